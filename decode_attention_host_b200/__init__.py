"""Python binding of libdkv: zero-copy host/HBM split-KV decode attention on B200.

Argument marshalling only.  Every step of the decode path runs in the CUDA
kernels of ``libdkv.so`` (built in-tree by ``python
decode_attention_host_b200/build.py``); importing this package fails loudly if
the library is missing, and there is no CPU fallback.  PyTorch is used for
device memory and streams.

The functions ``dkv_*`` mirror the C ABI in ``include/dkv.h`` one to one and
raise :class:`DkvError` when the C call returns a nonzero code.  The classes
below them (:class:`HostPool`, :class:`PagedKV`, :class:`DecodeAttention`)
only bundle those calls for the tests and the benchmark.
"""
from __future__ import annotations

import ctypes
import os
from pathlib import Path

import numpy as np

_PKG = Path(__file__).resolve().parent
# DKV_LIB_PATH selects another build of the same library (e.g. one compiled
# with different DKV_* build-time knobs) for side-by-side timing.
LIB_PATH = Path(os.environ.get("DKV_LIB_PATH", str(_PKG / "libdkv.so")))

DKV_OK = 0
DKV_ERR_INVALID_ARG = -1
DKV_ERR_UNSUPPORTED = -2
DKV_ERR_CUDA = -3
DKV_ERR_NO_MEMORY = -4
DKV_STATUS_BAD_BLOCK_ID = 1
DKV_STATUS_BAD_SEQ_LEN = 2
DKV_STATUS_COPY_TIMEOUT = 4
DKV_STATUS_INTERNAL = 8
DKV_KV_F16 = 0
DKV_KV_BF16 = 1
DKV_PLACE_PREFIX_HOST = 0
DKV_PLACE_RANDOM = 1

EXPORTED = ("dkv_create", "dkv_destroy", "dkv_attn_decode", "dkv_get_status", "dkv_last_error_string",
            "dkv_last_launch_count", "dkv_query_plan", "dkv_host_pool_alloc", "dkv_host_pool_free",
            "dkv_plan_blocks", "dkv_pack_kv", "dkv_profile_begin", "dkv_profile_end",
            "dkv_attn_decode_noalloc", "dkv_plan_offload", "dkv_attn_decode_staged", "dkv_append_kv",
            "dkv_attn_decode_multi", "dkv_debug_rope", "dkv_profile_timeline", "dkv_debug_fail_alloc",
            "dkv_debug_stall_copy")


class DkvConfig(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("kv_dtype", ctypes.c_int32), ("rope_base", ctypes.c_double),
                ("scale", ctypes.c_double), ("max_batch", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32),
                ("device", ctypes.c_int32), ("host_ctas", ctypes.c_int32)]


class DkvPlanParams(ctypes.Structure):
    _fields_ = [("block_size", ctypes.c_int32), ("placement", ctypes.c_int32), ("host_fraction", ctypes.c_double),
                ("shuffle_ids", ctypes.c_int32), ("seed", ctypes.c_uint64)]


class DkvPlanResult(ctypes.Structure):
    _fields_ = [("host_split", ctypes.c_int32), ("num_dev_blocks", ctypes.c_int32),
                ("host_tokens", ctypes.c_int64), ("dev_tokens", ctypes.c_int64)]


class DkvOffloadPlan(ctypes.Structure):
    _fields_ = [("host_fraction", ctypes.c_double), ("step_seconds", ctypes.c_double),
                ("hbm_bytes_freed", ctypes.c_double), ("time_optimal_fraction", ctypes.c_double)]


class DkvError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"libdkv error {code}: {message}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not LIB_PATH.exists():
        raise ImportError(f"{LIB_PATH} is missing: build it with `python decode_attention_host_b200/build.py`")
    lib = ctypes.CDLL(str(LIB_PATH))
    c, vp, i32, i64 = ctypes, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    sig = {
        "dkv_create": [c.POINTER(DkvConfig), c.POINTER(vp)],
        "dkv_destroy": [vp],
        "dkv_attn_decode": [vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32],
        "dkv_attn_decode_staged": [vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, vp, vp],
        "dkv_append_kv": [vp, vp, vp, vp, i32, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32],
        "dkv_attn_decode_multi": [vp, i32, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32],
        "dkv_get_status": [vp, c.POINTER(i32)],
        "dkv_last_error_string": [],
        "dkv_last_launch_count": [vp, c.POINTER(i32)],
        "dkv_query_plan": [vp, i32, i32, c.POINTER(i32), c.POINTER(i32)],
        "dkv_host_pool_alloc": [c.c_size_t, c.POINTER(vp)],
        "dkv_host_pool_free": [vp],
        "dkv_plan_blocks": [c.POINTER(DkvPlanParams), vp, i32, vp, i32, c.POINTER(DkvPlanResult)],
        "dkv_pack_kv": [vp, vp, i64, vp, i32, i32, i32, i32, vp, i32, i32, i32, vp, vp, vp, vp],
        "dkv_profile_begin": [vp, i32],
        "dkv_plan_offload": [c.c_double, c.c_double, c.c_double, c.c_double, c.c_double, c.POINTER(DkvOffloadPlan)],
        "dkv_attn_decode_noalloc": [c.POINTER(DkvConfig), vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, i32, i32,
                                    i32],
        "dkv_profile_end": [vp, c.POINTER(c.c_float), c.POINTER(i32)],
        "dkv_debug_rope": [i32, i32, c.c_double, vp, vp, i32, vp, vp, vp, i32, vp, vp],
        "dkv_profile_timeline": [vp, i32, c.POINTER(c.c_float)],
        "dkv_debug_fail_alloc": [i32],
        "dkv_debug_stall_copy": [i32],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "dkv_last_error_string" else ctypes.c_int
    return lib


lib = _load()


def _check(rc: int) -> None:
    if rc != DKV_OK:
        raise DkvError(rc, lib.dkv_last_error_string().decode())


def _p(x) -> int | None:
    """Address of a numpy array, torch tensor, int or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()


# ----------------------------------------------------------------------------- C ABI, one to one

def dkv_create(cfg: DkvConfig) -> int:
    h = ctypes.c_void_p()
    _check(lib.dkv_create(ctypes.byref(cfg), ctypes.byref(h)))
    return h.value


def dkv_destroy(h: int) -> None:
    _check(lib.dkv_destroy(h))


def dkv_attn_decode(h, q, k_host, v_host, k_dev, v_dev, block_table, seq_lens, host_split, out, stream,
                    batch, block_table_stride, num_dev_blocks) -> None:
    _check(lib.dkv_attn_decode(h, _p(q), _p(k_host), _p(v_host), _p(k_dev), _p(v_dev), _p(block_table),
                               _p(seq_lens), int(host_split), _p(out), stream, int(batch),
                               int(block_table_stride), int(num_dev_blocks)))


def dkv_attn_decode_staged(h, q, k_host, v_host, k_dev, v_dev, block_table, seq_lens, host_split, out, stream,
                           batch, block_table_stride, num_dev_blocks, k_stage, v_stage) -> None:
    _check(lib.dkv_attn_decode_staged(h, _p(q), _p(k_host), _p(v_host), _p(k_dev), _p(v_dev), _p(block_table),
                                      _p(seq_lens), int(host_split), _p(out), stream, int(batch),
                                      int(block_table_stride), int(num_dev_blocks), _p(k_stage), _p(v_stage)))


def dkv_append_kv(h, x, w_k, w_v, hidden, block_table, seq_lens, host_split, k_host, v_host, k_dev, v_dev, stream,
                  batch, block_table_stride, num_dev_blocks) -> None:
    _check(lib.dkv_append_kv(h, _p(x), _p(w_k), _p(w_v), int(hidden), _p(block_table), _p(seq_lens), int(host_split),
                             _p(k_host), _p(v_host), _p(k_dev), _p(v_dev), stream, int(batch),
                             int(block_table_stride), int(num_dev_blocks)))


def dkv_attn_decode_multi(h, num_queries, q, k_host, v_host, k_dev, v_dev, block_table, seq_lens, host_split, out,
                          stream, batch, block_table_stride, num_dev_blocks) -> None:
    _check(lib.dkv_attn_decode_multi(h, int(num_queries), _p(q), _p(k_host), _p(v_host), _p(k_dev), _p(v_dev),
                                     _p(block_table), _p(seq_lens), int(host_split), _p(out), stream, int(batch),
                                     int(block_table_stride), int(num_dev_blocks)))


def dkv_get_status(h: int) -> int:
    s = ctypes.c_int32()
    _check(lib.dkv_get_status(h, ctypes.byref(s)))
    return s.value


def dkv_last_error_string() -> str:
    return lib.dkv_last_error_string().decode()


def dkv_last_launch_count(h: int) -> int:
    n = ctypes.c_int32()
    _check(lib.dkv_last_launch_count(h, ctypes.byref(n)))
    return n.value


def dkv_query_plan(h: int, batch: int, block_table_stride: int) -> tuple[int, int]:
    ns, bps = ctypes.c_int32(), ctypes.c_int32()
    _check(lib.dkv_query_plan(h, batch, block_table_stride, ctypes.byref(ns), ctypes.byref(bps)))
    return ns.value, bps.value


def dkv_host_pool_alloc(nbytes: int) -> int:
    p = ctypes.c_void_p()
    _check(lib.dkv_host_pool_alloc(nbytes, ctypes.byref(p)))
    return p.value


def dkv_host_pool_free(ptr: int) -> None:
    _check(lib.dkv_host_pool_free(ptr))


def dkv_plan_blocks(params: DkvPlanParams, seq_lens: np.ndarray, block_table: np.ndarray) -> DkvPlanResult:
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    assert block_table.dtype == np.int32 and block_table.flags.c_contiguous and block_table.ndim == 2
    res = DkvPlanResult()
    _check(lib.dkv_plan_blocks(ctypes.byref(params), _p(seq_lens), len(seq_lens), _p(block_table),
                               block_table.shape[1], ctypes.byref(res)))
    return res


def dkv_plan_offload(kv_bytes: float, host_gbs: float, hbm_gbs: float, hbm_budget_bytes: float = -1.0,
                     hbm_alone_gbs: float = -1.0) -> DkvOffloadPlan:
    plan = DkvOffloadPlan()
    _check(lib.dkv_plan_offload(float(kv_bytes), float(host_gbs), float(hbm_gbs), float(hbm_budget_bytes),
                                float(hbm_alone_gbs), ctypes.byref(plan)))
    return plan


def dkv_pack_kv(k_logical, v_logical, seq_lens, num_kv_heads, head_dim, block_size, block_table, host_split,
                num_dev_blocks, k_host, v_host, k_dev_stage, v_dev_stage) -> None:
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    _check(lib.dkv_pack_kv(_p(k_logical), _p(v_logical), int(k_logical.shape[2]), _p(seq_lens), len(seq_lens),
                           num_kv_heads, head_dim, block_size, _p(block_table), block_table.shape[1],
                           int(host_split), int(num_dev_blocks), _p(k_host), _p(v_host), _p(k_dev_stage),
                           _p(v_dev_stage)))


def dkv_attn_decode_noalloc(cfg: DkvConfig, q, k_host, v_host, k_dev, v_dev, block_table, seq_lens, host_split,
                            out, status_out, stream, batch, block_table_stride, num_dev_blocks) -> None:
    """The allocation-free decode entry point (fixed scratch compiled into the library)."""
    _check(lib.dkv_attn_decode_noalloc(ctypes.byref(cfg), _p(q), _p(k_host), _p(v_host), _p(k_dev), _p(v_dev),
                                       _p(block_table), _p(seq_lens), int(host_split), _p(out), _p(status_out),
                                       stream, int(batch), int(block_table_stride), int(num_dev_blocks)))


def dkv_debug_fail_alloc(nth: int) -> None:
    """Test only: the nth device allocation of the next dkv_create on this thread fails (0 disarms)."""
    _check(lib.dkv_debug_fail_alloc(int(nth)))


def dkv_debug_stall_copy(enable: bool) -> None:
    """Test only: the next HBM launch on this thread leaves one tile copy unissued (its wait runs out)."""
    _check(lib.dkv_debug_stall_copy(1 if enable else 0))


def dkv_debug_rope(kv_dtype, head_dim, rope_base, k, tile_pos, num_tiles, k_out, q, q_pos, num_q, q_out,
                   stream) -> None:
    """Test only: the decode kernels' RoPE steps on given key tiles and queries."""
    _check(lib.dkv_debug_rope(int(kv_dtype), int(head_dim), float(rope_base), _p(k), _p(tile_pos), int(num_tiles),
                              _p(k_out), _p(q), _p(q_pos), int(num_q), _p(q_out), stream))


def dkv_profile_begin(h: int, max_calls: int) -> None:
    _check(lib.dkv_profile_begin(h, int(max_calls)))


def dkv_profile_timeline(h: int, call: int) -> list[float]:
    """(start, stop) in ms of the host-stream kernel, the HBM kernel and the merge of one recorded call,
    from the earliest start; -1 for a kernel that did not run."""
    t = (ctypes.c_float * 6)()
    _check(lib.dkv_profile_timeline(h, int(call), t))
    return list(t)


def dkv_profile_end(h: int) -> tuple[list[float], list[int]]:
    """Summed device ms and launch counts of (host-stream kernel, HBM split-K kernel, merge)."""
    ms = (ctypes.c_float * 3)()
    counts = (ctypes.c_int32 * 3)()
    _check(lib.dkv_profile_end(h, ms, counts))
    return list(ms), list(counts)


# ----------------------------------------------------------------------------- bundles

class HostPool:
    """Mapped pinned host memory from dkv_host_pool_alloc, viewed as a uint16 numpy array."""

    def __init__(self, nelems: int):
        self.nbytes = max(2, 2 * int(nelems))
        self.ptr = dkv_host_pool_alloc(self.nbytes)
        buf = (ctypes.c_uint16 * (self.nbytes // 2)).from_address(self.ptr)
        self.array = np.ctypeslib.as_array(buf)

    def free(self) -> None:
        if self.ptr:
            self.array = None
            dkv_host_pool_free(self.ptr)
            self.ptr = 0

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


class PagedKV:
    """A paged KV cache split between a mapped pinned host pool and an HBM pool.

    Built from logical K/V bits ``[B, Hkv, Lmax, D]`` with dkv_plan_blocks and
    dkv_pack_kv; the device pool is uploaded once with a torch copy.
    """

    def __init__(self, k_logical, v_logical, seq_lens, block_size: int, placement: int, host_fraction: float,
                 shuffle: bool = False, seed: int = 0, stride: int | None = None, device: int = 0):
        import torch
        B, Hkv, Lmax, D = k_logical.shape
        self.batch, self.num_kv_heads, self.head_dim, self.block_size = B, Hkv, D, block_size
        self.seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        need = int(max(1, -(-int(self.seq_lens.max(initial=0)) // block_size)))
        self.stride = stride or need
        self.table = np.full((B, self.stride), -1, dtype=np.int32)
        params = DkvPlanParams(block_size, placement, float(host_fraction), int(shuffle), int(seed))
        self.plan = dkv_plan_blocks(params, self.seq_lens, self.table)
        self.host_split = self.plan.host_split
        self.num_dev_blocks = self.plan.num_dev_blocks
        blk = Hkv * block_size * D
        self.k_host = HostPool(self.host_split * blk)
        self.v_host = HostPool(self.host_split * blk)
        k_stage = np.zeros(max(1, self.num_dev_blocks * blk), dtype=np.uint16)
        v_stage = np.zeros_like(k_stage)
        dkv_pack_kv(k_logical, v_logical, self.seq_lens, Hkv, D, block_size, self.table, self.host_split,
                    self.num_dev_blocks, self.k_host.array, self.v_host.array, k_stage, v_stage)
        dev = torch.device("cuda", device)
        self.k_dev = torch.from_numpy(k_stage.view(np.int16)).to(dev)
        self.v_dev = torch.from_numpy(v_stage.view(np.int16)).to(dev)
        del k_stage, v_stage
        self.table_dev = torch.from_numpy(self.table).to(dev)
        self.seq_lens_dev = torch.from_numpy(self.seq_lens).to(dev)

    @property
    def host_bytes(self) -> int:
        """K+V bytes of valid tokens in host blocks."""
        return 2 * self.plan.host_tokens * self.num_kv_heads * self.head_dim * 2

    @property
    def dev_bytes(self) -> int:
        return 2 * self.plan.dev_tokens * self.num_kv_heads * self.head_dim * 2

    def free(self) -> None:
        self.k_host.free()
        self.v_host.free()


class DecodeAttention:
    """A libdkv handle for one model shape."""

    def __init__(self, num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int, kv_dtype: int,
                 rope_base: float, max_batch: int, max_blocks_per_seq: int, scale: float = 0.0, device: int = 0,
                 host_ctas: int = 0):
        self.cfg = DkvConfig(num_q_heads, num_kv_heads, head_dim, block_size, kv_dtype, float(rope_base),
                             float(scale), max_batch, max_blocks_per_seq, device, host_ctas)
        self.handle = dkv_create(self.cfg)

    def __call__(self, q, kv: PagedKV, out, stream=None) -> None:
        """out[B, Hq, D] = decode attention of q[B, Hq, D] over the cache ``kv`` (async on ``stream``)."""
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(q.device)
        dkv_attn_decode(self.handle, q, kv.k_host.ptr or None, kv.v_host.ptr or None,
                        kv.k_dev if kv.num_dev_blocks else None, kv.v_dev if kv.num_dev_blocks else None,
                        kv.table_dev, kv.seq_lens_dev, kv.host_split, out, stream.cuda_stream, kv.batch,
                        kv.stride, kv.num_dev_blocks)

    def staged(self, q, kv: PagedKV, out, k_stage, v_stage, stream=None) -> None:
        """The staged-prefetch comparator: copy the host pools into HBM, then run HBM kernels only."""
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(q.device)
        dkv_attn_decode_staged(self.handle, q, kv.k_host.ptr or None, kv.v_host.ptr or None,
                               kv.k_dev if kv.num_dev_blocks else None, kv.v_dev if kv.num_dev_blocks else None,
                               kv.table_dev, kv.seq_lens_dev, kv.host_split, out, stream.cuda_stream, kv.batch,
                               kv.stride, kv.num_dev_blocks, k_stage, v_stage)

    def append(self, x, w_k, w_v, kv: PagedKV, stream=None) -> None:
        """Project x[B, hidden] with w_k, w_v [Hkv*D, hidden] and store at position seq_lens[b] of the cache."""
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(x.device)
        dkv_append_kv(self.handle, x, w_k, w_v, x.shape[1], kv.table_dev, kv.seq_lens_dev, kv.host_split,
                      kv.k_host.ptr or None, kv.v_host.ptr or None, kv.k_dev if kv.num_dev_blocks else None,
                      kv.v_dev if kv.num_dev_blocks else None, stream.cuda_stream, kv.batch, kv.stride,
                      kv.num_dev_blocks)

    def multi(self, q, kv: PagedKV, out, stream=None) -> None:
        """q, out [B, Tq, Hq, D]: query i of sequence b at position seq_lens[b] + i, causal over the cache."""
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(q.device)
        dkv_attn_decode_multi(self.handle, q.shape[1], q, kv.k_host.ptr or None, kv.v_host.ptr or None,
                              kv.k_dev if kv.num_dev_blocks else None, kv.v_dev if kv.num_dev_blocks else None,
                              kv.table_dev, kv.seq_lens_dev, kv.host_split, out, stream.cuda_stream, kv.batch,
                              kv.stride, kv.num_dev_blocks)

    def status(self) -> int:
        return dkv_get_status(self.handle)

    def launches(self) -> int:
        return dkv_last_launch_count(self.handle)

    def plan(self, batch: int, stride: int) -> tuple[int, int]:
        return dkv_query_plan(self.handle, batch, stride)

    def close(self) -> None:
        if self.handle:
            dkv_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
