"""The decode kernels' NeoX RoPE, element by element against the fp64 oracle (needs a B200).

dkv_debug_rope runs the split kernel's own rotation steps (fp64-reduced seed
angle, 4-position fp32 recurrence, a fresh seed at least every 16 tiles) on
given key tiles and queries.  The angle p * base^(-2i/D) reaches about 10^6
rad at the longest context, where one fp32 ulp of the angle is 0.0625 rad, so
this is where a rotation done in fp32 would break.

Error bound of the rotated value, relative to the pair's magnitude |(x, y)|:
the seed's angle is reduced in fp64 and rounded to fp32 (<= 2^-24 * pi) and
__sincosf on [-pi, pi] is accurate to ~2^-21.4 absolute; each of the at most
63 recurrence steps multiplies by a 4-position step factor carrying the same
~2^-21.4 error, so the phase and magnitude drift by at most ~64 * 4e-7 = 2.6e-5.
The test asserts 5e-5 * |pair| + 1e-6 per element.
"""
import json
import os

import numpy as np
import pytest
import torch

import decode_attention_host_b200 as dkv
import kvgen
import oracle

pytestmark = pytest.mark.gpu

REL = 5e-5
ABS = 1e-6


def _tiles(starts_and_counts):
    """Tile start positions: runs of consecutive 16-token tiles."""
    pos = []
    for start, count in starts_and_counts:
        pos.extend(start + 16 * i for i in range(count))
    return np.array(pos, dtype=np.int32)


# runs of consecutive tiles: from position 0 across two reseeds (tiles 16 and 32
# of the chain), around 511/512 and 32767/32768, a run that ends at 2^20 - 1,
# a single tile at the end of the 2^30-token capacity, and jumps between runs
RUNS = [(0, 40), (512 - 64, 8), (32768 - 48, 20), ((1 << 20) - 16 * 20, 20), ((1 << 30) - 16, 1), (7, 3)]
Q_POS = [0, 1, 511, 512, 32767, 32768, (1 << 20) - 1, 1 << 20, (1 << 30) - 1]


@pytest.mark.parametrize("d,dt,base", [(128, kvgen.BF16, 5e5), (64, kvgen.F16, 1e4), (128, kvgen.F16, 1e4),
                                       (64, kvgen.BF16, 5e5)])
def test_rope_matches_oracle_at_large_positions(d, dt, base):
    rng = np.random.default_rng(d + (1 if dt == kvgen.BF16 else 0))
    tile_pos = _tiles(RUNS)
    n = len(tile_pos)
    k_bits = kvgen.to_bits(rng.standard_normal((n, 16, d)).astype(np.float32), dt)
    q = rng.standard_normal((len(Q_POS), d)).astype(np.float32)
    q_pos = np.array(Q_POS, dtype=np.int32)
    dev = torch.device("cuda")
    k_out = torch.full((n, 16, d), float("nan"), dtype=torch.float32, device=dev)
    q_out = torch.full((len(Q_POS), d), float("nan"), dtype=torch.float32, device=dev)
    dkv.dkv_debug_rope(dkv.DKV_KV_BF16 if dt == kvgen.BF16 else dkv.DKV_KV_F16, d, base,
                       torch.from_numpy(k_bits.view(np.int16)).to(dev), torch.from_numpy(tile_pos).to(dev), n, k_out,
                       torch.from_numpy(q).to(dev), torch.from_numpy(q_pos).to(dev), len(Q_POS), q_out,
                       torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    got_k, got_q = k_out.cpu().numpy().astype(np.float64), q_out.cpu().numpy().astype(np.float64)
    k_f = kvgen.bits_to_f32(k_bits, dt).astype(np.float64)

    def worst(got, x, pos):
        want = oracle.rope(x, float(pos), base)
        mag = np.hypot(x[: d // 2], x[d // 2:])
        bound = REL * np.concatenate([mag, mag]) + ABS
        err = np.abs(got - want)
        assert (err <= bound).all(), f"position {pos}: err {err.max():.3e} above bound"
        return float((err / (np.concatenate([mag, mag]) + 1e-30)).max())

    rel = 0.0
    for i in range(n):
        for r in range(16):
            rel = max(rel, worst(got_k[i, r], k_f[i, r], int(tile_pos[i]) + r))
    qrel = max(worst(got_q[j], q[j].astype(np.float64), Q_POS[j]) for j in range(len(Q_POS)))
    log = os.environ.get("DKV_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"test": "rope", "head_dim": d, "dtype": dt, "base": base,
                                "max_rel_err_k": rel, "max_rel_err_q": qrel}) + "\n")


def test_rope_rejects_bad_arguments():
    s = torch.cuda.current_stream().cuda_stream
    buf = torch.zeros(16 * 128, dtype=torch.float32, device="cuda")
    for args, code in [((dkv.DKV_KV_BF16, 96, 1e4), dkv.DKV_ERR_UNSUPPORTED),
                       ((dkv.DKV_KV_BF16, 128, 1.0), dkv.DKV_ERR_INVALID_ARG),
                       ((5, 128, 1e4), dkv.DKV_ERR_INVALID_ARG)]:
        with pytest.raises(dkv.DkvError) as e:
            dkv.dkv_debug_rope(*args, buf, buf, 1, buf, None, None, 0, None, s)
        assert e.value.code == code
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_debug_rope(dkv.DKV_KV_BF16, 128, 1e4, None, None, 1, None, None, None, 0, None, s)
    assert e.value.code == dkv.DKV_ERR_INVALID_ARG
