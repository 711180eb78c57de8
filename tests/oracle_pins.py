"""Pins of the fp64 oracle against things other than itself.

Each ``pin_*`` function takes an oracle library handle and raises
AssertionError when the oracle disagrees with what the mathematics or a
library routine fixes.  ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on deliberately broken copies of the
oracle to show that each plausible mistake is caught by at least one pin.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import kvgen
import oracle
from tests import independent as ind

F16, BF16 = oracle.KV_F16, oracle.KV_BF16


def _widen(bits: np.ndarray, dt: int) -> np.ndarray:
    if dt == BF16:
        return torch.from_numpy(bits.astype(np.int16).copy()).view(torch.bfloat16).double().numpy()
    return bits.view(np.float16).astype(np.float64)


def _case(rng, B, Hq, Hkv, D, Lmax, dt, std=1.0, lens=None):
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    x = rng.standard_normal((2, B, Hkv, Lmax, D)).astype(np.float32) * np.float32(std)
    conv = kvgen.f32_to_bf16_bits if dt == BF16 else kvgen.f32_to_f16_bits
    k, v = conv(x[0]), conv(x[1])
    if lens is None:
        lens = np.full(B, Lmax, dtype=np.int32)
    return q, k, v, np.asarray(lens, dtype=np.int32)


# ----------------------------------------------------------------------------- storage decode

def pin_f16_decode_exhaustive(lib):
    """Every binary16 bit pattern decodes to numpy's float16 value."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    want = bits.view(np.float16).astype(np.float64)
    got = np.array([lib.oracle_f16_to_f64(int(b)) for b in bits])
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all(), f"fp16 decode differs at {np.flatnonzero(~same)[:5]}"


def pin_bf16_decode_exhaustive(lib):
    """Every bfloat16 bit pattern decodes to torch.bfloat16's value."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    want = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([lib.oracle_bf16_to_f64(int(b)) for b in bits])
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all(), f"bf16 decode differs at {np.flatnonzero(~same)[:5]}"


# ----------------------------------------------------------------------------- RoPE

def pin_rope_closed_forms(lib):
    """D=2: theta_0 = p.  D=4: theta_1 = p / sqrt(base).  p=0 and base=0 are the identity."""
    for p in (0.0, 1.0, 2.5, 1000.0, 1048575.0):
        y = oracle.rope(np.array([1.0, 0.0]), p, 1e4, lib=lib)
        assert np.allclose(y, [math.cos(p), math.sin(p)], atol=1e-12, rtol=0), (p, y)
        y = oracle.rope(np.array([0.0, 1.0]), p, 1e4, lib=lib)
        assert np.allclose(y, [-math.sin(p), math.cos(p)], atol=1e-12, rtol=0), (p, y)
        base = 500000.0
        th1 = p / math.sqrt(base)
        y = oracle.rope(np.array([0.3, 0.7, -1.1, 2.0]), p, base, lib=lib)
        want = [0.3 * math.cos(p) + 1.1 * math.sin(p), 0.7 * math.cos(th1) - 2.0 * math.sin(th1),
                -1.1 * math.cos(p) + 0.3 * math.sin(p), 2.0 * math.cos(th1) + 0.7 * math.sin(th1)]
        assert np.allclose(y, want, atol=1e-9, rtol=0), (p, y, want)
    x = np.random.default_rng(0).standard_normal(128)
    assert np.array_equal(oracle.rope(x, 0.0, 5e5, lib=lib), x)
    assert np.array_equal(oracle.rope(x, 12345.0, 0.0, lib=lib), x)


def pin_rope_vs_complex(lib):
    """Matches the complex-number formulation to 1e-12 for D in {8, 64, 128}, p up to 2^20."""
    rng = np.random.default_rng(1)
    for D in (8, 64, 128):
        for base in (1e4, 5e5):
            for p in (0, 1, 7, 511, 512, 32767, 1 << 20):
                x = rng.standard_normal(D)
                want = ind.rope_complex(x[None, :], np.array([p]), base)[0]
                got = oracle.rope(x, float(p), base, lib=lib)
                assert np.allclose(got, want, atol=1e-10 * max(1, p / 1e4), rtol=0), (D, base, p)


def pin_rope_vs_hf(lib):
    """HF's rotate-half RoPE with its own fp32 frequency table agrees at small positions."""
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb
    from transformers import LlamaConfig
    D = 64
    cfg = LlamaConfig(hidden_size=D * 2, num_attention_heads=2, num_key_value_heads=2, head_dim=D,
                      rope_theta=10000.0, max_position_embeddings=4096)
    try:
        cfg.rope_parameters = {"rope_type": "default", "rope_theta": 10000.0}
    except Exception:
        pass
    emb = LlamaRotaryEmbedding(cfg)
    pos = torch.arange(0, 300, dtype=torch.int64)[None]
    x = torch.tensor(np.random.default_rng(2).standard_normal((1, 1, 300, D)), dtype=torch.float32)
    cos, sin = emb(x, pos)
    xr, _ = apply_rotary_pos_emb(x, x, cos, sin)
    for p in (0, 1, 17, 299):
        got = oracle.rope(x[0, 0, p].double().numpy(), float(p), 10000.0, lib=lib)
        assert np.allclose(got, xr[0, 0, p].double().numpy(), atol=2e-4, rtol=0), p


def pin_rope_invariants(lib):
    """Norm preserved; <RoPE(q,a), RoPE(k,b)> depends only on a - b."""
    rng = np.random.default_rng(3)
    for D in (8, 128):
        q, k = rng.standard_normal(D), rng.standard_normal(D)
        for a, b, c in ((5, 3, 11), (1000, 2, 70000), (0, 900000, 148576)):
            y = oracle.rope(q, a, 5e5, lib=lib)
            assert abs(np.linalg.norm(y) - np.linalg.norm(q)) < 1e-12
            d0 = oracle.rope(q, a, 5e5, lib=lib) @ oracle.rope(k, b, 5e5, lib=lib)
            d1 = oracle.rope(q, a + c, 5e5, lib=lib) @ oracle.rope(k, b + c, 5e5, lib=lib)
            assert abs(d0 - d1) < 1e-8, (D, a, b, c, d0, d1)


# ----------------------------------------------------------------------------- attention

def pin_attention_vs_numpy(lib):
    """Oracle equals the numpy/scipy formulation (<= 1e-12) on small GQA/MHA cases."""
    rng = np.random.default_rng(4)
    for (B, Hq, Hkv, D, Lmax, dt, base) in ((2, 4, 1, 8, 9, F16, 1e4), (3, 8, 2, 16, 40, BF16, 5e5),
                                           (2, 4, 4, 64, 33, F16, 1e4), (1, 6, 3, 128, 17, BF16, 0.0)):
        lens = rng.integers(1, Lmax + 1, size=B).astype(np.int32)
        q, k, v, lens = _case(rng, B, Hq, Hkv, D, Lmax, dt, lens=lens)
        got = oracle.decode(q, k, v, lens, dt, base, lib=lib)
        want = ind.attend_numpy(q, _widen(k, dt), _widen(v, dt), lens, base)
        err = np.abs(got - want).max()
        assert err < 1e-12, (B, Hq, Hkv, D, err)


def pin_attention_vs_torch_hf(lib):
    """Oracle equals HF rotate-half + repeat_kv + torch SDPA in fp64 (<= 1e-12)."""
    rng = np.random.default_rng(5)
    for (B, Hq, Hkv, D, Lmax, dt, base) in ((2, 8, 2, 32, 21, BF16, 5e5), (1, 4, 1, 64, 64, F16, 1e4),
                                           (2, 2, 2, 16, 5, F16, 1e4)):
        lens = rng.integers(1, Lmax + 1, size=B).astype(np.int32)
        q, k, v, lens = _case(rng, B, Hq, Hkv, D, Lmax, dt, lens=lens)
        got = oracle.decode(q, k, v, lens, dt, base, lib=lib)
        want = ind.attend_torch_hf(q, _widen(k, dt), _widen(v, dt), lens, base)
        err = np.abs(got - want).max()
        assert err < 1e-12, (B, Hq, Hkv, D, err)


def pin_special_cases(lib):
    """L=1 -> v_0; constant V -> that constant; no information in scores -> mean of V; L=0 -> 0."""
    rng = np.random.default_rng(6)
    B, Hq, Hkv, D, Lmax = 2, 8, 2, 64, 37
    q, k, v, lens = _case(rng, B, Hq, Hkv, D, Lmax, BF16)
    G = Hq // Hkv
    vf = _widen(v, BF16)
    # L = 1
    out = oracle.decode(q, k, v, np.array([1, 1], np.int32), BF16, 5e5, lib=lib)
    for b in range(B):
        for hq in range(Hq):
            assert np.allclose(out[b, hq], vf[b, hq // G, 0], atol=1e-14, rtol=0)
    # L = 0 -> zeros, untouched batch row unaffected
    out = oracle.decode(q, k, v, np.array([0, Lmax], np.int32), BF16, 5e5, lib=lib)
    assert np.all(out[0] == 0.0)
    # all V rows equal c
    c = kvgen.f32_to_bf16_bits(rng.standard_normal(D).astype(np.float32))
    vc = np.broadcast_to(c, v.shape).copy()
    out = oracle.decode(q, k, vc, lens, BF16, 5e5, lib=lib)
    assert np.allclose(out, np.broadcast_to(_widen(c, BF16), out.shape), atol=1e-13, rtol=0)
    # identical keys without RoPE, zero keys with RoPE, zero queries with RoPE -> mean of V
    mean = np.repeat(vf.mean(axis=2), G, axis=1)
    kid = np.broadcast_to(k[:, :, :1, :], k.shape).copy()
    for (qq, kk, base) in ((q, kid, 0.0), (q, np.zeros_like(k), 5e5), (np.zeros_like(q), k, 5e5)):
        out = oracle.decode(qq, kk, v, lens, BF16, base, lib=lib)
        assert np.allclose(out, mean, atol=1e-13, rtol=0)


def pin_dominant_key(lib):
    """A key built as alpha * R(p_q - p_j) q gives a score gap >= 30: output ~= v_j."""
    rng = np.random.default_rng(7)
    D, L, base = 128, 50, 5e5
    q = rng.standard_normal((1, 1, D)).astype(np.float32)
    k = kvgen.f32_to_bf16_bits(rng.standard_normal((1, 1, L, D)).astype(np.float32) * 0.1)
    v = kvgen.f32_to_bf16_bits(rng.standard_normal((1, 1, L, D)).astype(np.float32))
    for j in (0, 23, L - 1):
        kd = ind.rope_complex(q[0].astype(np.float64), np.array([L - j]), base)[0]    # R(p_q - p_j) q
        alpha = 40.0 * math.sqrt(D) / float(q[0, 0] @ q[0, 0])
        kk = k.copy()
        kk[0, 0, j] = kvgen.f32_to_bf16_bits((alpha * kd).astype(np.float32))
        out = oracle.decode(q, kk, v, np.array([L], np.int32), BF16, base, lib=lib)
        assert np.allclose(out[0, 0], _widen(v, BF16)[0, 0, j], atol=1e-9, rtol=0), j


def pin_gqa_equals_repeated_mha(lib):
    """Hq=8 over Hkv=2 equals Hq=8 over 8 KV heads that repeat each group head consecutively."""
    rng = np.random.default_rng(8)
    q, k, v, lens = _case(rng, 2, 8, 2, 32, 19, F16, lens=[19, 7])
    a = oracle.decode(q, k, v, lens, F16, 1e4, lib=lib)
    b = oracle.decode(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), lens, F16, 1e4, lib=lib)
    assert np.array_equal(a, b)


def pin_ignores_tokens_past_length(lib):
    """Storage past L_b (even NaN bit patterns) does not reach the output."""
    rng = np.random.default_rng(9)
    q, k, v, lens = _case(rng, 1, 4, 2, 16, 30, BF16, lens=[20])
    a = oracle.decode(q, k, v, lens, BF16, 5e5, lib=lib)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 20:] = 0x7FC0
    v2[:, :, 20:] = 0x7FC0
    b = oracle.decode(q, k2, v2, lens, BF16, 5e5, lib=lib)
    assert np.array_equal(a, b)


def pin_linear_in_v(lib):
    """Doubling V (exact in 16-bit) doubles the output."""
    rng = np.random.default_rng(10)
    q, k, v, lens = _case(rng, 1, 4, 1, 32, 25, F16, std=0.25)
    a = oracle.decode(q, k, v, lens, F16, 1e4, lib=lib)
    v2 = kvgen.f32_to_f16_bits(kvgen.bits_to_f32(v, kvgen.F16) * 2)
    b = oracle.decode(q, k, v2, lens, F16, 1e4, lib=lib)
    assert np.allclose(b, 2 * a, atol=1e-14, rtol=0)


def pin_explicit_scale(lib):
    """An explicit scale of 1/sqrt(D) equals the default; another scale matches the numpy formulation."""
    rng = np.random.default_rng(11)
    q, k, v, lens = _case(rng, 1, 4, 2, 32, 12, BF16)
    a = oracle.decode(q, k, v, lens, BF16, 5e5, scale=0.0, lib=lib)
    b = oracle.decode(q, k, v, lens, BF16, 5e5, scale=1.0 / math.sqrt(32), lib=lib)
    assert np.allclose(a, b, atol=1e-15, rtol=0)
    c = oracle.decode(q, k, v, lens, BF16, 5e5, scale=0.05, lib=lib)
    want = ind.attend_numpy(q, _widen(k, BF16), _widen(v, BF16), lens, 5e5, scale=0.05)
    assert np.abs(c - want).max() < 1e-12


def pin_projection(lib):
    """The K/V projection equals numpy's matmul of the widened weights; one-hot x picks a weight column."""
    rng = np.random.default_rng(12)
    for dt, B, R, H in ((BF16, 3, 40, 96), (F16, 2, 17, 64)):
        x = rng.standard_normal((B, H)).astype(np.float32)
        conv = kvgen.f32_to_bf16_bits if dt == BF16 else kvgen.f32_to_f16_bits
        w = conv(rng.standard_normal((R, H)).astype(np.float32))
        got = oracle.project(x, w, dt, lib=lib)
        want = x.astype(np.float64) @ _widen(w, dt).T
        assert np.abs(got - want).max() < 1e-12
        e = np.zeros((1, H), np.float32)
        e[0, 5] = 1.0
        assert np.array_equal(oracle.project(e, w, dt, lib=lib)[0], _widen(w, dt)[:, 5])


ALL_PINS = [pin_f16_decode_exhaustive, pin_bf16_decode_exhaustive, pin_rope_closed_forms, pin_rope_vs_complex,
            pin_rope_vs_hf, pin_rope_invariants, pin_attention_vs_numpy, pin_attention_vs_torch_hf,
            pin_special_cases, pin_dominant_key, pin_gqa_equals_repeated_mha, pin_ignores_tokens_past_length,
            pin_linear_in_v, pin_explicit_scale, pin_projection]
