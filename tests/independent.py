"""Independent formulations used to pin the fp64 oracle.

None of this shares code with ``oracle/``: RoPE is written with complex
numbers (each rotate-half pair (x_i, x_{i+D/2}) is the complex number
x_i + 1j*x_{i+D/2}, turned by exp(1j*theta)), the GQA head mapping comes from
``np.repeat`` (or HF ``repeat_kv``), and softmax / attention come from library
routines (``scipy.special.softmax`` and ``torch``'s
``scaled_dot_product_attention`` in fp64).
"""
from __future__ import annotations

import numpy as np
import scipy.special
import torch


def inv_freq(D: int, base: float) -> np.ndarray:
    return 1.0 / np.power(float(base), np.arange(0, D, 2, dtype=np.float64) / D)


def rope_complex(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """x[..., n, D] rotated at positions pos[n] (complex-number formulation)."""
    if base == 0:
        return np.array(x, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    h = x.shape[-1] // 2
    z = x[..., :h] + 1j * x[..., h:]
    theta = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq(x.shape[-1], base)[None, :]
    z = z * np.exp(1j * theta)
    return np.concatenate([z.real, z.imag], axis=-1)


def attend_numpy(q: np.ndarray, k: np.ndarray, v: np.ndarray, seq_lens, base: float,
                 scale: float | None = None) -> np.ndarray:
    """Decode attention with numpy/scipy.

    q [B, Hq, D] (float), k/v [B, Hkv, Lmax, D] (already-widened float values).
    """
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    kr = np.repeat(np.asarray(k, dtype=np.float64), G, axis=1)   # HF repeat_kv order
    vr = np.repeat(np.asarray(v, dtype=np.float64), G, axis=1)
    out = np.zeros((B, Hq, D))
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        qh = rope_complex(q[b][:, None, :], np.array([L]), base)[:, 0, :]          # [Hq, D]
        kh = rope_complex(kr[b, :, :L, :], np.arange(L), base)                     # [Hq, L, D]
        s = np.einsum("hd,hld->hl", qh, kh) * scale
        p = scipy.special.softmax(s, axis=-1)
        out[b] = np.einsum("hl,hld->hd", p, vr[b, :, :L, :])
    return out


def attend_torch_hf(q: np.ndarray, k: np.ndarray, v: np.ndarray, seq_lens, base: float,
                    scale: float | None = None) -> np.ndarray:
    """Decode attention from HF's rotate-half RoPE + repeat_kv and torch SDPA, all fp64."""
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb, repeat_kv
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((B, Hq, D))
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        qt = torch.tensor(np.asarray(q[b], dtype=np.float64))[None, :, None, :]   # [1, Hq, 1, D]
        kt = torch.tensor(np.asarray(k[b, :, :L], dtype=np.float64))[None]        # [1, Hkv, L, D]
        vt = torch.tensor(np.asarray(v[b, :, :L], dtype=np.float64))[None]
        if base != 0:
            f = torch.tensor(inv_freq(D, base))
            def cs(pos):
                th = torch.tensor(np.asarray(pos, dtype=np.float64))[:, None] * f[None, :]
                emb = torch.cat([th, th], dim=-1)[None]                            # [1, n, D]
                return emb.cos(), emb.sin()
            cq, sq = cs([L])
            ck, sk = cs(np.arange(L))
            qt, _ = apply_rotary_pos_emb(qt, qt, cq, sq)
            kt, _ = apply_rotary_pos_emb(kt, kt, ck, sk)
        kt = repeat_kv(kt, G)
        vt = repeat_kv(vt, G)
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=float(scale))
        out[b] = o[0, :, 0, :].numpy()
    return out
