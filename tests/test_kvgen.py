"""The seeded input generator: rounding, determinism, shapes and the outlier recipe."""
import numpy as np
import torch

import kvgen


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(200000).astype(np.float32) * 3
    x[:4] = [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]   # ties round to even
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(kvgen.f32_to_bf16_bits(x), want)


def test_f16_rounding_matches_torch():
    x = np.random.default_rng(1).standard_normal(200000).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(kvgen.f32_to_f16_bits(x), want)


def test_deterministic_and_sliceable():
    w = kvgen.OPT_6_7B.replace(batch=3, ctx=(16, 40))
    lens = kvgen.gen_seq_lens(w)
    assert lens.dtype == np.int32 and (lens >= 16).all() and (lens <= 40).all()
    k1, v1 = kvgen.gen_kv(w, lens)
    k2, v2 = kvgen.gen_kv(w, lens)
    assert np.array_equal(k1, k2) and np.array_equal(v1, v2)
    assert k1.shape == (3, 32, int(lens.max()), 128)
    b, h = 2, 5
    assert np.array_equal(k1[b, h, :lens[b]], kvgen.gen_kv_slice(w, "k", b, h, int(lens[b])))
    assert not k1[b, h, lens[b]:].any()
    std = kvgen.bits_to_f32(v1[0, :, :lens[0]], w.kv_dtype).std()
    assert 0.45 < std < 0.55


def test_outliers_scale_keys_by_eight():
    cell = kvgen.sweep_cells()[0]
    assert cell.outlier_p == 0.01 and cell.kv_dtype == kvgen.BF16
    plain = cell.replace(outlier_p=0.0)
    L = 4096
    mask = kvgen.outlier_tokens(cell, 1, L)
    assert 10 < mask.sum() < 90
    a = kvgen.bits_to_f32(kvgen.gen_kv_slice(cell, "k", 1, 3, L), cell.kv_dtype)
    b = kvgen.bits_to_f32(kvgen.gen_kv_slice(plain, "k", 1, 3, L), cell.kv_dtype)
    assert np.array_equal(a[mask], 8 * b[mask]) and np.array_equal(a[~mask], b[~mask])


def test_sweep_has_twenty_cells_with_distinct_seeds():
    cells = kvgen.sweep_cells()
    assert len(cells) == 20 and len({c.seed for c in cells}) == 20
    assert {c.host_fraction for c in cells} == set(kvgen.SWEEP_HOST_FRACTION)


def test_threaded_generation_matches_serial_slices():
    """gen_kv draws large workloads on a thread pool: every slice must equal its serial draw."""
    w = kvgen.LLAMA3_8B.replace(batch=2, num_kv_heads=4, num_q_heads=16, ctx=(40000, 70000), seed=9)
    lens = kvgen.gen_seq_lens(w)
    k, v = kvgen.gen_kv(w, lens)
    assert k.nbytes >= (64 << 20)   # large enough to take the threaded path
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            L = int(lens[b])
            assert np.array_equal(k[b, h, :L], kvgen.gen_kv_slice(w, "k", b, h, L))
            assert np.array_equal(v[b, h, :L], kvgen.gen_kv_slice(w, "v", b, h, L))
            assert not k[b, h, L:].any() and not v[b, h, L:].any()
