"""Stored oracle output for the tiny GQA workload still matches (oracle and generator unchanged)."""
import os

import numpy as np

import kvgen
import oracle
from tests.golden.make_golden import input_digest

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden():
    digest, rows = None, []
    with open(os.path.join(HERE, "tiny_gqa_oracle.txt")) as f:
        for line in f:
            if line.startswith("# inputs_sha256"):
                digest = line.split()[-1]
            elif not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    return digest, np.array(rows)


def test_tiny_gqa_golden():
    w = kvgen.TINY_GQA
    q = kvgen.gen_q(w)
    lens = kvgen.gen_seq_lens(w)
    k, v = kvgen.gen_kv(w, lens)
    digest, want = load_golden()
    assert digest == input_digest(q, k, v, lens), "seeded generator output changed"
    got = oracle.decode(q, k, v, lens, oracle.KV_F16, w.rope_base)[0]
    assert want.shape == (4, 64)
    assert np.abs(got - want).max() < 1e-13
