"""Write the stored expected values under tests/golden/ (calls only oracle/ and kvgen).

The pages print no worked numerical example for decode attention, so the
stored values are the fp64 oracle's outputs on the seeded tiny GQA workload
(batch 1, 4 query heads over 1 KV head, head dim 64, context 512, fp16 K/V,
RoPE base 1e4, seed 0).  They pin later runs of the oracle and of the input
generator against silent change, and give the GPU smoke check an expected
answer.  Run:  python tests/golden/make_golden.py
"""
import hashlib
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import kvgen    # noqa: E402
import oracle   # noqa: E402


def input_digest(q, k, v, lens) -> str:
    h = hashlib.sha256()
    for a in (q, k, v, lens):
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()


def main():
    w = kvgen.TINY_GQA
    q = kvgen.gen_q(w)
    lens = kvgen.gen_seq_lens(w)
    k, v = kvgen.gen_kv(w, lens)
    out = oracle.decode(q, k, v, lens, oracle.KV_F16, w.rope_base)
    path = os.path.join(HERE, "tiny_gqa_oracle.txt")
    with open(path, "w") as f:
        f.write("# fp64 oracle output, tiny GQA decode workload (B=1, Hq=4, Hkv=1, D=64, L=512,\n")
        f.write("# fp16 K/V ~ N(0,1), q fp32 ~ N(0,1), NeoX RoPE base 1e4, q at position 512, seed 0)\n")
        f.write("# written by tests/golden/make_golden.py (oracle/ + kvgen only)\n")
        f.write(f"# inputs_sha256 {input_digest(q, k, v, lens)}\n")
        f.write("# rows: query head, columns: head dim\n")
        for hq in range(w.num_q_heads):
            f.write(" ".join(f"{x:.17g}" for x in out[0, hq]) + "\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
