"""Write the stored expected values under tests/golden/ from the oracle alone.

Run from the repository root:  python tests/golden/make_golden.py

tiny_block_index.txt: the block-sparse index of the tiny workload (1 head,
1024 tokens, head_dim 64, top-4 blocks per query block including the sink and
diagonal blocks), generated on the CPU with the seeded recipe in synth/ and
selected by oracle.block_index.  Selection rule: MInference 1.0 page, method
section (mean-pooled Q and K; pooling commutes with MatMul), with the sink and
diagonal blocks always kept.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import synth  # noqa: E402


def main():
    w = synth.make_prefill("tiny-1h-1k-d64", device="cpu")
    q, k = synth.to_f64(w.q), synth.to_f64(w.k)
    lists, _, _ = oracle.block_index(q, k, k_fixed=4)
    with open(os.path.join(HERE, "tiny_block_index.txt"), "w") as f:
        f.write("# tiny-1h-1k-d64: query_block: kept key blocks (ascending); oracle.block_index, k=4\n")
        f.write("# planted key blocks: " + " ".join(map(str, w.planted[0])) + "\n")
        for i in sorted(lists[0]):
            f.write(f"{i}: " + " ".join(map(str, lists[0][i].tolist())) + "\n")


if __name__ == "__main__":
    main()
