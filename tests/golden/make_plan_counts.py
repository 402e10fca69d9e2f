"""Writes plan_counts.json: for every named workload, the block-CSR size and
the number of attended (query, key) token pairs per head, both computed by the
fp64 oracle alone (the pair count token by token, O(N^2), about a minute).

Run from the repository root:  python tests/golden/make_plan_counts.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from block_sparse_attention_rope_b200 import synthetic  # noqa: E402


def main():
    out = {}
    for name, w in synthetic.WORKLOADS.items():
        rp, _ = oracle.block_csr(w.T, w.H, w.W, w.block, w.local, w.stride, w.n_cond)
        N, Nc = w.n_tokens, w.n_cond_tokens
        pairs = oracle.count_token_pairs(N, Nc, w.block, w.local, w.stride)
        if w.cached:  # queries are the noisy tokens only
            pairs -= Nc * Nc
        out[name] = {"nnz": int(rp[-1]), "q_blocks": int(len(rp) - 1),
                     "attended_token_pairs_per_head": int(pairs)}
        print(name, out[name], flush=True)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "plan_counts.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main()
