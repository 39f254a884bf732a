"""Write the oracle's outputs for the tiny fp32 workload to config1_oracle.json.

Calls only ``oracle/`` and the seeded input generator; nothing here touches the CUDA
library.  The file is a regression lock on the oracle: the pages print no worked example,
so these numbers carry no authority beyond the pinned oracle that produced them.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from hstu_attention_b200 import inputs as gen  # noqa: E402


def compute():
    pc = gen.config1_tiny()
    ck, cv, cpt = pc.compact_pool()
    out = oracle.hstu_paged(pc.q_new, pc.k_new, pc.v_new, pc.u_new, ck, cv, cpt, pc.cached_lens,
                            pc.new_lens, pc.num_targets, pc.rab, pc.n_max, pc.eps, nthreads=1)
    return {
        "workload": "tiny fp32 paged cache hit: 2 users, cached {37, 64}, 4 candidates each, "
                    "H=2, D=32, P=16, pool 32, NB=32, n_max=68, seed 1001",
        "shape": list(out.shape),
        "out_row0_head0": out[0, 0].tolist(),
        "out_row7_head1": out[7, 1].tolist(),
        "out_sum": float(out.sum()),
        "out_abs_sum": float(np.abs(out).sum()),
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "config1_oracle.json"), "w") as f:
        json.dump(compute(), f, indent=1)
