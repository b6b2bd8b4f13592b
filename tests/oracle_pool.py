"""Worker functions for running the oracle in a spawn-context process pool
(the oracle is single-threaded numpy; the full-size quantise workload needs it
on many cores).  Test infrastructure only."""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def quant_expert_and_oracle(args):
    """Expert j of the seeded quantise workload (bf16 bits [n, k]) and the
    oracle's quantisation of it: (w, q, s, G)."""
    seed, j, n, k = args
    import moe_inputs as gen
    from oracle import quantize as Q
    w = gen.make_quant_expert(seed, j, n, k)
    q, s, g = Q.quantize_tensor(w)
    return w, q, s, g


def pool(workers=None):
    import concurrent.futures as cf
    import multiprocessing as mp
    n = workers or max(1, min(32, len(os.sched_getaffinity(0))))
    return cf.ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"))
