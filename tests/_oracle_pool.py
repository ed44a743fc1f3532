"""Oracle work items for a process pool (spawned, so it can start after CUDA is in use):
the full-size backward checks need the oracle on many independent (sequence, head) pairs.
Each item gets its own slices and runs the oracle on them unchanged."""
import multiprocessing as mp
import os

import numpy as np


def _ref():
    from oracle import ref
    return ref


def dsink_term(args):
    """The d_sink contribution of one (sequence, q head): -sum_i p_sink,i (dout_i . out_i)."""
    qh, kh, vh, doh, sink_h, scale, causal, wl, wr = args
    ref = _ref()
    r = ref.attend_head(qh, kh, vh, sink_h, scale, ref.allowed_mask(len(qh), len(kh), causal, wl, wr))
    D = (r["out"] * doh.astype(np.float64)).sum(1)
    return -float((r["p_sink"] * D).sum())


def group_bwd(args):
    """ref.bwd_sequence_group on one sequence's slices of one kv head and its q heads."""
    q, k, v, dout, sink, scale, causal, wl, wr = args
    ref = _ref()
    cu_q = np.array([0, len(q)], np.int64)
    cu_k = np.array([0, len(k)], np.int64)
    return ref.bwd_sequence_group(q, k, v, dout, cu_q, cu_k, sink, scale, causal, wl, wr, b=0, g=0)


def pool_map(fn, items, workers=None):
    """fn over items in a spawned pool of `workers` processes (default: a quarter of the
    cores, at least 1, at most 8: each item holds a few full score matrices)."""
    if workers is None:
        workers = max(1, min(8, (os.cpu_count() or 4) // 4))
    with mp.get_context("spawn").Pool(workers) as pool:
        return pool.map(fn, items, chunksize=1)
