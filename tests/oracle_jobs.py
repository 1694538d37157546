"""Oracle runs split over query heads in a process pool (test infrastructure only).

The full-size parity tests compare every output element of a workload with the
fp64 oracle.  The oracle's extend functions are per-head loops, so the heads are
spread over worker processes.  The pool uses the ``spawn`` start method: a pool
forked after the parent has touched the GPU can hang, a spawned one cannot.
Each worker limits its BLAS library to one thread so the workers do not
oversubscribe the host's cores.
"""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np


def _one_blas_thread():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def _extend_head(args):
    """One query head (q [T, 1, D]) against its KV head's pools ([slots, 1, D])."""
    from oracle import attention as oa
    h, qb, cu, kb, vb, table, lens, page_size, scale = args
    o, l = oa.extend(qb, cu, kb, vb, table, lens, page_size, scale)
    return h, o[:, 0], l[:, 0]


def _sage_extend_head(args):
    """One query head and its KV head's 8-bit pools, scales and v_mean (head axis of size 1)."""
    from oracle import sage as osg
    h, q8, sfq, cu, k8, v8, sfk, sfv, vm, table, lens = args
    return h, osg.sage_extend(q8, sfq, cu, k8, v8, sfk, sfv, vm, table, lens, 64)[:, 0]


def workers():
    return max(1, min(16, (os.cpu_count() or 2) - 1))


def pool():
    return ProcessPoolExecutor(max_workers=workers(), mp_context=mp.get_context("spawn"),
                               initializer=_one_blas_thread)


def extend_all_heads(qb, cu, kb, vb, table, lens, page_size, scale):
    """oracle.attention.extend over every query head: (O [T, Hq, D], lse [T, Hq])."""
    T, Hq, D = qb.shape
    G = Hq // kb.shape[1]
    out = np.zeros((T, Hq, D))
    lse = np.zeros((T, Hq))
    # each job carries only its own head's slices (the pools are sliced to one KV head)
    kv = {hk: (np.ascontiguousarray(kb[:, hk:hk + 1]), np.ascontiguousarray(vb[:, hk:hk + 1]))
          for hk in range(kb.shape[1])}
    jobs = [(h, qb[:, h:h + 1], cu) + kv[h // G] + (table, lens, page_size, scale) for h in range(Hq)]
    with pool() as ex:
        for h, o, l in ex.map(_extend_head, jobs):
            out[:, h] = o
            lse[:, h] = l
    return out, lse


def sage_extend_all_heads(q8, sfq, cu, k8, v8, sfk, sfv, vm, table, lens):
    """oracle.sage.sage_extend over every query head: O [T, Hq, D]."""
    T, Hq, D = q8.shape
    G = Hq // k8.shape[1]
    out = np.zeros((T, Hq, D))
    jobs = []
    for h in range(Hq):
        hk = h // G
        jobs.append((h, q8[:, h:h + 1], sfq[:, h:h + 1], cu, np.ascontiguousarray(k8[:, hk:hk + 1]),
                     np.ascontiguousarray(v8[:, hk:hk + 1]), np.ascontiguousarray(sfk[:, hk:hk + 1]),
                     sfv[hk:hk + 1], None if vm is None else vm[hk:hk + 1], table, lens))
    with pool() as ex:
        for h, o in ex.map(_sage_extend_head, jobs):
            out[:, h] = o
    return out
