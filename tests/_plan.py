"""Reference builders for the tensor-core kernels' work plans (test helper).

These are layouts of this library's CUDA engine, not definitions from the
pages, so they live with the tests rather than in the oracle: the GPU tests
compare the plans that ``bsl_pack`` builds on the device with the ones
built here by plain loops, and ``test_plan_layout.py`` checks these builders
against independent properties (every stored block covered exactly once,
group counts found by walking the columns).
"""
from __future__ import annotations

import bisect

import numpy as np


def group_plan(ptr, idx, order, G: int, blk=None):
    """Plan of the forward (segments = block rows) or input gradient
    (segments = block columns) engine.

    Segments are taken G at a time in ``order`` (longest first).  For each
    group the members' block coordinates are merged into one ascending list
    of distinct values ("entries"); an entry records which members hold a
    block there (bit i = i-th member).  The blocks of the present members are
    listed entry by entry, members in group order.  ``blk`` maps a segment
    position to its BSR block (None: the position itself).

    Returns (grp_ptr, grp_bptr, ent, blk_list) with ent = coordinate | (mask << 24).
    """
    ptr = [int(v) for v in ptr]
    idx = [int(v) for v in idx]
    order = [int(v) for v in order]
    nseg = len(ptr) - 1
    ngroups = (nseg + G - 1) // G
    grp_ptr, grp_bptr, ent, blk_list = [0], [0], [], []
    for g in range(ngroups):
        members = order[g * G:(g + 1) * G]
        coords = {}
        for i, sgm in enumerate(members):
            for j in range(ptr[sgm], ptr[sgm + 1]):
                coords.setdefault(idx[j], {})[i] = j
        for c in sorted(coords):
            present = coords[c]
            mask = 0
            for i in sorted(present):
                mask |= 1 << i
                j = present[i]
                blk_list.append(j if blk is None else int(blk[j]))
            ent.append(c | (mask << 24))
        grp_ptr.append(len(ent))
        grp_bptr.append(len(blk_list))
    i32 = lambda v: np.asarray(v, dtype=np.int64).astype(np.int32)
    return i32(grp_ptr), i32(grp_bptr), i32(ent), i32(blk_list)


def stream_bounds(row_ptr, U: int) -> np.ndarray:
    """CTA ranges of the weight-streaming forward, ``[U, b_0, ..., b_U]``.

    Bound c stays within q = floor(nnz / (2U)) blocks of its equal share
    t = floor(c * nnz / U): on one of the block-row starts inside the window
    [t - q, t + q] when there is any, else at t itself.  Among those choices
    the bounds are the ones that reach the end with the smallest largest
    range L, taking for each CTA in turn the largest allowed bound at most L
    past the previous one.  With q = 0 the bounds are the equal shares."""
    row_ptr = [int(v) for v in row_ptr]
    nnz = row_ptr[-1]
    q = nnz // (2 * U)
    t = [c * nnz // U for c in range(U + 1)]
    if q == 0:
        return np.asarray([U] + t, dtype=np.int32)
    inside = [sorted({v for v in row_ptr[bisect.bisect_left(row_ptr, t[c] - q):bisect.bisect_right(row_ptr, t[c] + q)]})
              for c in range(U)]

    def largest(c, x):
        if not inside[c]:
            return t[c] if t[c] <= x else -1
        i = bisect.bisect_right(inside[c], x)
        return inside[c][i - 1] if i else -1

    def bounds_for(L):
        b = [0]
        for c in range(1, U):
            v = largest(c, b[-1] + L)
            if v < b[-1]:
                return None
            b.append(v)
        return b + [nnz] if nnz - b[-1] <= L else None

    lo, hi = -(-nnz // U), nnz  # bounds_for(nnz) always succeeds
    while lo < hi:
        mid = (lo + hi) // 2
        if bounds_for(mid) is None:
            lo = mid + 1
        else:
            hi = mid
    return np.asarray([U] + bounds_for(lo), dtype=np.int32)
