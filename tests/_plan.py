"""Reference builders for the tensor-core kernels' work plans (test helper).

These are layouts of this library's CUDA engine, not definitions from the
pages, so they live with the tests rather than in the oracle: the GPU tests
compare the plans that ``bsl_pack`` builds on the device with the ones
built here by plain loops, and ``test_plan_layout.py`` checks these builders
against independent properties (every stored block covered exactly once,
group counts found by walking the columns).
"""
from __future__ import annotations

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

    CTA c starts at its equal share t = floor(c * nnz / U), moved to the start
    of the block row holding block t or of the next row, whichever is nearer
    (the row's own start on a tie), when that is at most q = floor(nnz / (2U))
    blocks away; otherwise it starts at t."""
    row_ptr = [int(v) for v in row_ptr]
    nnz = row_ptr[-1]
    q = nnz // (2 * U)
    out = [U]
    for c in range(U + 1):
        t = c * nnz // U
        bound = t
        if 0 < t < nnz and q > 0:
            r = max(i for i in range(len(row_ptr) - 1) if row_ptr[i] <= t)  # the row holding block t
            da, dz = t - row_ptr[r], row_ptr[r + 1] - t
            if da <= dz:
                if da <= q:
                    bound = t - da
            elif dz <= q:
                bound = t + dz
        out.append(bound)
    return np.asarray(out, dtype=np.int32)
