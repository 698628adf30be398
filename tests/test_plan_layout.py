"""CPU checks of the plan builders in tests/_plan.py (the reference the GPU
tests hold the device-built plans to).  Each is checked against a property
found independently: a walk over the stored blocks, not the same formula."""
import numpy as np
import pytest

import oracle
import synth
from tests import _plan


def test_group_plan_covers_every_block_once(oracle_lib):
    """Each stored block appears exactly once, under its own coordinate and
    member, and entries are strictly ascending inside a group."""
    b, R, C, G = 4, 11, 9, 4
    mask = synth.mask_uniform(R, C, 37, np.random.default_rng(31))
    mask[5, :] = 0
    W = synth.bf16_bits(np.random.default_rng(31).standard_normal((R * b, C * b), dtype=np.float32))
    pk = oracle.pack(W, mask, b)
    order = oracle.schedule_order(pk["row_ptr"])
    gp, gb, ent, blk = _plan.group_plan(pk["row_ptr"], pk["col_idx"], order, G)
    assert sorted(blk.tolist()) == list(range(pk["nnz"]))
    seen = set()
    for g in range(len(gp) - 1):
        members = order[g * G:(g + 1) * G]
        cols = [int(e) & 0xFFFFFF for e in ent[gp[g]:gp[g + 1]]]
        assert cols == sorted(set(cols))
        q = gb[g]
        for e in ent[gp[g]:gp[g + 1]]:
            c, m = int(e) & 0xFFFFFF, int(e) >> 24
            for i in range(G):
                if m >> i & 1:
                    p = blk[q]
                    q += 1
                    r = members[i]
                    assert pk["row_ptr"][r] <= p < pk["row_ptr"][r + 1] and pk["col_idx"][p] == c
                    seen.add((r, c))
        assert q == gb[g + 1]
    assert seen == set(zip(*np.nonzero(mask)))
    # transposed plan over the CSC index maps to the same blocks
    corder = oracle.schedule_order(pk["col_ptr"])
    gp, gb, ent, blk = _plan.group_plan(pk["col_ptr"], pk["row_idx"], corder, G, blk=pk["csc_to_bsr"])
    assert sorted(blk.tolist()) == list(range(pk["nnz"]))


@pytest.mark.parametrize("R,C,nnz,U,seed", [
    (344, 128, 11008, 148, 1),   # the decode weight's shape and density
    (224, 64, 1434, 148, 2),
    (40, 30, 900, 148, 3),       # fewer blocks per CTA than rows are long
    (12, 7, 50, 148, 4),         # fewer blocks than CTAs: equal shares
    (64, 64, 4096, 16, 5),       # density 1
])
def test_stream_bounds_are_a_partition_that_keeps_short_rows_whole(R, C, nnz, U, seed):
    mask = synth.mask_uniform(R, C, nnz, np.random.default_rng(seed))
    mask[0, :] = 0
    mask[R // 2, :] = 0
    row_ptr = np.concatenate([[0], np.cumsum(mask.sum(axis=1))]).astype(np.int64)
    nnz = int(row_ptr[-1])
    sb = _plan.stream_bounds(row_ptr, U)
    assert sb[0] == U and len(sb) == U + 2
    b = sb[1:].astype(np.int64)
    assert b[0] == 0 and b[-1] == nnz
    assert np.all(np.diff(b) >= 0)
    q = nnz // (2 * U)
    t = np.arange(U + 1) * nnz // U
    assert np.all(np.abs(b - t) <= q)
    starts = set(int(v) for v in row_ptr)
    for c in range(U + 1):
        if b[c] != t[c]:
            assert int(b[c]) in starts  # only ever moved onto a row start
    # a row of at most 2q + 1 blocks always has a row start within q of any
    # block inside it, so no bound falls strictly inside it
    for r in range(R):
        lo, hi = int(row_ptr[r]), int(row_ptr[r + 1])
        if hi - lo <= 2 * q + 1:
            assert not np.any((b > lo) & (b < hi)), r
    if q == 0:
        assert np.array_equal(b, t)
        return
    # where the window [t - q, t + q] holds a row start the bound is one
    for c in range(1, U):
        if any(t[c] - q <= v <= t[c] + q for v in starts):
            assert int(b[c]) in starts
    # the largest range is the minimum over every allowed choice of bounds:
    # a dynamic programme over the candidates of each bound, written here
    cands = [[0]] + [sorted({int(v) for v in row_ptr if t[c] - q <= v <= t[c] + q} or {int(t[c])})
                     for c in range(1, U)]
    best = {0: 0}
    for c in range(1, U):
        best = {v: min(max(m, v - u) for u, m in best.items() if u <= v) for v in cands[c]}
    optimum = min(max(m, nnz - u) for u, m in best.items())
    assert np.diff(b).max() == optimum
