"""Plain CPU oracle for the block-sparse linear layer (fp64).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  It shares no
code with the CUDA library ``sparse_gemm_b200`` and imports nothing from it.

Sources it restates (page title + section):

* Hugging Face pytorch_block_sparse release note, "Block-Sparse
  Implementation and Usage": a linear layer whose weight W[N,K] keeps only
  its nonzero b x b blocks; Y = X W^T as in nn.Linear (no bias here).
* torchao sparsity README, introduction: pruned weights are handed over as a
  dense tensor with zeros at the pruned positions, and the sparse matmul is
  numerically the dense matmul with that tensor -> the contractions below are
  that dense definition, evaluated in fp64 by ``bsl_oracle.c``.
* torchao sparsity README, Table 4.1, rows BSR and CSR/CSC: blocks stored as
  data blocks plus an index (column indices per block row with a row pointer
  array; the transposed index per block column) -> :func:`pack`.
* torchao sparsity README, "Pruning Criteria", out-of-place mask updates:
  the masked weight gradient is dW (.) Mask -> :func:`backward_weight`
  evaluates dW = dY^T X at the mask's blocks only.

The contractions run in ``bsl_oracle.c`` (plain loops, OpenMP over output
rows/blocks).  The pack and the schedule order are plain Python loops.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsl_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile ``bsl_oracle.c`` with gcc (fp64, OpenMP) into liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC",
                               "-Wall", "-Wextra", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.bsl_oracle_dense_weight.argtypes = [_i64, _i64, _i64, _p, _p, _p]
        lib.bsl_oracle_widen.argtypes = [_i64, _p, _p]
        lib.bsl_oracle_forward_rows.argtypes = [_i64, _i64, _i64, _p, _p, _p, _i64, _p, _p]
        lib.bsl_oracle_backward_input_rows.argtypes = [_i64, _i64, _i64, _p, _p, _p, _i64, _p, _p]
        lib.bsl_oracle_backward_weight_blocks.argtypes = [_i64, _i64, _i64, _i64, _p, _p,
                                                          _p, _p, _i64, _p, _p]
        lib.bsl_oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().bsl_oracle_num_threads())


def widen(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().bsl_oracle_widen(bits.size, _ptr(bits), _ptr(out))
    return out


def dense_weight(W: np.ndarray, mask: np.ndarray, b: int) -> np.ndarray:
    """W with zeros outside the block mask, as float64 [N, K]."""
    W = np.ascontiguousarray(W, dtype=np.uint16)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    N, K = W.shape
    if N % b or K % b or mask.shape != (N // b, K // b):
        raise ValueError("shape mismatch between W, mask and b")
    out = np.empty((N, K), dtype=np.float64)
    _load().bsl_oracle_dense_weight(N, K, b, _ptr(W), _ptr(mask), _ptr(out))
    return out


def _rows(rows, M):
    if rows is None:
        rows = np.arange(M)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= M):
        raise ValueError("row index out of range")
    return rows


def forward(X, W, mask, b, rows=None, *, Xd=None, Wt=None):
    """Y[rows] = X[rows] Wt^T in fp64, and sum_k |x w| per output.

    ``X``/``W`` are bf16 bit arrays; ``Xd``/``Wt`` may pass already widened
    operands to skip the conversion.  Returns (Y, Yabs), shape [len(rows), N].
    """
    Xd = widen(X) if Xd is None else Xd
    Wt = dense_weight(W, mask, b) if Wt is None else Wt
    M, K = Xd.shape
    N = Wt.shape[0]
    rows = _rows(rows, M)
    Y = np.empty((rows.size, N))
    A = np.empty((rows.size, N))
    _load().bsl_oracle_forward_rows(M, N, K, _ptr(Xd), _ptr(Wt), _ptr(rows), rows.size,
                                    _ptr(Y), _ptr(A))
    return Y, A


def backward_input(dY, W, mask, b, rows=None, *, dYd=None, Wt=None):
    """dX[rows] = dY[rows] Wt in fp64, and sum_n |dy w| per output."""
    dYd = widen(dY) if dYd is None else dYd
    Wt = dense_weight(W, mask, b) if Wt is None else Wt
    M, N = dYd.shape
    K = Wt.shape[1]
    rows = _rows(rows, M)
    dX = np.empty((rows.size, K))
    A = np.empty((rows.size, K))
    _load().bsl_oracle_backward_input_rows(M, N, K, _ptr(dYd), _ptr(Wt), _ptr(rows),
                                           rows.size, _ptr(dX), _ptr(A))
    return dX, A


def backward_weight(dY, X, mask, b, blocks=None, *, dYd=None, Xd=None):
    """dW = dY^T X at mask blocks, in fp64, as [nblocks, b, b].

    ``blocks`` is a sequence of (block_row, block_col); by default every
    block of the mask in BSR order (row-major scan of the mask).  Returns
    (dW_blocks, abs_sums).
    """
    dYd = widen(dY) if dYd is None else dYd
    Xd = widen(X) if Xd is None else Xd
    M, N = dYd.shape
    K = Xd.shape[1]
    if blocks is None:
        rr, cc = np.nonzero(np.asarray(mask))
        blocks = list(zip(rr.tolist(), cc.tolist()))
    br = np.ascontiguousarray([r for r, _ in blocks], dtype=np.int64)
    bc = np.ascontiguousarray([c for _, c in blocks], dtype=np.int64)
    out = np.empty((len(blocks), b, b))
    A = np.empty((len(blocks), b, b))
    _load().bsl_oracle_backward_weight_blocks(M, N, K, b, _ptr(dYd), _ptr(Xd), _ptr(br),
                                              _ptr(bc), len(blocks), _ptr(out), _ptr(A))
    return out, A


def pack(W, mask, b):
    """Block-sparse storage of W (.) mask, by plain loops.

    BSR (torchao README, Table 4.1, BSR and CSR rows): blocks kept in
    row-major order of the mask; ``row_ptr[r]`` is the position of block row
    r's first block, ``col_idx[p]`` the block column of block p (ascending
    inside a row), ``values[p]`` the b x b block copied from W, row-major.
    The transposed index (Table 4.1, CSC row) lists, for each block column c,
    the block rows holding a block (ascending) in ``row_idx``, delimited by
    ``col_ptr``; ``csc_to_bsr[j]`` is the BSR position of the j-th CSC entry,
    so the values are stored once.
    """
    mask = np.asarray(mask)
    W = np.asarray(W)
    R, C = mask.shape
    row_ptr = [0]
    col_idx = []
    where = {}
    for r in range(R):
        for c in range(C):
            if mask[r, c]:
                where[(r, c)] = len(col_idx)
                col_idx.append(c)
        row_ptr.append(len(col_idx))
    nnz = len(col_idx)
    values = np.zeros((nnz, b, b), dtype=W.dtype)
    for (r, c), p in where.items():
        values[p] = W[r * b:(r + 1) * b, c * b:(c + 1) * b]
    col_ptr = [0]
    row_idx = []
    csc_to_bsr = []
    for c in range(C):
        for r in range(R):
            if mask[r, c]:
                row_idx.append(r)
                csc_to_bsr.append(where[(r, c)])
        col_ptr.append(len(row_idx))
    i32 = lambda v: np.asarray(v, dtype=np.int32)
    return {
        "nnz": nnz, "row_ptr": i32(row_ptr), "col_idx": i32(col_idx), "values": values,
        "col_ptr": i32(col_ptr), "row_idx": i32(row_idx), "csc_to_bsr": i32(csc_to_bsr),
    }


def schedule_order(ptr) -> np.ndarray:
    """Segments (block rows or block columns) sorted by block count,
    largest first, ties by lower id: the longest-first order in which a
    persistent kernel hands out its work."""
    ptr = [int(v) for v in ptr]
    counts = [ptr[i + 1] - ptr[i] for i in range(len(ptr) - 1)]
    return np.asarray(sorted(range(len(counts)), key=lambda i: (-counts[i], i)), dtype=np.int32)


def group_plan(ptr, idx, order, G: int, blk=None):
    """Work plan of the tensor-core forward (segments = block rows) or input
    gradient (segments = block columns).

    Segments are taken G at a time in ``order`` (longest first).  For each
    group, the block coordinates of its members are merged into one
    ascending list of distinct values ("entries"); each entry records which
    members hold a block there (bit i = i-th member of the group).  The
    blocks of the present members are listed entry by entry, members in
    group order.  ``ptr``/``idx`` are the segment pointer and per-entry
    coordinate arrays (BSR row_ptr/col_idx, or CSC col_ptr/row_idx); ``blk``
    maps a segment entry to its BSR block (None: the entry position itself).

    Returns (grp_ptr, grp_bptr, ent, blk_list) with ent = coordinate |
    (mask << 24).
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


def dw_group_ptr(col_ptr, group: int) -> np.ndarray:
    """Exclusive prefix over block columns of ceil(blocks_in_column / group):
    the weight-gradient kernel processes the blocks of one column in groups
    of ``group`` (= 128 / b) sharing the column's X strip."""
    col_ptr = [int(v) for v in col_ptr]
    out = [0]
    for c in range(len(col_ptr) - 1):
        n = col_ptr[c + 1] - col_ptr[c]
        out.append(out[-1] + (n + group - 1) // group)
    return np.asarray(out, dtype=np.int32)
