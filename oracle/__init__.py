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
* torchao sparsity README, Table 4.1, row "NVIDIA 2:4 compressed
  representation" (with the 2:4 semi-structured pattern of the README's
  introduction and of the "Lecture 11: Sparsity" summary, 8:02 and 12:52: two
  of every four consecutive elements are zero): the weight kept as a dense
  matrix of half the width holding the unpruned elements plus 2-bit indices
  -> :func:`compress24` / :func:`decompress24`; its product is the dense
  product with the weight it came from -> :func:`semi24_forward`.

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
        lib.bsl_oracle_forward_rows_blockskip.argtypes = [_i64, _i64, _i64, _i64, _p, _p, _p, _p,
                                                          _i64, _p, _p]
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


def forward(X, W, mask, b, rows=None, *, Xd=None, Wt=None, bias=None):
    """Y[rows] = X[rows] Wt^T (+ bias) in fp64, and sum_k |x w| (+ |bias|) per output.

    ``X``/``W`` are bf16 bit arrays; ``Xd``/``Wt`` may pass already widened
    operands to skip the conversion.  ``bias`` (bf16 bits, [N]) is the bias
    of nn.Linear, which BlockSparseLinear replaces as a drop-in (Hugging Face
    pytorch_block_sparse release note, "Block-Sparse Implementation and
    Usage"): one added term per output column.  Returns (Y, Yabs), shape
    [len(rows), N].
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
    if bias is not None:
        bd = widen(bias).reshape(-1)
        if bd.size != N:
            raise ValueError("bias must have N entries")
        Y += bd[None, :]
        A += np.abs(bd)[None, :]
    return Y, A


def bias_grad(dY, *, dYd=None):
    """Gradient of the bias: dbias[n] = sum_m dY[m][n] in fp64 (a column sum,
    rows added in increasing m), and sum_m |dY[m][n]|.  Returns (dbias, abs)."""
    dYd = widen(dY) if dYd is None else dYd
    M, N = dYd.shape
    s = np.zeros(N)
    a = np.zeros(N)
    for m in range(M):
        s += dYd[m]
        a += np.abs(dYd[m])
    return s, a


def forward_blockskip(X, W, mask, b, rows=None, *, Xd=None, Wt=None):
    """The forward of :func:`forward` visiting only the kept blocks (the
    stored blocks' work only; bit-identical results).  Returns (Y, Yabs)."""
    Xd = widen(X) if Xd is None else Xd
    Wt = dense_weight(W, mask, b) if Wt is None else Wt
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    M, K = Xd.shape
    N = Wt.shape[0]
    if mask.shape != (N // b, K // b):
        raise ValueError("mask shape does not match W and b")
    rows = _rows(rows, M)
    Y = np.empty((rows.size, N))
    A = np.empty((rows.size, N))
    _load().bsl_oracle_forward_rows_blockskip(M, N, K, b, _ptr(Xd), _ptr(Wt), _ptr(mask), _ptr(rows),
                                              rows.size, _ptr(Y), _ptr(A))
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


# ---------------------------------------------------------------- 2:4 semi-structured

_SEMI24_CODES = (0x4, 0x8, 0xC, 0x9, 0xD, 0xE)  # i0 | i1 << 2 for the six pairs i0 < i1


def compress24(W):
    """NVIDIA 2:4 compressed representation of a dense weight with zeros in
    place (torchao sparsity README, Table 4.1, row "NVIDIA 2:4 compressed
    representation": a compressed dense matrix of half the size holding the
    unpruned elements, plus 2-bit indices).

    ``W``: bf16 bits (uint16) [N, K], K a multiple of 16.  Every group of four
    consecutive elements of a row (columns 4g .. 4g+3) may hold at most two
    nonzeros; +0 and -0 both count as zero.  Returns ``(values, meta)``:

    * ``values`` uint16 [N, K/2]: group g's two kept elements at columns
      2g and 2g+1, in index order, copied bit for bit;
    * ``meta`` uint16 [N, K/16]: entry (n, c) holds the kept positions of
      groups 4c .. 4c+3 of row n, group 4c+j in bits 4j .. 4j+3 as
      i0 | i1 << 2 (positions inside the group, i0 < i1).

    The kept positions are the nonzero ones; when a group has fewer than two
    nonzeros the lowest-indexed zeros complete the pair.  Raises ValueError
    when a group holds more than two nonzeros.
    """
    W = np.ascontiguousarray(W, dtype=np.uint16)
    N, K = W.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    v = W.reshape(N, K // 4, 4)
    nz = (v & 0x7FFF) != 0
    cnt = nz.sum(axis=2)
    if (cnt > 2).any():
        n, g = np.argwhere(cnt > 2)[0]
        raise ValueError(f"row {n}, group {g} holds {cnt[n, g]} nonzeros: not 2:4")
    need = 2 - cnt                                   # zeros that complete the pair
    zero = ~nz
    zeros_before = np.cumsum(zero, axis=2) - zero    # zeros at lower positions of the group
    kept = nz | (zero & (zeros_before < need[:, :, None]))
    pos = np.nonzero(kept)[2].reshape(N, K // 4, 2)  # two kept positions per group, ascending
    values = np.take_along_axis(v, pos, axis=2).reshape(N, K // 2)
    code = (pos[:, :, 0] | (pos[:, :, 1] << 2)).astype(np.uint16).reshape(N, K // 16, 4)
    meta = code[:, :, 0] | (code[:, :, 1] << 4) | (code[:, :, 2] << 8) | (code[:, :, 3] << 12)
    return values.astype(np.uint16), meta.astype(np.uint16)


def decompress24(values, meta):
    """Dense bf16 bits [N, K] from the compressed form of :func:`compress24`:
    each kept element back at its position, zeros (+0) elsewhere."""
    values = np.ascontiguousarray(values, dtype=np.uint16)
    meta = np.ascontiguousarray(meta, dtype=np.uint16)
    N, half = values.shape
    K = 2 * half
    if meta.shape != (N, K // 16):
        raise ValueError("meta must be [N, K/16]")
    code = np.stack([(meta >> (4 * j)) & 0xF for j in range(4)], axis=2).reshape(N, K // 4)
    i0, i1 = code & 3, code >> 2
    if ((i0 >= i1)).any():
        raise ValueError("meta holds a pair that is not ascending")
    out = np.zeros((N, K // 4, 4), dtype=np.uint16)
    pair = values.reshape(N, K // 4, 2)
    np.put_along_axis(out, i0[:, :, None].astype(np.int64), pair[:, :, :1], axis=2)
    np.put_along_axis(out, i1[:, :, None].astype(np.int64), pair[:, :, 1:], axis=2)
    return out.reshape(N, K)


def compress24_blocks(values):
    """2:4 compressed form of packed b x b blocks ([nnz, b, b] bf16 bits, as
    :func:`pack` returns them), block by block along each block row: the
    "50% sparse pattern within blocks" of the Hugging Face release note
    ("Future Development Roadmap") stored as Table 4.1's compressed
    representation.  Returns (values [nnz, b, b/2], meta [nnz, b, b/16])."""
    values = np.ascontiguousarray(values, dtype=np.uint16)
    nnz, b, _ = values.shape
    v, m = compress24(values.reshape(nnz * b, b))
    return v.reshape(nnz, b, b // 2), m.reshape(nnz, b, b // 16)


def semi24_forward(X, values, meta, rows=None, *, Xd=None, bias=None):
    """Y[rows] = X[rows] W^T (+ bias) in fp64 with W the dense weight that
    the compressed form stands for: the sparse product is the dense product
    with zeros in place (torchao sparsity README, introduction).  Returns
    (Y, Yabs) like :func:`forward`."""
    Wt = widen(decompress24(values, meta))
    return forward(X, None, None, None, rows, Xd=Xd, Wt=Wt, bias=bias)
