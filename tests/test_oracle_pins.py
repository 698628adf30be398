"""Pins for the fp64 CPU oracle (no GPU).

Each pin checks the oracle against something other than itself: exact
integer arithmetic done here with Python ints, library routines (numpy
matmul, scipy.sparse BSR/CSC builders, numpy lexsort) on the special cases
that reduce to them, the pages' 4x storage figure, and invariants of the
definitions (block permutations, adjoint identities, empty rows).  The last
test plants mistakes in copies of the oracle and checks that a pin fails for
each of them.
"""
import json
import os

import numpy as np
import pytest
import scipy.sparse as sp

import oracle
import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def int_case(M, N, K, b, nnz, seed, **kw):
    return synth.random_case(M, N, K, b, nnz, seed, integer_values=True, **kw)


def as_int(bits):
    return synth.bits_to_f32(bits).astype(np.int64)


def brute_forward(X, W, mask, b):
    """Python-int forward, looping only over kept blocks' entries."""
    Xi, Wi = as_int(X).tolist(), as_int(W).tolist()
    M, K = len(Xi), len(Xi[0])
    N = len(Wi)
    Y = [[0] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            s = 0
            for k in range(K):
                if mask[n // b][k // b]:
                    s += Xi[m][k] * Wi[n][k]
            Y[m][n] = s
    return np.array(Y, dtype=np.int64)


def brute_backward_input(dY, W, mask, b):
    dYi, Wi = as_int(dY).tolist(), as_int(W).tolist()
    M, N = len(dYi), len(dYi[0])
    K = len(Wi[0])
    out = [[0] * K for _ in range(M)]
    for m in range(M):
        for k in range(K):
            s = 0
            for n in range(N):
                if mask[n // b][k // b]:
                    s += dYi[m][n] * Wi[n][k]
            out[m][k] = s
    return np.array(out, dtype=np.int64)


def brute_backward_weight(dY, X, mask, b):
    dYi, Xi = as_int(dY).tolist(), as_int(X).tolist()
    M = len(dYi)
    R, C = len(mask), len(mask[0])
    blocks = []
    for r in range(R):
        for c in range(C):
            if mask[r][c]:
                blk = [[sum(dYi[m][r * b + u] * Xi[m][c * b + v] for m in range(M))
                        for v in range(b)] for u in range(b)]
                blocks.append(blk)
    return np.array(blocks, dtype=np.int64).reshape(-1, b, b)


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("M,N,K,b,nnz,seed", [
    (5, 8, 12, 4, 3, 0), (7, 12, 8, 2, 11, 1), (3, 6, 6, 3, 2, 2), (9, 16, 24, 4, 10, 3),
])
def test_forward_matches_integer_brute_force(oracle_lib, M, N, K, b, nnz, seed):
    case = int_case(M, N, K, b, nnz, seed)
    Y, _ = oracle.forward(case["X"], case["W"], case["mask"], b)
    assert np.array_equal(Y, brute_forward(case["X"], case["W"], case["mask"].tolist(), b))


@pytest.mark.parametrize("M,N,K,b,nnz,seed", [(5, 8, 12, 4, 3, 4), (6, 12, 8, 2, 9, 5)])
def test_backward_input_matches_integer_brute_force(oracle_lib, M, N, K, b, nnz, seed):
    case = int_case(M, N, K, b, nnz, seed)
    dX, _ = oracle.backward_input(case["dY"], case["W"], case["mask"], b)
    assert np.array_equal(dX, brute_backward_input(case["dY"], case["W"], case["mask"].tolist(), b))


@pytest.mark.parametrize("M,N,K,b,nnz,seed", [(5, 8, 12, 4, 3, 6), (11, 12, 8, 2, 9, 7)])
def test_backward_weight_matches_integer_brute_force(oracle_lib, M, N, K, b, nnz, seed):
    case = int_case(M, N, K, b, nnz, seed)
    dW, _ = oracle.backward_weight(case["dY"], case["X"], case["mask"], b)
    assert np.array_equal(dW, brute_backward_weight(case["dY"], case["X"], case["mask"].tolist(), b))


def test_abs_sums_match_integer_brute_force(oracle_lib):
    case = int_case(4, 8, 8, 4, 2, 8)
    X, W, mask = case["X"], case["W"], case["mask"]
    _, A = oracle.forward(X, W, mask, 4)
    Xi, Wi = as_int(X), as_int(W)
    keep = np.kron(mask, np.ones((4, 4), dtype=np.int64))
    want = np.array([[int(sum(abs(int(Xi[m, k]) * int(Wi[n, k])) for k in range(8) if keep[n, k]))
                      for n in range(8)] for m in range(4)])
    assert np.array_equal(A, want)


# -------------------------------------------------- library routines at d = 1

def test_density_one_equals_numpy_matmul(oracle_lib):
    rng = np.random.default_rng(11)
    M, N, K, b = 33, 64, 96, 32
    X = synth.bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    W = synth.bf16_bits(rng.standard_normal((N, K), dtype=np.float32))
    dY = synth.bf16_bits(rng.standard_normal((M, N), dtype=np.float32))
    mask = np.ones((N // b, K // b), dtype=np.uint8)
    Xf, Wf, dYf = (synth.bits_to_f32(a).astype(np.float64) for a in (X, W, dY))
    Y, _ = oracle.forward(X, W, mask, b)
    np.testing.assert_allclose(Y, Xf @ Wf.T, rtol=1e-12, atol=1e-12)
    dX, _ = oracle.backward_input(dY, W, mask, b)
    np.testing.assert_allclose(dX, dYf @ Wf, rtol=1e-12, atol=1e-12)
    dW, _ = oracle.backward_weight(dY, X, mask, b)
    full = dYf.T @ Xf
    R, C = N // b, K // b
    want = full.reshape(R, b, C, b).transpose(0, 2, 1, 3).reshape(R * C, b, b)
    np.testing.assert_allclose(dW, want, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------- pack

def test_pack_matches_scipy_bsr_and_csc(oracle_lib):
    rng = np.random.default_rng(12)
    b, R, C = 4, 9, 7
    mask = synth.mask_uniform(R, C, 23, rng)
    mask[3, :] = 0                      # an empty block row
    mask[:, 5] = 0                      # an empty block column
    mask[6, :] = 1                      # a full block row
    W = synth.bf16_bits(rng.standard_normal((R * b, C * b), dtype=np.float32))
    pk = oracle.pack(W, mask, b)
    Wf = synth.bits_to_f32(W) * np.kron(mask, np.ones((b, b), dtype=np.float32))
    bsr = sp.bsr_matrix(Wf, blocksize=(b, b))
    bsr.sort_indices()
    assert np.array_equal(pk["row_ptr"], bsr.indptr)
    assert np.array_equal(pk["col_idx"], bsr.indices)
    assert np.array_equal(synth.bits_to_f32(pk["values"]), bsr.data)
    pos = sp.csr_matrix((np.arange(1, pk["nnz"] + 1), pk["col_idx"], pk["row_ptr"]), shape=(R, C))
    csc = pos.tocsc()
    csc.sort_indices()
    assert np.array_equal(pk["col_ptr"], csc.indptr)
    assert np.array_equal(pk["row_idx"], csc.indices)
    assert np.array_equal(pk["csc_to_bsr"], csc.data - 1)


def test_pack_closed_forms_and_4x_saving(oracle_lib):
    with open(os.path.join(HERE, "golden", "memory_saving_75pct_sparse.json")) as f:
        gold = json.load(f)
    for R, C, b, seed in [(12, 8, 4, 0), (96, 24, 2, 1), (16, 16, 8, 2)]:
        nnz = synth.round_half_even(gold["density"] * R * C)
        mask = synth.mask_uniform(R, C, nnz, np.random.default_rng(seed))
        W = synth.bf16_bits(np.random.default_rng(seed).standard_normal((R * b, C * b),
                                                                        dtype=np.float32))
        pk = oracle.pack(W, mask, b)
        assert pk["values"].size == nnz * b * b
        assert W.nbytes / pk["values"].nbytes == gold["dense_bytes_over_packed_value_bytes"]
        assert pk["row_ptr"][-1] == nnz and pk["col_ptr"][-1] == nnz
        assert sorted(pk["csc_to_bsr"].tolist()) == list(range(nnz))
        for c in range(C):       # every CSC entry points at a block in column c of row row_idx
            for j in range(pk["col_ptr"][c], pk["col_ptr"][c + 1]):
                p = pk["csc_to_bsr"][j]
                r = pk["row_idx"][j]
                assert pk["col_idx"][p] == c and pk["row_ptr"][r] <= p < pk["row_ptr"][r + 1]


def test_schedule_order_matches_lexsort(oracle_lib):
    rng = np.random.default_rng(13)
    counts = rng.integers(0, 6, size=50)
    ptr = np.concatenate([[0], np.cumsum(counts)])
    want = np.lexsort((np.arange(50), -counts))
    assert np.array_equal(oracle.schedule_order(ptr), want)


# --------------------------------------------------------------- invariants

def _permute_block_cols(a, perm, b):
    n = a.shape[1] // b
    return a.reshape(a.shape[0], n, b)[:, perm, :].reshape(a.shape)


def test_block_column_permutation_leaves_forward_unchanged(oracle_lib):
    b = 4
    case = int_case(6, 16, 20, b, 9, 21)
    perm = np.random.default_rng(0).permutation(5)
    Y0, _ = oracle.forward(case["X"], case["W"], case["mask"], b)
    Y1, _ = oracle.forward(_permute_block_cols(case["X"], perm, b),
                           _permute_block_cols(case["W"], perm, b),
                           case["mask"][:, perm], b)
    assert np.array_equal(Y0, Y1)


def test_block_row_permutation_permutes_output_blocks(oracle_lib):
    b = 4
    case = int_case(6, 24, 12, b, 8, 22)
    perm = np.random.default_rng(1).permutation(6)
    W1 = case["W"].reshape(6, b, 12)[perm].reshape(24, 12)
    Y0, _ = oracle.forward(case["X"], case["W"], case["mask"], b)
    Y1, _ = oracle.forward(case["X"], W1, case["mask"][perm], b)
    assert np.array_equal(Y1, Y0.reshape(6, 6, b)[:, perm, :].reshape(6, 24))


def test_adjoint_identities_exact_on_integers(oracle_lib):
    b = 4
    case = int_case(7, 16, 12, b, 6, 23)
    X, W, dY, mask = case["X"], case["W"], case["dY"], case["mask"]
    Y, _ = oracle.forward(X, W, mask, b)
    dX, _ = oracle.backward_input(dY, W, mask, b)
    dW, _ = oracle.backward_weight(dY, X, mask, b)
    pk = oracle.pack(W, mask, b)
    a = int(np.sum(as_int(dY) * Y.astype(np.int64)))
    bb = int(np.sum(as_int(X) * dX.astype(np.int64)))
    c = int(np.sum(synth.bits_to_f32(pk["values"]).astype(np.int64) * dW.astype(np.int64)))
    assert a == bb == c


def test_adjoint_identities_on_seeded_floats(oracle_lib):
    b = 32
    case = synth.random_case(48, 96, 128, b, 5, 24)
    X, W, dY, mask = case["X"], case["W"], case["dY"], case["mask"]
    Y, _ = oracle.forward(X, W, mask, b)
    dX, _ = oracle.backward_input(dY, W, mask, b)
    dW, _ = oracle.backward_weight(dY, X, mask, b)
    pk = oracle.pack(W, mask, b)
    a = np.sum(oracle.widen(dY) * Y)
    bb = np.sum(oracle.widen(X) * dX)
    c = np.sum(oracle.widen(pk["values"]) * dW)
    assert abs(a - bb) <= 1e-10 * abs(a) and abs(a - c) <= 1e-10 * abs(a)


def test_empty_rows_and_columns_give_exact_zeros(oracle_lib):
    b = 4
    case = synth.random_case(5, 16, 16, b, 10, 25, empty_rows=(1,), empty_cols=(2,))
    Y, A = oracle.forward(case["X"], case["W"], case["mask"], b)
    assert np.all(Y[:, 4:8] == 0) and np.all(A[:, 4:8] == 0)
    dX, A = oracle.backward_input(case["dY"], case["W"], case["mask"], b)
    assert np.all(dX[:, 8:12] == 0) and np.all(A[:, 8:12] == 0)


def test_row_subset_equals_full(oracle_lib):
    case = synth.random_case(40, 64, 64, 32, 3, 26)
    Yf, _ = oracle.forward(case["X"], case["W"], case["mask"], 32)
    Ys, _ = oracle.forward(case["X"], case["W"], case["mask"], 32, rows=[39, 0, 17])
    assert np.array_equal(Ys, Yf[[39, 0, 17]])
    dXf, _ = oracle.backward_input(case["dY"], case["W"], case["mask"], 32)
    dXs, _ = oracle.backward_input(case["dY"], case["W"], case["mask"], 32, rows=[5, 38])
    assert np.array_equal(dXs, dXf[[5, 38]])


def test_blockskip_forward_is_bit_identical_and_matches_brute_force(oracle_lib):
    """The block-skipping forward (the CPU baseline that does only the stored
    blocks' work) must give the dense-with-zeros result bit for bit, and the
    exact integer result on integer inputs."""
    b = 4
    case = int_case(6, 16, 20, b, 9, 28)
    got, A = oracle.forward_blockskip(case["X"], case["W"], case["mask"], b)
    assert np.array_equal(got, brute_forward(case["X"], case["W"], case["mask"].tolist(), b))
    case = synth.random_case(9, 256, 320, 32, 23, 29, empty_rows=(2,))
    want, wa = oracle.forward(case["X"], case["W"], case["mask"], 32)
    got, ga = oracle.forward_blockskip(case["X"], case["W"], case["mask"], 32)
    assert np.array_equal(got, want) and np.array_equal(ga, wa)


def test_bias_matches_integer_brute_force(oracle_lib):
    """Y = X Wt^T + bias and dbias = column sums of dY, against Python ints."""
    b = 4
    case = int_case(6, 16, 12, b, 5, 30)
    bias = synth.bf16_bits(np.random.default_rng(30).integers(-3, 4, size=16).astype(np.float32))
    Y, A = oracle.forward(case["X"], case["W"], case["mask"], b, bias=bias)
    want = brute_forward(case["X"], case["W"], case["mask"].tolist(), b) + as_int(bias)[None, :]
    assert np.array_equal(Y, want)
    Y0, A0 = oracle.forward(case["X"], case["W"], case["mask"], b)
    assert np.array_equal(A, A0 + np.abs(as_int(bias))[None, :])
    dYi = as_int(case["dY"])[:, :16]
    db, dba = oracle.bias_grad(case["dY"][:, :16].copy())
    assert db.tolist() == [sum(int(dYi[m][n]) for m in range(6)) for n in range(16)]
    assert dba.tolist() == [sum(abs(int(dYi[m][n])) for m in range(6)) for n in range(16)]


def test_bias_adjoint_identity(oracle_lib):
    """<dY, Y(bias)> = <dY, Y(0)> + <dbias, bias>: pins the bias term and its
    gradient against each other (exact on integers)."""
    b = 4
    case = int_case(7, 12, 8, b, 4, 31)
    bias = synth.bf16_bits(np.random.default_rng(31).integers(-3, 4, size=12).astype(np.float32))
    dY = case["dY"][:, :12].copy()
    Yb, _ = oracle.forward(case["X"], case["W"], case["mask"], b, bias=bias)
    Y0, _ = oracle.forward(case["X"], case["W"], case["mask"], b)
    db, _ = oracle.bias_grad(dY)
    dyd = oracle.widen(dY)
    assert float((dyd * Yb).sum()) == float((dyd * Y0).sum()) + float((db * oracle.widen(bias)).sum())


# ----------------------------------------------------------- planted mistakes

def _mutants():
    """Copies of the oracle's forward with one plausible mistake each."""
    def transposed_mask(X, W, mask, b):
        n, k = W.shape
        return oracle.forward(X, W, mask.T.copy() if mask.shape[0] == mask.shape[1] else mask[::-1].copy(), b)[0]

    def mask_ignored(X, W, mask, b):
        return oracle.forward(X, W, np.ones_like(mask), b)[0]

    def last_block_dropped(X, W, mask, b):
        m = mask.copy()
        r, c = np.argwhere(m)[-1]
        m[r, c] = 0
        return oracle.forward(X, W, m, b)[0]

    def sign_flipped(X, W, mask, b):
        return -oracle.forward(X, W, mask, b)[0]

    def operand_shifted(X, W, mask, b):
        Xs = np.roll(X, 1, axis=1)
        return oracle.forward(Xs, W, mask, b)[0]

    return [transposed_mask, mask_ignored, last_block_dropped, sign_flipped, operand_shifted]


def _bias_mutants():
    """Copies of the oracle's biased forward with one plausible mistake each."""
    def bias_ignored(X, W, mask, b, bias):
        return oracle.forward(X, W, mask, b)[0]

    def bias_reversed(X, W, mask, b, bias):
        return oracle.forward(X, W, mask, b, bias=bias[::-1].copy())[0]

    def bias_twice(X, W, mask, b, bias):
        Y, _ = oracle.forward(X, W, mask, b, bias=bias)
        return Y + oracle.widen(bias)[None, :]

    return [bias_ignored, bias_reversed, bias_twice]


@pytest.mark.parametrize("mutant", _bias_mutants(), ids=lambda f: f.__name__)
def test_bias_pin_catches_planted_mistakes(oracle_lib, mutant):
    b = 4
    case = int_case(5, 16, 16, b, 7, 32)
    bias = synth.bf16_bits(np.arange(-8, 8).astype(np.float32))
    want = brute_forward(case["X"], case["W"], case["mask"].tolist(), b) + as_int(bias)[None, :]
    assert np.array_equal(oracle.forward(case["X"], case["W"], case["mask"], b, bias=bias)[0], want)
    assert not np.array_equal(mutant(case["X"], case["W"], case["mask"], b, bias), want)


@pytest.mark.parametrize("mutant", _mutants(), ids=lambda f: f.__name__)
def test_pins_catch_planted_mistakes(oracle_lib, mutant):
    b = 4
    case = int_case(5, 16, 16, b, 7, 27)
    want = brute_forward(case["X"], case["W"], case["mask"].tolist(), b)
    assert np.array_equal(oracle.forward(case["X"], case["W"], case["mask"], b)[0], want)
    assert not np.array_equal(mutant(case["X"], case["W"], case["mask"], b), want)
