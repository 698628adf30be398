"""Pins for the oracle's 2:4 semi-structured functions (no GPU).

The compressed form (torchao sparsity README, Table 4.1, row "NVIDIA 2:4
compressed representation") is checked against a brute-force enumeration
written here: for each group of four, the kept pair is the smallest
ascending pair of positions (in lexicographic order) that contains every
nonzero position, which is an independent statement of "the nonzeros,
completed by the lowest-indexed zeros".  The product is checked against
Python-int arithmetic on the dense weight the compressed form came from and
against numpy's matmul.  Planted mistakes in the compressed form must fail
the brute-force pin.
"""
import itertools

import numpy as np
import pytest

import oracle
import synth

PAIRS = [(i0, i1) for i0, i1 in itertools.combinations(range(4), 2)]  # lexicographic


def brute_compress(W):
    """Plain loops: kept pair = smallest ascending pair covering the nonzeros."""
    N, K = W.shape
    values = np.zeros((N, K // 2), dtype=np.uint16)
    meta = np.zeros((N, K // 16), dtype=np.uint16)
    for n in range(N):
        for g in range(K // 4):
            grp = [int(W[n, 4 * g + i]) for i in range(4)]
            nonzero = {i for i in range(4) if grp[i] & 0x7FFF}
            pair = next(p for p in PAIRS if nonzero <= set(p))
            values[n, 2 * g] = grp[pair[0]]
            values[n, 2 * g + 1] = grp[pair[1]]
            meta[n, g // 4] |= (pair[0] + 4 * pair[1]) << (4 * (g % 4))
    return values, meta


def seeded_w(N, K, seed, **kw):
    return synth.semi24_weight(N, K, np.random.default_rng(seed), **kw)


@pytest.mark.parametrize("N,K,fewer,seed", [(3, 16, 0.0, 1), (5, 64, 0.4, 2), (8, 48, 0.8, 3),
                                            (2, 32, 1.0, 4)])
def test_compress_matches_brute_force(N, K, fewer, seed):
    W = seeded_w(N, K, seed, fewer=fewer)
    v, m = oracle.compress24(W)
    bv, bm = brute_compress(W)
    assert np.array_equal(v, bv)
    assert np.array_equal(m, bm)


def test_hand_worked_groups():
    # one row, four groups: nonzeros at {0, 3}; none; {2} with -0 at 1; {3}
    W = np.array([[0x3F80, 0, 0, 0x4000, 0, 0, 0, 0, 0, 0x8000, 0x3F80, 0, 0, 0, 0, 0x4040]],
                 dtype=np.uint16)
    v, m = oracle.compress24(W)
    assert v.tolist() == [[0x3F80, 0x4000, 0, 0, 0, 0x3F80, 0, 0x4040]]
    # pairs (0,3), (0,1), (0,2), (0,3) -> codes 0xC, 0x4, 0x8, 0xC, group j at bits 4j
    assert m.tolist() == [[0xC | 0x4 << 4 | 0x8 << 8 | 0xC << 12]]


def test_codes_are_ascending_pairs_and_storage_is_nine_sixteenths():
    N, K = 16, 256
    W = seeded_w(N, K, 7, fewer=0.3)
    v, m = oracle.compress24(W)
    valid = {i0 | i1 << 2 for i0, i1 in PAIRS}
    nibbles = {(int(x) >> (4 * j)) & 0xF for x in m.ravel() for j in range(4)}
    assert nibbles <= valid
    # half the elements plus 2 bits per kept element (Table 4.1's "half the size" + "2bit indices")
    assert v.shape == (N, K // 2) and m.shape == (N, K // 16)
    assert v.nbytes + m.nbytes == W.nbytes * 9 // 16


def test_round_trip():
    W = seeded_w(12, 128, 8)  # no signed zeros: bit-exact round trip
    assert np.array_equal(oracle.decompress24(*oracle.compress24(W)), W)
    Wz = seeded_w(12, 128, 9, fewer=0.5)  # dropped -0 comes back as +0: equal values
    back = oracle.decompress24(*oracle.compress24(Wz))
    assert np.array_equal(oracle.widen(back), oracle.widen(Wz))


@pytest.mark.parametrize("count", [3, 4])
def test_rejects_groups_with_more_than_two_nonzeros(count):
    W = seeded_w(4, 32, 10)
    W[2, 8:12] = 0
    W[2, 8:8 + count] = 0x3F80
    with pytest.raises(ValueError, match="not 2:4"):
        oracle.compress24(W)


def test_forward_equals_integer_product_with_the_dense_weight(oracle_lib):
    rng = np.random.default_rng(11)
    M, N, K = 5, 7, 64
    W = synth.semi24_weight(N, K, rng, fewer=0.3, integer_values=True)
    X = synth.bf16_bits(rng.integers(-3, 4, size=(M, K)).astype(np.float32))
    bias = synth.bf16_bits(rng.integers(-3, 4, size=N).astype(np.float32))
    v, m = oracle.compress24(W)
    Y, _ = oracle.semi24_forward(X, v, m, bias=bias)
    Xi = synth.bits_to_f32(X).astype(np.int64).tolist()
    Wi = synth.bits_to_f32(W).astype(np.int64).tolist()
    bi = synth.bits_to_f32(bias).astype(np.int64).tolist()
    want = [[sum(Xi[i][k] * Wi[n][k] for k in range(K)) + bi[n] for n in range(N)] for i in range(M)]
    assert np.array_equal(Y, np.asarray(want, dtype=np.float64))


def test_forward_equals_numpy_matmul(oracle_lib):
    rng = np.random.default_rng(12)
    M, N, K = 9, 24, 96
    W = synth.semi24_weight(N, K, rng, std=0.2)
    X = synth.bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    Y, A = oracle.semi24_forward(X, *oracle.compress24(W), rows=np.arange(2, 9))
    ref = synth.bits_to_f32(X).astype(np.float64) @ synth.bits_to_f32(W).astype(np.float64).T
    assert np.allclose(Y, ref[2:9], rtol=0, atol=1e-12)
    assert np.all(A >= np.abs(Y))


MUTANTS = {
    "nibble fields swapped": lambda v, m: (v, ((m & 0x3333) << 2 | (m & 0xCCCC) >> 2).astype(np.uint16)),
    "group order reversed": lambda v, m: (v, (
        (m & 0xF) << 12 | (m & 0xF0) << 4 | (m & 0xF00) >> 4 | (m & 0xF000) >> 12).astype(np.uint16)),
    "kept values swapped": lambda v, m: (v.reshape(v.shape[0], -1, 2)[:, :, ::-1].reshape(v.shape), m),
    "pad with the highest zeros": None,
}


def pad_high(W):
    """Mutant compressor: complete short groups with the highest zeros."""
    N, K = W.shape
    v = np.zeros((N, K // 2), dtype=np.uint16)
    m = np.zeros((N, K // 16), dtype=np.uint16)
    for n in range(N):
        for g in range(K // 4):
            grp = [int(W[n, 4 * g + i]) for i in range(4)]
            keep = [i for i in range(4) if grp[i] & 0x7FFF]
            for i in (3, 2, 1, 0):
                if len(keep) < 2 and i not in keep:
                    keep.append(i)
            keep.sort()
            v[n, 2 * g:2 * g + 2] = [grp[keep[0]], grp[keep[1]]]
            m[n, g // 4] |= (keep[0] | keep[1] << 2) << (4 * (g % 4))
    return v, m


@pytest.mark.parametrize("name", list(MUTANTS))
def test_brute_force_pin_catches_planted_mistakes(name):
    W = seeded_w(6, 64, 13, fewer=0.4)
    if MUTANTS[name] is None:
        v, m = pad_high(W)
    else:
        v, m = MUTANTS[name](*oracle.compress24(W))
    bv, bm = brute_compress(W)
    assert not (np.array_equal(v, bv) and np.array_equal(m, bm))


def test_block_compression_is_the_dense_compression_restricted_to_blocks():
    """For a block-sparse weight with 2:4 along K (b a multiple of 16), the
    compressed form of each kept block is the matching slice of the
    compressed form of the whole weight with zeros outside the blocks."""
    b, R, C = 16, 3, 4
    rng = np.random.default_rng(14)
    W = synth.semi24_weight(R * b, C * b, rng, fewer=0.3)
    mask = synth.mask_uniform(R, C, 7, rng)
    packed = oracle.pack(W, mask, b)
    v, m = oracle.compress24_blocks(packed["values"])
    Wz = W.copy()
    for r in range(R):
        for c in range(C):
            if not mask[r, c]:
                Wz[r * b:(r + 1) * b, c * b:(c + 1) * b] = 0
    dv, dm = oracle.compress24(Wz)
    p = 0
    for r in range(R):
        for c in range(C):
            if mask[r, c]:
                assert np.array_equal(v[p], dv[r * b:(r + 1) * b, c * b // 2:(c + 1) * b // 2])
                assert np.array_equal(m[p], dm[r * b:(r + 1) * b, c * b // 16:(c + 1) * b // 16])
                p += 1
    assert p == packed["nnz"]
