"""GPU parity of the 2:4 semi-structured path against the fp64 oracle.

The compressed form (values and positions) must match the oracle bit for
bit; the forward must match the oracle's product element by element within
the bound of tests/_parity.py.  Shapes span several tiles (256 features x
224 tokens) with ragged tails, one token, more tiles than SMs (so a CTA
walks several tiles and the rings wrap), and the full workload size on
sampled rows (the first and last token of every 224-token tile).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu import bits, to_dev, to_f64
from _parity import assert_parity

pytestmark = pytest.mark.gpu

sg = pytest.importorskip("sparse_gemm_b200")


def case(M, N, K, seed, *, fewer=0.2, integer_values=False):
    rng = np.random.default_rng(seed)
    W = synth.semi24_weight(N, K, rng, std=(2.0 / K) ** 0.5, fewer=fewer, integer_values=integer_values)
    if integer_values:
        X = synth.bf16_bits(rng.integers(-3, 4, size=(M, K)).astype(np.float32))
    else:
        X = synth.bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    bias = synth.bf16_bits(rng.standard_normal(N).astype(np.float32))
    return X, W, bias


def check_compress(W, w):
    v, m = oracle.compress24(W)
    assert np.array_equal(bits(w.values), v)
    assert np.array_equal(w.meta.cpu().numpy().view(np.uint16), m)
    assert sg.semi24_status(w) == 0


@pytest.mark.parametrize("N,K,fewer,seed", [(8, 64, 0.0, 1), (136, 320, 0.3, 2), (1000, 1024, 0.9, 3)])
def test_compress_bit_exact(N, K, fewer, seed):
    W = synth.semi24_weight(N, K, np.random.default_rng(seed), fewer=fewer)
    check_compress(W, sg.compress24(to_dev(W)))


def test_compress_reports_groups_with_more_than_two_nonzeros():
    W = synth.semi24_weight(64, 128, np.random.default_rng(4))
    W[17, 40:44] = [0x3F80, 0x4000, 0xBF80, 0]
    w = sg.compress24(to_dev(W))
    assert sg.semi24_status(w) == 8  # BSL_ERR_NOT_2_4
    assert sg.semi24_status(w) == 0  # read and cleared
    # every other row is still compressed as the oracle does
    W2 = W.copy()
    W2[17] = 0
    v, m = oracle.compress24(W2)
    rows = [r for r in range(64) if r != 17]
    assert np.array_equal(bits(w.values)[rows], v[rows])


FWD_CASES = [
    # M, N, K, bias, seed
    (1, 8, 64, False, 10),
    (5, 200, 128, True, 11),
    (224, 256, 64, False, 12),
    (225, 264, 192, True, 13),
    (400, 520, 320, True, 14),
    (700, 1032, 1024, False, 15),   # 16 stages per tile: the metadata ring wraps
    (3400, 2560, 128, True, 16),    # 160 tiles: CTAs walk several tiles
]


@pytest.mark.parametrize("M,N,K,with_bias,seed", FWD_CASES)
def test_forward_parity(M, N, K, with_bias, seed):
    X, W, bias = case(M, N, K, seed)
    w = sg.compress24(to_dev(W))
    Y = sg.forward24(to_dev(X), w, bias=to_dev(bias) if with_bias else None)
    torch.cuda.synchronize()
    assert sg.semi24_status(w) == 0
    v, m = oracle.compress24(W)
    ref, refabs = oracle.semi24_forward(X, v, m, bias=bias if with_bias else None)
    assert_parity(to_f64(Y), ref, refabs, f"semi24 forward M={M} N={N} K={K}")


def test_forward_exact_on_integers():
    """Integer values: fp32 accumulation is exact, so Y is the exact product
    rounded once to bf16."""
    M, N, K = 300, 392, 256
    X, W, _ = case(M, N, K, 20, integer_values=True, fewer=0.3)
    w = sg.compress24(to_dev(W))
    Y = sg.forward24(to_dev(X), w)
    ref, _ = oracle.semi24_forward(X, *oracle.compress24(W))
    want = torch.from_numpy(ref).to(torch.float32).to(torch.bfloat16)
    assert torch.equal(Y.cpu(), want)


def test_forward_is_deterministic_and_replays_from_a_cuda_graph():
    M, N, K = 520, 776, 512
    X, W, bias = case(M, N, K, 21)
    w = sg.compress24(to_dev(W))
    Xd, bd = to_dev(X), to_dev(bias)
    Y1 = sg.forward24(Xd, w, bias=bd)
    Y2 = sg.forward24(Xd, w, bias=bd)
    assert torch.equal(Y1, Y2)
    out = torch.empty_like(Y1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        sg.forward24(Xd, w, bias=bd, out=out)  # warm-up outside the capture
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            sg.forward24(Xd, w, bias=bd, out=out)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, Y1)
    assert sg.semi24_status(w) == 0


def test_full_workload_sampled_rows():
    wl = synth.SEMI24_WORKLOADS["semi24_fwd"]
    inp = synth.make_semi24_inputs(wl)
    X, W = inp["X"], inp["W"]
    w = sg.compress24(to_dev(W))
    check_compress(W, w)
    Y = sg.forward24(to_dev(X), w)
    torch.cuda.synchronize()
    assert sg.semi24_status(w) == 0
    rows = sorted({r for t in range(0, wl.M, 224) for r in (t, min(t + 223, wl.M - 1))})
    v, m = oracle.compress24(W)
    ref, refabs = oracle.semi24_forward(X, v, m, rows=np.asarray(rows))
    assert_parity(to_f64(Y[rows]), ref, refabs, "semi24 forward, full size, sampled rows")


def test_semi24_linear_module():
    """The inference module: leading dimensions kept, bias added, output equal
    to the oracle within the bound; a weight that is not 2:4 is refused."""
    rng = np.random.default_rng(22)
    W = synth.semi24_weight(136, 192, rng, std=0.1)
    bias = synth.bf16_bits(rng.standard_normal(136).astype(np.float32))
    X = synth.bf16_bits(rng.standard_normal((2 * 3 * 5, 192)).astype(np.float32))
    mod = sg.Semi24Linear.from_dense(to_dev(W), bias=to_dev(bias))
    y = mod(to_dev(X).reshape(2, 3, 5, 192))
    assert y.shape == (2, 3, 5, 136)
    ref, refabs = oracle.semi24_forward(X, *oracle.compress24(W), bias=bias)
    assert_parity(to_f64(y.reshape(30, 136)), ref, refabs, "Semi24Linear")
    bad = W.copy()
    bad[0, 0:4] = [0x3F80, 0x3F80, 0x3F80, 0]
    with pytest.raises(sg.BslError, match="NOT_2_4"):
        sg.Semi24Linear.from_dense(to_dev(bad))


def test_all_zero_weight_gives_the_bias_exactly():
    """Degenerate weight: every group has no nonzero (kept pair (0, 1) over
    zeros); the output is the bias alone, exactly, or exact zeros."""
    M, N, K = 230, 264, 128
    rng = np.random.default_rng(23)
    W = np.zeros((N, K), dtype=np.uint16)
    X = synth.bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    bias = synth.bf16_bits(rng.standard_normal(N).astype(np.float32))
    w = sg.compress24(to_dev(W))
    check_compress(W, w)
    Y0 = sg.forward24(to_dev(X), w)
    Yb = sg.forward24(to_dev(X), w, bias=to_dev(bias))
    assert not Y0.float().abs().max().item()
    assert np.array_equal(bits(Yb), np.broadcast_to(bias, (M, N)))
