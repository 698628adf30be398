"""GPU parity of the block-sparse layer with 2:4 inside its blocks.

The compressed blocks must match the oracle bit for bit (block by block, the
zero block after them); the forward must match the oracle's block-sparse
product (the dense product with zeros outside the kept blocks) element by
element within the bound of tests/_parity.py.  Cases, for block sizes 64
and 32: one token, ragged token tiles (224 tokens per tile), empty block rows
(a group without entries, whose rows must come out as the bias alone), a
block-row count that leaves the last group short, more tiles than SMs, and
the full workload on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu import bits, mask_dev, to_dev, to_f64
from _parity import assert_parity

pytestmark = pytest.mark.gpu

sg = pytest.importorskip("sparse_gemm_b200")


def case(M, N, K, nnz, seed, *, b=64, empty_rows=(), fewer=0.2):
    rng = np.random.default_rng(seed)
    mask = synth.mask_uniform(N // b, K // b, nnz, rng)
    for r in empty_rows:
        mask[r, :] = 0
    W = synth.semi24_weight(N, K, rng, std=(2.0 / K) ** 0.5, fewer=fewer)
    X = synth.bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    bias = synth.bf16_bits(rng.standard_normal(N).astype(np.float32))
    return X, W, mask, bias


def run(X, W, mask, bias=None, b=64):
    Wp = sg.pack(to_dev(W), mask_dev(mask), b)
    w24 = sg.compress_bsr24(Wp)
    Y = sg.forward_bsr24(to_dev(X), w24, bias=None if bias is None else to_dev(bias))
    torch.cuda.synchronize()
    assert sg.device_status(Wp) == 0
    return Wp, w24, Y


def check_blocks(W, mask, w24, b=64):
    packed = oracle.pack(W, mask, b)
    v, m = oracle.compress24_blocks(packed["values"])
    nnz = packed["nnz"]
    got_v = bits(w24.values)
    assert np.array_equal(got_v[:nnz], v)
    assert not got_v[nnz].any()  # the zero block
    if nnz:
        assert np.array_equal(w24.meta.cpu().numpy().view(np.uint16)[:nnz], m)


FWD_CASES = [
    # b, M, N, K, nnz, bias, empty block rows, seed
    (64, 1, 256, 256, 5, False, (), 30),
    (64, 225, 512, 384, 20, True, (), 31),
    (64, 300, 640, 1024, 40, True, (0, 1, 6), 32),  # block rows 0 and 1 form an empty group
    (64, 448, 320, 512, 12, False, (), 33),         # 5 block rows: the last group has one member
    (64, 5000, 1024, 512, 60, True, (), 34),        # 8 groups x 23 token tiles > SMs
    (32, 1, 128, 128, 5, False, (), 40),
    (32, 225, 512, 384, 60, True, (), 41),
    (32, 300, 640, 1024, 120, True, (0, 1, 2, 3, 9), 42),  # rows 0-3: an empty group of four
    (32, 448, 224, 512, 30, False, (), 43),         # 7 block rows: the last group has three members
    (32, 5000, 2048, 256, 200, True, (), 44),       # 16 groups x 23 token tiles > SMs
]


@pytest.mark.parametrize("b,M,N,K,nnz,with_bias,empty,seed", FWD_CASES)
def test_forward_parity(b, M, N, K, nnz, with_bias, empty, seed):
    X, W, mask, bias = case(M, N, K, nnz, seed, b=b, empty_rows=empty)
    Wp, w24, Y = run(X, W, mask, bias if with_bias else None, b=b)
    check_blocks(W, mask, w24, b=b)
    ref, refabs = oracle.forward(X, W, mask, b, bias=bias if with_bias else None)
    assert_parity(to_f64(Y), ref, refabs, f"2:4-block forward b={b} M={M} N={N} K={K} nnz={nnz}")


def test_compress_reports_groups_with_more_than_two_nonzeros():
    X, W, mask, _ = case(8, 256, 256, 6, 35)
    r, c = np.argwhere(mask)[0]
    W[r * 64 + 3, c * 64 + 8:c * 64 + 12] = [0x3F80, 0x4000, 0xBF80, 0]
    Wp = sg.pack(to_dev(W), mask_dev(mask), 64)
    sg.compress_bsr24(Wp)
    assert sg.device_status(Wp) == 8  # BSL_ERR_NOT_2_4


def test_deterministic_and_replays_from_a_cuda_graph():
    X, W, mask, bias = case(700, 768, 1024, 50, 37)
    Wp = sg.pack(to_dev(W), mask_dev(mask), 64)
    w24 = sg.compress_bsr24(Wp)
    Xd, bd = to_dev(X), to_dev(bias)
    Y1 = sg.forward_bsr24(Xd, w24, bias=bd)
    Y2 = sg.forward_bsr24(Xd, w24, bias=bd)
    assert torch.equal(Y1, Y2)
    out = torch.empty_like(Y1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        sg.forward_bsr24(Xd, w24, bias=bd, out=out)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            sg.forward_bsr24(Xd, w24, bias=bd, out=out)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, Y1)
    assert sg.device_status(Wp) == 0


def test_full_workload_sampled_rows():
    wl = synth.BSR24_WORKLOADS["bsr24_fwd"]
    inp = synth.make_bsr24_inputs(wl)
    X, W, mask = inp["X"], inp["W"], inp["mask"]
    Wp, w24, Y = run(X, W, mask)
    check_blocks(W, mask, w24)
    rows = sorted({r for t in range(0, wl.M, 224) for r in (t, min(t + 223, wl.M - 1))})
    ref, refabs = oracle.forward(X, W, mask, wl.b, rows=np.asarray(rows))
    assert_parity(to_f64(Y[rows]), ref, refabs, "2:4-block forward, full size, sampled rows")


@pytest.mark.parametrize("b", [64, 32])
def test_weight_without_blocks_gives_the_bias_exactly(b):
    """Degenerate mask: no kept block, so every group is empty and the forward
    writes the bias alone (exactly) without any MMA."""
    M, N, K = 300, 256, 256
    X, W, mask, bias = case(M, N, K, 1, 45, b=b)
    mask[:] = 0
    Wp, w24, Y = run(X, W, mask, bias, b=b)
    assert Wp.nnz == 0
    assert np.array_equal(bits(Y), np.broadcast_to(bias, (M, N)))
