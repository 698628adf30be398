"""Chains of calls on one stream, each consuming the previous call's output.

Every hot kernel may be launched while the kernel before it in the stream is
still finishing, and waits for that grid before touching global memory; a
missing or misplaced wait would let a consumer read its input before the
producer wrote it.  The chain here runs without synchronisation between
calls, eagerly and as a replayed CUDA graph, with every intermediate and
output first filled with NaN, and is compared bit for bit with the same chain
computed by the oracle.

Values are small integers (inputs and weights in {-1, 0, 1}), so every fp32
accumulation on the GPU and every fp64 sum in the oracle is exact, and each
layer's bf16 output is the exact sum rounded once (round to nearest even) on
both sides; the oracle chain rounds its own outputs before the next layer, so
no GPU value ever enters it.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu import bits, mask_dev, to_dev

pytestmark = pytest.mark.gpu

sg = pytest.importorskip("sparse_gemm_b200")

N = K = 256
B = 32
NNZ = 16
NAN = 0x7FC0


def sign_bits(a_bits):
    """bf16 bits -> bf16 bits of sign(value): keeps every zero (2:4 patterns stay)."""
    return synth.bf16_bits(np.sign(synth.bits_to_f32(a_bits)).astype(np.float32))


def exact_bf16(y):
    """fp64 exact integer sums -> bf16 bits, rounded once (RNE)."""
    assert np.abs(y).max() < 2 ** 24, "sums must stay exact in fp32"
    return synth.bf16_bits(y.astype(np.float32))


def make_chain(M, seed):
    rng = np.random.default_rng(seed)
    X0 = synth.bf16_bits(rng.integers(-1, 2, size=(M, K)).astype(np.float32))
    W1 = synth.bf16_bits(rng.integers(-1, 2, size=(N, K)).astype(np.float32))
    m1 = synth.mask_uniform(N // B, K // B, NNZ, rng)
    b1 = synth.bf16_bits(rng.integers(-1, 2, size=N).astype(np.float32))
    S2 = sign_bits(synth.semi24_weight(N, K, rng, integer_values=True, fewer=0.2))
    W3 = sign_bits(synth.semi24_weight(N, K, rng, integer_values=True, fewer=0.2))
    m3 = synth.mask_uniform(N // B, K // B, NNZ, rng)
    return X0, W1, m1, b1, S2, W3, m3


def oracle_chain(X0, W1, m1, b1, S2, W3, m3):
    Y1 = exact_bf16(oracle.forward(X0, W1, m1, B, bias=b1)[0])
    Y2 = exact_bf16(oracle.semi24_forward(Y1, *oracle.compress24(S2))[0])
    Y3 = exact_bf16(oracle.forward(Y2, W3, m3, B)[0])
    dX = exact_bf16(oracle.backward_input(Y1, W1, m1, B)[0])
    dW = exact_bf16(oracle.backward_weight(Y2, X0, m1, B)[0])
    return {"Y1": Y1, "Y2": Y2, "Y3": Y3, "dX": dX, "dW": dW}


@pytest.mark.parametrize("M", [16, 300])  # small-M streaming kernel / tensor-core engine for layer 1
def test_dependent_chain_eager_and_graph(M):
    X0, W1, m1, b1, S2, W3, m3 = make_chain(M, 60 + M)
    want = oracle_chain(X0, W1, m1, b1, S2, W3, m3)

    Wp1 = sg.pack(to_dev(W1), mask_dev(m1), B)
    w2 = sg.compress24(to_dev(S2))
    Wp3 = sg.pack(to_dev(W3), mask_dev(m3), B)
    w3 = sg.compress_bsr24(Wp3)
    Xd, bd = to_dev(X0), to_dev(b1)
    bf = dict(dtype=torch.bfloat16, device=Xd.device)
    out = {"Y1": torch.empty((M, N), **bf), "Y2": torch.empty((M, N), **bf), "Y3": torch.empty((M, N), **bf),
           "dX": torch.empty((M, K), **bf), "dW": torch.empty((Wp1.nnz, B, B), **bf)}

    def chain():
        sg.forward(Xd, Wp1, bias=bd, out=out["Y1"])
        sg.forward24(out["Y1"], w2, out=out["Y2"])
        sg.forward_bsr24(out["Y2"], w3, out=out["Y3"])
        sg.backward_input(out["Y1"], Wp1, out=out["dX"])
        sg.backward_weight(out["Y2"], Xd, Wp1, out=out["dW"])

    def poison():
        for t in out.values():
            t.view(torch.int16).fill_(NAN)

    def check(tag):
        torch.cuda.synchronize()
        for k, v in want.items():
            got = bits(out[k]).reshape(v.shape)
            assert np.array_equal(got, v), f"{tag}: {k} differs from the oracle chain"
        for st in (sg.device_status(Wp1), sg.semi24_status(w2), sg.device_status(Wp3)):
            assert st == 0

    torch.cuda.synchronize()
    poison()
    chain()
    check("eager")

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            chain()
    torch.cuda.current_stream().wait_stream(s)
    for rep in range(3):
        poison()
        g.replay()
        check(f"graph replay {rep}")


@pytest.mark.parametrize("M", [16, 300])
def test_calls_right_after_an_in_place_repack_see_the_new_weight(M):
    """The pack's kernels write the weight and its plans; the contractions
    launched right behind them (no synchronisation) must read what they
    wrote, not the previous pattern."""
    X0, W1, m1, b1, _, _, _ = make_chain(M, 80 + M)
    rng = np.random.default_rng(90 + M)
    m2 = synth.mask_uniform(N // B, K // B, NNZ, rng)  # same block count, new pattern
    assert not np.array_equal(m1, m2)
    W2 = synth.bf16_bits(rng.integers(-1, 2, size=(N, K)).astype(np.float32))
    dY = synth.bf16_bits(rng.integers(-1, 2, size=(M, N)).astype(np.float32))
    want_y = exact_bf16(oracle.forward(X0, W2, m2, B, bias=b1)[0])
    want_dx = exact_bf16(oracle.backward_input(dY, W2, m2, B)[0])
    want_dw = exact_bf16(oracle.backward_weight(dY, X0, m2, B)[0])

    Wp = sg.pack(to_dev(W1), mask_dev(m1), B)
    Xd, bd, dYd = to_dev(X0), to_dev(b1), to_dev(dY)
    sg.forward(Xd, Wp, bias=bd)  # the old pattern is in use just before the re-pack
    W2d, m2d = to_dev(W2), mask_dev(m2)
    torch.cuda.synchronize()
    Wp.repack(W2d, m2d)
    Y = sg.forward(Xd, Wp, bias=bd)
    dX = sg.backward_input(dYd, Wp)
    dW = sg.backward_weight(dYd, Xd, Wp)
    torch.cuda.synchronize()
    assert sg.device_status(Wp) == 0
    assert np.array_equal(bits(Y), want_y)
    assert np.array_equal(bits(dX), want_dx)
    assert np.array_equal(bits(dW).reshape(want_dw.shape), want_dw)
