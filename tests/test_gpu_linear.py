"""GPU parity of the drop-in nn.Linear pieces and of re-packing in place.

The layer is a drop-in for torch.nn.Linear (Hugging Face pytorch_block_sparse
release note, "Block-Sparse Implementation and Usage"), so the forward takes
nn.Linear's bias and the backward returns its gradient; the sparsity pattern
may change during training (release note, "Future Development Roadmap";
torchao README, "Pruning Criteria", out-of-place mask updates), which the
weight supports by re-packing into its existing buffers.  Every value output
is compared element by element with the fp64 oracle through the C ABI.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _plan
from tests._gpu import bits, mask_dev, to_dev, to_f64
from tests._parity import assert_parity

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_gemm_b200 as sg


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_gemm_b200 import build
    build.build()
    oracle.build()
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


def _bias_bits(N, seed):
    return synth.bf16_bits(np.random.default_rng(seed).standard_normal(N, dtype=np.float32))


BIAS_CASES = [
    # (M, N, K, b, nnz, seed, empty_rows)
    (1, 256, 256, 32, 16, 61, (1,)),
    (130, 384, 512, 32, 100, 62, (0, 11)),
    (300, 640, 448, 64, 30, 63, (2,)),
    (257, 1024, 768, 64, 0, 64, ()),          # no block at all: Y = bias
]


@pytest.mark.parametrize("case_args", BIAS_CASES)
def test_forward_with_bias_tc(case_args):
    M, N, K, b, nnz, seed, er = case_args
    case = synth.random_case(M, N, K, b, nnz, seed, empty_rows=er)
    bias = _bias_bits(N, seed)
    Wp = sg.pack(to_dev(case["W"]), mask_dev(case["mask"]), b)
    Y = sg.forward_tc(to_dev(case["X"]), Wp, bias=to_dev(bias))
    torch.cuda.synchronize()
    assert sg.device_status(Wp) == 0
    ref, S = oracle.forward(case["X"], case["W"], case["mask"], b, bias=bias)
    assert_parity(to_f64(Y), ref, S, "forward_tc + bias")


@pytest.mark.parametrize("case_args", BIAS_CASES)
def test_forward_with_bias_stream(case_args):
    M, N, K, b, nnz, seed, er = case_args
    M = min(M, 32)
    case = synth.random_case(M, N, K, b, nnz, seed, empty_rows=er)
    bias = _bias_bits(N, seed)
    Wp = sg.pack(to_dev(case["W"]), mask_dev(case["mask"]), b)
    Y = sg.forward_stream(to_dev(case["X"]), Wp, bias=to_dev(bias))
    torch.cuda.synchronize()
    assert sg.device_status(Wp) == 0
    ref, S = oracle.forward(case["X"], case["W"], case["mask"], b, bias=bias)
    assert_parity(to_f64(Y), ref, S, "forward_stream + bias")


@pytest.mark.parametrize("M,N", [(1, 32), (77, 96), (4096, 3072), (8192, 14336)])
def test_bias_grad(M, N):
    dY = synth.bf16_bits(np.random.default_rng(M + N).standard_normal((M, N), dtype=np.float32))
    got = sg.bias_grad(to_dev(dY))
    torch.cuda.synchronize()
    ref, S = oracle.bias_grad(dY)
    assert_parity(to_f64(got), ref, S, "bias_grad")
    again = sg.bias_grad(to_dev(dY))
    assert torch.equal(got.view(torch.int16), again.view(torch.int16))


def test_module_matches_oracle_and_sees_in_place_updates():
    M, N, K, b = 96, 512, 384, 32
    case = synth.random_case(M, N, K, b, 40, 65, empty_rows=(2,))
    bias = _bias_bits(N, 65)
    layer = sg.BlockSparseLinear.from_dense(to_dev(case["W"]), mask_dev(case["mask"]), b,
                                            bias=to_dev(bias))
    X = to_dev(case["X"]).reshape(4, 24, K).requires_grad_(True)   # leading dims are kept
    Y = layer(X)
    assert Y.shape == (4, 24, N)
    Y.backward(to_dev(case["dY"]).reshape(4, 24, N))
    ref, S = oracle.forward(case["X"], case["W"], case["mask"], b, bias=bias)
    assert_parity(to_f64(Y.detach().reshape(M, N)), ref, S, "module Y")
    ref, S = oracle.backward_input(case["dY"], case["W"], case["mask"], b)
    assert_parity(to_f64(X.grad.reshape(M, K)), ref, S, "module dX")
    ref, S = oracle.backward_weight(case["dY"], case["X"], case["mask"], b)
    assert_parity(to_f64(layer.values.grad).reshape(ref.shape), ref, S, "module dW")
    ref, S = oracle.bias_grad(case["dY"])
    assert_parity(to_f64(layer.bias.grad), ref, S, "module dbias")
    # an optimizer-style in-place update of the values is what the next call uses
    with torch.no_grad():
        layer.values.mul_(2.0)
        layer.bias.zero_()
    with torch.no_grad():
        Y2 = layer(X.detach())
    W2 = synth.bf16_bits((synth.bits_to_f32(case["W"]) * 2.0).astype(np.float32))
    ref, S = oracle.forward(case["X"], W2, case["mask"], b)
    assert_parity(to_f64(Y2.reshape(M, N)), ref, S, "module Y after update")


@pytest.mark.parametrize("M,N,K,b,nnz", [(300, 640, 448, 64, 30), (260, 768, 512, 32, 90)])
def test_repack_in_place_with_a_new_mask(M, N, K, b, nnz):
    first = synth.random_case(M, N, K, b, nnz, 66)
    second = synth.random_case(M, N, K, b, nnz, 67)
    # same block count, different pattern: block rows 0 and 9 emptied, their
    # blocks moved to the free positions of other rows
    m = second["mask"].copy()
    moved = int(m[0].sum() + m[9].sum())
    m[0] = 0
    m[9] = 0
    free = np.argwhere(m == 0)
    free = free[(free[:, 0] != 0) & (free[:, 0] != 9)][:moved]
    m[free[:, 0], free[:, 1]] = 1
    second["mask"] = m
    assert int(m.sum()) == nnz
    assert not np.array_equal(first["mask"], second["mask"])
    Wp = sg.pack(to_dev(first["W"]), mask_dev(first["mask"]), b)
    sg.forward_tc(to_dev(first["X"]), Wp)
    ptrs = {name: getattr(Wp, name).data_ptr() for name in ("values", "col_idx", "rgrp_ent", "sched")}
    Wp.repack(to_dev(second["W"]), mask_dev(second["mask"]))
    X = to_dev(second["X"])
    Y = sg.forward_tc(X, Wp)
    Ys = sg.forward_stream(X[:20].contiguous(), Wp)
    dX = sg.backward_input(to_dev(second["dY"]), Wp)
    torch.cuda.synchronize()
    assert sg.device_status(Wp) == 0
    assert {name: getattr(Wp, name).data_ptr() for name in ptrs} == ptrs   # same buffers
    want = oracle.pack(second["W"], second["mask"], b)
    for key in ("row_ptr", "col_ptr"):
        assert np.array_equal(getattr(Wp, key).cpu().numpy(), want[key]), key
    for key in ("col_idx", "row_idx", "csc_to_bsr"):
        assert np.array_equal(getattr(Wp, key)[:nnz].cpu().numpy(), want[key]), key
    assert np.array_equal(bits(Wp.block_values()), want["values"].reshape(nnz, b, b))
    gp, gb, ent, blk = _plan.group_plan(want["row_ptr"], want["col_idx"], oracle.schedule_order(want["row_ptr"]),
                                        128 // b)
    assert np.array_equal(Wp.rgrp_ptr.cpu().numpy(), gp)
    assert np.array_equal(Wp.rgrp_ent[:len(ent)].cpu().numpy(), ent)
    U = torch.cuda.get_device_properties(X.device).multi_processor_count
    assert np.array_equal(Wp.sbounds[:U + 2].cpu().numpy(), _plan.stream_bounds(want["row_ptr"], U))
    ref, S = oracle.forward(second["X"], second["W"], second["mask"], b)
    assert_parity(to_f64(Y), ref, S, "forward after repack")
    assert_parity(to_f64(Ys), ref[:20], S[:20], "stream forward after repack")
    ref, S = oracle.backward_input(second["dY"], second["W"], second["mask"], b)
    assert_parity(to_f64(dX), ref, S, "dX after repack")
    with pytest.raises(ValueError):
        Wp.repack(to_dev(first["W"]), mask_dev(np.ones_like(first["mask"])))
