"""GPU parity: every kernel against the fp64 CPU oracle, through the C ABI.

Index and byte outputs (the pack) must be bit-exact.  Value outputs must
satisfy |y - y_ref| <= 2^-7 |y_ref| + 1e-4 S (S = sum of |terms|), with
exact zeros where S = 0.  Small cases are compared element by element and
span several tiles plus a ragged tail; the full-size workloads run in the
same launch configuration as bench.py and are compared on sampled rows
(forward, dX) and sampled blocks (dW).
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


def pack_dev(case, b, nnz=None):
    return sg.pack(to_dev(case["W"]), mask_dev(case["mask"]), b, nnz)


def check_pack(Wp, case, b):
    want = oracle.pack(case["W"], case["mask"], b)
    nnz = want["nnz"]
    assert Wp.nnz == nnz
    for key in ("row_ptr", "col_ptr"):
        assert np.array_equal(getattr(Wp, key).cpu().numpy(), want[key]), key
    for key in ("col_idx", "row_idx", "csc_to_bsr"):
        assert np.array_equal(getattr(Wp, key)[:nnz].cpu().numpy(), want[key]), key
    assert np.array_equal(bits(Wp.block_values()), want["values"].reshape(nnz, b, b))
    assert np.array_equal(Wp.row_order.cpu().numpy(), oracle.schedule_order(want["row_ptr"]))
    assert np.array_equal(Wp.col_order.cpu().numpy(), oracle.schedule_order(want["col_ptr"]))
    rplan = _plan.group_plan(want["row_ptr"], want["col_idx"], oracle.schedule_order(want["row_ptr"]), 128 // b)
    cplan = _plan.group_plan(want["col_ptr"], want["row_idx"], oracle.schedule_order(want["col_ptr"]), 128 // b,
                              blk=want["csc_to_bsr"])
    for pre, plan in (("rgrp", rplan), ("cgrp", cplan)):
        gp, gb, ent, blk = plan
        assert np.array_equal(getattr(Wp, pre + "_ptr").cpu().numpy(), gp), pre
        assert np.array_equal(getattr(Wp, pre + "_bptr").cpu().numpy(), gb), pre
        assert np.array_equal(getattr(Wp, pre + "_ent")[:len(ent)].cpu().numpy(), ent), pre
        assert np.array_equal(getattr(Wp, pre + "_blk")[:nnz].cpu().numpy(), blk), pre
    U = torch.cuda.get_device_properties(Wp.values.device).multi_processor_count
    assert np.array_equal(Wp.sbounds[:U + 2].cpu().numpy(), _plan.stream_bounds(want["row_ptr"], U))
    assert sg.device_status(Wp) == 0


# ------------------------------------------------------------------ pack (a1-a4)

PACK_CASES = [
    # (M, N, K, b, nnz, seed, empty_rows, empty_cols)
    (8, 256, 256, 32, 16, 1, (), ()),
    (8, 512, 384, 32, 1, 2, (), ()),
    (8, 640, 448, 64, 30, 3, (1, 4), (2,)),
    (8, 1024, 2048, 32, 2048, 4, (), ()),       # density 1
    (8, 96 * 32, 24 * 32, 32, 576, 5, (0, 95), (23,)),
]


@pytest.mark.parametrize("case_args", PACK_CASES)
def test_pack_bit_exact(case_args):
    M, N, K, b, nnz, seed, er, ec = case_args
    case = synth.random_case(M, N, K, b, nnz, seed, empty_rows=er, empty_cols=ec)
    Wp = pack_dev(case, b)
    check_pack(Wp, case, b)


@pytest.mark.parametrize("name", ["tiny_fwd", "enc_fwd", "large_fwd", "decode_fwd", "enc_train_d0.1"])
def test_pack_bit_exact_workload_masks(name):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, M=1)
    case = {"W": inp["W"], "mask": inp["mask"]}
    Wp = pack_dev(case, w.b)
    assert Wp.nnz == w.nnz
    check_pack(Wp, case, w.b)


def test_pack_full_row_and_single_block():
    b = 64
    mask = np.zeros((6, 5), dtype=np.uint8)
    mask[2, :] = 1
    mask[5, 3] = 1
    rng = np.random.default_rng(7)
    W = synth.bf16_bits(rng.standard_normal((6 * b, 5 * b), dtype=np.float32))
    case = {"W": W, "mask": mask}
    check_pack(pack_dev(case, b), case, b)


def test_pack_nnz_mismatch_sets_status_and_stays_in_bounds():
    case = synth.random_case(8, 256, 256, 32, 10, 9)
    Wp = pack_dev(case, 32, nnz=7)
    assert sg.device_status(Wp) == 5
    assert sg.device_status(Wp) == 0  # cleared by the read
    ci = Wp.col_idx[:7].cpu().numpy()
    assert ci.min() >= 0 and ci.max() < 8


def test_count_blocks():
    case = synth.random_case(8, 640, 448, 64, 17, 10)
    assert sg.count_blocks(mask_dev(case["mask"])) == 17


# --------------------------------------------------------- small element-wise cases

def run_forward(fn, case, b, M):
    Wp = pack_dev(case, b)
    X = to_dev(case["X"])
    Y = fn(X, Wp)
    torch.cuda.synchronize()
    assert sg.device_status(Wp) == 0
    return to_f64(Y)


FWD_CASES = [
    # (M, N, K, b, nnz, seed, empty_rows)
    (1, 256, 256, 32, 16, 11, ()),
    (17, 512, 384, 32, 40, 12, (3,)),
    (130, 384, 512, 32, 100, 13, (0, 11)),
    (300, 640, 448, 64, 30, 14, (2,)),
    (257, 1024, 768, 64, 96, 15, ()),
    (64, 256, 256, 32, 64, 16, ()),           # density 1
    (128, 1024, 2048, 64, 7, 17, ()),
]


@pytest.mark.parametrize("case_args", FWD_CASES)
def test_forward_tc_parity(case_args):
    M, N, K, b, nnz, seed, er = case_args
    case = synth.random_case(M, N, K, b, nnz, seed, empty_rows=er)
    got = run_forward(sg.forward_tc, case, b, M)
    ref, S = oracle.forward(case["X"], case["W"], case["mask"], b)
    assert_parity(got, ref, S, "forward_tc")


STREAM_CASES = [
    (1, 256, 256, 32, 16, 21, ()),
    (3, 512, 384, 32, 40, 22, (3, 4)),
    (16, 1024, 512, 32, 200, 23, (0,)),
    (17, 640, 448, 64, 30, 24, (2,)),
    (32, 1024, 768, 64, 96, 25, ()),
    (7, 2048, 4096, 32, 1, 26, ()),           # one block: most warps idle
    (16, 4096, 4096, 32, 5000, 27, ()),       # rows cut across many warp shares
    (9, 512, 416, 32, 30, 28, (1,)),          # K = 13 block columns, an empty block row
]


@pytest.mark.parametrize("case_args", STREAM_CASES)
def test_forward_stream_parity(case_args):
    M, N, K, b, nnz, seed, er = case_args
    case = synth.random_case(M, N, K, b, nnz, seed, empty_rows=er)
    got = run_forward(sg.forward_stream, case, b, M)
    ref, S = oracle.forward(case["X"], case["W"], case["mask"], b)
    assert_parity(got, ref, S, "forward_stream")


def long_row_case(M, R, C, b, long_rows, per_row, seed):
    """A weight whose rows in ``long_rows`` hold every block column and whose
    other rows hold ``per_row`` blocks: the long rows reach across the ranges
    of many CTAs of the weight-streaming forward."""
    case = synth.random_case(M, R * b, C * b, b, R * per_row, seed)
    rng = np.random.default_rng(seed)
    mask = np.zeros((R, C), dtype=np.uint8)
    for r in range(R):
        if r in long_rows:
            mask[r, :] = 1
        else:
            mask[r, rng.choice(C, per_row, replace=False)] = 1
    case["mask"] = mask
    return case


LONG_ROW_CASES = [
    # (M, R, C, b, long rows, blocks per other row, seed)
    (16, 32, 256, 32, (0,), 4, 41),          # fewer blocks than 4 per CTA: equal shares
    (5, 64, 256, 32, (5, 40), 8, 42),        # CTA bounds moved onto nearby row starts
    (32, 48, 128, 64, (47,), 6, 43),
]


@pytest.mark.parametrize("case_args", LONG_ROW_CASES)
@pytest.mark.parametrize("with_bias", [False, True])
def test_forward_stream_rows_across_many_ctas(case_args, with_bias):
    M, R, C, b, long_rows, per_row, seed = case_args
    case = long_row_case(M, R, C, b, long_rows, per_row, seed)
    Wp = pack_dev(case, b)
    check_pack(Wp, case, b)
    bias = None
    if with_bias:  # the last CTA on a shared row adds the bias once
        bias = synth.bf16_bits(np.random.default_rng(seed + 500).standard_normal(R * b, dtype=np.float32))
    got = to_f64(sg.forward_stream(to_dev(case["X"]), Wp, bias=None if bias is None else to_dev(bias)))
    assert sg.device_status(Wp) == 0
    ref, S = oracle.forward(case["X"], case["W"], case["mask"], b, bias=bias)
    assert_parity(got, ref, S, "forward_stream" + (" + bias" if with_bias else ""))


def test_stream_bounds_with_more_block_rows_than_fit_in_shared_memory():
    """8400 block rows: the pack's bound search reads row_ptr from global
    memory instead of its shared-memory copy (8192 entries); the bounds must
    still equal the host model's and the forward the oracle's."""
    M, R, C, b = 16, 8400, 4, 32
    rng = np.random.default_rng(47)
    mask = (rng.random((R, C)) < 0.5).astype(np.uint8)
    mask[rng.integers(0, R, size=40), :] = 1  # some full rows
    mask[rng.integers(0, R, size=40), :] = 0  # some empty rows
    W = synth.bf16_bits((rng.standard_normal((R * b, C * b)) / np.sqrt(C * b)).astype(np.float32))
    X = synth.bf16_bits(rng.standard_normal((M, C * b)).astype(np.float32))
    Wp = sg.pack(to_dev(W), mask_dev(mask), b)
    row_ptr = np.concatenate([[0], np.cumsum(mask.sum(axis=1))]).astype(np.int64)
    assert np.array_equal(Wp.row_ptr.cpu().numpy(), row_ptr)
    U = torch.cuda.get_device_properties(Wp.values.device).multi_processor_count
    assert np.array_equal(Wp.sbounds[:U + 2].cpu().numpy(), _plan.stream_bounds(row_ptr, U))
    got = to_f64(sg.forward_stream(to_dev(X), Wp))
    assert sg.device_status(Wp) == 0
    ref, S = oracle.forward(X, W, mask, b)
    assert_parity(got, ref, S, "forward_stream, 8400 block rows")


def test_forward_stream_replayed_from_a_cuda_graph():
    # every call leaves the cross-CTA counters at zero, so every replay of a
    # captured call finds them fresh (a row whose count were carried over
    # would be left unwritten), with new inputs each time
    M, R, C, b = 16, 32, 256, 32
    case = long_row_case(M, R, C, b, (0, 9), 4, 44)
    Wp = pack_dev(case, b)
    X = to_dev(case["X"])
    Y = torch.zeros((M, R * b), dtype=torch.bfloat16, device=X.device)
    ws = torch.zeros(sg.forward_workspace_bytes(M, Wp), dtype=torch.uint8, device=X.device)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        sg.forward_stream(X, Wp, out=Y, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        sg.forward_stream(X, Wp, out=Y, workspace=ws)
    for k in range(3):
        Xk = synth.random_case(M, R * b, C * b, b, 4, 100 + k)["X"]
        X.copy_(to_dev(Xk))
        Y.zero_()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        ref, S = oracle.forward(Xk, case["W"], case["mask"], b)
        assert_parity(to_f64(Y), ref, S, f"graph replay {k}")
    assert sg.device_status(Wp) == 0
    del g


BWD_CASES = [
    # (M, N, K, b, nnz, seed, empty_rows, empty_cols)
    (1, 256, 256, 32, 16, 31, (), ()),
    (100, 512, 384, 32, 40, 32, (3,), (5,)),
    (257, 384, 640, 64, 25, 33, (0,), (1, 9)),
    (130, 1024, 512, 32, 512, 34, (), ()),    # density 1
    (64, 768, 1024, 64, 96, 35, (), ()),
    (40, 96, 32, 32, 2, 36, (), ()),          # one block column, three block rows: strips past the edge
]


@pytest.mark.parametrize("case_args", BWD_CASES)
def test_backward_input_parity(case_args):
    M, N, K, b, nnz, seed, er, ec = case_args
    case = synth.random_case(M, N, K, b, nnz, seed, empty_rows=er, empty_cols=ec)
    Wp = pack_dev(case, b)
    got = to_f64(sg.backward_input(to_dev(case["dY"]), Wp))
    assert sg.device_status(Wp) == 0
    ref, S = oracle.backward_input(case["dY"], case["W"], case["mask"], b)
    assert_parity(got, ref, S, "backward_input")


@pytest.mark.parametrize("case_args", BWD_CASES)
def test_backward_weight_parity(case_args):
    M, N, K, b, nnz, seed, er, ec = case_args
    case = synth.random_case(M, N, K, b, nnz, seed, empty_rows=er, empty_cols=ec)
    Wp = pack_dev(case, b)
    got = to_f64(sg.backward_weight(to_dev(case["dY"]), to_dev(case["X"]), Wp).reshape(-1, b))
    assert sg.device_status(Wp) == 0
    ref, S = oracle.backward_weight(case["dY"], case["X"], case["mask"], b)
    assert_parity(got.reshape(ref.shape), ref, S, "backward_weight")


# ---------------------------------------------------------------- edge cases

def test_empty_mask_gives_zeros():
    case = synth.random_case(70, 256, 256, 32, 0, 40)
    Wp = pack_dev(case, 32)
    X = to_dev(case["X"])
    assert torch.count_nonzero(sg.forward_tc(X, Wp)) == 0
    assert torch.count_nonzero(sg.forward_stream(X[:9], Wp)) == 0
    assert torch.count_nonzero(sg.backward_input(to_dev(case["dY"]), Wp)) == 0
    assert sg.backward_weight(to_dev(case["dY"]), X, Wp).numel() == 0


def test_outputs_stay_inside_their_buffers():
    M, N, K, b = 130, 512, 384, 32
    case = synth.random_case(M, N, K, b, 60, 41)
    Wp = pack_dev(case, b)
    canary = -12345.0
    buf = torch.full((M * N + 4096,), canary, dtype=torch.bfloat16, device="cuda")
    Y = buf[: M * N].view(M, N)
    sg.forward_tc(to_dev(case["X"]), Wp, out=Y)
    buf2 = torch.full((5 * N + 4096,), canary, dtype=torch.bfloat16, device="cuda")
    sg.forward_stream(to_dev(case["X"][:5]), Wp, out=buf2[: 5 * N].view(5, N))
    dbuf = torch.full((M * K + 4096,), canary, dtype=torch.bfloat16, device="cuda")
    sg.backward_input(to_dev(case["dY"]), Wp, out=dbuf[: M * K].view(M, K))
    wbuf = torch.full((Wp.nnz * b * b + 4096,), canary, dtype=torch.bfloat16, device="cuda")
    sg.backward_weight(to_dev(case["dY"]), to_dev(case["X"]), Wp,
                       out=wbuf[: Wp.nnz * b * b].view(Wp.nnz, b, b))
    torch.cuda.synchronize()
    for t in (buf, buf2, dbuf, wbuf):
        assert torch.all(t[-4096:] == canary)


def test_results_are_deterministic():
    case = synth.random_case(300, 1024, 768, 64, 96, 42)
    Wp = pack_dev(case, 64)
    X, dY = to_dev(case["X"]), to_dev(case["dY"])
    a = [sg.forward_tc(X, Wp), sg.forward_stream(X[:20], Wp), sg.backward_input(dY, Wp),
         sg.backward_weight(dY, X, Wp)]
    b = [sg.forward_tc(X, Wp), sg.forward_stream(X[:20], Wp), sg.backward_input(dY, Wp),
         sg.backward_weight(dY, X, Wp)]
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.int16), v.view(torch.int16))


def test_work_counters_with_more_units_than_ctas():
    """More units than CTAs: each CTA's first unit is its own index and the
    counter hands out the rest; after every launch (forward and dX, several
    M) the counters are back at zero and repeated results are bit-identical."""
    case = synth.random_case(5000, 2048, 1024, 64, 300, 48)
    Wp = pack_dev(case, 64)
    X, dY = to_dev(case["X"]), to_dev(case["dY"])
    ncta = torch.cuda.get_device_properties(X.device).multi_processor_count
    assert (2048 // 128) * ((5000 + 255) // 256) > ncta  # forward units
    assert (1024 // 128) * ((5000 + 255) // 256) > ncta  # dX units
    first = None
    for M in (5000, 4500, 5000):
        y = sg.forward_tc(X[:M].contiguous(), Wp)
        dx = sg.backward_input(dY[:M].contiguous(), Wp)
        torch.cuda.synchronize()
        assert int(Wp.sched.abs().sum()) == 0, M
        assert sg.device_status(Wp) == 0
        if M == 5000:
            if first is None:
                first = (y, dx)
                ref, S = oracle.forward(case["X"], case["W"], case["mask"], 64, rows=np.arange(0, 5000, 97))
                assert_parity(to_f64(y[::97]), ref, S, "forward, more units than CTAs")
            else:
                assert torch.equal(y.view(torch.int16), first[0].view(torch.int16))
                assert torch.equal(dx.view(torch.int16), first[1].view(torch.int16))


def test_work_counters_return_to_zero_after_every_launch():
    """The persistent kernels take units from counters in the packed weight,
    and the small-M forward counts CTAs in on rows they share in its
    workspace.  No memset precedes a launch: every launch leaves its
    counters at zero, so later launches of any M (ragged or not) take every
    unit and results stay bit-identical."""
    case = synth.random_case(700, 1024, 768, 64, 120, 44)
    Wp = pack_dev(case, 64)
    X, dY = to_dev(case["X"]), to_dev(case["dY"])
    ws = torch.zeros(sg.forward_workspace_bytes(32, Wp), dtype=torch.uint8, device=X.device)
    first = None
    for M in (700, 256, 1, 700, 33, 700):
        y = sg.forward_tc(X[:M].contiguous(), Wp)
        dx = sg.backward_input(dY[:M].contiguous(), Wp)
        ys = sg.forward_stream(X[:min(M, 32)].contiguous(), Wp, workspace=ws)
        torch.cuda.synchronize()
        assert int(Wp.sched.abs().sum()) == 0, M
        ncnt = torch.cuda.get_device_properties(X.device).multi_processor_count
        assert int(ws[:4 * ncnt].view(torch.int32).abs().sum()) == 0, M
        if M == 700:
            if first is None:
                first = (y.clone(), dx.clone(), ys.clone())
            else:
                assert torch.equal(y.view(torch.int16), first[0].view(torch.int16))
                assert torch.equal(dx.view(torch.int16), first[1].view(torch.int16))
                assert torch.equal(ys.view(torch.int16), first[2].view(torch.int16))
    ref, S = oracle.forward(case["X"], case["W"], case["mask"], 64)
    assert_parity(to_f64(first[0]), ref, S, "forward, repeated launches")
    ref32, S32 = oracle.forward(case["X"][:32], case["W"], case["mask"], 64)
    assert_parity(to_f64(first[2]), ref32, S32, "forward_stream, repeated launches")
    assert sg.device_status(Wp) == 0


def test_forward_tc_replayed_from_a_cuda_graph():
    # each replay of a captured call takes every unit again (the counter a
    # launch used is back at zero when the next one starts)
    M, N, K, b = 600, 1024, 768, 64
    case = synth.random_case(M, N, K, b, 120, 45)
    Wp = pack_dev(case, b)
    X = to_dev(case["X"])
    Y = torch.zeros((M, N), dtype=torch.bfloat16, device=X.device)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        sg.forward_tc(X, Wp, out=Y)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        sg.forward_tc(X, Wp, out=Y)
    for k in range(3):
        Xk = synth.random_case(M, N, K, b, 4, 200 + k)["X"]
        X.copy_(to_dev(Xk))
        Y.zero_()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        rows = np.arange(0, M, 7)
        ref, S = oracle.forward(Xk, case["W"], case["mask"], b, rows=rows)
        assert_parity(to_f64(Y)[rows], ref, S, f"graph replay {k}")
    assert int(Wp.sched.abs().sum()) == 0
    assert sg.device_status(Wp) == 0
    del g


def test_density_one_matches_cublas():
    M, N, K, b = 512, 1024, 768, 64
    case = synth.random_case(M, N, K, b, (N // b) * (K // b), 43)
    Wp = pack_dev(case, b)
    X, W = to_dev(case["X"]), to_dev(case["W"])
    got = to_f64(sg.forward_tc(X, Wp))
    lib = to_f64(torch.matmul(X, W.t()))
    ref, S = oracle.forward(case["X"], case["W"], case["mask"], b)
    assert_parity(got, ref, S, "forward vs oracle")
    assert_parity(lib, ref, S, "cuBLAS vs oracle")


def test_bounded_wait_reports_timeout():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sg.debug_wait_timeout(status, 2000)
    torch.cuda.synchronize()
    assert int(status.item()) == 4
    # the context is still usable afterwards
    assert torch.ones(4, device="cuda").sum().item() == 4


def test_autograd_function_matches_oracle():
    M, N, K, b = 96, 512, 384, 32
    case = synth.random_case(M, N, K, b, 40, 44)
    Wp = pack_dev(case, b)
    X = to_dev(case["X"]).requires_grad_(True)
    vals = torch.nn.Parameter(Wp.block_values())  # the packed values themselves (the kernels read them)
    Y = sg.BlockSparseLinearFunction.apply(X, vals, Wp)
    Y.backward(to_dev(case["dY"]))
    ref, S = oracle.forward(case["X"], case["W"], case["mask"], b)
    assert_parity(to_f64(Y.detach()), ref, S, "autograd forward")
    ref, S = oracle.backward_input(case["dY"], case["W"], case["mask"], b)
    assert_parity(to_f64(X.grad), ref, S, "autograd dX")
    ref, S = oracle.backward_weight(case["dY"], case["X"], case["mask"], b)
    assert_parity(to_f64(vals.grad).reshape(ref.shape), ref, S, "autograd dW")


# ----------------------------------------------------- full-size workloads (sampled)

def _sample_rows(M, n, seed, tile=128):
    """Rows checked at full size: the first and last row of every `tile`-row
    tile of M (every work unit of the tensor-core kernels starts and ends on
    such a boundary, so a unit that is skipped, duplicated or shifted shows
    up at its edges), plus `n` random rows."""
    rng = np.random.default_rng(seed)
    rows = {0, M - 1} | set(rng.choice(M, size=min(n, M), replace=False).tolist())
    for t0 in range(0, M, tile):
        rows |= {t0, min(M, t0 + tile) - 1}
    return np.array(sorted(rows))


def _dw_check_blocks(mask, seed, G):
    """Blocks checked at full size for the weight gradient: every block of
    the heaviest block column, every block of a column whose block count is
    not a multiple of G (the weight-gradient kernel works on G blocks of a
    column at a time, so this covers a short last group), the first and last
    block, and a random sample.  Returned as BSR positions."""
    rr, cc = np.nonzero(mask)                    # BSR order (row-major scan)
    counts = mask.sum(0)
    cols = {int(np.argmax(counts))}
    ragged = [c for c in range(mask.shape[1]) if counts[c] % G]
    if ragged:
        cols.add(int(ragged[0]))
    pick = set(np.nonzero(np.isin(cc, list(cols)))[0].tolist())
    pick |= {0, len(rr) - 1}
    rng = np.random.default_rng(seed)
    pick |= set(rng.choice(len(rr), size=min(24, len(rr)), replace=False).tolist())
    return np.array(sorted(pick)), rr, cc


@pytest.mark.parametrize("name", ["tiny_fwd", "enc_fwd", "large_fwd", "decode_fwd"])
def test_workload_forward(name):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w)
    Wp = pack_dev(inp, w.b)
    X = to_dev(inp["X"])
    Y = sg.forward(X, Wp)          # the entry point bench.py times
    torch.cuda.synchronize()
    assert sg.device_status(Wp) == 0
    rows = np.arange(w.M) if w.M <= 64 else _sample_rows(w.M, 16, w.seed)
    ref, S = oracle.forward(inp["X"], inp["W"], inp["mask"], w.b, rows=rows)
    assert_parity(to_f64(Y[torch.from_numpy(rows).cuda()]), ref, S, name)


@pytest.mark.parametrize("d", ["1.0", "0.5", "0.25", "0.1"])
def test_workload_training_step(d):
    w = synth.WORKLOADS[f"enc_train_d{d}"]
    inp = synth.make_inputs(w)
    Wp = pack_dev(inp, w.b)
    X, dY = to_dev(inp["X"]), to_dev(inp["dY"])
    Y = sg.forward(X, Wp)
    dX = sg.backward_input(dY, Wp)
    dW = sg.backward_weight(dY, X, Wp)
    torch.cuda.synchronize()
    assert sg.device_status(Wp) == 0
    rows = _sample_rows(w.M, 12, w.seed)
    Wt = oracle.dense_weight(inp["W"], inp["mask"], w.b)
    ref, S = oracle.forward(inp["X"], inp["W"], inp["mask"], w.b, rows=rows, Wt=Wt)
    assert_parity(to_f64(Y[torch.from_numpy(rows).cuda()]), ref, S, "Y")
    ref, S = oracle.backward_input(inp["dY"], inp["W"], inp["mask"], w.b, rows=rows, Wt=Wt)
    assert_parity(to_f64(dX[torch.from_numpy(rows).cuda()]), ref, S, "dX")
    pick, rr, cc = _dw_check_blocks(inp["mask"], w.seed, 128 // w.b)
    ref, S = oracle.backward_weight(inp["dY"], inp["X"], inp["mask"], w.b,
                                    blocks=[(int(rr[i]), int(cc[i])) for i in pick])
    got = to_f64(dW[torch.from_numpy(pick).cuda()])
    assert_parity(got, ref, S, "dW")


def test_calls_from_another_host_thread():
    """The autograd engine calls backward kernels from its own thread."""
    import threading
    case = synth.random_case(96, 512, 384, 32, 40, 45)
    Wp = pack_dev(case, 32)
    X, dY = to_dev(case["X"]), to_dev(case["dY"])
    out, err = {}, []

    def work():
        try:
            out["Y"] = sg.forward_tc(X, Wp)
            out["dX"] = sg.backward_input(dY, Wp)
            out["dW"] = sg.backward_weight(dY, X, Wp)
            torch.cuda.synchronize()
        except Exception as e:  # noqa: BLE001
            err.append(repr(e))

    t = threading.Thread(target=work)
    t.start()
    t.join()
    assert not err, err
    ref, S = oracle.backward_input(case["dY"], case["W"], case["mask"], 32)
    assert_parity(to_f64(out["dX"]), ref, S, "dX from a second thread")
