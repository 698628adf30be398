"""The allocation-free small-M forward (bsl_forward_stream_noalloc).

Some callers cannot allocate device memory once they run: a serving loop
under a fixed memory budget, where an allocation can stall or fail, or a
plug-in inside a framework that owns every allocation and gives the library
no allocator.  They call this entry point instead of bsl_forward_stream: its
scratch is a fixed array inside the library.  The test calls it through the
C ABI twice in a row (the second call finds the first call's partial sums
still in the array) and checks both results bit for bit against the regular
entry point, which runs the same kernels with a scratch buffer from the
caller, and element by element against the fp64 oracle.  This file is named
so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import oracle
import synth
from tests._gpu import mask_dev, to_dev, to_f64
from tests._parity import assert_parity

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 * 1024 * 1024  # BSL_NOALLOC_SCRATCH_BYTES in include/bsl.h


@pytest.fixture(scope="module")
def sg():
    from sparse_gemm_b200 import build
    build.build()
    oracle.build()
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sparse_gemm_b200
    return sparse_gemm_b200


def _noalloc(sg, X, Wp, Y):
    lib = sg.library()
    fn = lib.bsl_forward_stream_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(sg._BSR), ctypes.c_void_p,
                   ctypes.c_void_p]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(X.data_ptr(), X.shape[0], Wp.cref(), Y.data_ptr(), stream)


@pytest.mark.parametrize("name,M", [("decode_fwd", 16), ("decode_fwd", 5), ("small", 27)])
def test_noalloc_matches_caller_scratch_entry_point(sg, name, M):
    if name == "decode_fwd":
        w = synth.WORKLOADS[name]
        inp = synth.make_inputs(w, M=M)
        b = w.b
    else:
        b = 32
        inp = synth.random_case(M, 2048, 1024, b, 700, 51, empty_rows=(3,))
    Wp = sg.pack(to_dev(inp["W"]), mask_dev(inp["mask"]), b)
    X = to_dev(inp["X"])
    want = sg.forward_stream(X, Wp)
    ref, S = oracle.forward(inp["X"], inp["W"], inp["mask"], b)
    assert_parity(to_f64(want), ref, S, "caller-scratch entry point vs oracle")
    for _ in range(2):
        Y = torch.full_like(want, 7.0)
        assert _noalloc(sg, X, Wp, Y) == 0
        torch.cuda.synchronize()
        assert sg.device_status(Wp) == 0
        # same kernels, same fixed summation order: identical bits
        assert torch.equal(Y.view(torch.int16), want.view(torch.int16))
        assert_parity(to_f64(Y), ref, S, "no-alloc vs oracle")
    # the Python wrapper reaches the same entry point
    Y2 = sg.forward_stream_noalloc(X, Wp)
    torch.cuda.synchronize()
    assert torch.equal(Y2.view(torch.int16), want.view(torch.int16))


def test_noalloc_takes_the_largest_supported_call(sg):
    """b = 64 with 32 tokens is the largest scratch need of the small-M
    forward (SMs x 16 KiB); it fits the fixed array, runs, and matches the
    caller-scratch entry point bit for bit and the oracle element by element."""
    b, M = 64, 32
    inp = synth.random_case(M, 1024, 512, b, 40, 52, empty_rows=(5,))
    Wp = sg.pack(to_dev(inp["W"]), mask_dev(inp["mask"]), b)
    assert sg.forward_workspace_bytes(M, Wp) <= SCRATCH_BYTES
    X = to_dev(inp["X"])
    want = sg.forward_stream(X, Wp)
    Y = torch.full((M, 1024), 3.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(sg, X, Wp, Y) == 0
    torch.cuda.synchronize()
    assert sg.device_status(Wp) == 0
    assert torch.equal(Y.view(torch.int16), want.view(torch.int16))
    ref, S = oracle.forward(inp["X"], inp["W"], inp["mask"], b)
    assert_parity(to_f64(Y), ref, S, "no-alloc, b = 64, M = 32")


def test_noalloc_rejects_bad_arguments_before_any_launch(sg):
    """Arguments the entry point cannot serve come back as a status, with
    nothing launched and the output untouched: too many tokens for the
    small-M kernel, a null output."""
    b = 32
    inp = synth.random_case(40, 256, 256, b, 16, 53)
    Wp = sg.pack(to_dev(inp["W"]), mask_dev(inp["mask"]), b)
    Y = torch.zeros((40, 256), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(sg, to_dev(inp["X"]), Wp, Y) == 2   # BSL_ERR_UNSUPPORTED: M > small_m_max
    lib = sg.library()
    fn = lib.bsl_forward_stream_noalloc
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert fn(to_dev(inp["X"][:8]).data_ptr(), 8, Wp.cref(), None, stream) == 1   # null Y
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y) == 0
