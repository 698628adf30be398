"""The allocation-free small-M forward (bsl_forward_stream_noalloc).

Callers that cannot allocate device memory (a serving loop under a fixed
memory budget, a plug-in inside a framework that owns every allocation) use
this entry point instead of bsl_forward_stream; its scratch is a fixed array
inside the library.  The test calls it through the C ABI twice in a row (the
second call finds the first call's partial sums still in the array) and
checks both results against the regular entry point, which receives its
scratch from the caller, within the parity bound of the other GPU tests.
This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from tests._gpu import mask_dev, to_dev, to_f64
from tests._parity import assert_parity

pytestmark = pytest.mark.gpu


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
    ref = to_f64(want)
    _, S = oracle.forward(inp["X"], inp["W"], inp["mask"], b)
    for _ in range(2):
        Y = torch.full_like(want, 7.0)
        assert _noalloc(sg, X, Wp, Y) == 0
        torch.cuda.synchronize()
        assert sg.device_status(Wp) == 0
        assert_parity(to_f64(Y), ref, S, "no-alloc vs caller scratch")


def test_noalloc_rejects_calls_needing_more_scratch(sg):
    # b = 64 with 27 tokens needs more partial-sum scratch than the fixed
    # array on a 148-SM part; the call must fail cleanly and launch nothing
    b = 64
    inp = synth.random_case(27, 1024, 512, b, 40, 52)
    Wp = sg.pack(to_dev(inp["W"]), mask_dev(inp["mask"]), b)
    need = sg.forward_workspace_bytes(27, Wp)
    Y = torch.zeros((27, 1024), dtype=torch.bfloat16, device="cuda")
    st = _noalloc(sg, to_dev(inp["X"]), Wp, Y)
    if need > 16 * 1024 * 1024:
        assert st == 7  # BSL_ERR_SCRATCH_TOO_SMALL
        torch.cuda.synchronize()
        assert torch.count_nonzero(Y) == 0
    else:
        assert st == 0
    assert np.isfinite(to_f64(Y)).all()
