"""C-ABI checks that need no GPU: the library loads, exports every entry
point declared in include/bsl.h, and rejects bad arguments on the host
before touching a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from sparse_gemm_b200 import build
    build.build()
    import sparse_gemm_b200 as sg
    return sg.library()


def declared_entry_points():
    text = open(os.path.join(ROOT, "include", "bsl.h")).read()
    return sorted(set(re.findall(r"^BSL_API\s+[^;(]*?\b(bsl_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for required in ("bsl_pack", "bsl_pack_count", "bsl_forward", "bsl_backward_input",
                     "bsl_backward_weight", "bsl_get_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_entry_points() if not hasattr(lib, n)]
    assert not missing, missing


def _bsr(**kw):
    import sparse_gemm_b200 as sg
    s = sg._BSR()
    s.N, s.K, s.b, s.nnz = kw.get("N", 256), kw.get("K", 256), kw.get("b", 32), kw.get("nnz", 4)
    for name, _ in sg._BSR._fields_[4:]:
        setattr(s, name, kw.get(name, 4096))
    return s


@pytest.mark.parametrize("bad,code", [
    (dict(b=48), 2), (dict(b=16), 2), (dict(N=250), 1), (dict(K=100), 1), (dict(nnz=-1), 1),
    (dict(nnz=65), 1), (dict(row_ptr=0), 1), (dict(values=0), 1), (dict(values=4104), 1),
    (dict(status=0), 1), (dict(sbounds=0), 1),
])
def test_bad_weight_descriptor_is_rejected_on_host(lib, bad, code):
    s = _bsr(**bad)
    assert lib.bsl_forward_tc(4096, 64, ctypes.byref(s), None, 4096, None) == code
    assert lib.bsl_backward_input(4096, 64, ctypes.byref(s), 4096, None) == code


def test_bad_matrices_are_rejected_on_host(lib):
    s = _bsr()
    assert lib.bsl_forward_tc(0, 64, ctypes.byref(s), None, 4096, None) == 1       # null X
    assert lib.bsl_forward_tc(4096, 0, ctypes.byref(s), None, 4096, None) == 1     # M = 0
    assert lib.bsl_forward_tc(4104, 64, ctypes.byref(s), None, 4096, None) == 1    # misaligned X
    assert lib.bsl_forward_tc(4096, 64, ctypes.byref(s), 4104, 4096, None) == 1    # misaligned bias
    assert lib.bsl_backward_weight(4096, 0, 8, ctypes.byref(s), 4096, None) == 1
    assert lib.bsl_forward_stream(4096, 64, ctypes.byref(s), None, 4096, 4096, 1 << 20, None) == 2  # M too big
    assert lib.bsl_bias_grad(4096, 64, 100, 4096, None) == 1                        # N not a multiple of 32
    assert lib.bsl_bias_grad(4096, 64, 256, 0, None) == 1                           # null output
    assert lib.bsl_pack_count(0, 4, 4, 4096, ctypes.byref(ctypes.c_int32()), None) == 1


def test_status_strings(lib):
    assert lib.bsl_status_string(0) == b"BSL_OK"
    assert lib.bsl_status_string(4) == b"BSL_ERR_TIMEOUT"
    assert lib.bsl_small_m_max() == 32


def test_binding_struct_matches_the_header():
    """The ctypes mirror lists bsl_bsr's fields in the header's order and
    sizes sbounds as BSL_SBOUNDS_LEN."""
    import re
    import sparse_gemm_b200 as sg
    text = open(os.path.join(ROOT, "include", "bsl.h")).read()
    body = text[text.index("typedef struct {"):text.index("} bsl_bsr;")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = re.findall(r"\*?\s*(\w+)\s*[;,]", body)
    assert [n for n, _ in sg._BSR._fields_] == names
    m = re.search(r"#define BSL_SBOUNDS_LEN (\d+)", text)
    assert m and int(m.group(1)) == sg.SBOUNDS_LEN


def _semi24(**kw):
    import sparse_gemm_b200 as sg
    s = sg._SEMI24()
    s.N, s.K = kw.get("N", 256), kw.get("K", 256)
    for name in ("values", "meta", "status"):
        setattr(s, name, kw.get(name, 4096))
    return s


@pytest.mark.parametrize("bad", [dict(N=0), dict(N=252), dict(K=96), dict(K=0), dict(values=0),
                                 dict(values=4104), dict(meta=4100), dict(status=0)])
def test_bad_semi24_descriptor_is_rejected_on_host(lib, bad):
    s = _semi24(**bad)
    assert lib.bsl_semi24_forward(4096, 64, ctypes.byref(s), None, 4096, None) == 1
    assert lib.bsl_semi24_compress(4096, ctypes.byref(s), None) == 1


def test_bad_semi24_matrices_are_rejected_on_host(lib):
    s = _semi24()
    assert lib.bsl_semi24_forward(0, 64, ctypes.byref(s), None, 4096, None) == 1      # null X
    assert lib.bsl_semi24_forward(4096, 0, ctypes.byref(s), None, 4096, None) == 1    # M = 0
    assert lib.bsl_semi24_forward(4096, 64, ctypes.byref(s), 4100, 4096, None) == 1   # misaligned bias
    assert lib.bsl_semi24_forward(4096, 64, ctypes.byref(s), None, 0, None) == 1      # null Y
    assert lib.bsl_semi24_compress(0, ctypes.byref(s), None) == 1                     # null W
    assert lib.bsl_semi24_get_status(None, ctypes.byref(ctypes.c_int32()), None) == 1
    assert lib.bsl_status_string(8) == b"BSL_ERR_NOT_2_4"


def test_semi24_binding_struct_matches_the_header():
    import sparse_gemm_b200 as sg
    text = open(os.path.join(ROOT, "include", "bsl.h")).read()
    start = text.index("typedef struct {", text.index("2:4 semi-structured"))
    body = text[start:text.index("} bsl_semi24;")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = re.findall(r"\*?\s*(\w+)\s*[;,]", body)
    assert [n for n, _ in sg._SEMI24._fields_] == names


def test_bsr24_entry_points_check_arguments_on_host(lib):
    s = _bsr(b=64)
    assert lib.bsl_bsr24_forward(4096, 64, ctypes.byref(s), 0, 4096, None, 4096, None) == 1     # null values24
    assert lib.bsl_bsr24_forward(4096, 64, ctypes.byref(s), 4096, 4100, None, 4096, None) == 1  # misaligned meta
    assert lib.bsl_bsr24_forward(4096, 0, ctypes.byref(s), 4096, 4096, None, 4096, None) == 1   # M = 0
    assert lib.bsl_bsr24_forward(4096, 64, ctypes.byref(_bsr(b=48)), 4096, 4096, None, 4096, None) == 2
    assert lib.bsl_bsr24_compress(ctypes.byref(s), 4104, 4096, None) == 1                         # misaligned
    assert lib.bsl_bsr24_compress(ctypes.byref(_bsr(b=48)), 4096, 4096, None) == 2
