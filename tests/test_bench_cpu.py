"""The bench's measurement definitions, on the CPU.

These pin what `roofline.achieved` divides by: the algorithmic FLOPs
(2·M·b²·nnz = 2·M·N·K·density) and the minimum HBM bytes of each
contraction (every operand read once, every output written once), at the
workload sizes the pages' configurations name, and the bound each
workload is reported against.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402

PEAKS = {"hbm_gbs": 6527.8, "bf16_tflops": 1642.8, "bf16_tflops_sustained": 1384.4, "source": "test"}


def test_flops_are_dense_flops_times_density():
    for name in ("tiny_fwd", "enc_fwd", "large_fwd", "decode_fwd", "enc_train_d0.25"):
        w = synth.WORKLOADS[name]
        alg = bench.algorithmic(w, w.nnz)
        density = w.nnz / ((w.N // w.b) * (w.K // w.b))
        for kind in ("fwd", "dx", "dw"):
            assert alg[kind]["flops"] == pytest.approx(2 * w.M * w.N * w.K * density, rel=1e-12)


def test_large_forward_work_and_bytes():
    w = synth.WORKLOADS["large_fwd"]
    alg = bench.algorithmic(w, w.nnz)["fwd"]
    assert alg["flops"] == 96_234_110_976                       # 96.23 GFLOP
    x, y = 8192 * 4096 * 2, 8192 * 14336 * 2
    values, index = 1434 * 64 * 64 * 2, (224 + 1 + 1434) * 4
    assert alg["bytes"] == x + values + index + y              # 313.7 MB
    assert alg["bytes"] == pytest.approx(313.74e6, rel=1e-4)


def test_decode_bytes_are_the_compressed_weight_plus_activations():
    w = synth.WORKLOADS["decode_fwd"]
    alg = bench.algorithmic(w, w.nnz)["fwd"]
    assert alg["bytes"] == pytest.approx(23.07e6, rel=2e-3)    # values 22.54 MB + index + X + Y


@pytest.mark.parametrize("name,kind,bound", [
    ("large_fwd", "fwd", "tensor"),
    ("decode_fwd", "fwd", "hbm"),
    ("enc_fwd", "fwd", "hbm"),
    ("enc_train_d1.0", "dx", "tensor"),
    ("enc_train_d0.1", "dw", "hbm"),
])
def test_reported_bound(name, kind, bound):
    w = synth.WORKLOADS[name]
    r = bench.roofline_entry(kind, bench.algorithmic(w, w.nnz)[kind], 1.0, PEAKS)
    assert r["bound"] == bound
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], abs=6e-5)  # frac is rounded to 4 places


def test_traffic_entries_name_their_sources():
    for (wname, kind), t in bench.TRAFFIC.items():
        assert (wname in synth.WORKLOADS or wname in synth.SEMI24_WORKLOADS or wname in synth.BSR24_WORKLOADS) \
            and kind in ("fwd", "dx", "dw")
        assert t["bytes"] > 0 and len(t["src_sha"]) == 16
        assert set(t) == {"bytes", "src_sha", "files"}
        for f in t["files"]:
            assert os.path.exists(os.path.join(ROOT, "sparse_gemm_b200", "csrc", f))


def test_semi24_work_bytes_and_bound():
    """2:4 forward: kept products 2·M·N·(K/2); bytes X + half-width values +
    4 bits of positions per group + Y; at the LLM-MLP size it is tensor-bound
    against the dense peak (the kept products run at twice the dense rate)."""
    w = synth.SEMI24_WORKLOADS["semi24_fwd"]
    alg = bench.algorithmic_semi24(w)
    assert alg["flops"] == 2 * w.M * w.N * (w.K // 2)
    assert alg["bytes"] == w.M * w.K * 2 + w.N * w.K + w.N * w.K // 8 + w.M * w.N * 2
    assert bench.roofline_entry("fwd", alg, 0.5, PEAKS)["bound"] == "tensor"


def test_bsr24_work_and_bytes():
    """2:4 inside blocks: kept products M*b*b*nnz; bytes X + compressed blocks
    (b*b/2 values and b*b/16 words each) + BSR index + Y."""
    w = synth.BSR24_WORKLOADS["bsr24_fwd"]
    alg = bench.algorithmic_bsr24(w, w.nnz)
    assert alg["flops"] == bench.algorithmic(w, w.nnz)["fwd"]["flops"] // 2
    b, R = w.b, w.N // w.b
    assert alg["bytes"] == (w.M * w.K * 2 + w.nnz * b * b + w.nnz * b * b // 8 + (R + 1 + w.nnz) * 4
                            + w.M * w.N * 2)
