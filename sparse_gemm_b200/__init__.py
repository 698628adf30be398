"""sparse_gemm_b200 -- block-sparse linear layer on B200 (sm_100a).

Thin ctypes binding over ``libbsl.so`` (C ABI in ``include/bsl.h``).  The
binding only marshals arguments: it checks dtypes and shapes, allocates
outputs with torch on the tensors' device and passes raw pointers plus the
current CUDA stream.  Every step of the computation runs in the library's
CUDA kernels; there is no fallback.  If the library is missing or the
device is not an sm_100 GPU the calls raise.

Layer (Hugging Face pytorch_block_sparse release note, "Block-Sparse
Implementation and Usage"): a linear layer whose weight W[N, K] keeps only
its nonzero b x b blocks.  Forward Y = X W^T, input gradient dX = dY W,
weight gradient dW = dY^T X at the kept blocks only.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "BslError", "BsrWeight", "library", "count_blocks", "pack", "forward", "forward_tc",
    "forward_stream", "forward_workspace_bytes", "backward_input", "backward_weight",
    "device_status", "set_wait_timeout_us", "debug_wait_timeout", "small_m_max",
    "forward_stream_noalloc", "bias_grad",
    "BlockSparseLinearFunction", "BlockSparseLinear",
    "Semi24Weight", "compress24", "forward24", "semi24_status", "Semi24Linear",
    "Bsr24Weight", "compress_bsr24", "forward_bsr24",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsl.so")

STATUS_NAMES = {
    0: "BSL_OK", 1: "BSL_ERR_INVALID_ARG", 2: "BSL_ERR_UNSUPPORTED", 3: "BSL_ERR_CUDA",
    4: "BSL_ERR_TIMEOUT", 5: "BSL_ERR_NNZ_MISMATCH", 6: "BSL_ERR_NO_DEVICE",
    7: "BSL_ERR_SCRATCH_TOO_SMALL", 8: "BSL_ERR_NOT_2_4",
}


class BslError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS_NAMES.get(self.status, self.status)}")


class _BSR(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("b", ctypes.c_int32),
                ("nnz", ctypes.c_int32)] + [
        (name, ctypes.c_void_p) for name in
        ("row_ptr", "col_idx", "values", "col_ptr", "row_idx", "csc_to_bsr", "row_order",
         "col_order", "rgrp_ptr", "rgrp_bptr", "rgrp_ent", "rgrp_blk", "cgrp_ptr",
         "cgrp_bptr", "cgrp_ent", "cgrp_blk", "status", "sched", "sbounds")]

class _SEMI24(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("values", ctypes.c_void_p),
                ("meta", ctypes.c_void_p), ("status", ctypes.c_void_p)]


# int32 entries of bsl_bsr.sbounds (BSL_SBOUNDS_LEN in include/bsl.h)
SBOUNDS_LEN = 1026


_lib = None


def library() -> ctypes.CDLL:
    """Load libbsl.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m sparse_gemm_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I32, SZ, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_uint64
        BP = ctypes.POINTER(_BSR)
        SP = ctypes.POINTER(_SEMI24)
        sig = {
            "bsl_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "bsl_last_cuda_error": (ctypes.c_char_p, []),
            "bsl_pack_count": (ctypes.c_int, [P, I32, I32, P, ctypes.POINTER(I32), P]),
            "bsl_pack": (ctypes.c_int, [P, P, BP, P]),
            "bsl_forward": (ctypes.c_int, [P, I32, BP, P, P, P, SZ, P]),
            "bsl_small_m_max": (I32, []),
            "bsl_forward_workspace_bytes": (SZ, [I32, BP]),
            "bsl_forward_tc": (ctypes.c_int, [P, I32, BP, P, P, P]),
            "bsl_forward_stream": (ctypes.c_int, [P, I32, BP, P, P, P, SZ, P]),
            "bsl_bias_grad": (ctypes.c_int, [P, I32, I32, P, P]),
            "bsl_backward_input": (ctypes.c_int, [P, I32, BP, P, P]),
            "bsl_backward_weight": (ctypes.c_int, [P, P, I32, BP, P, P]),
            "bsl_get_device_status": (ctypes.c_int, [BP, ctypes.POINTER(I32), P]),
            "bsl_set_wait_timeout_us": (None, [U64]),
            "bsl_debug_wait_timeout": (ctypes.c_int, [P, U64, P]),
            "bsl_forward_stream_noalloc": (ctypes.c_int, [P, I32, BP, P, P]),
            "bsl_semi24_compress": (ctypes.c_int, [P, SP, P]),
            "bsl_semi24_forward": (ctypes.c_int, [P, I32, SP, P, P, P]),
            "bsl_semi24_get_status": (ctypes.c_int, [SP, ctypes.POINTER(I32), P]),
            "bsl_bsr24_compress": (ctypes.c_int, [BP, P, P, P]),
            "bsl_bsr24_forward": (ctypes.c_int, [P, I32, BP, P, P, P, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(st: int, where: str):
    if st != 0:
        detail = library().bsl_last_cuda_error().decode() if st == 3 else ""
        raise BslError(st, f"{where} [{detail}]" if detail else where)


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _cuda_bf16_2d(t: torch.Tensor, name: str, cols: int | None = None):
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 2):
        raise TypeError(f"{name} must be a 2-D bfloat16 CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")
    if cols is not None and t.shape[1] != cols:
        raise ValueError(f"{name} has {t.shape[1]} columns, expected {cols}")


class BsrWeight:
    """Packed block-sparse weight: device tensors of the bsl_bsr struct."""

    def __init__(self, N: int, K: int, b: int, nnz: int, device):
        if b not in (32, 64) or N % b or K % b:
            raise ValueError("b must be 32 or 64 and divide N and K")
        self.N, self.K, self.b, self.nnz = int(N), int(K), int(b), int(nnz)
        R, C = N // b, K // b
        i32 = dict(dtype=torch.int32, device=device)
        self.row_ptr = torch.empty(R + 1, **i32)
        self.col_idx = torch.empty(max(nnz, 1), **i32)
        self.values = torch.empty((max(nnz, 1), b, b), dtype=torch.bfloat16, device=device)
        self.col_ptr = torch.empty(C + 1, **i32)
        self.row_idx = torch.empty(max(nnz, 1), **i32)
        self.csc_to_bsr = torch.empty(max(nnz, 1), **i32)
        self.row_order = torch.empty(R, **i32)
        self.col_order = torch.empty(C, **i32)
        G = 128 // b   # block rows (forward) / block columns (input gradient) per group
        nrg, ncg = (R + G - 1) // G, (C + G - 1) // G
        self.rgrp_ptr = torch.empty(nrg + 1, **i32)
        self.rgrp_bptr = torch.empty(nrg + 1, **i32)
        self.rgrp_ent = torch.empty(max(nnz, 1), **i32)
        self.rgrp_blk = torch.empty(max(nnz, 1), **i32)
        self.cgrp_ptr = torch.empty(ncg + 1, **i32)
        self.cgrp_bptr = torch.empty(ncg + 1, **i32)
        self.cgrp_ent = torch.empty(max(nnz, 1), **i32)
        self.cgrp_blk = torch.empty(max(nnz, 1), **i32)
        self.status = torch.zeros(1, **i32)
        self.sched = torch.zeros(8, **i32)
        self.sbounds = torch.zeros(SBOUNDS_LEN, **i32)
        self._c = _BSR(self.N, self.K, self.b, self.nnz,
                       *[t.data_ptr() for t in (self.row_ptr, self.col_idx, self.values, self.col_ptr,
                                                self.row_idx, self.csc_to_bsr, self.row_order,
                                                self.col_order, self.rgrp_ptr,
                                                self.rgrp_bptr, self.rgrp_ent, self.rgrp_blk,
                                                self.cgrp_ptr, self.cgrp_bptr, self.cgrp_ent,
                                                self.cgrp_blk, self.status, self.sched, self.sbounds)])

    @property
    def R(self):
        return self.N // self.b

    @property
    def C(self):
        return self.K // self.b

    @property
    def device(self):
        return self.values.device

    def block_values(self) -> torch.Tensor:
        """Packed values [nnz, b, b] (empty view when nnz == 0)."""
        return self.values[: self.nnz]

    def repack(self, W: torch.Tensor, mask: torch.Tensor) -> "BsrWeight":
        """Re-pack a new dense weight and block mask with the same number of
        kept blocks into this weight's existing device arrays (no
        allocation, the tensors keep their addresses): the pattern can move
        during training (release note, "Future Development Roadmap"; torchao
        README, "Pruning Criteria", out-of-place mask updates) while every
        buffer, CUDA graph and optimizer state that refers to it stays
        valid.  Raises if the mask keeps a different number of blocks."""
        _cuda_bf16_2d(W, "W", self.K)
        if W.shape[0] != self.N:
            raise ValueError(f"W has {W.shape[0]} rows, expected {self.N}")
        m = _mask_u8(mask, self.R, self.C)
        n = count_blocks(m)
        if n != self.nnz:
            raise ValueError(f"mask keeps {n} blocks; this weight holds {self.nnz}")
        _check(library().bsl_pack(W.data_ptr(), m.data_ptr(), self.cref(), _stream(W)), "bsl_pack")
        self._mask = m
        return self

    def cref(self):
        return ctypes.byref(self._c)


def _mask_u8(mask: torch.Tensor, R: int, C: int) -> torch.Tensor:
    if not (mask.is_cuda and mask.dim() == 2 and tuple(mask.shape) == (R, C)):
        raise ValueError(f"mask must be a CUDA tensor of shape ({R}, {C})")
    return mask.to(torch.uint8).contiguous()


def count_blocks(mask: torch.Tensor) -> int:
    """Number of kept blocks in a [R, C] block mask (synchronises the stream)."""
    R, C = mask.shape
    m = _mask_u8(mask, R, C)
    tmp = torch.empty(R + 1, dtype=torch.int32, device=m.device)
    out = ctypes.c_int32(0)
    _check(library().bsl_pack_count(m.data_ptr(), R, C, tmp.data_ptr(), ctypes.byref(out), _stream(m)),
           "bsl_pack_count")
    return int(out.value)


def pack(W: torch.Tensor, mask: torch.Tensor, b: int, nnz: int | None = None) -> BsrWeight:
    """Pack a dense bf16 weight [N, K] with a block mask [N/b, K/b] (kept = nonzero)."""
    _cuda_bf16_2d(W, "W")
    N, K = W.shape
    m = _mask_u8(mask, N // b, K // b)
    if nnz is None:
        nnz = count_blocks(m)
    Wp = BsrWeight(N, K, b, nnz, W.device)
    _check(library().bsl_pack(W.data_ptr(), m.data_ptr(), Wp.cref(), _stream(W)), "bsl_pack")
    Wp._mask = m  # keep the mask alive until the stream has consumed it
    return Wp


def small_m_max() -> int:
    return int(library().bsl_small_m_max())


def forward_workspace_bytes(M: int, Wp: BsrWeight) -> int:
    return int(library().bsl_forward_workspace_bytes(M, Wp.cref()))


def _out(M, cols, like):
    return torch.empty((M, cols), dtype=torch.bfloat16, device=like.device)


def _bias_ptr(bias, N: int, like: torch.Tensor):
    if bias is None:
        return None
    if not (isinstance(bias, torch.Tensor) and bias.is_cuda and bias.dtype == torch.bfloat16
            and bias.dim() == 1 and bias.shape[0] == N and bias.is_contiguous()):
        raise TypeError(f"bias must be a contiguous 1-D bfloat16 CUDA tensor of {N} entries")
    if bias.device != like.device:
        raise ValueError("bias must be on the same device as X")
    return bias.data_ptr()


def forward(X: torch.Tensor, Wp: BsrWeight, out: torch.Tensor | None = None,
            workspace: torch.Tensor | None = None, bias: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X W^T (+ bias), kernel chosen by M (weight streaming for M <= small_m_max())."""
    _cuda_bf16_2d(X, "X", Wp.K)
    bptr = _bias_ptr(bias, Wp.N, X)
    M = X.shape[0]
    Y = _out(M, Wp.N, X) if out is None else out
    nbytes = forward_workspace_bytes(M, Wp)
    if nbytes and workspace is None:
        workspace = torch.zeros(nbytes, dtype=torch.uint8, device=X.device)
    wptr = workspace.data_ptr() if workspace is not None else None
    wlen = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(library().bsl_forward(X.data_ptr(), M, Wp.cref(), bptr, Y.data_ptr(), wptr, wlen, _stream(X)),
           "bsl_forward")
    return Y


def forward_tc(X: torch.Tensor, Wp: BsrWeight, out: torch.Tensor | None = None,
               bias: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X W^T (+ bias) on the tensor-core kernel (any M)."""
    _cuda_bf16_2d(X, "X", Wp.K)
    bptr = _bias_ptr(bias, Wp.N, X)
    M = X.shape[0]
    Y = _out(M, Wp.N, X) if out is None else out
    _check(library().bsl_forward_tc(X.data_ptr(), M, Wp.cref(), bptr, Y.data_ptr(), _stream(X)),
           "bsl_forward_tc")
    return Y


def forward_stream(X: torch.Tensor, Wp: BsrWeight, out: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None, bias: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X W^T (+ bias) on the weight-streaming kernel (M <= small_m_max())."""
    _cuda_bf16_2d(X, "X", Wp.K)
    bptr = _bias_ptr(bias, Wp.N, X)
    M = X.shape[0]
    Y = _out(M, Wp.N, X) if out is None else out
    nbytes = forward_workspace_bytes(M, Wp)
    if workspace is None:
        workspace = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=X.device)
    _check(library().bsl_forward_stream(X.data_ptr(), M, Wp.cref(), bptr, Y.data_ptr(), workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(), _stream(X)),
           "bsl_forward_stream")
    return Y


def forward_stream_noalloc(X: torch.Tensor, Wp: BsrWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X W^T on the weight-streaming kernel without a caller-provided
    workspace (for callers that cannot allocate device memory): the scratch
    is the library's fixed per-GPU array; overlapping calls race on it."""
    _cuda_bf16_2d(X, "X", Wp.K)
    M = X.shape[0]
    Y = _out(M, Wp.N, X) if out is None else out
    _check(library().bsl_forward_stream_noalloc(X.data_ptr(), M, Wp.cref(), Y.data_ptr(), _stream(X)),
           "bsl_forward_stream_noalloc")
    return Y


def backward_input(dY: torch.Tensor, Wp: BsrWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    """dX = dY W (tensor-core kernel over the CSC index)."""
    _cuda_bf16_2d(dY, "dY", Wp.N)
    M = dY.shape[0]
    dX = _out(M, Wp.K, dY) if out is None else out
    _check(library().bsl_backward_input(dY.data_ptr(), M, Wp.cref(), dX.data_ptr(), _stream(dY)),
           "bsl_backward_input")
    return dX


def backward_weight(dY: torch.Tensor, X: torch.Tensor, Wp: BsrWeight,
                    out: torch.Tensor | None = None) -> torch.Tensor:
    """dW at the kept blocks, [nnz, b, b] in BSR order."""
    _cuda_bf16_2d(dY, "dY", Wp.N)
    _cuda_bf16_2d(X, "X", Wp.K)
    if dY.shape[0] != X.shape[0]:
        raise ValueError("dY and X must have the same number of rows")
    dW = torch.empty((max(Wp.nnz, 1), Wp.b, Wp.b), dtype=torch.bfloat16, device=X.device) \
        if out is None else out
    _check(library().bsl_backward_weight(dY.data_ptr(), X.data_ptr(), X.shape[0], Wp.cref(),
                                         dW.data_ptr(), _stream(X)), "bsl_backward_weight")
    return dW[: Wp.nnz]


def bias_grad(dY: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """dbias = column sums of dY [M, N] (the gradient of the forward's bias), bf16 [N]."""
    _cuda_bf16_2d(dY, "dY")
    M, N = dY.shape
    db = torch.empty(N, dtype=torch.bfloat16, device=dY.device) if out is None else out
    _check(library().bsl_bias_grad(dY.data_ptr(), M, N, db.data_ptr(), _stream(dY)), "bsl_bias_grad")
    return db


def device_status(Wp: BsrWeight) -> int:
    """Read and clear the device status word (synchronises the stream)."""
    out = ctypes.c_int32(0)
    _check(library().bsl_get_device_status(Wp.cref(), ctypes.byref(out), _stream(Wp.values)),
           "bsl_get_device_status")
    return int(out.value)


def set_wait_timeout_us(us: int) -> None:
    library().bsl_set_wait_timeout_us(int(us))


def debug_wait_timeout(status: torch.Tensor, us: int) -> None:
    """Run the bounded-wait test kernel; it writes BSL_ERR_TIMEOUT (4) to status[0]."""
    if not (status.is_cuda and status.dtype == torch.int32):
        raise TypeError("status must be an int32 CUDA tensor")
    _check(library().bsl_debug_wait_timeout(status.data_ptr(), int(us), _stream(status)),
           "bsl_debug_wait_timeout")


class BlockSparseLinearFunction(torch.autograd.Function):
    """Autograd wrapper: forward Y = X W^T (+ bias); backward dX, dW at the
    kept blocks and dbias.

    ``values`` must be the packed weight's own value tensor
    (``Wp.block_values()``, the parameter being trained: the kernels read
    the weight from it, so an in-place update is seen by the next call); its
    gradient comes back in the same [nnz, b, b] layout.  ``bias`` is a bf16
    [N] tensor or None.
    """

    @staticmethod
    def forward(ctx, X, values, Wp, bias=None):
        if values.data_ptr() != Wp.values.data_ptr():
            raise ValueError("values must be the packed weight's block_values()")
        ctx.save_for_backward(X)
        ctx.Wp = Wp
        ctx.has_bias = bias is not None
        return forward(X.contiguous(), Wp, bias=bias)

    @staticmethod
    def backward(ctx, dY):
        (X,) = ctx.saved_tensors
        Wp = ctx.Wp
        dY = dY.contiguous()
        dX = backward_input(dY, Wp) if ctx.needs_input_grad[0] else None
        dW = backward_weight(dY, X.contiguous(), Wp) if ctx.needs_input_grad[1] else None
        db = bias_grad(dY) if ctx.has_bias and ctx.needs_input_grad[3] else None
        return dX, dW, None, db


class BlockSparseLinear(torch.nn.Module):
    """Drop-in for ``torch.nn.Linear`` with a block-sparse weight (Hugging
    Face pytorch_block_sparse release note, "Block-Sparse Implementation and
    Usage"): ``in_features`` -> ``out_features``, weight kept as its b x b
    blocks under a block mask, optional bias, bf16 on an sm_100 GPU.

    Build it from a dense weight (zeros in place or not) and a block mask
    with :meth:`from_dense`.  The trainable parameters are ``values`` (the
    packed blocks, [nnz, b, b], BSR order) and ``bias`` ([out_features]).
    Inputs may have any leading dimensions; the last one is in_features.
    """

    def __init__(self, packed: BsrWeight, bias: torch.Tensor | None = None):
        super().__init__()
        self.packed = packed
        self.in_features, self.out_features = packed.K, packed.N
        self.values = torch.nn.Parameter(packed.block_values(), requires_grad=True)
        if bias is not None:
            if bias.shape != (packed.N,):
                raise ValueError("bias must have out_features entries")
            bias = torch.nn.Parameter(bias.detach().to(device=packed.device, dtype=torch.bfloat16).contiguous())
        self.bias = bias

    @classmethod
    def from_dense(cls, weight: torch.Tensor, mask: torch.Tensor, block: int,
                   bias: torch.Tensor | None = None) -> "BlockSparseLinear":
        return cls(pack(weight.detach().to(torch.bfloat16).contiguous(), mask, block), bias)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features)
        if x2.dtype != torch.bfloat16:
            x2 = x2.to(torch.bfloat16)
        y = BlockSparseLinearFunction.apply(x2, self.values, self.packed, self.bias)
        return y.reshape(*lead, self.out_features)

    def extra_repr(self) -> str:
        return (f"in_features={self.in_features}, out_features={self.out_features}, "
                f"block={self.packed.b}, nnz_blocks={self.packed.nnz}, bias={self.bias is not None}")


# ---------------------------------------------------------------- 2:4 semi-structured


class Semi24Weight:
    """A weight with the 2:4 semi-structured pattern in its compressed form
    (torchao sparsity README, Table 4.1, "NVIDIA 2:4 compressed
    representation"): ``values`` bf16 [N, K/2], the two kept elements of every
    group of four, and ``meta`` [N, K/16] (16-bit words held in an int16
    tensor), their 2-bit positions; layout in include/bsl.h (bsl_semi24)."""

    def __init__(self, N: int, K: int, device):
        if N <= 0 or K <= 0 or N % 8 or K % 64:
            raise ValueError("N must be a positive multiple of 8 and K of 64")
        self.N, self.K = int(N), int(K)
        self.values = torch.empty((N, K // 2), dtype=torch.bfloat16, device=device)
        self.meta = torch.empty((N, K // 16), dtype=torch.int16, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self._c = _SEMI24(self.N, self.K, self.values.data_ptr(), self.meta.data_ptr(),
                          self.status.data_ptr())

    @property
    def device(self):
        return self.values.device

    def cref(self):
        return ctypes.byref(self._c)


def compress24(W: torch.Tensor, out: Semi24Weight | None = None) -> Semi24Weight:
    """Compress a dense bf16 weight [N, K] with zeros in place and at most two
    nonzeros per group of four along K.  A group with more nonzeros is
    reported by :func:`semi24_status` (BSL_ERR_NOT_2_4)."""
    _cuda_bf16_2d(W, "W")
    N, K = W.shape
    w = Semi24Weight(N, K, W.device) if out is None else out
    if (w.N, w.K) != (N, K):
        raise ValueError(f"out holds a [{w.N}, {w.K}] weight, W is [{N}, {K}]")
    _check(library().bsl_semi24_compress(W.data_ptr(), w.cref(), _stream(W)), "bsl_semi24_compress")
    return w


def forward24(X: torch.Tensor, w: Semi24Weight, bias: torch.Tensor | None = None,
              out: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X W^T (+ bias) on the sparse tensor-core kernel."""
    _cuda_bf16_2d(X, "X", w.K)
    bptr = _bias_ptr(bias, w.N, X)
    M = X.shape[0]
    Y = _out(M, w.N, X) if out is None else out
    _check(library().bsl_semi24_forward(X.data_ptr(), M, w.cref(), bptr, Y.data_ptr(), _stream(X)),
           "bsl_semi24_forward")
    return Y


def semi24_status(w: Semi24Weight) -> int:
    """Read and clear the weight's device status word (synchronises the stream)."""
    out = ctypes.c_int32(0)
    _check(library().bsl_semi24_get_status(w.cref(), ctypes.byref(out), _stream(w.values)),
           "bsl_semi24_get_status")
    return int(out.value)


class Semi24Linear(torch.nn.Module):
    """Inference ``nn.Linear`` with a 2:4 semi-structured weight: the torchao
    sparsity README's flow (introduction and its example) converts a trained
    linear layer's weight, pruned to two nonzeros in every four along K, into
    the compressed form and multiplies with the sparse tensor cores.  Built
    with :meth:`from_dense`; inputs may have any leading dimensions."""

    def __init__(self, weight24: Semi24Weight, bias: torch.Tensor | None = None):
        super().__init__()
        self.weight24 = weight24
        self.in_features, self.out_features = weight24.K, weight24.N
        if bias is not None:
            if bias.shape != (weight24.N,):
                raise ValueError("bias must have out_features entries")
            bias = bias.detach().to(device=weight24.device, dtype=torch.bfloat16).contiguous()
        self.register_buffer("bias", bias)

    @classmethod
    def from_dense(cls, weight: torch.Tensor, bias: torch.Tensor | None = None) -> "Semi24Linear":
        """Compress a [out_features, in_features] weight with at most two
        nonzeros in every group of four along in_features; raises BslError
        (BSL_ERR_NOT_2_4) if a group holds more."""
        w24 = compress24(weight.detach().to(torch.bfloat16).contiguous())
        st = semi24_status(w24)
        if st != 0:
            raise BslError(st, "Semi24Linear.from_dense")
        return cls(w24, bias)

    @torch.no_grad()
    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features)
        if x2.dtype != torch.bfloat16:
            x2 = x2.to(torch.bfloat16)
        y = forward24(x2.contiguous(), self.weight24, bias=self.bias)
        return y.reshape(*lead, self.out_features)


# ---------------------------------------------------------------- 2:4 inside blocks


class Bsr24Weight:
    """The kept blocks of a packed block-sparse weight in 2:4 compressed form
    ("50% sparse pattern within blocks", release note, "Future Development
    Roadmap"): ``values`` bf16 [nnz + 1, b, b/2] (the last block zeros) and
    ``meta`` [nnz, b, b/16] (16-bit position words held in an int16 tensor),
    beside the packed weight whose index and plan drive the kernel."""

    def __init__(self, packed: BsrWeight):
        b, nnz = packed.b, packed.nnz
        self.packed = packed
        self.values = torch.zeros((nnz + 1, b, b // 2), dtype=torch.bfloat16, device=packed.device)
        self.meta = torch.zeros((max(nnz, 1), b, b // 16), dtype=torch.int16, device=packed.device)

    @property
    def nnz(self):
        return self.packed.nnz


def compress_bsr24(Wp: BsrWeight, out: Bsr24Weight | None = None) -> Bsr24Weight:
    """Compress the kept blocks of ``Wp`` (2:4 along K inside each block).  A
    group with more than two nonzeros is reported by :func:`device_status`
    (BSL_ERR_NOT_2_4)."""
    w = Bsr24Weight(Wp) if out is None else out
    _check(library().bsl_bsr24_compress(Wp.cref(), w.values.data_ptr(), w.meta.data_ptr(),
                                        _stream(Wp.values)), "bsl_bsr24_compress")
    return w


def forward_bsr24(X: torch.Tensor, w: Bsr24Weight, bias: torch.Tensor | None = None,
                  out: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X W^T (+ bias) for a block-sparse weight with 2:4 blocks (b = 32 or 64)."""
    Wp = w.packed
    _cuda_bf16_2d(X, "X", Wp.K)
    bptr = _bias_ptr(bias, Wp.N, X)
    M = X.shape[0]
    Y = _out(M, Wp.N, X) if out is None else out
    _check(library().bsl_bsr24_forward(X.data_ptr(), M, Wp.cref(), w.values.data_ptr(), w.meta.data_ptr(),
                                       bptr, Y.data_ptr(), _stream(X)), "bsl_bsr24_forward")
    return Y
