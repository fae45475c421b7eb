"""ctypes binding of libqlora_nf4.so (the C ABI in include/qlora_nf4.h).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.  There is
no fallback: if the library is missing, every call raises.
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "qlora_nf4.h")

QLORA_F32, QLORA_BF16 = 0, 1
STATUS_BYTES = 256
GEMV_MAX_M = 16

STATUS_NAMES = {
    0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARGUMENT", 2: "QLORA_ERR_UNSUPPORTED_SHAPE",
    3: "QLORA_ERR_MISALIGNED", 4: "QLORA_ERR_WORKSPACE_TOO_SMALL", 5: "QLORA_ERR_NONFINITE",
    6: "QLORA_ERR_TIMEOUT", 7: "QLORA_ERR_CUDA", 8: "QLORA_ERR_NO_DEVICE",
}


class QLoRAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")


class NF4TensorC(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("codes", ctypes.c_void_p),
                ("scale_codes", ctypes.c_void_p), ("c2", ctypes.c_void_p), ("scale_format", ctypes.c_int32)]


# qlora_scale_format
SCALE_FORMATS = {"e4m3": 0, "e5m2": 1, "u8": 2}


class LoraC(ctypes.Structure):
    _fields_ = [("r", ctypes.c_int32), ("alpha", ctypes.c_float), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p)]


class AdamWC(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float)]


_lib = None


def lib():
    """Loads the library once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with `python -m bit_nf4_quantized_27_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    pT, pL = ctypes.POINTER(NF4TensorC), ctypes.POINTER(LoraC)
    sigs = {
        "qlora_abi_version": (ctypes.c_int, []),
        "qlora_nf4_codebook": (None, [ctypes.POINTER(ctypes.c_float)]),
        "qlora_nf4_storage_bytes": (sz, [i64, i64, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz)]),
        "qlora_workspace_bytes": (sz, [i64, i64, i64, i32, ctypes.c_int]),
        "qlora_workspace_bytes_multi": (sz, [i64, i64, i64, i32]),
        "qlora_nf4_quantize": (ctypes.c_int, [vp, ctypes.c_int, pT, vp, vp]),
        "qlora_nf4_dequantize": (ctypes.c_int, [pT, vp, ctypes.c_int, vp]),
        "qlora_linear_fwd": (ctypes.c_int, [pT, pL, vp, i64, vp, ctypes.c_int, vp, vp, sz, vp]),
        "qlora_linear_bwd": (ctypes.c_int, [pT, pL, vp, vp, i64, vp, vp, ctypes.c_int, vp, vp, ctypes.c_int, vp,
                                            sz, vp]),
        "qlora_workspace_bytes_dropout": (sz, [i64, i64, i64, i32, ctypes.c_int]),
        "qlora_linear_fwd_dropout": (ctypes.c_int, [pT, pL, vp, vp, ctypes.c_float, i64, vp, ctypes.c_int, vp, vp,
                                                    sz, vp]),
        "qlora_linear_bwd_dropout": (ctypes.c_int, [pT, pL, vp, vp, vp, ctypes.c_float, i64, vp, vp, ctypes.c_int,
                                                    vp, vp, ctypes.c_int, vp, sz, vp]),
        "qlora_linear_fwd_multi": (ctypes.c_int, [pT, pL, i32, ctypes.POINTER(i32), vp, i64, vp, ctypes.c_int, vp,
                                                  sz, vp]),
        "qlora_lora_merge": (ctypes.c_int, [pT, pL, vp, vp]),
        "qlora_adamw_step": (ctypes.c_int, [vp, vp, vp, vp, vp, i64, ctypes.POINTER(AdamWC), i64, vp]),
        "qlora_selftest_bounded_wait": (ctypes.c_int, [vp, ctypes.c_uint32, vp]),
        "qlora_clear_status": (ctypes.c_int, [vp, vp]),
        "qlora_read_status": (ctypes.c_int, [vp, vp]),
        "qlora_read_library_status": (ctypes.c_int, [vp]),
        "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def header_functions() -> list[str]:
    """Names of the functions include/qlora_nf4.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_\w+)\s*\(", text)))


def _check(code: int, where: str):
    if code != 0:
        raise QLoRAError(code, where)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(dt):
    if dt == torch.float32:
        return QLORA_F32
    if dt == torch.bfloat16:
        return QLORA_BF16
    raise ValueError(f"unsupported dtype {dt}")


# ---------------------------------------------------------------------------
def codebook() -> list[float]:
    out = (ctypes.c_float * 16)()
    lib().qlora_nf4_codebook(out)
    return list(out)


def storage_bytes(rows: int, cols: int):
    c, s, g = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    total = lib().qlora_nf4_storage_bytes(rows, cols, ctypes.byref(c), ctypes.byref(s), ctypes.byref(g))
    return total, c.value, s.value, g.value


def workspace_bytes(m: int, n: int, k: int, r: int, backward: bool) -> int:
    return int(lib().qlora_workspace_bytes(m, n, k, r, 1 if backward else 0))


class NF4Weight:
    """A quantised [rows, cols] weight: three device buffers owned by torch."""

    def __init__(self, rows: int, cols: int, device="cuda", scale_format: str = "e4m3"):
        total, cb, sb, gb = storage_bytes(rows, cols)
        if total == 0:
            raise ValueError("cols must be a positive multiple of 64")
        if scale_format not in SCALE_FORMATS:
            raise ValueError(f"scale_format must be one of {sorted(SCALE_FORMATS)}")
        self.rows, self.cols = rows, cols
        self.scale_format = scale_format
        self.codes = torch.empty(cb, dtype=torch.uint8, device=device)
        self.scale_codes = torch.empty(sb, dtype=torch.uint8, device=device)
        self.c2 = torch.empty(gb // 4, dtype=torch.float32, device=device)

    def c_struct(self) -> NF4TensorC:
        return NF4TensorC(self.rows, self.cols, self.codes.data_ptr(), self.scale_codes.data_ptr(),
                          self.c2.data_ptr(), SCALE_FORMATS[self.scale_format])

    def nbytes(self) -> int:
        return self.codes.numel() + self.scale_codes.numel() + 4 * self.c2.numel()


def new_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    ws = torch.zeros(max(nbytes, STATUS_BYTES), dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def quantize(w: torch.Tensor, out: NF4Weight | None = None, ws: torch.Tensor | None = None,
             stream=None, scale_format: str | None = None) -> NF4Weight:
    """NF4 codes with double-quantised block scales; scale_format (default the
    weight's own, E4M3 for a new one) picks the 8-bit scale format."""
    assert w.is_cuda and w.is_contiguous() and w.dim() == 2
    q = out if out is not None else NF4Weight(w.shape[0], w.shape[1], w.device, scale_format or "e4m3")
    if scale_format is not None:
        q.scale_format = scale_format
    if ws is None:
        ws = new_workspace(STATUS_BYTES, w.device)
    t = q.c_struct()
    _check(lib().qlora_nf4_quantize(_ptr(w), _dtype_code(w.dtype), ctypes.byref(t), _ptr(ws), _stream(stream)),
           "qlora_nf4_quantize")
    q._status_ws = ws
    return q


def dequantize(q: NF4Weight, dtype=torch.bfloat16, out: torch.Tensor | None = None, stream=None):
    y = out if out is not None else torch.empty(q.rows, q.cols, dtype=dtype, device=q.codes.device)
    t = q.c_struct()
    _check(lib().qlora_nf4_dequantize(ctypes.byref(t), _ptr(y), _dtype_code(y.dtype), _stream(stream)),
           "qlora_nf4_dequantize")
    return y


def _lora(A: torch.Tensor, B: torch.Tensor, alpha: float) -> LoraC:
    assert A.dtype == torch.bfloat16 and B.dtype == torch.bfloat16
    assert A.is_contiguous() and B.is_contiguous()
    return LoraC(A.shape[0], float(alpha), A.data_ptr(), B.data_ptr())


def linear_fwd(q: NF4Weight, A, B, alpha: float, X, y_dtype=torch.bfloat16, save_t: bool = True,
               ws: torch.Tensor | None = None, out: torch.Tensor | None = None, t_out=None, stream=None):
    """Y = X W'^T + (alpha/r) (X A^T) B^T.  Returns (Y, T or None); T is the
    [2, M, r] bf16 pair (hi, lo) with hi + lo = X A^T."""
    M = X.shape[0]
    r = A.shape[0]
    assert X.dtype == torch.bfloat16 and X.is_contiguous() and X.shape[1] == q.cols
    Y = out if out is not None else torch.empty(M, q.rows, dtype=y_dtype, device=X.device)
    T = t_out if t_out is not None else (torch.empty(2, M, r, dtype=torch.bfloat16, device=X.device) if save_t else None)
    need = workspace_bytes(M, q.rows, q.cols, r, False)
    if ws is None:
        ws = new_workspace(need, X.device)
    t, ad = q.c_struct(), _lora(A, B, alpha)
    _check(lib().qlora_linear_fwd(ctypes.byref(t), ctypes.byref(ad), _ptr(X), M, _ptr(Y), _dtype_code(Y.dtype),
                                  _ptr(T), _ptr(ws), ws.numel(), _stream(stream)), "qlora_linear_fwd")
    return Y, T


def linear_bwd(q: NF4Weight, A, B, alpha: float, X, dY, T=None, dx_dtype=torch.bfloat16,
               grad_dtype=torch.bfloat16, ws: torch.Tensor | None = None, outs=None, stream=None):
    """Returns (dX, dA, dB) for upstream gradient dY."""
    M = X.shape[0]
    r = A.shape[0]
    assert dY.dtype == torch.bfloat16 and dY.is_contiguous() and dY.shape == (M, q.rows)
    if outs is not None:
        dX, dA, dB = outs
    else:
        dX = torch.empty(M, q.cols, dtype=dx_dtype, device=X.device)
        dA = torch.empty(r, q.cols, dtype=grad_dtype, device=X.device)
        dB = torch.empty(q.rows, r, dtype=grad_dtype, device=X.device)
    need = workspace_bytes(M, q.rows, q.cols, r, True)
    if ws is None:
        ws = new_workspace(need, X.device)
    t, ad = q.c_struct(), _lora(A, B, alpha)
    _check(lib().qlora_linear_bwd(ctypes.byref(t), ctypes.byref(ad), _ptr(X), _ptr(dY), M, _ptr(T), _ptr(dX),
                                  _dtype_code(dX.dtype), _ptr(dA), _ptr(dB), _dtype_code(dA.dtype), _ptr(ws),
                                  ws.numel(), _stream(stream)), "qlora_linear_bwd")
    return dX, dA, dB


def selftest_bounded_wait(ws: torch.Tensor, limit_us: int, stream=None):
    """Runs the device-side give-up protocol once: records QLORA_ERR_TIMEOUT in ws."""
    _check(lib().qlora_selftest_bounded_wait(_ptr(ws), int(limit_us), _stream(stream)),
           "qlora_selftest_bounded_wait")


def clear_status(ws: torch.Tensor, stream=None):
    _check(lib().qlora_clear_status(_ptr(ws), _stream(stream)), "qlora_clear_status")


def read_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns the device status code (0 = ok)."""
    return int(lib().qlora_read_status(_ptr(ws), _stream(stream)))


def read_library_status(stream=None) -> int:
    """Synchronises the stream, returns and clears the status code of the calls
    without a workspace (the merged export) on the current device (0 = ok)."""
    return int(lib().qlora_read_library_status(_stream(stream)))


class QLoRALinearFunction(torch.autograd.Function):
    """Autograd wrapper: the frozen NF4 weight gets no gradient; A, B and X do."""

    @staticmethod
    def forward(ctx, X, A, B, q: NF4Weight, alpha: float):
        Y, T = linear_fwd(q, A, B, alpha, X.contiguous())
        ctx.save_for_backward(X, A, B, T)
        ctx.q, ctx.alpha = q, alpha
        return Y

    @staticmethod
    def backward(ctx, dY):
        X, A, B, T = ctx.saved_tensors
        dX, dA, dB = linear_bwd(ctx.q, A, B, ctx.alpha, X, dY.contiguous().to(torch.bfloat16), T)
        return dX, dA, dB, None, None


def merge(q: NF4Weight, A, B, alpha: float, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Merged export W_merged [N, K] bf16 = bf16(W' + (alpha/r) B A)."""
    if out is None:
        out = torch.empty(q.rows, q.cols, dtype=torch.bfloat16, device=A.device)
    t, ad = q.c_struct(), _lora(A, B, alpha)
    _check(lib().qlora_lora_merge(ctypes.byref(t), ctypes.byref(ad), _ptr(out), _stream(stream)), "qlora_lora_merge")
    return out


def adamw_step(p: torch.Tensor, g: torch.Tensor, m: torch.Tensor, v: torch.Tensor, step: int, lr: float,
               beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
               p_bf16: torch.Tensor | None = None, stream=None) -> None:
    """One AdamW step in place on flat float32 tensors p, m, v with gradient g;
    writes bf16(p) to p_bf16 if given."""
    for t in (p, g, m, v):
        assert t.dtype == torch.float32 and t.is_contiguous() and t.numel() == p.numel()
    if p_bf16 is not None:
        assert p_bf16.dtype == torch.bfloat16 and p_bf16.is_contiguous() and p_bf16.numel() == p.numel()
    hp = AdamWC(lr, beta1, beta2, eps, weight_decay)
    _check(lib().qlora_adamw_step(_ptr(p), _ptr(p_bf16), _ptr(g), _ptr(m), _ptr(v), p.numel(), ctypes.byref(hp),
                                  step, _stream(stream)), "qlora_adamw_step")


def linear_fwd_multi(q: NF4Weight, adapters, adapter_of_token, X, y_dtype=torch.bfloat16,
                     ws: torch.Tensor | None = None, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode forward of one base serving several adapters: adapters is a list of
    (A, B, alpha) of one rank; token t uses adapters[adapter_of_token[t]]."""
    M = X.shape[0]
    r = adapters[0][0].shape[0]
    Y = out if out is not None else torch.empty(M, q.rows, dtype=y_dtype, device=X.device)
    arr = (LoraC * len(adapters))(*[_lora(a, b, alpha) for a, b, alpha in adapters])
    idx = (ctypes.c_int32 * M)(*[int(i) for i in adapter_of_token])
    if ws is None:
        ws = new_workspace(workspace_bytes_multi(M, q.rows, q.cols, r), X.device)
    t = q.c_struct()
    _check(lib().qlora_linear_fwd_multi(ctypes.byref(t), arr, len(adapters), idx, _ptr(X), M, _ptr(Y),
                                        _dtype_code(Y.dtype), _ptr(ws), ws.numel(), _stream(stream)),
           "qlora_linear_fwd_multi")
    return Y


def workspace_bytes_multi(m: int, n: int, k: int, r: int) -> int:
    return int(lib().qlora_workspace_bytes_multi(m, n, k, r))


def workspace_bytes_dropout(m: int, n: int, k: int, r: int, backward: bool) -> int:
    return int(lib().qlora_workspace_bytes_dropout(m, n, k, r, 1 if backward else 0))


def linear_fwd_dropout(q: NF4Weight, A, B, alpha: float, X, keep: torch.Tensor, p: float, y_dtype=torch.bfloat16,
                       save_t: bool = True, ws: torch.Tensor | None = None, stream=None):
    """Forward with LoRA dropout on the adapter input; keep is the packed
    uint8 [M, K/8] mask.  Returns (Y, T pair or None) as linear_fwd."""
    M, K = X.shape
    r = A.shape[0]
    assert keep.dtype == torch.uint8 and keep.is_contiguous() and tuple(keep.shape) == (M, K // 8)
    Y = torch.empty(M, q.rows, dtype=y_dtype, device=X.device)
    T = torch.empty(2, M, r, dtype=torch.bfloat16, device=X.device) if save_t else None
    if ws is None:
        ws = new_workspace(workspace_bytes_dropout(M, q.rows, q.cols, r, False), X.device)
    t, ad = q.c_struct(), _lora(A, B, alpha)
    _check(lib().qlora_linear_fwd_dropout(ctypes.byref(t), ctypes.byref(ad), _ptr(X), _ptr(keep), float(p), M,
                                          _ptr(Y), _dtype_code(Y.dtype), _ptr(T), _ptr(ws), ws.numel(),
                                          _stream(stream)), "qlora_linear_fwd_dropout")
    return Y, T


def linear_bwd_dropout(q: NF4Weight, A, B, alpha: float, X, dY, keep: torch.Tensor, p: float, T=None,
                       dx_dtype=torch.bfloat16, grad_dtype=torch.bfloat16, ws: torch.Tensor | None = None, stream=None):
    """Gradients (dX, dA, dB) of linear_fwd_dropout for upstream dY."""
    M, K = X.shape
    r = A.shape[0]
    dX = torch.empty(M, K, dtype=dx_dtype, device=X.device)
    dA = torch.empty(r, K, dtype=grad_dtype, device=X.device)
    dB = torch.empty(q.rows, r, dtype=grad_dtype, device=X.device)
    if ws is None:
        ws = new_workspace(workspace_bytes_dropout(M, q.rows, q.cols, r, True), X.device)
    t, ad = q.c_struct(), _lora(A, B, alpha)
    _check(lib().qlora_linear_bwd_dropout(ctypes.byref(t), ctypes.byref(ad), _ptr(X), _ptr(dY), _ptr(keep), float(p),
                                          M, _ptr(T), _ptr(dX), _dtype_code(dx_dtype), _ptr(dA), _ptr(dB),
                                          _dtype_code(grad_dtype), _ptr(ws), ws.numel(), _stream(stream)),
           "qlora_linear_bwd_dropout")
    return dX, dA, dB
