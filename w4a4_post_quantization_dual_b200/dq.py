"""Thin Python binding of libdq.so (include/dq.h), same names as the C ABI.

Argument marshalling only: tensors are passed as raw device pointers with the
current torch CUDA stream; every step of the computation runs in the CUDA
kernels of libdq.so.  There is no CPU or PyTorch fallback: if the library is
missing or no GPU is present the call raises.
"""
import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libdq.so")

DQ_INT4, DQ_MXINT4, DQ_MXFP4, DQ_NVFP4 = 0, 1, 2, 3
DQ_INT8, DQ_MXINT8, DQ_MXFP8 = 4, 5, 6
EIGHT_BIT = (DQ_INT8, DQ_MXINT8, DQ_MXFP8)
DQ_F32, DQ_BF16 = 0, 1
FORMATS = {"int4": DQ_INT4, "mxint4": DQ_MXINT4, "mxfp4": DQ_MXFP4, "nvfp4": DQ_NVFP4,
           "int8": DQ_INT8, "mxint8": DQ_MXINT8, "mxfp8": DQ_MXFP8}
STATUS = {0: "DQ_OK", 1: "DQ_ERR_ARG", 2: "DQ_ERR_UNSUPPORTED", 3: "DQ_ERR_CUDA",
          4: "DQ_ERR_DEVICE_TIMEOUT", 5: "DQ_ERR_WORKSPACE"}

_lib = None
_vp, _i64, _int, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/dq.h
SIGNATURES = {
    "dq_status_string": (ctypes.c_char_p, [_int]),
    "dq_native_group": (_int, [_int]),
    "dq_scales_bytes": (_sz, [_i64, _i64, _int, _int]),
    "dq_solve_workspace_size": (_sz, [_int]),
    "dq_solve_scales": (_int, [_vp, _int, _i64, _i64, _int, _int, _int, _vp, _vp, _vp, _vp, _vp,
                               _sz, _vp]),
    "dq_solve_scales_ex": (_int, [_vp, _int, _i64, _i64, _int, _int, _int, ctypes.c_uint, _vp,
                                  _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "dq_quantize_weight": (_int, [_vp, _int, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp,
                                  _vp]),
    "dq_quantize_act": (_int, [_vp, _int, _i64, _i64, _vp, _int, _int, _vp, _vp, _vp, _vp]),
    "dq_w4a4_linear": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64,
                              _int, _vp]),
    "dq_solve_scales_noalloc": (_int, [_vp, _int, _i64, _i64, _int, _int, _int, _vp, _vp, _vp,
                                       _vp, _vp]),
    "dq_solve_batched_workspace_size": (_sz, [_int, _int]),
    "dq_solve_scales_batched": (_int, [_int, _vp, _int, _vp, _vp, _int, _int, _int, ctypes.c_uint,
                                       _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "dq_w4a4_linear_fused": (_int, [_vp, _int, _vp, _vp, _vp, _vp, _vp, _vp, _int, _i64, _i64,
                                    _i64, _int, _vp]),
    "dq_act_quant_error": (_int, [_vp, _int, _i64, _i64, _vp, _int, _int, _vp, _vp, _vp, _vp,
                                  _vp]),
    "dq_device_error": (_int, [_int]),
    "dq_set_wait_limit": (_int, [ctypes.c_uint64]),
    "dq_version": (_int, []),
}


class DQError(RuntimeError):
    pass


def lib():
    """Load libdq.so; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise DQError(f"{LIB_PATH} is missing: run python -m w4a4_post_quantization_dual_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status, what):
    if status != 0:
        raise DQError(f"{what}: {lib().dq_status_string(status).decode()}")


def _fmt(f):
    return FORMATS[f] if isinstance(f, str) else int(f)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise DQError("device tensor expected")
    if not t.is_contiguous():
        raise DQError("contiguous tensor expected")
    return t.data_ptr()


def _dtype(t):
    if t.dtype == torch.bfloat16:
        return DQ_BF16
    if t.dtype == torch.float32:
        return DQ_F32
    raise DQError(f"unsupported dtype {t.dtype}")


def _stream(stream):
    return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream


def native_group(fmt):
    return lib().dq_native_group(_fmt(fmt))


def scales_bytes(rows, k, fmt, group=0):
    return lib().dq_scales_bytes(rows, k, _fmt(fmt), group)


def solve_workspace_size(T):
    return lib().dq_solve_workspace_size(T)


def dq_solve_scales(W, fmt, T, r, c, s_tensor, mse_trace=None, workspace=None, group=0,
                    stream=None):
    """Algorithm 1 on W (m x n, bf16 or f32 CUDA tensor) into r, c, s_tensor."""
    m, n = W.shape
    if workspace is None:
        raise DQError("workspace required (solve_workspace_size(T) bytes)")
    _check(lib().dq_solve_scales(_ptr(W), _dtype(W), m, n, _fmt(fmt), group, T, _ptr(r), _ptr(c),
                                 _ptr(s_tensor), _ptr(mse_trace), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "dq_solve_scales")


DQ_SOLVE_ALPHA_ONLY, DQ_SOLVE_BETA_ONLY, DQ_SOLVE_KEEP_TENSOR_SCALE = 1, 2, 4
DQ_SOLVE_TRACE_CODES = 8


def dq_solve_scales_ex(W, fmt, T, r, c, s_tensor, flags=0, r0=None, c0=None, mse_trace=None,
                       workspace=None, group=0, stream=None):
    """Algorithm 1 with an ablation mode (DQ_SOLVE_ALPHA_ONLY / _BETA_ONLY),
    optional initial scales r0 / c0 and DQ_SOLVE_KEEP_TENSOR_SCALE (s_tensor
    read as input) -- see include/dq.h."""
    m, n = W.shape
    if workspace is None:
        raise DQError("workspace required (solve_workspace_size(T) bytes)")
    _check(lib().dq_solve_scales_ex(_ptr(W), _dtype(W), m, n, _fmt(fmt), group, T, flags,
                                    _ptr(r0), _ptr(c0), _ptr(r), _ptr(c), _ptr(s_tensor),
                                    _ptr(mse_trace), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(),
                                    _stream(stream)),
           "dq_solve_scales_ex")


def solve_batched_workspace_size(nw, T):
    return lib().dq_solve_batched_workspace_size(nw, T)


def dq_solve_scales_batched(Ws, fmt, T, rs, cs, sTs, traces=None, workspace=None, flags=0,
                            group=0, stream=None):
    """dq_solve_scales on a list of weights (same dtype) in few launches."""
    nw = len(Ws)
    if workspace is None:
        raise DQError("workspace required (solve_batched_workspace_size(nw, T) bytes)")
    if len({W.dtype for W in Ws}) != 1:
        raise DQError("all weights of a batch share one dtype")
    arr = lambda ts: (ctypes.c_void_p * nw)(*[_ptr(t) for t in ts])
    m = (ctypes.c_int64 * nw)(*[W.shape[0] for W in Ws])
    n = (ctypes.c_int64 * nw)(*[W.shape[1] for W in Ws])
    tr = arr(traces) if traces is not None else None
    _check(lib().dq_solve_scales_batched(nw, arr(Ws), _dtype(Ws[0]), m, n, _fmt(fmt), group, T,
                                         flags, arr(rs), arr(cs), arr(sTs), tr, _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(stream)),
           "dq_solve_scales_batched")


def dq_solve_scales_noalloc(W, fmt, T, r, c, s_tensor, mse_trace=None, group=0, stream=None):
    """dq_solve_scales without a workspace: the library's fixed scratch array
    is used instead (T <= 2045; calls on one device must not overlap)."""
    m, n = W.shape
    _check(lib().dq_solve_scales_noalloc(_ptr(W), _dtype(W), m, n, _fmt(fmt), group, T, _ptr(r),
                                         _ptr(c), _ptr(s_tensor), _ptr(mse_trace),
                                         _stream(stream)),
           "dq_solve_scales_noalloc")


def dq_quantize_weight(W, fmt, r, c, s_tensor, codes, scales, group=0, stream=None):
    m, n = W.shape
    _check(lib().dq_quantize_weight(_ptr(W), _dtype(W), m, n, _fmt(fmt), group, _ptr(r), _ptr(c),
                                    _ptr(s_tensor), _ptr(codes), _ptr(scales), _stream(stream)),
           "dq_quantize_weight")


def dq_quantize_act(X, fmt, c, codes, scales, s_tok=None, group=0, stream=None):
    M, K = X.shape
    _check(lib().dq_quantize_act(_ptr(X), _dtype(X), M, K, _ptr(c), _fmt(fmt), group, _ptr(codes),
                                 _ptr(scales), _ptr(s_tok), _stream(stream)),
           "dq_quantize_act")


def dq_w4a4_linear(A, sA, s_tok, B, sB, s_w, Y, fmt, r_row=None, stream=None):
    M, KB = A.shape                 # code bytes per row: K/2 (4-bit) or K (8-bit)
    N = B.shape[0]
    K = KB if _fmt(fmt) in (DQ_INT8, DQ_MXINT8, DQ_MXFP8) else 2 * KB
    _check(lib().dq_w4a4_linear(_ptr(A), _ptr(sA), _ptr(s_tok), _ptr(B), _ptr(sB), _ptr(s_w),
                                _ptr(r_row), _ptr(Y), _dtype(Y), M, N, K, _fmt(fmt),
                                _stream(stream)),
           "dq_w4a4_linear")


def dq_act_quant_error(X, fmt, c, codes, scales, s_tok, sums, group=0, stream=None):
    """sums[0] = sum x^2, sums[1] = sum (x - x^)^2 of the activation path (include/dq.h)."""
    M, K = X.shape
    _check(lib().dq_act_quant_error(_ptr(X), _dtype(X), M, K, _ptr(c), _fmt(fmt), group,
                                    _ptr(codes), _ptr(scales), _ptr(s_tok), _ptr(sums),
                                    _stream(stream)),
           "dq_act_quant_error")


def dq_w4a4_linear_fused(X, c, B, sB, s_w, Y, fmt, r_row=None, stream=None):
    """Activation quantisation + linear in one kernel (small M, NVFP4, bf16 X)."""
    M, K = X.shape
    N = B.shape[0]
    _check(lib().dq_w4a4_linear_fused(_ptr(X), _dtype(X), _ptr(c), _ptr(B), _ptr(sB), _ptr(s_w),
                                      _ptr(r_row), _ptr(Y), _dtype(Y), M, N, K, _fmt(fmt),
                                      _stream(stream)),
           "dq_w4a4_linear_fused")


def dq_device_error(clear=True):
    return lib().dq_device_error(1 if clear else 0)


def dq_set_wait_limit(ns=0):
    """Limit of the device-side bounded waits in ns (0: the 2 s default)."""
    _check(lib().dq_set_wait_limit(int(ns)), "dq_set_wait_limit")


# ----------------------------------------------------------------------------
# Convenience: allocate outputs (torch) and run the calls above.
# ----------------------------------------------------------------------------
class QuantizedLinear:
    """Artefacts of one linear layer (Section 4.4): packed codes What, encoded
    row-block scales (alpha^-1), column scales c (beta^-1) and the NVFP4
    per-tensor scale -- all device tensors."""

    def __init__(self, codes, scales, c, s_tensor, fmt, group, shape):
        self.codes, self.scales, self.c, self.s_tensor = codes, scales, c, s_tensor
        self.fmt, self.group, self.shape = _fmt(fmt), group, shape


def quantize_linear(W, fmt, T, group=0, mse_trace=False):
    """Solve the dual scales of W and pack it.  Returns (QuantizedLinear, r, trace)."""
    dev = W.device
    m, n = W.shape
    G = group or native_group(fmt)
    r = torch.empty((m, n // G), dtype=torch.float32, device=dev)
    c = torch.empty(n, dtype=torch.float32, device=dev)
    sT = torch.empty(1, dtype=torch.float32, device=dev)
    tr = torch.empty(T + 1, dtype=torch.float64, device=dev) if mse_trace else None
    ws = torch.empty(solve_workspace_size(T), dtype=torch.uint8, device=dev)
    dq_solve_scales(W, fmt, T, r, c, sT, tr, ws, group=G)
    codes = torch.empty((m, n if _fmt(fmt) in EIGHT_BIT else n // 2), dtype=torch.uint8,
                        device=dev)
    scales = torch.empty(scales_bytes(m, n, fmt, G), dtype=torch.uint8, device=dev)
    dq_quantize_weight(W, fmt, r, c, sT, codes, scales, group=G)
    return QuantizedLinear(codes, scales, c, sT, fmt, G, (m, n)), r, tr


def act_sqnr_db(X, fmt, c=None, group=0):
    """Activation SQNR (dB) of the W4A4 activation path on device activations X:
    rescale by c (None: without beta), quantise, and compare the dequantised
    activations mapped back by 1/c with X (Appendix E, Table 6)."""
    M, K = X.shape
    dev = X.device
    G = group or native_group(fmt)
    A = torch.empty((M, K if _fmt(fmt) in EIGHT_BIT else K // 2), dtype=torch.uint8,
                    device=dev)
    sA = torch.empty(scales_bytes(M, K, fmt, G), dtype=torch.uint8, device=dev)
    st = torch.empty(M, dtype=torch.float32, device=dev) if _fmt(fmt) == DQ_NVFP4 else None
    sums = torch.empty(2, dtype=torch.float64, device=dev)
    dq_quantize_act(X, fmt, c, A, sA, st, group=G)
    dq_act_quant_error(X, fmt, c, A, sA, st, sums, group=G)
    s = sums.cpu()
    return 10.0 * math.log10(float(s[0]) / float(s[1])) if float(s[1]) > 0 else math.inf


def linear(X, q: QuantizedLinear, out_dtype=torch.bfloat16, r_row=None):
    """Y = X W^T through the W4A4 path: fused rescale+quantise, block-scaled GEMM."""
    M, K = X.shape
    dev = X.device
    A = torch.empty((M, K if q.fmt in EIGHT_BIT else K // 2), dtype=torch.uint8, device=dev)
    sA = torch.empty(scales_bytes(M, K, q.fmt, q.group), dtype=torch.uint8, device=dev)
    st = torch.empty(M, dtype=torch.float32, device=dev) if q.fmt == DQ_NVFP4 else None
    dq_quantize_act(X, q.fmt, q.c, A, sA, st, group=q.group)
    Y = torch.empty((M, q.shape[0]), dtype=out_dtype, device=dev)
    dq_w4a4_linear(A, sA, st, q.codes, q.scales, q.s_tensor, Y, q.fmt, r_row=r_row)
    return Y
