"""Helpers for the GPU parity tests: move seeded host inputs to the device,
call the C ABI through the binding, and bring results back as numpy."""
import numpy as np
import torch

from w4a4_post_quantization_dual_b200 import dq

DEV = "cuda"


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(DEV)


EIGHT_BIT = (dq.DQ_INT8, dq.DQ_MXINT8, dq.DQ_MXFP8)
BF16_SCALED = (dq.DQ_INT4, dq.DQ_INT8)


def gpu_act(X, c, fmt, G, xdtype=torch.bfloat16):
    M, K = X.shape
    Xd = to_dev(X.astype(np.float32), xdtype)
    cd = to_dev(np.asarray(c, np.float32)) if c is not None else None
    codes = torch.empty((M, K if fmt in EIGHT_BIT else K // 2), dtype=torch.uint8, device=DEV)
    nbytes = dq.scales_bytes(M, K, fmt, G)
    scales = torch.full((nbytes,), 0xAB, dtype=torch.uint8, device=DEV)  # poison padding
    st = torch.full((M,), -1.0, dtype=torch.float32, device=DEV) if fmt == dq.DQ_NVFP4 else None
    dq.dq_quantize_act(Xd, fmt, cd, codes, scales, st, group=G)
    torch.cuda.synchronize()
    sc = scales.cpu().numpy()
    if fmt in BF16_SCALED:
        sc = sc.view(np.uint16).reshape(M, K // G)
    return codes.cpu().numpy(), sc, (st.cpu().numpy() if st is not None else None)


def gpu_pack(W, r, c, sT, fmt, G, wdtype=torch.bfloat16):
    m, n = W.shape
    Wd = to_dev(W.astype(np.float32), wdtype)
    codes = torch.empty((m, n if fmt in EIGHT_BIT else n // 2), dtype=torch.uint8, device=DEV)
    scales = torch.full((dq.scales_bytes(m, n, fmt, G),), 0xAB, dtype=torch.uint8, device=DEV)
    sTd = to_dev(np.array([sT], np.float32))
    dq.dq_quantize_weight(Wd, fmt, to_dev(np.asarray(r, np.float32)),
                          to_dev(np.asarray(c, np.float32)), sTd, codes, scales, group=G)
    torch.cuda.synchronize()
    sc = scales.cpu().numpy()
    if fmt in BF16_SCALED:
        sc = sc.view(np.uint16).reshape(m, n // G)
    return codes.cpu().numpy(), sc


def gpu_solve(W, fmt, G, T, wdtype=torch.bfloat16, trace=True):
    m, n = W.shape
    Wd = to_dev(W.astype(np.float32), wdtype)
    r = torch.full((m, n // G), -1.0, dtype=torch.float32, device=DEV)
    c = torch.full((n,), -1.0, dtype=torch.float32, device=DEV)
    sT = torch.zeros(1, dtype=torch.float32, device=DEV)
    tr = torch.full((T + 1,), -1.0, dtype=torch.float64, device=DEV) if trace else None
    ws = torch.full((dq.solve_workspace_size(T),), 0x5A, dtype=torch.uint8, device=DEV)
    dq.dq_solve_scales(Wd, fmt, T, r, c, sT, tr, ws, group=G)
    torch.cuda.synchronize()
    return (r.cpu().numpy(), c.cpu().numpy(), float(sT.cpu()[0]),
            tr.cpu().numpy() if trace else None)


def gpu_linear(A, sA, st, B, sB, sW, M, N, K, fmt, yt=torch.float32, r_row=None):
    Y = torch.full((M, N), float("nan"), dtype=yt, device=DEV)
    dq.dq_w4a4_linear(to_dev(A), to_dev(sA), to_dev(st) if st is not None else None, to_dev(B),
                      to_dev(sB), to_dev(np.array([sW], np.float32)), Y, fmt,
                      r_row=to_dev(np.asarray(r_row, np.float32)) if r_row is not None else None)
    torch.cuda.synchronize()
    return Y.float().cpu().numpy()


def bf16_round(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def gpu_solve_ex(W, fmt, G, T, flags=0, r0=None, c0=None, s_T=None, wdtype=torch.bfloat16):
    """dq_solve_scales_ex on seeded host inputs; r0 / c0 / s_T (host) are
    copied into the output buffers, which the call reads in place."""
    m, n = W.shape
    Wd = to_dev(W.astype(np.float32), wdtype)
    r = (to_dev(np.asarray(r0, np.float32).reshape(m, n // G)) if r0 is not None else
         torch.full((m, n // G), -1.0, dtype=torch.float32, device=DEV))
    c = (to_dev(np.asarray(c0, np.float32).reshape(n)) if c0 is not None else
         torch.full((n,), -1.0, dtype=torch.float32, device=DEV))
    sT = to_dev(np.array([s_T if s_T is not None else 0.0], np.float32))
    tr = torch.full((T + 1,), -1.0, dtype=torch.float64, device=DEV)
    ws = torch.full((dq.solve_workspace_size(T),), 0x5A, dtype=torch.uint8, device=DEV)
    dq.dq_solve_scales_ex(Wd, fmt, T, r, c, sT, flags=flags,
                          r0=r if r0 is not None else None, c0=c if c0 is not None else None,
                          mse_trace=tr, workspace=ws, group=G)
    torch.cuda.synchronize()
    return r.cpu().numpy(), c.cpu().numpy(), float(sT.cpu()[0]), tr.cpu().numpy()
