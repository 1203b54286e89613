"""Whole-model quantisation sweep: solve and pack every linear weight of a
model, in one format, with the weights partitioned over ranks.

DualQuant, Appendix I: the deployed model has all 224 linears of
Llama-3.1-8B quantised (q, k, v, o, gate, up, down in each of 32 layers),
solved offline and packed.  Every weight is an independent problem, so on N
ranks each rank takes its round-robin share and solves it with no exchange;
only the bookkeeping (which weight went where, what it packed to) is
gathered afterwards.  This module is orchestration: the solve and the
packing run in libdq.so's kernels through the dq binding.
"""
import torch

from . import dist

# (name, rows m = output features, columns n = input features)
LLAMA8B_LAYER = (("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
                 ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336))


def llama8b_linears(layers=32):
    """[(name, m, n)] of the linear weights of a Llama-3.1-8B-shaped model."""
    return [(f"layers.{l}.{name}", m, n) for l in range(layers) for name, m, n in LLAMA8B_LAYER]


def student_t_weight(m, n, seed, device, std=0.02):
    """A random bf16 m x n weight, Student-t(4) with standard deviation `std`,
    drawn on the device (t4 = z / sqrt(chi2_4 / 4), chi2_4 a sum of four
    squared normals; t4 has variance 2)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    z = torch.randn(m, n, device=device, generator=g)
    chi = torch.zeros(m, n, device=device)
    for _ in range(4):
        e = torch.randn(m, n, device=device, generator=g)
        chi.addcmul_(e, e)
    w = z.mul_(torch.rsqrt(chi.mul_(0.25))).mul_(std / 2 ** 0.5)
    return w.to(torch.bfloat16)


def solve_and_pack(weights, fmt, T, group=0, stream=None):
    """Solve the dual scales of every weight (one dq_solve_scales_batched call,
    which groups weights of one row count into shared launches) and pack each.
    Returns a list of dq.QuantizedLinear, one per weight, in order."""
    from . import dq
    if not weights:
        return []
    dev = weights[0].device
    G = group or dq.native_group(fmt)
    rs = [torch.empty((W.shape[0], W.shape[1] // G), dtype=torch.float32, device=dev)
          for W in weights]
    cs = [torch.empty(W.shape[1], dtype=torch.float32, device=dev) for W in weights]
    sTs = [torch.empty(1, dtype=torch.float32, device=dev) for _ in weights]
    ws = torch.empty(dq.solve_batched_workspace_size(len(weights), T), dtype=torch.uint8,
                     device=dev)
    dq.dq_solve_scales_batched(weights, fmt, T, rs, cs, sTs, None, ws, group=G, stream=stream)
    eight = dq._fmt(fmt) in dq.EIGHT_BIT
    out = []
    for W, r, c, sT in zip(weights, rs, cs, sTs):
        m, n = W.shape
        codes = torch.empty((m, n if eight else n // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty(dq.scales_bytes(m, n, fmt, G), dtype=torch.uint8, device=dev)
        dq.dq_quantize_weight(W, fmt, r, c, sT, codes, scales, group=G, stream=stream)
        out.append(dq.QuantizedLinear(codes, scales, c, sT, fmt, G, (m, n)))
    return out


def run(linears, make_weight, solve, rank=0, world=1):
    """This rank's share of a sweep.  linears: [(name, m, n)]; make_weight(i)
    gives weight i; solve(list of weights) gives one result per weight.
    Returns {name: result} for the weights this rank owns."""
    mine = dist.shard(len(linears), rank, world)
    results = solve([make_weight(i) for i in mine])
    return {linears[i][0]: res for i, res in zip(mine, results)}


def packed_summary(q):
    """Host-side bookkeeping of one packed weight: its shape and byte counts."""
    return {"shape": list(q.shape), "code_bytes": q.codes.numel(),
            "scale_bytes": q.scales.numel(), "c_bytes": 4 * q.c.numel()}


def gather(local, rank=0, world=1):
    """{name: host-side summary} of every rank, merged on every rank (a
    collective of small host objects; nothing on the data path)."""
    if world == 1 or not torch.distributed.is_initialized():
        return dict(local)
    parts = [None] * world
    torch.distributed.all_gather_object(parts, local)
    merged = {}
    for p in parts:
        for k, v in p.items():
            if k in merged:
                raise RuntimeError(f"weight {k} solved by two ranks")
            merged[k] = v
    return merged
