"""Seeded synthetic inputs for the HySparse2 hybrid-block hot path.

This module holds no arithmetic of the method: it only draws random tensors,
rounds them to the storage dtype and plants "needle" keys.  Both the CUDA path
and the CPU oracle consume what it produces; it imports neither.

The shapes follow the agent workload the pages describe (short actions, long
observations, a context that keeps growing to one million tokens; Agentik
explainer, "1. Agentic inference as the driving workload").  The retrieval
benchmarks the pages quote are not available here; planted keys stand in for
the "truly relevant content" that token-level selection should find.

Draws use torch generators seeded per (seed, stream): on the CPU for small
cases, on the GPU for the full-size workloads (a host draw of ~1e9 normals takes
minutes).  Values are drawn in fp32 and rounded to nearest-even bf16 by torch.
"""
from dataclasses import dataclass, field, replace
from typing import List, Optional

import torch

WINDOW = 128
BUDGET = 1024

# stream ids so every tensor has its own reproducible sub-stream
_S_QFULL, _S_QSPARSE, _S_K, _S_V, _S_NEEDLE, _S_HIDDEN, _S_W = range(7)


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q: int                 # query rows per sequence (1 = decode)
    ctx: int                 # keys visible to the last query row (cache rows in use)
    heads: int
    head_dim: int
    kv_dtype: str            # "f32" | "bf16" | "e4m3"
    n_sparse: int = 3
    window: int = WINDOW
    budget: int = BUDGET
    kv_std: float = 1.0      # std of the noise keys/values
    needles: int = 0         # planted keys per sequence (decode workloads)
    needle_norm: float = 0.0  # norm of a planted key (along the summed-query direction)
    needle_layout: str = "uniform"   # "uniform" | "one_per_block" | "packed16"
    n_new: int = 0           # rows produced by the KV-bridge projection (prefill)
    d_model: int = 0         # hidden size feeding the projection
    block_size: int = 1      # 1 = token-level selection, 64 = block-level arm

    @property
    def q_pos0(self) -> int:
        return self.ctx - self.n_q

    @property
    def q_dtype(self) -> str:
        return "f32" if self.kv_dtype == "f32" else "bf16"


# The five workloads (the first is small enough for the oracle on every row).
TINY = Workload("tiny_prefill_ctx2048_h8_d64_f32", batch=1, n_q=2048, ctx=2048, heads=8,
                head_dim=64, kv_dtype="f32", n_sparse=1)
DECODE_128K = Workload("decode_b32_ctx131072_h16_d128_bf16", batch=32, n_q=1, ctx=131072,
                       heads=16, head_dim=128, kv_dtype="bf16", kv_std=128 ** -0.5,
                       needles=16, needle_norm=4.0)
PREFILL_AGENT = Workload("prefill_b4_ctx65536+8192_h16_d128_bf16", batch=4, n_q=8192,
                         ctx=65536 + 8192, heads=16, head_dim=128, kv_dtype="bf16",
                         n_new=8192, d_model=2048)
DECODE_1M_FP8 = Workload("decode_b4_ctx1048576_h16_d128_e4m3", batch=4, n_q=1, ctx=1 << 20,
                         heads=16, head_dim=128, kv_dtype="e4m3", needles=32,
                         needle_norm=4.0 * 128 ** 0.5)


# Not one of the five: the 128K decode shape with the e4m3 cache recipe of the 1M workload
# (the single-launch decode kernel on an e4m3 cache; informational in the bench).
DECODE_128K_FP8 = Workload("decode_b32_ctx131072_h16_d128_e4m3", batch=32, n_q=1, ctx=131072,
                           heads=16, head_dim=128, kv_dtype="e4m3", needles=16,
                           needle_norm=4.0 * 128 ** 0.5)


# Not one of the five: the agent-round prefill shape against an e4m3 cache (all rows of
# the N(0,1) source quantized per token; the bridge's e4m3 output is timed on its own).
PREFILL_AGENT_FP8 = Workload("prefill_b4_ctx65536+8192_h16_d128_e4m3", batch=4, n_q=8192,
                             ctx=65536 + 8192, heads=16, head_dim=128, kv_dtype="e4m3")


def sweep(ctx: int, block_size: int = 1, layout: str = "one_per_block") -> Workload:
    """Selection-granularity sweep: one sequence, decode at p = ctx - 1, 64 planted tokens."""
    return Workload(f"sweep_ctx{ctx}_{'token' if block_size == 1 else 'block%d' % block_size}",
                    batch=1, n_q=1, ctx=ctx, heads=16, head_dim=128, kv_dtype="bf16",
                    n_sparse=1, needles=64, needle_norm=4.0 * 128 ** 0.5,
                    needle_layout=layout, block_size=block_size)


SWEEP_CTX = (4096, 32768, 262144, 1 << 20)


def shrink(wl: Workload, **kw) -> Workload:
    """Same workload recipe at other sizes (parity cases the oracle finishes quickly)."""
    return replace(wl, **kw)


@dataclass
class Inputs:
    wl: Workload
    q_full: torch.Tensor                 # [B, n_q, H, D] q dtype
    q_sparse: List[torch.Tensor]         # n_sparse x [B, n_q, H, D]
    k: Optional[torch.Tensor] = None     # [B, ctx, D] f32 or bf16 (None for e4m3 before quantizing)
    v: Optional[torch.Tensor] = None
    k_src: Optional[torch.Tensor] = None  # [B, ctx, D] fp32 source values (e4m3 workloads)
    v_src: Optional[torch.Tensor] = None
    hidden: Optional[torch.Tensor] = None  # [B, n_new, d_model] bf16 (prefill)
    w_kv: Optional[torch.Tensor] = None    # [d_model, 2D] bf16
    needle_pos: Optional[torch.Tensor] = None  # [B, needles] int64
    extra: dict = field(default_factory=dict)


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1000003 + stream * 7919) % (2 ** 63))
    return g


def _normal(shape, std, seed, stream, device, chunk_rows=None):
    g = _gen(seed, stream, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).mul_(std)


def _needle_positions(wl: Workload, seed: int, device) -> torch.Tensor:
    """Planted positions, all before the forced window (so only global selection finds them)."""
    g = _gen(seed, _S_NEEDLE, "cpu")
    hi = wl.ctx - wl.window          # candidates are [0, ctx - W - 1] for p = ctx - 1
    out = []
    for _ in range(wl.batch):
        if wl.needle_layout == "uniform":
            pos = torch.randperm(hi, generator=g)[:wl.needles]
        else:
            bs = 64
            nb = hi // bs
            if wl.needle_layout == "one_per_block":
                # distinct blocks while there are enough of them (a short context
                # with fewer blocks than planted tokens reuses blocks, never positions)
                reps = -(-wl.needles // nb)
                blocks = torch.cat([torch.randperm(nb, generator=g) for _ in range(reps)])[:wl.needles]
                perm = torch.stack([torch.randperm(bs, generator=g) for _ in range(nb)])
                occ = torch.arange(wl.needles) // nb
                pos = blocks * bs + perm[blocks, occ]
            else:   # packed16: 16 planted tokens in each of needles/16 blocks
                nblk = wl.needles // 16
                blocks = torch.randperm(nb, generator=g)[:nblk]
                pos = torch.cat([b * bs + torch.randperm(bs, generator=g)[:16] for b in blocks])
        out.append(torch.sort(pos.to(torch.int64)).values)
    return torch.stack(out).to(device)


def make_inputs(wl: Workload, seed: int = 0, device="cpu") -> Inputs:
    B, n, H, D, T = wl.batch, wl.n_q, wl.heads, wl.head_dim, wl.ctx
    qdt = torch.float32 if wl.q_dtype == "f32" else torch.bfloat16
    q_full = _normal((B, n, H, D), 1.0, seed, _S_QFULL, device).to(qdt)
    q_sparse = [_normal((B, n, H, D), 1.0, seed, _S_QSPARSE * 100 + l, device).to(qdt)
                for l in range(wl.n_sparse)]
    k = _normal((B, T, D), wl.kv_std, seed, _S_K, device)
    v = _normal((B, T, D), wl.kv_std, seed, _S_V, device)
    inp = Inputs(wl=wl, q_full=q_full, q_sparse=q_sparse)

    if wl.needles:
        pos = _needle_positions(wl, seed, device)
        u = q_full[:, -1].float().sum(dim=1)                 # [B, D] summed query direction
        u = u / u.norm(dim=1, keepdim=True)
        for b in range(B):
            k[b, pos[b]] = wl.needle_norm * u[b]
        inp.needle_pos = pos

    if wl.n_new:
        # rows [ctx - n_new, ctx) are produced by the bridge projection of hidden states;
        # hidden ~ N(0,1), W ~ N(0, 1/d_model) so the projected rows are ~N(0,1) like the rest
        inp.hidden = _normal((B, wl.n_new, wl.d_model), 1.0, seed, _S_HIDDEN, device).to(torch.bfloat16)
        inp.w_kv = _normal((wl.d_model, 2 * D), wl.d_model ** -0.5, seed, _S_W, device).to(torch.bfloat16)
        k[:, T - wl.n_new:] = 0
        v[:, T - wl.n_new:] = 0

    if wl.kv_dtype == "e4m3":
        inp.k_src, inp.v_src = k, v
    elif wl.kv_dtype == "bf16":
        inp.k, inp.v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    else:
        inp.k, inp.v = k, v
    return inp


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


__all__ = ["Workload", "Inputs", "make_inputs", "shrink", "sweep", "TINY", "DECODE_128K",
           "PREFILL_AGENT", "PREFILL_AGENT_FP8", "DECODE_1M_FP8", "SWEEP_CTX", "WINDOW", "BUDGET", "bf16_bits"]
