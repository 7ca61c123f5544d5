"""Shared helpers of the GPU parity tests: run the hot path through the C ABI,
hand the same bytes to the CPU oracle, and compare.

Comparison rules (floating point: tolerances derived in the design notes; integer
work: exact):
  - outputs O: max |gpu - oracle| <= 2e-2 (bf16/f32 cache) or 6e-2 (e4m3 cache)
    and ||gpu - oracle||_2 / ||oracle||_2 <= 1e-2
  - importance scores: |gpu - oracle| <= 1e-4 * |oracle| + 1e-8 (fp32 logits,
    fp32 exp and sums over 16 heads)
  - selection: counts exact; the forced window always present; the global picks
    equal the oracle's except for positions whose oracle score lies within 1e-6
    of the oracle's cutoff score (several selections are then correct)
"""
import numpy as np
import torch

import kv_shared_b200 as hs
import oracle

TOL_MAXABS = {"f32": 2e-2, "bf16": 2e-2, "e4m3": 6e-2}
TOL_RELL2 = 1e-2
TIE_BAND = 1e-6


def f64(t):
    return t.detach().double().cpu().numpy()


def dtype_code(s):
    return {"f32": hs.HS2_F32, "bf16": hs.HS2_BF16, "e4m3": hs.HS2_E4M3}[s]


def compare_out(gpu, ref, kv_dtype, what="O"):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), what + ": non-finite values"
    err = np.abs(gpu - ref)
    rel = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err.max() <= TOL_MAXABS[kv_dtype], f"{what}: max abs err {err.max():.3e}"
    assert rel <= TOL_RELL2, f"{what}: rel L2 err {rel:.3e}"
    return float(err.max()), float(rel)


def compare_scores(gpu, ref, pos):
    """gpu/ref [rows, >= p+1]; only entries 0..p of each row are defined."""
    worst = 0.0
    for r, p in enumerate(pos):
        g = np.asarray(gpu[r, :p + 1], dtype=np.float64)
        o = ref[r, :p + 1]
        bad = np.abs(g - o) > 1e-4 * np.abs(o) + 1e-8
        assert not bad.any(), f"row {r}: {bad.sum()} scores out of tolerance, e.g. j={np.flatnonzero(bad)[:5]}"
        worst = max(worst, float((np.abs(g - o) / (np.abs(o) + 1e-30)).max()))
    return worst


def check_selection(g_idx, g_cnt, o_idx, o_cnt, o_scores, pos, W, band=TIE_BAND):
    """Returns the number of rows whose index set differs (all differences inside the tie band)."""
    g_idx = np.asarray(g_idx)
    g_cnt = np.asarray(g_cnt)
    np.testing.assert_array_equal(g_cnt, o_cnt)
    differing = 0
    for r, p in enumerate(pos):
        c = int(o_cnt[r])
        gi = g_idx[r, :c]
        assert (g_idx[r, c:] == -1).all(), f"row {r}: padding"
        assert (np.diff(gi) > 0).all(), f"row {r}: not ascending/unique"
        win = np.arange(max(p - W + 1, 0), p + 1)
        assert np.isin(win, gi).all(), f"row {r}: window missing"
        if np.array_equal(gi, o_idx[r, :c]):
            continue
        differing += 1
        gs = set(gi.tolist()) - set(win.tolist())
        os_ = set(o_idx[r, :c].tolist()) - set(win.tolist())
        assert len(gs) == len(os_)
        tau = min(o_scores[r, j] for j in os_)
        for j in gs ^ os_:
            assert abs(o_scores[r, j] - tau) <= band, \
                f"row {r}: position {j} differs, score {o_scores[r, j]:.9g} vs cutoff {tau:.9g}"
    return differing


class Dev:
    """Device copies of one workload's inputs in the cache layouts of the C ABI."""

    def __init__(self, inp, quantize_on_gpu=True):
        wl = inp.wl
        self.wl = wl
        dev = "cuda"
        self.q_full = inp.q_full.to(dev).contiguous()
        self.q_sparse = [q.to(dev).contiguous() for q in inp.q_sparse]
        self.k_scale = self.v_scale = None
        self.k_src, self.v_src = inp.k_src, inp.v_src      # generator output (host or device)
        self.k_in, self.v_in = inp.k, inp.v
        if wl.kv_dtype == "e4m3":
            ks = inp.k_src.to(dev).contiguous()
            vs = inp.v_src.to(dev).contiguous()
            B, T, D = ks.shape
            self.k = torch.empty((B, T, D), dtype=torch.uint8, device=dev)
            self.v = torch.empty_like(self.k)
            self.k_scale = torch.empty((B, T), dtype=torch.float32, device=dev)
            self.v_scale = torch.empty_like(self.k_scale)
            hs.hs2_kv_quantize_fp8(ks, B * T, D, self.k, self.k_scale)
            hs.hs2_kv_quantize_fp8(vs, B * T, D, self.v, self.v_scale)
        else:
            self.k = inp.k.to(dev).contiguous()
            self.v = inp.v.to(dev).contiguous()
        self.q_pos0 = torch.full((wl.batch,), wl.q_pos0, dtype=torch.int32, device=dev)
        qd = dtype_code(wl.q_dtype)
        self.desc = hs.make_desc(wl.batch, wl.n_q, wl.heads, wl.head_dim, wl.window, wl.budget,
                                 q_dtype=qd, kv_dtype=dtype_code(wl.kv_dtype), max_ctx=wl.ctx)
        self.ws = hs.alloc_workspace(self.desc, scores_in_workspace=False)
        B, n, H, D = self.q_full.shape
        odt = torch.float32 if wl.q_dtype == "f32" else torch.bfloat16
        self.o_full = torch.empty((B, n, H, D), dtype=odt, device=dev)
        self.lse = torch.empty((B, n, H), dtype=torch.float32, device=dev)
        self.scores = torch.zeros((B, n, wl.ctx), dtype=torch.float32, device=dev)
        self.idx = torch.empty((B, n, self.desc.idx_stride), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((B, n), dtype=torch.int32, device=dev)
        self.o_sparse = [torch.empty_like(self.o_full) for _ in self.q_sparse]

    def full(self):
        hs.hs2_full_attn_select(self.desc, self.q_full, self.k, self.v, self.k_scale, self.v_scale,
                                self.q_pos0, self.o_full, self.lse, self.idx, self.cnt, self.scores,
                                self.ws)

    def sparse(self, layer, idx=None, cnt=None, lse=None):
        hs.hs2_sparse_attn(self.desc, self.q_sparse[layer], self.k, self.v, self.k_scale, self.v_scale,
                           self.idx if idx is None else idx, self.cnt if cnt is None else cnt,
                           self.o_sparse[layer], lse, self.ws)

    def status(self):
        return hs.hs2_last_status(self.ws)

    # ---- oracle inputs: the generator's bytes; an e4m3 cache is quantized by the oracle itself
    def kv_f64(self, b):
        if self.wl.kv_dtype == "e4m3":
            out = []
            for src in (self.k_src, self.v_src):
                codes, scales = oracle.fp8_quantize(src[b].cpu().numpy())
                out.append(oracle.fp8_dequantize(codes, scales))
            return out[0], out[1]
        return f64(self.k_in[b]), f64(self.v_in[b])
