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


def compare_scores(gpu, ref, pos, bridged_from=None):
    """gpu/ref [rows, >= p+1]; only entries 0..p of each row are defined.

    Keys at positions >= bridged_from come from the KV-bridge projection, whose GPU
    result may differ from the oracle's by one bf16 ulp in an element (fp32 versus
    exact accumulation before rounding); one ulp (<= 2^-7 relative) moves that key's
    logit by <= scale * sum_d |q_d| |k_d| 2^-7, i.e. up to ~1e-2 relative in its
    probabilities at these magnitudes, so those keys get rtol 1e-2."""
    worst = 0.0
    for r, p in enumerate(pos):
        g = np.asarray(gpu[r, :p + 1], dtype=np.float64)
        o = ref[r, :p + 1]
        rtol = np.full(p + 1, 1e-4)
        if bridged_from is not None:
            rtol[bridged_from:] = 1e-2
        bad = np.abs(g - o) > rtol * np.abs(o) + 1e-8
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
        """Oracle K/V of sequence b (fp64) from the generator's bytes."""
        if self.wl.kv_dtype == "e4m3":
            out = []
            for src in (self.k_src, self.v_src):
                codes, scales = oracle.fp8_quantize(src[b].cpu().numpy())
                out.append(oracle.fp8_dequantize(codes, scales))
            return out[0], out[1]
        return f64(self.k_in[b]), f64(self.v_in[b])


def _dev_bridge(self):
    """KV bridging on the GPU: rows [ctx - n_new, ctx) of every sequence's cache."""
    wl = self.wl
    self.pos0_new = torch.full((wl.batch,), wl.ctx - wl.n_new, dtype=torch.int32, device="cuda")
    hs.hs2_kv_bridge_proj(self.hidden, self.w_kv, wl.batch, wl.n_new, wl.d_model, wl.head_dim,
                          self.pos0_new, wl.ctx, self.k, self.v)


def _oracle_bridged_kv(self, b, k, v):
    """The oracle's own bridge rows (fp64 product rounded to bf16) replace the placeholders."""
    wl = self.wl
    kk, vv = oracle.bridge(f64(self.hidden_in[b]), f64(self.w_in), wl.head_dim)
    k = k.copy()
    v = v.copy()
    k[wl.ctx - wl.n_new:] = oracle.bf16_to_f64(oracle.round_bf16(kk))
    v[wl.ctx - wl.n_new:] = oracle.bf16_to_f64(oracle.round_bf16(vv))
    return k, v


Dev.bridge = _dev_bridge
Dev.oracle_bridged_kv = _oracle_bridged_kv


def block_parity(wl, seed, seqs=None, device="cpu", rows=None, pos0=None):
    """Runs the hybrid block through the C ABI and checks it against the oracle on the
    given sequences and query rows (all by default).  `pos0` gives each sequence its own
    first query position (ragged batch); by default every sequence ends at the context."""
    import synth
    inp = synth.make_inputs(wl, seed=seed, device=device)
    dev = Dev(inp)
    if pos0 is not None:
        dev.q_pos0 = torch.tensor(pos0, dtype=torch.int32, device="cuda")
    if wl.n_new:
        dev.hidden_in, dev.w_in = inp.hidden, inp.w_kv
        dev.hidden = inp.hidden.to("cuda").contiguous()
        dev.w_kv = inp.w_kv.to("cuda").contiguous()
        dev.bridge()
    dev.full()
    for l in range(wl.n_sparse):
        dev.sparse(l)
    assert dev.status() == hs.HS2_OK
    seqs = range(wl.batch) if seqs is None else seqs
    rows = np.arange(wl.n_q) if rows is None else np.asarray(rows)
    report = {"differing_rows": 0, "rows": 0}
    for b in seqs:
        pos = (wl.q_pos0 if pos0 is None else int(pos0[b])) + rows
        k, v = dev.kv_f64(b)
        if wl.n_new:
            k, v = dev.oracle_bridged_kv(b, k, v)
        qf = f64(inp.q_full[b])[rows]
        o_ref, lse_ref, sc_ref = oracle.full_attn(qf, k, v, pos)
        compare_out(f64(dev.o_full[b])[rows], o_ref, wl.kv_dtype, "O_full")
        np.testing.assert_allclose(dev.lse[b].cpu().numpy()[rows], lse_ref, rtol=1e-4, atol=1e-4)
        compare_scores(dev.scores[b, torch.from_numpy(rows).cuda()].cpu().numpy(), sc_ref, pos,
                       bridged_from=(wl.ctx - wl.n_new) if wl.n_new else None)
        o_idx, o_cnt = oracle.select_rows(sc_ref, pos, wl.window, wl.budget, block_size=wl.block_size)
        g_idx = dev.idx[b].cpu().numpy()[rows]
        g_cnt = dev.cnt[b].cpu().numpy()[rows]
        report["differing_rows"] += check_selection(g_idx, g_cnt, o_idx, o_cnt, sc_ref, pos, wl.window)
        report["rows"] += len(rows)
        if inp.needle_pos is not None and wl.block_size == 1 and pos0 is None:
            sel = set(g_idx[-1, :g_cnt[-1]].tolist())
            assert set(inp.needle_pos[b].tolist()) <= sel, "planted key not selected"
        same = np.array([np.array_equal(g_idx[r], o_idx[r]) for r in range(len(rows))])
        oi = torch.from_numpy(o_idx[None]).cuda()
        oc = torch.from_numpy(o_cnt[None]).cuda()
        rsel = torch.from_numpy(rows).cuda()
        for l in range(wl.n_sparse):
            o_sp_ref = oracle.sparse_attn(f64(inp.q_sparse[l][b])[rows], k, v, o_idx, o_cnt)
            # end to end (GPU indices) where the index sets agree
            if same.any():
                compare_out(f64(dev.o_sparse[l][b])[rows][same], o_sp_ref[same], wl.kv_dtype, f"O_sparse{l}")
            # and the kernel alone on the oracle's selection, every sampled row
            desc1 = hs.make_desc(1, len(rows), wl.heads, wl.head_dim, wl.window, wl.budget,
                                 q_dtype=dev.desc.q_dtype, kv_dtype=dev.desc.kv_dtype, max_ctx=wl.ctx)
            q1 = dev.q_sparse[l][b][rsel].unsqueeze(0).contiguous()
            o1 = torch.empty_like(q1)
            ws1 = hs.alloc_workspace(desc1)
            ks = dev.k_scale[b:b + 1] if dev.k_scale is not None else None
            vs = dev.v_scale[b:b + 1] if dev.v_scale is not None else None
            hs.hs2_sparse_attn(desc1, q1, dev.k[b:b + 1].contiguous(), dev.v[b:b + 1].contiguous(), ks, vs,
                               oi, oc, o1, None, ws1)
            compare_out(f64(o1[0]), o_sp_ref, wl.kv_dtype, f"O_sparse{l}_oracle_idx")
    return report
