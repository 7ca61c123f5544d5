"""Pins for the oracle's number formats (CPU only).

bf16 rounding against torch's float32 -> bfloat16 cast (exact for inputs that
are float32 values) and against a brute-force nearest-value search; e4m3
decoding and encoding against torch.float8_e4m3fn and a brute-force search over
all finite codes; the per-token FP8 quantizer against torch's fp32 division and
cast, and its error bound.
"""
import numpy as np
import torch

import oracle


def test_bf16_to_f64_matches_torch():
    bits = np.arange(0, 65536, dtype=np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    ours = oracle.bf16_to_f64(bits)
    finite = np.isfinite(t)
    np.testing.assert_array_equal(ours[finite], t[finite])


def test_round_bf16_matches_torch_on_float32_values():
    rng = np.random.default_rng(0)
    x32 = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                          (rng.standard_normal(1000) * 1e-38).astype(np.float32),
                          np.array([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8), 0.0, -0.0], np.float32)])
    ours = oracle.round_bf16(x32.astype(np.float64))
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_round_bf16_ties_to_even():
    vals = np.array([1 + 2**-8, 1 + 3 * 2**-8, 2 + 2**-7, 1 + 2**-8 + 2**-40])
    got = oracle.bf16_to_f64(oracle.round_bf16(vals))
    np.testing.assert_array_equal(got, [1.0, 1 + 2**-6, 2.0, 1 + 2**-7])


def test_round_bf16_brute_force_on_doubles():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(2000) * 3
    table_bits = np.arange(0, 0x7F80, dtype=np.uint16)          # all finite non-negative
    table = oracle.bf16_to_f64(table_bits)
    got = oracle.round_bf16(x)
    for xi, gi in zip(x, got):
        a = abs(xi)
        j = np.searchsorted(table, a)
        lo, hi = table[j - 1], table[j]
        if a - lo < hi - a:
            want = table_bits[j - 1]
        elif a - lo > hi - a:
            want = table_bits[j]
        else:
            want = table_bits[j - 1] if table_bits[j - 1] % 2 == 0 else table_bits[j]
        if xi < 0:
            want |= 0x8000
        assert gi == want


def test_e4m3_decode_matches_torch():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(oracle.e4m3_decode(codes), ref)
    assert oracle.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert oracle.e4m3_decode(np.array([0x01]))[0] == 2.0**-9


def test_e4m3_encode_matches_torch_and_brute_force():
    rng = np.random.default_rng(2)
    y = np.concatenate([rng.uniform(-448, 448, 20000), rng.standard_normal(20000),
                        rng.standard_normal(5000) * 2**-7]).astype(np.float32)
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_decode(finite)
    # midpoints between adjacent codes must go to the even code
    pos_codes = np.arange(0, 0x7E, dtype=np.uint8)
    pv = oracle.e4m3_decode(pos_codes)
    mids = ((pv[:-1] + pv[1:]) / 2).astype(np.float32)
    y = np.concatenate([y, mids, -mids])
    ours = oracle.e4m3_encode(y)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)
    # brute force: nearest finite value, ties to the even code
    for yi, ci in zip(y[:3000], ours[:3000]):
        d = np.abs(vals - float(yi))
        best = np.flatnonzero(d == d.min())
        cands = finite[best]
        if len(cands) > 1:
            cands = [c for c in cands if c % 2 == 0] or list(cands)
            if yi == 0:
                cands = [0x80 if np.signbit(yi) else 0x00]
        assert ci in list(cands), (yi, ci, cands)


def test_e4m3_encode_saturates():
    y = np.array([448.0, 449.0, 464.0, 500.0, 1e30, -600.0], dtype=np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(y), [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE])


def test_fp8_quantize_matches_torch_and_error_bound():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((500, 128)).astype(np.float32)
    x[7] = 0.0
    x[9, :5] = [1e-30, -2e-20, 0, 0, 3e-25]
    codes, scales = oracle.fp8_quantize(x)
    xt = torch.from_numpy(x)
    amax = xt.abs().amax(dim=1, keepdim=True)
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    np.testing.assert_array_equal(scales, s[:, 0].numpy())
    ref = (xt / s).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, ref)
    deq = oracle.fp8_dequantize(codes, scales)
    # error bound: half an e4m3 step, relative 2^-4 for normals, absolute 2^-10 * s below
    err = np.abs(deq - x.astype(np.float64))
    bound = np.maximum(np.abs(x) * 2.0**-4, 2.0**-10 * scales[:, None].astype(np.float64)) * (1 + 1e-6)
    assert (err <= bound).all()
    # the row maximum is represented exactly (448 * s ~= amax to fp32 rounding)
    rows = np.flatnonzero(np.abs(x).max(axis=1) > 0)
    top = np.abs(deq[rows]).max(axis=1)
    np.testing.assert_allclose(top, np.abs(x[rows]).max(axis=1), rtol=1e-6)
