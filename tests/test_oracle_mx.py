"""Pins of the oracle's MX (block-scaled) formats and MX expert FFN.

The pages name MXFP8 / MXFP4 ([MegaFlux] §2.1 'Persistent MoE execution',
§4.1 'Setup'; [MoonEP] "A bandwidth-only model": one scale per 32 elements)
without defining them; the oracle reads them as the OCP Microscaling
formats. These tests pin the oracle's encoder against the format's own
facts and against brute force over the code table, and pin the MX FFN
against the plain bf16 oracle on inputs that the quantization leaves
unchanged."""
import numpy as np
import pytest

from oracle import oracle as O



def _table():
    """Every non-negative finite E4M3 code with its value."""
    codes = np.arange(0, 0x7F)
    return codes, np.array([O.e4m3_value(int(c)) for c in codes])


def test_e4m3_landmarks():
    # the format's own facts: bias 7, 3 mantissa bits, subnormals, one NaN pattern per sign
    assert O.e4m3_value(0x7E) == 448.0            # largest finite
    assert O.e4m3_value(0x08) == 2.0 ** -6        # smallest normal
    assert O.e4m3_value(0x01) == 2.0 ** -9        # smallest subnormal
    assert O.e4m3_value(0x07) == 7 * 2.0 ** -9    # largest subnormal
    assert O.e4m3_value(0x38) == 1.0
    assert O.e4m3_value(0x39) == 1.125
    assert O.e4m3_value(0xB8) == -1.0
    assert np.isnan(O.e4m3_value(0x7F)) and np.isnan(O.e4m3_value(0xFF))
    codes, vals = _table()
    assert np.all(np.diff(vals) > 0)              # strictly increasing with the code
    # eight equally spaced values in every binade from 2^-6 up
    for e in range(-6, 9):
        b = vals[(vals >= 2.0 ** e) & (vals < 2.0 ** (e + 1))]
        assert len(b) == (7 if e == 8 else 8)     # 2^8 binade ends at 448 (480 is the NaN pattern)
        assert np.allclose(np.diff(b), 2.0 ** (e - 3))


def _nearest_by_search(v, codes, vals):
    a = abs(v)
    if a >= 448.0:
        c = 0x7E
    else:
        dist = np.abs(vals - a)
        best = np.flatnonzero(dist == dist.min())
        c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])   # ties: even code
    return c | (0x80 if np.signbit(v) else 0)


def test_e4m3_encode_is_nearest_ties_to_even():
    codes, vals = _table()
    rng = np.random.default_rng(7)
    mags = np.concatenate([2.0 ** rng.uniform(-12, 9.5, 4000), (vals[:-1] + vals[1:]) / 2, vals,
                           [448.0, 449.0, 463.9, 464.0, 1e6, 0.0]])
    for m in mags:
        for v in (m, -m):
            assert O.e4m3_encode(v) == _nearest_by_search(v, codes, vals), v


def test_scale_code_maps_the_block_maximum_into_256_512():
    rng = np.random.default_rng(3)
    for amax in 2.0 ** rng.uniform(-100, 100, 3000):
        s = O.mx_scale_code(amax)
        X = 2.0 ** (s - 127)
        assert 256.0 <= amax / X < 512.0
    assert O.mx_scale_code(0.0) == 0
    assert O.mx_scale_code(2.0 ** -140) == 0      # clamped at the smallest scale
    assert O.mx_scale_code(1.0) == 127 - 8
    assert O.mx_scale_code(448.0) == 127


def _bf16(a):
    return np.array([O.double_to_bf16(float(v)) for v in a.ravel()], np.uint16).reshape(a.shape)


def test_quantize_error_bound_and_requantize():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((16, 256)) * (2.0 ** rng.integers(-20, 20, (16, 1)))
    xb = _bf16(x)
    xv = O.bf16_bits_to_f64(xb)
    q, s = O.mx_quantize(xb, O.BF16)
    dq = O.mx_dequantize(q, s)
    for r in range(16):
        for b in range(256 // 32):
            blk = xv[r, 32 * b:32 * b + 32]
            X = 2.0 ** (int(s[r, b]) - 127)
            assert 256.0 <= np.abs(blk).max() / X < 512.0
            for i in range(32):
                v, w = blk[i] / X, dq[r, 32 * b + i] / X
                if abs(v) > 448.0:
                    assert w == np.sign(v) * 448.0
                else:
                    # half a step of the binade of |v| (steps of 2^-9 below 2^-6)
                    step = 2.0 ** (max(np.floor(np.log2(abs(v))), -6) - 3) if v != 0 else 2.0 ** -9
                    assert abs(w - v) <= step / 2
    # values already on the grid quantize to themselves
    q2, s2 = O.mx_quantize(dq.astype(np.float32), O.FP32)
    assert np.array_equal(q2, q) and np.array_equal(s2, s)


def _grid_matrix(rng, rows, K):
    """[rows, K] values that MXFP8 represents exactly: E4M3 grid values whose
    32-blocks each hold one element in [256, 448], times a power of two per block."""
    codes, vals = _table()
    v = rng.choice(np.concatenate([vals, -vals]), size=(rows, K))
    v = v.reshape(rows, K // 32, 32)
    top = rng.choice(vals[(vals >= 256) & (vals <= 448)], size=(rows, K // 32))
    v[:, :, 0] = top * rng.choice([-1.0, 1.0], size=(rows, K // 32))
    v = v * 2.0 ** rng.integers(-12, -6, size=(rows, K // 32, 1))
    return v.reshape(rows, K).astype(np.float32)


def test_grid_inputs_quantize_to_themselves():
    rng = np.random.default_rng(5)
    a = _grid_matrix(rng, 8, 128)
    q, s = O.mx_quantize(a, O.FP32)
    assert np.array_equal(O.mx_dequantize(q, s), a.astype(np.float64))


def test_mx_ffn_matches_the_bf16_oracle_on_exact_inputs():
    """On inputs MXFP8 represents exactly, the MX FFN's h equals the plain
    oracle's h (bf16-rounded) bit for bit, and y stays within the error that
    quantizing h to MXFP8 can add."""
    rng = np.random.default_rng(1)
    E, d, F, T = 3, 64, 96, 5
    x = _grid_matrix(rng, T, d)
    w_gu = _grid_matrix(rng, E * 2 * F, d).reshape(E, 2 * F, d)
    w_dn = _grid_matrix(rng, E * d, F).reshape(E, d, F)
    xq, xs = O.mx_quantize(x, O.FP32)
    w1q, w1s, w2q, w2s = O.mx_weights(w_gu, w_dn, O.FP32)
    tokens = np.repeat(np.arange(T), E)
    experts = np.tile(np.arange(E), T)
    h, hq, hs, y = O.mx_entry_ffn(tokens, experts, xq, xs, w1q, w1s, w2q, w2s, F)
    h_ref, y_ref = O.entry_ffn(tokens, experts, x, w_gu, w_dn, O.FP32, O.ROUND_BF16)
    assert np.array_equal(h, h_ref)
    hdq = O.mx_dequantize(hq, hs)
    assert np.array_equal(O.mx_dequantize(*O.mx_quantize(h.astype(np.float32), O.FP32)), hdq)
    # y: the effect of h's quantization, bounded by |h - hdq| . |W2|, plus bf16 rounding
    for n in range(len(tokens)):
        W2 = w_dn[experts[n]].astype(np.float64)
        bound = np.abs(W2) @ np.abs(h[n] - hdq[n]) + np.abs(y_ref[n]) * 2.0 ** -8 + np.abs(y[n]) * 2.0 ** -8
        assert np.all(np.abs(y[n] - y_ref[n]) <= bound + 1e-30)
        # the bound is not vacuous: h really was requantized for some entries
    assert np.any(h != hdq)


def test_mx_token_out_is_the_weighted_sum_of_its_entries():
    rng = np.random.default_rng(2)
    E, d, F, T, K = 4, 64, 64, 6, 2
    x = _bf16(rng.standard_normal((T, d)))
    w_gu = _bf16(rng.standard_normal((E, 2 * F, d)) * 0.1)
    w_dn = _bf16(rng.standard_normal((E, d, F)) * 0.1)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    w = rng.random((T, K)).astype(np.float32)
    xq, xs = O.mx_quantize(x, O.BF16)
    w1q, w1s, w2q, w2s = O.mx_weights(w_gu, w_dn, O.BF16)
    out = O.mx_token_out(np.arange(T), xq, xs, idx, w, w1q, w1s, w2q, w2s, F)
    _, _, _, y = O.mx_entry_ffn(np.repeat(np.arange(T), K), idx.ravel(), xq, xs, w1q, w1s, w2q, w2s, F)
    ref = (w.astype(np.float64)[:, :, None] * y.reshape(T, K, d)).sum(1)
    assert np.array_equal(out, O.bf16_bits_to_f64(_bf16(ref)))


def test_mx_fc1_and_fc2_rows_compose_to_the_entry_ffn():
    rng = np.random.default_rng(4)
    E, d, F, T = 3, 64, 64, 4
    x = _bf16(rng.standard_normal((T, d)))
    w_gu = _bf16(rng.standard_normal((E, 2 * F, d)) * 0.2)
    w_dn = _bf16(rng.standard_normal((E, d, F)) * 0.2)
    xq, xs = O.mx_quantize(x, O.BF16)
    w1q, w1s, w2q, w2s = O.mx_weights(w_gu, w_dn, O.BF16)
    tokens = np.repeat(np.arange(T), E)
    experts = np.tile(np.arange(E), T)
    h, hq, hs, y = O.mx_entry_ffn(tokens, experts, xq, xs, w1q, w1s, w2q, w2s, F)
    h1, hq1, hs1 = O.mx_fc1_rows(tokens, experts, xq, xs, w1q, w1s, F)
    assert np.array_equal(h1, h) and np.array_equal(hq1, hq) and np.array_equal(hs1, hs)
    assert np.array_equal(O.mx_fc2_rows(experts, hq, hs, w2q, w2s, d), y)


# ---------------------------------------------------------------- MXFP4 (E2M1) weights

def test_e2m1_table():
    # the format's own facts: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit, subnormal 0.5
    assert [O.e2m1_value(c) for c in range(8)] == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert [O.e2m1_value(c) for c in range(8, 16)] == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_e2m1_encode_ties_and_saturation():
    # midpoints go to the even code (mantissa bit 0)
    for v, c in ((0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6), (6.0, 7), (7.0, 7),
                 (100.0, 7), (0.2, 0), (0.3, 1), (-1.3, 8 | 3), (-0.1, 8)):
        assert O.e2m1_encode(v) == c, v
    rng = np.random.default_rng(9)
    vals = np.array([O.e2m1_value(c) for c in range(8)])
    for v in rng.uniform(-7, 7, 2000):
        c = O.e2m1_encode(v)
        d = np.abs(vals - abs(v))
        assert abs(O.e2m1_value(c & 7) - abs(v)) == d.min() or abs(v) > 6
        assert (c >= 8) == (v < 0)


def test_mxfp4_scale_and_error_bound():
    rng = np.random.default_rng(12)
    for amax in 2.0 ** rng.uniform(-60, 60, 2000):
        X = 2.0 ** (O.mx_scale_code_fmt(amax, O.MX_E2M1) - 127)
        assert 4.0 <= amax / X < 8.0          # the block maximum lands in E2M1's top binade (or saturates)
    x = rng.standard_normal((8, 128)).astype(np.float32)
    q, s = O.mx_quantize_fmt(x, O.FP32, O.MX_E2M1)
    assert q.max() < 16
    dq = O.mx_dequantize_fmt(q, s, O.MX_E2M1)
    X = np.repeat(2.0 ** (s.astype(np.int64) - 127), 32, axis=1)
    v = x.astype(np.float64) / X
    err = np.abs(dq / X - v)
    # half a step of the value's binade (steps 0.5 below 2, 1 in [2, 4), 2 in [4, 6]); saturation above 6
    step = np.where(np.abs(v) < 2, 0.5, np.where(np.abs(v) < 4, 1.0, 2.0))
    assert np.all((err <= step / 2 + 1e-12) | (np.abs(v) > 6))


def test_mx_ffn_with_mxfp4_weights_on_exact_inputs():
    """MXFP4 weights that E2M1 represents exactly: the MX FFN's h equals the plain oracle's h."""
    rng = np.random.default_rng(6)
    E, d, F, T = 2, 64, 64, 3
    vals = np.array([O.e2m1_value(c) for c in range(16)])

    def grid(rows, K):
        v = rng.choice(vals, size=(rows, K // 32, 32))
        v[:, :, 0] = rng.choice([4.0, 6.0, -4.0, -6.0], size=(rows, K // 32))
        return (v * 2.0 ** rng.integers(-9, -5, size=(rows, K // 32, 1))).reshape(rows, K).astype(np.float32)

    x = _grid_matrix(rng, T, d)
    w_gu = grid(E * 2 * F, d).reshape(E, 2 * F, d)
    w_dn = grid(E * d, F).reshape(E, d, F)
    xq, xs = O.mx_quantize(x, O.FP32)
    w1q, w1s, w2q, w2s = O.mx_weights(w_gu, w_dn, O.FP32, O.MX_E2M1)
    assert np.array_equal(O.mx_dequantize_fmt(w1q, w1s, O.MX_E2M1), w_gu.reshape(E * 2 * F, d).astype(np.float64))
    tokens = np.repeat(np.arange(T), E)
    experts = np.tile(np.arange(E), T)
    h, hq, hs, y = O.mx_entry_ffn(tokens, experts, xq, xs, w1q, w1s, w2q, w2s, F, O.MX_E2M1)
    h_ref, _ = O.entry_ffn(tokens, experts, x, w_gu, w_dn, O.FP32, O.ROUND_BF16)
    assert np.array_equal(h, h_ref)
    y2 = O.mx_fc2_rows(experts, hq, hs, w2q, w2s, d, O.MX_E2M1)
    assert np.array_equal(y2, y)


def test_e4m3_encode_matches_torch_float8_e4m3fn():
    """The oracle's encoder against a library conversion (PyTorch's
    float8_e4m3fn, round to nearest even) on values within the finite range,
    including every midpoint between neighbouring codes and subnormals."""
    import torch
    codes, vals = _table()
    rng = np.random.default_rng(21)
    mags = np.concatenate([2.0 ** rng.uniform(-12, np.log2(448.0), 6000), (vals[:-1] + vals[1:]) / 2, vals])
    v = np.concatenate([mags, -mags]).astype(np.float32)   # fp32-representable inputs for both sides
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.e4m3_encode(float(t)) for t in v], np.uint8)
    assert np.array_equal(got, ref)
