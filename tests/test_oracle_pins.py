"""Pins of the CPU oracle to what the pages and the mathematics fix.

None of these tests compares the oracle with itself or with a retyped copy of
its formulas: every expected value is printed on a page (tests/golden, cited
there), follows from a closed form or an invariant of the definition, or comes
from an independent implementation (numpy / torch binary16 and bfloat16
conversion, exact rational arithmetic with ``fractions``).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# --------------------------------------------------------------------------
# binary16 / bfloat16 conversions, against numpy and torch
# --------------------------------------------------------------------------

def test_f16_to_f32_all_65536_patterns():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_bits_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_f16_dense_sample_and_every_tie():
    # a dense stride over all fp32 bit patterns
    bits = np.arange(0, 2**32, 251, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    ours = oracle.f32_to_f16_bits(x)
    with np.errstate(over="ignore", invalid="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    finite = np.isfinite(x)
    assert np.array_equal(ours[finite], ref[finite])
    assert np.all(np.isnan(ours[~finite & np.isnan(x)].view(np.float16)))
    # every exact midpoint between consecutive positive binary16 values, and
    # one fp32 ulp either side of it: this is where rounding mistakes show
    h = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.all(mid.astype(np.float64) == (lo + hi) / 2)  # exact in fp32
    for probe in (mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9))):
        for sgn in (1, -1):
            p = (probe * sgn).astype(np.float32)
            assert np.array_equal(oracle.f32_to_f16_bits(p), p.astype(np.float16).view(np.uint16))


def test_f16_overflow_boundary():
    # 65504 is the largest binary16; 65520 is the midpoint to 2^16 and rounds
    # (ties to even) to infinity
    assert oracle.lib().orc_f32_to_f16(65504.0) == 0x7BFF
    assert oracle.lib().orc_f32_to_f16(65519.99609375) == 0x7BFF
    assert oracle.lib().orc_f32_to_f16(65520.0) == 0x7C00
    assert oracle.lib().orc_f32_to_f16(2.0 ** -25) == 0x0000     # tie -> even (zero)
    assert oracle.lib().orc_f32_to_f16(3 * 2.0 ** -26) == 0x0001  # above the tie


def test_bf16_against_torch():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 20)
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([oracle.f32_to_bf16_bits(float(v)) for v in x.numpy()[:20000]], np.uint16)
    assert np.array_equal(ours, ref[:20000])
    back = np.array([oracle.bf16_bits_to_f32(int(b)) for b in ref[:5000]], np.float32)
    assert np.array_equal(back, x[:5000].to(torch.bfloat16).float().numpy())


# --------------------------------------------------------------------------
# sizes and layouts printed on the pages
# --------------------------------------------------------------------------

def test_block_sizes_and_bits_per_weight():
    rows = {r[0]: r[1:] for r in read_golden("formats.txt")}
    n, nbytes, bpw = int(rows["q4_0"][0]), int(rows["q4_0"][1]), float(rows["q4_0"][2])
    assert oracle.q4_0_bytes(n) == nbytes and nbytes * 8 / n == bpw
    assert oracle.q4_0_bytes(4096 * n) == 4096 * nbytes
    assert oracle.q4_0_bytes(n + 1) == 0 and oracle.q4_0_bytes(16) == 0
    n, nbytes, bpw = int(rows["ksb"][0]), int(rows["ksb"][1]), float(rows["ksb"][2])
    assert oracle.ksb_bytes(n) == nbytes and nbytes * 8 / n == bpw
    assert oracle.ksb_bytes(n + 32) == 0
    assert round(18 / (32 * 4), 2) == float(rows["fp32_fraction_q4_0"][0])


def _golden_values(rows, key):
    return np.array([float(v) for v in rows[key]], np.float32)


def test_q4_0_nibble_order_and_dequant_rule():
    rows = {r[0]: r[1:] for r in read_golden("q4_0_nibble_order.txt")}
    for tag in "AB":
        blk = np.array([int(b, 16) for b in rows["bytes_" + tag]], np.uint8)
        want = _golden_values(rows, "values_" + tag)
        assert blk.size == 18 and want.size == 32
        got = oracle.dequantize_q4_0(blk, 32)
        assert np.array_equal(got, want), (tag, got, want)


def test_ksb_layout_hand_built():
    rows = {r[0]: r[1:] for r in read_golden("ksb_layout.txt")}
    exc = [r[1:] for r in read_golden("ksb_layout.txt") if r[0] == "exception"]
    blk = np.zeros(138, np.uint8)
    s = int(rows["S_bits"][0], 16)
    blk[0], blk[1] = s & 0xFF, s >> 8
    blk[2:10] = [int(v) for v in rows["q"]]
    blk[10:] = 0x9A
    blk[10 + 16 * 3 + 0] = 0x07
    want = np.zeros(256, np.float32)
    for j in range(8):
        want[32 * j:32 * j + 16] = float(rows["lowval"][j])
        want[32 * j + 16:32 * j + 32] = float(rows["highval"][j])
    for idx, val in exc:
        want[int(idx)] = float(val)
    got = oracle.dequantize_ksb(blk, 256)
    assert np.array_equal(got, want)


# --------------------------------------------------------------------------
# the worked super-scale example of the K-quants post
# --------------------------------------------------------------------------

def test_ksb_worked_example_codes_and_reconstruction():
    rows = read_golden("ksb_worked_example.txt")
    table = [r for r in rows if r[0][0].isdigit()]
    meta = {r[0]: float(r[1]) for r in rows if not r[0][0].isdigit()}
    scales = np.array([float(r[0]) for r in table], np.float32)
    page_q = np.array([int(r[1]) for r in table])
    page_rec = np.array([float(r[2]) for r in table])
    d16 = oracle.f32_to_f16_bits(scales)                  # "FP16" block scales
    S16, q = oracle.ksb_scale_step(d16)
    S = float(oracle.f16_bits_to_f32([S16])[0])
    assert np.array_equal(q.astype(int), page_q)          # exactly the page's INT8
    assert abs(S - meta["super_scale"]) < 5e-6            # page prints 0.00142
    rec = q.astype(np.float64) * S
    # the page multiplies by its rounded 0.00142 and prints 4 decimals; ours
    # uses the FP16 S, so the two differ by at most q*|S - 0.00142| + 0.5e-4
    allowed = q * abs(S - meta["super_scale"]) + 0.5e-4 + 1e-9
    assert np.all(np.abs(rec - page_rec) <= allowed)
    err = np.abs(rec - oracle.f16_bits_to_f32(d16))
    assert err.max() <= meta["error_max"] + 1e-4
    # the largest sub-scale always lands on the top INT8 code
    assert q[np.argmax(scales)] == 127


def test_ksb_worked_example_through_full_quantizer():
    # build a super-block whose eight sub-block absmax values are 7x the page's
    # FP16 scales, so absmax/7 reproduces exactly those scales
    rows = read_golden("ksb_worked_example.txt")
    table = [r for r in rows if r[0][0].isdigit()]
    d = oracle.f16_bits_to_f32(oracle.f32_to_f16_bits(
        np.array([float(r[0]) for r in table], np.float32)))
    x = np.zeros(256, np.float32)
    for j in range(8):
        x[32 * j] = np.float32(7.0) * d[j]
        x[32 * j + 5] = -0.5 * d[j]
    q, flags = oracle.quantize_ksb(x)
    assert flags == 0
    assert np.array_equal(q[2:10].view(np.int8), np.array([int(r[1]) for r in table], np.int8))


# --------------------------------------------------------------------------
# Q4_0 quantizer: the rule fixed for this build and the page's reference rule
# --------------------------------------------------------------------------

def _u16(q, off):
    return int(q[off]) | (int(q[off + 1]) << 8)


def _outlier_block():
    # the demo input of the Q4_0 chapter, section 4.5
    return np.array([0.01 * (i - 15) / 15 for i in range(31)] + [10.0], np.float32)


def test_outlier_demo_page_reference_rule():
    # section 4.5: d = 10 / -8 = -1.25; the small values all collapse onto one
    # code; the outlier lands on the end of the code range (section 4.4: for a
    # positive max the extreme value maps to q = 0)
    q, flags = oracle.quantize_q4_0(_outlier_block(), rule=oracle.RULE_LLAMA)
    d = float(oracle.f16_bits_to_f32([_u16(q, 0)])[0])
    assert d == -1.25 and flags == 0
    codes = np.concatenate([q[2:] & 0xF, q[2:] >> 4])
    assert codes[31] == 0
    assert len(set(codes[:31].tolist())) == 1 and codes[0] == 8
    rec = oracle.dequantize_q4_0(q, 32)
    assert rec[31] == 10.0 and np.all(rec[:31] == 0.0)


@pytest.mark.parametrize("first_sign", [1.0, -1.0])
def test_reference_rule_hand_worked_block(first_sign):
    # a block worked by hand under section 4.4's printed rule, with values
    # whose products with 1/d are exact in fp32: the max magnitude 4 occurs
    # twice with opposite signs and the first one sets d = max / -8;
    # codes are min(15, trunc(x / d + 8.5)) -- truncation, not rounding
    s = first_sign
    x = np.zeros(32, np.float32)
    x[5], x[9] = 4.0 * s, -4.0 * s        # tie in magnitude: position 5 wins
    x[1], x[2], x[3], x[4] = 1.0 * s, -1.0 * s, 0.75 * s, 0.5 * s
    x[6], x[7] = 0.25 * s, -0.25 * s
    q, flags = oracle.quantize_q4_0(x, rule=oracle.RULE_LLAMA)
    assert flags == 0
    d = float(oracle.f16_bits_to_f32([_u16(q, 0)])[0])
    assert d == -0.5 * s                  # 4s / -8
    codes = np.concatenate([q[2:] & 0xF, q[2:] >> 4])
    # x / d = -2x/s: 4s -> -8 + 8.5 = 0.5 -> 0; -4s -> 16.5 -> min(15, 16) = 15;
    # s -> 6.5 -> 6; -s -> 10.5 -> 10; 0.75s -> 7.0 -> 7; 0.5s -> 7.5 -> 7;
    # 0.25s -> 8.0 -> 8; -0.25s -> 9.0 -> 9; 0 -> 8.5 -> 8
    want = {5: 0, 9: 15, 1: 6, 2: 10, 3: 7, 4: 7, 6: 8, 7: 9}
    for i in range(32):
        assert codes[i] == want.get(i, 8), (i, codes[i])


def test_reference_rule_zero_and_truncation_edges():
    # a zero block: d = 0 / -8 = -0, the inverse scale is taken as 0, every
    # code is trunc(8.5) = 8 and the stored scale is FP16 -0
    q, _ = oracle.quantize_q4_0(np.zeros(32, np.float32), rule=oracle.RULE_LLAMA)
    assert _u16(q, 0) == 0x8000 and np.all(q[2:] == 0x88)
    # max 8 -> d = -1, id = -1: x = 0.4 gives 8.1 -> 8, x = -0.6 gives 9.1 -> 9
    # (round-to-nearest would give 8 and 9 as well; x = -0.4 gives 8.9 -> 8,
    # where rounding would give 9)
    x = np.zeros(32, np.float32)
    x[0], x[1], x[2], x[3] = 8.0, 0.4, -0.6, -0.4
    q, _ = oracle.quantize_q4_0(x, rule=oracle.RULE_LLAMA)
    codes = np.concatenate([q[2:] & 0xF, q[2:] >> 4])
    assert _u16(q, 0) == 0xBC00           # FP16 -1.0
    assert codes[0] == 0 and codes[1] == 8 and codes[2] == 9 and codes[3] == 8


def test_outlier_demo_build_rule():
    # the build's rule d = FP16(absmax/7): the outlier still takes the top code
    # and every small value collapses to zero (the failure mode the page shows)
    q, flags = oracle.quantize_q4_0(_outlier_block())
    codes = np.concatenate([q[2:] & 0xF, q[2:] >> 4])
    assert flags == 0
    assert codes[31] == 15 and np.all(codes[:31] == 8)
    rec = oracle.dequantize_q4_0(q, 32)
    assert abs(rec[31] - 10.0) < 10.0 / 7 / 2


def test_rint_ties_go_to_even():
    # absmax 1.75 gives d = 0.25 exactly; x = (k + 0.5) * 0.25 makes x/d an
    # exact tie, and round-half-to-even picks the even neighbour
    k = np.arange(-7, 7)
    x = np.zeros(32, np.float32)
    x[:14] = (k + 0.5) * 0.25
    x[14] = 1.75
    q, _ = oracle.quantize_q4_0(x)
    assert _u16(q, 0) == 0x3400                 # 0.25 in binary16
    codes = np.concatenate([q[2:] & 0xF, q[2:] >> 4])
    want = [int(np.round(v + 0.5)) + 8 for v in k]      # numpy rounds half to even
    assert codes[:14].tolist() == want == [2, 2, 4, 4, 6, 6, 8, 8, 10, 10, 12, 12, 14, 14]
    assert codes[14] == 15


def test_absmax_maps_to_top_code_and_sign():
    rng = np.random.default_rng(3)
    for _ in range(200):
        x = rng.standard_normal(32).astype(np.float32) * rng.uniform(1e-3, 1e3)
        i = int(np.argmax(np.abs(x)))
        q, _ = oracle.quantize_q4_0(x)
        codes = np.concatenate([q[2:] & 0xF, q[2:] >> 4])
        assert codes[i] == (15 if x[i] > 0 else 1)


def test_round_trip_bound_q4_0():
    w = synth.gaussian_weights(64, 1024, seed=11).numpy().ravel()
    q, flags = oracle.quantize_q4_0(w)
    assert flags == 0
    rec = oracle.dequantize_q4_0(q, w.size)
    d = oracle.f16_bits_to_f32(q.reshape(-1, 18)[:, :2].copy().view(np.uint16).ravel())
    d = np.repeat(d, 32).astype(np.float64)
    t = np.where(d > 0, w / np.where(d > 0, d, 1), 0)
    unclipped = np.abs(np.rint(t)) <= 7
    err = np.abs(w.astype(np.float64) - rec)
    assert np.all(err[unclipped] <= d[unclipped] * (0.5 + 2.0 ** -20))
    # the outlier mask makes clipping possible only through FP16 rounding of d
    assert unclipped.mean() > 0.999


def test_zero_tiny_and_range_blocks():
    q, f = oracle.quantize_q4_0(np.zeros(32, np.float32))
    assert f == 0 and q[0] == 0 and q[1] == 0 and np.all(q[2:] == 0x88)
    # a subnormal FP16 scale: absmax 7 * 2^-20 -> d = 2^-20 (0x0010)
    x = np.zeros(32, np.float32)
    x[3] = 7 * 2.0 ** -20
    x[20] = -3 * 2.0 ** -20
    q, f = oracle.quantize_q4_0(x)
    assert f == 0 and _u16(q, 0) == 0x0010
    rec = oracle.dequantize_q4_0(q, 32)
    assert rec[3] == x[3] and rec[20] == x[20]
    # absmax/7 at or above 65520 overflows the FP16 scale
    x = np.zeros(32, np.float32)
    x[0] = 7 * 65520.0
    _, f = oracle.quantize_q4_0(x)
    assert f & oracle.RANGE
    x[0] = np.nan
    _, f = oracle.quantize_q4_0(x)
    assert f & oracle.NONFINITE


# --------------------------------------------------------------------------
# ksb quantizer
# --------------------------------------------------------------------------

def test_round_trip_bound_ksb():
    w = synth.logstd_weights(32, 2048, seed=2).numpy().ravel()
    q, flags = oracle.quantize_ksb(w)
    assert flags == 0
    rec = oracle.dequantize_ksb(q, w.size).astype(np.float64)
    blk = q.reshape(-1, 138)
    S = oracle.f16_bits_to_f32(blk[:, :2].copy().view(np.uint16).ravel()).astype(np.float64)
    st = S[:, None] * blk[:, 2:10].view(np.int8).astype(np.float64)   # [nsb, 8]
    st = np.repeat(st.ravel(), 32)
    t = np.where(st > 0, w / np.where(st > 0, st, 1), 0)
    unclipped = np.abs(np.rint(t)) <= 7
    err = np.abs(w - rec)
    assert np.all(err[unclipped] <= st[unclipped] * (0.5 + 2.0 ** -20))
    # the largest sub-block scale of every super-block takes INT8 code 127
    assert np.all(blk[:, 2:10].view(np.int8).max(axis=1) == 127)


def test_ksb_zero_superblock():
    q, f = oracle.quantize_ksb(np.zeros(256, np.float32))
    assert f == 0 and np.all(q[:10] == 0) and np.all(q[10:] == 0x88)
    assert np.all(oracle.dequantize_ksb(q, 256) == 0)


# --------------------------------------------------------------------------
# products: exact rational brute force and closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("fmt,M,K", [(oracle.FMT_Q4_0, 5, 96), (oracle.FMT_KSB, 3, 512)])
def test_gemm_against_exact_rationals(fmt, M, K):
    W = synth.gaussian_weights(M, K, seed=7, frac=0.05).numpy()
    q, _ = oracle.quantize(fmt, W.ravel())
    X = synth.activations(3, K, seed=8, dtype=torch.float16).numpy()
    Y, bound = oracle.gemm(fmt, q, M, K, X)
    What = oracle.dequantize(fmt, q, M * K).reshape(M, K)
    for b in range(3):
        for m in range(M):
            exact = sum(Fraction(float(What[m, k])) * Fraction(float(X[b, k])) for k in range(K))
            absum = sum(abs(Fraction(float(What[m, k])) * Fraction(float(X[b, k]))) for k in range(K))
            assert abs(Fraction(Y[b, m]) - exact) <= Fraction(2.0 ** -50) * absum
            assert abs(Fraction(bound[b, m]) - absum) <= Fraction(2.0 ** -50) * absum


def test_gemm_closed_form_constant_codes():
    # every block: d = 0.5, every code 11 -> every weight 1.5; y = 1.5 * sum(x)
    M, K = 4, 64
    blk = np.array([0x00, 0x38] + [0xBB] * 16, np.uint8)
    W = np.tile(blk, M * K // 32)
    X = synth.activations(2, K, seed=1, dtype=torch.float32).numpy()
    Y, _ = oracle.gemm(oracle.FMT_Q4_0, W, M, K, X)
    want = 1.5 * X.astype(np.float64).sum(axis=1)
    assert np.allclose(Y, want[:, None], rtol=1e-14, atol=0)


def test_gemm_identity_columns_give_dequantized_columns():
    M, K = 6, 256
    W = synth.logstd_weights(M, K, seed=4).numpy()
    q, _ = oracle.quantize_ksb(W.ravel())
    X = np.zeros((5, K), np.float32)
    cols = [0, 17, 100, 200, 255]
    for b, c in enumerate(cols):
        X[b, c] = 1.0
    Y, _ = oracle.gemm(oracle.FMT_KSB, q, M, K, X)
    What = oracle.dequantize_ksb(q, M * K).reshape(M, K)
    for b, c in enumerate(cols):
        assert np.array_equal(Y[b], What[:, c].astype(np.float64))


def test_gemm_rows_matches_full_product_and_bf16_input():
    M, K = 40, 512
    W = synth.gaussian_weights(M, K, seed=9).numpy()
    q, _ = oracle.quantize_q4_0(W.ravel())
    Xb = synth.activations(2, K, seed=3, dtype=torch.bfloat16)
    Xbits = Xb.view(torch.int16).numpy().view(np.uint16)
    Y, bound = oracle.gemm(oracle.FMT_Q4_0, q, M, K, Xbits, xt=oracle.BF16)
    Yf, _ = oracle.gemm(oracle.FMT_Q4_0, q, M, K, Xb.float().numpy())
    assert np.array_equal(Y, Yf)                       # bf16 widening is exact
    rows = np.array([39, 0, 17])
    Yr, br = oracle.gemm_rows(oracle.FMT_Q4_0, q, M, K, Xbits, rows, xt=oracle.BF16)
    assert np.array_equal(Yr, Y[:, rows]) and np.array_equal(br, bound[:, rows])


# ------------------------------------------------------------- tiled storage
def test_tiled_layout_hand_worked_positions():
    # each listed byte of the tiled storage holds the canonical byte worked out
    # by hand from the layout definition (tests/golden/tiled_layout.txt)
    rows = read_golden("tiled_layout.txt")
    assert len(rows) == 24
    for fmt, M, K, toff, coff in ((int(r[0]), int(r[1]), int(r[2]), int(r[3]), int(r[4]))
                                  for r in rows):
        rb = oracle.q4_0_bytes(K) if fmt == oracle.FMT_Q4_0 else oracle.ksb_bytes(K)
        W = (np.arange(M * rb) * 7919 % 256).astype(np.uint8)
        # make the probed canonical byte unique in the matrix
        W[W == 255] = 254
        W[coff] = 255
        T = oracle.repack(fmt, W, M, K)
        assert T[toff] == 255 and np.count_nonzero(T == 255) == 1, (fmt, M, K, toff, coff)


@pytest.mark.parametrize("fmt,M,K", [(oracle.FMT_Q4_0, 16, 64), (oracle.FMT_Q4_0, 48, 4160),
                                     (oracle.FMT_KSB, 32, 2304), (oracle.FMT_KSB, 16, 11008)])
def test_tiled_is_a_byte_permutation(fmt, M, K):
    # M a multiple of 16: same size, and the inverse restores every byte; with
    # distinct 16-bit markers split over byte pairs, every tiled position is
    # filled from exactly one canonical position
    rb = oracle.q4_0_bytes(K) if fmt == oracle.FMT_Q4_0 else oracle.ksb_bytes(K)
    assert oracle.tiled_bytes(fmt, M, K) == M * rb
    rng = np.random.default_rng(M + K)
    W = rng.integers(0, 256, M * rb, dtype=np.uint8)
    T = oracle.repack(fmt, W, M, K)
    assert np.array_equal(oracle.unrepack(fmt, T, M, K), W)
    assert np.array_equal(np.sort(T), np.sort(W))


@pytest.mark.parametrize("fmt,M,K", [(oracle.FMT_Q4_0, 17, 128), (oracle.FMT_KSB, 33, 512)])
def test_tiled_ragged_rows_are_zero(fmt, M, K):
    # rows past M in the last group of 16 are stored as zeros
    rb = oracle.q4_0_bytes(K) if fmt == oracle.FMT_Q4_0 else oracle.ksb_bytes(K)
    W = np.full(M * rb, 0xA5, dtype=np.uint8)
    T = oracle.repack(fmt, W, M, K)
    assert T.size == (M + 15) // 16 * 16 * rb
    assert np.count_nonzero(T == 0xA5) == M * rb
    assert np.count_nonzero(T == 0) == T.size - M * rb
    assert np.array_equal(oracle.unrepack(fmt, T, M, K), W)


def test_tiled_rejects_partial_units():
    assert oracle.tiled_bytes(oracle.FMT_Q4_0, 16, 96) == -1
    assert oracle.tiled_bytes(oracle.FMT_KSB, 16, 128) == -1


def test_tiled_dequantizes_to_the_same_weights():
    # a tiled matrix, turned back into rows, decodes to the canonical weights
    M, K = 32, 2304
    for fmt in (oracle.FMT_Q4_0, oracle.FMT_KSB):
        w = synth.gaussian_weights(M, K, seed=5).numpy().ravel()
        q, _ = oracle.quantize(fmt, w)
        back = oracle.unrepack(fmt, oracle.repack(fmt, q, M, K), M, K)
        assert np.array_equal(oracle.dequantize(fmt, back, M * K).view(np.uint32),
                              oracle.dequantize(fmt, q, M * K).view(np.uint32))


def test_thread_count_does_not_change_results():
    # the timing runs change the oracle's thread count; every output is one
    # thread's loop, so quantized bytes and products are the same bytes
    w = synth.logstd_weights(96, 2048, seed=21).numpy().ravel()
    x = synth.activations(3, 2048, seed=22, dtype=torch.float16).numpy()
    res, n0 = [], oracle.num_threads()
    for th in (1, 3, n0):
        oracle.set_threads(th)
        q4, _ = oracle.quantize(oracle.FMT_Q4_0, w)
        qk, _ = oracle.quantize(oracle.FMT_KSB, w)
        y, b = oracle.gemm(oracle.FMT_KSB, qk, 96, 2048, x)
        res.append((q4.tobytes(), qk.tobytes(), y.tobytes(), b.tobytes()))
    oracle.set_threads(n0)
    assert res[0] == res[1] == res[2]
