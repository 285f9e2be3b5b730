"""GPU quantize / dequantize against the oracle, byte for byte and bit for bit."""
import numpy as np
import pytest
import torch

import bit_gemv_q4_b200 as gq
import oracle
import synth
from gpu_helpers import KSB, Q40

pytestmark = pytest.mark.gpu


def gpu_quantize(fmt, w: torch.Tensor):
    x = w.reshape(-1).float().contiguous().cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    f = gq.gq_quantize_q4_0 if fmt == Q40 else gq.gq_quantize_ksb
    q = f(x, dev_status=st)
    torch.cuda.synchronize()
    return q.cpu().numpy(), int(st.item())


def gpu_dequantize(fmt, q: np.ndarray, n: int):
    f = gq.gq_dequantize_q4_0 if fmt == Q40 else gq.gq_dequantize_ksb
    out = f(torch.from_numpy(q).cuda(), n)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def assert_bytes_equal(got, want, blk):
    if not np.array_equal(got, want):
        diff = np.nonzero(got != want)[0]
        b = diff[0] // blk
        raise AssertionError(f"{diff.size} bytes differ; first in block {b}: gpu "
                             f"{got[b * blk:(b + 1) * blk].tolist()} oracle "
                             f"{want[b * blk:(b + 1) * blk].tolist()}")


CASES = [
    # (format, rows, cols, generator) -- the five workloads' shapes plus ragged tails
    (Q40, 256, 1024, "gauss"),     # tiny workload (seed 0)
    (Q40, 1, 32, "gauss"),         # one block
    (Q40, 67, 32, "gauss"),        # 67 blocks: ragged CTA tile
    (Q40, 4096, 4096, "gauss"),    # decode shape
    (Q40, 11008, 4096, "logstd"),
    (KSB, 256, 1024, "gauss"),
    (KSB, 1, 256, "gauss"),
    (KSB, 9, 256, "logstd"),       # ragged CTA tile
    (KSB, 11008, 4096, "logstd"),  # MLP shape
    (KSB, 4096, 11008, "gauss"),
]


@pytest.mark.parametrize("fmt,M,K,gen", CASES)
def test_quantize_bit_exact(fmt, M, K, gen):
    seed = 0 if (M, K) == (256, 1024) else M + K
    w = (synth.gaussian_weights if gen == "gauss" else synth.logstd_weights)(M, K, seed=seed)
    got, st = gpu_quantize(fmt, w)
    want, flags = oracle.quantize(fmt, w.numpy().ravel())
    assert st == 0 and flags == 0
    assert_bytes_equal(got, want, 18 if fmt == Q40 else 138)


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_dequantize_bit_exact(fmt):
    # oracle-made blocks, plus arbitrary byte patterns with finite scales
    w = synth.logstd_weights(333, 512, seed=5)
    q, _ = oracle.quantize(fmt, w.numpy().ravel())
    n = w.numel()
    assert np.array_equal(gpu_dequantize(fmt, q, n).view(np.uint32),
                          oracle.dequantize(fmt, q, n).view(np.uint32))
    rng = np.random.default_rng(1)
    blk = 18 if fmt == Q40 else 138
    nb = 4099 if fmt == Q40 else 515
    r = rng.integers(0, 256, size=nb * blk, dtype=np.uint8).reshape(nb, blk)
    r[:, 1] &= 0x7B  # keep the FP16 scale finite
    q = r.ravel().copy()
    n = nb * (32 if fmt == Q40 else 256)
    assert np.array_equal(gpu_dequantize(fmt, q, n).view(np.uint32),
                          oracle.dequantize(fmt, q, n).view(np.uint32))


def _edge_blocks():
    rows = []
    rows.append(np.zeros(32))                                   # all zero
    x = np.zeros(32); x[3] = 7 * 2.0 ** -20; x[20] = -3 * 2.0 ** -20
    rows.append(x)                                              # subnormal FP16 scale
    x = np.zeros(32); x[:14] = (np.arange(-7, 7) + 0.5) * 0.25; x[14] = 1.75
    rows.append(x)                                              # exact ties
    rows.append(np.array([0.01 * (i - 15) / 15 for i in range(31)] + [10.0]))  # outlier demo
    x = np.zeros(32); x[5] = -1e-30
    rows.append(x)                                              # scale underflows to 0
    x = np.linspace(-3e4, 3e4, 32)
    rows.append(x)                                              # large but in range
    x = np.full(32, -0.0)
    rows.append(x)
    return np.concatenate(rows).astype(np.float32)


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_quantize_edge_blocks(fmt):
    x = _edge_blocks()
    if fmt == KSB:
        x = np.concatenate([x, np.zeros(256 - x.size % 256, np.float32)])
    got, st = gpu_quantize(fmt, torch.from_numpy(x))
    want, flags = oracle.quantize(fmt, x)
    assert st == flags == 0
    assert_bytes_equal(got, want, 18 if fmt == Q40 else 138)


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_quantize_status_flags(fmt):
    n = 32 * 64 if fmt == Q40 else 256 * 8
    x = np.zeros(n, np.float32)
    x[40] = 7 * 70000.0      # absmax/7 overflows FP16 -> range
    _, st = gpu_quantize(fmt, torch.from_numpy(x))
    _, flags = oracle.quantize(fmt, x)
    assert st == flags == gq.GQ_DEV_RANGE
    x[40] = 1.0
    for bad in (np.nan, np.inf, -np.inf):
        x[300] = bad
        _, st = gpu_quantize(fmt, torch.from_numpy(x))
        assert st & gq.GQ_DEV_NONFINITE
        assert gq.gq_status_from_dev(st) == 5
    # a block of NaNs only, and a non-finite value as the last of a tile
    x[:] = 0.0
    x[-32:] = np.nan
    _, st = gpu_quantize(fmt, torch.from_numpy(x))
    assert st & gq.GQ_DEV_NONFINITE
    x[:] = 0.0
    x[-1] = -np.inf
    _, st = gpu_quantize(fmt, torch.from_numpy(x))
    assert st & gq.GQ_DEV_NONFINITE


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_quantize_1e9_sampled(fmt):
    """Quantize of 1e9 fp32 weights N(0, 0.02^2) generated on the device (the
    throughput workload); a random sample of blocks is checked byte for byte
    against the oracle on the same input values."""
    n = 1_000_000_000
    rows = n // 8000
    w = synth.gaussian_weights(rows, 8000, seed=4, frac=0.0, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    f = gq.gq_quantize_q4_0 if fmt == Q40 else gq.gq_quantize_ksb
    q = f(w.view(-1), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    blk_w, blk_b = (32, 18) if fmt == Q40 else (256, 138)
    nblk = n // blk_w
    rng = np.random.default_rng(9)
    pick = np.unique(np.concatenate([rng.integers(0, nblk, 3000), [0, nblk - 1]]))
    idx = torch.from_numpy(pick).cuda()
    xin = w.view(-1, blk_w)[idx].cpu().numpy()
    got = q.view(-1, blk_b)[idx].cpu().numpy()
    want, _ = oracle.quantize(fmt, xin.ravel())
    assert_bytes_equal(got.ravel(), want, blk_b)
    del w, q
    torch.cuda.empty_cache()


def _boundary_values(rng, step, limit, n):
    """n fp32 values on and one or two ulps around (k + 1/2) * step, |v| <= limit."""
    ks = rng.integers(-8, 8, size=n)
    base = ((ks + 0.5) * np.float64(step)).astype(np.float32)
    nudge = rng.integers(-2, 3, size=n)
    v = base.copy()
    for i in range(n):
        for _ in range(abs(int(nudge[i]))):
            v[i] = np.nextafter(v[i], np.float32(np.inf if nudge[i] > 0 else -np.inf))
    return np.where(np.abs(v) <= limit, v, np.float32(0.0)).astype(np.float32)


def test_q4_0_codes_at_rounding_boundaries():
    # every block: one element fixes absmax (so d = FP16(absmax / 7)), the
    # others sit exactly on a half-way point (k + 1/2) * d -- ties go to even
    # -- or one or two ulps from it; scales from FP16-subnormal to large
    rng = np.random.default_rng(2024)
    nb = 20000
    absmax = (2.0 ** rng.uniform(-26, 14, size=nb)).astype(np.float32)
    d = oracle.f16_bits_to_f32(oracle.f32_to_f16_bits(absmax / np.float32(7.0)))
    x = np.empty((nb, 32), dtype=np.float32)
    for b in range(nb):
        x[b] = _boundary_values(rng, d[b], absmax[b], 32)
        x[b, rng.integers(0, 32)] = absmax[b] * (1 if rng.random() < 0.5 else -1)
    want, _ = oracle.quantize(Q40, x.ravel())
    got, st = gpu_quantize(Q40, torch.from_numpy(x))
    assert st == 0
    assert_bytes_equal(got, want, 18)


def test_ksb_codes_at_rounding_boundaries():
    # each sub-block's absmax is 7 * d_j, so its FP16 scale is exactly d_j;
    # the other values sit on and around half-way points of the rebuilt
    # scale S * q_j that the codes are taken against
    rng = np.random.default_rng(7)
    nsb = 2500
    x = np.empty((nsb, 256), dtype=np.float32)
    for s in range(nsb):
        e = rng.uniform(-20, 10)
        d = oracle.f16_bits_to_f32(oracle.f32_to_f16_bits(
            (2.0 ** (e + rng.uniform(-3, 0, size=8))).astype(np.float32)))
        s_bits, q = oracle.ksb_scale_step(oracle.f32_to_f16_bits(d))
        S = oracle.f16_bits_to_f32(np.array([s_bits], np.uint16))[0]
        for j in range(8):
            st = np.float32(S) * np.float32(q[j])
            limit = np.float32(7.0) * d[j]
            x[s, 32 * j:32 * (j + 1)] = _boundary_values(rng, st if st > 0 else d[j], limit, 32)
            x[s, 32 * j + rng.integers(0, 32)] = limit
    want, _ = oracle.quantize(KSB, x.ravel())
    got, st = gpu_quantize(KSB, torch.from_numpy(x))
    assert st == 0
    assert_bytes_equal(got, want, 138)


def _nudge32(v, k):
    """v moved by k fp32 ulps (elementwise)."""
    v = v.astype(np.float32).copy()
    for i in range(v.size):
        for _ in range(abs(int(k[i]))):
            v[i] = np.nextafter(v[i], np.float32(np.inf if k[i] > 0 else -np.inf))
    return v


def test_q4_0_scales_at_fp16_midpoints():
    # absmax = 7 * m for m half-way between two FP16 values (exact in fp32),
    # then 0-3 fp32 ulps either side: absmax / 7 lands on or next to an FP16
    # rounding midpoint, so the FP16 scale depends on the last bit of the fp32
    # quotient; FP16-subnormal scales up to the largest finite one
    rng = np.random.default_rng(31)
    nb = 20000
    h = rng.integers(1, 0x7BFF, size=nb).astype(np.uint16)
    lo = oracle.f16_bits_to_f32(h).astype(np.float64)
    hi = oracle.f16_bits_to_f32((h + 1).astype(np.uint16)).astype(np.float64)
    absmax = _nudge32((7.0 * (lo + hi) / 2.0).astype(np.float32), rng.integers(-3, 4, size=nb))
    x = (rng.uniform(-0.9, 0.9, size=(nb, 32)) * absmax[:, None]).astype(np.float32)
    pos = rng.integers(0, 32, size=nb)
    x[np.arange(nb), pos] = absmax * np.where(rng.random(nb) < 0.5, 1, -1).astype(np.float32)
    want, flags = oracle.quantize(Q40, x.ravel())
    got, st = gpu_quantize(Q40, torch.from_numpy(x))
    assert st == flags == 0
    assert_bytes_equal(got, want, 18)


def test_ksb_subscales_at_half_integers():
    # the largest sub-block scale is 127 * S0 for S0 of 3 significant bits, so
    # the super-scale is exactly S0 and S0 * (k + 1/2) is an FP16 value: the
    # other seven sub-block scales sit on such a tie (rounded half to even
    # into q_j) or one FP16 ulp either side of it
    rng = np.random.default_rng(37)
    nsb = 4000
    e = rng.integers(-24, 1, size=nsb).astype(np.float64)
    s0 = (2.0 ** e) * (1.0 + rng.integers(0, 4, size=nsb) / 4.0)
    dmax = 127.0 * s0
    x = np.empty((nsb, 256), dtype=np.float32)
    for s in range(nsb):
        k = rng.integers(0, 127, size=8)
        dj = oracle.f32_to_f16_bits((s0[s] * (k + 0.5)).astype(np.float32))
        dj = np.clip(dj.astype(np.int64) + rng.integers(-1, 2, size=8), 1, 0x7BFF)
        d = oracle.f16_bits_to_f32(dj.astype(np.uint16)).astype(np.float64)
        d[0] = dmax[s]
        d = np.minimum(d, dmax[s])
        limit = (7.0 * d).astype(np.float32)  # exact: d has at most 11 bits
        blk = rng.uniform(-0.9, 0.9, size=(8, 32)) * limit[:, None]
        blk[np.arange(8), rng.integers(0, 32, size=8)] = limit
        x[s] = blk.astype(np.float32).ravel()
    want, flags = oracle.quantize(KSB, x.ravel())
    got, st = gpu_quantize(KSB, torch.from_numpy(x))
    assert st == flags == 0
    assert_bytes_equal(got, want, 138)


# ------------------------------------------------------------------------
# The page's reference quantizer (Q4_0 chapter 4.4; GQ_QUANT_REF_RULE)

def gpu_quantize_ref(x: np.ndarray):
    xt = torch.from_numpy(np.ascontiguousarray(x, np.float32).ravel()).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = gq.gq_quantize_q4_0_ex(xt, gq.GQ_QUANT_REF_RULE, dev_status=st)
    torch.cuda.synchronize()
    return q.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("rows,cols,seed", [(64, 1024, 0), (4096, 4096, 1), (7, 96, 2)])
def test_ref_rule_random(rows, cols, seed):
    w = synth.gaussian_weights(rows, cols, seed=seed).numpy()
    want, flags = oracle.quantize_q4_0(w.ravel(), rule=oracle.RULE_LLAMA)
    got, st = gpu_quantize_ref(w)
    assert st == flags
    assert_bytes_equal(got, want, 18)


def test_ref_rule_outlier_demo_and_ties():
    rng = np.random.default_rng(5)
    blocks = []
    # the page's outlier demo (section 4.5): 31 small values and one 10
    blocks.append(np.array([0.01 * (i - 15) / 15 for i in range(31)] + [10.0], np.float32))
    # equal magnitudes of both signs: the first one sets the sign of d
    for _ in range(200):
        b = rng.uniform(-1, 1, 32).astype(np.float32)
        m = np.float32(rng.uniform(1, 4))
        i, j = sorted(rng.choice(32, 2, replace=False))
        b[i], b[j] = (m, -m) if rng.random() < 0.5 else (-m, m)
        blocks.append(b)
    # zeros (signed and unsigned), a single value, subnormals, huge values
    blocks.append(np.zeros(32, np.float32))
    blocks.append(-np.zeros(32, np.float32))
    z = np.zeros(32, np.float32); z[17] = -3.0; blocks.append(z)
    blocks.append((rng.standard_normal(32) * 1e-40).astype(np.float32))
    blocks.append((rng.standard_normal(32) * 1e30).astype(np.float32))
    x = np.stack(blocks)
    want, flags = oracle.quantize_q4_0(x.ravel(), rule=oracle.RULE_LLAMA)
    got, st = gpu_quantize_ref(x)
    assert st == flags
    assert_bytes_equal(got, want, 18)


def test_ref_rule_code_boundaries():
    # values placed so that x * id + 8.5 lands on and beside integers, where
    # truncation decides the code
    rng = np.random.default_rng(11)
    nb = 20000
    vmax = (2.0 ** rng.uniform(-20, 10, nb)).astype(np.float32) * np.where(
        rng.random(nb) < 0.5, 1, -1).astype(np.float32)
    d = vmax / np.float32(-8.0)
    x = np.empty((nb, 32), np.float32)
    for b in range(nb):
        k = rng.integers(-8, 8, 32).astype(np.float64)
        v = ((k - 0.5) * np.float64(d[b])).astype(np.float32)     # x * id + 8.5 ~ k + 8
        nudge = rng.integers(-2, 3, 32)
        for i in range(32):
            for _ in range(abs(int(nudge[i]))):
                v[i] = np.nextafter(v[i], np.float32(np.inf if nudge[i] > 0 else -np.inf))
        v = np.where(np.abs(v) < np.abs(vmax[b]), v, np.float32(0.0))
        v[rng.integers(0, 32)] = vmax[b]
        x[b] = v
    want, flags = oracle.quantize_q4_0(x.ravel(), rule=oracle.RULE_LLAMA)
    got, st = gpu_quantize_ref(x)
    assert st == flags
    assert_bytes_equal(got, want, 18)


def test_ref_rule_flags_and_default_unchanged():
    x = np.zeros(32 * 64, np.float32)
    x[40] = 8 * 70000.0                      # |d| = 70000 overflows FP16
    _, st = gpu_quantize_ref(x)
    _, flags = oracle.quantize_q4_0(x, rule=oracle.RULE_LLAMA)
    assert st == flags == gq.GQ_DEV_RANGE
    x[40] = 1.0
    x[300] = np.nan
    _, st = gpu_quantize_ref(x)
    assert st & gq.GQ_DEV_NONFINITE
    # flags = 0 is the default rule, byte for byte
    w = synth.gaussian_weights(32, 512, seed=3)
    a = gq.gq_quantize_q4_0_ex(w.view(-1).cuda(), 0).cpu().numpy()
    b = gq.gq_quantize_q4_0(w.view(-1).cuda()).cpu().numpy()
    assert np.array_equal(a, b)
