"""GPU dequantize-fused GEMV against the oracle's fp64 product.

Tolerance, per output: |y - y_ref| <= 1e-4 * sum_k |w_hat||x| plus one unit in
the last place of the output type (the fp32 result is rounded once to fp16 /
bf16).  Weights are quantized by the oracle, so every input byte of the GPU
product comes from the oracle side."""
import numpy as np
import pytest
import torch

import bit_gemv_q4_b200 as gq
import oracle
import synth
from gpu_helpers import KSB, Q40, assert_product_close, x_for_oracle

pytestmark = pytest.mark.gpu

_cache = {}


def packed(fmt, M, K, gen="gauss", seed=None):
    key = (fmt, M, K, gen, seed)
    if key not in _cache:
        s = (M * 7 + K) if seed is None else seed
        w = (synth.gaussian_weights if gen == "gauss" else synth.logstd_weights)(M, K, seed=s)
        q, _ = oracle.quantize(fmt, w.numpy().ravel())
        _cache[key] = q
    return _cache[key]


def run_gemv(fmt, q, M, K, x, ydt, flags=0):
    f = gq.gq_gemv_q4_0 if fmt == Q40 else gq.gq_gemv_ksb
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = f(torch.from_numpy(q).cuda(), M, K, x.cuda(), y_dtype=ydt, flags=flags, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return y


def check(fmt, M, K, B, xdt, ydt, gen="gauss", flags=0, seed=None):
    q = packed(fmt, M, K, gen, seed)
    x = synth.activations(B, K, seed=B + K, dtype=xdt)
    y = run_gemv(fmt, q, M, K, x, ydt, flags)
    xo, xt = x_for_oracle(x)
    Y, bound = oracle.gemm(fmt, q, M, K, xo, xt)
    return assert_product_close(y, Y, bound)


# the five workloads' product shapes
def test_tiny_fp32_in_fp32_out():
    # W 256x1024 (seed 0) N(0, 0.02^2) with 0.1 % x10 outliers; x fp32; y fp32
    check(Q40, 256, 1024, 1, torch.float32, torch.float32, seed=0)


def test_decode_4096x4096_fp16():
    check(Q40, 4096, 4096, 1, torch.float16, torch.float16)


@pytest.mark.parametrize("B", [1, 8])
def test_ksb_mlp_11008x4096(B):
    check(KSB, 11008, 4096, B, torch.float16, torch.float16, gen="logstd")


@pytest.mark.parametrize("fmt", [Q40, KSB])
@pytest.mark.parametrize("M,K", [(4096, 11008), (11008, 4096)])
def test_metric_shapes(fmt, M, K):
    # both orientations of the 4096x11008 headline shape, with and without PDL
    check(fmt, M, K, 1, torch.float16, torch.float16)
    check(fmt, M, K, 1, torch.float16, torch.float16, flags=gq.GQ_GEMV_PDL)


# edge shapes: ragged row tiles, single blocks, K chunks with ragged tails
@pytest.mark.parametrize("fmt,M,K", [
    (Q40, 1, 32), (Q40, 7, 64), (Q40, 17, 288), (Q40, 33, 1056), (Q40, 4097, 2080),
    (Q40, 5, 3072 + 32), (KSB, 1, 256), (KSB, 15, 512), (KSB, 17, 1280), (KSB, 129, 2304),
])
def test_edge_shapes(fmt, M, K):
    check(fmt, M, K, 1, torch.float16, torch.float16)


@pytest.mark.parametrize("B", [1, 2, 3, 5, 7, 8])
@pytest.mark.parametrize("xdt", [torch.float16, torch.bfloat16, torch.float32])
def test_batches_and_dtypes(B, xdt):
    ydt = {torch.float16: torch.float32, torch.bfloat16: torch.bfloat16,
           torch.float32: torch.float16}[xdt]
    check(Q40, 100, 2048, B, xdt, ydt)
    check(KSB, 100, 2048, B, xdt, ydt, gen="logstd")


def test_wide_batch_window():
    # fp32 activations of 8 rows at K = 20480 (ten 2048-weight chunks): a
    # chunk of x alone fills the shared memory left beside the ring, so a
    # K split would need more than 8 CTAs per cluster; x is streamed in
    # windows instead
    check(Q40, 40, 20480, 8, torch.float32, torch.float32)
    check(KSB, 24, 20480, 8, torch.float32, torch.float16, gen="logstd")


# Batches whose activations do not fit beside the ring: K is split over a
# cluster of 2..8 CTAs, each with its slice of x resident, the partial sums
# added in rank order through distributed shared memory.
@pytest.mark.parametrize("fmt,M,K,B,xdt,ydt", [
    (Q40, 4096, 11008, 8, torch.float16, torch.float16),   # 2 CTAs, 3 chunks each
    (KSB, 300, 11008, 8, torch.float16, torch.float32),    # unaligned rows
    (Q40, 300, 11008, 6, torch.bfloat16, torch.bfloat16),
    (KSB, 129, 11008, 7, torch.float16, torch.float16),
    (Q40, 64, 11008, 8, torch.float32, torch.float32),     # 6 CTAs, one chunk each
    (KSB, 48, 11008, 8, torch.float16, torch.float32),
    (KSB, 33, 16384, 8, torch.float16, torch.float16),     # 2 CTAs, 4 chunks each
    (Q40, 17, 16384, 2, torch.float32, torch.float32),
    (Q40, 1, 11008, 8, torch.float16, torch.float32),      # one row
    (Q40, 7, 16448, 5, torch.float32, torch.float32),      # ragged last chunk, 5 CTAs
])
@pytest.mark.parametrize("flags", [0, 1])
def test_k_split_over_cluster(fmt, M, K, B, xdt, ydt, flags):
    check(fmt, M, K, B, xdt, ydt, gen="gauss" if fmt == Q40 else "logstd", flags=flags)


def test_k_split_deterministic():
    # rank 0 adds the other ranks' sums in rank order: repeated calls agree
    # bit for bit
    M, K, B = 1000, 11008, 8
    q = torch.from_numpy(packed(KSB, M, K)).cuda()
    x = synth.activations(B, K, seed=3, dtype=torch.float16).cuda()
    ys = [gq.gq_gemv_ksb(q, M, K, x, y_dtype=torch.float32, flags=gq.GQ_GEMV_PDL)
          for _ in range(4)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


def test_k_zero_writes_zeros():
    y = torch.full((2, 5), 7.0, device="cuda")
    W = torch.zeros(16, dtype=torch.uint8, device="cuda")
    x = torch.zeros((2, 0), dtype=torch.float16, device="cuda")
    gq.gq_gemv_q4_0(W, 5, 0, x, y_dtype=torch.float32, out=y)
    torch.cuda.synchronize()
    assert torch.all(y == 0)


def test_constant_codes_closed_form():
    # every block d = 0.5, every code 11 -> y = 1.5 * sum(x)
    M, K = 40, 4096
    blk = np.array([0x00, 0x38] + [0xBB] * 16, np.uint8)
    q = np.tile(blk, M * K // 32)
    x = synth.activations(3, K, seed=3, dtype=torch.float16)
    y = run_gemv(Q40, q, M, K, x, torch.float32)
    want = 1.5 * x.double().sum(dim=1)
    assert torch.allclose(y.double().cpu(), want[:, None].expand(3, M), rtol=1e-5, atol=1e-4)


# the batch-1 fp16 kernel: K a multiple of 64 (Q4_0) or 256 (super-blocks), up
# to 16384; super-block rows of odd K / 256 are grouped by parity; ragged M
@pytest.mark.parametrize("fmt,M,K", [
    (Q40, 1, 64), (Q40, 3, 128), (Q40, 17, 1088), (Q40, 33, 16384), (Q40, 7, 16448),
    (KSB, 1, 768), (KSB, 33, 256), (KSB, 47, 2816), (KSB, 65, 16384), (KSB, 31, 4352),
])
@pytest.mark.parametrize("flags", [0, 1])
def test_batch1_fp16_shapes(fmt, M, K, flags):
    check(fmt, M, K, 1, torch.float16, torch.float32, flags=flags)


@pytest.mark.parametrize("fmt,M,K", [(Q40, 64, 16384), (KSB, 48, 11008), (Q40, 300, 11008),
                                     (KSB, 129, 16384)])
def test_batch1_tensor_memory_stash(fmt, M, K):
    # few row groups over a long K: each CTA's share is more stages than the
    # shared-memory ring holds, so with PDL the first stages go through
    # tensor memory; three launches back to back on different matrices, each
    # free to start while the previous one runs
    qs = [packed(fmt, M, K, seed=M + K + i) for i in range(3)]
    x = synth.activations(1, K, seed=K, dtype=torch.float16)
    f = gq.gq_gemv_q4_0 if fmt == Q40 else gq.gq_gemv_ksb
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Wd = [torch.from_numpy(q).cuda() for q in qs]
    xd = x.cuda()
    ys = [f(W, M, K, xd, y_dtype=torch.float32, flags=gq.GQ_GEMV_PDL, dev_status=st) for W in Wd]
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    xo, xt = x_for_oracle(x)
    for q, y in zip(qs, ys):
        Y, bound = oracle.gemm(fmt, q, M, K, xo, xt)
        assert_product_close(y, Y, bound)


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_batch1_extreme_activations(fmt):
    # activations spanning the fp16 range: outliers near 3e4, values near 1e-3,
    # fp16 subnormals, exact zeros and both signs
    M, K = 96, 4096
    q = packed(fmt, M, K)
    g = torch.Generator().manual_seed(11)
    x = torch.randn((1, K), generator=g)
    idx = torch.randperm(K, generator=g)
    x[0, idx[:8]] = torch.tensor([3.0e4, -2.5e4, 1.2e4, -6.0e3, 900.0, -700.0, 4.0e3, -3.3e4])
    x[0, idx[8:200]] *= 1e-3
    x[0, idx[200:260]] = torch.randint(-1023, 1024, (60,), generator=g).float() * 2.0 ** -24
    x[0, idx[260:300]] = 0.0
    x = x.to(torch.float16)
    for flags in (0, gq.GQ_GEMV_PDL):
        y = run_gemv(fmt, q, M, K, x, torch.float32, flags)
        Y, bound = oracle.gemm(fmt, q, M, K, *x_for_oracle(x))
        assert_product_close(y, Y, bound)


def test_misaligned_rows_large_k():
    # K = 11008 super-blocks give 5934-byte rows, so most rows start off a
    # 16-byte boundary; an offset view of W shifts them all
    M, K = 40, 11008
    q = packed(KSB, M, K)
    x = synth.activations(1, K, seed=1, dtype=torch.float16)
    y = run_gemv(KSB, q, M, K, x, torch.float32)
    Y, bound = oracle.gemm(KSB, q, M, K, *x_for_oracle(x))
    assert_product_close(y, Y, bound)


def test_concurrent_host_threads():
    # several host threads launch products of different shapes (different
    # shared-memory sizes and kernel configurations) on their own streams at
    # once; every result equals the same call made alone
    import threading
    # (the last case splits K over clusters of 2 CTAs)
    cases = [(Q40, 4096, 4096, 1), (KSB, 300, 11008, 1), (Q40, 1000, 2048, 8), (KSB, 129, 4352, 3),
             (KSB, 200, 11008, 8)]
    data = []
    for fmt, M, K, B in cases:
        q = torch.from_numpy(packed(fmt, M, K)).cuda()
        x = synth.activations(B, K, seed=M + B, dtype=torch.float16).cuda()
        f = gq.gq_gemv_q4_0 if fmt == Q40 else gq.gq_gemv_ksb
        ref = f(q, M, K, x, y_dtype=torch.float32)
        data.append((f, q, M, K, x, ref))
    torch.cuda.synchronize()
    errors = []

    def worker(i):
        try:
            f, q, M, K, x, ref = data[i % len(data)]
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(20):
                    y = f(q, M, K, x, y_dtype=torch.float32, stream=s)
            s.synchronize()
            if not torch.equal(y, ref):
                errors.append(i)
        except Exception as e:  # reported below
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(8)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
