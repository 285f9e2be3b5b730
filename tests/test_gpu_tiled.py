"""Tiled storage on the GPU: gq_repack_* against the oracle's repack byte for
byte, and the batch-1 GEMV on tiled storage against the oracle's fp64 product
of the canonical rows (tolerance as in test_gpu_gemv.py: 1e-4 * sum|w||x| plus
one unit in the last place of the output type).  Weights are quantized by the
oracle; the repack under test is the only step that makes the tiled bytes."""
import numpy as np
import pytest
import torch

import bit_gemv_q4_b200 as gq
import oracle
import synth
from gpu_helpers import KSB, Q40, assert_product_close, x_for_oracle

pytestmark = pytest.mark.gpu

_cache = {}


def packed(fmt, M, K, seed=None):
    key = (fmt, M, K, seed)
    if key not in _cache:
        s = (M * 13 + K) if seed is None else seed
        gen = synth.gaussian_weights if fmt == Q40 else synth.logstd_weights
        q, _ = oracle.quantize(fmt, gen(M, K, seed=s).numpy().ravel())
        _cache[key] = q
    return _cache[key]


def tiled(fmt, q, M, K):
    T = gq.gq_repack(fmt, torch.from_numpy(q).cuda(), M, K)
    torch.cuda.synchronize()
    return T


def run(fmt, T, M, K, x, ydt, flags=0):
    f = gq.gq_gemv_q4_0_tiled if fmt == Q40 else gq.gq_gemv_ksb_tiled
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = f(T, M, K, x.cuda(), y_dtype=ydt, flags=flags, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return y


@pytest.mark.parametrize("fmt,M,K", [
    (Q40, 16, 64), (Q40, 17, 4160), (Q40, 4096, 11008), (Q40, 11008, 4096),
    (KSB, 1, 256), (KSB, 33, 2304), (KSB, 4096, 11008), (KSB, 11008, 4096),
])
def test_repack_matches_oracle(fmt, M, K):
    q = packed(fmt, M, K)
    T = tiled(fmt, q, M, K)
    want = oracle.repack(fmt, q, M, K)
    assert T.numel() == want.size == gq.gq_tiled_bytes(fmt, M, K)
    assert np.array_equal(T.cpu().numpy(), want)


@pytest.mark.parametrize("fmt,M,K", [
    (Q40, 4096, 11008), (Q40, 11008, 4096), (Q40, 4096, 4096),
    (KSB, 4096, 11008), (KSB, 11008, 4096),
])
@pytest.mark.parametrize("flags", [0, 1])
def test_tiled_gemv_workload_shapes(fmt, M, K, flags):
    q = packed(fmt, M, K)
    x = synth.activations(1, K, seed=K + 1, dtype=torch.float16)
    y = run(fmt, tiled(fmt, q, M, K), M, K, x, torch.float16, flags)
    Y, bound = oracle.gemm(fmt, q, M, K, *x_for_oracle(x))
    assert_product_close(y, Y, bound)


@pytest.mark.parametrize("fmt,M,K", [
    (Q40, 1, 64), (Q40, 3, 128), (Q40, 17, 1088), (Q40, 33, 16384), (Q40, 129, 2112),
    (KSB, 1, 256), (KSB, 15, 512), (KSB, 47, 2816), (KSB, 65, 16384), (KSB, 31, 4352),
])
@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16])
def test_tiled_gemv_edge_shapes(fmt, M, K, ydt):
    q = packed(fmt, M, K)
    x = synth.activations(1, K, seed=M, dtype=torch.float16)
    T = tiled(fmt, q, M, K)
    Y, bound = oracle.gemm(fmt, q, M, K, *x_for_oracle(x))
    for flags in (0, gq.GQ_GEMV_PDL):
        assert_product_close(run(fmt, T, M, K, x, ydt, flags), Y, bound)


@pytest.mark.parametrize("fmt,M,K", [(Q40, 64, 16384), (KSB, 48, 11008), (Q40, 300, 11008),
                                     (KSB, 129, 16384), (Q40, 4096, 11008)])
def test_tiled_gemv_chain_with_stash(fmt, M, K):
    # each CTA's share is more tiles than the ring holds, so with PDL the
    # first tiles go through tensor memory; four launches on different
    # matrices back to back, each free to start while the previous one runs
    qs = [packed(fmt, M, K, seed=M + K + i) for i in range(4)]
    Ts = [tiled(fmt, q, M, K) for q in qs]
    x = synth.activations(1, K, seed=K, dtype=torch.float16)
    xd = x.cuda()
    f = gq.gq_gemv_q4_0_tiled if fmt == Q40 else gq.gq_gemv_ksb_tiled
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ys = [f(T, M, K, xd, y_dtype=torch.float32, flags=gq.GQ_GEMV_PDL, dev_status=st) for T in Ts]
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for q, y in zip(qs, ys):
        Y, bound = oracle.gemm(fmt, q, M, K, *x_for_oracle(x))
        assert_product_close(y, Y, bound)


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_tiled_gemv_extreme_activations(fmt):
    # activations spanning the fp16 range: outliers near 3e4, values near 1e-3,
    # fp16 subnormals, exact zeros, both signs
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
    T = tiled(fmt, q, M, K)
    Y, bound = oracle.gemm(fmt, q, M, K, *x_for_oracle(x))
    for flags in (0, gq.GQ_GEMV_PDL):
        assert_product_close(run(fmt, T, M, K, x, torch.float32, flags), Y, bound)


@pytest.mark.parametrize("fmt,M,K", [(Q40, 33, 4160), (KSB, 40, 11008)])
def test_tiled_stays_in_bounds(fmt, M, K):
    # repack writes exactly gq_tiled_bytes bytes and the GEMV exactly M outputs:
    # sentinel bytes on both sides of each output stay untouched
    guard, sent = 512, 0xA5
    q = torch.from_numpy(packed(fmt, M, K)).cuda()
    n = gq.gq_tiled_bytes(fmt, M, K)
    tb = torch.full((n + 2 * guard,), sent, dtype=torch.uint8, device="cuda")
    T = tb[guard:guard + n]
    gq.gq_repack(fmt, q, M, K, out=T)
    yb = torch.full((4 * M + 2 * guard,), sent, dtype=torch.uint8, device="cuda")
    y = yb[guard:guard + 4 * M].view(torch.float32).view(1, M)
    x = synth.activations(1, K, seed=1, dtype=torch.float16).cuda()
    q0 = q.clone()
    f = gq.gq_gemv_q4_0_tiled if fmt == Q40 else gq.gq_gemv_ksb_tiled
    f(T, M, K, x, y_dtype=torch.float32, out=y, flags=gq.GQ_GEMV_PDL)
    torch.cuda.synchronize()
    for b in (tb, yb):
        assert bool((b[:guard] == sent).all()) and bool((b[-guard:] == sent).all())
    assert torch.equal(q, q0)


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_tiled_gemv_table_batches(fmt):
    # K = 16384 leaves room for six row groups in the partial-sum table, and
    # 16576 rows are 1036 row groups, seven per CTA on 148 SMs: the table is
    # filled, reduced and filled again
    M, K = 16576, 16384
    q = packed(fmt, M, K)
    x = synth.activations(1, K, seed=5, dtype=torch.float16)
    T = tiled(fmt, q, M, K)
    Y, bound = oracle.gemm(fmt, q, M, K, *x_for_oracle(x))
    for flags in (0, gq.GQ_GEMV_PDL):
        assert_product_close(run(fmt, T, M, K, x, torch.float32, flags), Y, bound)


@pytest.mark.parametrize("fmt", [Q40, KSB])
@pytest.mark.parametrize("bad", [float("inf"), float("-inf"), float("nan")])
def test_tiled_gemv_nonfinite_activation(fmt, bad):
    # one non-finite activation reaches every output row: each row multiplies
    # it by a decoded weight, and the block's -8 * sum(x) correction carries
    # it even where the code is 8 (weight zero)
    M, K = 48, 2048
    q = packed(fmt, M, K)
    x = synth.activations(1, K, seed=4, dtype=torch.float16)
    x[0, 777] = bad
    T = tiled(fmt, q, M, K)
    for flags in (0, gq.GQ_GEMV_PDL):
        y = run(fmt, T, M, K, x, torch.float32, flags)
        assert not bool(torch.isfinite(y).any())


def grouped(fmt):
    return gq.gq_gemv_q4_0_tiled_grouped if fmt == Q40 else gq.gq_gemv_ksb_tiled_grouped


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_tiled_grouped_decoder_layer(fmt):
    # the seven projections of one decoder layer of the 4096 / 11008 model
    # that share one input (four 4096-row, three 11008-row matrices, K = 4096)
    # in one call; each output is bit for bit the single-matrix tiled GEMV's
    K = 4096
    Ms = [4096] * 4 + [11008] * 3
    qs = [packed(fmt, M, K, seed=100 + i) for i, M in enumerate(Ms)]
    Ts = [tiled(fmt, q, M, K) for q, M in zip(qs, Ms)]
    x = synth.activations(1, K, seed=21, dtype=torch.float16)
    xd = x.cuda()
    for flags in (0, gq.GQ_GEMV_PDL):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        ys = grouped(fmt)(Ts, Ms, K, xd, y_dtype=torch.float32, flags=flags, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for q, T, M, y in zip(qs, Ts, Ms, ys):
            Y, bound = oracle.gemm(fmt, q, M, K, *x_for_oracle(x))
            assert_product_close(y, Y, bound)
            assert torch.equal(y, run(fmt, T, M, K, x, torch.float32, flags))


@pytest.mark.parametrize("fmt,K", [(Q40, 1088), (KSB, 2304), (Q40, 16384), (KSB, 16384)])
def test_tiled_grouped_ragged(fmt, K):
    # ragged row counts (one row, a partial group, exact groups), an empty
    # entry in the middle, and bfloat16 outputs
    Ms = [1, 17, 0, 48, 333, 16]
    qs = [packed(fmt, M, K, seed=7 * i + K) if M else None for i, M in enumerate(Ms)]
    Ts = [tiled(fmt, q, M, K) if M else torch.empty(0, dtype=torch.uint8, device="cuda")
          for q, M in zip(qs, Ms)]
    x = synth.activations(1, K, seed=K + 3, dtype=torch.float16)
    for flags in (0, gq.GQ_GEMV_PDL):
        ys = grouped(fmt)(Ts, Ms, K, x.cuda(), y_dtype=torch.bfloat16, flags=flags)
        torch.cuda.synchronize()
        for q, M, y in zip(qs, Ms, ys):
            if M == 0:
                assert y.numel() == 0
                continue
            Y, bound = oracle.gemm(fmt, q, M, K, *x_for_oracle(x))
            assert_product_close(y, Y, bound)


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_tiled_grouped_more_than_one_launch(fmt):
    # 300 matrices: more than one launch's table of 256, in stream order
    K = 1024 if fmt == Q40 else 2048
    Ms = [16 + (i % 5) * 7 for i in range(300)]
    q = packed(fmt, max(Ms), K, seed=9)
    rb = len(q) // max(Ms)
    T_by_M = {M: tiled(fmt, q[:M * rb], M, K) for M in set(Ms)}
    x = synth.activations(1, K, seed=2, dtype=torch.float16)
    ys = grouped(fmt)([T_by_M[M] for M in Ms], Ms, K, x.cuda(), y_dtype=torch.float32,
                      flags=gq.GQ_GEMV_PDL)
    torch.cuda.synchronize()
    want = {M: oracle.gemm(fmt, q[:M * rb], M, K, *x_for_oracle(x)) for M in set(Ms)}
    for M, y in zip(Ms, ys):
        assert_product_close(y, *want[M])


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_tiled_grouped_stays_in_bounds(fmt):
    # every output of the table gets exactly its M values: sentinel bytes
    # around each output stay untouched
    K = 2048
    Ms = [33, 16, 70]
    guard, sent = 256, 0xA5
    qs = [packed(fmt, M, K, seed=40 + M) for M in Ms]
    Ts = [tiled(fmt, q, M, K) for q, M in zip(qs, Ms)]
    bufs = [torch.full((4 * M + 2 * guard,), sent, dtype=torch.uint8, device="cuda") for M in Ms]
    outs = [b[guard:guard + 4 * M].view(torch.float32).view(1, M) for b, M in zip(bufs, Ms)]
    x = synth.activations(1, K, seed=8, dtype=torch.float16)
    grouped(fmt)(Ts, Ms, K, x.cuda(), outs=outs, flags=gq.GQ_GEMV_PDL)
    torch.cuda.synchronize()
    for b in bufs:
        assert bool((b[:guard] == sent).all()) and bool((b[-guard:] == sent).all())
    for q, M, y in zip(qs, Ms, outs):
        assert_product_close(y, *oracle.gemm(fmt, q, M, K, *x_for_oracle(x)))



@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_tiled_grouped_table_batches(fmt):
    # K = 16384 leaves room for six row groups in the partial-sum table;
    # two 16576-row matrices are 2072 row groups, seven per CTA on two CTAs
    # per SM of 148 SMs: the table is filled, reduced and filled again.  The
    # same weights twice, so both outputs must match the oracle and each other.
    M, K = 16576, 16384
    q = packed(fmt, M, K)
    T = tiled(fmt, q, M, K)
    x = synth.activations(1, K, seed=6, dtype=torch.float16)
    Y, bound = oracle.gemm(fmt, q, M, K, *x_for_oracle(x))
    for flags in (0, gq.GQ_GEMV_PDL):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        ys = grouped(fmt)([T, T], [M, M], K, x.cuda(), y_dtype=torch.float32, flags=flags,
                          dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert_product_close(ys[0], Y, bound)
        assert torch.equal(ys[0], ys[1])


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_tiled_grouped_chained_layers(fmt):
    # one grouped call per layer, three layers chained with PDL, so that each
    # launch stages its first tiles (six tiles per row group at K = 11008,
    # more than the ring holds) while the previous one still runs; every
    # output equals the same call made alone, and one matrix is checked
    # against the oracle
    K = 11008
    Ms = [256] * 4 + [688] * 3
    qs = [[packed(fmt, M, K, seed=500 + 10 * l + i) for i, M in enumerate(Ms)] for l in range(3)]
    Ts = [[tiled(fmt, q, M, K) for q, M in zip(ql, Ms)] for ql in qs]
    x = synth.activations(1, K, seed=31, dtype=torch.float16)
    xd = x.cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ys = [grouped(fmt)(Tl, Ms, K, xd, y_dtype=torch.float32, flags=gq.GQ_GEMV_PDL, dev_status=st)
          for Tl in Ts]
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for Tl, yl in zip(Ts, ys):
        alone = grouped(fmt)(Tl, Ms, K, xd, y_dtype=torch.float32)
        torch.cuda.synchronize()
        for a, b in zip(yl, alone):
            assert torch.equal(a, b)
    Y, bound = oracle.gemm(fmt, qs[2][5], Ms[5], K, *x_for_oracle(x))
    assert_product_close(ys[2][5], Y, bound)
