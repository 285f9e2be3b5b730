"""GPU dequant-GEMM against the oracle's fp64 product: batches above 16 run
on the tcgen05 kernel, batches up to 16 on the warp-MMA product.

Tolerance per output: |Y - Y_ref| <= 1e-4 * sum_k |w_hat||x| plus one unit in
the last place of the output type.  Weights are quantized by the oracle."""
import numpy as np
import pytest
import torch

import bit_gemv_q4_b200 as gq
import oracle
import synth
from gpu_helpers import KSB, Q40, assert_product_close, x_for_oracle

pytestmark = pytest.mark.gpu

_cache = {}


def packed(fmt, M, K, gen="gauss"):
    key = (fmt, M, K, gen)
    if key not in _cache:
        w = (synth.gaussian_weights if gen == "gauss" else synth.logstd_weights)(M, K, seed=M + 3 * K)
        _cache[key] = oracle.quantize(fmt, w.numpy().ravel())[0]
    return _cache[key]


def run_gemm(fmt, q, M, K, X, ydt=torch.float32):
    f = gq.gq_gemm_q4_0 if fmt == Q40 else gq.gq_gemm_ksb
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = f(torch.from_numpy(q).cuda(), M, K, X.cuda(), y_dtype=ydt, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return Y


def check(fmt, M, K, B, ydt=torch.float32, gen="gauss", rows=None):
    q = packed(fmt, M, K, gen)
    X = synth.activations(B, K, seed=K + B, dtype=torch.bfloat16)
    Y = run_gemm(fmt, q, M, K, X, ydt)
    xo, xt = x_for_oracle(X)
    if rows is None:
        Yr, bound = oracle.gemm(fmt, q, M, K, xo, xt)
        return assert_product_close(Y, Yr, bound)
    Yr, bound = oracle.gemm_rows(fmt, q, M, K, xo, rows, xt)
    return assert_product_close(Y[:, torch.from_numpy(rows).cuda()], Yr, bound)


@pytest.mark.parametrize("fmt,M,K,B", [
    (Q40, 128, 256, 16), (Q40, 128, 512, 16), (Q40, 100, 1024, 7), (Q40, 300, 544, 33),
    (Q40, 1, 96, 1), (Q40, 257, 4096, 64), (KSB, 128, 512, 16), (KSB, 200, 1280, 48),
    (KSB, 129, 4352, 256),
])
def test_gemm_shapes(fmt, M, K, B):
    check(fmt, M, K, B)


@pytest.mark.parametrize("ydt", [torch.float16, torch.bfloat16])
def test_gemm_output_dtypes(ydt):
    check(Q40, 160, 1024, 24, ydt=ydt)


@pytest.mark.parametrize("fmt", [Q40, KSB])
@pytest.mark.parametrize("B", [16, 64, 256])
def test_gemm_batched_workload(fmt, B):
    # W 11008x4096 times X bf16 [B, 4096] ~ N(0,1); outputs checked on a
    # sample of rows spanning every 128-row tile and the ragged last tile
    M, K = 11008, 4096
    rows = np.unique(np.concatenate([np.arange(0, M, 37), [M - 1]])).astype(np.int64)
    check(fmt, M, K, B, gen="gauss" if fmt == Q40 else "logstd", rows=rows)


def test_gemm_matches_gemv_small_batch():
    M, K = 256, 2048
    q = packed(Q40, M, K)
    X = synth.activations(4, K, seed=5, dtype=torch.bfloat16).cuda()
    Wt = torch.from_numpy(q).cuda()
    y1 = gq.gq_gemm_q4_0(Wt, M, K, X)
    y2 = gq.gq_gemv_q4_0(Wt, M, K, X, y_dtype=torch.float32)
    torch.cuda.synchronize()
    Yr, bound = oracle.gemm(Q40, q, M, K, *x_for_oracle(X))
    assert_product_close(y1, Yr, bound)
    assert_product_close(y2, Yr, bound)


def test_gemm_stream_k_deterministic_and_reusable():
    # 1000 x 4096 with 36 k-steps per tile spread over every SM: most tiles
    # are cut between CTAs; their parts are summed in CTA order, so repeated
    # calls on one workspace give identical bits
    M, K, B = 1000, 4096, 40
    q = packed(Q40, M, K)
    X = synth.activations(B, K, seed=9, dtype=torch.bfloat16).cuda()
    Wt = torch.from_numpy(q).cuda()
    ws = torch.zeros(gq.gq_gemm_workspace_bytes(Q40, M, K, B), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        outs.append(gq.gq_gemm_q4_0(Wt, M, K, X, workspace=ws, dev_status=st))
        torch.cuda.synchronize()
        assert int(st.item()) == 0
    assert torch.equal(outs[0].view(torch.int32), outs[1].view(torch.int32))
    assert torch.equal(outs[0].view(torch.int32), outs[2].view(torch.int32))
    Yr, bound = oracle.gemm(Q40, q, M, K, *x_for_oracle(X))
    assert_product_close(outs[0], Yr, bound)


@pytest.mark.parametrize("M,K,B", [(20000, 64, 16), (8192, 256, 16), (3000, 1024, 256)])
def test_gemm_split_shapes(M, K, B):
    # one k-step per tile (whole tiles only), short rows with cuts inside
    # tiles, and the widest batch; checked on rows spanning every tile
    rows = np.unique(np.concatenate([np.arange(0, M, 29), [M - 1]])).astype(np.int64)
    check(Q40, M, K, B, rows=rows)


@pytest.mark.parametrize("fmt,M,K,B,ydt", [
    (Q40, 333, 2080, 9, torch.float32),      # ragged chunk, unaligned rows, odd batch
    (KSB, 150, 2304, 13, torch.bfloat16),
    (Q40, 4096, 4096, 16, torch.float32),
    (KSB, 1000, 4096, 12, torch.float16),
    (Q40, 17, 8192, 11, torch.float32),
    (Q40, 4096, 11008, 16, torch.float32),   # x beside the ring would need 399 KB:
    (KSB, 1000, 11008, 12, torch.float16),   # K split over clusters of 3 CTAs
    (Q40, 40, 16384, 16, torch.bfloat16),    # ... and of 4 CTAs
])
def test_gemm_warp_mma_batches(fmt, M, K, B, ydt):
    # batches 9..16 take two n8 tiles of the warp MMA (every code decoded once
    # for all 16 columns); columns past B are never stored
    check(fmt, M, K, B, ydt=ydt)


def test_gemm_refuses_short_workspace():
    M, K, B = 256, 512, 16
    Wt = torch.from_numpy(packed(Q40, M, K)).cuda()
    X = torch.zeros((B, K), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(gq.gq_gemm_workspace_bytes(Q40, M, K, B) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(gq.GQError):
        gq.gq_gemm_q4_0(Wt, M, K, X, workspace=ws)
