"""Grouped GEMV (gq_gemv_*_grouped): several matrices sharing K and x in one
launch.  Every output is compared with the oracle's fp64 product (tolerance as
in test_gpu_gemv.py).  Tables with fewer than 8 row groups per SM run on the
single-matrix configuration and agree with the single-matrix entry point bit
for bit; larger tables run on the large-table configuration (four small CTAs
per SM), whose sums differ only in the order of fp32 additions."""
import numpy as np
import pytest
import torch

import bit_gemv_q4_b200 as gq
import oracle
import synth
from gpu_helpers import KSB, Q40, assert_product_close, x_for_oracle

pytestmark = pytest.mark.gpu


def _mats(fmt, Ms, K, seed):
    qs = []
    for i, M in enumerate(Ms):
        if M == 0:
            qs.append(np.zeros(0, np.uint8))
            continue
        w = synth.gaussian_weights(M, K, seed=seed + i).numpy().ravel()
        q, _ = oracle.quantize(fmt, w)
        qs.append(q)
    return qs


def _grouped(fmt, Wd, Ms, K, x, ydt, flags=0):
    f = gq.gq_gemv_q4_0_grouped if fmt == Q40 else gq.gq_gemv_ksb_grouped
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = f(Wd, Ms, K, x, y_dtype=ydt, flags=flags, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return outs


def _single(fmt, W, M, K, x, ydt):
    f = gq.gq_gemv_q4_0 if fmt == Q40 else gq.gq_gemv_ksb
    y = f(W, M, K, x, y_dtype=ydt)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("fmt,K,B,xdt,ydt", [
    (Q40, 4096, 1, torch.float16, torch.float16),
    (Q40, 2080, 3, torch.bfloat16, torch.float32),   # ragged chunks, unaligned rows
    (KSB, 4096, 1, torch.float16, torch.float16),
    (KSB, 2304, 2, torch.float32, torch.bfloat16),
])
def test_grouped_matches_oracle_and_single(fmt, K, B, xdt, ydt):
    Ms = [4096, 17, 0, 1, 300, 33, 2048]
    qs = _mats(fmt, Ms, K, seed=100 + K)
    Wd = [torch.from_numpy(q).cuda() if q.size else None for q in qs]
    x = synth.activations(B, K, seed=5, dtype=xdt).cuda()
    outs = _grouped(fmt, Wd, Ms, K, x, ydt)
    xo, xt = x_for_oracle(x)
    for q, W, M, y in zip(qs, Wd, Ms, outs):
        assert tuple(y.shape) == (B, M)
        if M == 0:
            continue
        Y, bound = oracle.gemm(fmt, q, M, K, xo, xt)
        assert_product_close(y, Y, bound)
        ys = _single(fmt, W, M, K, x, ydt)
        assert torch.equal(y.view(torch.int16) if y.dtype != torch.float32 else y.view(torch.int32),
                           ys.view(torch.int16) if ys.dtype != torch.float32 else ys.view(torch.int32))


def test_grouped_more_matrices_than_one_launch():
    # 300 matrices (more than one launch's table), with PDL between launches
    K = 512
    Ms = [(i * 37) % 70 + 1 for i in range(300)]
    qs = _mats(Q40, Ms, K, seed=7)
    Wd = [torch.from_numpy(q).cuda() for q in qs]
    x = synth.activations(1, K, seed=3, dtype=torch.float16).cuda()
    outs = _grouped(Q40, Wd, Ms, K, x, torch.float16, flags=gq.GQ_GEMV_PDL)
    xo, xt = x_for_oracle(x)
    for q, M, y in zip(qs, Ms, outs):
        Y, bound = oracle.gemm(Q40, q, M, K, xo, xt)
        assert_product_close(y, Y, bound)


def _every_group_rows(M):
    """One row in every 16-row group (its position inside the group varies)
    plus the last row."""
    g = np.arange((M + 15) // 16)
    rows = np.minimum(16 * g + (5 * g) % 16, M - 1)
    return np.unique(np.concatenate([rows, [M - 1]])).astype(np.int64)


def _large_table_case(fmt, Ms, K, seed, ydt=torch.float16):
    """Oracle-quantized matrices in one grouped call that takes the
    large-table configuration; each output checked on one row of every 16-row
    group against the oracle's fp64 product."""
    assert sum((M + 15) // 16 for M in Ms) >= 8 * torch.cuda.get_device_properties(0).multi_processor_count
    x = synth.activations(1, K, seed=seed, dtype=torch.float16).cuda()
    qs = _mats(fmt, Ms, K, seed=seed)
    Wd = [torch.from_numpy(q).cuda() for q in qs]
    outs = _grouped(fmt, Wd, Ms, K, x, ydt, flags=gq.GQ_GEMV_PDL)
    xo, xt = x_for_oracle(x)
    for q, M, y in zip(qs, Ms, outs):
        rows = _every_group_rows(M)
        Yr, bound = oracle.gemm_rows(fmt, q, M, K, xo, rows, xt)
        assert_product_close(y[:, torch.from_numpy(rows).cuda()], Yr, bound)


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_grouped_model_layer_shapes(fmt):
    # one decoder layer of the whole-model stream (4 x 4096^2 and 3 x
    # 11008x4096, 3088 row groups: the large-table configuration) with one x.
    # K = 4096 makes both formats' rows whole 16-byte granules (2304 / 2208
    # bytes), so the super-block case runs the compile-time word-offset
    # branch of that configuration.
    _large_table_case(fmt, [4096, 4096, 4096, 4096, 11008, 11008, 4096], 4096, seed=30000)


def test_grouped_large_table_unaligned_q4_0_rows():
    # the large-table configuration on Q4_0 rows that do not start on 16-byte
    # boundaries: K = 2080 is 65 blocks, 1170-byte rows (1280 row groups)
    _large_table_case(Q40, [4096] * 5, 2080, seed=41000, ydt=torch.float32)


def test_grouped_large_table_unaligned_ksb_rows():
    # super-block rows of K = 11008 (5934 bytes, starting at every even
    # offset mod 16) on the large-table configuration (1376 row groups)
    _large_table_case(KSB, [11008, 11008], 11008, seed=42000)


@pytest.mark.parametrize("fmt", [Q40, KSB])
def test_grouped_large_table_ragged(fmt):
    # 1300 matrices of 1..40 rows (about 2000 row groups: the large-table
    # configuration, in six launches of up to 256 matrices) against the oracle
    K = 512 if fmt == Q40 else 768
    rng = np.random.default_rng(3)
    Ms = [int(m) for m in rng.integers(1, 41, size=1300)]
    assert sum((M + 15) // 16 for M in Ms) >= 8 * torch.cuda.get_device_properties(0).multi_processor_count
    w = synth.gaussian_weights(sum(Ms), K, seed=17).numpy()
    qs, r0 = [], 0
    for M in Ms:
        q, _ = oracle.quantize(fmt, w[r0:r0 + M].ravel())
        qs.append(q)
        r0 += M
    Wd = [torch.from_numpy(q).cuda() for q in qs]
    x = synth.activations(2, K, seed=4, dtype=torch.bfloat16).cuda()
    outs = _grouped(fmt, Wd, Ms, K, x, torch.float32, flags=gq.GQ_GEMV_PDL)
    xo, xt = x_for_oracle(x)
    for q, M, y in zip(qs, Ms, outs):
        Y, bound = oracle.gemm(fmt, q, M, K, xo, xt)
        assert_product_close(y, Y, bound)
