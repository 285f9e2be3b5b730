"""The batch-1 integer tensor-core GEMV path (Q4_0, fp16 x, a workspace)
against the oracle's fp64 product, and its workspace contract.

The path splits x exactly into signed 7-bit digit columns and multiplies
unsigned codes on the integer MMA, so its only rounding is the fp32
accumulation; the tolerance is the same as for every GEMV:
|y - y_ref| <= 1e-4 * sum_k |w_hat||x| plus one ulp of the output type."""
import numpy as np
import pytest
import torch

import bit_gemv_q4_b200 as gq
import oracle
import synth
from gpu_helpers import Q40, assert_product_close, x_for_oracle

pytestmark = pytest.mark.gpu


def packed(M, K, seed):
    w = synth.gaussian_weights(M, K, seed=seed)
    q, _ = oracle.quantize(Q40, w.numpy().ravel())
    return q


def workspace(M, K):
    need = gq.gq_gemv_workspace_bytes(Q40, M, K, 1, torch.float16)
    assert need > 0
    return torch.zeros(need, dtype=torch.uint8, device="cuda")


def run(q, M, K, x, ydt, ws, flags=0):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = gq.gq_gemv_q4_0(torch.from_numpy(q).cuda(), M, K, x.cuda(), y_dtype=ydt, flags=flags,
                        dev_status=st, workspace=ws)
    torch.cuda.synchronize()
    return y, int(st.item())


def check(M, K, ydt=torch.float16, seed=1, x=None, flags=0):
    q = packed(M, K, seed)
    if x is None:
        x = synth.activations(1, K, seed=seed + 1, dtype=torch.float16)
    ws = workspace(M, K)
    y, st = run(q, M, K, x, ydt, ws, flags)
    assert st == 0
    Y, bound = oracle.gemm(Q40, q, M, K, *x_for_oracle(x))
    assert_product_close(y, Y, bound)
    return q, x, ws, y


@pytest.mark.parametrize("M,K", [
    (4096, 11008), (11008, 4096), (4096, 4096),      # the benchmark shapes
    (1, 256), (17, 256), (33, 512), (100, 2048),     # ragged row groups, one slice
    (4097, 2048), (40, 14336), (3, 1536 * 8),        # cut row groups, ragged M, longest K
])
def test_parity(M, K):
    check(M, K)


def test_long_rows_take_the_other_path():
    # activation fragments of K > 14336 do not stay resident: no workspace
    assert gq.gq_gemv_workspace_bytes(Q40, 40, 65536, 1, torch.float16) == 0
    assert gq.gq_gemv_workspace_bytes(Q40, 40, 14336, 1, torch.float16) > 0


def test_fp32_and_bf16_outputs_and_pdl():
    check(300, 4096, ydt=torch.float32)
    check(300, 4096, ydt=torch.bfloat16, flags=gq.GQ_GEMV_PDL)


def test_deterministic_and_workspace_reusable():
    # row groups cut between CTAs: the parts are combined in CTA order
    # whatever CTA finishes last, and a workspace serves call after call
    M, K = 2000, 11008
    q, x, ws, y0 = check(M, K, ydt=torch.float32)
    for _ in range(3):
        y, st = run(q, M, K, x, torch.float32, ws)
        assert st == 0
        assert torch.equal(y.view(torch.int32), y0.view(torch.int32))


def test_same_result_class_as_path_without_workspace():
    M, K = 512, 4096
    q = packed(M, K, 5)
    x = synth.activations(1, K, seed=6, dtype=torch.float16)
    Y, bound = oracle.gemm(Q40, q, M, K, *x_for_oracle(x))
    y_ws, st = run(q, M, K, x, torch.float32, workspace(M, K))
    y_nows, st2 = run(q, M, K, x, torch.float32, None)
    assert st == 0 and st2 == 0
    assert_product_close(y_ws, Y, bound)
    assert_product_close(y_nows, Y, bound)


def test_extreme_activations_are_split_exactly():
    # the largest fp16 value, the smallest subnormal, the smallest normal and
    # values near each power of two: the digit split is exact for all of them
    K = 4096
    vals = torch.tensor([65504.0, -65504.0, 2.0 ** -24, -(2.0 ** -24), 2.0 ** -14, 6.0e-5,
                         1.0, -1.0, 0.5, 3.0, -1024.0, 2047.0, 0.0, -0.0], dtype=torch.float32)
    x = synth.activations(1, K, seed=9, dtype=torch.float32)
    x[0, :vals.numel()] = vals
    x[0, 1000:1000 + vals.numel()] = vals * 0.75
    x = x.to(torch.float16)
    check(64, K, ydt=torch.float32, x=x)


def test_constant_codes_closed_form():
    # every block d = 0.5, every code 11 -> y = 1.5 * sum(x), for all rows
    M, K = 40, 4096
    blk = np.array([0x00, 0x38] + [0xBB] * 16, np.uint8)
    q = np.tile(blk, M * K // 32)
    x = synth.activations(1, K, seed=3, dtype=torch.float16)
    y, st = run(q, M, K, x, torch.float32, workspace(M, K))
    assert st == 0
    want = 1.5 * x.double().sum()
    assert torch.allclose(y.double().cpu(), want.expand(1, M), rtol=1e-6, atol=1e-5)


def test_nonfinite_activation_gives_nan():
    M, K = 64, 2048
    q = packed(M, K, 2)
    x = synth.activations(1, K, seed=4, dtype=torch.float16)
    x[0, 77] = float("inf")
    ws = workspace(M, K)
    y, st = run(q, M, K, x, torch.float32, ws)
    assert st & gq.GQ_DEV_NONFINITE
    assert torch.isnan(y).all()
    # the workspace is still usable afterwards
    x[0, 77] = 0.5
    y, st = run(q, M, K, x, torch.float32, ws)
    assert st == 0
    Y, bound = oracle.gemm(Q40, q, M, K, *x_for_oracle(x))
    assert_product_close(y, Y, bound)


def test_ineligible_calls_ignore_the_workspace():
    # batch 2, bf16 x and K % 256 != 0 take the path without a workspace
    M = 96
    for K, B, xdt in ((4096, 2, torch.float16), (4096, 1, torch.bfloat16), (288, 1, torch.float16)):
        q = packed(M, K, 7)
        x = synth.activations(B, K, seed=8, dtype=xdt)
        ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
        y = gq.gq_gemv_q4_0(torch.from_numpy(q).cuda(), M, K, x.cuda(), y_dtype=torch.float32,
                            workspace=ws)
        torch.cuda.synchronize()
        Y, bound = oracle.gemm(Q40, q, M, K, *x_for_oracle(x))
        assert_product_close(y, Y, bound)
        assert int(ws.count_nonzero()) == 0  # untouched


def test_small_workspace_is_refused():
    M, K = 64, 2048
    q = torch.from_numpy(packed(M, K, 3)).cuda()
    x = torch.ones((1, K), dtype=torch.float16, device="cuda")
    need = gq.gq_gemv_workspace_bytes(Q40, M, K, 1, torch.float16)
    ws = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(gq.GQError):
        gq.gq_gemv_q4_0(q, M, K, x, workspace=ws)


def test_workspace_shared_across_shapes():
    # one buffer serves calls of different shapes in turn (its size does not
    # depend on the shape)
    shapes = [(4096, 11008), (11008, 4096), (300, 2048), (4096, 11008)]
    assert len({gq.gq_gemv_workspace_bytes(Q40, M, K, 1, torch.float16) for M, K in shapes}) == 1
    need = max(gq.gq_gemv_workspace_bytes(Q40, M, K, 1, torch.float16) for M, K in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for i, (M, K) in enumerate(shapes):
        q = packed(M, K, 20 + i)
        x = synth.activations(1, K, seed=30 + i, dtype=torch.float16)
        y, st = run(q, M, K, x, torch.float32, ws)
        assert st == 0
        Y, bound = oracle.gemm(Q40, q, M, K, *x_for_oracle(x))
        assert_product_close(y, Y, bound)
