"""Failure detection without a GPU fault: a GEMV whose first pipeline stage is
never filled (a flag nothing sets) must end on its own after a ~1 ms bounded
wait, report GQ_DEV_TIMEOUT, and leave the context usable."""
import numpy as np
import pytest
import torch

import bit_gemv_q4_b200 as gq
import oracle
import synth
from gpu_helpers import Q40, assert_product_close, x_for_oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    M, K = 48, 8192
    w = synth.gaussian_weights(M, K, seed=3)
    q, _ = oracle.quantize_q4_0(w.numpy().ravel())
    Wt = torch.from_numpy(q).cuda()
    x = synth.activations(1, K, seed=4, dtype=torch.float16).cuda()
    y = torch.empty((1, M), dtype=torch.float16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gq.gq_selftest_gemv_timeout(Wt, M, K, x, y, st)
    torch.cuda.synchronize()
    assert int(st.item()) & gq.GQ_DEV_TIMEOUT
    assert gq.gq_status_from_dev(int(st.item())) == 7
    # the same buffers through the normal path: correct, no status bits
    st.zero_()
    y2 = gq.gq_gemv_q4_0(Wt, M, K, x, y_dtype=torch.float32, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    Y, bound = oracle.gemm(Q40, q, M, K, *x_for_oracle(x))
    assert_product_close(y2, Y, bound)
