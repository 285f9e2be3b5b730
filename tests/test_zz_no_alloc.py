"""gq_gemv_q4_0_noalloc -- the batch-1 integer GEMV path with the library's
static scratch -- against the same path through gq_gemv_q4_0 with a caller
workspace, on two consecutive calls per shape (the second call runs on the
scratch the first one used).  Collected last on purpose: it must pass after
every other test has run in the same process, as well as alone."""
import numpy as np
import pytest
import torch

import bit_gemv_q4_b200 as gq
import oracle
import synth
from gpu_helpers import Q40, assert_product_close, x_for_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K", [(4096, 11008), (11008, 4096), (300, 2048), (17, 256)])
def test_noalloc_matches_workspace_path(M, K):
    w = synth.gaussian_weights(M, K, seed=M + K)
    q, _ = oracle.quantize(Q40, w.numpy().ravel())
    Wt = torch.from_numpy(q).cuda()
    need = gq.gq_gemv_workspace_bytes(Q40, M, K, 1, torch.float16)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for call in range(2):
        x = synth.activations(1, K, seed=call + 5, dtype=torch.float16).cuda()
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        y_ref = gq.gq_gemv_q4_0(Wt, M, K, x, y_dtype=torch.float32, workspace=ws)
        y = gq.gq_gemv_q4_0_noalloc(Wt, M, K, x, y_dtype=torch.float32, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        # same kernel, same partition, same order of every sum: identical bits
        assert torch.equal(y.view(torch.int32), y_ref.view(torch.int32)), call
        Y, bound = oracle.gemm(Q40, q, M, K, *x_for_oracle(x.cpu()))
        assert_product_close(y, Y, bound)


def test_noalloc_refuses_what_it_cannot_run():
    x = torch.zeros((1, 288), dtype=torch.float16, device="cuda")
    W = torch.zeros(64 * 9 * 18, dtype=torch.uint8, device="cuda")
    with pytest.raises(gq.GQError):  # K % 256 != 0
        gq.gq_gemv_q4_0_noalloc(W, 64, 288, x)
    x = torch.zeros((1, 16384), dtype=torch.float16, device="cuda")
    W = torch.zeros(4 * 512 * 18, dtype=torch.uint8, device="cuda")
    with pytest.raises(gq.GQError):  # K beyond the resident activation split
        gq.gq_gemv_q4_0_noalloc(W, 4, 16384, x)
