"""Out-of-bounds writes, checked without a sanitizer.

Every kernel writes its result into a view that sits inside a larger buffer
filled with a sentinel byte; after the call the bytes on both sides of the
view must be untouched, and the call's inputs must be unchanged.  Shapes are
ragged on purpose: row counts that leave partial 16-row groups and 128-row
tiles, K that leaves a partial pipeline chunk, super-block rows that start
off 16-byte boundaries, and sizes that leave a partial quantizer tile.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

GUARD = 512  # bytes on each side; a multiple of 16 keeps the views aligned
SENTINEL = 0xA5


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_gemv_q4_b200 as m
    return m


class Guarded:
    """A view of `nbytes` bytes with GUARD sentinel bytes before and after."""

    def __init__(self, nbytes, dtype=torch.uint8, shape=None):
        self.nbytes = nbytes
        self.buf = torch.full((nbytes + 2 * GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        v = self.buf[GUARD:GUARD + nbytes]
        v = v.view(dtype)
        self.view = v.view(shape) if shape is not None else v

    def intact(self):
        torch.cuda.synchronize()
        lo = self.buf[:GUARD]
        hi = self.buf[GUARD + self.nbytes:]
        return bool((lo == SENTINEL).all()) and bool((hi == SENTINEL).all())


def weights(M, K, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn((M, K), generator=g, device="cuda", dtype=torch.float32) * 0.02


@pytest.mark.parametrize("fmt,n", [("q4_0", 32 * 1001), ("q4_0", 32), ("ksb", 256 * 37),
                                   ("ksb", 256)])
def test_quantize_dequantize_stay_in_bounds(gq, fmt, n):
    x = weights(1, n, seed=n).view(-1)
    x0 = x.clone()
    qbytes = gq.gq_q4_0_bytes(n) if fmt == "q4_0" else gq.gq_ksb_bytes(n)
    q = Guarded(qbytes)
    (gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb)(x, out=q.view)
    assert q.intact()
    assert torch.equal(x, x0)
    q0 = q.view.clone()
    d = Guarded(4 * n, torch.float32)
    (gq.gq_dequantize_q4_0 if fmt == "q4_0" else gq.gq_dequantize_ksb)(q.view, n, out=d.view)
    assert d.intact()
    assert torch.equal(q.view, q0)


def test_reference_rule_quantizer_stays_in_bounds(gq):
    n = 32 * 777
    x = weights(1, n, seed=5).view(-1)
    q = Guarded(gq.gq_q4_0_bytes(n))
    gq.gq_quantize_q4_0_ex(x, gq.GQ_QUANT_REF_RULE, out=q.view)
    assert q.intact()


GEMV_CASES = [
    ("q4_0", 17, 288, 1, torch.float16, torch.float16),
    ("q4_0", 4097, 2080, 1, torch.float16, torch.float32),
    ("q4_0", 33, 11008, 3, torch.bfloat16, torch.bfloat16),
    ("q4_0", 129, 4096, 5, torch.float16, torch.float16),
    ("ksb", 40, 11008, 1, torch.float16, torch.float16),
    ("ksb", 23, 2304, 8, torch.float32, torch.float32),
]


@pytest.mark.parametrize("fmt,M,K,B,xt,yt", GEMV_CASES)
def test_gemv_stays_in_bounds(gq, fmt, M, K, B, xt, yt):
    quant = gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb
    W = quant(weights(M, K, seed=M + K).view(-1))
    W0 = W.clone()
    x = torch.randn((B, K), device="cuda").to(xt)
    x0 = x.clone()
    esz = torch.tensor([], dtype=yt).element_size()
    y = Guarded(B * M * esz, yt, (B, M))
    f = gq.gq_gemv_q4_0 if fmt == "q4_0" else gq.gq_gemv_ksb
    for flags in (0, gq.GQ_GEMV_PDL):
        f(W, M, K, x, y_dtype=yt, out=y.view, flags=flags)
        assert y.intact()
    assert torch.equal(W, W0) and torch.equal(x, x0)


def test_integer_path_stays_in_bounds(gq):
    M, K = 300, 4096
    W = gq.gq_quantize_q4_0(weights(M, K, seed=3).view(-1))
    x = torch.randn((1, K), device="cuda").half()
    y = Guarded(M * 2, torch.float16, (1, M))
    ws = torch.zeros(gq.gq_gemv_workspace_bytes(gq.GQ_FMT_Q4_0, M, K, 1, torch.float16),
                     dtype=torch.uint8, device="cuda")
    gq.gq_gemv_q4_0(W, M, K, x, y_dtype=torch.float16, out=y.view, workspace=ws)
    assert y.intact()


@pytest.mark.parametrize("fmt", ["q4_0", "ksb"])
def test_grouped_gemv_stays_in_bounds(gq, fmt):
    K = 2048
    Ms = [17, 300, 16, 1]
    quant = gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb
    Ws = [quant(weights(M, K, seed=40 + i).view(-1)) for i, M in enumerate(Ms)]
    x = torch.randn((2, K), device="cuda").half()
    outs = [Guarded(2 * M * 2, torch.float16, (2, M)) for M in Ms]
    fg = gq.gq_gemv_q4_0_grouped if fmt == "q4_0" else gq.gq_gemv_ksb_grouped
    fg(Ws, Ms, K, x, outs=[o.view for o in outs])
    assert all(o.intact() for o in outs)


@pytest.mark.parametrize("fmt,M,B", [("q4_0", 300, 17), ("q4_0", 129, 64), ("ksb", 200, 40),
                                     ("q4_0", 1000, 256)])
def test_gemm_stays_in_bounds(gq, fmt, M, B):
    K = 1024
    quant = gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb
    W = quant(weights(M, K, seed=M + B).view(-1))
    X = torch.randn((B, K), device="cuda").bfloat16()
    X0 = X.clone()
    code = gq.GQ_FMT_Q4_0 if fmt == "q4_0" else gq.GQ_FMT_KSB
    ws = torch.zeros(max(gq.gq_gemm_workspace_bytes(code, M, K, B), 1), dtype=torch.uint8,
                     device="cuda")
    Y = Guarded(B * M * 4, torch.float32, (B, M))
    f = gq.gq_gemm_q4_0 if fmt == "q4_0" else gq.gq_gemm_ksb
    f(W, M, K, X, out=Y.view, workspace=ws)
    f(W, M, K, X, out=Y.view, workspace=ws)  # the workspace is ready for a second call
    assert Y.intact()
    assert torch.equal(X, X0)
