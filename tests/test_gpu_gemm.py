"""GPU parity of the library's tensor-core GEMM (gtr_gemm_fwd, through the C
ABI) against the product in float64 on the CPU (numpy), with the bias and
residual added in float64.

Tolerance: max|err| / max|ref| <= 2e-3 for fp16 (the result is rounded once
to fp16, a relative error of at most 2^-11 = 4.9e-4 of each element, and the
fp32 sums over K <= 3072 products add far less), 1e-2 for bf16 (2^-8)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = {torch.float16: 2e-3, torch.bfloat16: 1e-2}


def ref(x, w, b, r):
    y = x.double().numpy() @ w.double().numpy().T
    if b is not None:
        y = y + b.double().numpy()
    if r is not None:
        y = y + r.double().numpy()
    return y


def rel(a, b):
    return float(np.max(np.abs(a.double().cpu().numpy() - b)) / np.max(np.abs(b)))


@pytest.mark.parametrize("M,N,K,bias,resid,dtype", [
    (1600, 3072, 384, False, False, torch.float16),   # SwiGLU gate/value projection, 640x640 grid, C = 384
    (1600, 384, 1536, True, True, torch.float16),     # down projection with bias and residual
    (1600, 1920, 384, False, False, torch.bfloat16),  # the layer's fused q/k/v/gate/output-gate projection
    (1000, 136, 72, True, False, torch.float16),      # ragged M, N and K tails
    (1, 8, 8, True, True, torch.float16),             # one row
    (3333, 512, 256, False, True, torch.bfloat16),
    (300, 256, 1000, True, True, torch.float16),      # K not a multiple of 64 (the last block zero-filled)
    (1600, 768, 3072, False, False, torch.bfloat16),  # long K
    (3840, 768, 512, True, True, torch.float16),      # 192-wide tiles
    (3840, 760, 256, False, True, torch.bfloat16),    # 192-wide tiles with a column tail
])
def test_gemm_matches_float64(M, N, K, bias, resid, dtype):
    from recurrent_vision_backbone_chunkwise_b200 import gemm, gla

    g = torch.Generator().manual_seed(M + N + K)
    x = torch.randn(M, K, generator=g).to(dtype)
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(dtype)
    b = (0.1 * torch.randn(N, generator=g)).to(dtype) if bias else None
    r = torch.randn(M, N, generator=g).to(dtype) if resid else None
    dev = [t.cuda() if t is not None else None for t in (x, w, b, r)]
    y = gemm.gtr_gemm_fwd(*dev)
    assert gla.gtr_gla_status() == 0
    assert rel(y, ref(x, w, b, r)) <= TOL[dtype]


def test_gemm_accumulates_in_place():
    """resid = out: out += x . w^T (the residual branches of the layer)."""
    from recurrent_vision_backbone_chunkwise_b200 import gemm, gla

    g = torch.Generator().manual_seed(1)
    x = torch.randn(700, 384, generator=g).half()
    w = (torch.randn(384, 384, generator=g) / 20).half()
    r = torch.randn(700, 384, generator=g).half()
    out = r.cuda()
    gemm.gtr_gemm_fwd(x.cuda(), w.cuda(), resid=out, out=out)
    assert gla.gtr_gla_status() == 0
    assert rel(out, ref(x, w, None, r)) <= TOL[torch.float16]


def test_gemm_is_deterministic():
    """Fixed accumulation order: two calls agree bit for bit."""
    from recurrent_vision_backbone_chunkwise_b200 import gemm, gla

    g = torch.Generator().manual_seed(3)
    x = torch.randn(1600, 1536, generator=g).half().cuda()
    w = (torch.randn(384, 1536, generator=g) / 40).half().cuda()
    a = gemm.gtr_gemm_fwd(x, w)
    b = gemm.gtr_gemm_fwd(x, w)
    torch.cuda.synchronize()
    assert gla.gtr_gla_status() == 0
    assert torch.equal(a, b)
