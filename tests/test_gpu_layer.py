"""GPU parity of the backbone layer and the direction-cycled stack (through
the C ABI) against the fp64 oracle (oracle/backbone.py), on seeded synthetic
weights.

Tolerance: max|err| / max|ref| <= 1e-2 after one layer and after a stack.
Every layer rounds its activations to fp16 about ten times on the way (the
normalised input, the fused projection, q / k / v / z, the attention output,
the tail, the two residual sums, the SwiGLU's gate / value projection and its
product), each a relative error of at most 2^-11 = 4.9e-4 of the value rounded;
with the fp32 accumulations in between that is a few 1e-3 of max|ref| per
layer, so 1e-2 leaves room for five layers and still fails a wrong weight, a
wrong direction or a dropped term (each of which moves the output by O(1)
relative).  bf16 has 8 bits fewer in the mantissa: 5e-2.
"""
import numpy as np
import pytest
import torch

import oracle.backbone as bb
from recurrent_vision_backbone_chunkwise_b200.inputs import make_backbone_params

pytestmark = pytest.mark.gpu

TOL = {"f16": 1e-2, "bf16": 5e-2}
TDT = {"f16": torch.float16, "bf16": torch.bfloat16}


def _x0(B, gh, gw, C, dtype, seed):
    g = torch.Generator().manual_seed(seed + 1)
    return torch.randn(B, gh, gw, C, generator=g).to(TDT[dtype])


def _err(y, ref):
    return float(np.max(np.abs(y - ref)) / np.max(np.abs(ref)))


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_layer_matches_oracle(direction):
    from recurrent_vision_backbone_chunkwise_b200 import gla, layer

    B, gh, gw, C, F = 1, 6, 7, 128, 512
    params = make_backbone_params(C, F, 1, "f16", seed=direction)
    x0 = _x0(B, gh, gw, C, "f16", direction)
    x = x0.cuda()
    layer.gtr_layer_fwd(x, layer.pack_weights(params[0], "cuda"), direction)
    assert gla.gtr_gla_status() == 0
    ref = bb.layer_forward(x0, params[0], direction)
    assert _err(x.double().cpu().numpy(), ref) <= TOL["f16"]


@pytest.mark.parametrize("dtype,shape", [("f16", (2, 9, 11, 192, 768)), ("bf16", (1, 8, 8, 128, 512))])
def test_stack_matches_oracle(dtype, shape):
    """Five layers: the fifth scans L->R again, so the cycle's order is pinned."""
    from recurrent_vision_backbone_chunkwise_b200 import gla, layer

    B, gh, gw, C, F = shape
    params = make_backbone_params(C, F, 5, dtype, seed=3)
    x0 = _x0(B, gh, gw, C, dtype, 3)
    x = x0.cuda()
    layers = [layer.pack_weights(p, "cuda", TDT[dtype]) for p in params]
    layer.gtr_backbone_fwd(x, layers)
    assert gla.gtr_gla_status() == 0
    ref = bb.backbone_forward(x0, params)
    assert _err(x.double().cpu().numpy(), ref) <= TOL[dtype]


def test_stack_in_cuda_graph_matches_eager():
    """The 12-layer stack captured in one CUDA graph replays to the eager result
    bit for bit (same kernels, same order, fixed reduction orders)."""
    from recurrent_vision_backbone_chunkwise_b200 import gla, layer

    B, gh, gw, C, F = 1, 10, 12, 128, 512
    layers = [layer.pack_weights(p, "cuda") for p in make_backbone_params(C, F, 12, "f16", seed=5)]
    x0 = _x0(B, gh, gw, C, "f16", 5).cuda()
    ws = torch.zeros(layer.gtr_layer_workspace_size(B, gh, gw, C, F), dtype=torch.uint8, device="cuda")
    eager = x0.clone()
    layer.gtr_backbone_fwd(eager, layers, workspace=ws)
    torch.cuda.synchronize()
    xg = x0.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on the capture stream
        layer.gtr_backbone_fwd(xg, layers, workspace=ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        layer.gtr_backbone_fwd(xg, layers, workspace=ws, stream=s)
    xg.copy_(x0)
    g.replay()
    torch.cuda.synchronize()
    assert gla.gtr_gla_status() == 0
    assert torch.equal(xg, eager)


def test_binding_rejects_wrong_weights():
    from recurrent_vision_backbone_chunkwise_b200 import layer

    params = make_backbone_params(128, 512, 1, "f16", seed=0)
    w = layer.pack_weights(params[0], "cuda")
    x = torch.zeros(1, 4, 4, 192, dtype=torch.float16, device="cuda")
    with pytest.raises(ValueError):
        layer.gtr_layer_fwd(x, w, 0)  # C of x does not match the weights
    w.tensors["b_a"] = w.tensors["b_a"].half()
    with pytest.raises(ValueError):
        layer.gtr_layer_fwd(torch.zeros(1, 4, 4, 128, dtype=torch.float16, device="cuda"), w, 0)
