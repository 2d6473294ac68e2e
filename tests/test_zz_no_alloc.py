"""The entry point that allocates nothing (gtr_gla_fwd_noalloc).

It serves callers that cannot allocate device memory while they run, such as
a deployment with a fixed, pre-planned memory budget or host code without a
device allocator of its own: its scratch is a fixed array inside the library.
This file is collected last on purpose, and the test passes both alone in a
fresh process and after the other tests.  It calls the new entry point through
the C ABI twice in a row and compares each result with the library's default
entry point, gtr_gla_fwd, at the fp16 tolerance the parity tests use (5e-3 of
max |reference|)."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = 5e-3


def rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).abs().max() / b.abs().max())


def test_noalloc_matches_default_entry_point_on_two_calls():
    from recurrent_vision_backbone_chunkwise_b200 import gla
    from recurrent_vision_backbone_chunkwise_b200.inputs import CONFIGS, make_inputs

    shape, _ = CONFIGS["640_b1"]
    q, k, v, la = (t.cuda() for t in make_inputs(shape, "f16", seed=11))
    vp = ctypes.c_void_p
    stream = torch.cuda.current_stream().cuda_stream
    for direction in (2, 1):  # two calls in a row
        ref_o, ref_s = gla.gtr_gla_fwd(q, k, v, la, direction)
        out = torch.full_like(v, float("nan"))
        fs = torch.full((shape.B, shape.H, shape.d_k, shape.d_v), float("nan"), device="cuda")
        rc = gla._lib.gtr_gla_fwd_noalloc(vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()),
                                          vp(la.data_ptr()), vp(out.data_ptr()), vp(fs.data_ptr()),
                                          shape.B, shape.H, shape.grid_h, shape.grid_w,
                                          shape.d_k, shape.d_v, direction, vp(stream))
        assert rc == 0, gla.gtr_gla_strerror(rc)
        assert gla.gtr_gla_status() == 0
        assert torch.isfinite(out).all() and torch.isfinite(fs).all()
        assert rel(out, ref_o) <= TOL
        assert rel(fs, ref_s) <= TOL


def test_noalloc_rejects_unsupported_head_size():
    from recurrent_vision_backbone_chunkwise_b200 import gla

    x = torch.zeros((1, 1, 4, 4, 128), dtype=torch.float16, device="cuda")
    la = torch.zeros((1, 1, 4, 4, 128), device="cuda")
    out = torch.empty_like(x)
    with pytest.raises(gla.GlaError) as e:
        gla.gtr_gla_fwd_noalloc(x, x.clone(), x.clone(), la, 0, out)
    assert e.value.code == -3
