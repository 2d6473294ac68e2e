"""The entry point that allocates nothing (gtr_gla_fwd_noalloc).

It serves callers that cannot allocate device memory while they run, such as
a deployment with a fixed, pre-planned memory budget or host code without a
device allocator of its own: its scratch is a fixed array inside the library.
This file is collected last on purpose, and the test passes both alone in a
fresh process and after the other tests.  It calls the new entry point through
the C ABI twice in a row and compares each result with the library's default
entry point, gtr_gla_fwd, and with the fp64 oracle, at the fp16 tolerance the
parity tests use (5e-3 of max |reference|); after its first (set-up) call the
entry point must leave the device's free memory unchanged."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = 5e-3


def rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).abs().max() / b.abs().max())


def test_noalloc_matches_default_entry_point_on_two_calls():
    import oracle
    from recurrent_vision_backbone_chunkwise_b200 import gla
    from recurrent_vision_backbone_chunkwise_b200.inputs import CONFIGS, make_inputs

    shape, _ = CONFIGS["640_b1"]
    host = make_inputs(shape, "f16", seed=11)
    q, k, v, la = (t.cuda() for t in host)
    vp = ctypes.c_void_p
    stream = torch.cuda.current_stream().cuda_stream
    directions = (2, 1)  # two calls in a row
    # references first, then the library's own workspace is released, so that
    # nothing but the entry point under test could allocate below
    refs = {d: tuple(t.clone() for t in gla.gtr_gla_fwd(q, k, v, la, d)) for d in directions}
    gla.gtr_gla_release()
    outs = [torch.full_like(v, float("nan")) for _ in directions]
    fss = [torch.full((shape.B, shape.H, shape.d_k, shape.d_v), float("nan"), device="cuda")
           for _ in directions]
    torch.cuda.synchronize()
    free_after_setup = None
    for i, direction in enumerate(directions):
        rc = gla._lib.gtr_gla_fwd_noalloc(vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()),
                                          vp(la.data_ptr()), vp(outs[i].data_ptr()),
                                          vp(fss[i].data_ptr()), shape.B, shape.H, shape.grid_h,
                                          shape.grid_w, shape.d_k, shape.d_v, direction,
                                          vp(stream))
        assert rc == 0, gla.gtr_gla_strerror(rc)
        torch.cuda.synchronize()
        free_now = torch.cuda.mem_get_info()[0]
        if free_after_setup is None:
            free_after_setup = free_now
        else:
            assert free_now == free_after_setup, "the call allocated device memory"
    assert gla.gtr_gla_status() == 0
    for i, direction in enumerate(directions):
        out, fs = outs[i], fss[i]
        ref_o, ref_s = refs[direction]
        assert torch.isfinite(out).all() and torch.isfinite(fs).all()
        assert rel(out, ref_o) <= TOL
        assert rel(fs, ref_s) <= TOL
    # one direction against the fp64 oracle directly
    o_ref, s_ref = oracle.forward(*host, directions[0])
    got = outs[0].double().cpu().numpy()
    assert np.max(np.abs(got - o_ref)) / np.max(np.abs(o_ref)) <= TOL
    got_s = fss[0].double().cpu().numpy()
    assert np.max(np.abs(got_s - s_ref)) / np.max(np.abs(s_ref)) <= TOL


def test_noalloc_rejects_unsupported_head_size():
    from recurrent_vision_backbone_chunkwise_b200 import gla

    x = torch.zeros((1, 1, 4, 4, 128), dtype=torch.float16, device="cuda")
    la = torch.zeros((1, 1, 4, 4, 128), device="cuda")
    out = torch.empty_like(x)
    with pytest.raises(gla.GlaError) as e:
        gla.gtr_gla_fwd_noalloc(x, x.clone(), x.clone(), la, 0, out)
    assert e.value.code == -3
