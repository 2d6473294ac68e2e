"""C-ABI checks that need no GPU: the library loads, exports every entry point
that include/*.h declares, and rejects bad arguments before touching memory
(fake pointer values are never dereferenced on those paths)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def gla():
    from recurrent_vision_backbone_chunkwise_b200 import build

    build.build()
    from recurrent_vision_backbone_chunkwise_b200 import gla as g

    return g


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(gtr_(?:gla|swiglu|output_tail|layer|backbone|gemm)_\w+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("gtr_gla_fwd", "gtr_gla_fwd_ex", "gtr_gla_workspace_size", "gtr_gla_status",
              "gtr_gla_strerror", "gtr_gla_release", "gtr_gla_launch_count",
              "gtr_swiglu_fwd", "gtr_swiglu_workspace_size", "gtr_output_tail_fwd",
              "gtr_layer_fwd", "gtr_backbone_fwd", "gtr_layer_workspace_size", "gtr_gemm_fwd"):
        assert n in names


def test_library_exports_every_declared_symbol(gla):
    lib = ctypes.CDLL(gla.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
        # the binding forwards under the same name
        from recurrent_vision_backbone_chunkwise_b200 import gemm, layer, output_tail, swiglu

        mod = (swiglu if n.startswith("gtr_swiglu_") else output_tail if n.startswith("gtr_output_tail_")
               else layer if n.startswith(("gtr_layer_", "gtr_backbone_"))
               else gemm if n.startswith("gtr_gemm_") else gla)
        assert hasattr(mod, n), n


def test_strerror_and_count(gla):
    assert gla.gtr_gla_strerror(0) == "ok"
    assert "direction" in gla.gtr_gla_strerror(-4)
    assert gla.gtr_gla_strerror(12345) == "unknown error code"
    for code in range(-13, 0):  # every declared code has its own text
        assert gla.gtr_gla_strerror(code) != "unknown error code", code
    assert "workspace header" in gla.gtr_gla_strerror(-12)
    assert "timed out" in gla.gtr_gla_strerror(-10)
    assert gla.gtr_gla_launch_count() >= 0


def test_workspace_size(gla):
    assert gla.gtr_gla_workspace_size(1, 6, 40, 40, 64, 64, gla.F16, 64) > 0
    # invalid shapes report 0
    assert gla.gtr_gla_workspace_size(0, 6, 40, 40, 64, 64, gla.F16, 64) == 0
    assert gla.gtr_gla_workspace_size(1, 6, 40, 40, 48, 64, gla.F16, 64) == 0
    # the header (64 KiB) at least; beyond it the size follows the segment plan
    # (which may hold fewer segment states for more planes), not the batch
    for B in (1, 2, 8):
        assert gla.gtr_gla_workspace_size(B, 12, 128, 128, 64, 64, gla.F16, 64) >= 65536


# fake, 256-aligned, non-overlapping "device" addresses; never dereferenced
Q, K, V, LA, OUT, FS, WS = (0x10000000 * (i + 1) for i in range(7))


def call_ex(gla, **kw):
    a = dict(q=Q, k=K, v=V, la=LA, out=OUT, fs=FS, B=1, H=2, gh=4, gw=4, dk=64, dv=64,
             dir=0, dtype=gla.F16, chunk=64, ws=WS, wsb=1 << 30)
    a.update(kw)
    vp = ctypes.c_void_p
    return gla._lib.gtr_gla_fwd_ex(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["la"]),
                                   vp(a["out"]), vp(a["fs"]), a["B"], a["H"], a["gh"],
                                   a["gw"], a["dk"], a["dv"], a["dir"], a["dtype"],
                                   a["chunk"], vp(a["ws"]), a["wsb"], vp(0))


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(la=0), -1), (dict(out=0), -1),
    (dict(B=0), -2), (dict(gh=-1), -2), (dict(H=70000), -2),
    (dict(H=1024, gh=2048, gw=1024), -2),  # 2^31 token rows in all
    (dict(dk=32), -3), (dict(dv=96), -3),
    (dict(dir=4), -4), (dict(dir=-1), -4),
    (dict(q=Q + 8), -5), (dict(fs=FS + 4), -5),
    (dict(dtype=3), -6),
    (dict(chunk=48), -7), (dict(chunk=16), -7),
    (dict(ws=0), -8), (dict(wsb=16), -8), (dict(ws=WS + 16), -8),
    (dict(out=Q + 256), -11), (dict(fs=OUT), -11),
    (dict(ws=OUT), -11), (dict(ws=LA + 4096), -11), (dict(ws=FS), -11),  # workspace on a tensor
])
def test_argument_errors_return_before_launch(gla, kw, code):
    assert call_ex(gla, **kw) == code


def test_chunk_128_needs_dk_64(gla):
    # chunk 128 is supported only with d_k = 64 (shared-memory bound); the
    # calls below are rejected before anything is launched
    for dtype in (gla.F16, gla.BF16, gla.F32):
        assert call_ex(gla, dtype=dtype, chunk=128, dk=128, dv=128) == -7
        assert call_ex(gla, dtype=dtype, chunk=128, dk=128, dv=64) == -7


def test_noalloc_rejects_before_touching_memory(gla):
    vp = ctypes.c_void_p
    args = [vp(Q), vp(K), vp(V), vp(LA), vp(OUT), vp(FS)]
    # d = 128 is not a problem the allocation-free entry point handles
    assert gla._lib.gtr_gla_fwd_noalloc(*args, 1, 2, 4, 4, 128, 128, 0, vp(0)) == -3
    assert gla._lib.gtr_gla_fwd_noalloc(*args, 1, 2, 4, 4, 64, 64, 7, vp(0)) == -4
    assert gla._lib.gtr_gla_fwd_noalloc(vp(0), *args[1:], 1, 2, 4, 4, 64, 64, 0, vp(0)) == -1


def test_swiglu_argument_errors_before_launch(gla):
    """Spatial SwiGLU entry point: every argument error is reported before
    anything is launched (the fake pointers are never dereferenced)."""
    import ctypes as C

    from recurrent_vision_backbone_chunkwise_b200 import swiglu

    lib = swiglu._lib
    p = C.c_void_p(1 << 20)  # 16-byte aligned fake address

    def call(ptrs=None, B=1, gh=4, gw=4, Cc=64, F=256, dtype=gla.F16, ws=p, wsb=1 << 40):
        ptrs = ptrs or [p] * 8
        return lib.gtr_swiglu_fwd(*ptrs, B, gh, gw, Cc, F, dtype, ws, wsb, None)

    assert call(ptrs=[p] * 7 + [None]) == -1          # y NULL
    assert call(B=0) == -2 and call(Cc=60) == -2 and call(F=100) == -2
    assert call(dtype=gla.F32) == -6
    assert call(ptrs=[p] * 6 + [C.c_void_p((1 << 20) + 4), p]) == -5   # b_down misaligned
    assert call(ptrs=[p] * 8) == -11                  # y aliases the inputs
    q = [C.c_void_p((1 << 20) + (i << 32)) for i in range(8)]
    assert call(ptrs=q, ws=None) == -8                 # no workspace
    assert call(ptrs=q, wsb=16) == -8                  # workspace too small
    assert call(ptrs=q) == -11                         # workspace on x
    assert call(ptrs=q, ws=q[3]) == -11                # workspace on the depthwise taps
    assert swiglu.gtr_swiglu_workspace_size(1, 4, 4, 60, 256) == 0
    assert swiglu.gtr_swiglu_workspace_size(1, 40, 40, 384, 1536) > 1600 * 3 * 1536 * 2


def test_output_tail_argument_errors_before_launch(gla):
    """Output-tail entry point: every argument error is reported before
    anything is launched (the fake pointers are never dereferenced)."""
    import ctypes as C

    from recurrent_vision_backbone_chunkwise_b200 import output_tail

    lib = output_tail._lib
    q = [C.c_void_p((1 << 20) + (i << 32)) for i in range(4)]  # distinct, 16-byte aligned

    def call(ptrs=None, B=1, H=2, gh=4, gw=4, dv=64, eps=1e-5, dtype=gla.F16):
        return lib.gtr_output_tail_fwd(*(ptrs or q), B, H, gh, gw, dv, eps, dtype, None)

    assert call(ptrs=q[:3] + [None]) == -1              # y NULL
    assert call(B=0) == -2 and call(H=-1) == -2 and call(gw=0) == -2
    assert call(eps=-1.0) == -2 and call(eps=float("nan")) == -2 and call(eps=float("inf")) == -2
    assert call(dv=32) == -3 and call(dv=96) == -3
    assert call(dtype=gla.F32) == -6
    assert call(ptrs=q[:2] + [C.c_void_p((1 << 20) + (2 << 32) + 8), q[3]]) == -5   # w misaligned
    assert call(ptrs=q[:3] + [q[0]]) == -11              # y is o


def _tensors(dt=None):
    import torch

    dt = dt or torch.float16
    q = torch.zeros((1, 2, 4, 5, 64), dtype=dt)
    return q, q.clone(), torch.zeros((1, 2, 4, 5, 64), dtype=dt), torch.zeros((1, 2, 4, 5, 64))


@pytest.mark.parametrize("bad", ["la_f16", "k_shape", "v_dtype", "out_small", "out_strided",
                                 "fs_f16", "fs_shape", "cpu"])
def test_binding_checks_tensors_before_any_call(gla, bad):
    """The binding rejects tensors whose dtype, shape, layout or device would
    make the library read or write outside them, before calling it (these
    checks need no GPU: every tensor here is a CPU tensor, and the device is
    checked last)."""
    import torch

    q, k, v, la = _tensors()
    out, fs = None, None
    if bad == "la_f16":
        la = la.half()
    elif bad == "k_shape":
        k = k[..., :32].contiguous()
    elif bad == "v_dtype":
        v = v.bfloat16()
    elif bad == "out_small":
        out = torch.zeros((1, 2, 4, 4, 64), dtype=torch.float16)
    elif bad == "out_strided":
        out = torch.zeros((1, 2, 4, 5, 128), dtype=torch.float16)[..., ::2]
    elif bad == "fs_f16":
        fs = torch.zeros((1, 2, 64, 64), dtype=torch.float16)
    elif bad == "fs_shape":
        fs = torch.zeros((1, 2, 64, 32))
    before = gla.gtr_gla_launch_count()
    for fn in (gla.gtr_gla_fwd, gla.gtr_gla_fwd_ex):
        with pytest.raises(ValueError) as e:
            fn(q, k, v, la, 0, out=out, final_state=fs)
        if bad == "cpu":
            assert "CUDA device" in str(e.value)
    with pytest.raises(ValueError):
        gla.gtr_gla_fwd_noalloc(q, k, v, la, 0, out if out is not None else torch.zeros_like(v), fs)
    assert gla.gtr_gla_launch_count() == before


# ---------------------------------------------------------------- backbone layer

def _layer_struct(layer, base=0x40000000, **override):
    vals = {n: base + 0x100000 * i for i, n in enumerate(layer._FIELDS)}
    vals.update(override)
    return layer.GtrLayerWeights(*[ctypes.c_void_p(vals[n]) for n in layer._FIELDS])


def call_layer(gla, **kw):
    from recurrent_vision_backbone_chunkwise_b200 import layer

    a = dict(x=0x20000000, w=_layer_struct(layer), B=1, gh=6, gw=7, C=128, F=512, dir=0,
             dtype=gla.F16, ws=0x30000000, wsb=1 << 34)
    a.update(kw)
    w = a["w"]
    return gla._lib.gtr_layer_fwd(ctypes.c_void_p(a["x"]), None if w is None else ctypes.byref(w), a["B"],
                                  a["gh"], a["gw"], a["C"], a["F"], a["dir"], a["dtype"],
                                  ctypes.c_void_p(a["ws"]), a["wsb"], None)


def test_layer_workspace_size(gla):
    from recurrent_vision_backbone_chunkwise_b200 import layer

    a = layer.gtr_layer_workspace_size(1, 40, 40, 384, 1536, gla.F16)
    assert a > 0 and layer.gtr_layer_workspace_size(8, 40, 40, 384, 1536, gla.F16) > a
    assert layer.gtr_layer_workspace_size(1, 40, 40, 100, 400, gla.F16) == 0  # C not a multiple of 64
    assert layer.gtr_layer_workspace_size(1, 40, 40, 128, 0, gla.F16) == 0
    assert layer.gtr_layer_workspace_size(1, 40, 40, 128, 512, gla.F32) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(x=0), -1), (dict(w=None), -1), ("w_o_null", -1),
    (dict(C=100), -2), (dict(C=4096), -2), (dict(F=0), -2), (dict(F=12), -2), (dict(B=0), -2),
    (dict(dir=4), -4), (dict(dtype=2), -6), (dict(x=0x20000008), -5), ("w_gu_misaligned", -5),
    (dict(ws=0), -8), (dict(wsb=1024), -8), (dict(ws=0x30000010), -8),
    (dict(x=0x30000000), -11),            # x inside the workspace
    ("w_o_on_x", -11), ("w_dw_in_ws", -11),
])
def test_layer_argument_errors(gla, kw, code):
    from recurrent_vision_backbone_chunkwise_b200 import layer

    if kw == "w_o_null":
        kw = dict(w=_layer_struct(layer, w_o=0))
    elif kw == "w_gu_misaligned":
        kw = dict(w=_layer_struct(layer, w_gu=0x50000004))
    elif kw == "w_o_on_x":
        kw = dict(w=_layer_struct(layer, w_o=0x20000000 - 4096))  # [C, C] fp16 runs into x
    elif kw == "w_dw_in_ws":
        kw = dict(w=_layer_struct(layer, w_dw=0x30000100))
    assert call_layer(gla, **kw) == code



def test_backbone_argument_errors(gla):
    from recurrent_vision_backbone_chunkwise_b200 import layer

    arr = (layer.GtrLayerWeights * 2)(_layer_struct(layer), _layer_struct(layer, b_dw=0))
    vp = ctypes.c_void_p
    f = gla._lib.gtr_backbone_fwd
    assert f(vp(0x20000000), arr, 2, 1, 6, 7, 128, 512, gla.F16, vp(0x30000000), 1 << 34, None) == -1
    assert f(vp(0x20000000), None, 2, 1, 6, 7, 128, 512, gla.F16, vp(0x30000000), 1 << 34, None) == -1
    assert f(vp(0x20000000), arr, 0, 1, 6, 7, 128, 512, gla.F16, vp(0x30000000), 1 << 34, None) == -2
    assert f(vp(0x20000000), arr, 1, 1, 6, 7, 128, 512, gla.F16, vp(0x30000000), 1024, None) == -8
    arr2 = (layer.GtrLayerWeights * 2)(_layer_struct(layer), _layer_struct(layer, b_down=0x20000000))
    assert f(vp(0x20000000), arr2, 2, 1, 6, 7, 128, 512, gla.F16, vp(0x30000000), 1 << 34, None) == -11


# ------------------------------------------------------------ fused output tail

def call_tail(gla, **kw):
    a = dict(q=Q, k=K, v=V, la=LA, z=0x80000000, w=0x90000000, eps=1e-5, y=OUT, fs=FS, B=1, H=2, gh=4,
             gw=4, dk=64, dv=64, dir=0, dtype=gla.F16, ws=WS, wsb=1 << 30)
    a.update(kw)
    vp = ctypes.c_void_p
    return gla._lib.gtr_gla_fwd_tail(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["la"]), vp(a["z"]), vp(a["w"]),
                                     a["eps"], vp(a["y"]), vp(a["fs"]), a["B"], a["H"], a["gh"], a["gw"],
                                     a["dk"], a["dv"], a["dir"], a["dtype"], vp(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(z=0), -1), (dict(w=0), -1), (dict(y=0), -1), (dict(q=0), -1),
    (dict(eps=-1.0), -2), (dict(eps=float("nan")), -2), (dict(eps=float("inf")), -2), (dict(B=0), -2),
    (dict(dk=48), -3), (dict(dir=5), -4), (dict(z=0x80000008), -5), (dict(w=0x90000004), -5),
    (dict(dtype=2), -6), (dict(wsb=0), -8), (dict(ws=0), -8),
    (dict(z=OUT + 64), -11), (dict(y=Q), -11), (dict(w=OUT + 256), -11),
    (dict(ws=0x80000000), -11), (dict(ws=K), -11), (dict(ws=OUT), -11),  # workspace on z, k, y
])
def test_tail_argument_errors(gla, kw, code):
    assert call_tail(gla, **kw) == code


def test_tail_workspace_size(gla):
    a = gla.gtr_gla_tail_workspace_size(1, 6, 40, 40, 64, 64, gla.F16)
    assert a == gla.gtr_gla_workspace_size(1, 6, 40, 40, 64, 64, gla.F16, 64)  # fused: no o buffer
    b = gla.gtr_gla_tail_workspace_size(1, 6, 40, 40, 128, 128, gla.F16)
    assert b >= gla.gtr_gla_workspace_size(1, 6, 40, 40, 128, 128, gla.F16, 64) + 1600 * 6 * 128 * 2
    assert gla.gtr_gla_tail_workspace_size(1, 6, 40, 40, 64, 64, gla.F32) == 0


def test_checked_build_exports_every_declared_symbol(gla):
    from recurrent_vision_backbone_chunkwise_b200 import build

    path = build.build(checked=True)
    lib = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(lib, n), n
    lib.gtr_gla_strerror.restype = ctypes.c_char_p
    assert b"index check" in lib.gtr_gla_strerror(-13)



@pytest.mark.parametrize("kw,code", [
    (dict(x=0), -1), (dict(w=0), -1), (dict(out=0), -1), (dict(M=0), -2), (dict(N=12), -2), (dict(K=20), -2),
    (dict(dtype=2), -6), (dict(x=0x20000004), -5), (dict(bias=0x60000002), -5),
    (dict(out=0x20000000 + 64), -11), (dict(resid=0x70000000 + 128), -11),
])
def test_gemm_argument_errors(gla, kw, code):
    a = dict(x=0x20000000, w=0x40000000, bias=0x60000000, resid=0, out=0x70000000, M=100, N=64, K=64,
             dtype=gla.F16)
    a.update(kw)
    vp = ctypes.c_void_p
    assert gla._lib.gtr_gemm_fwd(vp(a["x"]), vp(a["w"]), vp(a["bias"]), vp(a["resid"]), vp(a["out"]),
                                 ctypes.c_longlong(a["M"]), a["N"], a["K"], a["dtype"], None) == code


# ---------------------------------------------------------------- backward pass

@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(dla=0), -1), (dict(B=0), -2), (dict(dk=128), -3), (dict(dir=4), -4),
    (dict(dq=Q + 8), -5), (dict(dtype=3), -6), (dict(ws=0), -8), (dict(wsb=16), -8),
    (dict(dq=K), -11), (dict(dv=0xA0000000 + 256), -11), (dict(dla=LA), -11),
    (dict(ws=0xB0000000), -11), (dict(ws=FS), -11), (dict(ws=Q), -11),  # workspace on dk, dS_final, q
])
def test_backward_argument_errors(gla, kw, code):
    a = dict(q=Q, k=K, v=V, la=LA, dO=OUT, dsf=FS, dq=0xA0000000, dk=0xB0000000, dv=0xC0000000,
             dla=0xD0000000, B=1, H=2, gh=4, gw=4, dk_=64, dv_=64, dir=0, dtype=gla.F16, ws=WS, wsb=1 << 30)
    if "dk" in kw and isinstance(kw["dk"], int) and kw["dk"] == 128:
        kw = dict(dk_=128)
    a.update(kw)
    vp = ctypes.c_void_p
    assert gla._lib.gtr_gla_bwd(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["la"]), vp(a["dO"]), vp(a["dsf"]),
                                vp(a["dq"]), vp(a["dk"]), vp(a["dv"]), vp(a["dla"]), a["B"], a["H"], a["gh"],
                                a["gw"], a["dk_"], a["dv_"], a["dir"], a["dtype"], vp(a["ws"]), a["wsb"],
                                None) == code


def test_backward_workspace_size(gla):
    assert gla.gtr_gla_bwd_workspace_size(1, 6, 40, 40) > 0
    assert gla.gtr_gla_bwd_workspace_size(1, 6, 40, 40, 128, 128) == 0
