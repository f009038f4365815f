"""The C-ABI library loads and exports every function include/*.h declares; host-only entry
points validate their arguments without touching a GPU."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from resolution_vit_vision_b200 import build as b
    if not os.path.exists(b.LIB):
        b.build()
    from resolution_vit_vision_b200 import native as nv
    return nv.lib()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, re.M):
            names.add(m.group(1))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"vit_encode", "mrope_index", "vit_weights_create", "vit_op_gemm", "vit_op_attention"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_status_strings(lib):
    from resolution_vit_vision_b200 import native as nv
    for code in range(10):
        assert lib.vit_status_string(code)
    assert b"unknown" in lib.vit_status_string(99)


def test_encode_sizes_host_only(lib):
    from resolution_vit_vision_b200 import native as nv
    from resolution_vit_vision_b200 import synthetic as syn
    for wl in syn.WORKLOADS.values():
        P, M = nv.encode_sizes(wl.grids)
        assert P == syn.n_patches(wl.grids) and M == P // 4
    assert nv.encode_sizes([(1, 32, 32)]) == (1024, 256)
    assert nv.encode_sizes([(1, 48, 48)]) == (2304, 576)
    for bad, code in [([(1, 7, 8)], nv.VIT_ERR_GRID), ([(0, 8, 8)], nv.VIT_ERR_GRID),
                      ([(1, 8, 8194)], nv.VIT_ERR_LIMIT)]:
        with pytest.raises(nv.VitError) as e:
            nv.encode_sizes(bad)
        assert e.value.code == code


def test_weights_create_rejects_bad_descriptors_before_cuda(lib):
    from resolution_vit_vision_b200 import native as nv
    d = nv.VitWeightsDesc()
    h = ctypes.c_void_p()
    assert lib.vit_weights_create(None, ctypes.byref(h)) == nv.VIT_ERR_ARG
    d.depth, d.out_dim, d.ln_eps, d.patch_order = 0, 1536, 1e-6, 0
    assert lib.vit_weights_create(ctypes.byref(d), ctypes.byref(h)) == nv.VIT_ERR_ARG
    d.depth, d.out_dim = 1, 1537
    assert lib.vit_weights_create(ctypes.byref(d), ctypes.byref(h)) == nv.VIT_ERR_ARG
    layers = (nv.VitLayerW * 1)()
    d.out_dim, d.layers = 1536, layers
    assert lib.vit_weights_create(ctypes.byref(d), ctypes.byref(h)) == nv.VIT_ERR_ARG   # null weights
    fake = 0x10000
    for k in ("pe_w", "lnq_w", "m0_w", "m2_w"):
        setattr(d, k, fake)
    for k in ("ln1_w", "qkv_w", "proj_w", "ln2_w", "fc1_w", "fc2_w"):
        setattr(layers[0], k, fake)
    layers[0].qkv_w = fake + 2
    assert lib.vit_weights_create(ctypes.byref(d), ctypes.byref(h)) == nv.VIT_ERR_ALIGN
    layers[0].qkv_w = fake
    for bad_window in (-2, 7, 8194):                      # windows: even, 2 .. max side
        d.window = bad_window
        assert lib.vit_weights_create(ctypes.byref(d), ctypes.byref(h)) == nv.VIT_ERR_ARG


def test_window_ops_reject_bad_arguments_before_cuda(lib):
    from resolution_vit_vision_b200 import native as nv
    g = np.array([[1, 8, 8]], np.int32)
    p = ctypes.c_void_p(0x10000)
    n = ctypes.c_int(-1)
    assert lib.vit_op_window_attention(p, 64, p, 0, p, None, None) == nv.VIT_ERR_ARG       # no windows
    assert lib.vit_op_window_attention(p, 64, p, 17, p, None, None) == nv.VIT_ERR_ARG      # > P / 4
    assert lib.vit_op_window_attention(p, 64, None, 1, p, None, None) == nv.VIT_ERR_ARG
    assert lib.vit_op_window_attention(ctypes.c_void_p(0x10002), 64, p, 1, p, None, None) == nv.VIT_ERR_ALIGN
    assert lib.vit_op_window_attention(p, (1 << 21) + 4, p, 1, p, None, None) == nv.VIT_ERR_LIMIT
    assert lib.vit_op_window_positions(nv._gp(g), 1, 0, 5, p, p, p, p, ctypes.byref(n), None) == nv.VIT_ERR_ARG
    assert lib.vit_op_window_positions(nv._gp(g), 1, 2, 8, p, p, p, p, ctypes.byref(n), None) == nv.VIT_ERR_ARG
    assert lib.vit_op_window_positions(nv._gp(g), 1, 0, 8, p, p, p, p, None, None) == nv.VIT_ERR_ARG
    bad = np.array([[1, 7, 8]], np.int32)
    assert lib.vit_op_window_positions(nv._gp(bad), 1, 0, 8, p, p, p, p, ctypes.byref(n), None) == nv.VIT_ERR_GRID
    assert n.value == -1                                   # nothing written on an error
    assert lib.vit_op_gather_rows(p, p, p, 4, 2352 + 8, None) == nv.VIT_ERR_ALIGN


def test_mrope_rejects_bad_arguments(lib):
    from resolution_vit_vision_b200 import native as nv
    g = np.array([[1, 3, 4]], np.int32)
    assert lib.mrope_index(None, 5, None, 0, None, None, None, None) == nv.VIT_ERR_ARG
    # grid values are checked on the device and only for consumed grids: no host-side refusal
    assert lib.mrope_index(ctypes.c_void_p(16), (1 << 30) + 1, nv._gp(g), 1, ctypes.c_void_p(16), None, None,
                           None) == nv.VIT_ERR_LIMIT
    assert lib.mrope_index(ctypes.c_void_p(16), 5, None, 1, ctypes.c_void_p(16), None, None, None) == nv.VIT_ERR_ARG
    assert lib.mrope_index(ctypes.c_void_p(16), -1, None, 0, ctypes.c_void_p(16), None, None, None) == nv.VIT_ERR_ARG


def test_decoder_steps_reject_bad_arguments_before_cuda(lib):
    from resolution_vit_vision_b200 import native as nv
    p = ctypes.c_void_p(0x10000)
    sec = np.array([16, 24, 24], np.int32)
    bad_sec = np.array([16, 24, 23], np.int32)
    ok = sec.ctypes.data_as(nv.c_i32p)
    assert lib.mrope_apply(p, 28, p, 4, 128, p, 10, 1e6, bad_sec.ctypes.data_as(nv.c_i32p), None) == nv.VIT_ERR_ARG
    assert lib.mrope_apply(p, 28, p, 4, 120, p, 10, 1e6, ok, None) == nv.VIT_ERR_ARG           # not a multiple of 16
    assert lib.mrope_apply(None, 28, p, 4, 128, p, 10, 1e6, ok, None) == nv.VIT_ERR_ARG        # q missing
    assert lib.mrope_apply(p, 28, p, 4, 128, None, 10, 1e6, ok, None) == nv.VIT_ERR_ARG        # positions missing
    assert lib.mrope_apply(ctypes.c_void_p(0x10008), 28, p, 4, 128, p, 10, 1e6, ok, None) == nv.VIT_ERR_ALIGN
    assert lib.scatter_vision_tokens(p, 10, p, 100, 12, p, 2, p, None, None) == nv.VIT_ERR_ARG  # dim % 8
    assert lib.scatter_vision_tokens(p, (1 << 18) + 1, p, 100, 64, p, 2, p, None, None) == nv.VIT_ERR_ARG
    assert lib.scatter_vision_tokens(p, 10, p, 100, 64, None, 2, p, None, None) == nv.VIT_ERR_ARG
    assert lib.scatter_vision_tokens(p, 10, ctypes.c_void_p(0x10004), 100, 64, p, 2, p, None, None) == nv.VIT_ERR_ALIGN


def test_fp8_entry_points_reject_bad_arguments_before_cuda(lib):
    from resolution_vit_vision_b200 import native as nv
    p = ctypes.c_void_p(0x10000)
    # vit_quantize_fp8: width a multiple of 8 in 8..65536, pointers present and 16-byte aligned
    assert lib.vit_quantize_fp8(p, 4, 12, p, p, None) == nv.VIT_ERR_ARG
    assert lib.vit_quantize_fp8(p, 4, 65544, p, p, None) == nv.VIT_ERR_ARG
    assert lib.vit_quantize_fp8(None, 4, 64, p, p, None) == nv.VIT_ERR_ARG
    assert lib.vit_quantize_fp8(p, -1, 64, p, p, None) == nv.VIT_ERR_ARG
    assert lib.vit_quantize_fp8(ctypes.c_void_p(0x10008), 4, 64, p, p, None) == nv.VIT_ERR_ALIGN
    assert lib.vit_quantize_fp8(p, 0, 64, None, None, None) == nv.VIT_OK       # nothing to do
    # vit_op_gemm_fp8: scales required, K a multiple of 16, QKV_ROPE only for N = 3840
    args = dict(A=p, sa=p, B=p, sb=p, bias=None, C=p, M=64, N=256, K=128, epi=nv.EPI_ADD_F32)

    def call(**kw):
        a = dict(args, **kw)
        return lib.vit_op_gemm_fp8(a["A"], a["sa"], a["B"], a["sb"], a["bias"], a["C"], a["M"], a["N"], a["K"],
                                   a["epi"], None, None, None, None)
    assert call(sa=None) == nv.VIT_ERR_ARG
    assert call(sb=None) == nv.VIT_ERR_ARG
    assert call(K=120) == nv.VIT_ERR_ARG
    assert call(N=250) == nv.VIT_ERR_ARG
    assert call(epi=nv.EPI_QKV_ROPE) == nv.VIT_ERR_ARG
    assert call(epi=9) == nv.VIT_ERR_ARG
    assert call(sb=ctypes.c_void_p(0x10004)) == nv.VIT_ERR_ALIGN
    assert call(M=(1 << 30) + 1) == nv.VIT_ERR_LIMIT
    # vit_op_layernorm_fp8
    assert lib.vit_op_layernorm_fp8(p, p, None, p, None, 4, 1e-6, None) == nv.VIT_ERR_ARG
    assert lib.vit_op_layernorm_fp8(p, p, None, p, p, 4, 0.0, None) == nv.VIT_ERR_ARG
    assert lib.vit_op_layernorm_fp8(ctypes.c_void_p(0x10008), p, None, p, p, 4, 1e-6, None) == nv.VIT_ERR_ALIGN
    # vit_op_exp2_fma
    assert lib.vit_op_exp2_fma(None, p, 4, None) == nv.VIT_ERR_ARG
    assert lib.vit_op_exp2_fma(p, p, -1, None) == nv.VIT_ERR_ARG
    assert lib.vit_op_exp2_fma(None, None, 0, None) == nv.VIT_OK


def test_weights_create_validates_fp8_layers_before_cuda(lib):
    # an fp8 descriptor with a missing code pointer is refused before any device call
    from resolution_vit_vision_b200 import native as nv
    p = 0x10000
    layers = (nv.VitLayerW * 1)()
    for k in ("ln1_w", "ln2_w"):
        setattr(layers[0], k, p)
    q8 = (nv.VitLayerFp8 * 1)()
    for f, _ in nv.VitLayerFp8._fields_:
        setattr(q8[0], f, p)
    d = nv.VitWeightsDesc()
    d.depth, d.out_dim, d.ln_eps, d.patch_order = 1, 1536, 1e-6, 0
    d.pe_w = d.lnq_w = d.m0_w = d.m2_w = p
    d.layers = layers
    d.fp8_layers = q8
    h = ctypes.c_void_p()
    q8[0].fc2_q = None
    assert lib.vit_weights_create(ctypes.byref(d), ctypes.byref(h)) == nv.VIT_ERR_ARG
    q8[0].fc2_q = p + 8
    assert lib.vit_weights_create(ctypes.byref(d), ctypes.byref(h)) == nv.VIT_ERR_ALIGN
    d.fp8_layers = None                                  # bf16 tower: the linears are then required
    assert lib.vit_weights_create(ctypes.byref(d), ctypes.byref(h)) == nv.VIT_ERR_ARG
