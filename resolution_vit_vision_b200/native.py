"""ctypes binding of ``libvit_b200.so`` (the C ABI in ``include/vit.h`` and ``include/vit_ops.h``).

Argument marshalling only: torch supplies device memory and streams; every step of the encoder
runs in the library's CUDA kernels. There is no fallback: if the library is missing or the
device is not an sm_100 GPU, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import numpy as np
import torch

from . import synthetic as syn

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvit_b200.so")

VIT_OK, VIT_ERR_ARG, VIT_ERR_GRID, VIT_ERR_ALIGN, VIT_ERR_NOMEM, VIT_ERR_CUDA, VIT_ERR_TOKENS, \
    VIT_ERR_TIMEOUT, VIT_ERR_UNSUPPORTED, VIT_ERR_LIMIT = range(10)
EPI_STORE_F32, EPI_ADD_F32, EPI_STORE_BF16, EPI_GELU_BF16, EPI_QKV_ROPE = range(5)

c_void_p, c_int, c_int64, c_float = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
c_i32p = ctypes.POINTER(ctypes.c_int32)


class VitLayerW(ctypes.Structure):
    _fields_ = [(k, c_void_p) for k in syn.LAYER_KEYS]


FP8_LINEARS = ("qkv", "proj", "fc1", "fc2")


class VitLayerFp8(ctypes.Structure):
    _fields_ = [(f"{k}_{x}", c_void_p) for k in FP8_LINEARS for x in ("q", "s")]


class VitWeightsDesc(ctypes.Structure):
    _fields_ = [("depth", c_int), ("out_dim", c_int), ("ln_eps", c_float), ("patch_order", c_int),
                ("pe_w", c_void_p), ("pe_b", c_void_p), ("layers", ctypes.POINTER(VitLayerW)),
                ("lnq_w", c_void_p), ("lnq_b", c_void_p), ("m0_w", c_void_p), ("m0_b", c_void_p),
                ("m2_w", c_void_p), ("m2_b", c_void_p), ("window", c_int),
                ("full_attention", ctypes.POINTER(ctypes.c_uint8)),
                ("fp8_layers", ctypes.POINTER(VitLayerFp8))]

# The Qwen2.5-VL tower's full-attention blocks (0-based) when windows are on
QWEN25_FULL_BLOCKS = (7, 15, 23, 31)


_SIGS = {
    "vit_status_string": (ctypes.c_char_p, [c_int]),
    "vit_encode_sizes": (c_int, [c_i32p, c_int, ctypes.POINTER(c_int64), ctypes.POINTER(c_int64)]),
    "vit_weights_create": (c_int, [ctypes.POINTER(VitWeightsDesc), ctypes.POINTER(c_void_p)]),
    "vit_weights_destroy": (None, [c_void_p]),
    "vit_reserve": (c_int, [c_void_p, c_int64]),
    "vit_encode": (c_int, [c_void_p, c_i32p, c_int, c_void_p, c_void_p, c_void_p]),
    "vit_encode_host": (c_int, [c_void_p, c_i32p, c_int, c_void_p, c_void_p, c_void_p]),
    "vit_encode_noalloc": (c_int, [c_void_p, c_i32p, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "mrope_index": (c_int, [c_void_p, c_int64, c_i32p, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "vit_device_status": (c_int, [c_void_p, c_void_p, c_i32p]),
    "vit_launch_count": (c_int64, [c_void_p]),
    "vit_graph_enable": (c_int, [c_void_p, c_int]),
    "vit_profile_enable": (c_int, [c_void_p, c_int]),
    "vit_profile_read": (c_int, [c_void_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(c_int64), c_int]),
    "vit_profile_name": (ctypes.c_char_p, [c_int]),
    "vit_op_gemm": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int, c_int, c_int, c_void_p,
                            c_void_p, c_void_p, c_void_p]),
    "vit_op_rope_table": (c_int, [c_void_p, c_int, c_void_p]),
    "vit_op_positions": (c_int, [c_i32p, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "vit_op_layernorm": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_float, c_void_p, c_void_p]),
    "vit_op_attention": (c_int, [c_void_p, c_int64, c_i32p, c_int, c_void_p, c_void_p, c_void_p]),
    "vit_op_wait_selftest": (c_int, [c_void_p, c_int64, c_void_p]),
    "vit_op_exp2_fma": (c_int, [c_void_p, c_void_p, c_int64, c_void_p]),
    "vit_quantize_fp8": (c_int, [c_void_p, c_int64, c_int, c_void_p, c_void_p, c_void_p]),
    "vit_op_gemm_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int, c_int,
                                c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "vit_op_layernorm_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_float,
                                     c_void_p]),
    "mrope_apply": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_void_p, c_int64, ctypes.c_double, c_i32p,
                            c_void_p]),
    "scatter_vision_tokens": (c_int, [c_void_p, c_int64, c_void_p, c_int64, c_int, c_void_p, c_int64, c_void_p,
                                      c_void_p, c_void_p]),
    "vit_op_window_positions": (c_int, [c_i32p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                        ctypes.POINTER(c_int), c_void_p]),
    "vit_op_gather_rows": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_int, c_void_p]),
    "vit_op_window_attention": (c_int, [c_void_p, c_int64, c_void_p, c_int, c_void_p, c_void_p, c_void_p]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Loads the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m resolution_vit_vision_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


class VitError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {lib().vit_status_string(code).decode()} (status {code})")


def check(rc: int, what: str) -> None:
    if rc != VIT_OK:
        raise VitError(rc, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _grid_arg(grid_thw) -> np.ndarray:
    g = np.ascontiguousarray(np.asarray(grid_thw, dtype=np.int32).reshape(-1, 3))
    return g


def _gp(g: np.ndarray):
    return g.ctypes.data_as(c_i32p)


def encode_sizes(grid_thw):
    g = _grid_arg(grid_thw)
    P, M = c_int64(), c_int64()
    check(lib().vit_encode_sizes(_gp(g), g.shape[0], ctypes.byref(P), ctypes.byref(M)), "vit_encode_sizes")
    return P.value, M.value


# ------------------------------------------------------------------------------------------------
def weights_to_device(w_np: Dict, device="cuda") -> Dict:
    """bf16-bit numpy weights (synthetic.make_weights) -> dict of bf16 CUDA tensors."""
    def t(a):
        if a is None:
            return None
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(device)
    out = {k: t(v) for k, v in w_np.items() if k != "layers"}
    out["layers"] = [{k: t(v) for k, v in L.items()} for L in w_np["layers"]]
    return out


def random_weights_device(depth: int, out_dim: int, seed: int, device="cuda", std: float = 0.02) -> Dict:
    """Same shapes and distribution as synthetic.make_weights (N(0, 0.02) matrices, zero biases,
    unit gamma), drawn on the device with a seeded torch generator (fast, for benchmarking)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)

    def mat(shape):
        return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)

    def zeros(n):
        return torch.zeros(n, device=device, dtype=torch.bfloat16)

    def ones(n):
        return torch.ones(n, device=device, dtype=torch.bfloat16)

    w = {"pe_w": mat((syn.WIDTH, syn.PATCH_K)), "pe_b": None}
    layers = []
    for _ in range(depth):
        L = {}
        for k in syn.LAYER_KEYS:
            shape = syn.LAYER_SHAPES[k]
            L[k] = ones(shape[0]) if k in ("ln1_w", "ln2_w") else (zeros(shape[0]) if len(shape) == 1 else mat(shape))
        layers.append(L)
    w["layers"] = layers
    w["lnq_w"], w["lnq_b"] = ones(syn.WIDTH), zeros(syn.WIDTH)
    w["m0_w"], w["m0_b"] = mat((syn.MERGE_K, syn.MERGE_K)), zeros(syn.MERGE_K)
    w["m2_w"], w["m2_b"] = mat((out_dim, syn.MERGE_K)), zeros(out_dim)
    return w


def quantize_fp8(x: torch.Tensor, stream=None):
    """E4M3 codes (uint8, same shape) and per-row power-of-two scales (fp32 [rows]) of a bf16
    [rows, cols] device tensor, by vit_quantize_fp8."""
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous() and x.dim() == 2
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scales = torch.empty((x.shape[0],), dtype=torch.float32, device=x.device)
    check(lib().vit_quantize_fp8(_ptr(x), x.shape[0], x.shape[1], _ptr(codes), _ptr(scales), _stream(stream)),
          "vit_quantize_fp8")
    return codes, scales


def fp8_layers_device(weights: Dict, stream=None):
    """Per layer {"qkv": (codes, scales), "proj": ..., "fc1": ..., "fc2": ...} of the device bf16
    weights' four block linears, quantised on the device."""
    return [{k: quantize_fp8(L[f"{k}_w"], stream) for k in FP8_LINEARS} for L in weights["layers"]]


class VisionEncoder:
    """A validated weight view (vit_handle) and its workspace; ``encode`` runs vit_encode.
    window > 0 makes the windowed (Qwen2.5-VL) tower: blocks in ``full_blocks`` attend over the
    whole frame, the others inside window x window patches. fp8: per layer the E4M3 codes and
    scales of the four block linears (``fp8_layers_device``): the fp8 tower."""

    def __init__(self, weights: Dict, out_dim: int, eps: float = 1e-6, patch_order: int = 0, window: int = 0,
                 full_blocks: Sequence[int] = (), fp8=None):
        self.weights = weights          # keeps the device tensors alive
        self.out_dim = out_dim
        depth = len(weights["layers"])
        self._layers = (VitLayerW * depth)()
        for i, L in enumerate(weights["layers"]):
            for k in syn.LAYER_KEYS:
                setattr(self._layers[i], k, _ptr(L.get(k)))
        d = VitWeightsDesc()
        d.depth, d.out_dim, d.ln_eps, d.patch_order = depth, out_dim, eps, patch_order
        d.pe_w, d.pe_b = _ptr(weights["pe_w"]), _ptr(weights.get("pe_b"))
        d.layers = self._layers
        for k in ("lnq_w", "lnq_b", "m0_w", "m0_b", "m2_w", "m2_b"):
            setattr(d, k, _ptr(weights.get(k)))
        d.window = int(window)
        self._full = (ctypes.c_uint8 * depth)(*[1 if l in set(full_blocks) else 0 for l in range(depth)])
        d.full_attention = ctypes.cast(self._full, ctypes.POINTER(ctypes.c_uint8))
        self._fp8 = fp8                 # keeps the codes and scales alive
        if fp8 is not None:
            self._fp8_layers = (VitLayerFp8 * depth)()
            for i, Lq in enumerate(fp8):
                for k in FP8_LINEARS:
                    setattr(self._fp8_layers[i], f"{k}_q", _ptr(Lq[k][0]))
                    setattr(self._fp8_layers[i], f"{k}_s", _ptr(Lq[k][1]))
            d.fp8_layers = self._fp8_layers
        self._desc = d
        h = c_void_p()
        check(lib().vit_weights_create(ctypes.byref(d), ctypes.byref(h)), "vit_weights_create")
        self._h = h

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().vit_weights_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def reserve(self, max_patches: int):
        check(lib().vit_reserve(self._h, int(max_patches)), "vit_reserve")

    def encode(self, patches: torch.Tensor, grid_thw, out: Optional[torch.Tensor] = None, stream=None):
        g = _grid_arg(grid_thw)
        P, M = encode_sizes(g)
        assert patches.dtype == torch.bfloat16 and patches.is_cuda and patches.is_contiguous()
        assert patches.shape == (P, syn.PATCH_K), (patches.shape, P)
        if out is None:
            out = torch.empty((M, self.out_dim), dtype=torch.bfloat16, device=patches.device)
        check(lib().vit_encode(_ptr(patches), _gp(g), g.shape[0], self._h, _ptr(out), _stream(stream)), "vit_encode")
        return out

    def encode_host(self, patches_host: torch.Tensor, grid_thw, out_host: torch.Tensor, stream=None):
        g = _grid_arg(grid_thw)
        check(lib().vit_encode_host(_ptr(patches_host), _gp(g), g.shape[0], self._h, _ptr(out_host),
                                    _stream(stream)), "vit_encode_host")
        return out_host

    def device_status(self, stream=None) -> int:
        v = ctypes.c_int32()
        check(lib().vit_device_status(self._h, _stream(stream), ctypes.byref(v)), "vit_device_status")
        return v.value

    def graph_enable(self, on: bool = True):
        check(lib().vit_graph_enable(self._h, 1 if on else 0), "vit_graph_enable")

    def launch_count(self) -> int:
        return int(lib().vit_launch_count(self._h))

    def profile_enable(self, on: bool = True):
        check(lib().vit_profile_enable(self._h, 1 if on else 0), "vit_profile_enable")

    def profile_read(self) -> Dict[str, Dict[str, float]]:
        n = 16
        ms = (ctypes.c_double * n)()
        cnt = (c_int64 * n)()
        k = lib().vit_profile_read(self._h, ms, cnt, n)
        return {lib().vit_profile_name(i).decode(): {"ms": ms[i], "launches": cnt[i]} for i in range(k)}


def mrope_index(input_ids: torch.Tensor, grid_thw, out=None, delta=None, status=None, stream=None):
    """3-D M-RoPE ids [3, L] int32 and delta [1] int32 (device tensors)."""
    assert input_ids.dtype == torch.int32 and input_ids.is_cuda
    g = _grid_arg(grid_thw) if grid_thw is not None else np.zeros((0, 3), np.int32)
    L = input_ids.numel()
    if out is None:
        out = torch.empty((3, L), dtype=torch.int32, device=input_ids.device)
    if delta is None:
        delta = torch.empty((1,), dtype=torch.int32, device=input_ids.device)
    check(lib().mrope_index(_ptr(input_ids), L, _gp(g), g.shape[0], _ptr(out), _ptr(delta), _ptr(status),
                            _stream(stream)), "mrope_index")
    return out, delta


# ------------------------------------------------------------------------------------------------
# kernel-level ops (include/vit_ops.h)
def op_gemm(A, B, bias, C, epilogue, pos=None, rope_cs=None, status=None, stream=None):
    M, K = A.shape
    N = B.shape[0]
    check(lib().vit_op_gemm(_ptr(A), _ptr(B), _ptr(bias), _ptr(C), M, N, K, epilogue, _ptr(pos), _ptr(rope_cs),
                            _ptr(status), _stream(stream)), "vit_op_gemm")
    return C


def op_rope_table(n_pos: int, device="cuda", stream=None):
    cs = torch.empty((n_pos, 20, 2), dtype=torch.float32, device=device)
    check(lib().vit_op_rope_table(_ptr(cs), n_pos, _stream(stream)), "vit_op_rope_table")
    return cs


def op_positions(grid_thw, patch_order: int, device="cuda", stream=None):
    g = _grid_arg(grid_thw)
    P, _ = encode_sizes(g)
    pos = torch.empty(P, dtype=torch.int32, device=device)
    mr = torch.empty(P, dtype=torch.int32, device=device)
    check(lib().vit_op_positions(_gp(g), g.shape[0], patch_order, _ptr(pos), _ptr(mr), _stream(stream)),
          "vit_op_positions")
    return pos, mr


def op_layernorm(X, gamma, beta, Y, eps=1e-6, out_row=None, stream=None):
    check(lib().vit_op_layernorm(_ptr(X), _ptr(gamma), _ptr(beta), _ptr(Y), X.shape[0], eps, _ptr(out_row),
                                 _stream(stream)), "vit_op_layernorm")
    return Y


def op_attention(qkv, cu_seqlens: Sequence[int], out, status=None, stream=None):
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    check(lib().vit_op_attention(_ptr(qkv), qkv.shape[0], cu.ctypes.data_as(c_i32p), cu.shape[0] - 1, _ptr(out),
                                 _ptr(status), _stream(stream)), "vit_op_attention")
    return out


def op_gemm_fp8(A, a_scale, B, b_scale, bias, C, epilogue, pos=None, rope_cs=None, status=None, stream=None):
    M, K = A.shape
    N = B.shape[0]
    check(lib().vit_op_gemm_fp8(_ptr(A), _ptr(a_scale), _ptr(B), _ptr(b_scale), _ptr(bias), _ptr(C), M, N, K,
                                epilogue, _ptr(pos), _ptr(rope_cs), _ptr(status), _stream(stream)), "vit_op_gemm_fp8")
    return C


def op_layernorm_fp8(X, gamma, beta, eps=1e-6, stream=None):
    rows = X.shape[0]
    codes = torch.empty((rows, syn.WIDTH), dtype=torch.uint8, device=X.device)
    scales = torch.empty((rows,), dtype=torch.float32, device=X.device)
    check(lib().vit_op_layernorm_fp8(_ptr(X), _ptr(gamma), _ptr(beta), _ptr(codes), _ptr(scales), rows, eps,
                                     _stream(stream)), "vit_op_layernorm_fp8")
    return codes, scales


def op_exp2_fma(x: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The attention softmax's FMA-pipe exponential 2^x, elementwise on fp32 device tensors."""
    assert x.dtype == torch.float32 and x.is_cuda and x.is_contiguous()
    y = torch.empty_like(x) if y is None else y
    check(lib().vit_op_exp2_fma(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "vit_op_exp2_fma")
    return y


def op_window_positions(grid_thw, patch_order: int, window: int, device="cuda", stream=None):
    """(pos, merge_row, src_row) of the window-order rows, int32 [P] each, and the window table
    int32 [n_windows, 2] = (first row, rows)."""
    g = _grid_arg(grid_thw)
    P, _ = encode_sizes(g)
    pos, mr, src = (torch.empty(P, dtype=torch.int32, device=device) for _ in range(3))
    tab = torch.empty((P // 4 + 1, 2), dtype=torch.int32, device=device)
    n = c_int(0)
    check(lib().vit_op_window_positions(_gp(g), g.shape[0], patch_order, window, _ptr(pos), _ptr(mr), _ptr(src),
                                        _ptr(tab), ctypes.byref(n), _stream(stream)), "vit_op_window_positions")
    return pos, mr, src, tab[:n.value]


def op_gather_rows(src, src_row, dst, stream=None):
    row_bytes = src.shape[1] * src.element_size()
    check(lib().vit_op_gather_rows(_ptr(src), _ptr(src_row), _ptr(dst), dst.shape[0], row_bytes, _stream(stream)),
          "vit_op_gather_rows")
    return dst


def op_window_attention(qkv, win_table, out, status=None, stream=None):
    """win_table: int32 [n_windows, 2] device (first row, rows), as op_window_positions returns."""
    check(lib().vit_op_window_attention(_ptr(qkv), qkv.shape[0], _ptr(win_table), win_table.shape[0], _ptr(out),
                                        _ptr(status), _stream(stream)), "vit_op_window_attention")
    return out


MROPE_THETA = 1.0e6
MROPE_SECTIONS = (16, 24, 24)


def mrope_apply(q, k, pos, theta: float = MROPE_THETA, sections=MROPE_SECTIONS, stream=None):
    """3-D M-RoPE in place on q [L, heads, head_dim] and k [L, kv_heads, head_dim] (bf16, either may
    be None); pos int32 [3, L] from mrope_index."""
    x = q if q is not None else k
    L, D = x.shape[0], x.shape[2]
    sec = np.ascontiguousarray(np.asarray(sections, dtype=np.int32))
    check(lib().mrope_apply(_ptr(q), 0 if q is None else q.shape[1], _ptr(k), 0 if k is None else k.shape[1], D,
                            _ptr(pos), L, float(theta), sec.ctypes.data_as(c_i32p), _stream(stream)), "mrope_apply")
    return q, k


def scatter_vision_tokens(input_ids, embed_table, vision, out=None, status=None, stream=None):
    """The decoder's input rows: vision tokens at the image / video placeholders, embeddings elsewhere."""
    L, (V, D) = input_ids.shape[0], embed_table.shape
    if out is None:
        out = torch.empty((L, D), dtype=embed_table.dtype, device=embed_table.device)
    n_vis = 0 if vision is None else vision.shape[0]
    check(lib().scatter_vision_tokens(_ptr(input_ids), L, _ptr(embed_table), V, D, _ptr(vision), n_vis, _ptr(out),
                                      _ptr(status), _stream(stream)), "scatter_vision_tokens")
    return out


def op_wait_selftest(status, limit_cycles: int, stream=None):
    check(lib().vit_op_wait_selftest(_ptr(status), int(limit_cycles), _stream(stream)), "vit_op_wait_selftest")
