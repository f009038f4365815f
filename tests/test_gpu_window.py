"""Windowed attention (the Qwen2.5-VL tower) on a B200, through the C ABI, against the fp64 oracle.

"Qwen2.5-VL-7B-Instruct" (inference-research model record), architecture note: windows of 112 px
(8 x 8 patches), full attention at blocks 7, 15, 23 and 31. The CUDA path keeps the rows in window
order (a permutation of the packed patches); the oracle builds the windows as index sets in the
packed order. Kernel parity: window-order positions / source rows / merge rows (bit-exact), the
row gather (bit-exact), the packed window-attention kernel (attention bound). Encoder parity: the
whole windowed tower at the encoder bar, small ragged cases and the mixed batch at full depth.
"""
import numpy as np
import pytest
import torch

from oracle import vit_oracle as vo
from resolution_vit_vision_b200 import native as nv
from resolution_vit_vision_b200 import synthetic as syn
from tests.parity import assert_attention_close, assert_encoder_close, bf16_bits_to_torch, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
FULL = nv.QWEN25_FULL_BLOCKS

RAGGED = [(1, 20, 12), (2, 6, 10), (1, 2, 2), (1, 18, 4), (1, 16, 16)]


def _window_cu(grids, order, window):
    return np.concatenate([[0], np.cumsum([len(g) for g in vo.window_groups(grids, order, window)])])


# ------------------------------------------------------------------ positions, gather
@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("window", [8, 4, 16])
def test_window_positions(order, window):
    grids = RAGGED
    pos, mr, src, tab = (to_np(t).astype(np.int64) for t in nv.op_window_positions(grids, order, window))
    groups = vo.window_groups(grids, order, window)
    cu = _window_cu(grids, order, window)
    np.testing.assert_array_equal(tab[:, 0], cu[:-1])      # the window table: first row, rows
    np.testing.assert_array_equal(tab[:, 1], np.diff(cu))
    for i, g in enumerate(groups):      # window i is the contiguous run cu[i] .. cu[i + 1]
        assert sorted(src[cu[i]:cu[i + 1]].tolist()) == g.tolist()
    if order == 0:
        np.testing.assert_array_equal(src, np.concatenate(groups))
    hp, wp = vo.patch_positions(grids, order)
    np.testing.assert_array_equal(pos >> 16, hp[src])
    np.testing.assert_array_equal(pos & 0xFFFF, wp[src])
    block_of = np.arange(src.size) if order == 0 else np.argsort(vo.merge_groups(grids, 1).reshape(-1))
    np.testing.assert_array_equal(mr, block_of[src])
    # four consecutive window-order rows are one merge group, in (dh, dw) order
    q = mr.reshape(-1, 4)
    assert (q[:, 0] % 4 == 0).all() and (q - q[:, :1] == np.arange(4)).all()


def test_gather_rows_bit_exact():
    P = 777
    src = bf16_bits_to_torch(syn.make_matrix((P, 1176), 71, 1.0))
    perm = torch.from_numpy(np.random.Generator(np.random.PCG64(72)).permutation(P).astype(np.int32)).to(DEV)
    dst = torch.empty_like(src)
    nv.op_gather_rows(src, perm, dst)
    torch.cuda.synchronize()
    assert torch.equal(dst.view(torch.int16), src[perm.long()].view(torch.int16))


# ------------------------------------------------------------------ the window kernel
WIN_CASES = [
    ([(1, 8, 8)], 8),                    # one window: the tile's second half is empty
    ([(1, 20, 12)], 8),                  # border windows 32 and 16 rows
    (RAGGED, 8),
    (RAGGED, 4),
    (RAGGED, 2),
    ([(1, 14, 22), (1, 2, 30)], 6),
]


@pytest.mark.parametrize("grids,window", WIN_CASES)
def test_window_attention_kernel(grids, window):
    P = syn.n_patches(grids)
    cu = _window_cu(grids, 0, window)
    qkv = syn.make_matrix((P, 3840), 73 + P, 1.0)
    out = torch.full((P, 1280), float("nan"), dtype=torch.bfloat16, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    tab = nv.op_window_positions(grids, 0, window)[3]
    nv.op_window_attention(bf16_bits_to_torch(qkv), tab, out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x = vo._f64(qkv)
    q, k, v = (x[:, i * 1280:(i + 1) * 1280].reshape(P, 16, 80) for i in range(3))
    segs = [(int(cu[i]), int(cu[i + 1] - cu[i]), 0, 0) for i in range(len(cu) - 1)]
    ref = vo.varlen_attention(q, k, v, segs)
    assert_attention_close(to_np(out), ref, np.abs(v).max(), f"window attention {grids} w{window}")


def test_window_attention_kernel_full_mixed_batch_peaked():
    # the mixed 8-image batch (17696 rows, 279 windows, 140 tiles x 16 heads: several items per
    # CTA through the whole 3-stage ring) with sharply peaked scores
    grids = syn.WORKLOADS["mixed8"].grids
    P = syn.n_patches(grids)
    cu = _window_cu(grids, 0, 8)
    assert len(cu) - 1 == 279
    qkv = syn.make_matrix((P, 3840), 74, 4.0)
    out = torch.empty((P, 1280), dtype=torch.bfloat16, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    tab = nv.op_window_positions(grids, 0, 8)[3]
    nv.op_window_attention(bf16_bits_to_torch(qkv), tab, out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x = vo._f64(qkv)
    q, k, v = (x[:, i * 1280:(i + 1) * 1280].reshape(P, 16, 80) for i in range(3))
    segs = [(int(cu[i]), int(cu[i + 1] - cu[i]), 0, 0) for i in range(len(cu) - 1)]
    assert_attention_close(to_np(out), vo.varlen_attention(q, k, v, segs), np.abs(v).max(), "mixed8 windows")


# ------------------------------------------------------------------ the windowed encoder
def _encode(grids, depth, out_dim, seed, order, window, full, affine=True, patches=None, wts=None):
    wts = wts if wts is not None else syn.make_weights(depth, out_dim, seed, affine=affine)
    patches = patches if patches is not None else syn.make_patches(grids, seed)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), out_dim, 1e-6, order, window=window, full_blocks=full)
    out = enc.encode(bf16_bits_to_torch(patches), grids)
    assert enc.device_status() == 0
    return to_np(out), wts, patches, enc


@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("window", [8, 4, 16])
def test_windowed_encoder_ragged(order, window):
    grids = RAGGED
    got, wts, patches, _ = _encode(grids, 2, 1536, 75, order, window, (1,))
    ref = vo.vit_encode(patches, grids, wts, patch_order=order, window=window, full_blocks=(1,))
    assert_encoder_close(got, ref, f"windowed order {order} window {window}")


def test_windowed_encoder_all_full_blocks_equals_plain_tower():
    # every block full-attention: the window-order layout alone must not change the tokens beyond
    # rounding (same kernels, rows permuted)
    grids = [(1, 20, 12), (1, 6, 10)]
    wts = syn.make_weights(2, 1536, 76)
    patches = syn.make_patches(grids, 76)
    a, *_ = _encode(grids, 2, 1536, 76, 0, 8, (0, 1), wts=wts, patches=patches)
    b, *_ = _encode(grids, 2, 1536, 76, 0, 0, (), wts=wts, patches=patches)
    ref = vo.vit_encode(patches, grids, wts)
    assert_encoder_close(a, ref, "all full blocks, window layout")
    assert_encoder_close(b, ref, "plain tower")


def test_windowed_encoder_graph_replay_and_host():
    grids = [(1, 20, 12), (2, 6, 10)]
    got, wts, patches, enc = _encode(grids, 2, 1536, 77, 0, 8, (1,))
    enc.graph_enable(True)
    p = bf16_bits_to_torch(patches)
    out = torch.empty((got.shape[0], 1536), dtype=torch.bfloat16, device=DEV)
    enc.encode(p, grids, out=out)
    enc.encode(p, grids, out=out)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(out), got)
    enc.graph_enable(False)
    hp = torch.from_numpy(patches.copy()).view(torch.bfloat16).pin_memory()
    ho = torch.empty((got.shape[0], 1536), dtype=torch.bfloat16).pin_memory()
    enc.encode_host(hp, grids, ho)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ho.float().numpy(), got)


def test_noalloc_rejects_windowed_handle():
    wts = syn.make_weights(1, 1536, 78)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), 1536, window=8)
    g = np.array([[1, 8, 8]], np.int32)
    p = torch.zeros((64, 1176), dtype=torch.bfloat16, device=DEV)
    out = torch.zeros((16, 1536), dtype=torch.bfloat16, device=DEV)
    rc = nv.lib().vit_encode_noalloc(p.data_ptr(), nv._gp(g), 1, enc.handle, out.data_ptr(), None,
                                     torch.cuda.current_stream().cuda_stream)
    assert rc == nv.VIT_ERR_ARG


@pytest.mark.slow
def test_windowed_mixed8_full_depth_sampled_images():
    # the Qwen2.5-VL tower shape on the mixed batch, depth 32, full attention at 7, 15, 23, 31
    wl = syn.WORKLOADS["mixed8"]
    got, wts, patches, _ = _encode(wl.grids, wl.depth, wl.out_dim, wl.seed, 0, 8, FULL, affine=False)
    assert got.shape == (4424, 3584)
    starts = np.cumsum([0] + [t * h * w for t, h, w in wl.grids])
    for i in (5, 2):
        ref = vo.vit_encode(patches[starts[i]:starts[i + 1]], [wl.grids[i]], wts, window=8, full_blocks=FULL)
        assert_encoder_close(got[starts[i] // 4:starts[i + 1] // 4], ref, f"windowed mixed8 image {i}")
    assert np.isfinite(got).all()


@pytest.mark.slow
def test_windowed_hires_1792():
    # 16384 patches, 256 windows: four blocks with a full-attention block last, whole image
    wl = syn.WORKLOADS["hires_1792"]
    wts = syn.make_weights(4, wl.out_dim, wl.seed)
    got, _, patches, _ = _encode(wl.grids, 4, wl.out_dim, wl.seed, 0, 8, (3,), wts=wts)
    ref = vo.vit_encode(patches, wl.grids, wts, window=8, full_blocks=(3,))
    assert_encoder_close(got, ref, "windowed 1792^2 depth 4")
