"""Pins for the oracle's patch embed, 2x2 merge and whole tower (CPU only).

* T7: the patch-embed GEMM on patches flattened (c, t, ph, pw) equals torch's Conv3d with
  kernel = stride = (2, 14, 14) on the image, and, with the two frames identical, the Conv2d with
  the summed temporal kernel ("Qwen2-VL-2B-Instruct -- LiteRT-LM", Conversion notes).
* 2x2 grouping equals torch's pixel_unshuffle(2) (space-to-depth), reordered to (dh, dw, c).
* T8: raster-ordered and block-ordered patches give the same merged tokens (Conversion notes,
  "No GATHER_ND": ordering is irrelevant when every patch keeps its own 2-D rope).
* T3/T4: block-diagonal attention: images are independent and their order only permutes rows.
* T1: printed shapes (tests/golden/page_shapes.json).
* T14: the whole tower against a second float64 restatement in torch built from different
  primitives (conv3d patch embed, masked SDPA, complex-number rope, F.layer_norm, F.gelu).
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import vit_oracle as vo
from resolution_vit_vision_b200 import synthetic as syn

HERE = os.path.dirname(__file__)


def _small_weights(depth, out_dim=64, seed=3, affine=True):
    """Full-width tower weights (the widths are fixed) with a small merger output."""
    return syn.make_weights(depth, out_dim, seed, affine=affine)


def _image_to_patches(img, order):
    """img [3, 2, H, W] -> patches [P, 1176] flattened (c, t, ph, pw), in the given patch order."""
    C, T, H, W = img.shape
    h, w = H // 14, W // 14
    x = img.reshape(C, T, h, 14, w, 14).transpose(2, 4, 0, 1, 3, 5)   # h, w, c, t, ph, pw
    hp, wp = vo.frame_positions(h, w, order)
    return x[hp, wp].reshape(-1, 1176)


# ------------------------------------------------------------------ T7
@pytest.mark.parametrize("order", [0, 1])
def test_patch_embed_is_conv3d(order):
    r = np.random.Generator(np.random.PCG64(21))
    H, W = 4 * 14, 6 * 14
    img = r.uniform(-1, 1, (3, 2, H, W))
    wpe = syn.bf16_bits_to_f64(syn.make_matrix((1280, 1176), 22, 0.02))
    got = vo.patch_embed(_image_to_patches(img, order), wpe)
    ref = F.conv3d(torch.from_numpy(img)[None], torch.from_numpy(wpe).reshape(1280, 3, 2, 14, 14),
                   stride=(2, 14, 14))[0, :, 0]                       # [1280, h, w]
    hp, wp = vo.frame_positions(4, 6, order)
    np.testing.assert_allclose(got, ref.numpy()[:, hp, wp].T, rtol=1e-11, atol=1e-11)


def test_patch_embed_conv3d_to_conv2d_fold():
    r = np.random.Generator(np.random.PCG64(23))
    H, W = 2 * 14, 4 * 14
    frame = r.uniform(-1, 1, (3, H, W))
    img = np.stack([frame, frame], axis=1)                            # a still image, both frames
    wpe = syn.bf16_bits_to_f64(syn.make_matrix((1280, 1176), 24, 0.02))
    got = vo.patch_embed(_image_to_patches(img, 1), wpe)
    k = torch.from_numpy(wpe).reshape(1280, 3, 2, 14, 14)
    ref = F.conv2d(torch.from_numpy(frame)[None], k[:, :, 0] + k[:, :, 1], stride=14)[0]
    np.testing.assert_allclose(got, ref.numpy().reshape(1280, -1).T, rtol=1e-11, atol=1e-11)


# ------------------------------------------------------------------ 2x2 grouping
def test_merge_groups_equal_pixel_unshuffle():
    h, w, C = 6, 8, 5
    r = np.random.Generator(np.random.PCG64(25))
    feat = r.standard_normal((h, w, C))
    for order in (0, 1):
        hp, wp = vo.frame_positions(h, w, order)
        rows = feat[hp, wp]                                           # packed rows in that order
        g = vo.merge_groups([(1, h, w)], order)
        merged = rows[g].reshape(-1, 4 * C)                           # K order (dh, dw, c)
        ref = F.pixel_unshuffle(torch.from_numpy(feat).permute(2, 0, 1)[None], 2)[0]   # [C*4, h/2, w/2]
        ref = ref.reshape(C, 2, 2, h // 2, w // 2).permute(3, 4, 1, 2, 0).reshape(-1, 4 * C)
        np.testing.assert_array_equal(merged, ref.numpy())


# ------------------------------------------------------------------ T8, T3, T4
def test_raster_and_block_order_give_same_tokens():
    grids = [(1, 4, 6), (2, 2, 4)]
    wts = _small_weights(1)
    r = np.random.Generator(np.random.PCG64(26))
    P = syn.n_patches(grids)
    # one set of patches per (frame, h, w); pack it twice
    by_pos = {}
    raw = r.uniform(-1, 1, (P, 1176))
    i = 0
    for gi, (t, h, w) in enumerate(grids):
        for f in range(t):
            for a in range(h):
                for b in range(w):
                    by_pos[(gi, f, a, b)] = raw[i]; i += 1
    packs = {}
    for order in (0, 1):
        rows = []
        for gi, (t, h, w) in enumerate(grids):
            hp, wp = vo.frame_positions(h, w, order)
            for f in range(t):
                rows += [by_pos[(gi, f, a, b)] for a, b in zip(hp, wp)]
        packs[order] = np.array(rows)
    out0 = vo.vit_encode(packs[0], grids, wts, patch_order=0)
    out1 = vo.vit_encode(packs[1], grids, wts, patch_order=1)
    np.testing.assert_allclose(out1, out0, rtol=1e-10, atol=1e-12)


def test_images_independent_and_permutable():
    grids = [(1, 4, 4), (1, 2, 6), (1, 6, 2)]
    wts = _small_weights(2, seed=5)
    patches = syn.bf16_bits_to_f64(syn.make_patches(grids, 7))
    packed = vo.vit_encode(patches, grids, wts)
    starts = np.cumsum([0] + [t * h * w for t, h, w in grids])
    tok = np.cumsum([0] + [t * h * w // 4 for t, h, w in grids])
    # T4: each image alone
    for i, g in enumerate(grids):
        alone = vo.vit_encode(patches[starts[i]:starts[i + 1]], [g], wts)
        np.testing.assert_allclose(packed[tok[i]:tok[i + 1]], alone, rtol=1e-11, atol=1e-13)
    # T3: reversed image order permutes the output blocks
    perm = [2, 0, 1]
    p2 = np.concatenate([patches[starts[i]:starts[i + 1]] for i in perm])
    out2 = vo.vit_encode(p2, [grids[i] for i in perm], wts)
    ref = np.concatenate([packed[tok[i]:tok[i + 1]] for i in perm])
    np.testing.assert_allclose(out2, ref, rtol=1e-11, atol=1e-13)


# ------------------------------------------------------------------ T1
def test_printed_shapes():
    items = json.load(open(os.path.join(HERE, "golden", "page_shapes.json")))["items"]
    for it in items:
        if "image_hw" not in it:
            continue
        H, W = it["image_hw"]
        grid = (1, H // 14, W // 14)
        P = syn.n_patches([grid])
        if "patches" in it:
            assert P == it["patches"], it["cite"]
        if "merged" in it:
            assert P // 4 == it["merged"] == H * W // 784, it["cite"]
    # every workload image follows tokens = pixels / 784 (images are H x W = 14h x 14w)
    for wl in syn.WORKLOADS.values():
        for t, h, w in wl.grids:
            assert (t * h * w) // 4 == t * (14 * h) * (14 * w) // 784


@pytest.mark.parametrize("hw,out_dim", [((448, 448), 3584), ((672, 672), 1536)])
def test_oracle_output_shapes(hw, out_dim):
    H, W = hw
    grids = [(1, H // 14, W // 14)]
    wts = syn.make_weights(1, out_dim, 1)
    patches = syn.make_patches(grids, 1)
    out, hidden = vo.vit_encode(patches, grids, wts, return_hidden=True)
    assert hidden.shape == (H * W // 196, 1280)
    assert out.shape == (H * W // 784, out_dim)
    assert np.isfinite(out).all()


def test_config_table_matches_constants():
    cfg = json.load(open(os.path.join(HERE, "golden", "qwen2vl_config.json")))
    assert (vo.WIDTH, vo.HEADS, vo.HEAD_DIM) == (cfg["vision_embed_dim"], cfg["vision_num_heads"],
                                                 cfg["vision_embed_dim"] // cfg["vision_num_heads"])
    assert syn.MLP == cfg["vision_mlp_ratio"] * cfg["vision_embed_dim"]
    assert syn.PATCH_K == cfg["in_channels"] * cfg["temporal_patch_size"] * cfg["patch_size"] ** 2
    assert syn.MERGE_K == cfg["spatial_merge_size"] ** 2 * cfg["vision_embed_dim"]
    assert (syn.IMAGE_TOKEN, syn.VIDEO_TOKEN, syn.VISION_START, syn.VISION_END) == (
        cfg["image_token_id"], cfg["video_token_id"], cfg["vision_start_token_id"], cfg["vision_end_token_id"])
    assert syn.WORKLOADS["2b_448"].out_dim == cfg["merger_out_2b"]
    assert syn.WORKLOADS["mixed8"].out_dim == cfg["merger_out_7b"]
    assert all(wl.depth == cfg["vision_depth"] for k, wl in syn.WORKLOADS.items() if k != "tiny")


# ------------------------------------------------------------------ T14
def _torch_tower(patches, grids, wts, eps):
    """A second float64 statement of the tower in torch, from different primitives."""
    d = torch.float64
    T = lambda a: torch.from_numpy(syn.bf16_bits_to_f64(a) if a.dtype == np.uint16 else a).to(d)
    g = [tuple(x) for x in grids]
    # patch embed as a Conv3d over each patch seen as a (3, 2, 14, 14) volume
    pe_b = T(wts["pe_b"]) if wts.get("pe_b") is not None else None
    x = F.conv3d(T(patches).reshape(-1, 3, 2, 14, 14), T(wts["pe_w"]).reshape(1280, 3, 2, 14, 14), pe_b).reshape(-1, 1280)
    P = x.shape[0]
    # positions and block-diagonal mask
    hp, wp, seg_id, sid = [], [], [], 0
    for t, h, w in g:
        for _ in range(t):
            bh = torch.arange(h // 2).repeat_interleave(2 * w)                      # bh slowest
            bw = torch.arange(w // 2).repeat_interleave(4).repeat(h // 2)
            dh = torch.tensor([0, 0, 1, 1]).repeat(h * w // 4)
            dw = torch.tensor([0, 1, 0, 1]).repeat(h * w // 4)
            hp.append(2 * bh + dh); wp.append(2 * bw + dw)
            seg_id.append(torch.full((h * w,), sid)); sid += 1
    hp, wp, seg_id = torch.cat(hp), torch.cat(wp), torch.cat(seg_id)
    mask = seg_id[:, None] == seg_id[None, :]
    inv = 1.0 / (10000.0 ** (torch.arange(0, 40, 2, dtype=d) / 40))
    ang = torch.cat([hp.to(d)[:, None] * inv, wp.to(d)[:, None] * inv], 1)       # [P, 40]
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]

    def rope(z):                                                                   # z [P, 16, 80]
        c = torch.complex(z[..., :40], z[..., 40:]) * rot
        return torch.cat([c.real, c.imag], -1)

    for L in wts["layers"]:
        h = F.layer_norm(x, (1280,), T(L["ln1_w"]), T(L["ln1_b"]), eps)
        qkv = F.linear(h, T(L["qkv_w"]), T(L["qkv_b"])).reshape(P, 3, 16, 80)
        q, k, v = rope(qkv[:, 0]), rope(qkv[:, 1]), qkv[:, 2]
        a = F.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1), attn_mask=mask)
        x = x + F.linear(a.transpose(0, 1).reshape(P, 1280), T(L["proj_w"]), T(L["proj_b"]))
        h = F.layer_norm(x, (1280,), T(L["ln2_w"]), T(L["ln2_b"]), eps)
        x = x + F.linear(F.gelu(F.linear(h, T(L["fc1_w"]), T(L["fc1_b"]))), T(L["fc2_w"]), T(L["fc2_b"]))
    y = F.layer_norm(x, (1280,), T(wts["lnq_w"]), T(wts["lnq_b"]), eps).reshape(P // 4, 5120)
    return F.linear(F.gelu(F.linear(y, T(wts["m0_w"]), T(wts["m0_b"]))), T(wts["m2_w"]), T(wts["m2_b"])).numpy()


def test_tower_matches_torch_restatement():
    grids = [(1, 4, 6), (2, 2, 2), (1, 8, 4)]
    wts = _small_weights(2, out_dim=96, seed=31, affine=True)
    patches = syn.make_patches(grids, 32)
    ref = _torch_tower(patches, grids, wts, 1e-6)
    got = vo.vit_encode(patches, grids, wts, eps=1e-6)
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-11)


def test_tiny_workload_runs():
    wl = syn.WORKLOADS["tiny"]
    wts = syn.make_weights(wl.depth, wl.out_dim, wl.seed)
    out = vo.vit_encode(syn.make_patches(wl.grids, wl.seed), wl.grids, wts)
    assert out.shape == (16, 1536) and np.isfinite(out).all()
