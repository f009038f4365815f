"""Whole-encoder parity on a B200 through vit_encode (include/vit.h) against the fp64 oracle.

Bar: max|err| <= 3e-2 * max|ref| and per-token cosine >= 0.999 on the bf16 output.
Full sizes, all at depth 32 in the launch configuration the benchmark uses: the 2B-shaped single
image is checked whole against the oracle run in the test; the 8-image mixed batch, the 1792^2
image and the video batch against the oracle's stored full-depth outputs
(``tests/golden/full_depth_*.npz``, written by ``tests/golden/make_full_depth.py`` from the oracle
alone): sampled rows of every image and video frame element by element, every row through its
norm and random projections, plus whole images the oracle can compute in the test.
"""
import numpy as np
import pytest
import torch

from oracle import vit_oracle as vo
from resolution_vit_vision_b200 import native as nv
from resolution_vit_vision_b200 import synthetic as syn
from tests.parity import assert_encoder_close, bf16_bits_to_torch, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(grids, depth, out_dim, seed, order=0, affine=False, patches=None, wts=None):
    wts = wts if wts is not None else syn.make_weights(depth, out_dim, seed, affine=affine)
    patches = patches if patches is not None else syn.make_patches(grids, seed)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), out_dim, 1e-6, order)
    out = enc.encode(bf16_bits_to_torch(patches), grids)
    assert enc.device_status() == 0
    return to_np(out), wts, patches, enc


def test_tiny_workload():
    wl = syn.WORKLOADS["tiny"]
    got, wts, patches, _ = _run(wl.grids, wl.depth, wl.out_dim, wl.seed)
    ref = vo.vit_encode(patches, wl.grids, wts)
    assert got.shape == (16, 1536)
    assert_encoder_close(got, ref, "tiny")


@pytest.mark.parametrize("order", [0, 1])
def test_ragged_multi_image_affine(order):
    grids = [(1, 10, 14), (2, 4, 6), (1, 6, 2), (1, 16, 12)]   # 140 + 48 + 12 + 192 = 392 patches
    got, wts, patches, _ = _run(grids, 2, 1536, 7, order=order, affine=True)
    ref = vo.vit_encode(patches, grids, wts, patch_order=order)
    assert_encoder_close(got, ref, f"ragged order {order}")


def test_raster_equals_block_order():
    # T8: the same patches packed raster vs 2x2-block give the same merged tokens
    grids = [(1, 6, 10), (1, 4, 4)]
    wts = syn.make_weights(2, 1536, 8)
    raw = syn.make_patches(grids, 8)              # taken as raster order
    hp, wp = vo.patch_positions(grids, 0)
    rows, start = [], 0
    for t, h, w in grids:
        fh, fw = vo.frame_positions(h, w, 0)
        rows.append(start + fh * w + fw)
        start += h * w
    block = raw[np.concatenate(rows)]
    g0, *_ = _run(grids, 2, 1536, 8, order=0, patches=block, wts=wts)
    g1, *_ = _run(grids, 2, 1536, 8, order=1, patches=raw, wts=wts)
    assert_encoder_close(g1, g0, "raster vs block")


def test_permuting_images_permutes_outputs():
    # T3 / T4: attention never crosses images, so the order of images only permutes output rows
    grids = [(1, 8, 8), (1, 4, 12), (1, 10, 6)]
    wts = syn.make_weights(2, 1536, 9)
    patches = syn.make_patches(grids, 9)
    out, *_ = _run(grids, 2, 1536, 9, patches=patches, wts=wts)
    starts = np.cumsum([0] + [t * h * w for t, h, w in grids])
    tok = starts // 4
    perm = [2, 0, 1]
    p2 = np.concatenate([patches[starts[i]:starts[i + 1]] for i in perm])
    out2, *_ = _run([grids[i] for i in perm], 2, 1536, 9, patches=p2, wts=wts)
    ref = np.concatenate([out[tok[i]:tok[i + 1]] for i in perm])
    np.testing.assert_array_equal(out2, ref)      # same kernels, same per-image work: bit-equal
    alone, *_ = _run([grids[1]], 2, 1536, 9, patches=patches[starts[1]:starts[2]], wts=wts)
    np.testing.assert_array_equal(alone, out[tok[1]:tok[2]])


def test_more_segments_than_one_attention_launch():
    # a 600-frame video of 2 x 4 patches plus an image: 601 attention segments, more than one
    # attention launch holds, through the whole encoder against the oracle
    grids = [(600, 2, 4), (1, 4, 4)]
    got, wts, patches, _ = _run(grids, 2, 1536, 16)
    ref = vo.vit_encode(patches, grids, wts)
    assert got.shape == (1204, 1536)
    assert_encoder_close(got, ref, "601 segments")


def test_encode_host_matches_device():
    grids = [(1, 8, 12), (1, 6, 6)]
    got, wts, patches, enc = _run(grids, 2, 1536, 10)
    hp = torch.from_numpy(patches.copy()).view(torch.bfloat16).pin_memory()
    ho = torch.empty((got.shape[0], 1536), dtype=torch.bfloat16).pin_memory()
    enc.encode_host(hp, grids, ho)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ho.float().numpy(), got)


def test_repeat_calls_identical_and_growth():
    grids = [(1, 8, 8)]
    wts = syn.make_weights(1, 1536, 11)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), 1536)
    p_small = bf16_bits_to_torch(syn.make_patches(grids, 11))
    a = to_np(enc.encode(p_small, grids))
    big = [(1, 32, 32), (1, 8, 8)]
    pb = bf16_bits_to_torch(syn.make_patches(big, 12))
    enc.encode(pb, big)                            # grows the workspace
    b = to_np(enc.encode(p_small, grids))
    np.testing.assert_array_equal(a, b)


def test_boundary_errors():
    wts = syn.make_weights(1, 1536, 13)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), 1536)
    p = torch.zeros((64, 1176), dtype=torch.bfloat16, device=DEV)
    out = torch.zeros((16, 1536), dtype=torch.bfloat16, device=DEV)
    L = nv.lib()
    g = np.array([[1, 8, 8]], np.int32)
    s = torch.cuda.current_stream().cuda_stream
    assert L.vit_encode(p.data_ptr(), nv._gp(g), 1, enc.handle, None, s) == nv.VIT_ERR_ARG
    assert L.vit_encode(p.data_ptr(), nv._gp(g), 0, enc.handle, out.data_ptr(), s) == nv.VIT_ERR_ARG
    for bad in ([1, 7, 8], [0, 8, 8], [1, 8, 0]):
        gb = np.array([bad], np.int32)
        assert L.vit_encode(p.data_ptr(), nv._gp(gb), 1, enc.handle, out.data_ptr(), s) == nv.VIT_ERR_GRID
    assert L.vit_encode(p.data_ptr() + 2, nv._gp(g), 1, enc.handle, out.data_ptr(), s) == nv.VIT_ERR_ALIGN
    n0 = enc.launch_count()
    assert L.vit_encode(p.data_ptr(), nv._gp(g), 1, enc.handle, out.data_ptr(), s) == 0
    assert enc.launch_count() > n0


# ------------------------------------------------------------------ full sizes
@pytest.mark.slow
def test_2b_448_full_depth():
    wl = syn.WORKLOADS["2b_448"]
    got, wts, patches, _ = _run(wl.grids, wl.depth, wl.out_dim, wl.seed)
    ref = vo.vit_encode(patches, wl.grids, wts)
    assert got.shape == (256, 1536)
    assert_encoder_close(got, ref, "2B 448x448 depth 32")


def _check_full_depth_golden(name, got):
    """The stored full-depth oracle output of a workload (tests/golden/make_full_depth.py):
    sampled rows element by element at the encoder bar (scale: max|ref| over the whole batch),
    and every row through its norm and 16 random +-1 projections."""
    from tests.golden.make_full_depth import N_PROJ, path_for, projection_matrix
    wl = syn.WORKLOADS[name]
    g = np.load(path_for(name))
    assert [tuple(r) for r in g["grids"].tolist()] == [tuple(r) for r in wl.grids]
    assert int(g["depth"]) == wl.depth and int(g["seed"]) == wl.seed
    assert got.shape == (g["norm"].shape[0], wl.out_dim)
    rows, ref = g["rows"], g["ref_rows"].astype(np.float64)
    sub = got[rows]
    err = np.abs(sub - ref).max()
    assert err <= 3e-2 * float(g["max_abs"]), f"{name}: max|err| {err:.3e} on {rows.size} sampled rows"
    cos = (sub * ref).sum(1) / (np.linalg.norm(sub, axis=1) * np.linalg.norm(ref, axis=1))
    assert cos.min() >= 0.999, f"{name}: min cosine {cos.min():.6f} on the sampled rows"
    # every row: a per-token cosine of 0.999 allows |got - ref| up to ~0.045 |ref|. The norms must
    # agree to that, and the error estimated from the projections (chi-square with 16 degrees of
    # freedom: within a factor 2 of the true error with overwhelming probability) must stay below
    # twice it
    norm = g["norm"].astype(np.float64)
    assert np.all(np.abs(np.linalg.norm(got, axis=1) - norm) <= 0.045 * norm), f"{name}: row norms"
    est = np.linalg.norm(got @ projection_matrix(wl.out_dim) - g["proj"], axis=1) / np.sqrt(N_PROJ)
    assert np.all(est <= 0.09 * norm), f"{name}: worst estimated row error {np.max(est / norm):.3e} of |ref|"
    return err / float(g["max_abs"]), float(cos.min()), float(np.max(est / norm))


@pytest.mark.slow
def test_mixed8_full_depth_every_image():
    # all 8 images at depth 32 against the stored oracle output, in the benchmark's configuration;
    # the 336x336 image also whole against the oracle run here
    wl = syn.WORKLOADS["mixed8"]
    got, wts, patches, _ = _run(wl.grids, wl.depth, wl.out_dim, wl.seed)
    assert got.shape == (4424, 3584)
    _check_full_depth_golden("mixed8", got)
    starts = np.cumsum([0] + [t * h * w for t, h, w in wl.grids])
    i = 5
    ref = vo.vit_encode(patches[starts[i]:starts[i + 1]], [wl.grids[i]], wts)
    assert_encoder_close(got[starts[i] // 4:starts[i + 1] // 4], ref, f"mixed8 image {i}")


@pytest.mark.slow
def test_video_batch_full_depth_every_item():
    # the four frames of the video and both images at depth 32 against the stored oracle output;
    # the last image also whole against the oracle run here, and each frame is its own segment:
    # frame 3 alone equals its rows of the batch
    wl = syn.WORKLOADS["video_2img"]
    got, wts, patches, _ = _run(wl.grids, wl.depth, wl.out_dim, wl.seed)
    assert got.shape == (1792, 3584)
    _check_full_depth_golden("video_2img", got)
    s = 4096 + 1536
    ref = vo.vit_encode(patches[s:], [wl.grids[2]], wts)
    assert_encoder_close(got[s // 4:], ref, "video batch, image 2")
    one = [(1, 32, 32)]
    g1, *_ = _run(one, wl.depth, wl.out_dim, wl.seed, patches=patches[3072:4096], wts=wts)
    np.testing.assert_array_equal(g1, got[768:1024])


def test_graph_replay_matches_direct_launches():
    grids = [(1, 8, 12), (2, 4, 6)]
    wts = syn.make_weights(2, 1536, 14)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), 1536)
    p1 = bf16_bits_to_torch(syn.make_patches(grids, 14))
    ref = to_np(enc.encode(p1, grids))
    enc.graph_enable(True)
    out = torch.empty((ref.shape[0], 1536), dtype=torch.bfloat16, device=DEV)
    n0 = enc.launch_count()
    enc.encode(p1, grids, out=out)                 # records and launches
    enc.encode(p1, grids, out=out)                 # replays
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(out), ref)
    assert (enc.launch_count() - n0) % 2 == 0 and enc.launch_count() > n0
    # host buffers through the replayed graph
    hp = p1.cpu().pin_memory()
    ho = torch.empty((ref.shape[0], 1536), dtype=torch.bfloat16).pin_memory()
    for _ in range(2):
        enc.encode_host(hp, grids, ho)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(ho.float().numpy(), ref)
    # new data in the same buffers is encoded by the replay
    p2 = bf16_bits_to_torch(syn.make_patches(grids, 15))
    p1.copy_(p2)
    enc.encode(p1, grids, out=out)
    enc.graph_enable(False)
    ref2 = to_np(enc.encode(p2, grids))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(out), ref2)
    assert enc.device_status() == 0


def test_back_to_back_encodes_on_one_stream():
    # Different batches encoded one after another on one stream with nothing synchronising them:
    # every kernel may start while its predecessor drains (programmatic dependent launch), so a
    # kernel touching memory before its wait would let one encode read or overwrite another's
    # positions, activations or output. Each result must equal the same batch encoded alone.
    wts = syn.make_weights(2, 1536, 16)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), 1536)
    batches = [[(1, 12, 16), (2, 4, 6)], [(1, 8, 8)], [(1, 20, 10), (1, 6, 6), (3, 4, 4)]]
    ins = [bf16_bits_to_torch(syn.make_patches(g, 16 + i)) for i, g in enumerate(batches)]
    refs = []
    for p, g in zip(ins, batches):               # one at a time (this also grows the workspace)
        refs.append(to_np(enc.encode(p, g)))
    outs = [torch.full((r.shape[0], 1536), float("nan"), dtype=torch.bfloat16, device=DEV) for r in refs]
    for graphs in (False, True):
        enc.graph_enable(graphs)
        for _ in range(3):
            for p, g, o in zip(ins, batches, outs):
                enc.encode(p, g, out=o)
        torch.cuda.synchronize()
        for o, r in zip(outs, refs):
            np.testing.assert_array_equal(to_np(o), r)
    enc.graph_enable(False)
    assert enc.device_status() == 0


@pytest.mark.slow
def test_hires_1792_single_segment():
    # 16384 patches in one attention segment: the full depth-32 encode against the stored oracle
    # output, and the whole image against the oracle run here at depth 1
    wl = syn.WORKLOADS["hires_1792"]
    got, wts, patches, _ = _run(wl.grids, wl.depth, wl.out_dim, wl.seed)
    assert got.shape == (4096, 3584)
    _check_full_depth_golden("hires_1792", got)
    wts1 = dict(wts, layers=wts["layers"][:1])
    got1, *_ = _run(wl.grids, 1, wl.out_dim, wl.seed, wts=wts1, patches=patches)
    ref = vo.vit_encode(patches, wl.grids, wts1)
    assert_encoder_close(got1, ref, "1792^2 depth 1")
