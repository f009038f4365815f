"""vit_encode_noalloc, the encoder entry point for callers that cannot allocate device memory
(their GPU memory belongs to another allocator, or allocation after start-up is forbidden).

It keeps the activations in a fixed array inside the library instead of a cudaMalloc'd
workspace; its tokens must match vit_encode's on the same inputs. Two calls in a row (a
full-size 1024-patch image, then a smaller multi-image batch) also show that the shared array's
leftovers from one call do not leak into the next. This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from resolution_vit_vision_b200 import native as nv
from resolution_vit_vision_b200 import synthetic as syn
from tests.parity import assert_encoder_close, bf16_bits_to_torch, to_np

pytestmark = pytest.mark.gpu


def _noalloc(enc, patches, grids, out, status):
    g = np.ascontiguousarray(np.asarray(grids, np.int32).reshape(-1, 3))
    return nv.lib().vit_encode_noalloc(patches.data_ptr(), nv._gp(g), g.shape[0], enc.handle, out.data_ptr(),
                                       status.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_vit_encode_two_calls_in_a_row():
    wts = syn.make_weights(2, 1536, 41, affine=True)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), 1536)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for grids, seed in (([(1, 32, 32)], 42), ([(1, 8, 12), (2, 4, 6), (1, 6, 10)], 43)):
        patches = bf16_bits_to_torch(syn.make_patches(grids, seed))
        ref = to_np(enc.encode(patches, grids))
        out = torch.full((ref.shape[0], 1536), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(enc, patches, grids, out, status) == nv.VIT_OK
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_encoder_close(to_np(out), ref, f"noalloc vs vit_encode, grids {grids}")


def test_noalloc_raster_order_two_calls_and_no_allocation():
    # raster-ordered patches (the merge gathers 2x2 groups through the merge-row table); the
    # second call must leave the device's free memory and torch's allocator untouched
    wts = syn.make_weights(2, 1536, 45)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), 1536, 1e-6, 1)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i, (grids, seed) in enumerate((([(1, 16, 24), (1, 10, 6)], 46), ([(2, 8, 8), (1, 12, 20)], 47))):
        patches = bf16_bits_to_torch(syn.make_patches(grids, seed))
        ref = to_np(enc.encode(patches, grids))
        out = torch.full((ref.shape[0], 1536), float("nan"), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        free0, stats0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_stats().get("allocation.all.allocated", 0)
        assert _noalloc(enc, patches, grids, out, status) == nv.VIT_OK
        torch.cuda.synchronize()
        if i == 1:   # the first call may set the array up; the later one allocates nothing
            assert torch.cuda.mem_get_info()[0] == free0
            assert torch.cuda.memory_stats().get("allocation.all.allocated", 0) == stats0
        assert int(status.item()) == 0
        assert_encoder_close(to_np(out), ref, f"noalloc raster order vs vit_encode, grids {grids}")


def test_noalloc_rejects_overflowing_grid_rows():
    # factors whose product would overflow 64 bits are refused before the product is formed
    wts = syn.make_weights(1, 1536, 48)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), 1536)
    patches = torch.zeros((64, 1176), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((16, 1536), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bad in ([1 << 28, 1 << 17, 1 << 18], [1, 1 << 30, 2], [1 << 30, 2, 2], [1, 1024, 1024]):
        assert _noalloc(enc, patches, [bad], out, status) == nv.VIT_ERR_LIMIT, bad


def test_noalloc_rejects_batches_beyond_its_limit():
    wts = syn.make_weights(1, 1536, 44)
    enc = nv.VisionEncoder(nv.weights_to_device(wts), 1536)
    grids = [(1, 32, 32), (1, 2, 2)]                       # 1028 patches > 1024
    patches = torch.zeros((1028, 1176), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((257, 1536), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _noalloc(enc, patches, grids, out, status) == nv.VIT_ERR_LIMIT
