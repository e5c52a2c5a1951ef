"""vit_forward_noalloc: the forward for callers that may not allocate device memory while they
run (a plug-in whose host owns every allocation, a latency-critical loop where an allocation
could stall the device).  Its workspace is a fixed array inside the library, so this test
checks, through the C ABI, that two calls in a row give the same outputs as vit_forward with a
caller-provided workspace, and that a batch too large for the fixed array is refused.

The file name sorts last so that a run stopping at the first failure has already run every
other test; it passes alone in a fresh process and after the rest of the suite."""
import ctypes

import numpy as np
import torch

import synthetic as S
from parity import DESC_COS_MIN, desc_cos, gpu, need_cuda

pytestmark = gpu


def _outputs(V, outs):
    o = V.VitOutputs()
    o.desc = outs["desc"].data_ptr()
    o.patch_tokens = outs["patch_tokens"].data_ptr()
    o.patch_fp32 = 1
    return o


def test_noalloc_matches_vit_forward_twice():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.VITS16_336
    B = 3
    enc = V.VitEncoder(spec, S.make_weights(spec, 91), max_batch=B)
    images = S.make_images(spec, B, 92).cuda()
    ref = enc.forward(images, desc=True, patch=True, patch_fp32=True)
    torch.cuda.synchronize()
    lib = V.load_library()
    stream = torch.cuda.current_stream().cuda_stream or None
    for call in range(2):
        got = enc.alloc_outputs(B, desc=True, patch=True, patch_fp32=True)
        st = lib.vit_forward_noalloc(enc.handle, images.data_ptr(), B, ctypes.byref(_outputs(V, got)), stream)
        assert st == V.VIT_OK, lib.vit_last_error()
        torch.cuda.synchronize()
        enc.poll()
        for i in range(B):
            assert desc_cos(got["desc"][i].double().cpu().numpy(), ref["desc"][i].double().cpu().numpy()) >= DESC_COS_MIN
        diff = (got["patch_tokens"] - ref["patch_tokens"]).abs().max().item()
        assert diff <= 1e-5 * max(1.0, ref["patch_tokens"].abs().max().item()), (call, diff)
        assert torch.isfinite(got["patch_tokens"]).all()
    enc.close()


NOALLOC_BYTES = 64 << 20        # the fixed array's size, as the header states
NOALLOC_VITS16_336_MAX_BATCH = 24  # the largest ViT-S/16@336 batch the header says fits


def test_noalloc_boundary_of_the_fixed_scratch():
    """The largest batch whose workspace fits the fixed array runs and matches vit_forward; one
    image more is refused with VIT_E_WORKSPACE before anything is launched."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.VITS16_336
    enc = V.VitEncoder(spec, S.make_weights(spec, 93), max_batch=40)
    bmax = max(b for b in range(1, 41) if enc.workspace_size(b) <= NOALLOC_BYTES)
    assert bmax == NOALLOC_VITS16_336_MAX_BATCH, bmax
    lib = V.load_library()
    big = torch.zeros(bmax + 1, 3, spec.img_h, spec.img_w, device="cuda")
    outs = enc.alloc_outputs(bmax + 1, desc=True, patch=True, patch_fp32=True)
    st = lib.vit_forward_noalloc(enc.handle, big.data_ptr(), bmax + 1, ctypes.byref(_outputs(V, outs)), None)
    assert st == V.VIT_E_WORKSPACE
    assert b"fixed" in lib.vit_last_error()
    images = S.make_images(spec, bmax, 94).cuda()
    ref = enc.forward(images, desc=True, patch=True, patch_fp32=True)
    got = enc.alloc_outputs(bmax, desc=True, patch=True, patch_fp32=True)
    st = lib.vit_forward_noalloc(enc.handle, images.data_ptr(), bmax, ctypes.byref(_outputs(V, got)), None)
    assert st == V.VIT_OK, lib.vit_last_error()
    torch.cuda.synchronize()
    enc.poll()
    assert torch.equal(got["desc"], ref["desc"])
    assert torch.equal(got["patch_tokens"], ref["patch_tokens"])
    enc.close()


def test_noalloc_refuses_another_current_device():
    """With another GPU current the call is refused before any launch: the fixed array of that GPU
    must never be paired with this model's weights."""
    need_cuda()
    if torch.cuda.device_count() < 2:
        import pytest
        pytest.skip("needs two visible GPUs")
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s16"]
    torch.cuda.set_device(0)
    enc = V.VitEncoder(spec, S.make_weights(spec, 95), max_batch=1)
    images = S.make_images(spec, 1, 96).cuda(0)
    outs = enc.alloc_outputs(1, desc=True, patch=True, patch_fp32=True)
    lib = V.load_library()
    with torch.cuda.device(1):
        st = lib.vit_forward_noalloc(enc.handle, images.data_ptr(), 1, ctypes.byref(_outputs(V, outs)), None)
    assert st == V.VIT_E_INVALID_ARG
    assert b"device" in lib.vit_last_error()
    enc.close()
