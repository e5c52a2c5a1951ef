"""End-to-end parity of vit_forward against the fp64 oracle, per configuration.

Small shapes are compared on every image; the full-size workloads run in the launch
configuration the bench times (whole batch on the GPU) and are compared on sampled images,
which the oracle computes one by one."""
import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import assert_forward_parity, gpu, need_cuda, run_gpu

pytestmark = gpu


@pytest.mark.parametrize("name,batch", [("tiny_s16", 2), ("tiny_s14", 3), ("small_s16", 2)])
def test_small_configs_all_images(name, batch):
    need_cuda()
    spec = S.PRESETS[name]
    w = S.make_weights(spec, 31)
    im = S.make_images(spec, batch, 32)
    g = run_gpu(spec, w, im)
    ref = O.forward(im, w, spec, record_hidden=True)
    assert_forward_parity(g, ref, spec, list(range(batch)))


def test_vits16_336_b1():
    need_cuda()
    spec, w, im = S.make_workload("vits16_336_b1")
    g = run_gpu(spec, w, im)
    ref = O.forward(im, w, spec, record_hidden=True)
    assert_forward_parity(g, ref, spec, [0])


def test_vits16_336_b64_attention_sink():
    """kornia/dinov3 card, "Build BF16, not FP16": block-1 logits of ~2.2e6, no NaN anywhere."""
    need_cuda()
    spec, w, im = S.make_workload("vits16_336_b64_outlier")
    idx = [0, 37, 63]
    g = run_gpu(spec, w, im, keep=idx)
    assert g["hidden_finite"] and np.isfinite(g["desc"]).all()
    ref = O.forward(im, w, spec, record_hidden=True, image_indices=idx)
    assert_forward_parity(g, ref, spec, idx)


def test_vits14_518_b8_taps():
    need_cuda()
    spec, w, im = S.make_workload("vits14_518_b8_taps")
    g = run_gpu(spec, w, im)
    for t in g["taps"]:
        assert t.shape == (8, 384, 37, 37)
    idx = [0, 7]
    ref = O.forward(im, w, spec, record_hidden=True, image_indices=idx)
    assert_forward_parity(g, ref, spec, idx)


@pytest.mark.slow
def test_vitl16_1024_b8():
    need_cuda()
    spec, w, im = S.make_workload("vitl16_1024_b8")
    idx = [5]
    g = run_gpu(spec, w, im, hidden=True, keep=idx)
    assert g["hidden_finite"]
    ref = O.forward(im, w, spec, record_hidden=True, image_indices=idx)
    assert_forward_parity(g, ref, spec, idx)


@pytest.mark.slow
def test_vitl16_1024_b1():
    """ViT-L/16@1024, batch 1: the batch of the DINOv3 deployment article's latency table (§3.2).
    At M = 4,101 rows the residual GEMMs run on single-CTA 128 x 256 tiles, not the paired tiles
    that batch 8 takes, so this shape is checked on its own."""
    need_cuda()
    spec, w, im = S.make_workload("vitl16_1024_b1")
    g = run_gpu(spec, w, im, hidden=True)
    assert np.isfinite(g["hidden"]).all()
    ref = O.forward(im, w, spec, record_hidden=True)
    assert_forward_parity(g, ref, spec, [0])


def _ln_rows(x):
    """Plain per-row LayerNorm (no affine), fp64: what a folded LayerNorm hands its GEMM."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(-1, keepdims=True)
    return (x - mu) / np.sqrt(((x - mu) ** 2).mean(-1, keepdims=True) + 1e-6)


def _offset_rows(spec, w, seed):
    """CLS and register rows (and, through the patch bias, every patch row) whose mean is large
    against their spread.  kornia/dinov3 card, "Build BF16, not FP16": activations of the encoder
    stay below ~1.8e3, so the largest offset here is 1,500."""
    g = torch.Generator().manual_seed(seed)
    D = spec.dim
    w = dict(w)
    w["cls"] = S.to_bf16(15.0 + 1.5 * torch.randn(D, generator=g))
    if spec.registers:
        offs = [150.0, 1500.0, -150.0] + [0.0] * (spec.registers - 3)
        reg = torch.stack([o + 1.5 * torch.randn(D, generator=g) for o in offs[:spec.registers]])
        w["reg"] = S.to_bf16(reg)
    w["patch_b"] = S.to_bf16(w["patch_b"].float() + 20.0)
    return w


@pytest.mark.parametrize("name", ["tiny_s16", "small_s16", "vitb14_224"])
def test_rows_with_large_mean(name):
    """The folded LayerNorm multiplies a bf16 copy of the residual stream.  Rows whose mean is
    large against their spread (|mean|/std from ~10 to several hundred here) lose their spread
    to bf16 rounding unless that copy is re-centred; the check is on what the LayerNorm sees:
    every row of every block's output, normalised, against the oracle's."""
    need_cuda()
    spec = S.PRESETS[name]
    w = _offset_rows(spec, S.make_weights(spec, 83), 84)
    im = S.make_images(spec, 2, 85)
    g = run_gpu(spec, w, im)
    ref = O.forward(im, w, spec, record_hidden=True)
    assert_forward_parity(g, ref, spec, [0, 1])
    ratio = 0.0
    for l in range(spec.depth):
        for i in range(2):
            xr = ref["hidden"][l, i]
            r = np.abs(xr.mean(-1)) / xr.std(-1)
            ratio = max(ratio, float(r.max()))
            a, b = _ln_rows(g["hidden"][l, i]), _ln_rows(xr)
            err = np.abs(a - b).max(-1) / np.abs(b).max(-1)
            assert err.max() <= 2e-2, f"block {l + 1} image {i}: row {int(err.argmax())} normalised rel err {err.max():.3e}"
    assert ratio >= (300.0 if spec.registers else 5.0), ratio


def test_forward_host_matches_device_path():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]
    w = S.make_weights(spec, 41)
    im = S.make_images(spec, 3, 42)
    enc = V.VitEncoder(spec, w, max_batch=3)
    dev = enc.forward(im.cuda(), desc=True, patch=True)
    ih = im.pin_memory()
    dh = torch.empty(3, spec.dim, dtype=torch.float32).pin_memory()
    ph = torch.empty(3, spec.n_patches, spec.dim, dtype=torch.bfloat16).pin_memory()
    enc.forward_host(ih, dh, ph)
    torch.cuda.synchronize()
    enc.poll()
    assert torch.equal(dh, dev["desc"].cpu())
    assert torch.equal(ph, dev["patch_tokens"].cpu())
    enc.close()


def test_repeated_calls_are_deterministic_and_launch_count():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s14"]
    w = S.make_weights(spec, 51)
    im = S.make_images(spec, 2, 52).cuda()
    enc = V.VitEncoder(spec, w, max_batch=2)
    a = enc.forward(im, desc=True, patch=True, taps=True)
    b = enc.forward(im, desc=True, patch=True, taps=True)
    torch.cuda.synchronize()
    enc.poll()
    assert torch.equal(a["desc"], b["desc"]) and torch.equal(a["patch_tokens"], b["patch_tokens"])
    # im2col, patch GEMM, prefix rows, 5 per block, one per tap, final LayerNorm
    assert enc.last_launch_count() == 3 + 5 * spec.depth + len(spec.taps) + 1
    enc.close()


def test_forward_replays_from_a_cuda_graph():
    """vit_forward enqueues only kernel launches on the caller's stream, so it can be captured into
    a CUDA graph (the bench times small batches that way); the replay must match an eager call."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]
    w = S.make_weights(spec, 61)
    x = S.make_images(spec, 2, 62).cuda()
    enc = V.VitEncoder(spec, w, max_batch=2)
    ws = torch.empty(enc.workspace_size(2), dtype=torch.uint8, device="cuda")
    eager = enc.forward(x, desc=True, patch=True)
    outs = enc.alloc_outputs(2, desc=True, patch=True)
    enc.forward_into(x, outs, ws=ws)          # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        enc.forward_into(x, outs, ws=ws)
    outs["desc"].zero_()
    g.replay()
    torch.cuda.synchronize()
    enc.poll()
    assert torch.equal(outs["desc"], eager["desc"]) and torch.equal(outs["patch_tokens"], eager["patch_tokens"])
    del g
    enc.close()


@pytest.mark.parametrize("name", ["vitb14_224", "vitg14_224"])
def test_other_widths(name):
    """ViT-B/14 and ViT-G/14 widths (DINOv2 blog's model-variant table) through the same kernels."""
    need_cuda()
    spec = S.PRESETS[name]
    w = S.make_weights(spec, 71)
    im = S.make_images(spec, 2, 72)
    g = run_gpu(spec, w, im)
    ref = O.forward(im, w, spec, record_hidden=True)
    assert_forward_parity(g, ref, spec, [0, 1])


def test_vitb14_224_b64_paired_gemms():
    """Batch 64 of ViT-B/14 (M = 16,448 rows): every block GEMM runs on paired 256 x 256 tiles."""
    need_cuda()
    spec = S.PRESETS["vitb14_224"]
    w = S.make_weights(spec, 73)
    im = S.make_images(spec, 64, 74)
    keep = [0, 37, 63]
    g = run_gpu(spec, w, im, keep=keep)
    assert g["hidden_finite"]
    ref = O.forward(im, w, spec, record_hidden=True, image_indices=keep)
    assert_forward_parity(g, ref, spec, keep)



def test_nonfinite_input_is_reported_by_poll():
    """A NaN pixel propagates through the encoder; the final LayerNorm flags the non-finite rows and
    vit_poll reports VIT_E_NONFINITE once (the flag is cleared by the poll)."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s16"]
    enc = V.VitEncoder(spec, S.make_weights(spec, 81), max_batch=2)
    im = S.make_images(spec, 2, 82).cuda()
    enc.forward(im)
    enc.poll()                                  # clean input: no error
    bad = im.clone()
    bad[1, 0, 5, 7] = float("nan")
    enc.forward(bad)
    with pytest.raises(V.VitError) as e:
        enc.poll()
    assert e.value.status == V.VIT_E_NONFINITE
    enc.forward(im)
    enc.poll()                                  # flag cleared
    enc.close()


def test_forward_rejects_bad_arguments():
    """vit_forward validates on the host before any launch: a batch outside 1..max_batch, a
    workspace below vit_workspace_size and pointers that are not 16-byte aligned are refused with
    their status codes, and the model still gives the same descriptors afterwards."""
    need_cuda()
    import ctypes
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s16"]
    enc = V.VitEncoder(spec, S.make_weights(spec, 61), max_batch=2)
    im = S.make_images(spec, 3, 62).cuda().contiguous()
    before = enc.forward(im[:2], desc=True)["desc"].clone()
    desc = torch.empty(2, spec.dim, dtype=torch.float32, device="cuda")
    need = enc.workspace_size(2)
    ws = torch.empty(need + 256, dtype=torch.uint8, device="cuda")

    def call(img_ptr, B, ws_bytes, desc_ptr):
        o = V.VitOutputs()
        o.desc = desc_ptr
        return enc.lib.vit_forward(enc.handle, ctypes.c_void_p(img_ptr), B, ctypes.byref(o),
                                   ctypes.c_void_p(ws.data_ptr()), ws_bytes, None)

    ok_img, ok_desc = im.data_ptr(), desc.data_ptr()
    assert call(ok_img, 0, need, ok_desc) == V.VIT_E_SHAPE
    assert call(ok_img, 3, need, ok_desc) == V.VIT_E_SHAPE
    assert call(ok_img, 2, need - 1, ok_desc) == V.VIT_E_WORKSPACE
    assert call(ok_img + 4, 2, need, ok_desc) == V.VIT_E_INVALID_ARG
    assert call(ok_img, 2, need, ok_desc + 4) == V.VIT_E_INVALID_ARG
    assert call(0, 2, need, ok_desc) == V.VIT_E_INVALID_ARG
    torch.cuda.synchronize()
    enc.poll()
    assert call(ok_img, 2, need, ok_desc) == V.VIT_OK
    torch.cuda.synchronize()
    enc.poll()
    assert torch.equal(desc, before)
    enc.close()


_PDL_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import synthetic as S, vision_transformer_encoder_fwd_b200 as V
spec = S.PRESETS["small_s16"]
enc = V.VitEncoder(spec, S.make_weights(spec, 191), max_batch=2)
o = enc.forward(S.make_images(spec, 2, 192).cuda(), desc=True, patch=True)
torch.cuda.synchronize()
enc.poll()
np.save(sys.argv[2], o["patch_tokens"].float().cpu().numpy())
enc.close()
"""


def test_programmatic_dependent_launch_changes_nothing(tmp_path):
    """The GEMM and attention kernels are launched with programmatic dependent launch unless
    VIT_B200_PDL=0; a forward in a child process with it off must give the same bits."""
    need_cuda()
    import os
    import subprocess
    import sys
    import vision_transformer_encoder_fwd_b200 as V
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = tmp_path / "off.npy"
    env = dict(os.environ, VIT_B200_PDL="0")
    subprocess.run([sys.executable, "-c", _PDL_CHILD, root, str(out)], env=env, check=True, timeout=600)
    spec = S.PRESETS["small_s16"]
    enc = V.VitEncoder(spec, S.make_weights(spec, 191), max_batch=2)
    o = enc.forward(S.make_images(spec, 2, 192).cuda(), desc=True, patch=True)
    torch.cuda.synchronize()
    enc.poll()
    on = o["patch_tokens"].float().cpu().numpy()
    enc.close()
    assert np.array_equal(on, np.load(out))
