"""Zero-shot patch-text scoring (vit_seg_zero_shot) against the fp64 oracle: whole and slide
modes (dino.txt zero-shot segmentation article, whole/slide section)."""
import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import ARGMAX_AGREE_MIN, gpu, need_cuda

pytestmark = gpu


def assert_valid_argmax(labels, scores, tol):
    """Every label must be an argmax of `scores` [C, H, W] up to `tol` (near-ties may resolve
    either way between fp32 and fp64; what is unique is the maximal score)."""
    best = scores.max(axis=0)
    picked = np.take_along_axis(scores, labels[None].astype(np.int64), axis=0)[0]
    assert (best - picked).max() <= tol, (best - picked).max()


def _gpu_tokens(enc, crops):
    outs = enc.forward(crops, desc=False, patch=True, patch_fp32=True)
    torch.cuda.synchronize()
    return outs["patch_tokens"].double().cpu().numpy()


def _crops(image, side, stride):
    _, H, W = image.shape
    return torch.stack([image[:, y:y + side, x:x + side] for y in O.window_origins(H, side, stride)
                        for x in O.window_origins(W, side, stride)]).contiguous()


def test_seg_whole_small():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]
    w = S.make_weights(spec, 61)
    im = S.make_images(spec, 1, 62)
    text = S.make_text_feats(20, spec.dim, 63)
    enc = V.VitEncoder(spec, w, max_batch=1)
    probs, labels = enc.seg(im[0].cuda(), text.cuda(), mode=V.VIT_SEG_WHOLE)
    torch.cuda.synchronize()
    enc.poll()
    ref = O.forward(im, w, spec)
    rs, rl = O.seg_whole_from_tokens(ref["patch_tokens"][0], text.double().numpy(), spec.img_h, spec.img_w,
                                     ref["grid"])
    g = probs.double().cpu().numpy()
    assert np.abs(g - rs).max() < 2e-3
    agree = (labels.cpu().numpy() == rl).mean()
    assert agree >= ARGMAX_AGREE_MIN, agree
    # the head alone on the GPU's own tokens: bilinear/argmax logic must agree (almost) exactly
    tok = _gpu_tokens(enc, im.cuda())
    hs, hl = O.seg_whole_from_tokens(tok[0], text.double().numpy(), spec.img_h, spec.img_w, ref["grid"])
    assert np.abs(g - hs).max() < 1e-5
    assert (labels.cpu().numpy() == hl).mean() >= 0.999
    assert_valid_argmax(labels.cpu().numpy(), hs, 2e-5)
    enc.close()


def test_seg_slide_small():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]          # 224 x 224 windows
    w = S.make_weights(spec, 71)
    H, W, side, stride = 320, 480, 224, 112
    im = S.make_images(spec, 1, 72, H, W)[0]
    text = S.make_text_feats(30, spec.dim, 73)
    nwin = len(O.window_origins(H, side, stride)) * len(O.window_origins(W, side, stride))
    enc = V.VitEncoder(spec, w, max_batch=nwin)
    probs, labels = enc.seg(im.cuda(), text.cuda(), mode=V.VIT_SEG_SLIDE, side=side, stride=stride)
    torch.cuda.synchronize()
    enc.poll()
    rp, rl, _ = O.seg_slide(im, w, spec, text, side, stride)
    g = probs.double().cpu().numpy()
    assert np.abs(g.sum(0) - 1).max() < 1e-4
    assert np.abs(g - rp).max() < 2e-3
    assert (labels.cpu().numpy() == rl).mean() >= ARGMAX_AGREE_MIN
    tok = _gpu_tokens(enc, _crops(im.cuda(), side, stride))
    hp, hl = O.seg_slide_from_tokens(tok, text.double().numpy(), H, W, side, stride, (spec.grid_h, spec.grid_w))
    assert np.abs(g - hp).max() < 1e-5
    assert (labels.cpu().numpy() == hl).mean() >= 0.999
    assert_valid_argmax(labels.cpu().numpy(), hp, 2e-5)
    enc.close()


@pytest.mark.parametrize("side,stride", [(112, 112), (160, 64), (96, 40), (224, 64), (128, 96)])
def test_seg_slide_window_overlaps(side, stride):
    """Window overlaps from none to five per axis (pixels covered by 1 to 12 windows, clamped last
    windows): the GPU head on the GPU's own window tokens against the oracle's."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]
    w = S.make_weights(spec, 75)
    H, W = 256, 400
    im = S.make_images(spec, 1, 76, H, W)[0]
    text = S.make_text_feats(11, spec.dim, 77)
    nwin = len(O.window_origins(H, side, stride)) * len(O.window_origins(W, side, stride))
    enc = V.VitEncoder(spec, w, max_batch=nwin)
    probs, labels = enc.seg(im.cuda(), text.cuda(), mode=V.VIT_SEG_SLIDE, side=side, stride=stride)
    torch.cuda.synchronize()
    enc.poll()
    tok = _gpu_tokens(enc, _crops(im.cuda(), side, stride))
    g = side // spec.patch
    hp, hl = O.seg_slide_from_tokens(tok, text.double().numpy(), H, W, side, stride, (g, g))
    gp = probs.double().cpu().numpy()
    assert np.abs(gp - hp).max() < 1e-5
    assert np.abs(gp.sum(0) - 1).max() < 1e-4
    assert_valid_argmax(labels.cpu().numpy(), hp, 2e-5)
    enc.close()


@pytest.mark.parametrize("C", [1, 160, 161, 300])
@pytest.mark.parametrize("slide", [False, True])
def test_seg_class_counts(C, slide):
    """Class counts from 1 to 300: one and several 64-class tiles of the cosine GEMM, and the tiled
    slide-scoring kernel's 160-class limit on both sides (beyond it the per-pixel kernel runs),
    checked against the oracle's head on the GPU's own tokens."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]
    w = S.make_weights(spec, 85)
    H, W, side, stride = (256, 400, 224, 112) if slide else (spec.img_h, spec.img_w, 0, 0)
    im = S.make_images(spec, 1, 86, H, W)
    text = S.make_text_feats(C, spec.dim, 87)
    nwin = len(O.window_origins(H, side, stride)) * len(O.window_origins(W, side, stride)) if slide else 1
    enc = V.VitEncoder(spec, w, max_batch=nwin)
    if slide:
        scores, labels = enc.seg(im[0].cuda(), text.cuda(), mode=V.VIT_SEG_SLIDE, side=side, stride=stride)
        tok = _gpu_tokens(enc, _crops(im[0].cuda(), side, stride))
        hs, _ = O.seg_slide_from_tokens(tok, text.double().numpy(), H, W, side, stride,
                                        (side // spec.patch, side // spec.patch))
    else:
        scores, labels = enc.seg(im[0].cuda(), text.cuda(), mode=V.VIT_SEG_WHOLE)
        tok = _gpu_tokens(enc, im.cuda())
        hs, _ = O.seg_whole_from_tokens(tok[0], text.double().numpy(), H, W, (spec.grid_h, spec.grid_w))
    torch.cuda.synchronize()
    enc.poll()
    assert np.abs(scores.double().cpu().numpy() - hs).max() < 1e-5
    assert_valid_argmax(labels.cpu().numpy(), hs, 2e-5)
    enc.close()


@pytest.mark.slow
def test_seg_slide_vitl16_512x1024():
    """The full zero-shot workload: ViT-L/16 on 2 x 5 windows of 384 at stride 192, 150 classes."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec, w, im = S.make_workload("vitl16_slide_512x1024")
    text = S.make_text_feats(S.SLIDE_CLASSES, spec.dim)
    H, W = S.SLIDE_IMAGE
    enc = V.VitEncoder(spec, w, max_batch=10)
    probs, labels = enc.seg(im[0].cuda(), text.cuda(), mode=V.VIT_SEG_SLIDE, side=S.SLIDE_SIDE, stride=S.SLIDE_STRIDE)
    torch.cuda.synchronize()
    enc.poll()
    g = probs.double().cpu().numpy()
    gl = labels.cpu().numpy()
    assert np.isfinite(g).all()
    rp, rl, _ = O.seg_slide(im[0], w, spec, text, S.SLIDE_SIDE, S.SLIDE_STRIDE)
    agree = (gl == rl).mean()
    assert agree >= ARGMAX_AGREE_MIN, agree
    assert np.abs(g - rp).max() < 5e-3
    tok = _gpu_tokens(enc, _crops(im[0].cuda(), S.SLIDE_SIDE, S.SLIDE_STRIDE))
    hp, hl = O.seg_slide_from_tokens(tok, text.double().numpy(), H, W, S.SLIDE_SIDE, S.SLIDE_STRIDE,
                                     (spec.grid_h, spec.grid_w))
    assert (gl == hl).mean() >= 0.999
    assert_valid_argmax(gl, hp, 2e-5)
    enc.close()


def test_seg_rejects_bad_arguments():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]
    enc = V.VitEncoder(spec, S.make_weights(spec, 81), max_batch=2)
    im = torch.zeros(3, 320, 480, device="cuda")
    text = torch.zeros(4, spec.dim, device="cuda")
    with pytest.raises(V.VitError) as e:
        enc.seg(im, text, mode=V.VIT_SEG_SLIDE, side=224, stride=112)   # 8 windows > max_batch 2
    assert e.value.status == V.VIT_E_SHAPE
    with pytest.raises(V.VitError) as e:
        enc.seg(im, text, mode=V.VIT_SEG_SLIDE, side=400, stride=112)   # window taller than the image
    assert e.value.status == V.VIT_E_SHAPE
    with pytest.raises(V.VitError) as e:
        enc.seg(im, text, mode=V.VIT_SEG_SLIDE, side=8, stride=112)     # window smaller than a patch
    assert e.value.status == V.VIT_E_INVALID_ARG
    with pytest.raises(V.VitError) as e:
        enc.seg(im, text, mode=7)
    assert e.value.status == V.VIT_E_INVALID_ARG
    enc.close()
