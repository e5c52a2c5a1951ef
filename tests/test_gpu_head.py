"""The dino.txt vision head (dino.txt article, "Aligning 1024-d patch tokens with 2048-d text
embeddings": 2 extra self-attention blocks on the backbone's tokens before the cosine with the
text features) through vit_set_text_head / vit_forward_text_tokens / vit_seg_zero_shot,
against the fp64 oracle's text_head."""
import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import ARGMAX_AGREE_MIN, BLOCK_REL_MAX, block_rel_err, gpu, need_cuda

pytestmark = gpu


@pytest.mark.parametrize("name,hw,batch", [("tiny_s16", None, 2), ("tiny_s14", (98, 154), 3),
                                           ("small_s16", (320, 224), 2)])
def test_text_tokens_match_oracle(name, hw, batch):
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS[name]
    hw = hw or (spec.img_h, spec.img_w)
    w = S.make_weights(spec, 121)
    head = S.make_head_weights(spec, 122)
    im = S.make_images(spec, batch, 123, *hw)
    enc = V.VitEncoder(spec, w, max_batch=batch)
    enc.set_text_head(head)
    tok = enc.text_tokens(im.cuda().contiguous())
    torch.cuda.synchronize()
    enc.poll()
    n_launch = enc.last_launch_count()
    native = (hw[0] // spec.patch, hw[1] // spec.patch) == (spec.grid_h, spec.grid_w)
    assert n_launch == (0 if native else 1) + 3 + 5 * (spec.depth + 2) + 2
    g = tok.double().cpu().numpy()
    assert np.isfinite(g).all()
    ref = O.text_head(O.forward(im, w, spec)["final_tokens"], head, spec)
    for i in range(batch):
        e = block_rel_err(g[i], ref[i])
        assert e <= BLOCK_REL_MAX, f"image {i}: head tokens rel err {e:.3e}"
    enc.close()


def test_seg_whole_and_slide_with_head():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]
    w = S.make_weights(spec, 131)
    head = S.make_head_weights(spec, 132)
    text = S.make_text_feats(16, spec.dim, 133)
    H, W, side, stride = 288, 416, 224, 112
    im = S.make_images(spec, 1, 134, H, W)[0]
    nwin = len(O.window_origins(H, side, stride)) * len(O.window_origins(W, side, stride))
    enc = V.VitEncoder(spec, w, max_batch=nwin)
    enc.set_text_head(head)
    scores, labels = enc.seg(im.cuda(), text.cuda(), mode=V.VIT_SEG_WHOLE)
    probs, plabels = enc.seg(im.cuda(), text.cuda(), mode=V.VIT_SEG_SLIDE, side=side, stride=stride)
    torch.cuda.synchronize()
    enc.poll()
    rs, rl, _ = O.seg_whole(im, w, spec, text, head_blocks=head)
    assert np.abs(scores.double().cpu().numpy() - rs).max() < 2e-3
    assert (labels.cpu().numpy() == rl).mean() >= ARGMAX_AGREE_MIN
    rp, rpl, _ = O.seg_slide(im, w, spec, text, side, stride, head_blocks=head)
    g = probs.double().cpu().numpy()
    assert np.abs(g.sum(0) - 1).max() < 1e-4
    assert np.abs(g - rp).max() < 2e-3
    assert (plabels.cpu().numpy() == rpl).mean() >= ARGMAX_AGREE_MIN
    enc.close()


def test_head_argument_errors():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s16"]
    enc = V.VitEncoder(spec, S.make_weights(spec, 141), max_batch=1)
    im = S.make_images(spec, 1, 142).cuda()
    with pytest.raises(V.VitError) as e:
        enc.text_tokens(im)                          # no head attached yet
    assert e.value.status == V.VIT_E_INVALID_ARG
    enc.set_text_head(S.make_head_weights(spec, 143))
    with pytest.raises(V.VitError) as e:
        enc.set_text_head(S.make_head_weights(spec, 144))   # only once per model
    assert e.value.status == V.VIT_E_INVALID_ARG
    enc.close()


@pytest.mark.slow
def test_seg_slide_vitl16_512x1024_with_head():
    """The full zero-shot workload with the head: ViT-L/16 + 2 head blocks on 2 x 5 windows of 384
    at stride 192, 150 classes."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec, w, im = S.make_workload("vitl16_slide_512x1024")
    head = S.make_head_weights(spec, S.HEAD_SEED)
    text = S.make_text_feats(S.SLIDE_CLASSES, spec.dim)
    enc = V.VitEncoder(spec, w, max_batch=10)
    enc.set_text_head(head)
    probs, labels = enc.seg(im[0].cuda(), text.cuda(), mode=V.VIT_SEG_SLIDE, side=S.SLIDE_SIDE, stride=S.SLIDE_STRIDE)
    torch.cuda.synchronize()
    enc.poll()
    g = probs.double().cpu().numpy()
    assert np.isfinite(g).all()
    rp, rl, _ = O.seg_slide(im[0], w, spec, text, S.SLIDE_SIDE, S.SLIDE_STRIDE, head_blocks=head)
    assert (labels.cpu().numpy() == rl).mean() >= ARGMAX_AGREE_MIN
    assert np.abs(g - rp).max() < 5e-3
    enc.close()
