"""Dense head on the taps (LibreYOLO DINOv2 configuration diagram: "Projector P4", "Projector
Bottleneck", "Projector output ConvX", "Task head") through vit_set_dense_head /
vit_forward_dense, against the fp64 oracle's dense_head on the oracle's own taps.

Tolerance: projector features and logits within 2e-2 of their largest magnitude (the encoder's
per-block bar), although the GPU keeps the activations between the ten conv / norm stages in
bf16 (fp32 accumulation and statistics).  Class agreement: the seeded head gives nearly flat
logits over 19 classes, so many pixels have two classes within the error bar of each other;
there both answers are right at the stated precision.  The argmax must agree on at least 99.5%
of the pixels whose top-2 gap exceeds twice the error bar, and on at least 99% of all pixels."""
import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import block_rel_err, gpu, need_cuda

pytestmark = gpu
DENSE_REL_MAX = 2e-2


def _check(spec, w, hw, im, idx, out_hw):
    import vision_transformer_encoder_fwd_b200 as V
    enc = V.VitEncoder(spec, w, max_batch=im.shape[0])
    enc.set_dense_head(hw)
    logits, p4 = enc.forward_dense(im.cuda().contiguous(), p4=True)
    torch.cuda.synchronize()
    enc.poll()
    n_launch = enc.last_launch_count()
    g_logits = logits.double().cpu().numpy()
    g_p4 = p4.double().cpu().numpy()
    enc.close()
    assert np.isfinite(g_logits).all() and np.isfinite(g_p4).all()
    o = O.forward(im, w, spec, image_indices=idx)
    ref = O.dense_head(o["taps"], hw, spec, out_hw)
    for j, i in enumerate(idx):
        ep = block_rel_err(g_p4[i], ref["p4"][j])
        el = block_rel_err(g_logits[i], ref["logits"][j])
        r = ref["logits"][j]
        agree = (g_logits[i].argmax(0) == r.argmax(0)).mean()
        top2 = np.sort(r, axis=0)[-2:]
        clear = (top2[1] - top2[0]) > 2 * DENSE_REL_MAX * np.abs(r).max()
        agree_clear = (g_logits[i].argmax(0) == r.argmax(0))[clear].mean()
        print(f"dense head image {i}: p4 rel err {ep:.3e}, logits rel err {el:.3e}, argmax agreement "
              f"{agree:.5f} (all pixels), {agree_clear:.5f} on the {clear.mean():.3f} of pixels whose top-2 gap "
              f"exceeds twice the tolerance")
        assert ep <= DENSE_REL_MAX, f"image {i}: projector rel err {ep:.3e}"
        assert el <= DENSE_REL_MAX, f"image {i}: logits rel err {el:.3e}"
        assert agree_clear >= 0.995, agree_clear
        assert agree >= 0.99, agree
    return n_launch


@pytest.mark.parametrize("hw_in", [None, (98, 154)])
def test_dense_head_tiny(hw_in):
    need_cuda()
    spec = S.PRESETS["tiny_s14_dense"]
    hw_in = hw_in or (spec.img_h, spec.img_w)
    w = S.make_weights(spec, 151)
    hw = S.make_dense_head_weights(spec, 152)
    im = S.make_images(spec, 2, 153, *hw_in)
    n = _check(spec, w, hw, im, [0, 1], hw_in)
    native = (hw_in[0] // 14, hw_in[1] // 14) == (spec.grid_h, spec.grid_w)
    # encoder (+ position resize) + 4 tap rows, projector 2 + 3 x 6 + 2, features 1, head 3 + 4
    assert n == (0 if native else 1) + 3 + 5 * spec.depth + 4 + 2 + 18 + 2 + 1 + 3 + 4


def test_dense_head_vits14_518():
    """The diagram's configuration: ViT-S/14 at 518 x 518, taps 3/6/9/12, 37 x 37 grid, width 256,
    19 classes, logits at 518 x 518."""
    need_cuda()
    spec = S.PRESETS["vits14_518"]
    w = S.make_weights(spec, 161)
    hw = S.make_dense_head_weights(spec, S.DENSE_SEED)
    im = S.make_images(spec, 2, 162)
    _check(spec, w, hw, im, [1], (spec.img_h, spec.img_w))


def test_dense_head_argument_errors():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s14"]                          # two taps only
    enc = V.VitEncoder(spec, S.make_weights(spec, 171), max_batch=1)
    with pytest.raises(V.VitError) as e:
        enc.set_dense_head(S.make_dense_head_weights(spec, 172))
    assert e.value.status == V.VIT_E_UNSUPPORTED
    enc.close()
    spec = S.PRESETS["tiny_s14_dense"]
    enc = V.VitEncoder(spec, S.make_weights(spec, 173), max_batch=1)
    with pytest.raises(V.VitError) as e:
        enc.dense_workspace_size(1, spec.img_h, spec.img_w)   # no head attached
    assert e.value.status == V.VIT_E_INVALID_ARG
    enc.set_dense_head(S.make_dense_head_weights(spec, 174))
    with pytest.raises(V.VitError) as e:
        enc.set_dense_head(S.make_dense_head_weights(spec, 175))
    assert e.value.status == V.VIT_E_INVALID_ARG
    enc.close()
