"""Inputs at sizes other than the one the position embedding was learned for ([diagram]
"DINOv2-S encoder": the learned grid goes through "Bicubic interpolation" to the input's patch
grid): the resize kernel alone, the whole forward (vit_forward_hw) and zero-shot scoring at
such sizes, each against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import ARGMAX_AGREE_MIN, BLOCK_REL_MAX, assert_forward_parity, gpu, need_cuda

pytestmark = gpu


@pytest.mark.parametrize("grid0,grid,cls", [((24, 24), (32, 48), True), ((37, 37), (16, 40), False),
                                            ((6, 10), (8, 8), True), ((5, 7), (1, 1), False), ((14, 14), (14, 14), True)])
def test_pos_resize_stage(grid0, grid, cls):
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    D = 192
    rows0 = (1 if cls else 0) + grid0[0] * grid0[1]
    pos = torch.randn(rows0, D, generator=torch.Generator().manual_seed(sum(grid0) + sum(grid)), dtype=torch.float32)
    out = V.stage_pos_resize(pos.cuda(), grid0, grid, cls)
    torch.cuda.synchronize()
    ref = O.resize_pos_embed(pos.double().numpy(), grid0, grid, cls)
    # fp32 weights and sums of 16 taps: a few ulps of the O(1) inputs
    assert np.abs(out.double().cpu().numpy() - ref).max() < 2e-5


@pytest.mark.parametrize("name,hw,batch", [("tiny_s16", (128, 128), 2),     # 6x10 grid -> 8x8
                                           ("tiny_s16", (16, 16), 3),       # one patch: T = 1 + R + 1
                                           ("tiny_s16", (31, 400), 2),      # 1 x 25 grid, ragged pixels
                                           ("tiny_s14", (98, 154), 3),      # 9x9 -> 7x11
                                           ("tiny_s16", (100, 170), 2),     # floor grid 6x10: the native one
                                           ("small_s16", (288, 160), 2)])   # 14x14 -> 18x10
def test_forward_at_other_sizes(name, hw, batch):
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS[name]
    w = S.make_weights(spec, 91)
    im = S.make_images(spec, batch, 92, *hw)
    enc = V.VitEncoder(spec, w, max_batch=batch)
    outs = enc.forward(im.cuda().contiguous(), desc=True, patch=True, patch_fp32=True, taps=bool(spec.taps),
                       hidden=True)
    torch.cuda.synchronize()
    enc.poll()
    launches = enc.last_launch_count()
    gh, gw = hw[0] // spec.patch, hw[1] // spec.patch
    native = (gh, gw) == (spec.grid_h, spec.grid_w)
    assert outs["patch_tokens"].shape == (batch, gh * gw, spec.dim)
    assert launches == (0 if native else 1) + 3 + 5 * spec.depth + len(spec.taps) + 1
    g = {k: ([t.double().cpu().numpy() for t in v] if isinstance(v, list) else v.double().cpu().numpy())
         for k, v in outs.items()}
    ref = O.forward(im, w, spec, record_hidden=True)
    assert ref["grid"] == (gh, gw)
    assert_forward_parity(g, ref, spec, list(range(batch)))
    enc.close()


def test_vits14_518_weights_at_448x672():
    """The native-size preset of the taps workload on a 32 x 48 grid (1,541 tokens)."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["vits14_518"]
    w = S.make_weights(spec, 93)
    im = S.make_images(spec, 2, 94, 448, 672)
    enc = V.VitEncoder(spec, w, max_batch=2)
    outs = enc.forward(im.cuda().contiguous(), desc=True, patch=True, patch_fp32=True, taps=True, hidden=True)
    torch.cuda.synchronize()
    enc.poll()
    g = {k: ([t.double().cpu().numpy() for t in v] if isinstance(v, list) else v.double().cpu().numpy())
         for k, v in outs.items()}
    ref = O.forward(im[:1], w, spec, record_hidden=True)
    assert_forward_parity(g, ref, spec, [0])
    enc.close()


def test_hw_matches_native_entry_point_at_native_size():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s16"]
    w = S.make_weights(spec, 95)
    im = S.make_images(spec, 2, 96).cuda()
    enc = V.VitEncoder(spec, w, max_batch=2)
    a = enc.forward(im, patch=True)
    b = enc.alloc_outputs(2, patch=True)
    o = V.VitOutputs()
    o.desc, o.patch_tokens = V._ptr(b["desc"]), V._ptr(b["patch_tokens"])
    ws = torch.empty(enc.workspace_size(2, (spec.img_h, spec.img_w)) + 4096, dtype=torch.uint8, device="cuda")
    V._check("vit_forward_hw", enc.lib.vit_forward_hw(enc.handle, V._ptr(im), 2, spec.img_h, spec.img_w,
                                                      V.ctypes.byref(o), V._ptr(ws), ws.numel(), None))
    torch.cuda.synchronize()
    enc.poll()
    assert torch.equal(a["desc"], b["desc"]) and torch.equal(a["patch_tokens"], b["patch_tokens"])
    enc.close()


def test_forward_hw_rejects_bad_sizes():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s16"]
    enc = V.VitEncoder(spec, S.make_weights(spec, 97), max_batch=2)
    for hw in [(8, 160), (96, 15), (20000, 64)]:
        with pytest.raises(V.VitError) as e:
            enc.workspace_size(1, hw)
        assert e.value.status == V.VIT_E_SHAPE
    enc.close()


def test_seg_whole_at_other_size():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]
    w = S.make_weights(spec, 101)
    H, W = 320, 480                                      # 20 x 30 grid from a 14 x 14 position grid
    im = S.make_images(spec, 1, 102, H, W)
    text = S.make_text_feats(20, spec.dim, 103)
    enc = V.VitEncoder(spec, w, max_batch=1)
    scores, labels = enc.seg(im[0].cuda(), text.cuda(), mode=V.VIT_SEG_WHOLE)
    torch.cuda.synchronize()
    enc.poll()
    ref = O.forward(im, w, spec)
    rs, rl = O.seg_whole_from_tokens(ref["patch_tokens"][0], text.double().numpy(), H, W, ref["grid"])
    assert np.abs(scores.double().cpu().numpy() - rs).max() < 2e-3
    assert (labels.cpu().numpy() == rl).mean() >= ARGMAX_AGREE_MIN
    enc.close()


def test_seg_slide_with_windows_of_another_size():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]                        # learned for 224; windows of 160 (10 x 10 grid)
    w = S.make_weights(spec, 111)
    H, W, side, stride = 256, 400, 160, 96
    im = S.make_images(spec, 1, 112, H, W)[0]
    text = S.make_text_feats(12, spec.dim, 113)
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
    enc.close()
