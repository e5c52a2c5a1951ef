"""Guard bands around every buffer the library is handed (the stand-in for a memory checker,
which is closed on this machine): the workspace and each output sit inside a larger allocation
whose head and tail are filled with a known pattern, and after the call the pattern must be
intact -- no kernel writes outside the buffers it was given, at sizes with ragged tiles, with
paired tiles, at other input sizes, in the zero-shot scoring and in the dense head."""
import numpy as np
import pytest
import torch

import synthetic as S
from parity import gpu, need_cuda

pytestmark = gpu

GUARD = 64 * 1024          # bytes of guard on each side (a multiple of 1024: alignment is kept)
PATTERN = 0xA5


def _guarded(nbytes):
    """(whole uint8 buffer, inner uint8 view of nbytes) with the guards filled."""
    whole = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    return whole, whole[GUARD:GUARD + nbytes]


def _guarded_like(shape, dtype):
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    whole, inner = _guarded(n)
    return whole, inner.view(dtype).view(*shape)


def _intact(whole, nbytes):
    head = whole[:GUARD]
    tail = whole[GUARD + nbytes:]
    return bool((head == PATTERN).all().item()) and bool((tail == PATTERN).all().item())


@pytest.mark.parametrize("name,B,hw", [("small_s16", 3, None), ("tiny_s14", 2, None), ("vitb14_224", 64, None),
                                      ("small_s16", 2, (288, 160))])
def test_forward_writes_only_its_buffers(name, B, hw):
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS[name]
    hw = hw or (spec.img_h, spec.img_w)
    enc = V.VitEncoder(spec, S.make_weights(spec, 141), max_batch=B)
    im = S.make_images(spec, B, 142, *hw).cuda()
    gh, gw = hw[0] // spec.patch, hw[1] // spec.patch
    T = 1 + spec.registers + gh * gw
    bufs = {"desc": _guarded_like((B, spec.dim), torch.float32),
            "patch_tokens": _guarded_like((B, gh * gw, spec.dim), torch.bfloat16),
            "hidden": _guarded_like((spec.depth, B, T, spec.dim), torch.float32)}
    outs = {k: v[1] for k, v in bufs.items()}
    if spec.taps:
        taps = [_guarded_like((B, spec.dim, gh, gw), torch.float32) for _ in spec.taps]
        outs["taps"] = [t[1] for t in taps]
    need = enc.workspace_size(B, hw)
    ws_whole, ws = _guarded(need)
    enc.forward_into(im, outs, ws=ws)
    torch.cuda.synchronize()
    enc.poll()
    assert _intact(ws_whole, need), "workspace guard"
    for k, (whole, t) in bufs.items():
        assert _intact(whole, t.numel() * t.element_size()), f"{k} guard"
    for i, (whole, t) in enumerate(taps if spec.taps else []):
        assert _intact(whole, t.numel() * 4), f"tap {i} guard"
    enc.close()


@pytest.mark.parametrize("mode", ["whole", "slide"])
def test_zero_shot_writes_only_its_buffers(mode):
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s16"]
    H, W, side, stride, C = 80, 150, 48, 32, 19
    enc = V.VitEncoder(spec, S.make_weights(spec, 143), max_batch=12)
    enc.set_text_head(S.make_head_weights(spec, 144))
    img = S.make_images(spec, 1, 145, H, W)[0].cuda().contiguous()
    text = S.make_text_feats(C, spec.dim, 146).cuda()
    m = V.VIT_SEG_SLIDE if mode == "slide" else V.VIT_SEG_WHOLE
    need = enc.seg_workspace_size(H, W, C, m, side, stride)
    ws_whole, ws = _guarded(need)
    pw, probs = _guarded_like((C, H, W), torch.float32)
    lw, labels = _guarded_like((H, W), torch.int32)
    st = enc.lib.vit_seg_zero_shot(enc.handle, img.data_ptr(), H, W, text.data_ptr(), C, m, side, stride,
                                   probs.data_ptr(), labels.data_ptr(), ws.data_ptr(), need, None)
    assert st == V.VIT_OK, enc.lib.vit_last_error()
    torch.cuda.synchronize()
    enc.poll()
    assert _intact(ws_whole, need) and _intact(pw, probs.numel() * 4) and _intact(lw, labels.numel() * 4)
    assert int(labels.min()) >= 0 and int(labels.max()) < C
    enc.close()


def test_dense_head_writes_only_its_buffers():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s14_dense"]
    B = 2
    enc = V.VitEncoder(spec, S.make_weights(spec, 147), max_batch=B)
    enc.set_dense_head(S.make_dense_head_weights(spec, 148))
    im = S.make_images(spec, B, 149).cuda().contiguous()
    need = enc.dense_workspace_size(B, spec.img_h, spec.img_w)
    ws_whole, ws = _guarded(need)
    K = S.DENSE_CLASSES
    gh, gw = spec.grid_h, spec.grid_w
    lw, logits = _guarded_like((B, K, spec.img_h, spec.img_w), torch.float32)
    fw, p4 = _guarded_like((B, S.DENSE_WIDTH, gh, gw), torch.float32)
    st = enc.lib.vit_forward_dense(enc.handle, im.data_ptr(), B, spec.img_h, spec.img_w, logits.data_ptr(),
                                   p4.data_ptr(), ws.data_ptr(), need, None)
    assert st == V.VIT_OK, enc.lib.vit_last_error()
    torch.cuda.synchronize()
    enc.poll()
    assert _intact(ws_whole, need) and _intact(lw, logits.numel() * 4) and _intact(fw, p4.numel() * 4)
    enc.close()
