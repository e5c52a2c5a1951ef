"""Pins of the fp64 oracle against things other than itself: the pages' printed values,
closed forms, invariants, brute force on tiny inputs and fp64 library special cases.

Every test here runs on the CPU (no GPU marker).  The last group plants mistakes in the
oracle (monkeypatching one of its functions) and checks that some pin catches each one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
import oracle.vit_oracle as OV
import synthetic as S

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


# ------------------------------------------------------------------ independent torch composition
def torch_forward(images, weights, spec, record_hidden=False, head_blocks=None):
    """The encoder written with torch fp64 functional ops (F.conv2d, F.layer_norm, F.linear,
    F.scaled_dot_product_attention, F.gelu, F.normalize) -- shares no code with the oracle."""
    x = images.to(torch.bfloat16).double()
    W = {k: v.double() for k, v in weights.items() if k != "blocks"}
    e = F.conv2d(x, W["patch_w"], W["patch_b"], stride=spec.patch)
    B, D, gh, gw = e.shape
    if (gh, gw) != (spec.grid_h, spec.grid_w):
        start = 1 if spec.pos_on_cls else 0
        grid = W["pos"][start:].reshape(1, spec.grid_h, spec.grid_w, D).permute(0, 3, 1, 2)
        grid = F.interpolate(grid, size=(gh, gw), mode="bicubic", align_corners=False)
        W["pos"] = torch.cat([W["pos"][:start], grid.permute(0, 2, 3, 1).reshape(gh * gw, D)])
    e = e.flatten(2).transpose(1, 2)
    parts = [W["cls"].view(1, 1, D).expand(B, 1, D)]
    if spec.registers:
        parts.append(W["reg"].view(1, -1, D).expand(B, -1, D))
    if spec.pos_on_cls:
        parts[0] = parts[0] + W["pos"][0].view(1, 1, D)
        e = e + W["pos"][1:].unsqueeze(0)
    else:
        e = e + W["pos"].unsqueeze(0)
    h = torch.cat(parts + [e], dim=1)
    T = h.shape[1]
    hidden = []
    for bw in weights["blocks"]:
        h = torch_block(h, bw, spec)
        hidden.append(h.clone())
    n = F.layer_norm(h, (D,), W["norm_w"], W["norm_b"], spec.ln_eps)
    out = {"desc": F.normalize(n[:, 0], dim=-1).numpy(), "patch_tokens": n[:, 1 + spec.registers:].numpy()}
    if record_hidden:
        out["hidden"] = torch.stack(hidden).numpy()
    if head_blocks is not None:
        for bw in head_blocks:
            n = torch_block(n, bw, spec)
        out["head_tokens"] = n[:, 1 + spec.registers:].numpy()
    return out


def torch_block(h, bw, spec):
    B, T, D = h.shape
    b = {k: v.double() for k, v in bw.items()}
    u = F.layer_norm(h, (D,), b["ln1_w"], b["ln1_b"], spec.ln_eps)
    qkv = F.linear(u, b["qkv_w"], b["qkv_b"]).view(B, T, 3, spec.heads, 64).permute(2, 0, 3, 1, 4)
    o = F.scaled_dot_product_attention(qkv[0], qkv[1], qkv[2])
    o = o.transpose(1, 2).reshape(B, T, D)
    h = h + b["ls1"] * F.linear(o, b["proj_w"], b["proj_b"])
    u2 = F.layer_norm(h, (D,), b["ln2_w"], b["ln2_b"], spec.ln_eps)
    return h + b["ls2"] * F.linear(F.gelu(F.linear(u2, b["fc1_w"], b["fc1_b"])), b["fc2_w"], b["fc2_b"])


def _close(a, b, rtol=1e-9):
    a, b = np.asarray(a), np.asarray(b)
    return np.abs(a - b).max() <= rtol * max(1.0, np.abs(b).max())


# ------------------------------------------------------------------ bf16 rounding
def test_bf16_round_matches_torch_conversion():
    g = torch.Generator().manual_seed(0)
    vals = torch.cat([
        torch.randn(20000, generator=g) * 10.0 ** torch.randint(-30, 30, (20000,), generator=g).float(),
        torch.tensor([0.0, -0.0, 1.0, -1.0, 65504.0, 3.3895314e38, 1e-40, -1e-42, float("inf"), -float("inf")]),
    ])
    # exact ties: bf16 value + half an ulp, for even and odd kept mantissas
    base = torch.tensor([1.0, 1.0078125, 3.0, 3.015625], dtype=torch.float32)
    ulp = torch.tensor([2.0 ** -7, 2.0 ** -7, 2.0 ** -6, 2.0 ** -6])
    vals = torch.cat([vals, base + ulp / 2, -(base + ulp / 2)]).float()
    ours = O.bf16_round(vals.numpy())
    ref = vals.to(torch.bfloat16).double().numpy()
    assert np.array_equal(ours, ref)
    assert np.isnan(O.bf16_round(np.array([np.nan], np.float32)))[0]


def test_bf16_round_ties_to_even_by_hand():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to the even mantissa (1.0)
    assert O.bf16_round(np.float32(1 + 2 ** -8)) == 1.0
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even): rounds up
    assert O.bf16_round(np.float32(1 + 3 * 2 ** -8)) == 1 + 2 ** -6


# ------------------------------------------------------------------ patch embedding
def test_patch_embed_matches_conv2d():
    g = torch.Generator().manual_seed(1)
    for p, H, W in [(16, 48, 80), (14, 42, 28), (3, 9, 6)]:
        x = torch.randn(2, 3, H, W, generator=g, dtype=torch.float64)
        w = torch.randn(5, 3, p, p, generator=g, dtype=torch.float64)
        b = torch.randn(5, generator=g, dtype=torch.float64)
        ref = F.conv2d(x, w, b, stride=p).flatten(2).transpose(1, 2).numpy()
        ours = O.patch_embed(x.numpy(), w.numpy(), b.numpy(), p)
        assert _close(ours, ref, 1e-12)


@pytest.mark.parametrize("p,gh,gw", [(2, 2, 2), (2, 3, 2), (3, 2, 3)])
def test_patch_embed_brute_force_loops(p, gh, gw):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((1, 3, gh * p, gw * p))
    w = rng.standard_normal((4, 3, p, p))
    b = rng.standard_normal(4)
    ours = O.patch_embed(x, w, b, p)
    for gy in range(gh):
        for gx in range(gw):
            for d in range(4):
                acc = b[d]
                for c in range(3):
                    for ky in range(p):
                        for kx in range(p):
                            acc += w[d, c, ky, kx] * x[0, c, gy * p + ky, gx * p + kx]
                assert abs(ours[0, gy * gw + gx, d] - acc) < 1e-12


def test_patch_order_is_row_major():
    # a single bright pixel at patch (gy, gx) must land in token gy * gw + gx
    p, gh, gw = 4, 3, 5
    x = np.zeros((1, 3, gh * p, gw * p))
    x[0, 1, 2 * p + 1, 3 * p + 2] = 1.0
    w = np.zeros((1, 3, p, p))
    w[0, 1, 1, 2] = 1.0
    out = O.patch_embed(x, w, np.zeros(1), p)[0, :, 0]
    assert out.argmax() == 2 * gw + 3 and out.sum() == 1.0


# ------------------------------------------------------------------ tokens
def test_token_assembly_order_and_pos():
    B, P, D, R = 2, 6, 3, 4
    e = np.arange(B * P * D, dtype=np.float64).reshape(B, P, D)
    cls, reg = np.full(D, 100.0), np.arange(R * D, dtype=np.float64).reshape(R, D) + 1000
    pos = np.arange((P + 1) * D, dtype=np.float64).reshape(P + 1, D) * 0.5
    x = O.assemble_tokens(e, cls, reg, pos[1:], pos_on_cls=False)
    assert x.shape == (B, 1 + R + P, D)
    assert np.array_equal(x[:, 0], np.broadcast_to(cls, (B, D)))
    assert np.array_equal(x[:, 1:1 + R], np.broadcast_to(reg, (B, R, D)))      # no pos on registers
    assert np.array_equal(x[:, 1 + R:], e + pos[1:])
    x2 = O.assemble_tokens(e, cls, None, pos, pos_on_cls=True)
    assert np.array_equal(x2[:, 0], np.broadcast_to(cls + pos[0], (B, D)))
    assert np.array_equal(x2[:, 1:], e + pos[1:])


# ------------------------------------------------------------------ LayerNorm, GELU
def test_layer_norm_matches_torch_and_closed_form():
    g = torch.Generator().manual_seed(3)
    x = torch.randn(7, 33, generator=g, dtype=torch.float64) * 3 + 5
    gam = torch.randn(33, generator=g, dtype=torch.float64)
    bet = torch.randn(33, generator=g, dtype=torch.float64)
    ref = F.layer_norm(x, (33,), gam, bet, 1e-6).numpy()
    assert _close(O.layer_norm(x.numpy(), gam.numpy(), bet.numpy(), 1e-6), ref, 1e-12)
    # gamma = 1, beta = 0: zero mean and variance var / (var + eps) exactly
    xs = x.numpy()
    n = O.layer_norm(xs, np.ones(33), np.zeros(33), 1e-6)
    var = xs.var(axis=1)
    assert np.abs(n.mean(axis=1)).max() < 1e-14
    assert np.abs(n.var(axis=1) - var / (var + 1e-6)).max() < 1e-13
    # a row [a, b]: normalised to [-1, 1] * |a-b|/2 / sqrt(((a-b)/2)^2 + eps)
    r = O.layer_norm(np.array([[3.0, 1.0]]), np.ones(2), np.zeros(2), 0.25)
    assert _close(r, np.array([[1.0, -1.0]]) / math.sqrt(1.25), 1e-15)


def test_gelu_matches_torch_and_closed_points():
    x = torch.linspace(-12, 12, 2001, dtype=torch.float64)
    assert _close(O.gelu(x.numpy()), F.gelu(x).numpy(), 1e-14)
    assert O.gelu(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu(np.array([20.0]))[0] - 20.0) < 1e-12
    assert abs(O.gelu(np.array([-20.0]))[0]) < 1e-12
    # x * Phi(x) at x = 1: Phi(1) = 0.841344746068543 (standard normal CDF table value)
    assert abs(O.gelu(np.array([1.0]))[0] - 0.841344746068543) < 1e-12


# ------------------------------------------------------------------ attention
def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal((50, 64)) * 4, rng.standard_normal((70, 64)) * 4
    a = O.attention_probs(q, k)
    assert np.abs(a.sum(axis=1) - 1).max() < 1e-14 and (a >= 0).all()


def test_attention_uniform_when_keys_equal_and_single_token():
    rng = np.random.default_rng(5)
    D, T = 128, 9
    u = rng.standard_normal((T, D))
    w = rng.standard_normal((3 * D, D)) * 0.1
    b = rng.standard_normal(3 * D) * 0.1
    w[D:2 * D] = 0.0          # all keys equal (k = bias only) -> uniform weights
    out = O.attention(u, w, b, heads=2)
    v = u @ w[2 * D:].T + b[2 * D:]
    assert _close(out, np.broadcast_to(v.mean(axis=0), (T, D)), 1e-13)
    w1 = rng.standard_normal((3 * D, D))
    out1 = O.attention(u[:1], w1, b, heads=2)
    assert _close(out1, u[:1] @ w1[2 * D:].T + b[2 * D:], 1e-13)   # T = 1 -> o = v


def test_attention_matches_sdpa():
    g = torch.Generator().manual_seed(6)
    T, D, H = 37, 192, 3
    u = torch.randn(T, D, generator=g, dtype=torch.float64)
    w = torch.randn(3 * D, D, generator=g, dtype=torch.float64) * 0.2
    b = torch.randn(3 * D, generator=g, dtype=torch.float64)
    qkv = F.linear(u, w, b).view(T, 3, H, 64).permute(1, 2, 0, 3)
    ref = F.scaled_dot_product_attention(qkv[0], qkv[1], qkv[2]).transpose(0, 1).reshape(T, D)
    assert _close(O.attention(u.numpy(), w.numpy(), b.numpy(), H), ref.numpy(), 1e-12)


def test_block_identity_when_layer_scale_zero():
    spec = S.TINY_S16
    w = O.to_f64_weights(S.make_weights(spec, 7))
    bw = dict(w["blocks"][0])
    bw["ls1"] = np.zeros_like(bw["ls1"])
    bw["ls2"] = np.zeros_like(bw["ls2"])
    x = np.random.default_rng(7).standard_normal((spec.tokens, spec.dim))
    assert np.array_equal(O.encoder_block(x, bw, spec.heads, spec.ln_eps), x)


# ------------------------------------------------------------------ whole encoder
@pytest.mark.parametrize("name", ["tiny_s16", "tiny_s14", "small_s16"])
def test_forward_matches_torch_composition(name):
    spec = S.PRESETS[name]
    w = S.make_weights(spec, 11)
    im = S.make_images(spec, 2, 12)
    ours = O.forward(im, w, spec, record_hidden=True)
    ref = torch_forward(im, w, spec, record_hidden=True)
    assert _close(ours["hidden"], ref["hidden"], 1e-10)
    assert _close(ours["desc"], ref["desc"], 1e-10)
    assert _close(ours["patch_tokens"], ref["patch_tokens"], 1e-10)


def test_permutation_equivariance_with_pos_zero():
    spec = S.TINY_S16
    w = S.make_weights(spec, 13)
    w["pos"] = torch.zeros_like(w["pos"])
    im = S.make_images(spec, 1, 14)
    p, gh, gw = spec.patch, spec.grid_h, spec.grid_w
    perm = np.random.default_rng(15).permutation(gh * gw)
    tiles = im.view(1, 3, gh, p, gw, p).permute(0, 2, 4, 1, 3, 5).reshape(1, gh * gw, 3, p, p)
    tiles2 = tiles[:, perm]
    im2 = tiles2.reshape(1, gh, gw, 3, p, p).permute(0, 3, 1, 4, 2, 5).reshape(1, 3, gh * p, gw * p)
    a = O.forward(im, w, spec, record_hidden=True)
    b = O.forward(im2, w, spec, record_hidden=True)
    R = spec.registers
    assert _close(b["patch_tokens"][0], a["patch_tokens"][0][perm], 1e-10)
    assert _close(b["hidden"][:, 0, :1 + R], a["hidden"][:, 0, :1 + R], 1e-10)
    assert _close(b["desc"], a["desc"], 1e-10)


def test_descriptor_is_unit_cls_direction():
    spec = S.TINY_S14
    out = O.forward(S.make_images(spec, 3, 16), S.make_weights(spec, 17), spec)
    assert np.abs(np.linalg.norm(out["desc"], axis=1) - 1).max() < 1e-14
    cosv = (out["desc"] * out["cls_norm"]).sum(1) / np.linalg.norm(out["cls_norm"], axis=1)
    assert np.abs(cosv - 1).max() < 1e-14      # the card's cos(pooler, CLS) = 1.000000


def test_taps_shapes_and_content():
    spec = S.TINY_S14
    w = S.make_weights(spec, 18)
    im = S.make_images(spec, 2, 19)
    out = O.forward(im, w, spec, record_hidden=True)
    wf = O.to_f64_weights(w)
    for l in spec.taps:
        t = out["taps"][l]
        assert t.shape == (2, spec.dim, spec.grid_h, spec.grid_w)
        n = F.layer_norm(torch.from_numpy(out["hidden"][l - 1]), (spec.dim,), torch.from_numpy(wf["norm_w"]),
                         torch.from_numpy(wf["norm_b"]), spec.ln_eps).numpy()[:, 1 + spec.registers:]
        # channel d, grid (gy, gx) == token gy * gw + gx, channel d
        assert _close(t.reshape(2, spec.dim, -1).transpose(0, 2, 1), n, 1e-12)


def test_page_shapes_vits16_336_and_vits14_518():
    f = GOLDEN["vits16_336"]
    spec = S.VITS16_336
    assert (spec.img_h, spec.patch, spec.grid_h, spec.registers) == (f["input"][2], f["patch"], f["grid"], f["registers"])
    assert spec.tokens == 1 + f["registers"] + f["grid"] ** 2 == 446
    assert tuple(S.IMAGENET_MEAN) == tuple(f["imagenet_mean"]) and tuple(S.IMAGENET_STD) == tuple(f["imagenet_std"])
    g = GOLDEN["vits14_518"]
    s2 = S.VITS14_518
    assert s2.grid_h == g["conv_out"][1] and s2.n_patches == g["flatten"][0] and s2.tokens == g["tokens"][0]
    assert s2.n_pos == g["pos_embed"][0] and s2.dim == g["tokens"][1] and s2.heads == g["heads_shape"][0]
    assert s2.mlp == g["mlp_hidden"][1] and list(s2.taps) == g["taps"] and s2.ln_eps == g["ln_eps"]
    for v, (dim, depth, heads) in {"ViT-S/14": (384, 12, 6), "ViT-L/14": (1024, 24, 16)}.items():
        gv = GOLDEN["variants"][v]
        assert (gv["dim"], gv["depth"], gv["heads"]) == (dim, depth, heads)
    assert (S.VITL16_1024.dim, S.VITL16_1024.depth, S.VITL16_1024.heads) == (1024, 24, 16)


def test_vits14_518_taps_shape_from_oracle():
    # one image through the real ViT-S/14@518 shape: taps are 384 x 37 x 37 after 3/6/9/12
    spec = S.VITS14_518
    out = O.forward(S.make_images(spec, 1, 3), S.make_weights(spec, 1003), spec, n_blocks=None)
    g = GOLDEN["vits14_518"]
    assert sorted(out["taps"]) == g["taps"]
    for t in out["taps"].values():
        assert list(t.shape[1:]) == g["tap_shape"]
    assert out["patch_tokens"].shape == (1, 1369, 384)


# ------------------------------------------------------------------ attention sink (card: bf16 vs fp16)
def test_attention_sink_magnitudes_and_fp16_nan():
    spec, w, im = S.make_workload("vits16_336_b64_outlier")
    diag = {}
    wf = O.to_f64_weights(w)
    out = O.forward(im[:8], wf, spec, n_blocks=1, diag=diag, record_hidden=True)
    f = GOLDEN["bf16_vs_fp16"]
    mx = max(diag["max_abs_logit"])
    assert 2.0e6 <= mx <= f["scaled_logit_max_natural_image"]
    head0_gaps = diag["min_top_gap"][0::spec.heads]
    assert min(head0_gaps) > 1e5
    assert max(diag["max_abs_qkv"]) < f["other_tensors_below"]
    assert max(diag["max_abs_ln"]) < f["other_tensors_below"] and max(diag["max_abs_h"]) < f["other_tensors_below"]
    assert np.isfinite(out["desc"]).all() and np.abs(out["hidden"]).max() < f["other_tensors_below"]
    # fp16 logits overflow (max 65504) -> inf - inf -> NaN, as the card reports
    assert mx > f["fp16_max"]
    bad = O.forward(im[:1], wf, spec, n_blocks=1, logit_dtype=np.float16)
    assert np.isnan(bad["desc"]).all()


def test_attention_sink_full_encoder_finite():
    spec, w, im = S.make_workload("vits16_336_b64_outlier")
    out = O.forward(im[:2], w, spec)
    assert np.isfinite(out["desc"]).all() and np.isfinite(out["patch_tokens"]).all()


# ------------------------------------------------------------------ zero-shot
@pytest.mark.parametrize("h,w,oh,ow", [(24, 24, 384, 384), (5, 7, 13, 3), (3, 3, 3, 3), (4, 6, 9, 16)])
def test_bilinear_matches_interpolate(h, w, oh, ow):
    x = torch.randn(3, h, w, generator=torch.Generator().manual_seed(h * w), dtype=torch.float64)
    ref = F.interpolate(x[None], size=(oh, ow), mode="bilinear", align_corners=False)[0].numpy()
    assert _close(O.bilinear_resize(x.numpy(), oh, ow), ref, 1e-13)


def test_slide_grid_and_counts():
    f = GOLDEN["slide"]
    H, W = f["image"]
    ys, xs = O.window_origins(H, f["side"], f["stride"]), O.window_origins(W, f["side"], f["stride"])
    assert [len(ys), len(xs)] == f["windows_grid"] and len(ys) * len(xs) == f["windows"]
    assert ys == [0, 128] and xs == [0, 192, 384, 576, 640]
    c = O.overlap_counts(H, W, f["side"], f["stride"])
    # closed form: count = (#y-windows covering y) * (#x-windows covering x)
    cy = np.array([sum(y0 <= y < y0 + 384 for y0 in ys) for y in range(H)])
    cx = np.array([sum(x0 <= x < x0 + 384 for x0 in xs) for x in range(W)])
    assert np.array_equal(c, np.outer(cy, cx))
    assert c.min() == 1 and c.max() == 6 and set(np.unique(c)) == {1, 2, 3, 4, 6}


def test_slide_single_window_reduces_to_softmax_of_whole():
    rng = np.random.default_rng(20)
    C, D, g = 5, 16, 3
    toks = rng.standard_normal((1, g * g, D))
    text = O.l2_normalize(rng.standard_normal((C, D)))
    probs, lab = O.seg_slide_from_tokens(toks, text, 48, 48, 48, 24, (g, g))
    scores, lab2 = O.seg_whole_from_tokens(toks[0], text, 48, 48, (g, g))
    e = np.exp(scores - scores.max(0))
    assert _close(probs, e / e.sum(0), 1e-14) and np.array_equal(lab, lab2)


def test_slide_constant_cos_gives_uniform_probs():
    C, D, g = 7, 8, 2
    toks = np.ones((10, g * g, D))
    text = np.tile(O.l2_normalize(np.ones((1, D))), (C, 1))
    probs, lab = O.seg_slide_from_tokens(toks, text, 64, 128, 48, 24, (g, g))
    assert np.abs(probs - 1.0 / C).max() < 1e-15 and (lab == 0).all()


@pytest.mark.parametrize("H,W", [(80, 144), (80, 150)])
def test_slide_crops_are_the_windows_in_row_major_order(H, W):
    """seg_slide's crop loop against crops cut independently: torch's unfold over rows, then over
    columns, for the regular part of the grid, and explicit slicing from the right edge for the
    last, clamped column of windows.  A non-square image, so a swapped y / x or a wrong window
    order changes which pixels a window sees."""
    spec = S.PRESETS["tiny_s16"]
    side, stride = 48, 32
    w = O.to_f64_weights(S.make_weights(spec, 131))
    img = S.make_images(spec, 1, 132, H, W)[0]
    text = S.make_text_feats(3, spec.dim, 133)
    _, _, toks = O.seg_slide(img, w, spec, text, side, stride)
    ys, xs = O.window_origins(H, side, stride), O.window_origins(W, side, stride)
    assert toks.shape[0] == len(ys) * len(xs)
    grid = img.unfold(1, side, stride).unfold(2, side, stride)      # [3, nY, nX, side, side]
    for iy, y in enumerate(ys):
        for ix, x in enumerate(xs):
            if ix < grid.shape[2] and x == ix * stride:
                crop = grid[:, iy, ix]
            else:                                                   # the clamped last column
                assert x == W - side
                crop = img[:, y:y + side, W - side:]
            ref = O.forward(crop[None].contiguous(), w, spec)["patch_tokens"][0]
            assert np.array_equal(toks[iy * len(xs) + ix], ref), (iy, ix)


def test_cos_map_is_cosine():
    rng = np.random.default_rng(21)
    toks = rng.standard_normal((6, 10)) * 5
    text = O.l2_normalize(rng.standard_normal((4, 10)))
    cm = O.cos_map(toks, text, 2, 3)
    ref = torch.nn.functional.cosine_similarity(torch.from_numpy(text)[:, None, :], torch.from_numpy(toks)[None], dim=-1)
    assert _close(cm.reshape(4, 6), ref.numpy(), 1e-14)


# ------------------------------------------------------------------ position-embedding resize
@pytest.mark.parametrize("h,w,oh,ow", [(21, 21, 32, 64), (24, 24, 16, 40), (5, 7, 11, 3), (4, 4, 1, 1)])
def test_bicubic_matches_interpolate(h, w, oh, ow):
    x = torch.randn(3, h, w, generator=torch.Generator().manual_seed(h + w), dtype=torch.float64)
    ref = F.interpolate(x[None], size=(oh, ow), mode="bicubic", align_corners=False)[0].numpy()
    assert _close(O.bicubic_resize(x.numpy(), oh, ow), ref, 1e-13)


def test_bicubic_identity_at_native_grid():
    # "DINOv2 n semantic" diagram: "Bicubic interpolation, 37x37 unchanged"
    g = GOLDEN["vits14_518"]["conv_out"][1]
    x = np.random.default_rng(30).standard_normal((5, g, g))
    assert np.array_equal(O.bicubic_resize(x, g, g), x)
    pos = np.random.default_rng(31).standard_normal((1 + g * g, 8))
    assert np.array_equal(O.resize_pos_embed(pos, (g, g), (g, g), True), pos)


def test_resize_keeps_cls_row_and_constant_fields():
    pos = np.random.default_rng(32).standard_normal((1 + 6 * 6, 4))
    pos[1:] = 2.5                                   # a constant grid stays constant (weights sum to 1)
    r = O.resize_pos_embed(pos, (6, 6), (9, 4), pos_on_cls=True)
    assert r.shape == (1 + 36, 4) and np.array_equal(r[0], pos[0]) and np.abs(r[1:] - 2.5).max() < 1e-14


@pytest.mark.parametrize("name,hw", [("tiny_s16", (128, 128)), ("tiny_s14", (98, 154))])
def test_forward_at_other_sizes_matches_torch_composition(name, hw):
    spec = S.PRESETS[name]
    w = S.make_weights(spec, 33)
    im = S.make_images(spec, 2, 34, *hw)
    ours = O.forward(im, w, spec, record_hidden=True)
    ref = torch_forward(im, w, spec, record_hidden=True)
    assert _close(ours["hidden"], ref["hidden"], 1e-10) and _close(ours["desc"], ref["desc"], 1e-10)


def test_planted_cubic_coefficient_mistake_is_caught(monkeypatch):
    # a = -0.5 (Catmull-Rom) instead of the -0.75 kernel: a plausible slip the pin must see
    orig = OV._cubic_weights
    x = np.random.default_rng(35).standard_normal((2, 21, 21))
    ref = F.interpolate(torch.from_numpy(x)[None], size=(32, 64), mode="bicubic", align_corners=False)[0].numpy()
    monkeypatch.setattr(OV, "_cubic_weights", lambda t, a=-0.5: orig(t, -0.5))
    assert not _close(OV.bicubic_resize(x, 32, 64), ref, 1e-6)


# ------------------------------------------------------------------ dino.txt vision head
@pytest.mark.parametrize("name,hw", [("tiny_s16", None), ("tiny_s14", (98, 154))])
def test_text_head_matches_torch_composition(name, hw):
    spec = S.PRESETS[name]
    w = S.make_weights(spec, 41)
    head = S.make_head_weights(spec, 42)
    im = S.make_images(spec, 2, 43, *(hw or (spec.img_h, spec.img_w)))
    o = O.forward(im, w, spec)
    ours = O.text_head(o["final_tokens"], head, spec)
    ref = torch_forward(im, w, spec, head_blocks=head)["head_tokens"]
    assert len(head) == 2 and ours.shape == ref.shape == o["patch_tokens"].shape
    assert _close(ours, ref, 1e-10)


def test_text_head_with_zero_layer_scale_is_the_identity():
    spec = S.PRESETS["tiny_s16"]
    w = S.make_weights(spec, 44)
    head = S.make_head_weights(spec, 45)
    for b in head:
        b["ls1"] = torch.zeros_like(b["ls1"])
        b["ls2"] = torch.zeros_like(b["ls2"])
    o = O.forward(S.make_images(spec, 1, 46), w, spec)
    assert np.array_equal(O.text_head(o["final_tokens"], head, spec), o["patch_tokens"])


def test_seg_whole_with_head_uses_head_tokens():
    spec = S.PRESETS["tiny_s16"]
    w = S.make_weights(spec, 47)
    head = S.make_head_weights(spec, 48)
    im = S.make_images(spec, 1, 49)[0]
    text = S.make_text_feats(7, spec.dim, 50)
    scores, labels, tok = O.seg_whole(im, w, spec, text, head_blocks=head)
    ref = torch_forward(im[None], w, spec, head_blocks=head)["head_tokens"][0]
    assert _close(tok, ref, 1e-10)
    t = ref / np.linalg.norm(ref, axis=1, keepdims=True)
    cos = (text.double().numpy() @ t.T).reshape(7, spec.grid_h, spec.grid_w)
    up = F.interpolate(torch.from_numpy(cos)[None], size=(spec.img_h, spec.img_w), mode="bilinear",
                       align_corners=False)[0].numpy()
    assert _close(scores, up, 1e-10) and np.array_equal(labels, up.argmax(0))


# ------------------------------------------------------------------ dense head on the taps
def torch_dense_head(taps, hw, layers, out_hw):
    """The projector and task head with torch fp64 ops (F.conv2d, F.layer_norm over channels,
    F.silu, F.group_norm, F.gelu, F.interpolate) -- shares no code with the oracle."""
    W = {k: ([t.double() for t in v] if isinstance(v, list) else v.double()) for k, v in hw.items()}

    def cln(x, g, b):
        return F.layer_norm(x.permute(0, 2, 3, 1), (x.shape[1],), g, b, 1e-6).permute(0, 3, 1, 2)

    def cls_(x, w, g, b, pad):
        return F.silu(cln(F.conv2d(x, w, padding=pad), g, b))

    x = torch.cat([torch.from_numpy(taps[l]) for l in layers], dim=1)
    y = cls_(x, W["cv1_w"], W["cv1_ln_w"], W["cv1_ln_b"], 0)
    a, b = y.chunk(2, dim=1)
    outs, cur = [a, b], b
    for i in range(3):
        cur = cls_(cur, W["bn_w"][2 * i], W["bn_ln_w"][2 * i], W["bn_ln_b"][2 * i], 1)
        cur = cls_(cur, W["bn_w"][2 * i + 1], W["bn_ln_w"][2 * i + 1], W["bn_ln_b"][2 * i + 1], 1)
        outs.append(cur)
    z = cls_(torch.cat(outs, dim=1), W["cv2_w"], W["cv2_ln_w"], W["cv2_ln_b"], 0)
    p4 = cln(z, W["out_ln_w"], W["out_ln_b"])
    h = F.conv2d(F.conv2d(p4, W["lat_w"], W["lat_b"]), W["smooth_w"], W["smooth_b"], padding=1)
    h = F.gelu(F.group_norm(h, 32, W["gn_w"], W["gn_b"], 1e-5))
    logits = F.interpolate(F.conv2d(h, W["pred_w"], W["pred_b"]), size=out_hw, mode="bilinear", align_corners=False)
    return p4.numpy(), logits.numpy()


def test_dense_head_matches_torch_composition():
    spec = S.PRESETS["tiny_s14_dense"]
    w = S.make_weights(spec, 51)
    hw = S.make_dense_head_weights(spec, 52)
    im = S.make_images(spec, 2, 53)
    o = O.forward(im, w, spec)
    layers = list(spec.taps)
    assert len(layers) == 4
    out = O.dense_head(o["taps"], hw, spec, (spec.img_h, spec.img_w))
    p4, logits = torch_dense_head(o["taps"], hw, layers, (spec.img_h, spec.img_w))
    assert out["logits"].shape == (2, 19, spec.img_h, spec.img_w)
    assert _close(out["p4"], p4, 1e-10) and _close(out["logits"], logits, 1e-10)


def test_conv2d_matches_brute_force_loops():
    rng = np.random.default_rng(54)
    x, w, b = rng.standard_normal((3, 5, 4)), rng.standard_normal((2, 3, 3, 3)), rng.standard_normal(2)
    ref = np.zeros((2, 5, 4))
    for o in range(2):
        for y in range(5):
            for xx in range(4):
                acc = b[o]
                for c in range(3):
                    for ky in range(3):
                        for kx in range(3):
                            yy, xs = y + ky - 1, xx + kx - 1
                            if 0 <= yy < 5 and 0 <= xs < 4:
                                acc += w[o, c, ky, kx] * x[c, yy, xs]
                ref[o, y, xx] = acc
    assert _close(O.conv2d(x, w, b, 1), ref, 1e-12)


def test_group_norm_and_channel_ln_special_cases():
    rng = np.random.default_rng(55)
    x = rng.standard_normal((8, 3, 5))
    one = np.ones(8)
    zero = np.zeros(8)
    # GroupNorm with one group per channel is instance norm; with one group, LayerNorm over (C, H, W)
    inst = (x - x.mean(axis=(1, 2), keepdims=True)) / np.sqrt(x.var(axis=(1, 2), keepdims=True) + 1e-5)
    assert _close(O.group_norm(x, 8, one, zero), inst, 1e-12)
    whole = (x - x.mean()) / np.sqrt(x.var() + 1e-5)
    assert _close(O.group_norm(x, 1, one, zero), whole, 1e-12)
    cl = O.channel_layer_norm(x, one, zero)
    assert np.abs(cl.mean(axis=0)).max() < 1e-12 and np.abs((cl ** 2).mean(axis=0) - 1).max() < 1e-5
    assert _close(O.silu(np.array([0.0, 1.0, -2.0])), np.array([0.0, 1 / (1 + np.exp(-1)), -2 / (1 + np.exp(2))]), 1e-15)


def test_planted_bottleneck_shortcut_is_caught(monkeypatch):
    # a residual inside the bottleneck (the C2f variant the diagram rules out) must not pass
    spec = S.PRESETS["tiny_s14_dense"]
    w = S.make_weights(spec, 56)
    hw = S.make_dense_head_weights(spec, 57)
    o = O.forward(S.make_images(spec, 1, 58), w, spec)
    p4, _ = torch_dense_head(o["taps"], hw, list(spec.taps), (spec.img_h, spec.img_w))
    orig = OV._conv_ln_silu
    calls = {"n": 0}

    def with_shortcut(x, wt, g, b, pad):
        y = orig(x, wt, g, b, pad)
        calls["n"] += 1
        return y + x if (pad == 1 and calls["n"] % 2 == 0) else y
    monkeypatch.setattr(OV, "_conv_ln_silu", with_shortcut)
    bad = O.dense_head(o["taps"], hw, spec, (spec.img_h, spec.img_w))["p4"]
    assert not _close(bad, p4, 1e-6)


# ------------------------------------------------------------------ planted mistakes
def _mut_gelu_tanh(x):
    return 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))


def _mut_ln_unbiased(x, g, b, eps):
    mu = x.mean(-1, keepdims=True)
    return (x - mu) / np.sqrt(x.var(-1, ddof=1, keepdims=True) + eps) * g + b


def _mut_probs_wrong_scale(q, k, logit_dtype=None):
    s = (q @ k.T) / math.sqrt(q.shape[-1] * 2)
    s = s - s.max(1, keepdims=True)
    a = np.exp(s)
    return a / a.sum(1, keepdims=True)


def _mut_bilinear_align(img, oh, ow):
    return F.interpolate(torch.from_numpy(img)[None], size=(oh, ow), mode="bilinear", align_corners=True)[0].numpy()


@pytest.mark.parametrize("fname", ["gelu", "layer_norm", "attention_probs", "patch_embed", "assemble_tokens"])
def test_planted_mistake_is_caught(monkeypatch, fname):
    spec = S.TINY_S16
    w = S.make_weights(spec, 22)
    im = S.make_images(spec, 1, 23)
    ref = torch_forward(im, w, spec)
    orig = getattr(OV, fname)
    muts = {
        "gelu": _mut_gelu_tanh,
        "layer_norm": _mut_ln_unbiased,
        "attention_probs": _mut_probs_wrong_scale,
        "patch_embed": lambda xb, wt, b, p: orig(xb, wt.transpose(0, 1, 3, 2), b, p),
        "assemble_tokens": lambda e, cls, reg, pos, poc: orig(e, cls, reg, np.roll(pos, 1, axis=0), poc),
    }
    monkeypatch.setattr(OV, fname, muts[fname])
    bad = OV.forward(im, w, spec)
    assert not _close(bad["patch_tokens"], ref["patch_tokens"], 1e-6)


def test_planted_bilinear_mistake_is_caught(monkeypatch):
    x = np.random.default_rng(24).standard_normal((2, 24, 24))
    ref = F.interpolate(torch.from_numpy(x)[None], size=(384, 384), mode="bilinear", align_corners=False)[0].numpy()
    monkeypatch.setattr(OV, "bilinear_resize", _mut_bilinear_align)
    assert not _close(OV.bilinear_resize(x, 384, 384), ref, 1e-6)
