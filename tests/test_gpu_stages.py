"""Stage-level parity of the hot kernels through the C ABI (vit_stage_linear,
vit_stage_attention) against the fp64 oracle's building blocks on the same bf16 inputs."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import gpu, need_cuda

pytestmark = gpu


def _ref_linear(A, W, b, gelu):
    r = A.double().numpy() @ W.double().numpy().T + b.double().numpy()
    return O.gelu(r) if gelu else r


@pytest.mark.parametrize("M,N,K,gelu", [
    (1, 128, 64, False),        # one row, one tile
    (129, 384, 384, False),     # ragged second M tile
    (446, 1152, 384, False),    # ViT-S/16 QKV shape
    (446, 1536, 384, True),     # ViT-S/16 FC1 with GELU
    (1000, 1024, 4096, False),  # long K (FC2-like), ragged M
    (5000, 4096, 1024, True),   # paired 256 x 256 tiles (2-CTA clusters), GELU
    (20000, 1024, 1024, False), # paired tiles; last tile: 32 rows on the first CTA, none on the second
    (10184, 3072, 1024, False), # paired tiles; last tile: 256 + 72 rows
    (4096, 768, 3072, False),   # paired tiles, N = 3 x 256, long K
    (28544, 1152, 384, False),  # ViT-S/16@336 b64 QKV: paired tiles, last column tile padded
    (10000, 384, 1536, True),   # padded paired tiles, long K, GELU; last row tile: 16 rows
    (9500, 640, 512, False),    # padded paired tiles, N = 2 x 256 + 128; last row tile: 28 rows
])
def test_linear_matches_oracle(M, N, K, gelu):
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    A = S.make_matrix((M, K), 1 + M, 1.0)
    W = S.make_matrix((N, K), 2 + N, 1.0 / math.sqrt(K))
    b = S.make_matrix((N,), 3, 0.5, torch.float32)
    out, st = V.stage_linear(A.cuda(), W.cuda(), b.cuda(), gelu=gelu)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g = out.double().cpu().numpy()
    r = _ref_linear(A, W, b, gelu)
    assert np.isfinite(g).all()
    err = np.abs(g - r).max()
    assert err <= 6e-3 * np.abs(r).max() + 1e-3, err


def _ref_attention(qkv, heads):
    B, T, _ = qkv.shape
    D = heads * 64
    x = qkv.double().numpy()
    out = np.empty((B, T, D))
    for b in range(B):
        for h in range(heads):
            q = x[b, :, h * 64:(h + 1) * 64]
            k = x[b, :, D + h * 64:D + (h + 1) * 64]
            v = x[b, :, 2 * D + h * 64:2 * D + (h + 1) * 64]
            out[b, :, h * 64:(h + 1) * 64] = O.attention_probs(q, k) @ v
    return out


@pytest.mark.parametrize("B,T,heads,qk_scale", [
    (1, 1, 1, 1.0),       # a single key: output = v
    (2, 65, 2, 1.0),      # one ragged KV tile
    (1, 129, 1, 3.0),     # two KV tiles, the second with one key; sharper softmax
    (1, 446, 6, 1.0),     # ViT-S/16@336 tokens
    (2, 1370, 6, 2.0),    # ViT-S/14@518 tokens
    (1, 4101, 2, 1.0),    # ViT-L/16@1024 tokens (two heads)
    (8, 1370, 6, 1.0),    # ViT-S/14@518 batch 8: a grid of several waves
])
def test_attention_matches_oracle(B, T, heads, qk_scale):
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    D = heads * 64
    qkv = S.make_matrix((B, T, 3 * D), 10 + T, 1.0).float()
    qkv[..., :2 * D] *= qk_scale
    qkv = qkv.to(torch.bfloat16)
    out, st = V.stage_attention(qkv.cuda(), heads)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g = out.double().cpu().numpy()
    r = _ref_attention(qkv, heads)
    assert np.isfinite(g).all()
    err = np.abs(g - r).max()
    assert err <= 1e-2 * np.abs(r).max() + 2e-3, err


def test_attention_long_sequence_sampled_rows():
    """16,389 tokens (ViT-S/16 at 2048 x 2048: 129 key blocks, a ragged last one): sampled query
    rows of every head against fp64 softmax(q K^T / 8) V computed row by row."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    B, T, heads = 1, 16389, 2
    D = heads * 64
    qkv = S.make_matrix((B, T, 3 * D), 2048, 1.0).to(torch.bfloat16)
    out, st = V.stage_attention(qkv.cuda(), heads)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g = out.double().cpu().numpy()[0]
    x = qkv.double().numpy()[0]
    rows = np.random.default_rng(7).choice(T, 48, replace=False).tolist() + [0, 127, 128, T - 5, T - 1]
    for h in range(heads):
        k = x[:, D + 64 * h:D + 64 * (h + 1)]
        v = x[:, 2 * D + 64 * h:2 * D + 64 * (h + 1)]
        for t in rows:
            q = x[t, 64 * h:64 * (h + 1)]
            a = O.attention_probs(q[None], k)[0]
            ref = a @ v
            err = np.abs(g[t, 64 * h:64 * (h + 1)] - ref).max()
            assert err <= 1e-2 * np.abs(ref).max() + 2e-3, (h, t, err)


def test_attention_huge_logits_stay_finite():
    """kornia/dinov3 card, "Build BF16, not FP16": scaled logits of ~2e6 must not overflow."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    B, T, heads = 1, 300, 1
    D = 64
    qkv = S.make_matrix((B, T, 3 * D), 99, 0.5).float()
    # every query has 1500 on the first 8 dims; key 1 has 1470 there: logit 8*1500*1470/8 = 2.2e6
    qkv[0, :, 0:8] = 1500.0
    qkv[0, 1, D:D + 8] = 1470.0
    qkv = qkv.to(torch.bfloat16)
    out, st = V.stage_attention(qkv.cuda(), heads)
    torch.cuda.synchronize()
    g = out.double().cpu().numpy()
    r = _ref_attention(qkv, heads)
    assert np.isfinite(g).all() and int(st.item()) == 0
    assert np.abs(g - r).max() <= 1e-2 * np.abs(r).max() + 2e-3
    # the sink takes all the weight: every row equals v of key 1
    assert np.abs(g[0] - qkv[0, 1, 2 * D:].double().numpy()).max() < 1e-2


def test_gelu_formula_against_exact_erf():
    """The epilogue's GELU (Abramowitz & Stegun 7.1.28 erf) against the exact erf form in fp64:
    the formula's error (at most 1.5e-7 |x|) plus single-precision evaluation (one reciprocal,
    four squarings, the fp32 result) stays within 3e-7 |x| + 5e-7 over [-12, 12]; exact signs
    and limits far out.  bf16 outputs resolve 3.9e-3 relative, four orders coarser."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    x = torch.linspace(-12, 12, 2_000_001, dtype=torch.float32)
    x = torch.cat([x, torch.tensor([0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0, 3e38, -3e38])])
    y = V.stage_gelu(x.cuda())
    torch.cuda.synchronize()
    xd = x.double().numpy()
    ref = O.gelu(xd)
    err = np.abs(y.double().cpu().numpy() - ref)
    assert np.isfinite(y.cpu().numpy()).all()
    assert (err <= 3e-7 * np.abs(xd) + 5e-7).all(), err.max()
    yl, rl = y.cpu().numpy()[-6:], ref[-6:]            # 1e-30, -1e-30, 40, -40, 3e38, -3e38
    assert yl[2] == 40.0 and yl[3] == 0.0 and yl[4] == np.float32(3e38) and yl[5] == 0.0 and abs(yl[0] - rl[0]) < 1e-37

