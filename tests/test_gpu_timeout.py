"""Failure detection without a GPU fault.  Every pipeline wait of the tensor-core kernels is
bounded; a wait that runs out makes its kernel record a status code, let the copies and MMAs it
has in flight land, free its tensor memory and return, and the kernels after it on the same
status word return without work.  These tests shorten the limit (a kernel argument, 2 s by
default) to a few hundred nanoseconds, far below any pipeline's latency, so that the waits run
out on purpose; they check the reported code and that the next call with the default limit is
correct.  Nothing traps and no memory outside the buffers is touched."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from parity import assert_forward_parity, gpu, need_cuda

pytestmark = gpu

SHORT_NS = 200


def test_forward_wait_expiry_is_reported_and_the_model_recovers():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["tiny_s16"]
    w = S.make_weights(spec, 111)
    im = S.make_images(spec, 2, 112)
    enc = V.VitEncoder(spec, w, max_batch=2)
    x = im.cuda()
    clean = enc.forward(x, desc=True, patch=True, patch_fp32=True)
    enc.poll()
    enc.set_wait_limit(SHORT_NS)
    enc.forward(x, desc=True, patch=True, patch_fp32=True)
    with pytest.raises(V.VitError) as e:
        enc.poll()
    assert e.value.status == V.VIT_E_DEVICE_TIMEOUT
    assert b"pipeline wait" in enc.lib.vit_last_error()
    enc.poll()                                   # the word was cleared by the poll that reported it
    enc.set_wait_limit(0)
    again = enc.forward(x, desc=True, patch=True, patch_fp32=True, hidden=True)
    enc.poll()
    assert torch.equal(again["desc"], clean["desc"]) and torch.equal(again["patch_tokens"], clean["patch_tokens"])
    g = {k: (v.double().cpu().numpy() if torch.is_tensor(v) else v) for k, v in again.items()}
    ref = O.forward(im, w, spec, record_hidden=True)
    assert_forward_parity(g, ref, spec, [0, 1])
    enc.close()


@pytest.mark.parametrize("M,N,K", [
    (300, 256, 128),     # single-CTA tiles
    (8192, 2048, 256),   # paired 256 x 256 tiles (2-CTA clusters)
])
def test_stage_linear_wait_expiry(M, N, K):
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    A = S.make_matrix((M, K), 5 + M, 1.0).cuda()
    W = S.make_matrix((N, K), 6 + N, 1.0 / math.sqrt(K)).cuda()
    b = S.make_matrix((N,), 7, 0.5, torch.float32).cuda()
    out, st = V.stage_linear(A, W, b, wait_ns=SHORT_NS)
    torch.cuda.synchronize()
    code = int(st.item())
    assert 0x100 < code < 0x200, hex(code)       # a GEMM wait site
    st.zero_()
    out, st = V.stage_linear(A, W, b, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    r = A.double() @ W.double().T + b.double()
    err = (out.double() - r).abs().max().item()
    assert err <= 6e-3 * r.abs().max().item() + 1e-3, err


def test_stage_attention_wait_expiry():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    B, T, heads = 2, 300, 2
    D = 64 * heads
    qkv = S.make_matrix((B, T, 3 * D), 113, 1.0).cuda()
    out, st = V.stage_attention(qkv, heads, wait_ns=SHORT_NS)
    torch.cuda.synchronize()
    code = int(st.item())
    assert 0x200 < code < 0x300, hex(code)       # an attention wait site
    st.zero_()
    out, st = V.stage_attention(qkv, heads, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x = qkv.double().cpu().numpy()
    g = out.double().cpu().numpy()
    for bi in range(B):
        for h in range(heads):
            q = x[bi, :, 64 * h:64 * (h + 1)]
            k = x[bi, :, D + 64 * h:D + 64 * (h + 1)]
            v = x[bi, :, 2 * D + 64 * h:2 * D + 64 * (h + 1)]
            ref = O.attention_probs(q, k) @ v
            err = np.abs(g[bi, :, 64 * h:64 * (h + 1)] - ref).max()
            assert err <= 1e-2 * np.abs(ref).max() + 2e-3, (bi, h, err)


def test_stage_attention_wait_expiry_full_grid():
    """The same expiry on a grid of several waves (ViT-S/14@518 batch 8, two CTAs per SM); the
    next call with the default limit is compared with the oracle on sampled rows."""
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    B, T, heads = 8, 1370, 6
    D = 64 * heads
    qkv = S.make_matrix((B, T, 3 * D), 117, 1.0).cuda()
    out, st = V.stage_attention(qkv, heads, wait_ns=SHORT_NS)
    torch.cuda.synchronize()
    code = int(st.item())
    assert 0x200 < code < 0x300, hex(code)
    st.zero_()
    out, st = V.stage_attention(qkv, heads, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x = qkv.double().cpu().numpy()
    g = out.double().cpu().numpy()
    rows = [0, 1, 127, 128, 640, T - 2, T - 1]
    for bi in (0, B - 1):
        for h in (0, heads - 1):
            q = x[bi, rows, 64 * h:64 * (h + 1)]
            k = x[bi, :, D + 64 * h:D + 64 * (h + 1)]
            v = x[bi, :, 2 * D + 64 * h:2 * D + 64 * (h + 1)]
            ref = O.attention_probs(q, k) @ v
            err = np.abs(g[bi, rows, 64 * h:64 * (h + 1)] - ref).max()
            assert err <= 6e-3 * np.abs(ref).max() + 1e-3, (bi, h, err)
