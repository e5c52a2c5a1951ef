"""Per-launch profiling (vit_profile_begin / vit_profile_end): the library records a CUDA event pair
around every kernel it launches, eagerly and under stream capture (where the pairs become
event-record nodes that every replay records again).  The per-kind launch counts must be those of
one forward, with positive times, and profiling must not change the outputs."""
import pytest
import torch

import synthetic as S
from parity import gpu, need_cuda

pytestmark = gpu


def _expected_counts(spec):
    # im2col, patch GEMM, token prep; per block QKV, attention, proj, FC1, FC2; final LayerNorm
    return {"im2col": 1, "patch_gemm": 1, "prefix": 1, "qkv_gemm": spec.depth, "attention": spec.depth,
            "proj_gemm": spec.depth, "fc1_gemm": spec.depth, "fc2_gemm": spec.depth}


def _check(prof, spec, reps):
    for k, n in _expected_counts(spec).items():
        assert k in prof, (k, sorted(prof))
        ms, cnt = prof[k]
        assert cnt == n * reps, (k, cnt, n * reps)
        assert ms > 0.0, (k, ms)


def test_profile_eager():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]
    enc = V.VitEncoder(spec, S.make_weights(spec, 181), max_batch=2)
    x = S.make_images(spec, 2, 182).cuda()
    ref = enc.forward(x, desc=True, patch=True)
    torch.cuda.synchronize()
    n = enc.last_launch_count()
    enc.profile_begin(2 * n + 4)
    outs = [enc.forward(x, desc=True, patch=True) for _ in range(2)]
    torch.cuda.synchronize()
    prof = enc.profile_end()
    enc.poll()
    _check(prof, spec, 2)
    assert sum(c for _, c in prof.values()) == 2 * n
    for o in outs:
        assert torch.equal(o["desc"], ref["desc"]) and torch.equal(o["patch_tokens"], ref["patch_tokens"])
    enc.close()


def test_profile_graph_replay():
    need_cuda()
    import vision_transformer_encoder_fwd_b200 as V
    spec = S.PRESETS["small_s16"]
    enc = V.VitEncoder(spec, S.make_weights(spec, 183), max_batch=2)
    x = S.make_images(spec, 2, 184).cuda()
    ws = torch.empty(enc.workspace_size(2), dtype=torch.uint8, device="cuda")
    outs = enc.alloc_outputs(2, desc=True, patch=True)
    enc.forward_into(x, outs, ws=ws)
    torch.cuda.synchronize()
    n = enc.last_launch_count()
    enc.profile_begin(n + 4)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        enc.forward_into(x, outs, ws=ws)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    prof = enc.profile_end()        # the slots hold the last replay's records
    enc.poll()
    _check(prof, spec, 1)
    del g
    enc.close()
