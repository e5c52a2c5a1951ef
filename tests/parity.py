"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, compare with
the fp64 oracle with the tolerances the encoder's accuracy target states (descriptor cosine
>= 0.9995, per-block hidden-state max relative error <= 2e-2, no NaN/Inf, zero-shot argmax
agreement >= 99.5% of pixels)."""
import numpy as np
import pytest
import torch

DESC_COS_MIN = 0.9995
BLOCK_REL_MAX = 2e-2
ARGMAX_AGREE_MIN = 0.995

gpu = pytest.mark.gpu


def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def block_rel_err(g, r):
    """max |x_gpu - x_ref| / max |x_ref| over one block's [T, D] output of one image."""
    return float(np.abs(g - r).max() / np.abs(r).max())


def desc_cos(g, r):
    return float((g * r).sum() / (np.linalg.norm(g) * np.linalg.norm(r)))


def run_gpu(spec, weights, images, hidden=True, patch=True, taps=None, keep=None):
    """Run vit_forward on the whole batch; ``keep`` (image indices) limits what is copied back
    of the per-block hidden states (the rest of the outputs come back whole)."""
    import vision_transformer_encoder_fwd_b200 as V
    B = images.shape[0]
    enc = V.VitEncoder(spec, weights, max_batch=B)
    outs = enc.forward(images.cuda().contiguous(), desc=True, patch=patch, patch_fp32=True,
                       taps=bool(spec.taps) if taps is None else taps, hidden=hidden)
    torch.cuda.synchronize()
    enc.poll()
    res = {}
    for k, v in outs.items():
        if k == "hidden" and keep is not None:
            res[k] = np.zeros((v.shape[0], v.shape[1]) + tuple(v.shape[2:]), dtype=np.float32)
            res["hidden_finite"] = bool(torch.isfinite(v).all().item())
            for i in keep:
                res[k][:, i] = v[:, i].cpu().numpy()
            continue
        res[k] = [t.double().cpu().numpy() for t in v] if isinstance(v, list) else v.double().cpu().numpy()
    res["launches"] = enc.last_launch_count()
    enc.close()
    return res


def assert_forward_parity(g, ref, spec, image_indices, report=None):
    """g: GPU outputs for the whole batch; ref: oracle outputs for ``image_indices``."""
    for k in ("desc", "patch_tokens"):
        assert np.isfinite(g[k]).all(), f"non-finite {k}"
    worst = 0.0
    for j, i in enumerate(image_indices):
        if "hidden" in g and "hidden" in ref:
            for l in range(ref["hidden"].shape[0]):
                e = block_rel_err(g["hidden"][l, i], ref["hidden"][l, j])
                worst = max(worst, e)
                assert e <= BLOCK_REL_MAX, f"image {i} block {l + 1}: rel err {e:.3e}"
        c = desc_cos(g["desc"][i], ref["desc"][j])
        assert c >= DESC_COS_MIN, f"image {i}: descriptor cosine {c:.6f}"
        assert abs(np.linalg.norm(g["desc"][i]) - 1) < 1e-4
        pe = block_rel_err(g["patch_tokens"][i], ref["patch_tokens"][j])
        assert pe <= BLOCK_REL_MAX, f"image {i}: patch tokens rel err {pe:.3e}"
        for t, l in enumerate(spec.taps):
            te = block_rel_err(g["taps"][t][i], ref["taps"][l][j])
            assert te <= BLOCK_REL_MAX, f"image {i}: tap {l} rel err {te:.3e}"
    if report is not None:
        report["worst_block_rel_err"] = worst
    return worst
