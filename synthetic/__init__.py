"""Seeded synthetic inputs for the ViT encoder forward: weights, images, text features.

This module is shared by the fp64 oracle (``oracle/``) and by the CUDA path's tests and bench.
It holds random draws, their rounding to bf16, the ImageNet input normalisation that the
caller applies before the encoder, and the attention-sink construction.  It holds none of
the encoder's own arithmetic (no patch embedding, LayerNorm, attention, MLP or scoring).

Everything is drawn on the CPU with ``torch.Generator`` so that a seed gives the same bytes on
any host.  Matrix parameters are returned as bf16 CPU tensors (the library consumes bf16
weights); images and text features are fp32.

Sources for the shapes and the distributions:
  * kornia/dinov3 model card, section "Model I/O": ViT-S/16 at 336 = 21 x 16, ImageNet
    mean/std normalised CHW input, CLS + 4 register tokens + patch grid.
  * "DINOv2 n semantic" diagram (libreyolo), panel "DINOv2-S encoder": ViT-S/14 at 518,
    37 x 37 patches, CLS, 1,370-row position embedding, zero register tokens, taps 3/6/9/12.
  * DINOv3 zero-shot segmentation article (dino.txt), sections on the embedding alignment
    and on whole/slide inference: ViT-L/16 patch tokens of width 1024, text features
    [num_classes, 1024], 150 ADE20K classes, side 384 / stride 192 windows.
  * DINOv2 ONNX/TensorRT blog, table "模型规格对比表" (model variants): widths, depths, heads.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch

IMAGENET_MEAN = (0.485, 0.456, 0.406)
IMAGENET_STD = (0.229, 0.224, 0.225)


@dataclass(frozen=True)
class ModelSpec:
    """Architecture of one encoder (all integers; head width is always 64)."""

    name: str
    patch: int
    img_h: int
    img_w: int
    dim: int
    depth: int
    heads: int
    mlp: int
    registers: int
    pos_on_cls: bool
    taps: Tuple[int, ...] = ()
    ln_eps: float = 1e-6

    @property
    def grid_h(self) -> int:
        return self.img_h // self.patch

    @property
    def grid_w(self) -> int:
        return self.img_w // self.patch

    @property
    def n_patches(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def tokens(self) -> int:
        return 1 + self.registers + self.n_patches

    @property
    def n_pos(self) -> int:
        return self.n_patches + (1 if self.pos_on_cls else 0)

    def with_image(self, h: int, w: int) -> "ModelSpec":
        return dataclasses.replace(self, img_h=h, img_w=w)


# Model presets.  DINOv3-style models carry 4 registers and a patch-only position embedding;
# the DINOv2-style ViT-S/14 has no registers and a position embedding that also covers CLS.
VITS16_336 = ModelSpec("vits16_336", 16, 336, 336, 384, 12, 6, 1536, 4, False)
VITS14_518 = ModelSpec("vits14_518", 14, 518, 518, 384, 12, 6, 1536, 0, True, (3, 6, 9, 12))
VITL16_1024 = ModelSpec("vitl16_1024", 16, 1024, 1024, 1024, 24, 16, 4096, 4, False)
VITL16_384 = ModelSpec("vitl16_384", 16, 384, 384, 1024, 24, 16, 4096, 4, False)

# Other widths of the DINOv2 family ("DINOv2模型服务" blog, model-variant table: ViT-B/14
# 768 / 12 blocks / 12 heads, ViT-G/14 1536 / 40 / 24), DINOv2-style (no registers, position
# embedding on CLS), MLP ratio 4 with GELU as in the blog's DinoVisionTransformer(mlp_ratio=4);
# at 224 x 224 (16 x 16 patches, 257 tokens) so the fp64 oracle stays fast.
VITB14_224 = ModelSpec("vitb14_224", 14, 224, 224, 768, 12, 12, 3072, 0, True)
VITG14_224 = ModelSpec("vitg14_224", 14, 224, 224, 1536, 40, 24, 6144, 0, True)

# Small shapes for fast parity runs (several GEMM tiles and a ragged tail, seconds in fp64).
TINY_S16 = ModelSpec("tiny_s16", 16, 96, 160, 128, 2, 2, 512, 4, False)            # T = 65
TINY_S14 = ModelSpec("tiny_s14", 14, 126, 126, 128, 3, 2, 256, 0, True, (1, 3))     # T = 82
TINY_S14_DENSE = ModelSpec("tiny_s14_dense", 14, 126, 126, 128, 4, 2, 256, 0, True, (1, 2, 3, 4))  # four taps
SMALL_S16 = ModelSpec("small_s16", 16, 224, 224, 256, 3, 4, 1024, 4, False, (2,))   # T = 201

PRESETS: Dict[str, ModelSpec] = {
    s.name: s for s in (VITS16_336, VITS14_518, VITL16_1024, VITL16_384, VITB14_224, VITG14_224, TINY_S16, TINY_S14, TINY_S14_DENSE,
                        SMALL_S16)
}


@dataclass(frozen=True)
class Workload:
    """One measured configuration: a model, a batch and the seeds of its inputs."""

    name: str
    spec: ModelSpec
    batch: int
    weight_seed: int
    image_seed: int
    outlier: bool = False


WORKLOADS: Dict[str, Workload] = {
    "vits16_336_b1": Workload("vits16_336_b1", VITS16_336, 1, 1001, 1),
    "vits16_336_b64_outlier": Workload("vits16_336_b64_outlier", VITS16_336, 64, 1002, 2, outlier=True),
    "vits14_518_b8_taps": Workload("vits14_518_b8_taps", VITS14_518, 8, 1003, 3),
    "vitl16_1024_b1": Workload("vitl16_1024_b1", VITL16_1024, 1, 1004, 4),
    "vitl16_1024_b8": Workload("vitl16_1024_b8", VITL16_1024, 8, 1004, 40),
    "vitl16_slide_512x1024": Workload("vitl16_slide_512x1024", VITL16_384, 1, 1005, 5),
}

SLIDE_IMAGE = (512, 1024)
SLIDE_SIDE = 384
SLIDE_STRIDE = 192
SLIDE_CLASSES = 150
TEXT_SEED = 5150
# dino.txt vision head: 2 extra blocks on the backbone's tokens before the cosine with the
# text features (dino.txt article, "Aligning 1024-d patch tokens with 2048-d text embeddings").
DINOTXT_HEAD_BLOCKS = 2
HEAD_SEED = 5151


def to_bf16(t: torch.Tensor) -> torch.Tensor:
    """Round fp32 draws to bf16 (round-to-nearest-even, torch's conversion)."""
    return t.to(torch.bfloat16)


def _normal(g: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def _uniform(g: torch.Generator, shape, lo: float, hi: float) -> torch.Tensor:
    return lo + (hi - lo) * torch.rand(*shape, generator=g, dtype=torch.float32)


def _block_weights(g: torch.Generator, D: int, F: int) -> Dict[str, torch.Tensor]:
    """One encoder block's weights in draw order (qkv left fp32 for the sink construction)."""
    return {
        "ln1_w": to_bf16(1.0 + _normal(g, (D,), 0.02)),
        "ln1_b": to_bf16(_normal(g, (D,), 0.02)),
        "qkv_w": _normal(g, (3 * D, D), 0.02),
        "qkv_b": _normal(g, (3 * D,), 0.02),
        "proj_w": to_bf16(_normal(g, (D, D), 0.02)),
        "proj_b": to_bf16(_normal(g, (D,), 0.02)),
        "ls1": to_bf16(_uniform(g, (D,), 0.1, 1.0)),
        "ln2_w": to_bf16(1.0 + _normal(g, (D,), 0.02)),
        "ln2_b": to_bf16(_normal(g, (D,), 0.02)),
        "fc1_w": to_bf16(_normal(g, (F, D), 0.02)),
        "fc1_b": to_bf16(_normal(g, (F,), 0.02)),
        "fc2_w": to_bf16(_normal(g, (D, F), 0.02)),
        "fc2_b": to_bf16(_normal(g, (D,), 0.02)),
        "ls2": to_bf16(_uniform(g, (D,), 0.1, 1.0)),
    }


def make_weights(spec: ModelSpec, seed: int, outlier: bool = False) -> Dict[str, object]:
    """Seeded bf16 weights of one encoder.

    Distributions: Linear/conv weights and biases N(0, 0.02); CLS, registers and position
    embedding N(0, 0.02); LayerNorm gamma 1 + N(0, 0.02) and beta N(0, 0.02); layer-scale
    U(0.1, 1).  Shapes follow nn.Linear ([out, in]) and nn.Conv2d ([D, 3, p, p]); the three
    attention projections are stacked as one [3D, D] matrix with rows q | k | v.

    Returns a dict with bf16 CPU tensors and a list ``blocks`` of per-block dicts.
    """
    g = torch.Generator().manual_seed(int(seed))
    D, F, p, R = spec.dim, spec.mlp, spec.patch, spec.registers
    w: Dict[str, object] = {}
    w["patch_w"] = to_bf16(_normal(g, (D, 3, p, p), 0.02))
    w["patch_b"] = to_bf16(_normal(g, (D,), 0.02))
    w["cls"] = to_bf16(_normal(g, (D,), 0.02))
    w["reg"] = to_bf16(_normal(g, (R, D), 0.02))
    w["pos"] = to_bf16(_normal(g, (spec.n_pos, D), 0.02))
    w["norm_w"] = to_bf16(1.0 + _normal(g, (D,), 0.02))
    w["norm_b"] = to_bf16(_normal(g, (D,), 0.02))
    blocks: List[Dict[str, torch.Tensor]] = [_block_weights(g, D, F) for _ in range(spec.depth)]
    if outlier:
        _inject_attention_sink(spec, w, blocks, seed)
    for b in blocks:
        b["qkv_w"] = to_bf16(b["qkv_w"]) if b["qkv_w"].dtype != torch.bfloat16 else b["qkv_w"]
        b["qkv_b"] = to_bf16(b["qkv_b"]) if b["qkv_b"].dtype != torch.bfloat16 else b["qkv_b"]
    w["blocks"] = blocks
    return w


def make_head_weights(spec: ModelSpec, seed: int, n_blocks: int = DINOTXT_HEAD_BLOCKS) -> List[Dict[str, torch.Tensor]]:
    """Seeded bf16 weights of the dino.txt vision head: ``n_blocks`` blocks of the encoder
    block's form and width, drawn like make_weights' blocks."""
    g = torch.Generator().manual_seed(int(seed))
    blocks = [_block_weights(g, spec.dim, spec.mlp) for _ in range(n_blocks)]
    for b in blocks:
        b["qkv_w"] = to_bf16(b["qkv_w"])
        b["qkv_b"] = to_bf16(b["qkv_b"])
    return blocks


DENSE_CLASSES = 19       # [diagram] "Predict Conv2d 1x1: 256 to 19 class logits"
DENSE_WIDTH = 256        # [diagram] "Projector P4": 1,536 to 256
DENSE_SEED = 5190


def make_dense_head_weights(spec: ModelSpec, seed: int, n_classes: int = DENSE_CLASSES,
                            width: int = DENSE_WIDTH) -> Dict[str, object]:
    """Seeded bf16 weights of the dense head on the taps (C2f projector P4 + semantic task head),
    drawn like make_weights: conv weights and biases N(0, 0.02), norm gamma 1 + N(0, 0.02) and
    beta N(0, 0.02).  Conv weights are [out, in, k, k]; ``bn_w`` lists the six 3x3 convs of the
    three bottlenecks in order."""
    g = torch.Generator().manual_seed(int(seed))
    C4, h = 4 * spec.dim, width // 2

    def ln(n):
        return to_bf16(1.0 + _normal(g, (n,), 0.02)), to_bf16(_normal(g, (n,), 0.02))

    w: Dict[str, object] = {}
    w["cv1_w"] = to_bf16(_normal(g, (width, C4, 1, 1), 0.02))
    w["cv1_ln_w"], w["cv1_ln_b"] = ln(width)
    w["bn_w"], w["bn_ln_w"], w["bn_ln_b"] = [], [], []
    for _ in range(6):
        w["bn_w"].append(to_bf16(_normal(g, (h, h, 3, 3), 0.02)))
        a, b = ln(h)
        w["bn_ln_w"].append(a)
        w["bn_ln_b"].append(b)
    w["cv2_w"] = to_bf16(_normal(g, (width, 5 * h, 1, 1), 0.02))
    w["cv2_ln_w"], w["cv2_ln_b"] = ln(width)
    w["out_ln_w"], w["out_ln_b"] = ln(width)
    w["lat_w"] = to_bf16(_normal(g, (width, width, 1, 1), 0.02))
    w["lat_b"] = to_bf16(_normal(g, (width,), 0.02))
    w["smooth_w"] = to_bf16(_normal(g, (width, width, 3, 3), 0.02))
    w["smooth_b"] = to_bf16(_normal(g, (width,), 0.02))
    w["gn_w"], w["gn_b"] = ln(width)
    w["pred_w"] = to_bf16(_normal(g, (n_classes, width, 1, 1), 0.02))
    w["pred_b"] = to_bf16(_normal(g, (n_classes,), 0.02))
    return w


# Attention-sink construction (kornia/dinov3 card, "Build BF16, not FP16": the scaled logits
# Q.K^T/8 of the first block reach about 2.1e6 -- 2.5e6 on a natural image -- while every
# other tensor stays below 1800; the register tokens absorb this sink).  The page gives only
# magnitudes, so the construction is ours:
#   * e_hat: a zero-mean unit direction; register 1 = SINK_REG_SCALE * e_hat, so block 1's
#     LayerNorm maps register 1 to about sqrt(D) * e_hat.
#   * e_q: a second zero-mean unit direction orthogonal to e_hat; block 1's LN1 beta gets
#     SINK_BETA * e_q, giving every token a component SINK_BETA along e_q.
#   * w: eight ones on the first eight channels of head 0.
#   * W_k += SINK_AK * w e_hat^T and W_q += SINK_AQ * w e_q^T (rank one each).
# Every head-0 query then carries ~SINK_AQ * SINK_BETA along w, register 1's key carries
# ~SINK_AK * sqrt(D) along w, and head 0 puts all its weight on register 1 with a margin of
# more than 1e6 over every other key -- robust to bf16 rounding of Q and K.
SINK_REG_SCALE = 40.0
SINK_BETA = 20.0
SINK_AQ = 67.5
SINK_AK = 75.5
SINK_SEED_OFFSET = 77


def _zero_mean_unit(g: torch.Generator, n: int) -> torch.Tensor:
    v = torch.randn(n, generator=g, dtype=torch.float64)
    v = v - v.mean()
    return v / v.norm()


def _inject_attention_sink(spec: ModelSpec, w, blocks, seed: int) -> None:
    if spec.registers < 1:
        raise ValueError("the attention-sink construction needs at least one register token")
    D = spec.dim
    g = torch.Generator().manual_seed(int(seed) + SINK_SEED_OFFSET)
    e_hat = _zero_mean_unit(g, D)
    e_q = _zero_mean_unit(g, D)
    e_q = e_q - (e_q @ e_hat) * e_hat
    e_q = e_q - e_q.mean()
    e_q = e_q / e_q.norm()
    wv = torch.zeros(D, dtype=torch.float64)
    wv[:8] = 1.0
    reg = w["reg"].to(torch.float32).clone()
    reg[0] = (SINK_REG_SCALE * e_hat).to(torch.float32)
    w["reg"] = to_bf16(reg)
    b0 = blocks[0]
    b0["ln1_b"] = to_bf16((SINK_BETA * e_q).to(torch.float32))
    qkv = b0["qkv_w"].to(torch.float64)
    qkv[0:D] += SINK_AQ * torch.outer(wv, e_q)
    qkv[D:2 * D] += SINK_AK * torch.outer(wv, e_hat)
    b0["qkv_w"] = qkv.to(torch.float32)


def make_images(spec: ModelSpec, batch: int, seed: int, h: Optional[int] = None,
                w: Optional[int] = None) -> torch.Tensor:
    """Pixels U[0,1) fp32, then ImageNet mean/std per channel -> [B, 3, H, W] fp32.

    The normalisation is the caller-side preprocessing the kornia/dinov3 card states for the
    model input ("Model I/O"); the library receives already-normalised images.
    """
    H = spec.img_h if h is None else h
    W = spec.img_w if w is None else w
    g = torch.Generator().manual_seed(int(seed))
    x = torch.rand(batch, 3, H, W, generator=g, dtype=torch.float32)
    mean = torch.tensor(IMAGENET_MEAN, dtype=torch.float32).view(1, 3, 1, 1)
    std = torch.tensor(IMAGENET_STD, dtype=torch.float32).view(1, 3, 1, 1)
    return (x - mean) / std


def make_text_feats(n_classes: int, dim: int, seed: int = TEXT_SEED) -> torch.Tensor:
    """Stand-in for dino.txt class embeddings: N(0,1) rows scaled to unit length -> fp32 [C, dim].

    The trained text tower is not available; these seeded unit vectors take its place.
    """
    g = torch.Generator().manual_seed(int(seed))
    t = torch.randn(n_classes, dim, generator=g, dtype=torch.float64)
    t = t / t.norm(dim=1, keepdim=True)
    return t.to(torch.float32)


def make_workload(name: str):
    """(spec, weights, images) of a named workload.  The slide workload's images are the one
    512 x 1024 picture that the windows are cut from."""
    wl = WORKLOADS[name]
    weights = make_weights(wl.spec, wl.weight_seed, wl.outlier)
    if name.startswith("vitl16_slide"):
        images = make_images(wl.spec, 1, wl.image_seed, *SLIDE_IMAGE)
    else:
        images = make_images(wl.spec, wl.batch, wl.image_seed)
    return wl.spec, weights, images


def as_numpy_f64(t) -> np.ndarray:
    """Exact upcast of a bf16/fp32 tensor to fp64 numpy (no rounding happens)."""
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to(torch.float64).cpu().numpy()


def make_matrix(shape, seed: int, std: float = 1.0, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, std^2) draws of the given shape, rounded to ``dtype`` (stage-level test inputs)."""
    g = torch.Generator().manual_seed(int(seed))
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).to(dtype)
