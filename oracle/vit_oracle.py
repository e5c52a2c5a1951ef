"""Plain, slow fp64 CPU oracle of the DINOv2/DINOv3 ViT encoder forward and of the
dino.txt zero-shot patch-text scoring.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference arm may import or run this module.  It shares no code with the CUDA
library: it reads the same seeded inputs (bf16 weights, fp32 images, fp32 text features)
and computes everything in float64 with numpy.  Library primitives used as single steps:
``numpy.matmul`` / ``@`` (a plain dense product), ``numpy.exp``, ``scipy.special.erf``.
There is no blocking, fusion or reordering beyond what each definition states.

Pages cited (title, then section / panel):
  [card]    "kornia/dinov3" model card (aimarketly.com): "Model I/O", "Build BF16, not FP16",
            "Usage".
  [diagram] "DINOv2 n semantic" architecture diagram (libreyolo.com): panels "DINOv2-S
            encoder", "Encoder block", "Encoder self-attention".
  [dinotxt] "DINOv3零样本分割实测：dino.txt补丁级匹配与双推理模式" (hotelren.com): sections
            "对齐 1024 维补丁令牌与 2048 维文本嵌入" (patch/text alignment) and
            "按分辨率切换 whole 与 slide 两种推理模式" (whole and slide modes).
  [blog]    "DINOv2模型服务：ONNX导出与TensorRT加速推理" (blog.gitcode.com): "DINOv2模型架构概览"
            (architecture overview, register_tokens / NestedTensorBlock / norm).

Readings taken where the pages are silent (each one is listed in the design notes):
  * Q/K/V, output projection and MLP linears carry biases (nn.Linear default).
  * LayerNorm uses the biased variance with eps inside the square root, eps = 1e-6
    ([diagram] "Encoder block": LayerNorm eps=1e-6).  The "(x-mean)/(std+eps)" layer in the
    blog's FAQ is a workaround for an export problem, not the model's norm, and is not used.
  * GELU is the exact erf form.
  * Register tokens sit between CLS and the patches and receive no position embedding
    ([card] "Model I/O": skip indices 1-4).  DINOv3-style models add the position embedding
    to the patches only; DINOv2-style (``pos_on_cls``) adds its first row to CLS as well
    ([diagram]: a 1,370 x 384 position embedding for 1 CLS + 1369 patches).
  * Taps apply the final LayerNorm's parameters ([diagram]: "Taps apply LayerNorm, remove
    CLS, reshape"); register tokens are removed with CLS.
  * The descriptor is F.normalize(final_norm(x)[CLS]) with eps 1e-12 ([card] "Usage":
    L2-normed; "Model I/O": the descriptor is the CLS token).
  * Slide windows: n = ceil((size - side) / stride) + 1 per axis, last origin clamped to
    size - side; 512 x 1024 gives 2 x 5 = 10 windows ([dinotxt] whole/slide section).
  * Whole mode: the scores are the upsampled cosine map (no softmax); argmax ties resolve
    to the lowest class index.

Parity status: every function below is pinned by tests in ``tests/test_oracle_pins.py``
(closed forms, invariants, brute force on tiny inputs and fp64 library special cases);
the composed forward is additionally cross-checked against an independent composition of
torch fp64 functional ops.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "bicubic_resize", "resize_pos_embed", "bf16_round", "to_f64_weights", "patch_embed", "assemble_tokens", "layer_norm", "gelu",
    "attention", "attention_probs", "encoder_block", "forward", "l2_normalize", "cos_map",
    "bilinear_resize", "window_origins", "overlap_counts", "seg_slide_from_tokens",
    "seg_whole_from_tokens", "seg_slide", "seg_whole", "text_head", "conv2d", "channel_layer_norm", "silu",
    "group_norm", "dense_projector", "dense_task_head", "dense_head", "HEAD_DIM",
]

HEAD_DIM = 64


# ---------------------------------------------------------------------------------------------
# Precision: [card] "Build BF16, not FP16" -- the engine computes in bf16.  The encoder input
# is fp32 ImageNet-normalised pixels ([card] "Model I/O"); the first thing the bf16 path does
# is round them to bf16, which this function restates bit by bit.
# ---------------------------------------------------------------------------------------------
def bf16_round(a) -> np.ndarray:
    """Round to the nearest bf16 value, ties to even; returns float64 holding bf16 values.

    A float32 keeps its top 16 bits; the discarded low half decides the rounding: add
    0x7FFF plus the lowest kept bit, then truncate.  NaN stays NaN.
    """
    a32 = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = a32.view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + keep_lsb) & np.uint64(0xFFFF0000)).astype(np.uint32)
    out = r.view(np.float32).astype(np.float64)
    out[np.isnan(a32)] = np.nan
    return out


def to_f64_weights(weights) -> Dict[str, object]:
    """Exact fp64 copy of a weight dict (bf16 torch tensors or arrays) -- no arithmetic."""
    def conv(t):
        if isinstance(t, np.ndarray):
            return t.astype(np.float64)
        return t.detach().double().cpu().numpy()
    out = {k: conv(v) for k, v in weights.items() if k != "blocks"}
    out["blocks"] = [{k: conv(v) for k, v in b.items()} for b in weights["blocks"]]
    return out


# ---------------------------------------------------------------------------------------------
# [diagram] "DINOv2-S encoder": "Position embedding 1,370 x 384" followed by "Bicubic
# interpolation, 37x37 unchanged" -- the learned grid is resized bicubically to the input's
# patch grid (the identity at the native size).  Reading: the convolution form of bicubic
# interpolation with a = -0.75, half-pixel centres (align_corners=False), source coordinates
# not clamped, taps clamped to the border -- the convention of F.interpolate(mode="bicubic").
# ---------------------------------------------------------------------------------------------
def _cubic_weights(t: np.ndarray, a: float = -0.75) -> np.ndarray:
    """Weights of the taps at offsets -1, 0, +1, +2 for fractional positions t in [0, 1)."""
    def k(x):
        x = np.abs(x)
        return np.where(x <= 1.0, ((a + 2.0) * x - (a + 3.0)) * x * x + 1.0,
                        np.where(x < 2.0, ((a * x - 5.0 * a) * x + 8.0 * a) * x - 4.0 * a, 0.0))
    return np.stack([k(1.0 + t), k(t), k(1.0 - t), k(2.0 - t)], axis=-1)


def bicubic_resize(img: np.ndarray, out_h: int, out_w: int) -> np.ndarray:
    """[C, h, w] -> [C, out_h, out_w], separable: rows, then columns."""
    C, h, w = img.shape

    def axis(n_in, n_out):
        src = (np.arange(n_out, dtype=np.float64) + 0.5) * (n_in / n_out) - 0.5
        i0 = np.floor(src).astype(np.int64)
        wts = _cubic_weights(src - i0)
        idx = np.clip(i0[:, None] + np.arange(-1, 3)[None, :], 0, n_in - 1)
        return idx, wts

    ry, wy = axis(h, out_h)
    rx, wx = axis(w, out_w)
    rows = (img[:, ry, :] * wy[None, :, :, None]).sum(axis=2)           # [C, out_h, w]
    return (rows[:, :, rx] * wx[None, None, :, :]).sum(axis=3)


def resize_pos_embed(pos: np.ndarray, grid0, grid, pos_on_cls: bool) -> np.ndarray:
    """Position embedding for a patch grid `grid` from the learned one for `grid0`: the patch rows
    are resized bicubically as a [D, gh0, gw0] image; a CLS row (pos_on_cls) is kept as is."""
    gh0, gw0 = grid0
    gh, gw = grid
    cls = pos[:1] if pos_on_cls else pos[:0]
    patch = pos[(1 if pos_on_cls else 0):]
    if (gh, gw) == (gh0, gw0):
        return pos.copy()
    D = patch.shape[1]
    img = patch.reshape(gh0, gw0, D).transpose(2, 0, 1)
    out = bicubic_resize(img, gh, gw).transpose(1, 2, 0).reshape(gh * gw, D)
    return np.concatenate([cls, out], axis=0)


# ---------------------------------------------------------------------------------------------
# [diagram] "DINOv2-S encoder": Conv2d p x p / p with bias, then "Flatten patch grid"
# (row-major over the g_h x g_w grid).  Written as the direct convolution: one kernel tap
# (c, ky, kx) at a time, each contributing W[:, c, ky, kx] * pixel(gy*p + ky, gx*p + kx).
# ---------------------------------------------------------------------------------------------
def patch_embed(xb: np.ndarray, w: np.ndarray, b: np.ndarray, p: int) -> np.ndarray:
    """xb [B, 3, H, W], w [D, 3, p, p], b [D] -> patch embeddings [B, gh*gw, D]."""
    B, C, H, W = xb.shape
    D = w.shape[0]
    gh, gw = H // p, W // p
    out = np.zeros((B, gh * gw, D), dtype=np.float64)
    for c in range(C):
        for ky in range(p):
            for kx in range(p):
                tap = xb[:, c, ky:gh * p:p, kx:gw * p:p]          # [B, gh, gw]
                out += tap.reshape(B, gh * gw, 1) * w[:, c, ky, kx].reshape(1, 1, D)
    out += b.reshape(1, 1, D)
    return out


def assemble_tokens(e: np.ndarray, cls: np.ndarray, reg: np.ndarray, pos: np.ndarray,
                    pos_on_cls: bool) -> np.ndarray:
    """[diagram] "Learned CLS", "Concat CLS and patches", "Position embedding" (+);
    [card] "Model I/O": 4 register tokens between CLS and the patch grid.

    Token order: CLS, registers 1..R, patches (row-major).  Returns [B, 1 + R + P, D].
    """
    B, P, D = e.shape
    R = 0 if reg is None else reg.shape[0]
    x = np.empty((B, 1 + R + P, D), dtype=np.float64)
    x[:, 0, :] = cls + (pos[0] if pos_on_cls else 0.0)
    if R:
        x[:, 1:1 + R, :] = reg
    x[:, 1 + R:, :] = e + pos[(1 if pos_on_cls else 0):]
    return x


def layer_norm(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float) -> np.ndarray:
    """[diagram] "Encoder block": LayerNorm, eps=1e-6.  Biased variance over the last axis,
    eps inside the square root, then the per-channel affine."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * g + b


def gelu(x: np.ndarray) -> np.ndarray:
    """[diagram] "Encoder block": GELU, exact form x * Phi(x) = x/2 * (1 + erf(x / sqrt 2))."""
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def attention_probs(q: np.ndarray, k: np.ndarray, logit_dtype=None) -> np.ndarray:
    """[diagram] "Encoder self-attention": MatMul Q K-transpose, Scale (divide by sqrt(64)),
    Softmax over keys.  q, k [T, 64] -> A [T, T], rows summing to one.

    ``logit_dtype`` (e.g. np.float16) casts the scaled logits before the softmax; it exists
    only to reproduce [card] "Build BF16, not FP16" (fp16 logits overflow to inf -> NaN).
    """
    s = (q @ k.T) / math.sqrt(q.shape[-1])
    if logit_dtype is not None:
        with np.errstate(over="ignore", invalid="ignore"):
            s = s.astype(logit_dtype)
    with np.errstate(over="ignore", invalid="ignore"):
        s = s - s.max(axis=1, keepdims=True)
        a = np.exp(s.astype(np.float64))
        a = a / a.sum(axis=1, keepdims=True)
    return a


def attention(u: np.ndarray, qkv_w: np.ndarray, qkv_b: np.ndarray, heads: int,
              logit_dtype=None, diag: Optional[dict] = None) -> np.ndarray:
    """[diagram] "Encoder self-attention" for one image: Linear Q, K, V (D -> D each; stacked
    rows q | k | v), reshape to heads x T x 64, softmax(Q K^T / 8) V per head, merge heads
    (head h -> channels 64h .. 64h + 63).  u [T, D] -> [T, D] (before the output Linear)."""
    T, D = u.shape
    qkv = u @ qkv_w.T + qkv_b
    q, k, v = qkv[:, :D], qkv[:, D:2 * D], qkv[:, 2 * D:]
    out = np.empty((T, D), dtype=np.float64)
    for h in range(heads):
        sl = slice(h * HEAD_DIM, (h + 1) * HEAD_DIM)
        if diag is not None:
            s = (q[:, sl] @ k[:, sl].T) / math.sqrt(HEAD_DIM)
            diag.setdefault("max_abs_logit", []).append(float(np.abs(s).max()))
            if T > 1:
                top2 = np.sort(s, axis=1)[:, -2:]
                diag.setdefault("min_top_gap", []).append(float((top2[:, 1] - top2[:, 0]).min()))
            diag.setdefault("max_abs_qkv", []).append(float(np.abs(qkv).max()))
        a = attention_probs(q[:, sl], k[:, sl], logit_dtype)
        out[:, sl] = a @ v[:, sl]
    return out


def encoder_block(x: np.ndarray, bw: Dict[str, np.ndarray], heads: int, eps: float,
                  logit_dtype=None, diag: Optional[dict] = None) -> np.ndarray:
    """[diagram] "Encoder block" (pre-LN) for one image, x [T, D]:
        x <- x + ls1 * (Attn(LN1(x)) W_o^T + b_o)
        x <- x + ls2 * (GELU(LN2(x) W_1^T + b_1) W_2^T + b_2)
    ("Multiply layer scale: 384 learned channel weights" on each branch before the +)."""
    u = layer_norm(x, bw["ln1_w"], bw["ln1_b"], eps)
    o = attention(u, bw["qkv_w"], bw["qkv_b"], heads, logit_dtype, diag)
    x = x + bw["ls1"] * (o @ bw["proj_w"].T + bw["proj_b"])
    u2 = layer_norm(x, bw["ln2_w"], bw["ln2_b"], eps)
    h = gelu(u2 @ bw["fc1_w"].T + bw["fc1_b"])
    if diag is not None:
        diag.setdefault("max_abs_ln", []).append(float(max(np.abs(u).max(), np.abs(u2).max())))
        diag.setdefault("max_abs_h", []).append(float(np.abs(h).max()))
    x = x + bw["ls2"] * (h @ bw["fc2_w"].T + bw["fc2_b"])
    return x


def l2_normalize(v: np.ndarray, eps: float = 1e-12) -> np.ndarray:
    """F.normalize(p=2) over the last axis: v / max(||v||_2, eps)."""
    n = np.sqrt((v * v).sum(axis=-1, keepdims=True))
    return v / np.maximum(n, eps)


def forward(images, weights, spec, n_blocks: Optional[int] = None, record_hidden: bool = False,
            logit_dtype=None, diag: Optional[dict] = None, image_indices: Optional[Sequence[int]] = None
            ) -> Dict[str, object]:
    """The encoder forward of ``spec`` on fp32 images [B, 3, H, W].

    Steps: bf16 rounding of the input; patch embedding; CLS / register / position tokens (the
    learned grid resized bicubically when the input's patch grid differs from the native one);
    ``depth`` encoder blocks (taps after the blocks listed in ``spec.taps``); final
    LayerNorm; outputs
      desc          [B, D]   L2-normalised final-norm CLS token ([card] "Usage")
      patch_tokens  [B, P, D] final-norm tokens of the patches (CLS and registers dropped)
      final_tokens  [B, T, D] the whole final-norm sequence (CLS, registers, patches)
      taps          {l: [B, D, gh, gw]} final-norm tokens after block l, CLS and registers
                    removed, channels first ([diagram] "Tap stage", "Taps apply LayerNorm,
                    remove CLS, reshape")
      hidden        [n_blocks, B, T, D] residual stream after each block (if requested)
    ``n_blocks`` < depth runs only the first blocks (used to time bounded samples); the
    outputs are then those of the truncated encoder.
    """
    w = weights if isinstance(weights.get("patch_w"), np.ndarray) else to_f64_weights(weights)
    imgs = images.detach().cpu().numpy() if hasattr(images, "detach") else np.asarray(images)
    if image_indices is not None:
        imgs = imgs[list(image_indices)]
    xb = bf16_round(imgs)
    p, D, R = spec.patch, spec.dim, spec.registers
    B = xb.shape[0]
    gh, gw = xb.shape[2] // p, xb.shape[3] // p
    P = gh * gw
    e = patch_embed(xb, w["patch_w"], w["patch_b"], p)
    pos = resize_pos_embed(w["pos"], (spec.grid_h, spec.grid_w), (gh, gw), spec.pos_on_cls)
    x = assemble_tokens(e, w["cls"], w["reg"] if R else None, pos, spec.pos_on_cls)
    L = spec.depth if n_blocks is None else n_blocks
    hidden = np.empty((L, B, x.shape[1], D)) if record_hidden else None
    taps: Dict[int, np.ndarray] = {}
    for l in range(1, L + 1):
        bw = w["blocks"][l - 1]
        for i in range(B):
            x[i] = encoder_block(x[i], bw, spec.heads, spec.ln_eps, logit_dtype,
                                 diag if (diag is not None and l == 1) else None)
        if record_hidden:
            hidden[l - 1] = x
        if l in spec.taps:
            n = layer_norm(x, w["norm_w"], w["norm_b"], spec.ln_eps)[:, 1 + R:, :]
            taps[l] = n.reshape(B, gh, gw, D).transpose(0, 3, 1, 2).copy()
    n = layer_norm(x, w["norm_w"], w["norm_b"], spec.ln_eps)
    out = {
        "desc": l2_normalize(n[:, 0, :]),
        "cls_norm": n[:, 0, :].copy(),
        "patch_tokens": n[:, 1 + R:, :].copy(),
        "final_tokens": n,
        "taps": taps,
        "grid": (gh, gw),
    }
    if record_hidden:
        out["hidden"] = hidden
    return out


# ---------------------------------------------------------------------------------------------
# Zero-shot scoring, [dinotxt] patch/text alignment and whole/slide sections.
# ---------------------------------------------------------------------------------------------
def cos_map(tokens: np.ndarray, text: np.ndarray, gh: int, gw: int) -> np.ndarray:
    """predict_whole's core: F.normalize the patch tokens, then einsum("cd,hwd->chw") with the
    (already unit) text features.  tokens [gh*gw, D], text [C, D] -> [C, gh, gw]."""
    t = l2_normalize(tokens)
    return (text @ t.T).reshape(text.shape[0], gh, gw)


def bilinear_resize(img: np.ndarray, out_h: int, out_w: int) -> np.ndarray:
    """F.interpolate(mode="bilinear", align_corners=False) of [C, h, w] -> [C, out_h, out_w].

    Source coordinate of output index i: (i + 0.5) * in/out - 0.5, clamped below at 0; the
    lower neighbour is its floor, the upper one floor + 1 clamped to in - 1; weights are the
    fractional part and its complement.  Separable: rows then columns.
    """
    C, h, w = img.shape

    def axis_weights(n_in, n_out):
        scale = n_in / n_out
        src = (np.arange(n_out, dtype=np.float64) + 0.5) * scale - 0.5
        src = np.maximum(src, 0.0)
        i0 = np.floor(src).astype(np.int64)
        i0 = np.minimum(i0, n_in - 1)
        i1 = np.minimum(i0 + 1, n_in - 1)
        lam = src - i0
        return i0, i1, lam

    y0, y1, ly = axis_weights(h, out_h)
    x0, x1, lx = axis_weights(w, out_w)
    rows = img[:, y0, :] * (1.0 - ly)[None, :, None] + img[:, y1, :] * ly[None, :, None]
    return rows[:, :, x0] * (1.0 - lx)[None, None, :] + rows[:, :, x1] * lx[None, None, :]


def window_origins(size: int, side: int, stride: int) -> List[int]:
    """Origins of the sliding windows along one axis (reading of [dinotxt]: side 384,
    stride 192, 512 x 1024 -> 2 x 5 windows): ceil((size - side) / stride) + 1 windows,
    the last one clamped to end at the border."""
    if size <= side:
        return [0]
    n = int(math.ceil((size - side) / stride)) + 1
    return [min(i * stride, size - side) for i in range(n)]


def overlap_counts(H: int, W: int, side: int, stride: int) -> np.ndarray:
    """counts[y, x] = number of windows covering pixel (y, x) ("counts[y1:y2, x1:x2] += 1")."""
    c = np.zeros((H, W), dtype=np.int64)
    for y in window_origins(H, side, stride):
        for x in window_origins(W, side, stride):
            c[y:y + min(side, H), x:x + min(side, W)] += 1
    return c


def _softmax_classes(s: np.ndarray) -> np.ndarray:
    s = s - s.max(axis=0, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=0, keepdims=True)


def seg_slide_from_tokens(window_tokens: np.ndarray, text: np.ndarray, H: int, W: int,
                          side: int, stride: int, grid: Tuple[int, int]) -> Tuple[np.ndarray, np.ndarray]:
    """predict_slide given each window's patch tokens (windows in row-major origin order):
    cos -> bilinear to the window size -> softmax over classes -> probs[:, win] += ,
    counts[win] += 1; finally probs /= counts and argmax over classes (lowest index on ties).
    window_tokens [n_win, gh*gw, D] -> (probs [C, H, W], labels [H, W] int64)."""
    C = text.shape[0]
    probs = np.zeros((C, H, W), dtype=np.float64)
    counts = np.zeros((H, W), dtype=np.float64)
    k = 0
    for y in window_origins(H, side, stride):
        for x in window_origins(W, side, stride):
            wh, ww = min(side, H), min(side, W)
            cos = cos_map(window_tokens[k], text, grid[0], grid[1])
            up = bilinear_resize(cos, wh, ww)
            probs[:, y:y + wh, x:x + ww] += _softmax_classes(up)
            counts[y:y + wh, x:x + ww] += 1.0
            k += 1
    probs /= counts[None]
    return probs, np.argmax(probs, axis=0)


# ---------------------------------------------------------------------------------------------
# [dino.txt article] "Aligning 1024-d patch tokens with 2048-d text embeddings": on the vision
# side the backbone's 1024-d patch tokens first go through 2 extra self-attention blocks
# (vision_model_num_head_blocks = 2), then meet the patch half of the text embedding in a
# cosine.  Readings: each head block has the encoder block's form and width (pre-LN attention
# and MLP branches with layer scale); it runs on the backbone's whole final-norm sequence
# (CLS, registers and patches attend to one another as in the backbone); the head's patch rows
# go to the cosine as they come out of the last block (the passage names no further norm, and
# the cosine divides by the token's length anyway).
# ---------------------------------------------------------------------------------------------
def text_head(final_tokens: np.ndarray, head_blocks, spec) -> np.ndarray:
    """final_tokens [B, T, D] (backbone final-norm sequence) -> head patch tokens [B, P, D]."""
    hb = to_f64_weights({"blocks": head_blocks})["blocks"]
    x = np.array(final_tokens, dtype=np.float64, copy=True)
    for bw in hb:
        for i in range(x.shape[0]):
            x[i] = encoder_block(x[i], bw, spec.heads, spec.ln_eps)
    return x[:, 1 + spec.registers:, :].copy()


def seg_whole_from_tokens(tokens: np.ndarray, text: np.ndarray, H: int, W: int,
                          grid: Tuple[int, int]) -> Tuple[np.ndarray, np.ndarray]:
    """predict_whole: cos map [C, h, w] upsampled bilinearly to [C, H, W]; argmax."""
    up = bilinear_resize(cos_map(tokens, text, grid[0], grid[1]), H, W)
    return up, np.argmax(up, axis=0)


def seg_slide(image, weights, spec, text, side: int, stride: int, n_windows: Optional[int] = None,
              head_blocks=None):
    """Full slide mode on one image [3, H, W] (or [1, 3, H, W]): crops every window, runs the
    encoder of ``spec`` on each (its position grid resized to side/p x side/p when the window is
    not the size it was learned for) and, if ``head_blocks`` is given, the dino.txt vision head
    (text_head), then scores.
    Returns (probs, labels, window_tokens)."""
    img = image.detach().cpu().numpy() if hasattr(image, "detach") else np.asarray(image)
    if img.ndim == 4:
        img = img[0]
    _, H, W = img.shape
    crops = []
    for y in window_origins(H, side, stride):
        for x in window_origins(W, side, stride):
            crops.append(img[:, y:y + side, x:x + side])
    crops = np.stack(crops)
    txt = text.detach().double().cpu().numpy() if hasattr(text, "detach") else np.asarray(text, np.float64)
    w = to_f64_weights(weights) if not isinstance(weights.get("patch_w"), np.ndarray) else weights
    toks = []
    for i in range(crops.shape[0]):
        o = forward(crops[i:i + 1], w, spec)
        toks.append(o["patch_tokens"][0] if head_blocks is None else text_head(o["final_tokens"], head_blocks, spec)[0])
    toks = np.stack(toks)
    probs, labels = seg_slide_from_tokens(toks, txt, H, W, side, stride, (side // spec.patch, side // spec.patch))
    return probs, labels, toks


def seg_whole(image, weights, spec, text, head_blocks=None):
    """Whole mode on one image [3, H, W]: one encoder pass at the image's own size (position grid
    resized as in forward), the dino.txt head if given, then seg_whole_from_tokens."""
    img = image.detach().cpu().numpy() if hasattr(image, "detach") else np.asarray(image)
    if img.ndim == 3:
        img = img[None]
    txt = text.detach().double().cpu().numpy() if hasattr(text, "detach") else np.asarray(text, np.float64)
    o = forward(img, weights, spec)
    tok = o["patch_tokens"][0] if head_blocks is None else text_head(o["final_tokens"], head_blocks, spec)[0]
    scores, labels = seg_whole_from_tokens(tok, txt, img.shape[2], img.shape[3], o["grid"])
    return scores, labels, tok


# ---------------------------------------------------------------------------------------------
# Dense head on the taps ([diagram] "Projector P4", "Projector Bottleneck", "Projector output
# ConvX", "Task head"; the LibreYOLO DINOv2 configuration): the four tap maps [D, g, g] are
# concatenated, projected by a C2f block (1x1 conv, channel LayerNorm, SiLU; split into two
# halves; three chained bottlenecks of two 3x3 conv / channel LN / SiLU each, no residual; all
# five pieces concatenated; 1x1 conv / channel LN / SiLU; a final channel LN), then the semantic
# head: lateral 1x1 conv, 3x3 smoothing conv, GroupNorm(32), GELU, dropout (identity at
# inference), 1x1 prediction conv to the class logits, bilinear resize to the input size.
# Readings: channel LayerNorm normalises each pixel over its channels with the biased variance
# and eps = 1e-6 (the only LayerNorm eps the diagram prints); GroupNorm uses eps = 1e-5 (the
# library default; none is printed); the prediction conv carries a bias (the diagram marks
# bias=False only on the projector's convs).
# ---------------------------------------------------------------------------------------------
CHANNEL_LN_EPS = 1e-6
GROUP_NORM_EPS = 1e-5


def conv2d(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray], pad: int) -> np.ndarray:
    """x [C, H, W], w [O, C, k, k], stride 1, zero padding `pad` -> [O, H', W'].  Written as
    the sum over kernel taps (ky, kx) of W[:, :, ky, kx] times the shifted input."""
    C, H, W = x.shape
    O, _, k, _ = w.shape
    xp = np.pad(x, ((0, 0), (pad, pad), (pad, pad)))
    Ho, Wo = H + 2 * pad - k + 1, W + 2 * pad - k + 1
    out = np.zeros((O, Ho * Wo))
    for ky in range(k):
        for kx in range(k):
            out += w[:, :, ky, kx] @ xp[:, ky:ky + Ho, kx:kx + Wo].reshape(C, Ho * Wo)
    if b is not None:
        out += b[:, None]
    return out.reshape(O, Ho, Wo)


def channel_layer_norm(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float = CHANNEL_LN_EPS) -> np.ndarray:
    """x [C, H, W]: each pixel's C values normalised (biased variance), then g * . + b."""
    mu = x.mean(axis=0, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=0, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * g[:, None, None] + b[:, None, None]


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def group_norm(x: np.ndarray, groups: int, g: np.ndarray, b: np.ndarray, eps: float = GROUP_NORM_EPS) -> np.ndarray:
    """x [C, H, W]: each group of C/groups channels normalised over its channels and pixels."""
    C, H, W = x.shape
    xg = x.reshape(groups, -1)
    mu = xg.mean(axis=1, keepdims=True)
    var = ((xg - mu) ** 2).mean(axis=1, keepdims=True)
    y = ((xg - mu) / np.sqrt(var + eps)).reshape(C, H, W)
    return y * g[:, None, None] + b[:, None, None]


def _conv_ln_silu(x, w, ln_g, ln_b, pad):
    return silu(channel_layer_norm(conv2d(x, w, None, pad), ln_g, ln_b))


def dense_projector(taps: Sequence[np.ndarray], hw: Dict[str, np.ndarray]) -> np.ndarray:
    """Projector P4 on one image: taps = four [D, g, g] maps -> [256, g, g]."""
    x = np.concatenate(list(taps), axis=0)
    y = _conv_ln_silu(x, hw["cv1_w"], hw["cv1_ln_w"], hw["cv1_ln_b"], 0)
    half = y.shape[0] // 2
    pieces = [y[:half], y[half:]]
    cur = pieces[1]
    for i in range(3):
        t = _conv_ln_silu(cur, hw["bn_w"][2 * i], hw["bn_ln_w"][2 * i], hw["bn_ln_b"][2 * i], 1)
        cur = _conv_ln_silu(t, hw["bn_w"][2 * i + 1], hw["bn_ln_w"][2 * i + 1], hw["bn_ln_b"][2 * i + 1], 1)
        pieces.append(cur)
    z = _conv_ln_silu(np.concatenate(pieces, axis=0), hw["cv2_w"], hw["cv2_ln_w"], hw["cv2_ln_b"], 0)
    return channel_layer_norm(z, hw["out_ln_w"], hw["out_ln_b"])


def dense_task_head(p4: np.ndarray, hw: Dict[str, np.ndarray], out_h: int, out_w: int) -> np.ndarray:
    """Semantic task head on one image: [256, g, g] -> class logits [n_classes, out_h, out_w]."""
    lat = conv2d(p4, hw["lat_w"], hw["lat_b"], 0)
    sm = conv2d(lat, hw["smooth_w"], hw["smooth_b"], 1)
    h = gelu(group_norm(sm, 32, hw["gn_w"], hw["gn_b"]))
    logits = conv2d(h, hw["pred_w"], hw["pred_b"], 0)
    return bilinear_resize(logits, out_h, out_w)


def dense_head(taps: Dict[int, np.ndarray], head_weights, spec, out_hw: Tuple[int, int]) -> Dict[str, np.ndarray]:
    """Projector + task head on a batch: taps {l: [B, D, g, g]} (forward's output, four layers of
    spec.taps in order) -> {"p4": [B, 256, g, g], "logits": [B, n_classes, H, W]}."""
    hw = {k: ([_to64(t) for t in v] if isinstance(v, (list, tuple)) else _to64(v)) for k, v in head_weights.items()}
    layers = list(spec.taps)
    B = taps[layers[0]].shape[0]
    p4, logits = [], []
    for i in range(B):
        p = dense_projector([taps[l][i] for l in layers], hw)
        p4.append(p)
        logits.append(dense_task_head(p, hw, out_hw[0], out_hw[1]))
    return {"p4": np.stack(p4), "logits": np.stack(logits)}


def _to64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().double().cpu().numpy()

