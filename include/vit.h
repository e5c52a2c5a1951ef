/*
 * vit.h -- C ABI of libvit_b200: the DINOv2/DINOv3 ViT encoder forward on one B200 (sm_100a).
 *
 * The interface follows the kornia/dinov3 model card ("Usage"): build a model from weights,
 * let the caller own the result buffers, enqueue the forward on a stream without
 * synchronising, and read an L2-normalised descriptor.  Errors come back as status codes,
 * never as process aborts; nothing here traps on the device.
 *
 * Pages cited (title, section / panel):
 *   [card]    "kornia/dinov3" model card: "Model I/O", "Build BF16, not FP16", "Usage".
 *   [diagram] "DINOv2 n semantic" architecture diagram: "DINOv2-S encoder", "Encoder block",
 *             "Encoder self-attention".
 *   [dinotxt] "DINOv3零样本分割实测：dino.txt补丁级匹配与双推理模式": patch/text alignment and
 *             the whole / slide inference modes.
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" are CUDA device memory of the current device; "host" are host
 *     memory (pinned memory makes the copies asynchronous).  All device pointers must be
 *     16-byte aligned.  The caller owns all memory passed in; the library never frees it.
 *   - bf16 means IEEE bfloat16 (2 bytes); matrices are row-major, nn.Linear weights [out, in].
 *   - Functions taking a cudaStream_t enqueue work on that stream and return without
 *     synchronising (except where stated).  Host validation happens before any launch; on a
 *     validation failure nothing is enqueued.
 *   - Device-side failures (a pipeline wait that ran out of time) set the model's status
 *     word; vit_poll() reads it.  No kernel traps.  The final LayerNorm (and the dino.txt
 *     head's) also flags any token row holding a NaN or an infinity; vit_poll() then returns
 *     VIT_E_NONFINITE.
 *   - The tensor-core kernels (GEMMs, attention) are launched with programmatic dependent
 *     launch: each may be scheduled (the GEMMs also set up their shared and tensor memory)
 *     while the kernel before it in the stream finishes, and touches global memory only once
 *     that kernel has completed.  Stream order, graph capture and results are unchanged.  Setting the
 *     environment variable VIT_B200_PDL=0 before the first launch turns it off.
 */
#ifndef VIT_B200_H
#define VIT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *vit_stream_t; /* == cudaStream_t; NULL = legacy default stream */

typedef enum vit_status {
  VIT_OK = 0,
  VIT_E_INVALID_ARG = 1,    /* null / misaligned pointer, bad value */
  VIT_E_SHAPE = 2,          /* sizes inconsistent with the model or with each other */
  VIT_E_UNSUPPORTED = 3,    /* a configuration this build does not implement */
  VIT_E_WORKSPACE = 4,      /* workspace smaller than vit_*_workspace_size reports */
  VIT_E_CUDA = 5,           /* a CUDA runtime / driver call failed */
  VIT_E_DEVICE_TIMEOUT = 6, /* a device pipeline wait gave up (read via vit_poll) */
  VIT_E_NONFINITE = 7       /* a NaN or infinity reached the final LayerNorm (read via vit_poll) */
} vit_status;

/* Encoder architecture.  [diagram] "DINOv2-S encoder" / "Encoder block"; [card] "Model I/O".
 * Constraints checked by vit_create: head width dim/heads == 64; dim and mlp_dim multiples of
 * 128; img_h, img_w multiples of patch; 1 <= patch <= 32; 0 <= n_registers <= 16;
 * 1 <= depth <= 64; max_batch >= 1; ln_eps > 0; at most 4 taps, all <= depth. */
typedef struct vit_config {
  int32_t patch;       /* p: patch side (16 DINOv3, 14 DINOv2) */
  int32_t img_h;       /* native input height in pixels (multiple of p) */
  int32_t img_w;       /* native input width in pixels (multiple of p) */
  int32_t dim;         /* D: token width */
  int32_t depth;       /* L: number of encoder blocks */
  int32_t heads;       /* D / 64 */
  int32_t mlp_dim;     /* F: MLP hidden width (4 D) */
  int32_t n_registers; /* R: register tokens between CLS and the patches (4 DINOv3, 0 DINOv2) */
  int32_t pos_on_cls;  /* 1: position embedding has 1 + P rows, row 0 added to CLS (DINOv2);
                          0: P rows, patches only (DINOv3) */
  int32_t max_batch;   /* largest batch vit_forward will be called with */
  float ln_eps;        /* LayerNorm eps (1e-6) */
  uint32_t tap_mask;   /* bit (l-1) set: tap after block l ([diagram] taps 3/6/9/12) */
} vit_config;

/* One encoder block's weights: device pointers to bf16 ([diagram] "Encoder block",
 * "Encoder self-attention").  The Q, K and V Linears are stacked: qkv_w [3D, D] with rows
 * q (0..D-1) | k (D..2D-1) | v (2D..3D-1); head h owns rows 64h..64h+63 of each part. */
typedef struct vit_block_weights {
  const void *ln1_w, *ln1_b;   /* [D] */
  const void *qkv_w, *qkv_b;   /* [3D, D], [3D] */
  const void *proj_w, *proj_b; /* [D, D], [D] */
  const void *ls1;             /* [D] layer scale of the attention branch */
  const void *ln2_w, *ln2_b;   /* [D] */
  const void *fc1_w, *fc1_b;   /* [F, D], [F] */
  const void *fc2_w, *fc2_b;   /* [D, F], [D] */
  const void *ls2;             /* [D] layer scale of the MLP branch */
} vit_block_weights;

/* Whole-model weights: device pointers to bf16, except `blocks`, a HOST array of `depth`
 * entries.  Borrowed: the device memory must stay valid and unchanged for the model's life.
 * The model also keeps derived copies it allocates itself (see vit_create). */
typedef struct vit_weights {
  const void *patch_w;  /* [D, 3, p, p] Conv2d weight */
  const void *patch_b;  /* [D] */
  const void *cls;      /* [D] learned CLS token */
  const void *reg;      /* [R, D] register tokens; may be NULL when R == 0 */
  const void *pos;      /* [pos_on_cls + gh*gw, D] learned additive position embedding */
  const void *norm_w, *norm_b; /* [D] final LayerNorm (also applied to the taps) */
  const vit_block_weights *blocks; /* host array [depth] */
} vit_weights;

/* Outputs of vit_forward; every pointer is optional (NULL = not wanted).  Device memory. */
typedef struct vit_outputs {
  float *desc;          /* [B, D] fp32: final-LN CLS token / max(||.||_2, 1e-12) ([card]) */
  void *patch_tokens;   /* [B, gh*gw, D] final-LN patch tokens (CLS and registers dropped),
                           fp32 if patch_fp32 else bf16 */
  int32_t patch_fp32;
  float *taps[4];       /* [B, D, gh, gw] fp32 each: final LayerNorm of the tokens after the
                           tapped blocks in ascending order, CLS and registers removed,
                           channels first ([diagram] "Taps apply LayerNorm, remove CLS, reshape") */
  float *hidden;        /* [depth, B, T, D] fp32 residual stream after every block
                           (T = 1 + R + gh*gw); a diagnostic for parity checks */
} vit_outputs;

typedef struct vit_model vit_model;

/* Validate the configuration, borrow the weights and prepare the derived weights the kernels
 * consume: the LayerNorm gammas folded into the QKV and FC1 matrices (bf16), the betas folded
 * into their biases (fp32), column sums of the folded matrices, the patch matrix padded to a
 * multiple of 64 columns, and fp32 copies of the vectors.  Runs on the current device and
 * synchronises it once.  On success *out receives the model. */
vit_status vit_create(const vit_config *cfg, const vit_weights *w, vit_model **out);

/* Bytes of device workspace vit_forward needs for `batch` images (batch <= max_batch). */
vit_status vit_workspace_size(const vit_model *m, int32_t batch, size_t *bytes);

/* The encoder forward ([diagram] "DINOv2-S encoder" with its blocks; [card] "Model I/O"):
 *   images  device fp32 [B, 3, img_h, img_w], ImageNet-normalised (the caller normalises);
 *           rounded to bf16 by the patch-embedding kernel.
 *   B       1 <= B <= max_batch.
 *   ws      device workspace of at least vit_workspace_size(m, B) bytes, 256-byte aligned;
 *           it must not be used concurrently by another call.
 * Enqueues on `stream`; returns without synchronising. */
vit_status vit_forward(vit_model *m, const float *images, int32_t B, const vit_outputs *out,
                       void *ws, size_t ws_bytes, vit_stream_t stream);

/* The same forward from host memory: copies `images_host` [B, 3, img_h, img_w] fp32 into the
 * workspace, runs vit_forward, and copies the descriptor [B, D] fp32 to `desc_host` and (if
 * non-NULL) the bf16 patch tokens [B, gh*gw, D] to `patch_tokens_host`.  Needs
 * vit_host_workspace_size bytes.  Enqueues on `stream`; the host buffers must stay valid until
 * the stream has been synchronised (pinned host memory makes the copies asynchronous). */
vit_status vit_host_workspace_size(const vit_model *m, int32_t batch, size_t *bytes);
vit_status vit_forward_host(vit_model *m, const float *images_host, int32_t B, float *desc_host,
                            void *patch_tokens_host, void *ws, size_t ws_bytes, vit_stream_t stream);

/* The encoder forward at an input size other than the one the model was created for
 * ([diagram] "DINOv2-S encoder": the learned position grid goes through "Bicubic
 * interpolation" to the input's patch grid, the identity at the native size).
 *   images  device fp32 [B, 3, H, W], ImageNet-normalised; patch <= H, W <= 16384.
 *   The patch grid is gh = floor(H / patch) by gw = floor(W / patch) (the stride-p
 *   convolution's; pixels past gh*patch, gw*patch are not read); T = 1 + R + gh*gw tokens.
 *   At a grid other than the native one, the first kernel writes the patch rows of the position
 *   embedding resized by separable cubic convolution (Keys' kernel, a = -0.75, half-pixel
 *   centres, taps clamped to the border; the CLS row, if any, copied) into the workspace.
 *   Outputs are sized by that grid: patch_tokens and taps [B, gh*gw, D], hidden [depth, B, T, D].
 *   ws  at least vit_workspace_size_hw(m, B, H, W) bytes, 256-byte aligned.
 * At the native size this is vit_forward.  Errors as vit_forward; VIT_E_SHAPE for H or W out of
 * range or B * T >= 2^30.  Enqueues on `stream`. */
vit_status vit_workspace_size_hw(const vit_model *m, int32_t batch, int32_t H, int32_t W, size_t *bytes);
vit_status vit_forward_hw(vit_model *m, const float *images, int32_t B, int32_t H, int32_t W,
                          const vit_outputs *out, void *ws, size_t ws_bytes, vit_stream_t stream);

/* dino.txt vision head ([dinotxt] "Aligning 1024-d patch tokens with 2048-d text embeddings":
 * the backbone's patch tokens pass through 2 extra self-attention blocks before the cosine
 * with the text features).  Each head block has the encoder block's form and width and takes
 * vit_block_weights like the backbone's; the head runs on the backbone's whole final-norm
 * sequence (CLS, registers, patches) and its patch rows, as the last block leaves them, are
 * the tokens the zero-shot scoring uses.
 *   vit_set_text_head: attaches n_blocks (1..8) head blocks, once per model (a second call
 *   returns VIT_E_INVALID_ARG); the weights are read as vit_create reads the backbone's (the
 *   folded QKV/FC1 copies are made now; proj_w and fc2_w are borrowed and must stay valid).
 *   Call it with the model's device current.  Once attached, vit_seg_zero_shot scores the
 *   head's tokens instead of the backbone's final-norm patch tokens.
 *   vit_forward_text_tokens: backbone + head on B images of H x W (any size as for
 *   vit_forward_hw; workspace vit_workspace_size_hw(m, B, H, W)); tokens: device fp32
 *   [B, floor(H/p) * floor(W/p), D].  VIT_E_INVALID_ARG if no head is attached. */
vit_status vit_set_text_head(vit_model *m, const vit_block_weights *blocks, int32_t n_blocks);
vit_status vit_forward_text_tokens(vit_model *m, const float *images, int32_t B, int32_t H, int32_t W,
                                   float *tokens, void *ws, size_t ws_bytes, vit_stream_t stream);

/* Dense head on the four taps (LibreYOLO DINOv2 configuration diagram: "Projector P4",
 * "Projector Bottleneck", "Projector output ConvX", "Task head").  bf16 device weights in
 * PyTorch layouts, borrowed as in vit_create except where noted; W = width, h = W / 2,
 * D4 = 4 * dim (the four taps concatenated in tap order). */
typedef struct vit_dense_head_weights {
  int32_t n_classes;                   /* K: prediction channels (19 in the diagram), 1..1024 */
  int32_t width;                       /* W: projector width (256 in the diagram); must be 256 */
  const void *cv1_w;                   /* [W, D4, 1, 1] 1x1 conv, no bias */
  const void *cv1_ln_w, *cv1_ln_b;     /* [W] channel LayerNorm */
  const void *bn_w[6];                 /* [h, h, 3, 3] bottleneck convs, no bias: bottleneck i uses 2i, 2i+1 */
  const void *bn_ln_w[6], *bn_ln_b[6]; /* [h] their channel LayerNorms */
  const void *cv2_w;                   /* [W, 5h, 1, 1] output ConvX, no bias */
  const void *cv2_ln_w, *cv2_ln_b;     /* [W] */
  const void *out_ln_w, *out_ln_b;     /* [W] final channel LayerNorm */
  const void *lat_w, *lat_b;           /* [W, W, 1, 1], [W] lateral conv */
  const void *smooth_w, *smooth_b;     /* [W, W, 3, 3], [W] smoothing conv */
  const void *gn_w, *gn_b;             /* [W] GroupNorm (32 groups) */
  const void *pred_w, *pred_b;         /* [K, W, 1, 1], [K] prediction conv */
} vit_dense_head_weights;

/* Attach the dense head (once per model; the model must have exactly four taps in tap_mask).
 * Makes the 3x3 weights' GEMM copies and fp32 copies of the vectors and of pred_w now; cv1_w,
 * cv2_w and lat_w are borrowed.  Call with the model's device current.
 * Projector: concat of the four final-norm taps -> 1x1 conv -> channel LN -> SiLU -> split in
 * halves a, b -> three chained bottlenecks on b (3x3 conv, channel LN, SiLU, twice; no
 * residual) -> concat a, b, the three bottleneck outputs -> 1x1 conv -> channel LN -> SiLU ->
 * final channel LN.  Task head: 1x1 lateral conv, 3x3 smoothing conv, GroupNorm(32), GELU,
 * (dropout: identity), 1x1 prediction conv, bilinear resize (align_corners = false) to H x W.
 * Channel LN: biased variance, eps 1e-6; GroupNorm eps 1e-5.  Activations between the convs
 * are bf16 (fp32 accumulation and statistics).  VIT_E_INVALID_ARG / VIT_E_UNSUPPORTED on bad
 * weights or configuration. */
vit_status vit_set_dense_head(vit_model *m, const vit_dense_head_weights *w);

/* Workspace of vit_forward_dense for B images of H x W (as vit_forward_hw's sizes). */
vit_status vit_dense_workspace_size(const vit_model *m, int32_t B, int32_t H, int32_t W, size_t *bytes);

/* Encoder + dense head on B images [B, 3, H, W] (device fp32, normalised):
 *   logits  device fp32 [B, K, H, W] class logits at the input resolution (required);
 *   p4      device fp32 [B, W, floor(H/p), floor(W/p)] projector output, or NULL.
 * Enqueues on `stream`.  VIT_E_INVALID_ARG if no dense head is attached. */
vit_status vit_forward_dense(vit_model *m, const float *images, int32_t B, int32_t H, int32_t W, float *logits,
                             float *p4, void *ws, size_t ws_bytes, vit_stream_t stream);

/* Zero-shot dense scoring ([dinotxt] patch/text alignment; whole and slide modes). */
enum { VIT_SEG_WHOLE = 0, VIT_SEG_SLIDE = 1 };

/* Workspace for vit_seg_zero_shot with these arguments (VIT_E_SHAPE / VIT_E_INVALID_ARG for
 * arguments vit_seg_zero_shot would reject). */
vit_status vit_seg_workspace_size(const vit_model *m, int32_t H, int32_t W, int32_t C, int32_t mode,
                                  int32_t side, int32_t stride, size_t *bytes);

/* image  device fp32 [3, H, W], ImageNet-normalised.
 * text   device fp32 [C, D] class embeddings (unit rows; used as given).
 * Tokens: the backbone's final-norm patch tokens, or the text head's (vit_set_text_head).
 * WHOLE: the encoder runs once on the H x W image (as vit_forward_hw: any H, W >= patch, the
 *        position embedding resized to the floor(H/p) x floor(W/p) grid); scores = bilinear
 *        (align_corners=False) upsample to H x W of the cosine map
 *        cos[c, i] = text[c] . t_i / max(||t_i||, 1e-12) over the final-LN patch tokens t.
 * SLIDE: side >= patch and side <= H, W (windows at a side other than the model's img_h x img_w
 *        use the resized position embedding); windows of side x side at `stride`, per axis
 *        ceil((size - side) / stride) + 1 origins with the last clamped to size - side; every
 *        window runs the encoder (all windows in one batch, so max_batch must cover them);
 *        per window the cosine map is upsampled to side x side, softmaxed over classes and
 *        accumulated; the sum is divided by the per-pixel window count.
 * probs  device fp32 [C, H, W] (scores in WHOLE mode, averaged probabilities in SLIDE) or NULL.
 * labels device int32 [H, W] argmax over classes (lowest index on ties) or NULL.
 * Enqueues on `stream`. */
vit_status vit_seg_zero_shot(vit_model *m, const float *image, int32_t H, int32_t W, const float *text,
                             int32_t C, int32_t mode, int32_t side, int32_t stride, float *probs,
                             int32_t *labels, void *ws, size_t ws_bytes, vit_stream_t stream);

/* The same forward as vit_forward for callers that may not allocate device memory while they
 * run (for example a plug-in whose host owns every allocation, or a latency-critical loop in
 * which an allocation could block or synchronise the device).  The pages have no counterpart:
 * this entry point is an addition of this library.
 *   The workspace comes from a fixed 64 MiB device array inside the library instead of from
 *   the caller; images and outputs are as for vit_forward and are still the caller's.  This
 *   entry point itself allocates nothing.
 *   Limit: batches whose vit_workspace_size exceeds 64 MiB are rejected with VIT_E_WORKSPACE
 *   and a message naming the size (ViT-S/16 at 336 x 336 needs about 2.8 MB per image, so up
 *   to 24 images fit; ViT-L/16 at 1024 x 1024 needs 67.5 MB and does not fit even one image).
 *   Every GPU that loads the library holds the 64 MiB until the process exits.
 *   vit_create looks up the array's device address (cudaGetSymbolAddress) on the model's
 *   device, with that device current, so a call never does that lookup itself.  The model's
 *   device must be current when this is called (VIT_E_INVALID_ARG otherwise, before any
 *   launch), so the array of another GPU is never paired with this model's weights.
 *   All calls share the one array, on every stream and model: calls whose work overlaps on
 *   the GPU race on it and must be serialised by the caller.  Nothing in it needs to start at
 *   zero; each call overwrites what it reads. */
vit_status vit_forward_noalloc(vit_model *m, const float *images, int32_t B, const vit_outputs *out,
                               vit_stream_t stream);

/* Synchronise `stream`, then read and clear the model's device status words.  Returns VIT_OK,
 * VIT_E_DEVICE_TIMEOUT if a kernel gave up on a pipeline wait since the last poll,
 * VIT_E_NONFINITE if a token row reaching the final LayerNorm held a NaN or an infinity, or
 * VIT_E_CUDA if the stream reports an error. */
vit_status vit_poll(vit_model *m, vit_stream_t stream);

/* Limit, in nanoseconds, of every pipeline wait in the model's later launches (0 restores the
 * default of 2 s, far above any real wait).  A wait that runs out makes its kernel record
 * VIT_E_DEVICE_TIMEOUT for vit_poll, let the copies and MMAs it has in flight land, free its
 * tensor memory and return; the kernels launched after it on the model find the status word
 * set and return without work until vit_poll clears it.  A limit shorter than the pipeline's
 * latency therefore exercises that path on purpose (the failure-detection test does this).
 * Host-side setting only: no launch, no synchronisation. */
vit_status vit_set_wait_limit(vit_model *m, uint64_t ns);

/* Number of kernel launches the last vit_forward / vit_forward_hw / vit_seg_zero_shot call made. */
int32_t vit_last_launch_count(const vit_model *m);

/* Per-launch timing on the caller's stream.  After vit_profile_begin(m, capacity) every kernel
 * launch of vit_forward / vit_seg_zero_shot (up to `capacity` launches in total) is bracketed by
 * two CUDA events recorded on the launch stream.  vit_profile_end synchronises those events,
 * adds up the elapsed times per kernel kind into total_ms[VIT_K_COUNT] (milliseconds) and
 * launches[VIT_K_COUNT], and switches profiling off.  Either output pointer may be NULL.
 * Launches captured into a CUDA graph while profiling is on keep their events as event-record
 * nodes: every replay records them again, and vit_profile_end reports the last replay. */
enum {
  VIT_K_IM2COL = 0, VIT_K_PATCH_GEMM, VIT_K_PREFIX, VIT_K_QKV_GEMM, VIT_K_ATTENTION, VIT_K_PROJ_GEMM,
  VIT_K_FC1_GEMM, VIT_K_FC2_GEMM, VIT_K_TAP, VIT_K_FINAL_LN, VIT_K_SEG_NORM, VIT_K_SEG_COS, VIT_K_SEG_MAP,
  VIT_K_POS_RESIZE, VIT_K_HEAD_OUT, VIT_K_DENSE_GEMM, VIT_K_DENSE_AUX, VIT_K_COUNT
};
vit_status vit_profile_begin(vit_model *m, int32_t capacity);
vit_status vit_profile_end(vit_model *m, float *total_ms, int32_t *launches);

void vit_destroy(vit_model *m);
const char *vit_status_str(vit_status s);
/* Text of the last host-side error of this thread (validation message or CUDA error). */
const char *vit_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* VIT_B200_H */
