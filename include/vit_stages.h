/*
 * vit_stages.h -- stage-level entry points of libvit_b200, exposed so that each hot kernel can
 * be checked on its own against the fp64 oracle.  They run the same kernels vit_forward runs.
 *
 * Conventions as in vit.h: device pointers, 16-byte aligned, caller-owned; work is enqueued on
 * `stream` without synchronising; `status` is a caller-allocated device int32 (zero-initialised)
 * that a kernel sets to a non-zero code if one of its pipeline waits gives up, and that every
 * kernel checks on entry (a non-zero status makes later kernels return without work).
 */
#ifndef VIT_B200_STAGES_H
#define VIT_B200_STAGES_H

#include "vit.h"

#ifdef __cplusplus
extern "C" {
#endif

/* out[M, N] = act(A[M, K] . W[N, K]^T + bias[N]) on the tcgen05 GEMM ("DINOv2 n semantic"
 * diagram, "Encoder block": the Linear layers; act = exact-erf GELU when gelu != 0).
 *   A, W: bf16, row-major, K contiguous;  bias: fp32 [N];  out: bf16 [M, N].
 *   Requires M >= 1, N a multiple of 128, K a multiple of 64.  VIT_E_SHAPE otherwise. */
vit_status vit_stage_linear(const void *A, const void *W, const float *bias, int32_t M, int32_t N, int32_t K,
                            int32_t gelu, void *out, int32_t *status, vit_stream_t stream);

/* vit_stage_linear with the limit of its pipeline waits given in nanoseconds (0: the default 2 s);
 * vit_stage_linear is this with 0.  When a wait runs out the kernel writes a non-zero code into
 * *status, lets its copies and MMAs in flight land, frees its tensor memory and returns. */
vit_status vit_stage_linear_bounded(const void *A, const void *W, const float *bias, int32_t M, int32_t N,
                                    int32_t K, int32_t gelu, void *out, int32_t *status, uint64_t wait_ns,
                                    vit_stream_t stream);

/* Multi-head self-attention core ("DINOv2 n semantic" diagram, "Encoder self-attention"):
 * for each image b and head h, out[b, :, 64h:64h+64] = softmax_keys(Q_h K_h^T / 8) V_h with
 * Q_h, K_h, V_h the 64-column slices h of the q, k and v parts of qkv[b] = [q | k | v].
 *   qkv: bf16 [B, T, 3 * 64 * heads];  out: bf16 [B, T, 64 * heads].  T >= 1, heads >= 1. */
vit_status vit_stage_attention(const void *qkv, int32_t B, int32_t T, int32_t heads, void *out, int32_t *status,
                               vit_stream_t stream);

/* vit_stage_attention with the limit of its pipeline waits given in nanoseconds (0: the default
 * 2 s), with the same behaviour on expiry as vit_stage_linear_bounded. */
vit_status vit_stage_attention_bounded(const void *qkv, int32_t B, int32_t T, int32_t heads, void *out,
                                       int32_t *status, uint64_t wait_ns, vit_stream_t stream);

/* GELU as the FC1 epilogue evaluates it ([diagram] "Encoder block": exact erf form, with erf from
 * Abramowitz & Stegun 7.1.28, absolute error <= 1.5e-7 |x| plus fp32 rounding):
 * y[i] = GELU(x[i]) for 0 <= i < n; x, y device fp32.  Enqueues on `stream`. */
vit_status vit_stage_gelu(const float *x, int64_t n, float *y, vit_stream_t stream);

/* Position-embedding resize ([diagram] "DINOv2-S encoder": "Bicubic interpolation" of the
 * learned grid to the input's patch grid), the kernel vit_forward_hw runs first:
 *   pos: fp32 [(pos_on_cls ? 1 : 0) + gh0 * gw0, D], the patch rows in row-major grid order;
 *   out: fp32 [(pos_on_cls ? 1 : 0) + gh * gw, D]; the CLS row (if any) is copied, the patch
 *   rows are the separable cubic-convolution resize (Keys' kernel, a = -0.75, half-pixel
 *   centres, taps clamped to the border) of the gh0 x gw0 grid to gh x gw.
 * Grids 1..4096 per side (VIT_E_SHAPE otherwise).  Enqueues on `stream`. */
vit_status vit_stage_pos_resize(const float *pos, int32_t gh0, int32_t gw0, int32_t gh, int32_t gw, int32_t D,
                                int32_t pos_on_cls, float *out, vit_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* VIT_B200_STAGES_H */
