// Dense head on the four taps (LibreYOLO DINOv2 configuration diagram: "Projector P4",
// "Projector Bottleneck", "Projector output ConvX", "Task head").  Activations are pixel-major
// bf16 rows [B * gh * gw, C]: every 1x1 conv is then a GEMM on the tcgen05 GEMM kernel, and
// every 3x3 conv a GEMM over an im2col matrix whose column k = (ky * 3 + kx) * C + c.  The
// kernels here are the memory-bound pieces around those GEMMs: building the tap concat,
// per-pixel channel LayerNorm (+ SiLU), the 3x3 im2col, GroupNorm + GELU, the 1x1 prediction
// conv to the class logits and the bilinear resize to the input size.
#pragma once

#include "aux_kernels.cuh"
#include "gelu.cuh"

namespace vit {

// [diagram] "Taps apply LayerNorm, remove CLS, reshape", "Concat four selected features":
// out[b * P + p, col0 + d] = bf16(LN_final(x[b, 1 + R + p])[d]).  One warp per patch row.
__global__ void tap_rows_kernel(const float* __restrict__ x, const float* __restrict__ g, const float* __restrict__ be,
                                int B, int T, int R, int D, float eps, __nv_bfloat16* __restrict__ out, int ld,
                                int col0) {
  const int P = T - 1 - R;
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= static_cast<long long>(B) * P) return;
  const int lane = threadIdx.x & 31;
  const int b = static_cast<int>(row / P);
  const int p = static_cast<int>(row - static_cast<long long>(b) * P);
  const float* xr = x + (static_cast<size_t>(b) * T + 1 + R + p) * D;
  float mean, rstd;
  row_mean_rstd(xr, D, eps, mean, rstd);
  __nv_bfloat16* o = out + static_cast<size_t>(row) * ld + col0;
  for (int n = lane; n < D; n += 32) o[n] = __float2bfloat16_rn((xr[n] - mean) * rstd * g[n] + be[n]);
}

// [diagram] "Channel LayerNorm" then "SiLU" on each pixel row of C channels (C = 128 or 256):
// biased variance, eps inside the square root.  mode 0: LN, SiLU.  mode 1 (projector output):
// LN, SiLU, then the final channel LN with (g2, b2).  Values are kept in registers (C / 32 per
// lane); one warp per row.
__global__ void row_ln_silu_kernel(const __nv_bfloat16* __restrict__ in, int ld_in, long long rows, int C,
                                   const float* __restrict__ g, const float* __restrict__ b, const float* __restrict__ g2,
                                   const float* __restrict__ b2, float eps, int mode, __nv_bfloat16* __restrict__ out,
                                   int ld_out, int col0) {
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const int per = C / 32;  // 4 or 8
  const __nv_bfloat16* r = in + static_cast<size_t>(row) * ld_in;
  float v[8];
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < per) {
      v[j] = __bfloat162float(r[j * 32 + lane]);
      s += v[j];
    }
  float mean = warp_sum(s) / static_cast<float>(C);
  float q = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < per) {
      const float d = v[j] - mean;
      q = fmaf(d, d, q);
    }
  float rstd = rsqrtf(warp_sum(q) / static_cast<float>(C) + eps);
  s = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < per) {
      const int n = j * 32 + lane;
      const float y = (v[j] - mean) * rstd * g[n] + b[n];
      v[j] = y / (1.f + __expf(-y));  // SiLU
      s += v[j];
    }
  if (mode == 1) {
    mean = warp_sum(s) / static_cast<float>(C);
    q = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < per) {
        const float d = v[j] - mean;
        q = fmaf(d, d, q);
      }
    rstd = rsqrtf(warp_sum(q) / static_cast<float>(C) + eps);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < per) {
        const int n = j * 32 + lane;
        v[j] = (v[j] - mean) * rstd * g2[n] + b2[n];
      }
  }
  __nv_bfloat16* o = out + static_cast<size_t>(row) * ld_out + col0;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < per) o[j * 32 + lane] = __float2bfloat16_rn(v[j]);
}

// im2col of a 3x3, stride-1, zero-padded conv on pixel-major rows: A[b * P + y * gw + x,
// (ky * 3 + kx) * C + c] = in[b, y + ky - 1, x + kx - 1, col0 + c] (0 outside the grid).
// 8 channels (16 bytes) per thread; C and col0 multiples of 8, ld_in a multiple of 8.
__global__ void im2col3x3_kernel(const __nv_bfloat16* __restrict__ in, int ld_in, int col0, int C, int B, int gh,
                                 int gw, __nv_bfloat16* __restrict__ A) {
  const int c8n = C / 8;
  const long long total = static_cast<long long>(B) * gh * gw * 9 * c8n;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c8 = static_cast<int>(i % c8n);
    const long long t = i / c8n;
    const int tap = static_cast<int>(t % 9);
    const long long pix = t / 9;
    const int P = gh * gw;
    const int b = static_cast<int>(pix / P);
    const int pi = static_cast<int>(pix - static_cast<long long>(b) * P);
    const int y = pi / gw + tap / 3 - 1, x = pi % gw + tap % 3 - 1;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (y >= 0 && y < gh && x >= 0 && x < gw)
      v = *reinterpret_cast<const uint4*>(in + (static_cast<size_t>(b) * P + y * gw + x) * ld_in + col0 + c8 * 8);
    *reinterpret_cast<uint4*>(A + static_cast<size_t>(pix) * 9 * C + tap * C + c8 * 8) = v;
  }
}

// Weight of a 3x3 conv [O, C, 3, 3] (bf16) as the GEMM's B operand [O, 9 C] with column
// (ky * 3 + kx) * C + c, matching im2col3x3_kernel.  Run once when the head is attached.
__global__ void conv3x3_weight_kernel(const __nv_bfloat16* __restrict__ w, int O, int C,
                                      __nv_bfloat16* __restrict__ out) {
  const long long total = static_cast<long long>(O) * 9 * C;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i % C);
    const long long t = i / C;
    const int tap = static_cast<int>(t % 9);
    const int o = static_cast<int>(t / 9);
    out[i] = w[(static_cast<size_t>(o) * C + c) * 9 + tap];
  }
}

// [diagram] "GroupNorm: 32 groups, 256 channels": per image and group, the mean and the sum of
// squared deviations over the group's C/G channels and all P pixels (two passes over the
// L2-resident rows).  One block per (group, image).
__global__ void group_norm_stats_kernel(const __nv_bfloat16* __restrict__ in, int P, int C, int G,
                                        float2* __restrict__ stats) {
  const int gi = blockIdx.x, b = blockIdx.y;
  const int cg = C / G;
  const long long n = static_cast<long long>(P) * cg;
  const __nv_bfloat16* base = in + static_cast<size_t>(b) * P * C + gi * cg;
  __shared__ float red[32];
  float s = 0.f;
  for (long long i = threadIdx.x; i < n; i += blockDim.x)
    s += __bfloat162float(base[(i / cg) * C + (i % cg)]);
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const float mean = red[0] / static_cast<float>(n);
  __syncthreads();
  float q = 0.f;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) {
    const float d = __bfloat162float(base[(i / cg) * C + (i % cg)]) - mean;
    q = fmaf(d, d, q);
  }
  q = warp_sum(q);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = q;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) stats[b * G + gi] = make_float2(mean, t);
  }
}

// GroupNorm affine + GELU ("Dropout2d (eval identity)" is the identity), bf16 in and out.
__global__ void group_norm_gelu_kernel(const __nv_bfloat16* __restrict__ in, long long rows, int P, int C, int G,
                                       const float2* __restrict__ stats, const float* __restrict__ g,
                                       const float* __restrict__ be, float eps, __nv_bfloat16* __restrict__ out) {
  const long long total = rows * C / 2;
  const int cg = C / G;
  const float inv_n = 1.f / static_cast<float>(static_cast<long long>(P) * cg);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long e = 2 * i;
    const int c = static_cast<int>(e % C);
    const int b = static_cast<int>((e / C) / P);
    const float2 st = stats[b * G + c / cg];  // c and c + 1 share a group (cg even)
    const float rstd = rsqrtf(st.y * inv_n + eps);
    const __nv_bfloat162 v = reinterpret_cast<const __nv_bfloat162*>(in)[i];
    const float y0 = (__bfloat162float(v.x) - st.x) * rstd * g[c] + be[c];
    const float y1 = (__bfloat162float(v.y) - st.x) * rstd * g[c + 1] + be[c + 1];
    const float2 r = gelu2(make_float2(y0, y1));
    reinterpret_cast<__nv_bfloat162*>(out)[i] = __floats2bfloat162_rn(r.x, r.y);
  }
}

// [diagram] "Predict Conv2d 1x1: 256 to 19 class logits": lr[b, k, p] = w[k] . h[b * P + p] +
// bias[k], fp32, channels first for the resize.  One warp per pixel: each lane holds 8 of the
// 256 channels, the dot products are reduced across the warp.
__global__ void predict_kernel(const __nv_bfloat16* __restrict__ h, long long rows, int P, int C,
                               const float* __restrict__ w, const float* __restrict__ bias, int K,
                               float* __restrict__ lr) {
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const int per = C / 32;
  float v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < per) v[j] = __bfloat162float(h[static_cast<size_t>(row) * C + j * 32 + lane]);
  const int b = static_cast<int>(row / P);
  const int p = static_cast<int>(row - static_cast<long long>(b) * P);
  for (int k = 0; k < K; ++k) {
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < per) s = fmaf(w[static_cast<size_t>(k) * C + j * 32 + lane], v[j], s);
    s = warp_sum(s);
    if (lane == 0) lr[(static_cast<size_t>(b) * K + k) * P + p] = s + bias[k];
  }
}

// [diagram] "Bilinear resize 19 x 518 x 518, align_corners=False": out[b, k, y, x] from the
// gh x gw logits, half-pixel centres with the source clamped at 0 (the convention of
// F.interpolate).  One thread per output pixel, looping over the K classes.
__global__ void resize_logits_kernel(const float* __restrict__ lr, int B, int K, int gh, int gw, int H, int W,
                                     float* __restrict__ out) {
  const long long total = static_cast<long long>(B) * H * W;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int x = static_cast<int>(i % W);
    const long long t = i / W;
    const int y = static_cast<int>(t % H);
    const int b = static_cast<int>(t / H);
    const Taps1D ty = bilinear_taps(y, gh, H);
    const Taps1D tx = bilinear_taps(x, gw, W);
    const float w00 = (1.f - ty.w1) * (1.f - tx.w1), w01 = (1.f - ty.w1) * tx.w1;
    const float w10 = ty.w1 * (1.f - tx.w1), w11 = ty.w1 * tx.w1;
    const int o00 = ty.i0 * gw + tx.i0, o01 = ty.i0 * gw + tx.i1, o10 = ty.i1 * gw + tx.i0, o11 = ty.i1 * gw + tx.i1;
    const size_t plane = static_cast<size_t>(H) * W;
    for (int k = 0; k < K; ++k) {
      const float* s = lr + (static_cast<size_t>(b) * K + k) * gh * gw;
      out[(static_cast<size_t>(b) * K + k) * plane + static_cast<size_t>(y) * W + x] =
          w00 * s[o00] + w01 * s[o01] + w10 * s[o10] + w11 * s[o11];
    }
  }
}

// Projector output as fp32 channels-first features [B, C, gh * gw] (optional output).
__global__ void rows_to_chw_kernel(const __nv_bfloat16* __restrict__ in, int B, int P, int C, float* __restrict__ out) {
  const long long total = static_cast<long long>(B) * P * C;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i % P);
    const long long t = i / P;
    const int c = static_cast<int>(t % C);
    const int b = static_cast<int>(t / C);
    out[i] = __bfloat162float(in[(static_cast<size_t>(b) * P + p) * C + c]);
  }
}

}  // namespace vit
