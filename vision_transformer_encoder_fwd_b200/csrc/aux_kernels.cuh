// Memory-bound kernels of the encoder forward and of the zero-shot scoring, plus the one-time
// weight preparation run by vit_create.  None of these touches tensor cores: they are
// HBM/L2-bound and laid out for coalesced 16-byte (or 4-byte per lane) accesses.
#pragma once

#include "common.cuh"
#include "gelu.cuh"

namespace vit {

// Source of the encoder's input pixels.  Image b of the batch is read at
//   ptr[b * img_stride + c * chan_stride + (oy + y) * row_stride + (ox + x)]
// with the window origin (oy, ox) of batch entry b = iy * nx + ix given by
//   oy = min(iy * win_stride, max_oy), ox = min(ix * win_stride, max_ox)
// (nx = 1, win_stride = 0 for a plain batch of images).
struct ImgSrc {
  const float* ptr;
  long long img_stride, chan_stride, row_stride;
  int nx, win_stride, max_oy, max_ox;
};

// kornia/dinov3 card "Model I/O" + "DINOv2 n semantic" diagram "Conv2d p x p / p": the
// patch convolution as a GEMM needs A[b*P + p, k] = bf16(pixel), k = c*p^2 + ky*p + kx, zero
// for k >= 3 p^2 up to Kpad.  Each thread writes 8 consecutive k (one 16-byte store).  VEC:
// p is a multiple of 8 and every row start, window origin and stride is a multiple of 4 floats,
// so the 8 pixels of a thread lie in one image row and load as two 16-byte vectors.
template <bool VEC>
__global__ void im2col_bf16_kernel(ImgSrc src, int B, int p, int gw, int P, int Kpad, __nv_bfloat16* __restrict__ A) {
  pdl_launch_dependents();
  const int kv = Kpad / 8;
  const long long total = static_cast<long long>(B) * P * kv;
  const int pp = p * p;
  const int K = 3 * pp;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int k8 = static_cast<int>(i % kv);
    const long long row = i / kv;
    const int b = static_cast<int>(row / P);
    const int pi = static_cast<int>(row - static_cast<long long>(b) * P);
    const int gy = pi / gw, gx = pi - gy * gw;
    const int iy = b / src.nx, ix = b - iy * src.nx;
    const int oy = min(iy * src.win_stride, src.max_oy) + gy * p;
    const int ox = min(ix * src.win_stride, src.max_ox) + gx * p;
    const float* base = src.ptr + b * src.img_stride;
    float v[8];
    if (VEC) {
      const int k = k8 * 8;
      if (k < K) {
        const int c = k / pp;
        const int rem = k - c * pp;
        const int ky = rem / p, kx = rem - ky * p;
        const float4* q = reinterpret_cast<const float4*>(base + c * src.chan_stride +
                                                          static_cast<long long>(oy + ky) * src.row_stride + (ox + kx));
        const float4 lo = __ldg(q), hi = __ldg(q + 1);
        v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
        v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = 0.f;
      }
    } else {
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int k = k8 * 8 + t;
        float x = 0.f;
        if (k < K) {
          const int c = k / pp;
          const int rem = k - c * pp;
          const int ky = rem / p, kx = rem - ky * p;
          x = __ldg(base + c * src.chan_stride + static_cast<long long>(oy + ky) * src.row_stride + (ox + kx));
        }
        v[t] = x;
      }
    }
    uint4 w;
    w.x = pack_bf16x2(v[0], v[1]);
    w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]);
    w.w = pack_bf16x2(v[6], v[7]);
    reinterpret_cast<uint4*>(A + row * Kpad)[k8] = w;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Token rows of the residual stream before block 1, whole rows at a time: the CLS and register
// rows are written here ([card] "Model I/O": CLS, then the registers, no position embedding on
// them; [diagram] position embedding row 0 on CLS for DINOv2), the patch rows were written by
// the patch GEMM.  For every row this kernel then writes what the folded LayerNorm of block 1
// reads: the (mean, M2) partial statistics of each group of gcols columns, the row mean as the
// centre, and the re-centred bf16 copy xb = bf16(x - centre).  One warp per row; lane l owns
// the columns 128 c + 4 l .. + 3 (float4 accesses); gcols is 64 or 128.
__global__ void token_prep_kernel(const float* __restrict__ cls, const float* __restrict__ reg,
                                  const float* __restrict__ pos, int pos_on_cls, long long rows, int T, int R, int D,
                                  int gcols, float* __restrict__ x, __nv_bfloat16* __restrict__ xb,
                                  float2* __restrict__ stats, float* __restrict__ ctr) {
  pdl_wait();  // launched to start early: global memory only after the previous kernel
  pdl_launch_dependents();
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const int t = static_cast<int>(row % T);
  float* xr = x + static_cast<size_t>(row) * D;
  const int lpg = gcols / 4;  // lanes per statistics group within a 128-column chunk
  const int ng = D / gcols;
  float lsum = 0.f;
  for (int c = 0; c < D / 128; ++c) {
    const int n = c * 128 + lane * 4;
    float4 v;
    if (t <= R) {
      if (t == 0) {
        v = *reinterpret_cast<const float4*>(cls + n);
        if (pos_on_cls) {
          const float4 p = *reinterpret_cast<const float4*>(pos + n);
          v.x += p.x;
          v.y += p.y;
          v.z += p.z;
          v.w += p.w;
        }
      } else {
        v = *reinterpret_cast<const float4*>(reg + static_cast<size_t>(t - 1) * D + n);
      }
      *reinterpret_cast<float4*>(xr + n) = v;
    } else {
      v = *reinterpret_cast<const float4*>(xr + n);
    }
    float s = (v.x + v.y) + (v.z + v.w);
    lsum += s;
    for (int o = lpg / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float gm = s / static_cast<float>(gcols);
    const float d0 = v.x - gm, d1 = v.y - gm, d2 = v.z - gm, d3 = v.w - gm;
    float q = (d0 * d0 + d1 * d1) + (d2 * d2 + d3 * d3);
    for (int o = lpg / 2; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    if (lane % lpg == 0) stats[static_cast<size_t>(row) * ng + (n / gcols)] = make_float2(gm, q);
  }
  const float centre = warp_sum(lsum) / static_cast<float>(D);
  for (int c = 0; c < D / 128; ++c) {
    const int n = c * 128 + lane * 4;
    const float4 v = *reinterpret_cast<const float4*>(xr + n);
    uint2 w;
    w.x = pack_bf16x2(v.x - centre, v.y - centre);
    w.y = pack_bf16x2(v.z - centre, v.w - centre);
    *reinterpret_cast<uint2*>(xb + static_cast<size_t>(row) * D + n) = w;
  }
  if (lane == 0) ctr[row] = centre;
}

// [diagram] "DINOv2-S encoder": the learned position grid goes through "Bicubic
// interpolation" to the input's patch grid.  Separable cubic convolution with Keys' kernel
// (a = -0.75), half-pixel centres (source coordinate (i + 1/2) * in/out - 1/2, not clamped),
// the four taps of each axis clamped to the border; a CLS row (pos_off = 1) is copied as is.
// One thread per output element, D innermost: a warp reads 32 consecutive floats of each of
// the 16 source rows it touches.
__device__ __forceinline__ void keys_cubic_weights(float t, float w[4]) {
  const float a = -0.75f;
  // |x| <= 1: ((a + 2)|x| - (a + 3)) x^2 + 1;   1 < |x| < 2: a|x|^3 - 5a x^2 + 8a|x| - 4a
  auto near = [a](float x) { return ((a + 2.f) * x - (a + 3.f)) * x * x + 1.f; };
  auto far = [a](float x) { return ((a * x - 5.f * a) * x + 8.f * a) * x - 4.f * a; };
  w[0] = far(1.f + t);
  w[1] = near(t);
  w[2] = near(1.f - t);
  w[3] = far(2.f - t);
}

__global__ void pos_resize_kernel(const float* __restrict__ pos0, int gh0, int gw0, int gh, int gw, int D, int pos_off,
                                  float* __restrict__ out) {
  const long long total = static_cast<long long>(pos_off + gh * gw) * D;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int d = static_cast<int>(i % D);
    const int r = static_cast<int>(i / D);
    if (r < pos_off) {
      out[i] = pos0[i];
      continue;
    }
    const int pi = r - pos_off, py = pi / gw, px = pi - py * gw;
    const float sy = (static_cast<float>(py) + 0.5f) * (static_cast<float>(gh0) / static_cast<float>(gh)) - 0.5f;
    const float sx = (static_cast<float>(px) + 0.5f) * (static_cast<float>(gw0) / static_cast<float>(gw)) - 0.5f;
    const float fy = floorf(sy), fx = floorf(sx);
    float wy[4], wx[4];
    keys_cubic_weights(sy - fy, wy);
    keys_cubic_weights(sx - fx, wx);
    const int iy = static_cast<int>(fy) - 1, ix = static_cast<int>(fx) - 1;
    const float* base = pos0 + static_cast<size_t>(pos_off) * D + d;
    float acc = 0.f;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int yy = min(max(iy + a, 0), gh0 - 1);
      float rowv = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int xx = min(max(ix + c, 0), gw0 - 1);
        rowv = fmaf(wx[c], base[static_cast<size_t>(yy * gw0 + xx) * D], rowv);
      }
      acc = fmaf(wy[a], rowv, acc);
    }
    out[i] = acc;
  }
}

// Row LayerNorm statistics with one warp per row, two passes over the row (L1/L2-resident on
// the second pass): biased variance, eps inside the square root ([diagram] "Encoder block").
__device__ __forceinline__ void row_mean_rstd(const float* __restrict__ xr, int D, float eps, float& mean, float& rstd) {
  const int lane = threadIdx.x & 31;
  float s = 0.f;
  for (int n = lane; n < D; n += 32) s += xr[n];
  mean = warp_sum(s) / static_cast<float>(D);
  float q = 0.f;
  for (int n = lane; n < D; n += 32) {
    const float d = xr[n] - mean;
    q = fmaf(d, d, q);
  }
  q = warp_sum(q);
  rstd = rsqrtf(q / static_cast<float>(D) + eps);
}

// Final LayerNorm and the encoder's outputs: the L2-normalised CLS descriptor ([card]
// "Usage": "L2-normed [384], cosine-ready"; "Model I/O": descriptor = CLS token) and the
// patch tokens (CLS and the R registers skipped, [card] "Model I/O").  One warp per
// (image, token) with token 0 (CLS) or 1 + R .. T - 1 (patches).
__global__ void final_ln_kernel(const float* __restrict__ x, const float* __restrict__ g, const float* __restrict__ be,
                                int B, int T, int R, int D, float eps, float* __restrict__ desc, void* __restrict__ patch,
                                int patch_fp32, int* __restrict__ nonfinite) {
  pdl_wait();  // launched to start early: global memory only after the previous kernel
  pdl_launch_dependents();
  const int P = T - 1 - R;
  const int warps_per_block = blockDim.x >> 5;
  const long long job = static_cast<long long>(blockIdx.x) * warps_per_block + (threadIdx.x >> 5);
  const long long njobs = static_cast<long long>(B) * (1 + P);
  if (job >= njobs) return;
  const int lane = threadIdx.x & 31;
  const int b = static_cast<int>(job / (1 + P));
  const int j = static_cast<int>(job - static_cast<long long>(b) * (1 + P));
  const int t = (j == 0) ? 0 : (j + R);
  const float* xr = x + (static_cast<size_t>(b) * T + t) * D;
  float mean, rstd;
  row_mean_rstd(xr, D, eps, mean, rstd);
  // a NaN or infinity anywhere in the row reaches its mean or its rstd
  if (lane == 0 && !(isfinite(mean) && isfinite(rstd))) atomicExch(nonfinite, 1);
  if (j == 0) {
    if (desc == nullptr) return;
    float q = 0.f;
    for (int n = lane; n < D; n += 32) {
      const float v = (xr[n] - mean) * rstd * g[n] + be[n];
      q = fmaf(v, v, q);
    }
    q = warp_sum(q);
    const float inv = 1.0f / fmaxf(sqrtf(q), 1e-12f);
    for (int n = lane; n < D; n += 32) desc[static_cast<size_t>(b) * D + n] = ((xr[n] - mean) * rstd * g[n] + be[n]) * inv;
  } else {
    if (patch == nullptr) return;
    const size_t o = (static_cast<size_t>(b) * P + (j - 1)) * D;
    if (patch_fp32) {
      float* dst = static_cast<float*>(patch) + o;
      for (int n = lane; n < D; n += 32) dst[n] = (xr[n] - mean) * rstd * g[n] + be[n];
    } else {
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(patch) + o;
      for (int n = lane; n < D; n += 32) dst[n] = __float2bfloat16_rn((xr[n] - mean) * rstd * g[n] + be[n]);
    }
  }
}

// [dino.txt article] the vision head's 2 blocks run on the backbone's final-norm sequence: the
// final LayerNorm applied in place to every row of the residual stream x (CLS, registers and
// patches), with the bf16 copy xb and the per-group (mean, M2) statistics that the first head
// block's folded LN1 reads -- the state a backbone block leaves behind.  One warp per row; each
// group of gcols (64 or 128) columns is kept in registers between its two passes.
__global__ void final_ln_stream_kernel(float* __restrict__ x, const float* __restrict__ g,
                                       const float* __restrict__ be, long long rows, int D, float eps, int gcols,
                                       __nv_bfloat16* __restrict__ xb, float2* __restrict__ stats,
                                       float* __restrict__ ctr, int* __restrict__ nonfinite) {
  pdl_wait();  // launched to start early: global memory only after the previous kernel
  pdl_launch_dependents();
  const int warps_per_block = blockDim.x >> 5;
  const long long row = static_cast<long long>(blockIdx.x) * warps_per_block + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  float* xr = x + static_cast<size_t>(row) * D;
  float mean, rstd;
  row_mean_rstd(xr, D, eps, mean, rstd);
  if (lane == 0 && !(isfinite(mean) && isfinite(rstd))) atomicExch(nonfinite, 1);
  __syncwarp();
  const int per = gcols / 32;  // 2 or 4
  const int ng = D / gcols;
  float tot = 0.f;
  for (int gi = 0; gi < ng; ++gi) {
    float v[4];
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j < per) {
        const int n = gi * gcols + j * 32 + lane;
        v[j] = (xr[n] - mean) * rstd * g[n] + be[n];
        s += v[j];
      }
    }
    const float gs = warp_sum(s);
    tot += gs;
    const float gm = gs / static_cast<float>(gcols);
    float q = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j < per) {
        const int n = gi * gcols + j * 32 + lane;
        const float d = v[j] - gm;
        q = fmaf(d, d, q);
        xr[n] = v[j];
      }
    }
    q = warp_sum(q);
    if (lane == 0) stats[static_cast<size_t>(row) * ng + gi] = make_float2(gm, q);
  }
  // the head's first folded LayerNorm reads the re-centred copy bf16(x - centre), centre = the
  // normalised row's mean (each lane re-reads the columns it has just written)
  const float centre = tot / static_cast<float>(D);
  for (int n = lane; n < D; n += 32) xb[static_cast<size_t>(row) * D + n] = __float2bfloat16_rn(xr[n] - centre);
  if (lane == 0) ctr[row] = centre;
}

// The patch rows of the residual stream, fp32: tok[b, p, :] = x[b, 1 + R + p, :] (the dino.txt
// head's output tokens, CLS and registers dropped).  float4 copies, grid-stride.
__global__ void patch_rows_kernel(const float* __restrict__ x, int B, int T, int R, int D, float* __restrict__ tok) {
  pdl_wait();  // launched to start early: global memory only after the previous kernel
  pdl_launch_dependents();
  const int P = T - 1 - R;
  const int d4 = D / 4;
  const long long total = static_cast<long long>(B) * P * d4;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i % d4);
    const long long r = i / d4;
    const int b = static_cast<int>(r / P);
    const int p = static_cast<int>(r - static_cast<long long>(b) * P);
    reinterpret_cast<float4*>(tok)[i] =
        reinterpret_cast<const float4*>(x + (static_cast<size_t>(b) * T + 1 + R + p) * D)[c];
  }
}

// Taps ([diagram] "Tap stage l: 384 x 37 x 37"; "Taps apply LayerNorm, remove CLS, reshape"):
// out[b, d, p] = LN_final(x[b, 1 + R + p])[d], channels first.  Block = 32 patches of one image:
// 8 warps compute the 32 row statistics, then 32 x 32 tiles are transposed through shared
// memory so that both the read (along d) and the write (along p) are coalesced.
__global__ void tap_kernel(const float* __restrict__ x, const float* __restrict__ g, const float* __restrict__ be, int T,
                           int R, int D, float eps, float* __restrict__ out) {
  pdl_wait();  // launched to start early: global memory only after the previous kernel
  pdl_launch_dependents();
  __shared__ float tile[32][33];
  __shared__ float s_mean[32], s_rstd[32];
  const int P = T - 1 - R;
  const int b = blockIdx.y;
  const int p0 = blockIdx.x * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = warp; i < 32; i += 8) {
    const int p = p0 + i;
    float mean = 0.f, rstd = 0.f;
    if (p < P) row_mean_rstd(x + (static_cast<size_t>(b) * T + 1 + R + p) * D, D, eps, mean, rstd);
    if (lane == 0) {
      s_mean[i] = mean;
      s_rstd[i] = rstd;
    }
  }
  __syncthreads();
  for (int d0 = 0; d0 < D; d0 += 32) {
    for (int i = warp; i < 32; i += 8) {
      const int p = p0 + i;
      const int d = d0 + lane;
      float v = 0.f;
      if (p < P) v = (x[(static_cast<size_t>(b) * T + 1 + R + p) * D + d] - s_mean[i]) * s_rstd[i] * g[d] + be[d];
      tile[i][lane] = v;
    }
    __syncthreads();
    for (int i = warp; i < 32; i += 8) {
      const int d = d0 + i;
      const int p = p0 + lane;
      if (p < P) out[(static_cast<size_t>(b) * D + d) * P + p] = tile[lane][i];
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ weight preparation
// LayerNorm folded into the following Linear (exact algebra, gamma/beta of the LayerNorm,
// W [N, K] of the Linear):
//   LN(x) W^T + b = rstd * (x Wg^T - mean * colsum(Wg)) + (b + W beta),  Wg[n, k] = gamma_k W[n, k]
// This kernel writes Wg in bf16, colsum over the bf16 Wg (so the mean term cancels the
// operand the MMA actually multiplies) and the folded bias in fp32.  One block per row n.
__global__ void fold_ln_weight_kernel(const __nv_bfloat16* __restrict__ W, const __nv_bfloat16* __restrict__ bias,
                                      const __nv_bfloat16* __restrict__ gamma, const __nv_bfloat16* __restrict__ beta,
                                      int N, int K, __nv_bfloat16* __restrict__ Wg, float* __restrict__ colsum,
                                      float* __restrict__ bias_out) {
  __shared__ double red[2][32];
  const int n = blockIdx.x;
  double cs = 0.0, bb = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const float w = __bfloat162float(W[static_cast<size_t>(n) * K + k]);
    const __nv_bfloat16 wg = __float2bfloat16_rn(w * __bfloat162float(gamma[k]));
    Wg[static_cast<size_t>(n) * K + k] = wg;
    cs += static_cast<double>(__bfloat162float(wg));
    bb += static_cast<double>(w) * static_cast<double>(__bfloat162float(beta[k]));
  }
  for (int o = 16; o > 0; o >>= 1) {
    cs += __shfl_xor_sync(0xffffffffu, cs, o);
    bb += __shfl_xor_sync(0xffffffffu, bb, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red[0][warp] = cs;
    red[1][warp] = bb;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, c = 0.0;
    for (int w = 0; w < (blockDim.x >> 5); ++w) {
      a += red[0][w];
      c += red[1][w];
    }
    colsum[n] = static_cast<float>(a);
    bias_out[n] = static_cast<float>(static_cast<double>(__bfloat162float(bias[n])) + c);
  }
}

// Patch-embedding weight [D, 3 p^2] copied into [D, Kpad] with zero columns past 3 p^2.
__global__ void pad_rows_bf16_kernel(const __nv_bfloat16* __restrict__ src, int rows, int K, int Kpad,
                                     __nv_bfloat16* __restrict__ dst) {
  const long long total = static_cast<long long>(rows) * Kpad;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / Kpad;
    const int k = static_cast<int>(i - r * Kpad);
    dst[i] = (k < K) ? src[r * K + k] : __float2bfloat16_rn(0.f);
  }
}

__global__ void bf16_to_f32_kernel(const __nv_bfloat16* __restrict__ src, long long n, float* __restrict__ dst) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    dst[i] = __bfloat162float(src[i]);
}

// ------------------------------------------------------------------ zero-shot scoring
// [dinotxt] patch/text alignment: cos[w, c, i] = text[c] . t_i / max(||t_i||, 1e-12) (F.normalize
// of the patch tokens, then einsum("cd,hwd->chw") with the unit text features), computed on the
// tensor cores as one bf16 GEMM whose operands carry fp32-grade values: each fp32 value v is split
// as v = hi + lo with hi = bf16(v) and lo = bf16(v - hi), and the K dimension is tripled so that
//   [hi_t | hi_t | lo_t] . [hi_c | lo_c | hi_c] = hi_t hi_c + hi_t lo_c + lo_t hi_c,
// which leaves out only lo_t lo_c (relative 2^-16 of each product) and the bf16 rounding of lo
// (2^-17): the cosines keep about 16 significant bits instead of bf16's 8.
//
// Step 1: the token rows, normalised and split: A3[r] = [hi | hi | lo] of t_r / max(||t_r||, 1e-12)
// (one warp per row, fp32).
__global__ void cos_split_tokens_kernel(const float* __restrict__ tok, long long rows, int D,
                                        __nv_bfloat16* __restrict__ a3) {
  const long long r = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const float* t = tok + r * D;
  float q = 0.f;
  for (int n = lane; n < D; n += 32) q = fmaf(t[n], t[n], q);
  const float inv = 1.0f / fmaxf(sqrtf(warp_sum(q)), 1e-12f);
  __nv_bfloat16* o = a3 + r * 3 * D;
  for (int n = lane; n < D; n += 32) {
    const float v = t[n] * inv;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    o[n] = hi;
    o[D + n] = hi;
    o[2 * D + n] = lo;
  }
}

// Step 2: the class rows, split the other way: B3[c] = [hi | lo | hi] of text[c] for c < C, zero
// rows up to Cpad (one warp per row).
__global__ void cos_split_text_kernel(const float* __restrict__ text, int C, int Cpad, int D,
                                      __nv_bfloat16* __restrict__ b3) {
  const int c = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (c >= Cpad) return;
  const int lane = threadIdx.x & 31;
  __nv_bfloat16* o = b3 + static_cast<size_t>(c) * 3 * D;
  for (int n = lane; n < D; n += 32) {
    const float v = (c < C) ? text[static_cast<size_t>(c) * D + n] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    o[n] = hi;
    o[D + n] = lo;
    o[2 * D + n] = hi;
  }
}
// Step 3 is the tcgen05 GEMM A3 . B3^T with the EPI_COS epilogue (gemm.cuh), which scatters the
// fp32 results to cos[w, c, p].

// Bilinear source taps of output index i for an in -> out resize with align_corners=False:
// src = (i + 0.5) * in / out - 0.5 clamped below at 0; neighbours floor(src) and
// min(floor + 1, in - 1); weight of the upper one = fractional part.
struct Taps1D {
  int i0, i1;
  float w1;
};
__device__ __forceinline__ Taps1D bilinear_taps(int i, int n_in, int n_out) {
  float src = (static_cast<float>(i) + 0.5f) * (static_cast<float>(n_in) / static_cast<float>(n_out)) - 0.5f;
  src = fmaxf(src, 0.f);
  int i0 = min(static_cast<int>(src), n_in - 1);
  Taps1D t;
  t.i0 = i0;
  t.i1 = min(i0 + 1, n_in - 1);
  t.w1 = src - static_cast<float>(i0);
  return t;
}

// Slide mode (dino.txt article, whole/slide section): for every pixel, the windows covering it
// (at most 6 here) each contribute softmax_c(bilinear(cos_w)) and the sum is divided by the
// covering count; label = argmax_c (lowest index on ties).  Gather form: each thread owns one
// pixel and visits its windows, so probs is written exactly once and no atomics are needed.
__global__ void seg_slide_kernel(const float* __restrict__ cosm, int C, int g, int H, int W, int side, int stride, int ny,
                                 int nx, float* __restrict__ probs, int* __restrict__ labels) {
  const long long pix = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (pix >= static_cast<long long>(H) * W) return;
  const int y = static_cast<int>(pix / W), x = static_cast<int>(pix - static_cast<long long>(y) * W);
  constexpr int MAXW = 16;
  int off[MAXW][4];
  float wt[MAXW][4];
  int nw = 0;
  for (int iy = 0; iy < ny; ++iy) {
    const int oy = min(iy * stride, H - side);
    if (y < oy || y >= oy + side) continue;
    const Taps1D ty = bilinear_taps(y - oy, g, side);
    for (int ix = 0; ix < nx; ++ix) {
      const int ox = min(ix * stride, W - side);
      if (x < ox || x >= ox + side || nw >= MAXW) continue;
      const Taps1D tx = bilinear_taps(x - ox, g, side);
      const int base = (iy * nx + ix) * C * g * g;
      off[nw][0] = base + ty.i0 * g + tx.i0;
      off[nw][1] = base + ty.i0 * g + tx.i1;
      off[nw][2] = base + ty.i1 * g + tx.i0;
      off[nw][3] = base + ty.i1 * g + tx.i1;
      wt[nw][0] = (1.f - ty.w1) * (1.f - tx.w1);
      wt[nw][1] = (1.f - ty.w1) * tx.w1;
      wt[nw][2] = ty.w1 * (1.f - tx.w1);
      wt[nw][3] = ty.w1 * tx.w1;
      ++nw;
    }
  }
  const int gg = g * g;
  float mx[MAXW], inv_sum[MAXW];
  for (int w = 0; w < nw; ++w) {
    float m = -INFINITY;
    for (int c = 0; c < C; ++c) {
      const float* cm = cosm + c * gg;
      const float v = wt[w][0] * __ldg(cm + off[w][0]) + wt[w][1] * __ldg(cm + off[w][1]) +
                      wt[w][2] * __ldg(cm + off[w][2]) + wt[w][3] * __ldg(cm + off[w][3]);
      m = fmaxf(m, v);
    }
    float s = 0.f;
    for (int c = 0; c < C; ++c) {
      const float* cm = cosm + c * gg;
      const float v = wt[w][0] * __ldg(cm + off[w][0]) + wt[w][1] * __ldg(cm + off[w][1]) +
                      wt[w][2] * __ldg(cm + off[w][2]) + wt[w][3] * __ldg(cm + off[w][3]);
      s += expf(v - m);
    }
    mx[w] = m;
    inv_sum[w] = 1.0f / s;
  }
  const float inv_count = 1.0f / static_cast<float>(nw);
  float best = -INFINITY;
  int best_c = 0;
  for (int c = 0; c < C; ++c) {
    const float* cm = cosm + c * gg;
    float p = 0.f;
    for (int w = 0; w < nw; ++w) {
      const float v = wt[w][0] * __ldg(cm + off[w][0]) + wt[w][1] * __ldg(cm + off[w][1]) +
                      wt[w][2] * __ldg(cm + off[w][2]) + wt[w][3] * __ldg(cm + off[w][3]);
      p += expf(v - mx[w]) * inv_sum[w];
    }
    p *= inv_count;
    if (probs) probs[static_cast<size_t>(c) * H * W + pix] = p;
    if (p > best) {
      best = p;
      best_c = c;
    }
  }
  if (labels) labels[pix] = best_c;
}

// Slide mode on 16 x 16 pixel tiles: the cosine values of every window covering the tile are
// first staged in shared memory (for each window the <= 4 x 4 grid cells the tile's pixels
// interpolate from, all classes), then each thread (pixel) runs the same three passes as
// seg_slide_kernel -- row maximum, exponential sum, then per class the average over windows of
// softmax(bilinear(cos)) with the argmax -- reading shared instead of global memory, with the
// exponential from the special-function unit (__expf: the arguments lie in [-2 max|cos|, 0]).
// Per-window statistics of each pixel also stay in shared memory.  Limits (the host falls back to
// seg_slide_kernel beyond them): at most SLIDE_TILE_WIN windows per tile, C <= SLIDE_TILE_C.
constexpr int SLIDE_TILE = 16;
constexpr int SLIDE_TILE_WIN = 6;
constexpr int SLIDE_TILE_C = 160;
constexpr int SLIDE_TILE_CELLS = 16;  // 4 x 4 grid cells per window
constexpr int SLIDE_TILE_SMEM =
    SLIDE_TILE_WIN * SLIDE_TILE_C * SLIDE_TILE_CELLS * 4 + SLIDE_TILE_WIN * SLIDE_TILE * SLIDE_TILE * 8;

__device__ __forceinline__ int slide_first(int lo, int side, int stride, int n) {
  // first window index whose [origin, origin + side) reaches pixel lo (origins clamped at size - side)
  return min(n - 1, (lo >= side) ? (lo - side) / stride + 1 : 0);
}

__global__ void seg_slide_tile_kernel(const float* __restrict__ cosm, int C, int g, int H, int W, int side, int stride,
                                      int ny, int nx, float* __restrict__ probs, int* __restrict__ labels) {
  extern __shared__ __align__(16) float sm[];
  float* scos = sm;                                                     // [win][C][16]
  float* sstat = sm + SLIDE_TILE_WIN * SLIDE_TILE_C * SLIDE_TILE_CELLS;  // [win][256][2]
  __shared__ int w_iy[SLIDE_TILE_WIN], w_ix[SLIDE_TILE_WIN], w_r0[SLIDE_TILE_WIN], w_c0[SLIDE_TILE_WIN];
  __shared__ int n_win;
  const int ty0 = blockIdx.y * SLIDE_TILE, tx0 = blockIdx.x * SLIDE_TILE;
  const int ty1 = min(H, ty0 + SLIDE_TILE) - 1, tx1 = min(W, tx0 + SLIDE_TILE) - 1;
  const int gg = g * g;
  if (threadIdx.x == 0) {
    // windows overlapping the tile, and for each the first grid row / column its pixels use
    int n = 0;
    const int iy_lo = slide_first(ty0, side, stride, ny), ix_lo = slide_first(tx0, side, stride, nx);
    for (int iy = iy_lo; iy < ny; ++iy) {
      const int oy = min(iy * stride, H - side);
      if (oy > ty1) break;
      if (oy + side <= ty0) continue;
      for (int ix = ix_lo; ix < nx; ++ix) {
        const int ox = min(ix * stride, W - side);
        if (ox > tx1) break;
        if (ox + side <= tx0) continue;
        if (n < SLIDE_TILE_WIN) {
          w_iy[n] = iy;
          w_ix[n] = ix;
          w_r0[n] = bilinear_taps(max(ty0, oy) - oy, g, side).i0;
          w_c0[n] = bilinear_taps(max(tx0, ox) - ox, g, side).i0;
        }
        ++n;
      }
    }
    n_win = n;
  }
  __syncthreads();
  const int nw = min(n_win, SLIDE_TILE_WIN);  // the host only launches tiles with <= SLIDE_TILE_WIN windows
  // stage the 4 x 4 cells of every window, all classes
  for (int i = threadIdx.x; i < nw * C * SLIDE_TILE_CELLS; i += blockDim.x) {
    const int w = i / (C * SLIDE_TILE_CELLS);
    const int rem = i - w * C * SLIDE_TILE_CELLS;
    const int c = rem / SLIDE_TILE_CELLS, cell = rem % SLIDE_TILE_CELLS;
    const int r = min(w_r0[w] + (cell >> 2), g - 1), q = min(w_c0[w] + (cell & 3), g - 1);
    scos[(w * SLIDE_TILE_C + c) * SLIDE_TILE_CELLS + cell] =
        __ldg(cosm + static_cast<size_t>(w_iy[w] * nx + w_ix[w]) * C * gg + static_cast<size_t>(c) * gg + r * g + q);
  }
  __syncthreads();
  const int y = ty0 + (threadIdx.x >> 4), x = tx0 + (threadIdx.x & 15);
  if (y >= H || x >= W) return;
  // per window: covered?, local tap offsets within the staged 4 x 4 cells, weights
  auto taps = [&](int w, int& o00, int& d01, int& d10, float& a00, float& a01, float& a10, float& a11) -> bool {
    const int oy = min(w_iy[w] * stride, H - side), ox = min(w_ix[w] * stride, W - side);
    if (y < oy || y >= oy + side || x < ox || x >= ox + side) return false;
    const Taps1D tyy = bilinear_taps(y - oy, g, side);
    const Taps1D txx = bilinear_taps(x - ox, g, side);
    o00 = (tyy.i0 - w_r0[w]) * 4 + (txx.i0 - w_c0[w]);
    d01 = txx.i1 - txx.i0;
    d10 = (tyy.i1 - tyy.i0) * 4;
    a00 = (1.f - tyy.w1) * (1.f - txx.w1);
    a01 = (1.f - tyy.w1) * txx.w1;
    a10 = tyy.w1 * (1.f - txx.w1);
    a11 = tyy.w1 * txx.w1;
    return true;
  };
  int covered = 0;
  for (int w = 0; w < nw; ++w) {
    int o00, d01, d10;
    float a00, a01, a10, a11;
    float m = -INFINITY, inv = 0.f;
    if (taps(w, o00, d01, d10, a00, a01, a10, a11)) {
      ++covered;
      const float* base = scos + w * SLIDE_TILE_C * SLIDE_TILE_CELLS + o00;
      for (int c = 0; c < C; ++c) {
        const float* q = base + c * SLIDE_TILE_CELLS;
        m = fmaxf(m, a00 * q[0] + a01 * q[d01] + a10 * q[d10] + a11 * q[d10 + d01]);
      }
      float sum = 0.f;
      for (int c = 0; c < C; ++c) {
        const float* q = base + c * SLIDE_TILE_CELLS;
        sum += __expf(a00 * q[0] + a01 * q[d01] + a10 * q[d10] + a11 * q[d10 + d01] - m);
      }
      inv = 1.0f / sum;
    }
    sstat[(w * 256 + threadIdx.x) * 2] = m;
    sstat[(w * 256 + threadIdx.x) * 2 + 1] = inv;
  }
  const float inv_count = 1.0f / static_cast<float>(covered);
  const long long pix = static_cast<long long>(y) * W + x;
  float best = -INFINITY;
  int best_c = 0;
  // classes in groups of 16: the window's taps are computed once per group, the group's partial
  // averages stay in registers
  constexpr int CG = 16;
  for (int c0 = 0; c0 < C; c0 += CG) {
    float acc[CG];
#pragma unroll
    for (int k = 0; k < CG; ++k) acc[k] = 0.f;
    for (int w = 0; w < nw; ++w) {
      int o00, d01, d10;
      float a00, a01, a10, a11;
      if (!taps(w, o00, d01, d10, a00, a01, a10, a11)) continue;
      const float m = sstat[(w * 256 + threadIdx.x) * 2], inv = sstat[(w * 256 + threadIdx.x) * 2 + 1];
      const float* base = scos + (w * SLIDE_TILE_C + c0) * SLIDE_TILE_CELLS + o00;
#pragma unroll
      for (int k = 0; k < CG; ++k) {
        if (c0 + k < C) {
          const float* q = base + k * SLIDE_TILE_CELLS;
          const float v = a00 * q[0] + a01 * q[d01] + a10 * q[d10] + a11 * q[d10 + d01];
          acc[k] += __expf(v - m) * inv;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < CG; ++k) {
      if (c0 + k < C) {
        const float p = acc[k] * inv_count;
        if (probs) probs[static_cast<size_t>(c0 + k) * H * W + pix] = p;
        if (p > best) {
          best = p;
          best_c = c0 + k;
        }
      }
    }
  }
  if (labels) labels[pix] = best_c;
}

__global__ void seg_whole_kernel(const float* __restrict__ cosm, int C, int gh, int gw, int H, int W,
                                 float* __restrict__ scores, int* __restrict__ labels) {
  const long long pix = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (pix >= static_cast<long long>(H) * W) return;
  const int y = static_cast<int>(pix / W), x = static_cast<int>(pix - static_cast<long long>(y) * W);
  const Taps1D ty = bilinear_taps(y, gh, H);
  const Taps1D tx = bilinear_taps(x, gw, W);
  const float w00 = (1.f - ty.w1) * (1.f - tx.w1), w01 = (1.f - ty.w1) * tx.w1;
  const float w10 = ty.w1 * (1.f - tx.w1), w11 = ty.w1 * tx.w1;
  float best = -INFINITY;
  int best_c = 0;
  for (int c = 0; c < C; ++c) {
    const float* cm = cosm + static_cast<size_t>(c) * gh * gw;
    const float v = w00 * __ldg(cm + ty.i0 * gw + tx.i0) + w01 * __ldg(cm + ty.i0 * gw + tx.i1) +
                    w10 * __ldg(cm + ty.i1 * gw + tx.i0) + w11 * __ldg(cm + ty.i1 * gw + tx.i1);
    if (scores) scores[static_cast<size_t>(c) * H * W + pix] = v;
    if (v > best) {
      best = v;
      best_c = c;
    }
  }
  if (labels) labels[pix] = best_c;
}

// y = GELU(x) elementwise with the epilogues' formula (gelu2), for checking it on its own.
__global__ void gelu_stage_kernel(const float* __restrict__ x, long long n, float* __restrict__ y) {
  for (long long i = 2 * (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x); i < n;
       i += 2LL * gridDim.x * blockDim.x) {
    const float2 g = gelu2(make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f));
    y[i] = g.x;
    if (i + 1 < n) y[i + 1] = g.y;
  }
}

}  // namespace vit

