// Persistent tcgen05 GEMM for sm_100a: C[M, N] = A[M, K] . B[N, K]^T with bf16 operands
// (both K-contiguous, nn.Linear layout for B) and an fp32 accumulator in tensor memory,
// followed by one of the encoder's fused epilogues.
//
// CTA = 10 warps, one CTA per SM, grid = min(#tiles, #SMs), tiles visited with stride gridDim:
//   warp 0 (one lane)  TMA producer: A tile 128 x 64 and B tile BN x 64 per stage, 128-byte
//                      swizzle, STAGES-deep ring guarded by full/empty mbarriers.
//   warp 1             allocates 512 TMEM columns (two BN-wide fp32 accumulators); one lane
//                      issues tcgen05.mma (M = 128, N = BN, K = 16) four times per stage and
//                      commits each stage back to the producer and each finished tile to
//                      the epilogue.
//   warps 2..9         epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31, i.e. one output
//                      row per thread, and half of the tile's columns (warps 2..5 the first
//                      half, 6..9 the second), 32 columns per tcgen05.ld.  Results are packed
//                      into a swizzled per-warp staging buffer in shared memory and written by
//                      TMA stores (the residual stream x is also read by TMA, one chunk ahead),
//                      so global memory only sees whole 128-byte lines.
// The double-buffered accumulator lets the epilogue of tile i overlap the MMAs of tile i+1.
#pragma once

#include "cluster.cuh"
#include "common.cuh"
#include "gelu.cuh"

namespace vit {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;
constexpr int GEMM_THREADS = 320;
constexpr int GEMM_EPI_WARPS = 8;
constexpr int GEMM_EPI_THREADS = 32 * GEMM_EPI_WARPS;
// Pipeline waits of the GEMMs poll with a 32 ns suspend-time hint: the threads react to a
// completed stage or accumulator sooner than with the default suspension (measured 2.5-5.5 %
// faster across the encoder's GEMM shapes, identical results).
constexpr int kGemmPoll = 32;

enum EpiMode : int {
  EPI_BIAS = 0,    // out_bf16 = act(acc + bias)
  EPI_LNFOLD = 1,  // out_bf16 = act(rstd * (acc + (ctr - mean) * colsum) + bias)  (LayerNorm folded)
  EPI_RESID = 2,   // x += ls * (acc + bias); xb = bf16(x - ctr); ctr; row partial stats of x
  EPI_PATCH = 3,   // x[token row] = acc + bias + pos (xb, ctr and stats: token_prep_kernel)
  EPI_COS = 4,     // cos[w, c, p] = acc (fp32, class-major per window; row m = w * P + p, column c)
};

struct EpiParams {
  int M, N;
  const float* bias;  // [N]
  int gelu;           // BIAS / LNFOLD: apply exact-erf GELU
  int ldo;
  // LNFOLD: per-row LayerNorm statistics rebuilt from partials written by the producer of x.
  // RESID: stats_in holds the partials of x before the update; their merged mean is the centre
  // of the new bf16 copy.
  const float* colsum;     // [N] column sums of the gamma-folded weight
  const float2* stats_in;  // [M, nt] (mean, M2) of column groups of nt_cols each (nt_cols = BN/2 of the producer)
  int nt, nt_cols, D;
  float eps;
  // The bf16 copy of x is stored re-centred, xb = bf16(x - ctr[row]): LNFOLD reads ctr, RESID
  // writes it (one writer per row: the warps of column group 0).
  float* ctr;              // [M]
  // RESID / PATCH
  float* x;              // [rows, N] fp32 residual stream (PATCH writes it directly)
  __nv_bfloat16* xb;     // [rows, N] bf16 copy of x (A operand of the next folded GEMM)
  const float* ls;       // [N] layer scale (RESID)
  float2* stats_out;     // [rows, N / stats_cols] (mean, M2) over each group of stats_cols columns
  int stats_cols;        // RESID: 32 x a power of two, dividing BN/2 (PATCH: always BN/2)
  // PATCH: GEMM row m = b * P + p goes to token row b * T + 1 + R + p, position row p + pos_off
  const float* pos;
  int P, T, R, pos_off;
  unsigned long long wait_ns;  // pipeline-wait limit (0: the default 2 s)
  // COS: the cosine map [windows, ncls, P] (P from above); columns >= ncls are padding
  float* cos;
  int ncls;
};

template <int BN, int MODE, int XBUF = 2>
struct GemmCfg {
  // 128-wide residual tiles have room for a fourth stage (ViT-S/16@336 b64 FC2 71 -> 64 us), a
  // fifth with one x buffer per warp (XBUF = 1)
  static constexpr int STAGES =
      (MODE == EPI_RESID) ? ((BN == 128) ? (XBUF == 1 ? 5 : 4) : 3) : ((BN == 256) ? 4 : 6);
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK * 2;
  static constexpr int B_BYTES = BN * GEMM_BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // per epilogue warp: RESID two 32 x 32 fp32 x buffers (128-byte rows, 128B swizzle) and one
  // 32 x 32 bf16 buffer (64-byte rows, 64B swizzle); BIAS / LNFOLD one 32 x 64 bf16 buffer
  static constexpr int EPI_WARP_BYTES =
      (MODE == EPI_RESID) ? (XBUF * 4096 + 2048) : ((MODE == EPI_PATCH || MODE == EPI_COS) ? 0 : 4096);
  static constexpr int OFF_EPI = STAGES * STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_EPI + GEMM_EPI_WARPS * EPI_WARP_BYTES;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(8 * (2 * STAGES + 5 + 2 * GEMM_EPI_WARPS) + 8 <= BAR_BYTES, "barrier area");
};

__device__ __forceinline__ void merge_stats(float& n, float& mean, float& m2, float nb, float mb, float m2b) {
  const float tot = n + nb;
  const float d = mb - mean;
  mean += d * (nb / tot);
  m2 += m2b + d * d * (n * nb / tot);
  n = tot;
}

// Mean and sum of squared deviations of 32 values, in four interleaved chains (the sum first,
// then the deviations from the mean): short dependency chains for the residual epilogue.
__device__ __forceinline__ void chunk_mean_m2(const float (&v)[32], float& mean, float& m2) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    s0 += v[j];
    s1 += v[j + 1];
    s2 += v[j + 2];
    s3 += v[j + 3];
  }
  mean = ((s0 + s1) + (s2 + s3)) * (1.0f / 32.0f);
  float q0 = 0.f, q1 = 0.f, q2 = 0.f, q3 = 0.f;
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float d0 = v[j] - mean, d1 = v[j + 1] - mean, d2 = v[j + 2] - mean, d3 = v[j + 3] - mean;
    q0 = fmaf(d0, d0, q0);
    q1 = fmaf(d1, d1, q1);
    q2 = fmaf(d2, d2, q2);
    q3 = fmaf(d3, d3, q3);
  }
  m2 = (q0 + q1) + (q2 + q3);
}

// Affine epilogue of one 32-column chunk for BIAS / LNFOLD: v <- act(rstd * v + shift * c + b)
// with shift = rstd * (ctr - mean) (the accumulator holds bf16(x - ctr) . W_gamma), two columns
// per packed f32x2 instruction.
template <int MODE>
__device__ __forceinline__ void epi_affine(const EpiParams& ep, float (&v)[32], int n, float shift, float rstd) {
  const float4* b4 = reinterpret_cast<const float4*>(ep.bias + n);
  if (MODE == EPI_LNFOLD) {
    const float4* c4 = reinterpret_cast<const float4*>(ep.colsum + n);
    const float2 nrm = make_float2(shift, shift);
    const float2 rs = make_float2(rstd, rstd);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 bb = __ldg(b4 + j);
      const float4 cc = __ldg(c4 + j);
      const float2 t0 = ffma2(nrm, make_float2(cc.x, cc.y), make_float2(bb.x, bb.y));
      const float2 t1 = ffma2(nrm, make_float2(cc.z, cc.w), make_float2(bb.z, bb.w));
      const float2 r0 = ffma2(rs, make_float2(v[4 * j + 0], v[4 * j + 1]), t0);
      const float2 r1 = ffma2(rs, make_float2(v[4 * j + 2], v[4 * j + 3]), t1);
      v[4 * j + 0] = r0.x;
      v[4 * j + 1] = r0.y;
      v[4 * j + 2] = r1.x;
      v[4 * j + 3] = r1.y;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 bb = __ldg(b4 + j);
      const float2 r0 = fadd2(make_float2(v[4 * j + 0], v[4 * j + 1]), make_float2(bb.x, bb.y));
      const float2 r1 = fadd2(make_float2(v[4 * j + 2], v[4 * j + 3]), make_float2(bb.z, bb.w));
      v[4 * j + 0] = r0.x;
      v[4 * j + 1] = r0.y;
      v[4 * j + 2] = r1.x;
      v[4 * j + 3] = r1.y;
    }
  }
  if (ep.gelu) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float2 g = gelu2(make_float2(v[2 * j], v[2 * j + 1]));
      v[2 * j] = g.x;
      v[2 * j + 1] = g.y;
    }
  }
}

// The row's mean and sum of squared deviations from the producer's partial (mean, M2) pairs.
// Every partial covers the same nt_cols columns, so the merged mean is the mean of the partial
// means and M2 = sum_i M2_i + nt_cols * sum_i (mean_i - mean)^2 (the pairwise update of Chan,
// Golub & LeVeque for equal counts, applied to all partials at once).  The deviations are summed
// around the first partial's mean, so no division sits in the chain (one reciprocal of nt); the
// loads go out eight at a time so their latencies overlap.
__device__ __forceinline__ void merge_row_stats(const EpiParams& ep, int row, float& mu, float& m2out) {
  const float2* s = ep.stats_in + static_cast<size_t>(row) * ep.nt;
  float c = 0.f, s1 = 0.f, s2 = 0.f, sm2 = 0.f;
  for (int t0 = 0; t0 < ep.nt; t0 += 8) {
    float2 st[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) st[u] = (t0 + u < ep.nt) ? s[t0 + u] : make_float2(0.f, 0.f);
    if (t0 == 0) c = st[0].x;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (t0 + u < ep.nt) {
        const float d = st[u].x - c;
        s1 += d;
        s2 = fmaf(d, d, s2);
        sm2 += st[u].y;
      }
    }
  }
  const float inv = 1.0f / static_cast<float>(ep.nt);
  mu = c + s1 * inv;
  m2out = sm2 + static_cast<float>(ep.nt_cols) * fmaxf(fmaf(-s1 * inv, s1, s2), 0.f);
}

// LNFOLD: rstd of the row and the shift rstd * (ctr - mean) that turns the accumulator of the
// re-centred operand into the accumulator of x - mean.
__device__ __forceinline__ void lnfold_row_stats(const EpiParams& ep, int row, float& shift, float& rstd) {
  float mu, m2;
  merge_row_stats(ep, row, mu, m2);
  rstd = rsqrtf(m2 / static_cast<float>(ep.D) + ep.eps);
  shift = rstd * (ep.ctr[row] - mu);
}

// Pulls the 128-byte lines of v[n0 .. n0 + cols - 1] (cols a multiple of 32) into L1, so that
// the epilogue's per-column vectors are L1 hits by the time the accumulator is ready.
__device__ __forceinline__ void prefetch_cols_l1(const float* v, int n0, int cols) {
  const int lane = threadIdx.x & 31;
  if (v != nullptr && lane < cols / 32) asm volatile("prefetch.global.L1 [%0];" ::"l"(v + n0 + lane * 32));
}

// Work a BIAS / LNFOLD epilogue warp does before it waits for its accumulator: the rows'
// LayerNorm statistics (LNFOLD) and the columns' bias / colsum lines.  (The same prefetch in the
// residual epilogue, whose x loads already run a chunk ahead, measured 1-2 % slower.)
//
// RESID: the centre of the row's new bf16 copy, the mean of x before this update (merged from
// stats_in), returned in `mu`.  Every CTA that writes a part of the row computes the same value.
template <int BN, int MODE>
__device__ __forceinline__ void epilogue_prologue(const EpiParams& ep, int row, int n0, float& mu, float& rstd) {
  mu = 0.f;
  rstd = 0.f;
  if (MODE == EPI_RESID) {
    float m2;
    if (row < ep.M) merge_row_stats(ep, row, mu, m2);
    return;
  }
  if (MODE != EPI_BIAS && MODE != EPI_LNFOLD) return;
  prefetch_cols_l1(ep.bias, n0, BN / 2);
  if (MODE == EPI_LNFOLD) prefetch_cols_l1(ep.colsum, n0, BN / 2);
  if (MODE == EPI_LNFOLD && row < ep.M) lnfold_row_stats(ep, row, mu, rstd);
}

// BIAS / LNFOLD: one warp's half of a tile (rows row0 .. row0 + 31, columns n0 .. n0 + BN/2 - 1),
// 64 columns per TMA store from the warp's staging buffer `obuf` (32 rows x 128 bytes, 128B
// swizzle: 16-byte chunk k of row r sits at chunk k ^ (r % 8)).  mu / rstd: this thread's row
// statistics (LNFOLD: mu carries the centre shift of lnfold_row_stats).
template <int BN, int MODE>
__device__ __forceinline__ void epilogue_store_bf16(const EpiParams& ep, const CUtensorMap* tmO, uint32_t taddr,
                                                    int row0, int n0, uint8_t* obuf, float mu, float rstd) {
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  for (int g = 0; g < BN / 128; ++g) {
    if (lane == 0) tma_store_wait_read0();  // the previous store has left the staging buffer
    __syncwarp();
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int c = 2 * g + cc;
      float v[32];
      tmem_ld32(taddr + c * 32, v);
      epi_affine<MODE>(ep, v, n0 + c * 32, mu, rstd);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * k + 0], v[8 * k + 1]);
        w.y = pack_bf16x2(v[8 * k + 2], v[8 * k + 3]);
        w.z = pack_bf16x2(v[8 * k + 4], v[8 * k + 5]);
        w.w = pack_bf16x2(v[8 * k + 6], v[8 * k + 7]);
        const int chunk = (cc * 4 + k) ^ (lane & 7);
        *reinterpret_cast<uint4*>(obuf + lane * 128 + chunk * 16) = w;
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmO, obuf, n0 + g * 64, row0);
      tma_store_commit();
    }
  }
}

// RESID: one warp's half of a tile.  x arrives by TMA into xbuf[c & 1] (32 rows x 128 bytes, 128B
// swizzle), chunk c + 1 is requested while chunk c is processed (XBUF = 1: one buffer, chunk c + 1
// requested after chunk c is stored, which frees shared memory for a deeper operand ring); the updated x goes back into the
// same buffer and, with its re-centred bf16 copy bf16(x - centre) (xbbuf: 32 rows x 64 bytes, 64B
// swizzle), out by TMA stores.  `centre` is this thread's row's mean of x before the update (the
// same value in every CTA that writes a part of the row); the warps of column group 0 record it
// in ep.ctr for the folded LayerNorm that reads the copy.  Row statistics (mean, M2) of the new x
// are written per row for each group of ep.stats_cols columns.
template <int BN, int XBUF = 2>
__device__ __forceinline__ void epilogue_resid(const EpiParams& ep, const CUtensorMap* tmX, const CUtensorMap* tmXb,
                                               uint32_t taddr, int row0, int n0, float centre, uint8_t* xbuf0,
                                               uint8_t* xbbuf, uint64_t* xfull, uint32_t (&xph)[2],
                                               bool (&xpending)[2], volatile int* abort_flag, int* gstatus, bool& ok) {
  constexpr int HALF = BN / 2;
  constexpr int CHUNKS = HALF / 32;
  const int lane = threadIdx.x & 31;
  const int row = row0 + lane;
  if (n0 == 0 && row < ep.M) ep.ctr[row] = centre;
  const float2 nc = make_float2(-centre, -centre);
  float run_n = 0.f, run_mean = 0.f, run_m2 = 0.f;
#pragma unroll 1
  for (int c = 0; c < CHUNKS; ++c) {
    const int buf = (XBUF == 2) ? (c & 1) : 0;
    const int n = n0 + c * 32;
    if (lane == 0) {
      tma_store_wait_read0();  // earlier stores have left the x buffer about to be filled and xbbuf
      if (XBUF == 2) {
        if (c + 1 < CHUNKS) {
          mbar_arrive_expect_tx(&xfull[buf ^ 1], 4096);
          tma_load_2d(xbuf0 + (buf ^ 1) * 4096, tmX, n + 32, row0, &xfull[buf ^ 1]);
          xpending[buf ^ 1] = true;
        }
      } else if (c > 0) {
        // one buffer: chunk c is requested once chunk c - 1 has been stored (chunk 0 was
        // requested before the accumulator wait)
        mbar_arrive_expect_tx(&xfull[0], 4096);
        tma_load_2d(xbuf0, tmX, n, row0, &xfull[0]);
        xpending[0] = true;
      }
    }
    __syncwarp();
    if (!mbar_wait<kGemmPoll>(&xfull[buf], xph[buf], abort_flag, gstatus, DEV_TIMEOUT_GEMM + 6, ep.wait_ns)) {
      ok = false;
      return;
    }
    xph[buf] ^= 1u;
    if (lane == 0) xpending[buf] = false;
    float v[32];
    __syncwarp();
    tmem_ld32(taddr + c * 32, v);
    uint8_t* xr = xbuf0 + buf * 4096 + lane * 128;
    const float4* b4 = reinterpret_cast<const float4*>(ep.bias + n);
    const float4* l4 = reinterpret_cast<const float4*>(ep.ls + n);
    // every load of the chunk is issued before the first use, so their latencies overlap
    float4 xo[8], bb[8], ll[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      xo[k] = *reinterpret_cast<const float4*>(xr + ((k ^ (lane & 7)) << 4));
      bb[k] = __ldg(b4 + k);
      ll[k] = __ldg(l4 + k);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 a0 = fadd2(make_float2(v[4 * k + 0], v[4 * k + 1]), make_float2(bb[k].x, bb[k].y));
      const float2 a1 = fadd2(make_float2(v[4 * k + 2], v[4 * k + 3]), make_float2(bb[k].z, bb[k].w));
      const float2 r0 = ffma2(make_float2(ll[k].x, ll[k].y), a0, make_float2(xo[k].x, xo[k].y));
      const float2 r1 = ffma2(make_float2(ll[k].z, ll[k].w), a1, make_float2(xo[k].z, xo[k].w));
      v[4 * k + 0] = r0.x;
      v[4 * k + 1] = r0.y;
      v[4 * k + 2] = r1.x;
      v[4 * k + 3] = r1.y;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k)
      *reinterpret_cast<float4*>(xr + ((k ^ (lane & 7)) << 4)) =
          make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 c0 = fadd2(make_float2(v[8 * k + 0], v[8 * k + 1]), nc);
      const float2 c1 = fadd2(make_float2(v[8 * k + 2], v[8 * k + 3]), nc);
      const float2 c2 = fadd2(make_float2(v[8 * k + 4], v[8 * k + 5]), nc);
      const float2 c3 = fadd2(make_float2(v[8 * k + 6], v[8 * k + 7]), nc);
      uint4 w;
      w.x = pack_bf16x2(c0.x, c0.y);
      w.y = pack_bf16x2(c1.x, c1.y);
      w.z = pack_bf16x2(c2.x, c2.y);
      w.w = pack_bf16x2(c3.x, c3.y);
      *reinterpret_cast<uint4*>(xbbuf + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4)) = w;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmX, xbuf0 + buf * 4096, n, row0);
      tma_store_2d(tmXb, xbbuf, n, row0);
      tma_store_commit();
    }
    float cm, q;
    chunk_mean_m2(v, cm, q);
    merge_stats(run_n, run_mean, run_m2, 32.f, cm, q);
    if ((n + 32) % ep.stats_cols == 0) {
      if (row < ep.M)
        ep.stats_out[static_cast<size_t>(row) * (ep.N / ep.stats_cols) + (n + 32) / ep.stats_cols - 1] =
            make_float2(run_mean, run_m2);
      run_n = 0.f;
      run_mean = 0.f;
      run_m2 = 0.f;
    }
  }
}

// PATCH: rows of the GEMM are scattered to token rows, so this epilogue writes x directly
// (x[b * T + 1 + R + p] = acc + bias + pos[p]); the bf16 copy, its centre and the row statistics
// follow in token_prep_kernel, which sees whole rows.
template <int BN>
__device__ __forceinline__ void epilogue_patch(const EpiParams& ep, uint32_t taddr, int row, int n0) {
  constexpr int HALF = BN / 2;
  const bool valid = row < ep.M;
  int xrow = row;
  const float* posrow = nullptr;
  if (valid) {
    const int b = row / ep.P;
    const int p = row - b * ep.P;
    xrow = b * ep.T + 1 + ep.R + p;
    posrow = ep.pos + static_cast<size_t>(p + ep.pos_off) * ep.N;
  }
#pragma unroll 1
  for (int c = 0; c < HALF / 32; ++c) {
    float v[32];
    const int n = n0 + c * 32;
    __syncwarp();
    tmem_ld32(taddr + c * 32, v);
    if (valid) {
      const float4* b4 = reinterpret_cast<const float4*>(ep.bias + n);
      const float4* p4 = reinterpret_cast<const float4*>(posrow + n);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 bb = __ldg(b4 + j);
        const float4 pp = __ldg(p4 + j);
        v[4 * j + 0] += bb.x + pp.x;
        v[4 * j + 1] += bb.y + pp.y;
        v[4 * j + 2] += bb.z + pp.z;
        v[4 * j + 3] += bb.w + pp.w;
      }
      float4* xp = reinterpret_cast<float4*>(ep.x + static_cast<size_t>(xrow) * ep.N + n);
#pragma unroll
      for (int j = 0; j < 8; ++j) xp[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
  }
}

// COS: the patch-text cosine map.  Row m = w * P + p of the GEMM (window w, patch p), column c
// (class) goes to cos[(w * ncls + c) * P + p]: for each column the 32 lanes of a warp write 32
// consecutive patches of one class row (128-byte segments).  Padding columns are skipped.
template <int BN>
__device__ __forceinline__ void epilogue_cos(const EpiParams& ep, uint32_t taddr, int row, int n0) {
  constexpr int HALF = BN / 2;
  float* base = nullptr;
  if (row < ep.M) {
    const int w = row / ep.P;
    const int p = row - w * ep.P;
    base = ep.cos + static_cast<size_t>(w) * ep.ncls * ep.P + p;
  }
#pragma unroll 1
  for (int c = 0; c < HALF / 32; ++c) {
    const int n = n0 + c * 32;
    if (n >= ep.ncls) break;  // warp-uniform: the rest of this half is padding
    float v[32];
    __syncwarp();
    tmem_ld32(taddr + c * 32, v);
    if (base != nullptr) {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (n + j < ep.ncls) base[static_cast<size_t>(n + j) * ep.P] = v[j];
    }
  }
}

// tmO1 / tmO2: BIAS / LNFOLD -> tmO1 = output [M, ldo] bf16 (box 64 x 32, 128B swizzle);
//              RESID -> tmO1 = x [M, N] fp32 (box 32 x 32, 128B swizzle), tmO2 = xb [M, N] bf16
//              (box 32 x 32, 64B swizzle); PATCH -> unused.
template <int BN, int MODE, int XBUF = 2>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmO1, const __grid_constant__ CUtensorMap tmO2, int M,
                        int N, int K, EpiParams ep, int* gstatus) {
  using Cfg = GemmCfg<BN, MODE, XBUF>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* sEpi = smem + Cfg::OFF_EPI;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* xfull = mma_done + 1;  // [GEMM_EPI_WARPS][2] (RESID)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(xfull + 2 * GEMM_EPI_WARPS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], GEMM_EPI_THREADS);
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < 2 * GEMM_EPI_WARPS; ++i) mbar_init(&xfull[i], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (MODE != EPI_PATCH && MODE != EPI_COS) tma_prefetch_desc(&tmO1);
    if (MODE == EPI_RESID) tma_prefetch_desc(&tmO2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  // everything above touches only this CTA's shared and tensor memory; global memory from here on
  pdl_wait();
  if (threadIdx.x == 0) *abort_flag = (*reinterpret_cast<volatile int*>(gstatus) != 0) ? 1 : 0;
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const bool skip = *abort_flag != 0;

  const int num_m = (M + GEMM_BM - 1) / GEMM_BM;
  const int num_n = N / BN;
  const int num_tiles = num_m * num_n;
  const int KB = K / GEMM_BK;

  if (!skip && warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int stage = 0;
    uint32_t phase = 0;
    int issued_parity[STAGES];
#pragma unroll
    for (int s = 0; s < STAGES; ++s) issued_parity[s] = -1;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mb = tile / num_n;
      const int nb = tile - mb * num_n;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait<kGemmPoll>(&empty[stage], phase ^ 1u, abort_flag, gstatus, DEV_TIMEOUT_GEMM + 1, ep.wait_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
        tma_load_2d(sA + stage * Cfg::A_BYTES, &tmA, kb * GEMM_BK, mb * GEMM_BM, &full[stage]);
        tma_load_2d(sB + stage * Cfg::B_BYTES, &tmB, kb * GEMM_BK, nb * BN, &full[stage]);
        issued_parity[stage] = static_cast<int>(phase);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
    if (*abort_flag) {
      // let every issued tile land before the CTA can exit and release its shared memory
      for (int s = 0; s < STAGES; ++s)
        if (issued_parity[s] >= 0) mbar_wait_drain(&full[s], static_cast<uint32_t>(issued_parity[s]));
    }
  } else if (!skip && warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(GEMM_BM, BN, false);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait<kGemmPoll>(&tempty[acc], acc_phase ^ 1u, abort_flag, gstatus, DEV_TIMEOUT_GEMM + 2, ep.wait_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait<kGemmPoll>(&full[stage], phase, abort_flag, gstatus, DEV_TIMEOUT_GEMM + 3, ep.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * Cfg::B_BYTES);
#pragma unroll
          for (int k = 0; k < GEMM_BK / 16; ++k) {
            tc_mma_ss(d_tmem, sdesc_sw128(a0 + k * 32, 16, 1024), sdesc_sw128(b0 + k * 32, 16, 1024), idesc,
                      (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      tc_commit(mma_done);
    }
    __syncwarp();
  } else if (!skip && warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int e = warp - 2;
    const int q = warp & 3;
    const int half = e >> 2;
    uint8_t* wbuf = sEpi + e * Cfg::EPI_WARP_BYTES;
    uint64_t* wxfull = xfull + 2 * e;
    uint32_t xph[2] = {0u, 0u};
    bool xpending[2] = {false, false};
    bool ok = true;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int mb = tile / num_n;
      const int nb = tile - mb * num_n;
      const int row0 = mb * GEMM_BM + q * 32;
      const int n0 = nb * BN + half * (BN / 2);
      if (MODE == EPI_RESID && lane == 0) {
        // the tile's first chunk of x, requested before the accumulator is ready
        tma_store_wait_read0();
        mbar_arrive_expect_tx(&wxfull[0], 4096);
        tma_load_2d(wbuf, &tmO1, n0, row0, &wxfull[0]);
        xpending[0] = true;
      }
      float mu, rstd;
      epilogue_prologue<BN, MODE>(ep, row0 + lane, n0, mu, rstd);
      if (!mbar_wait<kGemmPoll>(&tfull[acc], acc_phase, abort_flag, gstatus, DEV_TIMEOUT_GEMM + 4, ep.wait_ns)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + half * (BN / 2));
      __syncwarp();
      if (MODE == EPI_RESID) {
        epilogue_resid<BN, XBUF>(ep, &tmO1, &tmO2, taddr, row0, n0, mu, wbuf, wbuf + XBUF * 4096, wxfull, xph, xpending, abort_flag,
                           gstatus, ok);
        if (!ok) break;
      } else if (MODE == EPI_PATCH) {
        epilogue_patch<BN>(ep, taddr, row0 + lane, n0);
      } else if (MODE == EPI_COS) {
        epilogue_cos<BN>(ep, taddr, row0 + lane, n0);
      } else {
        epilogue_store_bf16<BN, MODE>(ep, &tmO1, taddr, row0, n0, wbuf, mu, rstd);
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) {
      if (MODE == EPI_RESID) {
        // x loads requested but not consumed (only after an abort) must land before exit
        for (int bb = 0; bb < 2; ++bb)
          if (xpending[bb]) mbar_wait_drain(&wxfull[bb], xph[bb]);
      }
      tma_store_wait0();  // every TMA store of this warp has completed
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 1) {
    if (!skip && lane == 0) {
      // all MMAs issued by this CTA have completed before TMEM is released
      mbar_wait_drain(mma_done, 0);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------------------
// Paired variant: a 2-CTA cluster computes one 256 x 256 tile with M = 256 tcgen05.mma
// (cta_group::2).  Each CTA loads its 128 rows of A and its 128 of the 256 B rows (16 KB + 16 KB
// per 64-deep stage instead of 16 KB + 32 KB), so per SM the tensor core consumes 131 instead of
// 87 FLOP per byte brought into shared memory.  Roles as in gemm_bf16_tc_kernel, with:
//   * both CTAs' producers fill their own stages and count the bytes on the leader's (rank 0)
//     full barrier; only the leader arms it (with both CTAs' bytes);
//   * the leader's lane issues the MMAs and commits stage / accumulator / final completion to
//     the barriers at the same offsets in both CTAs (multicast commit);
//   * each CTA's epilogue reads its own 128 accumulator rows from its own TMEM and releases the
//     accumulator by arriving (one arrive per warp) on the leader's tempty barrier.
// No TMA load uses cluster multicast.
template <int MODE, int XBUF = 2>
struct PairCfg {
  static constexpr int BN = 256;
  static constexpr int STAGES = (MODE == EPI_RESID) ? (XBUF == 1 ? 5 : 4) : 6;
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK * 2;
  static constexpr int B_BYTES = (BN / 2) * GEMM_BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_WARP_BYTES = (MODE == EPI_RESID) ? (XBUF * 4096 + 2048) : GemmCfg<256, MODE>::EPI_WARP_BYTES;
  static constexpr int OFF_EPI = STAGES * STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_EPI + GEMM_EPI_WARPS * EPI_WARP_BYTES;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(MODE != EPI_PATCH && MODE != EPI_COS, "the patch and cosine GEMMs run unpaired");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(8 * (2 * STAGES + 5 + 2 * GEMM_EPI_WARPS) + 8 <= BAR_BYTES, "barrier area");
};

__device__ __forceinline__ int ld_shared_cluster_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// Bounded pause (nanoseconds on the global timer) for copies whose completion this CTA cannot
// observe itself (its loads are counted on the peer's barrier); used only after an abort.
__device__ __forceinline__ void grace_wait_ns(unsigned long long ns) {
  const unsigned long long t0 = global_ns();
  while (global_ns() - t0 < ns) {
  }
}

template <int MODE, int XBUF = 2>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmO1, const __grid_constant__ CUtensorMap tmO2, int M, int N,
                     int K, EpiParams ep, int* gstatus) {
  using Cfg = PairCfg<MODE, XBUF>;
  constexpr int BN = Cfg::BN;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* sEpi = smem + Cfg::OFF_EPI;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* xfull = mma_done + 1;  // [GEMM_EPI_WARPS][2] (RESID)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(xfull + 2 * GEMM_EPI_WARPS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * GEMM_EPI_WARPS);  // one arrive per epilogue warp of each CTA
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < 2 * GEMM_EPI_WARPS; ++i) mbar_init(&xfull[i], 1);
    fence_mbar_init_cluster();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmO1);
    if (MODE == EPI_RESID) tma_prefetch_desc(&tmO2);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  // everything above touches only this cluster's shared and tensor memory; global memory from here on
  pdl_wait();
  if (threadIdx.x == 0) *abort_flag = (*reinterpret_cast<volatile int*>(gstatus) != 0) ? 1 : 0;
  pdl_launch_dependents();
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // the leader's view decides for both CTAs
  const bool skip = ld_shared_cluster_s32(mapa_shared(smem_u32(const_cast<int*>(abort_flag)), 0)) != 0;

  const int num_m = (M + 2 * GEMM_BM - 1) / (2 * GEMM_BM);
  // N a multiple of 128: when N = 256 k + 128 the last column tile is padded, its second half of
  // B rows is zero-filled by the loads and its second column half is neither computed into an
  // output nor stored
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int KB = K / GEMM_BK;
  const int cid = static_cast<int>(blockIdx.x >> 1);
  const int ncl = static_cast<int>(gridDim.x >> 1);

  if (!skip && warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    int issued_parity[STAGES];
#pragma unroll
    for (int s = 0; s < STAGES; ++s) issued_parity[s] = -1;
    bool issued_any = false;
    for (int tile = cid; tile < num_tiles; tile += ncl) {
      const int mb = tile / num_n;
      const int nb = tile - mb * num_n;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait<kGemmPoll>(&empty[stage], phase ^ 1u, abort_flag, gstatus, DEV_TIMEOUT_GEMM + 5, ep.wait_ns)) {
          ok = false;
          break;
        }
        if (leader) mbar_arrive_expect_tx(&full[stage], 2 * Cfg::STAGE_BYTES);
        const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
        tma_load_2d_pair(sA + stage * Cfg::A_BYTES, &tmA, kb * GEMM_BK, mb * 2 * GEMM_BM + static_cast<int>(rank) * GEMM_BM,
                         bar);
        tma_load_2d_pair(sB + stage * Cfg::B_BYTES, &tmB, kb * GEMM_BK, nb * BN + static_cast<int>(rank) * (BN / 2), bar);
        issued_parity[stage] = static_cast<int>(phase);
        issued_any = true;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
    if (*abort_flag) {
      // let every issued copy land before the CTA can exit: the leader sees both CTAs' bytes on
      // its full barriers; the peer cannot observe its own completions and pauses instead
      if (leader) {
        for (int s = 0; s < STAGES; ++s)
          if (issued_parity[s] >= 0) mbar_wait_drain(&full[s], static_cast<uint32_t>(issued_parity[s]));
      } else if (issued_any) {
        grace_wait_ns(200000ull);
      }
    }
  } else if (!skip && warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(2 * GEMM_BM, BN, false);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl) {
        if (!mbar_wait<kGemmPoll>(&tempty[acc], acc_phase ^ 1u, abort_flag, gstatus, DEV_TIMEOUT_GEMM + 6, ep.wait_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait<kGemmPoll>(&full[stage], phase, abort_flag, gstatus, DEV_TIMEOUT_GEMM + 7, ep.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * Cfg::B_BYTES);
#pragma unroll
          for (int k = 0; k < GEMM_BK / 16; ++k) {
            tc_mma_ss_pair(d_tmem, sdesc_sw128(a0 + k * 32, 16, 1024), sdesc_sw128(b0 + k * 32, 16, 1024), idesc,
                           (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(&tfull[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      tc_commit_pair_mc(mma_done, 0x3);
    }
    __syncwarp();
  } else if (!skip && warp >= 2) {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int e = warp - 2;
    const int q = warp & 3;
    const int half = e >> 2;
    uint8_t* wbuf = sEpi + e * Cfg::EPI_WARP_BYTES;
    uint64_t* wxfull = xfull + 2 * e;
    uint32_t xph[2] = {0u, 0u};
    bool xpending[2] = {false, false};
    bool ok = true;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cid; tile < num_tiles && ok; tile += ncl) {
      const int mb = tile / num_n;
      const int nb = tile - mb * num_n;
      const int row0 = mb * 2 * GEMM_BM + static_cast<int>(rank) * GEMM_BM + q * 32;
      const int n0 = nb * BN + half * (BN / 2);
      const bool active = n0 < N;  // false for the padding half of a last column tile
      if (MODE == EPI_RESID && active && lane == 0) {
        tma_store_wait_read0();
        mbar_arrive_expect_tx(&wxfull[0], 4096);
        tma_load_2d(wbuf, &tmO1, n0, row0, &wxfull[0]);
        xpending[0] = true;
      }
      float mu = 0.f, rstd = 0.f;
      if (active) epilogue_prologue<BN, MODE>(ep, row0 + lane, n0, mu, rstd);
      if (!mbar_wait<kGemmPoll>(&tfull[acc], acc_phase, abort_flag, gstatus, DEV_TIMEOUT_GEMM + 8, ep.wait_ns)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + half * (BN / 2));
      __syncwarp();
      if (MODE == EPI_RESID && active) {
        epilogue_resid<BN, XBUF>(ep, &tmO1, &tmO2, taddr, row0, n0, mu, wbuf, wbuf + XBUF * 4096, wxfull, xph,
                                 xpending, abort_flag, gstatus, ok);
        if (!ok) break;
      } else if (MODE != EPI_RESID && active) {
        epilogue_store_bf16<BN, MODE>(ep, &tmO1, taddr, row0, n0, wbuf, mu, rstd);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) {
      if (MODE == EPI_RESID) {
        for (int bb = 0; bb < 2; ++bb)
          if (xpending[bb]) mbar_wait_drain(&wxfull[bb], xph[bb]);
      }
      tma_store_wait0();
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 1 && !skip && lane == 0) {
    // every MMA of the pair (which reads this CTA's shared memory and writes its TMEM) is done
    mbar_wait_drain(mma_done, 0);
  }
  __syncwarp();
  tc_fence_before();
  // no CTA leaves while the other may still signal its barriers or use its TMEM
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace vit
