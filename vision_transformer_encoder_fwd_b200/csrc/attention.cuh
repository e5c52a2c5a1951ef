// Fused multi-head self-attention forward for sm_100a (tcgen05 + TMA), head width 64.
//
// "DINOv2 n semantic" diagram, panel "Encoder self-attention": per head, softmax over keys of
// Q K^T / sqrt(64), times V, heads merged.  kornia/dinov3 card, "Build BF16, not FP16": the
// scaled logits reach ~2.5e6, so Q, K, V and P stay bf16 but the logits, the running maximum
// and the running sum are fp32 (fp32's exponent range).
//
// One CTA per (128-query tile, head, image); 6 warps:
//   warp 0 (one lane)  TMA: the Q tile once, then K_j and V_j (128 keys x 64 dims each) into a
//                      2-deep ring, read straight from the stacked QKV activation [B, T, 3D]
//                      through a 3-D tensor map (rows past T are zero-filled).
//   warp 1             allocates 256 TMEM columns; one lane issues S = Q K_j^T (M=128, N=128)
//                      into TMEM columns 0..127 and O_j = P_j V_j (M=128, N=64, V as an
//                      MN-major operand) into columns 128 + 64 (j % 2).
//   warps 2..5         softmax, one query row per thread (TMEM lane = row): row maximum over
//                      the valid keys, exp2 of (s - max) * log2(e) / 8, P_j written to shared
//                      memory in the 128-byte-swizzled K-major layout the MMA reads, running
//                      sum; the fp32 output row is kept in registers and rescaled as
//                      O <- alpha O + P_j V_j when each P_j V_j lands.
// Two CTAs fit on one SM (112 KB shared memory and 256 TMEM columns each), so one CTA's
// softmax overlaps the other's MMAs.
#pragma once

#include "common.cuh"

namespace vit {

constexpr int ATT_BM = 128;
constexpr int ATT_BN = 128;
constexpr int ATT_THREADS = 192;

struct AttnCfg {
  static constexpr int Q_BYTES = ATT_BM * 64 * 2;  // 16 KB
  static constexpr int K_BYTES = ATT_BN * 64 * 2;  // 16 KB
  static constexpr int V_BYTES = ATT_BN * 64 * 2;  // 16 KB
  static constexpr int P_BYTES = ATT_BM * ATT_BN * 2;  // 32 KB: two 64-key swizzle atoms
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + 2 * K_BYTES;
  static constexpr int OFF_P = OFF_V + 2 * V_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 128;
  static constexpr uint32_t TMEM_COLS = 256;
};

// log2(e) / sqrt(64)
constexpr float kAttnScaleLog2 = 0.18033688011112042f;

__global__ void __launch_bounds__(ATT_THREADS, 2)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQKV, int T, int D, __nv_bfloat16* __restrict__ out,
                       int* gstatus) {
  extern __shared__ __align__(1024) uint8_t smem[];
  // The swizzled layouts assume 1024-byte aligned tiles; report and stop if the shared
  // window is not (uniform across the CTA, before anything is allocated).
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicExch(gstatus, DEV_TIMEOUT_ATTN + 15);
    return;
  }
  uint8_t* sQ = smem + AttnCfg::OFF_Q;
  uint8_t* sK = smem + AttnCfg::OFF_K;
  uint8_t* sV = smem + AttnCfg::OFF_V;
  uint8_t* sP = smem + AttnCfg::OFF_P;
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + AttnCfg::OFF_BAR);
  uint64_t* kv_full = q_full + 1;    // [2]
  uint64_t* kv_empty = q_full + 3;   // [2]
  uint64_t* s_full = q_full + 5;
  uint64_t* p_full = q_full + 6;
  uint64_t* pv_full = q_full + 7;    // [2]
  uint64_t* mma_done = q_full + 9;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(q_full + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qblk = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int nkv = (T + ATT_BN - 1) / ATT_BN;

  if (threadIdx.x == 0) {
    *abort_flag = (*reinterpret_cast<volatile int*>(gstatus) != 0) ? 1 : 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&pv_full[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQKV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, AttnCfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const bool skip = *abort_flag != 0;

  if (!skip && warp == 0 && lane == 0) {
    // ------------------------------------------------------------------ TMA producer
    int issued_parity[3] = {-1, -1, -1};  // q_full, kv_full[0], kv_full[1]
    mbar_arrive_expect_tx(q_full, AttnCfg::Q_BYTES);
    tma_load_3d(sQ, &tmQKV, h * 64, qblk * ATT_BM, b, q_full);
    issued_parity[0] = 0;
    for (int j = 0; j < nkv; ++j) {
      const int s = j & 1;
      const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1u;
      if (!mbar_wait(&kv_empty[s], ph ^ 1u, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 1)) break;
      mbar_arrive_expect_tx(&kv_full[s], AttnCfg::K_BYTES + AttnCfg::V_BYTES);
      tma_load_3d(sK + s * AttnCfg::K_BYTES, &tmQKV, D + h * 64, j * ATT_BN, b, &kv_full[s]);
      tma_load_3d(sV + s * AttnCfg::V_BYTES, &tmQKV, 2 * D + h * 64, j * ATT_BN, b, &kv_full[s]);
      issued_parity[1 + s] = static_cast<int>(ph);
    }
    if (*abort_flag) {
      if (issued_parity[0] >= 0) mbar_wait_drain(q_full, 0);
      for (int s = 0; s < 2; ++s)
        if (issued_parity[1 + s] >= 0) mbar_wait_drain(&kv_full[s], static_cast<uint32_t>(issued_parity[1 + s]));
    }
  } else if (!skip && warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(ATT_BM, ATT_BN, false);
      constexpr uint32_t idesc_o = idesc_bf16(ATT_BM, 64, true);
      const uint32_t q0 = smem_u32(sQ);
      const uint32_t k0 = smem_u32(sK);
      const uint32_t v0 = smem_u32(sV);
      const uint32_t p0 = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 2) &&
                mbar_wait(&kv_full[0], 0, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 3);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_ss(tmem_base, sdesc_sw128(q0 + k * 32, 16, 1024), sdesc_sw128(k0 + k * 32, 16, 1024), idesc_s,
                    k > 0 ? 1u : 0u);
        tc_commit(s_full);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        if (!mbar_wait(p_full, static_cast<uint32_t>(j) & 1u, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 4)) break;
        tc_fence_after();
        if (j + 1 < nkv) {
          const int s1 = (j + 1) & 1;
          if (!mbar_wait(&kv_full[s1], static_cast<uint32_t>((j + 1) >> 1) & 1u, abort_flag, gstatus,
                         DEV_TIMEOUT_ATTN + 5))
            break;
          tc_fence_after();
          const uint32_t kb = k0 + s1 * AttnCfg::K_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_ss(tmem_base, sdesc_sw128(q0 + k * 32, 16, 1024), sdesc_sw128(kb + k * 32, 16, 1024), idesc_s,
                      k > 0 ? 1u : 0u);
          tc_commit(s_full);
        }
        const int s = j & 1;
        const uint32_t vb = v0 + s * AttnCfg::V_BYTES;
        const uint32_t d_o = tmem_base + 128u + static_cast<uint32_t>(s * 64);
#pragma unroll
        for (int kk = 0; kk < ATT_BN / 16; ++kk) {
          const uint32_t pa = p0 + (kk >> 2) * (AttnCfg::P_BYTES / 2) + (kk & 3) * 32;
          tc_mma_ss(d_o, sdesc_sw128(pa, 16, 1024), sdesc_sw128(vb + kk * 2048, AttnCfg::V_BYTES, 1024), idesc_o,
                    kk > 0 ? 1u : 0u);
        }
        tc_commit(&pv_full[s]);
        tc_commit(&kv_empty[s]);
      }
      tc_commit(mma_done);
    }
    __syncwarp();
  } else if (!skip && warp >= 2) {
    // ------------------------------------------------------------------ softmax
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    float o[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f, alpha_prev = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait(s_full, static_cast<uint32_t>(j) & 1u, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 6)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int valid = min(ATT_BN, T - j * ATT_BN);
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < ATT_BN / 32; ++c) {
        float v[32];
        __syncwarp();
        tmem_ld32(lane_base + c * 32, v);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float sv = (c * 32 + t < valid) ? v[t] : -INFINITY;
          mx = fmaxf(mx, sv);
        }
      }
      const float m_new = fmaxf(m, mx);
      const float alpha = ex2_approx((m - m_new) * kAttnScaleLog2);
      const float mc = m_new * kAttnScaleLog2;
      if (j > 0) {
        const int s = (j - 1) & 1;
        if (!mbar_wait(&pv_full[s], static_cast<uint32_t>((j - 1) >> 1) & 1u, abort_flag, gstatus,
                       DEV_TIMEOUT_ATTN + 7)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float v[32];
          __syncwarp();
          tmem_ld32(lane_base + 128u + static_cast<uint32_t>(s * 64 + c * 32), v);
#pragma unroll
          for (int t = 0; t < 32; ++t) o[c * 32 + t] = fmaf(o[c * 32 + t], alpha_prev, v[t]);
        }
      }
      float rs = 0.f;
#pragma unroll 1
      for (int c = 0; c < ATT_BN / 32; ++c) {
        float v[32];
        __syncwarp();
        tmem_ld32(lane_base + c * 32, v);
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int k0 = c * 32 + 2 * t;
          const float e0 = (k0 < valid) ? ex2_approx(fmaf(v[2 * t], kAttnScaleLog2, -mc)) : 0.f;
          const float e1 = (k0 + 1 < valid) ? ex2_approx(fmaf(v[2 * t + 1], kAttnScaleLog2, -mc)) : 0.f;
          rs += e0 + e1;
          pk[t] = pack_bf16x2(e0, e1);
        }
        uint8_t* prow = sP + (c >> 1) * (AttnCfg::P_BYTES / 2) + r * 128;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int chunk = ((c & 1) * 4 + t) ^ (r & 7);
          *reinterpret_cast<uint4*>(prow + chunk * 16) = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
        }
      }
      l = fmaf(l, alpha, rs);
      m = m_new;
      alpha_prev = alpha;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && nkv > 0) {
      const int s = (nkv - 1) & 1;
      if (mbar_wait(&pv_full[s], static_cast<uint32_t>((nkv - 1) >> 1) & 1u, abort_flag, gstatus,
                    DEV_TIMEOUT_ATTN + 8)) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float v[32];
          __syncwarp();
          tmem_ld32(lane_base + 128u + static_cast<uint32_t>(s * 64 + c * 32), v);
#pragma unroll
          for (int t = 0; t < 32; ++t) o[c * 32 + t] = fmaf(o[c * 32 + t], alpha_prev, v[t]);
        }
        const int row = qblk * ATT_BM + r;
        if (row < T) {
          const float inv = 1.0f / l;
          uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<size_t>(b) * T + row) * D + h * 64);
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            dst[t] = make_uint4(pack_bf16x2(o[8 * t + 0] * inv, o[8 * t + 1] * inv),
                                pack_bf16x2(o[8 * t + 2] * inv, o[8 * t + 3] * inv),
                                pack_bf16x2(o[8 * t + 4] * inv, o[8 * t + 5] * inv),
                                pack_bf16x2(o[8 * t + 6] * inv, o[8 * t + 7] * inv));
          }
        }
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  __syncthreads();
  if (warp == 1) {
    if (!skip && lane == 0) mbar_wait_drain(mma_done, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, AttnCfg::TMEM_COLS);
  }
}

}  // namespace vit
