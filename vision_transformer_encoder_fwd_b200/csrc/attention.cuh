// Fused multi-head self-attention forward for sm_100a (tcgen05 + TMA), head width 64.
//
// "DINOv2 n semantic" diagram, panel "Encoder self-attention": per head, softmax over keys of
// Q K^T / sqrt(64), times V, heads merged.  kornia/dinov3 card, "Build BF16, not FP16": the
// scaled logits reach ~2.5e6, so Q, K, V and P stay bf16 while the logits, the running maximum
// and the running sum are fp32 (fp32's exponent range).
//
// One CTA per (128-query tile, head, image); 6 warps, two CTAs per SM:
//   warp 0 (one lane)  TMA: K_n and V_n (64 keys x 64 dims each) into a 6-deep ring, read from
//                      the stacked QKV activation [B, T, 3D] through a 3-D tensor map (rows past
//                      T are zero-filled).
//   warp 1             allocates 256 TMEM columns; one lane issues the MMAs.  The keys are taken
//                      in sub-blocks of 64, and S has two 64-column buffers that the sub-blocks
//                      alternate between:
//                        S_b = Q K_n^T              (A = Q from TMEM, B = K_n, N = 64)
//                        O  += P_n [V_n | 1]        (A = P from TMEM, B = V_n,
//                                                    MN-major, extended by a constant column of
//                                                    ones, N = 80)
//                      P of a sub-block overwrites the first 32 columns of its own S buffer, and
//                      the tensor pipe executes one thread's MMAs in issue order, so the S of
//                      sub-block n + 2 is issued into that buffer right after the PV of
//                      sub-block n: the S of the next sub-block is always computed while the
//                      softmax works on the current one.  Column 64 of O accumulates sum_k P_k
//                      in fp32 -- the softmax denominator of exactly the bf16 P that multiplies V.
//   warps 2..5         softmax, one query row per thread (TMEM lane = row).  First each thread
//                      copies its Q row from global memory into TMEM.  Per sub-block: one
//                      64-column load of S, row maximum over the valid keys, P = 2^((s - m)
//                      log2(e) / 8) -- exponent pairs from one packed fp32 FMA, the exponential
//                      from the special-function unit for most keys and from a cubic on the FMA
//                      pipe for the rest -- packed to bf16 and written over S.  The running
//                      maximum is only moved when it grows by more than 2^8 (O, including its
//                      sum column, is then rescaled in TMEM first), so every P stays <= 256.
// TMEM: S buffers [0,64) and [64,128), O [128,208), Q [208,240) of 256 (32-bit columns, lane =
// row; Q and P hold two bf16 per column).  Two CTAs share an SM, so one CTA's MMAs run while the
// other's softmax computes exponentials.
#pragma once

#include "common.cuh"

namespace vit {

constexpr int ATT_BM = 128;       // query rows per CTA
constexpr int ATT_BN = 64;        // keys per TMA stage: one sub-block
constexpr int ATT_SUB = 64;       // keys per S buffer
constexpr int ATT_THREADS = 192;
constexpr int ATT_KV_STAGES = 6;  // (three 128-key stages measured 3.5 % slower at ViT-L/16@1024 b8)

struct AttnCfg {
  static constexpr int K_BYTES = ATT_BN * 64 * 2;   // 8 KB
  static constexpr int V_BYTES = ATT_BN * 64 * 2;   // 8 KB
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + ATT_KV_STAGES * K_BYTES;
  // the constant "ones" MN-major atom that extends every V stage by 16 columns (1, 0, ..., 0)
  static constexpr int OFF_ONES = OFF_V + ATT_KV_STAGES * V_BYTES;
  static constexpr int OFF_BAR = OFF_ONES + V_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 256;
  static_assert(8 * (2 * ATT_KV_STAGES + 7) + 8 <= 256, "barrier area too small");
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr int O_COLS = 80;                 // 64 output columns + the sum column + padding
  static constexpr uint32_t TM_S = 0, TM_O = 128, TM_Q = 208;
};

// log2(e) / sqrt(64)
constexpr float kAttnScaleLog2 = 0.18033688011112042f;
// The running maximum moves only when a row's maximum grows by more than 2^8.
constexpr float kRescaleLog2 = 8.0f;

// The last key pair of every 16 takes the FMA-pipe exponential, the other 14 keys the
// special-function unit (all on the special-function unit, or 2 or 4 of every 8 on the FMA pipe,
// measured 0.7-8 % slower on the ViT-L/16@1024 shape).
constexpr int kPolyEvery = 16;

// 2^x on the FMA pipe for a pair of values: x = j + f with j = round(x) (add 1.5 * 2^23) and
// |f| <= 1/2, 2^f from a cubic (Remez fit of the relative error, max 7.5e-5; see
// gen_exp2_poly.py), 2^j added into the exponent field.  x is clamped at -125 so that the
// result stays a normal float.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = fadd2(x, make_float2(12582912.0f, 12582912.0f));
  const float2 j = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = fadd2(x, make_float2(-j.x, -j.y));
  float2 p = ffma2(make_float2(0.0551716685f, 0.0551716685f), f, make_float2(0.242611125f, 0.242611125f));
  p = ffma2(p, f, make_float2(0.693260968f, 0.693260968f));
  p = ffma2(p, f, make_float2(0.999928057f, 0.999928057f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Row maximum of 64 logits with four independent 3-input max chains.
__device__ __forceinline__ float row_max64(const float (&s)[64]) {
  float m0 = fmaxf(s[0], s[1]), m1 = fmaxf(s[2], s[3]), m2 = fmaxf(s[4], s[5]), m3 = fmaxf(s[6], s[7]);
#pragma unroll
  for (int t = 8; t < 64; t += 8) {
    m0 = fmax3(m0, s[t], s[t + 1]);
    m1 = fmax3(m1, s[t + 2], s[t + 3]);
    m2 = fmax3(m2, s[t + 4], s[t + 5]);
    m3 = fmax3(m3, s[t + 6], s[t + 7]);
  }
  return fmax3(m0, m1, fmaxf(m2, m3));
}

// P for one row of a 64-key sub-block: p = 2^(s * c - m * c) for pairs of keys (one packed fp32
// FMA forms the exponent pair); masked keys carry s = -inf and come out as 0 (the FMA-pipe path
// clamps them to 2^-125 and they are zeroed explicitly).  The 64 values are packed to bf16 and
// stored to the first 32 columns of the sub-block's S buffer (t_p); `full` is arrived on once the
// stores have completed.
template <bool MASK>
__device__ __forceinline__ void softmax_sub_p(const float (&s)[64], float mc, int valid, uint32_t t_p, uint64_t* full) {
  const float2 cc = make_float2(kAttnScaleLog2, kAttnScaleLog2);
  const float2 nm = make_float2(-mc, -mc);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int u = 0; u < 32; u += 2) {
      const int t = c * 32 + u;
      const float2 x = ffma2(make_float2(s[t], s[t + 1]), cc, nm);
      float2 e;
      if ((t & (kPolyEvery - 1)) == kPolyEvery - 2) {
        e = exp2_fma2(x);
        if (MASK) {
          e.x = (t < valid) ? e.x : 0.f;
          e.y = (t + 1 < valid) ? e.y : 0.f;
        }
      } else {
        e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      }
      pk[u >> 1] = pack_bf16x2(e.x, e.y);
    }
    tmem_st16_nowait(t_p + c * 16, pk);
  }
  tmem_st_wait();
  tc_fence_before();
  mbar_arrive(full);
}

// kBounded: the launch set a pipeline-wait limit (wait_ns); the default instantiation keeps the
// fixed 2 s limit out of every wait's fast path.
template <bool kBounded>
__global__ void __launch_bounds__(ATT_THREADS, 2)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQKV, const __nv_bfloat16* __restrict__ qkv, int T, int D,
                       __nv_bfloat16* __restrict__ out, int* gstatus, unsigned long long wait_ns) {
  const unsigned long long wlim = kBounded ? wait_ns : 0ull;  // 0: the default limit
  extern __shared__ __align__(1024) uint8_t smem[];
  // The swizzled layouts assume 1024-byte aligned tiles; report and stop if the shared window
  // is not (uniform across the CTA, before anything is allocated).
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicExch(gstatus, DEV_TIMEOUT_ATTN + 15);
    return;
  }
  uint8_t* sK = smem + AttnCfg::OFF_K;
  uint8_t* sV = smem + AttnCfg::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnCfg::OFF_BAR);
  uint64_t* kv_full = bars;                               // [ATT_KV_STAGES]
  uint64_t* kv_empty = kv_full + ATT_KV_STAGES;           // [ATT_KV_STAGES]
  uint64_t* s_full = kv_empty + ATT_KV_STAGES;            // [2]: S buffer b holds a new sub-block
  uint64_t* p_full = s_full + 2;                          // [2]: P of the sub-block in buffer b stored
  uint64_t* pv_done = p_full + 2;                         // 1: the PV MMAs issued so far completed
  uint64_t* mma_done = pv_done + 1;                       // 1
  uint64_t* q_ready = mma_done + 1;                       // 1: the Q tile copied into TMEM
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(q_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int nkv = (T + ATT_BN - 1) / ATT_BN;
  const int nsub = (T + ATT_SUB - 1) / ATT_SUB;

  // Launched to start early: wait for the previous kernel before anything else (setting up the
  // barriers and TMEM first, as the GEMMs do, measured slower here).
  pdl_wait();
  if (threadIdx.x == 0) {
    *abort_flag = (*reinterpret_cast<volatile int*>(gstatus) != 0) ? 1 : 0;
    mbar_init(q_ready, 128);
    for (int s = 0; s < ATT_KV_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQKV);
  }
  {
    // The ones atom: 64 key rows of 128 bytes in the 128-byte-swizzled MN-major layout, value
    // 1.0 at N position 0 of every row (16-byte chunk 0, swizzled to chunk r % 8), 0 elsewhere.
    uint4* ones = reinterpret_cast<uint4*>(smem + AttnCfg::OFF_ONES);
    for (int i = threadIdx.x; i < AttnCfg::V_BYTES / 16; i += blockDim.x) {
      const int row = i >> 3, chunk = i & 7;
      ones[i] = make_uint4((chunk == (row & 7)) ? 0x3F80u : 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, AttnCfg::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const bool skip = *abort_flag != 0;

  if (!skip && warp == 0 && lane == 0) {
    // ------------------------------------------------------------------ TMA producer
    int issued_parity[ATT_KV_STAGES];
    for (int s = 0; s < ATT_KV_STAGES; ++s) issued_parity[s] = -1;
    for (int j = 0; j < nkv; ++j) {
      const int s = j % ATT_KV_STAGES;
      const uint32_t ph = static_cast<uint32_t>(j / ATT_KV_STAGES) & 1u;
      if (!mbar_wait(&kv_empty[s], ph ^ 1u, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 1, wlim)) break;
      mbar_arrive_expect_tx(&kv_full[s], AttnCfg::K_BYTES + AttnCfg::V_BYTES);
      tma_load_3d(sK + s * AttnCfg::K_BYTES, &tmQKV, D + h * 64, j * ATT_BN, b, &kv_full[s]);
      tma_load_3d(sV + s * AttnCfg::V_BYTES, &tmQKV, 2 * D + h * 64, j * ATT_BN, b, &kv_full[s]);
      issued_parity[s] = static_cast<int>(ph);
    }
    if (*abort_flag) {
      for (int s = 0; s < ATT_KV_STAGES; ++s)
        if (issued_parity[s] >= 0) mbar_wait_drain(&kv_full[s], static_cast<uint32_t>(issued_parity[s]));
    }
  } else if (!skip && warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // (its waits poll with a 32 ns suspend-time hint: 0-4 % faster than the default suspension on
    // the measured shapes, the softmax and TMA waits keep the default)
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(ATT_BM, ATT_SUB, false);
      constexpr uint32_t idesc_o = idesc_bf16(ATT_BM, AttnCfg::O_COLS, true);
      const uint32_t k0 = smem_u32(sK);
      const uint32_t v0 = smem_u32(sV);
      const uint32_t ones0 = smem_u32(smem + AttnCfg::OFF_ONES);
      // Every MMA operand is built once: K and V descriptors per stage and K step (a K step only
      // moves the start address: +32 bytes for K, +2048 for V), TMEM addresses.  Stage st moves
      // the K start address by st * K_BYTES and the V start address by st * V_BYTES while the V
      // leading byte offset (distance to the ones atom) shrinks by the same amount: both are
      // linear in st, so the stage descriptors are one add away.
      uint64_t dk0[4], dv0[4];
      {
        const uint64_t d0 = sdesc_sw128(k0, 16, 1024);
        const uint64_t v0d = sdesc_sw128(v0, ones0 - v0, 1024);
#pragma unroll
        for (int k = 0; k < 4; ++k) dk0[k] = d0 + 2 * k;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) dv0[kk] = v0d + 128 * kk;
      }
      constexpr uint64_t kStepK = AttnCfg::K_BYTES >> 4;
      constexpr uint64_t kStepV = (AttnCfg::V_BYTES >> 4) - (static_cast<uint64_t>(AttnCfg::V_BYTES >> 4) << 16);
      const uint32_t t_s0 = tmem_base + AttnCfg::TM_S, t_q0 = tmem_base + AttnCfg::TM_Q;
      const uint32_t t_o0 = tmem_base + AttnCfg::TM_O;
      uint32_t aq[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) aq[k] = t_q0 + k * 8;
      // S of sub-block n (stage n % ATT_KV_STAGES) into buffer n % 2
      auto issue_s = [&](int n) {
        const int st = n % ATT_KV_STAGES;
        uint64_t dk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) dk[k] = dk0[k] + static_cast<uint64_t>(st) * kStepK;
        tc_mma_ts_chain4(t_s0 + ATT_SUB * (n & 1), aq, dk, idesc_s, 0u);
        tc_commit(&s_full[n & 1]);
      };
      bool ok = mbar_wait<32>(q_ready, 0, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 2, wlim) &&
                mbar_wait<32>(&kv_full[0], 0, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 3, wlim);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      if (ok && nsub > 1) {
        ok = mbar_wait<32>(&kv_full[1], 0, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 3, wlim);
        if (ok) {
          tc_fence_after();
          issue_s(1);
        }
      }
      for (int n = 0; ok && n < nsub; ++n) {
        const int buf = n & 1;
        const int st = n % ATT_KV_STAGES;
        if (!mbar_wait<32>(&p_full[buf], static_cast<uint32_t>(n >> 1) & 1u, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 4,
                       wlim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        {
          const uint32_t tp = t_s0 + ATT_SUB * buf;
          const uint32_t a_p[4] = {tp, tp + 8, tp + 16, tp + 24};
          uint64_t b_v[4];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            b_v[kk] = dv0[kk] + static_cast<uint64_t>(st) * kStepV;
          tc_mma_ts_chain4(t_o0, a_p, b_v, idesc_o, n > 0 ? 1u : 0u);
        }
        tc_commit(pv_done);
        if (n + 2 < nsub) {
          const int j2 = n + 2;
          if (!mbar_wait<32>(&kv_full[j2 % ATT_KV_STAGES], static_cast<uint32_t>(j2 / ATT_KV_STAGES) & 1u, abort_flag,
                         gstatus, DEV_TIMEOUT_ATTN + 5, wlim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(n + 2);
        }
        tc_commit(&kv_empty[st]);
      }
      tc_commit(mma_done);
    }
    __syncwarp();
  } else if (!skip && warp >= 2) {
    // ------------------------------------------------------------------ softmax
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t t_s = tmem_base + lane_off + AttnCfg::TM_S;
    const uint32_t t_o = tmem_base + lane_off + AttnCfg::TM_O;
    {
      // this thread's query row (64 bf16 = 32 columns, two per column) into TMEM
      const int qrow = tile * ATT_BM + r;
      uint32_t qv[32];
      if (qrow < T) {
        const uint4* src = reinterpret_cast<const uint4*>(qkv + (static_cast<size_t>(b) * T + qrow) * (3 * D) + h * 64);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const uint4 w = __ldg(src + t);
          qv[4 * t] = w.x;
          qv[4 * t + 1] = w.y;
          qv[4 * t + 2] = w.z;
          qv[4 * t + 3] = w.w;
        }
      } else {
#pragma unroll
        for (int t = 0; t < 32; ++t) qv[t] = 0u;
      }
      __syncwarp();
      tmem_st32(tmem_base + lane_off + AttnCfg::TM_Q, qv);
      tc_fence_before();
      mbar_arrive(q_ready);
    }
    float m = -INFINITY;
    bool ok = true;
    for (int n = 0; n < nsub; ++n) {
      const int buf = n & 1;
      if (!mbar_wait(&s_full[buf], static_cast<uint32_t>(n >> 1) & 1u, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 6,
                     wlim)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64];
      __syncwarp();
      tmem_ld64(t_s + ATT_SUB * buf, s);
      const int valid = min(ATT_SUB, T - n * ATT_SUB);
      if (valid < ATT_SUB) {
#pragma unroll
        for (int t = 0; t < 64; ++t) s[t] = (t < valid) ? s[t] : -INFINITY;
      }
      const float mx = row_max64(s);
      const float m_new = fmaxf(m, mx);
      const bool resc = (m_new - m) * kAttnScaleLog2 > kRescaleLog2;
      float alpha = 1.f;
      if (resc) {
        alpha = ex2_approx((m - m_new) * kAttnScaleLog2);
        m = m_new;
      }
      if (n > 0 && __any_sync(0xffffffffu, resc)) {
        // O holds the sub-blocks before n at the old maximum: wait for the last of them, rescale
        // (the sum column included) before this sub-block's P is released to the MMA.
        if (!mbar_wait(pv_done, static_cast<uint32_t>(n - 1) & 1u, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 7, wlim)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < AttnCfg::O_COLS; c += 16) {
          float o[16];
          tmem_ld16(t_o + c, o);
          uint32_t ob[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) ob[t] = __float_as_uint(o[t] * alpha);
          tmem_st16(t_o + c, ob);
        }
      }
      const float mc = m * kAttnScaleLog2;
      __syncwarp();
      if (valid < ATT_SUB)
        softmax_sub_p<true>(s, mc, valid, t_s + ATT_SUB * buf, &p_full[buf]);
      else
        softmax_sub_p<false>(s, mc, valid, t_s + ATT_SUB * buf, &p_full[buf]);
    }
    if (ok && mbar_wait(mma_done, 0, abort_flag, gstatus, DEV_TIMEOUT_ATTN + 8, wlim)) {
      tc_fence_after();
      float o[64], lsum[16];
      __syncwarp();
      tmem_ld64(t_o, o);
      tmem_ld16(t_o + 64, lsum);
      const int row = tile * ATT_BM + r;
      if (row < T) {
        const float inv = 1.0f / lsum[0];
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
