// libvit_b200: host side of the C ABI declared in include/vit.h and include/vit_stages.h.
//
// Plans and launches the encoder forward of the DINOv2/DINOv3 ViT ("DINOv2 n semantic"
// diagram; kornia/dinov3 card) and the dino.txt zero-shot scoring on one B200:
//   im2col -> patch GEMM (+bias +pos, token placement) -> CLS/register rows, row stats and the
//   re-centred bf16 copy of every token row
//   per block: QKV GEMM (LayerNorm folded) -> attention -> proj GEMM (+LS, residual, stats)
//              -> FC1 GEMM (LayerNorm folded, GELU) -> FC2 GEMM (+LS, residual, stats) [-> tap]
//   final LayerNorm -> descriptor / patch tokens
// All compute runs in the kernels of this library; this file only validates, lays out the
// workspace, encodes TMA descriptors and enqueues launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/vit.h"
#include "../../include/vit_stages.h"
#include "attention.cuh"
#include "aux_kernels.cuh"
#include "dense_head.cuh"
#include "gemm.cuh"

using namespace vit;

namespace {

thread_local std::string g_err;

void set_err(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
}

#define CK(call)                                                                              \
  do {                                                                                        \
    cudaError_t e_ = (call);                                                                  \
    if (e_ != cudaSuccess) {                                                                  \
      set_err("%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__, __LINE__);     \
      return VIT_E_CUDA;                                                                      \
    }                                                                                         \
  } while (0)

#define CKL()                                                                                 \
  do {                                                                                        \
    cudaError_t e_ = cudaGetLastError();                                                      \
    if (e_ != cudaSuccess) {                                                                  \
      set_err("kernel launch failed: %s (%s:%d)", cudaGetErrorString(e_), __FILE__, __LINE__); \
      return VIT_E_CUDA;                                                                      \
    }                                                                                         \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ------------------------------------------------------------------ TMA descriptor encoding
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 map over a row-major [rows, cols] matrix with leading dimension ld (elements);
// box = box_cols x box_rows with box_cols * 2 bytes == 128 (one 128-byte swizzle row).
bool tmap_2d(CUtensorMap* tm, const void* base, uint64_t cols, uint64_t rows, uint64_t ld, uint32_t box_cols,
             uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    set_err("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_err("cuTensorMapEncodeTiled(2d) failed with %d (cols %llu rows %llu ld %llu)", static_cast<int>(r),
            static_cast<unsigned long long>(cols), static_cast<unsigned long long>(rows),
            static_cast<unsigned long long>(ld));
    return false;
  }
  return true;
}

// 2-D map of an arbitrary element type for the epilogue's TMA stores and x loads: row-major
// [rows, cols] with leading dimension ld (elements), box box_cols x box_rows, given swizzle.
bool tmap_2d_any(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype, uint32_t elem_bytes, uint64_t cols,
                 uint64_t rows, uint64_t ld, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    set_err("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_err("cuTensorMapEncodeTiled(epilogue map) failed with %d", static_cast<int>(r));
    return false;
  }
  return true;
}
// bf16 output [M, ld] stored in boxes of 64 columns x 32 rows (one epilogue warp, 128B swizzle)
bool tmap_out_bf16(CUtensorMap* tm, const void* base, uint64_t cols, uint64_t rows, uint64_t ld) {
  return tmap_2d_any(tm, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cols, rows, ld, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
}
// fp32 residual stream [M, D] in boxes of 32 columns x 32 rows (128B swizzle)
bool tmap_x_f32(CUtensorMap* tm, const void* base, uint64_t cols, uint64_t rows) {
  return tmap_2d_any(tm, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, cols, rows, cols, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
}
// bf16 copy of x [M, D] in boxes of 32 columns x 32 rows (64B swizzle)
bool tmap_xb_bf16(CUtensorMap* tm, const void* base, uint64_t cols, uint64_t rows) {
  return tmap_2d_any(tm, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cols, rows, cols, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

// 3-D bf16 map over qkv [B, T, 3D]: dims {3D, T, B}, box {64, 128, 1}.
bool tmap_qkv3d(CUtensorMap* tm, const void* base, int B, int T, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    set_err("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(3 * D), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(3 * D) * 2, static_cast<cuuint64_t>(T) * 3 * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(ATT_BN), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_err("cuTensorMapEncodeTiled(3d) failed with %d", static_cast<int>(r));
    return false;
  }
  return true;
}

// ------------------------------------------------------------------ launch helpers
int device_sms(int dev) {
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

template <typename K>
cudaError_t set_smem_attr_once(K kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load() & bit) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit);
  return e;
}

// Programmatic dependent launch for the tensor-core kernels, which call pdl_wait before they touch
// global memory: each may be scheduled, and run its prologue (barrier set-up, tensor-memory
// allocation), while the kernel before it in the stream finishes.  VIT_B200_PDL=0 in the
// environment launches them in plain stream order instead.
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("VIT_B200_PDL");
    return !(e != nullptr && e[0] == '0');
  }();
  return on;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int BN, int MODE, int XBUF = 2>
cudaError_t launch_gemm_t(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o1, const CUtensorMap& o2,
                          int M, int N, int K, const EpiParams& ep, int* st, cudaStream_t s, int nsm) {
  static std::atomic<uint64_t> attr_done{0};
  constexpr int smem = GemmCfg<BN, MODE, XBUF>::SMEM_BYTES;
  cudaError_t e = set_smem_attr_once(gemm_bf16_tc_kernel<BN, MODE, XBUF>, smem, attr_done);
  if (e != cudaSuccess) return e;
  const int tiles = ((M + GEMM_BM - 1) / GEMM_BM) * (N / BN);
  const int grid = std::max(1, std::min(tiles, nsm));
  return launch_pdl(gemm_bf16_tc_kernel<BN, MODE, XBUF>, dim3(grid), dim3(GEMM_THREADS), smem, s, a, b, o1, o2, M, N, K,
                    ep, st);
}

// Tile code for the paired kernel (a 2-CTA cluster per 256 x 256 tile); its B map has 128-row boxes.
constexpr int BN_PAIR = 512;
// Host-side mode: the residual epilogue with one x buffer per warp and one more operand stage
// (paired and 128-wide tiles; 128 x 256 tiles run EPI_RESID).
constexpr int EPI_RESID_DEEP = 16;

template <int MODE, int XBUF = 2>
cudaError_t launch_gemm_pair_t(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o1,
                               const CUtensorMap& o2, int M, int N, int K, const EpiParams& ep, int* st, cudaStream_t s,
                               int nsm) {
  static std::atomic<uint64_t> attr_done{0};
  static std::atomic<int> max_clusters{0};
  constexpr int smem = PairCfg<MODE, XBUF>::SMEM_BYTES;
  cudaError_t e = set_smem_attr_once(gemm_pair_kernel<MODE, XBUF>, smem, attr_done);
  if (e != cudaSuccess) return e;
  int mc = max_clusters.load();
  if (mc == 0) {
    // how many 2-CTA clusters of this size fit on the device at once (the GPC layout can leave
    // an SM without a partner); the persistent grid never exceeds it
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (nsm / 2), 1, 1);
    cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<MODE, XBUF>, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = nsm / 2;
    }
    mc = std::max(1, std::min(n, nsm / 2));
    max_clusters.store(mc);
  }
  const int tiles = ((M + 2 * GEMM_BM - 1) / (2 * GEMM_BM)) * ((N + 255) / 256);
  const int clusters = std::max(1, std::min(tiles, mc));
  return launch_pdl(gemm_pair_kernel<MODE, XBUF>, dim3(2 * clusters), dim3(GEMM_THREADS), smem, s, a, b, o1, o2, M, N, K, ep,
                    st);
}

// o1 / o2: BIAS, LNFOLD: o1 = bf16 output map (tmap_out_bf16); RESID: o1 = x (tmap_x_f32),
// o2 = xb (tmap_xb_bf16); PATCH, COS: not read (any valid map).  bn: 128 or 256 (one CTA per tile,
// B map boxes of bn rows) or BN_PAIR (B map boxes of 128 rows; not for PATCH).
cudaError_t launch_gemm(int bn, int mode, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o1,
                        const CUtensorMap& o2, int M, int N, int K, const EpiParams& ep, int* st, cudaStream_t s,
                        int nsm) {
  if (bn == BN_PAIR) {
    switch (mode) {
      case EPI_BIAS: return launch_gemm_pair_t<EPI_BIAS>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
      case EPI_LNFOLD: return launch_gemm_pair_t<EPI_LNFOLD>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
      case EPI_RESID: return launch_gemm_pair_t<EPI_RESID>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
      case EPI_RESID_DEEP: return launch_gemm_pair_t<EPI_RESID, 1>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
      default: return cudaErrorInvalidValue;
    }
  }
  if (mode == EPI_RESID_DEEP && bn == 128)
    return launch_gemm_t<128, EPI_RESID, 1>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
  if (mode == EPI_RESID_DEEP) mode = EPI_RESID;  // 128 x 256 tiles have no room for a deeper ring
  if (bn == 256) {
    switch (mode) {
      case EPI_BIAS: return launch_gemm_t<256, EPI_BIAS>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
      case EPI_LNFOLD: return launch_gemm_t<256, EPI_LNFOLD>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
      case EPI_RESID: return launch_gemm_t<256, EPI_RESID>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
      default: return launch_gemm_t<256, EPI_PATCH>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
    }
  }
  switch (mode) {
    case EPI_BIAS: return launch_gemm_t<128, EPI_BIAS>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
    case EPI_LNFOLD: return launch_gemm_t<128, EPI_LNFOLD>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
    case EPI_RESID: return launch_gemm_t<128, EPI_RESID>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
    case EPI_COS: return launch_gemm_t<128, EPI_COS>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
    default: return launch_gemm_t<128, EPI_PATCH>(a, b, o1, o2, M, N, K, ep, st, s, nsm);
  }
}

// One CTA per (128-query tile, head, image), two CTAs per SM.
cudaError_t launch_attention(const CUtensorMap& tm, const __nv_bfloat16* qkv, int B, int T, int heads,
                             __nv_bfloat16* out, int* st, cudaStream_t s, unsigned long long wait_ns) {
  static std::atomic<uint64_t> attr_done{0}, attr_done_b{0};
  const int n_qtiles = (T + ATT_BM - 1) / ATT_BM;
  dim3 grid(n_qtiles, heads, B);
  if (wait_ns == 0) {
    cudaError_t e = set_smem_attr_once(attn_fwd_tc_kernel<false>, AttnCfg::SMEM_BYTES, attr_done);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_fwd_tc_kernel<false>, grid, dim3(ATT_THREADS), AttnCfg::SMEM_BYTES, s, tm, qkv, T,
                      heads * 64, out, st, 0ull);
  }
  cudaError_t e = set_smem_attr_once(attn_fwd_tc_kernel<true>, AttnCfg::SMEM_BYTES, attr_done_b);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_fwd_tc_kernel<true>, grid, dim3(ATT_THREADS), AttnCfg::SMEM_BYTES, s, tm, qkv, T, heads * 64,
                    out, st, wait_ns);
}

int grid_1d(long long work, int block, int nsm) {
  long long g = (work + block - 1) / block;
  return static_cast<int>(std::max(1LL, std::min(g, static_cast<long long>(nsm) * 32)));
}

// GEMM tiling: the paired 256 x 256 tile when the pairs fill the SMs (N = 256 k + 128 pads the
// last column tile: a tile of 256 x 256 per SM pair moves as many bytes through each SM's shared
// memory per k-step as one of 128 x 128 per SM, for twice the MMA work), else 128 x 256 per CTA
// when N allows it and that fills the SMs, else 128 x 128.
int pick_bn(int M, int N, int nsm) {
  const long long pairs = static_cast<long long>((M + 2 * GEMM_BM - 1) / (2 * GEMM_BM)) * ((N + 255) / 256);
  if (pairs >= nsm / 2) return BN_PAIR;
  if (N % 256 != 0) return 128;
  const long long tiles256 = static_cast<long long>((M + GEMM_BM - 1) / GEMM_BM) * (N / 256);
  return tiles256 >= nsm ? 256 : 128;
}

// Residual GEMMs (proj, FC2): N = D; the paired tile when D is a multiple of 256 and the pairs
// fill the SMs, else bn_res (whose half-width fixes the statistics groups).  A padded paired
// tile was measured slower here than 128 x 128 (ViT-S/16@336 b64 proj 46 against 38 us): the
// residual epilogue, not the MMA, sets these tiles' pace.
int pick_bn_res(int M, int D, int bn_res, int nsm) {
  if (bn_res != 256) return bn_res;
  const long long pairs = static_cast<long long>((M + 2 * GEMM_BM - 1) / (2 * GEMM_BM)) * (D / 256);
  return pairs >= nsm / 2 ? BN_PAIR : 256;
}

}  // namespace

// ------------------------------------------------------------------ model
struct BlockW {
  __nv_bfloat16* qkv_wg;  // [3D, D] gamma-folded (owned)
  float* qkv_c;           // [3D]
  float* qkv_b;           // [3D] beta-folded bias
  const __nv_bfloat16* proj_w;  // borrowed
  float* proj_b;
  float* ls1;
  __nv_bfloat16* fc1_wg;  // [F, D] (owned)
  float* fc1_c;
  float* fc1_b;
  const __nv_bfloat16* fc2_w;  // borrowed
  float* fc2_b;
  float* ls2;
  CUtensorMap tm_qkv[2], tm_fc1[2];  // [0]: box rows 128, [1]: 256
  CUtensorMap tm_proj, tm_fc2;       // box rows bn_res
  CUtensorMap tm_proj_h, tm_fc2_h;   // box rows 128 (paired tiles)
};

struct vit_model {
  vit_config cfg;
  int device = 0, nsm = 1;
  int gh = 0, gw = 0, P = 0, T = 0, K_pe = 0, Kpad = 0, bn_res = 128, stats_cols = 64, nt = 1;
  __nv_bfloat16* patch_w = nullptr;  // [D, Kpad]
  float *patch_b = nullptr, *pos = nullptr, *cls = nullptr, *reg = nullptr, *norm_w = nullptr, *norm_b = nullptr;
  CUtensorMap tm_patch;
  std::vector<BlockW> blocks;
  std::vector<BlockW> head;  // dino.txt vision head blocks (vit_set_text_head), empty if none
  struct DenseW {
    bool on = false;
    int K = 0, W = 0;
    const __nv_bfloat16 *cv1_w = nullptr, *cv2_w = nullptr, *lat_w = nullptr;  // borrowed [O, C]
    __nv_bfloat16* bn_wr[6] = {};     // [h, 9h] (owned)
    __nv_bfloat16* smooth_wr = nullptr;  // [W, 9W] (owned)
    float *cv1_ln_w = nullptr, *cv1_ln_b = nullptr, *bn_ln_w[6] = {}, *bn_ln_b[6] = {};
    float *cv2_ln_w = nullptr, *cv2_ln_b = nullptr, *out_ln_w = nullptr, *out_ln_b = nullptr;
    float *lat_b = nullptr, *smooth_b = nullptr, *gn_w = nullptr, *gn_b = nullptr;
    float *pred_w = nullptr, *pred_b = nullptr, *zero = nullptr;
  } dense;  // dense head on the taps (vit_set_dense_head)
  int* d_status = nullptr;
  unsigned long long wait_ns = 0;  // pipeline-wait limit of this model's launches (0: 2 s)
  int last_launches = 0;
  std::vector<void*> allocs;
  // per-launch profiling (vit_profile_begin / vit_profile_end)
  bool prof_on = false;
  std::vector<cudaEvent_t> prof_ev;  // 2 per slot
  std::vector<int> prof_kind;
  int prof_used = 0;
};

namespace {

struct WsLayout {
  size_t x, xb, stats, ctr, attn, big, pos, total;
};

// The token geometry of one forward: input H x W, patch grid gh x gw (the convolution's
// floor), P patch tokens, T = 1 + R + P tokens.  `native` is the size the position embedding
// was learned for; any other size reads a bicubically resized copy of it from the workspace.
struct Geom {
  int H, W, gh, gw, P, T;
  bool native;
};

Geom geom_for(const vit_model* m, int H, int W) {
  Geom g;
  g.H = H;
  g.W = W;
  g.gh = H / m->cfg.patch;
  g.gw = W / m->cfg.patch;
  g.P = g.gh * g.gw;
  g.T = 1 + m->cfg.n_registers + g.P;
  g.native = (g.gh == m->gh && g.gw == m->gw);
  return g;
}

Geom native_geom(const vit_model* m) { return geom_for(m, m->cfg.img_h, m->cfg.img_w); }

vit_status check_geom(const vit_model* m, int B, const Geom& g) {
  if (g.H < m->cfg.patch || g.W < m->cfg.patch || g.H > 16384 || g.W > 16384) {
    set_err("image %dx%d outside %d..16384 per side (patch %d)", g.H, g.W, m->cfg.patch, m->cfg.patch);
    return VIT_E_SHAPE;
  }
  // TMA row coordinates and the GEMMs' M are 32-bit
  if (static_cast<long long>(B) * g.T >= (1LL << 30)) {
    set_err("batch %d x %d tokens exceeds 2^30 rows", B, g.T);
    return VIT_E_SHAPE;
  }
  return VIT_OK;
}

WsLayout ws_layout(const vit_model* m, int B, const Geom& g) {
  const size_t M = static_cast<size_t>(B) * g.T, Mp = static_cast<size_t>(B) * g.P;
  const size_t D = m->cfg.dim, F = m->cfg.mlp_dim;
  WsLayout L;
  size_t off = 0;
  L.x = off;
  off = align_up(off + M * D * 4, 1024);
  L.xb = off;
  off = align_up(off + M * D * 2, 1024);
  // two statistics buffers: a residual GEMM reads the partials of x before its update (the centre
  // of the new bf16 copy) from one and writes those of the new x into the other
  L.stats = off;
  off = align_up(off + 2 * M * m->nt * 8, 1024);
  L.ctr = off;
  off = align_up(off + M * 4, 1024);
  L.attn = off;
  off = align_up(off + M * D * 2, 1024);
  L.big = off;
  off = align_up(off + std::max(std::max(M * 3 * D, M * F), Mp * static_cast<size_t>(m->Kpad)) * 2, 1024);
  L.pos = off;
  if (!g.native) off = align_up(off + (static_cast<size_t>(g.P) + (m->cfg.pos_on_cls ? 1 : 0)) * D * 4, 1024);
  L.total = off;
  return L;
}

// NVTX range names of the launch kinds (the VIT_K_* order of vit.h).
const char* const kKindName[VIT_K_COUNT] = {
    "vit/im2col",   "vit/patch_gemm", "vit/token_prep",  "vit/qkv_gemm", "vit/attention",  "vit/proj_gemm",
    "vit/fc1_gemm", "vit/fc2_gemm",   "vit/tap",         "vit/final_ln", "vit/seg_split",  "vit/seg_cos_gemm",
    "vit/seg_map",  "vit/pos_resize", "vit/head_tokens", "vit/dense_gemm", "vit/dense_aux"};

// Brackets around one launch: an NVTX range named after the launch kind (seen by Nsight tools
// when one is attached, a no-op otherwise) and, while per-launch profiling is on and capacity
// remains, two CUDA events on the launch stream.
// Under stream capture a profiling record must become an external event-record node, so that
// every replay of the graph records the event again; outside a capture that flag is refused, and
// the record is a plain one.
void prof_record(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  else
    cudaEventRecord(e, s);
}

int prof_open(vit_model* m, int kind, cudaStream_t s) {
  nvtxRangePushA(kKindName[kind]);
  if (!m->prof_on || m->prof_used >= static_cast<int>(m->prof_kind.size())) return -1;
  const int slot = m->prof_used++;
  m->prof_kind[slot] = kind;
  prof_record(m->prof_ev[2 * slot], s);
  return slot;
}
void prof_close(vit_model* m, int slot, cudaStream_t s) {
  if (slot >= 0) prof_record(m->prof_ev[2 * slot + 1], s);
  nvtxRangePop();
}

// Every launch of a model must run on the device whose memory holds its weights, derived
// copies and TMA descriptors; the caller picks the current device, so each entry point that
// launches checks it before anything is enqueued.
vit_status check_device(const vit_model* m, const char* fn) {
  int cur = 0;
  CK(cudaGetDevice(&cur));
  if (cur != m->device) {
    set_err("%s called with device %d current; the model lives on device %d", fn, cur, m->device);
    return VIT_E_INVALID_ARG;
  }
  return VIT_OK;
}

vit_status alloc_dev(vit_model* m, void** p, size_t bytes) {
  CK(cudaMalloc(p, std::max<size_t>(bytes, 16)));
  m->allocs.push_back(*p);
  return VIT_OK;
}

vit_status to_f32(vit_model* m, const void* src, size_t n, float** dst, cudaStream_t s) {
  vit_status st = alloc_dev(m, reinterpret_cast<void**>(dst), n * 4);
  if (st != VIT_OK) return st;
  if (n == 0) return VIT_OK;
  bf16_to_f32_kernel<<<grid_1d(static_cast<long long>(n), 256, m->nsm), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(src), static_cast<long long>(n), *dst);
  CKL();
  return VIT_OK;
}

vit_status validate_cfg(const vit_config* c) {
  if (!c) {
    set_err("config is NULL");
    return VIT_E_INVALID_ARG;
  }
  if (c->heads < 1 || c->dim != c->heads * 64) {
    set_err("dim (%d) must equal heads (%d) * 64", c->dim, c->heads);
    return VIT_E_UNSUPPORTED;
  }
  if (c->dim % 128 != 0 || c->mlp_dim % 128 != 0 || c->mlp_dim < 128) {
    set_err("dim (%d) and mlp_dim (%d) must be multiples of 128", c->dim, c->mlp_dim);
    return VIT_E_UNSUPPORTED;
  }
  if (c->patch < 1 || c->patch > 32 || c->img_h < c->patch || c->img_w < c->patch || c->img_h % c->patch ||
      c->img_w % c->patch) {
    set_err("image %dx%d must be a positive multiple of patch %d (1..32)", c->img_h, c->img_w, c->patch);
    return VIT_E_SHAPE;
  }
  if (c->n_registers < 0 || c->n_registers > 16 || c->depth < 1 || c->depth > 64 || c->max_batch < 1 ||
      !(c->ln_eps > 0.f)) {
    set_err("n_registers 0..16, depth 1..64, max_batch >= 1 and ln_eps > 0 required");
    return VIT_E_INVALID_ARG;
  }
  int ntaps = 0;
  for (int l = 0; l < 32; ++l)
    if (c->tap_mask & (1u << l)) {
      ++ntaps;
      if (l + 1 > c->depth) {
        set_err("tap after block %d exceeds depth %d", l + 1, c->depth);
        return VIT_E_INVALID_ARG;
      }
    }
  if (ntaps > 4) {
    set_err("at most 4 taps");
    return VIT_E_INVALID_ARG;
  }
  return VIT_OK;
}

// Device copies of one encoder block's weights: the LN-folded QKV and FC1 matrices with their
// column sums and folded biases, fp32 vectors, and the TMA maps of all four GEMM operands.
vit_status build_block(vit_model* m, const vit_block_weights& src, BlockW& b, cudaStream_t s) {
  const int D = m->cfg.dim, F = m->cfg.mlp_dim;
  vit_status e;
  if ((e = alloc_dev(m, reinterpret_cast<void**>(&b.qkv_wg), static_cast<size_t>(3) * D * D * 2)) != VIT_OK) return e;
  if ((e = alloc_dev(m, reinterpret_cast<void**>(&b.qkv_c), static_cast<size_t>(3) * D * 4)) != VIT_OK) return e;
  if ((e = alloc_dev(m, reinterpret_cast<void**>(&b.qkv_b), static_cast<size_t>(3) * D * 4)) != VIT_OK) return e;
  if ((e = alloc_dev(m, reinterpret_cast<void**>(&b.fc1_wg), static_cast<size_t>(F) * D * 2)) != VIT_OK) return e;
  if ((e = alloc_dev(m, reinterpret_cast<void**>(&b.fc1_c), static_cast<size_t>(F) * 4)) != VIT_OK) return e;
  if ((e = alloc_dev(m, reinterpret_cast<void**>(&b.fc1_b), static_cast<size_t>(F) * 4)) != VIT_OK) return e;
  fold_ln_weight_kernel<<<3 * D, 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(src.qkv_w), static_cast<const __nv_bfloat16*>(src.qkv_b),
      static_cast<const __nv_bfloat16*>(src.ln1_w), static_cast<const __nv_bfloat16*>(src.ln1_b), 3 * D, D, b.qkv_wg,
      b.qkv_c, b.qkv_b);
  CKL();
  fold_ln_weight_kernel<<<F, 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(src.fc1_w), static_cast<const __nv_bfloat16*>(src.fc1_b),
      static_cast<const __nv_bfloat16*>(src.ln2_w), static_cast<const __nv_bfloat16*>(src.ln2_b), F, D, b.fc1_wg,
      b.fc1_c, b.fc1_b);
  CKL();
  b.proj_w = static_cast<const __nv_bfloat16*>(src.proj_w);
  b.fc2_w = static_cast<const __nv_bfloat16*>(src.fc2_w);
  if ((e = to_f32(m, src.proj_b, D, &b.proj_b, s)) != VIT_OK) return e;
  if ((e = to_f32(m, src.ls1, D, &b.ls1, s)) != VIT_OK) return e;
  if ((e = to_f32(m, src.fc2_b, D, &b.fc2_b, s)) != VIT_OK) return e;
  if ((e = to_f32(m, src.ls2, D, &b.ls2, s)) != VIT_OK) return e;
  if (!tmap_2d(&b.tm_qkv[0], b.qkv_wg, D, 3 * D, D, 64, 128) || !tmap_2d(&b.tm_fc1[0], b.fc1_wg, D, F, D, 64, 128) ||
      !tmap_2d(&b.tm_proj, b.proj_w, D, D, D, 64, m->bn_res) ||
      !tmap_2d(&b.tm_fc2, b.fc2_w, F, D, F, 64, m->bn_res) || !tmap_2d(&b.tm_proj_h, b.proj_w, D, D, D, 64, 128) ||
      !tmap_2d(&b.tm_fc2_h, b.fc2_w, F, D, F, 64, 128))
    return VIT_E_CUDA;
  b.tm_qkv[1] = b.tm_qkv[0];
  b.tm_fc1[1] = b.tm_fc1[0];
  if ((3 * D) % 256 == 0 && !tmap_2d(&b.tm_qkv[1], b.qkv_wg, D, 3 * D, D, 64, 256)) return VIT_E_CUDA;
  if (F % 256 == 0 && !tmap_2d(&b.tm_fc1[1], b.fc1_wg, D, F, D, 64, 256)) return VIT_E_CUDA;
  return VIT_OK;
}

struct Scratch {
  float* x;
  __nv_bfloat16* xb;
  float2* stats[2];
  float* ctr;
  __nv_bfloat16* attn;
  __nv_bfloat16* big;
};

// The encoder forward on B images read through `src`; outputs per `out`.  With `head` (and a
// head attached) the dino.txt vision head runs after the backbone and `out->patch_tokens`
// (fp32) receives its patch rows; the descriptor is not written then.
vit_status run_forward(vit_model* m, const ImgSrc& src, int B, const Geom& g, const vit_outputs* out, void* ws,
                       size_t ws_bytes, cudaStream_t s, bool head = false, __nv_bfloat16* tap_rows = nullptr) {
  const vit_config& c = m->cfg;
  vit_status gst = check_device(m, "the forward");
  if (gst != VIT_OK) return gst;
  gst = check_geom(m, B, g);
  if (gst != VIT_OK) return gst;
  const WsLayout L = ws_layout(m, B, g);
  if (ws == nullptr || ws_bytes < L.total) {
    set_err("workspace of %zu bytes is smaller than the %zu required for batch %d", ws_bytes, L.total, B);
    return VIT_E_WORKSPACE;
  }
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) {
    set_err("workspace must be 256-byte aligned");
    return VIT_E_INVALID_ARG;
  }
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int D = c.dim, F = c.mlp_dim, T = g.T, P = g.P, R = c.n_registers;
  const int M = B * T, Mp = B * P;
  Scratch S{reinterpret_cast<float*>(w8 + L.x),
            reinterpret_cast<__nv_bfloat16*>(w8 + L.xb),
            {reinterpret_cast<float2*>(w8 + L.stats),
             reinterpret_cast<float2*>(w8 + L.stats) + static_cast<size_t>(M) * m->nt},
            reinterpret_cast<float*>(w8 + L.ctr),
            reinterpret_cast<__nv_bfloat16*>(w8 + L.attn),
            reinterpret_cast<__nv_bfloat16*>(w8 + L.big)};
  int cur = 0;  // S.stats[cur] holds the partial statistics of the current x
  int launches = 0;
  const float* pos = m->pos;
  if (!g.native) {
    float* rp = reinterpret_cast<float*>(w8 + L.pos);
    const long long n = static_cast<long long>(P + (c.pos_on_cls ? 1 : 0)) * D;
    { const int ps_ = prof_open(m, VIT_K_POS_RESIZE, s);
    pos_resize_kernel<<<grid_1d(n, 256, m->nsm), 256, 0, s>>>(m->pos, m->gh, m->gw, g.gh, g.gw, D,
                                                                c.pos_on_cls ? 1 : 0, rp);
    prof_close(m, ps_, s); }
    CKL();
    ++launches;
    pos = rp;
  }

  CUtensorMap tm_pe, tm_xb, tm_attn, tm_h, tm_qkv3, tm_qkv_out, tm_h_out, tm_x_ep, tm_xb_ep;
  if (!tmap_2d(&tm_pe, S.big, m->Kpad, Mp, m->Kpad, 64, GEMM_BM) || !tmap_2d(&tm_xb, S.xb, D, M, D, 64, GEMM_BM) ||
      !tmap_2d(&tm_attn, S.attn, D, M, D, 64, GEMM_BM) || !tmap_2d(&tm_h, S.big, F, M, F, 64, GEMM_BM) ||
      !tmap_qkv3d(&tm_qkv3, S.big, B, T, D) || !tmap_out_bf16(&tm_qkv_out, S.big, 3 * D, M, 3 * D) ||
      !tmap_out_bf16(&tm_h_out, S.big, F, M, F) || !tmap_x_f32(&tm_x_ep, S.x, D, M) ||
      !tmap_xb_bf16(&tm_xb_ep, S.xb, D, M))
    return VIT_E_CUDA;

  // patch embedding: im2col, GEMM with bias + position embedding, token placement
  { const int ps_ = prof_open(m, VIT_K_IM2COL, s);
  {
    // two 16-byte loads per thread when a thread's 8 pixels are one aligned run of an image row
    // (K = 3 p^2 is then a multiple of 8 too, so no thread straddles the end of K)
    const bool vec = c.patch % 8 == 0 && src.img_stride % 4 == 0 && src.chan_stride % 4 == 0 &&
                     src.row_stride % 4 == 0 && src.win_stride % 4 == 0 && src.max_ox % 4 == 0;
    const int grid = grid_1d(static_cast<long long>(Mp) * (m->Kpad / 8), 256, m->nsm);
    if (vec)
      im2col_bf16_kernel<true><<<grid, 256, 0, s>>>(src, B, c.patch, g.gw, P, m->Kpad, S.big);
    else
      im2col_bf16_kernel<false><<<grid, 256, 0, s>>>(src, B, c.patch, g.gw, P, m->Kpad, S.big);
  }
  prof_close(m, ps_, s); }
  CKL();
  ++launches;
  {
    EpiParams ep{};
    ep.wait_ns = m->wait_ns;
    ep.M = Mp;
    ep.N = D;
    ep.bias = m->patch_b;
    ep.x = S.x;
    ep.pos = pos;
    ep.P = P;
    ep.T = T;
    ep.R = R;
    ep.pos_off = c.pos_on_cls ? 1 : 0;
    { const int ps_ = prof_open(m, VIT_K_PATCH_GEMM, s);
    CK(launch_gemm(m->bn_res, EPI_PATCH, tm_pe, m->tm_patch, tm_pe, tm_pe, Mp, D, m->Kpad, ep, m->d_status, s, m->nsm));
    prof_close(m, ps_, s); }
    ++launches;
  }
  { const int ps_ = prof_open(m, VIT_K_PREFIX, s);
  CK(launch_pdl(token_prep_kernel, dim3(static_cast<unsigned>((M + 7) / 8)), dim3(256), 0, s,
                static_cast<const float*>(m->cls), static_cast<const float*>(m->reg), pos, c.pos_on_cls,
                static_cast<long long>(M), T, R, D, m->stats_cols, S.x, S.xb, S.stats[cur], S.ctr));
  prof_close(m, ps_, s); }
  CKL();
  ++launches;

  // One encoder block ([diagram] "Encoder block"): folded LN1 + QKV, attention, proj + layer
  // scale + residual, folded LN2 + FC1 + GELU, FC2 + layer scale + residual.
  auto run_block = [&](const BlockW& bw) -> vit_status {
    // LN1 (folded) + QKV
    {
      const int bn = pick_bn(M, 3 * D, m->nsm);
      EpiParams ep{};
      ep.wait_ns = m->wait_ns;
      ep.M = M;
      ep.N = 3 * D;
      ep.bias = bw.qkv_b;
      ep.colsum = bw.qkv_c;
      ep.stats_in = S.stats[cur];
      ep.ctr = S.ctr;
      ep.nt = m->nt;
      ep.nt_cols = m->stats_cols;
      ep.D = D;
      ep.eps = c.ln_eps;
      ep.ldo = 3 * D;
      { const int ps_ = prof_open(m, VIT_K_QKV_GEMM, s);
      CK(launch_gemm(bn, EPI_LNFOLD, tm_xb, bw.tm_qkv[bn == 256], tm_qkv_out, tm_qkv_out, M, 3 * D, D, ep, m->d_status, s,
                     m->nsm));
      prof_close(m, ps_, s); }
      ++launches;
    }
    { const int ps_ = prof_open(m, VIT_K_ATTENTION, s);
    CK(launch_attention(tm_qkv3, S.big, B, T, c.heads, S.attn, m->d_status, s, m->wait_ns));
    prof_close(m, ps_, s); }
    ++launches;
    // proj + layer scale + residual
    {
      EpiParams ep{};
      ep.wait_ns = m->wait_ns;
      ep.M = M;
      ep.N = D;
      ep.bias = bw.proj_b;
      ep.ls = bw.ls1;
      ep.x = S.x;
      ep.xb = S.xb;
      ep.ctr = S.ctr;
      ep.stats_in = S.stats[cur];
      ep.nt = m->nt;
      ep.nt_cols = m->stats_cols;
      ep.stats_out = S.stats[cur ^ 1];
      ep.stats_cols = m->stats_cols;
      const int bnr = pick_bn_res(M, D, m->bn_res, m->nsm);
      { const int ps_ = prof_open(m, VIT_K_PROJ_GEMM, s);
      CK(launch_gemm(bnr, EPI_RESID, tm_attn, bnr == BN_PAIR ? bw.tm_proj_h : bw.tm_proj, tm_x_ep, tm_xb_ep, M, D, D, ep,
                     m->d_status, s, m->nsm));
      prof_close(m, ps_, s); }
      ++launches;
      cur ^= 1;
    }
    // LN2 (folded) + FC1 + GELU
    {
      const int bn = pick_bn(M, F, m->nsm);
      EpiParams ep{};
      ep.wait_ns = m->wait_ns;
      ep.M = M;
      ep.N = F;
      ep.bias = bw.fc1_b;
      ep.colsum = bw.fc1_c;
      ep.stats_in = S.stats[cur];
      ep.ctr = S.ctr;
      ep.nt = m->nt;
      ep.nt_cols = m->stats_cols;
      ep.D = D;
      ep.eps = c.ln_eps;
      ep.ldo = F;
      ep.gelu = 1;
      { const int ps_ = prof_open(m, VIT_K_FC1_GEMM, s);
      CK(launch_gemm(bn, EPI_LNFOLD, tm_xb, bw.tm_fc1[bn == 256], tm_h_out, tm_h_out, M, F, D, ep, m->d_status, s,
                     m->nsm));
      prof_close(m, ps_, s); }
      ++launches;
    }
    // FC2 + layer scale + residual
    {
      EpiParams ep{};
      ep.wait_ns = m->wait_ns;
      ep.M = M;
      ep.N = D;
      ep.bias = bw.fc2_b;
      ep.ls = bw.ls2;
      ep.x = S.x;
      ep.xb = S.xb;
      ep.ctr = S.ctr;
      ep.stats_in = S.stats[cur];
      ep.nt = m->nt;
      ep.nt_cols = m->stats_cols;
      ep.stats_out = S.stats[cur ^ 1];
      ep.stats_cols = m->stats_cols;
      const int bnr = pick_bn_res(M, D, m->bn_res, m->nsm);
      { const int ps_ = prof_open(m, VIT_K_FC2_GEMM, s);
      // FC2's long K loop hides its epilogue: one x buffer per warp, the freed shared memory a
      // fifth operand stage
      CK(launch_gemm(bnr, EPI_RESID_DEEP, tm_h, bnr == BN_PAIR ? bw.tm_fc2_h : bw.tm_fc2, tm_x_ep, tm_xb_ep, M, D, F,
                     ep, m->d_status, s, m->nsm));
      prof_close(m, ps_, s); }
      ++launches;
      cur ^= 1;
    }
    return VIT_OK;
  };

  int tap_i = 0;
  for (int l = 0; l < c.depth; ++l) {
    const vit_status bst = run_block(m->blocks[l]);
    if (bst != VIT_OK) return bst;
    if (out && out->hidden)
      CK(cudaMemcpyAsync(out->hidden + static_cast<size_t>(l) * M * D, S.x, static_cast<size_t>(M) * D * 4,
                         cudaMemcpyDeviceToDevice, s));
    if (c.tap_mask & (1u << l)) {
      if (tap_rows) {
        // the dense head's input: final-norm tap rows, concatenated in tap order
        { const int ps_ = prof_open(m, VIT_K_TAP, s);
        tap_rows_kernel<<<static_cast<int>((static_cast<long long>(B) * P + 7) / 8), 256, 0, s>>>(
            S.x, m->norm_w, m->norm_b, B, T, R, D, c.ln_eps, tap_rows, 4 * D, tap_i * D);
        prof_close(m, ps_, s); }
        CKL();
        ++launches;
      } else if (out && out->taps[tap_i]) {
        { const int ps_ = prof_open(m, VIT_K_TAP, s);
        CK(launch_pdl(tap_kernel, dim3((P + 31) / 32, B), dim3(256), 0, s, static_cast<const float*>(S.x),
                      static_cast<const float*>(m->norm_w), static_cast<const float*>(m->norm_b), T, R, D, c.ln_eps,
                      out->taps[tap_i]));
        prof_close(m, ps_, s); }
        CKL();
        ++launches;
      }
      ++tap_i;
    }
  }
  if (head && !m->head.empty()) {
    // dino.txt vision head: final norm in place over the whole sequence, the head blocks, then
    // the head's patch rows (fp32) as the patch tokens
    const long long rows = static_cast<long long>(M);
    { const int ps_ = prof_open(m, VIT_K_FINAL_LN, s);
    CK(launch_pdl(final_ln_stream_kernel, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256), 0, s, S.x,
                  static_cast<const float*>(m->norm_w), static_cast<const float*>(m->norm_b), rows, D, c.ln_eps,
                  m->stats_cols, S.xb, S.stats[cur], S.ctr, m->d_status + 1));
    prof_close(m, ps_, s); }
    CKL();
    ++launches;
    for (const BlockW& hb : m->head) {
      const vit_status bst = run_block(hb);
      if (bst != VIT_OK) return bst;
    }
    if (out && out->patch_tokens) {
      { const int ps_ = prof_open(m, VIT_K_HEAD_OUT, s);
      CK(launch_pdl(patch_rows_kernel, dim3(grid_1d(static_cast<long long>(B) * P * (D / 4), 256, m->nsm)), dim3(256), 0,
                    s, static_cast<const float*>(S.x), B, T, R, D, static_cast<float*>(out->patch_tokens)));
      prof_close(m, ps_, s); }
      CKL();
      ++launches;
    }
  } else if (out && (out->desc || out->patch_tokens)) {
    const long long jobs = static_cast<long long>(B) * (1 + P);
    { const int ps_ = prof_open(m, VIT_K_FINAL_LN, s);
    CK(launch_pdl(final_ln_kernel, dim3(static_cast<unsigned>((jobs + 7) / 8)), dim3(256), 0, s,
                  static_cast<const float*>(S.x), static_cast<const float*>(m->norm_w),
                  static_cast<const float*>(m->norm_b), B, T, R, D, c.ln_eps, out->desc, out->patch_tokens,
                  out->patch_fp32, m->d_status + 1));
    prof_close(m, ps_, s); }
    CKL();
    ++launches;
  }
  m->last_launches = launches;
  return VIT_OK;
}

vit_status check_outputs(const vit_outputs* out) {
  if (!out) return VIT_OK;
  if (!aligned16(out->desc) || !aligned16(out->patch_tokens) || !aligned16(out->hidden)) {
    set_err("output pointers must be 16-byte aligned");
    return VIT_E_INVALID_ARG;
  }
  for (int i = 0; i < 4; ++i)
    if (!aligned16(out->taps[i])) {
      set_err("tap pointers must be 16-byte aligned");
      return VIT_E_INVALID_ARG;
    }
  return VIT_OK;
}

}  // namespace

// defined with the allocation-free forward at the end of this file
vit_status noalloc_resolve(int dev);

// ------------------------------------------------------------------ C ABI
extern "C" {

const char* vit_status_str(vit_status s) {
  switch (s) {
    case VIT_OK: return "ok";
    case VIT_E_INVALID_ARG: return "invalid argument";
    case VIT_E_SHAPE: return "shape mismatch";
    case VIT_E_UNSUPPORTED: return "unsupported configuration";
    case VIT_E_WORKSPACE: return "workspace too small";
    case VIT_E_CUDA: return "CUDA error";
    case VIT_E_DEVICE_TIMEOUT: return "device pipeline wait timed out";
    case VIT_E_NONFINITE: return "non-finite value";
  }
  return "unknown status";
}

const char* vit_last_error(void) { return g_err.c_str(); }

vit_status vit_create(const vit_config* cfg, const vit_weights* w, vit_model** out) {
  if (!out) {
    set_err("out is NULL");
    return VIT_E_INVALID_ARG;
  }
  *out = nullptr;
  vit_status st = validate_cfg(cfg);
  if (st != VIT_OK) return st;
  if (!w || !w->patch_w || !w->patch_b || !w->cls || !w->pos || !w->norm_w || !w->norm_b || !w->blocks ||
      (cfg->n_registers > 0 && !w->reg)) {
    set_err("missing weight pointer");
    return VIT_E_INVALID_ARG;
  }
  for (int l = 0; l < cfg->depth; ++l) {
    const vit_block_weights& b = w->blocks[l];
    const void* ptrs[] = {b.ln1_w, b.ln1_b, b.qkv_w, b.qkv_b, b.proj_w, b.proj_b, b.ls1,
                          b.ln2_w, b.ln2_b, b.fc1_w, b.fc1_b, b.fc2_w, b.fc2_b, b.ls2};
    for (const void* p : ptrs)
      if (!p || !aligned16(p)) {
        set_err("block %d: weight pointer NULL or not 16-byte aligned", l);
        return VIT_E_INVALID_ARG;
      }
  }
  vit_model* m = new vit_model();
  m->cfg = *cfg;
  CK(cudaGetDevice(&m->device));
  m->nsm = device_sms(m->device);
  const int D = cfg->dim, F = cfg->mlp_dim, p = cfg->patch;
  m->gh = cfg->img_h / p;
  m->gw = cfg->img_w / p;
  m->P = m->gh * m->gw;
  m->T = 1 + cfg->n_registers + m->P;
  m->K_pe = 3 * p * p;
  m->Kpad = static_cast<int>(align_up(m->K_pe, 64));
  m->bn_res = (D % 256 == 0) ? 256 : 128;
  m->stats_cols = m->bn_res / 2;  // each epilogue thread covers half of a tile's columns
  m->nt = D / m->stats_cols;

  cudaStream_t s;
  auto fail = [&](vit_status e) {
    vit_destroy(m);
    return e;
  };
  if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) {
    set_err("cudaStreamCreate failed");
    return fail(VIT_E_CUDA);
  }
  auto run = [&]() -> vit_status {
    vit_status e;
    if ((e = alloc_dev(m, reinterpret_cast<void**>(&m->d_status), 16)) != VIT_OK) return e;
    CK(cudaMemsetAsync(m->d_status, 0, 16, s));
    if ((e = alloc_dev(m, reinterpret_cast<void**>(&m->patch_w), static_cast<size_t>(D) * m->Kpad * 2)) != VIT_OK)
      return e;
    pad_rows_bf16_kernel<<<grid_1d(static_cast<long long>(D) * m->Kpad, 256, m->nsm), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(w->patch_w), D, m->K_pe, m->Kpad, m->patch_w);
    CKL();
    const size_t npos = static_cast<size_t>(m->P + (cfg->pos_on_cls ? 1 : 0)) * D;
    if ((e = to_f32(m, w->patch_b, D, &m->patch_b, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->pos, npos, &m->pos, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->cls, D, &m->cls, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->reg, static_cast<size_t>(cfg->n_registers) * D, &m->reg, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->norm_w, D, &m->norm_w, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->norm_b, D, &m->norm_b, s)) != VIT_OK) return e;
    if (!tmap_2d(&m->tm_patch, m->patch_w, m->Kpad, D, m->Kpad, 64, m->bn_res)) return VIT_E_CUDA;
    m->blocks.resize(cfg->depth);
    for (int l = 0; l < cfg->depth; ++l) {
      if ((e = build_block(m, w->blocks[l], m->blocks[l], s)) != VIT_OK) return e;
    }
    CK(cudaStreamSynchronize(s));
    // the allocation-free forward's scratch address on this device, looked up now, outside
    // any stream capture a caller might start later
    return noalloc_resolve(m->device);
  };
  st = run();
  cudaStreamDestroy(s);
  if (st != VIT_OK) return fail(st);
  *out = m;
  return VIT_OK;
}

void vit_destroy(vit_model* m) {
  if (!m) return;
  for (cudaEvent_t e : m->prof_ev) cudaEventDestroy(e);
  for (void* p : m->allocs) cudaFree(p);
  delete m;
}

vit_status vit_workspace_size(const vit_model* m, int32_t batch, size_t* bytes) {
  if (!m || !bytes) {
    set_err("NULL argument");
    return VIT_E_INVALID_ARG;
  }
  if (batch < 1 || batch > m->cfg.max_batch) {
    set_err("batch %d outside 1..max_batch (%d)", batch, m->cfg.max_batch);
    return VIT_E_SHAPE;
  }
  *bytes = ws_layout(m, batch, native_geom(m)).total;
  return VIT_OK;
}

vit_status vit_forward(vit_model* m, const float* images, int32_t B, const vit_outputs* out, void* ws, size_t ws_bytes,
                       vit_stream_t stream) {
  if (!m || !images || !aligned16(images)) {
    set_err("model or images NULL / images not 16-byte aligned");
    return VIT_E_INVALID_ARG;
  }
  if (B < 1 || B > m->cfg.max_batch) {
    set_err("batch %d outside 1..max_batch (%d)", B, m->cfg.max_batch);
    return VIT_E_SHAPE;
  }
  vit_status st = check_outputs(out);
  if (st != VIT_OK) return st;
  const vit_config& c = m->cfg;
  ImgSrc src{images, 3LL * c.img_h * c.img_w, static_cast<long long>(c.img_h) * c.img_w, c.img_w, 1, 0, 0, 0};
  return run_forward(m, src, B, native_geom(m), out, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

vit_status vit_workspace_size_hw(const vit_model* m, int32_t batch, int32_t H, int32_t W, size_t* bytes) {
  if (!m || !bytes) {
    set_err("NULL argument");
    return VIT_E_INVALID_ARG;
  }
  if (batch < 1 || batch > m->cfg.max_batch) {
    set_err("batch %d outside 1..max_batch (%d)", batch, m->cfg.max_batch);
    return VIT_E_SHAPE;
  }
  const Geom g = geom_for(m, H, W);
  vit_status st = check_geom(m, batch, g);
  if (st != VIT_OK) return st;
  *bytes = ws_layout(m, batch, g).total;
  return VIT_OK;
}

vit_status vit_forward_hw(vit_model* m, const float* images, int32_t B, int32_t H, int32_t W, const vit_outputs* out,
                          void* ws, size_t ws_bytes, vit_stream_t stream) {
  if (!m || !images || !aligned16(images)) {
    set_err("model or images NULL / images not 16-byte aligned");
    return VIT_E_INVALID_ARG;
  }
  if (B < 1 || B > m->cfg.max_batch) {
    set_err("batch %d outside 1..max_batch (%d)", B, m->cfg.max_batch);
    return VIT_E_SHAPE;
  }
  vit_status st = check_outputs(out);
  if (st != VIT_OK) return st;
  ImgSrc src{images, 3LL * H * W, static_cast<long long>(H) * W, W, 1, 0, 0, 0};
  return run_forward(m, src, B, geom_for(m, H, W), out, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

vit_status vit_set_text_head(vit_model* m, const vit_block_weights* blocks, int32_t n_blocks) {
  if (!m || (n_blocks > 0 && !blocks)) {
    set_err("NULL argument");
    return VIT_E_INVALID_ARG;
  }
  if (n_blocks < 1 || n_blocks > 8) {
    set_err("n_blocks %d outside 1..8", n_blocks);
    return VIT_E_INVALID_ARG;
  }
  if (!m->head.empty()) {
    set_err("a text head is already attached to this model");
    return VIT_E_INVALID_ARG;
  }
  for (int l = 0; l < n_blocks; ++l) {
    const vit_block_weights& b = blocks[l];
    const void* ptrs[] = {b.ln1_w, b.ln1_b, b.qkv_w, b.qkv_b, b.proj_w, b.proj_b, b.ls1,
                          b.ln2_w, b.ln2_b, b.fc1_w, b.fc1_b, b.fc2_w, b.fc2_b, b.ls2};
    for (const void* p : ptrs)
      if (!p || !aligned16(p)) {
        set_err("head block %d: weight pointer NULL or not 16-byte aligned", l);
        return VIT_E_INVALID_ARG;
      }
  }
  int cur = 0;
  CK(cudaGetDevice(&cur));
  if (cur != m->device) {
    set_err("vit_set_text_head called with device %d current; the model lives on device %d", cur, m->device);
    return VIT_E_INVALID_ARG;
  }
  cudaStream_t s;
  CK(cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking));
  std::vector<BlockW> head(n_blocks);
  vit_status st = VIT_OK;
  for (int l = 0; l < n_blocks && st == VIT_OK; ++l) st = build_block(m, blocks[l], head[l], s);
  const cudaError_t se = cudaStreamSynchronize(s);
  cudaStreamDestroy(s);
  if (st != VIT_OK) return st;
  if (se != cudaSuccess) {
    set_err("vit_set_text_head: %s", cudaGetErrorString(se));
    return VIT_E_CUDA;
  }
  m->head = std::move(head);
  return VIT_OK;
}

vit_status vit_forward_text_tokens(vit_model* m, const float* images, int32_t B, int32_t H, int32_t W, float* tokens,
                                   void* ws, size_t ws_bytes, vit_stream_t stream) {
  if (!m || !images || !tokens || !aligned16(images) || !aligned16(tokens)) {
    set_err("model, images or tokens NULL / not 16-byte aligned");
    return VIT_E_INVALID_ARG;
  }
  if (m->head.empty()) {
    set_err("no text head attached (vit_set_text_head)");
    return VIT_E_INVALID_ARG;
  }
  if (B < 1 || B > m->cfg.max_batch) {
    set_err("batch %d outside 1..max_batch (%d)", B, m->cfg.max_batch);
    return VIT_E_SHAPE;
  }
  vit_outputs o{};
  o.patch_tokens = tokens;
  o.patch_fp32 = 1;
  ImgSrc src{images, 3LL * H * W, static_cast<long long>(H) * W, W, 1, 0, 0, 0};
  return run_forward(m, src, B, geom_for(m, H, W), &o, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream),
                     /*head=*/true);
}

// ------------------------------------------------------------------ dense head on the taps
struct DenseLayout {
  size_t enc, xc, t, cc, t2, i3, p4, l, stats, lr, total;
};

static DenseLayout dense_layout(const vit_model* m, int B, const Geom& g) {
  const size_t Mp = static_cast<size_t>(B) * g.P, D4 = 4 * static_cast<size_t>(m->cfg.dim);
  const size_t W = m->dense.W, h = W / 2, K = m->dense.K;
  DenseLayout L;
  L.enc = ws_layout(m, B, g).total;
  size_t off = align_up(L.enc, 1024);
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 1024);
    return at;
  };
  L.xc = take(Mp * D4 * 2);
  L.t = take(Mp * W * 2);
  L.cc = take(Mp * 5 * h * 2);
  L.t2 = take(Mp * h * 2);
  L.i3 = take(Mp * 9 * W * 2);
  L.p4 = take(Mp * W * 2);
  L.l = take(Mp * W * 2);
  L.stats = take(static_cast<size_t>(B) * 32 * 8);
  L.lr = take(static_cast<size_t>(B) * K * g.P * 4);
  L.total = off;
  return L;
}

static vit_status run_dense(vit_model* m, const float* images, int B, const Geom& g, float* logits, float* p4out,
                            void* ws, size_t ws_bytes, cudaStream_t s) {
  const vit_config& c = m->cfg;
  const auto& dw = m->dense;
  vit_status st = check_geom(m, B, g);
  if (st != VIT_OK) return st;
  const DenseLayout DL = dense_layout(m, B, g);
  if (!ws || ws_bytes < DL.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) {
    set_err("dense workspace must be >= %zu bytes and 256-byte aligned", DL.total);
    return VIT_E_WORKSPACE;
  }
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(w8 + off); };
  __nv_bfloat16 *Xc = bf(DL.xc), *Tt = bf(DL.t), *Cc = bf(DL.cc), *T2 = bf(DL.t2), *I3 = bf(DL.i3), *P4 = bf(DL.p4),
                *Lb = bf(DL.l);
  float2* gstats = reinterpret_cast<float2*>(w8 + DL.stats);
  float* lr = reinterpret_cast<float*>(w8 + DL.lr);
  const int D4 = 4 * c.dim, W = dw.W, h = W / 2, K = dw.K, P = g.P;
  const long long Mp = static_cast<long long>(B) * P;

  ImgSrc src{images, 3LL * g.H * g.W, static_cast<long long>(g.H) * g.W, g.W, 1, 0, 0, 0};
  vit_outputs none{};
  st = run_forward(m, src, B, g, &none, ws, DL.enc, s, false, Xc);
  if (st != VIT_OK) return st;
  int launches = m->last_launches;

  auto gemm = [&](const __nv_bfloat16* A, int lda, int Kd, const __nv_bfloat16* Wt, int N, const float* bias,
                  __nv_bfloat16* out) -> vit_status {
    const int bn = pick_bn(static_cast<int>(Mp), N, m->nsm);
    CUtensorMap ta, tb, to;
    if (!tmap_2d(&ta, A, Kd, Mp, lda, 64, GEMM_BM) || !tmap_2d(&tb, Wt, Kd, N, Kd, 64, bn == BN_PAIR ? 128 : bn) ||
        !tmap_out_bf16(&to, out, N, Mp, N))
      return VIT_E_CUDA;
    EpiParams ep{};
    ep.wait_ns = m->wait_ns;
    ep.M = static_cast<int>(Mp);
    ep.N = N;
    ep.bias = bias;
    ep.ldo = N;
    { const int ps_ = prof_open(m, VIT_K_DENSE_GEMM, s);
    CK(launch_gemm(bn, EPI_BIAS, ta, tb, to, to, static_cast<int>(Mp), N, Kd, ep, m->d_status, s, m->nsm));
    prof_close(m, ps_, s); }
    ++launches;
    return VIT_OK;
  };
  const int rows_grid = static_cast<int>((Mp + 7) / 8);
  auto ln_silu = [&](const __nv_bfloat16* in, int C, const float* lg, const float* lb, const float* lg2,
                     const float* lb2, int mode, __nv_bfloat16* out, int ld_out, int col0) -> vit_status {
    { const int ps_ = prof_open(m, VIT_K_DENSE_AUX, s);
    row_ln_silu_kernel<<<rows_grid, 256, 0, s>>>(in, C, Mp, C, lg, lb, lg2, lb2, 1e-6f, mode, out, ld_out, col0);
    prof_close(m, ps_, s); }
    CKL();
    ++launches;
    return VIT_OK;
  };
  auto im2col = [&](const __nv_bfloat16* in, int ld_in, int col0, int C) -> vit_status {
    { const int ps_ = prof_open(m, VIT_K_DENSE_AUX, s);
    im2col3x3_kernel<<<grid_1d(Mp * 9 * (C / 8), 256, m->nsm), 256, 0, s>>>(in, ld_in, col0, C, B, g.gh, g.gw, I3);
    prof_close(m, ps_, s); }
    CKL();
    ++launches;
    return VIT_OK;
  };
#define DENSE_STEP(x)            \
  do {                           \
    const vit_status e_ = (x);   \
    if (e_ != VIT_OK) return e_; \
  } while (0)
  // projector P4
  DENSE_STEP(gemm(Xc, D4, D4, dw.cv1_w, W, dw.zero, Tt));
  DENSE_STEP(ln_silu(Tt, W, dw.cv1_ln_w, dw.cv1_ln_b, nullptr, nullptr, 0, Cc, 5 * h, 0));
  for (int i = 0; i < 3; ++i) {
    const int in_col = (i == 0) ? h : 2 * h + (i - 1) * h;
    DENSE_STEP(im2col(Cc, 5 * h, in_col, h));
    DENSE_STEP(gemm(I3, 9 * h, 9 * h, dw.bn_wr[2 * i], h, dw.zero, Tt));
    DENSE_STEP(ln_silu(Tt, h, dw.bn_ln_w[2 * i], dw.bn_ln_b[2 * i], nullptr, nullptr, 0, T2, h, 0));
    DENSE_STEP(im2col(T2, h, 0, h));
    DENSE_STEP(gemm(I3, 9 * h, 9 * h, dw.bn_wr[2 * i + 1], h, dw.zero, Tt));
    DENSE_STEP(ln_silu(Tt, h, dw.bn_ln_w[2 * i + 1], dw.bn_ln_b[2 * i + 1], nullptr, nullptr, 0, Cc, 5 * h,
                       2 * h + i * h));
  }
  DENSE_STEP(gemm(Cc, 5 * h, 5 * h, dw.cv2_w, W, dw.zero, Tt));
  DENSE_STEP(ln_silu(Tt, W, dw.cv2_ln_w, dw.cv2_ln_b, dw.out_ln_w, dw.out_ln_b, 1, P4, W, 0));
  if (p4out) {
    { const int ps_ = prof_open(m, VIT_K_DENSE_AUX, s);
    rows_to_chw_kernel<<<grid_1d(Mp * W, 256, m->nsm), 256, 0, s>>>(P4, B, P, W, p4out);
    prof_close(m, ps_, s); }
    CKL();
    ++launches;
  }
  // task head
  DENSE_STEP(gemm(P4, W, W, dw.lat_w, W, dw.lat_b, Lb));
  DENSE_STEP(im2col(Lb, W, 0, W));
  DENSE_STEP(gemm(I3, 9 * W, 9 * W, dw.smooth_wr, W, dw.smooth_b, Tt));
#undef DENSE_STEP
  { const int ps_ = prof_open(m, VIT_K_DENSE_AUX, s);
  group_norm_stats_kernel<<<dim3(32, B), 256, 0, s>>>(Tt, P, W, 32, gstats);
  prof_close(m, ps_, s); }
  CKL();
  { const int ps_ = prof_open(m, VIT_K_DENSE_AUX, s);
  group_norm_gelu_kernel<<<grid_1d(Mp * W / 2, 256, m->nsm), 256, 0, s>>>(Tt, Mp, P, W, 32, gstats, dw.gn_w, dw.gn_b,
                                                                         1e-5f, Lb);
  prof_close(m, ps_, s); }
  CKL();
  { const int ps_ = prof_open(m, VIT_K_DENSE_AUX, s);
  predict_kernel<<<rows_grid, 256, 0, s>>>(Lb, Mp, P, W, dw.pred_w, dw.pred_b, K, lr);
  prof_close(m, ps_, s); }
  CKL();
  { const int ps_ = prof_open(m, VIT_K_DENSE_AUX, s);
  resize_logits_kernel<<<grid_1d(static_cast<long long>(B) * g.H * g.W, 256, m->nsm), 256, 0, s>>>(
      lr, B, K, g.gh, g.gw, g.H, g.W, logits);
  prof_close(m, ps_, s); }
  CKL();
  launches += 4;
  m->last_launches = launches;
  return VIT_OK;
}

vit_status vit_set_dense_head(vit_model* m, const vit_dense_head_weights* w) {
  if (!m || !w) {
    set_err("NULL argument");
    return VIT_E_INVALID_ARG;
  }
  if (m->dense.on) {
    set_err("a dense head is already attached to this model");
    return VIT_E_INVALID_ARG;
  }
  if (__builtin_popcount(m->cfg.tap_mask) != 4) {
    set_err("the dense head needs exactly four taps (tap_mask has %d)", __builtin_popcount(m->cfg.tap_mask));
    return VIT_E_UNSUPPORTED;
  }
  if (w->width != 256 || w->n_classes < 1 || w->n_classes > 1024) {
    set_err("dense head: width must be 256 and n_classes 1..1024 (got %d, %d)", w->width, w->n_classes);
    return VIT_E_UNSUPPORTED;
  }
  const void* ptrs[] = {w->cv1_w, w->cv1_ln_w, w->cv1_ln_b, w->cv2_w, w->cv2_ln_w, w->cv2_ln_b, w->out_ln_w,
                        w->out_ln_b, w->lat_w, w->lat_b, w->smooth_w, w->smooth_b, w->gn_w, w->gn_b, w->pred_w,
                        w->pred_b};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) {
      set_err("dense head: weight pointer NULL or not 16-byte aligned");
      return VIT_E_INVALID_ARG;
    }
  for (int i = 0; i < 6; ++i)
    if (!w->bn_w[i] || !w->bn_ln_w[i] || !w->bn_ln_b[i] || !aligned16(w->bn_w[i])) {
      set_err("dense head: bottleneck %d weight pointer NULL or not 16-byte aligned", i);
      return VIT_E_INVALID_ARG;
    }
  int cur = 0;
  CK(cudaGetDevice(&cur));
  if (cur != m->device) {
    set_err("vit_set_dense_head called with device %d current; the model lives on device %d", cur, m->device);
    return VIT_E_INVALID_ARG;
  }
  const int W = w->width, h = W / 2, K = w->n_classes;
  auto& d = m->dense;
  cudaStream_t s;
  CK(cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking));
  auto run = [&]() -> vit_status {
    vit_status e;
    for (int i = 0; i < 6; ++i) {
      if ((e = alloc_dev(m, reinterpret_cast<void**>(&d.bn_wr[i]), static_cast<size_t>(h) * 9 * h * 2)) != VIT_OK)
        return e;
      conv3x3_weight_kernel<<<grid_1d(static_cast<long long>(h) * 9 * h, 256, m->nsm), 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(w->bn_w[i]), h, h, d.bn_wr[i]);
      CKL();
      if ((e = to_f32(m, w->bn_ln_w[i], h, &d.bn_ln_w[i], s)) != VIT_OK) return e;
      if ((e = to_f32(m, w->bn_ln_b[i], h, &d.bn_ln_b[i], s)) != VIT_OK) return e;
    }
    if ((e = alloc_dev(m, reinterpret_cast<void**>(&d.smooth_wr), static_cast<size_t>(W) * 9 * W * 2)) != VIT_OK)
      return e;
    conv3x3_weight_kernel<<<grid_1d(static_cast<long long>(W) * 9 * W, 256, m->nsm), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(w->smooth_w), W, W, d.smooth_wr);
    CKL();
    if ((e = to_f32(m, w->cv1_ln_w, W, &d.cv1_ln_w, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->cv1_ln_b, W, &d.cv1_ln_b, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->cv2_ln_w, W, &d.cv2_ln_w, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->cv2_ln_b, W, &d.cv2_ln_b, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->out_ln_w, W, &d.out_ln_w, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->out_ln_b, W, &d.out_ln_b, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->lat_b, W, &d.lat_b, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->smooth_b, W, &d.smooth_b, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->gn_w, W, &d.gn_w, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->gn_b, W, &d.gn_b, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->pred_w, static_cast<size_t>(K) * W, &d.pred_w, s)) != VIT_OK) return e;
    if ((e = to_f32(m, w->pred_b, K, &d.pred_b, s)) != VIT_OK) return e;
    if ((e = alloc_dev(m, reinterpret_cast<void**>(&d.zero), static_cast<size_t>(W) * 4)) != VIT_OK) return e;
    CK(cudaMemsetAsync(d.zero, 0, static_cast<size_t>(W) * 4, s));
    CK(cudaStreamSynchronize(s));
    return VIT_OK;
  };
  const vit_status st = run();
  cudaStreamDestroy(s);
  if (st != VIT_OK) return st;
  d.cv1_w = static_cast<const __nv_bfloat16*>(w->cv1_w);
  d.cv2_w = static_cast<const __nv_bfloat16*>(w->cv2_w);
  d.lat_w = static_cast<const __nv_bfloat16*>(w->lat_w);
  d.K = K;
  d.W = W;
  d.on = true;
  return VIT_OK;
}

vit_status vit_dense_workspace_size(const vit_model* m, int32_t B, int32_t H, int32_t W, size_t* bytes) {
  if (!m || !bytes) {
    set_err("NULL argument");
    return VIT_E_INVALID_ARG;
  }
  if (!m->dense.on) {
    set_err("no dense head attached (vit_set_dense_head)");
    return VIT_E_INVALID_ARG;
  }
  if (B < 1 || B > m->cfg.max_batch) {
    set_err("batch %d outside 1..max_batch (%d)", B, m->cfg.max_batch);
    return VIT_E_SHAPE;
  }
  const Geom g = geom_for(m, H, W);
  vit_status st = check_geom(m, B, g);
  if (st != VIT_OK) return st;
  *bytes = dense_layout(m, B, g).total;
  return VIT_OK;
}

vit_status vit_forward_dense(vit_model* m, const float* images, int32_t B, int32_t H, int32_t W, float* logits,
                             float* p4, void* ws, size_t ws_bytes, vit_stream_t stream) {
  if (!m || !images || !logits || !aligned16(images) || !aligned16(logits) || !aligned16(p4)) {
    set_err("model, images or logits NULL / a pointer not 16-byte aligned");
    return VIT_E_INVALID_ARG;
  }
  if (!m->dense.on) {
    set_err("no dense head attached (vit_set_dense_head)");
    return VIT_E_INVALID_ARG;
  }
  if (B < 1 || B > m->cfg.max_batch) {
    set_err("batch %d outside 1..max_batch (%d)", B, m->cfg.max_batch);
    return VIT_E_SHAPE;
  }
  return run_dense(m, images, B, geom_for(m, H, W), logits, p4, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

vit_status vit_host_workspace_size(const vit_model* m, int32_t batch, size_t* bytes) {
  size_t fw = 0;
  vit_status st = vit_workspace_size(m, batch, &fw);
  if (st != VIT_OK) return st;
  const size_t img = align_up(static_cast<size_t>(batch) * 3 * m->cfg.img_h * m->cfg.img_w * 4, 1024);
  const size_t desc = align_up(static_cast<size_t>(batch) * m->cfg.dim * 4, 1024);
  const size_t patch = align_up(static_cast<size_t>(batch) * m->P * m->cfg.dim * 2, 1024);
  *bytes = img + desc + patch + fw;
  return VIT_OK;
}

vit_status vit_forward_host(vit_model* m, const float* images_host, int32_t B, float* desc_host,
                            void* patch_tokens_host, void* ws, size_t ws_bytes, vit_stream_t stream) {
  if (!m || !images_host || !desc_host) {
    set_err("model, images_host or desc_host is NULL");
    return VIT_E_INVALID_ARG;
  }
  size_t need = 0;
  vit_status st = vit_host_workspace_size(m, B, &need);
  if (st != VIT_OK) return st;
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) {
    set_err("host-path workspace must be >= %zu bytes and 256-byte aligned", need);
    return VIT_E_WORKSPACE;
  }
  st = check_device(m, "vit_forward_host");
  if (st != VIT_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t img_b = static_cast<size_t>(B) * 3 * m->cfg.img_h * m->cfg.img_w * 4;
  const size_t img = align_up(img_b, 1024);
  const size_t desc_b = static_cast<size_t>(B) * m->cfg.dim * 4;
  const size_t desc = align_up(desc_b, 1024);
  const size_t patch_b = static_cast<size_t>(B) * m->P * m->cfg.dim * 2;
  const size_t patch = align_up(patch_b, 1024);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  float* d_img = reinterpret_cast<float*>(w8);
  float* d_desc = reinterpret_cast<float*>(w8 + img);
  void* d_patch = w8 + img + desc;
  CK(cudaMemcpyAsync(d_img, images_host, img_b, cudaMemcpyHostToDevice, s));
  vit_outputs o{};
  o.desc = d_desc;
  o.patch_tokens = patch_tokens_host ? d_patch : nullptr;
  o.patch_fp32 = 0;
  st = vit_forward(m, d_img, B, &o, w8 + img + desc + patch, ws_bytes - (img + desc + patch), stream);
  if (st != VIT_OK) return st;
  CK(cudaMemcpyAsync(desc_host, d_desc, desc_b, cudaMemcpyDeviceToHost, s));
  if (patch_tokens_host) CK(cudaMemcpyAsync(patch_tokens_host, d_patch, patch_b, cudaMemcpyDeviceToHost, s));
  return VIT_OK;
}

static int slide_count(int size, int side, int stride) {
  if (size <= side) return 1;
  return (size - side + stride - 1) / stride + 1;
}

// The view the encoder sees in each zero-shot mode: the whole image, or ny x nx windows of
// side x side (origins clamped so the last window ends on the border).
struct SegPlan {
  Geom g;
  int ny, nx;
};

static vit_status seg_plan(const vit_model* m, int32_t H, int32_t W, int32_t C, int32_t mode, int32_t side, int32_t stride,
                    SegPlan* p) {
  if (C < 1) {
    set_err("C (%d) must be >= 1", C);
    return VIT_E_INVALID_ARG;
  }
  if (mode == VIT_SEG_SLIDE) {
    if (stride < 1 || side < m->cfg.patch) {
      set_err("slide: stride must be >= 1 and side >= the patch size %d", m->cfg.patch);
      return VIT_E_INVALID_ARG;
    }
    if (H < side || W < side) {
      set_err("slide: window side %d must fit in the image %dx%d", side, H, W);
      return VIT_E_SHAPE;
    }
    p->ny = slide_count(H, side, stride);
    p->nx = slide_count(W, side, stride);
    p->g = geom_for(m, side, side);
  } else if (mode == VIT_SEG_WHOLE) {
    p->ny = p->nx = 1;
    p->g = geom_for(m, H, W);
  } else {
    set_err("mode must be VIT_SEG_WHOLE or VIT_SEG_SLIDE");
    return VIT_E_INVALID_ARG;
  }
  const int nwin = p->ny * p->nx;
  if (nwin > m->cfg.max_batch) {
    set_err("%d windows exceed max_batch (%d)", nwin, m->cfg.max_batch);
    return VIT_E_SHAPE;
  }
  return check_geom(m, nwin, p->g);
}

// Classes padded to the GEMM's column tile for the cosine map.
static int seg_cpad(int C) { return (C + 127) / 128 * 128; }

// Scoring scratch ahead of the encoder's workspace: fp32 tokens [rows, D], the split operands
// A3 [rows, 3D] and B3 [Cpad, 3D] (bf16) and the cosine map [windows, C, P] (fp32).
static size_t seg_head_bytes(const vit_model* m, const SegPlan& p, int C) {
  const size_t rows = static_cast<size_t>(p.ny) * p.nx * p.g.P;
  const size_t D = m->cfg.dim;
  return align_up(rows * D * 4, 1024) + align_up(rows * 3 * D * 2, 1024) +
         align_up(static_cast<size_t>(seg_cpad(C)) * 3 * D * 2, 1024) + align_up(rows * C * 4, 1024);
}

vit_status vit_seg_workspace_size(const vit_model* m, int32_t H, int32_t W, int32_t C, int32_t mode, int32_t side,
                                  int32_t stride, size_t* bytes) {
  if (!m || !bytes) {
    set_err("NULL argument");
    return VIT_E_INVALID_ARG;
  }
  SegPlan p;
  vit_status st = seg_plan(m, H, W, C, mode, side, stride, &p);
  if (st != VIT_OK) return st;
  *bytes = seg_head_bytes(m, p, C) + ws_layout(m, p.ny * p.nx, p.g).total;
  return VIT_OK;
}

vit_status vit_seg_zero_shot(vit_model* m, const float* image, int32_t H, int32_t W, const float* text, int32_t C,
                             int32_t mode, int32_t side, int32_t stride, float* probs, int32_t* labels, void* ws,
                             size_t ws_bytes, vit_stream_t stream) {
  if (!m || !image || !text || !aligned16(image) || !aligned16(text) || !aligned16(probs) || !aligned16(labels)) {
    set_err("NULL or misaligned pointer");
    return VIT_E_INVALID_ARG;
  }
  const vit_config& c = m->cfg;
  SegPlan plan;
  vit_status st = seg_plan(m, H, W, C, mode, side, stride, &plan);
  if (st != VIT_OK) return st;
  const size_t head = seg_head_bytes(m, plan, C);
  const size_t need = head + ws_layout(m, plan.ny * plan.nx, plan.g).total;
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) {
    set_err("seg workspace must be >= %zu bytes and 256-byte aligned", need);
    return VIT_E_WORKSPACE;
  }
  const int ny = plan.ny, nx = plan.nx, nwin = ny * nx, P = plan.g.P;
  const size_t rows = static_cast<size_t>(nwin) * P;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int D = c.dim, Cpad = seg_cpad(C);
  float* tok = reinterpret_cast<float*>(w8);
  size_t off = align_up(rows * D * 4, 1024);
  __nv_bfloat16* a3 = reinterpret_cast<__nv_bfloat16*>(w8 + off);
  off += align_up(rows * 3 * D * 2, 1024);
  __nv_bfloat16* b3 = reinterpret_cast<__nv_bfloat16*>(w8 + off);
  off += align_up(static_cast<size_t>(Cpad) * 3 * D * 2, 1024);
  float* cosm = reinterpret_cast<float*>(w8 + off);
  off += align_up(rows * C * 4, 1024);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  ImgSrc src{image, 0, static_cast<long long>(H) * W, W, nx, (mode == VIT_SEG_SLIDE) ? stride : 0,
             (mode == VIT_SEG_SLIDE) ? H - side : 0, (mode == VIT_SEG_SLIDE) ? W - side : 0};
  vit_outputs o{};
  o.patch_tokens = tok;
  o.patch_fp32 = 1;
  st = run_forward(m, src, nwin, plan.g, &o, w8 + off, ws_bytes - off, s, /*head=*/true);
  if (st != VIT_OK) return st;
  int launches = m->last_launches;
  // the cosine map on the tensor cores: split operands, then A3 . B3^T scattered to [w, c, p]
  { const int ps_ = prof_open(m, VIT_K_SEG_NORM, s);
  cos_split_tokens_kernel<<<static_cast<int>((rows + 7) / 8), 256, 0, s>>>(tok, static_cast<long long>(rows), D, a3);
  cos_split_text_kernel<<<(Cpad + 7) / 8, 256, 0, s>>>(text, C, Cpad, D, b3);
  prof_close(m, ps_, s); }
  CKL();
  {
    CUtensorMap ta, tb;
    if (!tmap_2d(&ta, a3, 3 * D, rows, 3 * D, 64, GEMM_BM) || !tmap_2d(&tb, b3, 3 * D, Cpad, 3 * D, 64, 128))
      return VIT_E_CUDA;
    EpiParams ep{};
    ep.wait_ns = m->wait_ns;
    ep.M = static_cast<int>(rows);
    ep.N = Cpad;
    ep.P = P;
    ep.cos = cosm;
    ep.ncls = C;
    { const int ps_ = prof_open(m, VIT_K_SEG_COS, s);
    CK(launch_gemm(128, EPI_COS, ta, tb, ta, ta, static_cast<int>(rows), Cpad, 3 * D, ep, m->d_status, s, m->nsm));
    prof_close(m, ps_, s); }
  }
  launches += 3;
  const long long pix = static_cast<long long>(H) * W;
  if (mode == VIT_SEG_SLIDE) {
    // the tiled kernel when every 16 x 16 tile meets at most SLIDE_TILE_WIN windows, the classes fit
    // its shared memory and a grid cell spans at least 8 pixels (a tile then needs <= 4 x 4 cells)
    auto tile_windows = [&](int size, int n) {
      int mx = 0;
      for (int t0 = 0; t0 < size; t0 += SLIDE_TILE) {
        const int t1 = std::min(size, t0 + SLIDE_TILE) - 1;
        int cnt = 0;
        for (int i = 0; i < n; ++i) {
          const int o = std::min(i * stride, size - side);
          if (o <= t1 && o + side > t0) ++cnt;
        }
        mx = std::max(mx, cnt);
      }
      return mx;
    };
    const int g = plan.g.gh;
    const bool tiled = C <= SLIDE_TILE_C && g * 8 <= side && tile_windows(H, ny) * tile_windows(W, nx) <= SLIDE_TILE_WIN;
    { const int ps_ = prof_open(m, VIT_K_SEG_MAP, s);
    if (tiled) {
      static std::atomic<uint64_t> attr_done{0};
      CK(set_smem_attr_once(seg_slide_tile_kernel, SLIDE_TILE_SMEM, attr_done));
      const dim3 grid((W + SLIDE_TILE - 1) / SLIDE_TILE, (H + SLIDE_TILE - 1) / SLIDE_TILE);
      seg_slide_tile_kernel<<<grid, SLIDE_TILE * SLIDE_TILE, SLIDE_TILE_SMEM, s>>>(cosm, C, g, H, W, side, stride, ny,
                                                                                    nx, probs, labels);
    } else {
      seg_slide_kernel<<<static_cast<int>((pix + 127) / 128), 128, 0, s>>>(cosm, C, g, H, W, side, stride, ny, nx,
                                                                           probs, labels);
    }
    prof_close(m, ps_, s); }
  } else {
    { const int ps_ = prof_open(m, VIT_K_SEG_MAP, s);
    seg_whole_kernel<<<static_cast<int>((pix + 127) / 128), 128, 0, s>>>(cosm, C, plan.g.gh, plan.g.gw, H, W, probs,
                                                                         labels);
    prof_close(m, ps_, s); }
  }
  CKL();
  m->last_launches = launches + 1;
  return VIT_OK;
}

vit_status vit_poll(vit_model* m, vit_stream_t stream) {
  if (!m) {
    set_err("model is NULL");
    return VIT_E_INVALID_ARG;
  }
  CK(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  int v[2] = {0, 0};
  CK(cudaMemcpy(v, m->d_status, 8, cudaMemcpyDeviceToHost));
  if (v[0] != 0 || v[1] != 0) CK(cudaMemset(m->d_status, 0, 8));
  if (v[0] != 0) {
    set_err("a kernel gave up on a pipeline wait (site 0x%x)", v[0]);
    return VIT_E_DEVICE_TIMEOUT;
  }
  if (v[1] != 0) {
    set_err("a non-finite value reached the final LayerNorm");
    return VIT_E_NONFINITE;
  }
  return VIT_OK;
}

vit_status vit_set_wait_limit(vit_model* m, uint64_t ns) {
  if (!m) {
    set_err("model is NULL");
    return VIT_E_INVALID_ARG;
  }
  m->wait_ns = ns;
  return VIT_OK;
}

int32_t vit_last_launch_count(const vit_model* m) { return m ? m->last_launches : 0; }

vit_status vit_profile_begin(vit_model* m, int32_t capacity) {
  if (!m || capacity < 1) {
    set_err("model is NULL or capacity < 1");
    return VIT_E_INVALID_ARG;
  }
  const size_t need = static_cast<size_t>(capacity) * 2;
  while (m->prof_ev.size() < need) {
    cudaEvent_t e;
    CK(cudaEventCreate(&e));
    m->prof_ev.push_back(e);
  }
  m->prof_kind.assign(capacity, -1);
  m->prof_used = 0;
  m->prof_on = true;
  return VIT_OK;
}

vit_status vit_profile_end(vit_model* m, float* total_ms, int32_t* launches) {
  if (!m) {
    set_err("model is NULL");
    return VIT_E_INVALID_ARG;
  }
  float acc[VIT_K_COUNT] = {};
  int32_t cnt[VIT_K_COUNT] = {};
  for (int i = 0; i < m->prof_used; ++i) {
    CK(cudaEventSynchronize(m->prof_ev[2 * i + 1]));
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, m->prof_ev[2 * i], m->prof_ev[2 * i + 1]));
    const int k = m->prof_kind[i];
    if (k >= 0 && k < VIT_K_COUNT) {
      acc[k] += ms;
      cnt[k] += 1;
    }
  }
  m->prof_on = false;
  m->prof_used = 0;
  if (total_ms) std::memcpy(total_ms, acc, sizeof(acc));
  if (launches) std::memcpy(launches, cnt, sizeof(cnt));
  return VIT_OK;
}

// ------------------------------------------------------------------ stage entry points
vit_status vit_stage_linear_bounded(const void* A, const void* W, const float* bias, int32_t M, int32_t N, int32_t K,
                                    int32_t gelu, void* out, int32_t* status, uint64_t wait_ns,
                                    vit_stream_t stream) {
  if (!A || !W || !bias || !out || !status || !aligned16(A) || !aligned16(W) || !aligned16(bias) || !aligned16(out)) {
    set_err("NULL or misaligned pointer");
    return VIT_E_INVALID_ARG;
  }
  if (M < 1 || N < 128 || N % 128 || K < 64 || K % 64) {
    set_err("need M >= 1, N multiple of 128, K multiple of 64 (got %d, %d, %d)", M, N, K);
    return VIT_E_SHAPE;
  }
  int dev = 0;
  CK(cudaGetDevice(&dev));
  const int nsm = device_sms(dev);
  const int bn = pick_bn(M, N, nsm);
  CUtensorMap ta, tb, to;
  if (!tmap_2d(&ta, A, K, M, K, 64, GEMM_BM) || !tmap_2d(&tb, W, K, N, K, 64, bn == BN_PAIR ? 128 : bn) ||
      !tmap_out_bf16(&to, out, N, M, N))
    return VIT_E_CUDA;
  EpiParams ep{};
  ep.M = M;
  ep.N = N;
  ep.bias = bias;
  ep.gelu = gelu;
  ep.ldo = N;
  ep.wait_ns = wait_ns;
  CK(launch_gemm(bn, EPI_BIAS, ta, tb, to, to, M, N, K, ep, status, reinterpret_cast<cudaStream_t>(stream), nsm));
  return VIT_OK;
}

vit_status vit_stage_linear(const void* A, const void* W, const float* bias, int32_t M, int32_t N, int32_t K,
                            int32_t gelu, void* out, int32_t* status, vit_stream_t stream) {
  return vit_stage_linear_bounded(A, W, bias, M, N, K, gelu, out, status, 0, stream);
}

vit_status vit_stage_attention_bounded(const void* qkv, int32_t B, int32_t T, int32_t heads, void* out,
                                       int32_t* status, uint64_t wait_ns, vit_stream_t stream) {
  if (!qkv || !out || !status || !aligned16(qkv) || !aligned16(out)) {
    set_err("NULL or misaligned pointer");
    return VIT_E_INVALID_ARG;
  }
  if (B < 1 || T < 1 || heads < 1) {
    set_err("need B, T, heads >= 1");
    return VIT_E_SHAPE;
  }
  CUtensorMap tm;
  if (!tmap_qkv3d(&tm, qkv, B, T, heads * 64)) return VIT_E_CUDA;
  CK(launch_attention(tm, static_cast<const __nv_bfloat16*>(qkv), B, T, heads, static_cast<__nv_bfloat16*>(out), status,
                      reinterpret_cast<cudaStream_t>(stream), wait_ns));
  return VIT_OK;
}

vit_status vit_stage_attention(const void* qkv, int32_t B, int32_t T, int32_t heads, void* out, int32_t* status,
                               vit_stream_t stream) {
  return vit_stage_attention_bounded(qkv, B, T, heads, out, status, 0, stream);
}

vit_status vit_stage_gelu(const float* x, int64_t n, float* y, vit_stream_t stream) {
  if (!x || !y || n < 0) {
    set_err("NULL pointer or negative n");
    return VIT_E_INVALID_ARG;
  }
  if (n == 0) return VIT_OK;
  int dev = 0;
  CK(cudaGetDevice(&dev));
  gelu_stage_kernel<<<grid_1d((n + 1) / 2, 256, device_sms(dev)), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x, static_cast<long long>(n), y);
  CKL();
  return VIT_OK;
}

vit_status vit_stage_pos_resize(const float* pos, int32_t gh0, int32_t gw0, int32_t gh, int32_t gw, int32_t D,
                                int32_t pos_on_cls, float* out, vit_stream_t stream) {
  if (!pos || !out) {
    set_err("NULL pointer");
    return VIT_E_INVALID_ARG;
  }
  if (gh0 < 1 || gw0 < 1 || gh < 1 || gw < 1 || D < 1 || gh > 4096 || gw > 4096 || gh0 > 4096 || gw0 > 4096) {
    set_err("grids must be 1..4096 per side and D >= 1");
    return VIT_E_SHAPE;
  }
  int dev = 0, nsm = 1;
  CK(cudaGetDevice(&dev));
  CK(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
  const long long n = static_cast<long long>(gh * gw + (pos_on_cls ? 1 : 0)) * D;
  pos_resize_kernel<<<grid_1d(n, 256, nsm), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      pos, gh0, gw0, gh, gw, D, pos_on_cls ? 1 : 0, out);
  CKL();
  return VIT_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ allocation-free forward
// Some callers may not allocate device memory at all once they are running: hosts that hand a
// plug-in a fixed memory budget and own every allocation themselves, or latency-critical
// loops where an allocation could block or synchronise the device.  For them
// vit_forward_noalloc runs the same forward as vit_forward with its workspace taken from the
// fixed array below instead of from the caller.  The array is part of the library's device
// image, so every GPU on which the library is loaded holds it until the process exits.
static constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(64) << 20;  // 64 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of g_noalloc_scratch, resolved once per device (the host-side symbol is only
// a stand-in and must never be handed to a kernel).
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};
}  // namespace

// Looks up the array's device address on the current device `dev` and caches it.  vit_create
// calls this on the model's device, so a vit_forward_noalloc call (which requires that device to
// be current) finds the address cached and never does the lookup itself, even under capture.
vit_status noalloc_resolve(int dev) {
  if (dev < 0 || dev >= 64) {
    set_err("device index %d out of range for the fixed scratch table", dev);
    return VIT_E_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    CK(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    g_noalloc_ptr[dev] = p;
  }
  return VIT_OK;
}

namespace {
// The cached address for the model's device.  Should it be missing (it cannot be after
// vit_create), the lookup is refused while `s` is being captured into a graph, where a symbol
// lookup (and the module load it may trigger) is not allowed.
vit_status noalloc_scratch(const vit_model* m, cudaStream_t s, void** ptr) {
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (m->device >= 0 && m->device < 64 && g_noalloc_ptr[m->device] != nullptr) {
      *ptr = g_noalloc_ptr[m->device];
      return VIT_OK;
    }
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  CK(cudaStreamIsCapturing(s, &cs));
  if (cs != cudaStreamCaptureStatusNone) {
    set_err("vit_forward_noalloc: the fixed scratch of device %d is not resolved yet and the stream is being "
            "captured; make one call outside the capture first",
            m->device);
    return VIT_E_INVALID_ARG;
  }
  const vit_status st = noalloc_resolve(m->device);
  if (st != VIT_OK) return st;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  *ptr = g_noalloc_ptr[m->device];
  return VIT_OK;
}
}  // namespace

extern "C" vit_status vit_forward_noalloc(vit_model* m, const float* images, int32_t B, const vit_outputs* out,
                                          vit_stream_t stream) {
  if (!m || !images || !aligned16(images)) {
    set_err("model or images NULL / images not 16-byte aligned");
    return VIT_E_INVALID_ARG;
  }
  if (B < 1 || B > m->cfg.max_batch) {
    set_err("batch %d outside 1..max_batch (%d)", B, m->cfg.max_batch);
    return VIT_E_SHAPE;
  }
  vit_status st = check_outputs(out);
  if (st != VIT_OK) return st;
  const size_t need = ws_layout(m, B, native_geom(m)).total;
  if (need > kNoAllocScratchBytes) {
    set_err("vit_forward_noalloc: batch %d of this model needs %zu bytes of scratch, more than the fixed %zu "
            "bytes; use vit_forward with a caller-provided workspace",
            B, need, kNoAllocScratchBytes);
    return VIT_E_WORKSPACE;
  }
  st = check_device(m, "vit_forward_noalloc");
  if (st != VIT_OK) return st;
  void* ws = nullptr;
  st = noalloc_scratch(m, reinterpret_cast<cudaStream_t>(stream), &ws);
  if (st != VIT_OK) return st;
  const vit_config& c = m->cfg;
  ImgSrc src{images, 3LL * c.img_h * c.img_w, static_cast<long long>(c.img_h) * c.img_w, c.img_w, 1, 0, 0, 0};
  return run_forward(m, src, B, native_geom(m), out, ws, kNoAllocScratchBytes, reinterpret_cast<cudaStream_t>(stream));
}
