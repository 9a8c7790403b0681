// moe_b200.cu - C ABI of the routed + shared-expert MoE layer (include/moe_b200.h).
//
// Host side of every call: validate the arguments (nothing is launched on an
// invalid argument), encode the TMA tensor maps, pick the kernel instance and
// launch it on the caller's stream. All kernels live in the headers included
// below and are compiled into this one translation unit.
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "moe_b200.h"
#include "gate.cuh"
#include "gemm.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "router.cuh"
#include "selftest.cuh"
#include "sort.cuh"

namespace {

thread_local char g_last_cuda_error[256] = "";

moe_status_t fail_cuda(cudaError_t e, const char* what) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", what, cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

#define MOE_CK(call)                                     \
  do {                                                   \
    cudaError_t e_ = (call);                             \
    if (e_ != cudaSuccess) return fail_cuda(e_, #call);  \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }
// block-scaled layers: MXFP8 throughout, or MXFP4 weights against MXFP8 tokens
inline bool is_mx_dtype(int dtype) { return dtype == MOE_DT_MXFP8_E4M3 || dtype == MOE_DT_MXFP4_E2M1; }
inline cudaStream_t as_stream(moe_stream_t s) { return static_cast<cudaStream_t>(s); }
inline bool valid_block_m(int bm) { return bm == 16 || bm == 32 || bm == 64 || bm == 128 || bm == 256; }

int num_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    int v = cache[dev].load();
    if (v) return v;
  }
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cache[dev].store(n);
  return n;
}

// ------------------------------------------------------------ TMA tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load();
  if (f) return f;
  void* p = nullptr;
  cudaDriverEntryPointQueryResult qr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) != cudaSuccess ||
      qr != cudaDriverEntryPointSuccess || p == nullptr)
    return nullptr;
  f = reinterpret_cast<EncodeTiledFn>(p);
  fn.store(f);
  return f;
}

// Tiled map with the 128-byte swizzle; dims/box innermost first, strides in
// bytes for dims 1..rank-1.
moe_status_t make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
                      const cuuint64_t* strides, const cuuint32_t* box,
                      CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn f = encode_fn();
  if (!f) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled unavailable");
    return MOE_ERR_CUDA;
  }
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUresult r = f(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box, es,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled failed (CUresult %d)",
             static_cast<int>(r));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Map of an MX scale-tile array (512-byte tiles) as rows of 128 bytes: one
// 128 x 4 box is one tile (four row requests), landing dense in shared memory
// (no swizzle).
moe_status_t make_sf_tile_map(CUtensorMap* m, const void* base, size_t tiles) {
  const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(tiles) * 4};
  const cuuint64_t st[1] = {128};
  const cuuint32_t box[2] = {128, 4};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, st, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// ------------------------------------------------------------ GEMM dispatch

template <int BN, int KIND, bool S1, int ST = 2>
constexpr int fit_stages() {
  if constexpr (ST < 16 && moe::GemmSmem<BN, ST + 1, KIND, S1>::kBytes <= 227 * 1024)
    return fit_stages<BN, KIND, S1, ST + 1>();
  else
    return ST;
}

template <int BN, int KIND, bool S1>
constexpr int stages_for() {
  // as many stages as fit in 227 KB of shared memory, one CTA per SM, except
  // bf16 / fp8 16-token tiles: 108 KB of operands in flight per SM (three
  // two-atom stages) streamed the weights faster than all that fit (decode
  // step 145.5 us either way for bf16, 177.8 against 193.5 us for fp8 at
  // T = 32), as a bulk-copy stream also peaks at 64-100 KB in flight per SM
  // and loses DRAM bandwidth beyond
  if constexpr (!moe::is_mx(KIND) && BN == 16) return 3;
  else return fit_stages<BN, KIND, S1>();
}

// Pair tiles: as many stages as fit in 227 KB (each CTA holds half the token rows).
template <int BN, int KIND, bool S1, int ST = 2>
constexpr int pair_stages() {
  if constexpr (ST < 16 && moe::GemmSmem<BN, ST + 1, KIND, S1, true>::kBytes <= 227 * 1024)
    return pair_stages<BN, KIND, S1, ST + 1>();
  else
    return ST;
}

// Whether a GEMM runs on CTA pairs (one MMA of M = 256 per 2-CTA cluster,
// each SM loading its 128 weight rows and half the token tile): opt-in with
// MOE_B200_PAIR=1, for 16- and 128-token tiles whose weight rows split into
// an even number of 128-row tiles, never the fp8 stage 1 (its per-row
// quantisation of h follows a grid barrier in a cooperative launch). Measured
// against one CTA per tile (two-atom stages both): MXFP8 prefill 4104 -> 4189
// us, bf16 decode 143.3 -> 146.8 us, MXFP4 decode 87.2 -> 105.1 us (a pair's
// MMA thread also moves the scale tiles), fp8 decode (T = 32) 175.3 -> 172.8
// us. Results do not depend on the choice.
bool use_pair(int dtype, int bm, int n_mt, bool s1) {
  static const bool enabled = [] {
    const char* v = getenv("MOE_B200_PAIR");
    return v && v[0] == '1';
  }();
  return enabled && (bm == 16 || bm == 128) && n_mt % 2 == 0 && !(s1 && dtype == MOE_DT_FP8_E4M3);
}

template <typename Kern>
moe_status_t set_smem_attr(Kern kern, int bytes, std::atomic<int>* attr_set) {
  int dev = 0;
  MOE_CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64 || !attr_set[dev].load()) {
    MOE_CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
    if (dev >= 0 && dev < 64) attr_set[dev].store(1);
  }
  return MOE_OK;
}

template <int BN, bool S1, int KIND>
moe_status_t launch_gemm_bn(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb16,
                            const moe::GemmArgs& g, int max_tiles, cudaStream_t s) {
  constexpr int ST = stages_for<BN, KIND, S1>();
  using L = moe::GemmSmem<BN, ST, KIND, S1>;
  static_assert(L::kBytes <= 227 * 1024, "shared memory per CTA");
  auto kern = moe::k_moe_gemm<BN, ST, S1, KIND, false>;
  static std::atomic<int> attr_set[64];
  const moe_status_t r = set_smem_attr(kern, L::kBytes, attr_set);
  if (r != MOE_OK) return r;
  int grid = max_tiles < num_sms() ? max_tiles : num_sms();
  if (grid < 1) grid = 1;
  // the scale-tile maps are read by pair kernels only
  if (g.quant_phase) {
    // every CTA resident at once (one per SM): the grid barrier's wait ends
    void* args[] = {const_cast<CUtensorMap*>(&ta), const_cast<CUtensorMap*>(&tb), const_cast<CUtensorMap*>(&tb16),
                    const_cast<CUtensorMap*>(&tb), const_cast<CUtensorMap*>(&tb), const_cast<moe::GemmArgs*>(&g)};
    MOE_CK(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid),
                                       dim3(moe::EpiCfg<BN, KIND, S1>::kThreads), args, L::kBytes, s));
  } else {
    kern<<<grid, moe::EpiCfg<BN, KIND, S1>::kThreads, L::kBytes, s>>>(ta, tb, tb16, tb, tb, g);
  }
  MOE_CK(cudaGetLastError());
  return MOE_OK;
}

// A GEMM on CTA pairs: 2-CTA clusters, as many as can be resident at once
// (cudaOccupancyMaxActiveClusters), each looping over pair tiles.
template <int BN, bool S1, int KIND>
moe_status_t launch_gemm_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb8,
                              const CUtensorMap& tsfa, const CUtensorMap& tsfb, const moe::GemmArgs& g,
                              int max_pair_tiles, cudaStream_t s) {
  constexpr int ST = pair_stages<BN, KIND, S1>();
  using L = moe::GemmSmem<BN, ST, KIND, S1, true>;
  static_assert(L::kBytes <= 227 * 1024, "shared memory per CTA");
  auto kern = moe::k_moe_gemm<BN, ST, S1, KIND, true>;
  constexpr int threads = moe::EpiCfg<BN, KIND, S1>::kThreads;
  static std::atomic<int> attr_set[64];
  moe_status_t r = set_smem_attr(kern, L::kBytes, attr_set);
  if (r != MOE_OK) return r;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = L::kBytes;
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  static std::atomic<int> max_clusters[64];
  int dev = 0;
  MOE_CK(cudaGetDevice(&dev));
  int mc = (dev >= 0 && dev < 64) ? max_clusters[dev].load() : 0;
  if (mc == 0) {
    cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1));
    if (cudaOccupancyMaxActiveClusters(&mc, reinterpret_cast<const void*>(kern), &cfg) != cudaSuccess || mc < 1) {
      cudaGetLastError();  // clear: fall back to one pair per two SMs
      mc = num_sms() / 2;
    }
    if (dev >= 0 && dev < 64) max_clusters[dev].store(mc);
  }
  int clusters = max_pair_tiles < mc ? max_pair_tiles : mc;
  if (clusters < 1) clusters = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
  void* args[] = {const_cast<CUtensorMap*>(&ta), const_cast<CUtensorMap*>(&tb), const_cast<CUtensorMap*>(&tb8),
                  const_cast<CUtensorMap*>(&tsfa), const_cast<CUtensorMap*>(&tsfb), const_cast<moe::GemmArgs*>(&g)};
  MOE_CK(cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(kern), args));
  MOE_CK(cudaGetLastError());
  return MOE_OK;
}

template <bool S1, int KIND>
moe_status_t launch_gemm(int bm, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb16,
                         const moe::GemmArgs& g, int max_tiles, cudaStream_t s) {
  switch (bm) {
    case 16: return launch_gemm_bn<16, S1, KIND>(ta, tb, tb16, g, max_tiles, s);
    case 32: return launch_gemm_bn<32, S1, KIND>(ta, tb, tb16, g, max_tiles, s);
    case 64: return launch_gemm_bn<64, S1, KIND>(ta, tb, tb16, g, max_tiles, s);
    case 128: return launch_gemm_bn<128, S1, KIND>(ta, tb, tb16, g, max_tiles, s);
    case 256:
      if constexpr (!moe::is_mx(KIND)) return launch_gemm_bn<256, S1, KIND>(ta, tb, tb16, g, max_tiles, s);
      break;
  }
  return MOE_ERR_INVALID_ARG;
}

template <bool S1>
moe_status_t launch_gemm_kind(int dtype, int bm, const CUtensorMap& ta, const CUtensorMap& tb,
                              const CUtensorMap& tb16, const moe::GemmArgs& g, int max_tiles, cudaStream_t s) {
  if (dtype == MOE_DT_FP8_E4M3) return launch_gemm<S1, moe::kFp8>(bm, ta, tb, tb16, g, max_tiles, s);
  if (dtype == MOE_DT_MXFP8_E4M3) return launch_gemm<S1, moe::kMx8>(bm, ta, tb, tb16, g, max_tiles, s);
  if (dtype == MOE_DT_MXFP4_E2M1) return launch_gemm<S1, moe::kMx4>(bm, ta, tb, tb16, g, max_tiles, s);
  return launch_gemm<S1, moe::kBf16>(bm, ta, tb, tb16, g, max_tiles, s);
}

template <int BN, bool S1>
moe_status_t launch_gemm_pair_bn(int dtype, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb8,
                                 const CUtensorMap& tsfa, const CUtensorMap& tsfb, const moe::GemmArgs& g,
                                 int max_pair_tiles, cudaStream_t s) {
  if (dtype == MOE_DT_MXFP8_E4M3)
    return launch_gemm_pair<BN, S1, moe::kMx8>(ta, tb, tb8, tsfa, tsfb, g, max_pair_tiles, s);
  if (dtype == MOE_DT_MXFP4_E2M1)
    return launch_gemm_pair<BN, S1, moe::kMx4>(ta, tb, tb8, tsfa, tsfb, g, max_pair_tiles, s);
  if constexpr (!S1) {
    if (dtype == MOE_DT_FP8_E4M3)
      return launch_gemm_pair<BN, S1, moe::kFp8>(ta, tb, tb8, tsfa, tsfb, g, max_pair_tiles, s);
  }
  if (dtype == MOE_DT_BF16) return launch_gemm_pair<BN, S1, moe::kBf16>(ta, tb, tb8, tsfa, tsfb, g, max_pair_tiles, s);
  return MOE_ERR_INVALID_ARG;
}

template <bool S1>
moe_status_t launch_gemm_pair_kind(int dtype, int bm, const CUtensorMap& ta, const CUtensorMap& tb,
                                   const CUtensorMap& tb8, const CUtensorMap& tsfa, const CUtensorMap& tsfb,
                                   const moe::GemmArgs& g, int max_pair_tiles, cudaStream_t s) {
  if (bm == 16) return launch_gemm_pair_bn<16, S1>(dtype, ta, tb, tb8, tsfa, tsfb, g, max_pair_tiles, s);
  if (bm == 128) return launch_gemm_pair_bn<128, S1>(dtype, ta, tb, tb8, tsfa, tsfb, g, max_pair_tiles, s);
  return MOE_ERR_INVALID_ARG;
}

// Padded sorted length bound T*k + E*(bm-1), rounded up to whole blocks.
size_t capacity(int T, int k, int E, int bm) {
  const size_t n = static_cast<size_t>(T) * k + static_cast<size_t>(E) * (bm - 1);
  return (n + bm - 1) / bm * bm;
}

// Stage-1 workspace, 256-byte aligned parts:
//  * fp8: unquantised fp32 h [rows, I], per-tile row amax [I/64][rows], one
//    arrival counter per token block, the grid barrier's two words;
//  * routed stage 1: token rows in sorted order [rows, H] (x's type);
//  * MXFP8 / MXFP4: token scale tiles [rows / block_m][H / 128][512].
struct Stage1Ws {
  size_t amax_off = 0, cnt_off = 0, bar_off = 0, xs_off = 0, xsf_off = 0, total = 0;
  Stage1Ws(int dtype, size_t rows, int H, int I, int bm) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    size_t o = 0;
    if (dtype == MOE_DT_FP8_E4M3) {
      amax_off = up(rows * static_cast<size_t>(I) * 4);
      cnt_off = amax_off + up(static_cast<size_t>((I + 63) / 64) * rows * 4);
      bar_off = cnt_off + up(rows / bm * 4);
      o = bar_off + 256;
    }
    xs_off = o;
    o += up(rows * static_cast<size_t>(H) * (dtype == MOE_DT_BF16 ? 2 : 1));
    xsf_off = o;
    if (is_mx_dtype(dtype)) o += up(rows / bm * static_cast<size_t>(H / 128) * moe::kSfTile);
    total = o;
  }
};

// Stage-2 workspace owned by the library, for callers that cannot allocate
// (moe_stage2_gemm_accumulate_static_ws). Zero at module load.
static __device__ __align__(256) unsigned char g_stage2_static_ws[MOE_STAGE2_STATIC_WS_BYTES];

// Device address of g_stage2_static_ws, looked up once per device with that
// device current. In host code the symbol is only a host-side stand-in.
std::mutex g_static_ws_mu;
void* g_static_ws_addr[64];

moe_status_t static_ws_address(void** out) {
  int dev = 0;
  MOE_CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_static_ws_mu);
  if (!g_static_ws_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_stage2_static_ws);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(g_stage2_static_ws)");
    g_static_ws_addr[dev] = p;
  }
  *out = g_static_ws_addr[dev];
  return MOE_OK;
}

}  // namespace

// ======================================================================== ABI

// Argument checks shared by the two routing entry points.
moe_status_t check_route(const float* correction_bias, int T, int E, int top_k, int mode, int n_group,
                         int topk_group, const int32_t* topk_ids, const float* topk_weights) {
  if (!topk_ids || !topk_weights) return MOE_ERR_INVALID_ARG;
  if (T < 1 || E < 1 || E > MOE_MAX_EXPERTS || top_k < 1 || top_k > E || top_k > MOE_MAX_TOPK)
    return MOE_ERR_INVALID_ARG;
  if (mode != MOE_ROUTE_SOFTMAX && mode != MOE_ROUTE_GROUPED_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (mode == MOE_ROUTE_GROUPED_SIGMOID) {
    if (n_group < 1 || n_group > 32 || E % n_group != 0) return MOE_ERR_INVALID_ARG;
    if (topk_group < 1 || topk_group > n_group) return MOE_ERR_INVALID_ARG;
    if (top_k > topk_group * (E / n_group)) return MOE_ERR_INVALID_ARG;
  } else if (correction_bias) {
    return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

template <int VPL, int TB, typename TX>
moe_status_t launch_router_gemm(moe::RouterGemmArgs a, cudaStream_t s) {
  auto kern = moe::k_router_gemm_topk<VPL, TB, TX>;
  const int c = a.H / moe::kRouterChunks;
  // W_r ring: up to 4 buffers of up to 64 rows, at least two sub-chunks per
  // chunk (both first buffers load at once); shrink the rows, then the number
  // of buffers, until the layout fits 227 KB
  int R = (c + 1) / 2 < 64 ? (c + 1) / 2 : 64;
  int NB = moe::kRouterMaxBuf;
  auto bytes = [&]() { return moe::RouterGemmSmem(TB, 32 * VPL, a.r.E, c, R, NB).total; };
  while (bytes() > 227u * 1024 && (R > 8 || NB > 2)) {
    if (NB > 2) --NB;
    else R /= 2;
  }
  const size_t smem = bytes();
  if (smem > 227u * 1024) return MOE_ERR_SHAPE;
  a.rows_per_stage = R;
  a.nbuf = NB;
  MOE_CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
  const dim3 grid(moe::kRouterChunks, (a.r.T + TB - 1) / TB);
  kern<<<grid, moe::kRouterGemmThreads, smem, s>>>(a);
  MOE_CK(cudaGetLastError());
  return MOE_OK;
}

template <typename TX>
moe_status_t launch_router_gemm_vpl(const moe::RouterGemmArgs& a, cudaStream_t s) {
  // 16 tokens per cluster once there are enough tokens to fill clusters of them
  // (W_r is then read once per 16 tokens), 4 otherwise (more clusters at decode)
  const int vpl = (a.r.E + 31) / 32;
  const bool wide = a.r.T >= 64 && vpl <= 8;
  if (vpl <= 1) return wide ? launch_router_gemm<1, 16, TX>(a, s) : launch_router_gemm<1, 4, TX>(a, s);
  if (vpl <= 2) return wide ? launch_router_gemm<2, 16, TX>(a, s) : launch_router_gemm<2, 4, TX>(a, s);
  if (vpl <= 4) return wide ? launch_router_gemm<4, 16, TX>(a, s) : launch_router_gemm<4, 4, TX>(a, s);
  if (vpl <= 8) return wide ? launch_router_gemm<8, 16, TX>(a, s) : launch_router_gemm<8, 4, TX>(a, s);
  return launch_router_gemm<16, 4, TX>(a, s);
}

// Argument checks of stage 2, shared by moe_stage2_gemm_accumulate and
// moe_stage2_gemm_accumulate_static_ws so that both accept and refuse the same
// calls, before anything is enqueued (the workspace is checked by each).
moe_status_t check_stage2(int dtype, const void* h, const void* h_scale, const void* w2, const void* w2_scale,
                          const void* weights, int weights_dtype, const int32_t* sorted_ids,
                          const int32_t* block_expert, const int32_t* num_padded, int T, int top_k, int H, int I,
                          int E, int block_m, const void* addend, const void* out) {
  const bool fp8 = dtype == MOE_DT_FP8_E4M3;
  const bool mx = is_mx_dtype(dtype);
  const bool w4 = dtype == MOE_DT_MXFP4_E2M1;
  if (dtype != MOE_DT_BF16 && !fp8 && !mx) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (!h || !w2 || !out) return MOE_ERR_INVALID_ARG;
  if (T < 1 || top_k < 1 || E < 1 || top_k > E || H < 1 || I < 1 || !valid_block_m(block_m))
    return MOE_ERR_INVALID_ARG;
  if (sorted_ids && (!block_expert || !num_padded)) return MOE_ERR_INVALID_ARG;
  if (!sorted_ids && top_k != 1) return MOE_ERR_INVALID_ARG;
  if ((fp8 || mx) && (!h_scale || !w2_scale)) return MOE_ERR_INVALID_ARG;
  if (mx && block_m > 128) return MOE_ERR_INVALID_ARG;
  if (weights && weights_dtype != MOE_DT_F32 && weights_dtype != MOE_DT_BF16 && weights_dtype != MOE_DT_FP16)
    return MOE_ERR_UNSUPPORTED_DTYPE;
  if (H % 128 != 0 || I % 64 != 0) return MOE_ERR_SHAPE;
  if (mx && I % 128 != 0) return MOE_ERR_ALIGNMENT;
  if (!aligned16(h) || !aligned16(w2) || !aligned16(out) || (addend && !aligned16(addend)) ||
      (mx && (!aligned16(h_scale) || !aligned16(w2_scale))) || (w4 && !aligned32(w2)))
    return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_DTYPE: return "MOE_ERR_UNSUPPORTED_DTYPE";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT";
    case MOE_ERR_SHAPE: return "MOE_ERR_SHAPE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
    case MOE_ERR_WORKSPACE_LIMIT: return "MOE_ERR_WORKSPACE_LIMIT";
  }
  return "MOE_ERR_UNKNOWN";
}

const char* moe_version(void) { return "moe_b200 0.1 (sm_100a)"; }

const char* moe_last_cuda_error(void) { return g_last_cuda_error; }

int moe_supports_output_addend(void) { return 1; }

moe_status_t moe_device_error(int* code, moe_stream_t stream) {
  if (!code) return MOE_ERR_INVALID_ARG;
  MOE_CK(cudaStreamSynchronize(as_stream(stream)));
  int v = 0;
  MOE_CK(cudaMemcpyFromSymbol(&v, moe::g_device_error, sizeof(int)));
  const int zero = 0;
  MOE_CK(cudaMemcpyToSymbol(moe::g_device_error, &zero, sizeof(int)));
  *code = v;
  return MOE_OK;
}

moe_status_t moe_selftest_wait_timeout(moe_stream_t stream) {
  moe::k_selftest_wait_timeout<<<1, 32, 0, as_stream(stream)>>>();
  MOE_CK(cudaGetLastError());
  return MOE_OK;
}

size_t moe_sorted_capacity(int T, int top_k, int E, int block_m) {
  if (T < 0 || top_k < 0 || E < 0 || block_m < 1) return 0;
  return capacity(T, top_k, E, block_m);
}

size_t moe_stage2_workspace_bytes(int T, int H) {
  if (T < 1 || H < 1) return 0;
  const size_t n_mt = (static_cast<size_t>(H) + moe::kTileM - 1) / moe::kTileM;
  return static_cast<size_t>(T) * H * sizeof(float) + static_cast<size_t>(T) * n_mt * sizeof(int);
}

size_t moe_stage1_workspace_bytes(int dtype, int T, int top_k, int E, int H, int I, int block_m) {
  if (dtype != MOE_DT_BF16 && dtype != MOE_DT_FP8_E4M3 && !is_mx_dtype(dtype)) return 0;
  if (T < 1 || top_k < 1 || E < 1 || H < 1 || I < 1 || !valid_block_m(block_m)) return 0;
  return Stage1Ws(dtype, capacity(T, top_k, E, block_m), H, I, block_m).total;
}

moe_status_t moe_router_gemm_topk(int dtype, const void* x, const void* w_r, const float* logit_bias,
                                  const float* correction_bias, int T, int H, int E, int top_k, int mode, int n_group,
                                  int topk_group, int renormalize, float routed_scaling_factor, float* logits,
                                  int32_t* topk_ids, float* topk_weights, moe_stream_t stream) {
  if (dtype != MOE_DT_BF16 && dtype != MOE_DT_FP16) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (!x || !w_r) return MOE_ERR_INVALID_ARG;
  const moe_status_t r = check_route(correction_bias, T, E, top_k, mode, n_group, topk_group, topk_ids, topk_weights);
  if (r != MOE_OK) return r;
  if (H < moe::kRouterChunks || H % moe::kRouterChunks != 0 || E % 8 != 0) return MOE_ERR_SHAPE;
  if (!aligned16(w_r)) return MOE_ERR_ALIGNMENT;  // W_r rows are bulk-copied
  moe::RouterGemmArgs a{};
  a.x = x;
  a.w = w_r;
  a.logit_bias = logit_bias;
  a.H = H;
  a.x_vec = (H % 64 == 0 && aligned16(x)) ? 1 : 0;
  a.logits_out = logits;
  a.r = moe::RouterArgs{nullptr, correction_bias, T, E, top_k, mode, n_group, topk_group, renormalize,
                        routed_scaling_factor, topk_ids, topk_weights};
  cudaStream_t s = as_stream(stream);
  return dtype == MOE_DT_BF16 ? launch_router_gemm_vpl<__nv_bfloat16>(a, s) : launch_router_gemm_vpl<__half>(a, s);
}

moe_status_t moe_router_topk(const float* logits, const float* correction_bias, int T, int E, int top_k, int mode,
                             int n_group, int topk_group, int renormalize, float routed_scaling_factor,
                             int32_t* topk_ids, float* topk_weights, moe_stream_t stream) {
  if (!logits) return MOE_ERR_INVALID_ARG;
  const moe_status_t r = check_route(correction_bias, T, E, top_k, mode, n_group, topk_group, topk_ids, topk_weights);
  if (r != MOE_OK) return r;
  moe::RouterArgs a{logits, correction_bias, T, E, top_k, mode, n_group, topk_group, renormalize,
                    routed_scaling_factor, topk_ids, topk_weights};
  const int vpl = (E + 31) / 32;
  const dim3 grid((T + moe::kRouterWarps - 1) / moe::kRouterWarps);
  const dim3 block(moe::kRouterWarps * 32);
  const size_t smem = static_cast<size_t>(moe::kRouterWarps) * 2 * E * sizeof(float);
  cudaStream_t s = as_stream(stream);
  if (vpl <= 1) moe::k_router_topk<1><<<grid, block, smem, s>>>(a);
  else if (vpl <= 2) moe::k_router_topk<2><<<grid, block, smem, s>>>(a);
  else if (vpl <= 4) moe::k_router_topk<4><<<grid, block, smem, s>>>(a);
  else if (vpl <= 8) moe::k_router_topk<8><<<grid, block, smem, s>>>(a);
  else moe::k_router_topk<16><<<grid, block, smem, s>>>(a);
  MOE_CK(cudaGetLastError());
  return MOE_OK;
}

moe_status_t moe_align_sort(const int32_t* topk_ids, int T, int top_k, int E, int block_m, int32_t* sorted_ids,
                            int32_t* block_expert, int32_t* expert_counts, int32_t* expert_offsets,
                            int32_t* num_padded, moe_stream_t stream) {
  if (!topk_ids || !sorted_ids || !block_expert || !expert_counts || !expert_offsets || !num_padded)
    return MOE_ERR_INVALID_ARG;
  if (T < 1 || top_k < 1 || E < 1 || E > MOE_MAX_EXPERTS || !valid_block_m(block_m)) return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * top_k > (1ll << 20)) return MOE_ERR_SHAPE;
  moe::SortArgs a{topk_ids, T * top_k, E, block_m, sorted_ids, block_expert, expert_counts, expert_offsets,
                  num_padded};
  const size_t smem = moe::sort_smem_bytes(E);
  const int smem_max = static_cast<int>(moe::sort_smem_bytes(MOE_MAX_EXPERTS));
  // a cluster of CTAs from kSortClusterMinSlots slots on (one CTA's 32 warps
  // take 32-slot steps one after another; the cluster splits them 8 ways)
  const bool cluster = a.N >= moe::kSortClusterMinSlots;
  if (cluster) {
    static std::atomic<int> attr_set[64];
    const moe_status_t r = set_smem_attr(moe::k_align_sort_cluster, smem_max, attr_set);
    if (r != MOE_OK) return r;
    moe::k_align_sort_cluster<<<moe::kSortCluster, moe::kSortThreads, smem, as_stream(stream)>>>(a);
  } else {
    static std::atomic<int> attr_set[64];
    const moe_status_t r = set_smem_attr(moe::k_align_sort, smem_max, attr_set);
    if (r != MOE_OK) return r;
    moe::k_align_sort<<<1, moe::kSortThreads, smem, as_stream(stream)>>>(a);
  }
  MOE_CK(cudaGetLastError());
  return MOE_OK;
}

moe_status_t moe_append_shared_slots(const int32_t* topk_ids, const float* topk_weights, int T, int top_k, int E,
                                     int m, const void* gate, int gate_dtype, int32_t* out_ids, float* out_weights,
                                     moe_stream_t stream) {
  if (!topk_ids || !topk_weights || !out_ids || !out_weights) return MOE_ERR_INVALID_ARG;
  if (T < 1 || top_k < 1 || E < 1 || m < 1 || E + m > MOE_MAX_EXPERTS || top_k + m > MOE_MAX_TOPK)
    return MOE_ERR_INVALID_ARG;
  if (gate && gate_dtype != MOE_DT_BF16 && gate_dtype != MOE_DT_FP16) return MOE_ERR_UNSUPPORTED_DTYPE;
  const int n = T * (top_k + m);
  moe::k_append_shared_slots<<<(n + 255) / 256, 256, 0, as_stream(stream)>>>(
      topk_ids, topk_weights, T, top_k, E, m, gate, gate_dtype == MOE_DT_FP16 ? 1 : 0, out_ids, out_weights);
  MOE_CK(cudaGetLastError());
  return MOE_OK;
}

moe_status_t moe_quantize_activations(int dtype, const void* x, int T, int H, void* codes, void* scale,
                                      moe_stream_t stream) {
  const bool mx = dtype == MOE_DT_MXFP8_E4M3;
  if (dtype != MOE_DT_FP8_E4M3 && !mx) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (!x || !codes || !scale || T < 1 || H < 1) return MOE_ERR_INVALID_ARG;
  if (H % (mx ? 32 : 8) != 0 || H > moe::kQuantXThreads * 8 * moe::kQuantXMaxV) return MOE_ERR_SHAPE;
  if (!aligned16(x) || reinterpret_cast<uintptr_t>(codes) % 8 != 0) return MOE_ERR_ALIGNMENT;
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* q = static_cast<uint8_t*>(codes);
  cudaStream_t s = as_stream(stream);
  if (mx) moe::k_quantize_x<true><<<T, moe::kQuantXThreads, 0, s>>>(xb, H, q, nullptr, static_cast<uint8_t*>(scale));
  else moe::k_quantize_x<false><<<T, moe::kQuantXThreads, 0, s>>>(xb, H, q, static_cast<float*>(scale), nullptr);
  MOE_CK(cudaGetLastError());
  return MOE_OK;
}

moe_status_t shared_expert_gate_dot(int dtype, const void* x, const void* w, int T, int K, int apply_sigmoid,
                                    void* out, moe_stream_t stream) {
  if (!x || !w || !out || T < 1 || K < 1) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DT_BF16 && dtype != MOE_DT_FP16) return MOE_ERR_UNSUPPORTED_DTYPE;
  const int vec_ok = (K % 8 == 0) && aligned16(x) && aligned16(w);
  cudaStream_t s = as_stream(stream);
  if (dtype == MOE_DT_BF16)
    moe::k_gate_dot<__nv_bfloat16><<<T, moe::kGateThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w), K, apply_sigmoid, vec_ok,
        static_cast<__nv_bfloat16*>(out));
  else
    moe::k_gate_dot<__half><<<T, moe::kGateThreads, 0, s>>>(static_cast<const __half*>(x),
                                                            static_cast<const __half*>(w), K, apply_sigmoid,
                                                            vec_ok, static_cast<__half*>(out));
  MOE_CK(cudaGetLastError());
  return MOE_OK;
}

moe_status_t moe_stage1_gemm(int dtype, const void* x, const void* x_scale, const void* w13, const void* w13_scale,
                             const int32_t* sorted_ids, const int32_t* block_expert, const int32_t* num_padded, int T,
                             int top_k, int H, int I, int E, int block_m, void* h, void* h_scale, void* ws,
                             moe_stream_t stream) {
  const bool fp8 = dtype == MOE_DT_FP8_E4M3;
  const bool mx = is_mx_dtype(dtype);
  const bool w4 = dtype == MOE_DT_MXFP4_E2M1;
  if (dtype != MOE_DT_BF16 && !fp8 && !mx) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (!x || !w13 || !h) return MOE_ERR_INVALID_ARG;
  if (T < 1 || top_k < 1 || E < 1 || top_k > E || H < 1 || I < 1 || !valid_block_m(block_m))
    return MOE_ERR_INVALID_ARG;
  if (sorted_ids && (!block_expert || !num_padded)) return MOE_ERR_INVALID_ARG;
  if (!sorted_ids && top_k != 1) return MOE_ERR_INVALID_ARG;
  // routed tiles read a copy of the token rows in sorted order
  const bool permute = sorted_ids != nullptr;
  if (fp8 && (!x_scale || !w13_scale || !h_scale)) return MOE_ERR_INVALID_ARG;
  if (mx && (!x_scale || !w13_scale || !h_scale)) return MOE_ERR_INVALID_ARG;
  if ((fp8 || mx || permute) && !ws) return MOE_ERR_INVALID_ARG;
  if (mx && block_m > 128) return MOE_ERR_INVALID_ARG;
  if (H % (dtype == MOE_DT_BF16 ? 64 : 128) != 0 || I % 64 != 0) return MOE_ERR_SHAPE;
  if (mx && I % 128 != 0) return MOE_ERR_ALIGNMENT;  // whole 4-block h scale tiles
  if (!aligned16(x) || !aligned16(w13) || !aligned16(h) || (ws && !aligned16(ws)) ||
      (mx && (!aligned16(x_scale) || !aligned16(w13_scale) || !aligned16(h_scale))) || (w4 && !aligned32(w13)))
    return MOE_ERR_ALIGNMENT;

  const bool b16 = dtype == MOE_DT_BF16;
  const int es = b16 ? 2 : 1;
  const int ke = b16 ? 64 : 128;
  const size_t rows_cap = capacity(T, top_k, E, block_m);  // identity routing: T rounded up to block_m
  // identity routing launches over the blocks that hold tokens only
  const int cap_blocks = sorted_ids ? static_cast<int>(rows_cap / block_m) : (T + block_m - 1) / block_m;
  const CUtensorMapDataType tdt = b16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;

  // W13 as 5-D (K, row-in-16, gate|up, 16-row group, expert): one box brings
  // 16 gate rows then the 16 matching up rows for four consecutive groups, so
  // the 128 weight rows of a tile pair gate and up inside each 32-lane quarter.
  const Stage1Ws L(dtype, rows_cap, H, I, block_m);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint8_t* xs = permute ? wsb + L.xs_off : nullptr;
  uint8_t* xsf = mx ? wsb + L.xsf_off : nullptr;
  const bool pair = use_pair(dtype, block_m, I / 64, true);
  CUtensorMap ta, tb, tb16, tsfa, tsfb;
  {
    // MXFP4: dims count e2m1 elements, strides bytes (two elements a byte);
    // the 16U4_ALIGN16B type spreads each 8 bytes over 16 in shared memory
    const size_t wrow = w4 ? static_cast<size_t>(H) / 2 : static_cast<size_t>(H) * es;
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(H), 16, 2, static_cast<cuuint64_t>(I / 16),
                                static_cast<cuuint64_t>(E)};
    const cuuint64_t st[4] = {wrow, static_cast<cuuint64_t>(I) * wrow, 16ull * wrow, 2ull * I * wrow};
    const cuuint32_t box[5] = {static_cast<cuuint32_t>(ke), 16, 2, 4, 1};
    moe_status_t r = make_map(&ta, w4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : tdt, 5, w13, dims, st, box);
    if (r != MOE_OK) return r;
  }
  {
    // token rows: one [block_m x 128 B] box per stage from the sorted copy,
    // or from x itself with identity routing (rows past T read as zeros);
    // tb16: the same rows in 16-row boxes, for tiles with fewer token rows.
    // A CTA pair splits the token rows: boxes of block_m / 2 rows, and 8-row
    // boxes for short tiles.
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(H), permute ? static_cast<cuuint64_t>(rows_cap)
                                                                    : static_cast<cuuint64_t>(T)};
    const cuuint64_t st[1] = {static_cast<cuuint64_t>(H) * es};
    const void* base = permute ? static_cast<const void*>(xs) : x;
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(ke), static_cast<cuuint32_t>(pair ? block_m / 2 : block_m)};
    moe_status_t r = make_map(&tb, tdt, 2, base, dims, st, box);
    if (r != MOE_OK) return r;
    const cuuint32_t box16[2] = {static_cast<cuuint32_t>(ke), pair ? 8u : 16u};
    r = make_map(&tb16, tdt, 2, base, dims, st, box16);
    if (r != MOE_OK) return r;
  }
  if (pair && mx) {
    // pairs load the scale tiles by TMA (their copies complete on rank 0's barrier)
    moe_status_t r = make_sf_tile_map(&tsfa, w13_scale, static_cast<size_t>(E) * (I / 64) * (H / 128));
    if (r != MOE_OK) return r;
    r = make_sf_tile_map(&tsfb, xsf, static_cast<size_t>(cap_blocks) * (H / 128));
    if (r != MOE_OK) return r;
  } else {
    tsfa = tb;  // not read
    tsfb = tb;
  }
  moe::GemmArgs g{};
  g.sorted_ids = sorted_ids;
  g.block_expert = block_expert;
  g.num_padded = num_padded;
  g.identity_rows = cap_blocks * block_m;
  g.cap_blocks = cap_blocks;
  g.T = T;
  g.top_k = top_k;
  g.H = H;
  g.I = I;
  g.E = E;
  g.n_mt = I / 64;
  g.num_kb = H / ke;
  g.rows_cap = static_cast<int>(rows_cap);
  if (fp8) {
    g.h32 = reinterpret_cast<float*>(wsb);
    g.h_amax = reinterpret_cast<float*>(wsb + L.amax_off);
    g.blk_cnt = reinterpret_cast<int*>(wsb + L.cnt_off);
    g.grid_bar = reinterpret_cast<unsigned*>(wsb + L.bar_off);
    // token blocks of 64 rows or more hold up to ~1.4 MB of fp32 h each: too
    // much for one warpgroup, so every warp quantises rows after a grid barrier
    g.quant_phase = block_m >= 64 ? 1 : 0;
    g.hq = static_cast<uint8_t*>(h);
    g.h_scale = static_cast<float*>(h_scale);
    g.x_scale = static_cast<const float*>(x_scale);
    g.w_scale = static_cast<const float*>(w13_scale);
  } else if (mx) {
    g.hq = static_cast<uint8_t*>(h);
    g.hsf = static_cast<uint8_t*>(h_scale);
    g.wsf = static_cast<const uint8_t*>(w13_scale);
    g.xsf = xsf;
  } else {
    g.h = static_cast<__nv_bfloat16*>(h);
  }
  cudaStream_t s = as_stream(stream);
  if (xs || xsf) {
    moe::PrepArgs p{};
    p.x = static_cast<const uint8_t*>(x);
    p.x_scale = static_cast<const uint8_t*>(x_scale);
    p.sorted_ids = sorted_ids;
    p.num_padded = num_padded;
    p.identity_rows = g.identity_rows;
    p.rows_cap = static_cast<int>(rows_cap);
    p.T = T;
    p.top_k = top_k;
    p.row_bytes = H * es;
    p.H = H;
    p.bm = block_m;
    p.xs = xs;
    p.xsf = xsf;
    const size_t want = (rows_cap + moe::kPrepWarps - 1) / moe::kPrepWarps;
    const int grid = static_cast<int>(want < 16u * num_sms() ? want : 16u * num_sms());
    moe::k_stage1_prep<<<grid, moe::kPrepWarps * 32, 0, s>>>(p);
    MOE_CK(cudaGetLastError());
  }
  const int max_tiles = cap_blocks * g.n_mt;
  if (pair) return launch_gemm_pair_kind<true>(dtype, block_m, ta, tb, tb16, tsfa, tsfb, g, max_tiles / 2, s);
  return launch_gemm_kind<true>(dtype, block_m, ta, tb, tb16, g, max_tiles, s);
}

moe_status_t moe_stage2_gemm_accumulate(int dtype, const void* h, const void* h_scale, const void* w2,
                                        const void* w2_scale, const void* weights, int weights_dtype,
                                        const int32_t* sorted_ids, const int32_t* block_expert,
                                        const int32_t* num_padded, int T, int top_k, int H, int I, int E,
                                        int block_m, const void* addend, moe_event_t addend_ready, void* acc_ws,
                                        void* out, moe_stream_t stream) {
  const moe_status_t chk = check_stage2(dtype, h, h_scale, w2, w2_scale, weights, weights_dtype, sorted_ids,
                                        block_expert, num_padded, T, top_k, H, I, E, block_m, addend, out);
  if (chk != MOE_OK) return chk;
  if (top_k > 1 && !acc_ws) return MOE_ERR_INVALID_ARG;
  if (acc_ws && !aligned16(acc_ws)) return MOE_ERR_ALIGNMENT;
  const bool fp8 = dtype == MOE_DT_FP8_E4M3;
  const bool mx = is_mx_dtype(dtype);
  const bool w4 = dtype == MOE_DT_MXFP4_E2M1;

  const bool b16 = dtype == MOE_DT_BF16;
  const int es = b16 ? 2 : 1;
  const int ke = b16 ? 64 : 128;
  const size_t rows_cap = capacity(T, top_k, E, block_m);
  // identity routing launches over the blocks that hold tokens only
  const int cap_blocks = sorted_ids ? static_cast<int>(rows_cap / block_m) : (T + block_m - 1) / block_m;
  const CUtensorMapDataType tdt = b16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const bool pair = use_pair(dtype, block_m, H / moe::kTileM, false);
  CUtensorMap ta, tb, tb16, tsfa, tsfb;
  {
    const size_t wrow = w4 ? static_cast<size_t>(I) / 2 : static_cast<size_t>(I) * es;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(I), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(E)};
    const cuuint64_t st[2] = {wrow, static_cast<cuuint64_t>(H) * wrow};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(ke), static_cast<cuuint32_t>(moe::kTileM), 1};
    moe_status_t r = make_map(&ta, w4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : tdt, 3, w2, dims, st, box);
    if (r != MOE_OK) return r;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(I), static_cast<cuuint64_t>(rows_cap)};
    const cuuint64_t st[1] = {static_cast<cuuint64_t>(I) * es};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(ke), static_cast<cuuint32_t>(pair ? block_m / 2 : block_m)};
    moe_status_t r = make_map(&tb, tdt, 2, h, dims, st, box);
    if (r != MOE_OK) return r;
    const cuuint32_t box16[2] = {static_cast<cuuint32_t>(ke), pair ? 8u : 16u};
    r = make_map(&tb16, tdt, 2, h, dims, st, box16);
    if (r != MOE_OK) return r;
  }
  if (pair && mx) {
    moe_status_t r = make_sf_tile_map(&tsfa, w2_scale, static_cast<size_t>(E) * (H / 128) * (I / 128));
    if (r != MOE_OK) return r;
    r = make_sf_tile_map(&tsfb, h_scale, static_cast<size_t>(cap_blocks) * (I / 128));
    if (r != MOE_OK) return r;
  } else {
    tsfa = tb;  // not read
    tsfb = tb;
  }
  cudaStream_t s = as_stream(stream);
  if (addend_ready) MOE_CK(cudaStreamWaitEvent(s, static_cast<cudaEvent_t>(addend_ready), 0));

  moe::GemmArgs g{};
  g.sorted_ids = sorted_ids;
  g.block_expert = block_expert;
  g.num_padded = num_padded;
  g.identity_rows = cap_blocks * block_m;
  g.cap_blocks = cap_blocks;
  g.T = T;
  g.top_k = top_k;
  g.H = H;
  g.I = I;
  g.E = E;
  g.n_mt = H / moe::kTileM;
  g.num_kb = (I + ke - 1) / ke;
  g.rows_cap = static_cast<int>(rows_cap);
  g.weights = weights;
  g.weights_dtype = weights_dtype;
  if (fp8) {
    g.h_scale = const_cast<float*>(static_cast<const float*>(h_scale));
    g.w_scale = static_cast<const float*>(w2_scale);
  } else if (mx) {
    g.hsf = const_cast<uint8_t*>(static_cast<const uint8_t*>(h_scale));
    g.wsf = static_cast<const uint8_t*>(w2_scale);
  }
  g.addend = static_cast<const __nv_bfloat16*>(addend);
  g.ws = static_cast<float*>(acc_ws);
  g.counters = acc_ws ? reinterpret_cast<int*>(static_cast<float*>(acc_ws) + static_cast<size_t>(T) * H) : nullptr;
  g.out = static_cast<__nv_bfloat16*>(out);
  const int max_tiles = cap_blocks * g.n_mt;
  if (pair) return launch_gemm_pair_kind<false>(dtype, block_m, ta, tb, tb16, tsfa, tsfb, g, max_tiles / 2, s);
  return launch_gemm_kind<false>(dtype, block_m, ta, tb, tb16, g, max_tiles, s);
}

size_t moe_mx_weight_scale_bytes(int which, int E, int H, int I) {
  if (E < 1 || H < 1 || I < 1 || H % 128 != 0 || I % 128 != 0) return 0;
  const size_t tiles = which == 0 ? static_cast<size_t>(I / 64) * (H / 128) : static_cast<size_t>(H / 128) * (I / 128);
  return static_cast<size_t>(E) * tiles * moe::kSfTile;
}

size_t moe_mx_h_scale_bytes(int T, int top_k, int E, int I, int block_m) {
  if (T < 1 || top_k < 1 || E < 1 || I < 1 || I % 128 != 0 || !valid_block_m(block_m) || block_m > 128) return 0;
  return capacity(T, top_k, E, block_m) / block_m * (I / 128) * moe::kSfTile;
}

moe_status_t moe_mx_pack_weight_scales(int which, const void* src, void* dst, int E, int H, int I,
                                       moe_stream_t stream) {
  if (!src || !dst || (which != 0 && which != 1)) return MOE_ERR_INVALID_ARG;
  if (E < 1 || H < 1 || I < 1) return MOE_ERR_INVALID_ARG;
  if (H % 128 != 0 || I % 128 != 0) return MOE_ERR_SHAPE;
  const int rows = which == 0 ? 2 * I : H;
  const int K = which == 0 ? H : I;
  const size_t n = moe_mx_weight_scale_bytes(which, E, H, I);
  const int blocks = static_cast<int>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  moe::k_mx_pack_weight_scales<<<blocks, 256, 0, as_stream(stream)>>>(
      static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), E, rows, K, I, which == 0 ? 1 : 0);
  MOE_CK(cudaGetLastError());
  return MOE_OK;
}

moe_status_t moe_stage2_gemm_accumulate_static_ws(int dtype, const void* h, const void* h_scale, const void* w2,
                                                  const void* w2_scale, const void* weights, int weights_dtype,
                                                  const int32_t* sorted_ids, const int32_t* block_expert,
                                                  const int32_t* num_padded, int T, int top_k, int H, int I, int E,
                                                  int block_m, const void* addend, moe_event_t addend_ready,
                                                  void* out, moe_stream_t stream) {
  // the checks of moe_stage2_gemm_accumulate first: nothing (not even the
  // clearing memset) is enqueued for a call that one of them refuses
  const moe_status_t chk = check_stage2(dtype, h, h_scale, w2, w2_scale, weights, weights_dtype, sorted_ids,
                                        block_expert, num_padded, T, top_k, H, I, E, block_m, addend, out);
  if (chk != MOE_OK) return chk;
  void* ws = nullptr;
  if (top_k > 1) {
    const size_t need = moe_stage2_workspace_bytes(T, H);
    if (need > MOE_STAGE2_STATIC_WS_BYTES) {
      snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
               "stage-2 workspace of %zu bytes exceeds the static %u bytes (T=%d, H=%d)", need,
               static_cast<unsigned>(MOE_STAGE2_STATIC_WS_BYTES), T, H);
      return MOE_ERR_WORKSPACE_LIMIT;
    }
    // the array used is the current device's: the stream must belong to it
    int dev = 0, sdev = 0;
    MOE_CK(cudaGetDevice(&dev));
    MOE_CK(cudaStreamGetDevice(as_stream(stream), &sdev));
    if (sdev != dev) {
      snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
               "stream of device %d while device %d is current", sdev, dev);
      return MOE_ERR_DEVICE;
    }
    const moe_status_t r = static_ws_address(&ws);
    if (r != MOE_OK) return r;
    MOE_CK(cudaMemsetAsync(ws, 0, need, as_stream(stream)));
  }
  return moe_stage2_gemm_accumulate(dtype, h, h_scale, w2, w2_scale, weights, weights_dtype, sorted_ids,
                                    block_expert, num_padded, T, top_k, H, I, E, block_m, addend, addend_ready, ws,
                                    out, stream);
}

}  // extern "C"
