// router.cuh - top-k routing, one warp per token.
//
// vllm-project/vllm PR 65207, "Purpose", commit 1: the routed scaling factor
// is applied to the top-k weights inside the top-k kernel (biased grouped
// top-k), so no multiply of the layer output follows.
#pragma once
#include <cooperative_groups.h>

#include "ptx.cuh"

namespace moe {

struct RouterArgs {
  const float* logits;  // [T,E]
  const float* bias;    // [E] or nullptr
  int T, E, k, mode, n_group, topk_group, renormalize;
  float rsf;
  int32_t* ids;  // [T,k]
  float* wts;    // [T,k]
};

// (value desc, index asc): does (va, ia) rank before (vb, ib)?
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Warp-wide arg-best of (v, i) under ranks_before; every lane gets the winner.
__device__ __forceinline__ void warp_argbest(float& v, int& i) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, off);
    const int oi = __shfl_xor_sync(0xffffffffu, i, off);
    if (ranks_before(ov, oi, v, i)) {
      v = ov;
      i = oi;
    }
  }
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

constexpr int kRouterWarps = 4;

// Top-k of token t from its logits row `l` (global or shared memory), run by
// one warp. VPL = values per lane = ceil(E / 32): expert e lives in lane
// e % 32, slot e / 32. c_sm / s_sm: E floats each of this warp's shared
// scratch (grouped mode).
template <int VPL>
__device__ void route_token(const RouterArgs& a, const float* l, float* c_sm, float* s_sm, int t, int lane) {
  const int E = a.E;
  const float NEG_INF = __int_as_float(0xff800000);

  float key[VPL];
  uint32_t avail = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = NEG_INF;
    if (e < E) {
      const float lv = l[e];
      if (a.mode == 0) {
        key[i] = lv;
      } else {
        // s = fp32(sigmoid(l)) evaluated in double, rounded once.
        const float s = static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(lv))));
        const float b = a.bias ? a.bias[e] : 0.0f;
        key[i] = __fadd_rn(s, b);
        c_sm[e] = key[i];
        s_sm[e] = s;
      }
      avail |= 1u << i;
    }
  }

  if (a.mode == 1) {
    __syncwarp();
    const int gsize = E / a.n_group;
    float score = NEG_INF;
    int gi = 0x7fffffff;
    if (lane < a.n_group) {
      const float* cg = c_sm + lane * gsize;
      if (gsize == 1) {
        score = cg[0];
      } else {
        float m1 = NEG_INF, m2 = NEG_INF;
        for (int i = 0; i < gsize; ++i) {
          const float v = cg[i];
          if (v > m1) {
            m2 = m1;
            m1 = v;
          } else if (v > m2) {
            m2 = v;
          }
        }
        score = __fadd_rn(m1, m2);
      }
      gi = lane;
    }
    uint32_t kept = 0;
    bool mine_taken = false;
    for (int r = 0; r < a.topk_group; ++r) {
      float v = mine_taken ? NEG_INF : score;
      int i = mine_taken ? 0x7fffffff : gi;
      warp_argbest(v, i);
      kept |= 1u << i;
      if (i == lane) mine_taken = true;
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((kept >> (e / gsize)) & 1u)) avail &= ~(1u << i);
    }
  }

  // k rounds of warp arg-best; lane j keeps the j-th pick.
  int my_sel = -1;
  float my_val = 0.f;
  for (int j = 0; j < a.k; ++j) {
    float v = NEG_INF;
    int idx = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      if (((avail >> i) & 1u) && ranks_before(key[i], e, v, idx)) {
        v = key[i];
        idx = e;
      }
    }
    warp_argbest(v, idx);
    if ((idx & 31) == lane) avail &= ~(1u << (idx >> 5));
    if (lane == j) {
      my_sel = idx;
      my_val = v;
    }
  }

  // Weights in double, rounded once to fp32; the scale is folded in here.
  const bool active = lane < a.k;
  double p = 0.0;
  double denom;
  if (a.mode == 0) {
    if (a.renormalize) {
      const float m = __shfl_sync(0xffffffffu, my_val, 0);
      p = active ? exp(static_cast<double>(my_val) - static_cast<double>(m)) : 0.0;
      denom = warp_sum_d(p);
    } else {
      float mx = NEG_INF;
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (lane + 32 * i < E) mx = fmaxf(mx, l[lane + 32 * i]);
      mx = warp_max_f(mx);
      double z = 0.0;
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (lane + 32 * i < E) z += exp(static_cast<double>(l[lane + 32 * i]) - static_cast<double>(mx));
      denom = warp_sum_d(z);
      p = active ? exp(static_cast<double>(my_val) - static_cast<double>(mx)) : 0.0;
    }
  } else {
    p = active ? static_cast<double>(s_sm[my_sel]) : 0.0;
    denom = a.renormalize ? warp_sum_d(p) : 1.0;
  }
  if (active) {
    const double w = p / denom * static_cast<double>(a.rsf);
    a.ids[static_cast<size_t>(t) * a.k + lane] = my_sel;
    a.wts[static_cast<size_t>(t) * a.k + lane] = static_cast<float>(w);
  }
}

template <int VPL>
__global__ void __launch_bounds__(kRouterWarps * 32) k_router_topk(const RouterArgs a) {
  extern __shared__ float rsm[];  // per warp: c[E], s[E] (grouped mode)
  const int wib = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouterWarps + wib;
  if (t >= a.T) return;
  float* c_sm = rsm + wib * 2 * a.E;
  route_token<VPL>(a, a.logits + static_cast<size_t>(t) * a.E, c_sm, c_sm + a.E, t, lane);
}


// ---------------------------------------------------------------------------
// Fused router linear + top-k: logits = x . W_r in one fixed fp32 order, then
// route_token. The pages give no router arithmetic (vllm-project/vllm
// PR 65207, "Purpose", passes the gate linear's output to the top-k); the
// order is this implementation's definition: H in kRouterChunks contiguous
// chunks, each summed in index order in fp32, the chunk sums added in chunk
// order, then the fp32 logit bias. Products of bf16/fp16 values are exact in
// fp32, so fmaf(x, w, acc) rounds exactly like acc + (x * w).
//
// One cluster of kRouterChunks CTAs per TB tokens: CTA j of the cluster sums
// chunk j for the cluster's tokens and all experts, streaming its rows of W_r
// through a two-buffer shared-memory ring (one bulk copy per sub-chunk of
// `rows_per_stage` rows), and writes the partial sums into CTA 0's shared
// memory (distributed shared memory); after the cluster barrier CTA 0 adds
// them in chunk order and its warps select the top-k of the TB tokens.

constexpr int kRouterChunks = 8;
constexpr int kRouterGemmThreads = 256;
constexpr int kRouterMaxBuf = 4;  // deepest W_r ring

struct RouterGemmArgs {
  const void* x;            // [T, H], bf16 or fp16
  const void* w;            // [H, E], same type (E % 8 == 0)
  const float* logit_bias;  // [E] or nullptr
  int H, rows_per_stage, nbuf;  // W_r ring: nbuf buffers of rows_per_stage rows
  int x_vec;          // 1: x and H / 8 allow 16-byte loads of every chunk row
  float* logits_out;  // [T, E] or nullptr
  RouterArgs r;       // routing parameters and outputs (r.logits unused)
};

__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_float(__half v) { return __half2float(v); }
template <typename TX>
__device__ __forceinline__ TX bits_as(unsigned short b);
template <>
__device__ __forceinline__ __nv_bfloat16 bits_as<__nv_bfloat16>(unsigned short b) {
  return __ushort_as_bfloat16(b);
}
template <>
__device__ __forceinline__ __half bits_as<__half>(unsigned short b) {
  return __ushort_as_half(b);
}
// The two values packed in a 32-bit word (low half first), without taking
// the address of a register.
__device__ __forceinline__ void unpack2(uint32_t w, __nv_bfloat16, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}
__device__ __forceinline__ void unpack2(uint32_t w, __half, float& lo, float& hi) {
  lo = __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xffffu)));
  hi = __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
}


// Shared-memory layout of k_router_gemm_topk (byte offsets; the W ring first,
// 128-byte aligned, then the partial sums, the selection scratch, x and the
// two ring barriers).
struct RouterGemmSmem {
  size_t w_off, part_off, cs_off, xs_off, bar_off, total;
  __host__ __device__ RouterGemmSmem(int TB, int EP, int E, int chunk, int rows, int nbuf) {
    auto up = [](size_t v) { return (v + 127) / 128 * 128; };
    w_off = 0;
    part_off = up(static_cast<size_t>(nbuf) * rows * E * 2);
    cs_off = part_off + up(static_cast<size_t>(kRouterChunks) * TB * EP * 4);
    xs_off = cs_off + up(static_cast<size_t>(kRouterGemmThreads / 32) * 2 * E * 4);
    bar_off = xs_off + up(static_cast<size_t>(chunk) * TB * 2);
    total = bar_off + 8 * kRouterMaxBuf;
  }
};

template <int VPL, int TB, typename TX>
__global__ void __cluster_dims__(kRouterChunks, 1, 1) __launch_bounds__(kRouterGemmThreads)
    k_router_gemm_topk(const RouterGemmArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int j = static_cast<int>(cluster.block_rank());
  const int E = a.r.E;
  const int H = a.H;
  const int c = H / kRouterChunks;
  const int R = a.rows_per_stage;
  const int NB = a.nbuf;
  const int nsub = (c + R - 1) / R;
  const int t0 = blockIdx.y * TB;
  const int tid = threadIdx.x;
  constexpr int EP = 32 * VPL;  // experts padded to whole lanes
  extern __shared__ __align__(128) uint8_t rg_raw[];
  const RouterGemmSmem L(TB, EP, E, c, R, NB);
  TX* wbuf = reinterpret_cast<TX*>(rg_raw + L.w_off);       // [NB][R][E]
  float* part = reinterpret_cast<float*>(rg_raw + L.part_off);  // [chunk][token][EP], CTA 0
  float* cs = reinterpret_cast<float*>(rg_raw + L.cs_off);      // per warp: c[E], s[E], CTA 0
  TX* xs = reinterpret_cast<TX*>(rg_raw + L.xs_off);            // [h][token]: x of chunk j, transposed
  uint64_t* bar = reinterpret_cast<uint64_t*>(rg_raw + L.bar_off);
  __shared__ int abort_sm;
  const TX* x = static_cast<const TX*>(a.x);
  const TX* wj = static_cast<const TX*>(a.w) + static_cast<size_t>(j) * c * E;

  auto issue = [&](int sub) {  // thread 0: rows [sub*R, sub*R + rows) of chunk j into buffer sub % NB
    const int rows = min(R, c - sub * R);
    const uint32_t bytes = static_cast<uint32_t>(rows) * E * 2;
    const int b = sub % NB;
    mbar_arrive_expect_tx(&bar[b], bytes);
    bulk_load(wbuf + b * R * E, wj + static_cast<size_t>(sub) * R * E, bytes, &bar[b], policy_evict_last());
  };
  if (tid == 0) {
    abort_sm = 0;
    for (int b = 0; b < NB; ++b) mbar_init(&bar[b], 1);
    fence_barrier_init();
    for (int sub = 0; sub < NB && sub < nsub; ++sub) issue(sub);
  }
  // x of chunk j for the cluster's tokens, transposed to [h][token]: 16-byte
  // loads (8 values) when every row segment is 16-byte aligned, all issued
  // before any is stored
  if (a.x_vec) {
    const int per_tok = c / 8;
    constexpr int kMaxV = 8;
    for (int base = tid; base < TB * per_tok; base += kRouterGemmThreads * kMaxV) {
      uint4 v[kMaxV];
#pragma unroll
      for (int u = 0; u < kMaxV; ++u) {
        const int i = base + u * kRouterGemmThreads;
        const int tt = i / per_tok;
        const int t = t0 + tt;
        v[u] = make_uint4(0, 0, 0, 0);
        if (i < TB * per_tok && t < a.r.T)
          v[u] = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H + j * c) + (i - tt * per_tok));
      }
#pragma unroll
      for (int u = 0; u < kMaxV; ++u) {
        const int i = base + u * kRouterGemmThreads;
        if (i < TB * per_tok) {
          const int tt = i / per_tok;
          const int h0 = (i - tt * per_tok) * 8;
          const uint32_t wv4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            xs[(h0 + 2 * q) * TB + tt] = bits_as<TX>(static_cast<unsigned short>(wv4[q] & 0xffffu));
            xs[(h0 + 2 * q + 1) * TB + tt] = bits_as<TX>(static_cast<unsigned short>(wv4[q] >> 16));
          }
        }
      }
    }
  } else {
    for (int i = tid; i < TB * c; i += kRouterGemmThreads) {
      const int tt = i / c;
      const int h = i - tt * c;
      const int t = t0 + tt;
      xs[h * TB + tt] = t < a.r.T ? x[static_cast<size_t>(t) * H + j * c + h] : TX(0.0f);
    }
  }
  __syncthreads();

  // Thread mapping: NE experts e_lo + k*EPT and TPT consecutive tokens
  // grp*TPT + u per thread; a warp shares its tokens (broadcast reads of x).
  constexpr int NE = EP > kRouterGemmThreads ? EP / kRouterGemmThreads : 1;
  constexpr int EPT = EP / NE;
  constexpr int G = kRouterGemmThreads / EPT;
  constexpr int TPT = TB >= G ? TB / G : 1;
  const int e_lo = tid % EPT;
  const int grp = tid / EPT;
  const bool has_tok = grp * TPT < TB;
  float acc[TPT][NE];
#pragma unroll
  for (int u = 0; u < TPT; ++u)
#pragma unroll
    for (int k = 0; k < NE; ++k) acc[u][k] = 0.f;
  bool live = true;
  for (int sub = 0; sub < nsub; ++sub) {
    if (live && !mbar_wait(&bar[sub % NB], static_cast<uint32_t>(sub / NB) & 1u, &abort_sm)) live = false;
    if (live && has_tok) {
      const TX* wb = wbuf + (sub % NB) * R * E;
      const TX* xr = xs + static_cast<size_t>(sub) * R * TB + grp * TPT;
      const int rows = min(R, c - sub * R);
#pragma unroll 4
      for (int i = 0; i < rows; ++i) {
        float xv[TPT];
        if constexpr (TPT % 8 == 0) {
#pragma unroll
          for (int v = 0; v < TPT / 8; ++v) {
            const uint4 q = *reinterpret_cast<const uint4*>(xr + i * TB + 8 * v);
            unpack2(q.x, TX(), xv[8 * v + 0], xv[8 * v + 1]);
            unpack2(q.y, TX(), xv[8 * v + 2], xv[8 * v + 3]);
            unpack2(q.z, TX(), xv[8 * v + 4], xv[8 * v + 5]);
            unpack2(q.w, TX(), xv[8 * v + 6], xv[8 * v + 7]);
          }
        } else if constexpr (TPT == 4) {
          const uint2 q = *reinterpret_cast<const uint2*>(xr + i * TB);
          unpack2(q.x, TX(), xv[0], xv[1]);
          unpack2(q.y, TX(), xv[2], xv[3]);
        } else if constexpr (TPT == 2) {
          unpack2(*reinterpret_cast<const uint32_t*>(xr + i * TB), TX(), xv[0], xv[1]);
        } else {
#pragma unroll
          for (int u = 0; u < TPT; ++u) xv[u] = to_float(xr[i * TB + u]);
        }
        float wv[NE];
#pragma unroll
        for (int k = 0; k < NE; ++k) {
          const int e = e_lo + k * EPT;
          wv[k] = e < E ? to_float(wb[i * E + e]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < TPT; ++u)
#pragma unroll
          for (int k = 0; k < NE; ++k) acc[u][k] = fmaf(xv[u], wv[k], acc[u][k]);
      }
    }
    __syncthreads();  // buffer sub % NB is no longer read
    if (tid == 0 && live && !abort_sm && sub + NB < nsub) issue(sub + NB);
  }
  if (tid == 0 && abort_sm) {
    // a wait gave up: let the copies still in flight land (bounded) before leaving
    for (int sub = 0; sub < nsub && sub < NB; ++sub) {
      const uint64_t t_start = globaltimer();
      while (!mbar_try_wait(smem_u32(&bar[sub % NB]), static_cast<uint32_t>(sub / NB) & 1u) &&
             globaltimer() - t_start < kWaitTimeoutNs) {
      }
    }
  }

  float* part0 = cluster.map_shared_rank(part, 0);
  if (has_tok) {
#pragma unroll
    for (int u = 0; u < TPT; ++u)
#pragma unroll
      for (int k = 0; k < NE; ++k) {
        const int e = e_lo + k * EPT;
        if (e < E) part0[(j * TB + grp * TPT + u) * EP + e] = acc[u][k];
      }
  }
  cluster.sync();
  if (j != 0) return;

  // chunk sums in chunk order (+ logit bias), written back into chunk 0's slot
  for (int q = tid; q < TB * EP; q += kRouterGemmThreads) {
    const int tt = q / EP;
    const int e = q - tt * EP;
    if (e >= E) continue;
    float v = part[tt * EP + e];
#pragma unroll
    for (int k = 1; k < kRouterChunks; ++k) v = __fadd_rn(v, part[(k * TB + tt) * EP + e]);
    if (a.logit_bias) v = __fadd_rn(v, a.logit_bias[e]);
    part[tt * EP + e] = v;
    const int t = t0 + tt;
    if (a.logits_out && t < a.r.T) a.logits_out[static_cast<size_t>(t) * E + e] = v;
  }
  __syncthreads();
  const int wib = tid >> 5;
  const int lane = tid & 31;
  float* c_sm = cs + wib * 2 * E;
  for (int tt = wib; tt < TB; tt += kRouterGemmThreads / 32)
    if (t0 + tt < a.r.T) route_token<VPL>(a.r, part + tt * EP, c_sm, c_sm + E, t0 + tt, lane);
}

// Fused shared expert (vllm-project/vllm PR 61503 "Fused heterogeneous MoE",
// "Overview"): the shared expert held as m always-selected routed experts
// E..E+m-1. Row t of the output top-k is the routed row followed by those m
// slots, each weighted by the shared gate g_t (1 without a gate).
__global__ void k_append_shared_slots(const int32_t* __restrict__ ids, const float* __restrict__ w, int T, int k,
                                      int E, int m, const void* __restrict__ gate, int gate_half,
                                      int32_t* __restrict__ ids2, float* __restrict__ w2) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int km = k + m;
  if (i >= T * km) return;
  const int t = i / km;
  const int j = i - t * km;
  if (j < k) {
    ids2[i] = ids[static_cast<size_t>(t) * k + j];
    w2[i] = w[static_cast<size_t>(t) * k + j];
  } else {
    ids2[i] = E + (j - k);
    float g = 1.0f;
    if (gate) g = gate_half ? __half2float(static_cast<const __half*>(gate)[t])
                            : __bfloat162float(static_cast<const __nv_bfloat16*>(gate)[t]);
    w2[i] = g;
  }
}

}  // namespace moe
