// router.cuh - top-k routing, one warp per token.
//
// vllm-project/vllm PR 65207, "Purpose", commit 1: the routed scaling factor
// is applied to the top-k weights inside the top-k kernel (biased grouped
// top-k), so no multiply of the layer output follows.
#pragma once
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

// VPL = values per lane = ceil(E / 32). Expert e lives in lane e % 32, slot e / 32.
template <int VPL>
__global__ void __launch_bounds__(kRouterWarps * 32) k_router_topk(const RouterArgs a) {
  extern __shared__ float rsm[];  // per warp: c[E], s[E] (grouped mode)
  const int wib = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouterWarps + wib;
  if (t >= a.T) return;
  const int E = a.E;
  float* c_sm = rsm + wib * 2 * E;
  float* s_sm = c_sm + E;
  const float* l = a.logits + static_cast<size_t>(t) * E;
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

}  // namespace moe
