// gate.cuh - shared-expert gate: out[t] = sigmoid(x[t] . w), one kernel.
//
// vllm-project/vllm PR 56789, "Summary" and "Commits": the 1 x 1 x K GEMM of
// shared_expert_gate becomes one fp32-accumulated dot with the sigmoid folded
// in; the scalar is stored in the input dtype so the store does the rounding.
// Here: one CTA per token, 16-byte vector loads, warp-shuffle + shared-memory
// reduction, sigmoid on the fp32 sum, one rounding at the store.
#pragma once
#include "ptx.cuh"

namespace moe {

constexpr int kGateThreads = 256;

template <typename T>
struct GateIO;
template <>
struct GateIO<__nv_bfloat16> {
  __device__ static float f(__nv_bfloat16 v) { return __bfloat162float(v); }
  __device__ static __nv_bfloat16 to(float v) { return __float2bfloat16_rn(v); }
  __device__ static float2 f2(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
  }
};
template <>
struct GateIO<__half> {
  __device__ static float f(__half v) { return __half2float(v); }
  __device__ static __half to(float v) { return __float2half_rn(v); }
  __device__ static float2 f2(uint32_t u) { return __half22float2(*reinterpret_cast<const __half2*>(&u)); }
};

template <typename T>
__global__ void __launch_bounds__(kGateThreads) k_gate_dot(const T* __restrict__ x, const T* __restrict__ w, int K,
                                                            int apply_sigmoid, int vec_ok, T* __restrict__ out) {
  __shared__ float part[kGateThreads / 32];
  const int t = blockIdx.x;
  const T* xr = x + static_cast<size_t>(t) * K;
  float acc = 0.f;
  if (vec_ok) {  // K % 8 == 0 and 16-byte aligned rows
    for (int i = threadIdx.x * 8; i < K; i += kGateThreads * 8) {
      const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xr + i));
      const uint4 wv = __ldg(reinterpret_cast<const uint4*>(w + i));
      const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
      const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 a = GateIO<T>::f2(xs[j]);
        const float2 b = GateIO<T>::f2(ws[j]);
        acc = fmaf(a.x, b.x, acc);
        acc = fmaf(a.y, b.y, acc);
      }
    }
  } else {
    for (int i = threadIdx.x; i < K; i += kGateThreads) acc = fmaf(GateIO<T>::f(xr[i]), GateIO<T>::f(w[i]), acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < kGateThreads / 32 ? part[threadIdx.x] : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (threadIdx.x == 0) {
      if (apply_sigmoid) v = 1.0f / (1.0f + expf(-v));
      out[t] = GateIO<T>::to(v);
    }
  }
}

}  // namespace moe
