// quant.cuh - bf16 activations to the stage-1 operand formats.
#pragma once
#include "gemm.cuh"

namespace moe {

// bf16 activations to the stage-1 operand formats (ROCm/aiter PR 6106,
// "Technical Details": per-token activation scales; MXFP8 BLOCK_K = 32), one
// CTA per token row: every thread loads its 16-byte chunks (8 values each,
// chunk c = tid + kQuantXThreads * v) at once and keeps them in registers.
//  fp8:   s = amax / 448 over the row (amax = 0: s = 1), code = e4m3_rn(x / s),
//         the fp32 quotient by IEEE division, saturating;
//  MXFP8: per 32 columns (chunks 4m..4m+3, held by four consecutive lanes)
//         X = mx_exponent(amax), byte X + 127, code = e4m3_rn(x * 2^-X).
constexpr int kQuantXThreads = 256;
constexpr int kQuantXMaxV = 8;  // chunks per thread: H <= 256 * 8 * 8 = 16384

__device__ __forceinline__ void bf16x8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

template <bool MX>
__global__ void __launch_bounds__(kQuantXThreads)
    k_quantize_x(const __nv_bfloat16* __restrict__ x, int H, uint8_t* __restrict__ codes,
                 float* __restrict__ scale, uint8_t* __restrict__ sbytes) {
  __shared__ float wmax[kQuantXThreads / 32];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const uint4* row = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H);
  uint2* out = reinterpret_cast<uint2*>(codes + static_cast<size_t>(t) * H);
  const int nc = H / 8;
  uint4 v[kQuantXMaxV];
#pragma unroll
  for (int u = 0; u < kQuantXMaxV; ++u) {
    const int c = tid + u * kQuantXThreads;
    v[u] = c < nc ? __ldg(row + c) : make_uint4(0, 0, 0, 0);
  }
  if (!MX) {
    float m = 0.f;
#pragma unroll
    for (int u = 0; u < kQuantXMaxV; ++u) {
      float f[8];
      bf16x8(v[u], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wmax[tid >> 5] = m;
    __syncthreads();
    m = wmax[0];
#pragma unroll
    for (int w = 1; w < kQuantXThreads / 32; ++w) m = fmaxf(m, wmax[w]);
    const float s = m > 0.f ? __fdiv_rn(m, 448.0f) : 1.0f;
    if (tid == 0) scale[t] = s;
#pragma unroll
    for (int u = 0; u < kQuantXMaxV; ++u) {
      const int c = tid + u * kQuantXThreads;
      if (c < nc) {
        float f[8];
        bf16x8(v[u], f);
        uint32_t q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = cvt_e4m3x2(__fdiv_rn(f[2 * i], s), __fdiv_rn(f[2 * i + 1], s));
        out[c] = make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
      }
    }
  } else {
    // nc % 4 == 0: the four lanes of a 32-column block are in or out together
#pragma unroll
    for (int u = 0; u < kQuantXMaxV; ++u) {
      const int c = tid + u * kQuantXThreads;
      float f[8];
      bf16x8(v[u], f);
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      if (c < nc) {
        const int X = mx_exponent(m);
        uint32_t q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = cvt_e4m3x2(ldexpf(f[2 * i], -X), ldexpf(f[2 * i + 1], -X));
        out[c] = make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
        if ((lane & 3) == 0) sbytes[static_cast<size_t>(t) * (H / 32) + c / 4] = static_cast<uint8_t>(X + 127);
      }
    }
  }
}

}  // namespace moe
