// moe_oracle.cpp - plain CPU oracle of the routed + shared-expert MoE layer.
//
// TEST INFRASTRUCTURE ONLY. This file is the slow, obviously-correct statement
// of what the GPU library computes, in plain C++17: scalar loops over tokens,
// experts, rows and columns in float64, every number format written from its
// definition, no BLAS, no SIMD intrinsics, no code or header shared with the
// CUDA library. It is built into oracle/liboracle.so and called through
// oracle/cpp.py by tests/, __graft_entry__.smoke() and the CPU legs of
// bench.py only; the product path never loads it.
//
// Sources (web pages; sections as printed on them):
//  * vllm-project/vllm PR 65207 "[ROCm][MoE] accumulate shared-expert output
//    in AITER stage 2": "Purpose" commit 1 (routed_scaling_factor folded into
//    the top-k weights of biased_grouped_topk), commit 2 (the shared-expert
//    output is the stage-2 addend, added before the output's one rounding);
//    reviewer measurements "Commits 2 and 3" (moe_sorting without zeroing).
//  * ROCm/aiter PR 6106 "[Triton/Gluon] Add per token scale to a8w8 moe gemm",
//    "Technical Details": a per-row activation scale and a per-expert weight
//    scale multiply the fp32 accumulator before the activation; the stage-1
//    output is quantised after the activation; MXFP8 with BLOCK_K = 32.
//  * vllm-project/vllm PR 56789 (shared_expert_gate as a tiny dot), "Summary"
//    and "Commits": sigmoid of a 1 x K dot with fp32 accumulation, stored in
//    the input dtype.
//  * vllm-project/vllm PR 61503 "Fused heterogeneous MoE", "Overview": the
//    shared expert computed as always-selected routed experts.
//
// Where the pages leave a step open, the reading is stated beside the code:
// tie rules of the two routers, the sort layout, the quantisation points, the
// MX exponent rule and the e2m1 nibble order.
//
// Compiled without fast-math and with -ffp-contract=off: every float operation
// below is one IEEE operation rounded in its own precision.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ------------------------------------------------------------------ formats

// A binary floating-point format: p significant bits (implicit bit included),
// smallest normal exponent emin, largest finite value max_finite; saturate
// clamps overflow to max_finite (the satfinite conversion), otherwise overflow
// gives infinity.
struct Format {
  int p;
  int emin;
  double max_finite;
  bool saturate;
};

const Format kBF16{8, -126, (2.0 - std::ldexp(1.0, -7)) * std::ldexp(1.0, 127), false};
const Format kFP16{11, -14, 65504.0, false};
const Format kFP32{24, -126, (2.0 - std::ldexp(1.0, -23)) * std::ldexp(1.0, 127), false};
// OCP 8-bit E4M3 ("fn": no infinity, one NaN pattern S.1111.111), bias 7,
// largest finite 1.75 * 2^8 = 448.
const Format kE4M3{4, -6, 448.0, true};
constexpr double kE4M3Max = 448.0;

// Nearest value of format f, ties to even. With x = m * 2^e (0.5 <= |m| < 1)
// the binade exponent is e - 1; representable values there are spaced
// 2^(max(e - 1, emin) - (p - 1)) apart (the lower bound gives the subnormal
// spacing). x / quantum is exact (a power of two), and nearbyint in the
// default rounding mode rounds half to even.
double round_to(double x, const Format& f) {
  if (x == 0.0 || std::isnan(x)) return x;
  int e = 0;
  std::frexp(x, &e);
  const int binade = std::max(e - 1, f.emin);
  const double quantum = std::ldexp(1.0, binade - (f.p - 1));
  double q = std::nearbyint(x / quantum) * quantum;
  if (std::fabs(q) > f.max_finite) q = f.saturate ? std::copysign(f.max_finite, q) : std::copysign(INFINITY, q);
  return q;
}

const Format& format_of(int code) {
  switch (code) {
    case 0: return kBF16;
    case 1: return kFP16;
    case 2: return kFP32;
    default: return kE4M3;
  }
}

// Value of an E4M3 byte: sign bit 7, exponent bits 3..6 (bias 7), mantissa
// bits 0..2; exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN.
double e4m3_value(uint8_t c) {
  const double sign = (c & 0x80) ? -1.0 : 1.0;
  const int ef = (c >> 3) & 0xF;
  const int mf = c & 0x7;
  if (ef == 15 && mf == 7) return NAN;
  if (ef == 0) return sign * (mf / 8.0) * std::ldexp(1.0, -6);
  return sign * (1.0 + mf / 8.0) * std::ldexp(1.0, ef - 7);
}

// Value of an E2M1 (FP4) code in bits 0..3: sign bit 3, exponent bits 1..2
// (bias 1), mantissa bit 0; exponent field 0 is subnormal (m/2 * 2^0). All
// sixteen patterns are finite (largest 6).
double e2m1_value(uint8_t c) {
  const double sign = (c & 0x8) ? -1.0 : 1.0;
  const int ef = (c >> 1) & 0x3;
  const int mf = c & 0x1;
  if (ef == 0) return sign * (mf / 2.0);
  return sign * (1.0 + mf / 2.0) * std::ldexp(1.0, ef - 1);
}

// An MX block scale byte b stands for 2^(b - 127).
double ue8m0_value(uint8_t b) { return std::ldexp(1.0, static_cast<int>(b) - 127); }

// bf16 is the upper half of an IEEE binary32.
double bf16_bits_value(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// IEEE binary16 from its fields: sign bit 15, exponent bits 10..14 (bias 15),
// fraction bits 0..9; exponent 0 is subnormal, 31 is infinity / NaN.
double fp16_bits_value(uint16_t b) {
  const double sign = (b & 0x8000) ? -1.0 : 1.0;
  const int ef = (b >> 10) & 0x1F;
  const int mf = b & 0x3FF;
  if (ef == 31) return mf ? NAN : sign * INFINITY;
  if (ef == 0) return sign * (mf / 1024.0) * std::ldexp(1.0, -14);
  return sign * (1.0 + mf / 1024.0) * std::ldexp(1.0, ef - 15);
}

// Shared exponent of one 32-element MX block of E4M3 elements (OCP MX v1.0
// conversion): X = floor(log2(amax)) - 8 (8 = largest E4M3 exponent), taken
// exactly from the binary exponent, clamped to [-127, 127]; an all-zero block
// takes X = -127 (byte 0).
int mx_exponent(double amax) {
  if (!(amax > 0.0)) return -127;
  int e = 0;
  std::frexp(amax, &e);
  const int x = e - 1 - 8;
  return x < -127 ? -127 : (x > 127 ? 127 : x);
}

// Code of a value that is already an E4M3 number (|v| <= 448): the
// non-negative codes 0x00..0x7E increase with their value; the sign bit comes
// from the value's sign, zero included (-0 encodes as 0x80). Returns -1 for a
// value that is not an E4M3 number.
int e4m3_code(double v) {
  const double mag = std::fabs(v);
  for (int c = 0; c <= 0x7E; ++c) {
    if (e4m3_value(static_cast<uint8_t>(c)) == mag) return c | (std::signbit(v) ? 0x80 : 0);
  }
  return -1;
}

double silu(double z) { return z / (1.0 + std::exp(-z)); }

// ------------------------------------------------------------------ operands

// Stored formats of the layer's operands.
enum LayerFmt : int { kFmtBf16 = 0, kFmtFp8 = 1, kFmtMx8 = 2, kFmtMx4 = 3 };

// A stored [rows x cols] matrix (one expert's slice or a whole tensor):
// bf16 bit patterns, E4M3 codes, E4M3 codes with one ue8m0 byte per 32
// columns, or E2M1 codes two per byte (element 2j in bits 0..3 of byte j,
// element 2j + 1 in bits 4..7) with one ue8m0 byte per 32 columns. The fp8
// per-tensor scale is not part of the values: the caller applies it after
// the matrix product.
struct Mat {
  int fmt;
  const uint8_t* data;
  const uint8_t* scale;  // MX: ue8m0 bytes [rows][cols / 32]
  int rows, cols;
};

Mat slice(int fmt, const void* data, const void* scale, int rows, int cols, size_t index) {
  Mat m{fmt, static_cast<const uint8_t*>(data), static_cast<const uint8_t*>(scale), rows, cols};
  const size_t n = static_cast<size_t>(rows) * cols;
  const size_t bytes = fmt == kFmtBf16 ? 2 * n : (fmt == kFmtMx4 ? n / 2 : n);
  m.data += index * bytes;
  if ((fmt == kFmtMx8 || fmt == kFmtMx4) && m.scale) m.scale += index * (n / 32);
  return m;
}

// Decoded row r of m (float64 values).
void decode_row(const Mat& m, int r, double* out) {
  const size_t base = static_cast<size_t>(r) * m.cols;
  for (int c = 0; c < m.cols; ++c) {
    double v = 0.0;
    if (m.fmt == kFmtBf16) {
      uint16_t b;
      std::memcpy(&b, m.data + 2 * (base + c), 2);
      v = bf16_bits_value(b);
    } else if (m.fmt == kFmtFp8) {
      v = e4m3_value(m.data[base + c]);
    } else if (m.fmt == kFmtMx8) {
      v = e4m3_value(m.data[base + c]) * ue8m0_value(m.scale[base / 32 + c / 32]);
    } else {
      const uint8_t byte = m.data[(base + c) / 2];
      const uint8_t code = ((base + c) % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      v = e2m1_value(code) * ue8m0_value(m.scale[base / 32 + c / 32]);
    }
    out[c] = v;
  }
}

double dot(const double* a, const double* b, int n) {
  double s = 0.0;
  for (int i = 0; i < n; ++i) s += a[i] * b[i];
  return s;
}

// ------------------------------------------------------------------ quantisation of h

// Quantisation point of the stage-1 output (values that stage 2 multiplies):
//  0 'bf16' : h stored as bf16;
//  1 'fp8'  : one scale per row, s = fp32(amax / 448) (amax = 0 gives s = 1),
//             q = e4m3_rn(h / s) with saturation, value q * s (ROCm/aiter PR
//             6106, "Technical Details": quantisation fused after the
//             activation, per-row scales);
//  2 'mxfp8': per 32 consecutive columns X = mx_exponent(amax),
//             q = e4m3_rn(h * 2^-X), value q * 2^X (BLOCK_K = 32).
void quantize_h(double* h, int n, int mode) {
  if (mode == 0) {
    for (int i = 0; i < n; ++i) h[i] = round_to(h[i], kBF16);
  } else if (mode == 1) {
    double amax = 0.0;
    for (int i = 0; i < n; ++i) amax = std::max(amax, std::fabs(h[i]));
    const double s = amax > 0.0 ? round_to(amax / kE4M3Max, kFP32) : 1.0;
    for (int i = 0; i < n; ++i) h[i] = round_to(h[i] / s, kE4M3) * s;
  } else {
    for (int b = 0; b + 32 <= n; b += 32) {
      double amax = 0.0;
      for (int i = b; i < b + 32; ++i) amax = std::max(amax, std::fabs(h[i]));
      const double scale = std::ldexp(1.0, mx_exponent(amax));
      for (int i = b; i < b + 32; ++i) h[i] = round_to(h[i] / scale, kE4M3) * scale;
    }
  }
}

// Stage-1 value of one expert on one token, before quantisation:
// acc = W13 . x (2I outputs); a = acc * s_x * s_w13 (scales on the accumulator
// before the activation); h = SiLU(a[:I]) * a[I:]. Rows 0..I-1 of W13 are the
// gate, rows I..2I-1 the up projection. `row` is a scratch row of W13's width.
void expert_hidden(const double* x, const Mat& w13, int I, double s_x, double s_w13, double* h, double* row) {
  std::vector<double> a(2 * static_cast<size_t>(I));
  for (int r = 0; r < 2 * I; ++r) {
    decode_row(w13, r, row);
    a[r] = dot(row, x, w13.cols) * s_x * s_w13;
  }
  for (int i = 0; i < I; ++i) h[i] = silu(a[i]) * a[I + i];
}

// One expert on one token, in the order the pages give: h = expert_hidden;
// h quantised (quantize_h); y = (W2 . h) * s_w2 (a per-row scale of h is
// already inside the dequantised h; MX block scales are inside the decoded
// operands).
// h_raw / h_q (optional, I values each): the stage-1 value before and after
// its quantisation.
void expert_forward(const double* x, const Mat& w13, const Mat& w2, int I, int hmode, double s_x, double s_w13,
                    double s_w2, double* y, double* h_raw = nullptr, double* h_q = nullptr) {
  std::vector<double> h(I), row(std::max(w13.cols, w2.cols));
  expert_hidden(x, w13, I, s_x, s_w13, h.data(), row.data());
  if (h_raw) std::memcpy(h_raw, h.data(), sizeof(double) * I);
  quantize_h(h.data(), I, hmode);
  if (h_q) std::memcpy(h_q, h.data(), sizeof(double) * I);
  for (int n = 0; n < w2.rows; ++n) {
    decode_row(w2, n, row.data());
    y[n] = dot(row.data(), h.data(), I) * s_w2;
  }
}

// ------------------------------------------------------------------ router

// k indices of the largest keys, in selection order: each round takes the
// largest remaining key, ties to the lower index. Keys equal to -inf are
// never taken while a finite key remains.
void topk_desc(const double* key, int n, int k, int* sel) {
  std::vector<char> used(n, 0);
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int i = 0; i < n; ++i) {
      if (used[i]) continue;
      if (best < 0 || key[i] > key[best]) best = i;
    }
    sel[j] = best;
    used[best] = 1;
  }
}

// Softmax top-k. Softmax is strictly increasing in the logit, so the k largest
// probabilities are the k largest fp32 logits (ties to the lower expert
// index). Weights: renormalised exp(l_j - m) / sum_sel exp(l_i - m) * rsf
// (m = largest selected logit), else the full softmax at the selected experts
// times rsf. vllm-project/vllm PR 65207 "Purpose", commit 1: the routed
// scaling factor is applied here, inside the top-k.
void route_softmax(const float* l, int E, int k, int renorm, double rsf, int32_t* ids, double* w) {
  std::vector<double> key(E);
  for (int e = 0; e < E; ++e) key[e] = l[e];
  std::vector<int> sel(k);
  topk_desc(key.data(), E, k, sel.data());
  if (renorm) {
    double sum = 0.0;
    std::vector<double> p(k);
    for (int j = 0; j < k; ++j) {
      p[j] = std::exp(key[sel[j]] - key[sel[0]]);
      sum += p[j];
    }
    for (int j = 0; j < k; ++j) w[j] = p[j] / sum * rsf;
  } else {
    double m = key[0];
    for (int e = 1; e < E; ++e) m = std::max(m, key[e]);
    double sum = 0.0;
    for (int e = 0; e < E; ++e) sum += std::exp(key[e] - m);
    for (int j = 0; j < k; ++j) w[j] = std::exp(key[sel[j]] - m) / sum * rsf;
  }
  for (int j = 0; j < k; ++j) ids[j] = sel[j];
}

// Router score s = sigmoid(l) evaluated in float64 and rounded once to fp32.
float sigmoid_fp32(float l) {
  return static_cast<float>(round_to(1.0 / (1.0 + std::exp(-static_cast<double>(l))), kFP32));
}

// Biased grouped sigmoid top-k (biased_grouped_topk of vllm-project/vllm PR
// 65207, "Purpose", commit 1), with the usual reading of its steps:
//  1. s_e = sigmoid(l_e) as fp32 (or the given fp32 scores);
//  2. choice key c_e = fp32(s_e + b_e) (b = correction bias, 0 if absent);
//  3. group score = fp32 sum of the two largest c of the group (the single c
//     of a one-expert group);
//  4. keep the topk_group groups of highest score (ties: lower group);
//  5. among the experts of kept groups pick k by (c desc, index asc);
//  6. weights from the unbiased scores: s_j / sum_sel s * rsf (renormalised)
//     or s_j * rsf: the routed scaling factor is applied inside the top-k.
void route_grouped(const float* l, const float* s_given, const float* bias, int E, int k, int n_group,
                   int topk_group, int renorm, double rsf, int32_t* ids, double* w) {
  const int gsize = E / n_group;
  std::vector<float> s(E), c(E);
  for (int e = 0; e < E; ++e) {
    s[e] = s_given ? s_given[e] : sigmoid_fp32(l[e]);
    const float b = bias ? bias[e] : 0.0f;
    c[e] = s[e] + b;  // one fp32 addition
  }
  std::vector<double> gscore(n_group);
  for (int g = 0; g < n_group; ++g) {
    if (gsize == 1) {
      gscore[g] = c[g];
      continue;
    }
    float m1 = -INFINITY, m2 = -INFINITY;  // the two largest values
    for (int i = g * gsize; i < (g + 1) * gsize; ++i) {
      if (c[i] > m1) {
        m2 = m1;
        m1 = c[i];
      } else if (c[i] > m2) {
        m2 = c[i];
      }
    }
    const float sc = m1 + m2;  // one fp32 addition
    gscore[g] = sc;
  }
  std::vector<int> kept(topk_group);
  topk_desc(gscore.data(), n_group, topk_group, kept.data());
  std::vector<double> key(E, -INFINITY);
  for (int q = 0; q < topk_group; ++q)
    for (int i = kept[q] * gsize; i < (kept[q] + 1) * gsize; ++i) key[i] = c[i];
  std::vector<int> sel(k);
  topk_desc(key.data(), E, k, sel.data());
  double sum = 0.0;
  for (int j = 0; j < k; ++j) sum += s[sel[j]];
  for (int j = 0; j < k; ++j) {
    ids[j] = sel[j];
    w[j] = (renorm ? s[sel[j]] / sum : static_cast<double>(s[sel[j]])) * rsf;
  }
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

// fmt: 0 bf16, 1 fp16, 2 fp32, 3 e4m3 (saturating).
void orc_round(const double* x, double* out, int64_t n, int fmt) {
  const Format& f = format_of(fmt);
  for (int64_t i = 0; i < n; ++i) out[i] = round_to(x[i], f);
}

void orc_e4m3_decode(const uint8_t* c, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(c[i]);
}

void orc_e2m1_decode(const uint8_t* c, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e2m1_value(c[i] & 0xF);
}

void orc_ue8m0_decode(const uint8_t* b, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = ue8m0_value(b[i]);
}

void orc_bf16_decode(const uint16_t* b, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_bits_value(b[i]);
}

void orc_fp16_decode(const uint16_t* b, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = fp16_bits_value(b[i]);
}

void orc_mx_exponent(const double* amax, int32_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = mx_exponent(amax[i]);
}

// Codes of values that are E4M3 numbers; returns the index of the first value
// that is not, or -1.
int64_t orc_e4m3_encode(const double* v, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) {
    const int c = e4m3_code(v[i]);
    if (c < 0) return i;
    out[i] = static_cast<uint8_t>(c);
  }
  return -1;
}

// Decoded stored matrix [rows x cols] (fmt: 0 bf16 bits, 1 e4m3 codes, 2 MX
// e4m3 + ue8m0, 3 MX e2m1 two per byte + ue8m0).
void orc_decode_matrix(int fmt, const void* data, const void* scale, int64_t rows, int cols, double* out) {
  const Mat m{fmt, static_cast<const uint8_t*>(data), static_cast<const uint8_t*>(scale), static_cast<int>(rows),
              cols};
  for (int64_t r = 0; r < rows; ++r) decode_row(m, static_cast<int>(r), out + r * cols);
}

// Quantisation of the layer's bf16 activations x [T, H] (given as float64
// values of bf16 numbers) to the stage-1 operand formats (ROCm/aiter PR 6106,
// "Technical Details": per-token scales; MXFP8 with BLOCK_K = 32).
// mode 0 'fp8': s = fp32(amax / 448) per row (amax = 0 gives s = 1); each
//   code is e4m3_rn(fp32(x / s)), the quotient an IEEE fp32 division (the
//   precision the kernel decides in), then one saturating E4M3 rounding;
//   scale_out is float [T].
// mode 1 'mxfp8': per 32 columns X = mx_exponent(amax), byte X + 127, codes
//   e4m3_rn(x * 2^-X) (exact scaling, then one rounding); scale_out is
//   uint8 [T, H/32].
void orc_quantize_activations(const double* x, int T, int H, int mode, uint8_t* codes, void* scale_out) {
  for (int t = 0; t < T; ++t) {
    const double* xr = x + static_cast<size_t>(t) * H;
    uint8_t* q = codes + static_cast<size_t>(t) * H;
    if (mode == 0) {
      double amax = 0.0;
      for (int h = 0; h < H; ++h) amax = std::max(amax, std::fabs(xr[h]));
      const double s = amax > 0.0 ? round_to(amax / kE4M3Max, kFP32) : 1.0;
      const float sf = static_cast<float>(s);
      for (int h = 0; h < H; ++h) {
        const float quot = static_cast<float>(xr[h]) / sf;  // IEEE fp32 division
        q[h] = static_cast<uint8_t>(e4m3_code(round_to(quot, kE4M3)));
      }
      static_cast<float*>(scale_out)[t] = sf;
    } else {
      uint8_t* sb = static_cast<uint8_t*>(scale_out) + static_cast<size_t>(t) * (H / 32);
      for (int b = 0; b < H / 32; ++b) {
        double amax = 0.0;
        for (int i = 32 * b; i < 32 * b + 32; ++i) amax = std::max(amax, std::fabs(xr[i]));
        const int X = mx_exponent(amax);
        for (int i = 32 * b; i < 32 * b + 32; ++i)
          q[i] = static_cast<uint8_t>(e4m3_code(round_to(xr[i] * std::ldexp(1.0, -X), kE4M3)));
        sb[b] = static_cast<uint8_t>(X + 127);
      }
    }
  }
}

// quantize_h on rows of h [n_rows, n] in place (mode 0 bf16, 1 fp8, 2 mxfp8).
void orc_quantize_h(double* h, int64_t n_rows, int n, int mode) {
  for (int64_t r = 0; r < n_rows; ++r) quantize_h(h + r * n, n, mode);
}

void orc_silu(const double* z, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = silu(z[i]);
}

// Router logits x . W_r in one fixed fp32 order (float result [T, E]). The
// pages give no arithmetic for the router linear (vllm-project/vllm PR 65207,
// "Purpose", passes the gating output to biased_grouped_topk); this order is
// the one the fused router defines, so that routing made from these logits
// can be compared bit for bit: with c = H / chunks, for each chunk j the fp32
// running sum of x_h * w_h over h = jc .. jc + c - 1 in index order, then the
// chunk sums added in chunk order, then + logit_bias[e] (fp32) when given.
// Every addition rounds to nearest fp32; products of bf16 / fp16 inputs are
// exact in fp32 (checked: returns 1 if a product is not, else 0).
int orc_router_logits(const double* x, const double* w_r, const float* bias, int T, int H, int E, int chunks,
                      float* out) {
  const int c = H / chunks;
  int inexact = 0;
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      float total = 0.0f;
      for (int j = 0; j < chunks; ++j) {
        float acc = 0.0f;
        for (int h = j * c; h < (j + 1) * c; ++h) {
          const double prod = x[static_cast<size_t>(t) * H + h] * w_r[static_cast<size_t>(h) * E + e];
          const float p32 = static_cast<float>(prod);
          if (static_cast<double>(p32) != prod) inexact = 1;
          acc = acc + p32;
        }
        total = (j == 0) ? acc : total + acc;
      }
      if (bias) total = total + bias[e];
      out[static_cast<size_t>(t) * E + e] = total;
    }
  }
  return inexact;
}

void orc_router_softmax_topk(const float* logits, int T, int E, int k, int renorm, double rsf, int32_t* ids,
                             double* w) {
  for (int t = 0; t < T; ++t)
    route_softmax(logits + static_cast<size_t>(t) * E, E, k, renorm, rsf, ids + static_cast<size_t>(t) * k,
                  w + static_cast<size_t>(t) * k);
}

void orc_sigmoid_fp32(const float* l, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = sigmoid_fp32(l[i]);
}

// Scores whose float64 sigmoid lies within 2^margin_log2 (relative) of an
// fp32 rounding midpoint: only these can round to different fp32 values on
// two machines whose float64 exp differs by a few ulps. other[i] receives the
// fp32 neighbour on the other side of the float64 value from the rounding
// taken by sigmoid_fp32 (the rounding another machine may take).
void orc_sigmoid_hazards(const float* l, int64_t n, int margin_log2, uint8_t* mask, float* other) {
  for (int64_t i = 0; i < n; ++i) {
    const double v = 1.0 / (1.0 + std::exp(-static_cast<double>(l[i])));
    const double r = round_to(v, kFP32);
    int e = 0;
    std::frexp(r, &e);
    const double half_ulp = std::ldexp(1.0, e - 1 - 24);
    const double mid = v >= r ? r + half_ulp : r - half_ulp;
    mask[i] = std::fabs(v - mid) < std::fabs(v) * std::ldexp(1.0, margin_log2) ? 1 : 0;
    const float rf = static_cast<float>(r);
    other[i] = v >= r ? std::nextafter(rf, INFINITY) : std::nextafter(rf, -INFINITY);
  }
}

// scores: NULL, or fp32 scores [T, E] that replace step 1 (used to evaluate
// the other rounding of a hazard score).
void orc_router_grouped_topk(const float* logits, const float* scores, const float* bias, int T, int E, int k,
                             int n_group, int topk_group, int renorm, double rsf, int32_t* ids, double* w) {
  for (int t = 0; t < T; ++t)
    route_grouped(logits + static_cast<size_t>(t) * E, scores ? scores + static_cast<size_t>(t) * E : nullptr, bias,
                  E, k, n_group, topk_group, renorm, rsf, ids + static_cast<size_t>(t) * k,
                  w + static_cast<size_t>(t) * k);
}

// Upper bound of the padded sorted length: every expert may add up to
// block_m - 1 padding slots.
int64_t orc_sorted_capacity(int T, int k, int E, int block_m) {
  return static_cast<int64_t>(T) * k + static_cast<int64_t>(E) * (block_m - 1);
}

// Stable counting sort of the flat slots f = t*k + j by expert (reading:
// segments in expert order 0..E-1; ascending f inside a segment; each segment
// padded to a multiple of block_m with the sentinel T*k; an expert with no
// slot gets no block; offsets = exclusive prefix sum of the padded sizes;
// block_expert[b] = owner of block b; num_padded = offsets[E]).
// vllm-project/vllm PR 65207, "Commits 2 and 3": moe_sorting without zeroing
// the output. sorted_ids needs orc_sorted_capacity entries, block_expert
// that divided by block_m. Returns 0, or -1 for an expert id out of range.
int orc_align_sort(const int32_t* ids, int T, int k, int E, int block_m, int32_t* sorted_ids,
                   int32_t* block_expert, int32_t* counts, int32_t* offsets, int32_t* num_padded) {
  const int n = T * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int f = 0; f < n; ++f) {
    if (ids[f] < 0 || ids[f] >= E) return -1;
    counts[ids[f]] += 1;
  }
  offsets[0] = 0;
  int nb = 0;
  for (int e = 0; e < E; ++e) {
    const int padded = (counts[e] + block_m - 1) / block_m * block_m;
    int pos = offsets[e];
    for (int f = 0; f < n; ++f)
      if (ids[f] == e) sorted_ids[pos++] = f;
    for (; pos < offsets[e] + padded; ++pos) sorted_ids[pos] = n;
    for (int b = 0; b < padded / block_m; ++b) block_expert[nb++] = e;
    offsets[e + 1] = offsets[e] + padded;
  }
  *num_padded = offsets[E];
  return 0;
}

// Shared-expert gate (vllm-project/vllm PR 56789, "Summary" and "Commits"):
// g_t = round_to(out format)( sigmoid( sum_h x[t,h] * w[h] ) ), the dot and
// the sigmoid in float64, one rounding at the store. out_fmt: 0 bf16, 1 fp16.
void orc_shared_gate(const double* x, const double* w, int T, int K, int apply_sigmoid, int out_fmt, double* g) {
  for (int t = 0; t < T; ++t) {
    const double d = dot(x + static_cast<size_t>(t) * K, w, K);
    const double v = apply_sigmoid ? 1.0 / (1.0 + std::exp(-d)) : d;
    g[t] = round_to(v, format_of(out_fmt));
  }
}

// One expert on one token from decoded float64 operands (x [H], w13 [2I, H],
// w2 [H, I]); hmode as quantize_h. Writes y [H] and, if h is not NULL, the
// unquantised stage-1 value h [I].
void orc_expert_forward(const double* x, const double* w13, const double* w2, int H, int I, int hmode, double s_x,
                        double s_w13, double s_w2, double* y, double* h_out) {
  std::vector<double> a(2 * static_cast<size_t>(I)), h(I);
  for (int r = 0; r < 2 * I; ++r) a[r] = dot(w13 + static_cast<size_t>(r) * H, x, H) * s_x * s_w13;
  for (int i = 0; i < I; ++i) h[i] = silu(a[i]) * a[I + i];
  if (h_out) std::memcpy(h_out, h.data(), sizeof(double) * I);
  quantize_h(h.data(), I, hmode);
  for (int n = 0; n < H; ++n) y[n] = dot(w2 + static_cast<size_t>(n) * I, h.data(), I) * s_w2;
}

// The layer's inputs, as stored (the same bytes the GPU library reads).
struct OrcLayer {
  int T, H, E, top_k, I, Is;
  int fmt;    // 0 bf16, 1 fp8 (per-token x scale, per-expert per-matrix W scale), 2 mxfp8, 3 mxfp4 weights
  int route;  // 0 softmax, 1 biased grouped sigmoid
  int n_group, topk_group, renormalize;
  double rsf;
  int shared_gate;           // 1: gated by sigmoid(x . w_gate)
  const float* logits;       // [T, E]
  const float* corr_bias;    // [E] or NULL
  const void* x;             // bf16 bits [T, H] or e4m3 codes [T, H]
  const void* x_scale;       // fp8: double [T] (the fp32 scales, widened); MX: ue8m0 [T, H/32]
  const uint16_t* w_gate;    // bf16 bits [H] or NULL
  const void* w13;           // [E, 2I, H] (mxfp4: [E, 2I, H/2])
  const void* w13_scale;     // fp8: double [E]; MX: ue8m0 [E, 2I, H/32]
  const void* w2;            // [E, H, I]
  const void* w2_scale;      // fp8: double [E]; MX: ue8m0 [E, H, I/32]
  const void* w13s;          // [2Is, H]
  const void* w13s_scale;    // fp8: double [1]; MX: ue8m0 [2Is, H/32]
  const void* w2s;           // [H, Is]
  const void* w2s_scale;     // fp8: double [1]; MX: ue8m0 [H, Is/32]
};

// Forward pass of one routed + shared-expert MoE layer, token by token.
// Routing (ids [T, k], weights [T, k]) is computed for every token; the other
// outputs for the listed tokens only (n_tok rows each, in list order):
//   g_t      = gate(x_t) if the layer has a shared gate, else 1
//   addend_t = bf16( g_t * SharedExpert(x_t) )
//   routed_t = sum over j = 0..k-1 of w_j * Expert_{ids_j}(x_t)
//   out_t    = bf16( addend_t + routed_t )
// (vllm-project/vllm PR 65207 "Purpose": the shared output is the addend of
// stage 2, so the routed sum and the addend meet before the one bf16
// rounding; commit 1: the routed scaling factor is already inside w.)
// shared_fused: the shared expert as always-selected routed experts
// (vllm-project/vllm PR 61503 "Fused heterogeneous MoE", "Overview"): cut into
// m = ceil(Is / I) pieces of I intermediate features (gate rows v*I .. with
// their up rows and W2 columns, zero-padded past Is), each computed like a
// routed expert (its h quantised on its own I columns) with weight g_t; then
// addend_t is the unrounded sum of the pieces and out_t = bf16(routed_t +
// addend_t). MXFP4 layers (fmt 3) hold e2m1 weights and MXFP8 x and h.
// Tokens run in parallel (OpenMP, `threads` threads; 0 = the default); each
// token's arithmetic is the same whatever the thread count.
// Returns 0, or -1 for an invalid argument.
// orc_moe_layer with optional outputs of the stage-1 values: h_raw_r / h_q_r
// [n_tok, k, I] (each routed slot's h before and after its quantisation) and
// h_raw_s / h_q_s [n_tok, Is] (the shared expert's; not filled in fused
// mode). Any of them may be NULL.
int orc_moe_layer_h(const OrcLayer* L, const int32_t* tokens, int n_tok, int shared_fused, int threads, int32_t* ids,
                    double* wts, double* gate, double* addend, double* routed, double* out, double* h_raw_r,
                    double* h_q_r, double* h_raw_s, double* h_q_s);

int orc_moe_layer(const OrcLayer* L, const int32_t* tokens, int n_tok, int shared_fused, int threads, int32_t* ids,
                  double* wts, double* gate, double* addend, double* routed, double* out) {
  return orc_moe_layer_h(L, tokens, n_tok, shared_fused, threads, ids, wts, gate, addend, routed, out, nullptr,
                         nullptr, nullptr, nullptr);
}

int orc_moe_layer_h(const OrcLayer* L, const int32_t* tokens, int n_tok, int shared_fused, int threads, int32_t* ids,
                    double* wts, double* gate, double* addend, double* routed, double* out, double* h_raw_r,
                    double* h_q_r, double* h_raw_s, double* h_q_s) {
  const int T = L->T, H = L->H, E = L->E, k = L->top_k, I = L->I, Is = L->Is;
  if (T < 1 || H < 1 || E < 1 || k < 1 || k > E || I < 1 || Is < 1 || L->fmt < 0 || L->fmt > 3) return -1;
  const int fmt = L->fmt;
  const bool mx = fmt == kFmtMx8 || fmt == kFmtMx4;
  const int afmt = mx ? kFmtMx8 : fmt;  // activations (MXFP4 layers: MXFP8)
  const int hmode = fmt == kFmtBf16 ? 0 : (fmt == kFmtFp8 ? 1 : 2);

  for (int t = 0; t < T; ++t) {
    if (L->route == 0)
      route_softmax(L->logits + static_cast<size_t>(t) * E, E, k, L->renormalize, L->rsf, ids + static_cast<size_t>(t) * k,
                    wts + static_cast<size_t>(t) * k);
    else
      route_grouped(L->logits + static_cast<size_t>(t) * E, nullptr, L->corr_bias, E, k, L->n_group, L->topk_group,
                    L->renormalize, L->rsf, ids + static_cast<size_t>(t) * k, wts + static_cast<size_t>(t) * k);
  }
  for (int i = 0; i < n_tok; ++i)
    if (tokens[i] < 0 || tokens[i] >= T) return -1;

  auto scale_of = [&](const void* p, int e) -> double {
    return fmt == kFmtFp8 ? static_cast<const double*>(p)[e] : 1.0;
  };
  const Mat xm = slice(afmt, L->x, L->x_scale, T, H, 0);
  const Mat w13s = slice(fmt, L->w13s, L->w13s_scale, 2 * Is, H, 0);
  const Mat w2s = slice(fmt, L->w2s, L->w2s_scale, H, Is, 0);
  const double s13s = scale_of(L->w13s_scale, 0), s2s = scale_of(L->w2s_scale, 0);

  // fused mode: the shared expert's pieces, decoded once into float64
  const int m = (Is + I - 1) / I;
  std::vector<double> p13, p2;
  if (shared_fused) {
    p13.assign(static_cast<size_t>(m) * 2 * I * H, 0.0);
    p2.assign(static_cast<size_t>(m) * H * I, 0.0);
    std::vector<double> row(std::max(H, Is));
    for (int v = 0; v < m; ++v) {
      const int lo = v * I, hi = std::min((v + 1) * I, Is);
      for (int r = lo; r < hi; ++r) {
        decode_row(w13s, r, row.data());  // gate row
        std::memcpy(&p13[(static_cast<size_t>(v) * 2 * I + (r - lo)) * H], row.data(), sizeof(double) * H);
        decode_row(w13s, Is + r, row.data());  // its up row
        std::memcpy(&p13[(static_cast<size_t>(v) * 2 * I + I + (r - lo)) * H], row.data(), sizeof(double) * H);
      }
      for (int n = 0; n < H; ++n) {
        decode_row(w2s, n, row.data());
        for (int c = lo; c < hi; ++c) p2[(static_cast<size_t>(v) * H + n) * I + (c - lo)] = row[c];
      }
    }
  }

  int status = 0;
#ifdef _OPENMP
  const int nthr = threads > 0 ? threads : omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthr)
#endif
  for (int i = 0; i < n_tok; ++i) {
    const int t = tokens[i];
    std::vector<double> x(H), y(H), wg(H), acc(H, 0.0);
    decode_row(xm, t, x.data());
    const double s_x = fmt == kFmtFp8 ? static_cast<const double*>(L->x_scale)[t] : 1.0;

    // gate (only gated layers carry one; bf16 x, stored in x's dtype)
    double g = 1.0;
    if (L->shared_gate && L->w_gate) {
      for (int h = 0; h < H; ++h) wg[h] = bf16_bits_value(L->w_gate[h]);
      const double d = dot(x.data(), wg.data(), H);
      g = round_to(1.0 / (1.0 + std::exp(-d)), fmt == kFmtBf16 ? kBF16 : kFP16);
    }
    gate[i] = g;

    // shared expert -> addend (fused: the unrounded sum over its pieces)
    double* add = addend + static_cast<size_t>(i) * H;
    if (shared_fused) {
      for (int n = 0; n < H; ++n) add[n] = 0.0;
      for (int v = 0; v < m; ++v) {
        // a piece is a float64 matrix: decode_row over a bf16 view is not
        // needed, so evaluate the expert from the decoded piece directly
        std::vector<double> a(2 * static_cast<size_t>(I)), hh(I);
        const double* P13 = &p13[static_cast<size_t>(v) * 2 * I * H];
        const double* P2 = &p2[static_cast<size_t>(v) * H * I];
        for (int r = 0; r < 2 * I; ++r) a[r] = dot(P13 + static_cast<size_t>(r) * H, x.data(), H) * s_x * s13s;
        for (int c = 0; c < I; ++c) hh[c] = silu(a[c]) * a[I + c];
        quantize_h(hh.data(), I, hmode);
        for (int n = 0; n < H; ++n) add[n] += g * (dot(P2 + static_cast<size_t>(n) * I, hh.data(), I) * s2s);
      }
    } else {
      expert_forward(x.data(), w13s, w2s, Is, hmode, s_x, s13s, s2s, y.data(),
                     h_raw_s ? h_raw_s + static_cast<size_t>(i) * Is : nullptr,
                     h_q_s ? h_q_s + static_cast<size_t>(i) * Is : nullptr);
      for (int n = 0; n < H; ++n) add[n] = round_to(g * y[n], kBF16);
    }

    // routed experts, j = 0..k-1
    for (int j = 0; j < k; ++j) {
      const int e = ids[static_cast<size_t>(t) * k + j];
      const Mat w13 = slice(fmt, L->w13, L->w13_scale, 2 * I, H, e);
      const Mat w2 = slice(fmt, L->w2, L->w2_scale, H, I, e);
      const size_t hoff = (static_cast<size_t>(i) * k + j) * I;
      expert_forward(x.data(), w13, w2, I, hmode, s_x, scale_of(L->w13_scale, e), scale_of(L->w2_scale, e),
                     y.data(), h_raw_r ? h_raw_r + hoff : nullptr, h_q_r ? h_q_r + hoff : nullptr);
      const double wj = wts[static_cast<size_t>(t) * k + j];
      for (int n = 0; n < H; ++n) acc[n] += wj * y[n];
    }
    double* rt = routed + static_cast<size_t>(i) * H;
    double* o = out + static_cast<size_t>(i) * H;
    for (int n = 0; n < H; ++n) {
      rt[n] = acc[n];
      o[n] = round_to(add[n] + acc[n], kBF16);
    }
  }
  return status;
}

// Units of the layer's work, one expert call each: unit u is the routed
// expert of slot uj[u] of token ut[u] (ids: the routing [T, k]), or, for
// uj[u] = -1, the token's shared expert (ungated). y receives [n, H]. Units run
// in parallel (OpenMP); this is the CPU reference's unit of timing.
int orc_layer_units(const OrcLayer* L, const int32_t* ids, const int32_t* ut, const int32_t* uj, int n, int threads,
                    double* y) {
  const int T = L->T, H = L->H, k = L->top_k, I = L->I, Is = L->Is;
  const int fmt = L->fmt;
  if (fmt < 0 || fmt > 3) return -1;
  const bool mx = fmt == kFmtMx8 || fmt == kFmtMx4;
  const int afmt = mx ? kFmtMx8 : fmt;
  const int hmode = fmt == kFmtBf16 ? 0 : (fmt == kFmtFp8 ? 1 : 2);
  auto scale_of = [&](const void* p, int e) -> double {
    return fmt == kFmtFp8 ? static_cast<const double*>(p)[e] : 1.0;
  };
  const Mat xm = slice(afmt, L->x, L->x_scale, T, H, 0);
  for (int u = 0; u < n; ++u)
    if (ut[u] < 0 || ut[u] >= T || uj[u] < -1 || uj[u] >= k) return -1;
#ifdef _OPENMP
  const int nthr = threads > 0 ? threads : omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthr)
#endif
  for (int u = 0; u < n; ++u) {
    const int t = ut[u];
    std::vector<double> x(H);
    decode_row(xm, t, x.data());
    const double s_x = fmt == kFmtFp8 ? static_cast<const double*>(L->x_scale)[t] : 1.0;
    double* yu = y + static_cast<size_t>(u) * H;
    if (uj[u] < 0) {
      const Mat w13 = slice(fmt, L->w13s, L->w13s_scale, 2 * Is, H, 0);
      const Mat w2 = slice(fmt, L->w2s, L->w2s_scale, H, Is, 0);
      expert_forward(x.data(), w13, w2, Is, hmode, s_x, scale_of(L->w13s_scale, 0), scale_of(L->w2s_scale, 0), yu);
    } else {
      const int e = ids[static_cast<size_t>(t) * k + uj[u]];
      const Mat w13 = slice(fmt, L->w13, L->w13_scale, 2 * I, H, e);
      const Mat w2 = slice(fmt, L->w2, L->w2_scale, H, I, e);
      expert_forward(x.data(), w13, w2, I, hmode, s_x, scale_of(L->w13_scale, e), scale_of(L->w2_scale, e), yu);
    }
  }
  return 0;
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
