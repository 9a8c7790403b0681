// gemm.cuh - grouped GEMMs of the MoE layer on tcgen05 tensor cores.
//
// Stage 1 (gate_up + SiLU-and-mul) and stage 2 (down + weighted scatter-reduce
// + shared-expert addend) share one persistent, warp-specialised kernel:
//
//   warp 0      TMA producer: per pipeline stage, the weight tile (128 rows
//               x 128 K-bytes per K atom; two atoms per stage up to 128-token
//               tiles) and, with one producer warp, the token tile (BN rows x
//               the same K-bytes). Stage-1 token rows come from a copy of x in
//               sorted order (k_stage1_prep). Block-scaled kernels add the
//               stage's 512-byte scale tiles.
//   warp 2      second producer (64+-token tiles, block-scaled kernels): the
//               token tile and its scale tiles, warp 0 keeping the weights'.
//   warp 1      TMEM allocator + MMA issuer (one thread): tcgen05.mma with the
//               weights as A (M = 128) and the tokens as B (N = BN), fp32
//               accumulator in TMEM, a ring of 2 to 4 across tiles.
//   warp 3      block-scaled kernels: copies each stage's scale tiles into
//               TMEM (tcgen05.cp) for the block-scaled MMA.
//   then        epilogue, one or two warpgroups taking alternate tiles:
//               tcgen05.ld of the accumulator, then
//               stage 1: operand scales, SiLU(gate) * up, store h in the
//               stage-2 operand format (bf16, e4m3 with a per-row scale, or
//               MXFP8 with a scale per 32 columns);
//               stage 2: scales x top-k weight, fp32 red.add into the token
//               row, and the CTA that brings a token's last slot adds the
//               addend, rounds once to bf16, writes out and re-zeroes.
//
// Weights on the MMA M side ("swap AB") keep the 128-row MMA fully used even
// when an expert holds a handful of tokens (decode), so the kernel streams
// weights at the rate the pipeline depth allows.
//
// Sources: vllm-project/vllm PR 65207 "Purpose" (commit 2: the shared-expert
// output is the stage-2 addend, accumulated in the GEMM2 epilogue; commit 1:
// the routed scale is already inside the top-k weights); ROCm/aiter PR 6106
// "Technical Details" (per-row activation scale x per-expert weight scale on
// the fp32 accumulator, before activation; rows follow the gather index;
// MXFP8 with BLOCK_K = 32).
#pragma once
#include "ptx.cuh"

namespace moe {

constexpr int kTileM = 128;       // weight rows per tile = MMA M
constexpr int kTileKBytes = 128;  // K bytes of one K atom = one 128-byte swizzle row
constexpr int kEpiThreads = 128;  // one epilogue warpgroup
constexpr int kSfTile = 512;      // bytes of one MXFP8 scale tile (128 rows x 4 K blocks)
constexpr int kSfSlots = 4;       // pairs: TMEM ring of scale tiles (8 columns per K atom: A then B)
constexpr int kFinBatch = 8;      // stage-2 finalisation: token columns per batch of loads
// kMx4: MXFP4 weights (e2m1, two per byte in memory; the tensor map unpacks
// each 16-element group into 16 bytes of shared memory, so a weight tile has
// the MXFP8 tile's shape there) against MXFP8 tokens, in the same block-scaled
// MMA with A declared e2m1.
enum Kind : int { kBf16 = 0, kFp8 = 1, kMx8 = 2, kMx4 = 3 };

__host__ __device__ constexpr bool is_mx(int kind) { return kind == kMx8 || kind == kMx4; }

// Epilogue warpgroups per CTA: two groups take alternate tiles so a tile's
// epilogue - atomics to L2 included - overlaps the next tiles' main loop, over
// a ring of TMEM accumulators (two per group where they fit). 256-token tiles
// fill TMEM with two accumulators and one group. Block-scaled stage 1 keeps
// one group from 64 tokens on (registers for the held h values); block-scaled
// stage 2 at 128 tokens shares three accumulators between its two groups, the
// scale ring taking TMEM's last columns.
//
// Copy issue: a thread needs about 130 cycles to issue one TMA copy, so where
// a stage holds four copies (block-scaled kernels: two operand tiles and their
// scale tiles) or a large token tile (64+ tokens), two producer warps share
// them: warp 0 loads the weight tile (and its MX scale tile), warp 2 the token
// tile (and its scale tile); both arm the stage's `full` barrier with their
// own bytes. The block-scaled kernels also give the two TMEM copies of a
// stage's scale tiles to warp 3, so that the MMA thread issues MMAs only.
template <int BN, int KIND, bool S1>
struct EpiCfg {
  static constexpr bool kMxWide = is_mx(KIND) && BN == 128 && !S1;
  static constexpr int kGroups = (is_mx(KIND) ? (BN <= 32 || !S1) : BN <= 128) ? 2 : 1;
  static constexpr int kAcc = kMxWide ? 3 : 2 * kGroups;
  static constexpr bool kSplit = BN >= 64 || is_mx(KIND);  // two producer warps
  static constexpr bool kSfWarp = is_mx(KIND);               // warp 3 copies scale tiles (one-CTA tiles)
  static constexpr int kLead = kSfWarp ? 128 : kSplit ? 96 : 64;  // threads before the epilogue warps
  static constexpr int kThreads = kLead + kEpiThreads * kGroups;
};

// 128-byte K atoms (one swizzle row of every operand row) per pipeline stage.
// Every stage costs each role a fixed amount of issue - a barrier wait, an
// expect-tx arrival, a commit, the loop: 200-500 cycles per role, measured -
// besides its copies and MMAs, and those fixed costs set the pace of these
// kernels. So a stage carries two atoms (two copies per operand into
// consecutive swizzle blocks, one scale-tile copy per operand for both, eight
// MMAs per barrier round trip). Measured against one atom per stage: MXFP8
// prefill layer 5178 -> 4278 us, MXFP4 prefill 4810 -> 3705 us, fp8 a8w8
// 506 -> 416 us, MXFP4 decode 101.6 -> 88.6 us, bf16 decode 150.1 -> 145.5
// us, fp8 decode (T = 32) 181.8 -> 177.8 us. 256-token tiles keep one atom:
// two would leave two stages of shared memory.
template <int BN, int KIND, bool PAIR>
__host__ __device__ constexpr int atoms_for() {
  return BN <= 128 ? 2 : 1;
}

struct GemmArgs {
  const int32_t* sorted_ids;  // nullptr: identity routing (row r = token r, expert 0)
  const int32_t* block_expert;
  const int32_t* num_padded;
  int identity_rows;  // identity routing: rows padded to BN
  int cap_blocks;     // token blocks the sorted buffers can hold
  int T, top_k, H, I;
  int E;       // experts the weight tensors hold (block_expert entries are checked against it)
  int n_mt;    // weight tiles per token block
  int num_kb;  // K stages per tile
  // stage 1 outputs
  __nv_bfloat16* h;  // bf16: h [rows, I]
  float* h32;        // fp8: the unquantised h [rows, I] in fp32 (workspace)
  float* h_amax;     // fp8: per-tile row amax [n_mt][rows_cap] (workspace)
  int* blk_cnt;      // fp8: finished weight tiles per token block (workspace, self-cleaning)
  int quant_phase;   // fp8: 1 = rows are quantised after a grid barrier by every warp (cooperative
                     // launch); 0 = by the epilogue that finishes a token block's last tile
  unsigned* grid_bar;  // fp8 quant_phase: arrival count, generation (workspace, self-cleaning)
  uint8_t* hq;       // fp8 / MXFP8: e4m3 codes of h [rows, I]
  int rows_cap;
  const float* x_scale;  // fp8: [T]
  const float* w_scale;  // fp8: [E] (stage 1: W13, stage 2: W2)
  float* h_scale;        // fp8: per-row scale of h [rows] (stage-1 output, stage-2 input)
  // MXFP8
  const uint8_t* wsf;  // weight scale tiles [E][n_mt][num_kb][512] (moe_mx_pack_weight_scales)
  uint8_t* hsf;        // h scale tiles [blocks][I/128][512] (stage-1 output, stage-2 input)
  const uint8_t* xsf;  // stage 1: token scale tiles [blocks][H/128][512] (k_stage1_prep)
  // stage 2
  const void* weights;  // [T*k] or nullptr
  int weights_dtype;    // 4 = f32, 0 = bf16, 1 = fp16
  const __nv_bfloat16* addend;
  float* ws;
  int* counters;
  __nv_bfloat16* out;
};

// PAIR: the tile is computed by a CTA pair (one MMA of M = 256); each CTA
// holds its 128 weight rows and half of the BN token rows of a stage.
template <int BN, int STAGES, int KIND, bool S1, bool PAIR = false>
struct GemmSmem {
  static constexpr bool kMx = is_mx(KIND);
  static constexpr int kGroups = EpiCfg<BN, KIND, S1>::kGroups;
  static constexpr int kAcc = EpiCfg<BN, KIND, S1>::kAcc;
  static constexpr int kAtoms = atoms_for<BN, KIND, PAIR>();
  static constexpr int kAtomA = kTileM * kTileKBytes;                 // one K atom of the weight tile
  static constexpr int kAtomB = (PAIR ? BN / 2 : BN) * kTileKBytes;  // one K atom of the token tile
  static constexpr int kABytes = kAtomA * kAtoms;
  static constexpr int kBBytes = kAtomB * kAtoms;
  static constexpr int kSfBytes = kMx ? 2 * kSfTile * kAtoms : 0;  // A scale tiles, then B's, one per atom
  static constexpr int kStageBytes = kABytes + kBBytes + kSfBytes;
  static_assert(kStageBytes % 1024 == 0, "stages start on 1024-byte swizzle boundaries");
  static constexpr int kBarOffset = STAGES * kStageBytes;
  // scale tiles in TMEM: copied by warp 3 into slot `stage` (one-CTA tiles;
  // 8 columns per atom: the A tiles, then the B tiles), else by the MMA
  // thread into a ring of kSfSlots (pairs; warp 3 idles)
  static constexpr bool kSfWarp = EpiCfg<BN, KIND, S1>::kSfWarp && !PAIR;
  static constexpr int kSfRing = kSfWarp ? STAGES : kSfSlots;
  // full[S], empty[S], acc_full[A], acc_empty[A], drain, then sf_full[S] with the scale-copy warp
  static constexpr int kNumBars = 2 * STAGES + 2 * kAcc + 1 + (kSfWarp ? STAGES : 0);
  static constexpr int kMiscOffset = kBarOffset + kNumBars * 8;
  // tmem slot, abort flag, grid-barrier flag, pad word; then per epilogue group: ok flag +
  // 3 pad words, tok[BN], wgt[BN], last[BN], amax_part[4][BN]
  static constexpr int kGroupWords = 4 + 7 * BN;
  static constexpr int kMiscBytes = 16 + kGroups * kGroupWords * 4;
  static constexpr int kBytes = kMiscOffset + kMiscBytes + 1024;  // + alignment slack
  static constexpr int kAccCols = kAcc * BN;
  static constexpr int kSfCol = kAccCols;  // first column of the scale ring
  static constexpr int kColsNeeded = kAccCols + (kMx ? 8 * kAtoms * kSfRing : 0);
  static constexpr int kTmemCols = kColsNeeded <= 32 ? 32 : kColsNeeded <= 64 ? 64 : kColsNeeded <= 128 ? 128
                                   : kColsNeeded <= 256 ? 256 : 512;
  static_assert(kColsNeeded <= 512, "TMEM");
};

__device__ __forceinline__ float load_weight(const void* w, int dt, int f) {
  if (w == nullptr) return 1.0f;
  if (dt == 4) return static_cast<const float*>(w)[f];
  if (dt == 0) return __bfloat162float(static_cast<const __nv_bfloat16*>(w)[f]);
  return __half2float(static_cast<const __half*>(w)[f]);
}

// Expert of token block `blk` (0 with identity routing). An entry outside
// [0, E) - a stale or foreign block_expert buffer - records kErrBlockExpert
// and reads as expert 0, so that no load or scale lookup leaves the weights.
__device__ __forceinline__ int block_expert_of(const GemmArgs& g, int blk) {
  if (!g.sorted_ids) return 0;
  const int e = g.block_expert[blk];
  if (e < 0 || e >= g.E) {
    set_device_error(kErrBlockExpert);
    return 0;
  }
  return e;
}

// Bounded wait that ignores the abort flag: used while unwinding, to let
// copies and MMAs already in flight land before the CTA exits.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer() - t0 > kWaitTimeoutNs) {
      set_device_error(kErrWaitTimeout);
      return;
    }
  }
}

__device__ __forceinline__ int atom_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// e4m3 with round-to-nearest-even and saturation to +-448 (two values).
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Shared exponent of an MXFP8 block: X = floor(log2(amax)) - 8, clamped to
// [-127, 127]; amax = 0 gives -127 (OCP MX v1.0 conversion for e4m3 elements).
__device__ __forceinline__ int mx_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  int e;
  frexpf(amax, &e);  // amax = m * 2^e, m in [0.5, 1): floor(log2 amax) = e - 1
  const int x = e - 1 - 8;
  return x < -127 ? -127 : (x > 127 ? 127 : x);
}

// mx_exponent from the bits of a finite non-negative amax: the biased
// exponent field e gives floor(log2 amax) = e - 127 for a normal amax; zero
// and subnormal amax (e = 0) give -135, clamped to -127 like the definition.
// (A finite fp32 amax gives at most 254 - 135 = 119.)
__device__ __forceinline__ int mx_exponent_bits(float amax) {
  const int x = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127 - 8;
  return x < -127 ? -127 : (x > 127 ? 127 : x);
}

// 2^-X as an fp32 number, for X in [-127, 126] (biased exponent 127 - X in [1, 254]).
__device__ __forceinline__ float pow2_neg(int X) { return __uint_as_float(static_cast<uint32_t>(127 - X) << 23); }

// Quantise the rows of token block `blk` that hold a slot from the
// unquantised fp32 h to e4m3 with one fp32 scale per row, s = amax / 448
// (amax = 0 -> s = 1), code = e4m3(h * (1 / s)) (round to nearest even,
// saturating; the fp32 reciprocal is taken once per row). Padding rows are
// left as they are: stage 2 skips their output columns, and each column of
// the MMA depends on its own row of h only. Run by one epilogue warpgroup
// (128 threads, named barrier `bar_id`) after it has acquired every weight
// tile of the block. `tok_sm` holds the token of each of the BN columns (-1 =
// padding); `rows_sm` (BN ints) and `inv_sm` (BN + 1 words) are its shared scratch.
// The pass reads the rows' fp32 values from L2, so every thread keeps
// kQuantUnroll chunks of loads in flight before converting any of them.
constexpr int kQuantUnroll = 8;
template <int BN>
__device__ __noinline__ void quantize_block_rows(const GemmArgs& g, int blk, int et, int bar_id, const int* tok_sm,
                                                 int* rows_sm, float* inv_sm) {
  named_bar_sync(bar_id, kEpiThreads);  // the caller's reads of rows_sm are done
  if (et < 32) {
    // compact the columns that hold a slot (ballot + prefix count, in order)
    int n = 0;
    for (int c0 = 0; c0 < BN; c0 += 32) {
      const int c = c0 + et;
      const bool v = c < BN && tok_sm[c] >= 0;
      const uint32_t mask = __ballot_sync(0xffffffffu, v);
      if (v) rows_sm[n + __popc(mask & ((1u << et) - 1u))] = c;
      n += __popc(mask);
    }
    if (et == 0) *reinterpret_cast<int*>(inv_sm + BN) = n;
  }
  named_bar_sync(bar_id, kEpiThreads);
  const int nrows = *reinterpret_cast<const int*>(inv_sm + BN);
  // row amax from the per-tile partials: TPR threads per row, combined by shuffles
  constexpr int TPR = BN >= kEpiThreads ? 1 : kEpiThreads / BN;
  for (int j0 = 0; j0 < nrows; j0 += kEpiThreads / TPR) {
    const int j = j0 + et / TPR;
    const int part = et % TPR;
    const int r = blk * BN + (j < nrows ? rows_sm[j] : 0);
    float m = 0.f;
    if (j < nrows) {
#pragma unroll 4
      for (int t = part; t < g.n_mt; t += TPR) m = fmaxf(m, __ldcg(g.h_amax + static_cast<size_t>(t) * g.rows_cap + r));
    }
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (part == 0 && j < nrows) {
      const float sc = m > 0.f ? m / 448.0f : 1.0f;
      inv_sm[j] = 1.0f / sc;
      g.h_scale[r] = sc;
    }
  }
  named_bar_sync(bar_id, kEpiThreads);
  const int chunks = g.I / 8;  // 8 columns per chunk: two 16-byte fp32 loads, one 8-byte e4m3 store
  const int total = nrows * chunks;
  const size_t row0 = static_cast<size_t>(blk) * BN;
  for (int base = et; base < total; base += kEpiThreads * kQuantUnroll) {
    float4 a[kQuantUnroll], b[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int i = base + u * kEpiThreads;
      if (i < total) {
        const int j = i / chunks;
        const size_t off = (row0 + rows_sm[j]) * g.I + static_cast<size_t>(i - j * chunks) * 8;
        a[u] = __ldcg(reinterpret_cast<const float4*>(g.h32 + off));
        b[u] = __ldcg(reinterpret_cast<const float4*>(g.h32 + off + 4));
      }
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int i = base + u * kEpiThreads;
      if (i < total) {
        const int j = i / chunks;
        const size_t off = (row0 + rows_sm[j]) * g.I + static_cast<size_t>(i - j * chunks) * 8;
        const float iv = inv_sm[j];
        const uint32_t q0 = cvt_e4m3x2(a[u].x * iv, a[u].y * iv), q1 = cvt_e4m3x2(a[u].z * iv, a[u].w * iv);
        const uint32_t q2 = cvt_e4m3x2(b[u].x * iv, b[u].y * iv), q3 = cvt_e4m3x2(b[u].z * iv, b[u].w * iv);
        *reinterpret_cast<uint2*>(g.hq + off) = make_uint2(q0 | (q1 << 16), q2 | (q3 << 16));
      }
    }
  }
}

// Byte offset of the scale of (row n, K block kb of the 4 in a stage) inside
// a 512-byte MXFP8 scale tile: 32 row positions x 16 bytes, each holding the
// 4 row groups (n / 32) x 4 K blocks. tcgen05.cp.32x128b.warpx4 moves the tile
// so that TMEM lane n % 32 (and its copies in the other lane quarters) holds,
// in column n / 32, the four K-block bytes of row n.
__host__ __device__ constexpr int sf_tile_offset(int n, int kb) { return (n % 32) * 16 + (n / 32) * 4 + kb; }

// Stage-1 operand preparation, run before the GEMM on the same stream.
// Row r of the sorted order (slot f = sorted_ids[r], token f / top_k; with
// identity routing token r) gets
//  * xs: a copy of its token's x row (routed layers), so that the GEMM loads
//    BN rows with one box per stage (tile::gather4 from x, four rows per
//    instruction, bounded the main loop at every tile size);
//  * xsf (MXFP8): its token's ue8m0 scale bytes, placed in the 512-byte tile
//    of (token block r / bm, stage c) at sf_tile_offset(r % bm, 0..3), the
//    layout the MMA's scale copy takes, so that the GEMM loads one tile per
//    stage as it does for the weights.
// Padding rows are skipped: the MMA column of a padding row is never read. A
// slot id that is neither a slot nor the padding value T * top_k sets
// kErrSlotRange.
struct PrepArgs {
  const uint8_t* x;           // [T][row_bytes]
  const uint8_t* x_scale;     // MXFP8: [T][H / 32]
  const int32_t* sorted_ids;  // nullptr: identity routing
  const int32_t* num_padded;
  int identity_rows, rows_cap, T, top_k, row_bytes, H, bm;
  uint8_t* xs;   // [rows_cap][row_bytes] or nullptr
  uint8_t* xsf;  // [rows_cap / bm][H / 128][512] or nullptr
};
constexpr int kPrepWarps = 8;
__global__ void __launch_bounds__(kPrepWarps * 32) k_stage1_prep(const PrepArgs a) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int rows = a.sorted_ids ? *a.num_padded : a.identity_rows;
  if (rows > a.rows_cap) rows = a.rows_cap;
  const int slots = a.T * a.top_k;
  const int stages = a.H / 128;
  for (int r = blockIdx.x * kPrepWarps + warp; r < rows; r += gridDim.x * kPrepWarps) {
    int t = -1;
    if (!a.sorted_ids) {
      if (r < a.T) t = r;
    } else {
      const int f = a.sorted_ids[r];
      if (f >= 0 && f < slots) t = f / a.top_k;
      else if (f != slots && lane == 0) set_device_error(kErrSlotRange);
    }
    if (t < 0) continue;
    if (a.xs) {
      const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.row_bytes);
      uint4* dst = reinterpret_cast<uint4*>(a.xs + static_cast<size_t>(r) * a.row_bytes);
      for (int i = lane; i < a.row_bytes / 16; i += 32) dst[i] = __ldg(src + i);
    }
    if (a.xsf) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(a.x_scale + static_cast<size_t>(t) * (a.H / 32));
      const int blk = r / a.bm;
      uint8_t* tiles = a.xsf + static_cast<size_t>(blk) * stages * kSfTile + sf_tile_offset(r - blk * a.bm, 0);
      for (int c = lane; c < stages; c += 32) *reinterpret_cast<uint32_t*>(tiles + static_cast<size_t>(c) * kSfTile) = src[c];
    }
  }
}

// Token columns of block `blk` that the tile computes: its rows that hold a
// slot, rounded up to 16 (a valid MMA N; at least 16). The slot rows of a
// sorted block are a prefix, since the sort puts each expert's padding after
// its slots; with identity routing they are the rows below T. Warp-collective.
template <int BN>
__device__ __forceinline__ int block_cols(const GemmArgs& g, int blk, int lane) {
  int v;
  if (!g.sorted_ids) {
    v = g.T - blk * BN;
  } else {
    const unsigned slots = static_cast<unsigned>(g.T * g.top_k);
    int c = 0;
    for (int i = lane; i < BN; i += 32) c += static_cast<unsigned>(g.sorted_ids[blk * BN + i]) < slots ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    v = c;
  }
  v = (v + 15) & ~15;
  return v < 16 ? 16 : (v > BN ? BN : v);
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Barrier over all CTAs of a cooperative launch (every CTA is resident, so
// the wait ends once each CTA has arrived). bar[0] counts arrivals and is
// reset by the last arrival, which then advances the generation bar[1]; the
// others wait for the generation to move. The wait is bounded: on timeout
// it records kErrWaitTimeout and returns false. Called by all threads.
__device__ bool grid_barrier(unsigned* bar, int* flag_sm) {
  if (threadIdx.x == 0) {
    const unsigned gen = ld_acquire_gpu(bar + 1);
    __threadfence();  // this CTA's writes (ordered before by the caller's __syncthreads) first
    int ok = 1;
    if (atomicAdd(bar, 1u) == gridDim.x - 1) {
      atomicExch(bar, 0u);
      __threadfence();
      atomicAdd(bar + 1, 1u);
    } else {
      const uint64_t t0 = globaltimer();
      while (ld_acquire_gpu(bar + 1) == gen) {
        if (globaltimer() - t0 > kWaitTimeoutNs) {
          set_device_error(kErrWaitTimeout);
          ok = 0;
          break;
        }
        __nanosleep(256);
      }
    }
    *flag_sm = ok;
  }
  __syncthreads();
  return *flag_sm != 0;
}

// fp8 stage 1, quant_phase: after every weight tile of every token block is
// done, each warp of the grid quantises whole rows of h (the rows holding a
// slot; padding rows are never read): row amax over the per-tile partials,
// s = amax / 448 (amax = 0 -> s = 1), codes e4m3(h * (1 / s)).
__device__ void quantize_rows_grid(const GemmArgs& g, int rows) {
  const int lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  const int slots = g.T * g.top_k;
  const int chunks = g.I / 8;  // 8 columns per chunk
  for (int r = blockIdx.x * nw + (threadIdx.x >> 5); r < rows; r += gridDim.x * nw) {
    const bool valid = g.sorted_ids ? (static_cast<unsigned>(g.sorted_ids[r]) < static_cast<unsigned>(slots)) : (r < g.T);
    if (!valid) continue;
    float m = 0.f;
    for (int t = lane; t < g.n_mt; t += 32) m = fmaxf(m, __ldcg(g.h_amax + static_cast<size_t>(t) * g.rows_cap + r));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float sc = m > 0.f ? m / 448.0f : 1.0f;
    const float iv = 1.0f / sc;
    if (lane == 0) g.h_scale[r] = sc;
    const float* src = g.h32 + static_cast<size_t>(r) * g.I;
    uint8_t* dst = g.hq + static_cast<size_t>(r) * g.I;
    for (int base = lane; base < chunks; base += 32 * kQuantUnroll) {
      float4 a[kQuantUnroll], b[kQuantUnroll];
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) {
        const int i = base + 32 * u;
        if (i < chunks) {
          a[u] = __ldcg(reinterpret_cast<const float4*>(src) + 2 * i);
          b[u] = __ldcg(reinterpret_cast<const float4*>(src) + 2 * i + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) {
        const int i = base + 32 * u;
        if (i < chunks) {
          const uint32_t q0 = cvt_e4m3x2(a[u].x * iv, a[u].y * iv), q1 = cvt_e4m3x2(a[u].z * iv, a[u].w * iv);
          const uint32_t q2 = cvt_e4m3x2(b[u].x * iv, b[u].y * iv), q3 = cvt_e4m3x2(b[u].z * iv, b[u].w * iv);
          reinterpret_cast<uint2*>(dst)[i] = make_uint2(q0 | (q1 << 16), q2 | (q3 << 16));
        }
      }
    }
  }
}

// PAIR = false: one CTA per tile (MMA M = 128). PAIR = true: a 2-CTA cluster
// per tile of 256 weight rows (rank r holds weight sub-tile 2 * wt + r, the
// sub-tile index the epilogue, the scale tiles and the fp8 partials use);
// rank 0 issues the M = 256 MMAs; each rank loads its 128 weight rows and
// half of the tile's token rows (split at ncols / 2), plus, for MX, its own
// A scale tile and the whole B scale tile. Stage pipeline: each rank waits on
// its own `empty` barriers; every load completes on rank 0's `full` barrier,
// armed by rank 0 with the bytes of both; the MMA commits to `empty` and
// `acc_full` of both ranks; every epilogue warp of both ranks arrives on rank
// 0's `acc_empty`.
template <int BN, int STAGES, bool S1, int KIND, bool PAIR = false>
__global__ void __launch_bounds__(EpiCfg<BN, KIND, S1>::kThreads, 1)
    k_moe_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmB16, const __grid_constant__ CUtensorMap tmSfa,
               const __grid_constant__ CUtensorMap tmSfb, const GemmArgs g) {
  using L = GemmSmem<BN, STAGES, KIND, S1, PAIR>;
  constexpr bool FP8 = KIND == kFp8;
  constexpr bool MX = is_mx(KIND);
  constexpr int G = L::kGroups;
  constexpr int NACC = L::kAcc;
  constexpr int KE = KIND == kBf16 ? 64 : 128;  // K elements per stage
  constexpr int kUmmaKBytes = 32;               // K bytes per MMA: 16 bf16 or 32 e4m3
  constexpr int kMmaM = PAIR ? 2 * kTileM : kTileM;
  constexpr bool SPLIT = EpiCfg<BN, KIND, S1>::kSplit;
  constexpr int kLead = EpiCfg<BN, KIND, S1>::kLead;
  constexpr bool SFW = L::kSfWarp;
  constexpr int KA = L::kAtoms;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "token tile");
  static_assert(!MX || BN <= 128, "MXFP8 scale tiles cover 128 token rows");
  static_assert(STAGES <= 32, "stage mask");
  static_assert(!PAIR || !(FP8 && S1), "fp8 stage 1 quantises h after a grid barrier: one CTA per tile");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + NACC;
  uint64_t* drain = acc_empty + NACC;
  uint64_t* sf_full = drain + 1;  // SFW: stage s's scale tiles are in TMEM slot s
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOffset);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* group_base = reinterpret_cast<int*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  // epilogue arrivals per accumulator phase: every thread (one CTA) or every
  // epilogue warp of both CTAs (pair)
  constexpr uint32_t kAccEmptyCount = PAIR ? 2 * (kEpiThreads / 32) : kEpiThreads;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], SPLIT ? 2 : 1);  // each producer warp arms it with its own bytes
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < NACC; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kAccEmptyCount);
    }
    mbar_init(drain, 1);
    if constexpr (SFW)
      for (int s = 0; s < STAGES; ++s) mbar_init(&sf_full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, L::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, L::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // shared::cluster addresses of rank 0's full / acc_empty barriers and of
  // both ranks' empty / acc_full barriers (pair only)
  uint32_t full0 = 0, acc_empty0 = 0, empty_r[2] = {0, 0}, acc_full_r[2] = {0, 0};
  if constexpr (PAIR) {
    full0 = mapa_shared(smem_u32(full), 0);
    acc_empty0 = mapa_shared(smem_u32(acc_empty), 0);
    empty_r[0] = mapa_shared(smem_u32(empty), 0);
    empty_r[1] = mapa_shared(smem_u32(empty), 1);
    acc_full_r[0] = mapa_shared(smem_u32(acc_full), 0);
    acc_full_r[1] = mapa_shared(smem_u32(acc_full), 1);
  }

  int n_blocks = g.sorted_ids ? (*g.num_padded) / BN : g.identity_rows / BN;
  if (n_blocks > g.cap_blocks) n_blocks = g.cap_blocks;
  // scheduling unit: one CTA (tile of 128 weight rows) or one pair (256 rows)
  const int n_wt = PAIR ? g.n_mt / 2 : g.n_mt;
  const int unit0 = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int n_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const int total = n_blocks * n_wt;
  const int slots = g.T * g.top_k;
  const int n_ks = (g.num_kb + KA - 1) / KA;  // pipeline stages per tile (the last may hold fewer atoms)

  if (warp == 0 || (SPLIT && warp == 2)) {
    // ------------------------------------------------------------ producer(s)
    const bool do_w = !SPLIT || warp == 0;  // weight tile (+ its MX scale tile)
    const bool do_t = !SPLIT || warp == 2;  // token tile (+ its MX scale tile)
    const uint64_t pol_w = policy_evict_first();  // weights stream through once
    const uint64_t pol_x = policy_evict_last();   // token rows are re-read per weight tile
    int stage = 0;
    uint32_t phase = 0;
    uint32_t pending = 0, pend_parity = 0;  // stages armed and not yet re-acquired
    bool ok = true;
    for (int tile = unit0; tile < total && ok; tile += n_units) {
      const int blk = tile / n_wt;
      const int mt = PAIR ? 2 * (tile - blk * n_wt) + static_cast<int>(rank) : tile - blk * n_wt;
      const int expert = do_w ? block_expert_of(g, blk) : 0;
      const int ncols = block_cols<BN>(g, blk, lane);  // token rows this tile loads and multiplies
      const int my_rows = PAIR ? ncols / 2 : ncols;    // token rows this CTA loads
      const int row0 = blk * BN + (PAIR ? static_cast<int>(rank) * my_rows : 0);
      // transaction bytes count what this warp's copies read from global
      // memory: half the shared-memory footprint for the packed e2m1 weight tile
      // (per K atom)
      uint32_t bytes = 0;
      if (do_w) bytes += (KIND == kMx4 ? L::kAtomA / 2 : L::kAtomA) + (MX ? kSfTile : 0);
      if (do_t) bytes += static_cast<uint32_t>(my_rows) * kTileKBytes + (MX ? kSfTile : 0);
      // A tile whose token rows come in one box needs lane 0 only: it runs the
      // tile's stages alone, and the warp re-joins at the tile's end. Short
      // tiles spread their row boxes over the lanes, stage by stage.
      const bool solo = ncols == BN || !do_t;
      for (int ks = 0; ks < n_ks; ++ks) {
        if (solo && lane != 0) break;
        const int kb0 = ks * KA;                                  // first K atom of the stage
        const int na = g.num_kb - kb0 < KA ? g.num_kb - kb0 : KA;  // atoms in the stage
        uint8_t* a_dst = smem + stage * L::kStageBytes;
        uint8_t* b_dst = a_dst + L::kABytes;
        uint8_t* sfa_dst = b_dst + L::kBBytes;
        uint8_t* sfb_dst = sfa_dst + KA * kSfTile;
        if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1u, abort_flag);
        if (!solo) ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if constexpr (PAIR) {
          const uint32_t fb = full0 + 8u * static_cast<uint32_t>(stage);
          if (lane == 0) {
            pending &= ~(1u << stage);
            // both CTAs' copies of this kind, per atom
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * bytes * static_cast<uint32_t>(na));
#pragma unroll
            for (int a = 0; a < KA; ++a) {
              if (a >= na) break;
              const int kb = kb0 + a;
              if (do_w) {
                uint8_t* dst = a_dst + a * L::kAtomA;
                if (S1) tma_load_5d_pair(dst, &tmA, fb, kb * KE, 0, 0, mt * 4, expert, pol_w);
                else tma_load_3d_pair(dst, &tmA, fb, kb * KE, mt * kTileM, expert, pol_w);
                if (MX)
                  tma_load_2d_pair(sfa_dst + a * kSfTile, &tmSfa, fb, 0, ((expert * g.n_mt + mt) * g.num_kb + kb) * 4,
                                   pol_w);
              }
              if (do_t) {
                if (ncols == BN) tma_load_2d_pair(b_dst + a * L::kAtomB, &tmB, fb, kb * KE, row0, pol_x);
                if (MX) tma_load_2d_pair(sfb_dst + a * kSfTile, &tmSfb, fb, 0, (blk * g.num_kb + kb) * 4, pol_x);
              }
            }
            pending |= 1u << stage;
            pend_parity = (pend_parity & ~(1u << stage)) | (phase << stage);
          }
          if (!solo) __syncwarp();
          // a short tile: this CTA's token rows in 8-row boxes, issued by the lanes
          if (do_t && ncols < BN) {
            const int boxes = my_rows / 8;  // per atom
            for (int q = lane; q < na * boxes; q += 32) {
              const int a = q / boxes;
              const int r = q - a * boxes;
              tma_load_2d_pair(b_dst + a * L::kAtomB + r * 8 * kTileKBytes, &tmB16, fb, (kb0 + a) * KE, row0 + r * 8,
                               pol_x);
            }
          }
        } else {
          if (lane == 0) {
            pending &= ~(1u << stage);
            mbar_arrive_expect_tx(&full[stage], bytes * static_cast<uint32_t>(na));
            // one copy per K atom and operand; the atoms' scale tiles are
            // consecutive in memory and come in one copy per operand
            if (do_w) {
#pragma unroll
              for (int a = 0; a < KA; ++a) {
                if (a < na) {
                  uint8_t* dst = a_dst + a * L::kAtomA;
                  if (S1) tma_load_5d(dst, &tmA, &full[stage], (kb0 + a) * KE, 0, 0, mt * 4, expert, pol_w);
                  else tma_load_3d(dst, &tmA, &full[stage], (kb0 + a) * KE, mt * kTileM, expert, pol_w);
                }
              }
              if (MX) {
                const size_t wt = (static_cast<size_t>(expert) * g.n_mt + mt) * g.num_kb + kb0;
                bulk_load(sfa_dst, g.wsf + wt * kSfTile, na * kSfTile, &full[stage], pol_w);
              }
            }
            if (do_t) {
              // token rows as one box per atom when the tile is full (B from x, the sorted copy, or h)
              if (ncols == BN) {
#pragma unroll
                for (int a = 0; a < KA; ++a)
                  if (a < na)
                    tma_load_2d(b_dst + a * L::kAtomB, &tmB, &full[stage], (kb0 + a) * KE, blk * BN, pol_x);
              }
              if (MX)
                bulk_load(sfb_dst, (S1 ? g.xsf : g.hsf) + (static_cast<size_t>(blk) * g.num_kb + kb0) * kSfTile,
                          na * kSfTile, &full[stage], pol_x);
            }
            pending |= 1u << stage;
            pend_parity = (pend_parity & ~(1u << stage)) | (phase << stage);
          }
          if (!solo) __syncwarp();
          // a short tile: its token rows in 16-row boxes, issued by the lanes of
          // the warp (the barrier was armed above with the stage's full byte count)
          if (do_t && ncols < BN) {
            const int boxes = ncols / 16;  // per atom
            for (int q = lane; q < na * boxes; q += 32) {
              const int a = q / boxes;
              const int r = q - a * boxes;
              tma_load_2d(b_dst + a * L::kAtomB + r * 16 * kTileKBytes, &tmB16, &full[stage], (kb0 + a) * KE,
                          blk * BN + r * 16, pol_x);
            }
          }
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (solo) {  // the other lanes take lane 0's ring position and status
        stage = __shfl_sync(0xffffffffu, stage, 0);
        phase = __shfl_sync(0xffffffffu, phase, 0);
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) {
      if (!PAIR || rank == 0) {
        for (int s = 0; s < STAGES; ++s)
          if ((pending >> s) & 1u) drain_wait(&full[s], (pend_parity >> s) & 1u);
      } else if (pending) {
        // rank 1's copies complete on rank 0's barriers, which it cannot wait
        // on: give copies in flight a bounded 2 ms to land before unwinding
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 2000000ull) __nanosleep(1000);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // (a pair's MMAs are all issued by rank 0). The warp computes each tile's
    // token-column count together; lane 0 alone then runs the tile's K stages
    // (issue is one thread's work, and per-stage warp shuffles and syncs cost
    // as much as an MMA issue).
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    uint32_t sf_slot = 0;
    int j = 0;  // local tile counter: accumulator j % NACC, use (j / NACC)
    const bool issuer = !PAIR || rank == 0;
    for (int tile = unit0; issuer && tile < total; tile += n_units, ++j) {
      const int ncols = block_cols<BN>(g, tile / n_wt, lane);
      if (lane == 0) {
        const int acc = j % NACC;
        const uint32_t acc_phase = static_cast<uint32_t>(j / NACC) & 1u;
        const uint32_t idesc = FP8 ? idesc_e4m3(kMmaM, ncols) : idesc_bf16(kMmaM, ncols);
        ok = mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag);
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        if (ok) tc_fence_after();
        for (int ks = 0; ok && ks < n_ks; ++ks) {
          const int na = g.num_kb - ks * KA < KA ? g.num_kb - ks * KA : KA;  // K atoms in the stage
          ok = mbar_wait(SFW ? &sf_full[stage] : &full[stage], phase, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * L::kStageBytes);
          const uint32_t b_addr = a_addr + L::kABytes;
          uint32_t tsfa = 0, tsfb = 0;
          if (SFW) {
            // slot `stage`: atom a's A scales in columns 4a.., its B scales 4 KA further
            tsfa = tmem_base + static_cast<uint32_t>(L::kSfCol + 8 * KA * stage);
            tsfb = tsfa + 4 * KA;
          } else if (MX) {
            // scale tiles of this stage -> TMEM ring slot (the atoms' A tiles in
            // 4 columns each, then their B tiles)
            tsfa = tmem_base + static_cast<uint32_t>(L::kSfCol) + sf_slot * 8 * KA;
            tsfb = tsfa + 4 * KA;
            const uint32_t sf_addr = a_addr + L::kABytes + L::kBBytes;
#pragma unroll
            for (int a = 0; a < KA; ++a) {
              if (a >= na) break;
              if constexpr (PAIR) {
                tmem_cp_32x128b_x4_pair(tsfa + 4 * a, plain_rows16_desc(sf_addr + a * kSfTile));
                tmem_cp_32x128b_x4_pair(tsfb + 4 * a, plain_rows16_desc(sf_addr + (KA + a) * kSfTile));
              } else {
                tmem_cp_32x128b_x4(tsfa + 4 * a, plain_rows16_desc(sf_addr + a * kSfTile));
                tmem_cp_32x128b_x4(tsfb + 4 * a, plain_rows16_desc(sf_addr + (KA + a) * kSfTile));
              }
            }
            sf_slot = (sf_slot + 1) % kSfSlots;
          }
#pragma unroll
          for (int a = 0; a < KA; ++a) {
            if (a >= na) break;
            const uint64_t adesc = sw128_kmajor_desc(a_addr + a * L::kAtomA);
            const uint64_t bdesc = sw128_kmajor_desc(b_addr + a * L::kAtomB);
            const uint32_t sfa = tsfa + 4 * a, sfb = tsfb + 4 * a;
#pragma unroll
            for (int kk = 0; kk < kTileKBytes / kUmmaKBytes; ++kk) {
              // +32 bytes along K inside the swizzle row: +2 in the (addr >> 4) field
              const uint64_t adv = static_cast<uint64_t>(kk * (kUmmaKBytes >> 4));
              const uint32_t accum = (ks | a | kk) != 0 ? 1u : 0u;
              if (MX) {
                // K block kk of the atom: byte kk of each scale column
                const uint32_t sel = static_cast<uint32_t>(kk) << 30;
                const uint32_t id = idesc_mx(kMmaM, ncols, kk, KIND == kMx4 ? kFmtE2M1 : kFmtE4M3);
                if constexpr (PAIR) umma_mx8_pair(d_tmem, adesc + adv, bdesc + adv, id, sfa | sel, sfb | sel, accum);
                else umma_mx8(d_tmem, adesc + adv, bdesc + adv, id, sfa | sel, sfb | sel, accum);
              } else if (FP8) {
                if constexpr (PAIR) umma_f8_pair(d_tmem, adesc + adv, bdesc + adv, idesc, accum);
                else umma_f8(d_tmem, adesc + adv, bdesc + adv, idesc, accum);
              } else {
                if constexpr (PAIR) umma_f16_pair(d_tmem, adesc + adv, bdesc + adv, idesc, accum);
                else umma_f16(d_tmem, adesc + adv, bdesc + adv, idesc, accum);
              }
            }
          }
          // smem stage free once these MMAs (and copies) finish: in both CTAs for a pair
          if constexpr (PAIR) {
            umma_commit_pair(empty_r[0] + 8u * static_cast<uint32_t>(stage));
            umma_commit_pair(empty_r[1] + 8u * static_cast<uint32_t>(stage));
          } else {
            umma_commit(&empty[stage]);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) {
          if constexpr (PAIR) {
            umma_commit_pair(acc_full_r[0] + 8u * static_cast<uint32_t>(acc));
            umma_commit_pair(acc_full_r[1] + 8u * static_cast<uint32_t>(acc));
          } else {
            umma_commit(&acc_full[acc]);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
    }
    if (!ok && lane == 0) {
      if constexpr (PAIR) umma_commit_pair(mapa_shared(smem_u32(drain), 0));
      else umma_commit(drain);
      drain_wait(drain, 0);
    }
  } else if (SFW && warp == 3) {
    // ------------------------------------------------------------ scale-tile copier
    // Lane 0 copies each stage's A and B scale tiles into TMEM slot `stage`
    // (columns kSfCol + 8 KA stage: the atoms' A tiles, then their B tiles) and commits the copies to
    // sf_full[stage], which the MMA thread waits on in place of `full`. A slot
    // needs no barrier of its own: stage s is refilled, and its `full` barrier
    // completes again, only after the MMAs that read slot s have finished
    // (the MMA thread's commit to empty[s]).
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int last = -1;  // stage of the last commit, drained on the way out
      uint32_t last_phase = 0;
      for (int tile = unit0; ok && tile < total; tile += n_units) {
        for (int ks = 0; ks < n_ks; ++ks) {
          const int na = g.num_kb - ks * KA < KA ? g.num_kb - ks * KA : KA;
          ok = mbar_wait(&full[stage], phase, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sf_addr = smem_u32(smem + stage * L::kStageBytes) + L::kABytes + L::kBBytes;
          const uint32_t tsfa = tmem_base + static_cast<uint32_t>(L::kSfCol + 8 * KA * stage);
#pragma unroll
          for (int a = 0; a < KA; ++a) {
            if (a < na) {
              tmem_cp_32x128b_x4(tsfa + 4 * a, plain_rows16_desc(sf_addr + a * kSfTile));
              tmem_cp_32x128b_x4(tsfa + 4 * (KA + a), plain_rows16_desc(sf_addr + (KA + a) * kSfTile));
            }
          }
          umma_commit(&sf_full[stage]);
          last = stage;
          last_phase = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every copy issued (the last commit tracks all of them) lands before TMEM is freed
      if (last >= 0) drain_wait(&sf_full[last], last_phase);
    }
    __syncwarp();
  } else if (warp >= kLead / 32) {
    // ------------------------------------------------------------ epilogue
    const int grp = (warp - kLead / 32) >> 2;     // epilogue group: tiles j with j % G == grp
    const int q = warp & 3;                       // TMEM lane quarter this warp may read
    const int et = threadIdx.x - kLead - kEpiThreads * grp;  // 0..127 inside the group
    const int bar_id = 1 + grp;                   // named barrier of this group
    int* gsm = group_base + grp * L::kGroupWords;
    volatile int* ok_sm = gsm;
    int* tok_sm = gsm + 4;                        // token of each column, -1 = padding
    float* wgt_sm = reinterpret_cast<float*>(tok_sm + BN);  // per-column factor: stage 1 fp8 x and W13 scales;
                                                            // stage 2 top-k weight (x h and W2 scales for fp8)
    int* last_sm = reinterpret_cast<int*>(wgt_sm + BN);
    float* amax_part = reinterpret_cast<float*>(last_sm + BN);
    // the accumulator is free again once this thread's (one CTA) or this
    // warp's (pair: every warp of both CTAs arrives on rank 0) reads are done
    auto release_acc = [&](int acc) {
      tc_fence_before();
      if constexpr (PAIR) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8u * static_cast<uint32_t>(acc));
      } else {
        mbar_arrive(&acc_empty[acc]);
      }
    };
    int j = 0;
    for (int tile = unit0; tile < total; tile += n_units, ++j) {
      if (j % G != grp) continue;
      const int blk = tile / n_wt;
      const int mt = PAIR ? 2 * (tile - blk * n_wt) + static_cast<int>(rank) : tile - blk * n_wt;
      const int acc = j % NACC;
      const uint32_t acc_phase = static_cast<uint32_t>(j / NACC) & 1u;
      const int expert = block_expert_of(g, blk);
      const int ncols = block_cols<BN>(g, blk, lane);  // accumulator columns the MMA wrote

      // per-column metadata, fetched while the accumulator is still being built
      for (int c = et; c < BN; c += kEpiThreads) {
        const int r = blk * BN + c;
        int f = r, t = -1;
        if (!g.sorted_ids) {
          if (r < g.T) t = r;
        } else {
          f = g.sorted_ids[r];
          if (f >= 0 && f < slots) t = f / g.top_k;
        }
        tok_sm[c] = t;
        float w = 0.f;
        if (t >= 0) {
          if (S1) w = FP8 ? g.x_scale[t] * g.w_scale[expert] : 1.0f;
          else w = load_weight(g.weights, g.weights_dtype, f) * (FP8 ? g.h_scale[r] * g.w_scale[expert] : 1.0f);
        }
        wgt_sm[c] = w;
      }
      if (et == 0) *ok_sm = mbar_wait(&acc_full[acc], acc_phase, abort_flag) ? 1 : 0;
      named_bar_sync(bar_id, kEpiThreads);
      if (!*ok_sm) break;  // same value in every thread of the group
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(acc * BN);

      if (S1) {
        // Lanes 0..15 of quarter q hold gate features 16q..16q+15 of this
        // 64-feature tile, lanes 16..31 the matching up features. Lanes 0..15
        // finish the even columns, lanes 16..31 the odd ones.
        const int feat = mt * 64 + 16 * q + (lane & 15);
        const bool lo = lane < 16;
        float hv_keep[MX ? BN / 2 : 1];  // MXFP8: h of this thread's columns until the block scale is known
        // (MXFP8 unrolls the column loop so that hv_keep stays in registers)
#pragma unroll(MX ? BN / 16 : 1)
        for (int c0 = 0; c0 < BN; c0 += 16) {
          if (c0 < ncols) {
          float v[16];
          tmem_ld16(t_row + static_cast<uint32_t>(c0), v);
          tmem_wait_ld();
          if (c0 + 16 >= ncols) release_acc(acc);
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const float o0 = __shfl_xor_sync(0xffffffffu, v[i], 16);
            const float o1 = __shfl_xor_sync(0xffffffffu, v[i + 1], 16);
            float gt = lo ? v[i] : o1;
            float up = lo ? o0 : v[i + 1];
            const int c = c0 + i + (lo ? 0 : 1);
            const int r = blk * BN + c;
            if (FP8) {
              const float sc = wgt_sm[c];
              gt *= sc;
              up *= sc;
            }
            // MXFP8 h is quantised to three mantissa bits next: the fast
            // exponential and division (relative error ~1e-6, as small as the
            // fp32 accumulation's) keep this loop short; bf16 and fp8 h use
            // the exact ones
            const float hv = MX ? __fdividef(gt, 1.0f + __expf(-gt)) * up : gt / (1.0f + expf(-gt)) * up;
            if (!MX && feat < g.I) {
              if (FP8) g.h32[static_cast<size_t>(r) * g.I + feat] = hv;
              else g.h[static_cast<size_t>(r) * g.I + feat] = __float2bfloat16_rn(hv);
            }
            if (MX) hv_keep[(c0 + i) / 2] = hv;
            if (FP8 || MX) {
              // amax over this half-warp's 16 features of column c
              float m = fabsf(hv);
              m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
              m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
              m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
              m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
              if ((lane & 15) == 0) amax_part[q * BN + c] = m;
            }
          }
          }
        }
        if (MX) {
          // One MX block = 32 features = lane quarters 2p and 2p+1 of the tile
          // (ROCm/aiter PR 6106: BLOCK_K = 32): shared exponent from the pair's
          // amax, codes e4m3(h * 2^-X), one ue8m0 byte X + 127 per (row, block),
          // written into stage 2's scale tile layout.
          named_bar_sync(bar_id, kEpiThreads);
          const int kblk = feat / 32;  // K block of stage 2
          const size_t tile_base = (static_cast<size_t>(blk) * (g.I / 128) + kblk / 4) * kSfTile;
#pragma unroll
          for (int i = 0; i < BN / 2; ++i) {
            if (2 * i >= ncols) continue;
            const int c = 2 * i + (lo ? 0 : 1);
            const float amax = fmaxf(amax_part[q * BN + c], amax_part[(q ^ 1) * BN + c]);
            const int X = mx_exponent_bits(amax);
            const float v = hv_keep[i] * pow2_neg(X);  // exact: a power of two in the normal range
            const uint8_t code = static_cast<uint8_t>(cvt_e4m3x2(v, 0.f) & 0xFF);
            if (feat < g.I) g.hq[static_cast<size_t>(blk * BN + c) * g.I + feat] = code;
            if ((q & 1) == 0 && (lane & 15) == 0)
              g.hsf[tile_base + sf_tile_offset(c, kblk & 3)] = static_cast<uint8_t>(X + 127);
          }
        }
        if (FP8) {
          named_bar_sync(bar_id, kEpiThreads);
          for (int c = et; c < ncols; c += kEpiThreads) {
            const float m = fmaxf(fmaxf(amax_part[c], amax_part[BN + c]),
                                  fmaxf(amax_part[2 * BN + c], amax_part[3 * BN + c]));
            g.h_amax[static_cast<size_t>(mt) * g.rows_cap + blk * BN + c] = m;
          }
          // The group that finishes the last weight tile of this token block
          // quantises the block's rows: one scale amax/448 per row over all I
          // columns (ROCm/aiter PR 6106, "Technical Details": quantisation
          // fused after the activation). The barrier orders this group's h and
          // amax stores before the counter's release; the acquire of the last
          // arrival makes every tile's stores visible.
          if (!g.quant_phase) {
            named_bar_sync(bar_id, kEpiThreads);
            if (et == 0) {
              int* cnt = g.blk_cnt + blk;
              const bool last = atom_add_acq_rel_gpu(cnt, 1) == g.n_mt - 1;
              if (last) *cnt = 0;
              last_sm[0] = last ? 1 : 0;
            }
            named_bar_sync(bar_id, kEpiThreads);
            if (last_sm[0]) quantize_block_rows<BN>(g, blk, et, bar_id, tok_sm, last_sm, amax_part);
          }
        }
      } else {
        const int n = mt * kTileM + 32 * q + lane;  // output feature
        const bool nvalid = n < g.H;
#pragma unroll 1
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          float v[16];
          tmem_ld16(t_row + static_cast<uint32_t>(c0), v);
          tmem_wait_ld();
          if (c0 + 16 >= ncols) release_acc(acc);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int t = tok_sm[c0 + i];
            if (t < 0 || !nvalid) continue;
            const float val = v[i] * wgt_sm[c0 + i];
            const size_t o = static_cast<size_t>(t) * g.H + n;
            if (g.top_k == 1) {
              float y = val;
              if (g.addend) y += __bfloat162float(g.addend[o]);
              g.out[o] = __float2bfloat16_rn(y);
            } else {
              red_add_f32(g.ws + o, val);
            }
          }
        }
        if (g.top_k > 1) {
          // Arrival count per (token, weight tile). The group barrier orders
          // every thread's red.add before the counter update, whose release
          // publishes them; the epilogue that brings a token's k-th slot
          // acquires all k contributions and finalises the 128 outputs.
          named_bar_sync(bar_id, kEpiThreads);
          for (int c = et; c < BN; c += kEpiThreads) {
            const int t = tok_sm[c];
            int flag = 0;
            if (t >= 0) {
              int* cnt = g.counters + static_cast<size_t>(t) * g.n_mt + mt;
              if (atom_add_acq_rel_gpu(cnt, 1) == g.top_k - 1) {
                flag = 1;
                *cnt = 0;
              }
            }
            last_sm[c] = flag;
          }
          // Finalise the columns this group brought last: their tokens' sums
          // are complete (acquired above). The columns are compacted first so
          // that each thread has kFinBatch independent loads in flight (one L2
          // round trip per batch instead of one per column).
          named_bar_sync(bar_id, kEpiThreads);
          int* list = reinterpret_cast<int*>(amax_part);  // BN column indices, then the count
          if (et < 32) {
            int cnt = 0;
            for (int c0 = 0; c0 < BN; c0 += 32) {
              const int c = c0 + et;
              const bool v = c < BN && last_sm[c];
              const uint32_t mask = __ballot_sync(0xffffffffu, v);
              if (v) list[cnt + __popc(mask & ((1u << et) - 1u))] = c;
              cnt += __popc(mask);
            }
            if (et == 0) list[BN] = cnt;
          }
          named_bar_sync(bar_id, kEpiThreads);
          const int nlast = list[BN];
          if (nvalid) {
            const __nv_bfloat16* add = g.addend;
            for (int j0 = 0; j0 < nlast; j0 += kFinBatch) {
              // addresses of the batch (a past-the-end entry repeats column
              // j0 and is loaded but not stored), then all workspace loads,
              // then all addend loads, then the stores
              float y[kFinBatch], a[kFinBatch];
              size_t o[kFinBatch];
#pragma unroll
              for (int u = 0; u < kFinBatch; ++u) {
                o[u] = static_cast<size_t>(tok_sm[list[j0 + u < nlast ? j0 + u : j0]]) * g.H + n;
                y[u] = 0.f;
                a[u] = 0.f;
              }
#pragma unroll
              for (int u = 0; u < kFinBatch; ++u)
                if (j0 + u < nlast) y[u] = __ldcg(g.ws + o[u]);
              if (add) {
#pragma unroll
                for (int u = 0; u < kFinBatch; ++u)
                  if (j0 + u < nlast) a[u] = __bfloat162float(add[o[u]]);
              }
#pragma unroll
              for (int u = 0; u < kFinBatch; ++u) {
                if (j0 + u < nlast) {
                  __stcg(g.ws + o[u], 0.0f);  // the workspace is left zeroed for the next call
                  g.out[o[u]] = __float2bfloat16_rn(y[u] + a[u]);
                }
              }
            }
          }
        }
      }
      named_bar_sync(bar_id, kEpiThreads);  // metadata of this tile no longer read
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // no CTA leaves while its peer may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, L::kTmemCols);
    else tmem_dealloc(tmem_base, L::kTmemCols);
  }
  if constexpr (FP8 && S1) {
    if (g.quant_phase && grid_barrier(g.grid_bar, reinterpret_cast<int*>(tmem_slot + 2)))
      quantize_rows_grid(g, n_blocks * BN);
  }
}

// Weight scale tiles for MXFP8 (one-off weight preparation). src is the
// row-major [E][rows][K/32] ue8m0 bytes; dst gets, per (expert, weight tile,
// stage), the 512-byte tile of the 128 A-operand rows x 4 K blocks in
// sf_tile_offset order. W13 tiles follow the stage-1 A layout, whose row m
// (m = rr + 16*gu + 32*qq) is W13 row gu*I + (4*mt + qq)*16 + rr; W2 tiles are
// 128 consecutive rows.
__global__ void k_mx_pack_weight_scales(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int E, int rows,
                                        int K, int I, int w13) {
  const int kbs = K / 32;    // K blocks per row
  const int n_kg = K / 128;  // stages per tile
  const int n_mt = w13 ? I / 64 : rows / 128;
  const size_t n_out = static_cast<size_t>(E) * n_mt * n_kg * kSfTile;
  for (size_t o = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; o < n_out;
       o += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int within = static_cast<int>(o % kSfTile);
    size_t t = o / kSfTile;
    const int kg = static_cast<int>(t % n_kg);
    t /= n_kg;
    const int mt = static_cast<int>(t % n_mt);
    const int e = static_cast<int>(t / n_mt);
    const int m0 = within / 16, m1 = (within % 16) / 4, kb = within % 4;
    const int m = m0 + 32 * m1;  // A-operand row of the tile
    int row;
    if (w13) {
      const int rr = m % 16, gu = (m / 16) % 2, qq = m / 32;
      row = gu * I + (4 * mt + qq) * 16 + rr;
    } else {
      row = mt * 128 + m;
    }
    dst[o] = src[(static_cast<size_t>(e) * rows + row) * kbs + kg * 4 + kb];
  }
}

}  // namespace moe
