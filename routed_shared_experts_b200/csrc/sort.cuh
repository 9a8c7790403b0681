// sort.cuh - align/sort of the routed slots by expert, one CTA of 32 warps.
//
// vllm-project/vllm PR 65207, reviewer measurements ("Commits 2 and 3"):
// moe_sorting is run without zeroing the layer output; here the sort never
// touches the output (the stage-2 epilogue writes every output row).
// ROCm/aiter PR 6106, "Technical Details": GEMM rows follow this gather index.
#pragma once
#include "ptx.cuh"

namespace moe {

constexpr int kSortThreads = 1024;
constexpr int kSortBatch = 8;  // 32-slot steps whose ids a warp loads at once

struct SortArgs {
  const int32_t* ids;  // [N] flat slots f = t*k + j
  int N, E, bm;
  int32_t* sorted;        // [capacity]
  int32_t* block_expert;  // [capacity / bm]
  int32_t* counts;        // [E]
  int32_t* offsets;       // [E+1]
  int32_t* num_padded;    // [1]
};

// Shared memory: cnt[E], base[E], warp_cnt[32][E], warp totals [32].
//
// Each warp owns one contiguous chunk of the flat slots (warp w: chunk w of
// 32), so that a stable order needs no barrier per round:
//   1. each warp counts its chunk's slots per expert into its own row of
//      warp_cnt (32 slots per step, __match_any_sync groups equal experts, the
//      lowest lane of a group adds the group's size: one writer per entry);
//   2. per expert, an exclusive prefix over the 32 warps' counts, and over
//      the experts an exclusive prefix of the padded segment sizes, turn each
//      warp_cnt entry into the absolute position of that warp's first slot of
//      that expert; counts, offsets, block owners and padding are written;
//   3. each warp walks its chunk again in order and places every slot at its
//      entry plus its rank among the equal experts of its 32-slot step, then
//      advances the entry: ascending f inside every expert segment.
__global__ void __launch_bounds__(kSortThreads) k_align_sort(const SortArgs a) {
  extern __shared__ int ssm[];
  const int E = a.E;
  int* cnt = ssm;
  int* base = cnt + E;
  int* warp_cnt = base + E;
  int* wsum = warp_cnt + 32 * E;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int chunk = (a.N + 31) / 32;
  const int f0 = warp * chunk;
  const int f1 = f0 + chunk < a.N ? f0 + chunk : a.N;
  int* my_cnt_row = warp_cnt + warp * E;

  for (int i = tid; i < 32 * E; i += kSortThreads) warp_cnt[i] = 0;
  __syncthreads();

  // 1. per-warp counts; the ids of kSortBatch steps are loaded before any is
  // used, so that a warp keeps that many loads in flight
  for (int b0 = f0; b0 < f1; b0 += 32 * kSortBatch) {
    int ev[kSortBatch];
#pragma unroll
    for (int u = 0; u < kSortBatch; ++u) {
      const int f = b0 + 32 * u + lane;
      ev[u] = f < f1 ? a.ids[f] : -1;
    }
#pragma unroll
    for (int u = 0; u < kSortBatch; ++u) {
      const int f = b0 + 32 * u + lane;
      int e = ev[u];
      if (e >= E || (f < f1 && e < 0)) {
        set_device_error(kErrExpertRange);
        e = -1;
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && (peers & ((1u << lane) - 1u)) == 0) my_cnt_row[e] += __popc(peers);
      __syncwarp();  // this step's counts before the next step's reads
    }
  }
  __syncthreads();

  // 2. exclusive prefix over warps (per expert), then over padded segments
  int my_cnt = 0;
  if (tid < E) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = warp_cnt[w * E + tid];
      warp_cnt[w * E + tid] = run;
      run += c;
    }
    my_cnt = run;
    cnt[tid] = run;
  }
  const int my_pad = tid < E ? (my_cnt + a.bm - 1) / a.bm * a.bm : 0;
  int incl = my_pad;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = wsum[lane];
    int s = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += o;
    }
    wsum[lane] = s - v;  // exclusive over warps
  }
  __syncthreads();
  const int excl = incl - my_pad + wsum[warp];
  if (tid < E) {
    base[tid] = excl;
    a.counts[tid] = my_cnt;
    a.offsets[tid] = excl;
    if (tid == E - 1) {
      a.offsets[E] = excl + my_pad;
      *a.num_padded = excl + my_pad;
    }
    for (int b = excl / a.bm; b < (excl + my_pad) / a.bm; ++b) a.block_expert[b] = tid;
    for (int p = excl + my_cnt; p < excl + my_pad; ++p) a.sorted[p] = a.N;  // sentinel
    for (int w = 0; w < 32; ++w) warp_cnt[w * E + tid] += excl;  // absolute start of warp w's slots of tid
  }
  __syncthreads();

  // 3. stable placement, each warp in its chunk's order (ids batched as above)
  for (int b0 = f0; b0 < f1; b0 += 32 * kSortBatch) {
    int ev[kSortBatch];
#pragma unroll
    for (int u = 0; u < kSortBatch; ++u) {
      const int f = b0 + 32 * u + lane;
      ev[u] = f < f1 ? a.ids[f] : -1;
    }
#pragma unroll
    for (int u = 0; u < kSortBatch; ++u) {
      const int f = b0 + 32 * u + lane;
      int e = ev[u];
      if (e >= E) e = -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      const uint32_t lower = peers & ((1u << lane) - 1u);
      int pos = 0;
      if (e >= 0) pos = my_cnt_row[e] + __popc(lower);
      __syncwarp();
      if (e >= 0) {
        a.sorted[pos] = f;
        if (lower == 0) my_cnt_row[e] += __popc(peers);
      }
      __syncwarp();
    }
  }
}

}  // namespace moe
