// sort.cuh - align/sort of the routed slots by expert, one CTA.
//
// vllm-project/vllm PR 65207, reviewer measurements ("Commits 2 and 3"):
// moe_sorting is run without zeroing the layer output; here the sort never
// touches the output (the stage-2 epilogue writes every output row).
// ROCm/aiter PR 6106, "Technical Details": GEMM rows follow this gather index.
#pragma once
#include "ptx.cuh"

namespace moe {

constexpr int kSortThreads = 1024;

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

  for (int e = tid; e < E; e += kSortThreads) cnt[e] = 0;
  __syncthreads();
  for (int f = tid; f < a.N; f += kSortThreads) {
    const int e = a.ids[f];
    if (e >= 0 && e < E) {
      atomicAdd(&cnt[e], 1);
    } else {
      set_device_error(kErrExpertRange);
    }
  }
  __syncthreads();

  // Exclusive prefix sum of the padded segment sizes (E <= 1024: one per thread).
  const int my_cnt = tid < E ? cnt[tid] : 0;
  const int my_pad = (my_cnt + a.bm - 1) / a.bm * a.bm;
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
  }
  __syncthreads();

  // Stable placement, 1024 slots per round: position = segment base + slots
  // of the same expert in earlier warps of this round + rank inside the warp.
  for (int start = 0; start < a.N; start += kSortThreads) {
    const int f = start + tid;
    int e = f < a.N ? a.ids[f] : -1;
    if (e >= E) e = -1;
    for (int i = tid; i < 32 * E; i += kSortThreads) warp_cnt[i] = 0;
    __syncthreads();
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rank == 0) warp_cnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (tid < E) {
      int run = base[tid];
      for (int w = 0; w < 32; ++w) {
        const int c = warp_cnt[w * E + tid];
        warp_cnt[w * E + tid] = run;
        run += c;
      }
      base[tid] = run;
    }
    __syncthreads();
    if (e >= 0) a.sorted[warp_cnt[warp * E + e] + rank] = f;
    __syncthreads();
  }
}

}  // namespace moe
