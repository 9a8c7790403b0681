// sort.cuh - align/sort of the routed slots by expert: one CTA of 32 warps
// for small batches, a cluster of kSortCluster such CTAs for large ones.
//
// vllm-project/vllm PR 65207, reviewer measurements ("Commits 2 and 3"):
// moe_sorting is run without zeroing the layer output; here the sort never
// touches the output (the stage-2 epilogue writes every output row).
// ROCm/aiter PR 6106, "Technical Details": GEMM rows follow this gather index.
#pragma once
#include "ptx.cuh"

namespace moe {

constexpr int kSortThreads = 1024;
constexpr int kSortCluster = 8;              // CTAs of the cluster sort
constexpr int kSortClusterMinSlots = 4096;   // slots from which the cluster sort runs
constexpr int kSortClusterBatch = 4;         // id loads per warp in flight (cluster sort)

struct SortArgs {
  const int32_t* ids;  // [N] flat slots f = t*k + j
  int N, E, bm;
  int32_t* sorted;        // [capacity]
  int32_t* block_expert;  // [capacity / bm]
  int32_t* counts;        // [E]
  int32_t* offsets;       // [E+1]
  int32_t* num_padded;    // [1]
};

// Shared memory of either kernel: tot[E] (this CTA's counts), seg_cnt[E] and
// seg_start[E] (every expert's count and padded segment start),
// warp_cnt[32][E], warp sums [32].
__host__ __device__ constexpr size_t sort_smem_bytes(int E) {
  return (3 * static_cast<size_t>(E) + 32 * static_cast<size_t>(E) + 32) * sizeof(int);
}

// Each warp owns one contiguous range [f0, f1) of the flat slots, so that a
// stable order needs no barrier per round:
//   1. the warp counts its range's slots per expert into its own row of
//      warp_cnt (32 slots per step, __match_any_sync groups equal experts, the
//      lowest lane of a group adds the group's size: one writer per entry);
//   2. exclusive prefixes - over the warps (and, in the cluster sort, over the
//      CTAs before this one) per expert, and over the experts' padded segment
//      sizes - turn each warp_cnt entry into the absolute position of that
//      warp's first slot of that expert; counts, offsets, block owners and
//      padding are written once;
//   3. the warp walks its range again in order and places every slot at its
//      entry plus its rank among the equal experts of its 32-slot step, then
//      advances the entry: ascending f inside every expert segment.
// B: 32-slot steps whose ids a warp loads before it uses any (B loads in
// flight instead of one per step; the single-CTA sort of small batches,
// whose warps take a step or two, is fastest with B = 1).
template <int B>
__device__ __forceinline__ void sort_count(const SortArgs& a, int f0, int f1, int* my_cnt_row) {
  const int lane = threadIdx.x & 31;
  for (int b0 = f0; b0 < f1; b0 += 32 * B) {
    int ev[B];
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int f = b0 + 32 * u + lane;
      ev[u] = f < f1 ? a.ids[f] : -1;
    }
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int f = b0 + 32 * u + lane;
      int e = ev[u];
      if (e >= a.E || (f < f1 && e < 0)) {
        set_device_error(kErrExpertRange);
        e = -1;
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && (peers & ((1u << lane) - 1u)) == 0) my_cnt_row[e] += __popc(peers);
      __syncwarp();  // this step's counts before the next step's reads
    }
  }
}

template <int B>
__device__ __forceinline__ void sort_place(const SortArgs& a, int f0, int f1, int* my_cnt_row) {
  const int lane = threadIdx.x & 31;
  for (int b0 = f0; b0 < f1; b0 += 32 * B) {
    int ev[B];
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int f = b0 + 32 * u + lane;
      ev[u] = f < f1 ? a.ids[f] : -1;
    }
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int f = b0 + 32 * u + lane;
      int e = ev[u];
      if (e >= a.E) e = -1;
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

// Per expert e = threadIdx.x < E: warp_cnt[w][e] becomes the exclusive prefix
// over warps; returns this CTA's count of e (0 for other threads).
__device__ __forceinline__ int sort_warp_prefix(int* warp_cnt, int E) {
  const int tid = threadIdx.x;
  int run = 0;
  if (tid < E) {
    for (int w = 0; w < 32; ++w) {
      const int c = warp_cnt[w * E + tid];
      warp_cnt[w * E + tid] = run;
      run += c;
    }
  }
  return run;
}

// Exclusive prefix over experts of the padded segment sizes (block-wide;
// every thread calls it); returns expert tid's segment start.
__device__ __forceinline__ int sort_segment_prefix(int my_pad, int* wsum) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int incl = my_pad;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = wsum[lane];
    int s = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += o;
    }
    wsum[lane] = s - v;  // exclusive over warps
  }
  __syncthreads();
  return incl - my_pad + wsum[warp];
}

// Expert tid's count and offset (and, for the last expert, the total).
__device__ __forceinline__ void sort_write_segment(const SortArgs& a, int e, int cnt, int excl, int pad) {
  a.counts[e] = cnt;
  a.offsets[e] = excl;
  if (e == a.E - 1) {
    a.offsets[a.E] = excl + pad;
    *a.num_padded = excl + pad;
  }
}

// Block owners and sentinel padding of one expert, by one thread: the
// single-CTA sort's way at token blocks of up to 32 (at most 31 padding
// slots), where it measured faster than sort_fill_padding (decode layer
// sort 6.6 -> 4.7 us).
__device__ __forceinline__ void sort_fill_expert(const SortArgs& a, int e, int cnt, int excl, int pad) {
  for (int b = excl / a.bm; b < (excl + pad) / a.bm; ++b) a.block_expert[b] = e;
  for (int p = excl + cnt; p < excl + pad; ++p) a.sorted[p] = a.N;  // sentinel
}

// Block owners and sentinel padding of every expert, from seg_cnt / seg_start
// in shared memory. The parts x 32 warps (every warp of every CTA taking part)
// share the experts: warp w of part r takes experts e = 32 r + w, then every
// (32 parts)-th after it, its lanes writing consecutive positions. (A segment
// has up to bm - 1 padding slots; one thread per expert would issue them as
// that many scattered stores, one after another.)
__device__ __forceinline__ void sort_fill_padding(const SortArgs& a, const int* seg_cnt, const int* seg_start,
                                                  int part, int parts) {
  const int lane = threadIdx.x & 31;
  const int gw = part * 32 + (threadIdx.x >> 5);
  for (int e = gw; e < a.E; e += parts * 32) {
    const int start = seg_start[e], cnt = seg_cnt[e];
    const int end = start + (cnt + a.bm - 1) / a.bm * a.bm;
    for (int b = start / a.bm + lane; b < end / a.bm; b += 32) a.block_expert[b] = e;
    for (int p = start + cnt + lane; p < end; p += 32) a.sorted[p] = a.N;  // sentinel
  }
}

// One CTA: warp w owns chunk w of 32 equal chunks of the slots.
__global__ void __launch_bounds__(kSortThreads) k_align_sort(const SortArgs a) {
  extern __shared__ int ssm[];
  const int E = a.E;
  int* seg_cnt = ssm + E;
  int* seg_start = seg_cnt + E;
  int* warp_cnt = seg_start + E;
  int* wsum = warp_cnt + 32 * E;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int chunk = (a.N + 31) / 32;
  const int f0 = warp * chunk;
  const int f1 = f0 + chunk < a.N ? f0 + chunk : a.N;
  int* my_cnt_row = warp_cnt + warp * E;

  for (int i = tid; i < 32 * E; i += kSortThreads) warp_cnt[i] = 0;
  __syncthreads();
  sort_count<1>(a, f0, f1, my_cnt_row);
  __syncthreads();
  const int cnt = sort_warp_prefix(warp_cnt, E);
  const int pad = tid < E ? (cnt + a.bm - 1) / a.bm * a.bm : 0;
  const int excl = sort_segment_prefix(pad, wsum);
  const bool per_thread_pad = a.bm <= 32;
  if (tid < E) {
    sort_write_segment(a, tid, cnt, excl, pad);
    if (per_thread_pad) sort_fill_expert(a, tid, cnt, excl, pad);
    seg_cnt[tid] = cnt;
    seg_start[tid] = excl;
    for (int w = 0; w < 32; ++w) warp_cnt[w * E + tid] += excl;  // absolute start of warp w's slots of tid
  }
  __syncthreads();
  if (!per_thread_pad) sort_fill_padding(a, seg_cnt, seg_start, 0, 1);
  sort_place<1>(a, f0, f1, my_cnt_row);
}

// kSortCluster CTAs: CTA r owns part r of kSortCluster equal parts of the
// slots, its warps 32 equal chunks of that part. After each CTA's counts, a
// cluster barrier makes every CTA's per-expert totals readable over
// distributed shared memory; each CTA adds up, per expert, the totals of all
// CTAs (the segment sizes, identical in every CTA) and of the CTAs before it
// (its start inside the segment). CTA 0 writes the counts and offsets; the
// padding of the segments is spread over the warps of all CTAs. A second
// cluster barrier, arrived at once the totals are read and waited on at the
// end, keeps every CTA's shared memory alive until the others have read it.
__global__ void __cluster_dims__(kSortCluster, 1, 1) __launch_bounds__(kSortThreads)
    k_align_sort_cluster(const SortArgs a) {
  extern __shared__ int ssm[];
  const int E = a.E;
  int* tot = ssm;  // this CTA's count of each expert, read by the cluster
  int* seg_cnt = ssm + E;
  int* seg_start = seg_cnt + E;
  int* warp_cnt = seg_start + E;
  int* wsum = warp_cnt + 32 * E;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int rank = static_cast<int>(cluster_ctarank());
  const int part = (a.N + kSortCluster - 1) / kSortCluster;
  const int p0 = rank * part < a.N ? rank * part : a.N;
  const int p1 = p0 + part < a.N ? p0 + part : a.N;
  const int chunk = (p1 - p0 + 31) / 32;
  const int f0 = p0 + warp * chunk < p1 ? p0 + warp * chunk : p1;
  const int f1 = f0 + chunk < p1 ? f0 + chunk : p1;
  int* my_cnt_row = warp_cnt + warp * E;

  for (int i = tid; i < 32 * E; i += kSortThreads) warp_cnt[i] = 0;
  __syncthreads();
  sort_count<kSortClusterBatch>(a, f0, f1, my_cnt_row);
  __syncthreads();
  const int mine = sort_warp_prefix(warp_cnt, E);
  if (tid < E) tot[tid] = mine;
  cluster_sync_all();  // every CTA's totals written and visible
  int cnt = 0, before = 0;
  if (tid < E) {
    // every remote load issued before any is used
    const uint32_t addr = smem_u32(tot + tid);
    int c[kSortCluster];
#pragma unroll
    for (int r = 0; r < kSortCluster; ++r) c[r] = ld_shared_cluster_s32(mapa_shared(addr, static_cast<uint32_t>(r)));
#pragma unroll
    for (int r = 0; r < kSortCluster; ++r) {
      if (r < rank) before += c[r];
      cnt += c[r];
    }
  }
  cluster_arrive_release();  // this CTA has read every other CTA's totals
  const int pad = tid < E ? (cnt + a.bm - 1) / a.bm * a.bm : 0;
  const int excl = sort_segment_prefix(pad, wsum);
  if (tid < E) {
    if (rank == 0) sort_write_segment(a, tid, cnt, excl, pad);
    seg_cnt[tid] = cnt;
    seg_start[tid] = excl;
    const int start = excl + before;
    for (int w = 0; w < 32; ++w) warp_cnt[w * E + tid] += start;
  }
  __syncthreads();
  sort_fill_padding(a, seg_cnt, seg_start, rank, kSortCluster);
  sort_place<kSortClusterBatch>(a, f0, f1, my_cnt_row);
  cluster_wait_acquire();  // no CTA leaves while another may still read its totals
}

}  // namespace moe
