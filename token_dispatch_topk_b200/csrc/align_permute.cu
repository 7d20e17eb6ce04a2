// align_permute.cu -- per-expert histogram, block-padded prefix and stable placement.
//
// Operation: "Upstream Reference: Deep-Spark xllm + vllm", "File Index"
// (moe_align_sum_kernels.cu: block alignment for scatter), with the expert-parallel
// remap of the 2026-07-16 MTP1 M=2 compact scheduler closure note (scheduler
// paragraph: each local expert's row count and remapped-row prefix come from topk_ids
// plus expert_map; coverage paragraph: an all-remote rank is valid).
//
// Slots s = t*k + j are cut into tiles of `tile_slots` consecutive slots.
//   count kernel (one CTA per tile): local expert of every slot, warp-aggregated
//     shared-memory histogram (match.any groups equal experts so one lane adds for
//     the whole group), tile counts to the workspace.  The CTA that finishes last
//     (completion ticket, no spinning) scans the tile counts per expert into
//     exclusive per-tile prefixes, writes counts, the block-padded offsets and
//     N_pad, and resets the ticket for the next call.
//   place kernel (one CTA per tile): every warp owns a contiguous run of the
//     tile's slots; per-warp histograms are scanned across warps, then each warp
//     walks its run in order and gives every slot the row
//        offsets[e] + tile prefix[e] + warp prefix[e] + rank among equal experts
//     in its 32-slot chunk (ballot-free: match.any + popc of the lower lanes).
//     Rows therefore follow (expert, slot) order exactly, with no dependence on
//     atomic ordering.  The same kernel writes the pad value into the pad rows,
//     the tail rows past N_pad, and expert_ids.
// When all slots fit one tile (decode, small batches), the count kernel does
// everything in one CTA and the place kernel is not launched.
// moe_align_permute takes these kernels above 65 536 slots (or 512 local experts), one
// thread-block cluster (align_cluster_kernel, below) up to 4096 slots, and between the two
// the tile kernels of the fused dispatch (route_fused.cu, moe_internal::align_tiles).
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "route_internal.h"

namespace {

constexpr int kAlignThreads = 512;
constexpr int kAlignWarps = kAlignThreads / 32;
constexpr int kWsHeaderBytes = 256;  // status word, ticket, padding

struct AlignArgs {
  const int32_t* topk_ids;
  const int32_t* expert_map;
  int64_t P;  // slots = T*k
  int E_global;
  int E_local;
  int bs;
  int64_t C;  // capacity rows
  int NB;     // blocks
  int tile_slots;
  int num_tiles;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_ids;
  int32_t* expert_ids;
  int32_t* n_pad;
  int32_t* inv_perm;
  int32_t* status;
  unsigned int* ticket;
  int32_t* tile_counts;  // [num_tiles][E_local]
};

// Local expert of slot s, or -1 (remote).  Bad ids are remote and flagged.
__device__ __forceinline__ int local_expert(const AlignArgs& a, int64_t s) {
  const int g = a.topk_ids[s];
  if (static_cast<unsigned>(g) >= static_cast<unsigned>(a.E_global)) {
    moe::record_status(a.status, MOE_ERR_BAD_EXPERT_ID);
    return -1;
  }
  const int le = a.expert_map != nullptr ? a.expert_map[g] : g;
  if (le < -1 || le >= a.E_local) {
    moe::record_status(a.status, MOE_ERR_BAD_EXPERT_ID);
    return -1;
  }
  return le;
}

// Lanes of this warp that hold the same value v >= 0, as a bit mask (0 for v < 0).  Uses a
// per-warp array of masks in shared memory, indexed by value, that is all zero on entry and is
// left all zero: one atomic OR, one read and one reset per lane, whatever the number of distinct
// values (match.any costs grow with it).
__device__ __forceinline__ unsigned peers_smem(unsigned* masks, int v, int lane) {
  if (v >= 0) atomicOr(&masks[v], 1u << lane);
  __syncwarp();
  const unsigned p = v >= 0 ? masks[v] : 0u;
  __syncwarp();
  if (v >= 0) masks[v] = 0u;
  __syncwarp();
  return p;
}

// Block-wide exclusive scan of n <= 2*kAlignThreads ints in shared memory (in place).
// Returns the total.  Every thread of the block must call it.
__device__ int block_exclusive_scan(int* data, int n, int* warp_sums) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i0 = 2 * tid, i1 = 2 * tid + 1;
  const int a = i0 < n ? data[i0] : 0;
  const int b = i1 < n ? data[i1] : 0;
  int incl = a + b;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kAlignWarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += v;
    }
    if (lane < kAlignWarps) warp_sums[lane] = w;  // inclusive warp prefix
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + incl - (a + b);
  const int total = warp_sums[kAlignWarps - 1];
  __syncthreads();
  if (i0 < n) data[i0] = before;
  if (i1 < n) data[i1] = before + a;
  __syncthreads();
  return total;
}

// counts (s_cnt) -> block-padded exclusive offsets (s_off, E_local+1 entries); writes the
// counts/offsets/N_pad outputs.  Block-wide.
__device__ void padded_offsets(const AlignArgs& a, const int* s_cnt, int* s_off, int* warp_sums) {
  for (int e = threadIdx.x; e < a.E_local; e += blockDim.x) {
    const int c = s_cnt[e];
    s_off[e] = ((c + a.bs - 1) / a.bs) * a.bs;
  }
  __syncthreads();
  const int total = block_exclusive_scan(s_off, a.E_local, warp_sums);
  if (threadIdx.x == 0) {
    s_off[a.E_local] = total;
    a.offsets[a.E_local] = total;
    a.n_pad[0] = total;
  }
  for (int e = threadIdx.x; e < a.E_local; e += blockDim.x) {
    a.offsets[e] = s_off[e];
    a.counts[e] = s_cnt[e];
  }
  __syncthreads();
}

// Pad value into every non-slot row, expert_ids for every block.  Work is split over
// `nworkers` CTAs; this CTA is `worker`.
__device__ void fill_pads_and_blocks(const AlignArgs& a, const int* s_cnt, const int* s_off, int worker,
                                     int nworkers) {
  const int npad = s_off[a.E_local];
  const int64_t pad_items = static_cast<int64_t>(a.E_local) * a.bs;
  const int64_t tail = a.C - npad;
  const int32_t pad_value = static_cast<int32_t>(a.P);
  const int64_t stride = static_cast<int64_t>(nworkers) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(worker) * blockDim.x + threadIdx.x; i < pad_items + tail; i += stride) {
    if (i < pad_items) {
      const int e = static_cast<int>(i / a.bs);
      const int r = static_cast<int>(i - static_cast<int64_t>(e) * a.bs);
      const int p = s_off[e] + s_cnt[e] + r;
      if (p < s_off[e + 1]) a.sorted_ids[p] = pad_value;
    } else {
      a.sorted_ids[npad + (i - pad_items)] = pad_value;
    }
  }
  // expert of each block: the largest e with offsets[e] <= b*bs (empty experts share offsets
  // with their successor, so the largest such e is the non-empty one), -1 past N_pad.
  for (int64_t b = static_cast<int64_t>(worker) * blockDim.x + threadIdx.x; b < a.NB; b += stride) {
    const int64_t row = b * a.bs;
    int e = -1;
    if (row < npad) {
      int lo = 0, hi = a.E_local - 1;  // invariant: s_off[lo] <= row
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= row) lo = mid; else hi = mid - 1;
      }
      e = lo;
    }
    a.expert_ids[b] = e;
  }
}

// Stable placement of one tile.  s_base[e] = first row of this tile's slots of expert e.
// s_whist: [kAlignWarps][E_local] scratch, s_le: [tile_slots] scratch, s_masks:
// [kAlignWarps][E_local] all-zero masks (left all zero).
__device__ void place_tile(const AlignArgs& a, int tile, const int* s_base, int* s_whist, int* s_le,
                           unsigned* s_masks) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t s0 = static_cast<int64_t>(tile) * a.tile_slots;
  const int64_t s1 = (s0 + a.tile_slots < a.P) ? s0 + a.tile_slots : a.P;
  const int per_warp = ((a.tile_slots / kAlignWarps) + 31) & ~31;
  const int64_t w0 = s0 + static_cast<int64_t>(warp) * per_warp;
  const int64_t w1 = (w0 + per_warp < s1) ? w0 + per_warp : s1;
  int* my_hist = s_whist + warp * a.E_local;
  unsigned* my_masks = s_masks + warp * a.E_local;

  for (int i = tid; i < kAlignWarps * a.E_local; i += blockDim.x) s_whist[i] = 0;
  __syncthreads();
  // pass 1: per-warp histogram of its own run
  for (int64_t s = w0 + lane; s < w1; s += 32) {
    const int le = local_expert(a, s);
    s_le[s - s0] = le;
    if (le >= 0) atomicAdd(&my_hist[le], 1);
  }
  __syncthreads();
  // pass 2: exclusive scan over warps, seeded with the tile's base row
  for (int e = tid; e < a.E_local; e += blockDim.x) {
    int run = s_base[e];
    for (int w = 0; w < kAlignWarps; ++w) {
      const int c = s_whist[w * a.E_local + e];
      s_whist[w * a.E_local + e] = run;
      run += c;
    }
  }
  __syncthreads();
  // pass 3: rows in slot order
  for (int64_t base = w0; base < w1; base += 32) {
    const int64_t s = base + lane;
    const int le = s < w1 ? s_le[s - s0] : -1;
    const unsigned peers = peers_smem(my_masks, le, lane);
    if (le >= 0) {
      const int row = my_hist[le] + __popc(peers & moe::lanemask_lt());
      a.sorted_ids[row] = static_cast<int32_t>(s);
      a.inv_perm[s] = row;
    } else if (s < w1) {
      a.inv_perm[s] = -1;
    }
    __syncwarp();
    if (le >= 0 && lane == __ffs(peers) - 1) my_hist[le] += __popc(peers);
    __syncwarp();
  }
}

// Shared-memory layout of both kernels (ints):
//   s_cnt[E_local] | s_off[E_local+1] | warp_sums[32] | s_whist[kAlignWarps*E_local] | s_le[tile_slots]
//   | s_tile_base[E_local] (place kernel) | s_masks[kAlignWarps*E_local]
__host__ __device__ inline size_t align_smem_ints(int E_local, int tile_slots) {
  return static_cast<size_t>(E_local) + (E_local + 1) + 32 + static_cast<size_t>(kAlignWarps) * E_local +
         tile_slots + E_local + static_cast<size_t>(kAlignWarps) * E_local;
}

__global__ void __launch_bounds__(kAlignThreads) align_count_kernel(AlignArgs a) {
  extern __shared__ int smem[];
  int* s_cnt = smem;
  int* s_off = s_cnt + a.E_local;
  int* warp_sums = s_off + a.E_local + 1;
  int* s_whist = warp_sums + 32;
  int* s_le = s_whist + kAlignWarps * a.E_local;
  unsigned* s_masks = reinterpret_cast<unsigned*>(s_le + a.tile_slots + a.E_local);
  __shared__ int s_is_last;

  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int64_t s0 = static_cast<int64_t>(tile) * a.tile_slots;
  const int64_t s1 = (s0 + a.tile_slots < a.P) ? s0 + a.tile_slots : a.P;

  for (int e = tid; e < a.E_local; e += blockDim.x) s_cnt[e] = 0;
  for (int i = tid; i < kAlignWarps * a.E_local; i += blockDim.x) s_masks[i] = 0u;
  __syncthreads();
  for (int64_t s = s0 + tid; s < s1; s += kAlignThreads) {
    const int le = local_expert(a, s);
    if (le >= 0) atomicAdd(&s_cnt[le], 1);
  }
  __syncthreads();

  if (a.num_tiles == 1) {
    // everything in this CTA
    padded_offsets(a, s_cnt, s_off, warp_sums);
    place_tile(a, 0, s_off, s_whist, s_le, s_masks);
    fill_pads_and_blocks(a, s_cnt, s_off, 0, 1);
    return;
  }

  int32_t* mine = a.tile_counts + static_cast<int64_t>(tile) * a.E_local;
  for (int e = tid; e < a.E_local; e += blockDim.x) mine[e] = s_cnt[e];
  __threadfence();
  __syncthreads();
  if (tid == 0) s_is_last = (atomicAdd(a.ticket, 1u) == static_cast<unsigned>(a.num_tiles - 1)) ? 1 : 0;
  __syncthreads();
  if (!s_is_last) return;
  __threadfence();

  // Last CTA: per-expert exclusive scan over tiles.  `parts` threads share one expert, each
  // scanning a contiguous range of tiles, so all threads work when E_local is small.
  int parts = 1;
  while (parts * 2 * a.E_local <= kAlignThreads && parts * 2 <= 32) parts *= 2;
  const int experts_per_pass = kAlignThreads / parts;
  const int part = tid % parts;
  const int per = (a.num_tiles + parts - 1) / parts;
  const int t0 = part * per;
  const int t1 = (t0 + per < a.num_tiles) ? t0 + per : a.num_tiles;
  for (int e0 = 0; e0 < a.E_local; e0 += experts_per_pass) {  // uniform trip count
    const int e = e0 + tid / parts;
    int sum = 0;
    if (e < a.E_local) {
      for (int t = t0; t < t1; ++t) sum += __ldcg(a.tile_counts + static_cast<int64_t>(t) * a.E_local + e);
    }
    // exclusive prefix of the part sums inside each group of `parts` lanes (groups never straddle a warp)
    int incl = sum;
    for (int off = 1; off < parts; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off, parts);
      if (part >= off) incl += v;
    }
    if (e < a.E_local) {
      int run = incl - sum;
      for (int t = t0; t < t1; ++t) {
        int32_t* p = a.tile_counts + static_cast<int64_t>(t) * a.E_local + e;
        const int c = __ldcg(p);
        *p = run;
        run += c;
      }
      if (part == parts - 1) s_cnt[e] = run;
    }
  }
  __syncthreads();
  padded_offsets(a, s_cnt, s_off, warp_sums);
  if (tid == 0) *a.ticket = 0u;  // ready for the next call
}

__global__ void __launch_bounds__(kAlignThreads) align_place_kernel(AlignArgs a) {
  extern __shared__ int smem[];
  int* s_cnt = smem;
  int* s_off = s_cnt + a.E_local;
  int* warp_sums = s_off + a.E_local + 1;
  int* s_whist = warp_sums + 32;
  int* s_le = s_whist + kAlignWarps * a.E_local;
  int* s_tile_base = s_le + a.tile_slots;  // [E_local]: first row of this tile's slots per expert
  unsigned* s_masks = reinterpret_cast<unsigned*>(s_tile_base + a.E_local);
  const int tile = blockIdx.x;
  for (int i = threadIdx.x; i < kAlignWarps * a.E_local; i += blockDim.x) s_masks[i] = 0u;
  for (int e = threadIdx.x; e <= a.E_local; e += blockDim.x) {
    s_off[e] = a.offsets[e];
    if (e < a.E_local) {
      s_cnt[e] = a.counts[e];
      s_tile_base[e] = a.offsets[e] + a.tile_counts[static_cast<int64_t>(tile) * a.E_local + e];
    }
  }
  __syncthreads();
  place_tile(a, tile, s_tile_base, s_whist, s_le, s_masks);
  __syncthreads();
  fill_pads_and_blocks(a, s_cnt, s_off, tile, a.num_tiles);
}

// ------------------------------------------------------------------------------------------
// Single-launch align on one thread-block cluster (up to 16 CTAs on distinct SMs), used up to
// 65536 slots with at most 512 local experts (larger batches take the two tile kernels above,
// which spread over every SM).  Global warp g = rank*32 + w owns the slot run [g*run, (g+1)*run).
//   1. every warp counts its run into its own shared-memory row (shared atomics; the ids of up
//      to 8 chunks are loaded at once and their experts kept for step 5);
//   2. per expert, the CTA turns its warp rows into exclusive prefixes and its CTA total;
//   3. every CTA pushes its totals into row `rank` of a table in the shared memory of every CTA
//      (16-byte st.shared::cluster stores); cluster barrier; each CTA scans its own table: the
//      sum over lower ranks is its base, the sum over all ranks is the expert's count;
//   4. block-padded offsets (each CTA computes them; rank 0 writes counts/offsets/N_pad);
//   5. every warp walks its run again and places its slots in order (peer masks from shared
//      memory, rank = earlier peers in the chunk);
//   6. pad rows, tail rows and expert_ids, split over the cluster.
// Steps 2 and 3 are warp shuffle scans: lane = warp index (32 warps) or lane = CTA rank; four
// experts are scanned at once to overlap the shuffle latencies.  The cluster barrier is the only
// inter-CTA synchronisation.
// ------------------------------------------------------------------------------------------
constexpr int kClusterThreads = 1024;
constexpr int kClusterWarps = kClusterThreads / 32;
constexpr int kMaxClusterCtas = 16;
constexpr int64_t kClusterMaxSlots = 65536;
constexpr int64_t kAlignTilesMinSlots = 4096;  // above this (up to kClusterMaxSlots): the tile kernels
constexpr int kClusterMaxExperts = 512;

// Exclusive scan of n <= 1024 ints in shared memory, one per thread of a 1024-thread block.
__device__ int block_exclusive_scan_1024(int* data, int n, int* warp_sums) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int v = tid < n ? data[tid] : 0;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += x;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += x;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + incl - v;
  const int total = warp_sums[31];
  __syncthreads();
  if (tid < n) data[tid] = before;
  __syncthreads();
  return total;
}

// Row stride of the per-warp counters and of the cluster table: odd, so that 32 lanes reading one
// expert column of 32 rows hit 32 different banks.
__host__ __device__ inline int warp_row_stride(int E_local) { return E_local | 1; }

// Row length of the cluster totals table: a multiple of 4 ints (16-byte rows for vector stores).
__host__ __device__ inline int table_row_ints(int E_local) { return (E_local + 3) & ~3; }

constexpr int kAlignBatch = 8;  // 32-slot chunks whose ids a warp loads at once

// Local experts of one batch of a warp's run: slot base + 32*b + lane for b < kAlignBatch.  All
// id loads (then all map loads) are issued before any is used.
__device__ __forceinline__ void load_batch(const AlignArgs& a, int64_t base, int64_t end, int lane,
                                           int (&le)[kAlignBatch]) {
  int g[kAlignBatch];
#pragma unroll
  for (int b = 0; b < kAlignBatch; ++b) {
    const int64_t s = base + 32 * b + lane;
    g[b] = s < end ? a.topk_ids[s] : -2;
  }
#pragma unroll
  for (int b = 0; b < kAlignBatch; ++b) {
    int v = -1;
    if (g[b] != -2) {
      if (static_cast<unsigned>(g[b]) >= static_cast<unsigned>(a.E_global)) {
        moe::record_status(a.status, MOE_ERR_BAD_EXPERT_ID);
      } else {
        v = a.expert_map != nullptr ? a.expert_map[g[b]] : g[b];
        if (v < -1 || v >= a.E_local) {
          moe::record_status(a.status, MOE_ERR_BAD_EXPERT_ID);
          v = -1;
        }
      }
    }
    le[b] = v;
  }
}

__global__ void __launch_bounds__(kClusterThreads) align_cluster_kernel(AlignArgs a, int64_t run) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int nc = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int El = a.E_local;
  const int ES = warp_row_stride(El);
  extern __shared__ int smem[];
  int* whist = smem;                                                          // [32][ES] counts, then prefixes
  unsigned* masks = reinterpret_cast<unsigned*>(whist + kClusterWarps * ES);  // [32][El] peer masks
  const int E4 = table_row_ints(El);
  int* table = reinterpret_cast<int*>(masks + kClusterWarps * El);  // [kMaxClusterCtas][E4] totals of every rank
  int* cta_cnt = table + kMaxClusterCtas * E4;                      // [E4] this CTA's totals
  int* s_cnt = cta_cnt + E4;                                        // [El] cluster counts
  int* s_off = s_cnt + El;                                          // [El+1] padded offsets
  int* s_base = s_off + El + 1;                                     // [El] this CTA's first rows
  int* warp_sums = s_base + El;                                     // [32]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t g = static_cast<int64_t>(rank) * kClusterWarps + warp;
  const int64_t w0 = g * run;
  const int64_t w1 = (w0 + run < a.P) ? w0 + run : a.P;
  int* my_hist = whist + warp * ES;
  unsigned* my_masks = masks + warp * El;
  const bool one_batch = run <= 32 * kAlignBatch;  // the whole run's experts stay in registers

  for (int i = tid; i < kClusterWarps * ES; i += kClusterThreads) whist[i] = 0;
  for (int i = tid; i < kClusterWarps * El; i += kClusterThreads) masks[i] = 0u;
  for (int i = El + tid; i < E4; i += kClusterThreads) cta_cnt[i] = 0;
  __syncthreads();
  // let the next kernel start now: it waits for this one in turn, and the first kernel of the
  // routing call has already waited for the producers of its inputs
  moe::pdl_launch_dependents();
  moe::pdl_wait();  // topk_ids come from the previous kernel
  // 1. per-warp counts of the warp's own run
  int le[kAlignBatch];
  for (int64_t base = w0; base < w1; base += 32 * kAlignBatch) {
    load_batch(a, base, w1, lane, le);
#pragma unroll
    for (int b = 0; b < kAlignBatch; ++b) {
      if (le[b] >= 0) atomicAdd(&my_hist[le[b]], 1);
    }
  }
  __syncthreads();
  // 2. per expert, exclusive prefix over this CTA's 32 warps (lane = warp index) and the CTA total
  for (int e0 = warp; e0 < El; e0 += 4 * kClusterWarps) {
    int c[4], incl[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = e0 + q * kClusterWarps;
      c[q] = e < El ? whist[lane * ES + e] : 0;
      incl[q] = c[q];
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int x = __shfl_up_sync(0xffffffffu, incl[q], off);
        if (lane >= off) incl[q] += x;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = e0 + q * kClusterWarps;
      if (e < El) {
        whist[lane * ES + e] = incl[q] - c[q];
        if (lane == 31) cta_cnt[e] = incl[q];
      }
    }
  }
  // 3. every CTA pushes its totals into row `rank` of the table of every CTA of the cluster
  //    (16-byte stores into distributed shared memory); after the cluster barrier each CTA scans
  //    its own table with lane = rank: the sum over lower ranks is its base, the sum over all
  //    ranks the count.  No CTA touches another's shared memory after that barrier.
  __syncthreads();
  if (nc > 1) {
    const int q4 = E4 / 4;
    for (int i = tid; i < nc * q4; i += kClusterThreads) {
      const int dst = i / q4;
      const int q = i - dst * q4;
      const uint4 v = *reinterpret_cast<const uint4*>(cta_cnt + 4 * q);
      moe::st_cluster_v4(table + rank * E4 + 4 * q, static_cast<uint32_t>(dst), v);
    }
    cluster.sync();
    for (int e0 = warp; e0 < El; e0 += 4 * kClusterWarps) {
      int c[4], incl[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = e0 + q * kClusterWarps;
        c[q] = (e < El && lane < nc) ? table[lane * E4 + e] : 0;
        incl[q] = c[q];
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int x = __shfl_up_sync(0xffffffffu, incl[q], off);
          if (lane >= off) incl[q] += x;
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = e0 + q * kClusterWarps;
        const int all = __shfl_sync(0xffffffffu, incl[q], 31);
        const int below = __shfl_sync(0xffffffffu, incl[q] - c[q], rank);
        if (lane == 0 && e < El) {
          s_base[e] = below;
          s_cnt[e] = all;
        }
      }
    }
  } else {
    for (int e = tid; e < El; e += kClusterThreads) {
      s_base[e] = 0;
      s_cnt[e] = cta_cnt[e];
    }
  }
  __syncthreads();
  // 4. block-padded offsets
  for (int e = tid; e < El; e += kClusterThreads) s_off[e] = ((s_cnt[e] + a.bs - 1) / a.bs) * a.bs;
  __syncthreads();
  const int total = block_exclusive_scan_1024(s_off, El, warp_sums);
  if (tid == 0) s_off[El] = total;
  __syncthreads();
  if (rank == 0) {
    for (int e = tid; e <= El; e += kClusterThreads) a.offsets[e] = s_off[e];
    for (int e = tid; e < El; e += kClusterThreads) a.counts[e] = s_cnt[e];
    if (tid == 0) a.n_pad[0] = total;
  }
  for (int e = tid; e < El; e += kClusterThreads) s_base[e] += s_off[e];
  __syncthreads();
  // 5. placement in slot order
  for (int64_t base = w0; base < w1; base += 32 * kAlignBatch) {
    if (!one_batch) load_batch(a, base, w1, lane, le);
    const int nb = static_cast<int>((w1 - base + 31) / 32);  // chunks of this batch that hold slots
#pragma unroll
    for (int b = 0; b < kAlignBatch; ++b) {
      if (b >= nb) break;  // uniform over the warp
      const int64_t s = base + 32 * b + lane;
      const unsigned peers = peers_smem(my_masks, le[b], lane);
      if (le[b] >= 0) {
        const int row = s_base[le[b]] + my_hist[le[b]] + __popc(peers & moe::lanemask_lt());
        a.sorted_ids[row] = static_cast<int32_t>(s);
        a.inv_perm[s] = row;
      } else if (s < w1) {
        a.inv_perm[s] = -1;
      }
      __syncwarp();
      if (le[b] >= 0 && lane == __ffs(peers) - 1) my_hist[le[b]] += __popc(peers);
      __syncwarp();
    }
  }
  // 6. pad rows (one warp per expert: fewer than bs rows each), tail rows, expert_ids
  const int32_t pad_value = static_cast<int32_t>(a.P);
  for (int e = rank * kClusterWarps + warp; e < El; e += nc * kClusterWarps) {
    const int p1 = s_off[e + 1];
    for (int p = s_off[e] + s_cnt[e] + lane; p < p1; p += 32) a.sorted_ids[p] = pad_value;
  }
  const uint32_t tail = static_cast<uint32_t>(a.C - total);
  for (uint32_t i = static_cast<uint32_t>(rank) * kClusterThreads + tid; i < tail;
       i += static_cast<uint32_t>(nc) * kClusterThreads)
    a.sorted_ids[total + i] = pad_value;
  for (int b = rank * kClusterThreads + tid; b < a.NB; b += nc * kClusterThreads) {
    const int64_t row = static_cast<int64_t>(b) * a.bs;
    int e = -1;
    if (row < total) {
      int lo = 0, hi = El - 1;  // largest e with s_off[e] <= row (empty experts share offsets)
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= row) lo = mid; else hi = mid - 1;
      }
      e = lo;
    }
    a.expert_ids[b] = e;
  }
}

__host__ inline size_t align_cluster_smem_bytes(int E_local) {
  const int E4 = table_row_ints(E_local);
  return (static_cast<size_t>(kClusterWarps) * warp_row_stride(E_local) + static_cast<size_t>(kClusterWarps) * E_local +
          static_cast<size_t>(kMaxClusterCtas + 1) * E4 + 3 * static_cast<size_t>(E_local) + 1 + 32) *
         sizeof(int);
}

// Tiling: one tile for up to 4096 slots (single-CTA path); otherwise tiles of 2048 slots,
// grown up to 8192 so that the last CTA's per-expert scan over tiles stays short.
int tile_slots_for(int64_t P) {
  if (P <= 4096) return 4096;
  int ts = 2048;
  while ((P + ts - 1) / ts > 256 && ts < 8192) ts *= 2;
  return ts;
}

int num_tiles_for(int64_t P, int ts) {
  const int64_t nt = (P + ts - 1) / ts;
  return nt < 1 ? 1 : static_cast<int>(nt);
}

}  // namespace

namespace {

// CTAs in the align cluster: one for small batches, else 8 (portable) or 16 when the device
// can co-schedule a 16-CTA cluster of this kernel.
int align_cluster_ctas(int64_t P, size_t smem) {
  if (P <= 4096) return 1;
  if (P <= 16384) return 8;
  if (cudaFuncSetAttribute(align_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    (void)cudaGetLastError();
    return 8;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kMaxClusterCtas);
  cfg.blockDim = dim3(kClusterThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kMaxClusterCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, align_cluster_kernel, &cfg) != cudaSuccess || clusters < 1) {
    (void)cudaGetLastError();
    return 8;
  }
  return kMaxClusterCtas;
}

moe_status_t launch_align_cluster(const AlignArgs& a, cudaStream_t st) {
  const size_t smem = align_cluster_smem_bytes(a.E_local);
  if (cudaFuncSetAttribute(align_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe_host::prefer_max_shared(reinterpret_cast<const void*>(align_cluster_kernel)) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int nc = align_cluster_ctas(a.P, smem);
  const int64_t warps = static_cast<int64_t>(nc) * kClusterWarps;
  int64_t run = (a.P + warps - 1) / warps;
  run = (run + 31) & ~int64_t{31};
  if (run < 32) run = 32;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nc);
  cfg.blockDim = dim3(kClusterThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nc;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  AlignArgs args = a;
  return cudaLaunchKernelEx(&cfg, align_cluster_kernel, args, run) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

extern "C" int64_t moe_align_capacity(int64_t T, int32_t k, int32_t E_local, int32_t block_size) {
  if (T < 0 || k < 1 || E_local < 1 || block_size < 1) return -1;
  if (T > (int64_t{1} << 40)) return -1;
  return T * k + static_cast<int64_t>(E_local) * (block_size - 1);
}

extern "C" int64_t moe_align_num_blocks(int64_t T, int32_t k, int32_t E_local, int32_t block_size) {
  const int64_t C = moe_align_capacity(T, k, E_local, block_size);
  if (C < 0) return -1;
  return (C + block_size - 1) / block_size;
}

namespace {
// Scratch of the count + place kernels and of the cluster kernel: header + per-tile (or per
// cluster rank) expert counters.
size_t count_place_scratch_bytes(int64_t T, int32_t k, int32_t E_local) {
  const int64_t P = T * k;
  const int ts = tile_slots_for(P);
  const int nt = num_tiles_for(P, ts);
  size_t rows = nt > 1 ? static_cast<size_t>(nt) : 0;  // per-tile counters of the tile kernels
  if (P > 4096 && rows < static_cast<size_t>(kMaxClusterCtas)) rows = kMaxClusterCtas;  // cluster table
  return kWsHeaderBytes + rows * static_cast<size_t>(E_local) * sizeof(int32_t);
}
}  // namespace

extern "C" size_t moe_align_workspace_bytes(int64_t T, int32_t k, int32_t E_local) {
  if (T < 0 || k < 1 || E_local < 1) return 0;
  const size_t own = count_place_scratch_bytes(T, k, E_local);
  const size_t tiles = moe_internal::align_tiles_workspace_bytes(T, E_local);  // the fused path's tile kernels
  return own > tiles ? own : tiles;
}

extern "C" moe_status_t moe_align_permute(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E_global,
                                          const int32_t* expert_map, int32_t E_local, int32_t block_size,
                                          int32_t* counts, int32_t* offsets, int32_t* sorted_token_ids,
                                          int32_t* expert_ids, int32_t* num_tokens_post_pad, int32_t* inv_perm,
                                          void* workspace, size_t workspace_bytes, void* stream) {
  if (T < 0 || k < 1 || E_global < 1 || E_local < 1 || block_size < 1) return MOE_ERR_INVALID_ARG;
  if (E_local > E_global) return MOE_ERR_INVALID_ARG;
  if (expert_map == nullptr && E_local != E_global) return MOE_ERR_INVALID_ARG;
  if (E_local > 1024) return MOE_ERR_UNSUPPORTED;
  const int64_t P = T * k;
  if (T > (int64_t{1} << 40) || P >= (int64_t{1} << 30)) return MOE_ERR_INVALID_ARG;
  const int64_t C = moe_align_capacity(T, k, E_local, block_size);
  if (C < 0 || C >= (int64_t{1} << 31)) return MOE_ERR_INVALID_ARG;
  if (counts == nullptr || offsets == nullptr || sorted_token_ids == nullptr || expert_ids == nullptr ||
      num_tokens_post_pad == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (P > 0 && (topk_ids == nullptr || inv_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < moe_align_workspace_bytes(T, k, E_local)) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return MOE_ERR_INVALID_ARG;

  AlignArgs a{};
  a.topk_ids = topk_ids;
  a.expert_map = expert_map;
  a.P = P;
  a.E_global = E_global;
  a.E_local = E_local;
  a.bs = block_size;
  a.C = C;
  a.NB = static_cast<int>((C + block_size - 1) / block_size);
  a.tile_slots = tile_slots_for(P);
  a.num_tiles = num_tiles_for(P, a.tile_slots);
  a.counts = counts;
  a.offsets = offsets;
  a.sorted_ids = sorted_token_ids;
  a.expert_ids = expert_ids;
  a.n_pad = num_tokens_post_pad;
  a.inv_perm = inv_perm;
  a.status = static_cast<int32_t*>(workspace);
  a.ticket = reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) + 4);
  a.tile_counts = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kWsHeaderBytes);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // mid-size batches: the tile kernels of the fused dispatch (per-tile ranks, a per-expert tile
  // scan, placement), measured faster there than the single cluster; small batches: one cluster;
  // above: count + place tile kernels over every SM
  if (P > kAlignTilesMinSlots && P <= kClusterMaxSlots)
    return moe_internal::align_tiles(topk_ids, T, k, E_global, expert_map, E_local, block_size, counts, offsets,
                                     sorted_token_ids, expert_ids, num_tokens_post_pad, inv_perm, workspace, st);
  if (P <= kClusterMaxSlots && E_local <= kClusterMaxExperts) return launch_align_cluster(a, st);
  // large batches or many local experts: count + place tile kernels over every SM
  const size_t smem = align_smem_ints(E_local, a.tile_slots) * sizeof(int);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(align_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(align_place_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (moe_host::prefer_max_shared(reinterpret_cast<const void*>(align_count_kernel)) != cudaSuccess ||
      moe_host::prefer_max_shared(reinterpret_cast<const void*>(align_place_kernel)) != cudaSuccess)
    return MOE_ERR_CUDA;
  align_count_kernel<<<a.num_tiles, kAlignThreads, smem, st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  if (a.num_tiles > 1) {
    align_place_kernel<<<a.num_tiles, kAlignThreads, smem, st>>>(a);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// ---------------------------------------------------------------------------------------------
// moe_align_permute_noalloc: the same two align kernels, with their scratch (completion ticket
// and per-tile expert counters) in a file-scope device array instead of a caller workspace.
// For callers that cannot allocate device memory at all (see the header).
// ---------------------------------------------------------------------------------------------
#include <cuda.h>  // CUcontext and CUresult for the two driver calls below (reached through the runtime)

#include <mutex>

namespace {
constexpr size_t kNoAllocScratchBytes = size_t{1} << 20;  // 1 MiB per device, held until process exit
constexpr int kNoAllocMaxDevices = 64;
}  // namespace

// Host code may not use this name as an address: it is a host-side stand-in.  The device address
// comes from cudaGetSymbolAddress, looked up once per CUDA context below.
static __device__ __align__(256) unsigned char g_align_noalloc_scratch[kNoAllocScratchBytes];

namespace {
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

std::mutex g_noalloc_mutex;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
struct NoAllocSlot {
  unsigned long long ctx_id;  // the context the address belongs to (ids are unique within a process)
  void* addr;
};
NoAllocSlot g_noalloc_slot[kNoAllocMaxDevices] = {};

// Unique id of the context current on this thread (the device's primary context once the runtime
// has made it current).  Caller holds g_noalloc_mutex.
moe_status_t current_context_id(unsigned long long* id) {
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 12000, cudaEnableDefault, &q1) != cudaSuccess ||
        cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &q2) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || f1 == nullptr || f2 == nullptr)
      return MOE_ERR_CUDA;
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return MOE_ERR_CUDA;
  return g_ctx_get_id(ctx, id) == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Device address of the scratch array in the current device's context.  Looked up with
// cudaGetSymbolAddress on the first call in each context and cached under the context's id, so
// that a reset device (a new primary context, where the module and the array may sit elsewhere)
// gets a fresh lookup instead of a stale address.
moe_status_t noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_UNSUPPORTED;
  if (cudaSetDevice(dev) != cudaSuccess) return MOE_ERR_CUDA;  // the device's primary context, current here
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  unsigned long long id = 0;
  const moe_status_t s = current_context_id(&id);
  if (s != MOE_OK) return s;
  NoAllocSlot& slot = g_noalloc_slot[dev];
  if (slot.addr == nullptr || slot.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_align_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    slot.ctx_id = id;
    slot.addr = p;
  }
  *out = slot.addr;
  return MOE_OK;
}
}  // namespace

extern "C" moe_status_t moe_align_permute_noalloc(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E_global,
                                                  const int32_t* expert_map, int32_t E_local, int32_t block_size,
                                                  int32_t* counts, int32_t* offsets, int32_t* sorted_token_ids,
                                                  int32_t* expert_ids, int32_t* num_tokens_post_pad,
                                                  int32_t* inv_perm, int32_t* device_status, void* stream) {
  if (T < 0 || k < 1 || E_global < 1 || E_local < 1 || block_size < 1) return MOE_ERR_INVALID_ARG;
  if (E_local > E_global) return MOE_ERR_INVALID_ARG;
  if (expert_map == nullptr && E_local != E_global) return MOE_ERR_INVALID_ARG;
  if (E_local > 1024) return MOE_ERR_UNSUPPORTED;
  const int64_t P = T * k;
  if (T > (int64_t{1} << 40) || P >= (int64_t{1} << 30)) return MOE_ERR_INVALID_ARG;
  const int64_t C = moe_align_capacity(T, k, E_local, block_size);
  if (C < 0 || C >= (int64_t{1} << 31)) return MOE_ERR_INVALID_ARG;
  if (counts == nullptr || offsets == nullptr || sorted_token_ids == nullptr || expert_ids == nullptr ||
      num_tokens_post_pad == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (P > 0 && (topk_ids == nullptr || inv_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  // the scratch these sizes need must fit the fixed array
  if (count_place_scratch_bytes(T, k, E_local) > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  const moe_status_t st_scratch = noalloc_scratch(&scratch);
  if (st_scratch != MOE_OK) return st_scratch;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the completion ticket must start at zero whatever an earlier call left behind
  if (cudaMemsetAsync(static_cast<char*>(scratch) + 4, 0, 4, st) != cudaSuccess) return MOE_ERR_CUDA;

  AlignArgs a{};
  a.topk_ids = topk_ids;
  a.expert_map = expert_map;
  a.P = P;
  a.E_global = E_global;
  a.E_local = E_local;
  a.bs = block_size;
  a.C = C;
  a.NB = static_cast<int>((C + block_size - 1) / block_size);
  a.tile_slots = tile_slots_for(P);
  a.num_tiles = num_tiles_for(P, a.tile_slots);
  a.counts = counts;
  a.offsets = offsets;
  a.sorted_ids = sorted_token_ids;
  a.expert_ids = expert_ids;
  a.n_pad = num_tokens_post_pad;
  a.inv_perm = inv_perm;
  a.status = device_status;
  a.ticket = reinterpret_cast<unsigned int*>(static_cast<char*>(scratch) + 4);
  a.tile_counts = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) + kWsHeaderBytes);

  const size_t smem = align_smem_ints(E_local, a.tile_slots) * sizeof(int);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(align_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(align_place_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (moe_host::prefer_max_shared(reinterpret_cast<const void*>(align_count_kernel)) != cudaSuccess ||
      moe_host::prefer_max_shared(reinterpret_cast<const void*>(align_place_kernel)) != cudaSuccess)
    return MOE_ERR_CUDA;
  align_count_kernel<<<a.num_tiles, kAlignThreads, smem, st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  if (a.num_tiles > 1) {
    align_place_kernel<<<a.num_tiles, kAlignThreads, smem, st>>>(a);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
