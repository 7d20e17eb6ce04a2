// route_fused.cu -- fused dispatch: gating, expert counting, the stable block-padded layout and the
// activation gather, with the kernel boundaries placed for latency.
//
// Operations: the FusedMoE pipeline of "Upstream Reference: Deep-Spark xllm + vllm", "File
// Index" (gate -> topk -> expand -> ...): topk_softmax (moe_topk_softmax_kernels.cuh), the
// block alignment for scatter (moe_align_sum_kernels.cu) and the permute-gather ("expand"),
// with the expert_map remap and the all-remote rank of the 2026-07-16 MTP1 M=2 compact
// scheduler closure note.  The outputs are exactly those of moe_topk_softmax +
// moe_align_permute + moe_gather; only the kernel boundaries move.
//
// Batches above the small-batch limits take three kernels, chained by programmatic dependent
// launch:
// gate_count_kernel (one CTA per tile of 16 or 32 tokens; 16 when the tiles of a batch fit on
// the SMs at once, so that each warp gates one row):
//   A. each warp gates rows of the tile (gate_row: one warp per row) and writes topk_weights and
//      topk_ids; the local expert of every slot of the tile goes to shared memory;
//   B. stable ranks inside the tile: each warp owns a contiguous run of the tile's slots, counts
//      it into its own shared-memory row, the rows are scanned across warps, and each slot's rank
//      = earlier warps' count + earlier peers in its warp; the rank is parked in inv_perm and the
//      tile's per-expert counts go to the workspace, expert-major ([E_local][tiles]).
//   gate_count_lanes_kernel replaces it for many short rows (moe_gate::lane_gating_fits): one
//   CTA per tile of 32 tokens, up to eight lanes per row (gate_lane.cuh), the same ranks and counts.
// tile_scan_kernel (one CTA per local expert): the expert's row of tile counts becomes the
//   exclusive prefix over the tiles (the tile bases) and its total goes to the workspace.
//   Nothing waits on another CTA: the kernel boundary is the only grid-wide step.
// place_gather_kernel (one warp per CTA, up to 8 tokens, TMA staging as in gather_tma_kernel):
//   bulk-loads its hidden rows first (hidden is an input of the call, complete before the first
//   kernel ran); scans the padded expert totals into the offsets itself (E_local values, in
//   shared memory); each slot's row = offsets[e] + tile base[e] + rank; writes sorted_token_ids
//   and inv_perm for its slots and bulk-stores the rows; the expert-owned outputs (counts,
//   offsets, expert_ids, pad rows) and the tail past N_pad are spread over the CTAs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "gate_lane.cuh"
#include "gate_row.cuh"
#include "route_internal.h"

namespace {

constexpr int kGcWarps = 16;
constexpr int kGcThreads = kGcWarps * 32;
constexpr int kWsHeaderBytes = 256;  // status word, test hooks (words 2 and 3), padding
constexpr int kRowsPerTile = 32;       // tile height of the lane kernel and of the align entry point
constexpr int kRowsPerTileSmall = 16;  // tile height of gate_count_kernel when all tiles fit at once
constexpr int kGcCtasPerSm = 4;        // gate_count_kernel CTAs resident per SM (2048 threads)
constexpr int kTsThreadsSmall = 128;  // tile_scan_kernel: threads per expert up to kTsWideTiles tiles
constexpr int kTsThreadsWide = 512;   // and above
constexpr int kTsWideTiles = 1024;
constexpr int kPgMaxTokens = 8;
constexpr uint32_t kPgCtaBytes = 32u * 1024u;
constexpr int kPgCtasPerSm = 4;  // place_gather_kernel CTAs resident per SM

struct DispatchArgs {
  const void* logits;
  int64_t T;
  int E;
  int k;
  int renormalize;  // scoring mode bits: moe_gate::kGateRenorm, moe_gate::kGateSigmoid
  int given_ids;  // topk_ids is an input: no gating, topk_weights untouched
  const int32_t* expert_map;
  int E_local;
  int bs;
  int bs_shift;  // log2(bs) when bs is a power of two, else -1
  int64_t P;  // T * k
  int64_t C;  // capacity rows
  int NB;     // blocks
  int rows_per_tile;
  int rt_shift;  // log2(rows_per_tile)
  int num_tiles;
  float* topk_weights;
  int32_t* topk_ids;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_ids;
  int32_t* expert_ids;
  int32_t* n_pad;
  int32_t* inv_perm;
  int32_t* status;
  int32_t* tile_counts;  // [E_local][num_tiles]: tile counts, then tile bases
  int32_t* totals;       // [E_local]
};

// Local expert of global expert g (or -1: remote); out-of-range values are flagged.
__device__ __forceinline__ int to_local(const DispatchArgs& a, int g) {
  if (static_cast<unsigned>(g) >= static_cast<unsigned>(a.E)) {
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

// Lanes of this warp holding the same value v >= 0 (0 for v < 0), through a per-warp array of
// masks in shared memory that is zero on entry and left zero.
__device__ __forceinline__ unsigned peers_of(unsigned* masks, int v, int lane) {
  if (v >= 0) atomicOr(&masks[v], 1u << lane);
  __syncwarp();
  const unsigned p = v >= 0 ? masks[v] : 0u;
  __syncwarp();
  if (v >= 0) masks[v] = 0u;
  __syncwarp();
  return p;
}

// Block-padded size of an expert with c slots: ceil(c / bs) * bs.
__device__ __forceinline__ int padded_rows(int c, int bs, int bs_shift) {
  if (c == 0) return 0;
  return bs_shift >= 0 ? (((c + bs - 1) >> bs_shift) << bs_shift) : ((c + bs - 1) / bs) * bs;
}

// Shared memory of gate_count_kernel (ints): s_le[rows_per_tile * k] | whist[kGcWarps][E_local] |
// masks[kGcWarps][E_local]
__host__ __device__ inline size_t gc_smem_ints(int rows_per_tile, int k, int E_local) {
  return static_cast<size_t>(rows_per_tile) * k + 2 * static_cast<size_t>(kGcWarps) * E_local;
}

// Stable ranks inside a tile, by the CTA's `nwarps` warps (all threads call this, after s_le is
// complete): warp w owns a contiguous run of the tile's 32-slot chunks and counts it into its row of
// `whist` ([nwarps][E_local], zero on entry); the rows are scanned across warps per expert (the
// tile's counts go to the workspace, expert-major); each slot's rank = earlier warps' count of its
// expert + the warp's running count + earlier peers in its chunk.  The rank is parked in inv_perm
// as (rank << 10) | local expert for place_gather_kernel; remote slots get -1.  `masks`
// ([nwarps][E_local]) is zero on entry and left zero.
__device__ __forceinline__ void rank_tile_slots(const DispatchArgs& a, const int* s_le, int nslots, int64_t row0,
                                                int tile, int* whist, unsigned* masks, int nwarps) {
  const int El = a.E_local, k = a.k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = nwarps * 32;
  const int nch = (nslots + 31) / 32;
  const int cpw = (nch + nwarps - 1) / nwarps;
  const int c0 = warp * cpw;
  const int c1 = (c0 + cpw < nch) ? c0 + cpw : nch;
  int* my_hist = whist + warp * El;
  unsigned* my_masks = masks + warp * El;
  for (int c = c0; c < c1; ++c) {
    const int i = c * 32 + lane;
    const int le = i < nslots ? s_le[i] : -1;
    if (le >= 0) atomicAdd(&my_hist[le], 1);
  }
  __syncthreads();
  for (int e = tid; e < El; e += nthreads) {
    int run = 0;
    for (int w = 0; w < nwarps; ++w) {
      const int c = whist[w * El + e];
      whist[w * El + e] = run;
      run += c;
    }
    a.tile_counts[static_cast<int64_t>(e) * a.num_tiles + tile] = run;
  }
  __syncthreads();
  for (int c = c0; c < c1; ++c) {
    const int i = c * 32 + lane;
    const int le = i < nslots ? s_le[i] : -1;
    const unsigned peers = peers_of(my_masks, le, lane);
    if (le >= 0) {
      a.inv_perm[row0 * k + i] = ((my_hist[le] + __popc(peers & moe::lanemask_lt())) << 10) | le;
    } else if (i < nslots) {
      a.inv_perm[row0 * k + i] = -1;
    }
    __syncwarp();
    if (le >= 0 && lane == __ffs(peers) - 1) my_hist[le] += __popc(peers);
    __syncwarp();
  }
}

template <typename TIn, int VEC, int CPL>
__global__ void __launch_bounds__(kGcThreads) gate_count_kernel(DispatchArgs a) {
  extern __shared__ int smem[];
  const int k = a.k, El = a.E_local, RT = a.rows_per_tile;
  int* s_le = smem;
  int* whist = s_le + RT * k;
  unsigned* masks = reinterpret_cast<unsigned*>(whist + kGcWarps * El);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x;
  const int64_t row0 = static_cast<int64_t>(tile) * RT;
  const int rows = static_cast<int>((a.T - row0) < RT ? (a.T - row0) : RT);
  for (int i = tid; i < kGcWarps * El; i += kGcThreads) {
    whist[i] = 0;
    masks[i] = 0u;
  }
  __syncthreads();
  moe::pdl_wait();  // the logits may come from the previous kernel
  moe::pdl_launch_dependents();

  // A. gating, one warp per row (or the routes the caller gave)
  const TIn* logits = static_cast<const TIn*>(a.logits);
  if (a.given_ids) {
    for (int i = tid; i < rows * k; i += kGcThreads) s_le[i] = to_local(a, a.topk_ids[row0 * k + i]);
  }
  for (int r = a.given_ids ? rows : warp; r < rows; r += kGcWarps) {
    const int64_t row = row0 + r;
    int my_e;
    float my_w;
    moe_gate::gate_row<TIn, VEC, CPL>(logits + row * static_cast<int64_t>(a.E), a.E, k, a.renormalize, lane, my_e,
                                      my_w);
    if (lane < k) {
      a.topk_weights[row * k + lane] = my_w;
      a.topk_ids[row * k + lane] = my_e;
      s_le[r * k + lane] = to_local(a, my_e);
    }
  }
  __syncthreads();

  // B. stable ranks inside the tile
  rank_tile_slots(a, s_le, rows * k, row0, tile, whist, masks, kGcWarps);
}

// One CTA of G warps per tile of kRowsPerTile tokens, G lanes per row: the tile's logits are staged
// in shared memory and each group of G lanes gates one row (moe_gate::lane_gate_row); then the G
// warps rank the tile's slots and write its per-expert counts (rank_tile_slots, as gate_count_kernel).
// Shared memory: staged rows [kRowsPerTile * stride chunks] | whist [G][E_local] | peer masks
// [G][E_local] | s_le [kRowsPerTile * K].
template <typename TIn, int K, int G>
__global__ void __launch_bounds__(32 * G) gate_count_lanes_kernel(DispatchArgs a, int cpr) {
  constexpr int NT = 32 * G;
  extern __shared__ __align__(16) uint4 s_rows[];
  const int El = a.E_local;
  const int stride = moe_gate::lane_tile_stride(cpr);
  int* whist = reinterpret_cast<int*>(s_rows + kRowsPerTile * stride);
  unsigned* masks = reinterpret_cast<unsigned*>(whist + G * El);
  int* s_le = reinterpret_cast<int*>(masks + G * El);
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int64_t row0 = static_cast<int64_t>(tile) * kRowsPerTile;
  const int rows = static_cast<int>((a.T - row0) < kRowsPerTile ? (a.T - row0) : kRowsPerTile);  // >= 1
  for (int e = tid; e < G * El; e += NT) {
    whist[e] = 0;
    masks[e] = 0u;
  }
  moe::pdl_wait();  // the logits may come from the previous kernel
  moe::pdl_launch_dependents();
  moe_gate::lane_tile_load(static_cast<const uint4*>(a.logits) + row0 * cpr, rows, cpr, stride, s_rows, tid, NT);
  __syncthreads();
  {
    const int r = tid / G, g = tid % G;
    const int rr = r < rows ? r : rows - 1;  // every lane takes part in the group's shuffles
    float w[K];
    int ids[K];
    moe_gate::lane_gate_row<TIn, K, G>(s_rows + rr * stride, cpr, a.renormalize, g, w, ids);
    if (r < rows && g == 0) {
      const int64_t o = (row0 + r) * K;
#pragma unroll
      for (int q = 0; q < K; ++q) {
        a.topk_weights[o + q] = w[q];
        a.topk_ids[o + q] = ids[q];
        s_le[r * K + q] = to_local(a, ids[q]);
      }
    }
  }
  __syncthreads();
  rank_tile_slots(a, s_le, rows * K, row0, tile, whist, masks, G);
}

using LanesKernel = void (*)(DispatchArgs, int);

template <typename TIn, int K>
LanesKernel lanes_kernel_g(int G) {
  switch (G) {
    case 1: return &gate_count_lanes_kernel<TIn, K, 1>;
    case 2: return &gate_count_lanes_kernel<TIn, K, 2>;
    case 4: return &gate_count_lanes_kernel<TIn, K, 4>;
    case 8: return &gate_count_lanes_kernel<TIn, K, 8>;
    default: return nullptr;
  }
}

template <typename TIn>
LanesKernel lanes_kernel_for(int k, int G) {
  switch (k) {
    case 1: return lanes_kernel_g<TIn, 1>(G);
    case 2: return lanes_kernel_g<TIn, 2>(G);
    case 3: return lanes_kernel_g<TIn, 3>(G);
    case 4: return lanes_kernel_g<TIn, 4>(G);
    case 5: return lanes_kernel_g<TIn, 5>(G);
    case 6: return lanes_kernel_g<TIn, 6>(G);
    case 7: return lanes_kernel_g<TIn, 7>(G);
    case 8: return lanes_kernel_g<TIn, 8>(G);
    default: return nullptr;
  }
}

// One CTA per local expert: its row of tile counts -> exclusive prefix over the tiles, in place;
// the total to `totals`.  Thread i owns a contiguous run of tiles; runs of up to kTsCache tiles
// are read once into registers (NT threads: up to 8 * NT tiles), longer ones are read again for the
// second pass.  The launcher takes 128 threads up to kTsWideTiles tiles: resident early (programmatic
// dependent launch), wider CTAs take SM room from the gating kernel.
constexpr int kTsCache = 8;
template <int NT>
__global__ void __launch_bounds__(NT) tile_scan_kernel(DispatchArgs a) {
  __shared__ int warp_sums[NT / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e = blockIdx.x;
  // let place_gather_kernel start now (it loads its hidden rows, then waits for this kernel,
  // which completes after gate_count_kernel)
  moe::pdl_launch_dependents();
  moe::pdl_wait();  // tile counts come from gate_count_kernel
  const int N = a.num_tiles;
  int32_t* col = a.tile_counts + static_cast<int64_t>(e) * N;
  const int per = (N + NT - 1) / NT;
  const int t0 = tid * per < N ? tid * per : N;
  const int t1 = t0 + per < N ? t0 + per : N;
  const bool cached = per <= kTsCache;
  int x[kTsCache];
  int sum = 0;
  if (cached) {
#pragma unroll
    for (int u = 0; u < kTsCache; ++u) x[u] = t0 + u < t1 ? col[t0 + u] : 0;
#pragma unroll
    for (int u = 0; u < kTsCache; ++u) sum += x[u];
  } else {
    for (int t = t0; t < t1; t += 8) {
      int y[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) y[u] = t + u < t1 ? col[t + u] : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) sum += y[u];
    }
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  int run = incl - sum, total = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const int ws = warp_sums[w];
    run += w < warp ? ws : 0;
    total += ws;
  }
  if (cached) {
#pragma unroll
    for (int u = 0; u < kTsCache; ++u) {
      if (t0 + u < t1) col[t0 + u] = run;
      run += x[u];
    }
  } else {
    for (int t = t0; t < t1; t += 8) {
      int y[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) y[u] = t + u < t1 ? col[t + u] : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (t + u < t1) col[t + u] = run;
        run += y[u];
      }
    }
  }
  if (tid == 0) a.totals[e] = total;
}

// One warp per CTA: slots of tokens [t0, t0 + n) get their rows, the hidden rows are staged with
// a bulk load and bulk-stored to every local row; then a share of the expert-owned outputs, the
// pad rows and the tail.  Shared memory: staged rows [tpc * row_bytes] | offsets [E_local + 1].
template <bool kGather>  // false: placement only (moe_align_permute), no hidden rows
__global__ void __launch_bounds__(32)
place_gather_kernel(DispatchArgs a, const uint8_t* __restrict__ hidden, uint32_t row_bytes, int tpc,
                    uint8_t* __restrict__ permuted) {
  extern __shared__ __align__(128) uint8_t rows[];
  __shared__ __align__(8) uint64_t bar;
  int* s_off = reinterpret_cast<int*>(rows + static_cast<size_t>(tpc) * row_bytes);
  const int lane = threadIdx.x;
  const int k = a.k, El = a.E_local, bs = a.bs, bs_shift = a.bs_shift;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * tpc;
  const int64_t left = a.T - t0;
  const int n = left <= 0 ? 0 : static_cast<int>(left < tpc ? left : tpc);
  // test hooks (zero in normal use): a withheld load makes the wait below run out after the limit
  const moe::WaitHooks hooks = kGather ? moe::read_hooks(a.status) : moe::WaitHooks{0u, moe::kWaitLimitNs};
  const bool withhold = (hooks.withhold & moe::kHookWithholdRowLoads) != 0u;
  if (kGather && lane == 0) {
    moe::mbar_init(&bar, 1);
    moe::fence_barrier_init();
  }
  __syncwarp();
  if (kGather && lane == 0 && n > 0 && !withhold) {  // hidden is an input of the call: complete before the first kernel ran
    moe::mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(n) * row_bytes);
    for (int i = 0; i < n; ++i) {
      moe::bulk_load(rows + static_cast<size_t>(i) * row_bytes, hidden + (t0 + i) * static_cast<int64_t>(row_bytes),
                     row_bytes, &bar, row_bytes <= moe::kEvictFirstMaxRowBytes);
    }
  }
  moe::pdl_launch_dependents();
  moe::pdl_wait();  // ranks (gate_count_kernel), tile bases and totals (tile_scan_kernel)

  // the slots' parked values (rank in the tile << 10 | local expert, or -1) and their tiles' bases
  // are loaded first, so that these loads are in flight during the offsets scan
  const int nslots = n * k;  // <= kPgMaxTokens * 32
  int pv[kPgMaxTokens];
  int base[kPgMaxTokens];
#pragma unroll
  for (int m = 0; m < kPgMaxTokens; ++m) {
    const int e = lane + 32 * m;
    pv[m] = e < nslots ? a.inv_perm[t0 * k + e] : -1;
  }
#pragma unroll
  for (int m = 0; m < kPgMaxTokens; ++m) {
    const int e = lane + 32 * m;
    base[m] = 0;
    if (pv[m] >= 0 && (pv[m] & 1023) < El) {
      const int64_t tile = (t0 + e / k) >> a.rt_shift;
      base[m] = a.tile_counts[static_cast<int64_t>(pv[m] & 1023) * a.num_tiles + tile];
    }
  }

  // expert offsets: exclusive scan of the block-padded totals; lane l owns a contiguous run
  {
    const int per = (El + 31) >> 5;
    const int e0 = lane * per < El ? lane * per : El;
    const int e1 = e0 + per < El ? e0 + per : El;
    int sum = 0;
    for (int e = e0; e < e1; ++e) {
      const int p = padded_rows(a.totals[e], bs, bs_shift);
      s_off[e] = p;
      sum += p;
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - sum;
    for (int e = e0; e < e1; ++e) {
      const int p = s_off[e];
      s_off[e] = run;
      run += p;
    }
    if (lane == 31) s_off[El] = incl;
    __syncwarp();
  }

  int32_t dst[kPgMaxTokens];
#pragma unroll
  for (int m = 0; m < kPgMaxTokens; ++m) {
    const int e = lane + 32 * m;
    int r = -1;
    const int v = pv[m];
    // a parked value names a local expert; anything else (buffers shared with a concurrent call)
    // is flagged and skipped, never used as an index
    if (v >= 0 && (v & 1023) >= El) {
      moe::record_status(a.status, MOE_ERR_BAD_ROW);
    } else if (v >= 0) {
      const int64_t s = t0 * k + e;
      r = s_off[v & 1023] + base[m] + (v >> 10);
      if (r < 0 || static_cast<int64_t>(r) >= a.C) {  // cannot happen for consistent inputs
        moe::record_status(a.status, MOE_ERR_BAD_ROW);
        r = -1;
      } else {
        a.sorted_ids[r] = static_cast<int32_t>(s);
        a.inv_perm[s] = r;
      }
    }
    dst[m] = r;
  }
  if (kGather && n > 0) {
    if (!moe::mbar_wait(&bar, 0, hooks.limit_ns)) {
      moe::record_status(a.status, MOE_ERR_TIMEOUT);
      if (!withhold) moe::mbar_wait(&bar, 0, hooks.limit_ns);  // one more bounded wait for the loads in flight
      return;
    }
#pragma unroll
    for (int m = 0; m < kPgMaxTokens; ++m) {
      const int e = lane + 32 * m;
      if (e < nslots && dst[m] >= 0) {
        moe::bulk_store(permuted + static_cast<int64_t>(dst[m]) * row_bytes,
                        rows + static_cast<size_t>(e / k) * row_bytes, row_bytes,
                        row_bytes <= moe::kEvictFirstMaxRowBytes);
      }
    }
    moe::bulk_commit();
  }

  // a share of the expert-owned outputs, the pad rows and the tail past N_pad
  const int G = gridDim.x, b = blockIdx.x;
  const int total = s_off[El];
  for (int e = b * 32 + lane; e < El; e += G * 32) {
    a.counts[e] = a.totals[e];
    a.offsets[e] = s_off[e];
  }
  if (b == 0 && lane == 0) {
    a.offsets[El] = total;
    a.n_pad[0] = total;
  }
  for (int64_t blk = static_cast<int64_t>(b) * 32 + lane; blk < a.NB; blk += static_cast<int64_t>(G) * 32) {
    const int64_t row = blk * bs;
    int e = -1;
    if (row < total) {
      int lo = 0, hi = El - 1;  // largest e with s_off[e] <= row (empty experts share offsets)
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= row) lo = mid; else hi = mid - 1;
      }
      e = lo;
    }
    a.expert_ids[blk] = e;
  }
  const int32_t pad_value = static_cast<int32_t>(a.P);
  for (int e = b; e < El; e += G) {
    const int p1 = s_off[e + 1];
    for (int p = s_off[e] + a.totals[e] + lane; p < p1; p += 32) a.sorted_ids[p] = pad_value;
  }
  const int64_t tail = a.C - total;
  for (int64_t i = static_cast<int64_t>(b) * 32 + lane; i < tail; i += static_cast<int64_t>(G) * 32)
    a.sorted_ids[total + i] = pad_value;
  if (kGather && n > 0) moe::bulk_wait_read_all();  // the staged rows must outlive the stores that read them
}

// ------------------------------------------------------------------------------------------
// Small batches (decode): one CTA per slot, each routing the whole batch by itself.
// A decode batch is a handful of tokens: its routing is a short chain of dependent steps, and one
// SM writing every hidden row to its slots would be bound by that SM's store bandwidth.  So the
// grid has one CTA per slot s = t*k + j; every CTA gates all T rows, ranks the slots and scans the
// local experts (no CTA waits for another); the routing outputs are shared out over the CTAs, so
// that no CTA's stores lengthen the chain; CTA s copies the hidden row of token t to the row of
// slot s when the slot is local.  The row is loaded into
// registers at kernel entry, so its memory latency overlaps the gating loads.  The phases are
// laid out for latency (few barriers, no serial searches):
//   A. hidden row -> registers; expert map -> shared memory; warp w gates rows w, w + 8, ...
//      (or reads the caller's routes);
//   B. per warp of 32 slots: local expert, rank among the warp's earlier slots of the same expert
//      and the warp's count of it (one match.any); the first slot of each expert in the
//      warp records the count in the warp's row of a histogram;
//   C. per expert (one per thread): count = sum of the warp rows, blocks = ceil(count/bs),
//      exclusive scan of the blocks over the experts; each CTA writes counts, offsets, expert_ids
//      and the pad rows of a contiguous share of the experts;
//   D. row of slot s = offset of its expert + its expert's slots in earlier warps + its rank;
//      CTA s writes sorted_token_ids[row] and inv_perm[s] and copies its row; the tail past
//      N_pad is shared out over the CTAs.
constexpr int kSmallThreads = 256;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kSmallMaxTokens = 32;
constexpr int kSmallMaxSlots = kSmallThreads;  // one slot per thread
constexpr int kSmallMaxExperts = 256;  // one expert per thread in every per-expert loop
constexpr int kSmallExpertsPerThread = kSmallMaxExperts / kSmallThreads;
constexpr int kSmallPrefetch = 4;  // 16-byte vectors per thread of the row held in registers while routing

template <typename TIn, int VEC, int CPL, bool kGivenIds>
__global__ void __launch_bounds__(kSmallThreads)
route_small_kernel(DispatchArgs a, const uint4* __restrict__ hidden, int nvec, uint4* __restrict__ permuted) {
  __shared__ int s_map[kSmallMaxExperts];
  __shared__ int whist[kSmallWarps * kSmallMaxExperts];  // [warp][E_local]: the warp's slots per expert
  __shared__ int s_off[kSmallMaxExperts];                // first row of each local expert
  __shared__ int s_ge[kSmallMaxSlots];
  __shared__ int s_le[kSmallMaxSlots];
  __shared__ int s_rk[kSmallMaxSlots];
  __shared__ int warp_sums[kSmallWarps];
  // every parameter, read into registers at entry (moe::pin), before the kernel waits for anything
  const int T = moe::pin(static_cast<int>(a.T)), k = moe::pin(a.k), E = moe::pin(a.E), El = moe::pin(a.E_local);
  const int bs = moe::pin(a.bs), bs_shift = moe::pin(a.bs_shift), NB = moe::pin(a.NB);
  const int renormalize = moe::pin(a.renormalize);
  const int64_t C = moe::pin(a.C);
  const TIn* logits = moe::pin(static_cast<const TIn*>(a.logits));
  const int32_t* expert_map = moe::pin(a.expert_map);
  int32_t* topk_ids = moe::pin(a.topk_ids);
  float* topk_weights = moe::pin(a.topk_weights);
  int32_t* counts = moe::pin(a.counts);
  int32_t* offsets = moe::pin(a.offsets);
  int32_t* sorted_ids = moe::pin(a.sorted_ids);
  int32_t* expert_ids = moe::pin(a.expert_ids);
  int32_t* n_pad = moe::pin(a.n_pad);
  int32_t* inv_perm = moe::pin(a.inv_perm);
  int32_t* status = moe::pin(a.status);
  hidden = moe::pin(hidden);
  permuted = moe::pin(permuted);
  nvec = moe::pin(nvec);
  const int P = T * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = (P + 31) >> 5;  // warps holding slots
  // grid (k, T): this CTA copies the row of slot tok * k + j (no CTA has a slot when P == 0)
  const int tok = blockIdx.y, slot = tok * k + static_cast<int>(blockIdx.x);
  const bool lead = blockIdx.x == 0 && blockIdx.y == 0;
  // the expert-owned outputs and the tail are shared out over the grid's CTAs (cta = slot)
  const int ncta = static_cast<int>(gridDim.x * gridDim.y), cta = slot;
  for (int i = tid; i < nw * El; i += kSmallThreads) whist[i] = 0;

  moe::pdl_wait();  // logits, routes and hidden may come from the previous kernel
  moe::pdl_launch_dependents();
  // A. this CTA's hidden row, the expert map and the gating loads, in flight together
  const uint4* src = hidden + static_cast<int64_t>(slot < P ? tok : 0) * nvec;
  uint4 pre[kSmallPrefetch];
#pragma unroll
  for (int i = 0; i < kSmallPrefetch; ++i) {
    const int v = tid + i * kSmallThreads;
    if (slot < P && v < nvec) pre[i] = __ldg(src + v);
  }
  int mv[kSmallExpertsPerThread];
#pragma unroll
  for (int i = 0; i < kSmallExpertsPerThread; ++i) {
    const int g = tid + i * kSmallThreads;
    mv[i] = g < E ? (expert_map != nullptr ? __ldg(expert_map + g) : g) : 0;
  }
  if constexpr (kGivenIds) {
    if (tid < P) s_ge[tid] = topk_ids[tid];
  } else {
    for (int row = warp; row < T; row += kSmallWarps) {
      int e;
      float w;
      moe_gate::gate_row<TIn, VEC, CPL>(logits + static_cast<int64_t>(row) * E, E, k, renormalize, lane, e, w);
      if (lane < k) {
        s_ge[row * k + lane] = e;
        if (lead) {
          topk_weights[row * k + lane] = w;
          topk_ids[row * k + lane] = e;
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kSmallExpertsPerThread; ++i) {
    const int g = tid + i * kSmallThreads;
    if (g < E) s_map[g] = mv[i];
  }
  __syncthreads();

  // B. local expert, rank inside the warp and the warp's count per expert (thread s owns slot s)
  int le = -1, rank = 0;
  if (warp < nw) {
    if (tid < P) {
      const int g = s_ge[tid];
      if (static_cast<unsigned>(g) >= static_cast<unsigned>(E)) {
        if (lead) moe::record_status(status, MOE_ERR_BAD_EXPERT_ID);
      } else {
        le = s_map[g];
        if (le < -1 || le >= El) {
          if (lead) moe::record_status(status, MOE_ERR_BAD_EXPERT_ID);
          le = -1;
        }
      }
    }
    const unsigned same = __match_any_sync(0xffffffffu, le);  // lanes of this warp with the same local expert
    rank = __popc(same & moe::lanemask_lt());
    if (le >= 0 && rank == 0) whist[warp * El + le] = __popc(same);
    if (tid < P) {
      s_le[tid] = le;
      s_rk[tid] = rank;
    }
  }
  __syncthreads();

  // C. per expert: count, blocks, exclusive scan of the blocks; each CTA writes the expert-owned
  //    outputs of its share of the experts
  const int ept = (El + kSmallThreads - 1) / kSmallThreads;  // experts per thread, consecutive
  const int e0 = tid * ept;
  const int epc = (El + ncta - 1) / ncta;  // experts per CTA, consecutive
  const int my_e0 = cta * epc, my_e1 = my_e0 + epc;
  int cnt_e[kSmallExpertsPerThread], nb_e[kSmallExpertsPerThread];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kSmallExpertsPerThread; ++i) {
    const int e = e0 + i;
    int c = 0;
    if (i < ept && e < El) {
      for (int w = 0; w < nw; ++w) c += whist[w * El + e];
    }
    cnt_e[i] = c;
    nb_e[i] = c == 0 ? 0 : bs_shift >= 0 ? (c + bs - 1) >> bs_shift : (c + bs - 1) / bs;
    sum += nb_e[i];
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  int before = incl - sum;
  int total_blocks = 0;
#pragma unroll
  for (int w = 0; w < kSmallWarps; ++w) {
    const int ws = warp_sums[w];
    before += (w < warp) ? ws : 0;
    total_blocks += ws;
  }
  const int total = total_blocks * bs;  // N_pad
  const int32_t pad_value = P;
#pragma unroll
  for (int i = 0; i < kSmallExpertsPerThread; ++i) {
    const int e = e0 + i;
    if (i < ept && e < El) {
      const int off = before * bs;
      s_off[e] = off;
      if (e >= my_e0 && e < my_e1) {
        counts[e] = cnt_e[i];
        offsets[e] = off;
        for (int b = 0; b < nb_e[i]; ++b) expert_ids[before + b] = e;
        for (int p = off + cnt_e[i]; p < off + nb_e[i] * bs; ++p) sorted_ids[p] = pad_value;
      }
    }
    before += nb_e[i];
  }
  if (lead && tid == 0) {
    offsets[El] = total;
    n_pad[0] = total;
  }
  __syncthreads();

  // D. this CTA's slot: its row (sorted_token_ids, inv_perm) and the copy of its hidden row; a share
  //    of the tail past N_pad
  if (slot < P) {
    const int le_s = s_le[slot];
    int row = -1;
    if (le_s >= 0) {
      row = s_off[le_s] + s_rk[slot];
      for (int w = 0; w < (slot >> 5); ++w) row += whist[w * El + le_s];
      if (static_cast<int64_t>(row) >= C) {  // < N_pad <= C for consistent inputs
        if (tid == 0) moe::record_status(status, MOE_ERR_BAD_ROW);
        row = -1;
      }
    }
    if (tid == 0) {
      inv_perm[slot] = row;
      if (row >= 0) sorted_ids[row] = slot;
    }
    if (row >= 0) {
      uint4* dst = permuted + static_cast<int64_t>(row) * nvec;
#pragma unroll
      for (int i = 0; i < kSmallPrefetch; ++i) {
        const int v = tid + i * kSmallThreads;
        if (v < nvec) dst[v] = pre[i];
      }
      for (int v = tid + kSmallPrefetch * kSmallThreads; v < nvec; v += kSmallThreads) dst[v] = __ldg(src + v);
    }
  }
  const int64_t stride = static_cast<int64_t>(ncta) * kSmallThreads;
  for (int64_t i = static_cast<int64_t>(total) + static_cast<int64_t>(cta) * kSmallThreads + tid; i < C; i += stride)
    sorted_ids[i] = pad_value;
  for (int64_t b = static_cast<int64_t>(total_blocks) + static_cast<int64_t>(cta) * kSmallThreads + tid; b < NB; b += stride)
    expert_ids[b] = -1;
}

// Decode batches of at most one warp of slots (P <= 32): the outputs of route_small_kernel with two
// CTA barriers instead of three, and the softmax weights off the routing chain.  Grid and row copy as
// in route_small_kernel (one CTA per slot).
//   A. hidden row -> registers; expert map -> shared memory; warp w selects the top-k of rows w, w + 8,
//      ... (moe_gate::gate_row_select; the selected keys go to shared memory), or reads the caller's
//      routes;
//   B. the last warp: local expert of each slot, its rank among earlier slots of the same expert and
//      the expert's count (one match.any), blocks per expert, exclusive scan of the blocks over the
//      local experts (one warp over shared memory).  Meanwhile the other warps of CTA 0 turn the
//      selected keys into the weights (moe_gate::gate_row_weights) and write topk_weights and topk_ids;
//   C. each CTA: its slot's row (offset of its expert + rank), sorted_token_ids and inv_perm, and the
//      copy of its hidden row; the expert-owned outputs of a contiguous share of the experts and a
//      share of the tail past N_pad.
constexpr int kDecodeMaxSlots = 32;
template <typename TIn, int VEC, int CPL, bool kGivenIds>
__global__ void __launch_bounds__(kSmallThreads)
route_decode_kernel(DispatchArgs a, const uint4* __restrict__ hidden, int nvec, uint4* __restrict__ permuted) {
  using KeyT = typename moe_gate::GateKey<TIn>::type;
  __shared__ int s_map[kSmallMaxExperts];
  __shared__ int s_cnt[kSmallMaxExperts];  // slots per local expert
  __shared__ int s_blk[kSmallMaxExperts];  // blocks per local expert, then their exclusive scan
  __shared__ int s_ge[kDecodeMaxSlots];
  __shared__ int s_le[kDecodeMaxSlots];
  __shared__ int s_rk[kDecodeMaxSlots];
  __shared__ KeyT s_key[kDecodeMaxSlots];    // selected keys, slot order
  __shared__ KeyT s_best[kDecodeMaxSlots];   // per row: its largest key
  __shared__ float s_z[kDecodeMaxSlots];     // per row: the full-row denominator (softmax without renormalising)
  __shared__ int s_total_blocks;
  // every parameter, read into registers at entry (moe::pin), before the kernel waits for anything
  const int T = moe::pin(static_cast<int>(a.T)), k = moe::pin(a.k), E = moe::pin(a.E), El = moe::pin(a.E_local);
  const int bs = moe::pin(a.bs), bs_shift = moe::pin(a.bs_shift), NB = moe::pin(a.NB);
  const int renormalize = moe::pin(a.renormalize);
  const int64_t C = moe::pin(a.C);
  const TIn* logits = moe::pin(static_cast<const TIn*>(a.logits));
  const int32_t* expert_map = moe::pin(a.expert_map);
  int32_t* topk_ids = moe::pin(a.topk_ids);
  float* topk_weights = moe::pin(a.topk_weights);
  int32_t* counts = moe::pin(a.counts);
  int32_t* offsets = moe::pin(a.offsets);
  int32_t* sorted_ids = moe::pin(a.sorted_ids);
  int32_t* expert_ids = moe::pin(a.expert_ids);
  int32_t* n_pad = moe::pin(a.n_pad);
  int32_t* inv_perm = moe::pin(a.inv_perm);
  int32_t* status = moe::pin(a.status);
  hidden = moe::pin(hidden);
  permuted = moe::pin(permuted);
  nvec = moe::pin(nvec);
  const int P = T * k;  // <= kDecodeMaxSlots
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tok = blockIdx.y, slot = tok * k + static_cast<int>(blockIdx.x);
  const bool lead = blockIdx.x == 0 && blockIdx.y == 0;
  const int ncta = static_cast<int>(gridDim.x * gridDim.y), cta = slot;
  for (int e = tid; e < El; e += kSmallThreads) {
    s_cnt[e] = 0;
    s_blk[e] = 0;
  }

  moe::pdl_wait();  // logits, routes and hidden may come from the previous kernel
  moe::pdl_launch_dependents();
  // A. this CTA's hidden row, the expert map and the gating loads, in flight together
  const uint4* src = hidden + static_cast<int64_t>(slot < P ? tok : 0) * nvec;
  uint4 pre[kSmallPrefetch];
#pragma unroll
  for (int i = 0; i < kSmallPrefetch; ++i) {
    const int v = tid + i * kSmallThreads;
    if (slot < P && v < nvec) pre[i] = __ldg(src + v);
  }
  int mv[kSmallExpertsPerThread];
#pragma unroll
  for (int i = 0; i < kSmallExpertsPerThread; ++i) {
    const int g = tid + i * kSmallThreads;
    mv[i] = g < E ? (expert_map != nullptr ? __ldg(expert_map + g) : g) : 0;
  }
  if constexpr (kGivenIds) {
    if (tid < P) s_ge[tid] = topk_ids[tid];
  } else {
    for (int row = warp; row < T; row += kSmallWarps) {
      KeyT key, best0;
      float z;
      moe_gate::gate_row_select<TIn, VEC, CPL>(logits + static_cast<int64_t>(row) * E, E, k, renormalize, lane, key,
                                               best0, z);
      if (lane < k) {
        s_ge[row * k + lane] = moe_gate::key_expert<TIn>(key);
        s_key[row * k + lane] = key;
      }
      if (lane == 0) {
        s_best[row] = best0;
        s_z[row] = z;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kSmallExpertsPerThread; ++i) {
    const int g = tid + i * kSmallThreads;
    if (g < E) s_map[g] = mv[i];
  }
  __syncthreads();

  // B. ranks, counts and the block scan (last warp); the weights (the other warps of CTA 0)
  if (warp == kSmallWarps - 1) {
    int le = -1;
    if (lane < P) {
      const int g = s_ge[lane];
      if (static_cast<unsigned>(g) >= static_cast<unsigned>(E)) {
        if (lead) moe::record_status(status, MOE_ERR_BAD_EXPERT_ID);
      } else {
        le = s_map[g];
        if (le < -1 || le >= El) {
          if (lead) moe::record_status(status, MOE_ERR_BAD_EXPERT_ID);
          le = -1;
        }
      }
    }
    const unsigned same = __match_any_sync(0xffffffffu, le);  // lanes with the same local expert
    const int rank = __popc(same & moe::lanemask_lt());
    if (le >= 0 && rank == 0) {
      const int c = __popc(same);
      s_cnt[le] = c;
      s_blk[le] = bs_shift >= 0 ? (c + bs - 1) >> bs_shift : (c + bs - 1) / bs;
    }
    if (lane < P) {
      s_le[lane] = le;
      s_rk[lane] = rank;
    }
    __syncwarp();
    const int per = (El + 31) >> 5;  // lane l scans a contiguous run of the local experts
    const int e0 = lane * per < El ? lane * per : El;
    const int e1 = e0 + per < El ? e0 + per : El;
    int sum = 0;
    for (int e = e0; e < e1; ++e) sum += s_blk[e];
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - sum;
    for (int e = e0; e < e1; ++e) {
      const int b = s_blk[e];
      s_blk[e] = run;
      run += b;
    }
    if (lane == 31) s_total_blocks = incl;
  } else if (!kGivenIds && lead) {
    for (int row = warp; row < T; row += kSmallWarps - 1) {
      int e;
      float w;
      moe_gate::gate_row_weights<TIn>(lane < k ? s_key[row * k + lane] : KeyT(0), s_best[row], s_z[row], k, renormalize,
                                      lane, e, w);
      if (lane < k) {
        topk_weights[row * k + lane] = w;
        topk_ids[row * k + lane] = e;
      }
    }
  }
  __syncthreads();

  // C. this CTA's slot and its row; a share of the expert-owned outputs and of the tail
  const int total_blocks = s_total_blocks;
  const int total = total_blocks * bs;  // N_pad
  const int32_t pad_value = P;
  if (slot < P) {
    const int le_s = s_le[slot];
    int row = -1;
    if (le_s >= 0) {
      row = s_blk[le_s] * bs + s_rk[slot];
      if (static_cast<int64_t>(row) >= C) {  // < N_pad <= C for consistent inputs
        if (tid == 0) moe::record_status(status, MOE_ERR_BAD_ROW);
        row = -1;
      }
    }
    if (tid == 0) {
      inv_perm[slot] = row;
      if (row >= 0) sorted_ids[row] = slot;
    }
    if (row >= 0) {
      uint4* dst = permuted + static_cast<int64_t>(row) * nvec;
#pragma unroll
      for (int i = 0; i < kSmallPrefetch; ++i) {
        const int v = tid + i * kSmallThreads;
        if (v < nvec) dst[v] = pre[i];
      }
      for (int v = tid + kSmallPrefetch * kSmallThreads; v < nvec; v += kSmallThreads) dst[v] = __ldg(src + v);
    }
  }
  const int epc = (El + ncta - 1) / ncta;  // experts per CTA, consecutive
  const int my_e1 = (cta + 1) * epc < El ? (cta + 1) * epc : El;
  for (int e = cta * epc + tid; e < my_e1; e += kSmallThreads) {
    const int c = s_cnt[e], b0 = s_blk[e];
    const int nb = c == 0 ? 0 : bs_shift >= 0 ? (c + bs - 1) >> bs_shift : (c + bs - 1) / bs;
    counts[e] = c;
    offsets[e] = b0 * bs;
    for (int b = 0; b < nb; ++b) expert_ids[b0 + b] = e;
    for (int p = b0 * bs + c; p < (b0 + nb) * bs; ++p) sorted_ids[p] = pad_value;
  }
  if (lead && tid == 0) {
    offsets[El] = total;
    n_pad[0] = total;
  }
  const int64_t stride = static_cast<int64_t>(ncta) * kSmallThreads;
  for (int64_t i = static_cast<int64_t>(total) + static_cast<int64_t>(cta) * kSmallThreads + tid; i < C; i += stride)
    sorted_ids[i] = pad_value;
  for (int64_t b = static_cast<int64_t>(total_blocks) + static_cast<int64_t>(cta) * kSmallThreads + tid; b < NB; b += stride)
    expert_ids[b] = -1;
}

// Kernel families instantiated per gating geometry (logits type, vector width, chunks per lane).
template <typename TIn, int VEC, int CPL>
struct GateCountFamily {
  using Fn = void (*)(DispatchArgs);
  static Fn get() { return &gate_count_kernel<TIn, VEC, CPL>; }
};
template <typename TIn, int VEC, int CPL>
struct SmallFamily {
  using Fn = void (*)(DispatchArgs, const uint4*, int, uint4*);
  static Fn get() { return &route_small_kernel<TIn, VEC, CPL, false>; }
};
template <typename TIn, int VEC, int CPL>
struct DecodeFamily {
  using Fn = void (*)(DispatchArgs, const uint4*, int, uint4*);
  static Fn get() { return &route_decode_kernel<TIn, VEC, CPL, false>; }
};
using GcKernel = GateCountFamily<float, 1, 1>::Fn;
using SmallKernel = SmallFamily<float, 1, 1>::Fn;

template <template <typename, int, int> class F, typename TIn, int VEC, int CPL>
typename F<float, 1, 1>::Fn family_instance() {
  if constexpr (VEC * CPL <= 32) {
    return F<TIn, VEC, CPL>::get();
  } else {
    return nullptr;
  }
}

template <template <typename, int, int> class F, typename TIn, int VEC>
typename F<float, 1, 1>::Fn family_pick_cpl(int cpl) {
  switch (cpl) {
    case 1: return family_instance<F, TIn, VEC, 1>();
    case 2: return family_instance<F, TIn, VEC, 2>();
    case 4: return family_instance<F, TIn, VEC, 4>();
    case 8: return family_instance<F, TIn, VEC, 8>();
    case 16: return family_instance<F, TIn, VEC, 16>();
    case 32: return family_instance<F, TIn, VEC, 32>();
    default: return nullptr;
  }
}

template <template <typename, int, int> class F, typename TIn>
typename F<float, 1, 1>::Fn family_pick(int vec, int cpl) {
  if constexpr (sizeof(TIn) == 2) {
    switch (vec) {
      case 8: return family_pick_cpl<F, TIn, 8>(cpl);
      case 4: return family_pick_cpl<F, TIn, 4>(cpl);
      case 2: return family_pick_cpl<F, TIn, 2>(cpl);
      default: return family_pick_cpl<F, TIn, 1>(cpl);
    }
  } else {
    switch (vec) {
      case 4: return family_pick_cpl<F, TIn, 4>(cpl);
      case 2: return family_pick_cpl<F, TIn, 2>(cpl);
      default: return family_pick_cpl<F, TIn, 1>(cpl);
    }
  }
}

moe_status_t launch_tile_scan(const DispatchArgs& a, int E_local, cudaStream_t st) {
  if (a.num_tiles > kTsWideTiles)
    return moe_host::launch_pdl_max_shared(tile_scan_kernel<kTsThreadsWide>, dim3(static_cast<unsigned>(E_local)),
                                           dim3(kTsThreadsWide), 0, st, a);
  return moe_host::launch_pdl_max_shared(tile_scan_kernel<kTsThreadsSmall>, dim3(static_cast<unsigned>(E_local)),
                                         dim3(kTsThreadsSmall), 0, st, a);
}

struct FusedLayout {
  int num_tiles;
  size_t tile_counts_off, totals_off, bytes;
};

FusedLayout fused_layout(int64_t T, int E_local, int rows_per_tile) {
  FusedLayout l{};
  const int64_t nt = (T + rows_per_tile - 1) / rows_per_tile;
  l.num_tiles = nt < 1 ? 1 : static_cast<int>(nt);
  l.tile_counts_off = kWsHeaderBytes;
  l.totals_off = l.tile_counts_off + ((static_cast<size_t>(l.num_tiles) * E_local * 4 + 255) & ~size_t{255});
  l.bytes = l.totals_off + static_cast<size_t>(E_local) * 4;
  return l;
}

}  // namespace

extern "C" size_t moe_route_dispatch_workspace_bytes(int64_t T, int32_t k, int32_t E_local) {
  if (T < 0 || k < 1 || E_local < 1) return 0;
  return fused_layout(T, E_local, kRowsPerTileSmall).bytes;  // the larger of the two tile heights' layouts
}

extern "C" moe_status_t moe_route_dispatch(const void* logits, moe_dtype_t dtype, const void* hidden, int64_t T,
                                           int32_t E, int32_t k, int32_t H, uint32_t flags, const int32_t* expert_map,
                                           int32_t E_local, int32_t block_size, float* topk_weights,
                                           int32_t* topk_ids, int32_t* counts, int32_t* offsets,
                                           int32_t* sorted_token_ids, int32_t* expert_ids,
                                           int32_t* num_tokens_post_pad, int32_t* inv_perm, void* permuted,
                                           void* workspace, size_t workspace_bytes, void* stream) {
  if (T < 0 || E < 1 || k < 1 || k > E || H < 1 || E_local < 1 || block_size < 1) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DTYPE_F32 && dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
  if ((flags & ~(MOE_RENORMALIZE | MOE_DISPATCH_GIVEN_IDS | MOE_SCORING_SIGMOID)) != 0u) return MOE_ERR_INVALID_ARG;
  const bool given_ids = (flags & MOE_DISPATCH_GIVEN_IDS) != 0u;
  if (E_local > E || (expert_map == nullptr && E_local != E)) return MOE_ERR_INVALID_ARG;
  if (E > 1024 || k > 32 || E_local > 1024) return MOE_ERR_UNSUPPORTED;
  if ((H % 8) != 0) return MOE_ERR_INVALID_ARG;
  const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
  if (row_bytes > 4u * kPgCtaBytes) return MOE_ERR_UNSUPPORTED;
  const int64_t P = T * k;
  if (T > (int64_t{1} << 40) || P >= (int64_t{1} << 30)) return MOE_ERR_INVALID_ARG;
  const int64_t C = moe_align_capacity(T, k, E_local, block_size);
  if (C < 0 || C >= (int64_t{1} << 31)) return MOE_ERR_INVALID_ARG;
  if (counts == nullptr || offsets == nullptr || sorted_token_ids == nullptr || expert_ids == nullptr ||
      num_tokens_post_pad == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (hidden == nullptr || topk_ids == nullptr || inv_perm == nullptr || permuted == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && !given_ids && (logits == nullptr || topk_weights == nullptr)) return MOE_ERR_INVALID_ARG;
  if ((hidden && !moe_host::aligned16(hidden)) || (permuted && !moe_host::aligned16(permuted)))
    return MOE_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < moe_route_dispatch_workspace_bytes(T, k, E_local))
    return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return MOE_ERR_INVALID_ARG;

  DispatchArgs a{};
  a.logits = logits;
  a.T = T;
  a.E = E;
  a.k = k;
  a.renormalize = ((flags & MOE_RENORMALIZE) ? moe_gate::kGateRenorm : 0) |
                  ((flags & MOE_SCORING_SIGMOID) ? moe_gate::kGateSigmoid : 0);
  a.given_ids = given_ids ? 1 : 0;
  a.expert_map = expert_map;
  a.E_local = E_local;
  a.bs = block_size;
  a.bs_shift = (block_size & (block_size - 1)) == 0 ? __builtin_ctz(static_cast<unsigned>(block_size)) : -1;
  a.P = P;
  a.C = C;
  a.NB = static_cast<int>((C + block_size - 1) / block_size);
  const int elem = dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const int sms = moe_host::sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  // the gating kernel and its tile height: one thread per row for many short rows (32-row tiles);
  // else one warp per row, in 16-row tiles when all of them fit on the SMs at once (then each warp
  // gates one row), 32-row tiles above
  const bool small_batch = T <= kSmallMaxTokens && P <= kSmallMaxSlots && E <= kSmallMaxExperts;
  const bool lanes = !small_batch && !given_ids && moe_gate::lane_gating_fits(T, E, k, elem, logits);
  int rt = kRowsPerTile;
  if (!lanes && (T + kRowsPerTileSmall - 1) / kRowsPerTileSmall <= static_cast<int64_t>(sms) * kGcCtasPerSm)
    rt = kRowsPerTileSmall;
  const FusedLayout lay = fused_layout(T, E_local, rt);
  a.rows_per_tile = rt;
  a.rt_shift = rt == kRowsPerTileSmall ? 4 : 5;
  a.num_tiles = lay.num_tiles;
  a.topk_weights = topk_weights;
  a.topk_ids = topk_ids;
  a.counts = counts;
  a.offsets = offsets;
  a.sorted_ids = sorted_token_ids;
  a.expert_ids = expert_ids;
  a.n_pad = num_tokens_post_pad;
  a.inv_perm = inv_perm;
  a.status = static_cast<int32_t*>(workspace);
  a.tile_counts = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + lay.tile_counts_off);
  a.totals = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + lay.totals_off);

  // gating geometry of the warp-per-row kernels: widest aligned vector that spreads the row over the warp
  int vec_max = 16 / elem;
  while (vec_max > 1 && ((E % vec_max) != 0 || (reinterpret_cast<uintptr_t>(logits) % (vec_max * elem)) != 0))
    vec_max >>= 1;
  int vec = 1;
  for (int v = vec_max; v >= 1; v >>= 1) {
    if ((E % v) == 0 && E / v >= 32) {
      vec = v;
      break;
    }
  }
  if (E < 32) vec = 1;
  const int n_chunks = E / vec;
  int cpl = 1;
  while (cpl * 32 < n_chunks) cpl <<= 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // small batches: one kernel, one CTA per slot
  if (small_batch) {
    // at most one warp of slots: route_decode_kernel (two CTA barriers); above: route_small_kernel
    const bool one_warp = P <= kDecodeMaxSlots;
    SmallKernel sk = given_ids ? (one_warp ? &route_decode_kernel<float, 1, 1, true> : &route_small_kernel<float, 1, 1, true>)
                     : one_warp ? (dtype == MOE_DTYPE_BF16 ? family_pick<DecodeFamily, __nv_bfloat16>(vec, cpl)
                                                          : family_pick<DecodeFamily, float>(vec, cpl))
                     : dtype == MOE_DTYPE_BF16 ? family_pick<SmallFamily, __nv_bfloat16>(vec, cpl)
                                               : family_pick<SmallFamily, float>(vec, cpl);
    if (sk == nullptr) return MOE_ERR_UNSUPPORTED;
    const dim3 grid = P > 0 ? dim3(static_cast<unsigned>(k), static_cast<unsigned>(T)) : dim3(1, 1);  // (j, t)
    return moe_host::launch_pdl(sk, grid, dim3(kSmallThreads), 0, st, a, static_cast<const uint4*>(hidden),
                                static_cast<int>(row_bytes / 16u), static_cast<uint4*>(permuted));
  }

  if (lanes) {
    const int cpr = E * elem / 16;
    const int G = moe_gate::lane_gate_lanes(cpr);
    LanesKernel lk = dtype == MOE_DTYPE_BF16 ? lanes_kernel_for<__nv_bfloat16>(k, G) : lanes_kernel_for<float>(k, G);
    if (lk == nullptr) return MOE_ERR_UNSUPPORTED;
    const size_t smem1 = static_cast<size_t>(kRowsPerTile) * moe_gate::lane_tile_stride(cpr) * sizeof(uint4) +
                         (2 * static_cast<size_t>(G) * E_local + static_cast<size_t>(kRowsPerTile) * k) * sizeof(int);
    if (smem1 > 48 * 1024 &&
        cudaFuncSetAttribute(reinterpret_cast<const void*>(lk), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem1)) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (moe_host::launch_pdl_max_shared(lk, dim3(static_cast<unsigned>(a.num_tiles)), dim3(32 * G), smem1, st, a, cpr) !=
        MOE_OK)
      return MOE_ERR_CUDA;
  } else {
    // the gating geometry does not matter when the routes are given (no row is gated)
    GcKernel gk = given_ids ? family_pick<GateCountFamily, float>(1, 1)
                  : dtype == MOE_DTYPE_BF16 ? family_pick<GateCountFamily, __nv_bfloat16>(vec, cpl)
                                            : family_pick<GateCountFamily, float>(vec, cpl);
    if (gk == nullptr) return MOE_ERR_UNSUPPORTED;
    const size_t smem1 = gc_smem_ints(a.rows_per_tile, k, E_local) * sizeof(int);
    if (smem1 > 48 * 1024 &&
        cudaFuncSetAttribute(reinterpret_cast<const void*>(gk), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem1)) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (moe_host::launch_pdl_max_shared(gk, dim3(static_cast<unsigned>(a.num_tiles)), dim3(kGcThreads), smem1, st, a) != MOE_OK)
      return MOE_ERR_CUDA;
  }
  if (launch_tile_scan(a, E_local, st) != MOE_OK) return MOE_ERR_CUDA;

  // tokens per CTA: at most kPgMaxTokens (and kPgCtaBytes of staged rows), chosen so that the CTAs
  // fill whole waves of kPgCtasPerSm per SM; shared memory sized so that no SM takes more
  int tpc = static_cast<int>(kPgCtaBytes / row_bytes);
  tpc = tpc < 1 ? 1 : (tpc > kPgMaxTokens ? kPgMaxTokens : tpc);
  tpc = moe_host::tokens_per_cta(T, tpc, static_cast<int64_t>(sms) * kPgCtasPerSm);
  int64_t blocks = (T + tpc - 1) / tpc;
  if (blocks < 1) blocks = 1;
  if (blocks > 0x7fffffff) return MOE_ERR_INVALID_ARG;
  const size_t smem2 = moe_host::smem_for_ctas_per_sm(
      static_cast<size_t>(tpc) * row_bytes + static_cast<size_t>(E_local + 1) * sizeof(int), kPgCtasPerSm);
  if (smem2 == 0) return MOE_ERR_CUDA;
  if (smem2 > 48 * 1024 &&
      cudaFuncSetAttribute(place_gather_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem2)) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  return moe_host::launch_pdl_max_shared(place_gather_kernel<true>, dim3(static_cast<unsigned>(blocks)), dim3(32), smem2, st, a,
                              static_cast<const uint8_t*>(hidden), row_bytes, tpc, static_cast<uint8_t*>(permuted));
}

// ---------------------------------------------------------------------------------------------
// moe_align_permute through the tile kernels above (given routes, no gather).
// ---------------------------------------------------------------------------------------------
size_t moe_internal::align_tiles_workspace_bytes(int64_t T, int32_t E_local) {
  return fused_layout(T, E_local, kRowsPerTile).bytes;
}

moe_status_t moe_internal::align_tiles(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E_global,
                                       const int32_t* expert_map, int32_t E_local, int32_t block_size,
                                       int32_t* counts, int32_t* offsets, int32_t* sorted_token_ids,
                                       int32_t* expert_ids, int32_t* num_tokens_post_pad, int32_t* inv_perm,
                                       void* workspace, cudaStream_t st) {
  DispatchArgs a{};
  a.T = T;
  a.E = E_global;
  a.k = k;
  a.given_ids = 1;
  a.expert_map = expert_map;
  a.E_local = E_local;
  a.bs = block_size;
  a.bs_shift = (block_size & (block_size - 1)) == 0 ? __builtin_ctz(static_cast<unsigned>(block_size)) : -1;
  a.P = T * k;
  a.C = moe_align_capacity(T, k, E_local, block_size);
  a.NB = static_cast<int>((a.C + block_size - 1) / block_size);
  const FusedLayout lay = fused_layout(T, E_local, kRowsPerTile);
  a.rows_per_tile = kRowsPerTile;
  a.rt_shift = 5;
  a.num_tiles = lay.num_tiles;
  a.topk_ids = const_cast<int32_t*>(topk_ids);  // read only: given_ids
  a.counts = counts;
  a.offsets = offsets;
  a.sorted_ids = sorted_token_ids;
  a.expert_ids = expert_ids;
  a.n_pad = num_tokens_post_pad;
  a.inv_perm = inv_perm;
  a.status = static_cast<int32_t*>(workspace);
  a.tile_counts = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + lay.tile_counts_off);
  a.totals = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + lay.totals_off);

  GcKernel gk = family_pick<GateCountFamily, float>(1, 1);  // no row is gated
  const size_t smem1 = gc_smem_ints(a.rows_per_tile, k, E_local) * sizeof(int);
  if (smem1 > 48 * 1024 &&
      cudaFuncSetAttribute(reinterpret_cast<const void*>(gk), cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem1)) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe_host::launch_pdl_max_shared(gk, dim3(static_cast<unsigned>(a.num_tiles)), dim3(kGcThreads), smem1, st, a) != MOE_OK)
    return MOE_ERR_CUDA;
  if (launch_tile_scan(a, E_local, st) != MOE_OK) return MOE_ERR_CUDA;
  // placement only: up to kPgMaxTokens tokens per one-warp CTA, the CTAs filling whole waves
  const int sms = moe_host::sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  const int tpc = moe_host::tokens_per_cta(T, kPgMaxTokens, static_cast<int64_t>(sms) * 16);
  int64_t blocks = (T + tpc - 1) / tpc;
  if (blocks < 1) blocks = 1;
  if (blocks > 0x7fffffff) return MOE_ERR_INVALID_ARG;
  const size_t smem2 = static_cast<size_t>(E_local + 1) * sizeof(int);
  return moe_host::launch_pdl_max_shared(place_gather_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(32), smem2, st,
                              a, static_cast<const uint8_t*>(nullptr), 0u, tpc, static_cast<uint8_t*>(nullptr));
}
