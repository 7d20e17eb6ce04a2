// gather_combine.cu -- activation permute-gather and top-k weighted combine.
//
// Operations: "Upstream Reference: Deep-Spark xllm + vllm", "File Index" -- the
// FusedMoE pipeline "gate -> topk -> expand -> gemm1 -> act -> gemm2 -> combine"
// (expand = the permute-gather into the expert-grouped layout, combine = the top-k
// weighted sum back to token order; moe_align_sum_kernels.cu names the "sum"), and
// the "final permuted gather" of the 2026-07-16 MTP1 M=2 compact scheduler closure note.
//
// Both stages are token-major and bandwidth-bound.  The main kernels move rows with TMA
// bulk copies (cp.async.bulk, no multicast) through shared memory:
//   gather_tma_kernel:  each hidden row is bulk-loaded once and bulk-stored to every
//                       local destination row of its token; rows loaded after the wait for
//                       inv_perm are only those of tokens with a local slot.
//   combine_tma_kernel: a producer warp bulk-loads the local slot rows of each (token,
//                       column chunk) into a ring of stages; consumer warps run the fp32
//                       fused multiply-adds in ascending slot order from +0 and store one
//                       bf16 round-to-nearest-even result.
// The register-staged gather_kernel (one warp per token or row segment, lane j < k holding
// the row of slot j) covers rows too long to stage; zero_pad_kernel fills pad rows on request.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace {

constexpr int kWarpsPerCta = 8;
constexpr int kGatherUnroll = 4;

// Row index of lane j's slot, or -1 (remote, absent, or out of range -> flagged).
__device__ __forceinline__ int lane_row(const int32_t* inv_perm, int64_t t, int k, int64_t capacity, int lane,
                                        int32_t* status) {
  int r = -1;
  if (lane < k) {
    r = inv_perm[t * k + lane];
    if (r < -1 || static_cast<int64_t>(r) >= capacity) {
      moe::record_status(status, MOE_ERR_BAD_ROW);
      r = -1;
    }
  }
  return r;
}

__global__ void __launch_bounds__(kWarpsPerCta * 32)
gather_kernel(const uint4* __restrict__ hidden, int64_t T, int NV, int k, int seg, int seg_len,
              const int32_t* __restrict__ inv_perm, int64_t capacity, uint4* __restrict__ permuted, int32_t* status) {
  moe::pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  const int64_t t = gw / seg;
  if (t >= T) return;  // uniform per warp
  const int sg = static_cast<int>(gw - t * seg);
  const int v0 = sg * seg_len;
  const int v1 = (v0 + seg_len < NV) ? v0 + seg_len : NV;
  const int myrow = lane_row(inv_perm, t, k, capacity, lane, status);
  const uint4* src = hidden + t * NV;

  for (int vb = v0; vb < v1; vb += 32 * kGatherUnroll) {
    uint4 x[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int v = vb + u * 32 + lane;
      if (v < v1) x[u] = moe::ld_stream(src + v);
    }
    for (int j = 0; j < k; ++j) {
      const int r = __shfl_sync(0xffffffffu, myrow, j);
      if (r < 0) continue;  // uniform: remote slot
      uint4* dst = permuted + static_cast<int64_t>(r) * NV;
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int v = vb + u * 32 + lane;
        if (v < v1) moe::st_plain(dst + v, x[u]);
      }
    }
  }
}

// +0 into every pad row below N_pad (rows whose slot id is the pad value P).
__global__ void __launch_bounds__(kWarpsPerCta * 32)
zero_pad_kernel(const int32_t* __restrict__ sorted_ids, const int32_t* __restrict__ n_pad, int64_t capacity, int NV,
                int32_t pad_value, uint4* __restrict__ permuted) {
  moe::pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t p = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  if (p >= capacity || p >= static_cast<int64_t>(n_pad[0])) return;
  if (sorted_ids[p] != pad_value) return;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  uint4* dst = permuted + p * NV;
  for (int v = lane; v < NV; v += 32) moe::st_plain(dst + v, z);
}

// ------------------------------------------------------------------------------------------
// TMA kernels.  Rows move as whole bulk copies through shared memory: the copy engine keeps
// many kilobytes in flight per SM without holding registers, which register-staged copies
// cannot (occupancy-limited, one dependent load/store phase per iteration).
// ------------------------------------------------------------------------------------------
constexpr int kGatherMaxTokensPerCta = 8;
constexpr uint32_t kGatherCtaBytes = 32u * 1024u;  // hidden rows staged per CTA
constexpr int kGatherCtasPerSm = 4;                 // gather_tma_kernel CTAs resident per SM

// One warp per CTA: lane 0 bulk-loads the CTA's `tokens_per_cta` hidden rows into shared memory
// while the lanes read the rows' destinations; then every lane bulk-stores the staged rows of its
// slots to their expert-grouped rows.
__global__ void __launch_bounds__(32)
gather_tma_kernel(const uint8_t* __restrict__ hidden, int64_t T, uint32_t row_bytes, int k, int tokens_per_cta,
                  const int32_t* __restrict__ inv_perm, int64_t capacity, uint8_t* __restrict__ permuted,
                  int32_t* status, int hidden_ready) {
  extern __shared__ __align__(128) uint8_t rows[];
  __shared__ __align__(8) uint64_t bar;
  const int lane = threadIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * tokens_per_cta;
  const int n = static_cast<int>((T - t0) < tokens_per_cta ? (T - t0) : tokens_per_cta);
  if (lane == 0) {
    moe::mbar_init(&bar, 1);
    moe::fence_barrier_init();
  }
  __syncwarp();
  const bool evict_first = row_bytes <= moe::kEvictFirstMaxRowBytes;
  auto load_rows = [&](unsigned mask) {  // bit i: load the row of token t0 + i
    if (lane == 0) {
      moe::mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(__popc(mask)) * row_bytes);
      for (int i = 0; i < n; ++i) {
        if ((mask >> i) & 1u)
          moe::bulk_load(rows + static_cast<size_t>(i) * row_bytes,
                         hidden + (t0 + i) * static_cast<int64_t>(row_bytes), row_bytes, &bar, evict_first);
      }
    }
  };
  const unsigned all_rows = n >= 32 ? 0xffffffffu : (1u << n) - 1u;
  if (hidden_ready) load_rows(all_rows);  // hidden predates the previous kernel: load it while that kernel finishes
  moe::pdl_launch_dependents();
  moe::pdl_wait();                 // inv_perm comes from the previous kernel
  const int nslots = n * k;  // <= 8 * 32
  int32_t dst[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int e = lane + 32 * m;
    int r = -1;
    if (e < nslots) {
      r = inv_perm[t0 * k + e];
      if (r < -1 || static_cast<int64_t>(r) >= capacity) {
        moe::record_status(status, MOE_ERR_BAD_ROW);
        r = -1;
      }
    }
    dst[m] = r;
  }
  if (!hidden_ready) {
    // loaded after the wait: only the rows of tokens with a local slot (a token whose slots are all
    // remote is never stored, and its row may sit in another GPU's memory)
    unsigned need = 0u;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      if (dst[m] >= 0) need |= 1u << ((lane + 32 * m) / k);
    }
    load_rows(__reduce_or_sync(0xffffffffu, need));
  }
  if (!moe::mbar_wait(&bar, 0)) {
    moe::record_status(status, MOE_ERR_TIMEOUT);
    moe::mbar_wait(&bar, 0);  // give the loads in flight one more bounded wait before leaving
    return;
  }
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int e = lane + 32 * m;
    if (e < nslots && dst[m] >= 0) {
      moe::bulk_store(permuted + static_cast<int64_t>(dst[m]) * row_bytes, rows + static_cast<size_t>(e / k) * row_bytes,
                      row_bytes, evict_first);
    }
  }
  moe::bulk_commit();
  moe::bulk_wait_read_all();  // the staged rows must outlive the stores that read them
}

constexpr int kCombineConsumerWarps = 8;
constexpr int kCombineMaxStages = 8;
constexpr uint32_t kCombineStageTarget = 32u * 1024u;  // bytes of slot rows per stage (about)
constexpr uint32_t kCombineRingTarget = 64u * 1024u;   // bytes of stages per CTA (about)

struct CombineArgs {
  const uint8_t* y;         // expert_out [capacity, H] bf16
  const float* w;           // [T, k]
  const int32_t* inv_perm;  // [T*k]
  int64_t T;
  int k;
  int tpu;                  // tokens per unit (tpu * k <= 32)
  int stages;               // depth of the shared-memory ring
  uint32_t row_bytes;       // H * 2
  uint32_t chunk_bytes;     // bytes of one row chunk (a unit covers one chunk of tpu tokens)
  int nchunks;
  int64_t units;            // ceil(T / tpu) * nchunks
  int64_t capacity;
  uint8_t* out;             // [T, H] bf16
  int32_t* status;
};

// Persistent, warp-specialised: warp 0 produces, warps 1..8 consume.  A unit is one column chunk
// of `tpu` consecutive tokens (tpu * k slot rows, about 32 KB).  The producer bulk-loads the chunk
// of every local slot row of the unit into a stage of a shared-memory ring (mbarrier `full`), with
// the slot weights and a validity mask beside it; one consumer thread waits for the stage and the
// consumer warps are released together by a named barrier (waiting warps take no issue slots).
// Consumers accumulate in fp32 (fmaf, ascending slot order, from +0), store the bf16 result and
// release the stage (mbarrier `empty`, one arrival per consumer warp).
template <int KU>  // slot loop unrolled KU times (k rounded up to 2, 4 or 8; blocks of 8 beyond)
__global__ void __launch_bounds__((1 + kCombineConsumerWarps) * 32) combine_tma_kernel(CombineArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int k = a.k;
  const int S = a.stages;
  const int spu = a.tpu * k;  // slot rows per unit (<= 32)
  const uint32_t stage_bytes = static_cast<uint32_t>(spu) * a.chunk_bytes;
  uint8_t* buf = smem;
  float* s_w = reinterpret_cast<float*>(smem + static_cast<size_t>(S) * stage_bytes);  // [S][32] slot weights
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(s_w + S * 32);                          // [S]
  uint64_t* full = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(s_mask + S) + 7) & ~uintptr_t(7));
  uint64_t* empty = full + S;
  __shared__ int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // an even share of the units (floor(b * units / G) up to floor((b + 1) * units / G)): every CTA
  // of the grid works, and the SMs, each holding the same number of CTAs, get the same bytes
  const int64_t u0 = static_cast<int64_t>(blockIdx.x) * a.units / gridDim.x;
  const int64_t u1 = static_cast<int64_t>(blockIdx.x + 1) * a.units / gridDim.x;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      moe::mbar_init(&full[s], 1);
      moe::mbar_init(&empty[s], kCombineConsumerWarps);
    }
    s_abort = 0;
    moe::fence_barrier_init();
  }
  __syncthreads();
  moe::pdl_launch_dependents();
  moe::pdl_wait();  // slot rows, weights and expert outputs come from earlier kernels
  if (u0 >= u1) return;

  if (warp == 0) {
    // ---- producer: lane l < spu handles slot l of the unit (token t0 + l / k, rank l % k)
    const bool evict_first = a.row_bytes <= moe::kEvictFirstMaxRowBytes;
    auto load_meta = [&](int64_t grp, int& r, float& w) {
      r = -1;
      w = 0.f;
      const int64_t t = grp * a.tpu + lane / k;
      if (lane < spu && t < a.T) {
        const int64_t s = t * k + lane % k;
        r = a.inv_perm[s];
        w = a.w[s];
        if (r < -1 || static_cast<int64_t>(r) >= a.capacity) {
          moe::record_status(a.status, MOE_ERR_BAD_ROW);
          r = -1;
        }
      }
    };
    int64_t grp = u0 / a.nchunks;  // token group of unit u (advanced without dividing)
    int c = static_cast<int>(u0 - grp * a.nchunks);
    int r_cur, r_next;
    float w_cur, w_next;
    load_meta(grp, r_cur, w_cur);
    load_meta(grp + 1, r_next, w_next);
    int s = 0;
    uint32_t round = 0;  // completed passes over the ring
    int64_t issued = 0;
    for (int64_t u = u0; u < u1; ++u, ++issued) {
      if (u != u0 && ++c == a.nchunks) {  // units are in group order: next group, prefetch the one after
        c = 0;
        ++grp;
        r_cur = r_next;
        w_cur = w_next;
        load_meta(grp + 1, r_next, w_next);
      }
      if (issued >= S && !moe::mbar_wait(&empty[s], (round - 1) & 1u)) {
        moe::record_status(a.status, MOE_ERR_TIMEOUT);
        s_abort = 1;
        break;
      }
      const uint32_t mask = __ballot_sync(0xffffffffu, r_cur >= 0);
      const uint32_t cb = (c == a.nchunks - 1) ? a.row_bytes - static_cast<uint32_t>(c) * a.chunk_bytes : a.chunk_bytes;
      s_w[s * 32 + lane] = w_cur;
      if (lane == 0) s_mask[s] = mask;
      __threadfence_block();
      __syncwarp();
      if (lane == 0) moe::mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(__popc(mask)) * cb);
      __syncwarp();
      if (r_cur >= 0) {
        moe::bulk_load(buf + static_cast<size_t>(s) * stage_bytes + static_cast<size_t>(lane) * a.chunk_bytes,
                       a.y + static_cast<int64_t>(r_cur) * a.row_bytes + static_cast<int64_t>(c) * a.chunk_bytes, cb,
                       &full[s], evict_first);
      }
      if (++s == S) {
        s = 0;
        ++round;
      }
    }
    if (s_abort && lane == 0) {
      // never leave with loads in flight into this CTA's shared memory: fills older than the
      // last S were consumed before their stage was refilled, so wait (bounded) for those S
      for (int64_t q = issued > S ? issued - S : 0; q < issued; ++q) {
        moe::mbar_wait(&full[q % S], static_cast<uint32_t>(q / S) & 1u);
      }
    }
    return;
  }

  // ---- consumers
  const int ct = tid - 32;
  constexpr int NCT = kCombineConsumerWarps * 32;
  int s = 0;
  uint32_t round = 0;
  int64_t grp = u0 / a.nchunks;  // token group of unit u (advanced without dividing)
  int c = static_cast<int>(u0 - grp * a.nchunks) - 1;
  for (int64_t u = u0; u < u1; ++u) {
    if (++c == a.nchunks) {
      c = 0;
      ++grp;
    }
    if (ct == 0 && !moe::mbar_wait(&full[s], round & 1u)) {
      moe::record_status(a.status, MOE_ERR_TIMEOUT);
      s_abort = 1;
    }
    moe::named_barrier(1, NCT);
    if (s_abort) break;
    while (!moe::mbar_try_wait(&full[s], round & 1u)) {
    }  // completed already: gives this thread its own acquire of the stage
    const uint32_t cb = (c == a.nchunks - 1) ? a.row_bytes - static_cast<uint32_t>(c) * a.chunk_bytes : a.chunk_bytes;
    const uint32_t mask = s_mask[s];
    const uint8_t* stage = buf + static_cast<size_t>(s) * stage_bytes;
    const int nvec = static_cast<int>(cb >> 4);
    for (int ti = 0; ti < a.tpu; ++ti) {
      const int64_t t = grp * a.tpu + ti;
      if (t >= a.T) break;
      const uint32_t tmask = mask >> (ti * k);
      const uint8_t* tok = stage + static_cast<size_t>(ti) * k * a.chunk_bytes;
      const float* wt = s_w + s * 32 + ti * k;
      uint8_t* dst = a.out + t * static_cast<int64_t>(a.row_bytes) + static_cast<int64_t>(c) * a.chunk_bytes;
      for (int v = ct; v < nvec; v += NCT) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        const uint8_t* col = tok + static_cast<size_t>(v) * 16;
        for (int j0 = 0; j0 < k; j0 += KU) {
#pragma unroll
        for (int jj = 0; jj < KU; ++jj) {
          const int j = j0 + jj;
          if (j < k && ((tmask >> j) & 1u)) {  // ascending slot order
            const uint4 yv = moe::lds128(col + static_cast<size_t>(j) * a.chunk_bytes);
            const float w = wt[j];
            acc[0] = fmaf(w, moe::bf16_lo(yv.x), acc[0]);
            acc[1] = fmaf(w, moe::bf16_hi(yv.x), acc[1]);
            acc[2] = fmaf(w, moe::bf16_lo(yv.y), acc[2]);
            acc[3] = fmaf(w, moe::bf16_hi(yv.y), acc[3]);
            acc[4] = fmaf(w, moe::bf16_lo(yv.z), acc[4]);
            acc[5] = fmaf(w, moe::bf16_hi(yv.z), acc[5]);
            acc[6] = fmaf(w, moe::bf16_lo(yv.w), acc[6]);
            acc[7] = fmaf(w, moe::bf16_hi(yv.w), acc[7]);
          }
        }
        }
        uint4 o;
        o.x = moe::pack_bf16x2(acc[0], acc[1]);
        o.y = moe::pack_bf16x2(acc[2], acc[3]);
        o.z = moe::pack_bf16x2(acc[4], acc[5]);
        o.w = moe::pack_bf16x2(acc[6], acc[7]);
        moe::st_plain(reinterpret_cast<uint4*>(dst + static_cast<size_t>(v) * 16), o);
      }
    }
    __syncwarp();
    if (lane == 0) moe::mbar_arrive(&empty[s]);
    if (++s == S) {
      s = 0;
      ++round;
    }
  }
}

// Small batches (decode): a batch of a few tokens is a chain of latencies (slot rows and weights,
// then the k expert rows), not a stream.  Grid (ceil(nvec / kCombineSmallThreads), T): thread v of
// token t reads the slot rows and weights of t (lane j holds slot j, passed around by shuffles),
// issues the loads of its 16-byte column of all the token's local slot rows together, then
// accumulates them in fp32 (fmaf, ascending slot order, from +0) and stores the bf16 result.
constexpr int kCombineSmallThreads = 128;

template <int KU>  // slots loaded together (k rounded up to 2, 4 or 8; blocks of 8 beyond)
__global__ void __launch_bounds__(kCombineSmallThreads)
combine_small_kernel(const uint4* __restrict__ y, const float* __restrict__ w, const int32_t* __restrict__ inv_perm,
                     int k, int nvec, int64_t capacity, uint4* __restrict__ out, int32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t t = blockIdx.y;
  const int v = blockIdx.x * kCombineSmallThreads + threadIdx.x;
  y = moe::pin(y);  // parameters into registers before waiting (moe::pin)
  w = moe::pin(w);
  inv_perm = moe::pin(inv_perm);
  k = moe::pin(k);
  nvec = moe::pin(nvec);
  capacity = moe::pin(capacity);
  out = moe::pin(out);
  status = moe::pin(status);
  moe::pdl_launch_dependents();
  moe::pdl_wait();  // slot rows, weights and expert outputs come from earlier kernels
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int j0 = 0; j0 < k; j0 += 32) {
    int r = -1;
    float wj = 0.f;
    if (j0 + lane < k) {
      r = inv_perm[t * k + j0 + lane];
      wj = w[t * k + j0 + lane];
      if (r < -1 || static_cast<int64_t>(r) >= capacity) {
        moe::record_status(status, MOE_ERR_BAD_ROW);
        r = -1;
      }
    }
    const int kb = (k - j0) < 32 ? (k - j0) : 32;
    for (int j1 = 0; j1 < kb; j1 += KU) {
      uint4 yv[KU];
      int rr[KU];
#pragma unroll
      for (int jj = 0; jj < KU; ++jj) {
        rr[jj] = __shfl_sync(0xffffffffu, r, (j1 + jj) & 31);
        if (j1 + jj >= kb) rr[jj] = -1;
        if (rr[jj] >= 0 && v < nvec) yv[jj] = __ldg(y + static_cast<int64_t>(rr[jj]) * nvec + v);
      }
#pragma unroll
      for (int jj = 0; jj < KU; ++jj) {
        const float wt = __shfl_sync(0xffffffffu, wj, (j1 + jj) & 31);
        if (rr[jj] >= 0 && v < nvec) {  // ascending slot order
          acc[0] = fmaf(wt, moe::bf16_lo(yv[jj].x), acc[0]);
          acc[1] = fmaf(wt, moe::bf16_hi(yv[jj].x), acc[1]);
          acc[2] = fmaf(wt, moe::bf16_lo(yv[jj].y), acc[2]);
          acc[3] = fmaf(wt, moe::bf16_hi(yv[jj].y), acc[3]);
          acc[4] = fmaf(wt, moe::bf16_lo(yv[jj].z), acc[4]);
          acc[5] = fmaf(wt, moe::bf16_hi(yv[jj].z), acc[5]);
          acc[6] = fmaf(wt, moe::bf16_lo(yv[jj].w), acc[6]);
          acc[7] = fmaf(wt, moe::bf16_hi(yv[jj].w), acc[7]);
        }
      }
    }
  }
  if (v < nvec) {
    uint4 o;
    o.x = moe::pack_bf16x2(acc[0], acc[1]);
    o.y = moe::pack_bf16x2(acc[2], acc[3]);
    o.z = moe::pack_bf16x2(acc[4], acc[5]);
    o.w = moe::pack_bf16x2(acc[6], acc[7]);
    out[t * nvec + v] = o;
  }
}

// Split each token row into `seg` segments of `seg_len` 16-byte vectors so that small
// batches still put enough warps on the GPU (about half its warp slots).
void segment_rows(int64_t T, int NV, int* seg, int* seg_len) {
  const int64_t target_warps = 148 * 32;
  int64_t s = (target_warps + T - 1) / (T > 0 ? T : 1);
  const int max_seg = (NV + 31) / 32;
  if (s < 1) s = 1;
  if (s > max_seg) s = max_seg;
  int len = static_cast<int>((NV + s - 1) / s);
  len = (len + 31) & ~31;
  *seg_len = len;
  *seg = (NV + len - 1) / len;
}

}  // namespace

extern "C" moe_status_t moe_gather(const void* hidden, int64_t T, int32_t H, int32_t k, const int32_t* inv_perm,
                                   const int32_t* sorted_token_ids, const int32_t* num_tokens_post_pad,
                                   int64_t capacity, uint32_t flags, void* permuted, int32_t* device_status,
                                   void* stream) {
  if (T < 0 || H < 1 || k < 1 || capacity < 0) return MOE_ERR_INVALID_ARG;
  if (k > 32) return MOE_ERR_UNSUPPORTED;
  if ((H % 8) != 0) return MOE_ERR_INVALID_ARG;
  if ((flags & ~(MOE_GATHER_ZERO_PAD | MOE_GATHER_HIDDEN_READY)) != 0u) return MOE_ERR_INVALID_ARG;
  const bool zero_pad = (flags & MOE_GATHER_ZERO_PAD) != 0u;
  if (T > (int64_t{1} << 40) || T * k >= (int64_t{1} << 30) || capacity >= (int64_t{1} << 31))
    return MOE_ERR_INVALID_ARG;
  if (zero_pad && (sorted_token_ids == nullptr || num_tokens_post_pad == nullptr)) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (hidden == nullptr || inv_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if ((T > 0 || zero_pad) && capacity > 0 && permuted == nullptr) return MOE_ERR_INVALID_ARG;
  if ((hidden && !moe_host::aligned16(hidden)) || (permuted && !moe_host::aligned16(permuted)))
    return MOE_ERR_INVALID_ARG;
  const int NV = H / 8;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
  if (T > 0 && row_bytes <= kGatherCtaBytes * 4u) {
    // tokens per CTA: at most kGatherMaxTokensPerCta (and kGatherCtaBytes of staged rows), chosen so
    // that the CTAs fill whole waves of kGatherCtasPerSm per SM; shared memory sized so that no SM
    // takes more (CTAs placed while the previous kernel runs would otherwise crowd its idle SMs)
    int tpc = static_cast<int>(kGatherCtaBytes / row_bytes);
    if (tpc < 1) tpc = 1;
    if (tpc > kGatherMaxTokensPerCta) tpc = kGatherMaxTokensPerCta;
    const int sms = moe_host::sm_count();
    if (sms <= 0) return MOE_ERR_CUDA;
    tpc = moe_host::tokens_per_cta(T, tpc, static_cast<int64_t>(sms) * kGatherCtasPerSm);
    const int64_t blocks = (T + tpc - 1) / tpc;
    const size_t smem = moe_host::smem_for_ctas_per_sm(static_cast<size_t>(tpc) * row_bytes, kGatherCtasPerSm);
    if (smem == 0) return MOE_ERR_CUDA;
    if (blocks > 0x7fffffff) return MOE_ERR_INVALID_ARG;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(gather_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess)
      return MOE_ERR_CUDA;
    const int ready = (flags & MOE_GATHER_HIDDEN_READY) ? 1 : 0;
    if (moe_host::launch_pdl_max_shared(gather_tma_kernel, dim3(static_cast<unsigned>(blocks)), dim3(32), smem, st,
                             static_cast<const uint8_t*>(hidden), T, row_bytes, k, tpc, inv_perm, capacity,
                             static_cast<uint8_t*>(permuted), device_status, ready) != MOE_OK)
      return MOE_ERR_CUDA;
  } else if (T > 0) {  // rows beyond 128 KB: register-staged copy
    int seg, seg_len;
    segment_rows(T, NV, &seg, &seg_len);
    const int64_t warps = T * seg;
    const int64_t blocks = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
    if (blocks > 0x7fffffff) return MOE_ERR_INVALID_ARG;
    if (moe_host::launch_pdl(gather_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kWarpsPerCta * 32), 0, st,
                             static_cast<const uint4*>(hidden), T, NV, k, seg, seg_len, inv_perm, capacity,
                             static_cast<uint4*>(permuted), device_status) != MOE_OK)
      return MOE_ERR_CUDA;
  }
  if (zero_pad && capacity > 0) {
    const int64_t blocks = (capacity + kWarpsPerCta - 1) / kWarpsPerCta;
    if (moe_host::launch_pdl(zero_pad_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kWarpsPerCta * 32), 0, st,
                             sorted_token_ids, num_tokens_post_pad, capacity, NV, static_cast<int32_t>(T * k),
                             static_cast<uint4*>(permuted)) != MOE_OK)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

extern "C" moe_status_t moe_combine(const void* expert_out, const float* topk_weights, const int32_t* inv_perm,
                                    int64_t T, int32_t k, int32_t H, int64_t capacity, void* out,
                                    int32_t* device_status, void* stream) {
  if (T < 0 || H < 1 || k < 1 || capacity < 0) return MOE_ERR_INVALID_ARG;
  if (k > 32) return MOE_ERR_UNSUPPORTED;
  if ((H % 8) != 0) return MOE_ERR_INVALID_ARG;
  if (T > (int64_t{1} << 40) || T * k >= (int64_t{1} << 30) || capacity >= (int64_t{1} << 31))
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (topk_weights == nullptr || inv_perm == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  if (capacity > 0 && expert_out == nullptr) return MOE_ERR_INVALID_ARG;
  if ((expert_out && !moe_host::aligned16(expert_out)) || !moe_host::aligned16(out)) return MOE_ERR_INVALID_ARG;
  CombineArgs a{};
  a.y = static_cast<const uint8_t*>(expert_out);
  a.w = topk_weights;
  a.inv_perm = inv_perm;
  a.T = T;
  a.k = k;
  a.row_bytes = static_cast<uint32_t>(H) * 2u;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int nvec = static_cast<int>(a.row_bytes / 16u);
  if (T * ((a.row_bytes + 4095u) / 4096u) < sms) {  // small batch: fewer 4 KB row chunks than SMs
    void (*ks)(const uint4*, const float*, const int32_t*, int, int, int64_t, uint4*, int32_t*) =
        k <= 2 ? combine_small_kernel<2> : k <= 4 ? combine_small_kernel<4> : combine_small_kernel<8>;
    const dim3 grid(static_cast<unsigned>((nvec + kCombineSmallThreads - 1) / kCombineSmallThreads),
                    static_cast<unsigned>(T));
    return moe_host::launch_pdl(ks, grid, dim3(kCombineSmallThreads), 0, static_cast<cudaStream_t>(stream),
                                static_cast<const uint4*>(expert_out), topk_weights, inv_perm, static_cast<int>(k),
                                nvec, capacity, static_cast<uint4*>(out), device_status);
  }
  // a unit: `tpu` tokens x k slot rows x one chunk of each row, about 32 KB
  const uint32_t chunk_cap = k <= 8 ? 4096u : (k <= 16 ? 2048u : 1024u);
  a.chunk_bytes = a.row_bytes < chunk_cap ? a.row_bytes : chunk_cap;
  a.nchunks = static_cast<int>((a.row_bytes + a.chunk_bytes - 1) / a.chunk_bytes);
  int tpu = static_cast<int>(kCombineStageTarget / (static_cast<uint32_t>(k) * a.chunk_bytes));
  if (tpu < 1) tpu = 1;
  if (tpu * k > 32) tpu = 32 / k;
  a.tpu = tpu;
  const uint32_t stage_bytes = static_cast<uint32_t>(tpu * k) * a.chunk_bytes;
  int stages = static_cast<int>(kCombineRingTarget / stage_bytes);
  stages = stages < 2 ? 2 : (stages > kCombineMaxStages ? kCombineMaxStages : stages);
  a.stages = stages;
  a.units = ((T + tpu - 1) / tpu) * a.nchunks;
  a.capacity = capacity;
  a.out = static_cast<uint8_t*>(out);
  a.status = device_status;
  const size_t smem = static_cast<size_t>(stages) * stage_bytes + static_cast<size_t>(stages) * 32 * sizeof(float) +
                      stages * sizeof(uint32_t) + 8 + 2 * stages * sizeof(uint64_t);
  int per_sm = static_cast<int>((200u * 1024u) / (smem + 1024));
  per_sm = per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm);
  // the fewest CTAs that still give no CTA more units than the resident maximum would: every CTA then
  // gets the same number of units (or one fewer for a few), so no handful of CTAs carries a last unit
  // alone while the rest have finished.  Measured on one GPU: the 4096 x 128 prefill combine 25.1 us
  // a launch against 26.8 us with every resident CTA (410 CTAs of 10 units against 444 of 9 or 10).
  const int64_t resident = static_cast<int64_t>(sms) * per_sm;
  const int64_t units_per_cta = (a.units + resident - 1) / resident;
  const int64_t grid = (a.units + units_per_cta - 1) / units_per_cta;
  void (*kern)(CombineArgs) = k <= 2 ? combine_tma_kernel<2> : k <= 4 ? combine_tma_kernel<4> : combine_tma_kernel<8>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return moe_host::launch_pdl_max_shared(kern, dim3(static_cast<unsigned>(grid)), dim3((1 + kCombineConsumerWarps) * 32), smem,
                              static_cast<cudaStream_t>(stream), a);
}
