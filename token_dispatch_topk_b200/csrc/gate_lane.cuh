// gate_lane.cuh -- fused softmax + top-k of router-logit rows, a few lanes per row.
//
// Operation: the fused softmax+topk of "Upstream Reference: Deep-Spark xllm + vllm", "File Index"
// (moe_topk_softmax_kernels.cuh; vLLM topk_softmax_kernels.cu), with the same selection order and
// weights as gate_row.cuh: the k largest logits, larger first, the lower expert index first among
// equal logits; softmax over the whole row (or over the k with renormalisation), or the logistic
// scores of the sigmoid variant (moe_topk_sigmoid_kernels.cuh).
//
// gate_row.cuh spends a warp on each row: k rounds of warp-wide reductions, a few hundred
// instructions per row, which makes gating of many short rows (say E = 60 experts, T = 16K tokens)
// bound by instruction issue.  Here a CTA stages 32 rows in shared memory and G lanes (up to 8)
// scan each row once.  bf16 logits become unique 32-bit keys, and their K largest come from sorting
// networks (a sort of each 16-byte chunk, then bitonic merges of the lists: about 5 instructions per
// logit for K = 8).  fp32 logits are inserted into a register-resident list of the K largest, as value
// and index (about 5 * K instructions per logit).  The G lists are merged with log2(G) shuffle rounds.
// That is several times fewer instructions per row than the warp-per-row kernel.
//
// Order: fp32 logits arrive in ascending expert order and a logit moves ahead only of kept logits it
// strictly exceeds, so among equal logits the lower index stays ahead (+0 and -0 compare equal); bf16
// keys hold the inverted index below the value, so the same order is the keys' order.
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "gate_row.cuh"

namespace moe_gate {

constexpr int kLaneGateMaxK = 8;            // K is a template parameter: 1..8
constexpr int kLaneGateMaxE = 64;           // rows of up to 64 logits: from 1024 rows on
constexpr int64_t kLaneGateMinRows = 1024;  // below this, the warp-per-row kernels have lower latency
constexpr int kLaneGateWideMaxE = 256;      // bf16 rows of up to 256 logits: from 16384 rows on
constexpr int64_t kLaneGateWideMinRows = 16384;

// Whether a batch of rows takes the lane gating (the same rule for every entry point, so that
// moe_topk_softmax and moe_route_dispatch choose the same arithmetic for the same batch).
// Rows must be whole 16-byte chunks and the logits 16-byte aligned.  Short rows take it from 1024
// rows on.  Wider bf16 rows take it only for large batches, where gating is bound by instruction
// issue: measured in back-to-back steps of the 4096 x 128 prefill batch, the lane kernel was
// slower than one warp per row there (65.9 against 63.6 us a step).
inline bool lane_gating_fits(int64_t T, int E, int k, int elem_bytes, const void* logits) {
  if (k > kLaneGateMaxK || (E * elem_bytes) % 16 != 0 || (reinterpret_cast<uintptr_t>(logits) & 15u) != 0)
    return false;
  if (E <= kLaneGateMaxE) return T >= kLaneGateMinRows;
  return elem_bytes == 2 && E <= kLaneGateWideMaxE && T >= kLaneGateWideMinRows;
}

// Shared-memory layout of a staged tile: row r starts at chunk r * stride, stride = chunks per row
// rounded up to odd, so lanes reading 16 bytes of different rows at the same offset hit distinct
// bank groups.
__host__ __device__ inline int lane_tile_stride(int cpr) { return cpr | 1; }

// Copy rows [0, rows) of a tile (contiguous in global memory, 16-byte aligned, cpr chunks a row)
// into shared memory with coalesced 16-byte loads, kLaneLoadBatch of them in flight per thread
// before the first store (the kernels stage at most 4 chunks per thread: one batch).
// Chunk c of the tile belongs to row c / cpr, computed as floor((c + 0.5) / cpr) in fp32: exact
// for the tile sizes here (c < 2^12, cpr <= 32: the fraction stays at least 1/64 from an integer,
// far above the rounding error).
constexpr int kLaneLoadBatch = 4;
__device__ __forceinline__ void lane_tile_load(const uint4* __restrict__ g, int rows, int cpr, int stride,
                                               uint4* __restrict__ s, int tid, int nthreads) {
  const int n = rows * cpr;
  const float inv = 1.f / static_cast<float>(cpr);
  for (int c0 = tid; c0 < n; c0 += kLaneLoadBatch * nthreads) {
    uint4 v[kLaneLoadBatch];
#pragma unroll
    for (int u = 0; u < kLaneLoadBatch; ++u) {
      const int c = c0 + u * nthreads;
      if (c < n) v[u] = __ldcs(g + c);
    }
#pragma unroll
    for (int u = 0; u < kLaneLoadBatch; ++u) {
      const int c = c0 + u * nthreads;
      if (c < n) {
        const int r = static_cast<int>((static_cast<float>(c) + 0.5f) * inv);
        s[r * stride + (c - r * cpr)] = v[u];
      }
    }
  }
}

// The K largest logits seen so far, larger first (v), with their experts (e).
template <int K>
struct LaneTopK {
  float v[K];
  int e[K];

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int p = 0; p < K; ++p) {
      v[p] = -INFINITY;
      e[p] = 0;
    }
  }

  // Logit x of expert i, experts arriving in ascending order.
  __device__ __forceinline__ void insert(float x, int i) {
    bool gt[K];
#pragma unroll
    for (int p = 0; p < K; ++p) gt[p] = x > v[p];
#pragma unroll
    for (int p = K - 1; p > 0; --p) {
      v[p] = gt[p - 1] ? v[p - 1] : (gt[p] ? x : v[p]);
      e[p] = gt[p - 1] ? e[p - 1] : (gt[p] ? i : e[p]);
    }
    v[0] = gt[0] ? x : v[0];
    e[0] = gt[0] ? i : e[0];
  }
};

// bf16 logits: the ordered 16-bit value above, 0xFFFF - expert below, so the keys of a row are
// unique and their order is the selection order (0 is below every key of a finite logit).  Keys being
// unique, the K largest of a set do not depend on the order in which its parts are combined, so they
// are found with sorting networks: each 16-byte chunk's 8 keys are sorted (Batcher's 19
// compare-exchanges), and two descending lists of KP keys (KP = K rounded up to a power of two,
// padded with 0) give the KP largest of both as max(a[i], b[KP-1-i]), a bitonic sequence that
// log2(KP) rounds of half-cleaners sort.  No chain runs through all the keys of a row, so most
// compare-exchanges are independent.
__device__ __forceinline__ uint32_t bf16_key(uint32_t bits16, int e) {
  return (ordered16(bits16) << 16) | (0xffffu - static_cast<uint32_t>(e));
}

template <int K>
struct KeyListSize {
  static constexpr int value = K <= 1 ? 1 : (K <= 2 ? 2 : (K <= 4 ? 4 : 8));
};

// v bitonic -> v sorted descending (half-cleaners at distance KP/2, ..., 1).
template <int KP>
__device__ __forceinline__ void bitonic_sort_desc(uint32_t (&v)[KP]) {
#pragma unroll
  for (int d = KP / 2; d >= 1; d >>= 1) {
#pragma unroll
    for (int i = 0; i < KP; ++i) {
      if ((i & d) == 0) {
        const uint32_t a = v[i], b = v[i + d];
        v[i] = a > b ? a : b;
        v[i + d] = a > b ? b : a;
      }
    }
  }
}

// l, o descending -> l = the KP largest of both, descending.
template <int KP>
__device__ __forceinline__ void merge_top_keys(uint32_t (&l)[KP], const uint32_t (&o)[KP]) {
#pragma unroll
  for (int i = 0; i < KP; ++i) {
    const uint32_t b = o[KP - 1 - i];
    l[i] = l[i] > b ? l[i] : b;
  }
  bitonic_sort_desc<KP>(l);
}

// The KP largest keys of one 16-byte chunk of bf16 logits (chunk j of the row), descending.
template <int KP>
__device__ __forceinline__ void chunk_top_keys(const uint4 q, int j, uint32_t (&out)[KP]) {
  const int i = 8 * j;
  uint32_t c[8] = {bf16_key(q.x & 0xffffu, i),     bf16_key(q.x >> 16, i + 1), bf16_key(q.y & 0xffffu, i + 2),
                   bf16_key(q.y >> 16, i + 3),     bf16_key(q.z & 0xffffu, i + 4), bf16_key(q.z >> 16, i + 5),
                   bf16_key(q.w & 0xffffu, i + 6), bf16_key(q.w >> 16, i + 7)};
  sort_desc<8>(c);
#pragma unroll
  for (int r = 0; r < KP; ++r) out[r] = c[r];
}

// Insert the logits of one 16-byte chunk (chunk j of the row) in ascending expert order.
template <typename TIn, int K>
__device__ __forceinline__ void lane_insert_chunk(LaneTopK<K>& t, const uint4 q, int j) {
  if constexpr (sizeof(TIn) == 4) {
    const int i = 4 * j;
    t.insert(__uint_as_float(q.x), i);
    t.insert(__uint_as_float(q.y), i + 1);
    t.insert(__uint_as_float(q.z), i + 2);
    t.insert(__uint_as_float(q.w), i + 3);
  } else {
    const int i = 8 * j;
    t.insert(moe::bf16_lo(q.x), i);
    t.insert(moe::bf16_hi(q.x), i + 1);
    t.insert(moe::bf16_lo(q.y), i + 2);
    t.insert(moe::bf16_hi(q.y), i + 3);
    t.insert(moe::bf16_lo(q.z), i + 4);
    t.insert(moe::bf16_hi(q.z), i + 5);
    t.insert(moe::bf16_lo(q.w), i + 6);
    t.insert(moe::bf16_hi(q.w), i + 7);
  }
}

// Lanes per row: G lanes share a row (G = 1, 2, 4, or 8 for rows of more than 16 chunks), lane g
// scanning chunks [g * cpr / G, (g + 1) * cpr / G) (one to four chunks each, read into registers
// once).  More lanes per row put more warps in flight for the same instructions per row: the scan
// is a chain of dependent inserts, and one lane per row leaves too few warps.
__host__ __device__ inline int lane_gate_lanes(int cpr) {
  return cpr > 16 ? 8 : (cpr >= 4 ? 4 : (cpr >= 2 ? 2 : 1));
}
constexpr int kLaneMaxChunks = 4;  // chunks one lane holds: cpr / G rounded up, <= 4 for cpr <= 32

// Gate one staged row (cpr 16-byte chunks of TIn logits; E = cpr * 16 / sizeof(TIn)) with the G
// lanes g = lane % G of a row group (consecutive lanes; every lane of the warp calls this).
// `mode`: kGateRenorm, kGateSigmoid.  Every lane of the group returns the K experts in selection
// order and their weights.
// Merge, after each lane's scan, pairwise over shuffle distance 1, 2, then 4:
//   bf16: the keys are unique, so the bitonic merge of the partner's list gives the K largest of both.
//   fp32: the list of the lower chunks is the base and the other is inserted into it in its own
//   order.  Every expert of the inserted list has a higher index than every expert of the base,
//   and among equal logits the inserted list keeps the lower index ahead, so the merged list is
//   the one a single scan in expert order would give.
template <typename TIn, int K, int G>
__device__ __forceinline__ void lane_gate_row(const uint4* __restrict__ srow, int cpr, int mode, int g,
                                              float (&w)[K], int (&ids)[K]) {
  const int j0 = (g * cpr) / G, j1 = ((g + 1) * cpr) / G;
  uint4 q[kLaneMaxChunks];
#pragma unroll
  for (int u = 0; u < kLaneMaxChunks; ++u) {
    if (j0 + u < j1) q[u] = srow[j0 + u];
  }
  LaneTopK<K> t;
  if constexpr (sizeof(TIn) == 2) {
    constexpr int KP = KeyListSize<K>::value;
    uint32_t kt[KP];
#pragma unroll
    for (int r = 0; r < KP; ++r) kt[r] = 0u;
#pragma unroll
    for (int u = 0; u < kLaneMaxChunks; ++u) {
      if (j0 + u < j1) {
        uint32_t c[KP];
        chunk_top_keys<KP>(q[u], j0 + u, c);
        merge_top_keys<KP>(kt, c);
      }
    }
#pragma unroll
    for (int d = 1; d < G; d <<= 1) {
      uint32_t o[KP];
#pragma unroll
      for (int r = 0; r < KP; ++r) o[r] = __shfl_xor_sync(0xffffffffu, kt[r], d);
      merge_top_keys<KP>(kt, o);
    }
#pragma unroll
    for (int r = 0; r < K; ++r) {
      t.v[r] = ordered16_to_float(kt[r] >> 16);
      t.e[r] = static_cast<int>(0xffffu - (kt[r] & 0xffffu));
    }
  } else {
    t.init();
#pragma unroll
    for (int u = 0; u < kLaneMaxChunks; ++u) {
      if (j0 + u < j1) lane_insert_chunk<TIn, K>(t, q[u], j0 + u);
    }
#pragma unroll
    for (int d = 1; d < G; d <<= 1) {
      LaneTopK<K> o;
#pragma unroll
      for (int r = 0; r < K; ++r) {
        o.v[r] = __shfl_xor_sync(0xffffffffu, t.v[r], d);
        o.e[r] = __shfl_xor_sync(0xffffffffu, t.e[r], d);
      }
      const bool upper = (g & d) != 0;  // this lane's chunks come after the partner's
      LaneTopK<K> base, add;
#pragma unroll
      for (int r = 0; r < K; ++r) {
        base.v[r] = upper ? o.v[r] : t.v[r];
        base.e[r] = upper ? o.e[r] : t.e[r];
        add.v[r] = upper ? t.v[r] : o.v[r];
        add.e[r] = upper ? t.e[r] : o.e[r];
      }
#pragma unroll
      for (int r = 0; r < K; ++r) base.insert(add.v[r], add.e[r]);
      t = base;
    }
  }
  const bool renormalize = (mode & kGateRenorm) != 0;
  const bool sigmoid = (mode & kGateSigmoid) != 0;
  const float m = t.v[0];
  float p[K];
  float den = 0.f;
#pragma unroll
  for (int r = 0; r < K; ++r) {
    p[r] = sigmoid ? 1.f / (1.f + expf(-t.v[r])) : expf(t.v[r] - m);
    den += p[r];
  }
  if (!renormalize && !sigmoid) {  // full-row denominator: each lane sums its chunks, then the group
    float z[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums (short dependency chains)
#pragma unroll
    for (int u = 0; u < kLaneMaxChunks; ++u) {
      if (j0 + u < j1) {
        if constexpr (sizeof(TIn) == 4) {
          z[0] += expf(__uint_as_float(q[u].x) - m);
          z[1] += expf(__uint_as_float(q[u].y) - m);
          z[2] += expf(__uint_as_float(q[u].z) - m);
          z[3] += expf(__uint_as_float(q[u].w) - m);
        } else {
          z[0] += expf(moe::bf16_lo(q[u].x) - m) + expf(moe::bf16_hi(q[u].x) - m);
          z[1] += expf(moe::bf16_lo(q[u].y) - m) + expf(moe::bf16_hi(q[u].y) - m);
          z[2] += expf(moe::bf16_lo(q[u].z) - m) + expf(moe::bf16_hi(q[u].z) - m);
          z[3] += expf(moe::bf16_lo(q[u].w) - m) + expf(moe::bf16_hi(q[u].w) - m);
        }
      }
    }
    den = (z[0] + z[1]) + (z[2] + z[3]);
#pragma unroll
    for (int d = 1; d < G; d <<= 1) den += __shfl_xor_sync(0xffffffffu, den, d);
  }
#pragma unroll
  for (int r = 0; r < K; ++r) {
    if (sigmoid) {
      w[r] = renormalize ? (den > 0.f ? p[r] / den : 1.f / static_cast<float>(K)) : p[r];
    } else {
      w[r] = p[r] / den;
    }
    ids[r] = t.e[r];
  }
}

}  // namespace moe_gate
