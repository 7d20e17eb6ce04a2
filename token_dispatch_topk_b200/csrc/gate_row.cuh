// gate_row.cuh -- fused softmax + top-k of one row of router logits by one warp.
//
// Operation: "Upstream Reference: Deep-Spark xllm + vllm", "File Index"
// (moe_topk_softmax_kernels.cuh: fused softmax+topk; vLLM topk_softmax_kernels.cu).
//
// Lane l holds chunks l, l+32, ... of VEC logits of the row.  bf16 logits fit a 32-bit key
// (ordered 16-bit value above, 0xFFFF - index below), so each selection round is a single
// warp-wide redux max; fp32 logits use a 64-bit key (ordered 32-bit value above, inverted index
// below), reduced as its high word, then the low word among the lanes holding that high word.
// Either way the round's maximum is the largest logit with the lowest index among equals, and the
// winner is retired (0 is below every real key).  With at most 8 keys per lane the keys are sorted
// once (a sorting network) so that a round is one redux of the lanes' top keys and a shift in the
// winning lane; with more, each round takes the lane maximum and zeroes the winner.  Lane j keeps round j's key;
// after the rounds each of lanes 0..k-1 takes one exp, and a warp sum gives the renormalising
// denominator (the full-row denominator Z is reduced in round 0 only when not renormalising).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moe_gate {

// Scoring mode bits of gate_row and the gating kernels.
constexpr int kGateRenorm = 1;   // renormalise the k weights to sum to 1
constexpr int kGateSigmoid = 2;  // score each expert with the logistic function instead of the softmax

__device__ __forceinline__ uint32_t ordered_bits(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) == 0u) u = 0u;  // -0 and +0 compare equal
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float ordered_to_float(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

__device__ __forceinline__ uint64_t make_key(float x, int e) {
  return (static_cast<uint64_t>(ordered_bits(x)) << 32) | static_cast<uint32_t>(0xffffffffu - static_cast<uint32_t>(e));
}

// Load VEC consecutive logits of a row as fp32.
template <typename TIn, int VEC>
struct VecLoad;

template <>
struct VecLoad<__nv_bfloat16, 8> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, float (&v)[8]) {
    uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    v[0] = moe::bf16_lo(u.x); v[1] = moe::bf16_hi(u.x); v[2] = moe::bf16_lo(u.y); v[3] = moe::bf16_hi(u.y);
    v[4] = moe::bf16_lo(u.z); v[5] = moe::bf16_hi(u.z); v[6] = moe::bf16_lo(u.w); v[7] = moe::bf16_hi(u.w);
  }
};
template <>
struct VecLoad<__nv_bfloat16, 4> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, float (&v)[4]) {
    uint2 u = __ldcs(reinterpret_cast<const uint2*>(p));
    v[0] = moe::bf16_lo(u.x); v[1] = moe::bf16_hi(u.x); v[2] = moe::bf16_lo(u.y); v[3] = moe::bf16_hi(u.y);
  }
};
template <>
struct VecLoad<__nv_bfloat16, 2> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, float (&v)[2]) {
    uint32_t u = __ldcs(reinterpret_cast<const unsigned int*>(p));
    v[0] = moe::bf16_lo(u); v[1] = moe::bf16_hi(u);
  }
};
template <>
struct VecLoad<__nv_bfloat16, 1> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, float (&v)[1]) {
    uint32_t u = __ldcs(reinterpret_cast<const unsigned short*>(p));
    v[0] = moe::bf16_lo(u);
  }
};
template <>
struct VecLoad<float, 4> {
  static __device__ __forceinline__ void run(const float* p, float (&v)[4]) {
    float4 u = __ldcs(reinterpret_cast<const float4*>(p));
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
};
template <>
struct VecLoad<float, 2> {
  static __device__ __forceinline__ void run(const float* p, float (&v)[2]) {
    float2 u = __ldcs(reinterpret_cast<const float2*>(p));
    v[0] = u.x; v[1] = u.y;
  }
};
template <>
struct VecLoad<float, 1> {
  static __device__ __forceinline__ void run(const float* p, float (&v)[1]) { v[0] = __ldcs(p); }
};

__device__ __forceinline__ uint32_t ordered16(uint32_t b) {
  b &= 0xffffu;
  if ((b & 0x7fffu) == 0u) b = 0u;  // -0 == +0
  return (b & 0x8000u) ? (~b & 0xffffu) : (b | 0x8000u);
}

__device__ __forceinline__ float ordered16_to_float(uint32_t o) {
  const uint32_t b = (o & 0x8000u) ? (o & 0x7fffu) : (~o & 0xffffu);
  return __uint_as_float(b << 16);
}

// Raw 16-bit patterns of VEC consecutive bf16 logits.
template <int VEC>
struct Bf16Bits;
template <>
struct Bf16Bits<8> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, uint32_t (&b)[8]) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    b[0] = u.x & 0xffffu; b[1] = u.x >> 16; b[2] = u.y & 0xffffu; b[3] = u.y >> 16;
    b[4] = u.z & 0xffffu; b[5] = u.z >> 16; b[6] = u.w & 0xffffu; b[7] = u.w >> 16;
  }
};
template <>
struct Bf16Bits<4> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, uint32_t (&b)[4]) {
    const uint2 u = __ldcs(reinterpret_cast<const uint2*>(p));
    b[0] = u.x & 0xffffu; b[1] = u.x >> 16; b[2] = u.y & 0xffffu; b[3] = u.y >> 16;
  }
};
template <>
struct Bf16Bits<2> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, uint32_t (&b)[2]) {
    const uint32_t u = __ldcs(reinterpret_cast<const unsigned int*>(p));
    b[0] = u & 0xffffu; b[1] = u >> 16;
  }
};
template <>
struct Bf16Bits<1> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, uint32_t (&b)[1]) {
    b[0] = __ldcs(reinterpret_cast<const unsigned short*>(p));
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Descending sorting networks for a lane's NV <= 8 keys (compare-exchange: larger key first).
template <typename K>
__device__ __forceinline__ void cas_desc(K& x, K& y) {
  const K hi = x > y ? x : y;
  const K lo = x > y ? y : x;
  x = hi;
  y = lo;
}

template <int NV, typename K>
__device__ __forceinline__ void sort_desc(K (&k)[NV]) {
  if constexpr (NV == 2) {
    cas_desc(k[0], k[1]);
  } else if constexpr (NV == 4) {
    cas_desc(k[0], k[1]); cas_desc(k[2], k[3]);
    cas_desc(k[0], k[2]); cas_desc(k[1], k[3]);
    cas_desc(k[1], k[2]);
  } else if constexpr (NV == 8) {  // Batcher odd-even merge sort, 19 comparators
    cas_desc(k[0], k[1]); cas_desc(k[2], k[3]); cas_desc(k[4], k[5]); cas_desc(k[6], k[7]);
    cas_desc(k[0], k[2]); cas_desc(k[1], k[3]); cas_desc(k[4], k[6]); cas_desc(k[5], k[7]);
    cas_desc(k[1], k[2]); cas_desc(k[5], k[6]);
    cas_desc(k[0], k[4]); cas_desc(k[1], k[5]); cas_desc(k[2], k[6]); cas_desc(k[3], k[7]);
    cas_desc(k[2], k[4]); cas_desc(k[3], k[5]);
    cas_desc(k[1], k[2]); cas_desc(k[3], k[4]); cas_desc(k[5], k[6]);
  }
}

// Retire the lane's top key when it won the round: shift the sorted keys up by one.
template <int NV, typename K>
__device__ __forceinline__ void pop_front_if(K (&k)[NV], bool hit) {
#pragma unroll
  for (int i = 0; i + 1 < NV; ++i) k[i] = hit ? k[i + 1] : k[i];
  k[NV - 1] = hit ? K(0) : k[NV - 1];
}

// The selection key of an expert: bf16 logits give a 32-bit key, fp32 logits a 64-bit one (see the
// file comment); 0 is below every real key.
template <typename TIn>
struct GateKey {
  using type = uint64_t;
};
template <>
struct GateKey<__nv_bfloat16> {
  using type = uint32_t;
};

template <typename TIn>
__device__ __forceinline__ int key_expert(typename GateKey<TIn>::type key) {
  if constexpr (sizeof(TIn) == 2) {
    return static_cast<int>(0xffffu - (key & 0xffffu));
  } else {
    return static_cast<int>(0xffffffffu - static_cast<uint32_t>(key));
  }
}

template <typename TIn>
__device__ __forceinline__ float key_value(typename GateKey<TIn>::type key) {
  if constexpr (sizeof(TIn) == 2) {
    return ordered16_to_float(key >> 16);
  } else {
    return ordered_to_float(static_cast<uint32_t>(key >> 32));
  }
}

// The selection half of gate_row (all 32 lanes of the warp call it): lanes 0..k-1 return the key of
// rank `lane` in my_key; every lane returns the row's largest key in best0 and, for the softmax
// without renormalisation, the full-row denominator Z (else 0).
template <typename TIn, int VEC, int CPL>
__device__ __forceinline__ void gate_row_select(const TIn* __restrict__ rp, int E, int k, int mode, int lane,
                                                typename GateKey<TIn>::type& my_key,
                                                typename GateKey<TIn>::type& best0, float& Z) {
  constexpr int NV = CPL * VEC;
  const int n_chunks = E / VEC;
  const bool full_row_z = (mode & (kGateRenorm | kGateSigmoid)) == 0;
  Z = 0.f;

  if constexpr (sizeof(TIn) == 2) {
    uint32_t key[NV];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const int chunk = lane + 32 * c;
      if (chunk < n_chunks) {
        uint32_t b[VEC];
        Bf16Bits<VEC>::run(rp + chunk * VEC, b);
#pragma unroll
        for (int i = 0; i < VEC; ++i) key[c * VEC + i] = (ordered16(b[i]) << 16) | (0xffffu - static_cast<uint32_t>(chunk * VEC + i));
      } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) key[c * VEC + i] = 0u;
      }
    }
    my_key = 0u;
    best0 = 0u;
    constexpr bool kSorted = NV <= 8;  // few keys per lane: keep them sorted, the lane's top is key[0]
    if constexpr (kSorted) sort_desc<NV>(key);
    for (int j = 0; j < k; ++j) {
      uint32_t best = 0u;
      if constexpr (kSorted) {
        best = key[0];
      } else {
#pragma unroll
        for (int i = 0; i < NV; ++i) best = key[i] > best ? key[i] : best;
      }
      best = __reduce_max_sync(0xffffffffu, best);
      if (j == 0) {
        best0 = best;
        if (full_row_z) {  // full-row denominator, from the keys before any is retired
          const float m = ordered16_to_float(best >> 16);
          float z = 0.f;
#pragma unroll
          for (int i = 0; i < NV; ++i) {
            if (key[i] != 0u) z += expf(ordered16_to_float(key[i] >> 16) - m);
          }
          Z = warp_sum(z);
        }
      }
      if constexpr (kSorted) {
        pop_front_if<NV>(key, key[0] == best);
      } else {
#pragma unroll
        for (int i = 0; i < NV; ++i) key[i] = (key[i] == best) ? 0u : key[i];
      }
      if (lane == j) my_key = best;
    }
  } else {
    uint64_t key[NV];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const int chunk = lane + 32 * c;
      if (chunk < n_chunks) {
        float v[VEC];
        VecLoad<TIn, VEC>::run(rp + chunk * VEC, v);
#pragma unroll
        for (int i = 0; i < VEC; ++i) key[c * VEC + i] = make_key(v[i], chunk * VEC + i);
      } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) key[c * VEC + i] = 0ull;
      }
    }
    my_key = 0ull;
    best0 = 0ull;
    constexpr bool kSorted = NV <= 8;
    if constexpr (kSorted) sort_desc<NV>(key);
    for (int j = 0; j < k; ++j) {
      uint64_t mine = 0ull;
      if constexpr (kSorted) {
        mine = key[0];
      } else {
#pragma unroll
        for (int i = 0; i < NV; ++i) mine = key[i] > mine ? key[i] : mine;
      }
      const uint32_t hi = __reduce_max_sync(0xffffffffu, static_cast<uint32_t>(mine >> 32));
      const uint32_t lo = __reduce_max_sync(0xffffffffu, static_cast<uint32_t>(mine >> 32) == hi
                                                             ? static_cast<uint32_t>(mine) : 0u);
      const uint64_t best = (static_cast<uint64_t>(hi) << 32) | lo;
      if (j == 0) {
        best0 = best;
        if (full_row_z) {
          const float m = ordered_to_float(hi);
          float z = 0.f;
#pragma unroll
          for (int i = 0; i < NV; ++i) {
            if (key[i] != 0ull) z += expf(ordered_to_float(static_cast<uint32_t>(key[i] >> 32)) - m);
          }
          Z = warp_sum(z);
        }
      }
      if constexpr (kSorted) {
        pop_front_if<NV>(key, key[0] == best);
      } else {
#pragma unroll
        for (int i = 0; i < NV; ++i) key[i] = (key[i] == best) ? 0ull : key[i];
      }
      if (lane == j) my_key = best;
    }
  }
}

// The weights half of gate_row (all 32 lanes call it, with gate_row_select's outputs): lanes 0..k-1
// return the expert of rank `lane` in my_e and its weight in my_w; other lanes' outputs are
// unspecified.  Softmax weights are exp(x - m) over Z (or over the k selected when renormalising);
// sigmoid weights are 1 / (1 + exp(-x)) each (or over their sum, 1/k if it is 0).
template <typename TIn>
__device__ __forceinline__ void gate_row_weights(typename GateKey<TIn>::type my_key, typename GateKey<TIn>::type best0,
                                                 float Z, int k, int mode, int lane, int& my_e, float& my_w) {
  const bool renormalize = (mode & kGateRenorm) != 0;
  const bool sigmoid = (mode & kGateSigmoid) != 0;
  const float m = key_value<TIn>(best0);
  float my_p = 0.f, S = 0.f;
  my_e = 0;
  if (lane < k) {
    const float xj = key_value<TIn>(my_key);
    my_p = sigmoid ? 1.f / (1.f + expf(-xj)) : expf(xj - m);
    my_e = key_expert<TIn>(my_key);
  }
  if (renormalize) S = warp_sum(my_p);
  if (sigmoid) {
    my_w = renormalize ? (S > 0.f ? my_p / S : 1.f / static_cast<float>(k)) : my_p;
  } else {
    my_w = my_p / (renormalize ? S : Z);
  }
}

// Top-k of one row (all 32 lanes of the warp call it).  Lanes 0..k-1 return the expert of rank
// `lane` in my_e and its weight in my_w; other lanes' outputs are unspecified.  `mode`: bits
// kGateRenorm and kGateSigmoid (see gate_row_weights).
template <typename TIn, int VEC, int CPL>
__device__ __forceinline__ void gate_row(const TIn* __restrict__ rp, int E, int k, int mode, int lane,
                                         int& my_e, float& my_w) {
  typename GateKey<TIn>::type key, best0;
  float Z;
  gate_row_select<TIn, VEC, CPL>(rp, E, k, mode, lane, key, best0, Z);
  gate_row_weights<TIn>(key, best0, Z, k, mode, lane, my_e, my_w);
}

}  // namespace moe_gate
