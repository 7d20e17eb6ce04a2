// gather_combine.cu -- activation permute-gather and top-k weighted combine.
//
// Operations: "Upstream Reference: Deep-Spark xllm + vllm", "File Index" -- the
// FusedMoE pipeline "gate -> topk -> expand -> gemm1 -> act -> gemm2 -> combine"
// (expand = the permute-gather into the expert-grouped layout, combine = the top-k
// weighted sum back to token order; moe_align_sum_kernels.cu names the "sum"), and
// the "final permuted gather" of the 2026-07-16 MTP1 M=2 compact scheduler closure note.
//
// Both kernels are token-major and bandwidth-bound: one warp owns one token (or one
// segment of a long row when there are too few tokens to fill the GPU).  Lane j < k
// holds the row inv_perm[t*k+j] of the token's j-th slot (and its weight) and hands
// it to the warp by shuffle, so the per-slot indices are read once per warp.
//   gather:  each hidden row is read once (16-byte loads, U vectors in flight per
//            lane) and stored to every local destination row.
//   combine: for each 16-byte column chunk, up to 8 slot rows are loaded before the
//            fp32 fused multiply-adds run in ascending j from +0, then one bf16
//            round-to-nearest-even store.
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
  const int lane = threadIdx.x & 31;
  const int64_t p = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  if (p >= capacity || p >= static_cast<int64_t>(n_pad[0])) return;
  if (sorted_ids[p] != pad_value) return;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  uint4* dst = permuted + p * NV;
  for (int v = lane; v < NV; v += 32) moe::st_plain(dst + v, z);
}

__global__ void __launch_bounds__(kWarpsPerCta * 32)
combine_kernel(const uint4* __restrict__ expert_out, const float* __restrict__ topk_weights,
               const int32_t* __restrict__ inv_perm, int64_t T, int NV, int k, int seg, int seg_len, int64_t capacity,
               uint4* __restrict__ out, int32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  const int64_t t = gw / seg;
  if (t >= T) return;  // uniform per warp
  const int sg = static_cast<int>(gw - t * seg);
  const int v0 = sg * seg_len;
  const int v1 = (v0 + seg_len < NV) ? v0 + seg_len : NV;
  const int myrow = lane_row(inv_perm, t, k, capacity, lane, status);
  const float myw = lane < k ? topk_weights[t * k + lane] : 0.f;
  uint4* dst = out + t * NV;

  for (int vb = v0; vb < v1; vb += 32) {
    const int v = vb + lane;
    const bool ok = v < v1;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j0 = 0; j0 < k; j0 += 8) {
      uint4 yv[8];
      int rr[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        rr[jj] = __shfl_sync(0xffffffffu, myrow, (j0 + jj) & 31);  // lanes >= k hold -1
        yv[jj] = make_uint4(0u, 0u, 0u, 0u);
        if (j0 + jj < k && rr[jj] >= 0 && ok) yv[jj] = moe::ld_stream(expert_out + static_cast<int64_t>(rr[jj]) * NV + v);
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const float w = __shfl_sync(0xffffffffu, myw, (j0 + jj) & 31);
        if (j0 + jj < k && rr[jj] >= 0) {
          acc[0] = fmaf(w, moe::bf16_lo(yv[jj].x), acc[0]);
          acc[1] = fmaf(w, moe::bf16_hi(yv[jj].x), acc[1]);
          acc[2] = fmaf(w, moe::bf16_lo(yv[jj].y), acc[2]);
          acc[3] = fmaf(w, moe::bf16_hi(yv[jj].y), acc[3]);
          acc[4] = fmaf(w, moe::bf16_lo(yv[jj].z), acc[4]);
          acc[5] = fmaf(w, moe::bf16_hi(yv[jj].z), acc[5]);
          acc[6] = fmaf(w, moe::bf16_lo(yv[jj].w), acc[6]);
          acc[7] = fmaf(w, moe::bf16_hi(yv[jj].w), acc[7]);
        }
      }
    }
    if (ok) {
      uint4 o;
      o.x = moe::pack_bf16x2(acc[0], acc[1]);
      o.y = moe::pack_bf16x2(acc[2], acc[3]);
      o.z = moe::pack_bf16x2(acc[4], acc[5]);
      o.w = moe::pack_bf16x2(acc[6], acc[7]);
      moe::st_plain(dst + v, o);
    }
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
  if ((flags & ~MOE_GATHER_ZERO_PAD) != 0u) return MOE_ERR_INVALID_ARG;
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
  if (T > 0) {
    int seg, seg_len;
    segment_rows(T, NV, &seg, &seg_len);
    const int64_t warps = T * seg;
    const int64_t blocks = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
    if (blocks > 0x7fffffff) return MOE_ERR_INVALID_ARG;
    gather_kernel<<<static_cast<unsigned>(blocks), kWarpsPerCta * 32, 0, st>>>(
        static_cast<const uint4*>(hidden), T, NV, k, seg, seg_len, inv_perm, capacity, static_cast<uint4*>(permuted),
        device_status);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (zero_pad && capacity > 0) {
    const int64_t blocks = (capacity + kWarpsPerCta - 1) / kWarpsPerCta;
    zero_pad_kernel<<<static_cast<unsigned>(blocks), kWarpsPerCta * 32, 0, st>>>(
        sorted_token_ids, num_tokens_post_pad, capacity, NV, static_cast<int32_t>(T * k),
        static_cast<uint4*>(permuted));
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
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
  const int NV = H / 8;
  int seg, seg_len;
  segment_rows(T, NV, &seg, &seg_len);
  const int64_t warps = T * seg;
  const int64_t blocks = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
  if (blocks > 0x7fffffff) return MOE_ERR_INVALID_ARG;
  combine_kernel<<<static_cast<unsigned>(blocks), kWarpsPerCta * 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(expert_out), topk_weights, inv_perm, T, NV, k, seg, seg_len, capacity,
      static_cast<uint4*>(out), device_status);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
