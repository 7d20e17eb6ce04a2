// topk_softmax.cu -- fused softmax + top-k gating over router logits.
//
// Operation: "Upstream Reference: Deep-Spark xllm + vllm", "File Index"
// (moe_topk_softmax_kernels.cuh: fused softmax+topk; vLLM topk_softmax_kernels.cu),
// placed by "Call Chain: MoE topk_softmax on BI-V100" between the router and the experts.
//
// Design (sm_100a).  Many rows of short logit rows and k <= 8 (moe_gate::lane_gating_fits): up
// to eight lanes per row (topk_lane_kernel below, gate_lane.cuh).  Otherwise rows of E >= 16 experts: one
// warp per row (topk_row_warp_kernel below), one warp-wide redux.sync max per selection round;
// short rows (E < 16): the sub-warp kernel described here.
// Sub-warp kernel: a sub-warp of G lanes (G a power of two, 1..32) owns one row.
// Each lane loads its share of the row with 16-byte vector loads (8-, 4- or
// 2-byte, or scalar, when the row length or base pointer does not allow 16),
// keeps it in registers as 64-bit ordered keys (value bits above, inverted
// index below), and the k experts are chosen by k rounds of a shuffle-xor max
// over the G lanes.  Because the key orders by value first and by lower index
// second, the round's maximum is the largest logit with the lowest index among
// equals, and the winner is retired by zeroing its key (0 is below every real
// key, so retired and padding slots can never win while k <= E).  Round 0 also
// yields the row maximum m, from which the full-row sum Z of exp(x - m) is
// reduced the same way.  Selected probabilities exp(x_j - m) are staged per
// warp in shared memory and written out with contiguous stores after the
// division by Z (or by their own sum when renormalising).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "gate_lane.cuh"
#include "gate_row.cuh"

namespace {

using namespace moe_gate;

constexpr int kMaxWarps = 8;


// One sub-warp of G = 2^g_log2 lanes per row; CPL vector chunks of VEC logits per lane.
template <typename TIn, int VEC, int CPL>
__global__ void __launch_bounds__(kMaxWarps * 32)
topk_softmax_kernel(const TIn* __restrict__ logits, int64_t T, int E, int k, int g_log2, int renormalize,
                    float* __restrict__ topk_weights, int32_t* __restrict__ topk_ids) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  constexpr int NV = CPL * VEC;
  const int G = 1 << g_log2;
  const int rows_per_warp = 32 >> g_log2;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane & (G - 1);
  const int sub = lane >> g_log2;

  moe::pdl_wait();
  moe::pdl_launch_dependents();
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp) * rows_per_warp;
  if (row0 >= T) return;  // uniform per warp

  // per-warp staging: ids, probabilities (rows_per_warp * k each), then one denominator per row
  const int stage = rows_per_warp * k;
  int32_t* s_id = reinterpret_cast<int32_t*>(smem_raw) + warp * (2 * stage + rows_per_warp);
  float* s_p = reinterpret_cast<float*>(s_id + stage);
  float* s_den = s_p + stage;

  const int64_t row = row0 + sub;
  const bool row_ok = row < T;
  const int n_chunks = E / VEC;
  const TIn* rp = logits + (row_ok ? row : row0) * static_cast<int64_t>(E);

  uint64_t key[NV];
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    const int chunk = g + c * G;
    if (row_ok && chunk < n_chunks) {
      float v[VEC];
      VecLoad<TIn, VEC>::run(rp + chunk * VEC, v);
#pragma unroll
      for (int i = 0; i < VEC; ++i) key[c * VEC + i] = make_key(v[i], chunk * VEC + i);
    } else {
#pragma unroll
      for (int i = 0; i < VEC; ++i) key[c * VEC + i] = 0ull;
    }
  }

  const bool renorm = (renormalize & kGateRenorm) != 0, sigmoid = (renormalize & kGateSigmoid) != 0;
  float m = 0.f, Z = 0.f, S = 0.f;
  for (int j = 0; j < k; ++j) {
    uint64_t best = 0ull;
#pragma unroll
    for (int i = 0; i < NV; ++i) best = key[i] > best ? key[i] : best;
    for (int off = G >> 1; off >= 1; off >>= 1) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
      best = o > best ? o : best;
    }
    const float xj = ordered_to_float(static_cast<uint32_t>(best >> 32));
    if (j == 0 && !sigmoid) {
      // the first winner is the row maximum; reduce Z = sum over the row of exp(x - m)
      m = xj;
      float z = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        if (key[i] != 0ull) z += expf(ordered_to_float(static_cast<uint32_t>(key[i] >> 32)) - m);
      }
      for (int off = G >> 1; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
      Z = z;
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) key[i] = (key[i] == best) ? 0ull : key[i];
    const float p = sigmoid ? 1.f / (1.f + expf(-xj)) : expf(xj - m);
    S += p;
    if (g == 0) {
      s_id[sub * k + j] = static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(best));
      s_p[sub * k + j] = p;
    }
  }
  if (g == 0) s_den[sub] = renorm ? S : (sigmoid ? 1.f : Z);
  __syncwarp();

  const int64_t rows_here = (T - row0) < rows_per_warp ? (T - row0) : rows_per_warp;
  const int n_out = static_cast<int>(rows_here) * k;
  float* wdst = topk_weights + row0 * k;
  int32_t* idst = topk_ids + row0 * k;
  for (int idx = lane; idx < n_out; idx += 32) {
    const int r = idx / k;
    const float den = s_den[r];
    wdst[idx] = den > 0.f ? s_p[idx] / den : 1.f / static_cast<float>(k);  // 0 only for sigmoid sums
    idst[idx] = s_id[idx];
  }
}

// ------------------------------------------------------------------------------------------
// One warp per row (E >= 16).  Lane l holds chunks l, l+32, ... of VEC logits.  bf16 logits fit
// a 32-bit key (ordered 16-bit value above, 0xFFFF - index below), so each round is a single
// warp-wide redux max; fp32 logits use the 64-bit key, reduced as its high word, then the low
// word among the lanes holding that high word.  Lane j keeps round j's key; after the rounds each
// of lanes 0..k-1 takes one exp, and a warp sum gives the renormalising denominator (the
// full-row denominator Z is reduced in round 0 only when not renormalising).
// ------------------------------------------------------------------------------------------
constexpr int kRowWarps = 4;


template <typename TIn, int VEC, int CPL>
__global__ void __launch_bounds__(kRowWarps * 32)
topk_row_warp_kernel(const TIn* __restrict__ logits, int64_t T, int E, int k, int g_log2_unused, int renormalize,
                     float* __restrict__ topk_weights, int32_t* __restrict__ topk_ids) {
  (void)g_log2_unused;
  const int lane = threadIdx.x & 31;
  moe::pdl_wait();  // the logits may come from the previous kernel (the router projection)
  moe::pdl_launch_dependents();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (row >= T) return;  // uniform per warp
  int my_e;
  float my_w;
  moe_gate::gate_row<TIn, VEC, CPL>(logits + row * static_cast<int64_t>(E), E, k, renormalize, lane, my_e, my_w);
  if (lane < k) {
    topk_weights[row * k + lane] = my_w;
    topk_ids[row * k + lane] = my_e;
  }
}

// ------------------------------------------------------------------------------------------
// G lanes per row (moe_gate::lane_gate_row): a CTA stages kLaneThreads / G consecutive rows in
// shared memory with coalesced 16-byte loads, then each group of G lanes gates one row and its
// first lane writes the K weights and ids.
// ------------------------------------------------------------------------------------------
constexpr int kLaneThreads = 128;

template <typename TIn, int K, int G>
__global__ void __launch_bounds__(kLaneThreads)
topk_lane_kernel(const TIn* __restrict__ logits, int64_t T, int cpr, int mode, float* __restrict__ topk_weights,
                 int32_t* __restrict__ topk_ids) {
  constexpr int kRows = kLaneThreads / G;
  extern __shared__ __align__(16) uint4 s_rows[];
  const int tid = threadIdx.x;
  const int stride = moe_gate::lane_tile_stride(cpr);
  moe::pdl_wait();  // the logits may come from the previous kernel (the router projection)
  moe::pdl_launch_dependents();
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kRows;
  const int rows = (T - row0) < kRows ? static_cast<int>(T - row0) : kRows;  // >= 1
  moe_gate::lane_tile_load(reinterpret_cast<const uint4*>(logits) + row0 * cpr, rows, cpr, stride, s_rows, tid,
                           kLaneThreads);
  __syncthreads();
  const int r = tid / G, g = tid % G;
  const int rr = r < rows ? r : rows - 1;  // every lane takes part in the group's shuffles
  float w[K];
  int ids[K];
  moe_gate::lane_gate_row<TIn, K, G>(s_rows + rr * stride, cpr, mode, g, w, ids);
  if (r < rows && g == 0) {
    const int64_t o = (row0 + r) * K;
#pragma unroll
    for (int q = 0; q < K; ++q) {
      topk_weights[o + q] = w[q];
      topk_ids[o + q] = ids[q];
    }
  }
}

using LaneKernel = void (*)(const void*, int64_t, int, int, float*, int32_t*);

template <typename TIn, int K>
LaneKernel lane_kernel_g(int G) {
  switch (G) {
    case 1: return reinterpret_cast<LaneKernel>(&topk_lane_kernel<TIn, K, 1>);
    case 2: return reinterpret_cast<LaneKernel>(&topk_lane_kernel<TIn, K, 2>);
    case 4: return reinterpret_cast<LaneKernel>(&topk_lane_kernel<TIn, K, 4>);
    case 8: return reinterpret_cast<LaneKernel>(&topk_lane_kernel<TIn, K, 8>);
    default: return nullptr;
  }
}

template <typename TIn>
LaneKernel lane_kernel_for(int k, int G) {
  switch (k) {
    case 1: return lane_kernel_g<TIn, 1>(G);
    case 2: return lane_kernel_g<TIn, 2>(G);
    case 3: return lane_kernel_g<TIn, 3>(G);
    case 4: return lane_kernel_g<TIn, 4>(G);
    case 5: return lane_kernel_g<TIn, 5>(G);
    case 6: return lane_kernel_g<TIn, 6>(G);
    case 7: return lane_kernel_g<TIn, 7>(G);
    case 8: return lane_kernel_g<TIn, 8>(G);
    default: return nullptr;
  }
}

using TopkKernel = void (*)(const void*, int64_t, int, int, int, int, float*, int32_t*);

// Launch a gating kernel (any instance, arguments as a void* array) with programmatic stream
// serialisation.
cudaError_t launch_topk(TopkKernel kern, int64_t grid, int block, size_t smem, cudaStream_t st, void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(kern), args);
}

template <typename TIn, int VEC, int CPL>
TopkKernel instance() {
  if constexpr (VEC * CPL <= 32) {
    return reinterpret_cast<TopkKernel>(&topk_softmax_kernel<TIn, VEC, CPL>);
  } else {
    return nullptr;
  }
}

template <typename TIn, int VEC>
TopkKernel pick_cpl(int cpl) {
  switch (cpl) {
    case 1: return instance<TIn, VEC, 1>();
    case 2: return instance<TIn, VEC, 2>();
    case 4: return instance<TIn, VEC, 4>();
    case 8: return instance<TIn, VEC, 8>();
    case 16: return instance<TIn, VEC, 16>();
    case 32: return instance<TIn, VEC, 32>();
    default: return nullptr;
  }
}

template <typename TIn, int VEC, int CPL>
TopkKernel row_instance() {
  if constexpr (VEC * CPL <= 32) {
    return reinterpret_cast<TopkKernel>(&topk_row_warp_kernel<TIn, VEC, CPL>);
  } else {
    return nullptr;
  }
}

template <typename TIn, int VEC>
TopkKernel pick_row_cpl(int cpl) {
  switch (cpl) {
    case 1: return row_instance<TIn, VEC, 1>();
    case 2: return row_instance<TIn, VEC, 2>();
    case 4: return row_instance<TIn, VEC, 4>();
    case 8: return row_instance<TIn, VEC, 8>();
    case 16: return row_instance<TIn, VEC, 16>();
    case 32: return row_instance<TIn, VEC, 32>();
    default: return nullptr;
  }
}

template <typename TIn>
TopkKernel pick_row_kernel(int vec, int cpl) {
  if constexpr (sizeof(TIn) == 2) {
    switch (vec) {
      case 8: return pick_row_cpl<TIn, 8>(cpl);
      case 4: return pick_row_cpl<TIn, 4>(cpl);
      case 2: return pick_row_cpl<TIn, 2>(cpl);
      default: return pick_row_cpl<TIn, 1>(cpl);
    }
  } else {
    switch (vec) {
      case 4: return pick_row_cpl<TIn, 4>(cpl);
      case 2: return pick_row_cpl<TIn, 2>(cpl);
      default: return pick_row_cpl<TIn, 1>(cpl);
    }
  }
}

template <typename TIn>
TopkKernel pick_kernel(int vec, int cpl) {
  if constexpr (sizeof(TIn) == 2) {
    switch (vec) {
      case 8: return pick_cpl<TIn, 8>(cpl);
      case 4: return pick_cpl<TIn, 4>(cpl);
      case 2: return pick_cpl<TIn, 2>(cpl);
      default: return pick_cpl<TIn, 1>(cpl);
    }
  } else {
    switch (vec) {
      case 4: return pick_cpl<TIn, 4>(cpl);
      case 2: return pick_cpl<TIn, 2>(cpl);
      default: return pick_cpl<TIn, 1>(cpl);
    }
  }
}

// Launch geometry for one logits layout: vector width, lanes per row, chunks per lane.
struct TopkGeometry {
  int vec, g_log2, cpl, warps, smem;
};

TopkGeometry topk_geometry(int elem_bytes, const void* logits, int E, int k) {
  TopkGeometry geo{};
  int vec = 16 / elem_bytes;
  while (vec > 1 && ((E % vec) != 0 || (reinterpret_cast<uintptr_t>(logits) % (vec * elem_bytes)) != 0)) vec >>= 1;
  const int n_chunks = E / vec;
  int G = 1, g_log2 = 0;
  while (G < n_chunks && G < 32) { G <<= 1; ++g_log2; }
  int cpl = 1;
  while (cpl * G < n_chunks) cpl <<= 1;
  geo.vec = vec;
  geo.g_log2 = g_log2;
  geo.cpl = cpl;
  const int rows_per_warp = 32 >> g_log2;
  const int per_warp = (2 * rows_per_warp * k + rows_per_warp) * 4;
  int warps = kMaxWarps;
  while (warps > 1 && warps * per_warp > 48 * 1024) warps >>= 1;
  geo.warps = warps;
  geo.smem = warps * per_warp;
  return geo;
}

}  // namespace

extern "C" moe_status_t moe_topk_softmax(const void* logits, moe_dtype_t dtype, int64_t T, int32_t E, int32_t k,
                                         uint32_t flags, float* topk_weights, int32_t* topk_ids, void* stream) {
  if (T < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DTYPE_F32 && dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
  if ((flags & ~(MOE_RENORMALIZE | MOE_SCORING_SIGMOID)) != 0u) return MOE_ERR_INVALID_ARG;
  if (E > 1024 || k > 32) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (logits == nullptr || topk_weights == nullptr || topk_ids == nullptr) return MOE_ERR_INVALID_ARG;
  if (T > (int64_t{1} << 40)) return MOE_ERR_INVALID_ARG;

  const int elem = dtype == MOE_DTYPE_BF16 ? 2 : 4;
  // scoring mode bits of the kernels (moe_gate::kGateRenorm, moe_gate::kGateSigmoid)
  int renorm_flag = ((flags & MOE_RENORMALIZE) ? moe_gate::kGateRenorm : 0) |
                    ((flags & MOE_SCORING_SIGMOID) ? moe_gate::kGateSigmoid : 0);
  if (moe_gate::lane_gating_fits(T, E, k, elem, logits)) {
    // G lanes per row
    const int cpr = E * elem / 16;
    const int G = moe_gate::lane_gate_lanes(cpr);
    LaneKernel lk = dtype == MOE_DTYPE_BF16 ? lane_kernel_for<__nv_bfloat16>(k, G) : lane_kernel_for<float>(k, G);
    if (lk == nullptr) return MOE_ERR_UNSUPPORTED;
    const int64_t rows_per_cta = kLaneThreads / G;
    const int64_t grid = (T + rows_per_cta - 1) / rows_per_cta;
    if (grid > 0x7fffffff) return MOE_ERR_INVALID_ARG;
    const size_t smem = static_cast<size_t>(rows_per_cta) * moe_gate::lane_tile_stride(cpr) * sizeof(uint4);
    return moe_host::launch_pdl_max_shared(lk, dim3(static_cast<unsigned>(grid)), dim3(kLaneThreads), smem,
                                static_cast<cudaStream_t>(stream), logits, T, cpr, renorm_flag, topk_weights,
                                topk_ids);
  }
  if (E >= 16) {
    // one warp per row: the widest aligned vector that still spreads the row over all 32 lanes
    int vec_max = 16 / elem;
    while (vec_max > 1 && ((E % vec_max) != 0 || (reinterpret_cast<uintptr_t>(logits) % (vec_max * elem)) != 0))
      vec_max >>= 1;
    int vec = 1;
    for (int v = vec_max; v >= 1; v >>= 1) {
      if ((E % v) == 0 && E / v >= 32) { vec = v; break; }
    }
    const int n_chunks = E / vec;
    int cpl = 1;
    while (cpl * 32 < n_chunks) cpl <<= 1;
    TopkKernel rk = dtype == MOE_DTYPE_BF16 ? pick_row_kernel<__nv_bfloat16>(vec, cpl) : pick_row_kernel<float>(vec, cpl);
    if (rk == nullptr) return MOE_ERR_UNSUPPORTED;
    const int64_t grid = (T + kRowWarps - 1) / kRowWarps;
    if (grid > 0x7fffffff) return MOE_ERR_INVALID_ARG;
    int unused = 0;
    const void* logits_arg = logits;
    void* args[] = {&logits_arg, &T, &E, &k, &unused, &renorm_flag, &topk_weights, &topk_ids};
    return launch_topk(rk, grid, kRowWarps * 32, 0, static_cast<cudaStream_t>(stream), args) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
  }
  const TopkGeometry geo = topk_geometry(elem, logits, E, k);
  TopkKernel kern = dtype == MOE_DTYPE_BF16 ? pick_kernel<__nv_bfloat16>(geo.vec, geo.cpl)
                                            : pick_kernel<float>(geo.vec, geo.cpl);
  if (kern == nullptr) return MOE_ERR_UNSUPPORTED;
  const int64_t rows_per_cta = static_cast<int64_t>(geo.warps) * (32 >> geo.g_log2);
  const int64_t grid = (T + rows_per_cta - 1) / rows_per_cta;
  if (grid > 0x7fffffff) return MOE_ERR_INVALID_ARG;
  int g_log2 = geo.g_log2;
  const void* logits_arg = logits;
  void* args[] = {&logits_arg, &T, &E, &k, &g_log2, &renorm_flag, &topk_weights, &topk_ids};
  return launch_topk(kern, grid, geo.warps * 32, static_cast<size_t>(geo.smem), static_cast<cudaStream_t>(stream),
                     args) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
