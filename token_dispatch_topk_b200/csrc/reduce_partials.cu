// reduce_partials.cu -- the exchange after an expert-parallel combine: the sum of the ranks'
// partial combines.
//
// Operation: under expert parallelism each rank keeps only the slots of its own experts
// ("b70-optimization-lab: 2026-07-16 MTP1 M=2 compact scheduler closure note", scheduler paragraph:
// each rank derives its local expert rows from topk_ids plus expert_map), so its combine is a
// partial sum over its local slots; the layer output is the sum of the ranks' partials.  The note
// leaves that collective out.  Reading: widen the bf16 partials to fp32, add them in ascending rank
// order from +0, round once to bf16 (round-to-nearest-even).
//
// The partials may live on other GPUs: with a rank's combine writing each owner's token range into
// that owner's buffers (a peer pointer given to moe_combine as `out`), the owner sums the partials it
// received with this kernel (a reduce-scatter whose transfer is the combine's own stores).  Plain
// 16-byte loads, which also read peer memory over NVLink; no TMA, no multicast.
//
// Bandwidth-bound: one 16-byte vector of the output per thread and grid-stride step; the n loads of a
// vector are issued together before the adds.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace {

constexpr int kMaxPartials = 16;
constexpr int kReduceThreads = 256;
constexpr int kReduceCtasPerSm = 8;

struct ReduceArgs {
  const uint4* p[kMaxPartials];  // partials, rank order
  int n;
  int64_t nvec;  // 16-byte vectors of the output
  uint4* out;
};

__global__ void __launch_bounds__(kReduceThreads) reduce_partials_kernel(ReduceArgs a) {
  moe::pdl_wait();  // the partials come from earlier work (the combines)
  moe::pdl_launch_dependents();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kReduceThreads;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * kReduceThreads + threadIdx.x; v < a.nvec; v += stride) {
    uint4 x[kMaxPartials];
#pragma unroll
    for (int r = 0; r < kMaxPartials; ++r) {
      if (r < a.n) x[r] = moe::ld_plain(a.p[r] + v);
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < kMaxPartials; ++r) {
      if (r < a.n) {  // ascending rank order
        acc[0] = acc[0] + moe::bf16_lo(x[r].x);
        acc[1] = acc[1] + moe::bf16_hi(x[r].x);
        acc[2] = acc[2] + moe::bf16_lo(x[r].y);
        acc[3] = acc[3] + moe::bf16_hi(x[r].y);
        acc[4] = acc[4] + moe::bf16_lo(x[r].z);
        acc[5] = acc[5] + moe::bf16_hi(x[r].z);
        acc[6] = acc[6] + moe::bf16_lo(x[r].w);
        acc[7] = acc[7] + moe::bf16_hi(x[r].w);
      }
    }
    uint4 o;
    o.x = moe::pack_bf16x2(acc[0], acc[1]);
    o.y = moe::pack_bf16x2(acc[2], acc[3]);
    o.z = moe::pack_bf16x2(acc[4], acc[5]);
    o.w = moe::pack_bf16x2(acc[6], acc[7]);
    moe::st_plain(a.out + v, o);
  }
}

}  // namespace

extern "C" moe_status_t moe_reduce_partials(const void* const* partials, int32_t n_partials, int64_t rows, int32_t H,
                                            void* out, void* stream) {
  if (n_partials < 1 || rows < 0 || H < 1 || (H % 8) != 0) return MOE_ERR_INVALID_ARG;
  if (n_partials > kMaxPartials) return MOE_ERR_UNSUPPORTED;
  if (rows > (int64_t{1} << 40) || rows > (int64_t{1} << 44) / (H / 8)) return MOE_ERR_INVALID_ARG;  // H >= 8
  if (rows == 0) return MOE_OK;
  if (partials == nullptr || out == nullptr || !moe_host::aligned16(out)) return MOE_ERR_INVALID_ARG;
  ReduceArgs a{};
  for (int r = 0; r < n_partials; ++r) {
    if (partials[r] == nullptr || !moe_host::aligned16(partials[r])) return MOE_ERR_INVALID_ARG;
    a.p[r] = static_cast<const uint4*>(partials[r]);
  }
  a.n = n_partials;
  a.nvec = rows * (H / 8);
  a.out = static_cast<uint4*>(out);
  const int sms = moe_host::sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  int64_t grid = (a.nvec + kReduceThreads - 1) / kReduceThreads;
  const int64_t cap = static_cast<int64_t>(sms) * kReduceCtasPerSm;
  if (grid > cap) grid = cap;
  return moe_host::launch_pdl(reduce_partials_kernel, dim3(static_cast<unsigned>(grid)), dim3(kReduceThreads), 0,
                              static_cast<cudaStream_t>(stream), a);
}
