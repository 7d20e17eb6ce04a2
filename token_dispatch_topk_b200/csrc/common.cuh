// common.cuh -- small device helpers shared by the routing kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "moe_route.h"

namespace moe {

// Record the first device-side error in a caller-provided status word (NULL = not collected).
__device__ __forceinline__ void record_status(int32_t* status, int32_t code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// 16-byte global accesses with cache-policy hints.
//   ld_stream: read-once data (evict-first in L1 and L2).
//   st_stream: write-once data.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream(uint4* p, const uint4& v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 ld_plain(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ void st_plain(uint4* p, const uint4& v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// bf16 <-> fp32.  Widening is exact (bf16 is the top half of a binary32).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Pack two fp32 into two bf16 (round-to-nearest-even), low element in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ---------------------------------------------------------------- TMA bulk copies + mbarriers --
// Non-tensor bulk copies (cp.async.bulk) between global and this CTA's shared memory, completed
// through an mbarrier (loads) or a bulk group (stores).  No cluster multicast anywhere.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0u;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for the phase with the given parity: false if it has not completed after about
// two seconds (every wait in this library completes in microseconds when the GPU is healthy).
// Between polls the warp sleeps (__nanosleep, 32 ns doubling to 256 ns) so that waiting warps
// take no issue slots from the warps doing the work.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  unsigned sleep_ns = 32;
  for (;;) {
    __nanosleep(sleep_ns);
    if (mbar_try_wait(bar, parity)) return true;
    if (sleep_ns < 256) sleep_ns <<= 1;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// Test hooks kept in words 2 and 3 of a dispatch workspace header (zero in normal use, which is what
// moe_workspace_init leaves): word 2 holds bits that withhold one event a bounded wait depends on, so
// that a test can make that wait run out and check the MOE_ERR_TIMEOUT it records; word 3 is the wait
// limit in microseconds (0: the default of about two seconds).
constexpr uint32_t kHookWithholdRowLoads = 1u;  // placement + gather: never issue the hidden-row loads
struct WaitHooks {
  uint32_t withhold;
  uint64_t limit_ns;
};
__device__ __forceinline__ WaitHooks read_hooks(const int32_t* ws_header) {
  const uint2 v = __ldcg(reinterpret_cast<const uint2*>(ws_header + 2));  // written by the host, not cached in L1
  WaitHooks h;
  h.withhold = v.x;
  h.limit_ns = v.y == 0u ? kWaitLimitNs : static_cast<uint64_t>(v.y) * 1000ull;
  return h;
}

// Named barrier over `nthreads` threads (a multiple of 32) of this CTA.
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Bulk copies of rows used once (hidden rows read by the gathers, expert-output rows read by the
// combine, gathered rows written for the expert GEMMs) may carry an L2 evict-first policy: those
// lines are the first to leave L2, ahead of lines that are still to be used.  The kernels ask for it
// when a row is at most kEvictFirstMaxRowBytes (one bulk copy per row).  Measured on one GPU in
// back-to-back steps: the 4096 x 128 prefill step (4 KB rows) takes 60.4 us with the policy on loads
// and stores, 63.3 with loads only, 63.2 with stores only, 63.5 without; the 16384 x 60 step (4 KB
// rows) 123.0 us with and without; the 65536 x 256 step (14 KB rows, which the combine copies in
// 4 KB pieces) 2672 us with and 2600 us without.
constexpr uint32_t kEvictFirstMaxRowBytes = 4096;

__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  return policy;
}

// global -> shared bulk copy; `bytes` and both addresses 16-byte aligned.
__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar,
                                          bool evict_first) {
  if (evict_first) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(evict_first_policy())
        : "memory");
  } else {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst_smem)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
  }
}

// shared -> global bulk copy, tracked by this thread's bulk groups.
__device__ __forceinline__ void bulk_store(void* dst, const void* src_smem, uint32_t bytes, bool evict_first) {
  if (evict_first) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(dst),
                 "r"(smem_addr(src_smem)), "r"(bytes), "l"(evict_first_policy())
                 : "memory");
  } else {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_addr(src_smem)),
                 "r"(bytes)
                 : "memory");
  }
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until this thread's bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(smem_addr(p)));
  return v;
}

// Packed fp32 pairs (sm_100 FFMA2): two independent IEEE fp32 fused multiply-adds.
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void f32x2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// acc + w * (bf16 pair in word u), element-wise in fp32, each a correctly rounded fma.
__device__ __forceinline__ uint64_t fma_bf16x2(uint64_t w2, uint32_t u, uint64_t acc) {
  const uint64_t y = f32x2(bf16_lo(u), bf16_hi(u));
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(w2), "l"(y), "l"(acc));
  return d;
}

__device__ __forceinline__ uint64_t lds64(const void* p) {
  uint64_t v;
  asm volatile("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(smem_addr(p)));
  return v;
}

// Programmatic dependent launch.  wait: block until the preceding kernel in the stream has
// completed and its writes are visible (returns at once when not launched as a dependent).
// launch_dependents: let the next kernel's CTAs be scheduled early (they wait in turn).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// Hold a value in a register from this point of the program on.  Kernel parameters are otherwise
// read from the constant bank where they are first used, and in a latency-bound kernel every first
// use of another parameter line is a constant-cache miss on the critical path; pinning them at
// entry issues those reads together, before the kernel waits for anything.
__device__ __forceinline__ int pin(int v) {
  asm volatile("" : "+r"(v));
  return v;
}
__device__ __forceinline__ int64_t pin(int64_t v) {
  asm volatile("" : "+l"(v));
  return v;
}
template <typename T>
__device__ __forceinline__ T* pin(T* p) {
  uint64_t u = reinterpret_cast<uint64_t>(p);
  asm volatile("" : "+l"(u));
  return reinterpret_cast<T*>(u);
}

// Store a 32-bit value into the same shared-memory variable of CTA `rank` of this cluster.
__device__ __forceinline__ void st_cluster_u32(const void* local_ptr, uint32_t rank, uint32_t v) {
  uint32_t raddr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(smem_addr(local_ptr)), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(raddr), "r"(v) : "memory");
}

// Store 16 bytes into the same shared-memory location of CTA `rank` of this cluster.
__device__ __forceinline__ void st_cluster_v4(const void* local_ptr, uint32_t rank, const uint4& v) {
  uint32_t raddr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(smem_addr(local_ptr)), "r"(rank));
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(raddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

}  // namespace moe

// Host-side helpers.
namespace moe_host {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Dynamic shared memory to request so that at most `per_sm` CTAs of a kernel fit on one SM:
// CTAs placed while other kernels still occupy SMs then spread evenly instead of piling onto the
// idle SMs (a streaming kernel is as fast as its most loaded SM).  Returns 0 on a CUDA error.
inline size_t smem_for_ctas_per_sm(size_t needed, int per_sm) {
  int dev = 0, smem_sm = 0, rsv = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
    return 0;
  // per_sm + 1 CTAs must not fit: (per_sm + 1) * (s + rsv) > smem_sm
  size_t s = static_cast<size_t>(smem_sm) / static_cast<size_t>(per_sm + 1) + 1;
  s = s > static_cast<size_t>(rsv) ? s - static_cast<size_t>(rsv) : 0;
  s = (s + 15) & ~size_t{15};
  return needed > s ? needed : s;
}

// Tokens per CTA for a one-pass kernel over T tokens with `slots` CTAs resident at a time and at
// most tpc_max tokens per CTA: the fewest full waves, each as evenly filled as possible.
inline int tokens_per_cta(int64_t T, int tpc_max, int64_t slots) {
  if (T <= 0 || slots <= 0) return tpc_max;
  const int64_t waves = (T + slots * tpc_max - 1) / (slots * tpc_max);
  const int64_t tpc = (T + slots * waves - 1) / (slots * waves);
  return tpc < 1 ? 1 : static_cast<int>(tpc);
}

inline int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return sms;
}

inline moe_status_t launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// The kernels of the large-batch chains (gating with the tile counts, tile scan, placement and
// gather, the TMA gather and combine, align) ask for the same split of each SM's L1 / shared
// memory: the most shared memory, which the staging kernels need.  An SM changes its split only
// when it is idle, so kernels with different splits chained by programmatic dependent launch would
// leave SMs unable to take the next kernel's CTAs until every CTA of the previous ones has left
// them.  The decode-sized kernels keep the default split, the one of the kernels around them.
inline cudaError_t prefer_max_shared(const void* kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                              static_cast<int>(cudaSharedmemCarveoutMaxShared));
}

// Launch with programmatic stream serialisation (the kernel may start while the previous kernel
// in the stream finishes; it calls moe::pdl_wait before reading that kernel's outputs).
template <typename... KArgs, typename... Args>
inline moe_status_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                               Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// launch_pdl for the kernels of the large-batch chains (the most shared memory, see above).
template <typename... KArgs, typename... Args>
inline moe_status_t launch_pdl_max_shared(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                          cudaStream_t st, Args&&... args) {
  if (prefer_max_shared(reinterpret_cast<const void*>(kernel)) != cudaSuccess) return MOE_ERR_CUDA;
  return launch_pdl(kernel, grid, block, smem, st, std::forward<Args>(args)...);
}

}  // namespace moe_host
