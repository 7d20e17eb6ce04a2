// route_internal.h -- library-internal entry points shared between the .cu files (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe_route.h"

namespace moe_internal {

// Workspace bytes of align_tiles for these sizes (a 256-byte header, per-tile expert counters,
// the expert totals).
size_t align_tiles_workspace_bytes(int64_t T, int32_t E_local);

// moe_align_permute through the fused dispatch's tile kernels: the given routes are counted and
// ranked per tile of tokens, the tile counts scanned per expert, and every slot placed.  The
// arguments are those of moe_align_permute, already validated by it; the workspace holds at least
// align_tiles_workspace_bytes and its first 4 bytes are the device status word.
moe_status_t align_tiles(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E_global, const int32_t* expert_map,
                         int32_t E_local, int32_t block_size, int32_t* counts, int32_t* offsets,
                         int32_t* sorted_token_ids, int32_t* expert_ids, int32_t* num_tokens_post_pad,
                         int32_t* inv_perm, void* workspace, cudaStream_t stream);

}  // namespace moe_internal
