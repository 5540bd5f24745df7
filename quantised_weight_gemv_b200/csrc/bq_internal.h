// bq_internal.h -- host-side helpers shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "bq.h"

namespace bq {

// Upper bound on CTAs of one streamed launch (2 per SM on up to 256 SMs); it
// sizes the cross-CTA partial-sum area of the workspace.
constexpr int kMaxCtas = 512;
// Two partial slots of up to 64 rows x 8 columns fp32 per CTA.
constexpr size_t kPartialBytesPerCta = 2 * 512 * sizeof(float);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Number of SMs of the current device (cached per device).  -1 on error.
int device_sm_count();

// Build a 2-D or 3-D tiled tensor map (no multicast).  `promotion` widens each
// L2 fill the copies cause.  Returns false on error.
bool encode_tensor_map(CUtensorMap *map, CUtensorMapDataType dtype, int rank,
                       const void *base, const uint64_t *dims, const uint64_t *strides_bytes,
                       const uint32_t *box, CUtensorMapSwizzle swizzle,
                       CUtensorMapL2promotion promotion);

// Launch `kernel` with the programmatic-dependent-launch attribute, as
// clusters of `cluster` CTAs along x when cluster > 1 (grid.x a multiple).
cudaError_t launch_pdl(const void *kernel, dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, void **args, int cluster = 1);

// Validation of a plane-layout matrix whose planes are device pointers.
int32_t check_qmat(const bq_qmat *W);

}  // namespace bq
