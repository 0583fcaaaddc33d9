// The compiled scan splits and the per-dtype scan units' entry points.
#pragma once

#include "launch.h"

namespace ssm {

// (states per lane, lanes per channel, channels per lane, scan warps per CTA)
#define SSM_SCAN_VARIANTS(X) \
    X(4, 4, 1, 4)            \
    X(4, 4, 2, 2)            \
    X(2, 8, 1, 2)            \
    X(2, 8, 2, 4)            \
    X(2, 4, 1, 4)            \
    X(1, 4, 1, 4)

// Launch one scan pass with the split `v` (scan_bf16.cu / scan_f32.cu).
cudaError_t launch_scan_bf16(const ScanVariant& v, bool tma, bool sum, bool packed,
                             const ScanMaps& maps, const ScanParams& p, dim3 grid,
                             cudaStream_t stream);
cudaError_t launch_scan_f32(const ScanVariant& v, bool tma, bool sum, bool packed,
                            const ScanMaps& maps, const ScanParams& p, dim3 grid,
                            cudaStream_t stream);

// Copy a unit's device error word into *code and clear it (asynchronous on `stream`).
cudaError_t take_error_scan_bf16(int* code, cudaStream_t stream);
cudaError_t take_error_scan_f32(int* code, cudaStream_t stream);

}  // namespace ssm
