// The compiled scan splits and the scan units' entry points.
#pragma once

#include "launch.h"

namespace ssm {

// (states per lane, lanes per channel, channels per lane, scan warps per CTA, EXT, M2):
// 2 lanes of 8 states (the default for wide batches), 4 lanes of 4, 8 lanes of 2 in
// CTAs of 8 or 12 channels (narrow batches);
// EXT splits also have packed-sequence and channel-last kernels; M2 = 1 splits also have
// kernels for A as one scalar per head and for time-invariant B/C, M2 = 2 splits for A
// per head only. 16 lanes of 4 or 8 states cover d_state 64 and 128; with A per head
// two channels per lane share each B/C load.
#define SSM_SCAN_VARIANTS(X) \
    X(4, 4, 1, 4, 1, 1)      \
    X(4, 4, 2, 2, 0, 0)      \
    X(2, 8, 1, 2, 1, 1)      \
    X(2, 8, 1, 3, 1, 1)      \
    X(8, 2, 1, 2, 1, 0)      \
    X(2, 8, 2, 4, 0, 0)      \
    X(2, 4, 1, 4, 1, 1)      \
    X(1, 4, 1, 4, 1, 1)      \
    X(4, 16, 1, 4, 1, 1)     \
    X(8, 16, 1, 4, 1, 1)     \
    X(4, 16, 2, 4, 0, 2)     \
    X(8, 16, 2, 4, 0, 2)     \
    X(8, 16, 2, 8, 0, 2)

// One scan pass with split `v`: one sequence per row in the (batch, dim, seqlen)
// layout (scan_bf16.cu / scan_f32.cu), packed sequences / channel-last
// (scan_bf16_ext.cu / scan_f32_ext.cu), or A per head / time-invariant B/C in either
// layout (scan_bf16_m2.cu / scan_f32_m2.cu).
#define SSM_SCAN_UNIT(SUF)                                                                  \
    cudaError_t launch_scan_##SUF(const ScanVariant& v, bool tma, bool sum, const ScanMaps& maps, \
                                  const ScanParams& p, dim3 grid, cudaStream_t stream);       \
    cudaError_t launch_scan_##SUF##_ext(const ScanVariant& v, bool tma, bool sum, bool packed,  \
                                        bool channel_last, const ScanMaps& maps,              \
                                        const ScanParams& p, dim3 grid, cudaStream_t stream); \
    cudaError_t launch_scan_##SUF##_m2(const ScanVariant& v, bool tma, bool sum,               \
                                       bool channel_last, int feat, const ScanMaps& maps,     \
                                       const ScanParams& p, dim3 grid, cudaStream_t stream);  \
    cudaError_t take_error_scan_##SUF(int* code, cudaStream_t stream);                         \
    cudaError_t take_error_scan_##SUF##_ext(int* code, cudaStream_t stream);                   \
    cudaError_t take_error_scan_##SUF##_m2(int* code, cudaStream_t stream);
SSM_SCAN_UNIT(bf16)
SSM_SCAN_UNIT(f32)
#undef SSM_SCAN_UNIT

}  // namespace ssm
