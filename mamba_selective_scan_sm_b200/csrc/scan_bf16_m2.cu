// Instantiations of the selective-scan kernel for bf16 activations: A as one scalar per head
// and / or time-invariant B/C, in the (batch, dim, seqlen) and channel-last layouts.
// (One translation unit per dtype and kind, so the variants compile in parallel.)
#define SSM_ERROR_WORD g_error_scan_bf16_m2
#include "scan_launch.cuh"
#include "scan_variants.h"

namespace ssm {

cudaError_t launch_scan_bf16_m2(const ScanVariant& v, bool tma, bool sum, bool cl, int feat,
                             const ScanMaps& maps, const ScanParams& p, dim3 grid,
                             cudaStream_t st) {
#define X(NP_, S_, KC_, SW_, EXT_, M2_)                                                     \
    if (v.np == NP_ && v.s == S_ && v.kc == KC_ && v.sw == SW_)                            \
        return launch_m2<__nv_bfloat16, NP_, S_, KC_, SW_, M2_>(tma, sum, cl, feat, maps, p, grid, st);
    SSM_SCAN_VARIANTS(X)
#undef X
    return cudaErrorInvalidValue;
}

cudaError_t take_error_scan_bf16_m2(int* code, cudaStream_t st) {
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(code, g_error_scan_bf16_m2, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbolAsync(g_error_scan_bf16_m2, &zero, sizeof(int), 0,
                                   cudaMemcpyHostToDevice, st);
}

}  // namespace ssm
