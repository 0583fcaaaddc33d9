// Instantiations of the selective-scan kernel for bf16 activations: one sequence per row, (batch, dim, seqlen) layout.
// (One translation unit per dtype and kind, so the variants compile in parallel.)
#define SSM_ERROR_WORD g_error_scan_bf16
#include "scan_launch.cuh"
#include "scan_variants.h"

namespace ssm {

cudaError_t launch_scan_bf16(const ScanVariant& v, bool tma, bool sum, const ScanMaps& maps,
                             const ScanParams& p, dim3 grid, cudaStream_t st) {
#define X(NP_, S_, KC_, SW_, EXT_, M2_)                                                       \
    if (v.np == NP_ && v.s == S_ && v.kc == KC_ && v.sw == SW_)                            \
        return launch_v<__nv_bfloat16, NP_, S_, KC_, SW_, false, false>(tma, sum, maps, p, grid, st);
    SSM_SCAN_VARIANTS(X)
#undef X
    return cudaErrorInvalidValue;
}

cudaError_t take_error_scan_bf16(int* code, cudaStream_t st) {
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(code, g_error_scan_bf16, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbolAsync(g_error_scan_bf16, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                                   st);
}

}  // namespace ssm
