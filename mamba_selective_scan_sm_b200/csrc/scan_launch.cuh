// Host launchers of the scan kernel's instantiations, included by each scan unit
// (scan_bf16.cu, scan_f32.cu, scan_bf16_ext.cu, scan_f32_ext.cu).
#pragma once

#include "scan_kernel.cuh"

namespace ssm {
namespace {

template <typename T, int NP, int S, int KC, int SW, bool TMA, bool SUM, bool VL, bool CL>
cudaError_t launch_one(const ScanMaps& maps, const ScanParams& p, dim3 grid, cudaStream_t st) {
    using Cfg = ScanCfg<T, NP, S, KC, SW>;
    auto* k = scan_fwd_kernel<T, NP, S, KC, SW, TMA, SUM, VL, CL>;
    static const cudaError_t attr =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (attr != cudaSuccess) return attr;
    k<<<grid, Cfg::NT, Cfg::SMEM, st>>>(maps, p);
    return cudaGetLastError();
}

// one scan pass of split (NP, S, KC, SW) for packed sequences VL / channel-last CL
template <typename T, int NP, int S, int KC, int SW, bool VL, bool CL>
cudaError_t launch_v(bool tma, bool sum, const ScanMaps& maps, const ScanParams& p, dim3 grid,
                     cudaStream_t st) {
    if (tma) return sum ? launch_one<T, NP, S, KC, SW, true, true, VL, CL>(maps, p, grid, st)
                        : launch_one<T, NP, S, KC, SW, true, false, VL, CL>(maps, p, grid, st);
    return sum ? launch_one<T, NP, S, KC, SW, false, true, VL, CL>(maps, p, grid, st)
               : launch_one<T, NP, S, KC, SW, false, false, VL, CL>(maps, p, grid, st);
}

// the packed-sequence and channel-last kernels exist only for splits marked EXT
template <typename T, int NP, int S, int KC, int SW, bool EXT>
cudaError_t launch_ext(bool tma, bool sum, bool vl, bool cl, const ScanMaps& maps,
                       const ScanParams& p, dim3 grid, cudaStream_t st) {
    if constexpr (EXT) {
        if (vl && cl) return launch_v<T, NP, S, KC, SW, true, true>(tma, sum, maps, p, grid, st);
        if (vl) return launch_v<T, NP, S, KC, SW, true, false>(tma, sum, maps, p, grid, st);
        if (cl) return launch_v<T, NP, S, KC, SW, false, true>(tma, sum, maps, p, grid, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace ssm
