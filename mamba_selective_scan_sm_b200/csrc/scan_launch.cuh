// Host launchers of the scan kernel's instantiations, included by each per-dtype scan
// unit (scan_bf16.cu, scan_f32.cu).
#pragma once

#include "scan_kernel.cuh"

namespace ssm {
namespace {

template <typename T, int NP, int S, int KC, int SW, bool TMA, bool SUM, bool VL>
cudaError_t launch_one(const ScanMaps& maps, const ScanParams& p, dim3 grid, cudaStream_t st) {
    using Cfg = ScanCfg<T, NP, S, KC, SW>;
    auto* k = scan_fwd_kernel<T, NP, S, KC, SW, TMA, SUM, VL>;
    static const cudaError_t attr =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (attr != cudaSuccess) return attr;
    k<<<grid, Cfg::NT, Cfg::SMEM, st>>>(maps, p);
    return cudaGetLastError();
}

template <typename T, int NP, int S, int KC, int SW, bool VL>
cudaError_t launch_v(bool tma, bool sum, const ScanMaps& maps, const ScanParams& p, dim3 grid,
                     cudaStream_t st) {
    if (tma) return sum ? launch_one<T, NP, S, KC, SW, true, true, VL>(maps, p, grid, st)
                        : launch_one<T, NP, S, KC, SW, true, false, VL>(maps, p, grid, st);
    return sum ? launch_one<T, NP, S, KC, SW, false, true, VL>(maps, p, grid, st)
               : launch_one<T, NP, S, KC, SW, false, false, VL>(maps, p, grid, st);
}

template <typename T, int NP, int S, int KC, int SW>
cudaError_t launch_t(bool tma, bool sum, bool vl, const ScanMaps& maps, const ScanParams& p,
                     dim3 grid, cudaStream_t st) {
    return vl ? launch_v<T, NP, S, KC, SW, true>(tma, sum, maps, p, grid, st)
              : launch_v<T, NP, S, KC, SW, false>(tma, sum, maps, p, grid, st);
}

}  // namespace
}  // namespace ssm
