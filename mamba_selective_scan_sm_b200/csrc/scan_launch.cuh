// Host launchers of the scan kernel's instantiations, included by each scan unit
// (scan_{bf16,f32}.cu, scan_{bf16,f32}_ext.cu, scan_{bf16,f32}_m2.cu).
#pragma once

#include "scan_kernel.cuh"

namespace ssm {
namespace {

template <typename T, int NP, int S, int KC, int SW, bool TMA, bool SUM, bool VL, bool CL,
          int FEAT>
cudaError_t launch_one(const ScanMaps& maps, const ScanParams& p, dim3 grid, cudaStream_t st) {
    using Cfg = ScanCfg<T, NP, S, KC, SW, VL>;
    auto* k = scan_fwd_kernel<T, NP, S, KC, SW, TMA, SUM, VL, CL, FEAT>;
    static const cudaError_t attr =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (attr != cudaSuccess) return attr;
    k<<<grid, Cfg::NT, Cfg::SMEM, st>>>(maps, p);
    return cudaGetLastError();
}

// one scan pass of split (NP, S, KC, SW) for packed sequences VL / channel-last CL /
// features FEAT (bit 0: A per head, bit 1: time-invariant B/C)
template <typename T, int NP, int S, int KC, int SW, bool VL, bool CL, int FEAT = 0>
cudaError_t launch_v(bool tma, bool sum, const ScanMaps& maps, const ScanParams& p, dim3 grid,
                     cudaStream_t st) {
    if (tma) return sum ? launch_one<T, NP, S, KC, SW, true, true, VL, CL, FEAT>(maps, p, grid, st)
                        : launch_one<T, NP, S, KC, SW, true, false, VL, CL, FEAT>(maps, p, grid, st);
    return sum ? launch_one<T, NP, S, KC, SW, false, true, VL, CL, FEAT>(maps, p, grid, st)
               : launch_one<T, NP, S, KC, SW, false, false, VL, CL, FEAT>(maps, p, grid, st);
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

// A per head / time-invariant B/C (feat 1..3), either layout: splits marked M2 = 1; A per
// head only (feat 1): splits marked M2 = 2
template <typename T, int NP, int S, int KC, int SW, int M2>
cudaError_t launch_m2(bool tma, bool sum, bool cl, int feat, const ScanMaps& maps,
                      const ScanParams& p, dim3 grid, cudaStream_t st) {
    if constexpr (M2 == 2) {
        if (feat == 1)
            return cl ? launch_v<T, NP, S, KC, SW, false, true, 1>(tma, sum, maps, p, grid, st)
                      : launch_v<T, NP, S, KC, SW, false, false, 1>(tma, sum, maps, p, grid, st);
    } else if constexpr (M2 == 1) {
        switch (feat | (cl ? 4 : 0)) {
            case 1: return launch_v<T, NP, S, KC, SW, false, false, 1>(tma, sum, maps, p, grid, st);
            case 2: return launch_v<T, NP, S, KC, SW, false, false, 2>(tma, sum, maps, p, grid, st);
            case 3: return launch_v<T, NP, S, KC, SW, false, false, 3>(tma, sum, maps, p, grid, st);
            case 5: return launch_v<T, NP, S, KC, SW, false, true, 1>(tma, sum, maps, p, grid, st);
            case 6: return launch_v<T, NP, S, KC, SW, false, true, 2>(tma, sum, maps, p, grid, st);
            case 7: return launch_v<T, NP, S, KC, SW, false, true, 3>(tma, sum, maps, p, grid, st);
            default: break;
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace ssm
