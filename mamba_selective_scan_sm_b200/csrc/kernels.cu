// Device code of the library: the conv, decode and self-test kernels, the choice of
// scan variant and the dispatch to the scan units (scan_bf16.cu, scan_f32.cu; for
// packed sequences and channel-last activations scan_bf16_ext.cu, scan_f32_ext.cu; for
// A per head and time-invariant B/C scan_bf16_m2.cu, scan_f32_m2.cu), which hold the
// scan kernels' instantiations and compile in parallel with this one.
#define SSM_ERROR_WORD g_error_main
#include "conv_kernel.cuh"
#include "decode_kernel.cuh"
#include "launch.h"
#include "scan_kernel.cuh"
#include "scan_variants.h"

namespace ssm {

namespace {

template <typename T, int NP, int S, int KC, int SW>
ScanVariant variant_of() {
    using Cfg = ScanCfg<T, NP, S, KC, SW>;
    using CfgV = ScanCfg<T, NP, S, KC, SW, true>;
    return ScanVariant{(int)sizeof(T), NP, S, KC, SW, Cfg::G, Cfg::NT, Cfg::TT, Cfg::HALO, Cfg::SMEM,
                       Cfg::MIN_CTAS, CfgV::TT, CfgV::SMEM, CfgV::MIN_CTAS};
}

template <typename T, int W>
cudaError_t launch_stream(const DecodeParams& p, dim3 grid, cudaStream_t st) {
    constexpr int smem = kStreamStages * StreamTile<T, W>::BYTES;
    auto* k = decode_stream_kernel<T, W>;
    static const cudaError_t attr =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr != cudaSuccess) return attr;
    k<<<grid, kStreamThreads, smem, st>>>(p);
    return cudaGetLastError();
}

template <typename T, int LPC>
cudaError_t launch_wide_stream(const DecodeParams& p, cudaStream_t st) {
    constexpr int smem = kStreamStages * WideTile<T, LPC>::BYTES;
    auto* k = decode_wide_stream_kernel<T, LPC>;
    static int per_sm = 0;                            // resident CTAs per SM
    if (per_sm == 0) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, 256, smem);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
    }
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // one wave: every CTA resident at once, each a contiguous range of tiles
    const int64_t tiles = p.rows / WideTile<T, LPC>::R;
    const int64_t grid = tiles < (int64_t)sms * per_sm ? tiles : (int64_t)sms * per_sm;
    k<<<(unsigned)grid, 256, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool scan_variant(int es, int np, int s, int kc, int sw, ScanVariant* v) {
#define X(NP_, S_, KC_, SW_, EXT_, M2_)                                     \
    if (np == NP_ && s == S_ && kc == KC_ && sw == SW_) {                   \
        *v = es == 2 ? variant_of<__nv_bfloat16, NP_, S_, KC_, SW_>()       \
                     : variant_of<float, NP_, S_, KC_, SW_>();              \
        return es == 2 || es == 4;                                          \
    }
    SSM_SCAN_VARIANTS(X)
#undef X
    return false;
}

cudaError_t launch_scan(const ScanVariant& v, bool tma, bool sum, bool vl, bool cl, int feat,
                        const ScanMaps& maps, const ScanParams& p, dim3 grid, cudaStream_t st) {
    if (feat) {
        if (vl) return cudaErrorInvalidValue;
        return v.elem_size == 2 ? launch_scan_bf16_m2(v, tma, sum, cl, feat, maps, p, grid, st)
                                : launch_scan_f32_m2(v, tma, sum, cl, feat, maps, p, grid, st);
    }
    if (vl || cl)
        return v.elem_size == 2 ? launch_scan_bf16_ext(v, tma, sum, vl, cl, maps, p, grid, st)
                                : launch_scan_f32_ext(v, tma, sum, vl, cl, maps, p, grid, st);
    return v.elem_size == 2 ? launch_scan_bf16(v, tma, sum, maps, p, grid, st)
                            : launch_scan_f32(v, tma, sum, maps, p, grid, st);
}

cudaError_t launch_conv_tail(int es, const ConvTailParams& p, cudaStream_t st) {
    const int64_t blocks = (p.rows + 255) / 256;
    if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
    if (es == 2) conv_tail_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(p);
    else conv_tail_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_conv(int es, bool vec, const ConvParams& p, cudaStream_t st) {
    const int v = kConvChunks * 16 / es;                            // outputs per thread
    const int64_t per_row = (p.seqlen + v - 1) / v;
    const unsigned bx = (unsigned)((per_row + kConvThreads - 1) / kConvThreads);
    const unsigned by = (unsigned)(p.rows < 65535 ? p.rows : 65535);
    const int64_t bz = (p.rows + 65534) / 65535;
    if (bz > 65535) return cudaErrorInvalidConfiguration;
    const dim3 grid(bx, by, (unsigned)bz);
    void (*k)(const ConvParams) = es == 2 ? (vec ? conv1d_kernel<__nv_bfloat16, true>
                                                 : conv1d_kernel<__nv_bfloat16, false>)
                                          : (vec ? conv1d_kernel<float, true> : conv1d_kernel<float, false>);
    // a programmatic dependent launch: the grid may start launching while the previous
    // one in the stream drains; the kernel waits for that grid before it touches memory
    return launch_dependent(k, grid, dim3(kConvThreads), 0, st, p);
}

cudaError_t launch_decode(int es, int dstate, const DecodeParams& p, cudaStream_t st) {
    if (p.stream) {
        // about four CTAs per SM, each a contiguous range of batch rows
        const int64_t groups = p.dim / kStreamRows, batch = p.rows / p.dim;
        int64_t split = (148 * 4 + groups - 1) / groups;
        if (split > batch) split = batch;
        if (split < 1) split = 1;
        const dim3 grid((unsigned)groups, (unsigned)split);
        const int W = p.conv_w ? p.conv_width : 0;
#define SSM_STREAM_W(T_, W_) \
        if (W == W_) return launch_stream<T_, W_>(p, grid, st);
        if (es == 2) {
            SSM_STREAM_W(__nv_bfloat16, 0) SSM_STREAM_W(__nv_bfloat16, 2)
            SSM_STREAM_W(__nv_bfloat16, 3) SSM_STREAM_W(__nv_bfloat16, 4)
        } else {
            SSM_STREAM_W(float, 0) SSM_STREAM_W(float, 2) SSM_STREAM_W(float, 3)
            SSM_STREAM_W(float, 4)
        }
#undef SSM_STREAM_W
        return cudaErrorInvalidValue;
    }
    if (p.bulk) {
        const dim3 grid((unsigned)(p.dim / kDecRows), (unsigned)(p.rows / p.dim));
        if (es == 2) decode_bulk_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(p);
        else decode_bulk_kernel<float><<<grid, 256, 0, st>>>(p);
        return cudaGetLastError();
    }
    // 4 lanes x 4 states covers dstate <= 16; 32-bit thread indices
    const int64_t threads = p.rows * 4;
    const int64_t blocks = (threads + 255) / 256;
    if (threads + 256 > 0x7fffffff) return cudaErrorInvalidConfiguration;
    (void)dstate;
    if (es == 2) decode_kernel<__nv_bfloat16, 4, 4><<<(unsigned)blocks, 256, 0, st>>>(p);
    else decode_kernel<float, 4, 4><<<(unsigned)blocks, 256, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_decode_warp(int es, const DecodeParams& p, cudaStream_t st) {
    if (p.stream) {                                   // d_state 32, 64, 128 in channel groups
        const int lpc = p.dstate / 16;
#define SSM_WIDE_LPC(T_, L_) \
        if (lpc == L_) return launch_wide_stream<T_, L_>(p, st);
        if (es == 2) {
            SSM_WIDE_LPC(__nv_bfloat16, 2) SSM_WIDE_LPC(__nv_bfloat16, 4)
            SSM_WIDE_LPC(__nv_bfloat16, 8)
        } else {
            SSM_WIDE_LPC(float, 2) SSM_WIDE_LPC(float, 4) SSM_WIDE_LPC(float, 8)
        }
#undef SSM_WIDE_LPC
        return cudaErrorInvalidValue;
    }
    // lanes per row: 16 states per lane
    const int lpr = p.dstate <= 16 ? 1 : p.dstate <= 32 ? 2 : p.dstate <= 64 ? 4 : 8;
    const int per_block = 8 * (32 / lpr);                       // channels per 8-warp block
    const int64_t batch = p.rows / p.dim;
    const int64_t bz = (batch + 65534) / 65535;
    if (bz > 65535) return cudaErrorInvalidConfiguration;
    const dim3 grid((unsigned)((p.dim + per_block - 1) / per_block),
                    (unsigned)(batch < 65535 ? batch : 65535), (unsigned)bz);
#define SSM_WARP_LPR(T_, L_) \
    if (lpr == L_) { decode_warp_kernel<T_, L_><<<grid, 256, 0, st>>>(p); return cudaGetLastError(); }
    if (es == 2) {
        SSM_WARP_LPR(__nv_bfloat16, 1) SSM_WARP_LPR(__nv_bfloat16, 2)
        SSM_WARP_LPR(__nv_bfloat16, 4) SSM_WARP_LPR(__nv_bfloat16, 8)
    } else {
        SSM_WARP_LPR(float, 1) SSM_WARP_LPR(float, 2) SSM_WARP_LPR(float, 4)
        SSM_WARP_LPR(float, 8)
    }
#undef SSM_WARP_LPR
    return cudaErrorInvalidValue;
}

// One thread waits, bounded by limit_ns, on an mbarrier that nothing arrives at: the
// wait runs out, sets the device error word and the kernel returns (a self-test of the
// failure path every kernel's waits share).
__global__ void wait_selftest_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait_bounded(&bar, 0, limit_ns);
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st) {
    wait_selftest_kernel<<<1, 1, 0, st>>>(limit_ns);
    return cudaGetLastError();
}

cudaError_t take_error_main(int* code, cudaStream_t st) {
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(code, g_error_main, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbolAsync(g_error_main, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
}

cudaError_t read_device_error(int* code, cudaStream_t st) {
    int w[7] = {0, 0, 0, 0, 0, 0, 0};
    cudaError_t e = take_error_main(&w[0], st);
    if (e == cudaSuccess) e = take_error_scan_bf16(&w[1], st);
    if (e == cudaSuccess) e = take_error_scan_f32(&w[2], st);
    if (e == cudaSuccess) e = take_error_scan_bf16_ext(&w[3], st);
    if (e == cudaSuccess) e = take_error_scan_f32_ext(&w[4], st);
    if (e == cudaSuccess) e = take_error_scan_bf16_m2(&w[5], st);
    if (e == cudaSuccess) e = take_error_scan_f32_m2(&w[6], st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    *code = w[0] | w[1] | w[2] | w[3] | w[4] | w[5] | w[6];
    return e;
}

}  // namespace ssm
