// Host-side launchers of the device kernels (defined in kernels.cu).
#pragma once

#include <cuda_runtime.h>

#include "scan_params.h"

namespace ssm {

// Static shape of one scan-kernel variant.
struct ScanVariant {
    int elem_size;      // 2 (bf16) or 4 (fp32)
    int np;             // states per lane
    int s;              // lanes per channel
    int kc;             // channels per lane
    int sw;             // scan warps per CTA
    int channels;       // channels per CTA
    int threads;        // threads per CTA
    int tile;           // time steps per tile (64 bytes of elements)
    int halo;           // conv history elements fetched with a tile
    int smem_bytes;     // dynamic shared memory per CTA
    int min_ctas;       // CTAs per SM the launch bounds are sized for
    int tile_vl;        // the same three for the packed-sequence kernels
    int smem_bytes_vl;
    int min_ctas_vl;
};

// Returns false if (elem_size, np, s, kc, sw) has no compiled kernel.
bool scan_variant(int elem_size, int np, int s, int kc, int sw, ScanVariant* v);

// feat: bit 0 A as one scalar per head, bit 1 time-invariant B/C (not with packed)
cudaError_t launch_scan(const ScanVariant& v, bool use_tma, bool summary, bool packed,
                        bool channel_last, int feat, const ScanMaps& maps, const ScanParams& p,
                        dim3 grid, cudaStream_t stream);

cudaError_t launch_conv(int elem_size, bool vec, const ConvParams& p, cudaStream_t stream);

cudaError_t launch_conv_tail(int elem_size, const ConvTailParams& p, cudaStream_t stream);

cudaError_t launch_decode(int elem_size, int dstate, const DecodeParams& p, cudaStream_t stream);

// Decode step for d_state up to 128 and A per head (p.head_dim), 16 states per lane.
cudaError_t launch_decode_warp(int elem_size, const DecodeParams& p, cudaStream_t stream);

// Replace the calling thread's ssm_last_error_detail() text.
void set_error_detail(const char* text);

// One bounded wait that runs out after limit_ns (self-test of the failure path).
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t stream);

// Read and clear the device error word (synchronises `stream`).
cudaError_t read_device_error(int* code, cudaStream_t stream);

}  // namespace ssm
