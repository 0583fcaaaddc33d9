// Standalone causal depthwise conv1d (+ SiLU) for sm_100a.
//
// out[b,d,t] = act(bias[d] + sum_k w[d,k] * x[b,d,t-W+1+k]), x[t<0] = 0: output t
// only sees inputs at positions <= t (qwerky.ai, "What We Built"). The op streams
// one read and one write per element, so it is HBM-bound: each thread produces 32
// bytes of consecutive outputs from two aligned 16-byte loads plus the 16-byte chunk
// before them (for the 3 preceding inputs; the neighbouring thread's chunk, an L1
// hit), with the taps, the conv and the SiLU on packed fp32 pairs.
#pragma once

#include "device_common.cuh"
#include "scan_params.h"

namespace ssm {


template <typename T, bool VEC>
__global__ void __launch_bounds__(128) conv1d_kernel(const ConvParams p) {
    using E = Elem<T>;
    constexpr int EPC = 16 / (int)sizeof(T);              // elements per 16-byte chunk
    constexpr int V = 2 * EPC;                            // outputs per thread (32 bytes)
    const int L = p.seqlen;
    // grid: x = runs of V outputs along the row, y = row (b, d) in slabs of 65535
    const int t0 = (int)(blockIdx.x * blockDim.x + threadIdx.x) * V;
    const int64_t row = (int64_t)blockIdx.z * 65535 + blockIdx.y;
    if (t0 >= L || row >= p.rows) return;
    const int d = row < 0xffffffffll ? (int)((uint32_t)row % (uint32_t)p.dim)
                                     : (int)(row % p.dim);
    const T* xr = static_cast<const T*>(p.x) + row * L;
    T* yr = static_cast<T*>(p.out) + row * L;

    uint64_t w2[4];                                       // right-aligned taps, as pairs
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int kk = k - (4 - p.width);
        const float wk = kk >= 0 ? p.w[(int64_t)d * p.width + kk] : 0.f;
        w2[k] = pk2(wk, wk);
    }
    const float bias = p.bias ? p.bias[d] : 0.f;

    if (VEC && t0 + V <= L) {
        // x[t0 - EPC .. t0 + V): the chunk before (for the 3 previous inputs) and the
        // thread's two chunks; position t0 - 3 + m is window element EPC - 3 + m
        const uint4 win[3] = {t0 >= EPC ? *reinterpret_cast<const uint4*>(xr + t0 - EPC)
                                        : make_uint4(0, 0, 0, 0),
                              *reinterpret_cast<const uint4*>(xr + t0),
                              *reinterpret_cast<const uint4*>(xr + t0 + EPC)};
        uint32_t ob[V / 2];                               // bf16 pairs, or fp32 bits
        float of[V];
#pragma unroll
        for (int i = 0; i < V; i += 2) {                  // outputs t0 + i, t0 + i + 1
            uint64_t acc = pk2(bias, bias);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                acc = fma2(w2[k], pk2(chunk_elem<T>(win, EPC - 3 + i + k),
                                      chunk_elem<T>(win, EPC - 2 + i + k)), acc);
            // SiLU with one SFU op per output (the reciprocal on the FMA pipe): 2 Newton
            // steps leave 1.2e-5 relative error, far below a bf16 output's rounding;
            // fp32 outputs take 3 (1.5e-10)
            if (p.silu) acc = sizeof(T) == 2 ? silu2_fma<2>(acc) : silu2_fma<3>(acc);
            const float2 y = upk2(acc);
            if constexpr (sizeof(T) == 2) {
                __nv_bfloat162 t2 = __floats2bfloat162_rn(y.x, y.y);
                ob[i / 2] = *reinterpret_cast<uint32_t*>(&t2);
            } else {
                of[i] = y.x;
                of[i + 1] = y.y;
            }
        }
        if constexpr (sizeof(T) == 2) {
            *reinterpret_cast<uint4*>(yr + t0) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
            *reinterpret_cast<uint4*>(yr + t0 + EPC) = make_uint4(ob[4], ob[5], ob[6], ob[7]);
        } else {
            *reinterpret_cast<float4*>(yr + t0) = make_float4(of[0], of[1], of[2], of[3]);
            *reinterpret_cast<float4*>(yr + t0 + 4) = make_float4(of[4], of[5], of[6], of[7]);
        }
        return;
    }
    // ragged or unaligned rows: element by element
    float w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = lo2(w2[k]);
    for (int m = 0; m < V && t0 + m < L; ++m) {
        const int t = t0 + m;
        float acc = bias;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int s = t - 3 + k;
            if (s >= 0) acc = fmaf(w[k], E::to_f(xr[s]), acc);
        }
        yr[t] = E::from_f(p.silu ? silu(acc) : acc);
    }
}

// The conv state a scan leaves for the next call: per row, the last `width` inputs
// of history ++ x, oldest first, zeros before both (one thread per row; a few
// bytes per row). Packed sequences (batch 1): per (sequence, channel), the last
// `width` inputs of that sequence, zeros before its start.
template <typename T>
__global__ void __launch_bounds__(256) conv_tail_kernel(const ConvTailParams p) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int W = p.width, L = p.seqlen;
    int64_t row = idx;
    int lo = 0, hi = L;                                // the row's sequence [lo, hi)
    if (p.cu) {
        if (idx >= (int64_t)p.nseq * p.dim) return;
        const int s = (int)(idx / p.dim);
        row = idx % p.dim;
        hi = min(max(p.cu[s + 1], 0), L);             // offsets clamped into [0, L]
        lo = min(max(p.cu[s], 0), hi);
    } else if (idx >= p.rows) {
        return;
    }
    // position t of the row: x[row * L + t], or channel-last x[(b * L + t) * stride + d]
    const int64_t base = p.stride ? (row / p.dim) * L * p.stride + row % p.dim : row * L;
    const int64_t step = p.stride ? p.stride : 1;
    const T* x = static_cast<const T*>(p.x) + base;
    const T* h = p.hist ? static_cast<const T*>(p.hist) + row * (W - 1) : nullptr;
    T* o = static_cast<T*>(p.out) + idx * W;
    for (int k = 0; k < W; ++k) {
        const int t = hi - W + k;                      // position in the sequence axis
        o[k] = t >= lo ? x[t * step] : (h && t >= -(W - 1) ? h[W - 1 + t] : T(0.f));
    }
}

}  // namespace ssm
