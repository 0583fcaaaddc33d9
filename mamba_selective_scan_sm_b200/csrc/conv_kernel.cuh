// Standalone causal depthwise conv1d (+ SiLU) for sm_100a.
//
// out[b,d,t] = act(bias[d] + sum_k w[d,k] * x[b,d,t-W+1+k]), x[t<0] = 0: output t
// only sees inputs at positions <= t (qwerky.ai, "What We Built"). The op streams
// one read and one write per element, so it is HBM-bound: each thread produces 8
// consecutive outputs from one aligned 16-byte (bf16) or 2 x 16-byte (fp32) vector
// plus the 3 preceding inputs, which the neighbouring thread also reads (L1 hit).
#pragma once

#include "device_common.cuh"
#include "scan_params.h"

namespace ssm {


template <typename T, bool VEC>
__global__ void __launch_bounds__(128) conv1d_kernel(const ConvParams p) {
    using E = Elem<T>;
    constexpr int V = 8;                                  // outputs per thread
    const int L = p.seqlen;
    // grid: x = chunks of 8 outputs along the row, y = row (b, d) in slabs of 65535
    const int t0 = (int)(blockIdx.x * blockDim.x + threadIdx.x) * V;
    const int64_t row = (int64_t)blockIdx.z * 65535 + blockIdx.y;
    if (t0 >= L || row >= p.rows) return;
    const int d = (int)((uint64_t)row % (uint32_t)p.dim);
    const T* xr = static_cast<const T*>(p.x) + row * L;
    T* yr = static_cast<T*>(p.out) + row * L;

    float w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {                          // right-aligned taps
        const int kk = k - (4 - p.width);
        w[k] = kk >= 0 ? p.w[(int64_t)d * p.width + kk] : 0.f;
    }
    const float bias = p.bias ? p.bias[d] : 0.f;

    float xv[V + 3];                                       // x[t0-3 .. t0+V-1]
    if (VEC && t0 + V <= L) {
        if constexpr (sizeof(T) == 2) {
            const uint4 cur = *reinterpret_cast<const uint4*>(xr + t0);
            const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&cur);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float2 f = __bfloat1622float2(c2[m]);
                xv[3 + 2 * m] = f.x;
                xv[4 + 2 * m] = f.y;
            }
        } else {
            const float4 a = *reinterpret_cast<const float4*>(xr + t0);
            const float4 bq = *reinterpret_cast<const float4*>(xr + t0 + 4);
            xv[3] = a.x; xv[4] = a.y; xv[5] = a.z; xv[6] = a.w;
            xv[7] = bq.x; xv[8] = bq.y; xv[9] = bq.z; xv[10] = bq.w;
        }
    } else {
#pragma unroll
        for (int m = 0; m < V; ++m) xv[3 + m] = (t0 + m < L) ? E::to_f(xr[t0 + m]) : 0.f;
    }
#pragma unroll
    for (int m = 0; m < 3; ++m) {
        const int t = t0 - 3 + m;
        xv[m] = t >= 0 ? E::to_f(xr[t]) : 0.f;
    }
    float y[V];
#pragma unroll
    for (int m = 0; m < V; ++m) {
        float acc = bias;
#pragma unroll
        for (int k = 0; k < 4; ++k) acc = fmaf(w[k], xv[m + k], acc);
        y[m] = p.silu ? silu(acc) : acc;
    }
    if (VEC && t0 + V <= L) {
        if constexpr (sizeof(T) == 2) {
            uint4 v;
            __nv_bfloat162* v2 = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
            for (int m = 0; m < 4; ++m) v2[m] = __floats2bfloat162_rn(y[2 * m], y[2 * m + 1]);
            *reinterpret_cast<uint4*>(yr + t0) = v;
        } else {
            *reinterpret_cast<float4*>(yr + t0) = make_float4(y[0], y[1], y[2], y[3]);
            *reinterpret_cast<float4*>(yr + t0 + 4) = make_float4(y[4], y[5], y[6], y[7]);
        }
    } else {
#pragma unroll
        for (int m = 0; m < V; ++m)
            if (t0 + m < L) yr[t0 + m] = E::from_f(y[m]);
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
    const T* x = static_cast<const T*>(p.x) + row * L;
    const T* h = p.hist ? static_cast<const T*>(p.hist) + row * (W - 1) : nullptr;
    T* o = static_cast<T*>(p.out) + idx * W;
    for (int k = 0; k < W; ++k) {
        const int t = hi - W + k;                      // position in the sequence axis
        o[k] = t >= lo ? x[t] : (h && t >= -(W - 1) ? h[W - 1 + t] : T(0.f));
    }
}

}  // namespace ssm
