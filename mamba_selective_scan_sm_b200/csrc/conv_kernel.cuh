// Standalone causal depthwise conv1d (+ SiLU) for sm_100a.
//
// out[b,d,t] = act(bias[d] + sum_k w[d,k] * x[b,d,t-W+1+k]), x[t<0] = 0: output t
// only sees inputs at positions <= t (qwerky.ai, "What We Built"). The op streams
// one read and one write per element, so it is HBM-bound: each thread produces 32
// bytes of consecutive outputs from two aligned 16-byte loads plus the 16-byte chunk
// before them (for the 3 preceding inputs; the neighbouring thread's chunk, an L1
// hit), with the taps as scalar FMAs and the SiLU on packed fp32 pairs.
#pragma once

#include "device_common.cuh"
#include "scan_params.h"

namespace ssm {


constexpr int kConvChunks = 2;                            // 16-byte output chunks per thread
constexpr int kConvThreads = 256 / kConvChunks;

template <typename T, bool VEC>
__global__ void __launch_bounds__(kConvThreads) conv1d_kernel(const ConvParams p) {
    using E = Elem<T>;
    constexpr int CH = kConvChunks;
    constexpr int EPC = 16 / (int)sizeof(T);              // elements per 16-byte chunk
    constexpr int V = CH * EPC;                           // outputs per thread
    grid_dependency_sync();                               // launched as a dependent
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
        uint4 win[CH + 1];
        win[0] = t0 >= EPC ? *reinterpret_cast<const uint4*>(xr + t0 - EPC) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int c = 0; c < CH; ++c) win[c + 1] = *reinterpret_cast<const uint4*>(xr + t0 + c * EPC);
        // the window widened once; the taps as scalar FMAs on it (a packed pair of
        // overlapping window elements would need register moves for every tap)
        float xf[(CH + 1) * EPC];
#pragma unroll
        for (int m = EPC - 3; m < (CH + 1) * EPC; ++m) xf[m] = chunk_elem<T>(win, m);
        float wk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) wk[k] = lo2(w2[k]);
        uint32_t ob[V / 2];                               // bf16 pairs, or fp32 bits
        float of[V];
#pragma unroll
        for (int i = 0; i < V; i += 2) {                  // outputs t0 + i, t0 + i + 1
            float a0 = bias, a1 = bias;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                a0 = fmaf(wk[k], xf[EPC - 3 + i + k], a0);
                a1 = fmaf(wk[k], xf[EPC - 2 + i + k], a1);
            }
            uint64_t acc = pk2(a0, a1);
            // SiLU with the exp and the reciprocal on the SFU: the kernel is issue-bound
            // before it is SFU-bound, and the FMA-pipe reciprocal (silu2_fma) takes
            // seven instructions per output against four
            if (p.silu) acc = silu2(acc);
            const float2 y = upk2(acc);
            if constexpr (sizeof(T) == 2) {
                __nv_bfloat162 t2 = __floats2bfloat162_rn(y.x, y.y);
                ob[i / 2] = *reinterpret_cast<uint32_t*>(&t2);
            } else {
                of[i] = y.x;
                of[i + 1] = y.y;
            }
        }
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            if constexpr (sizeof(T) == 2)
                *reinterpret_cast<uint4*>(yr + t0 + c * EPC) =
                    make_uint4(ob[4 * c], ob[4 * c + 1], ob[4 * c + 2], ob[4 * c + 3]);
            else
                *reinterpret_cast<float4*>(yr + t0 + c * EPC) =
                    make_float4(of[4 * c], of[4 * c + 1], of[4 * c + 2], of[4 * c + 3]);
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
