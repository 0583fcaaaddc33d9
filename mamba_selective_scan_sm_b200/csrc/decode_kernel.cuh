// Single-token selective state update (decode) for sm_100a.
//
// The step applies the scan's math to one token and updates the conv and SSM
// states in place (pyshine.com "Mamba" tour, the block paragraph on `step`;
// paperlayer.ai summary of arXiv 2603.09555, §3 Method, "Autoregressive cache").
//
// The step is HBM-bound on the fp32 state (read + write of dim * dstate floats per
// batch row). Four lanes share a channel and each moves a 16-byte slice of its
// state row, so a warp reads/writes 8 contiguous 64-byte rows per access; the
// four partial C.h sums meet through two xor-shuffles. A and the per-channel
// parameters are reused by every batch row and stay in L2.
#pragma once

#include "device_common.cuh"
#include "scan_params.h"

namespace ssm {


// LPC lanes per channel, NPL states per lane (LPC * NPL >= dstate).
template <typename T, int LPC, int NPL>
__global__ void __launch_bounds__(256) decode_kernel(const DecodeParams p) {
    using E = Elem<T>;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = gid / LPC;                 // (b, d)
    const int j = (int)(gid % LPC);
    const bool valid = row < p.rows;
    const int64_t rr = valid ? row : 0;
    const int d = (int)(rr % p.dim);
    const int64_t b = rr / p.dim;
    const int N = p.dstate;

    // conv window (every lane of the channel computes it; lane 0 writes it back)
    const float xt = E::to_f(static_cast<const T*>(p.x)[rr]);
    float xc;
    if (p.conv_w) {
        const int W = p.conv_width;
        T* cs = static_cast<T*>(p.conv_state) + rr * W;
        float win[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) win[k] = (k + 1 < W) ? E::to_f(cs[k + 1]) : 0.f;
        // window after the shift: [cs[1..W-1], x]
        float acc = p.conv_b ? p.conv_b[d] : 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k < W - 1) acc = fmaf(p.conv_w[(int64_t)d * W + k], win[k], acc);
        }
        acc = fmaf(p.conv_w[(int64_t)d * W + (W - 1)], xt, acc);
        xc = silu(acc);
        __syncwarp();                    // every lane has read the window before lane 0 writes
        if (valid && j == 0) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < W - 1) cs[k] = E::from_f(win[k]);
            cs[W - 1] = E::from_f(xt);
        }
    } else {
        xc = xt;
    }
    float dl = E::to_f(static_cast<const T*>(p.dt)[rr]) + (p.dt_bias ? p.dt_bias[d] : 0.f);
    if (p.softplus) dl = softplus(dl);
    const float du = dl * xc;

    float* st = p.state + rr * N + j * NPL;
    const float* Ar = p.A + (int64_t)d * N + j * NPL;
    const T* Bb = static_cast<const T*>(p.Bt) + b * N + j * NPL;
    const T* Cb = static_cast<const T*>(p.Ct) + b * N + j * NPL;
    float part = 0.f;
    if (NPL == 4 && p.vec) {
        float4 h4 = valid ? __ldcs(reinterpret_cast<const float4*>(st)) : make_float4(0, 0, 0, 0);
        const float4 a4 = __ldg(reinterpret_cast<const float4*>(Ar));
        float hv[4] = {h4.x, h4.y, h4.z, h4.w};
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float dA = ex2(dl * av[k] * kLog2e);
            hv[k] = fmaf(dA, hv[k], du * E::load(Bb + k));
            part = fmaf(E::load(Cb + k), hv[k], part);
        }
        if (valid) __stcs(reinterpret_cast<float4*>(st), make_float4(hv[0], hv[1], hv[2], hv[3]));
    } else {
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
            const int n = j * NPL + k;
            if (n < N) {
                const float dA = ex2(dl * Ar[k] * kLog2e);
                const float hn = fmaf(dA, valid ? st[k] : 0.f, du * E::load(Bb + k));
                if (valid) st[k] = hn;
                part = fmaf(E::load(Cb + k), hn, part);
            }
        }
    }
#pragma unroll
    for (int m = LPC / 2; m >= 1; m >>= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
    if (valid && j == 0) {
        float y = part + (p.D ? p.D[d] * xc : 0.f);
        if (p.z) y *= silu(E::to_f(static_cast<const T*>(p.z)[rr]));
        static_cast<T*>(p.out)[rr] = E::from_f(y);
    }
}

}  // namespace ssm
