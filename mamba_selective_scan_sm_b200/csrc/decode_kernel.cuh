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
    // 32-bit index arithmetic: the host guarantees batch * dim * LPC < 2^31
    const uint32_t gid = blockIdx.x * blockDim.x + threadIdx.x;
    const uint32_t row = gid / LPC;                // (b, d)
    const int j = (int)(gid % LPC);
    const bool valid = row < (uint32_t)p.rows;
    const int64_t rr = valid ? row : 0;
    const uint32_t r32 = (uint32_t)rr;
    const int d = (int)(r32 % (uint32_t)p.dim);
    const int64_t b = r32 / (uint32_t)p.dim;
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

// Bulk-copy variant: one CTA updates kDecRows consecutive channels of one batch row.
// Thread 0 moves the rows' state, conv state, x, dt and z into shared memory with
// 1-D bulk async copies (a handful of instructions for ~10 KB in flight per CTA);
// then, in three phases separated by CTA barriers:
//   1. one thread per row does the row's scalar work once: conv window + SiLU,
//      delta = softplus(dt + bias), delta * x, D * x and silu(z);
//   2. four lanes per row update the row's states in place (4 states each) and
//      reduce C.h with two xor-shuffles;
//   3. one thread per row forms y and shifts the conv window;
// and thread 0 writes state, conv state and y back with bulk stores. Requires
// dim % kDecRows == 0 and 16-byte aligned bases (checked on the host).
constexpr int kDecRows = 64;

template <typename T>
__global__ void __launch_bounds__(256) decode_bulk_kernel(const DecodeParams p) {
    using E = Elem<T>;
    __shared__ __align__(128) float s_state[kDecRows * 16];
    __shared__ __align__(128) T s_conv[kDecRows * 4];
    __shared__ __align__(16) T s_x[kDecRows];
    __shared__ __align__(16) T s_dt[kDecRows];
    __shared__ __align__(16) T s_z[kDecRows];
    __shared__ __align__(16) T s_y[kDecRows];
    __shared__ __align__(16) float2 s_p[kDecRows];    // {delta, delta * xc}
    __shared__ __align__(16) float2 s_e[kDecRows];    // {D * xc, silu(z)}
    __shared__ float s_part[kDecRows];                 // sum_n C_n h_n
    __shared__ uint64_t bar;

    const int tid = threadIdx.x;
    // grid: x = 64-channel group within a batch row (dim % 64 == 0), y = batch index
    const int64_t b = blockIdx.y;
    const int dbase = blockIdx.x * kDecRows;
    const int64_t r0 = b * p.dim + dbase;
    const int N = p.dstate, W = p.conv_width;
    const bool conv = p.conv_w != nullptr, gate = p.z != nullptr;
    const uint32_t st_bytes = kDecRows * N * 4, cs_bytes = conv ? kDecRows * W * sizeof(T) : 0;
    const uint32_t v_bytes = kDecRows * sizeof(T);

    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar, st_bytes + cs_bytes + v_bytes * (gate ? 3 : 2));
        bulk_load(s_state, p.state + r0 * N, st_bytes, &bar);
        if (conv) bulk_load(s_conv, static_cast<const T*>(p.conv_state) + r0 * W, cs_bytes, &bar);
        bulk_load(s_x, static_cast<const T*>(p.x) + r0, v_bytes, &bar);
        bulk_load(s_dt, static_cast<const T*>(p.dt) + r0, v_bytes, &bar);
        if (gate) bulk_load(s_z, static_cast<const T*>(p.z) + r0, v_bytes, &bar);
    }

    // parameters while the copies fly (L2-resident, shared by every batch row)
    const bool row_thread = tid < kDecRows;          // phases 1 and 3: thread = row
    const int c1 = tid;                               // its row
    float w[4] = {0.f, 0.f, 0.f, 0.f}, cb = 0.f, dbias = 0.f, Dv = 0.f;
    if (row_thread) {
        const int d = dbase + c1;
        if (conv) {
            // taps right-aligned: w[3] meets the newest input
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int kk = k - (4 - W);
                if (kk >= 0) w[k] = __ldg(p.conv_w + (int64_t)d * W + kk);
            }
            cb = p.conv_b ? __ldg(p.conv_b + d) : 0.f;
        }
        dbias = p.dt_bias ? __ldg(p.dt_bias + d) : 0.f;
        Dv = p.D ? __ldg(p.D + d) : 0.f;
    }
    const int c = tid >> 2, j = tid & 3;              // phase 2: four lanes per row
    float a[4], bt[4], ct[4];
    {
        const int d = dbase + c;
        if (p.vec) {
            const float4 a4 = __ldg(reinterpret_cast<const float4*>(p.A + (int64_t)d * 16) + j);
            a[0] = a4.x * kLog2e; a[1] = a4.y * kLog2e; a[2] = a4.z * kLog2e; a[3] = a4.w * kLog2e;
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int n = j * 4 + k;
                a[k] = n < N ? __ldg(p.A + (int64_t)d * N + n) * kLog2e : 0.f;
            }
        }
        const T* bp = static_cast<const T*>(p.Bt) + b * N;
        const T* cp = static_cast<const T*>(p.Ct) + b * N;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int n = j * 4 + k;
            bt[k] = n < N ? E::load(bp + n) : 0.f;
            ct[k] = n < N ? E::load(cp + n) : 0.f;
        }
    }

    bool ok = true;
    if (tid == 0) ok = mbar_wait_bounded(&bar, 0);   // one thread polls, the barrier releases all
    if (__syncthreads_or(!ok)) {
        if (tid == 0) mbar_wait_bounded(&bar, 0);   // drain the copies still in flight
        return;
    }
    if (tid != 0) mbar_try_wait(&bar, 0);           // acquire the completed phase in every thread

    // phase 1: per-row scalars
    if (row_thread) {
        const float xt = E::to_f(s_x[c1]);
        float xc = xt;
        if (conv) {
            // window after the shift: [conv_state[1 .. W-1], x]; tap k reads
            // conv_state[kk + 1] for kk = k - (4 - W) < W - 1
            float acc = fmaf(w[3], xt, cb);
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                const int kk = k - (4 - W);
                if (kk >= 0) acc = fmaf(w[k], E::to_f(s_conv[c1 * W + kk + 1]), acc);
            }
            xc = silu(acc);
        }
        float dl = E::to_f(s_dt[c1]) + dbias;
        if (p.softplus) dl = softplus(dl);
        s_p[c1] = make_float2(dl, dl * xc);
        s_e[c1] = make_float2(Dv * xc, gate ? silu(E::to_f(s_z[c1])) : 1.f);
    }
    __syncthreads();

    // phase 2: state update, four lanes per row
    {
        const float2 pd = s_p[c];
        float part = 0.f;
        if (p.vec) {
            float4* hp = reinterpret_cast<float4*>(s_state + c * 16) + j;
            float4 h = *hp;
            h.x = fmaf(ex2(pd.x * a[0]), h.x, pd.y * bt[0]);
            h.y = fmaf(ex2(pd.x * a[1]), h.y, pd.y * bt[1]);
            h.z = fmaf(ex2(pd.x * a[2]), h.z, pd.y * bt[2]);
            h.w = fmaf(ex2(pd.x * a[3]), h.w, pd.y * bt[3]);
            *hp = h;
            part = fmaf(ct[0], h.x, fmaf(ct[1], h.y, fmaf(ct[2], h.z, ct[3] * h.w)));
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int n = j * 4 + k;
                if (n < N) {
                    float& hs = s_state[c * N + n];
                    const float h = fmaf(ex2(pd.x * a[k]), hs, pd.y * bt[k]);
                    hs = h;
                    part = fmaf(ct[k], h, part);
                }
            }
        }
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        if (j == 0) s_part[c] = part;
    }
    __syncthreads();

    // phase 3: output and conv window shift
    if (row_thread) {
        const float2 e = s_e[c1];
        s_y[c1] = E::from_f((s_part[c1] + e.x) * e.y);
        if (conv) {
            for (int k = 0; k < W - 1; ++k) s_conv[c1 * W + k] = s_conv[c1 * W + k + 1];
            s_conv[c1 * W + W - 1] = s_x[c1];
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        bulk_store(p.state + r0 * N, s_state, st_bytes);
        if (conv) bulk_store(static_cast<T*>(p.conv_state) + r0 * W, s_conv, cs_bytes);
        bulk_store(static_cast<T*>(p.out) + r0, s_y, v_bytes);
        bulk_commit();
        bulk_wait_read();
    }
}

}  // namespace ssm
