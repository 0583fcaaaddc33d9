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

// Streaming variant (dstate 16): a CTA owns kStreamRows consecutive channels, one per
// thread, and walks a range of batch rows. Each thread keeps its channel's A (16
// values), conv taps, dt bias and D in registers for the whole range; each batch
// row's tile (the rows' fp32 state, conv state, x, dt, z, and the batch row's B_t and
// C_t) streams through a kStreamStages-deep ring of 1-D bulk copies, so several
// tiles are in flight per CTA while one is updated, and the updated state, conv
// state and y leave with bulk stores. A thread updates its row's 16 states as packed
// fp32 pairs; nothing is computed twice. One CTA barrier per tile. W is the conv
// width (0: no conv). Requires dim % kStreamRows == 0, dstate == 16 and 16-byte
// aligned bases (checked on the host).
constexpr int kStreamRows = 128;
constexpr int kStreamStages = 4;
constexpr int kStreamThreads = kStreamRows;

template <typename T, int W>
struct StreamTile {
    // byte offsets inside one stage (every part 16-byte aligned; bulk copies need it)
    static constexpr int ES = sizeof(T);
    static constexpr int STATE = 0;                                   // [rows][16] fp32
    static constexpr int CONV = STATE + kStreamRows * 16 * 4;         // [rows][W] T
    static constexpr int X = CONV + (kStreamRows * W * ES + 15) / 16 * 16;   // [rows] T
    static constexpr int DT = X + kStreamRows * ES;
    static constexpr int Z = DT + kStreamRows * ES;
    static constexpr int Y = Z + kStreamRows * ES;                    // output
    static constexpr int BT = Y + kStreamRows * ES;                   // [16] T
    static constexpr int CT = BT + 16 * ES;
    static constexpr int BYTES = (CT + 16 * ES + 127) / 128 * 128;
    static_assert(X % 16 == 0 && DT % 16 == 0 && Z % 16 == 0 && Y % 16 == 0 && BT % 16 == 0 &&
                  CT % 16 == 0, "bulk copies need 16-byte aligned parts");
};

// 4 values of T at an aligned shared address (8 or 16 bytes), widened to fp32
template <typename T>
__device__ __forceinline__ void load4(const uint8_t* src, float (&v)[4]) {
    if constexpr (sizeof(T) == 2) {
        const uint2 q = *reinterpret_cast<const uint2*>(src);
        v[0] = __uint_as_float(q.x << 16); v[1] = __uint_as_float(q.x & 0xffff0000u);
        v[2] = __uint_as_float(q.y << 16); v[3] = __uint_as_float(q.y & 0xffff0000u);
    } else {
        const float4 q = *reinterpret_cast<const float4*>(src);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
}

template <typename T, int W>
__global__ void __launch_bounds__(kStreamThreads, 4) decode_stream_kernel(const DecodeParams p) {
    using E = Elem<T>;
    using Tl = StreamTile<T, W>;
    constexpr bool CONV = W > 0;
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ uint64_t full[kStreamStages];

    const int tid = threadIdx.x, lane = tid & 31;
    const int dbase = blockIdx.x * kStreamRows;
    const int d = dbase + tid;                        // this thread's channel
    const int64_t nbatch = p.rows / p.dim;
    const int per = (int)((nbatch + gridDim.y - 1) / gridDim.y);
    const int64_t bfirst = (int64_t)blockIdx.y * per;
    const int ntiles = (int)max((int64_t)0, min((int64_t)per, nbatch - bfirst));
    if (ntiles == 0) return;                          // uniform over the CTA
    const bool gate = p.z != nullptr;
    const uint32_t cs_bytes = kStreamRows * W * sizeof(T);
    const uint32_t v_bytes = kStreamRows * sizeof(T);
    const uint32_t tile_bytes =
        kStreamRows * 64 + cs_bytes + v_bytes * (gate ? 3 : 2) + 2 * 16 * sizeof(T);

    auto stage = [&](int i) { return dsm + (i % kStreamStages) * Tl::BYTES; };
    auto issue = [&](int i) {                         // one thread: the loads of tile i
        uint8_t* s = stage(i);
        const int64_t b = bfirst + i;
        const int64_t r0 = b * p.dim + dbase;
        uint64_t* bar = &full[i % kStreamStages];
        mbar_arrive_expect_tx(bar, tile_bytes);
        bulk_load(s + Tl::STATE, p.state + r0 * 16, kStreamRows * 64, bar);
        if (CONV) bulk_load(s + Tl::CONV, static_cast<const T*>(p.conv_state) + r0 * W, cs_bytes, bar);
        bulk_load(s + Tl::X, static_cast<const T*>(p.x) + r0, v_bytes, bar);
        bulk_load(s + Tl::DT, static_cast<const T*>(p.dt) + r0, v_bytes, bar);
        if (gate) bulk_load(s + Tl::Z, static_cast<const T*>(p.z) + r0, v_bytes, bar);
        bulk_load(s + Tl::BT, static_cast<const T*>(p.Bt) + b * 16, 16 * sizeof(T), bar);
        bulk_load(s + Tl::CT, static_cast<const T*>(p.Ct) + b * 16, 16 * sizeof(T), bar);
    };

    int issued = 0;
    if (tid == 0) {
        for (int s = 0; s < kStreamStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
        for (; issued < min(kStreamStages, ntiles); ++issued) issue(issued);
    }

    // A thread walks its state row's four 16-byte chunks starting at chunk rot: the
    // eight lanes of a quarter-warp then touch eight different bank groups although
    // their rows are 64 bytes apart. A and B/C are read in the same rotated order.
    const int rot = (lane >> 1) & 3;
    // the channel's parameters, once for the whole range of batch rows
    uint64_t a2[8];                                   // A * log2(e), as pairs, rotated
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 a4 =
            __ldg(reinterpret_cast<const float4*>(p.A + (int64_t)d * 16) + ((q + rot) & 3));
        a2[2 * q] = pk2(a4.x * kLog2e, a4.y * kLog2e);
        a2[2 * q + 1] = pk2(a4.z * kLog2e, a4.w * kLog2e);
    }
    float w[W > 0 ? W : 1], cb = 0.f;
    if constexpr (CONV) {
#pragma unroll
        for (int k = 0; k < W; ++k) w[k] = __ldg(p.conv_w + (int64_t)d * W + k);
        cb = p.conv_b ? __ldg(p.conv_b + d) : 0.f;
    }
    const float dbias = p.dt_bias ? __ldg(p.dt_bias + d) : 0.f;
    const float Dv = p.D ? __ldg(p.D + d) : 0.f;

    // Tile i's data is complete when its barrier's phase (i / stages) & 1 completes.
    // Lane 0 of each warp polls (bounded), the CTA barrier shares the verdict, and
    // every thread then observes the phase itself (acquiring the copied bytes).
    auto wait_tile = [&](int i) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&full[i % kStreamStages], (i / kStreamStages) & 1);
        return ok;
    };
    auto drain = [&](int from) {                      // thread 0, on the way out
        if (tid != 0) return;
        for (int g = from; g < issued; ++g)
            mbar_wait_bounded(&full[g % kStreamStages], (g / kStreamStages) & 1);
        bulk_wait_read();
    };

    __syncthreads();                                  // barrier init before any wait
    if (__syncthreads_or(!wait_tile(0))) { drain(0); return; }
    for (int i = 0; i < ntiles; ++i) {
        uint8_t* s = stage(i);
        mbar_try_wait(&full[i % kStreamStages], (i / kStreamStages) & 1);
        const float xt = E::to_f(reinterpret_cast<const T*>(s + Tl::X)[tid]);
        float xc = xt;
        T* scv = reinterpret_cast<T*>(s + Tl::CONV) + tid * W;
        T win[W > 0 ? W : 1];
        if constexpr (CONV) {
            // window after the shift: [conv_state[1 .. W-1], x_t]; w[W-1] meets x_t
#pragma unroll
            for (int k = 0; k < W; ++k) win[k] = scv[k];
            float acc = fmaf(w[W - 1], xt, cb);
#pragma unroll
            for (int k = 0; k + 1 < W; ++k) acc = fmaf(w[k], E::to_f(win[k + 1]), acc);
            xc = silu(acc);
        }
        float dl = E::to_f(reinterpret_cast<const T*>(s + Tl::DT)[tid]) + dbias;
        if (p.softplus) dl = softplus(dl);
        const uint64_t dd = pk2(dl, dl), uu = pk2(dl * xc, dl * xc);
        float4* hp = reinterpret_cast<float4*>(s + Tl::STATE + tid * 64);
        uint64_t acc2 = pk2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int ch = (q + rot) & 3;             // state chunk: states 4ch .. 4ch+3
            float bv[4], cv[4];
            load4<T>(s + Tl::BT + ch * 4 * sizeof(T), bv);
            load4<T>(s + Tl::CT + ch * 4 * sizeof(T), cv);
            const float4 h4 = hp[ch];
            uint64_t h[2] = {pk2(h4.x, h4.y), pk2(h4.z, h4.w)};
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint64_t x = mul2(dd, a2[2 * q + k]);
                const uint64_t dA = pk2(ex2(lo2(x)), ex2(hi2(x)));
                h[k] = fma2(dA, h[k], mul2(uu, pk2(bv[2 * k], bv[2 * k + 1])));
                acc2 = fma2(pk2(cv[2 * k], cv[2 * k + 1]), h[k], acc2);
            }
            hp[ch] = make_float4(lo2(h[0]), hi2(h[0]), lo2(h[1]), hi2(h[1]));
        }
        float y = lo2(acc2) + hi2(acc2) + Dv * xc;
        if (gate) y *= silu(E::to_f(reinterpret_cast<const T*>(s + Tl::Z)[tid]));
        reinterpret_cast<T*>(s + Tl::Y)[tid] = E::from_f(y);
        if constexpr (CONV) {                         // shift the window, append x_t
#pragma unroll
            for (int k = 0; k + 1 < W; ++k) scv[k] = win[k + 1];
            scv[W - 1] = reinterpret_cast<const T*>(s + Tl::X)[tid];
        }
        fence_proxy_async_smem();                     // generic writes -> bulk-store reads
        const bool ok = i + 1 < ntiles ? wait_tile(i + 1) : true;
        if (__syncthreads_or(!ok)) { drain(i + 1); return; }
        if (tid == 0) {
            const int64_t r0 = (bfirst + i) * p.dim + dbase;
            bulk_store(p.state + r0 * 16, s + Tl::STATE, kStreamRows * 64);
            if (CONV) bulk_store(static_cast<T*>(p.conv_state) + r0 * W, s + Tl::CONV, cs_bytes);
            bulk_store(static_cast<T*>(p.out) + r0, s + Tl::Y, v_bytes);
            bulk_commit();
            // the stage of tile i - 1 is free once its stores have read it
            if (i >= 1 && issued < ntiles) {
                asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                issue(issued++);
            }
        }
    }
    if (tid == 0) bulk_wait_read();
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


// Decode step for d_state up to 128 and for A given per head. LPR lanes serve one (b, d)
// row, 16 states each (lane q of the row holds states 16q .. 16q + 15, four float4s), so
// a warp holds 32 / LPR rows (4 at d_state 128, 32 at d_state <= 16) and the per-row
// work (conv, softplus, gate, parameter loads) is shared by 16 states of every lane.
// With A per head the row's decay exp(delta * A_h) is one exp for all its states. Every
// lane takes part in the row's shuffle reduction, so no lane leaves early. Grid: x =
// groups of 8 * 32 / LPR channels, y (+ 65535 * z) = batch row: no index divisions.
template <typename T, int LPR>
__global__ void __launch_bounds__(256) decode_warp_kernel(const DecodeParams p) {
    using E = Elem<T>;
    constexpr int RPW = 32 / LPR;
    constexpr int NPL = 16;                                // states per lane
    const int lane = threadIdx.x & 31;
    const int dd = (blockIdx.x * 8 + (threadIdx.x >> 5)) * RPW + lane / LPR;
    const int64_t b0 = (int64_t)blockIdx.z * 65535 + blockIdx.y;
    const int q = lane % LPR;
    const bool live = dd < p.dim && b0 * p.dim < p.rows;
    const int d = live ? dd : 0;                           // dead lanes read row 0, store nothing
    const int64_t bb = live ? b0 : 0;
    const int64_t rr = bb * p.dim + d;
    const int N = p.dstate;
    const int n0 = NPL * q;
    // the state row first: its loads are the long ones and depend on nothing else (the
    // host rejects a conv state that overlaps the SSM state)
    float* st = p.state + rr * N;
    float h[NPL];
#pragma unroll
    for (int g = 0; g < NPL / 4; ++g) {
        const int n = n0 + 4 * g;
        if (p.vec && n + 3 < N) {                          // dstate % 4 == 0, aligned rows
            const float4 v = *reinterpret_cast<const float4*>(st + n);
            h[4 * g] = v.x; h[4 * g + 1] = v.y; h[4 * g + 2] = v.z; h[4 * g + 3] = v.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) h[4 * g + i] = n + i < N ? st[n + i] : 0.f;
        }
    }
    const T* Bt = static_cast<const T*>(p.Bt) + bb * N;
    const T* Ct = static_cast<const T*>(p.Ct) + bb * N;
    const float xt = E::to_f(static_cast<const T*>(p.x)[rr]);
    float dl = E::to_f(static_cast<const T*>(p.dt)[rr]) + (p.dt_bias ? p.dt_bias[d] : 0.f);
    float xc = xt;
    if (p.conv_w) {
        // the window after the shift: conv_state[1 .. W-1], then x_t (newest last)
        T* cs = static_cast<T*>(p.conv_state) + rr * p.conv_width;
        float win[4];
        float acc = p.conv_b ? p.conv_b[d] : 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k < p.conv_width) {
                win[k] = k < p.conv_width - 1 ? E::to_f(cs[k + 1]) : xt;
                acc = fmaf(p.conv_w[(int64_t)d * p.conv_width + k], win[k], acc);
            }
        }
        xc = silu(acc);
        __syncwarp();                                      // the row's lanes have read cs
        if (live && q == 0) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < p.conv_width) cs[k] = E::from_f(win[k]);   // exact: values of T
        }
    }
    if (p.softplus) dl = softplus(dl);
    const float du = dl * xc;
    const bool heads = p.head_dim != 0;
    const float dAh = heads ? ex2(dl * p.A[d / p.head_dim] * kLog2e) : 0.f;
    const float* Ar = p.A + (int64_t)d * N;
    float y = 0.f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int n = n0 + i;
        if (n < N) {
            const float dA = heads ? dAh : ex2(dl * Ar[n] * kLog2e);
            h[i] = fmaf(dA, h[i], du * E::to_f(Bt[n]));
            y = fmaf(E::to_f(Ct[n]), h[i], y);
        }
    }
    if (live) {
#pragma unroll
        for (int g = 0; g < NPL / 4; ++g) {
            const int n = n0 + 4 * g;
            if (p.vec && n + 3 < N) {
                *reinterpret_cast<float4*>(st + n) =
                    make_float4(h[4 * g], h[4 * g + 1], h[4 * g + 2], h[4 * g + 3]);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (n + i < N) st[n + i] = h[4 * g + i];
            }
        }
    }
#pragma unroll
    for (int m = LPR / 2; m >= 1; m >>= 1) y += __shfl_xor_sync(0xffffffffu, y, m);
    if (live && q == 0) {
        if (p.D) y = fmaf(p.D[d], xc, y);
        if (p.z) y *= silu(E::to_f(static_cast<const T*>(p.z)[rr]));
        static_cast<T*>(p.out)[rr] = E::from_f(y);
    }
}

// Streaming decode for d_state 32, 64 or 128 (LPC = d_state / 16 lanes per channel,
// 16 states per lane) with A per head or per (channel, state). A tile is one batch row's
// R = 256 / LPC consecutive channels: their fp32 state (R * d_state * 4 = 16 KB, one
// contiguous range), conv state, x, dt, z, and the batch row's B_t and C_t. Tiles stream
// through a kStreamStages-deep ring of 1-D bulk copies and leave with bulk stores, as in
// decode_stream_kernel; the grid is one wave of CTAs, each a contiguous range of the
// (channel group, batch row) tiles taken group-major, so the per-channel parameters stay
// in registers until the range crosses into the next group. Lane q of a channel holds,
// for g = 0..3, the four states n = 4 * (LPC * ch + q) .. + 3 of chunk ch = (g + c) & 3:
// the eight lanes of a quarter-warp then read 128 distinct bytes of shared memory. With
// A per head the decay exp(delta * A_h) is one exp per channel for all its states.
// Requires dim % R == 0, 16-byte aligned bases (checked on the host).
template <typename T, int LPC>
struct WideTile {
    static constexpr int ES = sizeof(T);
    static constexpr int R = 256 / LPC;                               // channels per tile
    static constexpr int N = 16 * LPC;                                // states per channel
    static constexpr int STATE = 0;                                   // [R][N] fp32
    static constexpr int CONV = STATE + R * N * 4;                    // [R][W] T, W <= 4
    static constexpr int X = CONV + R * 4 * ES;
    static constexpr int DT = X + R * ES;
    static constexpr int Z = DT + R * ES;
    static constexpr int Y = Z + R * ES;                              // output
    static constexpr int BT = Y + R * ES;                             // [N] T
    static constexpr int CT = BT + N * ES;
    static constexpr int BYTES = (CT + N * ES + 127) / 128 * 128;
    static_assert(CONV % 16 == 0 && X % 16 == 0 && DT % 16 == 0 && Z % 16 == 0 && Y % 16 == 0 &&
                  BT % 16 == 0 && CT % 16 == 0, "bulk copies need 16-byte aligned parts");
};

template <typename T, int LPC>
__global__ void __launch_bounds__(256, 3) decode_wide_stream_kernel(const DecodeParams p) {
    using E = Elem<T>;
    using Tl = WideTile<T, LPC>;
    constexpr int R = Tl::R, N = Tl::N, ES = Tl::ES;
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ uint64_t full[kStreamStages];

    const int tid = threadIdx.x, lane = tid & 31;
    const int c = tid / LPC, q = tid % LPC;           // channel within the tile, lane in it
    const int rot = c & 3;
    const int W = p.conv_w ? p.conv_width : 0;
    const bool gate = p.z != nullptr, heads = p.head_dim != 0;
    const int64_t batch = p.rows / p.dim;
    const int64_t ntot = batch * (p.dim / R);
    const int64_t tfirst = ntot * blockIdx.x / gridDim.x;
    const int ntiles = (int)(ntot * (blockIdx.x + 1) / gridDim.x - tfirst);
    if (ntiles == 0) return;                          // uniform over the CTA
    const int g0 = (int)(tfirst / batch);             // the range's first (group, batch row)
    const int64_t b0 = tfirst - (int64_t)g0 * batch;
    const uint32_t cs_bytes = R * W * ES, v_bytes = R * ES;
    const uint32_t tile_bytes = R * N * 4 + cs_bytes + v_bytes * (gate ? 3 : 2) + 2 * N * ES;

    auto stage = [&](int i) { return dsm + (i % kStreamStages) * Tl::BYTES; };
    int64_t ib = b0;                                  // the next tile to issue (thread 0)
    int ig = g0;
    auto issue = [&](int i) {
        uint8_t* s = stage(i);
        const int64_t r0 = ib * p.dim + (int64_t)ig * R;
        uint64_t* bar = &full[i % kStreamStages];
        mbar_arrive_expect_tx(bar, tile_bytes);
        bulk_load(s + Tl::STATE, p.state + r0 * N, R * N * 4, bar);
        if (W) bulk_load(s + Tl::CONV, static_cast<const T*>(p.conv_state) + r0 * W, cs_bytes, bar);
        bulk_load(s + Tl::X, static_cast<const T*>(p.x) + r0, v_bytes, bar);
        bulk_load(s + Tl::DT, static_cast<const T*>(p.dt) + r0, v_bytes, bar);
        if (gate) bulk_load(s + Tl::Z, static_cast<const T*>(p.z) + r0, v_bytes, bar);
        bulk_load(s + Tl::BT, static_cast<const T*>(p.Bt) + ib * N, N * ES, bar);
        bulk_load(s + Tl::CT, static_cast<const T*>(p.Ct) + ib * N, N * ES, bar);
        if (++ib == batch) { ib = 0; ++ig; }
    };

    int issued = 0;
    if (tid == 0) {
        for (int k = 0; k < kStreamStages; ++k) mbar_init(&full[k], 1);
        fence_mbar_init();
        for (; issued < min(kStreamStages, ntiles); ++issued) issue(issued);
    }

    // the channel's parameters, reloaded when the range enters the next channel group
    uint64_t a2[8];                                   // A * log2(e) as pairs, chunk-rotated
    float ah = 0.f, w4[4], cb = 0.f, dbias = 0.f, Dv = 0.f;
    auto load_params = [&](int grp) {
        const int d = grp * R + c;
        if (heads) {
            ah = __ldg(p.A + d / p.head_dim) * kLog2e;
        } else {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const int n0 = 4 * (LPC * ((g + rot) & 3) + q);
                const float4 a4 = __ldg(reinterpret_cast<const float4*>(p.A + (int64_t)d * N + n0));
                a2[2 * g] = pk2(a4.x * kLog2e, a4.y * kLog2e);
                a2[2 * g + 1] = pk2(a4.z * kLog2e, a4.w * kLog2e);
            }
        }
        // taps right-aligned: w4[3] meets the newest input
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int kk = k - (4 - W);
            w4[k] = kk >= 0 ? __ldg(p.conv_w + (int64_t)d * W + kk) : 0.f;
        }
        cb = W && p.conv_b ? __ldg(p.conv_b + d) : 0.f;
        dbias = p.dt_bias ? __ldg(p.dt_bias + d) : 0.f;
        Dv = p.D ? __ldg(p.D + d) : 0.f;
    };
    int grp = g0;
    load_params(grp);
    int64_t b = b0;

    auto wait_tile = [&](int i) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&full[i % kStreamStages], (i / kStreamStages) & 1);
        return ok;
    };
    auto drain = [&](int from) {                      // thread 0, on the way out
        if (tid != 0) return;
        for (int k = from; k < issued; ++k)
            mbar_wait_bounded(&full[k % kStreamStages], (k / kStreamStages) & 1);
        bulk_wait_read();
    };

    __syncthreads();                                  // barrier init before any wait
    if (__syncthreads_or(!wait_tile(0))) { drain(0); return; }
    for (int i = 0; i < ntiles; ++i) {
        uint8_t* s = stage(i);
        mbar_try_wait(&full[i % kStreamStages], (i / kStreamStages) & 1);
        const float xt = E::to_f(reinterpret_cast<const T*>(s + Tl::X)[c]);
        T* scv = reinterpret_cast<T*>(s + Tl::CONV) + c * W;
        float xc = xt;
        T win[3];                                     // conv_state[1 .. W-1], oldest first
        if (W) {
            float acc = fmaf(w4[3], xt, cb);
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                const int kk = k - (4 - W);           // window slot k + 1 - (4 - W) < W - 1
                win[k] = kk >= 0 ? scv[kk + 1] : E::from_f(0.f);
                if (kk >= 0) acc = fmaf(w4[k], E::to_f(win[k]), acc);
            }
            xc = silu(acc);
        }
        float dl = E::to_f(reinterpret_cast<const T*>(s + Tl::DT)[c]) + dbias;
        if (p.softplus) dl = softplus(dl);
        const uint64_t dd = pk2(dl, dl), uu = pk2(dl * xc, dl * xc);
        const float dAh = heads ? ex2(dl * ah) : 0.f;
        const uint64_t dA2h = pk2(dAh, dAh);
        float* hrow = reinterpret_cast<float*>(s + Tl::STATE) + c * N;
        uint64_t acc2 = pk2(0.f, 0.f);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int n0 = 4 * (LPC * ((g + rot) & 3) + q);
            float bv[4], cv[4];
            load4<T>(s + Tl::BT + n0 * ES, bv);
            load4<T>(s + Tl::CT + n0 * ES, cv);
            float4* hp = reinterpret_cast<float4*>(hrow + n0);
            const float4 h4 = *hp;
            uint64_t h[2] = {pk2(h4.x, h4.y), pk2(h4.z, h4.w)};
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                uint64_t dA = dA2h;
                if (!heads) {
                    const uint64_t x = mul2(dd, a2[2 * g + k]);
                    dA = pk2(ex2(lo2(x)), ex2(hi2(x)));
                }
                h[k] = fma2(dA, h[k], mul2(uu, pk2(bv[2 * k], bv[2 * k + 1])));
                acc2 = fma2(pk2(cv[2 * k], cv[2 * k + 1]), h[k], acc2);
            }
            *hp = make_float4(lo2(h[0]), hi2(h[0]), lo2(h[1]), hi2(h[1]));
        }
        float y = lo2(acc2) + hi2(acc2);
#pragma unroll
        for (int m = LPC / 2; m >= 1; m >>= 1) y += __shfl_xor_sync(0xffffffffu, y, m);
        __syncwarp();                                 // the channel's lanes have read its window
        if (q == 0) {
            y = fmaf(Dv, xc, y);
            if (gate) y *= silu(E::to_f(reinterpret_cast<const T*>(s + Tl::Z)[c]));
            reinterpret_cast<T*>(s + Tl::Y)[c] = E::from_f(y);
            if (W) {                                  // shift the window, append x_t
#pragma unroll
                for (int k = 0; k < 3; ++k)
                    if (k - (4 - W) >= 0) scv[k - (4 - W)] = win[k];
                scv[W - 1] = reinterpret_cast<const T*>(s + Tl::X)[c];
            }
        }
        fence_proxy_async_smem();                     // generic writes -> bulk-store reads
        const bool ok = i + 1 < ntiles ? wait_tile(i + 1) : true;
        if (__syncthreads_or(!ok)) { drain(i + 1); return; }
        if (tid == 0) {
            const int64_t r0 = b * p.dim + (int64_t)grp * R;
            bulk_store(p.state + r0 * N, s + Tl::STATE, R * N * 4);
            if (W) bulk_store(static_cast<T*>(p.conv_state) + r0 * W, s + Tl::CONV, cs_bytes);
            bulk_store(static_cast<T*>(p.out) + r0, s + Tl::Y, v_bytes);
            bulk_commit();
            // the stage of tile i - 1 is free once its stores have read it
            if (i >= 1 && issued < ntiles) {
                asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                issue(issued++);
            }
        }
        if (++b == batch && i + 1 < ntiles) {         // the next tile starts the next group
            b = 0;
            load_params(++grp);
        }
    }
    if (tid == 0) bulk_wait_read();
}

}  // namespace ssm
