// Selective-scan forward kernel for sm_100a.
//
// Work split. A CTA of 128 threads owns G = 128/S channels of one batch row and
// walks the sequence in tiles of TT = 32 time steps.
// The S lanes of a channel each keep NP = NS/S of the (padded) NS states in
// registers, so one channel's recurrence is spread over S lanes with no carry
// between them (A is diagonal: the states never interact).
//
// Per tile:
//   1. TMA brings the raw tiles (u or the pre-conv x with a 16-byte halo, dt, z,
//      B, C) into a 2-stage shared-memory ring; B and C are shared by the CTA's
//      channels (all channels of a batch row read the same B_t, C_t).
//   2. Prologue, once per (channel, t): conv + SiLU, delta = softplus(dt + bias),
//      delta*u, D*u and silu(z) -> fp32 staging buffers; B and C are transposed to
//      [t][n] fp32 so each lane reads its NP states with one vector load.
//   3. Scan: per (t, state) one ex2 on the SFU, then h = dA*h + delta*u*B and the
//      lane's partial C.h. Every 16 steps a butterfly transpose-reduce over the S
//      lanes leaves each lane owning 16/S consecutive outputs, which it gates and
//      stores with one vector store.
//
// Two-pass chunk carry (paperlayer.ai summary of arXiv 2603.09555, §3 Method,
// "Chunked recurrence"): with nchunks > 1, a SUMMARY launch scans every chunk but
// the last from a zero state and writes (prod dA, h_end) per state; the output
// launch starts chunk k from the carry H_k = P_{k-1} H_{k-1} + S_{k-1}.
#pragma once

#include <type_traits>

#include "device_common.cuh"
#include "scan_params.h"

namespace ssm {

// Steps whose state-independent operands are prepared together (a divisor of 16).
#ifndef SSM_SCAN_BATCH
#define SSM_SCAN_BATCH 2
#endif

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

template <typename T, int NP, int S, int KC>
struct ScanCfg {
    static constexpr int G = S == 4 ? 32 : 16;          // channels per CTA
    static constexpr int NT = G * S / KC;               // threads per CTA
    static constexpr int NS = NP * S;         // padded state count
    static constexpr int ES = sizeof(T);
    static constexpr int TT = 32;             // tile length (time steps)
    static constexpr int ROWB = TT * ES;      // bytes of one tile row: 64 (bf16) / 128 (fp32)
    static constexpr int SWZ = ROWB == 128 ? 7 : 3;   // TMA 128-B / 64-B swizzle mask
    static constexpr int HALO = 16 / ES;      // conv history, one 16-B TMA granule
    static constexpr int NSTAGE = 2;
    static constexpr int R = 16 / S;          // outputs owned per lane per 16-step block
    // raw stage (bytes from the 1024-aligned stage base)
    static constexpr int RAW_B = 0;                                   // [NS][TT], swizzled
    static constexpr int RAW_C = align_up(NS * ROWB, 1024);           // [NS][TT], swizzled
    static constexpr int RAW_X = align_up(RAW_C + NS * ROWB, 128);    // [G][TT(+HALO)]
    static constexpr int X_PITCH_MAX = (TT + HALO) * ES;
    static constexpr int RAW_DT = align_up(RAW_X + G * X_PITCH_MAX, 128);
    static constexpr int RAW_Z = align_up(RAW_DT + G * ROWB, 128);
    static constexpr int STAGE = align_up(RAW_Z + G * ROWB, 1024);
    // fp32 staging. P: per channel group of KC channels and step, KC x {delta, delta*u}.
    static constexpr int P_PITCH = TT * KC * 8 + 16;
    static constexpr int E_PITCH = TT * 8 + 16;           // per channel: {D*u, silu(z)}
    static constexpr int OFF_P = NSTAGE * STAGE;
    static constexpr int OFF_E = OFF_P + (G / KC) * P_PITCH;
    // Transposed B, C: [t][n] in the input type (bf16 stays bf16: exact, and half the
    // shared-memory bytes each lane reads per step; fp32 stays fp32).
    static constexpr int BCS = ES;
    static constexpr int OFF_BT = align_up(OFF_E + G * E_PITCH, 16);
    static constexpr int OFF_CT = OFF_BT + TT * NS * BCS;
    static constexpr int OFF_PAR = align_up(OFF_CT + TT * NS * BCS, 16);  // 16 floats per channel
    static constexpr int OFF_BAR = align_up(OFF_PAR + G * 64, 8);
    static constexpr int BYTES = OFF_BAR + NSTAGE * 8;
    static constexpr int SMEM = BYTES + 1024;             // slack for 1024-B alignment
    static_assert(TT % 16 == 0, "tile must hold whole 16-step blocks");
    static_assert(P_PITCH % 16 == 0 && E_PITCH % 16 == 0, "staging rows take 16-byte stores");
    static_assert(G % 2 == 0, "the prologue pairs channel rows");
    static_assert(NS <= 16, "at most 16 states");
    static_assert(KC == 1 || KC == 2, "one or two channels per lane");
};

// Byte offset of logical (row, byte) in a swizzled [rows][ROWB] tile. TMA's 128-B
// and 64-B swizzles XOR address bits [4, 4+k) with bits [7, 7+k) (k = 3 or 2) of
// the offset from a 1024-byte aligned tile base; SWZ is the k-bit mask.
template <int ROWB, int SWZ>
__device__ __forceinline__ int swz(int row, int byte_in_row) {
    const int off = row * ROWB + byte_in_row;
    return off ^ (((off >> 7) & SWZ) << 4);
}

// Recurrence state of one lane: NP states, held as fp32 pairs so the four
// per-state operations (delta*A, delta*u*B, the h update and C.h) issue as packed
// .f32x2 instructions.
template <int NP, bool SUMMARY>
struct LaneState {
    static constexpr int NPR = NP / 2;                   // packed pairs
    static constexpr bool ODD = (NP % 2) != 0;
    uint64_t h2[NPR > 0 ? NPR : 1], a2[NPR > 0 ? NPR : 1], pr2[NPR > 0 ? NPR : 1];
    float h1, a1, pr1;                                   // the unpaired state (NP odd)

    __device__ __forceinline__ void set_a(const float* a) {
#pragma unroll
        for (int k = 0; k < NPR; ++k) a2[k] = pk2(a[2 * k], a[2 * k + 1]);
        if (ODD) a1 = a[NP - 1];
    }
    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int k = 0; k < NPR; ++k) { h2[k] = pk2(0.f, 0.f); pr2[k] = pk2(1.f, 1.f); }
        h1 = 0.f;
        pr1 = 1.f;
    }
    __device__ __forceinline__ float get(int k) const {       // k is a compile-time index
        if (ODD && k == NP - 1) return h1;
        return (k & 1) ? hi2(h2[k >> 1]) : lo2(h2[k >> 1]);
    }
    __device__ __forceinline__ float get_pr(int k) const {
        if (ODD && k == NP - 1) return pr1;
        return (k & 1) ? hi2(pr2[k >> 1]) : lo2(pr2[k >> 1]);
    }
    __device__ __forceinline__ void set(const float* v) {
#pragma unroll
        for (int k = 0; k < NPR; ++k) h2[k] = pk2(v[2 * k], v[2 * k + 1]);
        if (ODD) h1 = v[NP - 1];
    }

    // Operands of one time step that do not depend on the state: the decay factors
    // exp2(delta*a2), delta*u*B and C. Computing them one step ahead of the state
    // update (software pipelining) overlaps the shared-memory loads and the SFU
    // latency with the previous step's dependent FMAs.
    struct In {
        uint64_t dA[NPR > 0 ? NPR : 1], bu[NPR > 0 ? NPR : 1], cc[NPR > 0 ? NPR : 1];
        float dA1, bu1, c1;
    };

    // dl = delta, du = delta*u of the step; b / cvv: this lane's NP fp32 B and C values.
    __device__ __forceinline__ In prep(float dl, float du, const float* b, const float* cvv) const {
        In in;
        const uint64_t dd = pk2(dl, dl), uu = pk2(du, du);
#pragma unroll
        for (int k = 0; k < NPR; ++k) {
            const uint64_t x = mul2(dd, a2[k]);
            in.dA[k] = pk2(ex2(lo2(x)), ex2(hi2(x)));
            in.bu[k] = mul2(uu, pk2(b[2 * k], b[2 * k + 1]));
            if (!SUMMARY) in.cc[k] = pk2(cvv[2 * k], cvv[2 * k + 1]);
        }
        if (ODD) {
            in.dA1 = ex2(dl * a1);
            in.bu1 = du * b[NP - 1];
            if (!SUMMARY) in.c1 = cvv[NP - 1];
        }
        return in;
    }

    // h = dA * h + delta*u*B; returns sum_k C_k h_k (SUMMARY: accumulates prod dA).
    __device__ __forceinline__ float update(const In& in) {
        uint64_t s = pk2(0.f, 0.f);
        float s1 = 0.f;
#pragma unroll
        for (int k = 0; k < NPR; ++k) {
            h2[k] = fma2(in.dA[k], h2[k], in.bu[k]);
            if (SUMMARY) pr2[k] = mul2(pr2[k], in.dA[k]);
            else s = (k == 0) ? mul2(in.cc[k], h2[k]) : fma2(in.cc[k], h2[k], s);
        }
        if (ODD) {
            h1 = fmaf(in.dA1, h1, in.bu1);
            if (SUMMARY) pr1 *= in.dA1;
            else s1 = in.c1 * h1;
        }
        if (SUMMARY) return 0.f;
        return (NPR > 0 ? lo2(s) + hi2(s) : 0.f) + s1;
    }
};

// Four CTAs per SM at least: 128 registers per thread with 128-thread CTAs, up to
// 255 with the 64-thread CTAs of the two-channel variant (shared memory allows 5).
template <typename T, int NP, int S, int KC, bool USE_TMA, bool SUMMARY>
__global__ void __launch_bounds__(ScanCfg<T, NP, S, KC>::NT, 4)
scan_fwd_kernel(const __grid_constant__ ScanMaps maps, const ScanParams p) {
    using Cfg = ScanCfg<T, NP, S, KC>;
    constexpr int NT = Cfg::NT;
    using E = Elem<T>;
    constexpr int G = Cfg::G, NS = Cfg::NS, TT = Cfg::TT, HALO = Cfg::HALO, R = Cfg::R;
    constexpr int ROWB = Cfg::ROWB, SWZ = Cfg::SWZ;
    constexpr int NSTAGE = Cfg::NSTAGE;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float2* Pbuf = reinterpret_cast<float2*>(smem + Cfg::OFF_P);
    float2* Ebuf = reinterpret_cast<float2*>(smem + Cfg::OFF_E);
    T* Bt = reinterpret_cast<T*>(smem + Cfg::OFF_BT);
    T* Ct = reinterpret_cast<T*>(smem + Cfg::OFF_CT);
    float* par = reinterpret_cast<float*>(smem + Cfg::OFF_PAR);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int lg = tid / S;         // lane group: channels lg*KC .. lg*KC + KC - 1 of the CTA
    const int j = tid % S;          // state group of this lane
    const int b = blockIdx.y;
    const int d0 = blockIdx.x * G;
    const int L = p.seqlen;
    const int chunk = blockIdx.z;
    const int cs = chunk * p.chunk_len;                    // first scan position
    const int ce = min(cs + p.chunk_len, L);               // one past the last
    const int ntl = (ce - cs + TT - 1) / TT;               // tiles per direction
    const int ndir = p.mode == 2 ? 2 : 1;
    const int nt = ntl * ndir;
    const bool has_z = !SUMMARY && p.z != nullptr;
    const bool conv = p.conv_w != nullptr;
    const int xpitch = conv ? Cfg::X_PITCH_MAX : TT * (int)sizeof(T);
    auto chan_d = [&](int k) { return d0 + lg * KC + k; };             // channel k of the lane
    auto chan_row = [&](int k) { return (int64_t)b * p.dim + chan_d(k); };  // its (b, d) row

    auto tile_rev = [&](int f) { return p.mode == 1 || (p.mode == 2 && f >= ntl); };
    // time of the first element of flat tile f
    auto tile_l0 = [&](int f) {
        const int jt = f % ntl;
        const int i0 = cs + jt * TT;
        return tile_rev(f) ? L - i0 - TT : i0;
    };

    if (USE_TMA && tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        prefetch_tensormap(&maps.x);
        prefetch_tensormap(&maps.dt);
        prefetch_tensormap(&maps.B);
        prefetch_tensormap(&maps.C);
        if (has_z) prefetch_tensormap(&maps.z);
    }

    auto issue = [&](int f) {   // one thread: TMA loads of flat tile f
        uint8_t* st = smem + (f % NSTAGE) * Cfg::STAGE;
        const int l0 = tile_l0(f);
        const bool rv = tile_rev(f);
        const uint32_t xbytes = G * xpitch;
        uint32_t bytes = 2u * NS * ROWB + xbytes + G * ROWB + (has_z ? G * ROWB : 0u);
        mbar_arrive_expect_tx(&bars[f % NSTAGE], bytes);
        tma_load_3d(st + Cfg::RAW_B, &maps.B, &bars[f % NSTAGE], l0, 0, b);
        tma_load_3d(st + Cfg::RAW_C, &maps.C, &bars[f % NSTAGE], l0, 0, b);
        tma_load_3d(st + Cfg::RAW_X, &maps.x, &bars[f % NSTAGE], (conv && !rv) ? l0 - HALO : l0,
                    d0, b);
        tma_load_3d(st + Cfg::RAW_DT, &maps.dt, &bars[f % NSTAGE], l0, d0, b);
        if (has_z) tma_load_3d(st + Cfg::RAW_Z, &maps.z, &bars[f % NSTAGE], l0, d0, b);
    };

    // Plain-load fallback (any alignment): fills stage 0 with the same layout.
    auto load_plain = [&](int f) {
        uint8_t* st = smem;
        const int l0 = tile_l0(f);
        const bool rv = tile_rev(f);
        const T* gB = static_cast<const T*>(p.Bm) + (int64_t)b * p.dstate * L;
        const T* gC = static_cast<const T*>(p.Cm) + (int64_t)b * p.dstate * L;
        for (int e = tid; e < NS * TT; e += NT) {
            const int n = e / TT, col = e % TT, t = l0 + col;
            const bool ok = n < p.dstate && t >= 0 && t < L;
            const int off = swz<ROWB, SWZ>(n, col * (int)sizeof(T));
            *reinterpret_cast<T*>(st + Cfg::RAW_B + off) = ok ? gB[(int64_t)n * L + t] : T(0.f);
            *reinterpret_cast<T*>(st + Cfg::RAW_C + off) = ok ? gC[(int64_t)n * L + t] : T(0.f);
        }
        const int xw = xpitch / (int)sizeof(T);
        const int xs = (conv && !rv) ? l0 - HALO : l0;
        for (int e = tid; e < G * xw; e += NT) {
            const int r = e / xw, col = e % xw, t = xs + col, dd = d0 + r;
            const bool ok = dd < p.dim && t >= 0 && t < L;
            const int64_t gi = ((int64_t)b * p.dim + dd) * L + t;
            reinterpret_cast<T*>(st + Cfg::RAW_X + r * xpitch)[col] =
                ok ? static_cast<const T*>(p.u)[gi] : T(0.f);
        }
        for (int e = tid; e < G * TT; e += NT) {
            const int r = e / TT, col = e % TT, t = l0 + col, dd = d0 + r;
            const bool ok = dd < p.dim && t >= 0 && t < L;
            const int64_t gi = ((int64_t)b * p.dim + dd) * L + t;
            reinterpret_cast<T*>(st + Cfg::RAW_DT)[r * TT + col] =
                ok ? static_cast<const T*>(p.delta)[gi] : T(0.f);
            if (has_z)
                reinterpret_cast<T*>(st + Cfg::RAW_Z)[r * TT + col] =
                    ok ? static_cast<const T*>(p.z)[gi] : T(0.f);
        }
    };

    // Per-direction channel parameters -> smem, 16 floats per channel slot, each value
    // stored twice so a 64-bit load yields the pair the packed prologue math needs:
    // {w0,w0, w1,w1, w2,w2, w3,w3, conv_b x2, dt_bias x2, D x2, 0, 0}.
    auto load_params = [&](int dir) {
        for (int e = tid; e < G; e += NT) {
            const int dd = d0 + e;
            float* q = par + e * 16;
            const bool ok = dd < p.dim;
            // conv taps right-aligned: tap 3 meets the newest input
            for (int k = 0; k < 4; ++k) {
                const int kk = k - (4 - p.conv_width);
                q[2 * k] = q[2 * k + 1] =
                    (ok && conv && kk >= 0) ? p.conv_w[(int64_t)dd * p.conv_width + kk] : 0.f;
            }
            q[8] = q[9] = (ok && p.conv_b) ? p.conv_b[dd] : 0.f;
            q[10] = q[11] = (ok && p.dbias[dir]) ? p.dbias[dir][dd] : 0.f;
            q[12] = q[13] = (ok && p.Dv[dir]) ? p.Dv[dir][dd] : 0.f;
            q[14] = q[15] = 0.f;
        }
    };

    LaneState<NP, SUMMARY> ls[KC];
    auto load_A = [&](int dir) {
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            const int d = chan_d(k);
            float a[NP];
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                const int n = j * NP + i;
                a[i] = (d < p.dim && n < p.dstate) ? p.A[dir][(int64_t)d * p.dstate + n] * kLog2e
                                                   : 0.f;
            }
            ls[k].set_a(a);
        }
    };
    // Initial state of this chunk: carry over the summaries of earlier chunks.
    auto init_state = [&]() {
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            ls[k].reset();
            if (!SUMMARY && chunk > 0 && chan_d(k) < p.dim) {
                float hv[NP];
#pragma unroll
                for (int i = 0; i < NP; ++i) hv[i] = 0.f;
                const int64_t stride = (int64_t)p.batch * p.dim * NS;
                for (int k2 = 0; k2 < chunk; ++k2) {
                    const float2* sm = p.summary + k2 * stride + chan_row(k) * NS + j * NP;
#pragma unroll
                    for (int i = 0; i < NP; ++i) {
                        const float2 ps = sm[i];
                        hv[i] = fmaf(ps.x, hv[i], ps.y);
                    }
                }
                ls[k].set(hv);
            }
        }
    };

    auto prologue = [&](int f, const uint8_t* st) {
        const bool rv = tile_rev(f);
        const int xoff = (conv && !rv) ? HALO : 0;
        // B, C: swizzled [n][t] -> [t][n] in the input type, one 16-byte chunk per thread
        constexpr int EPC = 16 / (int)sizeof(T);           // elements per 16-byte chunk
        constexpr int NCH = NS * ROWB / 16;                // chunks per tensor
        for (int e = tid; e < 2 * NCH; e += NT) {
            const int ten = e / NCH, ch = e % NCH;
            const int n = ch % NS, t0 = (ch / NS) * EPC;
            const uint8_t* src = st + (ten ? Cfg::RAW_C : Cfg::RAW_B) + swz<ROWB, SWZ>(n, t0 * (int)sizeof(T));
            T* dst = (ten ? Ct : Bt) + t0 * NS + n;
            const uint4 v = *reinterpret_cast<const uint4*>(src);
            const T* tv = reinterpret_cast<const T*>(&v);
#pragma unroll
            for (int m = 0; m < EPC; ++m) dst[m * NS] = tv[m];
        }
        // per (channel, t) quantities, two consecutive steps per lane in packed pairs:
        // 16 lanes cover one 32-step channel row, a warp two rows at a time
        for (int idx = warp; idx < G / 2; idx += NT / 32) {
            const int r = 2 * idx + (lane >> 4);
            const int tt = 2 * (lane & 15);                 // steps tt and tt + 1
            const T* xr = reinterpret_cast<const T*>(st + Cfg::RAW_X + r * xpitch);
            const uint64_t* q2 = reinterpret_cast<const uint64_t*>(par + r * 16);
            uint64_t u2;
            if (conv) {
                // forward: u_t = sum_k w_k x[t-3+k]; reverse: u_t = sum_k w_k x[t+3-k]
                float xv[5];
#pragma unroll
                for (int m = 0; m < 5; ++m)
                    xv[m] = E::to_f(rv ? xr[tt + 4 - m] : xr[xoff + tt - 3 + m]);
                uint64_t acc = q2[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    acc = fma2(q2[k], rv ? pk2(xv[k + 1], xv[k]) : pk2(xv[k], xv[k + 1]), acc);
                u2 = silu2(acc);
            } else {
                u2 = pk2(E::to_f(xr[tt]), E::to_f(xr[tt + 1]));
            }
            const T* dtr = reinterpret_cast<const T*>(st + Cfg::RAW_DT) + r * TT + tt;
            uint64_t dl2 = add2(pk2(E::to_f(dtr[0]), E::to_f(dtr[1])), q2[5]);
            if (p.softplus) dl2 = softplus2(dl2);
            const float2 dl = upk2(dl2), du = upk2(mul2(dl2, u2));
            uint8_t* prow = reinterpret_cast<uint8_t*>(Pbuf) + (r / KC) * Cfg::P_PITCH;
            if (KC == 1) {
                *reinterpret_cast<float4*>(prow + tt * 8) = make_float4(dl.x, du.x, dl.y, du.y);
            } else {
                *reinterpret_cast<float2*>(prow + tt * 16 + (r % KC) * 8) = make_float2(dl.x, du.x);
                *reinterpret_cast<float2*>(prow + tt * 16 + 16 + (r % KC) * 8) = make_float2(dl.y, du.y);
            }
            if (!SUMMARY) {
                uint64_t g2 = pk2(1.f, 1.f);
                if (has_z) {
                    const T* zr = reinterpret_cast<const T*>(st + Cfg::RAW_Z) + r * TT + tt;
                    g2 = silu2(pk2(E::to_f(zr[0]), E::to_f(zr[1])));
                }
                const float2 g = upk2(g2), dv = upk2(mul2(q2[6], u2));
                *reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(Ebuf) + r * Cfg::E_PITCH + tt * 8) =
                    make_float4(dv.x, g.x, dv.y, g.y);
            }
        }
    };

    const uint8_t* Prow = reinterpret_cast<uint8_t*>(Pbuf) + lg * Cfg::P_PITCH;
    const T* Bl = Bt + j * NP;
    const T* Cl = Ct + j * NP;
    // P of step tt for the lane's KC channels: pd[k] = {delta, delta*u}
    auto load_p = [&](int tt, float2 (&pd)[KC]) {
        if constexpr (KC == 2) {
            const float4 v = *reinterpret_cast<const float4*>(Prow + tt * 16);
            pd[0] = make_float2(v.x, v.y);
            pd[1] = make_float2(v.z, v.w);
        } else {
            pd[0] = *reinterpret_cast<const float2*>(Prow + tt * 8);
        }
    };
    // this lane's NP values of B and C at step tt (bf16 pairs are widened in registers:
    // the high half of a 32-bit word is already an fp32 bit pattern, the low half
    // shifted up by 16 is one)
    auto load_bc = [&](int tt, float (&bv)[NP], float (&cv)[NP]) {
        if constexpr (sizeof(T) == 2 && NP % 2 == 0) {
            uint32_t wb[NP / 2], wc[NP / 2];
            if constexpr (NP == 4) {
                const uint2 b2 = *reinterpret_cast<const uint2*>(Bl + tt * NS);
                wb[0] = b2.x; wb[1] = b2.y;
                if (!SUMMARY) {
                    const uint2 c2 = *reinterpret_cast<const uint2*>(Cl + tt * NS);
                    wc[0] = c2.x; wc[1] = c2.y;
                }
            } else {
#pragma unroll
                for (int i = 0; i < NP / 2; ++i) {
                    wb[i] = reinterpret_cast<const uint32_t*>(Bl + tt * NS)[i];
                    if (!SUMMARY) wc[i] = reinterpret_cast<const uint32_t*>(Cl + tt * NS)[i];
                }
            }
#pragma unroll
            for (int i = 0; i < NP / 2; ++i) {
                bv[2 * i] = __uint_as_float(wb[i] << 16);
                bv[2 * i + 1] = __uint_as_float(wb[i] & 0xffff0000u);
                if (!SUMMARY) {
                    cv[2 * i] = __uint_as_float(wc[i] << 16);
                    cv[2 * i + 1] = __uint_as_float(wc[i] & 0xffff0000u);
                }
            }
        } else if constexpr (sizeof(T) == 4 && NP % 4 == 0) {
#pragma unroll
            for (int i = 0; i < NP; i += 4) {
                const float4 b4 = *reinterpret_cast<const float4*>(Bl + tt * NS + i);
                bv[i] = b4.x; bv[i + 1] = b4.y; bv[i + 2] = b4.z; bv[i + 3] = b4.w;
                if (!SUMMARY) {
                    const float4 c4 = *reinterpret_cast<const float4*>(Cl + tt * NS + i);
                    cv[i] = c4.x; cv[i + 1] = c4.y; cv[i + 2] = c4.z; cv[i + 3] = c4.w;
                }
            }
        } else if constexpr (sizeof(T) == 4 && NP == 2) {
            const float2 b2 = *reinterpret_cast<const float2*>(Bl + tt * NS);
            bv[0] = b2.x; bv[1] = b2.y;
            if (!SUMMARY) {
                const float2 c2 = *reinterpret_cast<const float2*>(Cl + tt * NS);
                cv[0] = c2.x; cv[1] = c2.y;
            }
        } else {
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                bv[i] = E::to_f(Bl[tt * NS + i]);
                if (!SUMMARY) cv[i] = E::to_f(Cl[tt * NS + i]);
            }
        }
    };
    // gate, skip term, bidirectional partial and the store of R owned outputs
    auto epilogue = [&](int k, const float* acc, bool rv, int dir, int l0, int pos0, int nown) {
        const float2* Erow = reinterpret_cast<const float2*>(
            reinterpret_cast<uint8_t*>(Ebuf) + (lg * KC + k) * Cfg::E_PITCH);
        const int64_t row = chan_row(k);
        float yv[R];
#pragma unroll
        for (int m = 0; m < R; ++m) {
            const int ii = pos0 + m;
            const int tt = rv ? TT - 1 - ii : ii;
            const float2 e = Erow[tt];
            yv[m] = (acc[m] + e.x) * e.y;
        }
        if (chan_d(k) >= p.dim || nown <= 0) return;
        const int tmin = rv ? l0 + TT - 1 - (pos0 + R - 1) : l0 + pos0;
        float ya[R];                                      // time-ascending order
#pragma unroll
        for (int m = 0; m < R; ++m) ya[m] = rv ? yv[R - 1 - m] : yv[m];
        // valid ascending index range: forward [0, nown); reverse [R - nown, R)
        const int mlo = rv ? R - nown : 0;
        const int mhi = rv ? R : nown;
        const int64_t gbase = row * L + tmin;
        if (p.mode == 2 && dir == 1) {
#pragma unroll
            for (int m = 0; m < R; ++m)
                if (m >= mlo && m < mhi) ya[m] += p.partial[gbase + m];
        }
        if (p.mode == 2 && dir == 0) {
#pragma unroll
            for (int m = 0; m < R; ++m)
                if (m >= mlo && m < mhi) p.partial[gbase + m] = ya[m];
            return;
        }
        T* out = static_cast<T*>(p.out) + gbase;
        const bool full = (mlo == 0 && mhi == R) && p.vec_store;
        if (full && R * sizeof(T) == 16) {
            if constexpr (sizeof(T) == 4) {
                *reinterpret_cast<float4*>(out) = make_float4(ya[0], ya[1 % R], ya[2 % R], ya[3 % R]);
            } else {
                uint4 v;
                uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    __nv_bfloat162 t2 = __floats2bfloat162_rn(ya[(2 * m) % R], ya[(2 * m + 1) % R]);
                    w[m] = *reinterpret_cast<uint32_t*>(&t2);
                }
                *reinterpret_cast<uint4*>(out) = v;
            }
        } else if (full && R * sizeof(T) == 8) {
            if constexpr (sizeof(T) == 4) {
                *reinterpret_cast<float2*>(out) = make_float2(ya[0], ya[1 % R]);
            } else {
                __nv_bfloat162 t0 = __floats2bfloat162_rn(ya[0], ya[1 % R]);
                __nv_bfloat162 t1 = __floats2bfloat162_rn(ya[2 % R], ya[3 % R]);
                uint2 v;
                v.x = *reinterpret_cast<uint32_t*>(&t0);
                v.y = *reinterpret_cast<uint32_t*>(&t1);
                *reinterpret_cast<uint2*>(out) = v;
            }
        } else if (full && R * sizeof(T) == 4 && sizeof(T) == 2) {
            *reinterpret_cast<__nv_bfloat162*>(out) = __floats2bfloat162_rn(ya[0], ya[1 % R]);
        } else {
#pragma unroll
            for (int m = 0; m < R; ++m)
                if (m >= mlo && m < mhi) out[m] = E::from_f(ya[m]);
        }
    };

    // butterfly transpose-reduce over the S lanes of a channel: afterwards lane j
    // holds the sums of block positions [j*R, j*R + R) in acc[0 .. R)
    auto reduce_block = [&](float* acc) {
        int len = 16;
#pragma unroll
        for (int m = S / 2; m >= 1; m >>= 1) {
            const int half = len >> 1;
            const bool upper = (j & m) != 0;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float send = upper ? acc[i] : acc[i + half];
                const float keep = upper ? acc[i + half] : acc[i];
                acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
            len = half;
        }
    };

    // One tile in scan order. RV: walk time downwards. FULL: all TT steps valid
    // (no per-step predicate; shared-memory offsets are compile-time constants).
    auto scan_tile = [&](auto rv_tag, auto full_tag, int f) {
        constexpr bool RV = decltype(rv_tag)::value;
        constexpr bool FULL = decltype(full_tag)::value;
        const int dir = (p.mode == 2 && f >= ntl) ? 1 : 0;
        const int i0 = cs + (f % ntl) * TT;
        const int nvalid = FULL ? TT : min(TT, ce - i0);
        const int l0 = RV ? L - i0 - TT : i0;
#pragma unroll 1
        for (int blk = 0; blk < TT / 16; ++blk) {
            if (!FULL && blk * 16 >= nvalid) break;
            float acc[KC][16];
            if (FULL) {
                // KB steps at a time: their state-independent operands (shared-memory
                // loads, delta*A, the SFU exps, delta*u*B) are all prepared first, then the
                // KB dependent state updates run.
                // (two channels per lane already give two independent update streams)
                constexpr int KB = KC == 2 ? 1 : SSM_SCAN_BATCH;
#pragma unroll
                for (int q0 = 0; q0 < 16; q0 += KB) {
                    typename LaneState<NP, SUMMARY>::In in[KB][KC];
#pragma unroll
                    for (int u = 0; u < KB; ++u) {
                        const int tt = RV ? TT - 1 - (blk * 16 + q0 + u) : blk * 16 + q0 + u;
                        float2 pd[KC];
                        float bv[NP], cv[NP];
                        load_p(tt, pd);
                        load_bc(tt, bv, cv);
#pragma unroll
                        for (int k = 0; k < KC; ++k) in[u][k] = ls[k].prep(pd[k].x, pd[k].y, bv, cv);
                    }
#pragma unroll
                    for (int u = 0; u < KB; ++u)
#pragma unroll
                        for (int k = 0; k < KC; ++k) acc[k][q0 + u] = ls[k].update(in[u][k]);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int ii = blk * 16 + q;
                    const int tt = RV ? TT - 1 - ii : ii;
#pragma unroll
                    for (int k = 0; k < KC; ++k) acc[k][q] = 0.f;
                    if (ii < nvalid) {
                        float2 pd[KC];
                        float bv[NP], cv[NP];
                        load_p(tt, pd);
                        load_bc(tt, bv, cv);
#pragma unroll
                        for (int k = 0; k < KC; ++k)
                            acc[k][q] = ls[k].update(ls[k].prep(pd[k].x, pd[k].y, bv, cv));
                    }
                }
            }
            if (SUMMARY) continue;
            const int pos0 = blk * 16 + j * R;
#pragma unroll
            for (int k = 0; k < KC; ++k) {
                reduce_block(acc[k]);
                epilogue(k, acc[k], RV, dir, l0, pos0, FULL ? R : max(0, min(R, nvalid - pos0)));
            }
        }
    };

    auto finish_direction = [&](int dir) {
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            if (chan_d(k) >= p.dim) continue;
            const int64_t row = chan_row(k);
            if (SUMMARY) {
                float2* sm = p.summary + (int64_t)chunk * p.batch * p.dim * NS + row * NS + j * NP;
#pragma unroll
                for (int i = 0; i < NP; ++i) sm[i] = make_float2(ls[k].get_pr(i), ls[k].get(i));
            } else if (chunk == p.nchunks - 1 && p.final_state[dir]) {
                float* fs = p.final_state[dir] + row * p.dstate;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    const int n = j * NP + i;
                    if (n < p.dstate) fs[n] = ls[k].get(i);
                }
            }
        }
    };

    // ------------------------------------------------------------- main loop --
    load_params(0);
    load_A(0);
    init_state();
    if (USE_TMA) {
        __syncthreads();   // barrier init visible before any wait
        if (tid == 0)
            for (int f = 0; f < min(NSTAGE, nt); ++f) issue(f);
    }
    __syncthreads();

    for (int f = 0; f < nt; ++f) {
        if (p.mode == 2 && f == ntl) {       // second direction of the bidirectional sum
            finish_direction(0);
            __syncthreads();                 // params of direction 0 no longer read
            load_params(1);
            load_A(1);
#pragma unroll
            for (int k = 0; k < KC; ++k) ls[k].reset();
            __syncthreads();
        }
        bool ok = true;
        const uint8_t* st;
        if (USE_TMA) {
            // one lane per warp polls; __syncwarp hands the completed phase to the rest
            if (lane == 0) ok = mbar_wait_bounded(&bars[f % NSTAGE], (f / NSTAGE) & 1);
            __syncwarp();
            // each lane then observes the completed phase itself (one try_wait, which
            // succeeds at once), so the TMA writes are acquired by every reader
            if (lane != 0) mbar_try_wait(&bars[f % NSTAGE], (f / NSTAGE) & 1);
            st = smem + (f % NSTAGE) * Cfg::STAGE;
        } else {
            load_plain(f);
            __syncthreads();
            st = smem;
        }
        prologue(f, st);
        if (__syncthreads_or(!ok)) {
            // a tile never landed: drain what is still in flight (bounded), leave
            if (USE_TMA && tid == 0)
                for (int g2 = f; g2 < min(f + NSTAGE, nt); ++g2)
                    mbar_wait_bounded(&bars[g2 % NSTAGE], (g2 / NSTAGE) & 1);
            return;
        }
        if (USE_TMA && tid == 0 && f + NSTAGE < nt) issue(f + NSTAGE);
        const bool rv = tile_rev(f);
        const bool full = cs + (f % ntl) * TT + TT <= ce;
        using TrueT = std::integral_constant<bool, true>;
        using FalseT = std::integral_constant<bool, false>;
        if (full) {
            if (rv) scan_tile(TrueT{}, TrueT{}, f);
            else scan_tile(FalseT{}, TrueT{}, f);
        } else {
            if (rv) scan_tile(TrueT{}, FalseT{}, f);
            else scan_tile(FalseT{}, FalseT{}, f);
        }
        __syncthreads();
    }
    finish_direction(p.mode == 2 ? 1 : 0);
}

}  // namespace ssm
