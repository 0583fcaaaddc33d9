// Selective-scan forward kernel for sm_100a.
//
// Work split. A CTA owns G channels of one batch row and walks the sequence in
// tiles of TT steps (TT*sizeof(T) = 64 or 128 bytes). Its warps have two roles:
//
//  * 2 producer warps (6 beside 8 scan warps) own the TMA ring and the
//    once-per-(channel, t) prologue. For
//    each tile they wait for the raw tiles (u or the pre-conv x with a 16-byte halo,
//    dt, z, B, C; B and C are shared by all channels of a batch row), compute
//    conv + SiLU, delta = softplus(dt + bias), delta*u, D*u and silu(z) into one of
//    two staging buffers, transpose B and C to fp32 [t][n], and hand the buffer
//    over through an mbarrier;
//  * SW (2, 3, 4 or 8) scan warps run the recurrence. The S lanes of a channel each keep NP = NS/S
//    of the (padded) NS states in registers, so a channel's recurrence is spread
//    over S lanes with no carry between them (A is diagonal: the states never
//    interact); a lane serves KC channels with the same NP states, so each B and C
//    value it reads from shared memory feeds KC updates. Per (t, state) one ex2 on
//    the SFU, then h = dA*h + delta*u*B and the lane's partial C.h. Every 16 steps a
//    butterfly transpose-reduce over the S lanes leaves each lane owning 16/S
//    consecutive outputs of each of its channels, which it gates and stores with one
//    vector store. The buffer goes back to the producers through a second mbarrier.
//
// The scan warps never stop at a CTA-wide barrier: the prologue of tile f + 1 runs
// on the producer warps while the scan warps work through tile f. The scan is bound
// by the SFU (one exp per state and step), the issue slots and the shared-memory
// bandwidth together; serving KC channels per lane cuts the bytes each lane reads
// per update.
//
// Channel-last activations (CL): u, delta, z, out are (batch, seqlen, dim) and B, C
// (batch, seqlen, dstate), each with its own element stride between positions (so x
// and z may be views into one in_proj output). The TMA boxes are then (channels x
// steps): x/dt/z tiles land as [t][channel] and B/C tiles as [t][n], which the
// producers only widen (no transpose); a producer reads its channel's window with
// strided scalar loads (a warp's lanes read one row, conflict-free). The staged tile
// is the same for both layouts, so the scan warps run the same code; only the
// output and bidirectional-partial addresses differ.
//
// Packed sequences (VL): several sequences share the sequence axis of one batch row,
// starting at the offsets p.cu (p.cu[0] = 0, p.cu[nseq] = L). The state restarts from
// zero at every start, the fused conv reads nothing before its sequence's start, and
// each sequence's final state is written when its last step is done. One producer
// thread finds the starts near each tile with a binary search over p.cu and stages
// them as a bit mask with the tile.
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

// Bytes of one tile row in the splits of 8 lanes per channel with bf16 activations (the
// narrow batches): 128 (64-step tiles, half the per-tile overhead) or 64.
#ifndef SSM_NARROW_ROWB
#define SSM_NARROW_ROWB 128
#endif


// Steps whose state-independent operands are prepared together (a divisor of 16).
#ifndef SSM_SCAN_BATCH
#define SSM_SCAN_BATCH 2
#endif

constexpr int kProWarps = 2;                                // TMA + prologue warps
constexpr int kProWarpsWide = 6;                            // with 8 scan warps (one CTA per SM)
constexpr int kProBarrier = 1;                              // the producers' named barrier

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// VLK: the packed-sequence kernels (their tile length may differ).
template <typename T, int NP, int S, int KC, int SW, bool VLK = false>
struct ScanCfg {
    static constexpr int SCAN_THREADS = 32 * SW; // SW recurrence warps
    static constexpr bool ROWB_NARROW = sizeof(T) == 2 && S == 8 && NP * S == 16 && !VLK &&
                                        SSM_NARROW_ROWB == 128;   // 64-step tiles
    static constexpr int G = SCAN_THREADS / S * KC;   // channels per CTA
    // producer warps: 2; 6 beside 8 scan warps (d_state 128: one CTA per SM, and the
    // B/C transposes of 128 states per step are the producers' largest job)
    static constexpr int PRO_THREADS = 32 * (SW == 8 ? kProWarpsWide : kProWarps);
    static constexpr int NT = SCAN_THREADS + PRO_THREADS;   // threads per CTA
    // CTAs per SM the launch bounds ask for: three of 6 warps (96 registers per
    // thread), three of 4 warps with two channels per lane (168), five of 4 warps (96);
    // two for d_state 64 / 128 (their B/C tiles take up to 127 KB of shared memory), one
    // of 10 warps with 8 scan warps
    static constexpr int MIN_CTAS =
        SW == 8 ? 1 : NP * S > 16 ? 2 : (SW >= 3 || S == 2 || KC == 2 ? 3 : ROWB_NARROW ? 4 : 5);
    static constexpr int NS = NP * S;            // padded state count
    static constexpr int ES = sizeof(T);
    // bytes of one tile row: 64 (32 bf16 / 16 fp32 steps); 128 (64 bf16 steps) in the
    // narrow bf16 splits, where a CTA holds few channels and per-tile costs weigh most
    // (not for packed sequences: measured slower there)
    static constexpr int ROWB = ROWB_NARROW ? 128 : 64;
    static constexpr int TT = ROWB / ES;         // tile length in steps
    // TMA swizzle spanning one tile row (XOR of address bits [4, 4+w) with [7, 7+w)):
    // 64-byte (w = 2) or 128-byte (w = 3)
    static constexpr int SWZ = ROWB == 128 ? 7 : 3;
    static constexpr int HALO = 16 / ES;         // conv history, one 16-B TMA granule
    static constexpr int NSTAGE = 2;             // raw TMA stages
    static constexpr int NBUF = 2;               // staging buffers
    static constexpr int R = 16 / S;             // outputs owned per lane, channel and block
    // raw stage (bytes from the 1024-aligned stage base)
    static constexpr int RAW_B = 0;                                   // [NS][TT], swizzled
    static constexpr int RAW_C = align_up(NS * ROWB, 1024);           // [NS][TT], swizzled
    static constexpr int RAW_X = align_up(RAW_C + NS * ROWB, 128);    // [G][TT(+HALO)]
    static constexpr int X_PITCH_MAX = (TT + HALO) * ES;
    // delta / z tiles: swizzled like B / C in the (batch, dim, seqlen) layout
    static constexpr bool SWZDT = SSM_SWZ_DTZ != 0;
    static constexpr int RAW_DT = align_up(RAW_X + G * X_PITCH_MAX, SWZDT ? 1024 : 128);
    static constexpr int RAW_Z = align_up(RAW_DT + G * ROWB, SWZDT ? 1024 : 128);
    static constexpr int STAGE = align_up(RAW_Z + G * ROWB, 1024);
    // Staging buffer (fp32). P: per group of KC channels and step, KC x {delta,
    // delta*u} (one vector load per lane and step). E: per channel and step {D*u,
    // silu(z)}. B and C transposed to [t][n], so a lane reads its NP states of a
    // step with one vector load and no conversion.
    static constexpr int P_PITCH = TT * KC * 8 + 16;
    static constexpr int E_PITCH = TT * 8 + 16;
    static constexpr int BUF_P = 0;
    static constexpr int BUF_E = (G / KC) * P_PITCH;
    static constexpr int BUF_BT = BUF_E + G * E_PITCH;
    // B/C staging rows. A producer warp transposing 16-byte chunks writes, per store, the
    // same n of several rows EPC steps apart; with rows of 16 floats those rows share
    // banks. So the 2-state splits (8-byte loads) pad each row to NS + 2 floats, and the
    // splits that load 16 bytes keep NS floats and permute the rows: row t is stored at
    // t ^ ((t / EPC) & (BCW - 1)), BCW rows per 128 bytes (measured: the long sequence
    // 1.1 % and the 130M layer 0.9 % faster; the permutation in the 2-state splits slowed
    // the packed-sequence kernel by 4 %).
    static constexpr int BCP = NP == 2 ? NS + 2 : NS;   // row pitch (floats)
    // The prologue's SiLUs take the reciprocal on the FMA pipe (one SFU op per value) in
    // the 8 x 2 split, where the SFU is the busiest pipe (the 130M layer: 230 -> 226 µs);
    // elsewhere the SFU reciprocal measured faster.
    static constexpr bool SILU_FMA = NP == 8 && S == 2;
    static constexpr int EPC_ = 16 / (int)sizeof(T);
    static constexpr int BCW = NP % 4 == 0 && BCP < 32 ? (32 / BCP < EPC_ ? 32 / BCP : EPC_) : 1;
    __host__ __device__ static constexpr int bc_row(int t) { return t ^ ((t / EPC_) & (BCW - 1)); }
    static constexpr int BUF_CT = BUF_BT + TT * BCP * 4;
    // packed sequences: starts at positions [l0 - HALO, l0 + TT], bit i <-> l0 - HALO + i
    static constexpr int BUF_META = BUF_CT + TT * BCP * 4;
    static constexpr int BUF = align_up(BUF_META + 16, 128);
    static constexpr int OFF_BUF = NSTAGE * STAGE;
    static constexpr int OFF_PAR = OFF_BUF + NBUF * BUF;   // [2 directions][G][16] floats
    static constexpr int OFF_BAR = align_up(OFF_PAR + 2 * G * 64, 8);
    static constexpr int NBARS = NSTAGE + 2 * NBUF;        // raw full; buffer full, empty
    static constexpr int BYTES = OFF_BAR + NBARS * 8;
    static constexpr int SMEM = BYTES + 1024;              // slack for 1024-B alignment
    static_assert(TT % 16 == 0, "tile must hold whole 16-step blocks");
    static_assert(P_PITCH % 16 == 0 && E_PITCH % 16 == 0, "staging rows take 16-byte stores");
    static_assert(BUF_E % 16 == 0 && BUF_BT % 16 == 0 && BUF % 16 == 0, "16-byte aligned parts");
    static_assert(NS <= 128, "at most 128 states");
    static_assert(KC == 1 || KC == 2, "one or two channels per lane");
    static_assert(HALO + TT + 1 <= 128, "the packed-sequence window mask is 128 bits");
    static_assert(ROWB == 64 || ROWB == 128, "tile rows of 64 or 128 bytes");
    // packed sequences: sequence starts at positions [l0 - HALO, l0 + TT] (Mask) and the
    // tile's steps (Steps), one bit each
    using Mask = std::conditional_t<(HALO + TT + 1 > 64), unsigned __int128, uint64_t>;
    using Steps = std::conditional_t<(TT > 32), uint64_t, uint32_t>;
};

// Byte offset of logical (row, byte) in a swizzled [rows][ROWB] tile. TMA's 64-B
// swizzle XORs address bits [4, 6) with bits [7, 9) of the offset from a 1024-byte
// aligned tile base; SWZ is that 2-bit mask.
template <int ROWB, int SWZ>
__device__ __forceinline__ int swz(int row, int byte_in_row) {
    const int off = row * ROWB + byte_in_row;
    return off ^ (((off >> 7) & SWZ) << 4);
}

// Recurrence state of one lane: NP states, held as fp32 pairs so the four
// per-state operations (delta*A, delta*u*B, the h update and C.h) issue as packed
// .f32x2 instructions.
template <int NP, bool SUMMARY, bool SA = false>
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
    // A sequence starts: the state restarts from zero and no longer depends on the
    // state carried in (the chunk product drops to zero).
    __device__ __forceinline__ void cut() {
#pragma unroll
        for (int k = 0; k < NPR; ++k) { h2[k] = pk2(0.f, 0.f); pr2[k] = pk2(0.f, 0.f); }
        h1 = 0.f;
        pr1 = 0.f;
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
    // exp2(delta*a2), delta*u*B and C. Preparing several steps' operands before their
    // updates overlaps the shared-memory loads and the SFU latency with the
    // dependent FMAs.
    struct In {
        uint64_t dA[NPR > 0 ? NPR : 1], bu[NPR > 0 ? NPR : 1], cc[NPR > 0 ? NPR : 1];
        float dA1, bu1, c1;
    };

    // dl = delta (SA: the step's decay dA itself, the same for every state of a head),
    // du = delta*u of the step; b / cvv: this lane's NP fp32 B and C values.
    __device__ __forceinline__ In prep(float dl, float du, const float* b, const float* cvv) const {
        In in;
        const uint64_t dd = pk2(dl, dl), uu = pk2(du, du);
#pragma unroll
        for (int k = 0; k < NPR; ++k) {
            if (SA) {
                in.dA[k] = dd;
            } else {
                const uint64_t x = mul2(dd, a2[k]);
                in.dA[k] = pk2(ex2(lo2(x)), ex2(hi2(x)));
            }
            in.bu[k] = mul2(uu, pk2(b[2 * k], b[2 * k + 1]));
            if (!SUMMARY) in.cc[k] = pk2(cvv[2 * k], cvv[2 * k + 1]);
        }
        if (ODD) {
            in.dA1 = SA ? dl : ex2(dl * a1);
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

// Writes the caller's conv history (the inputs at positions -(W-1) .. -1) into the
// first forward tile's halo in shared memory. Out of line: it runs once per CTA and
// keeps its registers out of the producer loop.
template <typename T, int G, int HALO, int NTHR, bool CL>
__device__ __noinline__ void put_conv_history(const ScanParams& p, uint8_t* raw_x, int xpitch,
                                              int ptid, int b, int d0) {
    const int hw = p.conv_width - 1;
    for (int e = ptid; e < G * hw; e += NTHR) {
        const int r = e / hw, k = e % hw, dd = d0 + r;
        if (dd < p.dim) {
            const T v = static_cast<const T*>(p.conv_hist)[((int64_t)b * p.dim + dd) * hw + k];
            if (CL) reinterpret_cast<T*>(raw_x)[(HALO - hw + k) * G + r] = v;   // [t][channel]
            else reinterpret_cast<T*>(raw_x + r * xpitch)[HALO - hw + k] = v;
        }
    }
    fence_proxy_async_smem();                     // before the stage's next TMA write
}

template <typename T, int NP, int S, int KC, int SW, bool USE_TMA, bool SUMMARY, bool VL,
          bool CL, int FEAT>
__global__ void __launch_bounds__(ScanCfg<T, NP, S, KC, SW, VL>::NT,
                                  ScanCfg<T, NP, S, KC, SW, VL>::MIN_CTAS)
scan_fwd_kernel(const __grid_constant__ ScanMaps maps, const ScanParams p) {
    using Cfg = ScanCfg<T, NP, S, KC, SW, VL>;
    constexpr int kScanWarps = SW, kScanThreads = Cfg::SCAN_THREADS, kCtaThreads = Cfg::NT;
    using E = Elem<T>;
    constexpr int G = Cfg::G, NS = Cfg::NS, TT = Cfg::TT, HALO = Cfg::HALO, R = Cfg::R;
    constexpr int ROWB = Cfg::ROWB, SWZ = Cfg::SWZ;
    constexpr int NSTAGE = Cfg::NSTAGE;
    // FEAT bit 0 (SA): A is one scalar per head; the producers stage the step's decay
    // exp(delta A_h) in place of delta and the scan warps take no exps. Bit 1 (SB): B and
    // C are fp32 (dim, dstate), fixed per channel; no B/C tiles, each lane keeps its
    // channel's NP values of each in registers.
    constexpr bool SA = (FEAT & 1) != 0, SB = (FEAT & 2) != 0;
    static_assert(!SB || KC == 1, "time-invariant B/C: one channel per lane");

    // 1024-byte aligned base, reached by pointer arithmetic on the shared array (not
    // through an integer cast) so that every pointer derived from it stays in the
    // shared address space and its loads compile to shared loads, not generic ones
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* par = reinterpret_cast<float*>(smem + Cfg::OFF_PAR);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full_raw = bars;                    // [NSTAGE] TMA bytes landed (1 arrival + tx)
    uint64_t* full_buf = bars + NSTAGE;           // [NBUF] staging written (producer arrivals)
    uint64_t* empty_buf = bars + NSTAGE + Cfg::NBUF;   // [NBUF] staging read (scan arrivals)

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y;
    const int d0 = blockIdx.x * G;
    const int L = p.seqlen;
    const int chunk = blockIdx.z;
    // Scan range [cs + vbeg, ce) of this chunk, tiles from cs. Packed sequences in
    // sequence-aligned chunks (p.seq_aligned): the chunk runs from the first sequence
    // start at or after chunk * chunk_len to the first one at or after the next chunk's
    // position, so it starts from a zero state and needs no carry; cs is that start
    // rounded down to a tile, and the vbeg positions before it belong to the previous
    // chunk (scanned by it, skipped here).
    int cs = chunk * p.chunk_len;                          // first tile position
    int ce = min(cs + p.chunk_len, L);                     // one past the last position
    int vbeg = 0;
    if (VL && p.seq_aligned) {
        auto start_at_or_after = [&](int pos) {            // clamped to [0, L]
            int a = 0, z = p.nseq;
            while (a < z) {
                const int m = (a + z) >> 1;
                if (p.cu[m] < pos) a = m + 1; else z = m;
            }
            return min(max(p.cu[a], 0), L);
        };
        const int s0 = chunk == 0 ? 0 : start_at_or_after(cs);
        const int s1 = chunk == p.nchunks - 1 ? L : max(start_at_or_after(ce), s0);
        cs = s0 / TT * TT;
        vbeg = s0 - cs;
        ce = s1 > s0 ? s1 : cs;                             // empty: no tiles
    }
    const int ntl = (ce - cs + TT - 1) / TT;               // tiles per direction
    const int ndir = p.mode == 2 ? 2 : 1;
    const int nt = ntl * ndir;
    const bool has_z = !SUMMARY && p.z != nullptr;
    const bool conv = p.conv_w != nullptr;
    const int xpitch = conv ? Cfg::X_PITCH_MAX : TT * (int)sizeof(T);
    using TrueT = std::integral_constant<bool, true>;
    using FalseT = std::integral_constant<bool, false>;

    auto tile_rev = [&](int f) { return p.mode == 1 || (p.mode == 2 && f >= ntl); };
    auto tile_dir = [&](int f) { return (p.mode == 2 && f >= ntl) ? 1 : 0; };
    // time of the first element of flat tile f
    auto tile_l0 = [&](int f) {
        const int i0 = cs + (f % ntl) * TT;
        return tile_rev(f) ? L - i0 - TT : i0;
    };
    auto buf_of = [&](int f) { return smem + Cfg::OFF_BUF + (f & 1) * Cfg::BUF; };

    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) mbar_init(&full_raw[s], 1);
        for (int s = 0; s < Cfg::NBUF; ++s) {
            mbar_init(&full_buf[s], Cfg::PRO_THREADS);
            mbar_init(&empty_buf[s], kScanThreads);
        }
        fence_mbar_init();
    }
    // Channel parameters of both directions -> smem, 16 floats per channel slot, each
    // value twice so a 64-bit load yields the pair the packed prologue math needs:
    // {w0,w0, w1,w1, w2,w2, w3,w3, conv_b x2, dt_bias x2, D x2, 0, 0}.
    for (int e = tid; e < ndir * G; e += kCtaThreads) {
        const int dir = e / G, r = e % G, dd = d0 + r;
        float* q = par + (dir * G + r) * 16;
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
        q[14] = q[15] = (SA && ok) ? p.A[dir][dd / p.head_dim] * kLog2e : 0.f;   // A_h log2(e)
    }
    __syncthreads();   // barriers initialised and parameters written, for both roles

    if (warp >= kScanWarps) {
        // ============================================================ producers ==
        const int ptid = tid - kScanThreads;

        auto issue = [&](int f) {   // one thread: TMA loads of flat tile f
            uint8_t* st = smem + (f % NSTAGE) * Cfg::STAGE;
            const int l0 = tile_l0(f);
            const bool rv = tile_rev(f);
            const uint32_t bytes =
                (SB ? 0u : 2u * NS * ROWB) + G * xpitch + G * ROWB + (has_z ? G * ROWB : 0u);
            uint64_t* bar = &full_raw[f % NSTAGE];
            mbar_arrive_expect_tx(bar, bytes);
            const int lx = (conv && !rv) ? l0 - HALO : l0;
            if constexpr (CL) {               // maps over (channel, t, batch)
                if (!SB) {
                    tma_load_3d(st + Cfg::RAW_B, &maps.B, bar, 0, l0, b);
                    tma_load_3d(st + Cfg::RAW_C, &maps.C, bar, 0, l0, b);
                }
                tma_load_3d(st + Cfg::RAW_X, &maps.x, bar, d0, lx, b);
                tma_load_3d(st + Cfg::RAW_DT, &maps.dt, bar, d0, l0, b);
                if (has_z) tma_load_3d(st + Cfg::RAW_Z, &maps.z, bar, d0, l0, b);
            } else {                          // maps over (t, channel, batch)
                if (!SB) {
                    tma_load_3d(st + Cfg::RAW_B, &maps.B, bar, l0, 0, b);
                    tma_load_3d(st + Cfg::RAW_C, &maps.C, bar, l0, 0, b);
                }
                tma_load_3d(st + Cfg::RAW_X, &maps.x, bar, lx, d0, b);
                tma_load_3d(st + Cfg::RAW_DT, &maps.dt, bar, l0, d0, b);
                if (has_z) tma_load_3d(st + Cfg::RAW_Z, &maps.z, bar, l0, d0, b);
            }
        };

        // Plain-load fallback (any alignment or stride): fills stage 0 with the layout
        // the TMA path gives.
        auto load_plain_cl = [&](int f) {
            uint8_t* st = smem;
            const int l0 = tile_l0(f);
            const bool rv = tile_rev(f);
            const int64_t bL = (int64_t)b * L;
            for (int e = ptid; e < (SB ? 0 : NS * TT); e += Cfg::PRO_THREADS) {
                const int n = e % NS, row = e / NS, t = l0 + row;
                const bool ok = n < p.dstate && t >= 0 && t < L;
                reinterpret_cast<T*>(st + Cfg::RAW_B)[e] =
                    ok ? static_cast<const T*>(p.Bm)[(bL + t) * p.sB + n] : T(0.f);
                reinterpret_cast<T*>(st + Cfg::RAW_C)[e] =
                    ok ? static_cast<const T*>(p.Cm)[(bL + t) * p.sC + n] : T(0.f);
            }
            const int xrows = xpitch / (int)sizeof(T);
            const int xs = (conv && !rv) ? l0 - HALO : l0;
            const int hw = conv ? p.conv_width - 1 : 0;      // history length
            for (int e = ptid; e < G * xrows; e += Cfg::PRO_THREADS) {
                const int r = e % G, row = e / G, t = xs + row, dd = d0 + r;
                const bool ok = dd < p.dim && t >= 0 && t < L;
                const bool hist = p.conv_hist && !rv && dd < p.dim && t < 0 && t >= -hw;
                const int64_t hi = ((int64_t)b * p.dim + dd) * hw + hw + t;
                reinterpret_cast<T*>(st + Cfg::RAW_X)[e] =
                    ok ? static_cast<const T*>(p.u)[(bL + t) * p.su + dd]
                       : (hist ? static_cast<const T*>(p.conv_hist)[hi] : T(0.f));
            }
            for (int e = ptid; e < G * TT; e += Cfg::PRO_THREADS) {
                const int r = e % G, row = e / G, t = l0 + row, dd = d0 + r;
                const bool ok = dd < p.dim && t >= 0 && t < L;
                reinterpret_cast<T*>(st + Cfg::RAW_DT)[e] =
                    ok ? static_cast<const T*>(p.delta)[(bL + t) * p.sdl + dd] : T(0.f);
                if (has_z)
                    reinterpret_cast<T*>(st + Cfg::RAW_Z)[e] =
                        ok ? static_cast<const T*>(p.z)[(bL + t) * p.sz + dd] : T(0.f);
            }
        };
        auto load_plain = [&](int f) {
            if constexpr (CL) { load_plain_cl(f); return; }
            uint8_t* st = smem;
            const int l0 = tile_l0(f);
            const bool rv = tile_rev(f);
            const T* gB = static_cast<const T*>(p.Bm) + (int64_t)b * p.dstate * L;
            const T* gC = static_cast<const T*>(p.Cm) + (int64_t)b * p.dstate * L;
            for (int e = ptid; e < (SB ? 0 : NS * TT); e += Cfg::PRO_THREADS) {
                const int n = e / TT, col = e % TT, t = l0 + col;
                const bool ok = n < p.dstate && t >= 0 && t < L;
                const int off = swz<ROWB, SWZ>(n, col * (int)sizeof(T));
                *reinterpret_cast<T*>(st + Cfg::RAW_B + off) = ok ? gB[(int64_t)n * L + t] : T(0.f);
                *reinterpret_cast<T*>(st + Cfg::RAW_C + off) = ok ? gC[(int64_t)n * L + t] : T(0.f);
            }
            const int xw = xpitch / (int)sizeof(T);
            const int xs = (conv && !rv) ? l0 - HALO : l0;
            const int hw = conv ? p.conv_width - 1 : 0;      // history length
            for (int e = ptid; e < G * xw; e += Cfg::PRO_THREADS) {
                const int r = e / xw, col = e % xw, t = xs + col, dd = d0 + r;
                const bool ok = dd < p.dim && t >= 0 && t < L;
                const int64_t gi = ((int64_t)b * p.dim + dd) * L + t;
                // positions before 0 read the caller's conv history, if any
                const bool hist = p.conv_hist && !rv && dd < p.dim && t < 0 && t >= -hw;
                const int64_t hi = ((int64_t)b * p.dim + dd) * hw + hw + t;
                reinterpret_cast<T*>(st + Cfg::RAW_X + r * xpitch)[col] =
                    ok ? static_cast<const T*>(p.u)[gi]
                       : (hist ? static_cast<const T*>(p.conv_hist)[hi] : T(0.f));
            }
            for (int e = ptid; e < G * TT; e += Cfg::PRO_THREADS) {
                const int r = e / TT, col = e % TT, t = l0 + col, dd = d0 + r;
                const bool ok = dd < p.dim && t >= 0 && t < L;
                const int64_t gi = ((int64_t)b * p.dim + dd) * L + t;
                const int off = Cfg::SWZDT ? swz<ROWB, SWZ>(r, col * (int)sizeof(T))
                                           : (r * TT + col) * (int)sizeof(T);
                *reinterpret_cast<T*>(st + Cfg::RAW_DT + off) =
                    ok ? static_cast<const T*>(p.delta)[gi] : T(0.f);
                if (has_z)
                    *reinterpret_cast<T*>(st + Cfg::RAW_Z + off) =
                        ok ? static_cast<const T*>(p.z)[gi] : T(0.f);
            }
        };

        // Packed sequences: the starts at positions [l0 - HALO, l0 + TT] of (forward) tile f
        // as a bit mask (one thread).
        auto stage_starts = [&](int f, uint8_t* buf) {
            const int l0 = tile_l0(f);
            const int lo = l0 - HALO;
            int a = 0, z = p.nseq;                    // first i with cu[i] >= lo
            while (a < z) {
                const int m = (a + z) >> 1;
                if (p.cu[m] < lo) a = m + 1; else z = m;
            }
            typename Cfg::Mask wm = 0;
            for (int i = a; i <= p.nseq && i < a + 2 * (TT + HALO + 2); ++i) {
                const int s = p.cu[i];
                if (s > l0 + TT) break;
                if (s >= lo) wm |= typename Cfg::Mask(1) << (s - lo);
            }
            *reinterpret_cast<typename Cfg::Mask*>(buf + Cfg::BUF_META) = wm;
        };

        // Raw stage `st` of tile f -> staging buffer `buf`. Each producer thread owns a
        // segment of SEG consecutive steps of one channel row: it reads its window of x
        // (with the conv history), dt and z with 16-byte loads, keeps the channel's
        // parameters in registers, and works through SEG/2 independent step pairs.
        auto prologue = [&](auto rv_tag, auto conv_tag, int f, const uint8_t* st, uint8_t* buf) {
            constexpr bool RV = decltype(rv_tag)::value;
            constexpr bool CONV = decltype(conv_tag)::value;
            constexpr int EPC = 16 / (int)sizeof(T);          // elements per 16-byte chunk
            // steps per producer thread: whole 16-byte chunks, at least one (then not every
            // thread has a segment)
            constexpr int PER = TT * G / Cfg::PRO_THREADS;
            constexpr int SEG = PER <= EPC ? EPC : (PER + EPC - 1) / EPC * EPC;
            static_assert(TT % SEG == 0 && TT * G / SEG <= Cfg::PRO_THREADS, "segments tile the tile");
            [[maybe_unused]] constexpr int NSEG = TT * G / SEG;   // segments per tile
            constexpr int SUB = 2 * EPC < SEG ? 2 * EPC : SEG;  // steps per register window
            constexpr int NC = SUB / EPC;                     // dt / z chunks per window
            constexpr int NXC = CONV ? NC + 1 : NC;           // x chunks (+ the conv history)
            static_assert(SEG % SUB == 0 && SUB % EPC == 0 && SUB % 2 == 0, "windows of whole chunks");
            // B, C: swizzled [n][t] -> fp32 [t][n] (channel-last: already [t][n], widened
            // only), one 16-byte chunk per thread and pass
            [[maybe_unused]] constexpr int NCH = NS * ROWB / 16;   // chunks per tensor
            if constexpr (SB) {
                // time-invariant B/C: nothing staged per tile
            } else if constexpr (CL) {
                for (int e = ptid; e < 2 * NCH; e += Cfg::PRO_THREADS) {
                    const int ten = e / NCH, ch = e % NCH;
                    const uint4 v[1] = {reinterpret_cast<const uint4*>(
                        st + (ten ? Cfg::RAW_C : Cfg::RAW_B))[ch]};
                    // chunk ch holds positions ch * EPC .. + EPC - 1 of the [t][n] tile
                    const int t = ch * EPC / NS, n0 = ch * EPC % NS;
                    float* dst = reinterpret_cast<float*>(buf + (ten ? Cfg::BUF_CT : Cfg::BUF_BT)) +
                                 Cfg::bc_row(t) * Cfg::BCP + n0;
                    if constexpr (Cfg::BCP == NS) {
#pragma unroll
                        for (int m = 0; m < EPC; m += 4)
                            *reinterpret_cast<float4*>(dst + m) =
                                make_float4(chunk_elem<T>(v, m), chunk_elem<T>(v, m + 1),
                                            chunk_elem<T>(v, m + 2), chunk_elem<T>(v, m + 3));
                    } else {
#pragma unroll
                        for (int m = 0; m < EPC; m += 2)
                            *reinterpret_cast<float2*>(dst + m) =
                                make_float2(chunk_elem<T>(v, m), chunk_elem<T>(v, m + 1));
                    }
                }
            } else {
                // (braced: with an unbraced loop as the discarded branch, nvcc 12.9 also
                // dropped the statement after it, the early return below)
                for (int e = ptid; e < 2 * NCH; e += Cfg::PRO_THREADS) {
                    const int ten = e / NCH, ch = e % NCH;
                    const int n = ch % NS, c0 = (ch / NS) * EPC;
                    const uint8_t* src = st + (ten ? Cfg::RAW_C : Cfg::RAW_B) +
                                         swz<ROWB, SWZ>(n, c0 * (int)sizeof(T));
                    const uint4 v[1] = {*reinterpret_cast<const uint4*>(src)};
                    float* dst =
                        reinterpret_cast<float*>(buf + (ten ? Cfg::BUF_CT : Cfg::BUF_BT)) + c0 * Cfg::BCP + n;
                    const int k = (c0 / EPC) & (Cfg::BCW - 1);   // rows c0 + m land at c0 + (m ^ k)
#pragma unroll
                    for (int m = 0; m < EPC; ++m) dst[(m ^ k) * Cfg::BCP] = chunk_elem<T>(v, m);
                }
            }
            if (NSEG < Cfg::PRO_THREADS && ptid >= NSEG) return;
            const int r = ptid % G;                           // channel row
            const int t0 = (ptid / G) * SEG;                  // first step of the segment
            const uint4* q4 = reinterpret_cast<const uint4*>(par + (tile_dir(f) * G + r) * 16);
            const uint4 qa = q4[0], qb = q4[1], qc = q4[2], qd = q4[3];
            // duplicated pairs: {w0,w0} {w1,w1} {w2,w2} {w3,w3} {cb,cb} {bias,bias} {D,D}
            const uint64_t w2[4] = {pk2(__uint_as_float(qa.x), __uint_as_float(qa.y)),
                                    pk2(__uint_as_float(qa.z), __uint_as_float(qa.w)),
                                    pk2(__uint_as_float(qb.x), __uint_as_float(qb.y)),
                                    pk2(__uint_as_float(qb.z), __uint_as_float(qb.w))};
            const uint64_t cb2 = pk2(__uint_as_float(qc.x), __uint_as_float(qc.y));
            const uint64_t bias2 = pk2(__uint_as_float(qc.z), __uint_as_float(qc.w));
            const uint64_t D2 = pk2(__uint_as_float(qd.x), __uint_as_float(qd.y));
            [[maybe_unused]] const float aH = __uint_as_float(qd.z);   // SA: A_h log2(e)
            // P rows hold KC channels side by side: this channel's {delta, delta*u} slot
            uint8_t* prow_base = buf + Cfg::BUF_P + (r / KC) * Cfg::P_PITCH + (r % KC) * 8;
            // packed sequences: the conv of step ti reads no position before its start
            const typename Cfg::Mask wm =
                VL ? *reinterpret_cast<const typename Cfg::Mask*>(buf + Cfg::BUF_META) : 0;
            // first tap at or after the start for step s0 + i of the window, from the
            // window's slice of the mask (bit m <-> position s0 - 3 + m; SUB + 3 <= 32)
            static_assert(2 * EPC + 3 <= 32, "a register window's starts fit 32 bits");
            auto first_tap = [&](uint32_t wwin, int i) {
                const uint32_t w4 = (wwin >> i) & 0xFu;
                return w4 ? 31 - __clz(w4) : 0;
            };
#pragma unroll
            for (int s0 = t0; s0 < t0 + SEG; s0 += SUB) {
                [[maybe_unused]] const uint32_t wwin = VL ? (uint32_t)(wm >> (HALO + s0 - 3)) : 0u;
                // x window: row elements [s0, s0 + NXC*EPC). Forward rows start HALO steps
                // before the tile (the conv history), reverse rows end HALO steps after it.
                const uint4* xs = reinterpret_cast<const uint4*>(
                    st + Cfg::RAW_X + r * (CONV ? Cfg::X_PITCH_MAX : ROWB) + s0 * (int)sizeof(T));
                // 16-byte chunk c2 of the window in the delta / z rows (swizzled or not)
                auto dz_off = [&](int c2) {
                    const int byte = s0 * (int)sizeof(T) + c2 * 16;
                    return Cfg::SWZDT ? swz<ROWB, SWZ>(r, byte) : r * ROWB + byte;
                };
                [[maybe_unused]] uint4 xw[NXC], dw[NC], zw[NC];
                if constexpr (!CL) {
#pragma unroll
                    for (int c2 = 0; c2 < NXC; ++c2) xw[c2] = xs[c2];
#pragma unroll
                    for (int c2 = 0; c2 < NC; ++c2) {
                        dw[c2] = *reinterpret_cast<const uint4*>(st + Cfg::RAW_DT + dz_off(c2));
                        zw[c2] = has_z ? *reinterpret_cast<const uint4*>(st + Cfg::RAW_Z + dz_off(c2))
                                       : make_uint4(0, 0, 0, 0);
                    }
                }
                // element a of the window (raw row s0 + a of the channel): from the
                // registers, or (channel-last) a strided load from the [t][channel] tile
                const T* cx = reinterpret_cast<const T*>(st + Cfg::RAW_X) + r;
                const T* cd = reinterpret_cast<const T*>(st + Cfg::RAW_DT) + r;
                const T* cz = reinterpret_cast<const T*>(st + Cfg::RAW_Z) + r;
                auto X = [&](int a) {
                    if constexpr (CL) return E::to_f(cx[(s0 + a) * G]);
                    else return chunk_elem<T>(xw, a);
                };
                auto DT = [&](int a) {
                    if constexpr (CL) return E::to_f(cd[(s0 + a) * G]);
                    else return chunk_elem<T>(dw, a);
                };
                auto ZV = [&](int a) {
                    if constexpr (CL) return E::to_f(cz[(s0 + a) * G]);
                    else return chunk_elem<T>(zw, a);
                };
                uint8_t* prow = prow_base + s0 * KC * 8;
                uint8_t* erow = buf + Cfg::BUF_E + r * Cfg::E_PITCH + s0 * 8;
#pragma unroll
                for (int i = 0; i < SUB; i += 2) {           // steps s0 + i, s0 + i + 1
                    uint64_t u2;
                    if constexpr (CONV) {
                        // forward: u_t = sum_k w_k x[t-3+k]; reverse: u_t = sum_k w_k x[t+3-k]
                        uint64_t acc = cb2;
                        const int fa = VL ? first_tap(wwin, i) : 0, fb = VL ? first_tap(wwin, i + 1) : 0;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int a = RV ? i + 3 - k : HALO + i - 3 + k;
                            float xa = X(a), xb = X(a + 1);
                            if (VL) {
                                xa = k >= fa ? xa : 0.f;
                                xb = k >= fb ? xb : 0.f;
                            }
                            acc = fma2(w2[k], pk2(xa, xb), acc);
                        }
                        u2 = Cfg::SILU_FMA ? silu2_fma<sizeof(T) == 2 ? 2 : 3>(acc) : silu2(acc);
                    } else {
                        u2 = pk2(X(i), X(i + 1));
                    }
                    uint64_t dl2 = add2(pk2(DT(i), DT(i + 1)), bias2);
                    if (p.softplus) dl2 = softplus2(dl2);
                    float2 dl = upk2(dl2);
                    const float2 du = upk2(mul2(dl2, u2));
                    if (SA) dl = make_float2(ex2(dl.x * aH), ex2(dl.y * aH));   // the decay
                    if constexpr (KC == 1) {
                        *reinterpret_cast<float4*>(prow + i * 8) = make_float4(dl.x, du.x, dl.y, du.y);
                    } else {
                        *reinterpret_cast<float2*>(prow + i * KC * 8) = make_float2(dl.x, du.x);
                        *reinterpret_cast<float2*>(prow + (i + 1) * KC * 8) = make_float2(dl.y, du.y);
                    }
                    if (!SUMMARY) {
                        uint64_t g2 = pk2(1.f, 1.f);
                        if (has_z) {
                            const uint64_t z2 = pk2(ZV(i), ZV(i + 1));
                            g2 = Cfg::SILU_FMA ? silu2_fma<sizeof(T) == 2 ? 2 : 3>(z2) : silu2(z2);
                        }
                        const float2 g = upk2(g2), dv = upk2(mul2(D2, u2));
                        *reinterpret_cast<float4*>(erow + i * 8) = make_float4(dv.x, g.x, dv.y, g.y);
                    }
                }
            }
        };

        if (USE_TMA && ptid == 0) {
            prefetch_tensormap(&maps.x);
            prefetch_tensormap(&maps.dt);
            prefetch_tensormap(&maps.B);
            prefetch_tensormap(&maps.C);
            if (has_z) prefetch_tensormap(&maps.z);
            for (int f = 0; f < min(NSTAGE, nt); ++f) issue(f);
        }
        for (int f = 0; f < nt; ++f) {
            // Lane 0 of each warp polls (bounded); then every lane observes the completed
            // phase itself with one try_wait, acquiring the writes it guards. A phase
            // cannot move on before this warp's own part in the next round, so the
            // parity test is unambiguous.
            bool ok = true;
            if (f >= Cfg::NBUF) {     // the scan warps are done with this buffer (tile f - 2)
                const uint32_t par_e = ((f - Cfg::NBUF) / Cfg::NBUF) & 1;
                if (lane == 0) ok = mbar_wait_bounded(&empty_buf[f & 1], par_e);
                __syncwarp();
                if (lane != 0) mbar_try_wait(&empty_buf[f & 1], par_e);
            }
            const uint8_t* st = smem;
            if (USE_TMA) {
                const uint32_t par_r = (f / NSTAGE) & 1;
                if (lane == 0 && ok) ok = mbar_wait_bounded(&full_raw[f % NSTAGE], par_r);
                __syncwarp();
                if (lane != 0) mbar_try_wait(&full_raw[f % NSTAGE], par_r);
                st = smem + (f % NSTAGE) * Cfg::STAGE;
                // The first forward tile's conv halo (positions < 0) landed as zeros;
                // a continued sequence puts the caller's history there.
                if (conv && p.conv_hist && p.mode == 0 && chunk == 0 && f == 0)
                    put_conv_history<T, G, HALO, Cfg::PRO_THREADS, CL>(p, smem + Cfg::RAW_X, xpitch,
                                                                   ptid, b, d0);
            } else {
                // stage 0 was released by every producer at the end of tile f - 1
                load_plain(f);
            }
            if (VL && ptid == 0) stage_starts(f, buf_of(f));
            // one decision for all producers (this is also the barrier that orders the
            // plain loads and the start mask before the prologue): leave together if a
            // wait ran out
            if (named_bar_or(kProBarrier, Cfg::PRO_THREADS, !ok)) {
                if (USE_TMA && ptid == 0)     // drain the copies still in flight (bounded)
                    for (int g2 = f; g2 < min(f + NSTAGE, nt); ++g2)
                        mbar_wait_bounded(&full_raw[g2 % NSTAGE], (g2 / NSTAGE) & 1);
                return;
            }
            if (conv) {
                if (tile_rev(f)) prologue(TrueT{}, TrueT{}, f, st, buf_of(f));
                else prologue(FalseT{}, TrueT{}, f, st, buf_of(f));
            } else {
                if (tile_rev(f)) prologue(TrueT{}, FalseT{}, f, st, buf_of(f));
                else prologue(FalseT{}, FalseT{}, f, st, buf_of(f));
            }
            mbar_arrive(&full_buf[f & 1]);
            named_bar_sync(kProBarrier, Cfg::PRO_THREADS);   // every producer is done with the stage
            if (USE_TMA && ptid == 0 && f + NSTAGE < nt) issue(f + NSTAGE);
        }
        return;
    }

    // =============================================================== scan warps ==
    const int lg = tid / S;         // lane group: channels lg*KC .. lg*KC + KC - 1 of the CTA
    const int j = tid % S;          // state group of this lane
    auto chan_d = [&](int k) { return d0 + lg * KC + k; };                 // channel k of the lane
    auto chan_row = [&](int k) { return (int64_t)b * p.dim + chan_d(k); };  // its (b, d) row
    // The state in slot i of this lane. With NP a multiple of 4 the lanes interleave in
    // groups of 4 states, so that a quarter warp's 16-byte B/C loads are contiguous
    // (NP = 8 with lanes owning 8 consecutive states would put lanes j and j + 4 on the
    // same banks); otherwise lane j owns states j*NP .. j*NP + NP - 1.
    auto state_n = [&](int i) {
        return NP % 4 == 0 ? (i >> 2) * (4 * S) + 4 * j + (i & 3) : j * NP + i;
    };

    LaneState<NP, SUMMARY, SA> ls[KC];
    auto load_A = [&](int dir) {
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            const int d = chan_d(k);
            float a[NP];
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                const int n = state_n(i);
                a[i] = (!SA && d < p.dim && n < p.dstate)
                           ? p.A[dir][(int64_t)d * p.dstate + n] * kLog2e : 0.f;
            }
            ls[k].set_a(a);
        }
    };
    // SB: the lane's NP values of its channel's fixed B and C rows, for every step
    [[maybe_unused]] float sb_b[NP], sb_c[NP];
    if constexpr (SB) {
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            const int n = state_n(i);
            const bool ok = chan_d(0) < p.dim && n < p.dstate;
            const int64_t o = (int64_t)chan_d(0) * p.dstate + n;
            sb_b[i] = ok ? static_cast<const float*>(p.Bm)[o] : 0.f;
            sb_c[i] = ok ? static_cast<const float*>(p.Cm)[o] : 0.f;
        }
    }
    // Initial state of this chunk: carry over the summaries of earlier chunks.
    // A caller's initial state (a continued sequence) is the carry into chunk 0.
    auto init_state = [&]() {
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            ls[k].reset();
            if (!SUMMARY && ((chunk > 0 && !p.seq_aligned) || p.h0) && chan_d(k) < p.dim) {
                float hv[NP];
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    const int n = state_n(i);
                    hv[i] = (p.h0 && n < p.dstate) ? p.h0[chan_row(k) * p.dstate + n] : 0.f;
                }
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

    // gate, skip term, bidirectional partial and the store of R owned outputs of the
    // lane's channel k
    auto epilogue = [&](const uint8_t* buf, int k, const float* acc, bool rv, int dir, int l0,
                        int pos0, int nown, int nskip) {
        const float2* Erow =
            reinterpret_cast<const float2*>(buf + Cfg::BUF_E + (lg * KC + k) * Cfg::E_PITCH);
        float yv[R];
#pragma unroll
        for (int m = 0; m < R; ++m) {
            const int ii = pos0 + m;
            const int tt = rv ? TT - 1 - ii : ii;
            const float2 e = Erow[tt];
            yv[m] = (acc[m] + e.x) * e.y;
        }
        if (chan_d(k) >= p.dim || nown <= nskip) return;
        const int tmin = rv ? l0 + TT - 1 - (pos0 + R - 1) : l0 + pos0;
        float ya[R];                                      // time-ascending order
#pragma unroll
        for (int m = 0; m < R; ++m) ya[m] = rv ? yv[R - 1 - m] : yv[m];
        // valid ascending index range: forward [0, nown); reverse [R - nown, R)
        const int mlo = rv ? R - nown : nskip;   // (nskip: forward packed sequences only)
        const int mhi = rv ? R : nown;
        const int64_t gbase = chan_row(k) * L + tmin;
        // channel-last: position t of channel d at (b*L + t) * stride + d
        const int64_t cbase = (int64_t)b * L + tmin;
        auto pidx = [&](int m) {
            if constexpr (CL) return (cbase + m) * p.spart + chan_d(k);
            else return gbase + m;
        };
        if (p.mode == 2 && dir == 1) {
#pragma unroll
            for (int m = 0; m < R; ++m)
                if (m >= mlo && m < mhi) ya[m] += p.partial[pidx(m)];
        }
        if (p.mode == 2 && dir == 0) {
#pragma unroll
            for (int m = 0; m < R; ++m)
                if (m >= mlo && m < mhi) p.partial[pidx(m)] = ya[m];
            return;
        }
        if constexpr (CL) {
            T* oc = static_cast<T*>(p.out) + chan_d(k);
#pragma unroll
            for (int m = 0; m < R; ++m)
                if (m >= mlo && m < mhi) oc[(cbase + m) * p.sout] = E::from_f(ya[m]);
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

    // One tile in scan order from staging buffer `buf`. RV: walk time downwards.
    // FULL: all TT steps valid (no per-step predicate; shared-memory offsets are
    // compile-time constants).
    auto scan_tile = [&](auto rv_tag, auto full_tag, int f, const uint8_t* buf) {
        constexpr bool RV = decltype(rv_tag)::value;
        constexpr bool FULL = decltype(full_tag)::value;
        const int dir = tile_dir(f);
        const int i0 = cs + (f % ntl) * TT;
        const int nvalid = FULL ? TT : min(TT, ce - i0);
        const int vlo = (!FULL && f % ntl == 0) ? vbeg : 0;   // leading steps of another chunk
        const int l0 = RV ? L - i0 - TT : i0;
        const uint8_t* Prow = buf + Cfg::BUF_P + lg * Cfg::P_PITCH;
        // packed sequences: bit tt <-> step tt starts / ends a sequence
        const typename Cfg::Mask wm =
            VL ? *reinterpret_cast<const typename Cfg::Mask*>(buf + Cfg::BUF_META) : 0;
        using Steps = typename Cfg::Steps;
        const Steps starts = (Steps)(wm >> HALO), ends = (Steps)(wm >> (HALO + 1));
        // a sequence ended at step tt: its final state (the sequence is the last one whose
        // start is <= l0 + tt; empty sequences share their successor's start)
        auto seq_end = [&](int tt) {
            const int t = l0 + tt;
            int q = 0, r = p.nseq - 1;
            while (q < r) {
                const int m = (q + r + 1) >> 1;
                if (p.cu[m] <= t) q = m; else r = m - 1;
            }
#pragma unroll
            for (int k = 0; k < KC; ++k) {
                if (chan_d(k) >= p.dim || !p.final_state[0]) continue;
                float* fs = p.final_state[0] + ((int64_t)q * p.dim + chan_d(k)) * p.dstate;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    const int n = state_n(i);
                    if (n < p.dstate) fs[n] = ls[k].get(i);
                }
            }
        };
        // this lane's first B/C value of a step (its slot 0; see state_n)
        constexpr int kLaneOff = NP % 4 == 0 ? 4 : NP;
        [[maybe_unused]] const float* Bl =
            reinterpret_cast<const float*>(buf + Cfg::BUF_BT) + j * kLaneOff;
        [[maybe_unused]] const float* Cl =
            reinterpret_cast<const float*>(buf + Cfg::BUF_CT) + j * kLaneOff;
        // {delta, delta*u} of step tt for the lane's KC channels
        auto load_p = [&](int tt, float2 (&pd)[KC]) {
            if constexpr (KC == 2) {
                const float4 v = *reinterpret_cast<const float4*>(Prow + tt * 16);
                pd[0] = make_float2(v.x, v.y);
                pd[1] = make_float2(v.z, v.w);
            } else {
                pd[0] = *reinterpret_cast<const float2*>(Prow + tt * 8);
            }
        };
        // this lane's NP values of B and C at step tt
        auto load_bc = [&](int tt, float (&bv)[NP], float (&cv)[NP]) {
            if constexpr (SB) {
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    bv[i] = sb_b[i];
                    cv[i] = sb_c[i];
                }
            } else if constexpr (NP % 4 == 0) {
#pragma unroll
                for (int i = 0; i < NP; i += 4) {
                    const int o = Cfg::bc_row(tt) * Cfg::BCP + (i >> 2) * (4 * S);   // slots i .. i + 3
                    const float4 b4 = *reinterpret_cast<const float4*>(Bl + o);
                    bv[i] = b4.x; bv[i + 1] = b4.y; bv[i + 2] = b4.z; bv[i + 3] = b4.w;
                    if (!SUMMARY) {
                        const float4 c4 = *reinterpret_cast<const float4*>(Cl + o);
                        cv[i] = c4.x; cv[i + 1] = c4.y; cv[i + 2] = c4.z; cv[i + 3] = c4.w;
                    }
                }
            } else if constexpr (NP == 2) {
                const float2 b2 = *reinterpret_cast<const float2*>(Bl + Cfg::bc_row(tt) * Cfg::BCP);
                bv[0] = b2.x; bv[1] = b2.y;
                if (!SUMMARY) {
                    const float2 c2 = *reinterpret_cast<const float2*>(Cl + Cfg::bc_row(tt) * Cfg::BCP);
                    cv[0] = c2.x; cv[1] = c2.y;
                }
            } else {
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    bv[i] = Bl[Cfg::bc_row(tt) * Cfg::BCP + i];
                    if (!SUMMARY) cv[i] = Cl[Cfg::bc_row(tt) * Cfg::BCP + i];
                }
            }
        };
#pragma unroll 1
        for (int blk = 0; blk < TT / 16; ++blk) {
            if (!FULL && blk * 16 >= nvalid) break;
            float acc[KC][16];
            if (FULL) {
                // KB steps at a time: their state-independent operands (shared-memory
                // loads, delta*A, the SFU exps, delta*u*B) are all prepared first, then
                // the KB x KC independent state updates run. The packed-sequence kernels
                // take one step at a time (measured 11 % faster there; the same elsewhere,
                // slower with A per head).
                constexpr int KB = VL ? 1 : SSM_SCAN_BATCH;
#pragma unroll
                for (int q0 = 0; q0 < 16; q0 += KB) {
                    typename LaneState<NP, SUMMARY, SA>::In in[KB][KC];
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
                    for (int u = 0; u < KB; ++u) {
                        const int tt = RV ? TT - 1 - (blk * 16 + q0 + u) : blk * 16 + q0 + u;
                        if (VL && ((starts >> tt) & 1u)) {
#pragma unroll
                            for (int k = 0; k < KC; ++k) ls[k].cut();
                        }
#pragma unroll
                        for (int k = 0; k < KC; ++k) acc[k][q0 + u] = ls[k].update(in[u][k]);
                        if (VL && !SUMMARY && ((ends >> tt) & 1u)) seq_end(tt);
                    }
                }
            } else {
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int ii = blk * 16 + q;
                    const int tt = RV ? TT - 1 - ii : ii;
#pragma unroll
                    for (int k = 0; k < KC; ++k) acc[k][q] = 0.f;
                    if (ii < nvalid && ii >= vlo) {
                        float2 pd[KC];
                        float bv[NP], cv[NP];
                        load_p(tt, pd);
                        load_bc(tt, bv, cv);
                        if (VL && ((starts >> tt) & 1u)) {
#pragma unroll
                            for (int k = 0; k < KC; ++k) ls[k].cut();
                        }
#pragma unroll
                        for (int k = 0; k < KC; ++k)
                            acc[k][q] = ls[k].update(ls[k].prep(pd[k].x, pd[k].y, bv, cv));
                        if (VL && !SUMMARY && ((ends >> tt) & 1u)) seq_end(tt);
                    }
                }
            }
            if (SUMMARY) continue;
            const int pos0 = blk * 16 + j * R;
#pragma unroll
            for (int k = 0; k < KC; ++k) {
                reduce_block(acc[k]);
                epilogue(buf, k, acc[k], RV, dir, l0, pos0,
                         FULL ? R : max(0, min(R, nvalid - pos0)), FULL ? 0 : max(0, vlo - pos0));
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
            } else if (!VL && chunk == p.nchunks - 1 && p.final_state[dir]) {
                float* fs = p.final_state[dir] + row * p.dstate;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    const int n = state_n(i);
                    if (n < p.dstate) fs[n] = ls[k].get(i);
                }
            }
        }
    };

    load_A(0);
    init_state();
    for (int f = 0; f < nt; ++f) {
        if (p.mode == 2 && f == ntl) {       // second direction of the bidirectional sum
            finish_direction(0);
            load_A(1);
#pragma unroll
            for (int k = 0; k < KC; ++k) ls[k].reset();
        }
        // wait for the staging buffer of tile f (same polling scheme as the producers);
        // a warp whose wait ran out leaves, and the producers then run out of time on
        // the buffer it never releases
        const uint32_t par_f = (f / Cfg::NBUF) & 1;
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&full_buf[f & 1], par_f);
        if (__any_sync(0xffffffffu, !ok)) return;
        if (lane != 0) mbar_try_wait(&full_buf[f & 1], par_f);
        const uint8_t* buf = buf_of(f);
        const bool rv = tile_rev(f);
        const bool full = cs + (f % ntl) * TT + TT <= ce && !(f % ntl == 0 && vbeg > 0);
        if (full) {
            if (rv) scan_tile(TrueT{}, TrueT{}, f, buf);
            else scan_tile(FalseT{}, TrueT{}, f, buf);
        } else {
            if (rv) scan_tile(TrueT{}, FalseT{}, f, buf);
            else scan_tile(FalseT{}, FalseT{}, f, buf);
        }
        mbar_arrive(&empty_buf[f & 1]);      // the producers may refill it with tile f + 2
    }
    finish_direction(p.mode == 2 ? 1 : 0);
}

}  // namespace ssm
