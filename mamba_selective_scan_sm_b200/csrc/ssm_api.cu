// C ABI of the library (include/ssm.h): argument validation, variant choice,
// TMA descriptor encoding and kernel launch. Nothing here allocates, frees or
// synchronises (except ssm_device_error, which documents it).
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/ssm.h"
#include "launch.h"
#include "scan_params.h"

namespace {

thread_local std::string g_detail;

ssm_status_t fail(ssm_status_t s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_detail = buf;
    return s;
}

ssm_status_t ok() {
    g_detail.clear();
    return SSM_OK;
}

ssm_status_t cuda_fail(cudaError_t e, const char* what) {
    return fail(SSM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int elem_size(ssm_dtype_t t) { return t == SSM_BF16 ? 2 : 4; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    auto x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// ------------------------------------------------------------ TMA encoding --

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D tile map over a row-major (d2, d1, d0) tensor, d0 innermost.
bool encode_3d(CUtensorMap* map, int es, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
               uint32_t b0, uint32_t b1, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                    3, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D tile map with explicit byte strides of dims 1 and 2 (dim 0 innermost, dense).
bool encode_3d_strided(CUtensorMap* map, int es, const void* ptr, uint64_t d0, uint64_t d1,
                       uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1,
                       CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1, stride2};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                    3, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------- scan plan --

struct ScanPlan {
    ssm::ScanVariant v;
    int mode;            // 0 fwd, 1 rev, 2 bidir
    int nchunks;
    int chunk_len;
    size_t summary_bytes;
    size_t partial_bytes;
    size_t workspace;
};

int env_int(const char* name, int dflt) {
    const char* s = std::getenv(name);
    return s ? std::atoi(s) : dflt;
}

// SMs of a B200 (the automatic chunk count sizes the grid against them).
constexpr int kNumSMs = 148;

ssm_status_t plan_scan(const ssm_scan_args_t* a, ScanPlan* pl) {
    if (!a) return fail(SSM_ERR_NULL_ARG, "args is NULL");
    if (a->dtype != SSM_F32 && a->dtype != SSM_BF16)
        return fail(SSM_ERR_BAD_DTYPE, "dtype %d is not SSM_F32 or SSM_BF16", (int)a->dtype);
    if (a->batch < 0 || a->dim < 0 || a->seqlen < 0)
        return fail(SSM_ERR_BAD_SHAPE, "negative size (batch %lld, dim %lld, seqlen %lld)",
                    (long long)a->batch, (long long)a->dim, (long long)a->seqlen);
    if (a->dstate < 1 || a->dstate > SSM_MAX_SCAN_DSTATE)
        return fail(SSM_ERR_BAD_SHAPE, "dstate %lld outside 1..%d", (long long)a->dstate,
                    SSM_MAX_SCAN_DSTATE);
    if (a->a_heads < 0 || (a->a_heads > 0 && a->dim % a->a_heads != 0))
        return fail(SSM_ERR_BAD_SHAPE, "a_heads %d must be 0 or divide dim %lld", a->a_heads,
                    (long long)a->dim);
    if (a->bc_shared != 0 && a->bc_shared != 1)
        return fail(SSM_ERR_BAD_SHAPE, "bc_shared %d is not 0 or 1", a->bc_shared);
    if ((a->a_heads > 0 || a->bc_shared) && a->seq_starts)
        return fail(SSM_ERR_UNSUPPORTED,
                    "packed sequences need per-state A and input-dependent B, C");
    if (a->seqlen > 0x3fffffffLL || a->dim > 0x3fffffffLL)
        return fail(SSM_ERR_BAD_SHAPE, "seqlen and dim must be below 2^30");
    if (a->batch > 65535) return fail(SSM_ERR_UNSUPPORTED, "batch %lld > 65535", (long long)a->batch);
    if (a->conv_weight && (a->conv_width < 1 || a->conv_width > SSM_MAX_CONV_WIDTH))
        return fail(SSM_ERR_BAD_SHAPE, "conv_width %d outside 1..%d", a->conv_width,
                    SSM_MAX_CONV_WIDTH);
    if (a->num_chunks < 0) return fail(SSM_ERR_BAD_SHAPE, "num_chunks %d < 0", a->num_chunks);
    const bool bidir = a->A_rev != nullptr;
    if (a->final_state_rev && !bidir)
        return fail(SSM_ERR_UNSUPPORTED, "final_state_rev needs A_rev (bidirectional)");
    if (bidir && a->num_chunks > 1)
        return fail(SSM_ERR_UNSUPPORTED, "the bidirectional sum runs as a single pass");
    const bool cont = a->initial_state || a->conv_history || a->conv_state_out;
    if (cont && (bidir || a->reverse))
        return fail(SSM_ERR_UNSUPPORTED,
                    "initial_state, conv_history and conv_state_out need a forward scan");
    if ((a->conv_history || a->conv_state_out) && !a->conv_weight)
        return fail(SSM_ERR_NULL_ARG, "conv_history / conv_state_out need conv_weight");
    if (a->channel_last) {
        struct { int64_t s, w; const char* n; } sd[] = {
            {a->stride_u, a->dim, "stride_u"}, {a->stride_delta, a->dim, "stride_delta"},
            {a->stride_z, a->dim, "stride_z"}, {a->stride_out, a->dim, "stride_out"},
            {a->stride_B, a->dstate, "stride_B"}, {a->stride_C, a->dstate, "stride_C"}};
        for (auto& x : sd)
            if (x.s != 0 && (x.s < x.w || x.s > (1ll << 40)))
                return fail(SSM_ERR_BAD_SHAPE, "%s %lld: 0 or at least %lld", x.n,
                            (long long)x.s, (long long)x.w);
    }
    if (a->seq_starts) {
        if (a->num_seqs < 1 || a->num_seqs > 0x3fffffff)
            return fail(SSM_ERR_BAD_SHAPE, "num_seqs %d < 1", a->num_seqs);
        if (a->batch != 1)
            return fail(SSM_ERR_UNSUPPORTED, "packed sequences need batch 1 (got %lld)",
                        (long long)a->batch);
        if (bidir || a->reverse || a->initial_state || a->conv_history)
            return fail(SSM_ERR_UNSUPPORTED,
                        "packed sequences: forward scans without initial state or history");
    }

    const int es = elem_size(a->dtype);
    const int ns = a->dstate <= 4    ? 4
                   : a->dstate <= 8  ? 8
                   : a->dstate <= 16 ? 16
                   : a->dstate <= 64 ? 64
                                     : 128;
    int np = 4, s = 4, kc = 1, sw = 4;
    if (ns > 16) {
        // d_state 64 / 128: 16 lanes per channel of 4 / 8 states, 8 channels per CTA; with
        // A per head (and input-dependent B, C) each lane serves two channels, which share
        // its B/C loads (16 channels per CTA). SSM_CHANNELS_PER_LANE=1 keeps one.
        s = 16;
        np = ns / 16;
        kc = (a->a_heads > 0 && !a->bc_shared) ? env_int("SSM_CHANNELS_PER_LANE", 2) : 1;
        if (kc != 1 && kc != 2) kc = 2;
        // d_state 128 with two channels per lane: the staged tiles take 127 KB per CTA of
        // 4 scan warps, so one CTA fits an SM; CTAs of 8 scan warps (32 channels) keep 10
        // warps per SM instead of 6 (SSM_SCAN_WARPS=4 keeps the smaller CTA)
        if (ns == 128 && kc == 2) sw = env_int("SSM_SCAN_WARPS", 8) == 4 ? 4 : 8;
    } else if (ns == 16) {
        // Batch rows with enough channels for two 32-channel CTAs per SM: bf16, 2 lanes
        // per channel (8 states each) in CTAs of 2 scan warps; fp32 (16-step tiles), 4
        // lanes per channel (4 states each) in CTAs of 4 scan warps (32 channels both).
        // Fewer channels: 8 lanes per channel (2 states each) in CTAs of 8 or 12
        // channels, for more CTAs and warps. SSM_LANES_PER_CHANNEL (2, 4, 8) and
        // SSM_CHANNELS_PER_LANE (1, 2) pick another compiled split.
        const bool wide = a->batch * a->dim >= 2 * 148 * 32;
        const int s_wide = a->dtype == SSM_BF16 ? 2 : 4;
        s = env_int("SSM_LANES_PER_CHANNEL", wide ? s_wide : 8);
        if (s != 2 && s != 4 && s != 8) s = wide ? s_wide : 8;
        // A per head and time-invariant B/C have kernels in the 4-lane split only
        if (s == 2 && (a->a_heads > 0 || a->bc_shared)) s = 4;
        kc = env_int("SSM_CHANNELS_PER_LANE", 1);
        if (kc != 1 && kc != 2) kc = 1;
        if (s == 2 || a->seq_starts || a->channel_last || a->a_heads > 0 || a->bc_shared)
            kc = 1;                                     // the splits compiled for those
        np = 16 / s;
        sw = s == 2 ? 2 : (s == 4) == (kc == 1) ? 4 : 2;
        if (s == 8 && kc == 1) {
            // 8 or 12 channels per CTA (2 or 3 scan warps), whichever leaves the busiest SM
            // the fewest channels when every CTA is resident (long: 640 CTAs of 8 put 40
            // channels on some SMs, 427 of 12 at most 36, against an average of 34.6)
            auto busiest = [&](int64_t g) {
                const int64_t ctas = a->batch * ((a->dim + g - 1) / g);
                return (ctas + kNumSMs - 1) / kNumSMs * g;
            };
            const int64_t env_sw = env_int("SSM_SCAN_WARPS", 0);
            sw = env_sw == 2 || env_sw == 3 ? (int)env_sw : busiest(12) < busiest(8) ? 3 : 2;
        }
    } else if (ns == 8) {
        np = 2;
    } else {
        np = 1;
    }
    if (!ssm::scan_variant(es, np, s, kc, sw, &pl->v))
        return fail(SSM_ERR_UNSUPPORTED, "no kernel for elem %d np %d s %d kc %d sw %d", es, np, s,
                    kc, sw);
    pl->mode = bidir ? 2 : (a->reverse ? 1 : 0);
    if (a->seq_starts) {                      // the packed-sequence kernels' tile and size
        pl->v.tile = pl->v.tile_vl;
        pl->v.smem_bytes = pl->v.smem_bytes_vl;
        pl->v.min_ctas = pl->v.min_ctas_vl;
    }

    const int tile = pl->v.tile;
    const int64_t ntiles = (a->seqlen + tile - 1) / tile;
    int nch = a->num_chunks;
    if (nch == 0) {
        // Automatic: when batch * dim gives too few CTAs to fill the SMs, split the
        // sequence into chunks (two-pass carry) until the grid does. The summary pass
        // costs about one more scan over all but the last chunk, so only a grid at most
        // half as large as the SMs' CTA slots is split. Not for the bidirectional sum
        // (one pass), nor when the final state overwrites the initial state.
        const int64_t ctas = (a->dim + pl->v.channels - 1) / pl->v.channels * a->batch;
        const int64_t slots = (int64_t)kNumSMs * pl->v.min_ctas;
        const size_t stb = (size_t)a->batch * a->dim * a->dstate * sizeof(float);
        const bool inplace = a->initial_state && a->final_state &&
                             overlap(a->final_state, stb, a->initial_state, stb);
        nch = 1;
        if (a->seq_starts) {
            // packed sequences: chunks begin at sequence starts and need no carry, so
            // they cost nothing extra: as many as fill the SMs' CTA slots once (more
            // waves only add the tail of the chunks' unequal lengths: B1 D1536 L32768 in
            // 42 sequences took 1.09 ms in 4 chunks, 1.38 in 8 and 1.41 in 64)
            if (ctas > 0) nch = (int)std::max<int64_t>(1, (slots + ctas - 1) / ctas);
        } else if (!bidir && !inplace && ctas > 0 && 2 * ctas <= slots) {
            nch = (int)std::min<int64_t>(slots / ctas, 16);
        }
    }
    if (nch > ntiles) nch = (int)(ntiles > 0 ? ntiles : 1);
    if (nch > 65535) nch = 65535;
    const int64_t tiles_per_chunk = ntiles > 0 ? (ntiles + nch - 1) / nch : 1;
    pl->chunk_len = (int)(tiles_per_chunk * tile);
    pl->nchunks = ntiles > 0 ? (int)((ntiles + tiles_per_chunk - 1) / tiles_per_chunk) : 1;

    const int64_t rows = a->batch * a->dim;
    // packed sequences: sequence-aligned chunks carry nothing (no summary pass)
    pl->summary_bytes = pl->nchunks > 1 && !a->seq_starts
                            ? (size_t)(pl->nchunks - 1) * rows * ns * sizeof(float) * 2
                            : 0;
    pl->partial_bytes = (bidir && a->dtype != SSM_F32) ? (size_t)rows * a->seqlen * 4 : 0;
    // layout: [summaries][pad to 256][bidirectional fp32 partial]
    pl->workspace = pl->partial_bytes ? ((pl->summary_bytes + 255) / 256) * 256 + pl->partial_bytes
                                      : pl->summary_bytes;
    return SSM_OK;
}

}  // namespace

void ssm::set_error_detail(const char* text) { g_detail = text ? text : ""; }

extern "C" {

int ssm_abi_version(void) { return SSM_ABI_VERSION; }

const char* ssm_status_string(ssm_status_t s) {
    switch (s) {
        case SSM_OK: return "ok";
        case SSM_ERR_NULL_ARG: return "a required pointer is NULL";
        case SSM_ERR_BAD_SHAPE: return "a size is out of range";
        case SSM_ERR_BAD_DTYPE: return "unknown dtype";
        case SSM_ERR_MISALIGNED: return "a pointer is not aligned to its element size";
        case SSM_ERR_WORKSPACE: return "workspace missing or too small";
        case SSM_ERR_UNSUPPORTED: return "unsupported combination of arguments";
        case SSM_ERR_CUDA: return "CUDA runtime error";
        case SSM_ERR_TIMEOUT: return "a kernel-side bounded wait ran out";
        case SSM_ERR_ALIAS: return "output overlaps an input";
    }
    return "unknown status";
}

const char* ssm_last_error_detail(void) { return g_detail.c_str(); }

ssm_status_t ssm_selective_scan_workspace_size(const ssm_scan_args_t* a, size_t* bytes) {
    if (!bytes) return fail(SSM_ERR_NULL_ARG, "bytes is NULL");
    ScanPlan pl;
    ssm_status_t st = plan_scan(a, &pl);
    if (st != SSM_OK) return st;
    *bytes = pl.workspace;
    return ok();
}

ssm_status_t ssm_selective_scan_fwd(const ssm_scan_args_t* a, ssm_stream_t stream) {
    ScanPlan pl;
    ssm_status_t st = plan_scan(a, &pl);
    if (st != SSM_OK) return st;
    const bool bidir = pl.mode == 2;
    const int es = elem_size(a->dtype);
    const int64_t rows = a->batch * a->dim;
    const bool cl = a->channel_last != 0;
    // channel-last element strides between positions (0 = dense)
    const int64_t su = cl ? (a->stride_u ? a->stride_u : a->dim) : 0;
    const int64_t sdl = cl ? (a->stride_delta ? a->stride_delta : a->dim) : 0;
    const int64_t sz = cl ? (a->stride_z ? a->stride_z : a->dim) : 0;
    const int64_t sout = cl ? (a->stride_out ? a->stride_out : a->dim) : 0;
    const bool sb = a->bc_shared != 0;            // B, C fp32 (dim, dstate), fixed per channel
    const int64_t sB = (cl && !sb) ? (a->stride_B ? a->stride_B : a->dstate) : 0;
    const int64_t sC = (cl && !sb) ? (a->stride_C ? a->stride_C : a->dstate) : 0;
    // bytes each tensor spans: (batch, dim, seqlen) dense, or batch*seqlen positions at
    // their stride, the last one `width` elements long
    const int64_t npos = a->batch * a->seqlen;
    auto span = [&](int64_t stride, int64_t width) -> size_t {
        return npos > 0 ? (size_t)((npos - 1) * stride + width) * es : 0;
    };
    const size_t act = (size_t)rows * a->seqlen * es;
    const size_t bc = (size_t)a->batch * a->dstate * a->seqlen * es;
    const size_t act_u = cl ? span(su, a->dim) : act, act_dl = cl ? span(sdl, a->dim) : act;
    const size_t act_z = cl ? span(sz, a->dim) : act, act_out = cl ? span(sout, a->dim) : act;
    const size_t bc_fixed = (size_t)a->dim * a->dstate * sizeof(float);
    const size_t bc_B = sb ? bc_fixed : cl ? span(sB, a->dstate) : bc;
    const size_t bc_C = sb ? bc_fixed : cl ? span(sC, a->dstate) : bc;
    const bool empty = rows == 0 || a->seqlen == 0;

    if (!empty) {
        struct { const void* p; const char* n; } req[] = {
            {a->u, "u"}, {a->delta, "delta"}, {a->A, "A"}, {a->B, "B"}, {a->C, "C"},
            {a->out, "out"}};
        for (auto& r : req)
            if (!r.p) return fail(SSM_ERR_NULL_ARG, "%s is NULL", r.n);
    }
    // element alignment
    struct { const void* p; size_t al; const char* n; } al[] = {
        {a->u, (size_t)es, "u"}, {a->delta, (size_t)es, "delta"}, {a->z, (size_t)es, "z"},
        {a->B, sb ? 4 : (size_t)es, "B"}, {a->C, sb ? 4 : (size_t)es, "C"},
        {a->out, (size_t)es, "out"},
        {a->A, 4, "A"}, {a->D, 4, "D"}, {a->delta_bias, 4, "delta_bias"},
        {a->conv_weight, 4, "conv_weight"}, {a->conv_bias, 4, "conv_bias"},
        {a->A_rev, 4, "A_rev"}, {a->D_rev, 4, "D_rev"}, {a->delta_bias_rev, 4, "delta_bias_rev"},
        {a->final_state, 4, "final_state"}, {a->final_state_rev, 4, "final_state_rev"},
        {a->workspace, 16, "workspace"}, {a->initial_state, 4, "initial_state"},
        {a->conv_history, (size_t)es, "conv_history"},
        {a->conv_state_out, (size_t)es, "conv_state_out"}, {a->seq_starts, 4, "seq_starts"}};
    for (auto& x : al)
        if (x.p && !aligned(x.p, x.al))
            return fail(SSM_ERR_MISALIGNED, "%s is not %zu-byte aligned", x.n, x.al);
    if (!empty) {
        if (overlap(a->out, act_out, a->u, act_u) || overlap(a->out, act_out, a->delta, act_dl) ||
            overlap(a->out, act_out, a->z, act_z) || overlap(a->out, act_out, a->B, bc_B) ||
            overlap(a->out, act_out, a->C, bc_C))
            return fail(SSM_ERR_ALIAS, "out overlaps an input");
    }
    const bool packed = a->seq_starts != nullptr;
    // packed sequences: final state and conv state per sequence
    const int64_t out_rows = packed ? (int64_t)a->num_seqs * a->dim : rows;
    const size_t st_bytes = (size_t)rows * a->dstate * sizeof(float);
    const int cw = a->conv_weight ? a->conv_width : 0;
    const size_t hist_bytes = cw > 0 ? (size_t)rows * (cw - 1) * es : 0;
    const size_t tail_bytes = (size_t)out_rows * cw * es;
    if (a->conv_state_out &&
        (overlap(a->conv_state_out, tail_bytes, a->u, act_u) ||
         overlap(a->conv_state_out, tail_bytes, a->conv_history, hist_bytes) ||
         overlap(a->conv_state_out, tail_bytes, a->out, act_out)))
        return fail(SSM_ERR_ALIAS, "conv_state_out overlaps u, conv_history or out");
    // one pass reads a row's initial state before writing its final state; the two-pass
    // carry reads it in every chunk while the last chunk writes the final state
    if (pl.nchunks > 1 && overlap(a->final_state, st_bytes, a->initial_state, st_bytes))
        return fail(SSM_ERR_ALIAS, "final_state overlaps initial_state with a two-pass carry");
    if (pl.workspace > 0 && (!a->workspace || a->workspace_bytes < pl.workspace))
        return fail(SSM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", pl.workspace,
                    a->workspace ? a->workspace_bytes : (size_t)0);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the conv state the next call continues from (independent of the scan's results)
    auto conv_tail = [&]() -> ssm_status_t {
        if (!a->conv_state_out || rows == 0) return SSM_OK;
        ssm::ConvTailParams tp{a->u, a->conv_history, a->conv_state_out, out_rows, (int)a->seqlen,
                               cw, a->seq_starts, packed ? a->num_seqs : 0, (int)a->dim, su};
        cudaError_t e = ssm::launch_conv_tail(es, tp, s);
        return e == cudaSuccess ? SSM_OK : cuda_fail(e, "conv state launch");
    };
    if (packed && a->final_state) {
        // every sequence's final state is written at its last step; an empty sequence
        // has none and keeps the zero initial state
        const size_t fs = (size_t)out_rows * a->dstate * sizeof(float);
        cudaError_t e = cudaMemsetAsync(a->final_state, 0, fs, s);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    }
    if (empty) {
        // zero steps: the final state is the initial state, the conv state its history
        const size_t fs = (size_t)rows * a->dstate * sizeof(float);
        if (fs && a->final_state && a->initial_state) {
            if (a->final_state != a->initial_state) {
                cudaError_t e = cudaMemcpyAsync(a->final_state, a->initial_state, fs,
                                                cudaMemcpyDeviceToDevice, s);
                if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync");
            }
        } else if (fs && a->final_state && !packed) {
            cudaError_t e = cudaMemsetAsync(a->final_state, 0, fs, s);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
        }
        if (ssm_status_t t = conv_tail(); t != SSM_OK) return t;
        if (fs && a->final_state_rev) {
            cudaError_t e = cudaMemsetAsync(a->final_state_rev, 0, fs, s);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
        }
        return ok();
    }

    ssm::ScanParams p{};
    p.batch = (int)a->batch;
    p.dim = (int)a->dim;
    p.seqlen = (int)a->seqlen;
    p.dstate = (int)a->dstate;
    p.u = a->u;
    p.delta = a->delta;
    p.z = a->z;
    p.Bm = a->B;
    p.Cm = a->C;
    p.A[0] = a->A;
    p.Dv[0] = a->D;
    p.dbias[0] = a->delta_bias;
    p.A[1] = bidir ? a->A_rev : a->A;
    p.Dv[1] = bidir ? a->D_rev : a->D;
    p.dbias[1] = bidir ? a->delta_bias_rev : a->delta_bias;
    p.conv_w = a->conv_weight;
    p.conv_b = a->conv_weight ? a->conv_bias : nullptr;
    p.conv_width = a->conv_weight ? a->conv_width : 0;
    p.softplus = a->delta_softplus ? 1 : 0;
    p.mode = pl.mode;
    p.out = a->out;
    p.final_state[0] = a->final_state;
    p.final_state[1] = a->final_state_rev;
    p.chunk_len = pl.chunk_len;
    p.nchunks = pl.nchunks;
    p.seq_aligned = packed && pl.nchunks > 1 ? 1 : 0;
    uint8_t* ws = static_cast<uint8_t*>(a->workspace);
    p.summary = pl.summary_bytes ? reinterpret_cast<float2*>(ws) : nullptr;
    p.h0 = a->initial_state;
    p.conv_hist = a->conv_weight ? a->conv_history : nullptr;
    p.cu = a->seq_starts;
    p.nseq = packed ? a->num_seqs : 0;
    p.su = su;
    p.sdl = sdl;
    p.sz = sz;
    p.sout = sout;
    p.sB = sB;
    p.sC = sC;
    p.head_dim = a->a_heads > 0 ? (int)(a->dim / a->a_heads) : 0;
    const int feat = (a->a_heads > 0 ? 1 : 0) | (sb ? 2 : 0);
    if (bidir) {
        // the forward sweep's fp32 partial y: in `out` itself when fp32 (same layout and
        // stride), else in the workspace (dense, the activations' layout)
        p.partial = a->dtype == SSM_F32
                        ? static_cast<float*>(a->out)
                        : reinterpret_cast<float*>(ws + ((pl.summary_bytes + 255) / 256) * 256);
        p.spart = a->dtype == SSM_F32 ? sout : a->dim;
    }
    const bool row16 = (a->seqlen * es) % 16 == 0;
    p.vec_store = !cl && row16 && aligned(a->out, 16);

    // TMA needs 16-byte aligned bases and strides of a multiple of 16 bytes (and, in
    // channel-last, B/C rows of at least 16 bytes)
    const int ns_pad = pl.v.np * pl.v.s;
    const bool strides16 = cl ? ((su | sdl | sz | sB | sC) * es) % 16 == 0 &&
                                    (sb || ns_pad * es >= 16)
                              : row16;
    bool tma = strides16 && aligned(a->u, 16) && aligned(a->delta, 16) &&
               (sb || (aligned(a->B, 16) && aligned(a->C, 16))) && (!a->z || aligned(a->z, 16)) &&
               env_int("SSM_NO_TMA", 0) == 0;
    ssm::ScanMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (tma) {
        const auto& v = pl.v;
        const uint32_t xbox = a->conv_weight ? v.tile + v.halo : v.tile;
        const uint64_t L = a->seqlen, D = a->dim, Bn = a->batch, N = a->dstate;
        // B, C tiles use the swizzle whose span equals one tile row (64 B: 32 bf16 or 16
        // fp32 steps; 128 B: 64 bf16 steps)
        const int rowb = v.tile * es;
        if (rowb != 64 && rowb != 128)
            return fail(SSM_ERR_UNSUPPORTED, "tile rows must be 64 or 128 bytes");
        const CUtensorMapSwizzle bc =
            rowb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
        const CUtensorMapSwizzle none = CU_TENSOR_MAP_SWIZZLE_NONE;
        if (cl) {
            // (channel, t, batch) boxes: tiles land as [t][channel] and B/C as [t][n]
            auto map = [&](CUtensorMap* m, const void* ptr, uint64_t w, int64_t st,
                           uint32_t b0, uint32_t b1) {
                return encode_3d_strided(m, es, ptr, w, L, Bn, (uint64_t)st * es,
                                         (uint64_t)st * L * es, b0, b1, none);
            };
            tma = map(&maps.x, a->u, D, su, v.channels, xbox) &&
                  map(&maps.dt, a->delta, D, sdl, v.channels, v.tile) &&
                  (!a->z || map(&maps.z, a->z, D, sz, v.channels, v.tile)) &&
                  (sb || (map(&maps.B, a->B, N, sB, ns_pad, v.tile) &&
                          map(&maps.C, a->C, N, sC, ns_pad, v.tile)));
        } else {
            // delta and z rows land swizzled (the kernel reads them so)
            const CUtensorMapSwizzle dz = SSM_SWZ_DTZ ? bc : none;
            tma = encode_3d(&maps.x, es, a->u, L, D, Bn, xbox, v.channels, none) &&
                  encode_3d(&maps.dt, es, a->delta, L, D, Bn, v.tile, v.channels, dz) &&
                  (!a->z || encode_3d(&maps.z, es, a->z, L, D, Bn, v.tile, v.channels, dz)) &&
                  (sb || (encode_3d(&maps.B, es, a->B, L, N, Bn, v.tile, v.np * v.s, bc) &&
                          encode_3d(&maps.C, es, a->C, L, N, Bn, v.tile, v.np * v.s, bc)));
        }
    }

    const unsigned gx = (unsigned)((a->dim + pl.v.channels - 1) / pl.v.channels);
    cudaError_t e;
    if (pl.nchunks > 1 && !p.seq_aligned) {
        e = ssm::launch_scan(pl.v, tma, true, packed, cl, feat, maps, p,
                             dim3(gx, (unsigned)a->batch, pl.nchunks - 1), s);
        if (e != cudaSuccess) return cuda_fail(e, "summary pass launch");
    }
    e = ssm::launch_scan(pl.v, tma, false, packed, cl, feat, maps, p,
                         dim3(gx, (unsigned)a->batch, pl.nchunks), s);
    if (e != cudaSuccess) return cuda_fail(e, "scan launch");
    if (ssm_status_t t = conv_tail(); t != SSM_OK) return t;
    return ok();
}

ssm_status_t ssm_causal_conv1d_fwd(const void* x, const float* w, const float* bias, void* out,
                                   int64_t batch, int64_t dim, int64_t seqlen, int32_t width,
                                   int32_t apply_silu, ssm_dtype_t dtype, ssm_stream_t stream) {
    if (dtype != SSM_F32 && dtype != SSM_BF16)
        return fail(SSM_ERR_BAD_DTYPE, "dtype %d is not SSM_F32 or SSM_BF16", (int)dtype);
    if (batch < 0 || dim < 0 || seqlen < 0)
        return fail(SSM_ERR_BAD_SHAPE, "negative size");
    if (width < 1 || width > SSM_MAX_CONV_WIDTH)
        return fail(SSM_ERR_BAD_SHAPE, "width %d outside 1..%d", width, SSM_MAX_CONV_WIDTH);
    if (seqlen > 0x3fffffffLL || dim > 0x3fffffffLL)
        return fail(SSM_ERR_BAD_SHAPE, "seqlen and dim must be below 2^30");
    const int64_t rows = batch * dim;
    if (rows == 0 || seqlen == 0) return ok();
    if (!x || !w || !out) return fail(SSM_ERR_NULL_ARG, "%s is NULL", !x ? "x" : !w ? "w" : "out");
    const int es = elem_size(dtype);
    if (!aligned(x, es) || !aligned(out, es) || !aligned(w, 4) || (bias && !aligned(bias, 4)))
        return fail(SSM_ERR_MISALIGNED, "a pointer is not aligned to its element size");
    const size_t n = (size_t)rows * seqlen * es;
    if (overlap(x, n, out, n)) return fail(SSM_ERR_ALIAS, "out overlaps x");
    ssm::ConvParams p{x, w, bias, out, rows, (int)dim, (int)seqlen, width, apply_silu ? 1 : 0};
    const bool vec = (seqlen % 8 == 0) && aligned(x, 16) && aligned(out, 16);
    cudaError_t e = ssm::launch_conv(es, vec, p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "conv launch");
    return ok();
}

ssm_status_t ssm_selective_state_update(float* state, void* conv_state, const void* x,
                                        const void* dt, const float* A, const void* B_t,
                                        const void* C_t, const float* D, const void* z,
                                        const float* dt_bias, int32_t dt_softplus,
                                        const float* conv_weight, const float* conv_bias,
                                        int32_t conv_width, void* out, int64_t batch,
                                        int64_t dim, int64_t dstate, ssm_dtype_t dtype,
                                        ssm_stream_t stream) {
    if (dtype != SSM_F32 && dtype != SSM_BF16)
        return fail(SSM_ERR_BAD_DTYPE, "dtype %d is not SSM_F32 or SSM_BF16", (int)dtype);
    if (batch < 0 || dim < 0) return fail(SSM_ERR_BAD_SHAPE, "negative size");
    if (dstate < 1 || dstate > SSM_MAX_DSTATE)
        return fail(SSM_ERR_BAD_SHAPE, "dstate %lld outside 1..%d", (long long)dstate,
                    SSM_MAX_DSTATE);
    if (conv_weight && (conv_width < 1 || conv_width > SSM_MAX_CONV_WIDTH))
        return fail(SSM_ERR_BAD_SHAPE, "conv_width %d outside 1..%d", conv_width,
                    SSM_MAX_CONV_WIDTH);
    if (dim > 0x3fffffffLL) return fail(SSM_ERR_BAD_SHAPE, "dim must be below 2^30");
    const int64_t rows = batch * dim;
    if (rows == 0) return ok();
    if (rows > (int64_t)1 << 28)
        return fail(SSM_ERR_BAD_SHAPE, "batch * dim = %lld exceeds 2^28", (long long)rows);
    struct { const void* p; const char* n; } req[] = {
        {state, "state"}, {x, "x"}, {dt, "dt"}, {A, "A"}, {B_t, "B_t"}, {C_t, "C_t"}, {out, "out"}};
    for (auto& r : req)
        if (!r.p) return fail(SSM_ERR_NULL_ARG, "%s is NULL", r.n);
    if (conv_weight && !conv_state) return fail(SSM_ERR_NULL_ARG, "conv_state is NULL");
    const int es = elem_size(dtype);
    struct { const void* p; size_t al; const char* n; } al[] = {
        {state, 4, "state"}, {conv_state, (size_t)es, "conv_state"}, {x, (size_t)es, "x"},
        {dt, (size_t)es, "dt"}, {A, 4, "A"}, {B_t, (size_t)es, "B_t"}, {C_t, (size_t)es, "C_t"},
        {D, 4, "D"}, {z, (size_t)es, "z"}, {dt_bias, 4, "dt_bias"},
        {conv_weight, 4, "conv_weight"}, {conv_bias, 4, "conv_bias"}, {out, (size_t)es, "out"}};
    for (auto& q : al)
        if (q.p && !aligned(q.p, q.al))
            return fail(SSM_ERR_MISALIGNED, "%s is not %zu-byte aligned", q.n, q.al);
    const size_t on = (size_t)rows * es;
    if (overlap(out, on, x, on) || overlap(out, on, dt, on) || overlap(out, on, z, on) ||
        overlap(out, on, state, (size_t)rows * dstate * 4))
        return fail(SSM_ERR_ALIAS, "out overlaps an input");
    ssm::DecodeParams p{};
    p.state = state;
    p.conv_state = conv_weight ? conv_state : nullptr;
    p.x = x;
    p.dt = dt;
    p.A = A;
    p.Bt = B_t;
    p.Ct = C_t;
    p.D = D;
    p.z = z;
    p.dt_bias = dt_bias;
    p.conv_w = conv_weight;
    p.conv_b = conv_weight ? conv_bias : nullptr;
    p.out = out;
    p.rows = rows;
    p.dim = (int)dim;
    p.dstate = (int)dstate;
    p.conv_width = conv_weight ? conv_width : 0;
    p.softplus = dt_softplus ? 1 : 0;
    p.vec = dstate == 16 && aligned(state, 16) && aligned(A, 16);
    // Kernel choice. Streaming (the default where it applies): dstate 16, 128-channel
    // groups, conv width 2..4 or none, 16-byte aligned bases for its bulk copies. Else the bulk-copy kernel
    // (64-channel groups), else plain loads. SSM_DECODE_KERNEL = plain | bulk | stream
    // restricts the choice (tests compare the kernels).
    const bool base16 = aligned(state, 16) && aligned(x, 16) && aligned(dt, 16) &&
                        aligned(out, 16) && (!z || aligned(z, 16)) &&
                        (!conv_weight || aligned(conv_state, 16));
    const char* want = getenv("SSM_DECODE_KERNEL");
    const bool any = !want || !*want;
    const bool plain = !any && strcmp(want, "plain") == 0;
    p.stream = !plain && (any || strcmp(want, "stream") == 0) && dstate == 16 &&
               dim % 128 == 0 && (!conv_weight || conv_width >= 2) && base16 &&
               aligned(A, 16) && aligned(B_t, 16) && aligned(C_t, 16);
    p.bulk = !plain && !p.stream && (any || strcmp(want, "bulk") == 0) && dim % 64 == 0 &&
             batch <= 65535 && base16;
    cudaError_t e = ssm::launch_decode(es, (int)dstate, p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "state update launch");
    return ok();
}

ssm_status_t ssm_selective_state_update_ex(const ssm_update_args_t* a, ssm_stream_t stream) {
    if (!a) return fail(SSM_ERR_NULL_ARG, "args is NULL");
    if (a->a_heads < 0 || (a->a_heads > 0 && a->dim > 0 && a->dim % a->a_heads != 0))
        return fail(SSM_ERR_BAD_SHAPE, "a_heads %d must be 0 or divide dim %lld", a->a_heads,
                    (long long)a->dim);
    if (a->dstate <= SSM_MAX_DSTATE && a->a_heads == 0)
        return ssm_selective_state_update(a->state, a->conv_state, a->x, a->dt, a->A, a->B_t,
                                          a->C_t, a->D, a->z, a->dt_bias, a->dt_softplus,
                                          a->conv_weight, a->conv_bias, a->conv_width, a->out,
                                          a->batch, a->dim, a->dstate, a->dtype, stream);
    if (a->dtype != SSM_F32 && a->dtype != SSM_BF16)
        return fail(SSM_ERR_BAD_DTYPE, "dtype %d is not SSM_F32 or SSM_BF16", (int)a->dtype);
    if (a->batch < 0 || a->dim < 0) return fail(SSM_ERR_BAD_SHAPE, "negative size");
    if (a->dstate < 1 || a->dstate > SSM_MAX_SCAN_DSTATE)
        return fail(SSM_ERR_BAD_SHAPE, "dstate %lld outside 1..%d", (long long)a->dstate,
                    SSM_MAX_SCAN_DSTATE);
    if (a->conv_weight && (a->conv_width < 1 || a->conv_width > SSM_MAX_CONV_WIDTH))
        return fail(SSM_ERR_BAD_SHAPE, "conv_width %d outside 1..%d", a->conv_width,
                    SSM_MAX_CONV_WIDTH);
    if (a->dim > 0x3fffffffLL) return fail(SSM_ERR_BAD_SHAPE, "dim must be below 2^30");
    const int64_t rows = a->batch * a->dim;
    if (rows == 0) return ok();
    if (rows > (int64_t)1 << 28)
        return fail(SSM_ERR_BAD_SHAPE, "batch * dim = %lld exceeds 2^28", (long long)rows);
    struct { const void* p; const char* n; } req[] = {
        {a->state, "state"}, {a->x, "x"}, {a->dt, "dt"}, {a->A, "A"}, {a->B_t, "B_t"},
        {a->C_t, "C_t"}, {a->out, "out"}};
    for (auto& r : req)
        if (!r.p) return fail(SSM_ERR_NULL_ARG, "%s is NULL", r.n);
    if (a->conv_weight && !a->conv_state) return fail(SSM_ERR_NULL_ARG, "conv_state is NULL");
    const int es = elem_size(a->dtype);
    struct { const void* p; size_t al; const char* n; } al[] = {
        {a->state, 4, "state"}, {a->conv_state, (size_t)es, "conv_state"}, {a->x, (size_t)es, "x"},
        {a->dt, (size_t)es, "dt"}, {a->A, 4, "A"}, {a->B_t, (size_t)es, "B_t"},
        {a->C_t, (size_t)es, "C_t"}, {a->D, 4, "D"}, {a->z, (size_t)es, "z"},
        {a->dt_bias, 4, "dt_bias"}, {a->conv_weight, 4, "conv_weight"},
        {a->conv_bias, 4, "conv_bias"}, {a->out, (size_t)es, "out"}};
    for (auto& x : al)
        if (x.p && !aligned(x.p, x.al))
            return fail(SSM_ERR_MISALIGNED, "%s is not %zu-byte aligned", x.n, x.al);
    const size_t on = (size_t)rows * es;
    if (overlap(a->out, on, a->x, on) || overlap(a->out, on, a->dt, on) ||
        overlap(a->out, on, a->z, on) ||
        overlap(a->out, on, a->state, (size_t)rows * a->dstate * 4))
        return fail(SSM_ERR_ALIAS, "out overlaps an input");
    if (a->conv_weight && overlap(a->conv_state, (size_t)rows * a->conv_width * es, a->state,
                                  (size_t)rows * a->dstate * 4))
        return fail(SSM_ERR_ALIAS, "conv_state overlaps state");
    ssm::DecodeParams p{};
    p.state = a->state;
    p.conv_state = a->conv_weight ? a->conv_state : nullptr;
    p.x = a->x;
    p.dt = a->dt;
    p.A = a->A;
    p.Bt = a->B_t;
    p.Ct = a->C_t;
    p.D = a->D;
    p.z = a->z;
    p.dt_bias = a->dt_bias;
    p.conv_w = a->conv_weight;
    p.conv_b = a->conv_weight ? a->conv_bias : nullptr;
    p.out = a->out;
    p.rows = rows;
    p.dim = (int)a->dim;
    p.dstate = (int)a->dstate;
    p.conv_width = a->conv_weight ? a->conv_width : 0;
    p.softplus = a->dt_softplus ? 1 : 0;
    p.vec = a->dstate % 4 == 0 && aligned(a->state, 16);
    p.head_dim = a->a_heads > 0 ? (int)(a->dim / a->a_heads) : 0;
    // Streaming (the default where it applies): d_state 32, 64 or 128, channel groups of
    // 4096 / d_state, 16-byte aligned bases for its bulk copies. Else plain loads, one
    // warp per 32 / lanes-per-row rows. SSM_DECODE_KERNEL = plain restricts the choice.
    const int64_t group = a->dstate > 0 ? 4096 / a->dstate : 0;
    const char* want = getenv("SSM_DECODE_KERNEL");
    const bool plain = want && strcmp(want, "plain") == 0;
    p.stream = !plain && (a->dstate == 32 || a->dstate == 64 || a->dstate == 128) &&
               a->dim % group == 0 && aligned(a->state, 16) && aligned(a->x, 16) &&
               aligned(a->dt, 16) && aligned(a->out, 16) && aligned(a->B_t, 16) &&
               aligned(a->C_t, 16) && (!a->z || aligned(a->z, 16)) &&
               (!a->conv_weight || aligned(a->conv_state, 16)) &&
               (a->a_heads > 0 || aligned(a->A, 16));
    cudaError_t e = ssm::launch_decode_warp(es, p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "state update launch");
    return ok();
}

ssm_status_t ssm_wait_selftest(uint64_t limit_ns, ssm_stream_t stream) {
    if (limit_ns < 1000 || limit_ns > 1000000000ull)
        return fail(SSM_ERR_BAD_SHAPE, "limit_ns %llu outside 1 us .. 1 s",
                    (unsigned long long)limit_ns);
    cudaError_t e = ssm::launch_wait_selftest(limit_ns, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    return ok();
}

ssm_status_t ssm_device_error(int32_t* code, ssm_stream_t stream) {
    if (!code) return fail(SSM_ERR_NULL_ARG, "code is NULL");
    int c = 0;
    cudaError_t e = ssm::read_device_error(&c, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    *code = c;
    return ok();
}

}  // extern "C"
