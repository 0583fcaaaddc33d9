// Launch parameters of the kernels (host and device view).
#pragma once

#include <cuda.h>
#include <stdint.h>

// The (batch, dim, seqlen) layout's delta and z tiles (64-byte rows) land with the TMA
// 64-byte swizzle, so that the producers' 16-byte reads of consecutive rows hit distinct
// banks (unswizzled, every other row starts on the same bank: 4-way conflicts).
#ifndef SSM_SWZ_DTZ
#define SSM_SWZ_DTZ 1
#endif

namespace ssm {

// TMA descriptors of the streamed tensors (unused by the plain-load variant).
struct ScanMaps {
    CUtensorMap x;    // u or pre-conv x: dims (L, D, batch), box (TT [+halo], G, 1)
    CUtensorMap dt;   // delta:           dims (L, D, batch), box (TT, G, 1), 64-byte swizzle
    CUtensorMap z;    // gate input:      dims (L, D, batch), box (TT, G, 1), 64-byte swizzle
    CUtensorMap B;    // dims (L, N, batch), box (TT, NS, 1), swizzle spanning one tile row
    CUtensorMap C;    // dims (L, N, batch), box (TT, NS, 1), swizzle spanning one tile row
};

struct ScanParams {
    int batch, dim, seqlen, dstate;
    const void* u;
    const void* delta;
    const void* z;          // nullptr: no gate
    const void* Bm;
    const void* Cm;
    const float* A[2];      // per direction (index 1 only for the bidirectional sum)
    const float* Dv[2];
    const float* dbias[2];
    const float* conv_w;    // nullptr: no fused conv
    const float* conv_b;
    int conv_width;
    int softplus;
    int mode;               // 0 forward, 1 reverse, 2 bidirectional sum
    void* out;
    float* partial;         // bidirectional: fp32 buffer for the first direction
    float* final_state[2];
    int chunk_len;          // scan positions per chunk (multiple of the tile length)
    int nchunks;
    int seq_aligned;        // packed sequences: chunks begin at sequence starts (no carry)
    float2* summary;        // two-pass: [nchunks-1][batch*dim][NS] {prod dA, h_end}
    const float* h0;        // (batch, dim, dstate) state before position 0, or nullptr
    const void* conv_hist;  // (batch, dim, conv_width-1) inputs before position 0, or nullptr
    const int32_t* cu;      // packed sequences: nseq + 1 start offsets (cu[nseq] = seqlen)
    int nseq;
    // channel-last activations: element strides between consecutive positions
    int64_t su, sdl, sz, sout, sB, sC, spart;
    int vec_store;          // rows are 16-byte aligned: vector stores allowed
    // A as one scalar per head (kernels with FEAT bit 0): channels per head; A[dir] is
    // (dim / head_dim,) and channel d uses A[dir][d / head_dim]
    int head_dim;
    // time-invariant B, C (kernels with FEAT bit 1): Bm, Cm are fp32 (dim, dstate)
};

// The last conv_width inputs of history ++ x per row (the conv state a decode step
// continues from).
struct ConvTailParams {
    const void* x;          // (rows, seqlen)
    const void* hist;       // (rows, width-1) or nullptr
    void* out;              // (rows, width); packed sequences: (nseq, dim, width)
    int64_t rows;
    int seqlen, width;
    const int32_t* cu;      // packed sequences (batch 1): nseq + 1 start offsets, or nullptr
    int nseq, dim;
    int64_t stride;         // channel-last x: element stride between positions (0: rows of x)
};

// Standalone causal conv1d.
struct ConvParams {
    const void* x;
    const float* w;
    const float* bias;
    void* out;
    int64_t rows;      // batch * dim
    int dim, seqlen, width, silu;
};

// Single-token state update.
struct DecodeParams {
    float* state;
    void* conv_state;
    const void* x;
    const void* dt;
    const float* A;
    const void* Bt;
    const void* Ct;
    const float* D;
    const void* z;
    const float* dt_bias;
    const float* conv_w;
    const float* conv_b;
    void* out;
    int64_t rows;       // batch * dim
    int dim, dstate, conv_width, softplus;
    int vec;            // dstate == 16 and state / A rows 16-byte aligned
    int bulk;           // bulk-copy variant: rows % 64 == 0, 16-byte aligned bases
    int stream;         // streaming variant (bulk-copy ring): dstate 16 in 128-channel groups,
                        // or dstate 32 / 64 / 128 in 4096 / dstate channel groups; 16-byte
                        // aligned bases
    int head_dim;       // A one scalar per head (A[d / head_dim]); 0: A is (dim, dstate)
};

}  // namespace ssm
