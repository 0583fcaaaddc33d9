/*
 * ssm.h — C ABI of the B200 (sm_100a) Mamba selective-scan library.
 *
 * Three operations, following how the pages state the problem:
 *
 *  ssm_causal_conv1d_fwd
 *      The short causal depthwise convolution at the front of every Mamba block:
 *      output t depends only on inputs at positions <= t (qwerky.ai, "Bringing
 *      ... SSMs to the Modular MAX Framework", section "What We Built"; pyshine.com
 *      "Mamba" tour, the block paragraph: "runs a short causal convolution, then
 *      feeds the result to the selective scan").
 *
 *  ssm_selective_scan_fwd
 *      The selective-scan forward: delta = softplus(dt + delta_bias),
 *      dA = exp(delta*A) with A diagonal so the exponential is scalar (paperlayer.ai
 *      summary of arXiv 2603.09555, §3 Method, "State-space duality"),
 *      dBu = delta*B_t*u, h_t = dA*h_{t-1} + dBu (qwerky.ai, "Why State Space Models?
 *      Why Mamba?": a recurrence over a fixed-size hidden state), y = C_t.h_t + D*u,
 *      y *= silu(z). Optional: the causal conv + SiLU fused in front, the reverse
 *      direction, the bidirectional sum of both (kanishk-sama.me "ARM Selective-Scan
 *      Kernel", "What I built"), the final state, and a two-pass chunk-parallel
 *      carry for long sequences (paperlayer.ai §3 Method, "Chunked recurrence":
 *      chunk summaries combined by a light scan between chunks).
 *
 *  ssm_selective_state_update
 *      The single-token decode step: the same math on one token, with the conv and
 *      SSM states updated in place (pyshine.com tour, the block paragraph on
 *      `step`; paperlayer.ai §3 Method, "Autoregressive cache": fixed-size hidden and
 *      convolution states make each update O(1) in prefix length).
 *
 * Conventions for every entry point
 *  - Tensor pointers are DEVICE pointers, row-major and contiguous, with the
 *    sequence axis innermost: u, delta, z, out are (batch, dim, seqlen); B, C are
 *    (batch, dstate, seqlen); A is (dim, dstate); D, biases are (dim).
 *  - The caller owns all memory. The library never allocates, frees or
 *    synchronises; it only enqueues kernels on `stream` (a cudaStream_t value;
 *    NULL = the legacy default stream). Scratch memory is caller-provided
 *    (`workspace`, sized by ssm_selective_scan_workspace_size).
 *  - Activations (u, delta, z, B, C, out, x, dt, conv_state) use `dtype`
 *    (SSM_F32 or SSM_BF16). A, D, biases, conv weights and the SSM state are
 *    always fp32. Arithmetic is fp32 throughout; outputs are rounded to `dtype`
 *    once, at the store.
 *  - Every argument is validated on the host BEFORE anything is launched. On a
 *    bad argument the call returns an error code, launches nothing, and
 *    ssm_last_error_detail() describes the problem (thread-local text).
 *  - A launch failure reported by the CUDA runtime returns SSM_ERR_CUDA.
 *    Faults inside a kernel surface at the caller's next synchronisation.
 *  - Kernel-side waits are bounded. A wait that runs out sets a device-side error
 *    code, which ssm_device_error() reads and clears; the kernel then returns.
 *  - No C++ exception crosses this boundary. The library keeps no state between
 *    calls apart from the thread-local error text and the device error word.
 */
#ifndef SSM_B200_H
#define SSM_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported entry points keep default visibility when the library hides the rest. */
#if defined(__GNUC__)
#define SSM_API __attribute__((visibility("default")))
#else
#define SSM_API
#endif

#define SSM_ABI_VERSION 4
#define SSM_MAX_DSTATE 16        /* decode (ssm_selective_state_update) */
#define SSM_MAX_SCAN_DSTATE 128  /* scan (ssm_selective_scan_fwd) */
#define SSM_MAX_CONV_WIDTH 4

/* A cudaStream_t value, passed through untouched. */
typedef void* ssm_stream_t;

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype_t;

typedef enum {
    SSM_OK = 0,
    SSM_ERR_NULL_ARG = 1,     /* a required pointer is NULL */
    SSM_ERR_BAD_SHAPE = 2,    /* a size is out of range (negative, dstate > 16, ...) */
    SSM_ERR_BAD_DTYPE = 3,    /* dtype is not SSM_F32 / SSM_BF16 */
    SSM_ERR_MISALIGNED = 4,   /* a pointer is not aligned to its element size */
    SSM_ERR_WORKSPACE = 5,    /* workspace missing or smaller than required */
    SSM_ERR_UNSUPPORTED = 6,  /* valid but unsupported combination */
    SSM_ERR_CUDA = 7,         /* the CUDA runtime reported an error at launch */
    SSM_ERR_TIMEOUT = 8,      /* a kernel-side bounded wait ran out (ssm_device_error) */
    SSM_ERR_ALIAS = 9         /* out overlaps an input */
} ssm_status_t;

/* Version of this ABI (SSM_ABI_VERSION). */
SSM_API int ssm_abi_version(void);

/* Static text for a status code. Never NULL. */
SSM_API const char* ssm_status_string(ssm_status_t status);

/* Thread-local description of the last failure on the calling thread ("" if none).
 * The pointer stays valid until the next library call on that thread. */
SSM_API const char* ssm_last_error_detail(void);

/*
 * Causal depthwise conv1d (+ optional SiLU).
 *   out[b,d,t] = act( bias[d] + sum_{k<width} w[d,k] * x[b,d,t-width+1+k] ),
 *   x[b,d,s<0] = 0, act = SiLU if apply_silu else identity.
 * x, out: (batch, dim, seqlen) in dtype, device; w: (dim, width) fp32; bias: (dim)
 * fp32 or NULL. width in 1..4. batch, dim, seqlen >= 0 (zero sizes launch nothing).
 * out must not overlap x (SSM_ERR_ALIAS).
 */
SSM_API ssm_status_t ssm_causal_conv1d_fwd(const void* x, const float* w, const float* bias, void* out,
                                   int64_t batch, int64_t dim, int64_t seqlen, int32_t width,
                                   int32_t apply_silu, ssm_dtype_t dtype, ssm_stream_t stream);

/* Arguments of ssm_selective_scan_fwd. Zero-initialise, then fill. */
typedef struct {
    ssm_dtype_t dtype;        /* element type of u, delta, z, B, C, out */
    int64_t batch, dim, seqlen;
    int64_t dstate;           /* 1..SSM_MAX_SCAN_DSTATE */
    const void* u;            /* (batch, dim, seqlen); the pre-conv x when conv_weight != NULL */
    const void* delta;        /* (batch, dim, seqlen): raw dt */
    const float* A;           /* (dim, dstate), normally negative (A = -exp(A_log)); with
                                 a_heads > 0: (a_heads) */
    const void* B;            /* (batch, dstate, seqlen); with bc_shared: fp32 (dim, dstate) */
    const void* C;            /* (batch, dstate, seqlen); with bc_shared: fp32 (dim, dstate) */
    const float* D;           /* (dim) skip weight, or NULL (no skip term) */
    const void* z;            /* (batch, dim, seqlen) gate input, or NULL (no gate) */
    const float* delta_bias;  /* (dim) or NULL (zero) */
    int32_t delta_softplus;   /* nonzero: delta = softplus(dt + bias); zero: dt + bias */
    int32_t reverse;          /* nonzero: scan t = seqlen-1 .. 0 (ignored if bidirectional) */
    const float* conv_weight; /* (dim, conv_width) or NULL; non-NULL fuses conv + SiLU on u */
    const float* conv_bias;   /* (dim) or NULL */
    int32_t conv_width;       /* 1..SSM_MAX_CONV_WIDTH when conv_weight != NULL */
    const float* A_rev;       /* non-NULL selects the bidirectional sum: shaped as A */
    const float* D_rev;       /* (dim) or NULL: skip weight of the reverse direction */
    const float* delta_bias_rev; /* (dim) or NULL: dt bias of the reverse direction */
    void* out;                /* (batch, dim, seqlen) in dtype; must not overlap inputs */
    float* final_state;       /* (batch, dim, dstate) or NULL: state after the last step */
    float* final_state_rev;   /* (batch, dim, dstate) or NULL: bidirectional, reverse state
                                 after position 0 */
    void* workspace;          /* device scratch, >= ssm_selective_scan_workspace_size bytes */
    size_t workspace_bytes;
    int32_t num_chunks;       /* 0 = automatic; 1 = single pass; k > 1 = two-pass carry over
                                 k chunks of the sequence (one direction only) */
    /* Continuing a sequence that an earlier call (a scan or decode steps) stopped at;
     * forward single-direction scans only (ABI 2). */
    const float* initial_state; /* (batch, dim, dstate) fp32 state before position 0, or
                                   NULL (zeros) */
    const void* conv_history; /* (batch, dim, conv_width - 1) in dtype: the inputs at
                                 positions -(conv_width-1) .. -1, oldest first, that the
                                 fused conv reads instead of zeros; or NULL. Needs
                                 conv_weight. */
    void* conv_state_out;     /* (batch, dim, conv_width) in dtype, or NULL: the last
                                 conv_width inputs of conv_history ++ u, oldest first
                                 (zeros before both) -- the conv state a decode step or
                                 the next scan continues from. Needs conv_weight; must not
                                 overlap the inputs. */
    /* Packed sequences (batch 1, forward, no initial_state / conv_history): several
     * sequences share the sequence axis. The state restarts from zero at every start
     * and the fused conv reads nothing before its sequence's start. final_state is
     * then (num_seqs, dim, dstate) and conv_state_out (num_seqs, dim, conv_width), per
     * sequence; an empty sequence keeps zeros. */
    const int32_t* seq_starts; /* device, num_seqs + 1 offsets: 0 = s_0 <= s_1 <= ... <=
                                  s_num_seqs = seqlen; or NULL (one sequence per row).
                                  Offsets out of order or range give unspecified
                                  results (never an access outside the tensors). */
    int32_t num_seqs;
    /* Channel-last activations: nonzero puts u, delta, z, out in (batch, seqlen, dim)
     * and B, C in (batch, seqlen, dstate) instead. Each has an element stride between
     * consecutive positions (0 = dense: dim, or dstate for B and C; otherwise at least
     * that), so x and z can be views into one in_proj output (stride 2*dim) and B, C
     * views into an x_proj output; consecutive batch rows are seqlen strides apart.
     * The decode layouts, the conv history and conv_state_out are unchanged. With
     * 16-byte aligned bases and strides of a multiple of 16 bytes the tiles arrive by
     * TMA; otherwise by plain loads. */
    int32_t channel_last;
    int64_t stride_u, stride_delta, stride_z, stride_out, stride_B, stride_C;
    /* ABI 3. A as one scalar per head (Mamba-2's restriction of the diagonal A,
     * paperlayer.ai summary of arXiv 2603.09555, §3 Method, "State-space duality"):
     * a_heads > 0 (dividing dim) makes A and A_rev (a_heads) fp32, head h owning the
     * dim / a_heads consecutive channels from h * dim / a_heads; every state of those
     * channels decays by exp(delta * A[h]), one exp per (channel, step). 0: A is
     * (dim, dstate). */
    int32_t a_heads;
    /* Time-invariant B and C (the "variable or shared" B/C dispatch axis, pyshine.com
     * tour, CUDA-core paragraph): bc_shared = 1 makes B and C fp32 (dim, dstate), the
     * same at every position (stride_B / stride_C are then ignored); 0: input-dependent
     * as above. Neither a_heads nor bc_shared combines with seq_starts
     * (SSM_ERR_UNSUPPORTED); bad values give SSM_ERR_BAD_SHAPE. */
    int32_t bc_shared;
} ssm_scan_args_t;

/* Bytes of device workspace the call with these arguments needs (0 if none).
 * Needs the shape fields, dtype, A_rev and num_chunks; pointers are not read. */
SSM_API ssm_status_t ssm_selective_scan_workspace_size(const ssm_scan_args_t* args, size_t* bytes);

/* Selective-scan forward. See the file comment for the computation and the
 * struct fields for layouts. final_state is the state after the last step of the
 * scan direction (position seqlen-1 forward, position 0 reverse).
 * Continuation (forward, one direction): with initial_state and conv_history the
 * scan picks up a sequence where an earlier call stopped, so a prompt can be taken
 * in pieces and a prefill can follow decode steps or precede them; final_state and
 * conv_state_out are what the next call (a scan, or ssm_selective_state_update)
 * continues from. The pages carry these two states across calls for the step method
 * (pyshine.com tour, block paragraph; paperlayer.ai §3 Method, "Autoregressive
 * cache"). Packed sequences (seq_starts): the varlen dispatch axis of the upstream
 * kernel (pyshine.com tour, the CUDA-core paragraph), each sequence scanned as if
 * alone. Errors: SSM_ERR_UNSUPPORTED for any of initial_state, conv_history,
 * conv_state_out with reverse or the bidirectional sum, and for seq_starts with
 * batch != 1, reverse, the bidirectional sum, initial_state or conv_history;
 * SSM_ERR_BAD_SHAPE for num_seqs < 1 with seq_starts; SSM_ERR_NULL_ARG for
 * conv_history or conv_state_out without conv_weight; SSM_ERR_ALIAS when
 * conv_state_out overlaps u, conv_history or out. */
SSM_API ssm_status_t ssm_selective_scan_fwd(const ssm_scan_args_t* args, ssm_stream_t stream);

/*
 * Single-token decode update, in place on state and conv_state.
 *   conv_state <- [conv_state[1:], x]            (if conv_weight != NULL)
 *   xc = SiLU(conv_bias + sum_k conv_weight[k] * conv_state[k])   (else xc = x)
 *   delta = softplus(dt + dt_bias) (or dt + dt_bias)
 *   state = exp(delta*A) * state + delta * B_t * xc
 *   out = (C_t . state + D * xc) * silu(z)
 * state: (batch, dim, dstate) fp32, in/out. conv_state: (batch, dim, conv_width) in
 * dtype, newest last, in/out (ignored when conv_weight is NULL). x, dt, z, out:
 * (batch, dim) in dtype. B_t, C_t: (batch, dstate) in dtype. A: (dim, dstate) fp32.
 * D, dt_bias, conv_bias: (dim) fp32 or NULL. z may be NULL (no gate).
 */
SSM_API ssm_status_t ssm_selective_state_update(float* state, void* conv_state, const void* x,
                                        const void* dt, const float* A, const void* B_t,
                                        const void* C_t, const float* D, const void* z,
                                        const float* dt_bias, int32_t dt_softplus,
                                        const float* conv_weight, const float* conv_bias,
                                        int32_t conv_width, void* out, int64_t batch,
                                        int64_t dim, int64_t dstate, ssm_dtype_t dtype,
                                        ssm_stream_t stream);

/* Arguments of ssm_selective_state_update_ex. Zero-initialise, then fill. The fields
 * mean what the arguments of ssm_selective_state_update mean, plus: */
typedef struct {
    ssm_dtype_t dtype;
    int64_t batch, dim;
    int64_t dstate;           /* 1..SSM_MAX_SCAN_DSTATE */
    float* state;             /* (batch, dim, dstate) fp32, in/out */
    void* conv_state;         /* (batch, dim, conv_width) in dtype, in/out; or NULL */
    const void* x;            /* (batch, dim) */
    const void* dt;           /* (batch, dim) */
    const float* A;           /* (dim, dstate), or (a_heads) with a_heads > 0 */
    const void* B_t;          /* (batch, dstate) */
    const void* C_t;          /* (batch, dstate) */
    const float* D;           /* (dim) or NULL */
    const void* z;            /* (batch, dim) or NULL */
    const float* dt_bias;     /* (dim) or NULL */
    int32_t dt_softplus;
    const float* conv_weight; /* (dim, conv_width) or NULL */
    const float* conv_bias;   /* (dim) or NULL */
    int32_t conv_width;
    void* out;                /* (batch, dim) */
    /* A as one scalar per head, heads contiguous over the channels (the same reading as
     * ssm_scan_args_t.a_heads): every state of a channel of head h decays by
     * exp(delta * A[h]); 0: A is (dim, dstate). */
    int32_t a_heads;
} ssm_update_args_t;

/* The decode step of ssm_selective_state_update, for d_state up to SSM_MAX_SCAN_DSTATE
 * and A per head (the step method of the scan's per-head form). With d_state <= 16 and
 * a_heads = 0 it runs the same kernels as ssm_selective_state_update. With d_state 32, 64
 * or 128, dim a multiple of 4096 / d_state and 16-byte aligned state, conv_state, x, dt,
 * z, out, B_t, C_t (and A when it is per state), the step streams groups of channels
 * through shared memory with bulk copies; otherwise it uses plain loads. Same results
 * either way, within rounding. Errors as there; SSM_ERR_BAD_SHAPE also for a_heads < 0
 * or not dividing dim; SSM_ERR_ALIAS also when conv_state overlaps state. */
SSM_API ssm_status_t ssm_selective_state_update_ex(const ssm_update_args_t* args,
                                                   ssm_stream_t stream);

/*
 * Selective-scan forward that allocates nothing (the pages have no counterpart:
 * this is a deployment convenience). Same arguments and results as
 * ssm_selective_scan_fwd, except that `workspace` / `workspace_bytes` are ignored:
 * the scratch the call needs (two-pass chunk summaries, the bf16 bidirectional
 * partial) lives in a fixed device array of SSM_NOALLOC_SCRATCH_BYTES compiled
 * into the library. A device holds it until exit from the moment the library's
 * module is loaded there: with CUDA's default lazy module loading that is no later
 * than the first no-allocation call on the device (its address lookup loads the
 * module), with CUDA_MODULE_LOADING=EAGER when the context is created.
 * For callers that cannot call cudaMalloc (a runtime that hands out only fixed
 * buffers, a C caller with no allocator, a loop that must not risk an allocation's
 * implicit synchronisation).
 *  - A call needing more scratch than SSM_NOALLOC_SCRATCH_BYTES returns
 *    SSM_ERR_WORKSPACE and launches nothing.
 *  - The first call on each device looks the array's address up
 *    (cudaGetSymbolAddress, with that device current); make that first call before
 *    any stream capture. It allocates nothing, and neither do later calls.
 *  - Every call on a device shares the one array and it keeps the last call's
 *    contents; nothing in it needs to start at zero (each launch writes its
 *    scratch before reading it). Calls whose kernels overlap on the GPU (other
 *    streams, other threads) race on it: serialise them.
 */
#define SSM_NOALLOC_SCRATCH_BYTES (8u << 20)
SSM_API ssm_status_t ssm_selective_scan_fwd_noalloc(const ssm_scan_args_t* args,
                                                    ssm_stream_t stream);

/* Read and clear the device-side error word (0 = none; 1 = a bounded wait ran out).
 * Synchronises `stream`. */
SSM_API ssm_status_t ssm_device_error(int32_t* code, ssm_stream_t stream);

/* Self-test of the failure path (the pages have no counterpart): enqueues one thread
 * that waits, with the kernels' bounded-wait routine, on a barrier nothing completes.
 * After limit_ns (1e3 .. 1e9, else SSM_ERR_BAD_SHAPE) the wait gives up, sets the
 * device error word to 1 and the kernel returns; ssm_device_error() then reports it
 * and the context stays usable. */
SSM_API ssm_status_t ssm_wait_selftest(uint64_t limit_ns, ssm_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SSM_B200_H */
