/*
 * selscan.h -- C ABI of libselscan, the Mamba-1 selective scan for B200
 * (sm_100a).
 *
 * The operation (pages: "Mamba & State Space Models — Guide Complet" §1
 * "Discrétisation" and §4 "Implémentation du SSM sélectif (S6)";
 * "Mamba и State Space Models: альтернатива Transformer", "SSM as RNN",
 * "Discretization" and "Mamba Block"). For every batch row b, channel d and
 * state index n, with h = 0 before the first token:
 *
 *     Δ_t      = softplus(delta[b,t,d] + delta_bias[d])   (or no softplus)
 *     Abar_t   = exp(Δ_t · A[d,n])
 *     h_t[n]   = Abar_t · h_{t-1}[n] + Δ_t · B[b,t,n] · x[b,t,d]
 *     y[b,t,d] = (Σ_n C[b,t,n] · h_t[n] + D[d] · x[b,t,d]) · silu(z[b,t,d])
 *
 * Δ, B and C vary per token (the "selection"); A is diagonal per channel and
 * fixed; the input term is Δ·B ("SSM as RNN" scales B by delta); y reads the
 * state after the token's update; D·x is added before the gate.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device,
 *    row-major and contiguous, last index fastest. The caller owns every
 *    buffer; the library keeps no pointer after a call returns.
 *  - `dtype` is the element type of x, delta, z, B, C and y. A, D,
 *    delta_bias and all states are always float32. Arithmetic is float32.
 *    bf16 results are rounded to nearest even.
 *  - Pointers must be aligned to their element size; y must not overlap any
 *    input.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream). The return value reports argument validation and
 *    launch errors (cudaGetLastError after the launches), not completion.
 *  - "required" pointers may be NULL only when their tensor has zero
 *    elements.
 *  - Return values: SELSCAN_OK (0) or one of the negative SELSCAN_ERR_*
 *    codes; nothing is launched when validation fails.
 */
#ifndef SELSCAN_H_
#define SELSCAN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SELSCAN_API __attribute__((visibility("default")))
#else
#define SELSCAN_API
#endif

/* Same type as cudaStream_t; spelled out so that this header needs no CUDA
 * header. */
typedef struct CUstream_st *selscan_stream_t;

typedef enum {
    SELSCAN_F32 = 0,  /* float32 x, delta, z, B, C, y */
    SELSCAN_BF16 = 1  /* bfloat16 x, delta, z, B, C, y */
} selscan_dtype_t;

enum {
    SELSCAN_OK = 0,
    SELSCAN_ERR_NULL_ARG = -1,           /* a required pointer is NULL */
    SELSCAN_ERR_BAD_DIM = -2,            /* a size is negative or too large */
    SELSCAN_ERR_BAD_DTYPE = -3,          /* dtype is not a selscan_dtype_t */
    SELSCAN_ERR_MISALIGNED = -4,         /* a pointer is not element-aligned */
    SELSCAN_ERR_DSTATE_UNSUPPORTED = -5, /* dstate outside 1..SELSCAN_MAX_DSTATE
                                            (1..SELSCAN_MAX_DSTATE_BWD for selscan_bwd) */
    SELSCAN_ERR_CUDA = -6,               /* a CUDA call failed */
    SELSCAN_ERR_ALIAS = -7,              /* y overlaps an input */
    SELSCAN_ERR_WORKSPACE = -8           /* the given or static workspace is too small
                                            (selscan_fwd_noalloc, selscan_bwd_workspace) */
};

/* Largest d_state of the forward and decode entry points. d_state ≤ 16 takes
 * the TMA-staged and register-resident kernels; 17..256 take a kernel that
 * splits each chain's states over 2-16 lanes (one pass, no chunking,
 * batch ≤ 65535). The gradient (selscan_bwd) takes d_state ≤ 256 as well. */
#define SELSCAN_MAX_DSTATE 256
#define SELSCAN_MAX_DSTATE_BWD 256

/*
 * selscan_fwd -- selective scan over whole sequences (the forward pass).
 *
 *   x, delta      [batch, seqlen, dim]      dtype        required
 *   A             [dim, dstate]             float32      required; a channel
 *                                                        whose A[d,n] are all
 *                                                        within 2^-21 of
 *                                                        (n+1)·A[d,0] (the
 *                                                        S4D/Mamba −(1..N),
 *                                                        also −exp(log(1..N))
 *                                                        in float32) is scanned
 *                                                        with (n+1)·A[d,0]:
 *                                                        powers of one decay
 *                                                        per token, a relative
 *                                                        change of Δ·|A|·2^-21
 *                                                        in exp(Δ·A)
 *   B, C          [batch, seqlen, dstate]   dtype        required; shared by
 *                                                        all channels
 *   D             [dim]                     float32      NULL -> no skip term
 *   z             [batch, seqlen, dim]      dtype        NULL -> no gate
 *   delta_bias    [dim]                     float32      NULL -> zero bias
 *   softplus_flag nonzero -> Δ = softplus(delta + bias), zero -> Δ = delta + bias
 *   y             [batch, seqlen, dim]      dtype        required output
 *   final_state   [batch, dim, dstate]      float32      NULL -> not written;
 *                                                        else h after the
 *                                                        last token (zeros if
 *                                                        seqlen == 0)
 *   batch, seqlen, dim >= 0 (any of them 0 -> nothing to compute);
 *   1 <= dstate <= SELSCAN_MAX_DSTATE.
 *
 * The sequence is processed in chunks whose final states are carried to the
 * next chunk (the pages' blockwise scan with its state carried across blocks,
 * "Hardware-Aware Scan", and the associative operator of Guide Complet §4
 * "Parallel Associative Scan"). Depending on the sizes, chunks run one after
 * another with the state handed over on the device, or in parallel followed
 * by a carry pass. Either takes a stream-ordered device workspace
 * (cudaMallocAsync / cudaFreeAsync on `stream`; its size is reported by
 * selscan_fwd_plan); no other memory is allocated.
 */
SELSCAN_API int selscan_fwd(const void *x, const void *delta, const float *A,
                const void *B, const void *C, const float *D, const void *z,
                const float *delta_bias, int softplus_flag, void *y,
                float *final_state, int64_t batch, int64_t seqlen, int64_t dim,
                int64_t dstate, selscan_dtype_t dtype, selscan_stream_t stream);

/*
 * selscan_fwd_from_state -- selscan_fwd starting from a given state instead
 * of h = 0 before the first token: the state carried across blocks of a
 * sequence ("Mamba и State Space Models: альтернатива Transformer",
 * "Hardware-Aware Scan") handed in from outside, e.g. the final state of a
 * previous call on the preceding tokens or a state advanced by
 * selscan_state_update. Arguments as selscan_fwd, plus
 *   initial_state [batch, dim, dstate]   float32   NULL -> zero (== selscan_fwd)
 * initial_state may be the same buffer as final_state (the state is then
 * advanced in place); any other overlap with an output is rejected. With
 * seqlen == 0 the final state is a copy of the initial state.
 */
SELSCAN_API int selscan_fwd_from_state(const void *x, const void *delta, const float *A,
                                       const void *B, const void *C, const float *D,
                                       const void *z, const float *delta_bias,
                                       int softplus_flag, const float *initial_state,
                                       void *y, float *final_state, int64_t batch,
                                       int64_t seqlen, int64_t dim, int64_t dstate,
                                       selscan_dtype_t dtype, selscan_stream_t stream);

/*
 * selscan_fwd_conv -- the Mamba block's causal depthwise convolution and SiLU
 * in front of the scan, fused into it ("Mamba и State Space Models:
 * альтернатива Transformer", "Mamba Block": Conv1d with one filter per
 * channel and d_conv − 1 leading zeros; "Mamba & State Space Models — Guide
 * Complet" §7: kernel width 4, the first L outputs, Conv1D → SiLU → SSM).
 * The scan's x is
 *   x[b,t,d] = silu( conv_bias[d] + Σ_{k<K} conv_weight[d,k] · x_in[b, t−(K−1)+k, d] )
 * (x_in = 0 before the first token of each sequence; a cross-correlation like
 * torch's Conv1d), used both in Δ·B·x and in D·x; x itself is not written.
 *   x_in          [batch, seqlen, dim]      dtype        required
 *   conv_weight   [dim, conv_width]         float32      required
 *   conv_bias     [dim]                     float32      NULL -> zero
 *   conv_width    1 .. 4
 *   conv_init     [batch, dim, 3]           float32      NULL -> zero: the x_in
 *                 values of the 3 tokens before token 0, oldest first (with
 *                 initial_state, continues a sequence exactly: pass the last 3
 *                 x_in tokens of the preceding call)
 * Other arguments as selscan_fwd_from_state (initial_state may be NULL).
 */
SELSCAN_API int selscan_fwd_conv(const void *x_in, const float *conv_weight,
                                 const float *conv_bias, int conv_width,
                                 const float *conv_init, const void *delta,
                                 const float *A, const void *B, const void *C, const float *D,
                                 const void *z, const float *delta_bias, int softplus_flag,
                                 const float *initial_state, void *y, float *final_state,
                                 int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                                 selscan_dtype_t dtype, selscan_stream_t stream);

/* Input term of the discretisation. */
enum {
    SELSCAN_BBAR_DELTA = 0, /* Bbar·x = Δ·B·x ("SSM as RNN"; the default everywhere) */
    SELSCAN_BBAR_ZOH = 1    /* Bbar·x = (exp(Δ·A) − 1)/A · B·x, zero-order hold ("Mamba &
                               State Space Models — Guide Complet" §1 "Discrétisation",
                               diagonal A; Δ·B·x where A = 0) */
};

/* Options of selscan_fwd_ex; a zero-initialised struct (or NULL) is
 * selscan_fwd. Fields as in selscan_fwd_from_state and selscan_fwd_conv
 * (conv_width 0: no conv). */
typedef struct {
    const float *initial_state; /* [batch, dim, dstate] or NULL */
    const float *conv_weight;   /* [dim, conv_width] (conv_width > 0) */
    const float *conv_bias;     /* [dim] or NULL */
    const float *conv_init;     /* [batch, dim, 3] or NULL */
    int conv_width;             /* 0 .. 4 */
    int bbar_mode;              /* SELSCAN_BBAR_DELTA or SELSCAN_BBAR_ZOH */
} selscan_fwd_options_t;

/*
 * selscan_fwd_ex -- selscan_fwd with every option: an initial state, the
 * causal conv in front, and the input term (Δ·B·x or the zero-order-hold
 * term, both on the TMA-staged kernel where the shape allows it, else on the
 * generic kernels). options NULL: selscan_fwd. Unknown bbar_mode:
 * SELSCAN_ERR_BAD_DIM.
 */
SELSCAN_API int selscan_fwd_ex(const void *x, const void *delta, const float *A,
                               const void *B, const void *C, const float *D, const void *z,
                               const float *delta_bias, int softplus_flag,
                               const selscan_fwd_options_t *options, void *y,
                               float *final_state, int64_t batch, int64_t seqlen,
                               int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                               selscan_stream_t stream);

/*
 * selscan_fwd_noalloc -- selscan_fwd without any device allocation.
 *
 * The pages have no counterpart of this call; it exists for callers that
 * cannot allocate device memory while they run: code whose device memory is
 * all handed out by another allocator (a framework's caching allocator, an
 * arena reserved at start-up), latency-critical loops where an allocation may
 * block or fail, and processes without stream-ordered memory pools.
 *
 * Same arguments, results and launch plan as selscan_fwd. When the plan is
 * chunked, the chunk workspace is a fixed array inside the library of
 * SELSCAN_NOALLOC_WORKSPACE_BYTES bytes, held on every GPU that loads the
 * library until the process exits; sizes whose workspace (selscan_fwd_plan)
 * exceeds it are rejected with SELSCAN_ERR_WORKSPACE before anything runs.
 * This call never calls cudaMalloc, cudaMallocAsync or cudaFree.
 *  - Every call that needs the workspace looks up the array's device address
 *    on the current device (cudaGetSymbolAddress); nothing is cached, so a
 *    device reset or a re-created primary context, after which the array may
 *    sit at a new address, is picked up by the next call. The first such
 *    call on a device also loads the library's device code there; make it
 *    before any stream capture.
 *  - All calls on a device share the one array, and it keeps the contents
 *    of the last call. Calls that overlap on the GPU (e.g. on two streams
 *    without ordering between them) race on it and give wrong results; order
 *    them. The call itself clears, on `stream` and before its kernels, the
 *    counters that must start at zero (cudaMemsetAsync, no allocation); every
 *    other workspace element is written before it is read.
 */
#define SELSCAN_NOALLOC_WORKSPACE_BYTES (16u << 20)

SELSCAN_API int selscan_fwd_noalloc(const void *x, const void *delta, const float *A,
                                    const void *B, const void *C, const float *D,
                                    const void *z, const float *delta_bias,
                                    int softplus_flag, void *y, float *final_state,
                                    int64_t batch, int64_t seqlen, int64_t dim,
                                    int64_t dstate, selscan_dtype_t dtype,
                                    selscan_stream_t stream);

/*
 * selscan_fwd_plan -- the launch plan selscan_fwd would use for these sizes
 * with bf16 tensors on 16-byte boundaries (host only; no CUDA work). Writes,
 * through each non-NULL pointer, the number of sequence chunks (0 when there
 * is nothing to compute), the number of kernel launches (1 single pass; 3
 * chunked: chunk aggregates, carry, rescan) and the bytes of stream-ordered
 * workspace that call allocates. Returns SELSCAN_OK or the size errors of
 * selscan_fwd. The plan depends on the current device's SM count.
 */
SELSCAN_API int selscan_fwd_plan(int64_t batch, int64_t seqlen, int64_t dim,
                                 int64_t dstate, int64_t *chunks, int64_t *launches,
                                 int64_t *workspace_bytes);

/*
 * selscan_state_update -- one token of recurrent inference, in place
 * ("SSM as Convolution": recurrent mode for inference; Guide Complet §6: a
 * constant-size state instead of a growing cache).
 *
 *   state         [batch, dim, dstate]      float32      required, read and
 *                                                        overwritten with h_t
 *   x, delta      [batch, dim]              dtype        required
 *   A             [dim, dstate]             float32      required
 *   B, C          [batch, dstate]           dtype        required
 *   D             [dim]                     float32      NULL -> no skip term
 *   z             [batch, dim]              dtype        NULL -> no gate
 *   delta_bias    [dim]                     float32      NULL -> zero bias
 *   softplus_flag as for selscan_fwd
 *   y             [batch, dim]              dtype        required output
 *
 * A final_state from selscan_fwd is a valid `state`: steps continue the
 * sequence exactly where the scan stopped. No memory is allocated.
 */
SELSCAN_API int selscan_state_update(float *state, const void *x, const void *delta,
                         const float *A, const void *B, const void *C,
                         const float *D, const void *z,
                         const float *delta_bias, int softplus_flag, void *y,
                         int64_t batch, int64_t dim, int64_t dstate,
                         selscan_dtype_t dtype, selscan_stream_t stream);

/*
 * selscan_bwd -- gradient of selscan_fwd (the backward pass), with the
 * forward states recomputed instead of stored ("Mamba: co potrafią modele
 * przestrzeni stanów", "Cena selekcji": the backward pass recomputes the
 * intermediate states).
 *
 * For the loss Σ dy·y + Σ dfinal_state·final_state of the selscan_fwd call
 * with the same inputs, writes the loss's gradient with respect to each
 * input. With λ_t = ∂loss/∂h_t, λ after the last token = dfinal_state and
 * λ_t = ds_t·C_t + Abar_{t+1}·λ_{t+1}, ds_t = dy_t·silu(z_t):
 *
 *   x, delta, A, B, C, D, z, delta_bias, softplus_flag   as in selscan_fwd
 *   dy            [batch, seqlen, dim]      dtype        required
 *   dfinal_state  [batch, dim, dstate]      float32      NULL -> zero
 *   dx, ddelta    [batch, seqlen, dim]      dtype        required outputs
 *   dA            [dim, dstate]             float32      required output
 *                                                        (sum over batch and tokens)
 *   dB, dC        [batch, seqlen, dstate]   float32      required outputs
 *                                                        (sums over channels)
 *   dD            [dim]                     float32      NULL -> not written
 *   dz            [batch, seqlen, dim]      dtype        required iff z != NULL
 *   ddelta_bias   [dim]                     float32      NULL -> not written
 *   batch <= 65535, dstate 1..SELSCAN_MAX_DSTATE_BWD; other limits as in
 *   selscan_fwd.
 *
 * Every output is overwritten (not accumulated into); dB, dC, dA, dD and
 * ddelta_bias are float32 whatever `dtype` is. Results are deterministic
 * (fixed summation order, no atomics). Outputs must not overlap any input.
 * Takes a stream-ordered device workspace (cudaMallocAsync / cudaFreeAsync
 * on `stream`) of selscan_bwd_workspace_bytes() bytes: the state entering
 * every 8-token tile of every chain, and per-channel-tile partial sums of dB
 * and dC. Above 16 states the states go in groups of 16 computed side by
 * side; the workspace then holds every group's checkpoints and partials and
 * three float32 [batch, seqlen, dim] arrays per group, summed in group
 * order.
 */
SELSCAN_API int selscan_bwd(const void *x, const void *delta, const float *A,
                            const void *B, const void *C, const float *D, const void *z,
                            const float *delta_bias, int softplus_flag, const void *dy,
                            const float *dfinal_state, void *dx, void *ddelta, float *dA,
                            float *dB, float *dC, float *dD, void *dz, float *ddelta_bias,
                            int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                            selscan_dtype_t dtype, selscan_stream_t stream);

/* Host-only: device workspace bytes selscan_bwd takes for these sizes
 * (0 for empty or invalid sizes). */
SELSCAN_API int64_t selscan_bwd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t dim,
                                                int64_t dstate);

/*
 * selscan_bwd_workspace -- selscan_bwd on a workspace the caller provides
 * (e.g. from its own caching allocator) instead of one allocated on the
 * stream: same arguments and results, plus
 *   workspace        device buffer, 256-byte aligned, must not overlap any
 *                    input or output; NULL only when no token is processed
 *   workspace_bytes  its size: at least selscan_bwd_workspace_bytes() for
 *                    these sizes, else SELSCAN_ERR_WORKSPACE
 * Nothing is allocated. The workspace is free for reuse once the call's work
 * on `stream` has completed; its contents are not meaningful afterwards.
 */
SELSCAN_API int selscan_bwd_workspace(const void *x, const void *delta, const float *A,
                                      const void *B, const void *C, const float *D,
                                      const void *z, const float *delta_bias,
                                      int softplus_flag, const void *dy,
                                      const float *dfinal_state, void *dx, void *ddelta,
                                      float *dA, float *dB, float *dC, float *dD, void *dz,
                                      float *ddelta_bias, int64_t batch, int64_t seqlen,
                                      int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                                      void *workspace, int64_t workspace_bytes,
                                      selscan_stream_t stream);

/*
 * selscan_bwd_from_state -- the gradient of selscan_fwd_from_state: as
 * selscan_bwd_workspace, plus
 *   initial_state   [batch, dim, dstate]  float32  the forward's initial state
 *                                                  (NULL: zero)
 *   dinitial_state  [batch, dim, dstate]  float32  output: the loss's gradient
 *                                                  with respect to it (NULL: not
 *                                                  written); λ carried past the
 *                                                  first token, Abar_0·λ_0
 * workspace NULL: allocated on the stream as selscan_bwd does.
 */
SELSCAN_API int selscan_bwd_from_state(const void *x, const void *delta, const float *A,
                                       const void *B, const void *C, const float *D,
                                       const void *z, const float *delta_bias,
                                       int softplus_flag, const float *initial_state,
                                       const void *dy, const float *dfinal_state, void *dx,
                                       void *ddelta, float *dA, float *dB, float *dC,
                                       float *dD, void *dz, float *ddelta_bias,
                                       float *dinitial_state, int64_t batch, int64_t seqlen,
                                       int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                                       void *workspace, int64_t workspace_bytes,
                                       selscan_stream_t stream);

/*
 * selscan_bwd_conv -- the gradient of selscan_fwd_conv (conv_init NULL: the
 * conv sees zeros before token 0): as selscan_bwd_from_state with x_in, the
 * conv arguments, and
 *   dx_in          [batch, seqlen, dim]  dtype    output: gradient w.r.t. x_in
 *                                                 (through the conv and SiLU)
 *   dconv_weight   [dim, conv_width]     float32  output
 *   dconv_bias     [dim]                 float32  output (NULL: not written)
 * The workspace (NULL: allocated on the stream) needs
 * selscan_bwd_conv_workspace_bytes() bytes: besides the scan gradient's it
 * holds the conv output's gradient (float32 [batch, seqlen, dim]) and conv
 * partial sums. The conv output is recomputed, never stored.
 */
SELSCAN_API int selscan_bwd_conv(const void *x_in, const float *conv_weight,
                                 const float *conv_bias, int conv_width, const void *delta,
                                 const float *A, const void *B, const void *C, const float *D,
                                 const void *z, const float *delta_bias, int softplus_flag,
                                 const float *initial_state, const void *dy,
                                 const float *dfinal_state, void *dx_in, void *ddelta,
                                 float *dA, float *dB, float *dC, float *dD, void *dz,
                                 float *ddelta_bias, float *dinitial_state,
                                 float *dconv_weight, float *dconv_bias, int64_t batch,
                                 int64_t seqlen, int64_t dim, int64_t dstate,
                                 selscan_dtype_t dtype, void *workspace,
                                 int64_t workspace_bytes, selscan_stream_t stream);

/* Options of selscan_bwd_ex; zero-initialised (or NULL) is selscan_bwd. */
typedef struct {
    const float *initial_state;  /* [batch, dim, dstate] or NULL (the forward's) */
    float *dinitial_state;       /* [batch, dim, dstate] or NULL: its gradient */
    const float *conv_weight;    /* [dim, conv_width] (conv_width > 0): x is then the
                                    conv's input and dx its gradient */
    const float *conv_bias;      /* [dim] or NULL */
    int conv_width;              /* 0 .. 4 */
    float *dconv_weight;         /* [dim, conv_width] (conv_width > 0) */
    float *dconv_bias;           /* [dim] or NULL */
    int bbar_mode;               /* SELSCAN_BBAR_DELTA or SELSCAN_BBAR_ZOH */
} selscan_bwd_options_t;

/*
 * selscan_bwd_ex -- the gradient of selscan_fwd_ex with every option of the
 * forward that has one: initial state, the conv front end, and the input
 * term. With SELSCAN_BBAR_ZOH the forward input is c·B·x with
 * c = (exp(Δ·A[d,n]) − 1)/A[d,n] ("Mamba & State Space Models — Guide
 * Complet" §1, zero-order hold); its gradient uses ∂c/∂Δ = exp(Δ·A) and
 * ∂c/∂A = Δ²·f'(Δ·A), f(z) = (e^z − 1)/z. Arguments as selscan_bwd plus
 * the options; workspace NULL -> allocated on the stream, else at least
 * selscan_bwd_conv_workspace_bytes() (conv) or selscan_bwd_workspace_bytes()
 * bytes. Unknown bbar_mode or a negative conv_width: SELSCAN_ERR_BAD_DIM.
 */
SELSCAN_API int selscan_bwd_ex(const void *x, const void *delta, const float *A, const void *B,
                               const void *C, const float *D, const void *z,
                               const float *delta_bias, int softplus_flag, const void *dy,
                               const float *dfinal_state, const selscan_bwd_options_t *options,
                               void *dx, void *ddelta, float *dA, float *dB, float *dC, float *dD,
                               void *dz, float *ddelta_bias, int64_t batch, int64_t seqlen,
                               int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                               void *workspace, int64_t workspace_bytes, selscan_stream_t stream);

/* Host-only: workspace bytes selscan_bwd_conv takes (0 for empty or invalid sizes). */
SELSCAN_API int64_t selscan_bwd_conv_workspace_bytes(int64_t batch, int64_t seqlen,
                                                     int64_t dim, int64_t dstate);

/*
 * selscan_state_update_conv -- selscan_state_update with the causal conv +
 * SiLU of selscan_fwd_conv in front, for decoding after a selscan_fwd_conv
 * prefill: the token's x is silu(conv_bias + Σ_k conv_weight[d,k] · window),
 * the window being the 3 previous inputs kept in conv_state followed by
 * x_in; conv_state is then shifted to end with x_in.
 *   conv_state    [batch, dim, 3]           float32      in-out: the x_in values
 *                                                        of the 3 previous tokens,
 *                                                        oldest first
 *   x_in          [batch, dim]              dtype        required
 *   conv_weight   [dim, conv_width], conv_bias [dim] (NULL -> zero), conv_width 1..4
 * Other arguments as selscan_state_update. conv_state must not overlap any
 * other argument.
 */
SELSCAN_API int selscan_state_update_conv(float *state, float *conv_state, const void *x_in,
                                          const float *conv_weight, const float *conv_bias,
                                          int conv_width, const void *delta, const float *A,
                                          const void *B, const void *C, const float *D,
                                          const void *z, const float *delta_bias,
                                          int softplus_flag, void *y, int64_t batch,
                                          int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                                          selscan_stream_t stream);

/* Options of selscan_state_update_ex; zero-initialised (or NULL) is
 * selscan_state_update. Fields as in selscan_state_update_conv. */
typedef struct {
    float *conv_state;          /* [batch, dim, 3], in-out (conv_width > 0) */
    const float *conv_weight;   /* [dim, conv_width] */
    const float *conv_bias;     /* [dim] or NULL */
    int conv_width;             /* 0 .. 4 */
    int bbar_mode;              /* SELSCAN_BBAR_DELTA or SELSCAN_BBAR_ZOH */
} selscan_step_options_t;

/* selscan_state_update with every option (conv window, input term). */
SELSCAN_API int selscan_state_update_ex(float *state, const void *x, const void *delta,
                                        const float *A, const void *B, const void *C,
                                        const float *D, const void *z, const float *delta_bias,
                                        int softplus_flag, const selscan_step_options_t *options,
                                        void *y, int64_t batch, int64_t dim, int64_t dstate,
                                        selscan_dtype_t dtype, selscan_stream_t stream);

/*
 * selscan_ssd_fwd -- the scan with one scalar A per head, computed in the
 * chunked matrix form of "Mamba & State Space Models — Guide Complet" §5
 * ("SSD — State Space Dual": y = (L ◦ S)·u, a causal mask times a structured
 * semiseparable matrix). Channel d = h·headdim + p of head h:
 *   Δ_t = softplus(dt[b,t,h] + dt_bias[h]) (or no softplus),
 *   h_t[n] = exp(Δ_t·A[h])·h_{t−1}[n] + Δ_t·B[b,t,n]·x[b,t,d],
 *   y[b,t,d] = (Σ_n C[b,t,n]·h_t[n] + D[h]·x[b,t,d])·silu(z[b,t,d]),
 * i.e. selscan_fwd_from_state with delta, delta_bias, A and D broadcast from
 * the heads to their channels.
 *   x, z          [batch, seqlen, nheads·headdim]   dtype   (z NULL -> no gate)
 *   dt            [batch, seqlen, nheads]           dtype
 *   A, D, dt_bias [nheads]                          float32 (D, dt_bias nullable)
 *   B, C          [batch, seqlen, dstate]           dtype   (one group)
 *   initial_state, final_state [batch, nheads·headdim, dstate] float32, nullable
 *   headdim 1..64, dstate 1..128, batch and nheads ≤ 65535.
 * float32 I/O: 64-token chunks, products in float32 on the CUDA cores.
 * bfloat16 I/O: 128-token chunks on the tensor cores (tcgen05, float32
 * accumulators); the operands that are not inputs (the masked decay matrix
 * M, w ◦ x for the chunk states, the carried state h_in) are split into
 * bfloat16 high/low pairs, so the products keep about 16 significant bits.
 * Workspace (NULL: allocated on the stream) of selscan_ssd_workspace_bytes()
 * bytes; the caller owns every buffer. No output may overlap an input
 * (SELSCAN_ERR_ALIAS). Asynchronous like selscan_fwd.
 */
SELSCAN_API int selscan_ssd_fwd(const void *x, const void *dt, const float *A, const void *B,
                                const void *C, const float *D, const void *z,
                                const float *dt_bias, int softplus_flag,
                                const float *initial_state, void *y, float *final_state,
                                int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                                int64_t dstate, selscan_dtype_t dtype, void *workspace,
                                int64_t workspace_bytes, selscan_stream_t stream);

/* Host-only: workspace bytes selscan_ssd_fwd takes (0 for empty or invalid sizes). */
SELSCAN_API int64_t selscan_ssd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t nheads,
                                                int64_t headdim, int64_t dstate);

/*
 * selscan_device_status -- the library's sticky device-side error word on
 * the current device (synchronous: waits for prior work). 0 means no device
 * wait has given up; otherwise the code of the first one that did (1: a
 * sequence chunk waited too long for its predecessor's state; 2, 3: a
 * pipeline stage waited too long; 4: a tensor-core MMA or its operand copy
 * of selscan_ssd_fwd did not complete in time; 5: the state copy of a
 * selscan_state_update step did not complete in time). Every device-side wait in the library is
 * bounded (2 s); a wait that gives up records its code here and the kernel
 * returns instead of hanging, leaving its outputs undefined. `clear` nonzero
 * resets the word to 0 after reading it.
 */
SELSCAN_API int selscan_device_status(int *status, int clear);

/* Static, NUL-terminated description of a status code (never NULL). */
SELSCAN_API const char *selscan_status_string(int status);

/* Text of the CUDA error behind the calling thread's last SELSCAN_ERR_CUDA
 * (static storage; "no error" if none). */
SELSCAN_API const char *selscan_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SELSCAN_H_ */
