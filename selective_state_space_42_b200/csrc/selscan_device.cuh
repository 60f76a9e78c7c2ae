// selscan_device.cuh -- device-side helpers shared by the libselscan kernels:
// element loads/stores for the two I/O dtypes, the MUFU wrappers, softplus
// and silu in float32, and the launch-parameter structs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace selscan {

constexpr int kMaxN = 16;           // largest supported d_state
constexpr int kMaxConv = 4;         // widest causal conv in front of the scan
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// A[d, n] is taken as (n + 1)·A[d, 0], so that a token's decay factors are
// powers of one base, when the two differ by at most 2^−21 of A[d, n] (4 to
// 8 float32 ulps). exp(Δ·A) then changes by a relative Δ·|A|·2^−21: no more
// than the MUFU exponential's own error while Δ·|A| ≤ 1/2, and beyond that
// only in factors below e^−1/2. The pages' A = −exp(log(1..N)), which float32
// rounds a few ulps off the integers, qualifies.
__host__ __device__ __forceinline__ bool ladder_state(float an, float a0, int n) {
    return fabsf(an - (float)(n + 1) * a0) <= 0x1p-21f * fabsf(an);
}

// ---- element I/O -------------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);  // round to nearest even
}

template <typename T>
__device__ __forceinline__ float ldg_f32(const T *p) { return to_f32(__ldg(p)); }

// ---- special-function unit (MUFU) instructions ----------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(v) = max(v, 0) + log1p(w), w = exp(-|v|) in (0, 1].
// log1p(w): for w < 1/16 the alternating series w − w²/2 + … + w⁷/7 (truncation
// below w⁸/8 < 1e-10 relative); otherwise log2(1 + w)·ln 2, where 1 + w ≥ 1.0625
// keeps lg2's absolute error small relative to the result. Both branches are
// evaluated and one is selected, so warps never diverge here.
__device__ __forceinline__ float softplus_f32(float v) {
    const float w = ex2_approx(-fabsf(v) * kLog2e);
    float s = fmaf(w, -1.0f / 7.0f, 1.0f / 6.0f);
    s = fmaf(w, -s, 1.0f / 5.0f);
    s = fmaf(w, -s, 1.0f / 4.0f);
    s = fmaf(w, -s, 1.0f / 3.0f);
    s = fmaf(w, -s, 1.0f / 2.0f);
    s = fmaf(w, -s, 1.0f);
    const float series = w * s;
    const float viaLog = lg2_approx(1.0f + w) * kLn2;
    return fmaxf(v, 0.0f) + (w < 0.0625f ? series : viaLog);
}

__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// silu(z) = z · sigmoid(z) = z / (1 + e^-z); e^-z overflowing to +inf gives 0.
__device__ __forceinline__ float silu_f32(float z) {
    return z * rcp_approx(1.0f + ex2_approx(-z * kLog2e));
}

// silu(z) = z·(1 + tanh(z/2))/2 with one MUFU tanh, for bf16 outputs: tanh's
// absolute error (~5e-4 at most) gives |silu error| ≤ ~2.5e-4·|z|, well under
// the bf16 rounding of y for the gate values that matter.
__device__ __forceinline__ float silu_tanh(float z) {
    const float h = 0.5f * z;
    return fmaf(h, tanh_approx(h), h);
}

// Causal conv taps of one channel, right-aligned in four slots: slot 3
// multiplies the current token, slot 3 − j the token j steps back; slots
// before the filter's start are zero.
__device__ __forceinline__ void load_conv_taps(const float *w, int width, long long d,
                                               float (&cw)[kMaxConv]) {
#pragma unroll
    for (int k = 0; k < kMaxConv; ++k) {
        const int j = k - (kMaxConv - width);  // filter index of slot k
        cw[k] = j >= 0 ? w[d * width + j] : 0.0f;
    }
}

// Zero-order-hold input factor relative to Δ: (exp(z) − 1)/z with z = Δ·A,
// given a = exp(z). Below |z| = 1/32 a four-term series (truncation under
// z⁴/120 < 1e-8 relative); above, (a − 1)/z. The factor is 1 at z = 0, so
// the ZOH input term Δ·B·x·factor reduces to the Δ·B·x term there.
__device__ __forceinline__ float zoh_factor(float z, float a) {
    const float series = fmaf(z, fmaf(z, fmaf(z, 1.0f / 24.0f, 1.0f / 6.0f), 0.5f), 1.0f);
    return fabsf(z) < 0.03125f ? series : (a - 1.0f) / z;
}

// sigmoid(v) = 1 / (1 + e^-v); e^-v overflowing to +inf gives 0.
__device__ __forceinline__ float sigmoid_f32(float v) {
    return rcp_approx(1.0f + ex2_approx(-v * kLog2e));
}

// One step of the causal conv + SiLU: xw holds the three previous inputs
// (oldest first) and is shifted to include xi.
__device__ __forceinline__ float conv_step(const float (&cw)[kMaxConv], float cb,
                                           float (&xw)[kMaxConv - 1], float xi) {
    const float pre = fmaf(cw[0], xw[0], fmaf(cw[1], xw[1], fmaf(cw[2], xw[2], fmaf(cw[3], xi, cb))));
    xw[0] = xw[1];
    xw[1] = xw[2];
    xw[2] = xi;
    return silu_f32(pre);
}

// ---- launch parameters -------------------------------------------------------------
struct ScanParams {
    const void *x, *delta, *z, *B, *C;
    const float *A, *Dskip, *delta_bias;
    void *y;
    float *final_state;
    const float *h0;     // state before the first token, [batch][dim][dstate] (NULL: zero)
    const float *conv_w; // causal conv in front of the scan: [dim][conv_width] (NULL: none)
    const float *conv_b; // [dim] (NULL: zero)
    const float *conv_init;  // [batch][dim][kMaxConv − 1]: conv inputs before token 0 (NULL: zero)
    int conv_width;      // 0 (no conv) or 1..kMaxConv
    int zoh;             // input term: 0 Δ·B·x, 1 (exp(Δ·A) − 1)/A·B·x
    int64_t batch, seqlen, dim;
    int dstate;
    int softplus;
    int64_t chunk_len;   // tokens per chunk (== seqlen when not chunked)
    int nchunks;         // chunks per sequence
    int ntiles;          // channel tiles per batch row
    // chunk workspace, [batch][nchunks][dim][kMaxN] each (NULL if nchunks == 1):
    float *ws_P;         // pass 1: product of Abar over the chunk
    float *ws_H;         // pass 1: chunk state from zero; after carry: state entering the chunk
};

struct StepParams {
    float *state;
    const void *x, *delta, *z, *B, *C;
    const float *A, *Dskip, *delta_bias;
    void *y;
    float *conv_state;     // [batch][dim][kMaxConv − 1] conv inputs before the token (in-out)
    const float *conv_w;   // [dim][conv_width] (conv_width > 0)
    const float *conv_b;   // [dim] (NULL: zero)
    int conv_width;        // 0: no conv
    int zoh;               // input term: 0 Δ·B·x, 1 (exp(Δ·A) − 1)/A·B·x
    int64_t batch, dim;
    int dstate;
    int softplus;
};


// The library's device error word (defined with the TMA scan).
cudaError_t device_status_address(int **p);

// Persistent TMA-staged scan (scan_tma.cu).
// kModeCkpt: the one-pass plan's hand-off without y, writing instead the
// state entering every 8-token sub-tile (the gradient's checkpoints).
enum : int { kModeSeq = 0, kModeAgg = 1, kModeRescan = 2, kModeCkpt = 3 };

struct TmaScanParams {
    const void *B, *C;
    const float *A, *Dskip, *delta_bias;
    void *y;
    float *final_state;
    const float *h0;      // state before the first token, [batch][dim][dstate] (NULL: zero)
    const float *conv_w;  // causal conv in front of the scan: [dim][conv_width] (NULL: none)
    const float *conv_b;  // [dim] (NULL: zero)
    const float *conv_init;  // [batch][dim][kMaxConv − 1]: conv inputs before token 0 (NULL: zero)
    int conv_width;       // 0 (no conv) or 1..kMaxConv
    int zoh;              // input term: 0 Δ·B·x, 1 (exp(Δ·A) − 1)/A·B·x
    long long batch, seqlen, dim;
    int dstate;
    int softplus;
    int mode;             // kModeSeq | kModeAgg | kModeRescan
    int ntiles;           // 128-channel tiles per batch row
    long long chunk_len;  // tokens per unit (a multiple of the token tile)
    int nchunks;          // units per sequence
    long long groups;     // batch * ntiles
    int units;            // tickets handed out by this launch
    // workspace (zeroed counters + arrays)
    int *ticket;          // next ticket of this launch
    int *flags;           // kModeSeq: chunks completed, per group and consumer warp
    int *abort_all;       // set by any CTA whose wait gave up; stops the others
    float *ws_state;      // kModeSeq: [groups][128][16] state handed between units
    float *ws_P, *ws_H;   // chunked: [batch][nchunks][dim][16]
    unsigned long long timeout_ns;  // bound on every device-side wait
    int skip_release_chunk;  // fault-injection hook for tests: the kSeq units of this
                             // chunk publish no completion flag (-1: none)
    // kModeCkpt: [batch][ck_tiles][dim][16] float32, per (batch row, 8-token
    // tile, channel) the lower lane's states 0,2,4,6 | 8,10,12,14 then the upper
    // lane's 1,3,5,7 | 9,11,13,15 (the gradient kernel's layout)
    float *ckpt;
    long long ck_tiles;
};

cudaError_t launch_scan_tma(const TmaScanParams &p, bool bf16, const void *x, const void *dl,
                            const void *z, cudaStream_t stream);
cudaError_t read_device_status(int *out, bool clear);
int tma_tile_channels();
int tma_tile_tokens(bool bf16);
cudaError_t launch_carry(const ScanParams &p, cudaStream_t stream);

// Host-side launchers (one translation unit per kernel family).
cudaError_t launch_scan(const ScanParams &p, bool bf16, cudaStream_t stream);
cudaError_t launch_scan_wide(const ScanParams &p, bool bf16, cudaStream_t stream);
int wide_max_dstate();
cudaError_t launch_state_update(const StepParams &p, bool bf16, cudaStream_t stream);
int scan_channels_per_cta();
int scan_tile_tokens();

// Host-side helpers of the C ABI (api.cu).
int cuda_fail(cudaError_t e);  // records e for selscan_last_cuda_error

// A selscan_fwd call after validation: which kernels run, their parameters,
// and the workspace they need.
struct FwdPlan {
    bool tma = false;     // TMA-staged persistent kernel (else the generic kernels)
    ScanParams gp{};      // generic kernels (and the carry kernel)
    TmaScanParams tp{};   // TMA kernel
    const void *x = nullptr, *delta = nullptr, *z = nullptr;
    bool bf16 = false;
    bool wide = false;    // d_state above kMaxN: scan_wide.cu
    int chunks = 1;       // sequence chunks
    int launches = 0;     // kernel launches
    size_t ws_bytes = 0;  // workspace bytes
    size_t ws_clear = 0;  // leading workspace bytes zeroed before the launches
};

int fwd_setup(const void *x, const void *delta, const float *A, const void *B,
              const void *C, const float *D, const void *z, const float *delta_bias,
              int softplus_flag, const float *h0, const float *conv_w, const float *conv_b,
              const float *conv_init, int conv_width, int zoh, void *y, float *final_state,
              int64_t batch,
              int64_t seqlen, int64_t dim, int64_t dstate, int dtype,
              cudaStream_t stream, FwdPlan *plan, bool *done);
// Plans for the given sizes assuming 16-byte aligned tensors (selscan_fwd_plan).
void plan_for_sizes(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int dtype,
                    bool aligned, FwdPlan *plan);
// Points the plan at a workspace of plan->ws_bytes bytes and launches it.
cudaError_t fwd_run(FwdPlan *plan, void *ws, cudaStream_t stream);

}  // namespace selscan
