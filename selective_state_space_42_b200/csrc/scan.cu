// scan.cu -- selective-scan kernels for sm_100a.
//
// Pages: "Mamba & State Space Models — Guide Complet" §4 "Implémentation du
// SSM sélectif (S6)" (per-token Δ = softplus(·), Abar = exp(Δ·A), h = Abar·h +
// Bbar·x, y = C·h + D·x) and "Parallel Associative Scan" (operator
// (a,b)⊕(a',b') = (a·a', a·b' + b)); "Mamba и State Space Models: альтернатива
// Transformer", "SSM as RNN" (B scaled by delta) and "Hardware-Aware Scan"
// (the state carried across fixed blocks of the sequence); "Mamba: co potrafią
// modele przestrzeni stanów", "Cena selekcji" (discretize and recur in on-chip
// memory, never write the expanded state to HBM, fuse the steps in one kernel).
//
// Work decomposition. One thread owns one (batch row, channel) chain and keeps
// its d_state (≤ 16) float32 states in registers for the whole sequence (or
// chunk); a CTA of 128 threads covers 128 consecutive channels of one batch
// row, so every x/delta/z/y access of a warp is one contiguous 64-byte (bf16)
// or 128-byte (fp32) segment. B and C rows of a tile of tokens are staged once
// per CTA in shared memory as float32 and read by all 128 threads as
// broadcasts. Nothing of size L·D·N is ever written: Abar and Bbar·x live in
// registers only.
//
// Two exponent strategies, chosen per CTA at run time:
//  - general A: Abar[n] = 2^(Δ·A[d,n]·log2 e), one MUFU ex2 per element;
//  - A[d,n] = (n+1)·A[d,0] (within ladder_state's few ulps) for every n of
//    every channel of the CTA (the S4D/Mamba initialisation A = −(1..N), or
//    −exp(log(1..N)) in float32): Abar[n] = r^(n+1) with
//    r = 2^(Δ·A[d,0]·log2 e), i.e. one ex2 per token and a multiply per element.
//    Both are exp(Δ·A[d,n]) up to float32 rounding.
//
// Chunked plan (long sequences, few channels). Pass 1 scans every chunk from a
// zero state and stores its aggregate (P = Π Abar = 2^(A·log2e·ΣΔ), H = final
// state); the carry kernel composes the aggregates in order (the associative
// operator, later ∘ earlier) to give each chunk its incoming state; pass 2
// rescans every chunk from that state and writes y (and the final state).
#include "selscan_device.cuh"

namespace selscan {
namespace {

constexpr int kThreads = 128;  // channels per CTA
constexpr int kTileT = 64;     // tokens per shared-memory B/C tile

enum Mode { kModeScan = 0, kModeAggregate = 1 };

// Abar[n] for one token: either 16 ex2, or one ex2 and a power ladder of
// depth 4 (r, r², r³ = r²·r, r⁴ = r²·r², then doubling blocks).
template <bool kStruct>
__device__ __forceinline__ void discretize(float dt, const float (&A2)[kMaxN],
                                           float (&a)[kMaxN]) {
    if (kStruct) {
        const float r = ex2_approx(dt * A2[0]);
        a[0] = r;
        a[1] = r * r;
        a[2] = a[1] * r;
        a[3] = a[1] * a[1];
#pragma unroll
        for (int n = 4; n < 8; ++n) a[n] = a[n - 4] * a[3];
#pragma unroll
        for (int n = 8; n < 16; ++n) a[n] = a[n - 8] * a[7];
    } else {
#pragma unroll
        for (int n = 0; n < kMaxN; ++n) a[n] = ex2_approx(dt * A2[n]);
    }
}

template <typename T, bool kGate, int kMode, bool kStruct>
__device__ __forceinline__ void scan_tile(const ScanParams &p, int64_t b, int64_t d,
                                          int64_t t0, int nt,
                                          const float (*sB)[kMaxN],
                                          const float (*sC)[kMaxN],
                                          const float (&A2)[kMaxN], float dskip,
                                          float bias, float (&h)[kMaxN],
                                          float &dt_sum, bool conv,
                                          const float (&cw)[kMaxConv], float cb,
                                          float (&xw)[kMaxConv - 1]) {
    const T *__restrict__ xp = static_cast<const T *>(p.x);
    const T *__restrict__ dp = static_cast<const T *>(p.delta);
    const T *__restrict__ zp = static_cast<const T *>(p.z);
    T *__restrict__ yp = static_cast<T *>(p.y);
    const int64_t base = (b * p.seqlen + t0) * p.dim + d;
    constexpr int kU = 4;  // tokens whose loads are issued together
    for (int tt = 0; tt < nt; tt += kU) {
        float xv[kU], dv[kU], zv[kU];
#pragma unroll
        for (int k = 0; k < kU; ++k) {
            if (tt + k < nt) {
                const int64_t i = base + (int64_t)(tt + k) * p.dim;
                xv[k] = ldg_f32(xp + i);
                dv[k] = ldg_f32(dp + i);
                zv[k] = kGate ? ldg_f32(zp + i) : 0.0f;
            }
        }
#pragma unroll
        for (int k = 0; k < kU; ++k) {
            if (tt + k < nt) {
                if (conv) xv[k] = conv_step(cw, cb, xw, xv[k]);
                float dt = dv[k] + bias;
                if (p.softplus) dt = softplus_f32(dt);
                const float u = dt * xv[k];
                float a[kMaxN];
                discretize<kStruct>(dt, A2, a);
                const float *Bt0 = sB[tt + k];
                float Bz[kMaxN];  // B, times the ZOH factor in that mode
#pragma unroll
                for (int n = 0; n < kMaxN; ++n)
                    Bz[n] = p.zoh ? Bt0[n] * zoh_factor(dt * A2[n] * kLn2, a[n]) : Bt0[n];
                const float *Bt = Bz;
                if (kMode == kModeAggregate) {
                    dt_sum += dt;
#pragma unroll
                    for (int n = 0; n < kMaxN; ++n) h[n] = fmaf(a[n], h[n], u * Bt[n]);
                } else {
                    const float *Ct = sC[tt + k];
                    float y0 = 0.0f, y1 = 0.0f;
#pragma unroll
                    for (int n = 0; n < kMaxN; n += 2) {
                        h[n] = fmaf(a[n], h[n], u * Bt[n]);
                        h[n + 1] = fmaf(a[n + 1], h[n + 1], u * Bt[n + 1]);
                        y0 = fmaf(Ct[n], h[n], y0);
                        y1 = fmaf(Ct[n + 1], h[n + 1], y1);
                    }
                    float out = fmaf(dskip, xv[k], y0 + y1);
                    if (kGate) out *= silu_f32(zv[k]);
                    yp[base + (int64_t)(tt + k) * p.dim] = from_f32<T>(out);
                }
            }
        }
    }
}

template <typename T, bool kGate, int kMode>
__global__ void __launch_bounds__(kThreads)
scan_kernel(const ScanParams p) {
    __shared__ float sB[kTileT][kMaxN];
    __shared__ float sC[kTileT][kMaxN];

    // blockIdx.x = (b · nchunks + chunk) · ntiles + tile
    const int64_t blk = blockIdx.x;
    const int tile = (int)(blk % p.ntiles);
    const int64_t bc = blk / p.ntiles;
    const int chunk = (int)(bc % p.nchunks);
    const int64_t b = bc / p.nchunks;
    const int64_t d = (int64_t)tile * kThreads + threadIdx.x;
    const bool active = d < p.dim;
    const int64_t t_begin = (int64_t)chunk * p.chunk_len;
    const int64_t t_end = min(t_begin + p.chunk_len, p.seqlen);
    if (kMode == kModeAggregate && t_end >= p.seqlen) return;  // last chunk: unused

    // Per-channel constants. Padded states (n ≥ dstate) get A = 0 and B = C = 0,
    // so they stay exactly zero and add nothing to y.
    float A2[kMaxN];
    bool structured = true;
    float dskip = 0.0f, bias = 0.0f;
    if (active) {
        const float *Ar = p.A + d * p.dstate;
        const float a0 = Ar[0];
#pragma unroll
        for (int n = 0; n < kMaxN; ++n) {
            const float an = n < p.dstate ? Ar[n] : 0.0f;
            A2[n] = an * kLog2e;
            if (n < p.dstate) structured &= ladder_state(an, a0, n);
        }
        dskip = p.Dskip ? p.Dskip[d] : 0.0f;
        bias = p.delta_bias ? p.delta_bias[d] : 0.0f;
    } else {
#pragma unroll
        for (int n = 0; n < kMaxN; ++n) A2[n] = 0.0f;
    }
    structured = __syncthreads_and(structured);

    float h[kMaxN];
    const size_t ws_row = (((size_t)b * p.nchunks + chunk) * p.dim + (active ? d : 0)) * kMaxN;
    if (kMode == kModeScan && p.nchunks > 1 && active) {
#pragma unroll
        for (int n = 0; n < kMaxN; ++n) h[n] = p.ws_H[ws_row + n];  // carried-in state
    } else if (kMode == kModeScan && p.h0 && active) {
        const float *h0 = p.h0 + (b * p.dim + d) * p.dstate;
#pragma unroll
        for (int n = 0; n < kMaxN; ++n) h[n] = n < p.dstate ? h0[n] : 0.0f;
    } else {
#pragma unroll
        for (int n = 0; n < kMaxN; ++n) h[n] = 0.0f;
    }
    float dt_sum = 0.0f;

    // causal conv: this channel's taps and the inputs of the kMaxConv − 1
    // tokens before the chunk (zero before the sequence)
    const bool conv = p.conv_width > 0;
    float cw[kMaxConv] = {0.f, 0.f, 0.f, 0.f}, xw[kMaxConv - 1] = {0.f, 0.f, 0.f};
    float cb = 0.0f;
    if (conv && active) {
        load_conv_taps(p.conv_w, p.conv_width, d, cw);
        cb = p.conv_b ? p.conv_b[d] : 0.0f;
        const T *xp = static_cast<const T *>(p.x);
#pragma unroll
        for (int k = 0; k < kMaxConv - 1; ++k) {
            const int64_t t = t_begin - (kMaxConv - 1) + k;
            if (t >= 0)
                xw[k] = ldg_f32(xp + (b * p.seqlen + t) * p.dim + d);
            else if (p.conv_init)
                xw[k] = p.conv_init[(b * p.dim + d) * (kMaxConv - 1) + (t + kMaxConv - 1)];
        }
    }

    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);
    for (int64_t t0 = t_begin; t0 < t_end; t0 += kTileT) {
        const int nt = (int)min((int64_t)kTileT, t_end - t0);
        __syncthreads();  // previous tile fully consumed
        const T *Bt = Bp + (b * p.seqlen + t0) * p.dstate;
        const T *Ct = Cp + (b * p.seqlen + t0) * p.dstate;
        for (int i = threadIdx.x; i < kTileT * kMaxN; i += kThreads) {
            const int t = i / kMaxN, n = i % kMaxN;
            const bool in = t < nt && n < p.dstate;
            sB[t][n] = in ? ldg_f32(Bt + t * p.dstate + n) : 0.0f;
            if (kMode == kModeScan) sC[t][n] = in ? ldg_f32(Ct + t * p.dstate + n) : 0.0f;
        }
        __syncthreads();
        if (active) {
            if (structured)
                scan_tile<T, kGate, kMode, true>(p, b, d, t0, nt, sB, sC, A2, dskip,
                                                 bias, h, dt_sum, conv, cw, cb, xw);
            else
                scan_tile<T, kGate, kMode, false>(p, b, d, t0, nt, sB, sC, A2, dskip,
                                                  bias, h, dt_sum, conv, cw, cb, xw);
        }
    }

    if (!active) return;
    if (kMode == kModeAggregate) {
#pragma unroll
        for (int n = 0; n < kMaxN; ++n) {
            p.ws_P[ws_row + n] = ex2_approx(A2[n] * dt_sum);
            p.ws_H[ws_row + n] = h[n];
        }
    } else if (p.final_state && t_end >= p.seqlen) {
        float *fs = p.final_state + (b * p.dim + d) * p.dstate;
#pragma unroll
        for (int n = 0; n < kMaxN; ++n)
            if (n < p.dstate) fs[n] = h[n];
    }
}

// Chunk carry: hin_0 = h0 (or 0), hin_{c+1} = P_c · hin_c + H_c, hin_c
// written over H_c in place. Each chunk's aggregate is the affine map
// h ↦ P_c·h + H_c, and the maps compose associatively (later ∘ earlier:
// (P2, H2)∘(P1, H1) = (P2·P1, P2·H1 + H2)), so one warp per (b, d, group of
// 4 states) takes 32 chunks at a time, lane c chunk c0 + c: a warp-shuffle
// inclusive scan gives each lane the map from the block's start through its
// chunk, the exclusive map (the lane below's) applied to the state entering
// the block is its chunk's hin, and lane 31's map carries that state to the
// next block. Only the aggregates of chunks 0 .. nchunks-2 are read (pass 1
// skips the last chunk, which takes the identity map), so every workspace
// element is written before it is read.
__device__ __forceinline__ float4 fma4(float4 a, float4 b, float4 c) {
    return make_float4(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y), fmaf(a.z, b.z, c.z),
                       fmaf(a.w, b.w, c.w));
}
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
    return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}
__device__ __forceinline__ float4 shfl_up4(float4 v, int off) {
    return make_float4(__shfl_up_sync(0xffffffffu, v.x, off), __shfl_up_sync(0xffffffffu, v.y, off),
                       __shfl_up_sync(0xffffffffu, v.z, off), __shfl_up_sync(0xffffffffu, v.w, off));
}
__device__ __forceinline__ float4 shfl4(float4 v, int src) {
    return make_float4(__shfl_sync(0xffffffffu, v.x, src), __shfl_sync(0xffffffffu, v.y, src),
                       __shfl_sync(0xffffffffu, v.z, src), __shfl_sync(0xffffffffu, v.w, src));
}

constexpr int kCarryGroup = 4;  // states per lane

__global__ void carry_kernel(const ScanParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    constexpr int kGroups = kMaxN / kCarryGroup;
    if (gw >= p.batch * p.dim * kGroups) return;  // whole warps
    const int n0 = (int)(gw % kGroups) * kCarryGroup;
    const int64_t bd = gw / kGroups;
    const int64_t d = bd % p.dim, b = bd / p.dim;
    float hv[kCarryGroup];
#pragma unroll
    for (int k = 0; k < kCarryGroup; ++k)
        hv[k] = (p.h0 && n0 + k < p.dstate) ? p.h0[(b * p.dim + d) * p.dstate + n0 + k] : 0.0f;
    float4 h = make_float4(hv[0], hv[1], hv[2], hv[3]);
    const float4 one = make_float4(1.f, 1.f, 1.f, 1.f), zero = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < p.nchunks; c0 += 32) {
        const int c = c0 + lane;
        const size_t idx = (((size_t)b * p.nchunks + c) * p.dim + d) * kMaxN + n0;
        float4 P = one, H = zero;
        if (c + 1 < p.nchunks) {
            P = *reinterpret_cast<const float4 *>(p.ws_P + idx);
            H = *reinterpret_cast<const float4 *>(p.ws_H + idx);
        }
        // inclusive scan: lane c holds the map of chunks c0 .. c
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float4 Pp = shfl_up4(P, off), Hp = shfl_up4(H, off);
            if (lane >= off) {
                H = fma4(P, Hp, H);
                P = mul4(P, Pp);
            }
        }
        // exclusive: the map of chunks c0 .. c − 1, applied to the state
        // entering the block
        float4 Pe = shfl_up4(P, 1), He = shfl_up4(H, 1);
        if (lane == 0) {
            Pe = one;
            He = zero;
        }
        if (c < p.nchunks) *reinterpret_cast<float4 *>(p.ws_H + idx) = fma4(Pe, h, He);
        h = fma4(shfl4(P, 31), h, shfl4(H, 31));
    }
}

template <typename T, bool kGate, int kMode>
cudaError_t launch_one(const ScanParams &p, int64_t blocks, cudaStream_t stream) {
    scan_kernel<T, kGate, kMode><<<(unsigned)blocks, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const ScanParams &p, cudaStream_t stream) {
    const int64_t blocks = p.batch * p.nchunks * p.ntiles;
    cudaError_t e = cudaSuccess;
    if (p.nchunks > 1) {
        e = launch_one<T, false, kModeAggregate>(p, blocks, stream);
        if (e != cudaSuccess) return e;
        const int64_t threads = p.batch * p.dim * (kMaxN / kCarryGroup) * 32;
        carry_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (p.z)
        return launch_one<T, true, kModeScan>(p, blocks, stream);
    return launch_one<T, false, kModeScan>(p, blocks, stream);
}

}  // namespace

cudaError_t launch_carry(const ScanParams &p, cudaStream_t stream) {
    const int64_t threads = p.batch * p.dim * (kMaxN / kCarryGroup) * 32;
    carry_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(p);
    return cudaGetLastError();
}

int scan_channels_per_cta() { return kThreads; }
int scan_tile_tokens() { return kTileT; }

cudaError_t launch_scan(const ScanParams &p, bool bf16, cudaStream_t stream) {
    return bf16 ? launch_typed<__nv_bfloat16>(p, stream) : launch_typed<float>(p, stream);
}

}  // namespace selscan
