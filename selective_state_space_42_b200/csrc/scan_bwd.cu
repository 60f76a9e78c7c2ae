// scan_bwd.cu -- gradient of the selective scan: reverse sweep of the
// recurrence with the forward states recomputed from checkpoints.
//
// Pages: "Mamba: co potrafią modele przestrzeni stanów", "Cena selekcji"
// (the backward pass recomputes the intermediate states instead of storing
// them); the recurrence it differentiates is "Mamba & State Space Models —
// Guide Complet" §4 "Implémentation du SSM sélectif (S6)" and "Mamba и State
// Space Models: альтернатива Transformer", "SSM as RNN".
//
// With λ_t = ∂loss/∂h_t the reverse sweep is λ_t = ds_t·C_t + Abar_{t+1}·λ_{t+1}
// (λ after the last token = the final-state gradient), ds_t = dy_t·silu(z_t),
// and each token contributes
//   dB_t[n] += λ_t[n]·u_t,  dC_t[n] += ds_t·h_t[n]     (sums over channels)
//   du_t = Σ_n λ_t[n]·B_t[n],  dΔ_t = Σ_n λ_t[n]·A[n]·Abar_t[n]·h_{t−1}[n] + du_t·x_t
//   dA[n] += Δ_t·λ_t[n]·Abar_t[n]·h_{t−1}[n],  dx_t = du_t·Δ_t + ds_t·D,
//   dD += ds_t·x_t,  dz_t = dy_t·s_t·silu'(z_t),  ddelta_t = dΔ_t·σ(delta_t + bias)
// with u_t = Δ_t·x_t and s_t = Σ_n C_t[n]·h_t[n] + D·x_t.
//
// Organisation. A CTA owns 32 channels of one batch row for the whole
// sequence (no inter-CTA dependency). Lanes work in quads: lane (chain j,
// quarter q) holds states 4q..4q+3 of one chain. Tokens go in tiles of 16:
//  1. forward sweep: every tile's entering state is stored as a checkpoint
//     (float32, [batch][tiles][dim][16], 512 contiguous bytes per warp);
//  2. reverse sweep over the tiles, last first: recompute the tile's 16
//     states per lane from its checkpoint into registers, then walk the tile
//     backwards carrying λ in registers.
// Per-(token, channel) scalars (softplus, sigmoid, silu and its derivative,
// the decay base) are computed once by an owner thread into shared memory;
// the quad lanes read them. Channel sums of dB and dC are reduced within a
// warp by a shuffle reduce-scatter (8 values per lane → 1), across the 4
// warps in shared memory, and across channel tiles by a second kernel from a
// per-tile partial buffer (deterministic, no atomics). dA, dD and ddelta_bias
// are per-(batch row, channel) partials summed over batch rows the same way.
#include "selscan_device.cuh"

namespace selscan {
namespace {

constexpr int kSeg = 16;                 // tokens per tile (checkpoint interval)
constexpr int kChains = 32;              // channels per CTA
constexpr int kThreads = 4 * kChains;    // four lanes per channel
constexpr int kWarps = kThreads / 32;
constexpr int kVals = 2 * kMaxN;         // dB and dC values per token

struct BwdSmem {
    float4 sc[kSeg][kChains];   // Δ, u = Δ·x, ds = dy·silu(z), r = 2^(Δ·A[d,0]·log2 e)
    float4 so[kSeg][kChains];   // x, dy·silu'(z), σ(delta + bias), 0 (owner epilogue)
    float Bs[kSeg][kMaxN];      // B and C of the tile, float32, zero beyond dstate
    float Cs[kSeg][kMaxN];
    float s[kSeg][kChains];     // Σ_n C·h
    float2 duq[kSeg][kChains];  // Σ_n λ·B, Σ_n λ·A·Abar·h_prev
    float red[kWarps][kSeg][kVals];
};

// Decay factors Abar for the lane's four states at one token.
// Structured A (A[d, n] = (n+1)·A[d, 0]): powers of r; otherwise one ex2 each.
__device__ __forceinline__ void decay4(bool structured, int q, float dt, float r,
                                       const float (&Av)[4], float (&a)[4]) {
    if (structured) {
        const float r2 = r * r, r4 = r2 * r2, r8 = r4 * r4;
        const float base = q == 0 ? 1.0f : (q == 1 ? r4 : (q == 2 ? r8 : r8 * r4));
        a[0] = base * r;
        a[1] = a[0] * r;
        a[2] = a[1] * r;
        a[3] = a[2] * r;
    } else {
        const float dl = dt * kLog2e;
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = ex2_approx(dl * Av[i]);
    }
}

template <typename T>
__device__ __forceinline__ void load_bc(BwdSmem &S, const BwdParams &p, long long b,
                                        long long t0, bool withC) {
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);
    for (int e = threadIdx.x; e < kSeg * kMaxN; e += kThreads) {
        const int t = e / kMaxN, n = e % kMaxN;
        const long long tok = t0 + t;
        const bool ok = tok < p.seqlen && n < p.dstate;
        const long long idx = (b * p.seqlen + tok) * p.dstate + n;
        S.Bs[t][n] = ok ? ldg_f32(Bp + idx) : 0.0f;
        if (withC) S.Cs[t][n] = ok ? ldg_f32(Cp + idx) : 0.0f;
    }
}

// Owner step: per-(token, channel) scalars of tile t0 into shared memory.
// Tokens past the end and channels past dim get Δ = u = ds = 0 and r = 1,
// which leave every state and every gradient unchanged.
template <typename T, bool kGate, bool kSoftplus, bool kBwd>
__device__ __forceinline__ void owner_scalars(BwdSmem &S, const BwdParams &p, long long b,
                                              long long t0, int oc, int ot, long long od,
                                              float A0, float bias) {
    const T *xp = static_cast<const T *>(p.x);
    const T *dp = static_cast<const T *>(p.delta);
#pragma unroll
    for (int m = 0; m < kSeg / kWarps; ++m) {
        const int t = ot + kWarps * m;
        const long long tok = t0 + t;
        float4 sc = make_float4(0.f, 0.f, 0.f, 1.f);
        float4 so = make_float4(0.f, 0.f, 1.f, 0.f);
        if (od < p.dim && tok < p.seqlen) {
            const long long i = (b * p.seqlen + tok) * p.dim + od;
            const float xv = ldg_f32(xp + i);
            const float v = ldg_f32(dp + i) + bias;
            const float dt = kSoftplus ? softplus_f32(v) : v;
            sc.x = dt;
            sc.y = dt * xv;
            sc.w = ex2_approx(dt * A0 * kLog2e);
            if (kBwd) {
                const float dyv = ldg_f32(static_cast<const T *>(p.dy) + i);
                if (kGate) {
                    const float zv = ldg_f32(static_cast<const T *>(p.z) + i);
                    const float sg = sigmoid_f32(zv);
                    sc.z = dyv * zv * sg;
                    so.y = dyv * sg * fmaf(zv, 1.0f - sg, 1.0f);
                } else {
                    sc.z = dyv;
                }
                so.x = xv;
                so.z = kSoftplus ? sigmoid_f32(v) : 1.0f;
            }
        }
        S.sc[t][oc] = sc;
        if (kBwd) S.so[t][oc] = so;
    }
}

constexpr int kHalf = kSeg / 2;

// Shared-memory loads the compiler may neither merge with an earlier load of
// the same address nor move across one another: each token's operands are
// read when they are used, which keeps the per-token values of a half tile
// from all being live at once.
__device__ __forceinline__ float4 lds4(const void *ptr) {
    float4 v;
    const unsigned a = static_cast<unsigned>(__cvta_generic_to_shared(ptr));
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(a));
    return v;
}

// One token of the recurrence for the lane's four states.
__device__ __forceinline__ void fwd_token(const BwdSmem &S, int t, int jc, int q, bool structured,
                                          const float (&Av)[4], const float (&hin)[4],
                                          float (&hout)[4]) {
    const float4 sc = lds4(&S.sc[t][jc]);
    const float4 b4 = lds4(&S.Bs[t][4 * q]);
    float a[4];
    decay4(structured, q, sc.x, sc.w, Av, a);
    hout[0] = fmaf(a[0], hin[0], sc.y * b4.x);
    hout[1] = fmaf(a[1], hin[1], sc.y * b4.y);
    hout[2] = fmaf(a[2], hin[2], sc.y * b4.z);
    hout[3] = fmaf(a[3], hin[3], sc.y * b4.w);
}

// States through tokens kBase .. kBase + kHalf − 1 of the tile, nothing kept.
template <int kBase>
__device__ __forceinline__ void advance(const BwdSmem &S, int jc, int q, bool structured,
                                        const float (&Av)[4], float (&h)[4]) {
#pragma unroll
    for (int t = kBase; t < kBase + kHalf; ++t) {
        float hn[4];
        fwd_token(S, t, jc, q, structured, Av, h, hn);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = hn[i];
    }
}

// Tokens kBase .. kBase + kHalf − 1 of the tile: recompute their states from
// h (the state entering token kBase) into registers, store Σ_n C·h for the
// epilogue, then walk them backwards updating λ and the per-token gradients.
template <int kBase>
__device__ __forceinline__ void half_tile(BwdSmem &S, int jc, int q, int lane, int warp,
                                          bool structured, const float (&Av)[4],
                                          const float (&h)[4], float (&lam)[4],
                                          float (&dAacc)[4]) {
    float hs[kHalf + 1][4];  // hs[t + 1]: state after token kBase + t
#pragma unroll
    for (int i = 0; i < 4; ++i) hs[0][i] = h[i];
#pragma unroll
    for (int t = 0; t < kHalf; ++t) {
        fwd_token(S, kBase + t, jc, q, structured, Av, hs[t], hs[t + 1]);
        const float4 c4 = lds4(&S.Cs[kBase + t][4 * q]);
        float sp = c4.x * hs[t + 1][0];
        sp = fmaf(c4.y, hs[t + 1][1], sp);
        sp = fmaf(c4.z, hs[t + 1][2], sp);
        sp = fmaf(c4.w, hs[t + 1][3], sp);
        sp += __shfl_xor_sync(0xffffffffu, sp, 1);
        sp += __shfl_xor_sync(0xffffffffu, sp, 2);
        if (q == 0) S.s[kBase + t][jc] = sp;
    }
    const int jw = lane >> 2;
    const int b4bit = (lane >> 4) & 1, b3bit = (lane >> 3) & 1, b2bit = (lane >> 2) & 1;
#pragma unroll
    for (int t = kHalf - 1; t >= 0; --t) {
        const int tt = kBase + t;
        const float4 sc = lds4(&S.sc[tt][jc]);
        const float4 b4 = lds4(&S.Bs[tt][4 * q]);
        const float4 c4 = lds4(&S.Cs[tt][4 * q]);
        const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
        const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
        float a[4];
        decay4(structured, q, sc.x, sc.w, Av, a);
        float vals[8];
        float du = 0.f, qp = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            lam[i] = fmaf(sc.z, cv[i], lam[i]);     // λ_t
            const float hb = a[i] * hs[t][i];       // Abar_t·h_{t−1}
            const float lh = lam[i] * hb;
            du = fmaf(lam[i], bv[i], du);
            qp = fmaf(lh, Av[i], qp);
            dAacc[i] = fmaf(sc.x, lh, dAacc[i]);
            vals[i] = lam[i] * sc.y;                // dB
            vals[4 + i] = sc.z * hs[t + 1][i];      // dC
            lam[i] *= a[i];                         // Abar_t·λ_t, carried to token t − 1
        }
        du += __shfl_xor_sync(0xffffffffu, du, 1);
        du += __shfl_xor_sync(0xffffffffu, du, 2);
        qp += __shfl_xor_sync(0xffffffffu, qp, 1);
        qp += __shfl_xor_sync(0xffffffffu, qp, 2);
        if (q == 0) S.duq[tt][jc] = make_float2(du, qp);
        // reduce-scatter of the 8 values over the warp's 8 chains (lane bits
        // 4, 3, 2): afterwards lane (jw, q) holds value jw summed over them
        float w4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float keep = b4bit ? vals[4 + i] : vals[i];
            const float send = b4bit ? vals[i] : vals[4 + i];
            w4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
        float w2[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float keep = b3bit ? w4[2 + i] : w4[i];
            const float send = b3bit ? w4[i] : w4[2 + i];
            w2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
        const float keep = b2bit ? w2[1] : w2[0];
        const float send = b2bit ? w2[0] : w2[1];
        const float w1 = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        // value jw: 0..3 → dB[4q + jw], 4..7 → dC[4q + jw − 4]
        const int v = jw < 4 ? 4 * q + jw : kMaxN + 4 * q + (jw - 4);
        S.red[warp][tt][v] = w1;
    }
}

template <typename T, bool kGate, bool kSoftplus>
__global__ void __launch_bounds__(kThreads, 5) scan_bwd_kernel(const BwdParams p) {
    __shared__ BwdSmem S;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int q = lane & 3;                 // quarter: states 4q..4q+3
    const int jw = lane >> 2;               // chain within the warp
    const int jc = warp * 8 + jw;           // chain within the CTA
    const long long b = blockIdx.y;
    const long long d0 = (long long)blockIdx.x * kChains;
    const long long d = d0 + jc;
    const bool active = d < p.dim;
    const int oc = tid & 31, ot = tid >> 5;  // owner role: channel oc, tokens ot + 4m
    const long long od = d0 + oc;
    const int N = p.dstate;

    // this lane's A values (0 for states past dstate) and the structure test
    float Av[4];
    bool ok = true;
    const float A0 = active ? p.A[d * N] : 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int n = 4 * q + i;
        const bool has = active && n < N;
        Av[i] = has ? p.A[d * N + n] : 0.0f;
        if (has && Av[i] != (float)(n + 1) * A0) ok = false;
    }
    const bool structured = __all_sync(0xffffffffu, ok);
    const float oA0 = od < p.dim ? p.A[od * N] : 0.0f;
    const float obias = (od < p.dim && p.delta_bias) ? p.delta_bias[od] : 0.0f;
    const float oD = (od < p.dim && p.Dskip) ? p.Dskip[od] : 0.0f;
    const int K = p.ktiles;
    float4 *ck = reinterpret_cast<float4 *>(p.ckpt) + ((b * K) * p.dim + (active ? d : 0)) * 4 + q;
    const long long ck_stride = p.dim * 4;  // float4s between consecutive tiles

    // ---- 1. forward sweep: checkpoints ------------------------------------------
    {
        float h[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < K; ++k) {
            const long long t0 = (long long)k * kSeg;
            if (active) ck[k * ck_stride] = make_float4(h[0], h[1], h[2], h[3]);
            load_bc<T>(S, p, b, t0, false);
            owner_scalars<T, kGate, kSoftplus, false>(S, p, b, t0, oc, ot, od, oA0, obias);
            __syncthreads();
            advance<0>(S, jc, q, structured, Av, h);
            advance<kHalf>(S, jc, q, structured, Av, h);
            __syncthreads();
        }
    }

    // ---- 2. reverse sweep ---------------------------------------------------------
    float lam[4], dAacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int n = 4 * q + i;
        lam[i] = (active && n < N && p.dfinal) ? p.dfinal[(b * p.dim + d) * N + n] : 0.0f;
    }
    float accD = 0.f, accBias = 0.f;
    for (int k = K - 1; k >= 0; --k) {
        const long long t0 = (long long)k * kSeg;
        const float4 hc = active ? ck[k * ck_stride] : make_float4(0.f, 0.f, 0.f, 0.f);
        load_bc<T>(S, p, b, t0, true);
        owner_scalars<T, kGate, kSoftplus, true>(S, p, b, t0, oc, ot, od, oA0, obias);
        __syncthreads();

        // second half of the tile first, then the first half; each half
        // recomputes its 8 states into registers from the checkpoint
        float h[4] = {hc.x, hc.y, hc.z, hc.w};
        advance<0>(S, jc, q, structured, Av, h);
        half_tile<kHalf>(S, jc, q, lane, warp, structured, Av, h, lam, dAacc);
        h[0] = hc.x;
        h[1] = hc.y;
        h[2] = hc.z;
        h[3] = hc.w;
        half_tile<0>(S, jc, q, lane, warp, structured, Av, h, lam, dAacc);
        __syncthreads();

        // owner epilogue: dx, ddelta, dz; dD and ddelta_bias partials
#pragma unroll
        for (int m = 0; m < kSeg / kWarps; ++m) {
            const int t = ot + kWarps * m;
            const long long tok = t0 + t;
            if (od < p.dim && tok < p.seqlen) {
                const long long i = (b * p.seqlen + tok) * p.dim + od;
                const float4 sc = S.sc[t][oc];
                const float4 so = S.so[t][oc];
                const float2 dq = S.duq[t][oc];
                const float ddt = fmaf(dq.x, so.x, dq.y);
                const float dv = ddt * so.z;
                static_cast<T *>(p.dx)[i] = from_f32<T>(fmaf(dq.x, sc.x, sc.z * oD));
                static_cast<T *>(p.ddelta)[i] = from_f32<T>(dv);
                if (kGate) {
                    const float s = fmaf(oD, so.x, S.s[t][oc]);
                    static_cast<T *>(p.dz)[i] = from_f32<T>(s * so.y);
                }
                accD = fmaf(sc.z, so.x, accD);
                accBias += dv;
            }
        }
        // this tile's channel sums of dB and dC
        for (int e = tid; e < kSeg * kVals; e += kThreads) {
            const int t = e / kVals, v = e % kVals;
            const long long tok = t0 + t;
            if (tok < p.seqlen) {
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) sum += S.red[w][t][v];
                p.part[((b * p.ctiles + blockIdx.x) * p.seqlen + tok) * kVals + v] = sum;
            }
        }
        __syncthreads();
    }

    // per-(batch row, channel) partials
    if (active) {
#pragma unroll
        for (int i = 0; i < 4; ++i) p.pA[(b * p.dim + d) * kMaxN + 4 * q + i] = dAacc[i];
    }
    float *red = &S.red[0][0][0];
    red[tid] = accD;
    red[kThreads + tid] = accBias;
    __syncthreads();
    if (tid < kChains && od < p.dim) {
        float sd = 0.f, sb = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            sd += red[w * 32 + tid];
            sb += red[kThreads + w * 32 + tid];
        }
        p.pD[b * p.dim + od] = sd;
        p.pbias[b * p.dim + od] = sb;
    }
}

// dB[b, t, n] and dC[b, t, n]: sums of the channel-tile partials.
__global__ void bwd_reduce_bc_kernel(const BwdParams p) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = p.batch * p.seqlen * kVals;
    if (e >= total) return;
    const long long b = e / (p.seqlen * kVals);
    const long long rest = e - b * p.seqlen * kVals;  // tok * 32 + v
    const int v = (int)(rest % kVals);
    const long long tok = rest / kVals;
    const float *src = p.part + (b * p.ctiles) * p.seqlen * kVals + rest;
    float sum = 0.f;
    for (int c = 0; c < p.ctiles; ++c) sum += src[(long long)c * p.seqlen * kVals];
    const int n = v % kMaxN;
    if (n >= p.dstate) return;
    float *dst = v < kMaxN ? p.dB : p.dC;
    dst[(b * p.seqlen + tok) * p.dstate + n] = sum;
}

// dA[d, n], dD[d], ddelta_bias[d]: sums over batch rows.
__global__ void bwd_reduce_params_kernel(const BwdParams p) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= p.dim * kMaxN) return;
    const long long d = e / kMaxN;
    const int n = (int)(e % kMaxN);
    if (n < p.dstate) {
        float s = 0.f;
        for (long long b = 0; b < p.batch; ++b) s += p.pA[(b * p.dim + d) * kMaxN + n];
        p.dA[d * p.dstate + n] = s;
    }
    if (n == 0) {
        float sd = 0.f, sb = 0.f;
        for (long long b = 0; b < p.batch; ++b) {
            sd += p.pD[b * p.dim + d];
            sb += p.pbias[b * p.dim + d];
        }
        if (p.dD) p.dD[d] = sd;
        if (p.ddelta_bias) p.ddelta_bias[d] = sb;
    }
}

template <typename T, bool kGate>
cudaError_t launch_gate(const BwdParams &p, cudaStream_t stream) {
    const dim3 grid((unsigned)p.ctiles, (unsigned)p.batch);
    if (p.softplus)
        scan_bwd_kernel<T, kGate, true><<<grid, kThreads, 0, stream>>>(p);
    else
        scan_bwd_kernel<T, kGate, false><<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

int bwd_tile_tokens() { return kSeg; }
int bwd_tile_channels() { return kChains; }

cudaError_t launch_scan_bwd(const BwdParams &p, bool bf16, cudaStream_t stream) {
    cudaError_t e;
    if (bf16)
        e = p.z ? launch_gate<__nv_bfloat16, true>(p, stream)
                : launch_gate<__nv_bfloat16, false>(p, stream);
    else
        e = p.z ? launch_gate<float, true>(p, stream) : launch_gate<float, false>(p, stream);
    if (e != cudaSuccess) return e;
    const long long nbc = p.batch * p.seqlen * kVals;
    bwd_reduce_bc_kernel<<<(unsigned)((nbc + 255) / 256), 256, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long npar = p.dim * kMaxN;
    bwd_reduce_params_kernel<<<(unsigned)((npar + 255) / 256), 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace selscan
