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
// Organisation. One thread per (batch row, channel) chain holds its 16
// states in registers, two per packed f32x2 instruction; a CTA is one warp of
// 32 consecutive channels of one batch row and owns them for the whole
// sequence (no inter-CTA dependency). Tokens go in tiles of 8:
//  1. forward sweep: the state entering every tile is stored as a checkpoint
//     (float32, [batch][tiles][dim][16]);
//  2. reverse sweep over the tiles, last first: recompute the tile's states
//     from its checkpoint into shared memory (with the per-token scalars:
//     softplus, its derivative σ, silu(z) and its derivative, the decay base),
//     then walk the tile backwards carrying λ in registers.
// Global inputs of the next tile (x, delta, z, dy, B, C, the checkpoint) are
// loaded into registers while the current tile is computed. The channel sums
// of dB and dC are formed per token through shared memory (each lane writes
// its 32 values, swizzled so that the writes and the column reads are free of
// bank conflicts; eight lanes sum each group of four values over 8 channels,
// two shuffles finish the warp sum) and written as one 128-byte row per token
// to a per-channel-tile partial buffer, which a second kernel sums over the
// channel tiles: deterministic, no atomics. dA, dD and ddelta_bias are
// per-(batch row, channel) partials summed over batch rows the same way.
//
// Above 16 states the states go in groups of 16, one grid plane per group,
// each the pass above on its states. The recurrence, λ and the per-state
// gradients separate by state; the per-token sums over n (dx, dΔ and the
// pre-gate output s, which dz needs) are written per group and summed in
// group order by bwd_groups_finish_kernel, which also applies σ and silu'.
// The ZOH input term (p.zoh) scales B by f(Δ·A[n]) = (e^z − 1)/z in the
// recomputed forward and takes f and f' into dB, dx, dΔ and dA.
#include "bwd_params.cuh"

namespace selscan {
namespace {

constexpr int kSeg = 8;                  // tokens per tile (checkpoint interval)
constexpr int kChains = 32;              // channels per CTA: one warp
constexpr int kVals = 2 * kMaxN;         // dB and dC values per token
constexpr int kPairs = kMaxN / 2;        // f32x2 registers per state vector

__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 dup2(float v) { return make_float2(v, v); }

struct BwdSmem {
    float Bs[kSeg][kMaxN];             // B and C of the tile, float32, zero beyond dstate
    float Cs[kSeg][kMaxN];
    float4 sc[kSeg][kChains];          // Δ, u = Δ·x, ds = dy·silu(z), r = 2^(Δ·A[d,0]·log2 e)
    float4 so[kSeg][kChains];          // x, dy·silu'(z), σ(delta + bias), s = Σ C·h + D·x
    float4 hs[kSeg + 1][4][kChains];   // hs[0]: entering state; hs[t + 1]: after token t
    float4 red[kVals / 4][kChains];    // one token's dB (groups 0-3), dC (4-7), swizzled
};

// Raw per-token inputs of one tile for this lane's channel.
template <typename T> struct Raw {
    T x[kSeg], dl[kSeg], z[kSeg], dy[kSeg];
    T xh[kMaxConv - 1];  // conv: the inputs of the kMaxConv − 1 tokens before the tile
};

template <typename T, bool kGate, bool kBwd, bool kConv = false>
__device__ __forceinline__ void load_raw(Raw<T> &r, const BwdParams &p, long long b,
                                         long long t0, long long d, bool active) {
    const T zero = from_f32<T>(0.0f);
    if (kConv) {
#pragma unroll
        for (int k = 0; k < kMaxConv - 1; ++k) {
            const long long tok = t0 - (kMaxConv - 1) + k;
            const bool ok = active && tok >= 0 && tok < p.seqlen;
            r.xh[k] = ok ? __ldg(static_cast<const T *>(p.x) + (b * p.seqlen + tok) * p.dim + d)
                         : zero;
        }
    }
#pragma unroll
    for (int t = 0; t < kSeg; ++t) {
        const long long tok = t0 + t;
        const bool ok = active && tok < p.seqlen;
        const long long i = (b * p.seqlen + tok) * p.dim + d;
        r.x[t] = ok ? __ldg(static_cast<const T *>(p.x) + i) : zero;
        r.dl[t] = ok ? __ldg(static_cast<const T *>(p.delta) + i) : zero;
        if (kBwd) {
            r.dy[t] = ok ? __ldg(static_cast<const T *>(p.dy) + i) : zero;
            if (kGate) r.z[t] = ok ? __ldg(static_cast<const T *>(p.z) + i) : zero;
        }
    }
}

// Four B and four C elements of the tile for this lane: token lane / 4,
// states ng + 4·(lane % 4) .. + 3 of the 16-state group starting at ng (zero
// past the end or past dstate).
template <typename T>
__device__ __forceinline__ void load_bc(float (&bv)[4], float (&cv)[4], const BwdParams &p,
                                        long long b, long long t0, int lane, bool withC, int ng) {
    const int t = lane >> 2, n0 = ng + 4 * (lane & 3);
    const long long tok = t0 + t;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool ok = tok < p.seqlen && n0 + i < p.dstate;
        const long long idx = (b * p.seqlen + tok) * p.dstate + n0 + i;
        bv[i] = ok ? ldg_f32(static_cast<const T *>(p.B) + idx) : 0.0f;
        cv[i] = (ok && withC) ? ldg_f32(static_cast<const T *>(p.C) + idx) : 0.0f;
    }
}

__device__ __forceinline__ void store_bc(BwdSmem &S, const float (&bv)[4], const float (&cv)[4],
                                         int lane) {
    const int t = lane >> 2, n0 = 4 * (lane & 3);
    *reinterpret_cast<float4 *>(&S.Bs[t][n0]) = make_float4(bv[0], bv[1], bv[2], bv[3]);
    *reinterpret_cast<float4 *>(&S.Cs[t][n0]) = make_float4(cv[0], cv[1], cv[2], cv[3]);
}

// Abar for the 16 states at one token. Structured A: r^(n+1) by a power
// ladder; otherwise 2^(Δ·A[n]·log2 e) per state (Al = A·log2 e).
template <bool kStruct>
__device__ __forceinline__ void decay16(float dt, float r, const float2 (&Al)[kPairs],
                                        float2 (&a)[kPairs]) {
    if (kStruct) {
        const float r2 = r * r;
        a[0] = make_float2(r, r2);
        a[1] = mul2(a[0], dup2(r2));
        const float2 q4 = dup2(a[1].y);
        a[2] = mul2(a[0], q4);
        a[3] = mul2(a[1], q4);
        const float2 q8 = dup2(a[3].y);
#pragma unroll
        for (int j = 0; j < 4; ++j) a[4 + j] = mul2(a[j], q8);
    } else {
#pragma unroll
        for (int j = 0; j < kPairs; ++j)
            a[j] = make_float2(ex2_approx(dt * Al[j].x), ex2_approx(dt * Al[j].y));
    }
}

// Derivative of the ZOH factor f(z) = (e^z − 1)/z given a = e^z:
// f'(z) = (a·(z − 1) + 1)/z²; below |z| = 1/2 the series Σ_m (m + 1)·z^m /
// (m + 2)! to m = 7 (the next term is under 1e-8 of the sum), above the
// closed form (no cancellation there: a·(z − 1) + 1 ≥ 0.17).
__device__ __forceinline__ float zoh_factor_deriv(float z, float a) {
    float s = fmaf(z, 1.0f / 45360.0f, 1.0f / 5760.0f);
    s = fmaf(z, s, 1.0f / 840.0f);
    s = fmaf(z, s, 1.0f / 144.0f);
    s = fmaf(z, s, 1.0f / 30.0f);
    s = fmaf(z, s, 1.0f / 8.0f);
    s = fmaf(z, s, 1.0f / 3.0f);
    s = fmaf(z, s, 0.5f);
    return fabsf(z) < 0.5f ? s : fmaf(a, z - 1.0f, 1.0f) / (z * z);
}

// z = Δ·A[n] (natural units) of states 2j, 2j + 1: structured A[n] =
// (n + 1)·A[0]; otherwise Al = A·log2 e.
template <bool kStruct>
__device__ __forceinline__ float2 zoh_z(float dt, int j, float A0n, const float2 (&Al)[kPairs]) {
    return kStruct ? make_float2(dt * A0n * (float)(2 * j + 1), dt * A0n * (float)(2 * j + 2))
                   : make_float2(dt * Al[j].x * kLn2, dt * Al[j].y * kLn2);
}

// States 4q .. 4q+3 of a shared-memory row as two f32x2 pairs.
__device__ __forceinline__ void ld_quad(const float *base, int q, float2 &lo, float2 &hi) {
    const float4 v = *reinterpret_cast<const float4 *>(base + 4 * q);
    lo = make_float2(v.x, v.y);
    hi = make_float2(v.z, v.w);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// One pass over the chains' sequence for the 16-state group g (states
// ng = 16·g .. ng + 15). With one group the per-token outputs are written
// directly; with several, every group writes its parts of dΔ, dx and the
// pre-gate output to its own slice of p.acc, and bwd_groups_finish_kernel
// sums them.
template <typename T, bool kGate, bool kSoftplus, bool kStruct, bool kConv, bool kZoh>
__device__ __forceinline__ void bwd_body(BwdSmem &S, const BwdParams &p, int g) {
    const int lane = threadIdx.x;
    const long long b = blockIdx.y;
    const long long d = (long long)blockIdx.x * kChains + lane;
    const bool active = d < p.dim;
    const int N = p.dstate;
    const int ng = 16 * g;                  // first state of the group
    const long long dd = active ? d : 0;

    // A as 2^(·) exponents (general A) and the structured-A decay base
    float2 Al[kPairs];
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        const float a0 = (active && ng + 2 * j < N) ? p.A[dd * N + ng + 2 * j] : 0.0f;
        const float a1 = (active && ng + 2 * j + 1 < N) ? p.A[dd * N + ng + 2 * j + 1] : 0.0f;
        Al[j] = make_float2(a0 * kLog2e, a1 * kLog2e);
    }
    const float A0l = Al[0].x;
    const float A0n = A0l * kLn2;  // A[0] itself (natural units)
    const float bias = (active && p.delta_bias) ? p.delta_bias[dd] : 0.0f;
    const float Dv = (active && p.Dskip) ? p.Dskip[dd] : 0.0f;
    const int K = p.ktiles;
    // conv taps of this channel (the conv output is the scan's x)
    float cw[kMaxConv] = {0.f, 0.f, 0.f, 0.f}, cbias = 0.0f;
    if (kConv && active) {
        load_conv_taps(p.conv_w, p.conv_width, dd, cw);
        cbias = p.conv_b ? p.conv_b[dd] : 0.0f;
    }
    float4 *ck = reinterpret_cast<float4 *>(p.ckpt) +
                 ((((long long)g * p.batch + b) * K) * p.dim + dd) * 4;  // this group's region
    const long long ck_stride = p.dim * 4;  // float4s between consecutive tiles

    // ---- 1. forward sweep: checkpoints ------------------------------------------
    {
        float2 h[kPairs];
#pragma unroll
        for (int j = 0; j < kPairs; ++j) {
            const float *h0 = p.h0 + (b * p.dim + dd) * N + ng;
            h[j] = make_float2((active && p.h0 && ng + 2 * j < N) ? h0[2 * j] : 0.f,
                               (active && p.h0 && ng + 2 * j + 1 < N) ? h0[2 * j + 1] : 0.f);
        }
        Raw<T> cur, nxt;
        float bv[4], cv[4];
        load_raw<T, kGate, false>(cur, p, b, 0, dd, active);
        load_bc<T>(bv, cv, p, b, 0, lane, false, ng);
        float xw[kMaxConv - 1] = {0.f, 0.f, 0.f};  // conv window, zero before token 0
        for (int k = 0; k < K; ++k) {
            const long long t0 = (long long)k * kSeg;
            if (active) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    ck[k * ck_stride + j] =
                        make_float4(h[2 * j].x, h[2 * j].y, h[2 * j + 1].x, h[2 * j + 1].y);
            }
            __syncwarp();
            store_bc(S, bv, cv, lane);
            if (k + 1 < K) {
                load_raw<T, kGate, false>(nxt, p, b, t0 + kSeg, dd, active);
                load_bc<T>(bv, cv, p, b, t0 + kSeg, lane, false, ng);
            }
            __syncwarp();
#pragma unroll
            for (int t = 0; t < kSeg; ++t) {
                const float v = to_f32(cur.dl[t]) + bias;
                const bool live = active && t0 + t < p.seqlen;
                const float dt = live ? (kSoftplus ? softplus_f32(v) : v) : 0.0f;
                float xv = to_f32(cur.x[t]);
                if (kConv) xv = conv_step(cw, cbias, xw, xv);
                const float2 u2 = dup2(dt * xv);
                float2 a[kPairs];
                decay16<kStruct>(dt, ex2_approx(dt * A0l), Al, a);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float2 b0, b1;
                    ld_quad(S.Bs[t], q, b0, b1);
                    if (kZoh) {  // B·(e^z − 1)/z per state
                        const float2 z0 = zoh_z<kStruct>(dt, 2 * q, A0n, Al);
                        const float2 z1 = zoh_z<kStruct>(dt, 2 * q + 1, A0n, Al);
                        b0 = mul2(b0, make_float2(zoh_factor(z0.x, a[2 * q].x),
                                                  zoh_factor(z0.y, a[2 * q].y)));
                        b1 = mul2(b1, make_float2(zoh_factor(z1.x, a[2 * q + 1].x),
                                                  zoh_factor(z1.y, a[2 * q + 1].y)));
                    }
                    h[2 * q] = fma2(a[2 * q], h[2 * q], mul2(u2, b0));
                    h[2 * q + 1] = fma2(a[2 * q + 1], h[2 * q + 1], mul2(u2, b1));
                }
            }
            cur = nxt;
        }
    }

    // ---- 2. reverse sweep ---------------------------------------------------------
    float2 lam[kPairs], dA[kPairs];
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        const float l0 = (active && p.dfinal && ng + 2 * j < N)
                             ? p.dfinal[(b * p.dim + dd) * N + ng + 2 * j] : 0.f;
        const float l1 =
            (active && p.dfinal && ng + 2 * j + 1 < N) ? p.dfinal[(b * p.dim + dd) * N + ng + 2 * j + 1] : 0.f;
        lam[j] = make_float2(l0, l1);
        dA[j] = make_float2(0.f, 0.f);
    }
    float accD = 0.f, accBias = 0.f;
    const int kk = lane & 7, cg = lane >> 3;  // reduction role: value group kk, channels 8cg..8cg+7
    float *part = p.part + ((long long)g * p.batch * p.ctiles + b * p.ctiles + blockIdx.x) *
                               p.seqlen * kVals;
    Raw<T> cur, nxt;
    float bv[4], cv[4];
    float4 hc[4], hn[4];
    {
        const long long t0 = (long long)(K - 1) * kSeg;
        load_raw<T, kGate, true, kConv>(cur, p, b, t0, dd, active);
        load_bc<T>(bv, cv, p, b, t0, lane, true, ng);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            hc[j] = active ? ck[(K - 1) * ck_stride + j] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int k = K - 1; k >= 0; --k) {
        const long long t0 = (long long)k * kSeg;
        __syncwarp();
        store_bc(S, bv, cv, lane);
        if (k > 0) {
            load_raw<T, kGate, true, kConv>(nxt, p, b, t0 - kSeg, dd, active);
            load_bc<T>(bv, cv, p, b, t0 - kSeg, lane, true, ng);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                hn[j] = active ? ck[(k - 1) * ck_stride + j] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncwarp();

        // recompute the tile's states and per-token scalars
        float xw[kMaxConv - 1];
#pragma unroll
        for (int k = 0; k < kMaxConv - 1; ++k) xw[k] = kConv ? to_f32(cur.xh[k]) : 0.0f;
        float2 h[kPairs];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            h[2 * j] = make_float2(hc[j].x, hc[j].y);
            h[2 * j + 1] = make_float2(hc[j].z, hc[j].w);
            S.hs[0][j][lane] = hc[j];
        }
#pragma unroll
        for (int t = 0; t < kSeg; ++t) {
            const bool live = active && t0 + t < p.seqlen;
            float xv = to_f32(cur.x[t]);
            if (kConv) xv = conv_step(cw, cbias, xw, xv);
            const float v = to_f32(cur.dl[t]) + bias;
            const float dt = live ? (kSoftplus ? softplus_f32(v) : v) : 0.0f;
            const float u = dt * xv;
            const float dyv = to_f32(cur.dy[t]);
            float ds = dyv, dysz = 0.f;
            if (kGate) {
                const float zv = to_f32(cur.z[t]);
                const float sgz = sigmoid_f32(zv);
                ds = dyv * zv * sgz;
                dysz = dyv * sgz * fmaf(zv, 1.0f - sgz, 1.0f);
            }
            const float sg = kSoftplus ? sigmoid_f32(v) : 1.0f;
            const float r = ex2_approx(dt * A0l);
            float2 a[kPairs];
            decay16<kStruct>(dt, r, Al, a);
            const float2 u2 = dup2(u);
            float2 sacc = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float2 b0, b1, c0, c1;
                ld_quad(S.Bs[t], q, b0, b1);
                ld_quad(S.Cs[t], q, c0, c1);
                if (kZoh) {
                    const float2 z0 = zoh_z<kStruct>(dt, 2 * q, A0n, Al);
                    const float2 z1 = zoh_z<kStruct>(dt, 2 * q + 1, A0n, Al);
                    b0 = mul2(b0, make_float2(zoh_factor(z0.x, a[2 * q].x),
                                              zoh_factor(z0.y, a[2 * q].y)));
                    b1 = mul2(b1, make_float2(zoh_factor(z1.x, a[2 * q + 1].x),
                                              zoh_factor(z1.y, a[2 * q + 1].y)));
                }
                h[2 * q] = fma2(a[2 * q], h[2 * q], mul2(u2, b0));
                h[2 * q + 1] = fma2(a[2 * q + 1], h[2 * q + 1], mul2(u2, b1));
                sacc = fma2(c0, h[2 * q], sacc);
                sacc = fma2(c1, h[2 * q + 1], sacc);
            }
            S.sc[t][lane] = make_float4(dt, u, ds, r);
            // s = Σ_n C·h + D·x: the D term once, with the first group
            S.so[t][lane] = make_float4(xv, dysz, sg,
                                        fmaf(g == 0 ? Dv : 0.0f, xv, sacc.x + sacc.y));
#pragma unroll
            for (int j = 0; j < 4; ++j)
                S.hs[t + 1][j][lane] = make_float4(h[2 * j].x, h[2 * j].y, h[2 * j + 1].x, h[2 * j + 1].y);
        }

        // walk the tile backwards
#pragma unroll 1
        for (int t = kSeg - 1; t >= 0; --t) {
            const long long tok = t0 + t;
            const float4 sc = S.sc[t][lane];
            const float4 so = S.so[t][lane];
            float2 a[kPairs];
            decay16<kStruct>(sc.x, sc.w, Al, a);
            const float2 ds2 = dup2(sc.z), u2 = dup2(sc.y), dt2 = dup2(sc.x);
            // du2: Σ λ·c'·B over states for dx (c' = 1, or the ZOH factor f);
            // dd2: Σ λ·∂(c'Δ)/∂Δ·B for dΔ (ZOH: a; Δ·B·x: the same sum as du2)
            float2 du2 = make_float2(0.f, 0.f), dd2 = du2, qp2 = du2;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float4 hq = S.hs[t + 1][j][lane];    // h_t
                const float4 hp = S.hs[t][j][lane];        // h_{t−1}
                const float2 hh[2] = {make_float2(hq.x, hq.y), make_float2(hq.z, hq.w)};
                const float2 hprev[2] = {make_float2(hp.x, hp.y), make_float2(hp.z, hp.w)};
                float dbv[4], dcv[4];
                float2 bq[2], cq[2];
                ld_quad(S.Bs[t], j, bq[0], bq[1]);
                ld_quad(S.Cs[t], j, cq[0], cq[1]);
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int jj = 2 * j + e;
                    const float2 bb = bq[e];
                    lam[jj] = fma2(ds2, cq[e], lam[jj]);                    // λ_t
                    const float2 hb = mul2(a[jj], hprev[e]);                // Abar_t·h_{t−1}
                    const float2 lh = mul2(lam[jj], hb);
                    float2 lf = lam[jj];                                    // λ·f (ZOH) or λ
                    if (kZoh) {
                        const float2 zz = zoh_z<kStruct>(sc.x, jj, A0n, Al);
                        const float2 f = make_float2(zoh_factor(zz.x, a[jj].x),
                                                     zoh_factor(zz.y, a[jj].y));
                        const float2 fp = make_float2(zoh_factor_deriv(zz.x, a[jj].x),
                                                      zoh_factor_deriv(zz.y, a[jj].y));
                        lf = mul2(lam[jj], f);
                        dd2 = fma2(mul2(lam[jj], a[jj]), bb, dd2);
                        // ∂c/∂A = Δ²·f'(z): dA += λ·f'·Δ·u·B
                        dA[jj] = fma2(mul2(lam[jj], fp), mul2(mul2(dt2, u2), bb), dA[jj]);
                    }
                    du2 = fma2(lf, bb, du2);
                    if (kStruct)
                        qp2 = fma2(lh, make_float2((float)(2 * jj + 1), (float)(2 * jj + 2)), qp2);
                    else
                        qp2 = fma2(lh, Al[jj], qp2);
                    dA[jj] = fma2(dt2, lh, dA[jj]);
                    const float2 db = mul2(lf, u2);
                    const float2 dc = mul2(ds2, hh[e]);
                    dbv[2 * e] = db.x;
                    dbv[2 * e + 1] = db.y;
                    dcv[2 * e] = dc.x;
                    dcv[2 * e + 1] = dc.y;
                    lam[jj] = mul2(lam[jj], a[jj]);                       // carried to token t − 1
                }
                S.red[j][lane ^ j] = make_float4(dbv[0], dbv[1], dbv[2], dbv[3]);
                S.red[4 + j][lane ^ (4 + j)] = make_float4(dcv[0], dcv[1], dcv[2], dcv[3]);
            }
            const float du = du2.x + du2.y;
            const float dd = kZoh ? dd2.x + dd2.y : du;
            const float qsum = qp2.x + qp2.y;
            // Σ_n λ·hb·A[n]: structured A[n] = (n+1)·A[0]; otherwise Al = A·log2 e
            const float qp = kStruct ? qsum * A0l * kLn2 : qsum * kLn2;
            if (active && tok < p.seqlen) {
                const long long i = (b * p.seqlen + tok) * p.dim + d;
                float ddt = fmaf(dd, so.x, qp);
                float dxv = fmaf(du, sc.x, g == 0 ? sc.z * Dv : 0.0f);
                float sv = so.w;
                if (p.groups > 1) {  // this group's parts, summed by the finish kernel
                    const long long n3 = p.batch * p.seqlen * p.dim;
                    float *a = p.acc + (long long)g * 3 * n3;
                    a[i] = ddt;
                    a[n3 + i] = dxv;
                    a[2 * n3 + i] = sv;
                    if (g == 0) accD = fmaf(sc.z, so.x, accD);
                } else {
                    const float dv = ddt * so.z;
                    if (kConv)
                        p.dxc[i] = dxv;  // the conv's input gradient comes from conv_bwd_kernel
                    else
                        static_cast<T *>(p.dx)[i] = from_f32<T>(dxv);
                    static_cast<T *>(p.ddelta)[i] = from_f32<T>(dv);
                    if (kGate) static_cast<T *>(p.dz)[i] = from_f32<T>(sv * so.y);
                    accD = fmaf(sc.z, so.x, accD);
                    accBias += dv;
                }
            }
            __syncwarp();
            // channel sums of this token's 32 values
            float2 alo = make_float2(0.f, 0.f), ahi = alo;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 w = S.red[kk][(8 * cg + i) ^ kk];
                alo = add2(alo, make_float2(w.x, w.y));
                ahi = add2(ahi, make_float2(w.z, w.w));
            }
            float4 acc = make_float4(alo.x, alo.y, ahi.x, ahi.y);
#pragma unroll
            for (int m = 8; m <= 16; m <<= 1) {
                acc.x += __shfl_xor_sync(0xffffffffu, acc.x, m);
                acc.y += __shfl_xor_sync(0xffffffffu, acc.y, m);
                acc.z += __shfl_xor_sync(0xffffffffu, acc.z, m);
                acc.w += __shfl_xor_sync(0xffffffffu, acc.w, m);
            }
            const float mine = cg == 0 ? acc.x : (cg == 1 ? acc.y : (cg == 2 ? acc.z : acc.w));
            if (tok < p.seqlen) part[tok * kVals + 4 * kk + cg] = mine;
            __syncwarp();
        }
        cur = nxt;
#pragma unroll
        for (int j = 0; j < 4; ++j) hc[j] = hn[j];
    }

    // the initial state's gradient: λ carried past the first token
    if (active && p.dh0) {
        float *dh0 = p.dh0 + (b * p.dim + d) * N + ng;
#pragma unroll
        for (int j = 0; j < kPairs; ++j) {
            if (ng + 2 * j < N) dh0[2 * j] = lam[j].x;
            if (ng + 2 * j + 1 < N) dh0[2 * j + 1] = lam[j].y;
        }
    }
    // per-(batch row, channel) partials
    if (active) {
        float4 *pa = reinterpret_cast<float4 *>(p.pA + ((long long)g * p.batch * p.dim +
                                                         b * p.dim + d) * kMaxN);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            pa[j] = make_float4(dA[2 * j].x, dA[2 * j].y, dA[2 * j + 1].x, dA[2 * j + 1].y);
        if (g == 0) p.pD[b * p.dim + d] = accD;
        if (p.groups == 1) p.pbias[b * p.dim + d] = accBias;  // else: the finish kernel
    }
}

// A[d, n] = (n+1)·A[d, 0] (ladder_state) for every state of every channel of
// the warp selects the power-ladder decay (the A = −(1..N) initialisation).
template <typename T, bool kGate, bool kSoftplus, bool kConv, bool kZoh>
__global__ void __launch_bounds__(kChains, 6) scan_bwd_kernel(const BwdParams p) {
    __shared__ BwdSmem S;
    const long long d = (long long)blockIdx.x * kChains + threadIdx.x;
    bool ok = p.groups == 1;  // the power ladder covers states 1..16 of one group
    if (ok && d < p.dim) {
        const float a0 = p.A[d * p.dstate];
        for (int n = 1; n < p.dstate; ++n)
            if (!ladder_state(p.A[d * p.dstate + n], a0, n)) ok = false;
    }
    if (__all_sync(0xffffffffu, ok))
        bwd_body<T, kGate, kSoftplus, true, kConv, kZoh>(S, p, 0);
    else
        bwd_body<T, kGate, kSoftplus, false, kConv, kZoh>(S, p, (int)blockIdx.z);
}

// Above 16 states: the per-token sums over the state groups, in group order
// (deterministic), and what follows from them — dx (or the conv output's
// gradient), ddelta = dΔ·σ(delta + bias), dz = dy·s·silu'(z) — plus the
// per-(batch row, channel) sum of ddelta. One thread per (batch row,
// channel) walks the tokens; consecutive threads take consecutive channels.
template <typename T, bool kGate, bool kConv>
__global__ void bwd_groups_finish_kernel(const BwdParams p) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= p.batch * p.dim) return;
    const long long b = e / p.dim, d = e - b * p.dim;
    const long long n3 = p.batch * p.seqlen * p.dim;
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.0f;
    float sb = 0.0f;
    for (long long t = 0; t < p.seqlen; ++t) {
        const long long i = (b * p.seqlen + t) * p.dim + d;
        float ddt = 0.f, dxv = 0.f, sv = 0.f;
        for (int g = 0; g < p.groups; ++g) {
            const float *a = p.acc + (long long)g * 3 * n3;
            ddt += a[i];
            dxv += a[n3 + i];
            sv += a[2 * n3 + i];
        }
        const float v = ldg_f32(static_cast<const T *>(p.delta) + i) + bias;
        const float dv = p.softplus ? ddt * sigmoid_f32(v) : ddt;
        if (kConv)
            p.dxc[i] = dxv;
        else
            static_cast<T *>(p.dx)[i] = from_f32<T>(dxv);
        static_cast<T *>(p.ddelta)[i] = from_f32<T>(dv);
        if (kGate) {
            const float zv = ldg_f32(static_cast<const T *>(p.z) + i);
            const float dyv = ldg_f32(static_cast<const T *>(p.dy) + i);
            const float sgz = sigmoid_f32(zv);
            static_cast<T *>(p.dz)[i] = from_f32<T>(sv * (dyv * sgz * fmaf(zv, 1.0f - sgz, 1.0f)));
        }
        sb += dv;
    }
    p.pbias[b * p.dim + d] = sb;
}

// dB[b, t, n] and dC[b, t, n]: sums of the channel-tile partials (one
// thread per (batch row, token, four consecutive stored values, state
// group); 16-byte loads). Stored value e of a row holds dB (c = 0) or dC
// (c = 1) of state n: e = 16·c + n, or with part_lane_order
// e = 4·(4c + 2·(n & 1) + n / 8) + (n / 2) % 4.
__global__ void bwd_reduce_bc_kernel(const BwdParams p) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    constexpr int kQuads = kVals / 4;
    const long long per = p.batch * p.seqlen * kQuads;
    if (e >= per * p.groups) return;
    const int g = (int)(e / per);
    const long long eg = e - g * per;
    const long long b = eg / (p.seqlen * kQuads);
    const long long rest = eg - b * p.seqlen * kQuads;  // tok * 8 + f
    const int f = (int)(rest % kQuads);
    const long long tok = rest / kQuads;
    const float4 *src = reinterpret_cast<const float4 *>(
                            p.part + ((long long)g * p.batch * p.ctiles + b * p.ctiles) * p.seqlen * kVals) +
                        rest;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < p.ctiles; ++c) {
        const float4 v = src[(long long)c * p.seqlen * kQuads];
        sum.x += v.x;
        sum.y += v.y;
        sum.z += v.z;
        sum.w += v.w;
    }
    const float s[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int isC, m;
        if (p.part_lane_order) {
            isC = f >> 2;
            m = 8 * (f & 1) + 2 * i + ((f >> 1) & 1);
        } else {
            isC = (4 * f + i) / kMaxN;
            m = (4 * f + i) % kMaxN;
        }
        const int n = 16 * g + m;
        if (n < p.dstate) (isC ? p.dC : p.dB)[(b * p.seqlen + tok) * p.dstate + n] = s[i];
    }
}

// dA[d, n], dD[d], ddelta_bias[d]: sums over batch rows.
__global__ void bwd_reduce_params_kernel(const BwdParams p) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int width = kMaxN * p.groups;
    if (e >= p.dim * width) return;
    const long long d = e / width;
    const int n = (int)(e % width);
    if (n < p.dstate) {
        const float *src = p.pA + (long long)(n / kMaxN) * p.batch * p.dim * kMaxN + n % kMaxN;
        float s = 0.f;
        for (long long b = 0; b < p.batch; ++b) s += src[(b * p.dim + d) * kMaxN];
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

// Gradient of the causal conv + SiLU in front of the scan, from the
// gradient of its output (dxc, written by scan_bwd_kernel): with
// pre[t] = cb + Σ_k cw[k]·x_in[t − 3 + k] (taps right-aligned in 4 slots) and
// dpre[t] = dxc[t]·silu'(pre[t]),
//   dx_in[s] = Σ_k cw[k]·dpre[s + 3 − k],  dw[k] += dpre[t]·x_in[t − 3 + k],
//   db += dpre[t].
// A thread walks one channel over kConvTile tokens (3 more at the end for
// the dx_in of its last tokens), sliding windows of x_in and dpre in
// registers; dw and db go to a per-(batch row, token tile) partial buffer.
constexpr int kConvTile = 512;
constexpr int kConvThreads = 128;

template <typename T>
__global__ void __launch_bounds__(kConvThreads) conv_bwd_kernel(const BwdParams p) {
    const long long d = (long long)blockIdx.x * kConvThreads + threadIdx.x;
    const int tile = blockIdx.y;
    const long long b = blockIdx.z;
    if (d >= p.dim) return;
    const long long ta = (long long)tile * kConvTile;
    const long long tb = min(ta + kConvTile, p.seqlen);
    float cw[kMaxConv];
    load_conv_taps(p.conv_w, p.conv_width, d, cw);
    const float cb = p.conv_b ? p.conv_b[d] : 0.0f;
    const T *xp = static_cast<const T *>(p.x);
    const long long row = b * p.seqlen;
    float xw[kMaxConv - 1];
#pragma unroll
    for (int k = 0; k < kMaxConv - 1; ++k) {
        const long long t = ta - (kMaxConv - 1) + k;
        xw[k] = t >= 0 ? ldg_f32(xp + (row + t) * p.dim + d) : 0.0f;
    }
    float dq[kMaxConv] = {0.f, 0.f, 0.f, 0.f};  // dpre of the last 4 tokens, oldest first
    float dw[kMaxConv] = {0.f, 0.f, 0.f, 0.f}, db = 0.0f;
    T *dxp = static_cast<T *>(p.dx);
    for (long long t = ta; t < tb + (kMaxConv - 1); ++t) {
        float g = 0.0f;
        if (t < p.seqlen) {
            const long long i = (row + t) * p.dim + d;
            const float xi = ldg_f32(xp + i);
            const float pre =
                fmaf(cw[0], xw[0], fmaf(cw[1], xw[1], fmaf(cw[2], xw[2], fmaf(cw[3], xi, cb))));
            const float sg = sigmoid_f32(pre);
            g = p.dxc[i] * sg * fmaf(pre, 1.0f - sg, 1.0f);
            if (t < tb) {
                dw[0] = fmaf(g, xw[0], dw[0]);
                dw[1] = fmaf(g, xw[1], dw[1]);
                dw[2] = fmaf(g, xw[2], dw[2]);
                dw[3] = fmaf(g, xi, dw[3]);
                db += g;
            }
            xw[0] = xw[1];
            xw[1] = xw[2];
            xw[2] = xi;
        }
        dq[0] = dq[1];
        dq[1] = dq[2];
        dq[2] = dq[3];
        dq[3] = g;
        const long long s = t - (kMaxConv - 1);
        if (s >= ta && s < tb)
            dxp[(row + s) * p.dim + d] = from_f32<T>(
                fmaf(cw[3], dq[0], fmaf(cw[2], dq[1], fmaf(cw[1], dq[2], cw[0] * dq[3]))));
    }
    float *pc = p.pconv + ((b * p.conv_tiles + tile) * p.dim + d) * (kMaxConv + 1);
#pragma unroll
    for (int k = 0; k < kMaxConv; ++k) pc[k] = dw[k];
    pc[kMaxConv] = db;
}

// dconv_w[d, j] and dconv_b[d]: sums of the partials over batch rows and tiles.
__global__ void conv_reduce_kernel(const BwdParams p) {
    const long long d = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (d >= p.dim) return;
    float acc[kMaxConv + 1] = {0.f, 0.f, 0.f, 0.f, 0.f};
    for (long long r = 0; r < p.batch * p.conv_tiles; ++r) {
        const float *pc = p.pconv + (r * p.dim + d) * (kMaxConv + 1);
#pragma unroll
        for (int k = 0; k <= kMaxConv; ++k) acc[k] += pc[k];
    }
    for (int j = 0; j < p.conv_width; ++j)
        p.dconv_w[d * p.conv_width + j] = acc[j + kMaxConv - p.conv_width];
    if (p.dconv_b) p.dconv_b[d] = acc[kMaxConv];
}

template <typename T, bool kGate, bool kConv, bool kZoh>
cudaError_t launch_zoh(const BwdParams &p, cudaStream_t stream) {
    const dim3 grid((unsigned)p.ctiles, (unsigned)p.batch, (unsigned)p.groups);
    if (p.softplus)
        scan_bwd_kernel<T, kGate, true, kConv, kZoh><<<grid, kChains, 0, stream>>>(p);
    else
        scan_bwd_kernel<T, kGate, false, kConv, kZoh><<<grid, kChains, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T, bool kGate, bool kConv>
cudaError_t launch_conv(const BwdParams &p, cudaStream_t stream) {
    cudaError_t e = p.zoh ? launch_zoh<T, kGate, kConv, true>(p, stream)
                          : launch_zoh<T, kGate, kConv, false>(p, stream);
    if (e != cudaSuccess || p.groups == 1) return e;
    const long long n = p.batch * p.dim;
    bwd_groups_finish_kernel<T, kGate, kConv><<<(unsigned)((n + 127) / 128), 128, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T, bool kGate>
cudaError_t launch_gate(const BwdParams &p, cudaStream_t stream) {
    cudaError_t e = p.conv_width > 0 ? launch_conv<T, kGate, true>(p, stream)
                                     : launch_conv<T, kGate, false>(p, stream);
    if (e != cudaSuccess || p.conv_width == 0) return e;
    const dim3 grid((unsigned)((p.dim + kConvThreads - 1) / kConvThreads),
                    (unsigned)p.conv_tiles, (unsigned)p.batch);
    conv_bwd_kernel<T><<<grid, kConvThreads, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    conv_reduce_kernel<<<(unsigned)((p.dim + 255) / 256), 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

int bwd_tile_tokens() { return kSeg; }
int bwd_tile_channels() { return kChains; }
int bwd_conv_tile_tokens() { return kConvTile; }

cudaError_t launch_scan_bwd(const BwdParams &params, bool bf16, cudaStream_t stream) {
    cudaError_t e;
    BwdParams p = params;
    p.part_lane_order = bwd_pairs_supported(p, bf16) ? 1 : 0;
    if (p.part_lane_order) {
        // the two-lane kernel's channel tiles (its partial rows)
        p.ctiles = (int)((p.dim + bwd_pairs_tile_channels() - 1) / bwd_pairs_tile_channels());
        e = launch_scan_bwd_pairs(p, bf16, stream);
    }
    else if (bf16)
        e = p.z ? launch_gate<__nv_bfloat16, true>(p, stream)
                : launch_gate<__nv_bfloat16, false>(p, stream);
    else
        e = p.z ? launch_gate<float, true>(p, stream) : launch_gate<float, false>(p, stream);
    if (e != cudaSuccess) return e;
    const long long nbc = p.batch * p.seqlen * (kVals / 4) * p.groups;
    bwd_reduce_bc_kernel<<<(unsigned)((nbc + 255) / 256), 256, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long npar = p.dim * kMaxN * p.groups;
    bwd_reduce_params_kernel<<<(unsigned)((npar + 255) / 256), 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace selscan
