// scan_bwd2.cu -- gradient of the selective scan with two lanes per chain
// (d_state ≤ 16 in one group, no conv front end, Δ·B·x input term).
//
// Pages: "Mamba: co potrafią modele przestrzeni stanów", "Cena selekcji"
// (the backward pass recomputes the intermediate states instead of storing
// them); the recurrence it differentiates is "Mamba & State Space Models —
// Guide Complet" §4 "Implémentation du SSM sélectif (S6)" and "Mamba и State
// Space Models: альтернатива Transformer", "SSM as RNN".
//
// The sweeps and formulas are those of scan_bwd.cu (see its header): a
// forward sweep storing the state entering every 8-token tile, then a reverse
// sweep over the tiles that recomputes each tile's states from its checkpoint
// and walks the tile backwards carrying λ = ∂loss/∂h. The thread layout
// differs:
//  * lanes l and l + 16 of a warp share one channel, the lower lane keeping
//    the even states and the upper lane the odd ones (8 each), so a layer of
//    20,480 chains puts two warps where scan_bwd.cu has one;
//  * every per-token scalar (softplus and its derivative, silu(z) and its
//    derivative, the decay base, Δ·x) is formed once per token by one of the
//    two lanes (tokens 0–3 of a tile by the lower lane, 4–7 by the upper),
//    which also writes that token's dx, ddelta and dz at the end of the tile;
//  * the channel sums of dB and dC are formed per half tile, not per token:
//    the walk stores λ_t, the recompute has already stored h_t, and 32 lanes
//    each form 4 of the 4 tokens × 32 sums as Σ_c λ_t[c]·u_t[c] and
//    Σ_c ds_t[c]·h_t[c] (the products dB = λ·u and dC = ds·h are never formed
//    per chain); per tile the CTA's two warps add their rows and write one
//    128-byte row per token to the partial buffer of scan_bwd.cu, which its
//    reduction kernel sums over the channel tiles.
// With λa = λ_t·Abar_t (the λ carried to token t − 1), the per-state work of
// the walk is six f32x2 operations per state pair: λ_t = ds·C + λa_{t+1},
// du += λ_t·B, λa = λ_t·Abar_t, lh = λa·h_{t−1}, q += lh·A, dA += Δ·lh.
//
// A CTA is two warps = 32 consecutive channels of one batch row, the channel
// tile of scan_bwd.cu: the checkpoint, partial and per-channel buffers keep
// their sizes.
#include "bwd_params.cuh"

namespace selscan {
namespace {

constexpr int kSeg = 8;     // tokens per tile (checkpoint interval)
constexpr int kOwn = 4;     // tokens per tile whose scalars one lane forms
constexpr int kWarps = 2;   // warps per CTA
constexpr int kCh = 16;     // channels per warp
constexpr int kVals = 2 * kMaxN;
constexpr int kPairs = 4;   // f32x2 registers holding a lane's 8 states

__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 dup2(float v) { return make_float2(v, v); }

// A warp's shared memory. hs and lam rows hold one float4 per (lane, half):
// half 0 = state pairs 0, 1 of the lane, half 1 = pairs 2, 3; the slot of lane
// l is l ^ (4·half + 2·(l ≥ 16) + is_h), so that the reducer's column reads
// (8 lanes: both halves, both parities, λ and h, one channel) fall in 8
// distinct bank quads, while a lane reads back only the slots it wrote.
struct WarpSmem {
    float B[kSeg][kMaxN];            // float32; [0..7] the even states, [8..15] the odd ones
    float C[kSeg][kMaxN];
    float4 sc[kSeg][kCh + 1];        // Δ, u = Δ·x, ds = dy·silu(z), r = 2^(Δ·A[d,0]·log2 e)
    float4 hs[kSeg + 1][2][32];      // hs[0]: state entering the tile; hs[t + 1]: after token t
    float4 lam[kOwn][2][32];         // λ of the half tile being reduced
    float sv[kSeg][kCh];             // per token: s = Σ C·h (the D·x term is added later)
    float du[kSeg][kCh];             //   Σ_n λ·B
    float qp[kSeg][kCh];             //   Σ_n λ·Abar·h_{t−1}·A[n]
    float4 row[2][kSeg][kVals / 4];  // per-warp channel sums of the tile, double buffered
};

struct __align__(128) Smem {
    WarpSmem w[kWarps];
};

__device__ __forceinline__ int slot(int lane, int half, int is_h) {
    return lane ^ (4 * half + 2 * (lane >> 4) + is_h);
}

// The lane's 8 decay factors of one token: structured A (powers r^(n+1) of
// the lane's states n = 2i + odd) or one exp per state.
template <bool kStruct>
__device__ __forceinline__ void decay8(float dt, float r, bool odd, const float2 (&Al)[kPairs],
                                       float2 (&a)[kPairs]) {
    if (kStruct) {
        const float s = r * r;
        const float b = odd ? s : r;
        a[0] = make_float2(b, b * s);
        const float s2 = s * s;
        a[1] = mul2(a[0], dup2(s2));
        const float s4 = s2 * s2;
        a[2] = mul2(a[0], dup2(s4));
        a[3] = mul2(a[1], dup2(s4));
    } else {
#pragma unroll
        for (int q = 0; q < kPairs; ++q)
            a[q] = make_float2(ex2_approx(dt * Al[q].x), ex2_approx(dt * Al[q].y));
    }
}

// B and C of one tile: lane l fetches token l / 4, float4 slot l % 4 of the
// shared rows (slots 0, 1: the even states; 2, 3: the odd ones), a tile ahead
// into registers; C only in the reverse sweep.
template <typename T>
__device__ __forceinline__ void fetch_bc(float (&vb)[4], float (&vc)[4], const BwdParams &p,
                                         long long b, long long t0, int lane, bool withC) {
    const int s = lane & 3;
    const int odd = s >> 1, i0 = (s & 1) * 4;
    const long long tok = t0 + (lane >> 2);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int n = 2 * (i0 + e) + odd;
        const bool ok = tok < p.seqlen && n < p.dstate;
        const long long idx = (b * p.seqlen + tok) * p.dstate + n;
        vb[e] = ok ? ldg_f32(static_cast<const T *>(p.B) + idx) : 0.0f;
        vc[e] = (ok && withC) ? ldg_f32(static_cast<const T *>(p.C) + idx) : 0.0f;
    }
}

__device__ __forceinline__ void store_bc(WarpSmem &W, const float (&vb)[4], const float (&vc)[4],
                                         int lane, bool withC) {
    const int t = lane >> 2, s = lane & 3;
    *reinterpret_cast<float4 *>(&W.B[t][4 * s]) = make_float4(vb[0], vb[1], vb[2], vb[3]);
    if (withC)
        *reinterpret_cast<float4 *>(&W.C[t][4 * s]) = make_float4(vc[0], vc[1], vc[2], vc[3]);
}

// Raw inputs of the lane's 4 owned tokens of a tile (x, delta; z, dy in the
// reverse sweep), a tile ahead.
template <typename T> struct Raw {
    T x[kOwn], dl[kOwn], z[kOwn], dy[kOwn];
};

template <typename T, bool kGate, bool kBwd>
__device__ __forceinline__ void load_raw(Raw<T> &r, const BwdParams &p, long long b,
                                         long long tok0, long long d, bool active) {
    const T zero = from_f32<T>(0.0f);
    const long long i0 = (b * p.seqlen + tok0) * p.dim + d;
#pragma unroll
    for (int j = 0; j < kOwn; ++j) {
        const bool ok = active && tok0 + j < p.seqlen;
        const long long i = i0 + j * p.dim;
        r.x[j] = ok ? __ldg(static_cast<const T *>(p.x) + i) : zero;
        r.dl[j] = ok ? __ldg(static_cast<const T *>(p.delta) + i) : zero;
        if (kBwd) {
            r.dy[j] = ok ? __ldg(static_cast<const T *>(p.dy) + i) : zero;
            if (kGate) r.z[j] = ok ? __ldg(static_cast<const T *>(p.z) + i) : zero;
        }
    }
}

// One half tile's channel sums: lane (j, v) forms, for token base + j, the 4
// values of group v (v < 4: dB of states 8·(v & 1) + 2e + (v >> 1); v ≥ 4: dC
// of the same states for v − 4) summed over the warp's 16 channels.
__device__ __forceinline__ void reduce_half(WarpSmem &W, int buf, int base, int lane) {
    const int j = lane >> 3, v = lane & 7;
    const int is_h = v >> 2, par = (v >> 1) & 1, half = v & 1;
    const int t = base + j;
    const float4 *src = is_h ? &W.hs[t + 1][half][0] : &W.lam[j][half][0];
    const float *w = reinterpret_cast<const float *>(&W.sc[t][0]) + 1 + is_h;  // u or ds
    const int mask = 4 * half + 2 * par + is_h;
    float2 a01 = make_float2(0.f, 0.f), a23 = a01;
#pragma unroll
    for (int c = 0; c < kCh; ++c) {
        const float4 val = src[(16 * par + c) ^ mask];
        const float2 wc = dup2(w[4 * c]);
        a01 = fma2(make_float2(val.x, val.y), wc, a01);
        a23 = fma2(make_float2(val.z, val.w), wc, a23);
    }
    W.row[buf][t][v] = make_float4(a01.x, a01.y, a23.x, a23.y);
}

template <typename T, bool kGate, bool kSoftplus, bool kStruct>
__device__ __forceinline__ void bwd_pairs_body(Smem &S, const BwdParams &p) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool odd = lane >= 16;
    const int cl = lane & 15;
    const int own0 = odd ? kOwn : 0;  // first owned token of a tile
    WarpSmem &W = S.w[warp];
    const long long b = blockIdx.y;
    const long long d = (long long)blockIdx.x * (kWarps * kCh) + warp * kCh + cl;
    const bool active = d < p.dim;
    const int N = p.dstate;
    const long long dd = active ? d : 0;

    // A of this lane's states n = 4q + odd, 4q + 2 + odd as 2^(·) exponents,
    // and the coefficient of Σ_n A[n]·lh[n]: (n + 1) (structured, times A[0]
    // at the end) or A[n]·log2 e (times ln 2 at the end)
    float2 Al[kPairs], coef[kPairs];
#pragma unroll
    for (int q = 0; q < kPairs; ++q) {
        const int n0 = 4 * q + (odd ? 1 : 0), n1 = n0 + 2;
        Al[q] = make_float2((active && n0 < N) ? p.A[dd * N + n0] * kLog2e : 0.0f,
                            (active && n1 < N) ? p.A[dd * N + n1] * kLog2e : 0.0f);
        coef[q] = kStruct ? make_float2((float)(n0 + 1), (float)(n1 + 1)) : Al[q];
    }
    const float A0l = (active ? p.A[dd * N] : 0.0f) * kLog2e;
    const float bias = (active && p.delta_bias) ? p.delta_bias[dd] : 0.0f;
    const float Dv = (active && p.Dskip) ? p.Dskip[dd] : 0.0f;
    const int K = p.ktiles;
    // checkpoint of tile k: 4 float4 per (batch row, tile, channel), the lower
    // lane's 2 then the upper lane's
    float4 *ck = reinterpret_cast<float4 *>(p.ckpt) + ((b * K) * p.dim + dd) * 4 + (odd ? 2 : 0);
    const long long ck_stride = p.dim * 4;
    const int hs0 = slot(lane, 0, 1), hs1 = slot(lane, 1, 1);
    const int lm0 = slot(lane, 0, 0), lm1 = slot(lane, 1, 0);

    // ---- 1. forward sweep: checkpoints ------------------------------------------
    {
        float2 h[kPairs];
#pragma unroll
        for (int q = 0; q < kPairs; ++q) {
            const int n0 = 4 * q + (odd ? 1 : 0), n1 = n0 + 2;
            const float *h0 = p.h0 + (b * p.dim + dd) * N;
            h[q] = make_float2((active && p.h0 && n0 < N) ? h0[n0] : 0.f,
                               (active && p.h0 && n1 < N) ? h0[n1] : 0.f);
        }
        Raw<T> cur, nxt;
        float vb[4], vc[4];
        load_raw<T, kGate, false>(cur, p, b, own0, dd, active);
        fetch_bc<T>(vb, vc, p, b, 0, lane, false);
        for (int k = 0; k < K; ++k) {
            const long long t0 = (long long)k * kSeg;
            if (active) {
                ck[k * ck_stride] = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
                ck[k * ck_stride + 1] = make_float4(h[2].x, h[2].y, h[3].x, h[3].y);
            }
            store_bc(W, vb, vc, lane, false);
            if (k + 1 < K) {
                load_raw<T, kGate, false>(nxt, p, b, t0 + kSeg + own0, dd, active);
                fetch_bc<T>(vb, vc, p, b, t0 + kSeg, lane, false);
            }
#pragma unroll
            for (int j = 0; j < kOwn; ++j) {
                const float v = to_f32(cur.dl[j]) + bias;
                const bool live = active && t0 + own0 + j < p.seqlen;
                const float dt = live ? (kSoftplus ? softplus_f32(v) : v) : 0.0f;
                W.sc[own0 + j][cl] = make_float4(dt, dt * to_f32(cur.x[j]), 0.0f,
                                                 ex2_approx(dt * A0l));
            }
            __syncwarp();
#pragma unroll 2
            for (int t = 0; t < kSeg; ++t) {
                const float4 sc = W.sc[t][cl];
                float2 a[kPairs];
                decay8<kStruct>(sc.x, sc.w, odd, Al, a);
                const float2 u2 = dup2(sc.y);
                const float4 b0 = *reinterpret_cast<const float4 *>(&W.B[t][odd ? 8 : 0]);
                const float4 b1 = *reinterpret_cast<const float4 *>(&W.B[t][odd ? 12 : 4]);
                h[0] = fma2(a[0], h[0], mul2(u2, make_float2(b0.x, b0.y)));
                h[1] = fma2(a[1], h[1], mul2(u2, make_float2(b0.z, b0.w)));
                h[2] = fma2(a[2], h[2], mul2(u2, make_float2(b1.x, b1.y)));
                h[3] = fma2(a[3], h[3], mul2(u2, make_float2(b1.z, b1.w)));
            }
            __syncwarp();
            cur = nxt;
        }
    }

    // ---- 2. reverse sweep ---------------------------------------------------------
    float2 lam[kPairs], dA[kPairs];
#pragma unroll
    for (int q = 0; q < kPairs; ++q) {
        const int n0 = 4 * q + (odd ? 1 : 0), n1 = n0 + 2;
        const float *df = p.dfinal + (b * p.dim + dd) * N;
        lam[q] = make_float2((active && p.dfinal && n0 < N) ? df[n0] : 0.f,
                             (active && p.dfinal && n1 < N) ? df[n1] : 0.f);
        dA[q] = make_float2(0.f, 0.f);
    }
    float accD = 0.f, accBias = 0.f;
    float *part = p.part + (b * p.ctiles + blockIdx.x) * p.seqlen * kVals;
    Raw<T> cur, nxt;
    float vb[4], vc[4];
    float4 hc0, hc1, hn0, hn1;
    {
        const long long t0 = (long long)(K - 1) * kSeg;
        load_raw<T, kGate, true>(cur, p, b, t0 + own0, dd, active);
        fetch_bc<T>(vb, vc, p, b, t0, lane, true);
        hc0 = active ? ck[(K - 1) * ck_stride] : make_float4(0.f, 0.f, 0.f, 0.f);
        hc1 = active ? ck[(K - 1) * ck_stride + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int k = K - 1; k >= 0; --k) {
        const long long t0 = (long long)k * kSeg;
        const int buf = k & 1;
        store_bc(W, vb, vc, lane, true);
        if (k > 0) {
            load_raw<T, kGate, true>(nxt, p, b, t0 - kSeg + own0, dd, active);
            fetch_bc<T>(vb, vc, p, b, t0 - kSeg, lane, true);
            hn0 = active ? ck[(k - 1) * ck_stride] : make_float4(0.f, 0.f, 0.f, 0.f);
            hn1 = active ? ck[(k - 1) * ck_stride + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // owned tokens' scalars; x, dy·silu'(z) and σ stay in registers for
        // the tile's epilogue
        float xo[kOwn], dyso[kOwn], sgo[kOwn];
#pragma unroll
        for (int j = 0; j < kOwn; ++j) {
            const bool live = active && t0 + own0 + j < p.seqlen;
            const float xv = to_f32(cur.x[j]);
            const float v = to_f32(cur.dl[j]) + bias;
            const float dt = live ? (kSoftplus ? softplus_f32(v) : v) : 0.0f;
            const float dyv = to_f32(cur.dy[j]);
            float ds = dyv, dysz = 0.f;
            if (kGate) {
                const float zv = to_f32(cur.z[j]);
                const float sgz = sigmoid_f32(zv);
                ds = dyv * zv * sgz;
                dysz = dyv * sgz * fmaf(zv, 1.0f - sgz, 1.0f);
            }
            xo[j] = xv;
            dyso[j] = dysz;
            sgo[j] = kSoftplus ? sigmoid_f32(v) : 1.0f;
            W.sc[own0 + j][cl] = make_float4(dt, dt * xv, ds, ex2_approx(dt * A0l));
        }
        W.hs[0][0][hs0] = hc0;
        W.hs[0][1][hs1] = hc1;
        __syncwarp();

        // recompute the tile's states (this lane's 8) and Σ C·h per token
        {
            float2 h[kPairs] = {make_float2(hc0.x, hc0.y), make_float2(hc0.z, hc0.w),
                                make_float2(hc1.x, hc1.y), make_float2(hc1.z, hc1.w)};
#pragma unroll 2
            for (int t = 0; t < kSeg; ++t) {
                const float4 sc = W.sc[t][cl];
                float2 a[kPairs];
                decay8<kStruct>(sc.x, sc.w, odd, Al, a);
                const float2 u2 = dup2(sc.y);
                const float4 b0 = *reinterpret_cast<const float4 *>(&W.B[t][odd ? 8 : 0]);
                const float4 b1 = *reinterpret_cast<const float4 *>(&W.B[t][odd ? 12 : 4]);
                h[0] = fma2(a[0], h[0], mul2(u2, make_float2(b0.x, b0.y)));
                h[1] = fma2(a[1], h[1], mul2(u2, make_float2(b0.z, b0.w)));
                h[2] = fma2(a[2], h[2], mul2(u2, make_float2(b1.x, b1.y)));
                h[3] = fma2(a[3], h[3], mul2(u2, make_float2(b1.z, b1.w)));
                W.hs[t + 1][0][hs0] = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
                W.hs[t + 1][1][hs1] = make_float4(h[2].x, h[2].y, h[3].x, h[3].y);
                if (kGate) {  // dz needs the pre-gate output s = Σ C·h + D·x
                    const float4 c0 = *reinterpret_cast<const float4 *>(&W.C[t][odd ? 8 : 0]);
                    const float4 c1 = *reinterpret_cast<const float4 *>(&W.C[t][odd ? 12 : 4]);
                    float2 sacc = mul2(make_float2(c0.x, c0.y), h[0]);
                    sacc = fma2(make_float2(c0.z, c0.w), h[1], sacc);
                    sacc = fma2(make_float2(c1.x, c1.y), h[2], sacc);
                    sacc = fma2(make_float2(c1.z, c1.w), h[3], sacc);
                    float tot = sacc.x + sacc.y;
                    tot += __shfl_xor_sync(0xffffffffu, tot, 16);
                    W.sv[t][cl] = tot;  // both lanes store the same sum
                }
            }
        }

        // walk the tile backwards; the dB, dC sums per half tile
#pragma unroll 2
        for (int t = kSeg - 1; t >= 0; --t) {
            const float4 sc = W.sc[t][cl];
            float2 a[kPairs];
            decay8<kStruct>(sc.x, sc.w, odd, Al, a);
            const float2 ds2 = dup2(sc.z), dt2 = dup2(sc.x);
            const float4 hp0 = W.hs[t][0][hs0], hp1 = W.hs[t][1][hs1];
            const float2 hprev[kPairs] = {make_float2(hp0.x, hp0.y), make_float2(hp0.z, hp0.w),
                                          make_float2(hp1.x, hp1.y), make_float2(hp1.z, hp1.w)};
            const float4 b0 = *reinterpret_cast<const float4 *>(&W.B[t][odd ? 8 : 0]);
            const float4 b1 = *reinterpret_cast<const float4 *>(&W.B[t][odd ? 12 : 4]);
            const float4 c0 = *reinterpret_cast<const float4 *>(&W.C[t][odd ? 8 : 0]);
            const float4 c1 = *reinterpret_cast<const float4 *>(&W.C[t][odd ? 12 : 4]);
            const float2 bq[kPairs] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w),
                                       make_float2(b1.x, b1.y), make_float2(b1.z, b1.w)};
            const float2 cq[kPairs] = {make_float2(c0.x, c0.y), make_float2(c0.z, c0.w),
                                       make_float2(c1.x, c1.y), make_float2(c1.z, c1.w)};
            float2 du2 = make_float2(0.f, 0.f), qp2 = du2;
            float2 lt[kPairs];
#pragma unroll
            for (int q = 0; q < kPairs; ++q) {
                lam[q] = fma2(ds2, cq[q], lam[q]);        // λ_t
                lt[q] = lam[q];
                du2 = fma2(lam[q], bq[q], du2);
                lam[q] = mul2(lam[q], a[q]);              // λ_t·Abar_t, carried to t − 1
                const float2 lh = mul2(lam[q], hprev[q]);
                qp2 = fma2(lh, coef[q], qp2);
                dA[q] = fma2(dt2, lh, dA[q]);
            }
            W.lam[t & 3][0][lm0] = make_float4(lt[0].x, lt[0].y, lt[1].x, lt[1].y);
            W.lam[t & 3][1][lm1] = make_float4(lt[2].x, lt[2].y, lt[3].x, lt[3].y);
            float du = du2.x + du2.y, qs = qp2.x + qp2.y;
            du += __shfl_xor_sync(0xffffffffu, du, 16);
            qs += __shfl_xor_sync(0xffffffffu, qs, 16);
            W.du[t][cl] = du;  // both lanes store the same sums
            W.qp[t][cl] = kStruct ? qs * A0l * kLn2 : qs * kLn2;  // Σ_n λ·Abar·h·A[n]
            if ((t & 3) == 0) {  // a half tile is walked: its channel sums
                __syncwarp();
                reduce_half(W, buf, t, lane);
                __syncwarp();
            }
        }

        // the owned tokens' dx, ddelta, dz (the walk ended with a __syncwarp)
        {
            const long long tok0 = t0 + own0;
            const long long i0 = (b * p.seqlen + tok0) * p.dim + d;
#pragma unroll
            for (int j = 0; j < kOwn; ++j) {
                if (active && tok0 + j < p.seqlen) {
                    const int t = own0 + j;
                    const float4 sc = W.sc[t][cl];
                    const float du = W.du[t][cl];
                    const long long i = i0 + j * p.dim;
                    const float dv = fmaf(du, xo[j], W.qp[t][cl]) * sgo[j];
                    static_cast<T *>(p.dx)[i] = from_f32<T>(fmaf(du, sc.x, sc.z * Dv));
                    static_cast<T *>(p.ddelta)[i] = from_f32<T>(dv);
                    if (kGate)
                        static_cast<T *>(p.dz)[i] =
                            from_f32<T>(fmaf(Dv, xo[j], W.sv[t][cl]) * dyso[j]);
                    accD = fmaf(sc.z, xo[j], accD);
                    accBias += dv;
                }
            }
        }
        // the two warps' sums: one 128-byte row per token of the channel tile
        __syncthreads();
        {
            const int t = threadIdx.x >> 3, g = threadIdx.x & 7;
            const long long tok = t0 + t;
            if (tok < p.seqlen) {
                const float *r0 = reinterpret_cast<const float *>(&S.w[0].row[buf][t][0]);
                const float *r1 = reinterpret_cast<const float *>(&S.w[1].row[buf][t][0]);
                float o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int vv = 4 * g + i;  // natural index: 16·is_C + n
                    const int n = vv & 15;
                    const int e = 4 * (4 * (vv >> 4) + 2 * (n & 1) + (n >> 3)) + ((n >> 1) & 3);
                    o[i] = r0[e] + r1[e];
                }
                *reinterpret_cast<float4 *>(part + tok * kVals + 4 * g) =
                    make_float4(o[0], o[1], o[2], o[3]);
            }
        }
        cur = nxt;
        hc0 = hn0;
        hc1 = hn1;
    }

    // the initial state's gradient: λ carried past the first token
    if (active && p.dh0) {
        float *dh0 = p.dh0 + (b * p.dim + d) * N;
#pragma unroll
        for (int q = 0; q < kPairs; ++q) {
            const int n0 = 4 * q + (odd ? 1 : 0), n1 = n0 + 2;
            if (n0 < N) dh0[n0] = lam[q].x;
            if (n1 < N) dh0[n1] = lam[q].y;
        }
    }
    // per-(batch row, channel) partials: dA by state; dD and ddelta_bias
    // summed over the two lanes' tokens
    accD += __shfl_xor_sync(0xffffffffu, accD, 16);
    accBias += __shfl_xor_sync(0xffffffffu, accBias, 16);
    if (active) {
        float *pa = p.pA + (b * p.dim + d) * kMaxN;
#pragma unroll
        for (int q = 0; q < kPairs; ++q) {
            const int n0 = 4 * q + (odd ? 1 : 0);
            pa[n0] = dA[q].x;
            pa[n0 + 2] = dA[q].y;
        }
        if (!odd) {
            p.pD[b * p.dim + d] = accD;
            p.pbias[b * p.dim + d] = accBias;
        }
    }
}

template <typename T, bool kGate, bool kSoftplus>
__global__ void __launch_bounds__(kWarps * 32, 5) scan_bwd_pairs_kernel(const BwdParams p) {
    __shared__ Smem S;
    // A[d, n] == (n+1)·A[d, 0] for every state of every channel of the CTA
    // selects the power-ladder decay (two threads per channel check it)
    const long long d = (long long)blockIdx.x * (kWarps * kCh) + threadIdx.x / 2;
    bool ok = true;
    if (d < p.dim) {
        const float a0 = p.A[d * p.dstate];
        for (int n = 1 + (threadIdx.x & 1); n < p.dstate; n += 2)
            if (p.A[d * p.dstate + n] != (float)(n + 1) * a0) ok = false;
    }
    if (__syncthreads_and(ok))
        bwd_pairs_body<T, kGate, kSoftplus, true>(S, p);
    else
        bwd_pairs_body<T, kGate, kSoftplus, false>(S, p);
}

template <typename T, bool kGate, bool kSoftplus>
cudaError_t launch_one(const BwdParams &p, cudaStream_t stream) {
    // five CTAs per SM need the largest shared-memory carveout
    const cudaError_t e = cudaFuncSetAttribute(scan_bwd_pairs_kernel<T, kGate, kSoftplus>,
                                               cudaFuncAttributePreferredSharedMemoryCarveout,
                                               cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)p.ctiles, (unsigned)p.batch, 1);
    scan_bwd_pairs_kernel<T, kGate, kSoftplus><<<grid, kWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T, bool kGate>
cudaError_t launch_gate(const BwdParams &p, cudaStream_t stream) {
    return p.softplus ? launch_one<T, kGate, true>(p, stream) : launch_one<T, kGate, false>(p, stream);
}

}  // namespace

bool bwd_pairs_supported(const BwdParams &p) {
    return p.groups == 1 && p.dstate <= kMaxN && p.conv_width == 0 && !p.zoh;
}

cudaError_t launch_scan_bwd_pairs(const BwdParams &p, bool bf16, cudaStream_t stream) {
    if (bf16)
        return p.z ? launch_gate<__nv_bfloat16, true>(p, stream)
                   : launch_gate<__nv_bfloat16, false>(p, stream);
    return p.z ? launch_gate<float, true>(p, stream) : launch_gate<float, false>(p, stream);
}

}  // namespace selscan
