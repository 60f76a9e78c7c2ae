// scan_wide.cu -- the selective scan for d_state above 16 (up to 256).
//
// Pages: the same recurrence as scan.cu ("Mamba & State Space Models — Guide
// Complet" §4, "Mamba и State Space Models: альтернатива Transformer", "SSM
// as RNN"), at the larger state sizes the Guide's §5 ("Mamba-2") uses, where
// A is a per-head scalar (A[d, n] constant across n) and d_state is 64 to 256.
//
// Work decomposition. A chain's states are split over kLanes = d_state / 16
// (rounded up to a power of two) adjacent lanes of a warp, 16 states per lane
// in registers. Every lane computes the chain's per-token scalars itself (the
// loads of x, delta, z are broadcasts within the lane group), updates its 16
// states and forms its part of Σ_n C[n]·h[n]; log2(kLanes) xor-shuffles finish
// the sum and the group's first lane writes y. A CTA of 128 threads covers
// 128 / kLanes consecutive channels of one batch row; B and C of a 16-token
// tile are staged in shared memory as float32. One pass over the whole
// sequence per CTA (no chunking). The exponent strategy follows scan.cu: with
// A[d, n] = (n+1)·A[d, 0] (ladder_state) on every channel of the CTA, Abar[n] = r^(n+1) is
// a lane's base power r^(16·slice) times a ladder; otherwise one ex2 per
// element. Optional: initial state, causal conv in front, ZOH input term.
#include "selscan_device.cuh"

namespace selscan {
namespace {

constexpr int kThreads = 128;
constexpr int kTileT = 16;      // tokens per B/C tile
constexpr int kMaxWide = 256;   // largest d_state of this kernel
constexpr int kSlice = 16;      // states per lane

template <typename T, bool kGate, int kLanes, bool kZoh>
__global__ void __launch_bounds__(kThreads)
scan_wide_kernel(const ScanParams p) {
    constexpr int kWidth = kLanes * kSlice;  // padded d_state
    constexpr int kChainsPerCta = kThreads / kLanes;
    // B and C rows as [slice][16 + 4 pad]: a lane reads its 16 states as four
    // 16-byte loads, and the pad puts the 8 slices of a row on distinct banks
    constexpr int kRow = kSlice + 4;
    __shared__ __align__(16) float sB[kTileT][kLanes][kRow];
    __shared__ __align__(16) float sC[kTileT][kLanes][kRow];
    __shared__ float3 sX[kTileT][kChainsPerCta];  // x, delta, z of the tile per chain
    // without the conv, each (token, chain)'s scalars are computed once, by
    // one thread, before the lanes of the chain read them: Δ, Δ·x, the decay
    // base r = 2^(Δ·A[d,0]·log2 e), silu(z); and D·x·silu(z)
    __shared__ float4 sS[kTileT][kChainsPerCta];
    __shared__ float sY[kTileT][kChainsPerCta];
    const int tid = threadIdx.x;
    const int slice = tid % kLanes;
    const int64_t b = blockIdx.y;
    const int64_t d = (int64_t)blockIdx.x * kChainsPerCta + tid / kLanes;
    const bool active = d < p.dim;
    const int N = p.dstate;
    const int n0 = slice * kSlice;

    float A2[kSlice];
    bool structured = true, constant = true;
    float a0 = 0.0f;
    if (active) {
        a0 = p.A[d * N];
#pragma unroll
        for (int i = 0; i < kSlice; ++i) {
            const int n = n0 + i;
            const float an = n < N ? p.A[d * N + n] : 0.0f;
            A2[i] = an * kLog2e;
            if (n < N) {
                structured &= ladder_state(an, a0, n);
                constant &= (an == a0);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < kSlice; ++i) A2[i] = 0.0f;
    }
    // decay strategy for the whole CTA: A[d, n] = A[d, 0] (a per-head scalar,
    // one ex2 per token), A[d, n] = (n+1)·A[d, 0] (a power ladder), or general
    constant = __syncthreads_and(constant);
    structured = __syncthreads_and(structured);
    const float dskip = (active && p.Dskip) ? p.Dskip[d] : 0.0f;
    const float bias = (active && p.delta_bias) ? p.delta_bias[d] : 0.0f;

    float h[kSlice];
#pragma unroll
    for (int i = 0; i < kSlice; ++i) {
        const int n = n0 + i;
        h[i] = (active && p.h0 && n < N) ? p.h0[(b * p.dim + d) * N + n] : 0.0f;
    }

    const bool conv = p.conv_width > 0;
    float cw[kMaxConv] = {0.f, 0.f, 0.f, 0.f}, xw[kMaxConv - 1] = {0.f, 0.f, 0.f};
    float cb = 0.0f;
    if (conv && active) {
        load_conv_taps(p.conv_w, p.conv_width, d, cw);
        cb = p.conv_b ? p.conv_b[d] : 0.0f;
        if (p.conv_init) {
#pragma unroll
            for (int k = 0; k < kMaxConv - 1; ++k)
                xw[k] = p.conv_init[(b * p.dim + d) * (kMaxConv - 1) + k];
        }
    }

    const T *xp = static_cast<const T *>(p.x);
    const T *dp = static_cast<const T *>(p.delta);
    const T *zp = static_cast<const T *>(p.z);
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);
    T *yp = static_cast<T *>(p.y);
    // The next tile's B, C, x, delta, z are loaded into registers while the
    // current one is computed, then staged into shared memory.
    constexpr int kBCPer = kTileT * kWidth / kThreads;          // B (and C) values per thread
    constexpr int kXPer = kTileT * kChainsPerCta / kThreads;    // (x, delta, z) per thread
    float pb[kBCPer], pc[kBCPer];
    float3 px[kXPer];
    auto fetch = [&](int64_t t0) {
#pragma unroll
        for (int i = 0; i < kBCPer; ++i) {
            const int e = tid + i * kThreads;
            const int t = e / kWidth, n = e % kWidth;
            const bool in = t0 + t < p.seqlen && n < N;
            const int64_t idx = (b * p.seqlen + t0 + t) * N + n;
            pb[i] = in ? ldg_f32(Bp + idx) : 0.0f;
            pc[i] = in ? ldg_f32(Cp + idx) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < kXPer; ++i) {
            const int e = tid + i * kThreads;
            const int t = e / kChainsPerCta, cc = e % kChainsPerCta;
            const int64_t dc = (int64_t)blockIdx.x * kChainsPerCta + cc;
            const bool in = t0 + t < p.seqlen && dc < p.dim;
            const int64_t i2 = (b * p.seqlen + t0 + t) * p.dim + dc;
            px[i] = in ? make_float3(ldg_f32(xp + i2), ldg_f32(dp + i2),
                                     kGate ? ldg_f32(zp + i2) : 0.0f)
                       : make_float3(0.f, 0.f, 0.f);
        }
    };
    fetch(0);
    for (int64_t t0 = 0; t0 < p.seqlen; t0 += kTileT) {
        const int nt = (int)min((int64_t)kTileT, p.seqlen - t0);
        __syncthreads();  // the previous tile is consumed
#pragma unroll
        for (int i = 0; i < kBCPer; ++i) {
            const int e = tid + i * kThreads;
            const int t = e / kWidth, n = e % kWidth;
            sB[t][n / kSlice][n % kSlice] = pb[i];
            sC[t][n / kSlice][n % kSlice] = pc[i];
        }
#pragma unroll
        for (int i = 0; i < kXPer; ++i) {
            const int e = tid + i * kThreads;
            sX[e / kChainsPerCta][e % kChainsPerCta] = px[i];
        }
        if (t0 + kTileT < p.seqlen) fetch(t0 + kTileT);
        __syncthreads();
        if (!conv) {
#pragma unroll
            for (int i = 0; i < kXPer; ++i) {
                const int e = tid + i * kThreads;
                const int t = e / kChainsPerCta, c2 = e % kChainsPerCta;
                const int64_t dc = (int64_t)blockIdx.x * kChainsPerCta + c2;
                float4 sc = make_float4(0.f, 0.f, 1.f, 1.f);
                float dxg = 0.0f;
                if (dc < p.dim && t < nt) {
                    const float3 xdz = sX[t][c2];
                    float v = xdz.y + (p.delta_bias ? p.delta_bias[dc] : 0.0f);
                    if (p.softplus) v = softplus_f32(v);
                    const float g = kGate ? silu_f32(xdz.z) : 1.0f;
                    sc = make_float4(v, v * xdz.x, ex2_approx(v * p.A[dc * N] * kLog2e), g);
                    dxg = (p.Dskip ? p.Dskip[dc] : 0.0f) * xdz.x * g;
                }
                sS[t][c2] = sc;
                sY[t][c2] = dxg;
            }
            __syncthreads();
        }
        const int cc = tid / kLanes;
#pragma unroll 2
        for (int t = 0; t < nt; ++t) {
            float xv, dt, u, r, gate;
            if (conv) {
                const float3 xdz = sX[t][cc];
                xv = conv_step(cw, cb, xw, xdz.x);
                dt = active ? xdz.y + bias : 0.0f;
                if (p.softplus && active) dt = softplus_f32(dt);
                u = dt * xv;
                r = ex2_approx(dt * a0 * kLog2e);
                gate = kGate ? silu_f32(xdz.z) : 1.0f;
            } else {
                const float4 sc = sS[t][cc];
                xv = 0.0f;
                dt = sc.x;
                u = sc.y;
                r = sc.z;
                gate = sc.w;
            }
            float a[kSlice];
            if (constant) {
#pragma unroll
                for (int k = 0; k < kSlice; ++k) a[k] = r;
            } else if (structured) {
                // r^(n0 + 1 + i) = r^n0 · r^(i + 1), the powers by a ladder of depth 4
                const float base = ex2_approx(dt * a0 * kLog2e * (float)n0);
                float pw[kSlice];
                pw[0] = r;
                pw[1] = r * r;
                pw[2] = pw[1] * r;
                pw[3] = pw[1] * pw[1];
#pragma unroll
                for (int k = 4; k < 8; ++k) pw[k] = pw[k - 4] * pw[3];
#pragma unroll
                for (int k = 8; k < 16; ++k) pw[k] = pw[k - 8] * pw[7];
#pragma unroll
                for (int k = 0; k < kSlice; ++k) a[k] = base * pw[k];
            } else {
#pragma unroll
                for (int k = 0; k < kSlice; ++k) a[k] = ex2_approx(dt * A2[k]);
            }
            float part0 = 0.0f, part1 = 0.0f;
            const float4 *B4 = reinterpret_cast<const float4 *>(&sB[t][slice][0]);
            const float4 *C4 = reinterpret_cast<const float4 *>(&sC[t][slice][0]);
#pragma unroll
            for (int q = 0; q < kSlice / 4; ++q) {
                const float4 bq = B4[q], cq = C4[q];
                float bv[4] = {bq.x, bq.y, bq.z, bq.w};
                const float cv[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int k = 4 * q + i;
                    if (kZoh) bv[i] *= zoh_factor(dt * A2[k] * kLn2, a[k]);
                    h[k] = fmaf(a[k], h[k], u * bv[i]);
                    if (i & 1)
                        part1 = fmaf(cv[i], h[k], part1);
                    else
                        part0 = fmaf(cv[i], h[k], part0);
                }
            }
            float part = part0 + part1;
#pragma unroll
            for (int m = 1; m < kLanes; m <<= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
            if (active && slice == 0) {
                const float out = conv ? fmaf(dskip, xv, part) * gate
                                       : fmaf(part, gate, sY[t][cc]);
                yp[(b * p.seqlen + t0 + t) * p.dim + d] = from_f32<T>(out);
            }
        }
    }
    if (active && p.final_state) {
#pragma unroll
        for (int k = 0; k < kSlice; ++k)
            if (n0 + k < N) p.final_state[(b * p.dim + d) * N + n0 + k] = h[k];
    }
}

template <typename T, bool kGate, int kLanes>
cudaError_t launch_lanes(const ScanParams &p, cudaStream_t stream) {
    constexpr int kChainsPerCta = kThreads / kLanes;
    const dim3 grid((unsigned)((p.dim + kChainsPerCta - 1) / kChainsPerCta), (unsigned)p.batch);
    if (p.zoh)
        scan_wide_kernel<T, kGate, kLanes, true><<<grid, kThreads, 0, stream>>>(p);
    else
        scan_wide_kernel<T, kGate, kLanes, false><<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T, bool kGate>
cudaError_t launch_gate(const ScanParams &p, cudaStream_t stream) {
    if (p.dstate <= 32) return launch_lanes<T, kGate, 2>(p, stream);
    if (p.dstate <= 64) return launch_lanes<T, kGate, 4>(p, stream);
    if (p.dstate <= 128) return launch_lanes<T, kGate, 8>(p, stream);
    return launch_lanes<T, kGate, 16>(p, stream);
}

}  // namespace

int wide_max_dstate() { return kMaxWide; }

cudaError_t launch_scan_wide(const ScanParams &p, bool bf16, cudaStream_t stream) {
    if (bf16)
        return p.z ? launch_gate<__nv_bfloat16, true>(p, stream)
                   : launch_gate<__nv_bfloat16, false>(p, stream);
    return p.z ? launch_gate<float, true>(p, stream) : launch_gate<float, false>(p, stream);
}

}  // namespace selscan
