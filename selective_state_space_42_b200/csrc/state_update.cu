// state_update.cu -- single-token recurrent update (inference), in place.
//
// Pages: "Mamba и State Space Models: альтернатива Transformer", "SSM as
// Convolution" (recurrent mode for inference) and "SSM as RNN" (one step of
// the recurrence); "Mamba & State Space Models — Guide Complet" §6 (a
// constant-size state instead of a growing cache) and §4 (the step itself).
//
// The step is bound by HBM traffic: the float32 state [batch, dim, dstate]
// is read and written once, everything else is small. Lanes work in quads:
// the four lanes of a quad hold the four 16-byte quarters of one chain's
// 16 states, so each warp-wide access covers 8 whole chains = 512 contiguous
// bytes. Every lane serves kChainsPerLane chains (8 chains apart), issuing
// all of their state loads before any arithmetic so that enough bytes are in
// flight to cover DRAM latency. The partial outputs Σ_n C[n]·h[n] are
// combined across a quad with two xor-shuffles. Each state element is read
// and written by the same thread, which makes the in-place update safe.
#include "selscan_device.cuh"

namespace selscan {
namespace {

constexpr int kThreads = 256;
constexpr int kLanesPerChain = 4;
constexpr int kPerLane = kMaxN / kLanesPerChain;  // 4 states per lane
constexpr int kChainsPerLane = 4;                 // chains per lane, 8 apart
constexpr int kChainsPerWarp = 32 / kLanesPerChain * kChainsPerLane;  // 32

template <typename T, bool kGate>
__device__ __forceinline__ float token_scalars(const StepParams &p, int64_t chain, int64_t d,
                                               float &xv, float &zv) {
    const T *xp = static_cast<const T *>(p.x);
    const T *dp = static_cast<const T *>(p.delta);
    xv = ldg_f32(xp + chain);
    zv = kGate ? ldg_f32(static_cast<const T *>(p.z) + chain) : 0.0f;
    float dt = ldg_f32(dp + chain) + (p.delta_bias ? p.delta_bias[d] : 0.0f);
    if (p.softplus) dt = softplus_f32(dt);
    return dt;
}

// dstate == 16, state 16-byte aligned: vector path.
template <typename T, bool kGate>
__global__ void __launch_bounds__(kThreads)
state_update_vec_kernel(const StepParams p) {
    const int lane = threadIdx.x & 31;
    const int q = lane & 3;         // quarter of the chain's states
    const int j = lane >> 2;        // chain within an 8-chain group
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t total = p.batch * p.dim;
    const int64_t base = warp * kChainsPerWarp;

    float4 st[kChainsPerLane];
    bool act[kChainsPerLane];
#pragma unroll
    for (int k = 0; k < kChainsPerLane; ++k) {
        const int64_t chain = base + 8 * k + j;
        act[k] = chain < total;
        st[k] = act[k] ? *reinterpret_cast<const float4 *>(p.state + chain * kMaxN + 4 * q)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);
#pragma unroll
    for (int k = 0; k < kChainsPerLane; ++k) {
        const int64_t chain = act[k] ? base + 8 * k + j : 0;
        const int64_t b = chain / p.dim;
        const int64_t d = chain - b * p.dim;
        float xv = 0.f, zv = 0.f, dt = 0.f;
        float partial = 0.0f;
        if (act[k]) {
            dt = token_scalars<T, kGate>(p, chain, d, xv, zv);
            const float u = dt * xv;
            const float4 a4 = *reinterpret_cast<const float4 *>(p.A + d * kMaxN + 4 * q);
            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
            float h[4] = {st[k].x, st[k].y, st[k].z, st[k].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int n = 4 * q + i;
                const float a = ex2_approx(dt * av[i] * kLog2e);
                h[i] = fmaf(a, h[i], u * ldg_f32(Bp + b * kMaxN + n));
                partial = fmaf(ldg_f32(Cp + b * kMaxN + n), h[i], partial);
            }
            *reinterpret_cast<float4 *>(p.state + chain * kMaxN + 4 * q) =
                make_float4(h[0], h[1], h[2], h[3]);
        }
        // every lane takes part in the shuffles (inactive chains carry zeros)
        partial += __shfl_xor_sync(0xffffffffu, partial, 1);
        partial += __shfl_xor_sync(0xffffffffu, partial, 2);
        if (act[k] && q == 0) {
            float out = fmaf(p.Dskip ? p.Dskip[d] : 0.0f, xv, partial);
            if (kGate) out *= silu_f32(zv);
            static_cast<T *>(p.y)[chain] = from_f32<T>(out);
        }
    }
}

// Any dstate ≤ 16: one quad of lanes per chain, scalar accesses.
template <typename T, bool kGate>
__global__ void __launch_bounds__(kThreads)
state_update_kernel(const StepParams p) {
    const int64_t gid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t chain = gid / kLanesPerChain;
    const int q = (int)(gid % kLanesPerChain);
    const bool active = chain < p.batch * p.dim;
    const int64_t b = active ? chain / p.dim : 0;
    const int64_t d = active ? chain % p.dim : 0;
    const int n0 = q * kPerLane;
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);

    float partial = 0.0f, xv = 0.0f, zv = 0.0f;
    if (active) {
        const float dt = token_scalars<T, kGate>(p, chain, d, xv, zv);
        const float u = dt * xv;
        float *st = p.state + chain * p.dstate + n0;
#pragma unroll
        for (int k = 0; k < kPerLane; ++k) {
            const int n = n0 + k;
            if (n < p.dstate) {
                const float a = ex2_approx(dt * p.A[d * p.dstate + n] * kLog2e);
                const float h = fmaf(a, st[k], u * ldg_f32(Bp + b * p.dstate + n));
                st[k] = h;
                partial = fmaf(ldg_f32(Cp + b * p.dstate + n), h, partial);
            }
        }
    }
    partial += __shfl_xor_sync(0xffffffffu, partial, 1);
    partial += __shfl_xor_sync(0xffffffffu, partial, 2);
    if (active && q == 0) {
        float out = fmaf(p.Dskip ? p.Dskip[d] : 0.0f, xv, partial);
        if (kGate) out *= silu_f32(zv);
        static_cast<T *>(p.y)[chain] = from_f32<T>(out);
    }
}

template <typename T, bool kGate>
cudaError_t launch_gate(const StepParams &p, cudaStream_t stream) {
    const int64_t chains = p.batch * p.dim;
    const bool vec = p.dstate == kMaxN && (reinterpret_cast<uintptr_t>(p.state) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(p.A) & 15) == 0;
    if (vec) {
        const int64_t warps = (chains + kChainsPerWarp - 1) / kChainsPerWarp;
        const unsigned blocks = (unsigned)((warps * 32 + kThreads - 1) / kThreads);
        state_update_vec_kernel<T, kGate><<<blocks, kThreads, 0, stream>>>(p);
    } else {
        const int64_t threads = chains * kLanesPerChain;
        const unsigned blocks = (unsigned)((threads + kThreads - 1) / kThreads);
        state_update_kernel<T, kGate><<<blocks, kThreads, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const StepParams &p, cudaStream_t stream) {
    return p.z ? launch_gate<T, true>(p, stream) : launch_gate<T, false>(p, stream);
}

}  // namespace

cudaError_t launch_state_update(const StepParams &p, bool bf16, cudaStream_t stream) {
    return bf16 ? launch_typed<__nv_bfloat16>(p, stream) : launch_typed<float>(p, stream);
}

}  // namespace selscan
