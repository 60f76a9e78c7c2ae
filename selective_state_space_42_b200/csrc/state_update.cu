// state_update.cu -- single-token recurrent update (inference), in place.
//
// Pages: "Mamba и State Space Models: альтернатива Transformer", "SSM as
// Convolution" (recurrent mode for inference) and "SSM as RNN" (one step of
// the recurrence); "Mamba & State Space Models — Guide Complet" §6 (a
// constant-size state instead of a growing cache) and §4 (the step itself).
//
// The step is bound by HBM traffic: the float32 state [batch, dim, dstate] is
// read and written once, everything else is small. Four consecutive lanes own
// one (b, d) chain and four consecutive states each, so a warp reads and writes
// 8 whole chains = 512 contiguous bytes of state per access (16 bytes per lane
// when dstate == 16). The partial outputs Σ_n C[n]·h[n] are combined across the
// four lanes with two xor-shuffles. Each element of the state is read and
// written by the same thread, which makes the in-place update safe.
#include "selscan_device.cuh"

namespace selscan {
namespace {

constexpr int kThreads = 256;
constexpr int kLanesPerChain = 4;
constexpr int kPerLane = kMaxN / kLanesPerChain;  // 4 states per lane

template <typename T, bool kGate, bool kVec>
__global__ void __launch_bounds__(kThreads)
state_update_kernel(const StepParams p) {
    const int64_t gid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t chain = gid / kLanesPerChain;
    const int q = (int)(gid % kLanesPerChain);
    const bool active = chain < p.batch * p.dim;
    const int64_t b = active ? chain / p.dim : 0;
    const int64_t d = active ? chain % p.dim : 0;
    const int n0 = q * kPerLane;

    const T *__restrict__ xp = static_cast<const T *>(p.x);
    const T *__restrict__ dp = static_cast<const T *>(p.delta);
    const T *__restrict__ Bp = static_cast<const T *>(p.B);
    const T *__restrict__ Cp = static_cast<const T *>(p.C);

    float partial = 0.0f, xv = 0.0f;
    float h[kPerLane];
    float *st = p.state + chain * p.dstate + n0;
    if (active) {
        xv = ldg_f32(xp + chain);
        float dt = ldg_f32(dp + chain) + (p.delta_bias ? p.delta_bias[d] : 0.0f);
        if (p.softplus) dt = softplus_f32(dt);
        const float u = dt * xv;
        if (kVec) {
            const float4 s = *reinterpret_cast<const float4 *>(st);
            h[0] = s.x; h[1] = s.y; h[2] = s.z; h[3] = s.w;
        } else {
#pragma unroll
            for (int k = 0; k < kPerLane; ++k) h[k] = n0 + k < p.dstate ? st[k] : 0.0f;
        }
        const float *Ar = p.A + d * p.dstate;
#pragma unroll
        for (int k = 0; k < kPerLane; ++k) {
            const int n = n0 + k;
            if (kVec || n < p.dstate) {
                const float a = ex2_approx(dt * Ar[n] * kLog2e);
                h[k] = fmaf(a, h[k], u * ldg_f32(Bp + b * p.dstate + n));
                partial = fmaf(ldg_f32(Cp + b * p.dstate + n), h[k], partial);
            }
        }
        if (kVec) {
            *reinterpret_cast<float4 *>(st) = make_float4(h[0], h[1], h[2], h[3]);
        } else {
#pragma unroll
            for (int k = 0; k < kPerLane; ++k)
                if (n0 + k < p.dstate) st[k] = h[k];
        }
    }
    // all 32 lanes take part in the shuffles (inactive lanes carry zeros)
    partial += __shfl_xor_sync(0xffffffffu, partial, 1);
    partial += __shfl_xor_sync(0xffffffffu, partial, 2);
    if (active && q == 0) {
        float out = fmaf(p.Dskip ? p.Dskip[d] : 0.0f, xv, partial);
        if (kGate) out *= silu_f32(ldg_f32(static_cast<const T *>(p.z) + chain));
        static_cast<T *>(p.y)[chain] = from_f32<T>(out);
    }
}

template <typename T, bool kGate>
cudaError_t launch_gate(const StepParams &p, cudaStream_t stream) {
    const int64_t threads = p.batch * p.dim * kLanesPerChain;
    const unsigned blocks = (unsigned)((threads + kThreads - 1) / kThreads);
    const bool vec = p.dstate == kMaxN && (reinterpret_cast<uintptr_t>(p.state) & 15) == 0;
    if (vec)
        state_update_kernel<T, kGate, true><<<blocks, kThreads, 0, stream>>>(p);
    else
        state_update_kernel<T, kGate, false><<<blocks, kThreads, 0, stream>>>(p);
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
