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
// bytes. Every lane serves kChainsPerLane chains (8 chains apart). A CTA's
// 256 chains have contiguous states (16 KB): one bulk copy into shared
// memory, issued before anything else, brings them in, so the bytes in
// flight are not bounded by registers. The partial outputs Σ_n C[n]·h[n] are
// combined across a quad with two xor-shuffles. Each state element is
// written by the thread that read it, after the copy has landed, which makes
// the in-place update safe.
#include "selscan_device.cuh"
#include "tma_util.cuh"

namespace selscan {
namespace {

constexpr int kThreads = 256;
constexpr int kLanesPerChain = 4;
constexpr int kChainsPerLane = 4;                 // chains per lane, 8 apart
constexpr int kChainsPerWarp = 32 / kLanesPerChain * kChainsPerLane;  // 32
constexpr int kChainsPerCta = kThreads / 32 * kChainsPerWarp;          // 256
constexpr int kMinCtas = 6;                       // resident CTAs per SM the registers allow
constexpr int kStatusStateCopy = 5;               // device error code: the state copy timed out
constexpr uint64_t kStepWaitNs = 2000000000ull;   // bounded wait for the copy (2 s)
__device__ const int kNoAbortStep = 0;

// Contiguous global -> shared bulk copy (16-byte aligned, size a multiple of
// 16) completing on an mbarrier's transaction count.
__device__ __forceinline__ void bulk_copy_in(void *dst, const void *src, uint32_t bytes,
                                             uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// The causal conv + SiLU for one chain's token: reads the chain's window of
// the previous inputs, writes it back shifted by the new input.
template <typename T>
__device__ __forceinline__ float conv_token(const StepParams &p, int64_t chain, int64_t d) {
    const float xin = ldg_f32(static_cast<const T *>(p.x) + chain);
    float cw[kMaxConv];
    load_conv_taps(p.conv_w, p.conv_width, d, cw);
    float *cs = p.conv_state + chain * (kMaxConv - 1);
    float xw[kMaxConv - 1] = {cs[0], cs[1], cs[2]};
    const float xv = conv_step(cw, p.conv_b ? p.conv_b[d] : 0.0f, xw, xin);
#pragma unroll
    for (int k = 0; k < kMaxConv - 1; ++k) cs[k] = xw[k];
    return xv;
}

// x (after the conv, if any), z and Δ of one chain's token. With the conv,
// conv_x is the conv output computed by the caller.
template <typename T, bool kGate, bool kConv>
__device__ __forceinline__ float token_scalars(const StepParams &p, int64_t chain, int64_t d,
                                               float &xv, float &zv, float conv_x = 0.0f) {
    const T *xp = static_cast<const T *>(p.x);
    const T *dp = static_cast<const T *>(p.delta);
    xv = kConv ? conv_x : ldg_f32(xp + chain);
    zv = kGate ? ldg_f32(static_cast<const T *>(p.z) + chain) : 0.0f;
    float dt = ldg_f32(dp + chain) + (p.delta_bias ? p.delta_bias[d] : 0.0f);
    if (p.softplus) dt = softplus_f32(dt);
    return dt;
}

// Four consecutive elements of B or C, widened to float (16-byte aligned for
// float, 8-byte aligned for bf16).
__device__ __forceinline__ float4 ld4_f32(const float *p) {
    return __ldg(reinterpret_cast<const float4 *>(p));
}
__device__ __forceinline__ float4 ld4_f32(const __nv_bfloat16 *p) {
    const uint2 r = __ldg(reinterpret_cast<const uint2 *>(p));
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// dstate == 16 with state, A, B, C aligned for vector accesses.
//
// A warp serves 32 consecutive chains base..base+31. Lane (j = lane/4,
// q = lane%4) holds quarter q of the states of chains base + 8k + j,
// k = 0..3, and owns the per-token scalars of chain base + 8q + j: it loads
// that chain's x, delta and z (one 64-byte access per tensor per warp),
// computes Δ and Δ·x once, and hands them to the three other lanes of its
// quad that hold a quarter of that chain, by shuffle. After the quad
// reduction of Σ_n C[n]·h[n] every lane of the quad has the sum, and the
// owner writes the chain's y.
template <typename T, bool kGate, bool kConv, bool kZoh>
__global__ void __launch_bounds__(kThreads, kMinCtas)
state_update_vec_kernel(const StepParams p, int *status) {
    __shared__ __align__(128) float4 sst[kChainsPerCta * 4];  // the CTA's states, 16 KB
    __shared__ uint64_t bar;
    const int lane = threadIdx.x & 31;
    const int q = lane & 3;
    const int j = lane >> 2;
    const int quad0 = lane & ~3;
    const int wl = threadIdx.x >> 5;  // warp within the CTA
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t total = p.batch * p.dim;
    const int64_t base = warp * kChainsPerWarp;
    const int64_t cta0 = (int64_t)blockIdx.x * kChainsPerCta;

    // the CTA's states first: one copy of its contiguous chains
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        const uint32_t bytes = (uint32_t)(min((int64_t)kChainsPerCta, total - cta0) * kMaxN * 4);
        mbar_arrive_expect_tx(&bar, bytes);
        bulk_copy_in(sst, p.state + cta0 * kMaxN, bytes, &bar);
    }
    __syncthreads();

    // (b, d) of chain base + j by one division, then of base + 8k + j by steps of 8
    int64_t bk[kChainsPerLane], dk[kChainsPerLane];
    {
        int64_t b = (base + j) / p.dim;
        int64_t d = base + j - b * p.dim;
#pragma unroll
        for (int k = 0; k < kChainsPerLane; ++k) {
            bk[k] = b;
            dk[k] = d;
            d += 8;
            while (d >= p.dim) {
                d -= p.dim;
                ++b;
            }
        }
    }

    // per-token scalars of the owned chain base + 8q + j
    const int64_t own = base + 8 * q + j;
    int64_t own_d = dk[0];
#pragma unroll
    for (int k = 1; k < kChainsPerLane; ++k) own_d = (q == k) ? dk[k] : own_d;
    float dt_own = 0.f, u_own = 0.f, skip = 0.f, gate = 1.f;
    if (own < total) {
        float xv, zv;
        const float xc = kConv ? conv_token<T>(p, own, own_d) : 0.0f;
        dt_own = token_scalars<T, kGate, kConv>(p, own, own_d, xv, zv, xc);
        u_own = dt_own * xv;
        skip = (p.Dskip ? p.Dskip[own_d] : 0.0f) * xv;
        if (kGate) gate = silu_f32(zv);
    }

    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);
    if (!__all_sync(0xffffffffu, mbar_wait(&bar, 0, &kNoAbortStep, kStepWaitNs))) {
        // the warp agrees to give up: record it, give the copy one more
        // bounded wait to land, and leave the warp's chains as they were
        if (status) atomicCAS(status, 0, kStatusStateCopy);
        mbar_wait(&bar, 0, &kNoAbortStep, kStepWaitNs);
        return;
    }
    float mine = 0.f;
#pragma unroll
    for (int k = 0; k < kChainsPerLane; ++k) {
        const int64_t chain = base + 8 * k + j;
        const float dt = __shfl_sync(0xffffffffu, dt_own, quad0 | k);
        const float u = __shfl_sync(0xffffffffu, u_own, quad0 | k);
        float partial = 0.0f;
        if (chain < total) {
            const float4 a4 = __ldg(reinterpret_cast<const float4 *>(p.A + dk[k] * kMaxN + 4 * q));
            const float4 b4 = ld4_f32(Bp + bk[k] * kMaxN + 4 * q);
            const float4 c4 = ld4_f32(Cp + bk[k] * kMaxN + 4 * q);
            const float dl = dt * kLog2e;
            float4 h = sst[(wl * kChainsPerWarp + 8 * k + j) * 4 + q];
            const float e0 = ex2_approx(dl * a4.x), e1 = ex2_approx(dl * a4.y);
            const float e2 = ex2_approx(dl * a4.z), e3 = ex2_approx(dl * a4.w);
            float4 bz = b4;
            if (kZoh) {
                bz.x *= zoh_factor(dt * a4.x, e0);
                bz.y *= zoh_factor(dt * a4.y, e1);
                bz.z *= zoh_factor(dt * a4.z, e2);
                bz.w *= zoh_factor(dt * a4.w, e3);
            }
            h.x = fmaf(e0, h.x, u * bz.x);
            h.y = fmaf(e1, h.y, u * bz.y);
            h.z = fmaf(e2, h.z, u * bz.z);
            h.w = fmaf(e3, h.w, u * bz.w);
            *reinterpret_cast<float4 *>(p.state + chain * kMaxN + 4 * q) = h;
            partial = fmaf(c4.x, h.x, fmaf(c4.y, h.y, fmaf(c4.z, h.z, c4.w * h.w)));
        }
        // every lane takes part in the shuffles (inactive chains carry zeros)
        partial += __shfl_xor_sync(0xffffffffu, partial, 1);
        partial += __shfl_xor_sync(0xffffffffu, partial, 2);
        mine = (q == k) ? partial : mine;
    }
    if (own < total) {
        float out = skip + mine;
        if (kGate) out *= gate;
        static_cast<T *>(p.y)[own] = from_f32<T>(out);
    }
}

// Any dstate: one quad of lanes per chain, lane q taking states q, q + 4, ...
template <typename T, bool kGate, bool kConv, bool kZoh>
__global__ void __launch_bounds__(kThreads)
state_update_kernel(const StepParams p) {
    const int64_t gid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t chain = gid / kLanesPerChain;
    const int q = (int)(gid % kLanesPerChain);
    const bool active = chain < p.batch * p.dim;
    const int64_t b = active ? chain / p.dim : 0;
    const int64_t d = active ? chain % p.dim : 0;
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);

    float partial = 0.0f, xv = 0.0f, zv = 0.0f;
    // the conv window belongs to the chain: the quad's first lane advances it
    float xc = 0.0f;
    if (kConv) {
        if (active && q == 0) xc = conv_token<T>(p, chain, d);
        xc = __shfl_sync(0xffffffffu, xc, (threadIdx.x & 31) & ~3);
    }
    if (active) {
        const float dt = token_scalars<T, kGate, kConv>(p, chain, d, xv, zv, xc);
        const float u = dt * xv;
        float *st = p.state + chain * p.dstate;
        // lane q takes states q, q + 4, q + 8, ... (any d_state)
#pragma unroll 4
        for (int n = q; n < p.dstate; n += kLanesPerChain) {
            const float an = p.A[d * p.dstate + n];
            const float a = ex2_approx(dt * an * kLog2e);
            float bn = ldg_f32(Bp + b * p.dstate + n);
            if (kZoh) bn *= zoh_factor(dt * an, a);
            const float h = fmaf(a, st[n], u * bn);
            st[n] = h;
            partial = fmaf(ldg_f32(Cp + b * p.dstate + n), h, partial);
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

template <typename T, bool kGate, bool kConv, bool kZoh>
cudaError_t launch_zoh(const StepParams &p, cudaStream_t stream) {
    const int64_t chains = p.batch * p.dim;
    const uintptr_t bc_align = 4 * sizeof(T) - 1;
    const bool vec = p.dstate == kMaxN && (reinterpret_cast<uintptr_t>(p.state) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(p.A) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(p.B) & bc_align) == 0 &&
                     (reinterpret_cast<uintptr_t>(p.C) & bc_align) == 0;
    if (vec) {
        int *status = nullptr;
        const cudaError_t e = device_status_address(&status);
        if (e != cudaSuccess) return e;
        const int64_t warps = (chains + kChainsPerWarp - 1) / kChainsPerWarp;
        const unsigned blocks = (unsigned)((warps * 32 + kThreads - 1) / kThreads);
        state_update_vec_kernel<T, kGate, kConv, kZoh><<<blocks, kThreads, 0, stream>>>(p, status);
    } else {
        const int64_t threads = chains * kLanesPerChain;
        const unsigned blocks = (unsigned)((threads + kThreads - 1) / kThreads);
        state_update_kernel<T, kGate, kConv, kZoh><<<blocks, kThreads, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

template <typename T, bool kGate, bool kConv>
cudaError_t launch_conv(const StepParams &p, cudaStream_t stream) {
    return p.zoh ? launch_zoh<T, kGate, kConv, true>(p, stream)
                 : launch_zoh<T, kGate, kConv, false>(p, stream);
}

template <typename T, bool kGate>
cudaError_t launch_gate(const StepParams &p, cudaStream_t stream) {
    return p.conv_width > 0 ? launch_conv<T, kGate, true>(p, stream)
                            : launch_conv<T, kGate, false>(p, stream);
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
