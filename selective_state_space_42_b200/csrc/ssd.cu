// ssd.cu -- the scan with one scalar A per head, in chunked matrix form.
//
// Pages: "Mamba & State Space Models — Guide Complet" §5 "Mamba-2" / "SSD —
// State Space Dual": with a scalar A per head the scan's output is a
// lower-triangular (causal mask L) product with a structured semiseparable
// matrix, y = (L ◦ S)·u. Written out for one head (channels d = h·P + p,
// shared B and C, Δ and A per head), token i's output is
//   y_i = Σ_{j ≤ i} (C_i·B_j)·exp(Σ_{j<k≤i} Δ_k·A)·Δ_j·x_j + D·x_i,
// the same result as the recurrence h_t = exp(Δ_t·A)·h_{t−1} + Δ_t·B_t·x_t,
// y_t = C_t·h_t + D·x_t. Cut the sequence into chunks of Q tokens; inside a
// chunk the sum over j is a masked Q×Q matrix product, and the state carried
// in from earlier chunks adds C_i·exp(Acum_i)·h_in (Acum = the within-chunk
// prefix sum of Δ·A). Three kernels:
//   ssd_chunk_kernel  per (batch row, head, chunk): G = C·Bᵀ (Q×Q over N),
//                     M = G ◦ exp(Acum_i − Acum_j)·Δ_j on j ≤ i, the chunk's
//                     own output M·X (Q×P), and its final state from zero,
//                     S = Bᵀ·(w ◦ X) (N×P) with w_j = exp(Acum_end − Acum_j)·Δ_j;
//   ssd_state_kernel  per (batch row, head, state element): the states carried
//                     between chunks, h_c = exp(Acum_end,c)·h_{c−1} + S_c, and
//                     the final state;
//   ssd_out_kernel    per chunk again: y = M·X + exp(Acum_i)·C·h_in + D·x,
//                     times silu(z).
// The products are FP32 (register-blocked 4×4 per thread from shared memory);
// chunks are independent, so the whole sequence runs in parallel except for
// the element-wise carry. These kernels serve float32 I/O (64-token chunks);
// bfloat16 I/O goes to the tensor-core kernels of ssd_tc.cu (launch_ssd
// below chooses).
#include "ssd_params.cuh"

namespace selscan {
namespace {

constexpr int kQ = 64;           // tokens per chunk
constexpr int kP = 64;           // largest head dimension
constexpr int kNS = 128;         // largest d_state
constexpr int kThr = 256;

struct SsdSmem {
    float B[kQ][kNS + 1];
    float C[kQ][kNS + 1];
    float X[kQ][kP + 1];
    float M[kQ][kQ + 1];
    float dt[kQ];
    float acum[kQ];
};

// Δ (softplus of dt + bias, or dt + bias) and the within-chunk prefix sums
// of Δ·A for the chunk's tokens; zero past the sequence end.
template <typename T>
__device__ __forceinline__ void chunk_dt(SsdSmem &S, const SsdParams &p, long long b, int h,
                                         long long t0, int nq) {
    const T *dtp = static_cast<const T *>(p.dt);
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.0f;
    if (threadIdx.x < kQ) {
        const int q = threadIdx.x;
        float v = 0.0f;
        if (q < nq) {
            v = ldg_f32(dtp + (b * p.seqlen + t0 + q) * p.nheads + h) + bias;
            if (p.softplus) v = softplus_f32(v);
        }
        S.dt[q] = v;
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // inclusive prefix sum of Δ·A over the 64 tokens
        const int l = threadIdx.x;
        const float A = p.A[h];
        float a0 = S.dt[2 * l] * A, a1 = S.dt[2 * l + 1] * A;
        float s = a0 + a1;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const float o = __shfl_up_sync(0xffffffffu, s, m);
            if (l >= m) s += o;
        }
        const float before = s - (a0 + a1);
        S.acum[2 * l] = before + a0;
        S.acum[2 * l + 1] = before + a0 + a1;
    }
    __syncthreads();
}

template <typename T>
__device__ __forceinline__ void load_rows(float (*dst)[kNS + 1], const T *src, long long row0,
                                          int nq, int N) {
    for (int e = threadIdx.x; e < kQ * kNS; e += kThr) {
        const int q = e / kNS, n = e % kNS;
        dst[q][n] = (q < nq && n < N) ? ldg_f32(src + (row0 + q) * N + n) : 0.0f;
    }
}

template <typename T>
__device__ __forceinline__ void load_x(SsdSmem &S, const SsdParams &p, long long b, int h,
                                       long long t0, int nq) {
    const T *xp = static_cast<const T *>(p.x);
    const long long D = (long long)p.nheads * p.headdim;
    for (int e = threadIdx.x; e < kQ * kP; e += kThr) {
        const int q = e / kP, pp = e % kP;
        S.X[q][pp] = (q < nq && pp < p.headdim)
                         ? ldg_f32(xp + (b * p.seqlen + t0 + q) * D + (long long)h * p.headdim + pp)
                         : 0.0f;
    }
}

// M = (C·Bᵀ) ◦ exp(Acum_i − Acum_j)·Δ_j on j ≤ i (zero above the diagonal
// and past the chunk's tokens); thread tile 4×4.
__device__ __forceinline__ void build_M(SsdSmem &S, int nq, int N) {
    const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
    float g[4][4] = {};
    for (int n = 0; n < N; ++n) {
        float cv[4], bv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            cv[r] = S.C[4 * ti + r][n];
            bv[r] = S.B[4 * tj + r][n];
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) g[r][c] = fmaf(cv[r], bv[c], g[r][c]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = 4 * ti + r;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int j = 4 * tj + c;
            float m = 0.0f;
            if (j <= i && i < nq) m = g[r][c] * __expf(S.acum[i] - S.acum[j]) * S.dt[j];
            S.M[i][j] = m;
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kThr) ssd_chunk_kernel(const SsdParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SsdSmem &S = *reinterpret_cast<SsdSmem *>(smem_raw);
    const int c = blockIdx.x, h = blockIdx.y;
    const long long b = blockIdx.z;
    const long long t0 = (long long)c * kQ;
    const int nq = (int)min((long long)kQ, p.seqlen - t0);
    const int N = p.dstate, P = p.headdim;
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);
    load_rows<T>(S.B, Bp, b * p.seqlen + t0, nq, N);
    load_rows<T>(S.C, Cp, b * p.seqlen + t0, nq, N);
    load_x<T>(S, p, b, h, t0, nq);
    chunk_dt<T>(S, p, b, h, t0, nq);  // ends with __syncthreads
    build_M(S, nq, N);
    __syncthreads();

    const long long D = (long long)p.nheads * P;
    // the chunk's own output Y = M·X (Q×P), into the float32 partial output
    {
        const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
        float y[4][4] = {};
        for (int j = 0; j < kQ; ++j) {
            float mv[4], xv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                mv[r] = S.M[4 * ti + r][j];
                xv[r] = S.X[j][4 * tj + r];
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) y[r][cc] = fmaf(mv[r], xv[cc], y[r][cc]);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = 4 * ti + r;
            if (i >= nq) continue;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int pp = 4 * tj + cc;
                if (pp < P) p.ypart[(b * p.seqlen + t0 + i) * D + (long long)h * P + pp] = y[r][cc];
            }
        }
    }
    // the chunk's final state from zero: S = Bᵀ·(w ◦ X), N×P, thread tile 8×4
    {
        const float aend = S.acum[nq - 1];
        const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;  // n rows 8·ti.., p cols 4·tj..
        float s[8][4] = {};
        for (int j = 0; j < nq; ++j) {
            const float w = __expf(aend - S.acum[j]) * S.dt[j];
            float bv[8], xv[4];
#pragma unroll
            for (int r = 0; r < 8; ++r) bv[r] = S.B[j][8 * ti + r] * w;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) xv[cc] = S.X[j][4 * tj + cc];
#pragma unroll
            for (int r = 0; r < 8; ++r)
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) s[r][cc] = fmaf(bv[r], xv[cc], s[r][cc]);
        }
        float *dst = p.chunk_state + (((b * p.nheads + h) * p.nchunks + c) * kNS) * kP;
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) dst[(8 * ti + r) * kP + 4 * tj + cc] = s[r][cc];
        if (threadIdx.x == 0)
            p.chunk_decay[(b * p.nheads + h) * p.nchunks + c] = __expf(aend);
    }
}

// States between chunks, one thread per (batch row, head, n, p):
// h_in[c] = state before chunk c; h_{c} = decay_c·h_{c−1} + S_c.
__global__ void ssd_state_kernel(const SsdParams p) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long per = (long long)kNS * kP;
    if (e >= (long long)p.batch * p.nheads * per) return;
    const long long bh = e / per;
    const int n = (int)((e % per) / kP), pp = (int)(e % kP);
    const long long b = bh / p.nheads;
    const int h = (int)(bh % p.nheads);
    float st = 0.0f;
    if (p.h0 && n < p.dstate && pp < p.headdim)
        st = p.h0[((b * p.nheads + h) * (long long)p.headdim + pp) * p.dstate + n];
    for (int c = 0; c < p.nchunks; ++c) {
        const long long idx = ((bh * p.nchunks + c) * kNS + n) * kP + pp;
        p.state_in[idx] = st;
        st = fmaf(p.chunk_decay[bh * p.nchunks + c], st, p.chunk_state[idx]);
    }
    if (p.final_state && n < p.dstate && pp < p.headdim)
        p.final_state[((b * p.nheads + h) * (long long)p.headdim + pp) * p.dstate + n] = st;
}

// y = Y_chunk + exp(Acum_i)·C·h_in + D·x, gated; per (chunk, head, batch row).
template <typename T, bool kGate>
__global__ void __launch_bounds__(kThr) ssd_out_kernel(const SsdParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SsdSmem &S = *reinterpret_cast<SsdSmem *>(smem_raw);
    const int c = blockIdx.x, h = blockIdx.y;
    const long long b = blockIdx.z;
    const long long t0 = (long long)c * kQ;
    const int nq = (int)min((long long)kQ, p.seqlen - t0);
    const int N = p.dstate, P = p.headdim;
    load_rows<T>(S.C, static_cast<const T *>(p.C), b * p.seqlen + t0, nq, N);
    // h_in (N×P, [n][p]) in the B buffer, which this kernel does not use
    static_assert(sizeof(float) * kNS * kP <= sizeof(SsdSmem::B), "h_in fits the B buffer");
    const float *hin = p.state_in + (((b * p.nheads + h) * p.nchunks + c) * kNS) * kP;
    float(*H)[kP] = reinterpret_cast<float(*)[kP]>(&S.B[0][0]);
    for (int e = threadIdx.x; e < kNS * kP; e += kThr) H[e / kP][e % kP] = hin[e];
    chunk_dt<T>(S, p, b, h, t0, nq);  // ends with __syncthreads

    const long long D = (long long)p.nheads * P;
    const T *xp = static_cast<const T *>(p.x);
    const T *zp = static_cast<const T *>(p.z);
    T *yp = static_cast<T *>(p.y);
    const float dsk = p.Dskip ? p.Dskip[h] : 0.0f;
    const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
    float y[4][4] = {};
    for (int n = 0; n < N; ++n) {
        float cv[4], hv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            cv[r] = S.C[4 * ti + r][n];
            hv[r] = H[n][4 * tj + r];
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) y[r][cc] = fmaf(cv[r], hv[cc], y[r][cc]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = 4 * ti + r;
        if (i >= nq) continue;
        const float dec = __expf(S.acum[i]);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const int pp = 4 * tj + cc;
            if (pp >= P) continue;
            const long long idx = (b * p.seqlen + t0 + i) * D + (long long)h * P + pp;
            const float xv = ldg_f32(xp + idx);
            float out = fmaf(dec, y[r][cc], p.ypart[idx]) + dsk * xv;
            if (kGate) out *= silu_f32(ldg_f32(zp + idx));
            yp[idx] = from_f32<T>(out);
        }
    }
}

cudaError_t launch_state(const SsdParams &p, cudaStream_t stream) {
    const long long nst = (long long)p.batch * p.nheads * kNS * kP;
    ssd_state_kernel<<<(unsigned)((nst + 255) / 256), 256, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_f32(const SsdParams &p, cudaStream_t stream) {
    const size_t smem = sizeof(SsdSmem);
    static bool configured[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(ssd_chunk_kernel<float>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(ssd_out_kernel<float, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(ssd_out_kernel<float, false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const dim3 grid((unsigned)p.nchunks, (unsigned)p.nheads, (unsigned)p.batch);
    ssd_chunk_kernel<float><<<grid, kThr, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_state(p, stream);
    if (e != cudaSuccess) return e;
    if (p.z)
        ssd_out_kernel<float, true><<<grid, kThr, smem, stream>>>(p);
    else
        ssd_out_kernel<float, false><<<grid, kThr, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

int ssd_chunk_tokens() { return kQ; }
int ssd_max_headdim() { return kP; }
int ssd_max_dstate() { return kNS; }

// float32 I/O: the float32 chunk kernels above with 64-token chunks.
// bfloat16 I/O: the tensor-core chunk kernels (ssd_tc.cu) with 128-token
// chunks; the element-wise carry between chunks is the same kernel.
cudaError_t launch_ssd(const SsdParams &p_in, bool bf16, cudaStream_t stream) {
    SsdParams p = p_in;
    if (!bf16) {
        p.nchunks = (int)((p.seqlen + kQ - 1) / kQ);
        return launch_f32(p, stream);
    }
    if (!ssd_tc_supported(p.headdim, p.dstate)) return cudaErrorInvalidValue;
    const int q = ssd_tc_chunk_tokens();
    p.nchunks = (int)((p.seqlen + q - 1) / q);
    cudaError_t e = launch_ssd_tc_state(p, stream);
    if (e != cudaSuccess) return e;
    e = launch_ssd_tc_carry(p, stream);
    if (e != cudaSuccess) return e;
    return launch_ssd_tc_out(p, stream);
}

}  // namespace selscan
