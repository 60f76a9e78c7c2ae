// ssd_tc.cu -- the chunked matrix form of the scalar-A-per-head scan on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Pages: "Mamba & State Space Models — Guide Complet" §5 "Mamba-2" / "SSD —
// State Space Dual": with one scalar A per head the scan is a masked product
// with a semiseparable matrix, so each chunk's work is dense matrix products.
// For one head (channels d = h·P + p; Δ and A per head; B, C shared) and a
// chunk of Q = 128 tokens with within-chunk prefix sums Acum of Δ·A:
//   chunk state from zero   S  = Bᵀ·(w ◦ X),  w_j = exp(Acum_end − Acum_j)·Δ_j   (N×P)
//   chunk output            y  = M·X + diag(exp(Acum_i))·C·h_in + D·x,
//                           M  = (C·Bᵀ) ◦ [j ≤ i]·exp(Acum_i − Acum_j)·Δ_j        (Q×Q)
// and h_in, the state entering each chunk, comes from the element-wise carry
// h_c = exp(Acum_end,c)·h_{c−1} + S_c (ssd.cu). Two kernels here:
//   ssd_tc_state_kernel  S for one (chunk, head, batch row): MMAs of
//                        M=128 (state n) × N=64 (head channel p) × K=2×128
//                        (token; w ◦ X as a bfloat16 high/low pair)
//   ssd_tc_out_kernel    G = C·Bᵀ (128×128, K = d_state) and C·h_in (128×64) on
//                        the tensor cores (h_in as a bfloat16 high/low pair),
//                        M built from G by the 128 threads
//                        (thread i = token i = tensor-memory lane i) and
//                        written back to shared memory as a bfloat16 pair
//                        M_hi + M_lo, then M·X (128×64, K = 2×128) and the
//                        epilogue y = M·X + exp(Acum_i)·C·h_in + D·x, gated
//                        by silu(z).
// Operands are bfloat16 in shared memory, written by the threads (no TMA: the
// Δ-dependent scalings are applied while staging) in the interleaved layout
// the MMA reads without swizzling: 8×8 core matrices of 128 contiguous bytes,
// eight rows of 16 bytes along the tile's contiguous dimension. Accumulators
// are float32 in tensor memory; one elected thread issues every MMA and a
// tcgen05.commit to an mbarrier tells the CTA they are done.
#include "selscan_device.cuh"
#include "tma_util.cuh"

namespace selscan {
namespace {

constexpr int kQ = 128;   // tokens per chunk (= MMA M, one tensor-memory lane per token)
constexpr int kPp = 64;   // head dimension, zero-padded
constexpr int kNp = 128;  // d_state, zero-padded
constexpr int kThr = 128;
constexpr uint64_t kWaitNs = 2000000000ull;  // bounded MMA-completion wait (2 s)
constexpr int kStatusMmaWait = 4;             // device error code: an MMA wait gave up

__device__ const int kNoAbortTc = 0;

typedef __nv_bfloat16 bf16;

// Byte offset of element (r, c) in an interleaved tile with kCols columns:
// core matrix (r/8, c/8) at ((r/8)·(kCols/8) + c/8)·128, row r%8 at 16 bytes.
template <int kCols>
__device__ __forceinline__ uint32_t core_off(int r, int c) {
    return (uint32_t)(((r >> 3) * (kCols >> 3) + (c >> 3)) * 128 + (r & 7) * 16 + (c & 7) * 2);
}

// Shared-memory matrix descriptor, no swizzle: start address, leading byte
// offset (stride between core matrices along K), stride byte offset (along
// M or N), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::f16: bfloat16 A and B, float32 D, shape
// M×N, each operand K-major (0) or M/N-major (1).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        ::"r"(smem_addr(bar))
        : "memory");
}

// Whole-warp tensor-memory allocation of ncols columns (a power of two ≥ 32);
// the base address lands in *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_addr(dst)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive float32 columns of this thread's lane (shape 32x32b: the
// warp reads its own 32 lanes).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// Eight floats as bfloat16 pairs v = hi + lo: hi = bf16(v), lo = bf16(v − hi).
__device__ __forceinline__ void split8(const float (&v)[8], uint4 &hi, uint4 &lo) {
    float r[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = v[e] - __bfloat162float(__float2bfloat16_rn(v[e]));
    hi = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
    lo = make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]), pack_bf16x2(r[4], r[5]),
                    pack_bf16x2(r[6], r[7]));
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        f[2 * k] = __uint_as_float(w[k] << 16);
        f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
}

// Eight consecutive bfloat16 of a row from column c0, zero past ncols; one
// 16-byte load where the row allows it.
__device__ __forceinline__ uint4 ld8(const bf16 *row, int c0, int ncols, bool vec) {
    if (vec && c0 + 8 <= ncols) return __ldg(reinterpret_cast<const uint4 *>(row + c0));
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t lo = c0 + 2 * k < ncols
                                ? (uint32_t)__bfloat16_as_ushort(__ldg(row + c0 + 2 * k)) : 0u;
        const uint32_t hi = c0 + 2 * k + 1 < ncols
                                ? (uint32_t)__bfloat16_as_ushort(__ldg(row + c0 + 2 * k + 1)) : 0u;
        w[k] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void st_smem16(void *base, uint32_t off, const uint4 &v) {
    *reinterpret_cast<uint4 *>(static_cast<char *>(base) + off) = v;
}

// Δ_t for this thread's token t (zero past the sequence end) and the
// inclusive prefix sums of Δ·A over the chunk into acum[].
__device__ __forceinline__ float chunk_delta(const SsdParams &p, long long b, int h,
                                             long long t0, int nq, float *acum, float *wsum) {
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    float d = 0.0f;
    if (t < nq) {
        d = ldg_f32(static_cast<const bf16 *>(p.dt) + (b * p.seqlen + t0 + t) * p.nheads + h) +
            (p.dt_bias ? p.dt_bias[h] : 0.0f);
        if (p.softplus) d = softplus_f32(d);
    }
    float s = d * p.A[h];
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, s, m);
        if (lane >= m) s += o;
    }
    if (lane == 31) wsum[w] = s;
    __syncthreads();
    for (int k = 0; k < w; ++k) s += wsum[k];
    acum[t] = s;
    __syncthreads();
    return d;
}

__device__ __forceinline__ bool wait_mma(uint64_t *bar, uint32_t parity, int *status) {
    if (mbar_wait(bar, parity, &kNoAbortTc, kWaitNs)) return true;
    if (status) atomicCAS(status, 0, kStatusMmaWait);
    return false;
}

// ---- chunk states -----------------------------------------------------------------
struct TcStateSmem {
    bf16 Bt[kQ * kNp];  // rows token j, columns state n
    bf16 Xw[kQ * kPp];  // rows token j, columns channel p: w_j·x, bfloat16 high part
    bf16 Xl[kQ * kPp];  // the low part, w_j·x − high
    float acum[kQ];
    float wsum[4];
    uint64_t bar;
    uint32_t tmem;
};

__global__ void __launch_bounds__(kThr) ssd_tc_state_kernel(const SsdParams p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    TcStateSmem &S = *reinterpret_cast<TcStateSmem *>(smem_raw);
    const int c = blockIdx.x, h = blockIdx.y;
    const long long b = blockIdx.z;
    const long long t0 = (long long)c * kQ;
    const int nq = (int)min((long long)kQ, p.seqlen - t0);
    const int t = threadIdx.x, warp = t >> 5;
    const int N = p.dstate, P = p.headdim;
    const long long D = (long long)p.nheads * P;

    if (warp == 0) tmem_alloc(&S.tmem, 64);
    if (t == 0) {
        mbar_init(&S.bar, 1);
        fence_barrier_init();
    }
    const float d = chunk_delta(p, b, h, t0, nq, S.acum, S.wsum);
    const float aend = S.acum[kQ - 1];
    const float w = __expf(aend - S.acum[t]) * d;  // 0 past the sequence end (Δ = 0)

    // row j = t of B (states) and of w ◦ X (channels)
    {
        const bool live = t < nq;
        const bf16 *brow = static_cast<const bf16 *>(p.B) + (b * p.seqlen + t0 + t) * N;
#pragma unroll 4
        for (int k8 = 0; k8 < kNp / 8; ++k8) {
            const uint4 v = live ? ld8(brow, 8 * k8, N, p.vec_bc) : make_uint4(0, 0, 0, 0);
            st_smem16(S.Bt, core_off<kNp>(t, 8 * k8), v);
        }
        const bf16 *xrow = static_cast<const bf16 *>(p.x) + (b * p.seqlen + t0 + t) * D +
                           (long long)h * P;
#pragma unroll
        for (int k8 = 0; k8 < kPp / 8; ++k8) {
            uint4 hi = make_uint4(0, 0, 0, 0), lo = hi;
            if (live) {
                float f[8];
                unpack8(ld8(xrow, 8 * k8, P, p.vec_x), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] *= w;
                split8(f, hi, lo);
            }
            st_smem16(S.Xw, core_off<kPp>(t, 8 * k8), hi);
            st_smem16(S.Xl, core_off<kPp>(t, 8 * k8), lo);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;

    if (t == 0) {
        // A = Bᵀ: M = state n (contiguous), K = token j  -> M/N-major; core
        // matrices along n 128 bytes apart, along j (kNp/8)·128 bytes apart.
        // B = w ◦ X (high, then low part): N = channel p (contiguous), K =
        // token j -> M/N-major. The pair keeps the chunk state to about 16
        // significant bits: it is carried over the whole sequence.
        const uint32_t a0 = smem_addr(S.Bt), bh = smem_addr(S.Xw), bl = smem_addr(S.Xl);
        constexpr uint32_t kRowB = (kNp / 8) * 128, kRowX = (kPp / 8) * 128;
        constexpr uint32_t id = idesc_bf16(128, kPp, 1, 1);
#pragma unroll
        for (int k = 0; k < kQ / 16; ++k)
            umma_bf16(tmem, umma_desc(a0 + k * 2 * kRowB, kRowB, 128),
                      umma_desc(bh + k * 2 * kRowX, kRowX, 128), id, k > 0);
#pragma unroll
        for (int k = 0; k < kQ / 16; ++k)
            umma_bf16(tmem, umma_desc(a0 + k * 2 * kRowB, kRowB, 128),
                      umma_desc(bl + k * 2 * kRowX, kRowX, 128), id, 1);
        umma_commit(&S.bar);
    }
    const bool ok = __syncthreads_and(wait_mma(&S.bar, 0, p.status));
    tc_fence_after();
    if (ok) {
        // lane t holds state row n = t: S[n][0..63]
        float *dst = p.chunk_state + (((b * p.nheads + h) * p.nchunks + c) * 128 + t) * 64;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32 * half, v);
#pragma unroll
            for (int k = 0; k < 32; k += 4)
                *reinterpret_cast<float4 *>(dst + 32 * half + k) =
                    make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
        }
        if (t == 0) p.chunk_decay[(b * p.nheads + h) * p.nchunks + c] = __expf(aend);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

// ---- chunk outputs ----------------------------------------------------------------
struct TcOutSmem {
    bf16 C[kQ * kNp];   // C (rows token i, columns state n), then M_lo (rows i, columns j)
    bf16 BM[kQ * kNp];  // B (rows token j, columns n), then M_hi (rows i, columns j)
    bf16 HX[kNp * kPp]; // h_in high part (rows state n, columns channel p), then X
                        // (rows token j, columns p)
    bf16 Hl[kNp * kPp]; // h_in low part
    float acum[kQ];
    float dt[kQ];
    float wsum[4];
    uint64_t bar[2];
    uint32_t tmem;
};
static_assert(kQ == kNp, "M reuses the B tile");

// Tensor-memory columns of the accumulators.
constexpr uint32_t kColG = 0, kColYd = 128, kColYo = 192;

template <bool kGate>
__global__ void __launch_bounds__(kThr) ssd_tc_out_kernel(const SsdParams p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    TcOutSmem &S = *reinterpret_cast<TcOutSmem *>(smem_raw);
    const int c = blockIdx.x, h = blockIdx.y;
    const long long b = blockIdx.z;
    const long long t0 = (long long)c * kQ;
    const int nq = (int)min((long long)kQ, p.seqlen - t0);
    const int t = threadIdx.x, warp = t >> 5;
    const int N = p.dstate, P = p.headdim;
    const long long D = (long long)p.nheads * P;

    if (warp == 0) tmem_alloc(&S.tmem, 256);
    if (t == 0) {
        mbar_init(&S.bar[0], 1);
        mbar_init(&S.bar[1], 1);
        fence_barrier_init();
    }
    S.dt[t] = chunk_delta(p, b, h, t0, nq, S.acum, S.wsum);

    {
        const bool live = t < nq;
        const long long row = b * p.seqlen + t0 + t;
        const bf16 *crow = static_cast<const bf16 *>(p.C) + row * N;
        const bf16 *brow = static_cast<const bf16 *>(p.B) + row * N;
#pragma unroll 4
        for (int k8 = 0; k8 < kNp / 8; ++k8) {
            const uint4 z4 = make_uint4(0, 0, 0, 0);
            st_smem16(S.C, core_off<kNp>(t, 8 * k8), live ? ld8(crow, 8 * k8, N, p.vec_bc) : z4);
            st_smem16(S.BM, core_off<kNp>(t, 8 * k8), live ? ld8(brow, 8 * k8, N, p.vec_bc) : z4);
        }
        // h_in row n = t (float32, zero for n ≥ d_state and p ≥ headdim) as a
        // bfloat16 pair: the carried state can dominate y early in a chunk
        const float *hrow = p.state_in + (((b * p.nheads + h) * p.nchunks + c) * 128 + t) * 64;
#pragma unroll
        for (int k8 = 0; k8 < kPp / 8; ++k8) {
            const float4 u = __ldg(reinterpret_cast<const float4 *>(hrow + 8 * k8));
            const float4 v = __ldg(reinterpret_cast<const float4 *>(hrow + 8 * k8 + 4));
            const float f[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
            uint4 hi, lo;
            split8(f, hi, lo);
            st_smem16(S.HX, core_off<kPp>(t, 8 * k8), hi);
            st_smem16(S.Hl, core_off<kPp>(t, 8 * k8), lo);
        }
    }
    // x row j = t, held in registers until h_in's tile is free
    uint4 xr[kPp / 8];
    {
        const bf16 *xrow = static_cast<const bf16 *>(p.x) + (b * p.seqlen + t0 + t) * D +
                           (long long)h * P;
#pragma unroll
        for (int k8 = 0; k8 < kPp / 8; ++k8)
            xr[k8] = t < nq ? ld8(xrow, 8 * k8, P, p.vec_x) : make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;
    const int ksteps_n = (N + 15) / 16;  // K = d_state in steps of 16 (zero-padded)
    constexpr uint32_t kRowN = (kNp / 8) * 128, kRowP = (kPp / 8) * 128;

    if (t == 0) {
        // G = C·Bᵀ: A = C (M = token i, K = n, K-major), B = B (N = token j, K = n, K-major)
        // C·h_in:  A = C, B = h_in (N = channel p contiguous, K = n: M/N-major)
        const uint32_t c0 = smem_addr(S.C), b0 = smem_addr(S.BM);
        const uint32_t hh = smem_addr(S.HX), hl = smem_addr(S.Hl);
        for (int k = 0; k < ksteps_n; ++k) {
            const uint64_t a = umma_desc(c0 + k * 256, 128, kRowN);
            umma_bf16(tmem + kColG, a, umma_desc(b0 + k * 256, 128, kRowN),
                      idesc_bf16(128, 128, 0, 0), k > 0);
            umma_bf16(tmem + kColYo, a, umma_desc(hh + k * 2 * kRowP, kRowP, 128),
                      idesc_bf16(128, kPp, 0, 1), k > 0);
            umma_bf16(tmem + kColYo, a, umma_desc(hl + k * 2 * kRowP, kRowP, 128),
                      idesc_bf16(128, kPp, 0, 1), 1);
        }
        umma_commit(&S.bar[0]);
    }
    bool ok = __syncthreads_and(wait_mma(&S.bar[0], 0, p.status));
    tc_fence_after();

    // M row i = t from G row i: (C_i·B_j)·exp(Acum_i − Acum_j)·Δ_j for j ≤ i,
    // stored as two bfloat16 parts M = M_hi + M_lo (M_hi into the B tile, M_lo
    // into the C tile: both are free once the first MMAs are done). Single
    // products M_ij·x_j can be far larger than y_i, so one bfloat16 rounding
    // of M would cost more than the output's own rounding; the pair keeps
    // about 16 significant bits.
    if (ok) {
        const float ai = S.acum[t];
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
        for (int cb = 0; cb < kQ / 32; ++cb) {
            float g[32];
            tmem_ld32(lane_base + kColG + 32 * cb, g);
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
                float m[8], r[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = 32 * cb + 8 * k8 + e;
                    m[e] = (j <= t && t < nq) ? g[8 * k8 + e] * __expf(ai - S.acum[j]) * S.dt[j]
                                              : 0.0f;
                    r[e] = m[e] - __bfloat162float(__float2bfloat16_rn(m[e]));
                }
                const uint32_t off = core_off<kQ>(t, 32 * cb + 8 * k8);
                st_smem16(S.BM, off,
                          make_uint4(pack_bf16x2(m[0], m[1]), pack_bf16x2(m[2], m[3]),
                                     pack_bf16x2(m[4], m[5]), pack_bf16x2(m[6], m[7])));
                st_smem16(S.C, off,
                          make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]),
                                     pack_bf16x2(r[4], r[5]), pack_bf16x2(r[6], r[7])));
            }
        }
    }
    // X row j = t into the h_in tile (its MMAs are done)
#pragma unroll
    for (int k8 = 0; k8 < kPp / 8; ++k8) st_smem16(S.HX, core_off<kPp>(t, 8 * k8), xr[k8]);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t == 0 && ok) {
        // M·X = M_hi·X + M_lo·X: A = M part (M = token i, K = token j,
        // K-major), B = X (N = channel p, K = j: M/N-major)
        const uint32_t mh = smem_addr(S.BM), ml = smem_addr(S.C), x0 = smem_addr(S.HX);
#pragma unroll
        for (int k = 0; k < kQ / 16; ++k)
            umma_bf16(tmem + kColYd, umma_desc(mh + k * 256, 128, kRowN),
                      umma_desc(x0 + k * 2 * kRowP, kRowP, 128), idesc_bf16(128, kPp, 0, 1),
                      k > 0);
#pragma unroll
        for (int k = 0; k < kQ / 16; ++k)
            umma_bf16(tmem + kColYd, umma_desc(ml + k * 256, 128, kRowN),
                      umma_desc(x0 + k * 2 * kRowP, kRowP, 128), idesc_bf16(128, kPp, 0, 1), 1);
        umma_commit(&S.bar[1]);
    }
    ok = __syncthreads_and(ok && wait_mma(&S.bar[1], 0, p.status));
    tc_fence_after();

    // every lane loads its accumulator rows (tcgen05.ld is warp-wide); rows
    // past the sequence end store nothing
    if (ok) {
        const bool live = t < nq;
        const long long row = b * p.seqlen + t0 + t;
        const bf16 *xrow = static_cast<const bf16 *>(p.x) + row * D + (long long)h * P;
        const bf16 *zrow = kGate ? static_cast<const bf16 *>(p.z) + row * D + (long long)h * P
                                 : nullptr;
        bf16 *yrow = static_cast<bf16 *>(p.y) + row * D + (long long)h * P;
        const float dec = __expf(S.acum[t]);
        const float dsk = p.Dskip ? p.Dskip[h] : 0.0f;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            if (32 * half >= P) break;
            float yd[32], yo[32];
            tmem_ld32(lane_base + kColYd + 32 * half, yd);
            tmem_ld32(lane_base + kColYo + 32 * half, yo);
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
                const int c0 = 32 * half + 8 * k8;
                if (c0 >= P) break;
                float xv[8] = {}, zv[8] = {}, o[8];
                if (live) {
                    unpack8(ld8(xrow, c0, P, p.vec_x), xv);
                    if (kGate) unpack8(ld8(zrow, c0, P, p.vec_x), zv);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float v = fmaf(dec, yo[8 * k8 + e], yd[8 * k8 + e]) + dsk * xv[e];
                    if (kGate) v *= silu_f32(zv[e]);
                    o[e] = v;
                }
                if (!live) continue;
                if (p.vec_x && c0 + 8 <= P) {
                    *reinterpret_cast<uint4 *>(yrow + c0) =
                        make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                   pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (c0 + e < P) yrow[c0 + e] = __float2bfloat16_rn(o[e]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

bool ssd_tc_supported(int headdim, int dstate) {
    return headdim >= 1 && headdim <= kPp && dstate >= 1 && dstate <= kNp;
}

int ssd_tc_chunk_tokens() { return kQ; }

cudaError_t launch_ssd_tc_state(const SsdParams &p, cudaStream_t stream) {
    static bool configured[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = set_smem(ssd_tc_state_kernel, sizeof(TcStateSmem));
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const dim3 grid((unsigned)p.nchunks, (unsigned)p.nheads, (unsigned)p.batch);
    ssd_tc_state_kernel<<<grid, kThr, sizeof(TcStateSmem), stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_ssd_tc_out(const SsdParams &p, cudaStream_t stream) {
    static bool configured[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = set_smem(ssd_tc_out_kernel<true>, sizeof(TcOutSmem));
        if (e == cudaSuccess) e = set_smem(ssd_tc_out_kernel<false>, sizeof(TcOutSmem));
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const dim3 grid((unsigned)p.nchunks, (unsigned)p.nheads, (unsigned)p.batch);
    if (p.z)
        ssd_tc_out_kernel<true><<<grid, kThr, sizeof(TcOutSmem), stream>>>(p);
    else
        ssd_tc_out_kernel<false><<<grid, kThr, sizeof(TcOutSmem), stream>>>(p);
    return cudaGetLastError();
}

}  // namespace selscan
