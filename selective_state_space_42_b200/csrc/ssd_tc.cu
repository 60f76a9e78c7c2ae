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
// h_c = exp(Acum_end,c)·h_{c−1} + S_c. Three kernels:
//   ssd_tc_state_kernel  S for one (chunk, group of heads, batch row): B staged
//                        once, per head MMAs of M=128 (state n) × N=64 (head
//                        channel p) × K=2×128 (token; w ◦ X as a bfloat16
//                        high/low pair)
//   ssd_tc_carry_kernel  the element-wise carry over chunks, writing each h_in
//                        in the output kernel's operand layout
//   ssd_tc_out_kernel    G = C·Bᵀ (128×128, K = d_state) and C·h_in (128×64) on
//                        the tensor cores (h_in as a bfloat16 high/low pair),
//                        M built from G by the 256 threads (token row i =
//                        tensor-memory lane i, two threads per row) and
//                        written back to shared memory as a bfloat16 pair
//                        M_hi + M_lo, then M·X (128×64, K = 2×128) and the
//                        epilogue y = M·X + exp(Acum_i)·C·h_in + D·x, gated
//                        by silu(z).
// Operands are bfloat16 in shared memory: B and C by TMA into 128-byte
// swizzled slabs (or, where the rows do not allow TMA, by cp.async), h_in by
// one bulk copy, and the operands that carry a Δ-dependent scaling written
// by the threads; the last three in the interleaved layout the MMA reads
// without swizzling (8×8 core matrices of 128 contiguous bytes, eight rows
// of 16 bytes along the tile's contiguous dimension). Accumulators are
// float32 in tensor memory; one elected thread issues every MMA and a
// tcgen05.commit to an mbarrier tells the CTA they are done.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "ssd_params.cuh"
#include "tma_util.cuh"

#include <algorithm>
#include <cstddef>

namespace selscan {
namespace {

constexpr int kQ = 128;   // tokens per chunk (= MMA M, one tensor-memory lane per token)
constexpr int kPp = 64;   // head dimension, zero-padded
constexpr int kNp = 128;  // d_state, zero-padded
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

// The same for the 128-byte swizzled layout (layout type 2): 8-row atoms of
// 128-byte rows whose 16-byte chunks are permuted by the row index, as a
// 128B-swizzled TMA load writes them. K-major: the start advances by 32
// bytes per K step of 16 inside a 64-column slab; the stride byte offset is
// the distance between 8-row atoms (1024 bytes). M/N-major: leading byte
// offset = distance between 64-element slabs, stride byte offset = between
// 8-row atoms along K.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return umma_desc(saddr, lbo, sbo) | (2ull << 61);
}

// 3-D tiled TMA load (coordinates innermost first) completing on an mbarrier.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// The B or C tile of a chunk by TMA: two 64-column slabs of 128 token rows,
// 128-byte swizzled; rows past the sequence and columns past d_state (the
// whole second slab when d_state ≤ 64) are zero-filled by the copy.
constexpr uint32_t kBcTileBytes = 2u * kQ * 64 * 2;
__device__ __forceinline__ void tma_bc_tile(bf16 *tile, const CUtensorMap *map, uint64_t *bar,
                                            int t0, int b) {
    tma_load_3d(tile, map, bar, 0, t0, b);
    tma_load_3d(tile + kQ * 64, map, bar, 64, t0, b);
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

// Eight floats as bfloat16 pairs v = hi + lo: hi is v with its low 16 bits
// cleared (bfloat16 truncation, integer operations only) and lo = bf16(v − hi)
// rounded to nearest (v − hi is exact in float32), so |v − hi − lo| ≤
// 2⁻⁹·|v − hi| < 2⁻¹⁶·|v| without bias. One packed conversion per two
// elements: the conversions share the MUFU's issue rate.
__device__ __forceinline__ void split8(const float (&v)[8], uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t a = __float_as_uint(v[2 * k]) & 0xFFFF0000u;
        const uint32_t b = __float_as_uint(v[2 * k + 1]) & 0xFFFF0000u;
        h[k] = (a >> 16) | b;
        l[k] = pack_bf16x2(v[2 * k] - __uint_as_float(a), v[2 * k + 1] - __uint_as_float(b));
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
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

// 16-byte asynchronous global -> shared copy; src_bytes 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Contiguous global -> shared bulk copy (16-byte aligned, size a multiple of
// 16) completing on an mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Contiguous shared -> global bulk copy (16-byte aligned, size a multiple of
// 16) in this thread's bulk group.
__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(dst), "r"(smem_addr(src)), "r"(bytes)
                 : "memory");
}

constexpr int kThrTc = 256;  // threads of the two MMA kernels

// Work item k of this thread in a cooperative pass over a kQ-row tile with
// kCols columns: lane l of warp w takes row 8·g + l mod 8 and 8-column chunk
// 4·c + l / 8 of item (g, c) = w + 8·k, so that one warp instruction touches
// 8 row segments of 64 contiguous bytes in global memory and 4 whole core
// matrices (512 contiguous bytes) of the tile.
template <int kCols>
__device__ __forceinline__ void tile_item(int k, int &row, int &chunk) {
    constexpr int kQuads = kCols / 32;
    const int it = (int)(threadIdx.x >> 5) + (kThrTc / 32) * k;
    row = 8 * (it / kQuads) + (int)(threadIdx.x & 7);
    chunk = 4 * (it % kQuads) + (int)((threadIdx.x & 31) >> 3);
}
template <int kCols> constexpr int tile_items() { return (kQ / 8) * (kCols / 32) / (kThrTc / 32); }

// The whole tile from global rows base + row·stride (ncols valid bfloat16
// columns; rows ≥ nrows and columns ≥ ncols zero): asynchronous 16-byte
// copies where the rows allow them (vec: 16-byte aligned rows, ncols a
// multiple of 8), else loads and stores through registers. All threads.
template <int kCols>
__device__ __forceinline__ void stage_tile(bf16 *tile, const bf16 *base, long long stride,
                                           int nrows, int ncols, bool vec) {
    const uint32_t sbase = smem_addr(tile);
#pragma unroll
    for (int k = 0; k < tile_items<kCols>(); ++k) {
        int row, chunk;
        tile_item<kCols>(k, row, chunk);
        const bool in = row < nrows && 8 * chunk < ncols;
        const uint32_t off = core_off<kCols>(row, 8 * chunk);
        if (vec)
            cp_async16(sbase + off, in ? base + row * stride + 8 * chunk : base, in ? 16u : 0u);
        else
            st_smem16(tile, off, in ? ld8(base + row * stride, 8 * chunk, ncols, false)
                                    : make_uint4(0, 0, 0, 0));
    }
}

// This thread's items of such a tile into registers (zero outside).
template <int kCols>
__device__ __forceinline__ void load_tile_regs(uint4 (&v)[tile_items<kCols>()], const bf16 *base,
                                               long long stride, int nrows, int ncols, bool vec) {
#pragma unroll
    for (int k = 0; k < tile_items<kCols>(); ++k) {
        int row, chunk;
        tile_item<kCols>(k, row, chunk);
        v[k] = row < nrows ? ld8(base + row * stride, 8 * chunk, ncols, vec)
                           : make_uint4(0, 0, 0, 0);
    }
}

// dt + dt_bias of this thread's token (threads 0..kQ−1 of a chunk with nq
// tokens; 0 otherwise): issued early, consumed by chunk_delta.
__device__ __forceinline__ float chunk_dt_raw(const SsdParams &p, long long b, int h, long long t0,
                                              int nq) {
    const int t = threadIdx.x;
    if (t >= kQ || t >= nq) return 0.0f;
    return ldg_f32(static_cast<const bf16 *>(p.dt) + (b * p.seqlen + t0 + t) * p.nheads + h) +
           (p.dt_bias ? p.dt_bias[h] : 0.0f);
}

// Δ_t of the chunk's tokens t (zero past the sequence end; from chunk_dt_raw)
// into dt[], and the inclusive prefix sums of Δ·A over the chunk, times
// log2(e), into acum2[] (so exp(Acum_i − Acum_j) = 2^(acum2_i − acum2_j)).
// With F given, also F[t] = 2^(−acum2_t)·Δ_t and the per-warp maxima of
// |acum2| in wmax[4]. Threads 0..kQ−1 compute; every thread of the block
// takes part in the two barriers.
__device__ __forceinline__ void chunk_delta(const SsdParams &p, int h, int nq, float raw, float *dt,
                                            float *acum2, float *wsum, float *F = nullptr,
                                            float *wmax = nullptr) {
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    float d = 0.0f, s = 0.0f;
    if (t < kQ) {
        if (t < nq) d = p.softplus ? softplus_f32(raw) : raw;
        s = d * p.A[h] * kLog2e;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const float o = __shfl_up_sync(0xffffffffu, s, m);
            if (lane >= m) s += o;
        }
        if (lane == 31) wsum[w] = s;
    }
    __syncthreads();
    if (t < kQ) {
        for (int k = 0; k < w; ++k) s += wsum[k];
        acum2[t] = s;
        dt[t] = d;
        if (F) {
            F[t] = ex2_approx(-s) * d;  // used only when every |acum2| ≤ kFactorMax
            float m = fabsf(s);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) wmax[w] = m;
        }
    }
    __syncthreads();
}

// Largest |acum2| of a chunk for which 2^(acum2_i − acum2_j) may be taken as
// 2^acum2_i · 2^(−acum2_j): both factors stay normal float32 numbers and
// 2^(−acum2_j)·Δ_j stays finite for Δ_j < 2^27.
constexpr float kFactorMax = 100.0f;

__device__ __forceinline__ bool wait_mma(uint64_t *bar, uint32_t parity, int *status) {
    if (mbar_wait(bar, parity, &kNoAbortTc, kWaitNs)) return true;
    if (status) atomicCAS(status, 0, kStatusMmaWait);
    return false;
}

// ---- chunk states -----------------------------------------------------------------
// One CTA per (chunk, group of heads, batch row): B is staged once and used by
// every head of the group; per head the w ◦ x operand pair and the
// accumulator alternate between two buffers, so that the MMAs of head k run
// while head k − 1's result is stored and head k + 1's x is in flight.
// 256 threads; in the epilogue thread t reads state row n = t mod 128
// (tensor-memory lane n), column half t / 128, into the operand pair its
// head no longer needs (rows 0..63 over the high part, 64..127 over the low
// part), and one thread sends the 32 KB to global memory by two bulk copies.
// The chunk state is stored in 16-byte units swizzled within each row: the
// channels 4u .. 4u + 3 of state n sit at unit u ^ (n mod 8) of the row, so
// that the 32 rows a warp stages at once spread over all banks.

struct TcStateSmem {
    bf16 Bt[kQ * kNp];     // rows token j, columns state n
    bf16 Xw[2][kQ * kPp];  // rows token j, columns channel p: w_j·x, bfloat16 high part
    bf16 Xl[2][kQ * kPp];  // the low part, w_j·x − high
    float acum2[kQ];
    float dt[kQ];
    float wsum[4];
    uint64_t bar[2];
    uint64_t bar_b;       // the B tile's TMA
    uint32_t tmem;
};

__global__ void __launch_bounds__(kThrTc)
ssd_tc_state_kernel(const SsdParams p, const __grid_constant__ CUtensorMap tm_b) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    // 1024-byte aligned: the 128-byte swizzle pattern is taken from address bits 7..9
    TcStateSmem &S = *reinterpret_cast<TcStateSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int c = blockIdx.x;
    const int h_first = blockIdx.y * p.heads_per_cta;
    const int nh = min(p.heads_per_cta, p.nheads - h_first);
    const long long b = blockIdx.z;
    const long long t0 = (long long)c * kQ;
    const int nq = (int)min((long long)kQ, p.seqlen - t0);
    const int t = threadIdx.x, warp = t >> 5, r = t & (kQ - 1), hh = t / kQ;
    const int N = p.dstate, P = p.headdim;
    const long long D = (long long)p.nheads * P;

    if (warp == 0) tmem_alloc(&S.tmem, 128);
    if (t == 0) {
        mbar_init(&S.bar[0], 1);
        mbar_init(&S.bar[1], 1);
        mbar_init(&S.bar_b, 1);
        fence_barrier_init();
        if (p.tma_bc) {  // the chunk's B rows by TMA (128-byte swizzled slabs)
            mbar_arrive_expect_tx(&S.bar_b, kBcTileBytes);
            tma_bc_tile(S.Bt, &tm_b, &S.bar_b, (int)t0, (int)b);
        }
    }
    // else the chunk's B rows by asynchronous copies (interleaved layout);
    // the first head's x rows into registers
    const long long row0 = b * p.seqlen + t0;
    if (!p.tma_bc) {
        stage_tile<kNp>(S.Bt, static_cast<const bf16 *>(p.B) + row0 * N, N, nq, N, p.vec_bc);
        cp_async_commit();
    }
    const bf16 *xbase = static_cast<const bf16 *>(p.x) + row0 * D;
    uint4 xr[tile_items<kPp>()];
    load_tile_regs<kPp>(xr, xbase + (long long)h_first * P, D, nq, P, p.vec_x);
    float dt_raw = chunk_dt_raw(p, b, h_first, t0, nq);
    uint32_t tmem = 0;
    bool ok = true;
    float aend_prev = 0.0f;  // Acum_end·log2(e) of the previous head
    constexpr uint32_t kRowB = (kNp / 8) * 128, kRowX = (kPp / 8) * 128;

    for (int k = 0; k <= nh; ++k) {
        float aend2 = 0.0f;
        // the operand pair written below was sent out as head k − 2's state:
        // its copy must have read it (the barriers in chunk_delta publish this)
        if (t == 0 && k >= 2) bulk_wait_read<0>();
        if (k < nh) {
            const int h = h_first + k;
            chunk_delta(p, h, nq, dt_raw, S.dt, S.acum2, S.wsum);
            aend2 = S.acum2[kQ - 1];
            // w_j ◦ x_j as a bfloat16 pair (0 past the sequence end: Δ = 0)
            bf16 *xw = S.Xw[k & 1], *xl = S.Xl[k & 1];
#pragma unroll
            for (int i = 0; i < tile_items<kPp>(); ++i) {
                int j, chunk;
                tile_item<kPp>(i, j, chunk);
                const float w = ex2_approx(aend2 - S.acum2[j]) * S.dt[j];
                float f[8];
                unpack8(xr[i], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] *= w;
                uint4 hi, lo;
                split8(f, hi, lo);
                const uint32_t off = core_off<kPp>(j, 8 * chunk);
                st_smem16(xw, off, hi);
                st_smem16(xl, off, lo);
            }
            if (k + 1 < nh) {  // the next head's x and dt, in flight from here
                load_tile_regs<kPp>(xr, xbase + (long long)(h + 1) * P, D, nq, P, p.vec_x);
                dt_raw = chunk_dt_raw(p, b, h + 1, t0, nq);
            }
            if (k == 0 && !p.tma_bc) cp_async_wait_all();
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (k == 0) tmem = S.tmem;
            if (t == 0 && k == 0 && p.tma_bc) {
                ok = wait_mma(&S.bar_b, 0, p.status);  // B landed
                tc_fence_after();
            }
            if (t == 0 && ok) {
                // A = Bᵀ: M = state n (contiguous), K = token j -> M/N-major.
                // TMA tile: 64-state slabs 16 KB apart, 8-token atoms 1024
                // bytes apart; interleaved tile: core matrices along n 128
                // bytes apart, along j (kNp/8)·128 bytes apart.
                // B = w ◦ X (high, then low part): N = channel p (contiguous),
                // K = token j -> M/N-major. The pair keeps the chunk state to
                // about 16 significant bits: it is carried over the whole
                // sequence.
                const uint32_t a0 = smem_addr(S.Bt), bh = smem_addr(xw), bl = smem_addr(xl);
                const uint32_t d = tmem + 64u * (uint32_t)(k & 1);
                constexpr uint32_t id = idesc_bf16(128, kPp, 1, 1);
                auto adesc = [&](int q) {
                    return p.tma_bc ? umma_desc_sw128(a0 + q * 2048, kQ * 64 * 2, 1024)
                                    : umma_desc(a0 + q * 2 * kRowB, kRowB, 128);
                };
#pragma unroll
                for (int q = 0; q < kQ / 16; ++q)
                    umma_bf16(d, adesc(q), umma_desc(bh + q * 2 * kRowX, kRowX, 128), id, q > 0);
#pragma unroll
                for (int q = 0; q < kQ / 16; ++q)
                    umma_bf16(d, adesc(q), umma_desc(bl + q * 2 * kRowX, kRowX, 128), id, 1);
                umma_commit(&S.bar[k & 1]);
            }
        }
        if (k > 0) {  // the previous head's state, while this head's MMAs run
            const int kk = k - 1, h = h_first + kk;
            ok = __syncthreads_and(ok && wait_mma(&S.bar[kk & 1], (kk >> 1) & 1, p.status));
            tc_fence_after();
            if (ok) {
                // lane r holds state row n = r: this thread stages S[n][32·hh .. 32·hh + 31]
                float v[32];
                tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + 64u * (uint32_t)(kk & 1) +
                              32 * hh,
                          v);
                float4 *row = reinterpret_cast<float4 *>(r < 64 ? S.Xw[kk & 1] : S.Xl[kk & 1]) +
                              (r & 63) * 16;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    row[(8 * hh + i) ^ (r & 7)] =
                        make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                if (t == 0)
                    p.chunk_decay[(b * p.nheads + h) * p.nchunks + c] = ex2_approx(aend_prev);
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncthreads();
            if (t == 0 && ok) {
                char *dst = reinterpret_cast<char *>(
                    p.chunk_state + ((b * p.nheads + h) * p.nchunks + c) * 128ll * 64);
                bulk_store(dst, S.Xw[kk & 1], 16384);
                bulk_store(dst + 16384, S.Xl[kk & 1], 16384);
                bulk_commit();
            }
        }
        aend_prev = aend2;
    }
    if (t == 0) bulk_wait<0>();  // the last states are out before the CTA ends
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// ---- states entering the chunks ----------------------------------------------------
// h_in for every chunk, h_c = exp(Acum_end,c)·h_{c−1} + S_c from h_{−1} = h0
// (or zero), written per chunk as the bfloat16 pair (high, low) in the
// interleaved operand layout the output kernel's MMA reads: one 32 KB block
// per (batch row, head, chunk) = high tile [state n][channel p] then low
// tile. One CTA per (batch row, head, slab of 16 states): the slab of every
// chunk state (16 × 64 float32 = 4 KB, contiguous) streams through a ring of
// kCarryStages bulk copies, so that many chunks' loads are in flight without
// holding registers; thread t carries state n0 + t/16, channels 4·(t mod 16)
// to + 3, across the chunks.
constexpr int kCarryRows = 16, kCarryStages = 8, kCarryThreads = 256;
constexpr uint32_t kCarrySlab = kCarryRows * kPp * 4;
struct CarrySmem {
    float4 slab[kCarryStages][kCarryThreads];
    float dec[kCarryThreads];  // the decays of the next kCarryThreads chunks
    uint64_t full[kCarryStages];
};

__global__ void __launch_bounds__(kCarryThreads) ssd_tc_carry_kernel(const SsdParams p) {
    __shared__ __align__(128) CarrySmem S;
    constexpr int kSlabs = kNp / kCarryRows;
    const long long bh = blockIdx.x / kSlabs;
    const int n0 = (int)(blockIdx.x % kSlabs) * kCarryRows;
    const int t = threadIdx.x, n = n0 + t / 16, p0 = 4 * (t % 16);
    const long long b = bh / p.nheads;
    const int h = (int)(bh % p.nheads);
    const int N = p.dstate, P = p.headdim, nc = p.nchunks;
    const char *src0 = reinterpret_cast<const char *>(p.chunk_state) +
                       ((bh * nc * kNp + n0) * kPp) * 4ll;
    const long long chunk_bytes = (long long)kNp * kPp * 4;
    const int first = min(nc, kCarryStages);
    if (t == 0) {
        for (int s = 0; s < kCarryStages; ++s) mbar_init(&S.full[s], 1);
        fence_barrier_init();
        for (int c = 0; c < first; ++c) {
            mbar_arrive_expect_tx(&S.full[c], kCarrySlab);
            bulk_load(&S.slab[c][0], src0 + c * chunk_bytes, kCarrySlab, &S.full[c]);
        }
    }
    float st[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int pp = p0 + k;
        st[k] = (p.h0 && n < N && pp < P)
                    ? p.h0[((b * p.nheads + h) * (long long)P + pp) * N + n] : 0.0f;
    }
    __syncthreads();  // barriers initialised
    const uint32_t off = core_off<kPp>(n, p0);
    char *blk0 = reinterpret_cast<char *>(p.state_in) + bh * nc * 32768ll;
    const float *dec0 = p.chunk_decay + bh * nc;
    int c = 0;
    bool ok = true;
    for (; c < nc; ++c) {
        const int s = c % kCarryStages;
        if (c % kCarryThreads == 0) {  // one load per thread brings the next block of decays
            __syncthreads();
            S.dec[t] = c + t < nc ? dec0[c + t] : 0.0f;
            __syncthreads();
        }
        const float d = S.dec[c % kCarryThreads];
        const bool got = mbar_wait(&S.full[s], (uint32_t)(c / kCarryStages) & 1, &kNoAbortTc,
                                   kWaitNs);
        float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
        if (got) u = S.slab[s][(t & ~15) | ((t & 15) ^ (n & 7))];  // the rows' 16-byte swizzle
        // h_in of chunk c, then the state after it
        float v8[8] = {st[0], st[1], st[2], st[3], 0.f, 0.f, 0.f, 0.f};
        uint4 hi, lo;
        split8(v8, hi, lo);
        char *blk = blk0 + (long long)c * 32768;
        *reinterpret_cast<uint2 *>(blk + off) = make_uint2(hi.x, hi.y);
        *reinterpret_cast<uint2 *>(blk + 16384 + off) = make_uint2(lo.x, lo.y);
        st[0] = fmaf(d, st[0], u.x);
        st[1] = fmaf(d, st[1], u.y);
        st[2] = fmaf(d, st[2], u.z);
        st[3] = fmaf(d, st[3], u.w);
        // every thread has read stage s: refill it with chunk c + kCarryStages
        ok = __syncthreads_and(got) != 0;
        if (!ok) break;
        if (t == 0 && c + kCarryStages < nc) {
            mbar_arrive_expect_tx(&S.full[s], kCarrySlab);
            bulk_load(&S.slab[s][0], src0 + (c + kCarryStages) * chunk_bytes, kCarrySlab,
                      &S.full[s]);
        }
    }
    if (!ok) {
        // a wait gave up: record it, then let the copies still in flight into
        // this CTA's ring land (bounded) before the CTA exits
        if (t == 0) {
            if (p.status) atomicCAS(p.status, 0, kStatusMmaWait);
            for (int k = c; k < min(nc, c + kCarryStages); ++k)
                mbar_wait(&S.full[k % kCarryStages], (uint32_t)(k / kCarryStages) & 1,
                          &kNoAbortTc, kWaitNs);
        }
        __syncthreads();
        return;
    }
    if (p.final_state && n < N) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int pp = p0 + k;
            if (pp < P) p.final_state[((b * p.nheads + h) * (long long)P + pp) * N + n] = st[k];
        }
    }
}

// ---- chunk outputs ----------------------------------------------------------------
struct TcOutSmem {
    bf16 C[kQ * kNp];   // C (rows token i, columns state n), then M_lo (rows i, columns j)
    bf16 BM[kQ * kNp];  // B (rows token j, columns n), then M_hi (rows i, columns j)
    bf16 HX[kNp * kPp]; // h_in high part (rows state n, columns channel p), then X
                        // (rows token j, columns p)
    bf16 Hl[kNp * kPp]; // h_in low part, then z (rows token i, columns p)
    float acum2[kQ];
    float dt[kQ];
    float F[kQ];        // 2^(−acum2_j)·Δ_j
    float wsum[4];
    float wmax[4];
    uint64_t bar[4];    // first MMAs, second MMAs, h_in bulk copy, B and C TMA
    uint32_t tmem;
};
static_assert(kQ == kNp, "M reuses the B tile");
static_assert(offsetof(TcOutSmem, Hl) == offsetof(TcOutSmem, HX) + 2 * kNp * kPp,
              "h_in's two tiles are one contiguous copy");

// Tensor-memory columns of the accumulators.
constexpr uint32_t kColG = 0, kColYd = 128, kColYo = 192;

// 256 threads: thread t works on token row r = t mod 128 (tensor-memory lane
// r) and column half hh = t / 128 of every tile, of M and of y.
template <bool kGate>
__global__ void __launch_bounds__(kThrTc)
ssd_tc_out_kernel(const SsdParams p, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_c) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    // 1024-byte aligned: the 128-byte swizzle pattern is taken from address bits 7..9
    TcOutSmem &S = *reinterpret_cast<TcOutSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int c = blockIdx.x, h = blockIdx.y;
    const long long b = blockIdx.z;
    const long long t0 = (long long)c * kQ;
    const int nq = (int)min((long long)kQ, p.seqlen - t0);
    const int t = threadIdx.x, warp = t >> 5, r = t & (kQ - 1), hh = t / kQ;
    const int N = p.dstate, P = p.headdim;
    const long long D = (long long)p.nheads * P;
    const bool live = r < nq;
    const long long row = b * p.seqlen + t0 + r;
    const long long bh = b * p.nheads + h;
    const uint32_t lane_q = (uint32_t)((warp & 3) * 32) << 16;  // this warp's 32 lanes

    if (warp == 0) tmem_alloc(&S.tmem, 256);
    if (t == 0) {
        mbar_init(&S.bar[0], 1);
        mbar_init(&S.bar[1], 1);
        mbar_init(&S.bar[2], 1);
        mbar_init(&S.bar[3], 1);
        fence_barrier_init();
        if (p.tma_bc) {  // the chunk's C and B rows by TMA (128-byte swizzled slabs)
            mbar_arrive_expect_tx(&S.bar[3], 2 * kBcTileBytes);
            tma_bc_tile(S.C, &tm_c, &S.bar[3], (int)t0, (int)b);
            tma_bc_tile(S.BM, &tm_b, &S.bar[3], (int)t0, (int)b);
        }
        // h_in's (high, low) block for this chunk, already in operand layout
        mbar_arrive_expect_tx(&S.bar[2], 32768);
        bulk_load(S.HX, reinterpret_cast<const char *>(p.state_in) + (bh * p.nchunks + c) * 32768ll,
                  32768, &S.bar[2]);
    }
    // the chunk's C and B rows (asynchronous copies) and x rows (into
    // registers, until h_in's tile is free)
    const long long row0 = b * p.seqlen + t0;
    if (!p.tma_bc) {
        stage_tile<kNp>(S.C, static_cast<const bf16 *>(p.C) + row0 * N, N, nq, N, p.vec_bc);
        stage_tile<kNp>(S.BM, static_cast<const bf16 *>(p.B) + row0 * N, N, nq, N, p.vec_bc);
        cp_async_commit();
    }
    uint4 xr[tile_items<kPp>()];
    load_tile_regs<kPp>(xr, static_cast<const bf16 *>(p.x) + row0 * D + (long long)h * P, D, nq,
                        P, p.vec_x);
    const float dt_raw = chunk_dt_raw(p, b, h, t0, nq);
    if (!p.tma_bc) cp_async_wait_all();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;
    const int ksteps_n = (N + 15) / 16;  // K = d_state in steps of 16 (zero-padded)
    constexpr uint32_t kRowN = (kNp / 8) * 128, kRowP = (kPp / 8) * 128;
    const uint32_t c0 = smem_addr(S.C), b0 = smem_addr(S.BM);
    // K-major operand descriptors of the C and B tiles for K step k (16
    // states): 128-byte swizzled TMA slabs (32 bytes per step inside a
    // 64-column slab of 16 KB, 8-row atoms 1024 bytes apart), or the
    // interleaved layout (core matrices 128 bytes apart along K, 8-row
    // groups (kNp/8)·128 bytes apart)
    auto kdesc = [&](uint32_t base, int k) {
        return p.tma_bc ? umma_desc_sw128(base + (k >> 2) * (kQ * 64 * 2) + (k & 3) * 32, 16, 1024)
                        : umma_desc(base + k * 256, 128, kRowN);
    };

    // G = C·Bᵀ as soon as B and C are in: A = C (M = token i, K = n,
    // K-major), B = B (N = token j, K = n, K-major); the Δ prefix sums below
    // run while it executes
    bool ok = true;
    if (t == 0) {
        if (p.tma_bc) {
            ok = wait_mma(&S.bar[3], 0, p.status);  // B and C landed
            tc_fence_after();
        }
        for (int k = 0; ok && k < ksteps_n; ++k)
            umma_bf16(tmem + kColG, kdesc(c0, k), kdesc(b0, k), idesc_bf16(128, 128, 0, 0), k > 0);
    }
    chunk_delta(p, h, nq, dt_raw, S.dt, S.acum2, S.wsum, S.F, S.wmax);

    if (t == 0) {
        ok = ok && wait_mma(&S.bar[2], 0, p.status);  // h_in landed
        tc_fence_after();
        // C·h_in: A = C, B = h_in (N = channel p contiguous, K = n: M/N-major)
        const uint32_t hh0 = smem_addr(S.HX), hl0 = smem_addr(S.Hl);
        for (int k = 0; ok && k < ksteps_n; ++k) {
            const uint64_t a = kdesc(c0, k);
            umma_bf16(tmem + kColYo, a, umma_desc(hh0 + k * 2 * kRowP, kRowP, 128),
                      idesc_bf16(128, kPp, 0, 1), k > 0);
            umma_bf16(tmem + kColYo, a, umma_desc(hl0 + k * 2 * kRowP, kRowP, 128),
                      idesc_bf16(128, kPp, 0, 1), 1);
        }
        umma_commit(&S.bar[0]);  // tracks the G and C·h_in MMAs
    }
    ok = __syncthreads_and(ok && wait_mma(&S.bar[0], 0, p.status));
    tc_fence_after();

    // the chunk's z rows into h_in's low tile (its MMAs are done)
    if (kGate) {
        stage_tile<kPp>(S.Hl, static_cast<const bf16 *>(p.z) + row0 * D + (long long)h * P, D, nq,
                        P, p.vec_x);
        cp_async_commit();
    }
    // M row i = r, columns j in this thread's half, from G row i:
    // (C_i·B_j)·exp(Acum_i − Acum_j)·Δ_j for j ≤ i, stored as two bfloat16
    // parts M = M_hi + M_lo (M_hi into the B tile, M_lo into the C tile: both
    // are free once the first MMAs are done). Single products M_ij·x_j can be
    // far larger than y_i, so one bfloat16 rounding of M would cost more than
    // the output's own rounding; the pair keeps about 16 significant bits.
    // Column blocks above the diagonal for all of a warp's 32 rows are zero
    // (no tensor-memory read); the decay is 2^acum2_i · F_j when the chunk's
    // prefix sums allow it (no MUFU per element), else 2^(acum2_i − acum2_j).
    if (ok) {
        const int q = warp & 3;  // this warp's rows are 32q .. 32q + 31
        const float ai = S.acum2[r];
        const bool factored = fmaxf(fmaxf(S.wmax[0], S.wmax[1]), fmaxf(S.wmax[2], S.wmax[3])) <=
                              kFactorMax;
        const float ei = ex2_approx(ai);
#pragma unroll 1
        for (int cb = 2 * hh; cb < 2 * hh + 2; ++cb) {
            if (cb > q) {
                const uint4 z4 = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int k8 = 0; k8 < 4; ++k8) {
                    const uint32_t off = core_off<kQ>(r, 32 * cb + 8 * k8);
                    st_smem16(S.BM, off, z4);
                    st_smem16(S.C, off, z4);
                }
                continue;
            }
            float g[32];
            tmem_ld32(tmem + lane_q + kColG + 32 * cb, g);
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
                float m[8];
                if (factored) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 32 * cb + 8 * k8 + e;
                        m[e] = (j <= r && live) ? g[8 * k8 + e] * ei * S.F[j] : 0.0f;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 32 * cb + 8 * k8 + e;
                        m[e] = (j <= r && live)
                                   ? g[8 * k8 + e] * ex2_approx(ai - S.acum2[j]) * S.dt[j]
                                   : 0.0f;
                    }
                }
                uint4 hi, lo;
                split8(m, hi, lo);
                const uint32_t off = core_off<kQ>(r, 32 * cb + 8 * k8);
                st_smem16(S.BM, off, hi);
                st_smem16(S.C, off, lo);
            }
        }
    }
    // the x rows into h_in's high tile
#pragma unroll
    for (int k = 0; k < tile_items<kPp>(); ++k) {
        int j, chunk;
        tile_item<kPp>(k, j, chunk);
        st_smem16(S.HX, core_off<kPp>(j, 8 * chunk), xr[k]);
    }
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
    if (kGate) cp_async_wait_all();  // this thread's z copies (the barrier below publishes them)
    ok = __syncthreads_and(ok && wait_mma(&S.bar[1], 0, p.status));
    tc_fence_after();

    // every lane loads its accumulator rows (tcgen05.ld is warp-wide); rows
    // past the sequence end store nothing. x and z come from shared memory.
    if (ok && 32 * hh < P) {
        bf16 *yrow = static_cast<bf16 *>(p.y) + row * D + (long long)h * P;
        const float dec = ex2_approx(S.acum2[r]);
        const float dsk = p.Dskip ? p.Dskip[h] : 0.0f;
        float yd[32], yo[32];
        tmem_ld32(tmem + lane_q + kColYd + 32 * hh, yd);
        tmem_ld32(tmem + lane_q + kColYo + 32 * hh, yo);
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {
            const int c0 = 32 * hh + 8 * k8;
            if (c0 >= P || !live) break;
            const uint32_t off = core_off<kPp>(r, c0);
            float xv[8], zv[8], o[8];
            unpack8(*reinterpret_cast<const uint4 *>(reinterpret_cast<const char *>(S.HX) + off), xv);
            if (kGate)
                unpack8(*reinterpret_cast<const uint4 *>(reinterpret_cast<const char *>(S.Hl) + off), zv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float v = fmaf(dec, yo[8 * k8 + e], yd[8 * k8 + e]) + dsk * xv[e];
                if (kGate) v *= silu_tanh(zv[e]);  // one MUFU op; bfloat16 output
                o[e] = v;
            }
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
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// cuTensorMapEncodeTiled from the driver (through the runtime's entry-point
// query, so the library links against the runtime only).
PFN_cuTensorMapEncodeTiled_v12000 tma_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// A [batch][seqlen][dstate] bfloat16 tensor (B or C) as a 3-D map with
// 64-column × 128-token boxes, 128-byte swizzle, zero fill outside.
bool make_bc_map(CUtensorMap *m, const void *base, long long batch, long long seqlen, int dstate) {
    auto fn = tma_encode();
    if (!fn) return false;
    cuuint64_t gdim[3] = {(cuuint64_t)dstate, (cuuint64_t)seqlen, (cuuint64_t)batch};
    cuuint64_t gstride[2] = {(cuuint64_t)dstate * 2, (cuuint64_t)(seqlen * dstate * 2)};
    cuuint32_t box[3] = {64, (cuuint32_t)kQ, 1};
    cuuint32_t estride[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), gdim, gstride, box,
              estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
    static int sms_of[64] = {0};
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = set_smem(ssd_tc_state_kernel, sizeof(TcStateSmem) + 1024);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&sms_of[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const int sms = (dev >= 0 && dev < 64 && sms_of[dev] > 0) ? sms_of[dev] : 148;
    // heads per CTA (1..8): the fewest estimated CTA-time units, a CTA of g
    // heads taking (setup + g) with the setup (TMEM, barriers, the B tile)
    // about half a head, and the CTAs running in waves of two per SM
    SsdParams q = p;
    int best = 1;
    double best_cost = 1e300;
    for (int g = 1; g <= 8; ++g) {
        const long long ctas = (long long)p.nchunks * ((p.nheads + g - 1) / g) * p.batch;
        const long long waves = (ctas + 2LL * sms - 1) / (2LL * sms);
        const double cost = (double)waves * (0.5 + g);
        if (cost < best_cost) {
            best_cost = cost;
            best = g;
        }
    }
    q.heads_per_cta = best;
    const dim3 grid((unsigned)p.nchunks,
                    (unsigned)((p.nheads + q.heads_per_cta - 1) / q.heads_per_cta),
                    (unsigned)p.batch);
    CUtensorMap mb{};
    q.tma_bc = p.vec_bc && make_bc_map(&mb, p.B, p.batch, p.seqlen, p.dstate) ? 1 : 0;
    ssd_tc_state_kernel<<<grid, kThrTc, sizeof(TcStateSmem) + 1024, stream>>>(q, mb);
    return cudaGetLastError();
}

cudaError_t launch_ssd_tc_carry(const SsdParams &p, cudaStream_t stream) {
    const long long n = (long long)p.batch * p.nheads * (kNp / kCarryRows);
    ssd_tc_carry_kernel<<<(unsigned)n, kCarryThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_ssd_tc_out(const SsdParams &p, cudaStream_t stream) {
    static bool configured[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = set_smem(ssd_tc_out_kernel<true>, sizeof(TcOutSmem) + 1024);
        if (e == cudaSuccess) e = set_smem(ssd_tc_out_kernel<false>, sizeof(TcOutSmem) + 1024);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const dim3 grid((unsigned)p.nchunks, (unsigned)p.nheads, (unsigned)p.batch);
    SsdParams q = p;
    CUtensorMap mb{}, mc{};
    q.tma_bc = p.vec_bc && make_bc_map(&mb, p.B, p.batch, p.seqlen, p.dstate) &&
                       make_bc_map(&mc, p.C, p.batch, p.seqlen, p.dstate)
                   ? 1 : 0;
    if (p.z)
        ssd_tc_out_kernel<true><<<grid, kThrTc, sizeof(TcOutSmem) + 1024, stream>>>(q, mb, mc);
    else
        ssd_tc_out_kernel<false><<<grid, kThrTc, sizeof(TcOutSmem) + 1024, stream>>>(q, mb, mc);
    return cudaGetLastError();
}

}  // namespace selscan
