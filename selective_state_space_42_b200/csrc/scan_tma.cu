// scan_tma.cu -- persistent, TMA-staged selective-scan kernel for sm_100a.
//
// Pages: "Mamba & State Space Models — Guide Complet" §4 "Implémentation du
// SSM sélectif (S6)" (Δ = softplus(·), Abar = exp(Δ·A), h = Abar·h + Bbar·x,
// y = C·h + D·x) and "Parallel Associative Scan"; "Mamba и State Space Models:
// альтернатива Transformer", "SSM as RNN" and "Hardware-Aware Scan" (blocks of
// the sequence with the state carried between them); "Mamba: co potrafią
// modele przestrzeni stanów", "Cena selekcji" (fuse discretisation and
// recurrence on chip, never write the expanded state).
//
// Organisation. One CTA per SM, 4 consumer warps + 1 producer warp. A unit of
// work is (batch row b, 128-channel tile, chunk of the sequence). The producer
// takes units from a global ticket counter, streams each unit's x, delta and
// z tiles (kTile tokens × 128 channels) into a kStages-deep shared-memory ring
// with 2-D TMA loads, and converts the unit's B and C rows to float32 in the
// same ring slot. Each consumer thread owns one channel chain (16 float32
// states in registers) and walks the tokens of a tile in sub-tiles of kSub:
// first the per-token scalars (softplus, Δ·x, exp, gate) for all kSub tokens,
// then the recurrence, packed two states at a time (f32x2).
//
// Modes:
//  kSeq     single pass. Ticket i is chunk i / G of group i % G (G = batch ×
//           channel tiles), so a unit's predecessor was handed out G tickets
//           earlier to a running CTA; the unit waits (bounded) for the
//           predecessor's completion flag, reads its final state from a
//           per-group buffer in L2, and publishes its own when done. This
//           balances any number of groups over the SMs without extra work.
//           Each consumer warp hands over its own 32 channels (one flag per
//           group and warp), so no barrier spans warps.
//  kAgg     pass 1 of the chunked plan: chunks from a zero state, storing the
//           aggregate P = Π Abar = 2^(A·log2 e·ΣΔ) and the chunk state H.
//  kRescan  pass 2: chunks from the carried-in state; writes y.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "selscan_device.cuh"
#include "tma_util.cuh"

namespace selscan {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kChannels = 32 * kConsumerWarps;  // channels per tile (one per consumer thread)
constexpr int kBlock = kChannels + 32;          // + producer warp
constexpr int kMaxConsumerWarps = 8;            // flags per group in the workspace
#ifndef SELSCAN_TMA_STAGES
#define SELSCAN_TMA_STAGES 4
#endif
#ifndef SELSCAN_TMA_KSUB
#define SELSCAN_TMA_KSUB 8
#endif
constexpr int kStages = SELSCAN_TMA_STAGES;
constexpr int kSub = SELSCAN_TMA_KSUB;  // tokens per register sub-tile

template <typename T> struct TileCfg;
template <> struct TileCfg<__nv_bfloat16> { static constexpr int kTile = 32; };
template <> struct TileCfg<float> { static constexpr int kTile = 16; };

// Rows of x before a tile that the causal conv reads.
constexpr int kHalo = kMaxConv - 1;

// The x rows of a stage: with the conv, the kHalo tokens before the tile
// sit right before the tile's rows, so one TMA box fills both.
template <typename T, bool kConv> struct XRows;
template <typename T> struct XRows<T, false> {
    T x[TileCfg<T>::kTile][kChannels];
};
template <typename T> struct XRows<T, true> {
    T xh[kHalo][kChannels];
    T x[TileCfg<T>::kTile][kChannels];
};

template <typename T, bool kConv> struct alignas(128) Stage : XRows<T, kConv> {
    static constexpr int kTile = TileCfg<T>::kTile;
    T dl[kTile][kChannels];
    T z[kTile][kChannels];
    T Bs[kTile * kMaxN];  // TMA destination: the tile's B rows, dstate per row
    T Cs[kTile * kMaxN];
    float B[kTile][kMaxN];  // float32 copies read by the consumers (zero padded)
    float C[kTile][kMaxN];
};

// Two-lane float32 arithmetic (packed f32x2 instructions: one issue slot
// for two lanes of work).
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }

enum : int { kFirst = 1, kLast = 2, kEnd = 4 };

struct TileInfo {
    long long b, t0;
    int tile, chunk, nt, flags;
};

constexpr int kYBufs = 2;  // y staging tiles per consumer warp (TMA stores in flight)

template <typename T, bool kConv> struct alignas(128) Shared {
    Stage<T, kConv> stage[kStages];
    // per consumer warp: y of its 32 channels for one full tile, [kTile][32]
    alignas(128) T ybuf[kConsumerWarps][kYBufs][TileCfg<T>::kTile * 32];
    TileInfo info[kStages];
    uint64_t full[kStages];   // x/delta/z bytes + 32 producer arrivals (after B/C conversion)
    uint64_t empty[kStages];  // one arrival per consumer warp
    uint64_t bc[kStages];     // B/C TMA bytes of the stage
    int abort;
};

}  // namespace

// Sticky device-side error word of this library on each device: 0, or the
// code of the first wait that gave up (1 predecessor flag, 2 producer ring
// slot, 3 consumer ring slot). Read and cleared by selscan_device_status.
__device__ int g_device_status = 0;

namespace {

__device__ const int kNoAbort = 0;

// Records the failure, stops this CTA (shared abort word) and every other CTA
// of the launch (the launch's abort word in the workspace, polled by waits).
__device__ __forceinline__ void fail(const TmaScanParams &p, int *abort, int code) {
    atomicCAS(&g_device_status, 0, code);
    *reinterpret_cast<volatile int *>(abort) = 1;
    *reinterpret_cast<volatile int *>(p.abort_all) = 1;
}

// ---- producer warp -----------------------------------------------------------------
// Converts the B and C rows of stage s (landed by TMA as the I/O type, dstate
// per row) to float32 [kTile][16], zero for rows past nt and states past
// dstate. Lane l handles float4 slots l, l + 32, ...: consecutive lanes write
// consecutive 16-byte chunks.
template <typename T, bool kConv>
__device__ __forceinline__ void convert_bc(Stage<T, kConv> &st, int nt, int dstate, int lane) {
    constexpr int kTile = TileCfg<T>::kTile;
    constexpr int kSlots = kTile * kMaxN / 4;
#pragma unroll
    for (int i = lane; i < kSlots; i += 32) {
        const int t = i / (kMaxN / 4);
        const int n0 = (i % (kMaxN / 4)) * 4;
        float vb[4], vc[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool ok = t < nt && n0 + e < dstate;
            vb[e] = ok ? to_f32(st.Bs[t * dstate + n0 + e]) : 0.0f;
            vc[e] = ok ? to_f32(st.Cs[t * dstate + n0 + e]) : 0.0f;
        }
        reinterpret_cast<float4 *>(&st.B[0][0])[i] = make_float4(vb[0], vb[1], vb[2], vb[3]);
        reinterpret_cast<float4 *>(&st.C[0][0])[i] = make_float4(vc[0], vc[1], vc[2], vc[3]);
    }
}

// The producer issues every TMA of a stage as soon as the stage is free and
// converts its B/C kLag stages later, so it never waits on global memory
// latency itself; the stage is handed to the consumers (32 arrivals on
// `full`) after its conversion.
template <typename T, bool kGate, bool kConv>
__device__ void produce(Shared<T, kConv> &S, const TmaScanParams &p, const CUtensorMap *tm_x,
                        const CUtensorMap *tm_d, const CUtensorMap *tm_z,
                        const CUtensorMap *tm_b, const CUtensorMap *tm_c) {
    constexpr int kTile = TileCfg<T>::kTile;
    constexpr int kLag = kStages > 2 ? 2 : 1;
    const int lane = threadIdx.x & 31;
    if (lane == 0) {
        prefetch_tmap(tm_x);
        prefetch_tmap(tm_d);
        if (kGate) prefetch_tmap(tm_z);
        prefetch_tmap(tm_b);
        prefetch_tmap(tm_c);
    }
    constexpr uint32_t kTileBytes = kTile * kChannels * sizeof(T);
    constexpr uint32_t kXBytes = (kConv ? kHalo + kTile : kTile) * kChannels * sizeof(T);
    const uint32_t tx_bytes = (kGate ? 2u : 1u) * kTileBytes + kXBytes;
    const uint32_t bc_bytes = 2u * kTile * p.dstate * sizeof(T);
    int s = 0;                 // next stage to fill
    uint32_t phase = 0;
    int cs = 0;                // oldest stage awaiting conversion
    uint32_t cphase = 0;
    int npend = 0;             // stages issued but not yet converted / handed over

    // converts the oldest pending stage and hands it to the consumers
    auto convert_oldest = [&]() -> bool {
        if (!mbar_wait(&S.bc[cs], cphase, &S.abort, p.timeout_ns)) return false;
        convert_bc<T, kConv>(S.stage[cs], S.info[cs].nt, p.dstate, lane);
        __syncwarp();
        mbar_arrive(&S.full[cs]);
        if (++cs == kStages) {
            cs = 0;
            cphase ^= 1u;
        }
        --npend;
        return true;
    };
    // failure: record it, then wait (bounded) for this warp's copies in flight
    auto bail = [&]() {
        if (lane == 0) fail(p, &S.abort, 2);
        for (; npend > 0; --npend) {
            mbar_wait(&S.bc[cs], cphase, &kNoAbort, p.timeout_ns / 16);
            mbar_arrive(&S.full[cs]);
            mbar_wait(&S.full[cs], cphase, &kNoAbort, p.timeout_ns / 16);
            if (++cs == kStages) {
                cs = 0;
                cphase ^= 1u;
            }
        }
        __syncwarp();
    };

    for (;;) {
        int ticket = 0;
        if (lane == 0) ticket = atomicAdd(p.ticket, 1);
        ticket = __shfl_sync(0xffffffffu, ticket, 0);
        const bool end = ticket >= p.units;
        if (end) {
            while (npend > 0)
                if (!convert_oldest()) return bail();
            if (!mbar_wait(&S.empty[s], phase ^ 1u, &S.abort, p.timeout_ns)) return bail();
            if (lane == 0) S.info[s].flags = kEnd;
            __syncwarp();
            mbar_arrive(&S.full[s]);
            return;
        }
        const long long g = ticket % p.groups;
        const int chunk = (int)(ticket / p.groups);
        const long long b = g / p.ntiles;
        const int tile = (int)(g % p.ntiles);
        const long long t_begin = (long long)chunk * p.chunk_len;
        const long long t_end = min(t_begin + p.chunk_len, (long long)p.seqlen);
        const int ntl = (int)((t_end - t_begin + kTile - 1) / kTile);
        for (int j = 0; j < ntl; ++j) {
            if (!mbar_wait(&S.empty[s], phase ^ 1u, &S.abort, p.timeout_ns)) return bail();
            const long long t0 = t_begin + (long long)j * kTile;
            if (lane == 0) {
                TileInfo &inf = S.info[s];
                inf.b = b;
                inf.t0 = t0;
                inf.tile = tile;
                inf.chunk = chunk;
                inf.nt = (int)min((long long)kTile, t_end - t0);
                inf.flags = (j == 0 ? kFirst : 0) | (j == ntl - 1 ? kLast : 0);
                const int c1 = (int)(b * p.seqlen + t0);
                mbar_expect_tx(&S.full[s], tx_bytes);
                // with the conv the box starts kHalo rows early (a negative row
                // at the very start reads zeros; rows of the previous sequence
                // are ignored by the consumers)
                if constexpr (kConv)
                    tma_load_2d(&S.stage[s].xh[0][0], tm_x, &S.full[s], tile * kChannels,
                                c1 - kHalo);
                else
                    tma_load_2d(&S.stage[s].x[0][0], tm_x, &S.full[s], tile * kChannels, c1);
                tma_load_2d(&S.stage[s].dl[0][0], tm_d, &S.full[s], tile * kChannels, c1);
                if (kGate) tma_load_2d(&S.stage[s].z[0][0], tm_z, &S.full[s], tile * kChannels, c1);
                mbar_arrive_expect_tx(&S.bc[s], bc_bytes);
                tma_load_2d(&S.stage[s].Bs[0], tm_b, &S.bc[s], 0, c1);
                tma_load_2d(&S.stage[s].Cs[0], tm_c, &S.bc[s], 0, c1);
            }
            __syncwarp();
            if (++s == kStages) {
                s = 0;
                phase ^= 1u;
            }
            if (++npend > kLag)
                if (!convert_oldest()) return bail();
        }
    }
}

// ---- consumer warps ----------------------------------------------------------------
__device__ __forceinline__ float softplus_fast(float v) {
    // log(1 + e^v) through the MUFU pair; absolute error ~1e-7, enough for
    // bf16 I/O. Large v returns v.
    const float w = ex2_approx(v * kLog2e);
    const float s = lg2_approx(1.0f + w) * kLn2;
    return v > 15.0f ? v : s;
}

// One ring stage for this thread's channel. kFull: the stage holds kTile
// valid tokens and y goes to this warp's shared-memory tile `ys` (written to
// global memory by one TMA store per warp); otherwise tokens past nt leave
// the state unchanged and y goes straight to global memory.
template <typename T, bool kGate, int kMode, bool kStruct, bool kSoftplus, bool kFull,
          bool kConv>
__device__ __forceinline__ void consume_tile(const Stage<T, kConv> &st, int nt,
                                             float2 (&h)[kMaxN / 2],
                                             const float (&A2)[kMaxN], float dskip, float bias,
                                             float &dt_sum, T *ys, T *yp, long long ybase,
                                             long long ystride, bool active,
                                             const float (&cw)[kMaxConv], float cb,
                                             float (&xw)[kMaxConv - 1]) {
    constexpr int kTile = TileCfg<T>::kTile;
    constexpr bool kFastSp = sizeof(T) == 2;
    const int c = threadIdx.x;  // channel within the tile
    const int lane = c & 31;
#pragma unroll 1
    for (int sub = 0; sub < kTile; sub += kSub) {
        if (!kFull && sub >= nt) break;
        float uu[kSub], rr[kSub], gg[kSub], pp[kSub];
        // per-token scalars
#pragma unroll
        for (int k = 0; k < kSub; ++k) {
            const int t = sub + k;
            float xv = to_f32(st.x[t][c]);
            if (kConv) xv = conv_step(cw, cb, xw, xv);
            float dt = to_f32(st.dl[t][c]) + bias;
            if (kSoftplus) dt = kFastSp ? softplus_fast(dt) : softplus_f32(dt);
            if (!kFull) dt = t < nt ? dt : 0.0f;  // Abar = 1, no input: state unchanged
            uu[k] = dt * xv;
            rr[k] = kStruct ? ex2_approx(dt * A2[0]) : dt;
            if (kMode == kModeAgg) {
                dt_sum += dt;
            } else {
                const float g = kGate ? silu_f32(to_f32(st.z[t][c])) : 1.0f;
                gg[k] = g;
                pp[k] = dskip * xv * g;
            }
        }
        // recurrence
#pragma unroll
        for (int k = 0; k < kSub; ++k) {
            const int t = sub + k;
            float2 a[kMaxN / 2];
            if (kStruct) {
                const float r = rr[k];
                const float r2 = r * r;
                a[0] = make_float2(r, r2);
                a[1] = mul2(a[0], make_float2(r2, r2));
                const float r4 = a[1].y;
                const float2 q4 = make_float2(r4, r4);
                a[2] = mul2(a[0], q4);
                a[3] = mul2(a[1], q4);
                const float r8 = a[3].y;
                const float2 q8 = make_float2(r8, r8);
#pragma unroll
                for (int j = 0; j < 4; ++j) a[4 + j] = mul2(a[j], q8);
            } else {
#pragma unroll
                for (int j = 0; j < kMaxN / 2; ++j)
                    a[j] = make_float2(ex2_approx(rr[k] * A2[2 * j]),
                                       ex2_approx(rr[k] * A2[2 * j + 1]));
            }
            const float2 u2 = make_float2(uu[k], uu[k]);
            const float4 *B4 = reinterpret_cast<const float4 *>(&st.B[t][0]);
            if (kMode == kModeAgg) {
#pragma unroll
                for (int q = 0; q < kMaxN / 4; ++q) {
                    const float4 bq = B4[q];
                    h[2 * q] = fma2(a[2 * q], h[2 * q], mul2(u2, make_float2(bq.x, bq.y)));
                    h[2 * q + 1] = fma2(a[2 * q + 1], h[2 * q + 1], mul2(u2, make_float2(bq.z, bq.w)));
                }
            } else {
                const float4 *C4 = reinterpret_cast<const float4 *>(&st.C[t][0]);
                float2 y0 = make_float2(0.0f, 0.0f), y1 = y0;
#pragma unroll
                for (int q = 0; q < kMaxN / 4; ++q) {
                    const float4 bq = B4[q];
                    const float4 cq = C4[q];
                    h[2 * q] = fma2(a[2 * q], h[2 * q], mul2(u2, make_float2(bq.x, bq.y)));
                    h[2 * q + 1] = fma2(a[2 * q + 1], h[2 * q + 1], mul2(u2, make_float2(bq.z, bq.w)));
                    y0 = fma2(make_float2(cq.x, cq.y), h[2 * q], y0);
                    y1 = fma2(make_float2(cq.z, cq.w), h[2 * q + 1], y1);
                }
                const float2 yv = add2(y0, y1);
                const T out = from_f32<T>(fmaf(yv.x + yv.y, gg[k], pp[k]));
                if (kFull)
                    ys[t * 32 + lane] = out;
                else if (active && t < nt)
                    yp[ybase + (long long)t * ystride] = out;
            }
        }
    }
}

template <typename T, bool kGate, int kMode, bool kSoftplus, bool kConv>
__device__ void consume(Shared<T, kConv> &S, const TmaScanParams &p, const CUtensorMap *tm_y) {
    constexpr int kTile = TileCfg<T>::kTile;
    const int c = threadIdx.x;  // 0..127
    const int lane = c & 31;
    const int warp = c >> 5;
    int kbuf = 0;
    // before leaving: this warp's y stores must have finished reading shared memory
    auto drain = [&]() {
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    };
    T *yp = static_cast<T *>(p.y);
    int s = 0;
    uint32_t phase = 0;
    int cur_tile = -1;
    float A2[kMaxN];
    float dskip = 0.0f, bias = 0.0f;
    float cw[kMaxConv] = {0.f, 0.f, 0.f, 0.f}, cb = 0.0f;  // conv taps of this channel
    bool structured = false;
    float2 h[kMaxN / 2];
#pragma unroll
    for (int j = 0; j < kMaxN / 2; ++j) h[j] = make_float2(0.0f, 0.0f);
    float dt_sum = 0.0f;
    for (;;) {
        if (!mbar_wait(&S.full[s], phase, &S.abort, p.timeout_ns)) {
            if (lane == 0) fail(p, &S.abort, 3);
            return drain();
        }
        const TileInfo inf = S.info[s];
        if (inf.flags & kEnd) return drain();
        const long long d = (long long)inf.tile * kChannels + c;
        const bool active = d < p.dim;
        const long long g = inf.b * p.ntiles + inf.tile;
        if (inf.flags & kFirst) {
            if (inf.tile != cur_tile) {
                bool ok = true;
                if (active) {
                    const float *Ar = p.A + d * p.dstate;
                    const float a0 = Ar[0];
#pragma unroll
                    for (int n = 0; n < kMaxN; ++n) {
                        const float an = n < p.dstate ? Ar[n] : 0.0f;
                        A2[n] = an * kLog2e;
                        if (n < p.dstate) ok &= (an == (float)(n + 1) * a0);
                    }
                    dskip = p.Dskip ? p.Dskip[d] : 0.0f;
                    bias = p.delta_bias ? p.delta_bias[d] : 0.0f;
                    if (kConv) {
                        load_conv_taps(p.conv_w, p.conv_width, d, cw);
                        cb = p.conv_b ? p.conv_b[d] : 0.0f;
                    }
                } else {
#pragma unroll
                    for (int n = 0; n < kMaxN; ++n) A2[n] = 0.0f;
                    dskip = bias = 0.0f;
                }
                structured = __all_sync(0xffffffffu, ok);
                cur_tile = inf.tile;
            }
            dt_sum = 0.0f;
            float hs[kMaxN];
#pragma unroll
            for (int n = 0; n < kMaxN; ++n) hs[n] = 0.0f;
            if (kMode == kModeSeq && inf.chunk > 0) {
                // every lane acquires this warp's predecessor flag (bounded)
                const int *flag = p.flags + g * kMaxConsumerWarps + (c >> 5);
                const uint64_t start = global_ns();
                while (ld_acquire_gpu(flag) < inf.chunk) {
                    __nanosleep(64);
                    if (*reinterpret_cast<volatile int *>(&S.abort) ||
                        *reinterpret_cast<volatile int *>(p.abort_all) ||
                        global_ns() - start > p.timeout_ns) {
                        if (lane == 0) fail(p, &S.abort, 1);
                        break;
                    }
                }
                __syncwarp();
                if (active) {
                    const float *src = p.ws_state + (g * kChannels + c) * kMaxN;
#pragma unroll
                    for (int q = 0; q < kMaxN / 4; ++q) {
                        const float4 v = ld_cg_f4(src + 4 * q);
                        hs[4 * q] = v.x; hs[4 * q + 1] = v.y; hs[4 * q + 2] = v.z; hs[4 * q + 3] = v.w;
                    }
                }
            } else if (kMode == kModeSeq && p.h0 && active) {
                const float *src = p.h0 + (inf.b * p.dim + d) * p.dstate;
#pragma unroll
                for (int n = 0; n < kMaxN; ++n) hs[n] = n < p.dstate ? src[n] : 0.0f;
            } else if (kMode == kModeRescan && p.nchunks > 1 && active) {
                const float *src = p.ws_H + ((inf.b * p.nchunks + inf.chunk) * p.dim + d) * kMaxN;
#pragma unroll
                for (int n = 0; n < kMaxN; ++n) hs[n] = src[n];
            }
#pragma unroll
            for (int j = 0; j < kMaxN / 2; ++j) h[j] = make_float2(hs[2 * j], hs[2 * j + 1]);
        }

        const long long ybase = (inf.b * p.seqlen + inf.t0) * p.dim + d;
        // conv window: the inputs of the kHalo tokens before the tile (zero
        // before the sequence's first token)
        float xw[kMaxConv - 1] = {0.f, 0.f, 0.f};
        if constexpr (kConv) {
            if (inf.t0 > 0) {
#pragma unroll
                for (int k = 0; k < kHalo; ++k) xw[k] = to_f32(S.stage[s].xh[k][c]);
            } else if (p.conv_init && active) {
#pragma unroll
                for (int k = 0; k < kHalo; ++k)
                    xw[k] = p.conv_init[(inf.b * p.dim + d) * kHalo + k];
            }
        }
        if (inf.nt == kTile) {
            T *ys = S.ybuf[warp][kbuf];
            if (kMode != kModeAgg) {
                // the store that last read this staging tile has finished with it
                if (lane == 0) bulk_wait_read<kYBufs - 1>();
                __syncwarp();
            }
            if (structured)
                consume_tile<T, kGate, kMode, true, kSoftplus, true, kConv>(
                    S.stage[s], inf.nt, h, A2, dskip, bias, dt_sum, ys, yp, ybase, p.dim, active,
                    cw, cb, xw);
            else
                consume_tile<T, kGate, kMode, false, kSoftplus, true, kConv>(
                    S.stage[s], inf.nt, h, A2, dskip, bias, dt_sum, ys, yp, ybase, p.dim, active,
                    cw, cb, xw);
            if (kMode != kModeAgg) {
                fence_proxy_async_smem();
                __syncwarp();
                const int c0 = inf.tile * kChannels + warp * 32;
                if (lane == 0 && c0 < p.dim) {
                    tma_store_2d(tm_y, ys, c0, (int)(inf.b * p.seqlen + inf.t0));
                    bulk_commit();
                }
                kbuf ^= 1;
            }
        } else {
            if (structured)
                consume_tile<T, kGate, kMode, true, kSoftplus, false, kConv>(
                    S.stage[s], inf.nt, h, A2, dskip, bias, dt_sum, nullptr, yp, ybase, p.dim,
                    active, cw, cb, xw);
            else
                consume_tile<T, kGate, kMode, false, kSoftplus, false, kConv>(
                    S.stage[s], inf.nt, h, A2, dskip, bias, dt_sum, nullptr, yp, ybase, p.dim,
                    active, cw, cb, xw);
        }

        if (inf.flags & kLast) {
            const bool last_chunk = inf.chunk == p.nchunks - 1;
            if (kMode == kModeAgg) {
                if (active) {
                    const long long row = ((inf.b * p.nchunks + inf.chunk) * p.dim + d) * kMaxN;
#pragma unroll
                    for (int j = 0; j < kMaxN / 2; ++j) {
                        p.ws_P[row + 2 * j] = ex2_approx(A2[2 * j] * dt_sum);
                        p.ws_P[row + 2 * j + 1] = ex2_approx(A2[2 * j + 1] * dt_sum);
                        p.ws_H[row + 2 * j] = h[j].x;
                        p.ws_H[row + 2 * j + 1] = h[j].y;
                    }
                }
            } else if (last_chunk) {
                if (p.final_state && active) {
                    float *fs = p.final_state + (inf.b * p.dim + d) * p.dstate;
#pragma unroll
                    for (int j = 0; j < kMaxN / 2; ++j) {
                        if (2 * j < p.dstate) fs[2 * j] = h[j].x;
                        if (2 * j + 1 < p.dstate) fs[2 * j + 1] = h[j].y;
                    }
                }
            } else if (kMode == kModeSeq) {
                if (active) {
                    float *dst = p.ws_state + (g * kChannels + c) * kMaxN;
#pragma unroll
                    for (int q = 0; q < kMaxN / 4; ++q)
                        st_cg_f4(dst + 4 * q, make_float4(h[2 * q].x, h[2 * q].y, h[2 * q + 1].x,
                                                          h[2 * q + 1].y));
                }
                __threadfence();
                __syncwarp();
                if (lane == 0)
                    st_release_gpu(p.flags + g * kMaxConsumerWarps + (c >> 5), inf.chunk + 1);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[s]);
        if (++s == kStages) {
            s = 0;
            phase ^= 1u;
        }
    }
}

template <typename T, bool kGate, int kMode, bool kSoftplus, bool kConv>
__global__ void __launch_bounds__(kBlock, 1)
scan_tma_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_d,
                const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                const TmaScanParams p) {
    // Indexed straight off the __shared__ array so that every access compiles
    // to a shared-memory instruction (no generic addressing, no aliasing with
    // the global y stores).
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    Shared<T, kConv> &S = *reinterpret_cast<Shared<T, kConv> *>(smem_raw);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&S.full[i], 32);              // producer lanes (+ TMA bytes)
            mbar_init(&S.empty[i], kConsumerWarps);  // one arrival per consumer warp
            mbar_init(&S.bc[i], 1);
        }
        S.abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x >= kChannels)
        produce<T, kGate, kConv>(S, p, &tm_x, &tm_d, &tm_z, &tm_b, &tm_c);
    else
        consume<T, kGate, kMode, kSoftplus, kConv>(S, p, &tm_y);
}

// ---- host side -----------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2-D map over a row-major [rows][cols] tensor with boxes of
// box_cols × TileCfg<T>::kTile rows.
template <typename T>
bool make_map(CUtensorMap *m, const void *base, long long rows, long long cols,
              int box_cols = kChannels, int box_rows = TileCfg<T>::kTile) {
    auto fn = encode_fn();
    if (!fn) return false;
    const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t gstride[1] = {(cuuint64_t)(cols * sizeof(T))};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void *>(base), gdim, gstride, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int num_sms() {
    static std::atomic<int> cached[64];
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64 && (sms = cached[dev].load(std::memory_order_relaxed)) > 0) return sms;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    if (dev < 64) cached[dev].store(sms, std::memory_order_relaxed);
    return sms;
}

template <typename T, bool kGate, int kMode, bool kSoftplus, bool kConv>
cudaError_t launch_mode(const TmaScanParams &p, const void *x, const void *dl, const void *z,
                        cudaStream_t stream) {
    if (p.units <= 0) return cudaSuccess;
    CUtensorMap mx, md, mz, mb, mc, my;
    const long long rows = p.batch * p.seqlen;
    const int x_rows = kConv ? kHalo + TileCfg<T>::kTile : TileCfg<T>::kTile;
    if (!make_map<T>(&mx, x, rows, p.dim, kChannels, x_rows) ||
        !make_map<T>(&md, dl, rows, p.dim) ||
        !make_map<T>(&mb, p.B, rows, p.dstate, p.dstate) ||
        !make_map<T>(&mc, p.C, rows, p.dstate, p.dstate) ||
        !make_map<T>(&my, p.y, rows, p.dim, 32))
        return cudaErrorInvalidValue;
    if (kGate) {
        if (!make_map<T>(&mz, z, rows, p.dim)) return cudaErrorInvalidValue;
    } else {
        mz = md;
    }
    const size_t smem = sizeof(Shared<T, kConv>);
    auto kern = scan_tma_kernel<T, kGate, kMode, kSoftplus, kConv>;
    // the shared-memory opt-in is set once per device for this instantiation
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    const long long grid = min((long long)num_sms(), (long long)p.units);
    kern<<<(unsigned)grid, kBlock, smem, stream>>>(mx, md, mz, mb, mc, my, p);
    return cudaGetLastError();
}

template <typename T, bool kGate, bool kSoftplus, bool kConv>
cudaError_t launch_conv(const TmaScanParams &p, const void *x, const void *dl, const void *z,
                        cudaStream_t stream) {
    switch (p.mode) {
    case kModeSeq: return launch_mode<T, kGate, kModeSeq, kSoftplus, kConv>(p, x, dl, z, stream);
    case kModeAgg: return launch_mode<T, false, kModeAgg, kSoftplus, kConv>(p, x, dl, z, stream);
    default: return launch_mode<T, kGate, kModeRescan, kSoftplus, kConv>(p, x, dl, z, stream);
    }
}

template <typename T, bool kGate, bool kSoftplus>
cudaError_t launch_sp(const TmaScanParams &p, const void *x, const void *dl, const void *z,
                      cudaStream_t stream) {
    return p.conv_width > 0 ? launch_conv<T, kGate, kSoftplus, true>(p, x, dl, z, stream)
                            : launch_conv<T, kGate, kSoftplus, false>(p, x, dl, z, stream);
}

template <typename T, bool kGate>
cudaError_t launch_gate(const TmaScanParams &p, const void *x, const void *dl, const void *z,
                        cudaStream_t stream) {
    return p.softplus ? launch_sp<T, kGate, true>(p, x, dl, z, stream)
                      : launch_sp<T, kGate, false>(p, x, dl, z, stream);
}

}  // namespace

cudaError_t device_status_address(int **p) {
    return cudaGetSymbolAddress(reinterpret_cast<void **>(p), g_device_status);
}

cudaError_t read_device_status(int *out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_device_status, sizeof(int));
    if (e == cudaSuccess && clear) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
    }
    return e;
}

int tma_tile_channels() { return kChannels; }
int tma_tile_tokens(bool bf16) {
    return bf16 ? TileCfg<__nv_bfloat16>::kTile : TileCfg<float>::kTile;
}

cudaError_t launch_scan_tma(const TmaScanParams &p, bool bf16, const void *x, const void *dl,
                            const void *z, cudaStream_t stream) {
    if (bf16)
        return z ? launch_gate<__nv_bfloat16, true>(p, x, dl, z, stream)
                 : launch_gate<__nv_bfloat16, false>(p, x, dl, z, stream);
    return z ? launch_gate<float, true>(p, x, dl, z, stream)
             : launch_gate<float, false>(p, x, dl, z, stream);
}

}  // namespace selscan
