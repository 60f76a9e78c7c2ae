// api.cu -- the C ABI of libselscan (declared in include/selscan.h): argument
// validation, the launch plan, workspace handling and error reporting. Every
// step of the computation runs in the CUDA kernels of scan.cu and
// state_update.cu; this file only checks arguments and launches them.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "selscan.h"
#include "selscan_device.cuh"
#include "ssd_params.cuh"
#include "bwd_params.cuh"

namespace {

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

bool misaligned(const void *p, size_t a) {
    return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) != 0;
}

// Half-open byte ranges [a, a + na) and [b, b + nb) intersect.
bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a);
    const uintptr_t pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
}

// a · b ≤ limit for non-negative a, b, without overflow.
bool mul_le(int64_t a, int64_t b, int64_t limit) {
    return a == 0 || b <= limit / a;
}

constexpr int64_t kMaxElems = (int64_t)1 << 40;  // per tensor

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
        sms = 148;
    if (dev < 64) cached[dev] = sms;
    return sms;
}

// A set, non-"0" environment variable (tuning and testing switches).
bool env_flag(const char *name) {
    const char *v = getenv(name);
    return v && *v && strcmp(v, "0") != 0;
}

int64_t env_int(const char *name) {
    const char *v = getenv(name);
    return (v && *v) ? atoll(v) : 0;
}

int64_t round_up(int64_t a, int64_t m) { return (a + m - 1) / m * m; }

// Chunks of the generic kernels' plan. Each (batch row, channel) chain is one
// thread; with too few chains to keep every SM busy the sequence is split so
// that chains × chunks reaches a target of resident threads, each chunk at
// least kMinChunk tokens and a whole number of B/C tiles.
void plan_generic(int64_t batch, int64_t seqlen, int64_t dim, selscan::FwdPlan *pl) {
    constexpr int64_t kMinChunk = 256;
    constexpr int64_t kSinglePassChains = 16384;
    int64_t n = env_int("SELSCAN_CHUNKS");
    if (n <= 0) {
        const int64_t chains = batch * dim;
        const int64_t target = (int64_t)sm_count() * 512;
        n = 1;
        if (chains < kSinglePassChains && seqlen >= 2 * kMinChunk) {
            n = (target + chains - 1) / chains;
            n = n < seqlen / kMinChunk ? n : seqlen / kMinChunk;
        }
    }
    if (n < 1) n = 1;
    if (n > seqlen) n = seqlen > 0 ? seqlen : 1;
    const int64_t tileT = selscan::scan_tile_tokens();
    int64_t len = round_up((seqlen + n - 1) / n, tileT);
    if (len < 1) len = 1;
    selscan::ScanParams &g = pl->gp;
    g.chunk_len = len;
    g.nchunks = seqlen > 0 ? (int)((seqlen + len - 1) / len) : 1;
    const int64_t cpc = selscan::scan_channels_per_cta();
    g.ntiles = (int)((dim + cpc - 1) / cpc);
    pl->tma = false;
    pl->chunks = g.nchunks;
    pl->launches = g.nchunks > 1 ? 3 : 1;
    pl->ws_bytes = g.nchunks > 1
                       ? 2 * (size_t)(batch * g.nchunks * dim) * selscan::kMaxN * sizeof(float)
                       : 0;
    pl->ws_clear = 0;
}

// Plan of the TMA kernel. Groups = batch rows × 128-channel tiles. With at
// least ~60% as many groups as SMs: one pass, units of 1024 tokens handed
// from chunk to chunk (kModeSeq). With fewer: chunk aggregates, carry and
// rescan, with about 8 units per SM. SELSCAN_PATH=seq|chunked, SELSCAN_UNIT
// and SELSCAN_CHUNKS override (tuning only).
void plan_tma(int64_t batch, int64_t seqlen, int64_t dim, bool bf16, selscan::FwdPlan *pl) {
    const int64_t tileT = selscan::tma_tile_tokens(bf16);
    const int64_t cpt = selscan::tma_tile_channels();
    const int64_t ntiles = (dim + cpt - 1) / cpt;
    const int64_t groups = batch * ntiles;
    const int64_t sms = sm_count();
    const char *path = getenv("SELSCAN_PATH");
    bool seq = groups * 5 >= sms * 3;
    if (path && !strcmp(path, "seq")) seq = true;
    if (path && !strcmp(path, "chunked")) seq = false;
    int64_t len = 0;
    if (seq) {
        len = env_int("SELSCAN_UNIT");
        if (len <= 0) len = 1024;
    } else {
        int64_t n = env_int("SELSCAN_CHUNKS");
        if (n <= 0) n = (8 * sms + groups - 1) / groups;
        const int64_t nmax = seqlen / 256 > 1 ? seqlen / 256 : 1;
        n = n < nmax ? n : nmax;
        if (n < 2) seq = true;
        len = (seqlen + n - 1) / n;
    }
    len = round_up(len < seqlen ? len : seqlen, tileT);
    const int64_t nchunks = (seqlen + len - 1) / len;
    if (nchunks <= 1) seq = true;
    selscan::TmaScanParams &t = pl->tp;
    t.mode = seq ? selscan::kModeSeq : selscan::kModeAgg;
    t.ntiles = (int)ntiles;
    t.chunk_len = len;
    t.nchunks = (int)nchunks;
    t.groups = groups;
    t.timeout_ns = 2000000000ull;
    const int64_t tmo = env_int("SELSCAN_TIMEOUT_MS");
    if (tmo > 0) t.timeout_ns = (unsigned long long)tmo * 1000000ull;
    // Test hook (off unless set): the one-pass plan's units of this chunk do
    // not publish their completion flag, so their successors' bounded waits
    // run out; the fault-handling test uses it together with a short
    // SELSCAN_TIMEOUT_MS.
    const char *skip = getenv("SELSCAN_TEST_SKIP_RELEASE");
    t.skip_release_chunk = (skip && *skip) ? atoi(skip) : -1;
    pl->tma = true;
    pl->chunks = (int)nchunks;
    pl->launches = seq ? 1 : 3;
    // workspace: [0, 256) tickets; SEQ: flags at 256, states after them;
    // chunked: P and H arrays from 256.
    if (seq) {
        const size_t flags_end = round_up(256 + 4 * 8 * groups, 256);  // one per warp
        pl->ws_clear = flags_end;
        pl->ws_bytes = flags_end + (size_t)groups * cpt * selscan::kMaxN * sizeof(float);
    } else {
        pl->ws_clear = 256;
        pl->ws_bytes =
            256 + 2 * (size_t)(batch * nchunks * dim) * selscan::kMaxN * sizeof(float);
    }
}

}  // namespace

namespace selscan {

int cuda_fail(cudaError_t e) {
    g_last_cuda_error = e;
    return SELSCAN_ERR_CUDA;
}

void plan_for_sizes(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int dtype,
                    bool aligned, FwdPlan *pl) {
    const bool bf16 = dtype == SELSCAN_BF16;
    const int64_t es = bf16 ? 2 : 4;
    const char *path = getenv("SELSCAN_PATH");
    const bool forced_generic = path && !strcmp(path, "generic");
    // TMA rows must start on 16-byte boundaries and tiles are 128 channels.
    // B/C rows are TMA'd too: dstate·elem must be a multiple of 16 bytes.
    const bool eligible = aligned && !forced_generic && dim >= tma_tile_channels() &&
                          (dim * es) % 16 == 0 && (dstate * es) % 16 == 0 &&
                          batch * seqlen < ((int64_t)1 << 31) && dstate <= kMaxN;
    pl->bf16 = bf16;
    pl->wide = dstate > kMaxN;
    if (pl->wide) {  // one pass of scan_wide.cu, no workspace
        pl->tma = false;
        pl->chunks = 1;
        pl->launches = 1;
        pl->ws_bytes = 0;
        pl->ws_clear = 0;
        pl->gp.nchunks = 1;
        pl->gp.chunk_len = seqlen;
    } else if (eligible) {
        plan_tma(batch, seqlen, dim, bf16, pl);
    } else {
        plan_generic(batch, seqlen, dim, pl);
    }
}

// Argument validation and launch plan shared by the selscan_fwd entry points.
// On SELSCAN_OK fills *plan (workspace pointers left NULL); *done is set when
// no kernel has to run (empty sizes; for seqlen == 0 the final state has
// been cleared on stream).
int fwd_setup(const void *x, const void *delta, const float *A, const void *B,
              const void *C, const float *D, const void *z, const float *delta_bias,
              int softplus_flag, const float *h0, const float *conv_w, const float *conv_b,
              const float *conv_init, int conv_width, int zoh, void *y, float *final_state,
              int64_t batch,
              int64_t seqlen, int64_t dim, int64_t dstate, int dtype,
              cudaStream_t stream, FwdPlan *plan, bool *done) {
    *done = false;
    if (dtype != SELSCAN_F32 && dtype != SELSCAN_BF16) return SELSCAN_ERR_BAD_DTYPE;
    if (batch < 0 || seqlen < 0 || dim < 0) return SELSCAN_ERR_BAD_DIM;
    if (dstate < 1 || dstate > SELSCAN_MAX_DSTATE) return SELSCAN_ERR_DSTATE_UNSUPPORTED;
    if (!mul_le(batch, seqlen, kMaxElems) || !mul_le(batch * seqlen, dim, kMaxElems) ||
        !mul_le(batch, dim, kMaxElems))
        return SELSCAN_ERR_BAD_DIM;
    if (conv_width < 0 || conv_width > kMaxConv) return SELSCAN_ERR_BAD_DIM;
    if (dstate > kMaxN && batch > 65535) return SELSCAN_ERR_BAD_DIM;  // a grid dimension
    if (conv_width > 0 && dim > 0 && !conv_w) return SELSCAN_ERR_NULL_ARG;
    if (misaligned(conv_w, 4) || misaligned(conv_b, 4) || misaligned(conv_init, 4))
        return SELSCAN_ERR_MISALIGNED;
    // A tensor with zero elements may be passed as NULL.
    const bool has_tokens = batch * seqlen * dim > 0;
    if (has_tokens && (!x || !delta || !y || !B || !C)) return SELSCAN_ERR_NULL_ARG;
    if (dim > 0 && !A) return SELSCAN_ERR_NULL_ARG;
    const size_t es = dtype == SELSCAN_F32 ? 4 : 2;
    if (misaligned(x, es) || misaligned(delta, es) || misaligned(z, es) ||
        misaligned(B, es) || misaligned(C, es) || misaligned(y, es) ||
        misaligned(A, 4) || misaligned(D, 4) || misaligned(delta_bias, 4) ||
        misaligned(final_state, 4) || misaligned(h0, 4))
        return SELSCAN_ERR_MISALIGNED;
    const size_t nx = (size_t)(batch * seqlen * dim) * es;
    const size_t nbc = (size_t)(batch * seqlen * dstate) * es;
    const size_t ns = (size_t)(batch * dim * dstate) * sizeof(float);
    const size_t nci = (size_t)(batch * dim) * (kMaxConv - 1) * sizeof(float);
    if (overlaps(y, nx, x, nx) || overlaps(y, nx, delta, nx) || overlaps(y, nx, z, nx) ||
        overlaps(y, nx, B, nbc) || overlaps(y, nx, C, nbc) || overlaps(y, nx, h0, ns) ||
        (conv_width > 0 && overlaps(y, nx, conv_init, nci)))
        return SELSCAN_ERR_ALIAS;
    // the final state may overwrite the initial state in place, but not partly
    if (h0 && final_state && h0 != final_state && overlaps(h0, ns, final_state, ns))
        return SELSCAN_ERR_ALIAS;

    if (batch == 0 || dim == 0) {
        *done = true;
        return SELSCAN_OK;
    }
    if (seqlen == 0) {
        *done = true;
        if (final_state && final_state != h0) {
            // no token: the final state is the initial one
            cudaError_t e = h0 ? cudaMemcpyAsync(final_state, h0, ns, cudaMemcpyDeviceToDevice,
                                                 stream)
                               : cudaMemsetAsync(final_state, 0, ns, stream);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return SELSCAN_OK;
    }

    const bool aligned = !misaligned(x, 16) && !misaligned(delta, 16) && !misaligned(z, 16) &&
                         !misaligned(B, 16) && !misaligned(C, 16) && !misaligned(y, 16);
    plan_for_sizes(batch, seqlen, dim, dstate, dtype, aligned, plan);
    plan->x = x;
    plan->delta = delta;
    plan->z = z;

    ScanParams &g = plan->gp;
    g.x = x; g.delta = delta; g.z = z; g.B = B; g.C = C;
    g.A = A; g.Dskip = D; g.delta_bias = delta_bias;
    g.y = y; g.final_state = final_state; g.h0 = h0;
    g.conv_w = conv_width > 0 ? conv_w : nullptr;
    g.conv_b = conv_width > 0 ? conv_b : nullptr;
    g.conv_init = conv_width > 0 ? conv_init : nullptr;
    g.conv_width = conv_width;
    g.zoh = zoh ? 1 : 0;
    g.batch = batch; g.seqlen = seqlen; g.dim = dim; g.dstate = (int)dstate;
    g.softplus = softplus_flag ? 1 : 0;
    g.ws_P = g.ws_H = nullptr;
    if (plan->tma) {
        TmaScanParams &t = plan->tp;
        t.B = B; t.C = C; t.A = A; t.Dskip = D; t.delta_bias = delta_bias;
        t.y = y; t.final_state = final_state; t.h0 = h0;
        t.conv_w = g.conv_w; t.conv_b = g.conv_b; t.conv_init = g.conv_init;
        t.conv_width = conv_width;
        t.zoh = zoh ? 1 : 0;
        t.batch = batch; t.seqlen = seqlen; t.dim = dim; t.dstate = (int)dstate;
        t.softplus = g.softplus;
        const int64_t units = t.groups * t.nchunks;
        if (units >= INT32_MAX) return SELSCAN_ERR_BAD_DIM;
        // carry kernel parameters (chunked plan)
        g.nchunks = t.nchunks;
        g.chunk_len = t.chunk_len;
    } else if (!mul_le(batch * g.nchunks, g.ntiles, INT32_MAX)) {
        return SELSCAN_ERR_BAD_DIM;
    }
    return SELSCAN_OK;
}

cudaError_t fwd_run(FwdPlan *plan, void *ws, cudaStream_t stream) {
    if (plan->wide) return launch_scan_wide(plan->gp, plan->bf16, stream);
    if (!plan->tma) {
        ScanParams &g = plan->gp;
        if (g.nchunks > 1) {
            const size_t half = plan->ws_bytes / 2;
            g.ws_P = static_cast<float *>(ws);
            g.ws_H = reinterpret_cast<float *>(static_cast<char *>(ws) + half);
        }
        return launch_scan(g, plan->bf16, stream);
    }
    TmaScanParams &t = plan->tp;
    char *w = static_cast<char *>(ws);
    cudaError_t e = cudaMemsetAsync(w, 0, plan->ws_clear, stream);
    if (e != cudaSuccess) return e;
    int *tickets = reinterpret_cast<int *>(w);
    t.abort_all = tickets + 2;
    if (t.mode == kModeSeq) {
        t.ticket = tickets;
        t.flags = reinterpret_cast<int *>(w + 256);
        t.ws_state = reinterpret_cast<float *>(w + plan->ws_clear);
        t.units = (int)(t.groups * t.nchunks);
        return launch_scan_tma(t, plan->bf16, plan->x, plan->delta, plan->z, stream);
    }
    const size_t half = (plan->ws_bytes - 256) / 2;
    t.ws_P = reinterpret_cast<float *>(w + 256);
    t.ws_H = reinterpret_cast<float *>(w + 256 + half);
    // pass 1: aggregates of every chunk but the last
    t.mode = kModeAgg;
    t.ticket = tickets;
    t.units = (int)(t.groups * (t.nchunks - 1));
    e = launch_scan_tma(t, plan->bf16, plan->x, plan->delta, plan->z, stream);
    if (e != cudaSuccess) return e;
    ScanParams &g = plan->gp;
    g.ws_P = t.ws_P;
    g.ws_H = t.ws_H;
    e = launch_carry(g, stream);
    if (e != cudaSuccess) return e;
    // pass 2: every chunk from its carried-in state
    t.mode = kModeRescan;
    t.ticket = tickets + 1;
    t.units = (int)(t.groups * t.nchunks);
    e = launch_scan_tma(t, plan->bf16, plan->x, plan->delta, plan->z, stream);
    t.mode = kModeAgg;
    return e;
}

}  // namespace selscan

namespace {

struct BwdLayout {
    size_t ckpt, part, pA, pD, pbias, dxc, pconv, acc, tma, tma_bytes, total;
};

// 16-state groups the gradient walks per chain
int64_t bwd_groups(int64_t dstate) { return (dstate + 15) / 16; }

int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

BwdLayout bwd_layout(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                     bool conv = false) {
    const int64_t K = ceil_div64(seqlen, selscan::bwd_tile_tokens());
    const int64_t ct = ceil_div64(dim, selscan::bwd_tile_channels());
    const int64_t G = bwd_groups(dstate);
    BwdLayout l;
    size_t off = 0;
    l.ckpt = off;  // every group's checkpoints (the groups run side by side)
    off = align256(off + (size_t)(G * batch * K * dim) * selscan::kMaxN * sizeof(float));
    l.part = off;
    off = align256(off + (size_t)(G * batch * ct * seqlen) * 2 * selscan::kMaxN * sizeof(float));
    l.pA = off;
    off = align256(off + (size_t)(G * batch * dim) * selscan::kMaxN * sizeof(float));
    l.pD = off;
    off = align256(off + (size_t)(batch * dim) * sizeof(float));
    l.pbias = off;
    off = align256(off + (size_t)(batch * dim) * sizeof(float));
    l.dxc = l.pconv = off;
    if (conv) {  // the conv output's gradient and the conv-gradient partials
        const int64_t ctt = ceil_div64(seqlen, selscan::bwd_conv_tile_tokens());
        l.dxc = off;
        off = align256(off + (size_t)(batch * seqlen * dim) * sizeof(float));
        l.pconv = off;
        off = align256(off + (size_t)(batch * ctt * dim) * (selscan::kMaxConv + 1) *
                                 sizeof(float));
    }
    l.acc = off;
    if (G > 1) off = align256(off + 3 * (size_t)(G * batch * seqlen * dim) * sizeof(float));
    // the one-pass TMA plan's counters, flags and handed-over states, for the
    // checkpoint pass of the forward kernel (one 16-state group, no conv)
    l.tma = off;
    l.tma_bytes = 0;
    if (G == 1 && !conv && dim >= selscan::tma_tile_channels()) {
        const int64_t groups = batch * ceil_div64(dim, selscan::tma_tile_channels());
        l.tma_bytes = align256(256 + 4 * 8 * (size_t)groups) +
                      (size_t)groups * selscan::tma_tile_channels() * selscan::kMaxN * sizeof(float);
        off = align256(off + l.tma_bytes);
    }
    l.total = off;
    return l;
}

struct Span {
    const void *p;
    size_t n;
};

bool any_overlap(const Span *outs, int no, const Span *ins, int ni) {
    for (int i = 0; i < no; ++i) {
        for (int j = 0; j < ni; ++j)
            if (overlaps(outs[i].p, outs[i].n, ins[j].p, ins[j].n)) return true;
        for (int j = i + 1; j < no; ++j)
            if (overlaps(outs[i].p, outs[i].n, outs[j].p, outs[j].n)) return true;
    }
    return false;
}

}  // namespace

extern "C" {

const char *selscan_status_string(int status) {
    switch (status) {
    case SELSCAN_OK: return "ok";
    case SELSCAN_ERR_NULL_ARG: return "a required pointer argument is NULL";
    case SELSCAN_ERR_BAD_DIM: return "a size argument is negative or too large";
    case SELSCAN_ERR_BAD_DTYPE: return "dtype is not SELSCAN_F32 or SELSCAN_BF16";
    case SELSCAN_ERR_MISALIGNED: return "a pointer is not aligned to its element size";
    case SELSCAN_ERR_DSTATE_UNSUPPORTED: return "dstate must be between 1 and 16";
    case SELSCAN_ERR_CUDA: return "a CUDA runtime call failed (see selscan_last_cuda_error)";
    case SELSCAN_ERR_ALIAS: return "an output overlaps an input";
    case SELSCAN_ERR_WORKSPACE:
        return "the sizes need more chunk workspace than the static scratch array holds";
    default: return "unknown status";
    }
}

const char *selscan_last_cuda_error(void) {
    return g_last_cuda_error == cudaSuccess ? "no error"
                                            : cudaGetErrorString(g_last_cuda_error);
}

}  // extern "C"

namespace {

int fwd_entry(const void *x, const void *delta, const float *A, const void *B, const void *C,
              const float *D, const void *z, const float *delta_bias, int softplus_flag,
              const float *h0, const float *conv_w, const float *conv_b,
              const float *conv_init, int conv_width, int zoh, void *y, float *final_state,
              int64_t batch, int64_t seqlen, int64_t dim,
              int64_t dstate, selscan_dtype_t dtype, selscan_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    selscan::FwdPlan plan;
    bool done = false;
    const int st = selscan::fwd_setup(x, delta, A, B, C, D, z, delta_bias, softplus_flag, h0,
                                      conv_w, conv_b, conv_init, conv_width, zoh, y,
                                      final_state, batch,
                                      seqlen, dim, dstate, dtype, stream, &plan, &done);
    if (st != SELSCAN_OK || done) return st;
    void *ws = nullptr;
    if (plan.ws_bytes > 0) {
        cudaError_t e = cudaMallocAsync(&ws, plan.ws_bytes, stream);
        if (e != cudaSuccess) return selscan::cuda_fail(e);
    }
    cudaError_t e = selscan::fwd_run(&plan, ws, stream);
    if (ws) {
        cudaError_t ef = cudaFreeAsync(ws, stream);
        if (e == cudaSuccess) e = ef;
    }
    return e == cudaSuccess ? SELSCAN_OK : selscan::cuda_fail(e);
}

}  // namespace

extern "C" {

int selscan_fwd(const void *x, const void *delta, const float *A, const void *B,
                const void *C, const float *D, const void *z, const float *delta_bias,
                int softplus_flag, void *y, float *final_state, int64_t batch,
                int64_t seqlen, int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                selscan_stream_t stream) {
    return fwd_entry(x, delta, A, B, C, D, z, delta_bias, softplus_flag, nullptr, nullptr,
                     nullptr, nullptr, 0, 0, y, final_state, batch, seqlen, dim, dstate, dtype,
                     stream);
}

int selscan_fwd_from_state(const void *x, const void *delta, const float *A, const void *B,
                           const void *C, const float *D, const void *z,
                           const float *delta_bias, int softplus_flag,
                           const float *initial_state, void *y, float *final_state,
                           int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                           selscan_dtype_t dtype, selscan_stream_t stream) {
    return fwd_entry(x, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state,
                     nullptr, nullptr, nullptr, 0, 0, y, final_state, batch, seqlen, dim,
                     dstate, dtype, stream);
}

int selscan_fwd_conv(const void *x_in, const float *conv_weight, const float *conv_bias,
                     int conv_width, const float *conv_init, const void *delta, const float *A, const void *B,
                     const void *C, const float *D, const void *z, const float *delta_bias,
                     int softplus_flag, const float *initial_state, void *y,
                     float *final_state, int64_t batch, int64_t seqlen, int64_t dim,
                     int64_t dstate, selscan_dtype_t dtype, selscan_stream_t stream) {
    if (conv_width < 1) return SELSCAN_ERR_BAD_DIM;
    return fwd_entry(x_in, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state,
                     conv_weight, conv_bias, conv_init, conv_width, 0, y, final_state, batch,
                     seqlen, dim, dstate, dtype, stream);
}

int selscan_fwd_ex(const void *x, const void *delta, const float *A, const void *B,
                   const void *C, const float *D, const void *z, const float *delta_bias,
                   int softplus_flag, const selscan_fwd_options_t *options, void *y,
                   float *final_state, int64_t batch, int64_t seqlen, int64_t dim,
                   int64_t dstate, selscan_dtype_t dtype, selscan_stream_t stream) {
    selscan_fwd_options_t o{};
    if (options) o = *options;
    if (o.bbar_mode != SELSCAN_BBAR_DELTA && o.bbar_mode != SELSCAN_BBAR_ZOH)
        return SELSCAN_ERR_BAD_DIM;
    return fwd_entry(x, delta, A, B, C, D, z, delta_bias, softplus_flag, o.initial_state,
                     o.conv_weight, o.conv_bias, o.conv_init, o.conv_width,
                     o.bbar_mode == SELSCAN_BBAR_ZOH, y, final_state, batch, seqlen, dim,
                     dstate, dtype, stream);
}

int selscan_fwd_plan(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                     int64_t *chunks, int64_t *launches, int64_t *workspace_bytes_out) {
    if (batch < 0 || seqlen < 0 || dim < 0) return SELSCAN_ERR_BAD_DIM;
    if (dstate < 1 || dstate > SELSCAN_MAX_DSTATE) return SELSCAN_ERR_DSTATE_UNSUPPORTED;
    if (!mul_le(batch, seqlen, kMaxElems) || !mul_le(batch * seqlen, dim, kMaxElems))
        return SELSCAN_ERR_BAD_DIM;
    int64_t nc = 0, nl = 0, ws = 0;
    if (batch > 0 && dim > 0 && seqlen > 0) {
        selscan::FwdPlan plan;
        selscan::plan_for_sizes(batch, seqlen, dim, dstate, SELSCAN_BF16, true, &plan);
        nc = plan.chunks;
        nl = plan.launches;
        ws = (int64_t)plan.ws_bytes;
    }
    if (chunks) *chunks = nc;
    if (launches) *launches = nl;
    if (workspace_bytes_out) *workspace_bytes_out = ws;
    return SELSCAN_OK;
}

int64_t selscan_bwd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t dim,
                                    int64_t dstate) {
    if (batch <= 0 || seqlen <= 0 || dim <= 0 || dstate < 1 || dstate > SELSCAN_MAX_DSTATE_BWD)
        return 0;
    if (!mul_le(batch, seqlen, kMaxElems) || !mul_le(batch * seqlen, dim, kMaxElems))
        return 0;
    return (int64_t)bwd_layout(batch, seqlen, dim, dstate).total;
}

}  // extern "C"

namespace {

// Shared by selscan_bwd (workspace == NULL: allocated on the stream) and
// selscan_bwd_workspace (the caller's workspace).
int bwd_entry(const void *x, const void *delta, const float *A, const void *B, const void *C,
              const float *D, const void *z, const float *delta_bias, int softplus_flag,
              const void *dy, const float *dfinal_state, void *dx, void *ddelta, float *dA,
              float *dB, float *dC, float *dD, void *dz, float *ddelta_bias, int64_t batch,
              int64_t seqlen, int64_t dim, int64_t dstate, selscan_dtype_t dtype,
              const float *h0, float *dh0, const float *conv_w,
              const float *conv_b, int conv_width, float *dconv_w, float *dconv_b, void *workspace, int64_t workspace_bytes,
              bool allocate,
              selscan_stream_t stream_, int zoh = 0) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (dtype != SELSCAN_F32 && dtype != SELSCAN_BF16) return SELSCAN_ERR_BAD_DTYPE;
    if (batch < 0 || seqlen < 0 || dim < 0 || batch > 65535) return SELSCAN_ERR_BAD_DIM;
    if (dstate < 1 || dstate > SELSCAN_MAX_DSTATE_BWD) return SELSCAN_ERR_DSTATE_UNSUPPORTED;
    if (!mul_le(batch, seqlen, kMaxElems) || !mul_le(batch * seqlen, dim, kMaxElems) ||
        !mul_le(batch, dim, kMaxElems))
        return SELSCAN_ERR_BAD_DIM;
    const bool has_tokens = batch * seqlen * dim > 0;
    const bool has_bc = batch * seqlen > 0;
    if (has_tokens && (!x || !delta || !dy || !dx || !ddelta || (z && !dz)))
        return SELSCAN_ERR_NULL_ARG;
    if (has_bc && (!B || !C || !dB || !dC)) return SELSCAN_ERR_NULL_ARG;
    if (dim > 0 && (!A || !dA)) return SELSCAN_ERR_NULL_ARG;
    const size_t es = dtype == SELSCAN_F32 ? 4 : 2;
    if (misaligned(x, es) || misaligned(delta, es) || misaligned(z, es) ||
        misaligned(B, es) || misaligned(C, es) || misaligned(dy, es) || misaligned(dx, es) ||
        misaligned(ddelta, es) || misaligned(dz, es) || misaligned(A, 4) ||
        misaligned(D, 4) || misaligned(delta_bias, 4) || misaligned(dfinal_state, 4) ||
        misaligned(dA, 4) || misaligned(dB, 4) || misaligned(dC, 4) || misaligned(dD, 4) ||
        misaligned(ddelta_bias, 4) || misaligned(workspace, 256) || misaligned(h0, 4) ||
        misaligned(dh0, 4) || misaligned(conv_w, 4) || misaligned(conv_b, 4) ||
        misaligned(dconv_w, 4) || misaligned(dconv_b, 4))
        return SELSCAN_ERR_MISALIGNED;
    if (conv_width < 0 || conv_width > selscan::kMaxConv) return SELSCAN_ERR_BAD_DIM;
    if (conv_width > 0 && dim > 0 && (!conv_w || !dconv_w)) return SELSCAN_ERR_NULL_ARG;
    const size_t nx = (size_t)(batch * seqlen * dim) * es;
    const size_t nbc = (size_t)(batch * seqlen * dstate) * es;
    const size_t nbcf = (size_t)(batch * seqlen * dstate) * 4;
    const size_t na = (size_t)(dim * dstate) * 4, nd = (size_t)dim * 4;
    const size_t ns = (size_t)(batch * dim * dstate) * 4;
    const size_t ncw = (size_t)(dim * conv_width) * 4;
    const Span outs[] = {{dx, nx}, {ddelta, nx}, {dz, z ? nx : 0}, {dA, na}, {dB, nbcf},
                         {dC, nbcf}, {dD, nd}, {ddelta_bias, nd}, {dh0, ns},
                         {dconv_w, ncw}, {dconv_b, conv_width > 0 ? nd : 0}};
    const Span ins[] = {{x, nx}, {delta, nx}, {z, nx}, {dy, nx}, {B, nbc}, {C, nbc},
                        {A, na}, {D, nd}, {delta_bias, nd}, {dfinal_state, ns}, {h0, ns},
                        {conv_w, ncw}, {conv_b, conv_width > 0 ? nd : 0}};
    if (any_overlap(outs, 11, ins, 13)) return SELSCAN_ERR_ALIAS;

    if (!has_tokens) {
        // no token reaches the loss through a channel: the float32 gradients are 0
        cudaError_t e = cudaSuccess;
        if (e == cudaSuccess && has_bc) e = cudaMemsetAsync(dB, 0, nbcf, stream);
        if (e == cudaSuccess && has_bc) e = cudaMemsetAsync(dC, 0, nbcf, stream);
        if (e == cudaSuccess && dim > 0) e = cudaMemsetAsync(dA, 0, na, stream);
        if (e == cudaSuccess && dim > 0 && dD) e = cudaMemsetAsync(dD, 0, nd, stream);
        if (e == cudaSuccess && dim > 0 && ddelta_bias)
            e = cudaMemsetAsync(ddelta_bias, 0, nd, stream);
        // no token: the final state is the initial one
        if (e == cudaSuccess && conv_width > 0 && dim > 0)
            e = cudaMemsetAsync(dconv_w, 0, ncw, stream);
        if (e == cudaSuccess && conv_width > 0 && dconv_b && dim > 0)
            e = cudaMemsetAsync(dconv_b, 0, nd, stream);
        if (e == cudaSuccess && dh0 && ns > 0)
            e = dfinal_state ? cudaMemcpyAsync(dh0, dfinal_state, ns, cudaMemcpyDeviceToDevice,
                                               stream)
                             : cudaMemsetAsync(dh0, 0, ns, stream);
        return e == cudaSuccess ? SELSCAN_OK : selscan::cuda_fail(e);
    }

    const BwdLayout l = bwd_layout(batch, seqlen, dim, dstate, conv_width > 0);
    if (!allocate) {
        if (!workspace) return SELSCAN_ERR_NULL_ARG;
        if (workspace_bytes < (int64_t)l.total) return SELSCAN_ERR_WORKSPACE;
        const Span wsp[] = {{workspace, l.total}};
        if (any_overlap(wsp, 1, outs, 11) || any_overlap(wsp, 1, ins, 13))
            return SELSCAN_ERR_ALIAS;
    }
    selscan::BwdParams p{};
    p.x = x; p.delta = delta; p.z = z; p.B = B; p.C = C; p.dy = dy;
    p.A = A; p.Dskip = D; p.delta_bias = delta_bias; p.dfinal = dfinal_state;
    p.h0 = h0; p.dh0 = dh0;
    p.conv_width = conv_width;
    p.conv_w = conv_width > 0 ? conv_w : nullptr;
    p.conv_b = conv_width > 0 ? conv_b : nullptr;
    p.dconv_w = conv_width > 0 ? dconv_w : nullptr;
    p.dconv_b = conv_width > 0 ? dconv_b : nullptr;
    p.conv_tiles = (int)ceil_div64(seqlen, selscan::bwd_conv_tile_tokens());
    p.dx = dx; p.ddelta = ddelta; p.dz = dz;
    p.dA = dA; p.dB = dB; p.dC = dC; p.dD = dD; p.ddelta_bias = ddelta_bias;
    p.batch = batch; p.seqlen = seqlen; p.dim = dim; p.dstate = (int)dstate;
    p.softplus = softplus_flag ? 1 : 0;
    p.zoh = zoh ? 1 : 0;
    p.ktiles = (int)ceil_div64(seqlen, selscan::bwd_tile_tokens());
    p.ctiles = (int)ceil_div64(dim, selscan::bwd_tile_channels());
    if (!mul_le(p.ctiles, 1, INT32_MAX) || !mul_le(p.ktiles, 1, INT32_MAX))
        return SELSCAN_ERR_BAD_DIM;
    void *ws = workspace;
    cudaError_t e = cudaSuccess;
    if (allocate) {
        e = cudaMallocAsync(&ws, l.total, stream);
        if (e != cudaSuccess) return selscan::cuda_fail(e);
    }
    char *w = static_cast<char *>(ws);
    p.ckpt = reinterpret_cast<float *>(w + l.ckpt);
    p.part = reinterpret_cast<float *>(w + l.part);
    p.pA = reinterpret_cast<float *>(w + l.pA);
    p.pD = reinterpret_cast<float *>(w + l.pD);
    p.pbias = reinterpret_cast<float *>(w + l.pbias);
    p.groups = (int)bwd_groups(dstate);
    p.acc = p.groups > 1 ? reinterpret_cast<float *>(w + l.acc) : nullptr;
    p.dxc = conv_width > 0 ? reinterpret_cast<float *>(w + l.dxc) : nullptr;
    p.pconv = conv_width > 0 ? reinterpret_cast<float *>(w + l.pconv) : nullptr;
    // With the two-lane gradient kernel and the forward's one-pass TMA plan
    // both available, the TMA-staged forward kernel writes the checkpoints
    // (no y) and the gradient kernel skips its own forward sweep.
    const bool bf16 = dtype == SELSCAN_BF16;
    if (l.tma_bytes > 0 && selscan::bwd_pairs_supported(p, bf16) &&
        !env_flag("SELSCAN_BWD_OWN_SWEEP")) {
        const bool aligned = !misaligned(x, 16) && !misaligned(delta, 16) &&
                             !misaligned(B, 16) && !misaligned(C, 16);
        selscan::FwdPlan fp{};
        selscan::plan_for_sizes(batch, seqlen, dim, dstate, dtype, aligned, &fp);
        if (fp.tma && fp.tp.mode == selscan::kModeSeq && fp.ws_bytes <= l.tma_bytes) {
            selscan::TmaScanParams t = fp.tp;
            t.B = B; t.C = C; t.A = A; t.Dskip = D; t.delta_bias = delta_bias;
            t.y = nullptr; t.final_state = nullptr; t.h0 = h0;
            t.conv_w = t.conv_b = t.conv_init = nullptr;
            t.conv_width = 0;
            t.zoh = 0;
            t.batch = batch; t.seqlen = seqlen; t.dim = dim; t.dstate = (int)dstate;
            t.softplus = p.softplus;
            t.mode = selscan::kModeCkpt;
            t.ckpt = p.ckpt;
            t.ck_tiles = p.ktiles;
            char *tw = w + l.tma;
            e = cudaMemsetAsync(tw, 0, fp.ws_clear, stream);
            int *tickets = reinterpret_cast<int *>(tw);
            t.ticket = tickets;
            t.abort_all = tickets + 2;
            t.flags = reinterpret_cast<int *>(tw + 256);
            t.ws_state = reinterpret_cast<float *>(tw + fp.ws_clear);
            t.units = (int)(t.groups * t.nchunks);
            if (e == cudaSuccess) e = selscan::launch_scan_tma(t, bf16, x, delta, nullptr, stream);
            p.ckpt_ready = e == cudaSuccess ? 1 : 0;
            // a tensor map the driver refused: nothing launched, the gradient
            // kernel does its own forward sweep
            if (e == cudaErrorInvalidValue) e = cudaSuccess;
        }
    }
    if (e == cudaSuccess) e = selscan::launch_scan_bwd(p, bf16, stream);
    if (allocate) {
        cudaError_t ef = cudaFreeAsync(ws, stream);
        if (e == cudaSuccess) e = ef;
    }
    return e == cudaSuccess ? SELSCAN_OK : selscan::cuda_fail(e);
}

}  // namespace

extern "C" {

int selscan_bwd(const void *x, const void *delta, const float *A, const void *B, const void *C,
                const float *D, const void *z, const float *delta_bias, int softplus_flag,
                const void *dy, const float *dfinal_state, void *dx, void *ddelta, float *dA,
                float *dB, float *dC, float *dD, void *dz, float *ddelta_bias, int64_t batch,
                int64_t seqlen, int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                selscan_stream_t stream) {
    return bwd_entry(x, delta, A, B, C, D, z, delta_bias, softplus_flag, dy, dfinal_state, dx,
                     ddelta, dA, dB, dC, dD, dz, ddelta_bias, batch, seqlen, dim, dstate, dtype,
                     nullptr, nullptr, nullptr, nullptr, 0, nullptr, nullptr, nullptr, 0, true,
                     stream);
}

int selscan_bwd_workspace(const void *x, const void *delta, const float *A, const void *B,
                          const void *C, const float *D, const void *z,
                          const float *delta_bias, int softplus_flag, const void *dy,
                          const float *dfinal_state, void *dx, void *ddelta, float *dA,
                          float *dB, float *dC, float *dD, void *dz, float *ddelta_bias,
                          int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                          selscan_dtype_t dtype, void *workspace, int64_t workspace_bytes,
                          selscan_stream_t stream) {
    return bwd_entry(x, delta, A, B, C, D, z, delta_bias, softplus_flag, dy, dfinal_state, dx,
                     ddelta, dA, dB, dC, dD, dz, ddelta_bias, batch, seqlen, dim, dstate, dtype,
                     nullptr, nullptr, nullptr, nullptr, 0, nullptr, nullptr, workspace,
                     workspace_bytes, false, stream);
}

int selscan_bwd_from_state(const void *x, const void *delta, const float *A, const void *B,
                           const void *C, const float *D, const void *z,
                           const float *delta_bias, int softplus_flag,
                           const float *initial_state, const void *dy,
                           const float *dfinal_state, void *dx, void *ddelta, float *dA,
                           float *dB, float *dC, float *dD, void *dz, float *ddelta_bias,
                           float *dinitial_state, int64_t batch, int64_t seqlen, int64_t dim,
                           int64_t dstate, selscan_dtype_t dtype, void *workspace,
                           int64_t workspace_bytes, selscan_stream_t stream) {
    return bwd_entry(x, delta, A, B, C, D, z, delta_bias, softplus_flag, dy, dfinal_state, dx,
                     ddelta, dA, dB, dC, dD, dz, ddelta_bias, batch, seqlen, dim, dstate, dtype,
                     initial_state, dinitial_state, nullptr, nullptr, 0, nullptr, nullptr,
                     workspace, workspace_bytes, workspace == nullptr, stream);
}

int selscan_bwd_conv(const void *x_in, const float *conv_weight, const float *conv_bias,
                     int conv_width, const void *delta, const float *A, const void *B,
                     const void *C, const float *D, const void *z, const float *delta_bias,
                     int softplus_flag, const float *initial_state, const void *dy,
                     const float *dfinal_state, void *dx_in, void *ddelta, float *dA,
                     float *dB, float *dC, float *dD, void *dz, float *ddelta_bias,
                     float *dinitial_state, float *dconv_weight, float *dconv_bias,
                     int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                     selscan_dtype_t dtype, void *workspace, int64_t workspace_bytes,
                     selscan_stream_t stream) {
    if (conv_width < 1) return SELSCAN_ERR_BAD_DIM;
    return bwd_entry(x_in, delta, A, B, C, D, z, delta_bias, softplus_flag, dy, dfinal_state,
                     dx_in, ddelta, dA, dB, dC, dD, dz, ddelta_bias, batch, seqlen, dim, dstate,
                     dtype, initial_state, dinitial_state, conv_weight, conv_bias, conv_width,
                     dconv_weight, dconv_bias, workspace, workspace_bytes,
                     workspace == nullptr, stream);
}

int selscan_bwd_ex(const void *x, const void *delta, const float *A, const void *B,
                   const void *C, const float *D, const void *z, const float *delta_bias,
                   int softplus_flag, const void *dy, const float *dfinal_state,
                   const selscan_bwd_options_t *options, void *dx, void *ddelta, float *dA,
                   float *dB, float *dC, float *dD, void *dz, float *ddelta_bias, int64_t batch,
                   int64_t seqlen, int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                   void *workspace, int64_t workspace_bytes, selscan_stream_t stream) {
    selscan_bwd_options_t o{};
    if (options) o = *options;
    if (o.bbar_mode != SELSCAN_BBAR_DELTA && o.bbar_mode != SELSCAN_BBAR_ZOH)
        return SELSCAN_ERR_BAD_DIM;
    if (o.conv_width < 0) return SELSCAN_ERR_BAD_DIM;
    return bwd_entry(x, delta, A, B, C, D, z, delta_bias, softplus_flag, dy, dfinal_state, dx,
                     ddelta, dA, dB, dC, dD, dz, ddelta_bias, batch, seqlen, dim, dstate, dtype,
                     o.initial_state, o.dinitial_state, o.conv_weight, o.conv_bias,
                     o.conv_width, o.dconv_weight, o.dconv_bias, workspace, workspace_bytes,
                     workspace == nullptr, stream, o.bbar_mode == SELSCAN_BBAR_ZOH);
}

int64_t selscan_bwd_conv_workspace_bytes(int64_t batch, int64_t seqlen, int64_t dim,
                                         int64_t dstate) {
    if (batch <= 0 || seqlen <= 0 || dim <= 0 || dstate < 1 || dstate > SELSCAN_MAX_DSTATE_BWD)
        return 0;
    if (!mul_le(batch, seqlen, kMaxElems) || !mul_le(batch * seqlen, dim, kMaxElems))
        return 0;
    return (int64_t)bwd_layout(batch, seqlen, dim, dstate, true).total;
}

}  // extern "C"

namespace {

struct SsdLayout {
    size_t ypart, cstate, decay, sin, total;
};

SsdLayout ssd_layout(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim) {
    const int64_t nc = ceil_div64(seqlen, selscan::ssd_chunk_tokens());
    const size_t per = (size_t)selscan::ssd_max_dstate() * selscan::ssd_max_headdim();
    SsdLayout l;
    size_t off = 0;
    l.ypart = off;
    off = align256(off + (size_t)(batch * seqlen * nheads * headdim) * sizeof(float));
    l.cstate = off;
    off = align256(off + (size_t)(batch * nheads * nc) * per * sizeof(float));
    l.decay = off;
    off = align256(off + (size_t)(batch * nheads * nc) * sizeof(float));
    l.sin = off;
    off = align256(off + (size_t)(batch * nheads * nc) * per * sizeof(float));
    l.total = off;
    return l;
}

}  // namespace

extern "C" {

int64_t selscan_ssd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t nheads,
                                    int64_t headdim, int64_t dstate) {
    if (batch <= 0 || seqlen <= 0 || nheads <= 0 || headdim <= 0 ||
        headdim > selscan::ssd_max_headdim() || dstate < 1 || dstate > selscan::ssd_max_dstate())
        return 0;
    if (!mul_le(batch, seqlen, kMaxElems) || !mul_le(batch * seqlen, nheads * headdim, kMaxElems))
        return 0;
    return (int64_t)ssd_layout(batch, seqlen, nheads, headdim).total;
}

int selscan_ssd_fwd(const void *x, const void *dt, const float *A, const void *B, const void *C,
                    const float *D, const void *z, const float *dt_bias, int softplus_flag,
                    const float *initial_state, void *y, float *final_state, int64_t batch,
                    int64_t seqlen, int64_t nheads, int64_t headdim, int64_t dstate,
                    selscan_dtype_t dtype, void *workspace, int64_t workspace_bytes,
                    selscan_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (dtype != SELSCAN_F32 && dtype != SELSCAN_BF16) return SELSCAN_ERR_BAD_DTYPE;
    if (batch < 0 || seqlen < 0 || nheads < 0 || batch > 65535 || nheads > 65535 ||
        headdim < 1 || headdim > selscan::ssd_max_headdim())
        return SELSCAN_ERR_BAD_DIM;
    if (dstate < 1 || dstate > selscan::ssd_max_dstate()) return SELSCAN_ERR_DSTATE_UNSUPPORTED;
    const int64_t dim = nheads * headdim;
    if (!mul_le(batch, seqlen, kMaxElems) || !mul_le(batch * seqlen, dim, kMaxElems) ||
        !mul_le(batch, dim * dstate, kMaxElems))
        return SELSCAN_ERR_BAD_DIM;
    const bool has_tokens = batch * seqlen * dim > 0;
    if (has_tokens && (!x || !dt || !A || !B || !C || !y)) return SELSCAN_ERR_NULL_ARG;
    const size_t es = dtype == SELSCAN_F32 ? 4 : 2;
    if (misaligned(x, es) || misaligned(dt, es) || misaligned(z, es) || misaligned(B, es) ||
        misaligned(C, es) || misaligned(y, es) || misaligned(A, 4) || misaligned(D, 4) ||
        misaligned(dt_bias, 4) || misaligned(initial_state, 4) || misaligned(final_state, 4) ||
        misaligned(workspace, 256))
        return SELSCAN_ERR_MISALIGNED;
    const size_t nx = (size_t)(batch * seqlen * dim) * es;
    const size_t ndt = (size_t)(batch * seqlen * nheads) * es;
    const size_t nbc = (size_t)(batch * seqlen * dstate) * es;
    const size_t ns = (size_t)(batch * dim * dstate) * sizeof(float);
    const Span outs[] = {{y, nx}, {final_state, ns}};
    const Span ins[] = {{x, nx}, {dt, ndt}, {z, nx}, {B, nbc}, {C, nbc}, {initial_state, ns}};
    if (any_overlap(outs, 2, ins, 6)) return SELSCAN_ERR_ALIAS;
    if (!has_tokens) {
        if (final_state && batch * dim > 0) {
            cudaError_t e = initial_state
                                ? cudaMemcpyAsync(final_state, initial_state, ns,
                                                  cudaMemcpyDeviceToDevice, stream)
                                : cudaMemsetAsync(final_state, 0, ns, stream);
            if (e != cudaSuccess) return selscan::cuda_fail(e);
        }
        return SELSCAN_OK;
    }
    const SsdLayout l = ssd_layout(batch, seqlen, nheads, headdim);
    void *ws = workspace;
    if (ws) {
        if (workspace_bytes < (int64_t)l.total) return SELSCAN_ERR_WORKSPACE;
        const Span wsp[] = {{ws, l.total}};
        if (any_overlap(wsp, 1, outs, 2) || any_overlap(wsp, 1, ins, 6)) return SELSCAN_ERR_ALIAS;
    } else {
        cudaError_t e = cudaMallocAsync(&ws, l.total, stream);
        if (e != cudaSuccess) return selscan::cuda_fail(e);
    }
    char *w = static_cast<char *>(ws);
    selscan::SsdParams p{};
    p.x = x; p.dt = dt; p.z = z; p.B = B; p.C = C;
    p.A = A; p.Dskip = D; p.dt_bias = dt_bias; p.h0 = initial_state;
    p.y = y; p.final_state = final_state;
    p.ypart = reinterpret_cast<float *>(w + l.ypart);
    p.chunk_state = reinterpret_cast<float *>(w + l.cstate);
    p.chunk_decay = reinterpret_cast<float *>(w + l.decay);
    p.state_in = reinterpret_cast<float *>(w + l.sin);
    p.batch = batch; p.seqlen = seqlen;
    p.nheads = (int)nheads; p.headdim = (int)headdim; p.dstate = (int)dstate;
    p.nchunks = (int)ceil_div64(seqlen, selscan::ssd_chunk_tokens());
    p.softplus = softplus_flag ? 1 : 0;
    p.vec_x = (headdim % 8 == 0) && !misaligned(x, 16) && !misaligned(y, 16) && !misaligned(z, 16);
    p.vec_bc = (dstate % 8 == 0) && !misaligned(B, 16) && !misaligned(C, 16);
    {
        cudaError_t es = selscan::device_status_address(&p.status);
        if (es != cudaSuccess) return selscan::cuda_fail(es);
    }
    cudaError_t e = selscan::launch_ssd(p, dtype == SELSCAN_BF16, stream);
    if (!workspace) {
        cudaError_t ef = cudaFreeAsync(ws, stream);
        if (e == cudaSuccess) e = ef;
    }
    return e == cudaSuccess ? SELSCAN_OK : selscan::cuda_fail(e);
}

int selscan_device_status(int *status, int clear) {
    if (!status) return SELSCAN_ERR_NULL_ARG;
    cudaError_t e = selscan::read_device_status(status, clear != 0);
    return e == cudaSuccess ? SELSCAN_OK : selscan::cuda_fail(e);
}

}  // extern "C"

namespace {

int step_entry(float *state, float *conv_state, const float *conv_w, const float *conv_b,
               int conv_width, int zoh, const void *x, const void *delta, const float *A,
               const void *B, const void *C, const float *D, const void *z,
               const float *delta_bias, int softplus_flag, void *y, int64_t batch, int64_t dim,
               int64_t dstate, selscan_dtype_t dtype, selscan_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (dtype != SELSCAN_F32 && dtype != SELSCAN_BF16) return SELSCAN_ERR_BAD_DTYPE;
    if (batch < 0 || dim < 0) return SELSCAN_ERR_BAD_DIM;
    if (dstate < 1 || dstate > SELSCAN_MAX_DSTATE) return SELSCAN_ERR_DSTATE_UNSUPPORTED;
    if (conv_width < 0 || conv_width > selscan::kMaxConv) return SELSCAN_ERR_BAD_DIM;
    if (batch * dim > 0 && (!state || !x || !delta || !A || !B || !C || !y))
        return SELSCAN_ERR_NULL_ARG;
    if (batch * dim > 0 && conv_width > 0 && (!conv_state || !conv_w))
        return SELSCAN_ERR_NULL_ARG;
    if (!mul_le(batch, dim, kMaxElems / 64)) return SELSCAN_ERR_BAD_DIM;
    const size_t es = dtype == SELSCAN_F32 ? 4 : 2;
    if (misaligned(x, es) || misaligned(delta, es) || misaligned(z, es) ||
        misaligned(B, es) || misaligned(C, es) || misaligned(y, es) ||
        misaligned(state, 4) || misaligned(A, 4) || misaligned(D, 4) ||
        misaligned(delta_bias, 4) || misaligned(conv_state, 4) || misaligned(conv_w, 4) ||
        misaligned(conv_b, 4))
        return SELSCAN_ERR_MISALIGNED;
    const size_t ny = (size_t)(batch * dim) * es;
    const size_t nbc = (size_t)(batch * dstate) * es;
    const size_t ns = (size_t)(batch * dim * dstate) * sizeof(float);
    const size_t ncs = conv_width > 0 ? (size_t)(batch * dim) * 3 * sizeof(float) : 0;
    if (overlaps(y, ny, x, ny) || overlaps(y, ny, delta, ny) || overlaps(y, ny, z, ny) ||
        overlaps(y, ny, B, nbc) || overlaps(y, ny, C, nbc) || overlaps(y, ny, state, ns) ||
        overlaps(y, ny, conv_state, ncs) || overlaps(conv_state, ncs, state, ns) ||
        overlaps(conv_state, ncs, x, ny))
        return SELSCAN_ERR_ALIAS;
    if (batch == 0 || dim == 0) return SELSCAN_OK;
    if (!mul_le(batch * dim, 4, (int64_t)INT32_MAX * 256)) return SELSCAN_ERR_BAD_DIM;

    selscan::StepParams p{};
    p.state = state; p.x = x; p.delta = delta; p.z = z; p.B = B; p.C = C;
    p.A = A; p.Dskip = D; p.delta_bias = delta_bias; p.y = y;
    p.conv_width = conv_width;
    p.conv_state = conv_width > 0 ? conv_state : nullptr;
    p.conv_w = conv_width > 0 ? conv_w : nullptr;
    p.conv_b = conv_width > 0 ? conv_b : nullptr;
    p.zoh = zoh ? 1 : 0;
    p.batch = batch; p.dim = dim; p.dstate = (int)dstate;
    p.softplus = softplus_flag ? 1 : 0;
    cudaError_t e = selscan::launch_state_update(p, dtype == SELSCAN_BF16, stream);
    return e == cudaSuccess ? SELSCAN_OK : selscan::cuda_fail(e);
}

}  // namespace

extern "C" {

int selscan_state_update(float *state, const void *x, const void *delta, const float *A,
                         const void *B, const void *C, const float *D, const void *z,
                         const float *delta_bias, int softplus_flag, void *y,
                         int64_t batch, int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                         selscan_stream_t stream) {
    return step_entry(state, nullptr, nullptr, nullptr, 0, 0, x, delta, A, B, C, D, z,
                      delta_bias, softplus_flag, y, batch, dim, dstate, dtype, stream);
}

int selscan_state_update_conv(float *state, float *conv_state, const void *x_in,
                              const float *conv_weight, const float *conv_bias, int conv_width,
                              const void *delta, const float *A, const void *B, const void *C,
                              const float *D, const void *z, const float *delta_bias,
                              int softplus_flag, void *y, int64_t batch, int64_t dim,
                              int64_t dstate, selscan_dtype_t dtype, selscan_stream_t stream) {
    if (conv_width < 1) return SELSCAN_ERR_BAD_DIM;
    return step_entry(state, conv_state, conv_weight, conv_bias, conv_width, 0, x_in, delta,
                      A, B, C, D, z, delta_bias, softplus_flag, y, batch, dim, dstate, dtype,
                      stream);
}

int selscan_state_update_ex(float *state, const void *x, const void *delta, const float *A,
                            const void *B, const void *C, const float *D, const void *z,
                            const float *delta_bias, int softplus_flag,
                            const selscan_step_options_t *options, void *y, int64_t batch,
                            int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                            selscan_stream_t stream) {
    selscan_step_options_t o{};
    if (options) o = *options;
    if (o.bbar_mode != SELSCAN_BBAR_DELTA && o.bbar_mode != SELSCAN_BBAR_ZOH)
        return SELSCAN_ERR_BAD_DIM;
    return step_entry(state, o.conv_state, o.conv_weight, o.conv_bias, o.conv_width,
                      o.bbar_mode == SELSCAN_BBAR_ZOH, x, delta, A, B, C, D, z, delta_bias,
                      softplus_flag, y, batch, dim, dstate, dtype, stream);
}

}  // extern "C"
