// api.cu -- the C ABI of libselscan (declared in include/selscan.h): argument
// validation, the launch plan, workspace handling and error reporting. Every
// step of the computation runs in the CUDA kernels of scan.cu and
// state_update.cu; this file only checks arguments and launches them.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include "selscan.h"
#include "selscan_device.cuh"

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

// Sequence split of one selscan_fwd call. Each (batch row, channel) chain is
// one thread; when there are too few chains to keep every SM busy, the
// sequence is split so that chains × chunks reaches a target of resident
// threads, each chunk at least kMinChunk tokens and a whole number of B/C
// tiles. SELSCAN_CHUNKS overrides the chunk count (tuning only).
struct Plan {
    int nchunks;
    int64_t chunk_len;
};

Plan plan_fwd(int64_t batch, int64_t seqlen, int64_t dim) {
    constexpr int64_t kMinChunk = 256;
    constexpr int64_t kSinglePassChains = 16384;
    const char *env = getenv("SELSCAN_CHUNKS");
    int64_t n = 0;
    if (env && *env) n = atoll(env);
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
    int64_t len = (seqlen + n - 1) / n;
    len = (len + tileT - 1) / tileT * tileT;
    if (len < 1) len = 1;
    Plan p;
    p.chunk_len = len;
    p.nchunks = seqlen > 0 ? (int)((seqlen + len - 1) / len) : 1;
    return p;
}

size_t workspace_bytes(int64_t batch, int64_t dim, int nchunks) {
    if (nchunks <= 1) return 0;
    return 2 * (size_t)(batch * nchunks * dim) * selscan::kMaxN * sizeof(float);
}

}  // namespace

namespace selscan {

int cuda_fail(cudaError_t e) {
    g_last_cuda_error = e;
    return SELSCAN_ERR_CUDA;
}

// Argument validation and launch plan shared by the selscan_fwd entry points.
// On SELSCAN_OK fills *p (workspace pointers left NULL) and *ws_bytes, the
// chunk workspace the plan needs; *done is set when no kernel has to run
// (empty sizes; for seqlen == 0 the final state has been cleared on stream).
int fwd_setup(const void *x, const void *delta, const float *A, const void *B,
              const void *C, const float *D, const void *z, const float *delta_bias,
              int softplus_flag, void *y, float *final_state, int64_t batch,
              int64_t seqlen, int64_t dim, int64_t dstate, int dtype,
              cudaStream_t stream, ScanParams *p, size_t *ws_bytes, bool *done) {
    *done = false;
    *ws_bytes = 0;
    if (dtype != SELSCAN_F32 && dtype != SELSCAN_BF16) return SELSCAN_ERR_BAD_DTYPE;
    if (batch < 0 || seqlen < 0 || dim < 0) return SELSCAN_ERR_BAD_DIM;
    if (dstate < 1 || dstate > SELSCAN_MAX_DSTATE) return SELSCAN_ERR_DSTATE_UNSUPPORTED;
    if (!mul_le(batch, seqlen, kMaxElems) || !mul_le(batch * seqlen, dim, kMaxElems) ||
        !mul_le(batch, dim, kMaxElems))
        return SELSCAN_ERR_BAD_DIM;
    // A tensor with zero elements may be passed as NULL.
    const bool has_tokens = batch * seqlen * dim > 0;
    if (has_tokens && (!x || !delta || !y || !B || !C)) return SELSCAN_ERR_NULL_ARG;
    if (dim > 0 && !A) return SELSCAN_ERR_NULL_ARG;
    const size_t es = dtype == SELSCAN_F32 ? 4 : 2;
    if (misaligned(x, es) || misaligned(delta, es) || misaligned(z, es) ||
        misaligned(B, es) || misaligned(C, es) || misaligned(y, es) ||
        misaligned(A, 4) || misaligned(D, 4) || misaligned(delta_bias, 4) ||
        misaligned(final_state, 4))
        return SELSCAN_ERR_MISALIGNED;
    const size_t nx = (size_t)(batch * seqlen * dim) * es;
    const size_t nbc = (size_t)(batch * seqlen * dstate) * es;
    if (overlaps(y, nx, x, nx) || overlaps(y, nx, delta, nx) || overlaps(y, nx, z, nx) ||
        overlaps(y, nx, B, nbc) || overlaps(y, nx, C, nbc))
        return SELSCAN_ERR_ALIAS;

    if (batch == 0 || dim == 0) {
        *done = true;
        return SELSCAN_OK;
    }
    if (seqlen == 0) {
        *done = true;
        if (final_state) {
            cudaError_t e = cudaMemsetAsync(final_state, 0,
                                            (size_t)(batch * dim * dstate) * sizeof(float),
                                            stream);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return SELSCAN_OK;
    }

    p->x = x; p->delta = delta; p->z = z; p->B = B; p->C = C;
    p->A = A; p->Dskip = D; p->delta_bias = delta_bias;
    p->y = y; p->final_state = final_state;
    p->batch = batch; p->seqlen = seqlen; p->dim = dim; p->dstate = (int)dstate;
    p->softplus = softplus_flag ? 1 : 0;
    const int64_t cpc = scan_channels_per_cta();
    p->ntiles = (int)((dim + cpc - 1) / cpc);
    const Plan plan = plan_fwd(batch, seqlen, dim);
    p->chunk_len = plan.chunk_len;
    p->nchunks = plan.nchunks;
    p->ws_P = p->ws_H = nullptr;
    if (!mul_le(batch * plan.nchunks, p->ntiles, INT32_MAX)) return SELSCAN_ERR_BAD_DIM;
    *ws_bytes = workspace_bytes(batch, dim, plan.nchunks);
    return SELSCAN_OK;
}

}  // namespace selscan

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
    case SELSCAN_ERR_ALIAS: return "the output y overlaps an input";
    case SELSCAN_ERR_WORKSPACE:
        return "the sizes need more chunk workspace than the static scratch array holds";
    default: return "unknown status";
    }
}

const char *selscan_last_cuda_error(void) {
    return g_last_cuda_error == cudaSuccess ? "no error"
                                            : cudaGetErrorString(g_last_cuda_error);
}

int selscan_fwd(const void *x, const void *delta, const float *A, const void *B,
                const void *C, const float *D, const void *z, const float *delta_bias,
                int softplus_flag, void *y, float *final_state, int64_t batch,
                int64_t seqlen, int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                selscan_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    selscan::ScanParams p{};
    size_t ws_bytes = 0;
    bool done = false;
    const int st = selscan::fwd_setup(x, delta, A, B, C, D, z, delta_bias, softplus_flag,
                                      y, final_state, batch, seqlen, dim, dstate, dtype,
                                      stream, &p, &ws_bytes, &done);
    if (st != SELSCAN_OK || done) return st;
    void *ws = nullptr;
    if (ws_bytes > 0) {
        cudaError_t e = cudaMallocAsync(&ws, ws_bytes, stream);
        if (e != cudaSuccess) return selscan::cuda_fail(e);
        p.ws_P = static_cast<float *>(ws);
        p.ws_H = reinterpret_cast<float *>(static_cast<char *>(ws) + ws_bytes / 2);
    }
    cudaError_t e = selscan::launch_scan(p, dtype == SELSCAN_BF16, stream);
    if (ws) {
        cudaError_t ef = cudaFreeAsync(ws, stream);
        if (e == cudaSuccess) e = ef;
    }
    return e == cudaSuccess ? SELSCAN_OK : selscan::cuda_fail(e);
}

int selscan_fwd_plan(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                     int64_t *chunks, int64_t *launches, int64_t *workspace_bytes_out) {
    if (batch < 0 || seqlen < 0 || dim < 0) return SELSCAN_ERR_BAD_DIM;
    if (dstate < 1 || dstate > SELSCAN_MAX_DSTATE) return SELSCAN_ERR_DSTATE_UNSUPPORTED;
    if (!mul_le(batch, seqlen, kMaxElems) || !mul_le(batch * seqlen, dim, kMaxElems))
        return SELSCAN_ERR_BAD_DIM;
    int64_t nc = 0, nl = 0;
    size_t ws = 0;
    if (batch > 0 && dim > 0 && seqlen > 0) {
        const Plan plan = plan_fwd(batch, seqlen, dim);
        nc = plan.nchunks;
        nl = plan.nchunks > 1 ? 3 : 1;
        ws = workspace_bytes(batch, dim, plan.nchunks);
    }
    if (chunks) *chunks = nc;
    if (launches) *launches = nl;
    if (workspace_bytes_out) *workspace_bytes_out = (int64_t)ws;
    return SELSCAN_OK;
}

int selscan_state_update(float *state, const void *x, const void *delta, const float *A,
                         const void *B, const void *C, const float *D, const void *z,
                         const float *delta_bias, int softplus_flag, void *y,
                         int64_t batch, int64_t dim, int64_t dstate, selscan_dtype_t dtype,
                         selscan_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (dtype != SELSCAN_F32 && dtype != SELSCAN_BF16) return SELSCAN_ERR_BAD_DTYPE;
    if (batch < 0 || dim < 0) return SELSCAN_ERR_BAD_DIM;
    if (dstate < 1 || dstate > SELSCAN_MAX_DSTATE) return SELSCAN_ERR_DSTATE_UNSUPPORTED;
    if (batch * dim > 0 && (!state || !x || !delta || !A || !B || !C || !y))
        return SELSCAN_ERR_NULL_ARG;
    if (!mul_le(batch, dim, kMaxElems / 64)) return SELSCAN_ERR_BAD_DIM;
    const size_t es = dtype == SELSCAN_F32 ? 4 : 2;
    if (misaligned(x, es) || misaligned(delta, es) || misaligned(z, es) ||
        misaligned(B, es) || misaligned(C, es) || misaligned(y, es) ||
        misaligned(state, 4) || misaligned(A, 4) || misaligned(D, 4) ||
        misaligned(delta_bias, 4))
        return SELSCAN_ERR_MISALIGNED;
    const size_t ny = (size_t)(batch * dim) * es;
    const size_t nbc = (size_t)(batch * dstate) * es;
    const size_t ns = (size_t)(batch * dim * dstate) * sizeof(float);
    if (overlaps(y, ny, x, ny) || overlaps(y, ny, delta, ny) || overlaps(y, ny, z, ny) ||
        overlaps(y, ny, B, nbc) || overlaps(y, ny, C, nbc) || overlaps(y, ny, state, ns))
        return SELSCAN_ERR_ALIAS;
    if (batch == 0 || dim == 0) return SELSCAN_OK;
    if (!mul_le(batch * dim, 4, (int64_t)INT32_MAX * 256)) return SELSCAN_ERR_BAD_DIM;

    selscan::StepParams p{};
    p.state = state; p.x = x; p.delta = delta; p.z = z; p.B = B; p.C = C;
    p.A = A; p.Dskip = D; p.delta_bias = delta_bias; p.y = y;
    p.batch = batch; p.dim = dim; p.dstate = (int)dstate;
    p.softplus = softplus_flag ? 1 : 0;
    cudaError_t e = selscan::launch_state_update(p, dtype == SELSCAN_BF16, stream);
    return e == cudaSuccess ? SELSCAN_OK : selscan::cuda_fail(e);
}

}  // extern "C"
