// ssd_params.cuh -- launch parameters and entry points of the scan with one
// scalar A per head in chunked matrix form (ssd.cu, ssd_tc.cu).
#pragma once

#include "selscan_device.cuh"

namespace selscan {

struct SsdParams {
    const void *x, *dt, *z, *B, *C;  // x, z [batch][seqlen][nheads·headdim]; dt [batch][seqlen][nheads]
    const float *A, *Dskip, *dt_bias;  // [nheads]
    const float *h0;                 // [batch][nheads·headdim][dstate] or NULL
    void *y;
    float *final_state;              // [batch][nheads·headdim][dstate] or NULL
    // workspace
    float *ypart;                    // [batch][seqlen][nheads·headdim]: each chunk's own output
    float *chunk_state;              // [batch][nheads][nchunks][128][64]: chunk states from zero
    float *chunk_decay;              // [batch][nheads][nchunks]
    float *state_in;                 // [batch][nheads][nchunks][128][64]: state entering each
                                     // chunk (float32 path), or per chunk the bfloat16 pair
                                     // (high, low) in MMA operand layout (tensor-core path)
    long long batch, seqlen;
    int nheads, headdim, dstate, nchunks;
    int softplus;
    int vec_x;                       // x, z, y rows allow 16-byte accesses (tensor-core path)
    int vec_bc;                      // B, C rows allow 16-byte accesses (tensor-core path)
    int *status;                     // the library's device error word
    int heads_per_cta;               // set by the launcher of the tensor-core state kernel
    int tma_bc;                      // tensor-core kernels: B and C tiles by TMA (set by the launchers)
};
// float32 I/O: the float32 chunk kernels; bfloat16 I/O: the tensor-core kernels.
cudaError_t launch_ssd(const SsdParams &p, bool bf16, cudaStream_t stream);
int ssd_chunk_tokens();  // chunk length of the float32 path (sizes the workspace)
int ssd_max_headdim();
int ssd_max_dstate();
// Tensor-core form for bfloat16 I/O (ssd_tc.cu): 128-token chunks.
bool ssd_tc_supported(int headdim, int dstate);
int ssd_tc_chunk_tokens();
cudaError_t launch_ssd_tc_state(const SsdParams &p, cudaStream_t stream);
cudaError_t launch_ssd_tc_carry(const SsdParams &p, cudaStream_t stream);
cudaError_t launch_ssd_tc_out(const SsdParams &p, cudaStream_t stream);

}  // namespace selscan
