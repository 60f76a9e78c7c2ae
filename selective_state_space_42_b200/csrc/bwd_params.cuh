// bwd_params.cuh -- launch parameters and host entry points of the gradient
// kernels (scan_bwd.cu).
#pragma once

#include "selscan_device.cuh"

namespace selscan {

// Gradient of the scan (scan_bwd.cu).
struct BwdParams {
    const void *x, *delta, *z, *B, *C, *dy;
    const float *A, *Dskip, *delta_bias, *dfinal;
    const float *h0;  // state before the first token (NULL: zero)
    float *dh0;       // its gradient (NULL: not written)
    const float *conv_w, *conv_b;  // causal conv in front (conv_width > 0)
    int conv_width;
    float *dxc;       // with the conv: gradient of the conv output, [batch][seqlen][dim]
    float *dconv_w, *dconv_b;      // conv gradients (outputs; dconv_b nullable)
    float *pconv;     // [batch][conv tiles][dim][kMaxConv + 1] conv-gradient partials
    int conv_tiles;   // token tiles of the conv-gradient kernel
    void *dx, *ddelta, *dz;
    float *dA, *dB, *dC, *dD, *ddelta_bias;  // outputs written by the reduction kernel
    // workspace
    float *ckpt;   // [groups][batch][ktiles][dim][16]: state of each 16-state group entering each token tile
    float *part;   // [groups][batch][ctiles][seqlen][32]: per channel tile, Σ over its channels
                   // of dB (0..15), dC (16..31) of the group's states; with part_lane_order
                   // value 16·c + n (c = 1 for dC) sits at 4·(4c + 2·(n & 1) + n / 8) + (n / 2) % 4
    int part_lane_order;  // set by launch_scan_bwd for the kernel it runs
    int ckpt_ready;       // ckpt already holds every tile's entering state (the two-lane
                          // kernel then skips its forward sweep)
    float *pA;     // [groups][batch][dim][16]: Σ over tokens of dA
    float *acc;    // groups > 1: [groups][3][batch][seqlen][dim] float32: each group's part of
                   // dΔ (before the softplus derivative), dx and the pre-gate output
    float *pD;     // [batch][dim]
    float *pbias;  // [batch][dim]
    long long batch, seqlen, dim;
    int dstate;
    int softplus;
    int zoh;       // input term (exp(Δ·A) − 1)/A·B·x instead of Δ·B·x
    int groups;    // ⌈dstate / 16⌉: 16-state groups, one grid plane each
    int ktiles;    // token tiles per sequence
    int ctiles;    // channel tiles per batch row
};

cudaError_t launch_scan_bwd(const BwdParams &p, bool bf16, cudaStream_t stream);
// Two lanes per chain (scan_bwd2.cu): one 16-state group, no conv, Δ·B·x input.
// Its CTAs cover bwd_pairs_tile_channels() channels (no fewer than the
// one-lane kernel's, so the workspace's partial rows suffice): the channel
// tiles of its partial sums when it runs.
bool bwd_pairs_supported(const BwdParams &p, bool bf16);
cudaError_t launch_scan_bwd_pairs(const BwdParams &p, bool bf16, cudaStream_t stream);
int bwd_pairs_tile_channels();
int bwd_tile_tokens();
int bwd_tile_channels();
int bwd_conv_tile_tokens();

}  // namespace selscan
