// Backward pass of the recurrence (fp32 adjoint scan): arguments and launcher.
#pragma once
#include "common.cuh"

namespace kda {

// Gradient arguments of the backward scan (device pointers; fp32 gradients in
// the layouts of the inputs they belong to).
struct BwdArgs {
    const void *d_o;      // dL/do [B,T,H,dv], input dtype
    const float *d_sf;    // dL/dS_final [N,H,dk,dv] or null
    float *dq, *dk, *dv, *dalpha, *dg1, *dg2;
    float *d_s0;          // dL/dS_initial [N,H,dk,dv] or null
    float *scratch;       // scan_bwd_scratch_bytes(a): the chunk's S_{t-1} per CTA
};

// a.snap must hold the forward's state snapshots (chunk slots).
size_t scan_bwd_scratch_bytes(const FwdArgs &a);
cudaError_t launch_scan_bwd(const FwdArgs &a, const BwdArgs &g, bool bf16, cudaStream_t st);

}  // namespace kda
