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
    const float *u;       // u_t of every token from the checkpoint scan, [B*T][H][dv] fp32
                          // (read by the kernels for d_k >= 32; may be null at d_k = 16)
};

// The forward token scan in its states-only form: a.snap receives the state
// after every 64 tokens (chunk slots) and u_save, if not null, u_t of every
// token (u_j = m_j - sum_i alpha_i a~_i S_ij, fp32, [B*T][H][d_v]).
cudaError_t launch_scan_checkpoints(const FwdArgs &a, float *u_save, bool bf16, cudaStream_t st);

// a.snap must hold the forward's state snapshots (chunk slots), g.u the
// checkpoint scan's u_t.
size_t scan_bwd_scratch_bytes(const FwdArgs &a);
cudaError_t launch_scan_bwd(const FwdArgs &a, const BwdArgs &g, bool bf16, cudaStream_t st);

}  // namespace kda
