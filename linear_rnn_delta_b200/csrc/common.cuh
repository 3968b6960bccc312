// Shared device helpers and internal launch declarations of the kda library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace kda {

enum Variant { KDA = 0, RDA = 1, GDN2 = 2 };

// Element loads/stores in the input dtype, arithmetic in fp32.
__device__ __forceinline__ float ld_f32(const float *p) { return *p; }
__device__ __forceinline__ float ld_f32(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_out(float *p, float x) { *p = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// Arguments shared by the forward kernels (device pointers, see include/kda.h).
struct FwdArgs {
    int variant;
    int B, T, H, dk, dv;
    const void *q, *k, *v, *alpha, *g1, *g2;
    const int32_t *cu_seqlens;
    int num_seqs;
    const float *s0;
    float *sf;
    void *o;
    unsigned prep = 0;   // PREP_* bits: input preparation done by the kernels
    int ext = 0;         // extended (Complex KDA) gate range: selects the activations
    float *snap = nullptr;   // optional: state after every 64 tokens, [slot][H][dk][dv] (chunk slots)
    int debug_stall = 0;     // testing aid (split form): one chain CTA's first wait runs out
};

// Chunk slot of chunk c (64 tokens) of sequence n whose first token is global
// row R_n: n + floor(R_n / 64) + c -- unique, increasing within a sequence and
// below N + ceil(rows / 64).  Workspace slots and state snapshots use it.
constexpr int SLOT_TOKENS = 64;
__device__ __forceinline__ int seq_row0(const FwdArgs &a, int n) { return a.cu_seqlens ? a.cu_seqlens[n] : n * a.T; }
__device__ __forceinline__ int seq_len(const FwdArgs &a, int n)
{
    return a.cu_seqlens ? a.cu_seqlens[n + 1] - a.cu_seqlens[n] : a.T;
}
__device__ __forceinline__ int slot_base(const FwdArgs &a, int n) { return n + seq_row0(a, n) / SLOT_TOKENS; }

// ---- input preparation (optional, applied once where the kernels read their inputs) ----
// PREP_LOGITS: alpha and the gates arrive as logits.  Standard range:
//   alpha = exp(-softplus(x)) = 1 / (1 + e^x),  gate = sigmoid(y);
// extended range: alpha = tanh(x),  gate = 2 sigmoid(y).
// PREP_L2NORM_K: k_t is replaced by k_t / max(||k_t||_2, 1e-6) per token and head.
// Prepared values are computed in fp32 and rounded to the input dtype, as a
// separate activation / normalisation pass would have stored them.
constexpr unsigned PREP_LOGITS = 1u, PREP_L2NORM_K = 2u;
constexpr float K_NORM_FLOOR = 1e-6f;

__device__ __forceinline__ float prep_alpha(float x, bool ext)
{
    return ext ? tanhf(x) : __fdividef(1.f, 1.f + __expf(x));   // e^x = inf -> 0
}
__device__ __forceinline__ float prep_gate(float y, bool ext)
{
    const float s = __fdividef(1.f, 1.f + __expf(-y));
    return ext ? 2.f * s : s;
}
__device__ __forceinline__ float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }
template <typename T> __device__ __forceinline__ float round_to(float x) { return x; }
template <> __device__ __forceinline__ float round_to<__nv_bfloat16>(float x) { return round_bf16(x); }
// 1 / max(||k||, floor) from the sum of squares
__device__ __forceinline__ float prep_kscale(float sumsq)
{
    return 1.f / fmaxf(sqrtf(sumsq), K_NORM_FLOOR);
}

// Internal launchers; each returns cudaSuccess or the launch error.
cudaError_t launch_scan_fwd(const FwdArgs &a, bool bf16, cudaStream_t st);
cudaError_t launch_decode_step(const FwdArgs &a, bool bf16, cudaStream_t st);
cudaError_t launch_chunk_fwd_sm100(const FwdArgs &a, cudaStream_t st);
// Two-kernel chunked path: `ws` holds chunk_split_workspace_bytes(a) bytes.
bool chunk_prefer_split(const FwdArgs &a);   // the shape-based default choice of form
size_t chunk_split_workspace_bytes(const FwdArgs &a);
cudaError_t launch_chunk_split_sm100(const FwdArgs &a, void *ws, cudaStream_t st);
// Split form with the fixed device scratch array as its workspace (no allocation).
size_t chunk_noalloc_capacity();
cudaError_t launch_chunk_split_noalloc(const FwdArgs &a, cudaStream_t st);
cudaError_t launch_check_gates(int variant, int gate_range, bool bf16, long long n_tok, int dk,
                               const void *alpha, const void *g1, int *d_count, cudaStream_t st);
cudaError_t launch_check_seqlens(const int32_t *cu, int num_seqs, long long total, int *d_count, cudaStream_t st);
// Synchronous input validation: counts gates outside the range (*bad_gates) and
// violations of the cu_seqlens contract (*bad_seqlens; cu may be NULL), waiting
// for the verdict on `st`.
cudaError_t validate_inputs(int variant, int gate_range, bool bf16, long long n_tok, int dk, const void *alpha,
                            const void *g1, const int32_t *cu, int num_seqs, long long total, cudaStream_t st,
                            int *bad_gates, int *bad_seqlens);
// Device failure word: read and cleared after `st` has drained.
cudaError_t take_device_status(cudaStream_t st, unsigned *bits);

}  // namespace kda
