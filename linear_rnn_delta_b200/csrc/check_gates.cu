// Device-side checks of the inputs' contracts.
//
// Gates against the declared range.  KDA range: alpha in (0,1], beta in
// [0,1]; Complex KDA range: alpha in [-1,1], beta in [0,2] ("Complex KDA"
// arXiv abstract: gates in [-1,1] and the delta-rule coefficient in [0,2]).
// The same intervals are applied to RDA's erase gate e and to GDN-2's erase
// vector b.  NaN counts as a violation.
//
// Packed document offsets (the "document reset" of the openarchlab page on
// GDN/KDA state updates, sec. 3): cu[0] = 0, cu[n] <= cu[n+1], cu[N] = total.
//
// Each check writes a count of violations to device memory and never traps.
#include <mutex>

#include "common.cuh"

namespace kda {
namespace {

template <typename TIn>
__global__ void check_gates_kernel(int variant, int extended, long long n_alpha, long long n_g1,
                                   const TIn *alpha, const TIn *g1, int *count)
{
    int bad = 0;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_alpha; e += stride) {
        const float x = ld_f32(alpha + e);
        const bool ok = extended ? (x >= -1.f && x <= 1.f) : (x > 0.f && x <= 1.f);
        bad += ok ? 0 : 1;
    }
    const float gmax = extended ? 2.f : 1.f;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_g1; e += stride) {
        const float x = ld_f32(g1 + e);
        bad += (x >= 0.f && x <= gmax) ? 0 : 1;
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, off);
    if ((threadIdx.x & 31) == 0 && bad) atomicAdd(count, bad);
    (void)variant;
}

// One count per violated condition: cu[0] != 0, each n with cu[n+1] < cu[n], cu[N] != total.
__global__ void check_seqlens_kernel(const int32_t *cu, int num_seqs, long long total, int *count)
{
    int bad = 0;
    const int stride = gridDim.x * blockDim.x;
    for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < num_seqs; n += stride)
        bad += cu[n + 1] < cu[n] ? 1 : 0;
    if (blockIdx.x == 0 && threadIdx.x == 0)
        bad += (cu[0] != 0 ? 1 : 0) + ((long long)cu[num_seqs] != total ? 1 : 0);
#pragma unroll
    for (int off = 16; off; off >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, off);
    if ((threadIdx.x & 31) == 0 && bad) atomicAdd(count, bad);
}

// Counters of the synchronous validation (calls hold the mutex below while they use them).
__device__ int g_validate_counts[2];

}  // namespace

cudaError_t launch_check_seqlens(const int32_t *cu, int num_seqs, long long total, int *d_count, cudaStream_t st)
{
    cudaError_t e = cudaMemsetAsync(d_count, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    long long blocks = ((long long)num_seqs + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    check_seqlens_kernel<<<(unsigned)blocks, 256, 0, st>>>(cu, num_seqs, total, d_count);
    return cudaGetLastError();
}

cudaError_t validate_inputs(int variant, int gate_range, bool bf16, long long n_tok, int dk, const void *alpha,
                            const void *g1, const int32_t *cu, int num_seqs, long long total, cudaStream_t st,
                            int *bad_gates, int *bad_seqlens)
{
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    int *counts = nullptr;
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(&counts), g_validate_counts);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(counts, 0, 2 * sizeof(int), st)) != cudaSuccess) return e;
    if (n_tok > 0 && (e = launch_check_gates(variant, gate_range, bf16, n_tok, dk, alpha, g1, counts, st)) !=
                         cudaSuccess)
        return e;
    if (cu && (e = launch_check_seqlens(cu, num_seqs, total, counts + 1, st)) != cudaSuccess) return e;
    int h[2] = {0, 0};
    if ((e = cudaMemcpyAsync(h, counts, sizeof(h), cudaMemcpyDeviceToHost, st)) != cudaSuccess) return e;
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
    *bad_gates = h[0];
    *bad_seqlens = h[1];
    return cudaSuccess;
}

cudaError_t launch_check_gates(int variant, int gate_range, bool bf16, long long n_tok, int dk,
                               const void *alpha, const void *g1, int *d_count, cudaStream_t st)
{
    cudaError_t e = cudaMemsetAsync(d_count, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    const long long n_alpha = n_tok * dk;
    const long long n_g1 = (variant == GDN2) ? n_tok * dk : n_tok;
    long long blocks = (n_alpha + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    if (bf16)
        check_gates_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
            variant, gate_range, n_alpha, n_g1, (const __nv_bfloat16 *)alpha, (const __nv_bfloat16 *)g1, d_count);
    else
        check_gates_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
            variant, gate_range, n_alpha, n_g1, (const float *)alpha, (const float *)g1, d_count);
    return cudaGetLastError();
}

}  // namespace kda
