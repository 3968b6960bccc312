// Device-side check of gate values against the declared range.
//
// KDA range: alpha in (0,1], beta in [0,1]; Complex KDA range: alpha in
// [-1,1], beta in [0,2] ("Complex KDA" arXiv abstract: gates in [-1,1] and the
// delta-rule coefficient in [0,2]).  The same intervals are applied to RDA's
// erase gate e and to GDN-2's erase vector b.  Writes the number of
// violations (NaN included) to caller memory.
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

}  // namespace

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
