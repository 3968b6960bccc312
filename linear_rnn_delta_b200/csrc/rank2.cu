// Rank-2 (DeltaProduct_2-style) steps -- two delta-rule transitions composed
// in one recurrent update, named as prior work in the Complex KDA arXiv
// abstract -- run on the rank-1 kernels as two sub-tokens per token:
//   sub-token 2t:   the token's decay alpha_t, (k, v, gates) of sub-step 1, readout discarded
//   sub-token 2t+1: decay 1, (k, v, gates) of sub-step 2, readout = o_t
// The caller's k, v and gate tensors carry the sub-step axis after T
// ([B,T,2,H,.]), which in memory is already the sub-token order [B,2T,H,.];
// only q and alpha are expanded, and o gathered, by the copy kernels here
// (16-byte vectors, grid-stride).  The gradient of rank-2 steps is the rank-1
// backward over the same sub-tokens with d_o spread onto the second sub-tokens,
// mapped back: dq from the second sub-tokens, dalpha from the first.
#include "rank2.cuh"

namespace kda {
namespace {

constexpr int COPY_THREADS = 256;
constexpr int COPY_MAX_BLOCKS = 148 * 8;

// One 16-byte vector of a row: `one` is the bit pattern of 1.0 repeated (bf16 or fp32).
__global__ void rank2_expand_kernel(const uint4 *q, const uint4 *alpha, uint4 *q2, uint4 *alpha2, long long tokens,
                                    int row_vecs, unsigned one, const int32_t *cu, int32_t *cu2, int n_cu)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long first = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long n = tokens * row_vecs;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u), ones = make_uint4(one, one, one, one);
    for (long long e = first; e < n; e += stride) {
        const long long tok = e / row_vecs, r = e % row_vecs;
        const long long even = 2 * tok * row_vecs + r, odd = even + row_vecs;
        q2[even] = zero;
        q2[odd] = q[e];
        alpha2[even] = alpha[e];
        alpha2[odd] = ones;
    }
    if (cu)
        for (long long i = first; i < n_cu; i += stride) cu2[i] = 2 * cu[i];
}

__global__ void rank2_gather_kernel(const uint4 *o2, uint4 *o, long long tokens, int row_vecs, int parity)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long n = tokens * row_vecs;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
        const long long tok = e / row_vecs, r = e % row_vecs;
        o[e] = o2[(2 * tok + parity) * row_vecs + r];
    }
}

// x2[2t] = 0, x2[2t+1] = x[t]: a per-token tensor onto the sub-tokens, present on the second
__global__ void rank2_spread_kernel(const uint4 *x, uint4 *x2, long long tokens, int row_vecs)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long n = tokens * row_vecs;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
        const long long tok = e / row_vecs, r = e % row_vecs;
        x2[2 * tok * row_vecs + r] = zero;
        x2[(2 * tok + 1) * row_vecs + r] = x[e];
    }
}

unsigned blocks_for(long long n)
{
    const long long b = (n + COPY_THREADS - 1) / COPY_THREADS;
    return (unsigned)(b < 1 ? 1 : (b > COPY_MAX_BLOCKS ? COPY_MAX_BLOCKS : b));
}

}  // namespace

cudaError_t launch_rank2_expand(bool bf16, const void *q, const void *alpha, void *q2, void *alpha2,
                                long long tokens, int row_elems, const int32_t *cu, int32_t *cu2, int n_cu,
                                cudaStream_t st)
{
    const int row_vecs = row_elems * (bf16 ? 2 : 4) / 16;   // row_elems is a multiple of 16
    const unsigned one = bf16 ? 0x3F803F80u : 0x3F800000u;
    const long long n = tokens * row_vecs > n_cu ? tokens * row_vecs : n_cu;
    rank2_expand_kernel<<<blocks_for(n), COPY_THREADS, 0, st>>>(
        static_cast<const uint4 *>(q), static_cast<const uint4 *>(alpha), static_cast<uint4 *>(q2),
        static_cast<uint4 *>(alpha2), tokens, row_vecs, one, cu, cu2, n_cu);
    return cudaGetLastError();
}

cudaError_t launch_rank2_gather(bool bf16, const void *o2, void *o, long long tokens, int row_elems, int parity,
                                cudaStream_t st)
{
    const int row_vecs = row_elems * (bf16 ? 2 : 4) / 16;
    if (tokens == 0) return cudaSuccess;
    rank2_gather_kernel<<<blocks_for(tokens * row_vecs), COPY_THREADS, 0, st>>>(
        static_cast<const uint4 *>(o2), static_cast<uint4 *>(o), tokens, row_vecs, parity);
    return cudaGetLastError();
}

cudaError_t launch_rank2_spread(bool bf16, const void *x, void *x2, long long tokens, int row_elems, cudaStream_t st)
{
    const int row_vecs = row_elems * (bf16 ? 2 : 4) / 16;
    if (tokens == 0) return cudaSuccess;
    rank2_spread_kernel<<<blocks_for(tokens * row_vecs), COPY_THREADS, 0, st>>>(
        static_cast<const uint4 *>(x), static_cast<uint4 *>(x2), tokens, row_vecs);
    return cudaGetLastError();
}

}  // namespace kda
