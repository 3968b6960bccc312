// Token-by-token fp32 scan of the gated delta-rule recurrence.
//
// Serves every shape/dtype the tensor-core chunked kernel does not (fp32
// inputs, head dims 16..128), and is the exact-order reference path on the
// GPU.  One CTA per (sequence, head); thread j owns value column j of the
// state and keeps S[:, j] (d_k fp32) in registers for the whole sequence.
// The columns of S evolve independently: the left operator
// (I - k a~^T) Diag(alpha) acts on every column alike and the written value
// m enters column j only through m_j (update equations on the
// Raon-1-mini-preview discussion page), so no thread talks to another except
// through the shared per-token vectors.
//
// Per token (decay, residual, write, readout):
//   u_j  = m_j - sum_i (alpha_i a~_i) S_ij
//   S_ij = alpha_i S_ij + k_i u_j
//   o_j  = sum_i q_i S_ij
// Token vectors are staged TB tokens at a time in shared memory so the inner
// loop runs without barriers; optional input preparation (gate activations,
// L2 norm of k) is applied while staging.
#include "common.cuh"

namespace kda {
namespace {

constexpr int TB = 16;  // tokens staged per barrier
constexpr int SB = 4;   // elements per thread loaded before any is widened (staging)

__device__ __forceinline__ float widen(float x) { return x; }
__device__ __forceinline__ float widen(__nv_bfloat16 x) { return __bfloat162float(x); }

// PREP: input preparation requested; without it that code is compiled out.
template <int DK, int DV, typename TIn, bool PREP>
__global__ void __launch_bounds__(DV)
scan_fwd_kernel(FwdArgs a)
{
    __shared__ __align__(16) float s_aa[TB][DK];   // alpha_i * a~_i
    __shared__ __align__(16) float s_al[TB][DK];   // alpha_i
    __shared__ __align__(16) float s_k[TB][DK];
    __shared__ __align__(16) float s_q[TB][DK];
    __shared__ __align__(16) float s_m[TB][DV];
    __shared__ float s_ksc[TB];   // 1 / ||k_t|| (input preparation)

    const int n = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int j = threadIdx.x;
    int b, t0, len;
    if (a.cu_seqlens) { b = 0; t0 = a.cu_seqlens[n]; len = a.cu_seqlens[n + 1] - t0; }
    else { b = n; t0 = 0; len = a.T; }

    const TIn *q = (const TIn *)a.q, *k = (const TIn *)a.k, *v = (const TIn *)a.v;
    const TIn *al = (const TIn *)a.alpha, *g1 = (const TIn *)a.g1, *g2 = (const TIn *)a.g2;
    const size_t soff = ((size_t)n * a.H + h) * DK * DV;

    float S[DK];
#pragma unroll
    for (int i = 0; i < DK; ++i) S[i] = a.s0 ? a.s0[soff + (size_t)i * DV + j] : 0.f;

    const bool logits = PREP && (a.prep & PREP_LOGITS), l2k = PREP && (a.prep & PREP_L2NORM_K), ext = a.ext != 0;
    for (int base = 0; base < len; base += TB) {
        const int nt = min(TB, len - base);
        __syncthreads();  // previous block of tokens fully consumed
        // loads are issued SB elements at a time and widened afterwards: widening
        // each one as it arrives would wait out every load's latency in turn
        for (int e0 = j; e0 < nt * DK; e0 += DV * SB) {
            TIn rk[SB], ra[SB], rg[SB], rq[SB];
#pragma unroll
            for (int bb = 0; bb < SB; ++bb) {
                const int e = e0 + bb * DV;
                if (e < nt * DK) {
                    const int tt = e / DK, i = e % DK;
                    const size_t tok = ((size_t)b * a.T + t0 + base + tt) * a.H + h;
                    rk[bb] = k[tok * DK + i];
                    ra[bb] = al[tok * DK + i];
                    rg[bb] = (a.variant == GDN2) ? g1[tok * DK + i] : g1[tok];
                    rq[bb] = q[tok * DK + i];
                }
            }
#pragma unroll
            for (int bb = 0; bb < SB; ++bb) {
                const int e = e0 + bb * DV;
                if (e < nt * DK) {
                    const int tt = e / DK, i = e % DK;
                    const float kk = widen(rk[bb]);
                    float aa = widen(ra[bb]), g = widen(rg[bb]);
                    if (logits) {
                        aa = round_to<TIn>(prep_alpha(aa, ext));
                        g = round_to<TIn>(prep_gate(g, ext));
                    }
                    s_k[tt][i] = kk;
                    s_al[tt][i] = aa;
                    s_aa[tt][i] = l2k ? aa * g : aa * (g * kk);   // times k once it is normalised
                    s_q[tt][i] = widen(rq[bb]);
                }
            }
        }
        for (int e0 = j; e0 < nt * DV; e0 += DV * SB) {
            TIn rv[SB], rw[SB];
#pragma unroll
            for (int bb = 0; bb < SB; ++bb) {
                const int e = e0 + bb * DV;
                if (e < nt * DV) {
                    const int tt = e / DV, jj = e % DV;
                    const size_t tok = ((size_t)b * a.T + t0 + base + tt) * a.H + h;
                    rw[bb] = a.variant == KDA ? g1[tok] : (a.variant == RDA ? g2[tok] : g2[tok * DV + jj]);
                    rv[bb] = v[tok * DV + jj];
                }
            }
#pragma unroll
            for (int bb = 0; bb < SB; ++bb) {
                const int e = e0 + bb * DV;
                if (e < nt * DV) {
                    float g = widen(rw[bb]);
                    if (logits) g = round_to<TIn>(prep_gate(g, ext));
                    s_m[e / DV][e % DV] = g * widen(rv[bb]);
                }
            }
        }
        __syncthreads();
        if (l2k) {   // k_t / ||k_t||, then a~ = (alpha g) (.) k
            for (int tt = j; tt < nt; tt += DV) {
                float ss = 0.f;
                for (int i = 0; i < DK; ++i) ss = fmaf(s_k[tt][i], s_k[tt][i], ss);
                s_ksc[tt] = prep_kscale(ss);
            }
            __syncthreads();
            for (int e = j; e < nt * DK; e += DV) {
                const int tt = e / DK, i = e % DK;
                const float kn = round_to<TIn>(s_k[tt][i] * s_ksc[tt]);
                s_k[tt][i] = kn;
                s_aa[tt][i] *= kn;
            }
            __syncthreads();
        }
        for (int tt = 0; tt < nt; ++tt) {
            float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll
            for (int i = 0; i < DK; i += 4) {
                const float4 c = *reinterpret_cast<const float4 *>(&s_aa[tt][i]);
                r0 = fmaf(c.x, S[i], r0);
                r1 = fmaf(c.y, S[i + 1], r1);
                r2 = fmaf(c.z, S[i + 2], r2);
                r3 = fmaf(c.w, S[i + 3], r3);
            }
            const float u = s_m[tt][j] - ((r0 + r1) + (r2 + r3));
            float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
#pragma unroll
            for (int i = 0; i < DK; i += 4) {
                const float4 av = *reinterpret_cast<const float4 *>(&s_al[tt][i]);
                const float4 kv = *reinterpret_cast<const float4 *>(&s_k[tt][i]);
                const float4 qv = *reinterpret_cast<const float4 *>(&s_q[tt][i]);
                S[i] = fmaf(av.x, S[i], kv.x * u);
                S[i + 1] = fmaf(av.y, S[i + 1], kv.y * u);
                S[i + 2] = fmaf(av.z, S[i + 2], kv.z * u);
                S[i + 3] = fmaf(av.w, S[i + 3], kv.w * u);
                o0 = fmaf(qv.x, S[i], o0);
                o1 = fmaf(qv.y, S[i + 1], o1);
                o2 = fmaf(qv.z, S[i + 2], o2);
                o3 = fmaf(qv.w, S[i + 3], o3);
            }
            const size_t tok = ((size_t)b * a.T + t0 + base + tt) * a.H + h;
            if (a.o) st_out((TIn *)a.o + tok * DV + j, (o0 + o1) + (o2 + o3));   // null: states only
            const int t = base + tt;   // token index within the sequence
            if (a.snap && ((t + 1) % SLOT_TOKENS == 0 || t + 1 == len)) {   // state after a 64-token chunk
                float *dst = a.snap + ((size_t)(slot_base(a, n) + t / SLOT_TOKENS) * a.H + h) * DK * DV + j;
#pragma unroll
                for (int i = 0; i < DK; ++i) dst[(size_t)i * DV] = S[i];
            }
        }
    }
    if (a.sf) {
#pragma unroll
        for (int i = 0; i < DK; ++i) a.sf[soff + (size_t)i * DV + j] = S[i];
    }
}

template <int DK, int DV>
cudaError_t launch_dims(const FwdArgs &a, bool bf16, cudaStream_t st)
{
    const int N = a.cu_seqlens ? a.num_seqs : a.B;
    dim3 grid((unsigned)(N * a.H)), block(DV);
    if (bf16) {
        if (a.prep) scan_fwd_kernel<DK, DV, __nv_bfloat16, true><<<grid, block, 0, st>>>(a);
        else scan_fwd_kernel<DK, DV, __nv_bfloat16, false><<<grid, block, 0, st>>>(a);
    } else {
        if (a.prep) scan_fwd_kernel<DK, DV, float, true><<<grid, block, 0, st>>>(a);
        else scan_fwd_kernel<DK, DV, float, false><<<grid, block, 0, st>>>(a);
    }
    return cudaGetLastError();
}

template <int DK>
cudaError_t launch_dv(const FwdArgs &a, bool bf16, cudaStream_t st)
{
    switch (a.dv) {
    case 16: return launch_dims<DK, 16>(a, bf16, st);
    case 32: return launch_dims<DK, 32>(a, bf16, st);
    case 64: return launch_dims<DK, 64>(a, bf16, st);
    case 128: return launch_dims<DK, 128>(a, bf16, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_scan_fwd(const FwdArgs &a, bool bf16, cudaStream_t st)
{
    switch (a.dk) {
    case 16: return launch_dv<16>(a, bf16, st);
    case 32: return launch_dv<32>(a, bf16, st);
    case 64: return launch_dv<64>(a, bf16, st);
    case 128: return launch_dv<128>(a, bf16, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda
