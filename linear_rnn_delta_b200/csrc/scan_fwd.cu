// Token-by-token fp32 scan of the gated delta-rule recurrence.
//
// Serves every shape/dtype the tensor-core chunked kernel does not (fp32
// inputs, head dims 16..128), writes the backward pass's fp32 checkpoints,
// and is the exact-order reference path on the GPU.
// The columns of S evolve independently: the left operator
// (I - k a~^T) Diag(alpha) acts on every column alike and the written value
// m enters column j only through m_j (update equations on the
// Raon-1-mini-preview discussion page), so a column needs nothing from the
// others but the shared per-token vectors.  Lanes work in groups of KS
// (16, or d_k / 4 below d_k = 64) adjacent lanes; a group owns CC = 4 (2 for
// the smallest heads) adjacent value columns, and lane p of it keeps rows
// i = 4 (m KS + p) + e (e < 4) of them in registers for the whole sequence.  The two sums over key rows are
// in-thread partial sums and log2(KS) butterfly shuffles, after which every
// lane of the group holds the same bits.  Per token a lane reads 3 d_k / KS
// floats of the shared token vectors and uses each for CC columns, so the
// shared-memory pipe, which bounds this kernel, delivers 3 d_k / CC floats
// per column and token (one float per lane and wavefront).  A CTA serves 64 columns (all of them when
// d_v < 64) of one (sequence, head).
//
// Per token (decay, residual, write, readout):
//   u_j  = m_j - sum_i (alpha_i a~_i) S_ij
//   S_ij = alpha_i S_ij + k_i u_j
//   o_j  = sum_i q_i S_ij
// Token vectors are staged TB tokens at a time in shared memory, double
// buffered, so the inner loop runs without barriers; optional input
// preparation (gate activations, L2 norm of k) is applied while staging.  Without an output (the backward's
// checkpoints) the readout is compiled out, and u_t of every token may be kept instead: with it the
// backward replays a chunk from its checkpoint by the update alone, bitwise as this scan ran it.
#include "common.cuh"
#include "scan_bwd.cuh"

namespace kda {
namespace {

constexpr int TB = 8;   // tokens per staged block (two blocks in shared memory)

__device__ __forceinline__ float widen(float x) { return x; }
__device__ __forceinline__ float widen(__nv_bfloat16 x) { return __bfloat162float(x); }

template <int DK, int DV> struct ScanShape {
    static constexpr int KS = DK >= 64 ? 16 : DK / 4;      // lanes per group (rows split KS ways)
    static constexpr int NG = DK / (4 * KS);               // float4 row groups per lane
    static constexpr int CB = DV < 64 ? DV : 64;           // value columns per CTA
    static constexpr int CC = CB / 4 * KS >= 32 ? 4 : 2;   // value columns per group (whole warps)
    static constexpr int NTH = CB / CC * KS;               // threads per CTA
    static constexpr int CTAS = DV / CB;                   // CTAs per (sequence, head)
    static_assert(NG >= 1 && NTH % 32 == 0, "scan shape");
};

// CC consecutive floats (16- or 8-byte aligned)
template <int CC> __device__ __forceinline__ void ld_cols(const float *p, float (&x)[CC])
{
    if constexpr (CC == 4) {
        const float4 t = *reinterpret_cast<const float4 *>(p);
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else {
        const float2 t = *reinterpret_cast<const float2 *>(p);
        x[0] = t.x; x[1] = t.y;
    }
}
template <int CC> __device__ __forceinline__ void st_cols(float *p, const float2 (&x)[CC / 2])
{
    if constexpr (CC == 4) *reinterpret_cast<float4 *>(p) = make_float4(x[0].x, x[0].y, x[1].x, x[1].y);
    else *reinterpret_cast<float2 *>(p) = x[0];
}

// Sum of x over the KS lanes of a group; every lane gets the same bits (each
// butterfly step adds the same two values, in one order or the other).
template <int KS>
__device__ __forceinline__ float group_sum(float x)
{
#pragma unroll
    for (int off = 1; off < KS; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// PREP: input preparation requested; OUT: o is written.  Without either, that
// code is compiled out.  u_save (states-only variant, may be null): u_t, fp32,
// in o's layout [B*T][H][d_v].
template <int DK, int DV, typename TIn, bool PREP, bool OUT>
__global__ void __launch_bounds__(ScanShape<DK, DV>::NTH)
scan_fwd_kernel(FwdArgs a, float *u_save)
{
    using SH = ScanShape<DK, DV>;
    constexpr int KS = SH::KS, NG = SH::NG, CB = SH::CB, CC = SH::CC, NTH = SH::NTH, CTAS = SH::CTAS;
    __shared__ __align__(16) float s_aa[2][TB][DK];   // alpha_i * a~_i (two blocks of tokens)
    __shared__ __align__(16) float s_al[2][TB][DK];   // alpha_i
    __shared__ __align__(16) float s_k[2][TB][DK];
    __shared__ __align__(16) float s_q[2][OUT ? TB : 1][DK];
    __shared__ __align__(16) float s_m[2][TB][CB];
    __shared__ float s_ksc[TB];   // 1 / ||k_t|| (input preparation)

    const int pair = blockIdx.x / CTAS, cblk = blockIdx.x % CTAS;
    const int n = pair / a.H, h = pair % a.H;
    const int tid = threadIdx.x, p = tid % KS, grp = tid / KS;
    const int cl = grp * CC;        // first of the group's columns within the CTA
    const int j = cblk * CB + cl;   // ... and within the head
    int b, t0, len;
    if (a.cu_seqlens) { b = 0; t0 = a.cu_seqlens[n]; len = a.cu_seqlens[n + 1] - t0; }
    else { b = n; t0 = 0; len = a.T; }

    const TIn *q = (const TIn *)a.q, *k = (const TIn *)a.k, *v = (const TIn *)a.v;
    const TIn *al = (const TIn *)a.alpha, *g1 = (const TIn *)a.g1, *g2 = (const TIn *)a.g2;
    const size_t soff = ((size_t)n * a.H + h) * DK * DV;
    auto row = [&](int m, int e) { return 4 * (m * KS + p) + e; };

    // S2[4 m + e][c] = (S_{row(m, e), j + 2c}, S_{row(m, e), j + 2c + 1})
    float2 S2[4 * NG][CC / 2];
#pragma unroll
    for (int m = 0; m < NG; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int c = 0; c < CC / 2; ++c)
                S2[4 * m + e][c] = a.s0 ? *reinterpret_cast<const float2 *>(a.s0 + soff + (size_t)row(m, e) * DV + j + 2 * c)
                                        : make_float2(0.f, 0.f);

    const bool logits = PREP && (a.prep & PREP_LOGITS), l2k = PREP && (a.prep & PREP_L2NORM_K), ext = a.ext != 0;
    // Token vectors of block b+1 are loaded into registers (raw) while block b
    // is computed, then widened, prepared and stored to the other buffer: the
    // loads' latency hides behind a block's arithmetic and each block costs
    // one barrier.
    constexpr int EK = (TB * DK + NTH - 1) / NTH, EM = (TB * CB + NTH - 1) / NTH;
    TIn pk[EK], pa[EK], pg[EK], pq[OUT ? EK : 1], pv[EM], pw[EM];
    auto fetch = [&](int base) {
        const int nt = min(TB, len - base);
#pragma unroll
        for (int x = 0; x < EK; ++x) {
            const int e = tid + x * NTH;
            if (e < nt * DK) {
                const int tt = e / DK, i = e % DK;
                const size_t tok = ((size_t)b * a.T + t0 + base + tt) * a.H + h;
                pk[x] = k[tok * DK + i];
                pa[x] = al[tok * DK + i];
                pg[x] = (a.variant == GDN2) ? g1[tok * DK + i] : g1[tok];
                if (OUT) pq[x] = q[tok * DK + i];
            }
        }
#pragma unroll
        for (int x = 0; x < EM; ++x) {
            const int e = tid + x * NTH;
            if (e < nt * CB) {
                const int tt = e / CB, jj = cblk * CB + e % CB;
                const size_t tok = ((size_t)b * a.T + t0 + base + tt) * a.H + h;
                pw[x] = a.variant == KDA ? g1[tok] : (a.variant == RDA ? g2[tok] : g2[tok * DV + jj]);
                pv[x] = v[tok * DV + jj];
            }
        }
    };
    auto commit = [&](int buf, int base) {
        const int nt = min(TB, len - base);
#pragma unroll
        for (int x = 0; x < EK; ++x) {
            const int e = tid + x * NTH;
            if (e < nt * DK) {
                const int tt = e / DK, i = e % DK;
                const float kk = widen(pk[x]);
                float aa = widen(pa[x]), g = widen(pg[x]);
                if (logits) {
                    aa = round_to<TIn>(prep_alpha(aa, ext));
                    g = round_to<TIn>(prep_gate(g, ext));
                }
                s_k[buf][tt][i] = kk;
                s_al[buf][tt][i] = aa;
                s_aa[buf][tt][i] = l2k ? aa * g : aa * (g * kk);   // times k once it is normalised
                if (OUT) s_q[buf][tt][i] = widen(pq[x]);
            }
        }
#pragma unroll
        for (int x = 0; x < EM; ++x) {
            const int e = tid + x * NTH;
            if (e < nt * CB) {
                float g = widen(pw[x]);
                if (logits) g = round_to<TIn>(prep_gate(g, ext));
                s_m[buf][e / CB][e % CB] = g * widen(pv[x]);
            }
        }
    };
    if (len > 0) {
        fetch(0);
        commit(0, 0);
    }
    __syncthreads();
    for (int base = 0, blk = 0; base < len; base += TB, ++blk) {
        const int nt = min(TB, len - base), buf = blk & 1;
        const bool more = base + TB < len;
        if (more) fetch(base + TB);
        if (l2k) {   // k_t / ||k_t||, then a~ = (alpha g) (.) k
            for (int tt = tid; tt < nt; tt += NTH) {
                float ss = 0.f;
                for (int i = 0; i < DK; ++i) ss = fmaf(s_k[buf][tt][i], s_k[buf][tt][i], ss);
                s_ksc[tt] = prep_kscale(ss);
            }
            __syncthreads();
            for (int e = tid; e < nt * DK; e += NTH) {
                const int tt = e / DK, i = e % DK;
                const float kn = round_to<TIn>(s_k[buf][tt][i] * s_ksc[tt]);
                s_k[buf][tt][i] = kn;
                s_aa[buf][tt][i] *= kn;
            }
            __syncthreads();
        }
        for (int tt = 0; tt < nt; ++tt) {
            // column pairs (2c, 2c + 1) go through the packed fp32 pipe: each
            // lane of a pair gets the same fused multiply-add as the scalar form
            float2 r[CC / 2][2];
#pragma unroll
            for (int c = 0; c < CC / 2; ++c) r[c][0] = r[c][1] = make_float2(0.f, 0.f);
#pragma unroll
            for (int m = 0; m < NG; ++m) {
                const float4 x = *reinterpret_cast<const float4 *>(&s_aa[buf][tt][row(m, 0)]);
#pragma unroll
                for (int c = 0; c < CC / 2; ++c) {
                    r[c][0] = __ffma2_rn(make_float2(x.x, x.x), S2[4 * m][c], r[c][0]);
                    r[c][1] = __ffma2_rn(make_float2(x.y, x.y), S2[4 * m + 1][c], r[c][1]);
                    r[c][0] = __ffma2_rn(make_float2(x.z, x.z), S2[4 * m + 2][c], r[c][0]);
                    r[c][1] = __ffma2_rn(make_float2(x.w, x.w), S2[4 * m + 3][c], r[c][1]);
                }
            }
            float u[CC];
            ld_cols<CC>(&s_m[buf][tt][cl], u);
#pragma unroll
            for (int c = 0; c < CC / 2; ++c) {
                u[2 * c] -= group_sum<KS>(r[c][0].x + r[c][1].x);
                u[2 * c + 1] -= group_sum<KS>(r[c][0].y + r[c][1].y);
            }
            const size_t tok = ((size_t)b * a.T + t0 + base + tt) * a.H + h;
            if (!OUT && u_save && p == 0) {   // every lane of the group holds the same bits
                float2 u2[CC / 2];
#pragma unroll
                for (int c = 0; c < CC / 2; ++c) u2[c] = make_float2(u[2 * c], u[2 * c + 1]);
                st_cols<CC>(u_save + tok * DV + j, u2);
            }
            float2 o[CC / 2][2];
#pragma unroll
            for (int c = 0; c < CC / 2; ++c) o[c][0] = o[c][1] = make_float2(0.f, 0.f);
#pragma unroll
            for (int m = 0; m < NG; ++m) {
                const float4 av = *reinterpret_cast<const float4 *>(&s_al[buf][tt][row(m, 0)]);
                const float4 kv = *reinterpret_cast<const float4 *>(&s_k[buf][tt][row(m, 0)]);
                const float a4[4] = {av.x, av.y, av.z, av.w}, k4[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
#pragma unroll
                    for (int c = 0; c < CC / 2; ++c) {
                        const float2 ku = __fmul2_rn(make_float2(k4[e], k4[e]), make_float2(u[2 * c], u[2 * c + 1]));
                        S2[4 * m + e][c] = __ffma2_rn(make_float2(a4[e], a4[e]), S2[4 * m + e][c], ku);
                    }
                if (OUT) {
                    const float4 qv = *reinterpret_cast<const float4 *>(&s_q[buf][tt][row(m, 0)]);
                    const float q4[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
#pragma unroll
                        for (int c = 0; c < CC / 2; ++c)
                            o[c][e & 1] = __ffma2_rn(make_float2(q4[e], q4[e]), S2[4 * m + e][c], o[c][e & 1]);
                }
            }
            if (OUT) {
                float ov[CC];
#pragma unroll
                for (int c = 0; c < CC / 2; ++c) {
                    ov[2 * c] = group_sum<KS>(o[c][0].x + o[c][1].x);
                    ov[2 * c + 1] = group_sum<KS>(o[c][0].y + o[c][1].y);
                }
                if (p == 0) {
#pragma unroll
                    for (int c = 0; c < CC; ++c) st_out((TIn *)a.o + tok * DV + j + c, ov[c]);
                }
            }
            const int t = base + tt;   // token index within the sequence
            if (a.snap && ((t + 1) % SLOT_TOKENS == 0 || t + 1 == len)) {   // state after a 64-token chunk
                float *dst = a.snap + ((size_t)(slot_base(a, n) + t / SLOT_TOKENS) * a.H + h) * DK * DV + j;
#pragma unroll
                for (int m = 0; m < NG; ++m)
#pragma unroll
                    for (int e = 0; e < 4; ++e) st_cols<CC>(dst + (size_t)row(m, e) * DV, S2[4 * m + e]);
            }
        }
        if (more) commit(buf ^ 1, base + TB);
        __syncthreads();   // block b consumed, block b+1 staged
    }
    if (a.sf) {
#pragma unroll
        for (int m = 0; m < NG; ++m)
#pragma unroll
            for (int e = 0; e < 4; ++e) st_cols<CC>(a.sf + soff + (size_t)row(m, e) * DV + j, S2[4 * m + e]);
    }
}

// Variants launched: with output, with or without input preparation; states
// only (the backward's checkpoints), without preparation.
template <int DK, int DV, typename TIn>
void launch_typed(const FwdArgs &a, float *u_save, dim3 grid, cudaStream_t st)
{
    constexpr int NTH = ScanShape<DK, DV>::NTH;
    if (a.prep) scan_fwd_kernel<DK, DV, TIn, true, true><<<grid, NTH, 0, st>>>(a, nullptr);
    else if (a.o) scan_fwd_kernel<DK, DV, TIn, false, true><<<grid, NTH, 0, st>>>(a, nullptr);
    else scan_fwd_kernel<DK, DV, TIn, false, false><<<grid, NTH, 0, st>>>(a, u_save);
}

template <int DK, int DV>
cudaError_t launch_dims(const FwdArgs &a, float *u_save, bool bf16, cudaStream_t st)
{
    if (a.prep && !a.o) return cudaErrorInvalidValue;   // no such variant (and no caller)
    const int N = a.cu_seqlens ? a.num_seqs : a.B;
    const dim3 grid((unsigned)(N * a.H * ScanShape<DK, DV>::CTAS));
    if (bf16) launch_typed<DK, DV, __nv_bfloat16>(a, u_save, grid, st);
    else launch_typed<DK, DV, float>(a, u_save, grid, st);
    return cudaGetLastError();
}

template <int DK>
cudaError_t launch_dv(const FwdArgs &a, float *u_save, bool bf16, cudaStream_t st)
{
    switch (a.dv) {
    case 16: return launch_dims<DK, 16>(a, u_save, bf16, st);
    case 32: return launch_dims<DK, 32>(a, u_save, bf16, st);
    case 64: return launch_dims<DK, 64>(a, u_save, bf16, st);
    case 128: return launch_dims<DK, 128>(a, u_save, bf16, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_any(const FwdArgs &a, float *u_save, bool bf16, cudaStream_t st)
{
    switch (a.dk) {
    case 16: return launch_dv<16>(a, u_save, bf16, st);
    case 32: return launch_dv<32>(a, u_save, bf16, st);
    case 64: return launch_dv<64>(a, u_save, bf16, st);
    case 128: return launch_dv<128>(a, u_save, bf16, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_scan_fwd(const FwdArgs &a, bool bf16, cudaStream_t st) { return launch_any(a, nullptr, bf16, st); }

cudaError_t launch_scan_checkpoints(const FwdArgs &a, float *u_save, bool bf16, cudaStream_t st)
{
    if (a.o || a.prep || !a.snap) return cudaErrorInvalidValue;   // the states-only variant
    return launch_any(a, u_save, bf16, st);
}

}  // namespace kda
