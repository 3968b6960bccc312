// Backward pass of the gated delta-rule recurrence: an fp32 adjoint scan.
//
// Forward step (update equations on the Raon-1-mini-preview discussion page):
//   S' = Diag(alpha) S_{t-1},  u = m - S'^T a~,  S_t = S' + k u^T,  o_t = S_t^T q_t.
// With G = dL/dS_t (the part flowing back from later tokens plus q_t do_t^T),
// the adjoint of one step is
//   dq = S_t do,  du = G^T k,  dk += G u,  dS' = G - a~ du^T,
//   dalpha = rowsum(S_{t-1} (.) dS'),  da~ = -S' du,  dm = du,
//   G <- Diag(alpha) dS'   (dL/dS_{t-1}),
// followed by the variant's gate algebra ((a~, m) = (beta k, beta v),
// (e k, w v) or (b (.) k, w (.) v)).  The backward needs S_{t-1} at every
// token: one CTA per (sequence, head) walks the sequence's 64-token chunks
// from last to first; each chunk is replayed forward from its checkpoint (the
// state snapshot the forward scan stored after the previous chunk), keeping
// every S_{t-1} and u_t of the chunk, then walked backwards.  S and G live in
// shared memory (rows padded to DV + 1 floats: row-wise and column-wise sweeps
// are both bank-conflict free); row sums (over value columns j) and column
// sums (over key channels i) are split over the CTA's 256 threads.
#include "scan_bwd.cuh"

namespace kda {
namespace {

constexpr int BNT = 256;       // threads per CTA
constexpr int BC = SLOT_TOKENS;  // tokens per checkpointed chunk

template <int DK, int DV>
struct BwdSmem {
    static constexpr int P = DV + 1;                  // padded row pitch of S and G
    static constexpr int RSPLIT = BNT / DK;           // threads per row sum
    static constexpr int CSPLIT = BNT / DV;           // threads per column sum
    static constexpr size_t S = 0;                    // S_{t-1} (forward replay: S)
    static constexpr size_t G = S + (size_t)DK * P;   // dL/dS
    static constexpr size_t U = G + (size_t)DK * P;   // u_t of the chunk [BC][DV]
    static constexpr size_t VK = U + (size_t)BC * DV; // token vectors over d_k: k, q, alpha, a~
    static constexpr size_t VV = VK + 4 * DK;         // over d_v: m, v, do, g2 part
    static constexpr size_t RED = VV + 4 * DV;        // partial sums [4][RSPLIT][DK] | [CSPLIT][DV]
    static constexpr size_t OUT = RED + 4 * (size_t)RSPLIT * DK + (size_t)CSPLIT * DV;   // du [DV], dat [DK], scalars
    static constexpr size_t FLOATS = OUT + DV + DK + 8;
};

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(BNT, 1) scan_bwd_kernel(FwdArgs a, BwdArgs g)
{
    using L = BwdSmem<DK, DV>;
    constexpr int P = L::P, RS = L::RSPLIT, CS = L::CSPLIT;
    extern __shared__ float smf[];
    float *S = smf + L::S, *G = smf + L::G, *Uc = smf + L::U;
    float *vk = smf + L::VK, *vv = smf + L::VV, *red = smf + L::RED, *out = smf + L::OUT;
    float *s_k = vk, *s_q = vk + DK, *s_al = vk + 2 * DK, *s_at = vk + 3 * DK;
    float *s_m = vv, *s_v = vv + DV, *s_do = vv + 2 * DV, *s_g2 = vv + 3 * DV;
    float *s_du = out, *s_dat = out + DV, *s_sc = out + DV + DK;   // s_sc: u.do, scalar gate sums

    const int n = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int tid = threadIdx.x;
    const int row0 = seq_row0(a, n), len = seq_len(a, n);
    const int nchunks = (len + BC - 1) / BC;
    const TIn *q = (const TIn *)a.q, *k = (const TIn *)a.k, *v = (const TIn *)a.v;
    const TIn *al = (const TIn *)a.alpha, *g1 = (const TIn *)a.g1, *g2 = (const TIn *)a.g2;
    const TIn *dO = (const TIn *)g.d_o;
    const size_t soff = ((size_t)n * a.H + h) * DK * DV;
    float *scratch = g.scratch + (size_t)blockIdx.x * BC * DK * DV;   // S_{t-1} of the chunk's tokens

    // the token's vectors (fp32): k, alpha, a~, m; with grads also q, v, do and the write gate
    auto stage = [&](int t, bool bwd) {
        const size_t tok = ((size_t)row0 + t) * a.H + h;
        for (int i = tid; i < DK; i += BNT) {
            const float kk = ld_f32(k + tok * DK + i);
            const float e = (a.variant == GDN2) ? ld_f32(g1 + tok * DK + i) : ld_f32(g1 + tok);
            s_k[i] = kk;
            s_al[i] = ld_f32(al + tok * DK + i);
            s_at[i] = e * kk;
            if (bwd) s_q[i] = ld_f32(q + tok * DK + i);
        }
        for (int j = tid; j < DV; j += BNT) {
            float w;
            if (a.variant == KDA) w = ld_f32(g1 + tok);
            else if (a.variant == RDA) w = ld_f32(g2 + tok);
            else w = ld_f32(g2 + tok * DV + j);
            const float vj = ld_f32(v + tok * DV + j);
            s_m[j] = w * vj;
            if (bwd) {
                s_v[j] = vj;
                s_g2[j] = w;
                s_do[j] = ld_f32(dO + tok * DV + j);
            }
        }
    };

    // G <- dL/dS_T
    for (int e = tid; e < DK * DV; e += BNT) {
        const int i = e / DV, j = e % DV;
        G[i * P + j] = g.d_sf ? g.d_sf[soff + (size_t)i * DV + j] : 0.f;
    }
    for (int c = nchunks - 1; c >= 0; --c) {
        const int t0 = c * BC, nt = min(BC, len - t0);
        // ---- checkpoint: the state before chunk c
        const float *ck = c == 0 ? (a.s0 ? a.s0 + soff : nullptr)
                                 : a.snap + ((size_t)(slot_base(a, n) + c - 1) * a.H + h) * DK * DV;
        for (int e = tid; e < DK * DV; e += BNT) {
            const int i = e / DV, j = e % DV;
            S[i * P + j] = ck ? ck[(size_t)i * DV + j] : 0.f;
        }
        __syncthreads();
        // ---- replay the chunk forward, keeping S_{t-1} (global scratch) and u_t (shared)
        for (int tt = 0; tt < nt; ++tt) {
            stage(t0 + tt, false);
            float *sc = scratch + (size_t)tt * DK * DV;
            for (int e = tid; e < DK * DV; e += BNT) sc[e] = S[(e / DV) * P + e % DV];
            __syncthreads();
            {   // u_j = m_j - sum_i alpha_i a~_i S_ij, split over CS threads per column
                const int j = tid % DV, part = tid / DV;
                float acc = 0.f;
                for (int i = part * (DK / CS); i < (part + 1) * (DK / CS); ++i)
                    acc = fmaf(s_al[i] * s_at[i], S[i * P + j], acc);
                red[part * DV + j] = acc;
            }
            __syncthreads();
            for (int j = tid; j < DV; j += BNT) {
                float acc = 0.f;
                for (int p = 0; p < CS; ++p) acc += red[p * DV + j];
                Uc[tt * DV + j] = s_m[j] - acc;
            }
            __syncthreads();
            for (int e = tid; e < DK * DV; e += BNT) {
                const int i = e / DV, j = e % DV;
                S[i * P + j] = fmaf(s_al[i], S[i * P + j], s_k[i] * Uc[tt * DV + j]);
            }
            __syncthreads();
        }
        // ---- adjoint steps, last token first
        for (int tt = nt - 1; tt >= 0; --tt) {
            const int t = t0 + tt;
            const size_t tok = ((size_t)row0 + t) * a.H + h;
            const float *uu = Uc + tt * DV;
            stage(t, true);
            const float *sc = scratch + (size_t)tt * DK * DV;
            for (int e = tid; e < DK * DV; e += BNT) S[(e / DV) * P + e % DV] = sc[e];   // S_{t-1}
            __syncthreads();
            // G += q do^T;  u . do
            for (int e = tid; e < DK * DV; e += BNT) {
                const int i = e / DV, j = e % DV;
                G[i * P + j] = fmaf(s_q[i], s_do[j], G[i * P + j]);
            }
            if (tid < 32) {
                float d = 0.f;
                for (int j = tid; j < DV; j += 32) d = fmaf(uu[j], s_do[j], d);
#pragma unroll
                for (int off = 16; off; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
                if (tid == 0) s_sc[0] = d;
            }
            __syncthreads();
            {   // row sums: sum_j S_{t-1,ij} do_j (for dq) and sum_j G_ij u_j (for dk)
                const int i = tid % DK, part = tid / DK;
                float a0 = 0.f, a1 = 0.f;
                for (int j = part * (DV / RS); j < (part + 1) * (DV / RS); ++j) {
                    a0 = fmaf(S[i * P + j], s_do[j], a0);
                    a1 = fmaf(G[i * P + j], uu[j], a1);
                }
                red[(0 * RS + part) * DK + i] = a0;
                red[(1 * RS + part) * DK + i] = a1;
            }
            {   // column sums: du_j = sum_i k_i G_ij
                const int j = tid % DV, part = tid / DV;
                float acc = 0.f;
                for (int i = part * (DK / CS); i < (part + 1) * (DK / CS); ++i) acc = fmaf(s_k[i], G[i * P + j], acc);
                red[4 * RS * DK + part * DV + j] = acc;
            }
            __syncthreads();
            float dq_i = 0.f, gu_i = 0.f;   // kept by threads tid < DK for the outputs below
            if (tid < DK) {
                const int i = tid;
                for (int p = 0; p < RS; ++p) {
                    dq_i += red[(0 * RS + p) * DK + i];
                    gu_i += red[(1 * RS + p) * DK + i];
                }
                // dq = S_t do with S_t = Diag(alpha) S_{t-1} + k u^T
                dq_i = fmaf(s_al[i], dq_i, s_k[i] * s_sc[0]);
            }
            for (int j = tid; j < DV; j += BNT) {
                float acc = 0.f;
                for (int p = 0; p < CS; ++p) acc += red[4 * RS * DK + p * DV + j];
                s_du[j] = acc;
            }
            __syncthreads();
            // dS' = G - a~ du^T (in place)
            for (int e = tid; e < DK * DV; e += BNT) {
                const int i = e / DV, j = e % DV;
                G[i * P + j] = fmaf(-s_at[i], s_du[j], G[i * P + j]);
            }
            __syncthreads();
            {   // row sums: dalpha_i = sum_j S_{t-1,ij} dS'_ij;  sum_j S_{t-1,ij} du_j (for da~)
                const int i = tid % DK, part = tid / DK;
                float a0 = 0.f, a1 = 0.f;
                for (int j = part * (DV / RS); j < (part + 1) * (DV / RS); ++j) {
                    a0 = fmaf(S[i * P + j], G[i * P + j], a0);
                    a1 = fmaf(S[i * P + j], s_du[j], a1);
                }
                red[(2 * RS + part) * DK + i] = a0;
                red[(3 * RS + part) * DK + i] = a1;
            }
            __syncthreads();
            // G <- Diag(alpha) dS' : dL/dS_{t-1}
            for (int e = tid; e < DK * DV; e += BNT) {
                const int i = e / DV, j = e % DV;
                G[i * P + j] *= s_al[i];
            }
            // per-token gradients
            if (tid < DK) {
                const int i = tid;
                float da = 0.f, sd = 0.f;
                for (int p = 0; p < RS; ++p) {
                    da += red[(2 * RS + p) * DK + i];
                    sd += red[(3 * RS + p) * DK + i];
                }
                const float dat = -s_al[i] * sd;   // da~ = -S' du = -Diag(alpha) S_{t-1} du
                s_dat[i] = dat;
                const float e = (a.variant == GDN2) ? ld_f32(g1 + tok * DK + i) : ld_f32(g1 + tok);
                g.dq[tok * DK + i] = dq_i;
                g.dk[tok * DK + i] = fmaf(e, dat, gu_i);   // a~ = e (.) k
                g.dalpha[tok * DK + i] = da;
                if (a.variant == GDN2) g.dg1[tok * DK + i] = s_k[i] * dat;   // db_i = k_i da~_i
            }
            for (int j = tid; j < DV; j += BNT) {
                g.dv[tok * DV + j] = s_g2[j] * s_du[j];                       // m = w (.) v: dv = w dm
                if (a.variant == GDN2) g.dg2[tok * DV + j] = s_v[j] * s_du[j];   // dw_j = v_j dm_j
            }
            __syncthreads();
            if (a.variant != GDN2 && tid < 32) {   // scalar gates: sums over the channels
                float sk = 0.f, sv = 0.f;
                for (int i = tid; i < DK; i += 32) sk = fmaf(s_k[i], s_dat[i], sk);
                for (int j = tid; j < DV; j += 32) sv = fmaf(s_v[j], s_du[j], sv);
#pragma unroll
                for (int off = 16; off; off >>= 1) {
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                    sv += __shfl_xor_sync(0xffffffffu, sv, off);
                }
                if (tid == 0) {
                    if (a.variant == KDA) g.dg1[tok] = sk + sv;   // a~ = beta k, m = beta v
                    else {                                         // RDA: a~ = e k, m = w v
                        g.dg1[tok] = sk;
                        g.dg2[tok] = sv;
                    }
                }
            }
            __syncthreads();
        }
    }
    if (g.d_s0) {
        for (int e = tid; e < DK * DV; e += BNT) {
            const int i = e / DV, j = e % DV;
            g.d_s0[soff + (size_t)i * DV + j] = G[i * P + j];
        }
    }
}

template <int DK, int DV>
cudaError_t launch_bwd_dims(const FwdArgs &a, const BwdArgs &g, bool bf16, cudaStream_t st)
{
    const size_t smem = BwdSmem<DK, DV>::FLOATS * sizeof(float);
    const int N = a.cu_seqlens ? a.num_seqs : a.B;
    cudaError_t e;
    if (bf16) {
        if ((e = cudaFuncSetAttribute(scan_bwd_kernel<DK, DV, __nv_bfloat16>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        scan_bwd_kernel<DK, DV, __nv_bfloat16><<<(unsigned)(N * a.H), BNT, smem, st>>>(a, g);
    } else {
        if ((e = cudaFuncSetAttribute(scan_bwd_kernel<DK, DV, float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        scan_bwd_kernel<DK, DV, float><<<(unsigned)(N * a.H), BNT, smem, st>>>(a, g);
    }
    return cudaGetLastError();
}

template <int DK>
cudaError_t launch_bwd_dv(const FwdArgs &a, const BwdArgs &g, bool bf16, cudaStream_t st)
{
    switch (a.dv) {
    case 16: return launch_bwd_dims<DK, 16>(a, g, bf16, st);
    case 32: return launch_bwd_dims<DK, 32>(a, g, bf16, st);
    case 64: return launch_bwd_dims<DK, 64>(a, g, bf16, st);
    case 128: return launch_bwd_dims<DK, 128>(a, g, bf16, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

size_t scan_bwd_scratch_bytes(const FwdArgs &a)
{
    const long long N = a.cu_seqlens ? a.num_seqs : a.B;
    return (size_t)N * a.H * BC * a.dk * a.dv * sizeof(float);
}

cudaError_t launch_scan_bwd(const FwdArgs &a, const BwdArgs &g, bool bf16, cudaStream_t st)
{
    switch (a.dk) {
    case 16: return launch_bwd_dv<16>(a, g, bf16, st);
    case 32: return launch_bwd_dv<32>(a, g, bf16, st);
    case 64: return launch_bwd_dv<64>(a, g, bf16, st);
    case 128: return launch_bwd_dv<128>(a, g, bf16, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda
