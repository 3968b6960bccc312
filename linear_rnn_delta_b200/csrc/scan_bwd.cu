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
// token: each sequence's 64-token chunks are walked from last to first; each
// chunk is replayed forward from its checkpoint (the state snapshot the forward
// scan stored after the previous chunk), then walked backwards.
//
// Both directions act on the columns of S and G independently (the left
// factors Diag(alpha) and I - k a~^T are shared by all value columns; m_j and
// do_j touch column j only).  The main kernel (d_k >= 32) therefore splits the
// d_v columns over a cluster of CTAs, 32 columns each (16 at d_v = 16), and
// gives every thread one row of S and G in registers: sums over value columns
// are in-thread, sums over key rows are a warp reduce-scatter plus one CTA
// barrier.  The per-row results (dq, dk, dalpha, k (.) da~) are partial sums
// over the CTA's columns; the cluster
// adds them through distributed shared memory every 8 tokens, in a fixed order
// (deterministic results).  The checkpoint scan also keeps u_t of every token,
// so the replay of a chunk is the state update alone (no sum over key rows, no
// barrier), bitwise the scan's own steps.  It keeps S_{t-1} only every 4 tokens
// (global scratch) with u_t in shared memory; the backward walk recomputes the
// states in between with the same fused multiply-adds, so they are bitwise
// those of the replay.  d_k = 16 uses a plain shared-memory kernel (one CTA per
// sequence and head) that replays with its own sums.
#include "scan_bwd.cuh"

#include <cooperative_groups.h>

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

// ---------------------------------------------------------------------------
// Row-resident kernel: a cluster of DV / DVB CTAs per (sequence, head), DK
// threads per CTA (thread i = row i), DVB value columns per CTA.

namespace cg = cooperative_groups;

constexpr int CKP = 4;   // tokens between stored states within a chunk
constexpr int RTB = 8;   // tokens per cross-CTA reduction block

template <int DK, int DVB>
struct RowSmem {
    static constexpr int NW = DK / 32;
    static constexpr size_t U = 0;                               // [BC][DVB] u_t of the chunk (from the scan)
    static constexpr size_t DO = U + (size_t)BC * DVB;           // [BC][DVB] do_t
    static constexpr size_t VV = DO + (size_t)BC * DVB;          // [BC][DVB] v_t
    static constexpr size_t WW = VV + (size_t)BC * DVB;          // [BC][DVB] write gate (scalar gates broadcast)
    static constexpr size_t PART = WW + (size_t)BC * DVB;        // [2][NW][DVB] per-warp column sums
    static constexpr size_t FIN = PART + 2 * NW * DVB;           // [NW][DVB] column totals, one copy per warp
    static constexpr size_t RING = FIN + NW * DVB;               // [2][RTB][4][DK] per-token row partials
    static constexpr size_t RINGV = RING + 2 * RTB * 4 * DK;     // [2][RTB] partial sum_j v_j du_j
    static constexpr size_t SRED = RINGV + 2 * RTB;              // [RTB][NW] warp sums of k_i da~_i
    static constexpr size_t TOK = SRED + RTB * NW;               // [2][RTB] token index (int)
    static constexpr size_t CKB = TOK + 2 * RTB;                 // [2][DVB/4][DK] float4: a group's stored state
    static constexpr size_t RSM = CKB + 2 * (size_t)DVB * DK;    // [CKP][4][DK] row scalars of a group
    static constexpr size_t UDO = RSM + (size_t)CKP * 4 * DK;    // [BC] sum_j u_j do_j over the CTA's columns
    static constexpr size_t FLOATS = UDO + BC;
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Sums x over the warp's 32 lanes for every column: on return x[0] holds the
// total of column lane / (32 / L) (a butterfly that halves the vector at each
// exchange; the last exchanges, when L < 32, add duplicates).
template <int L>
__device__ __forceinline__ void reduce_scatter(float (&x)[L], int lane)
{
#pragma unroll
    for (int half = L / 2, off = 16; half >= 1; half /= 2, off /= 2) {
        const bool upper = lane & off;
#pragma unroll
        for (int e = 0; e < half; ++e) {
            const float send = upper ? x[e] : x[e + half];
            const float keep = upper ? x[e + half] : x[e];
            x[e] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
#pragma unroll
    for (int off = 16 / L; off >= 1; off /= 2) x[0] += __shfl_xor_sync(0xffffffffu, x[0], off);
}

// Prefetched scalars stay in the input dtype until used: widening a bf16 load
// right away would wait for the load inside the barrier-delimited region that
// issued it.
__device__ __forceinline__ float widen(float x) { return x; }
__device__ __forceinline__ float widen(__nv_bfloat16 x) { return __bfloat162float(x); }

template <int DK, int DVB, typename TIn>
__global__ void __launch_bounds__(DK) scan_bwd_rows_kernel(FwdArgs a, BwdArgs g)
{
    using L = RowSmem<DK, DVB>;
    constexpr int NW = L::NW, LPC = 32 / DVB, NQ = DVB / 4;
    extern __shared__ __align__(16) float smf[];
    float *sU = smf + L::U, *sDO = smf + L::DO, *sV = smf + L::VV, *sW = smf + L::WW;
    int *tokrow = reinterpret_cast<int *>(smf + L::TOK);
    cg::cluster_group cl = cg::this_cluster();
    const int NB = a.dv / DVB;
    const int rank = (int)cl.block_rank();
    const int hh = blockIdx.x / NB, jb = blockIdx.x % NB;
    const int n = hh / a.H, h = hh % a.H;
    const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
    const bool owner = lane % LPC == 0;   // holds column lane / LPC after a reduce-scatter
    const int col = lane / LPC;
    const int row0 = seq_row0(a, n), len = seq_len(a, n);
    const TIn *q = (const TIn *)a.q, *k = (const TIn *)a.k, *v = (const TIn *)a.v;
    const TIn *al = (const TIn *)a.alpha, *g1 = (const TIn *)a.g1, *g2 = (const TIn *)a.g2;
    const TIn *dO = (const TIn *)g.d_o;
    const bool vec_gate = a.variant == GDN2;
    // row i of this CTA's column block in a [dk][dv] state
    const size_t srow = (((size_t)n * a.H + h) * DK + i) * a.dv + (size_t)jb * DVB;
    float4 *scr = reinterpret_cast<float4 *>(g.scratch) + (size_t)blockIdx.x * (BC / CKP) * NQ * DK;

    // row i of S and G, as column pairs (2p, 2p + 1): elementwise work goes
    // through the packed fp32 pipe, each lane with the scalar form's fused
    // multiply-add in the scalar form's order
    float2 S[DVB / 2], G[DVB / 2];
    auto load_row = [&](float2 (&dst)[DVB / 2], const float *src) {
#pragma unroll
        for (int c4 = 0; c4 < NQ; ++c4) {
            const float4 x = src ? reinterpret_cast<const float4 *>(src)[c4] : make_float4(0.f, 0.f, 0.f, 0.f);
            dst[2 * c4] = make_float2(x.x, x.y);
            dst[2 * c4 + 1] = make_float2(x.z, x.w);
        }
    };
    auto dup = [](float x) { return make_float2(x, x); };
    auto tok_of = [&](int t) { return ((size_t)row0 + t) * a.H + h; };
    auto gate_raw = [&](size_t tok) { return vec_gate ? g1[tok * DK + i] : g1[tok]; };
    // column sums over the CTA's rows of x (destroyed); returns nothing, leaves the
    // totals in `fin` (this warp's copy) after a CTA barrier and a warp barrier
    unsigned red_count = 0;
    auto column_sums = [&](float (&x)[DVB]) -> float * {
        reduce_scatter<DVB>(x, lane);
        float *part = smf + L::PART + (red_count & 1) * NW * DVB;
        ++red_count;
        if (owner) part[warp * DVB + col] = x[0];
        __syncthreads();
        float *fin = smf + L::FIN + warp * DVB;
        if (owner) {
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) acc += part[w * DVB + col];
            fin[col] = acc;
        }
        __syncwarp();
        return fin;
    };

    load_row(G, g.d_sf ? g.d_sf + srow : nullptr);
    int blk = 0, pos = 0;   // cross-CTA reduction block and position in it
    const int nchunks = (len + BC - 1) / BC;
    for (int c = nchunks - 1; c >= 0; --c) {
        const int t0 = c * BC, nt = min(BC, len - t0);
        __syncthreads();   // the previous chunk's readers of the staged vectors are done
        constexpr int SB = 8;   // elements per thread loaded before any is widened
        for (int e0 = i; e0 < nt * DVB; e0 += DK * SB) {
            TIn rv[SB], rw[SB], rd[SB];
            float ru[SB];
#pragma unroll
            for (int b = 0; b < SB; ++b) {
                const int e = e0 + b * DK;
                if (e < nt * DVB) {
                    const size_t tok = tok_of(t0 + e / DVB);
                    const size_t cj = tok * a.dv + (size_t)jb * DVB + e % DVB;
                    rv[b] = v[cj];
                    rw[b] = a.variant == KDA ? g1[tok] : (a.variant == RDA ? g2[tok] : g2[cj]);
                    rd[b] = dO[cj];
                    ru[b] = g.u[cj];
                }
            }
#pragma unroll
            for (int b = 0; b < SB; ++b) {
                const int e = e0 + b * DK;
                if (e < nt * DVB) {
                    sV[e] = widen(rv[b]);
                    sW[e] = widen(rw[b]);
                    sDO[e] = widen(rd[b]);
                    sU[e] = ru[b];
                }
            }
        }
        load_row(S, c == 0 ? (a.s0 ? a.s0 + srow : nullptr)
                           : a.snap + (((size_t)(slot_base(a, n) + c - 1) * a.H + h) * DK + i) * a.dv +
                                 (size_t)jb * DVB);
        __syncthreads();
        for (int tt = i; tt < nt; tt += DK) {   // per token: sum over the CTA's columns of u_j do_j (row-independent)
            const float4 *d4p = reinterpret_cast<const float4 *>(sDO + tt * DVB);
            const float4 *u4p = reinterpret_cast<const float4 *>(sU + tt * DVB);
            float2 udo = make_float2(0.f, 0.f);
#pragma unroll
            for (int c4 = 0; c4 < NQ; ++c4) {
                const float4 d4 = d4p[c4], u4 = u4p[c4];
                udo = __ffma2_rn(make_float2(u4.x, u4.y), make_float2(d4.x, d4.y), udo);
                udo = __ffma2_rn(make_float2(u4.z, u4.w), make_float2(d4.z, d4.w), udo);
            }
            smf[L::UDO + tt] = udo.x + udo.y;
        }
        // ---- replay: S_{t-1} every CKP tokens into scratch.  u_t comes from the checkpoint
        // scan, so a step is the update S_ij = alpha_i S_ij + k_i u_j alone (the scan's own
        // fused multiply-add: the replayed states are the scan's, bit for bit), with no sum
        // over rows and no barrier
        TIn n_al = TIn(0.f), n_k = TIn(0.f);   // next token's row scalars, raw
        if (nt > 0) {
            const size_t tok = tok_of(t0);
            n_al = al[tok * DK + i]; n_k = k[tok * DK + i];
        }
        for (int tt = 0; tt < nt; ++tt) {
            const float alpha_i = widen(n_al), k_i = widen(n_k);
            if (tt + 1 < nt) {
                const size_t tok = tok_of(t0 + tt + 1);
                n_al = al[tok * DK + i]; n_k = k[tok * DK + i];
            }
            if (tt % CKP == 0) {
#pragma unroll
                for (int c4 = 0; c4 < NQ; ++c4)
                    scr[((size_t)(tt / CKP) * NQ + c4) * DK + i] =
                        make_float4(S[2 * c4].x, S[2 * c4].y, S[2 * c4 + 1].x, S[2 * c4 + 1].y);
            }
            const float4 *u4p = reinterpret_cast<const float4 *>(sU + tt * DVB);
#pragma unroll
            for (int c4 = 0; c4 < NQ; ++c4) {
                const float4 u4 = u4p[c4];
                S[2 * c4] = __ffma2_rn(dup(alpha_i), S[2 * c4], __fmul2_rn(dup(k_i), make_float2(u4.x, u4.y)));
                S[2 * c4 + 1] = __ffma2_rn(dup(alpha_i), S[2 * c4 + 1], __fmul2_rn(dup(k_i), make_float2(u4.z, u4.w)));
            }
        }
        __syncthreads();   // the replay is done (and its scratch stores ordered) before the walk reads them back
        // ---- backward walk, last token first, in groups of CKP tokens (one stored state each)
        const int ngrp = (nt + CKP - 1) / CKP;
        float4 *ckb = reinterpret_cast<float4 *>(smf + L::CKB);   // [2][NQ][DK]: each thread its own row
        float c_al[CKP], c_k[CKP];   // alpha_i, k_i of the current group's tokens (recompute steps)
        float *rsm = smf + L::RSM;   // [CKP][4][DK]: alpha, k, q, e of the group's tokens, own row only
        TIn f_al[CKP], f_k[CKP], f_q[CKP], f_e[CKP];   // of the next group (prefetched, raw)
#pragma unroll
        for (int s = 0; s < CKP; ++s) f_al[s] = f_k[s] = f_q[s] = f_e[s] = TIn(0.f);
        // pass gi fetches group gi - 1 (stored state by cp.async, row scalars into
        // registers) while it works on group gi, fetched by the pass before
        for (int gi = ngrp; gi >= 0; --gi) {
            const int grp = gi, buf = gi & 1;
#pragma unroll
            for (int s = 0; s < CKP; ++s) {
                c_al[s] = widen(f_al[s]);
                c_k[s] = widen(f_k[s]);
                rsm[(s * 4 + 0) * DK + i] = c_al[s];
                rsm[(s * 4 + 1) * DK + i] = c_k[s];
                rsm[(s * 4 + 2) * DK + i] = widen(f_q[s]);
                rsm[(s * 4 + 3) * DK + i] = widen(f_e[s]);
            }
            cp_async_wait_all();
            if (gi > 0) {
                const int fg = gi - 1, fb = fg & 1;
#pragma unroll
                for (int c4 = 0; c4 < NQ; ++c4)
                    cp_async16(&ckb[((size_t)fb * NQ + c4) * DK + i], &scr[((size_t)fg * NQ + c4) * DK + i]);
                cp_async_commit();
                const int fn = min(CKP, nt - fg * CKP);
#pragma unroll
                for (int s = 0; s < CKP; ++s) {
                    if (s < fn) {
                        const size_t tok = tok_of(t0 + fg * CKP + s);
                        f_al[s] = al[tok * DK + i];
                        f_k[s] = k[tok * DK + i];
                        f_q[s] = q[tok * DK + i];
                        f_e[s] = gate_raw(tok);
                    }
                }
            }
            if (gi == ngrp) continue;
            const int ntok = min(CKP, nt - grp * CKP);
            for (int r = ntok - 1; r >= 0; --r) {
                const int tt = grp * CKP + r;
                // S_{t-1}: the group's stored state advanced over its first r tokens (the replay's own steps)
#pragma unroll
                for (int c4 = 0; c4 < NQ; ++c4) {
                    const float4 x = ckb[((size_t)buf * NQ + c4) * DK + i];
                    S[2 * c4] = make_float2(x.x, x.y);
                    S[2 * c4 + 1] = make_float2(x.z, x.w);
                }
                const float alpha_i = rsm[(r * 4 + 0) * DK + i], k_i = rsm[(r * 4 + 1) * DK + i];
                const float q_i = rsm[(r * 4 + 2) * DK + i], e_i = rsm[(r * 4 + 3) * DK + i];
#pragma unroll
                for (int s = 0; s < CKP - 1; ++s) {
                    if (s < r) {
                        const float4 *u4p = reinterpret_cast<const float4 *>(sU + (grp * CKP + s) * DVB);
#pragma unroll
                        for (int c4 = 0; c4 < NQ; ++c4) {
                            const float4 u4 = u4p[c4];
                            S[2 * c4] = __ffma2_rn(dup(c_al[s]), S[2 * c4],
                                                   __fmul2_rn(dup(c_k[s]), make_float2(u4.x, u4.y)));
                            S[2 * c4 + 1] = __ffma2_rn(dup(c_al[s]), S[2 * c4 + 1],
                                                       __fmul2_rn(dup(c_k[s]), make_float2(u4.z, u4.w)));
                        }
                    }
                }
                const int t = t0 + tt;
                const size_t tok = tok_of(t);
                const float4 *do4 = reinterpret_cast<const float4 *>(sDO + tt * DVB);
                const float4 *u4p = reinterpret_cast<const float4 *>(sU + tt * DVB);
                // G += q do^T;  row partials of S_t do (= alpha S_{t-1} do + k (u.do), u.do summed once
                // per token above) and G u (partial sums over even and odd columns in .x and .y)
                float2 sdo = make_float2(0.f, 0.f), gu = sdo;
#pragma unroll
                for (int c4 = 0; c4 < NQ; ++c4) {
                    const float4 d4 = do4[c4], u4 = u4p[c4];
                    const float2 dd[2] = {make_float2(d4.x, d4.y), make_float2(d4.z, d4.w)};
                    const float2 uu[2] = {make_float2(u4.x, u4.y), make_float2(u4.z, u4.w)};
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j2 = 2 * c4 + e;
                        G[j2] = __ffma2_rn(dup(q_i), dd[e], G[j2]);
                        sdo = __ffma2_rn(S[j2], dd[e], sdo);
                        gu = __ffma2_rn(G[j2], uu[e], gu);
                    }
                }
                // du_j = sum_i k_i G_ij
                float x[DVB];
#pragma unroll
                for (int j2 = 0; j2 < DVB / 2; ++j2) {
                    const float2 t = __fmul2_rn(dup(k_i), G[j2]);
                    x[2 * j2] = t.x;
                    x[2 * j2 + 1] = t.y;
                }
                float *fin = column_sums(x);
                if (warp == 0) {   // per-column outputs: dv = w du;  GDN-2 dw = v du;  scalar gates: sum_j v_j du_j
                    float vdu = 0.f;
                    if (owner) {
                        const float du = fin[col], vj = sV[tt * DVB + col];
                        const size_t cj = tok * a.dv + (size_t)jb * DVB + col;
                        g.dv[cj] = sW[tt * DVB + col] * du;
                        if (vec_gate) g.dg2[cj] = vj * du;
                        vdu = vj * du;
                    }
                    if (!vec_gate) {
#pragma unroll
                        for (int off = 16; off; off >>= 1) vdu += __shfl_xor_sync(0xffffffffu, vdu, off);
                        if (lane == 0) smf[L::RINGV + (blk & 1) * RTB + pos] = vdu;
                    }
                }
                // dS' = G - a~ du^T;  dalpha = rowsum(S_{t-1} dS');  S_{t-1} du;  G <- Diag(alpha) dS'
                const float at = e_i * k_i;
                float2 sds = make_float2(0.f, 0.f), sdu = sds;
#pragma unroll
                for (int c4 = 0; c4 < NQ; ++c4) {
                    const float4 du4 = reinterpret_cast<const float4 *>(fin)[c4];
                    const float2 du[2] = {make_float2(du4.x, du4.y), make_float2(du4.z, du4.w)};
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j2 = 2 * c4 + e;
                        G[j2] = __ffma2_rn(dup(-at), du[e], G[j2]);
                        sds = __ffma2_rn(S[j2], G[j2], sds);
                        sdu = __ffma2_rn(S[j2], du[e], sdu);
                        G[j2] = __fmul2_rn(G[j2], dup(alpha_i));
                    }
                }
                // this CTA's parts (its value columns) of dq, dk, dalpha and k (.) da~, da~ = -Diag(alpha) S_{t-1} du
                const float datp = -alpha_i * (sdu.x + sdu.y);
                float *ring = smf + L::RING + ((size_t)((blk & 1) * RTB + pos) * 4) * DK;
                ring[i] = fmaf(alpha_i, sdo.x + sdo.y, k_i * smf[L::UDO + tt]);
                ring[DK + i] = fmaf(e_i, datp, gu.x + gu.y);   // a~ = e (.) k: dk = G u + e da~
                ring[2 * DK + i] = sds.x + sds.y;
                ring[3 * DK + i] = k_i * datp;
                if (i == 0) tokrow[(blk & 1) * RTB + pos] = t;
                ++pos;
                if (pos == RTB || (c == 0 && tt == 0)) {   // add the cluster's parts for this block of tokens
                    const int rb = blk & 1, cnt = pos;
                    cl.sync();
                    for (int p = rank; p < cnt; p += NB) {
                        float sum[4] = {0.f, 0.f, 0.f, 0.f};
                        for (int cr = 0; cr < NB; ++cr) {
                            const float *rr =
                                cl.map_shared_rank(smf + L::RING + (size_t)((rb * RTB + p) * 4) * DK, cr);
#pragma unroll
                            for (int qd = 0; qd < 4; ++qd) sum[qd] += rr[qd * DK + i];
                        }
                        const size_t tk = tok_of(tokrow[rb * RTB + p]);
                        g.dq[tk * DK + i] = sum[0];
                        g.dk[tk * DK + i] = sum[1];
                        g.dalpha[tk * DK + i] = sum[2];
                        if (vec_gate) {
                            g.dg1[tk * DK + i] = sum[3];   // db_i = k_i da~_i
                        } else {
                            float sk = sum[3];
#pragma unroll
                            for (int off = 16; off; off >>= 1) sk += __shfl_xor_sync(0xffffffffu, sk, off);
                            if (lane == 0) smf[L::SRED + p * NW + warp] = sk;
                        }
                    }
                    if (!vec_gate) {
                        __syncthreads();
                        if (i < cnt && i % NB == rank) {   // scalar gates of token position i
                            const int p = i;
                            float sk = 0.f, sv = 0.f;
#pragma unroll
                            for (int w = 0; w < NW; ++w) sk += smf[L::SRED + p * NW + w];
                            for (int cr = 0; cr < NB; ++cr)
                                sv += *cl.map_shared_rank(smf + L::RINGV + rb * RTB + p, cr);
                            const size_t tk = tok_of(tokrow[rb * RTB + p]);
                            if (a.variant == KDA) {
                                g.dg1[tk] = sk + sv;   // a~ = beta k, m = beta v
                            } else {
                                g.dg1[tk] = sk;        // RDA: a~ = e k, m = w v
                                g.dg2[tk] = sv;
                            }
                        }
                    }
                    ++blk;
                    pos = 0;
                }
            }
        }
    }
    if (g.d_s0) {
        float4 *dst = reinterpret_cast<float4 *>(g.d_s0 + srow);
#pragma unroll
        for (int c4 = 0; c4 < NQ; ++c4) dst[c4] = make_float4(G[2 * c4].x, G[2 * c4].y, G[2 * c4 + 1].x, G[2 * c4 + 1].y);
    }
    cl.sync();   // no CTA leaves while the cluster may still read its shared memory
}

template <int DK, int DVB>
cudaError_t launch_rows_dims(const FwdArgs &a, const BwdArgs &g, bool bf16, cudaStream_t st)
{
    const size_t smem = RowSmem<DK, DVB>::FLOATS * sizeof(float);
    const int N = a.cu_seqlens ? a.num_seqs : a.B;
    const int NB = a.dv / DVB;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(N * a.H * NB));
    cfg.blockDim = dim3(DK);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NB;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (bf16) {
        auto *kern = scan_bwd_rows_kernel<DK, DVB, __nv_bfloat16>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        e = cudaLaunchKernelEx(&cfg, kern, a, g);
    } else {
        auto *kern = scan_bwd_rows_kernel<DK, DVB, float>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        e = cudaLaunchKernelEx(&cfg, kern, a, g);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int DK>
cudaError_t launch_rows_dv(const FwdArgs &a, const BwdArgs &g, bool bf16, cudaStream_t st)
{
    // 16 columns per CTA for d_v = 16, else 32 (clusters of 1, 2 or 4 CTAs)
    return a.dv == 16 ? launch_rows_dims<DK, 16>(a, g, bf16, st) : launch_rows_dims<DK, 32>(a, g, bf16, st);
}

}  // namespace

size_t scan_bwd_scratch_bytes(const FwdArgs &a)
{
    // d_k = 16: every S_{t-1} of a chunk; otherwise every CKP-th
    const long long N = a.cu_seqlens ? a.num_seqs : a.B;
    return (size_t)N * a.H * (a.dk == 16 ? BC : BC / CKP) * a.dk * a.dv * sizeof(float);
}

cudaError_t launch_scan_bwd(const FwdArgs &a, const BwdArgs &g, bool bf16, cudaStream_t st)
{
    if (a.dv % 16 != 0 || a.dv < 16 || a.dv > 128) return cudaErrorInvalidValue;
    switch (a.dk) {
    case 16: return launch_bwd_dv<16>(a, g, bf16, st);
    case 32: return launch_rows_dv<32>(a, g, bf16, st);
    case 64: return launch_rows_dv<64>(a, g, bf16, st);
    case 128: return launch_rows_dv<128>(a, g, bf16, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda
