// Chunked-parallel forward of the gated delta-rule recurrence on sm_100a
// tensor cores (bf16 inputs, d_k = d_v = 128, chunk C = 64).
//
// Recurrence (update equations on the Raon-1-mini-preview discussion page):
//   S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T,   u_t = m_t - (Diag(alpha_t) S_{t-1})^T a~_t,
//   o_t = S_t^T q_t,
// with (a~, m) = (beta k, beta v) for KDA / Complex KDA, (e k, w v) for RDA and
// (b (.) k, w (.) v) for GDN-2.  Unrolled over a chunk of C tokens that starts
// from state S0 (positions r, s in 0..C-1, all products forward, never divided):
//   Gamma_r      = prod_{t<=r} alpha_t                      (per key channel)
//   Lam_{r,s}    = prod_{s<t<=r} alpha_t
//   A_{r,s}      = sum_c a~_{r,c} Lam_{r,s,c} k_{s,c}        (s < r)
//   P_{r,s}      = sum_c q_{r,c}  Lam_{r,s,c} k_{s,c}        (s <= r)
//   T            = (I + A)^{-1}                             (UT transform)
//   W            = T (Gamma (.) A~),    U = T M - W S0        (WY form)
//   O            = (Gamma (.) Q) S0 + P U
//   S_C          = Diag(Gamma_C) S0 + Kbar^T U,   Kbar_s = Lam_{C-1,s} (.) k_s
// Because alpha may be negative or zero (Complex KDA gates in [-1,1]), no
// log-space cumulative sum and no ratio Gamma_r / Gamma_s is ever formed:
// A and P are built from "anchored" forward products.  At level L = 1..6 the
// chunk is cut into blocks of 2h tokens (h = 32 >> (L-1)); for a row r in a
// block's second half and a column s in its first half, with anchor
// a = last token of the first half,
//   Lam_{r,s} = (prod_{a<t<=r} alpha_t) (.) (prod_{s<t<=a} alpha_t),
// so that level's pairs are one dense product of "row factors" and "column
// factors" (a tensor-core GEMM with K = d_k).  The six levels cover every
// pair s < r exactly once; the diagonal P_{r,r} = q_r . k_r is a dot product.
//
// One CTA per (sequence, head); the d_k x d_v fp32 state lives in tensor
// memory (TMEM) for the whole sequence, transposed (lane = value column j,
// column = key channel i), so every state-dependent GEMM has M = d_v = 128.
// q, k, v, alpha tiles arrive by TMA; every other operand is produced on chip
// in 128-byte-swizzled shared-memory tiles.  Per chunk:
//   1. TMA raw tiles -> decay products, Gamma(.)Q, Gamma(.)A~, Kbar, M
//   2. level factors -> three tcgen05 GEMMs (M=128, N=64) -> A, P
//   3. T = (I + A)^{-1} by blocked forward substitution (fp32, SIMT)
//   4. tcgen05: W = T (Gamma(.)A~);  U^T = M^T T^T
//   5. tcgen05: U^T -= S0^T W^T;  O^T = S0^T (Gamma(.)Q)^T;  S^T *= Gamma_C
//   6. tcgen05: O^T += U^T P^T;  S^T += U^T Kbar  -> o to HBM, S^T -> bf16 copy
// The next chunk's TMA loads are issued as soon as step 2 has consumed the
// raw tiles.
#include <cuda.h>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {
using namespace sm100;

constexpr int C = 64;    // chunk length
constexpr int D = 128;   // d_k = d_v
constexpr int NT = 256;  // threads per CTA

// ---- shared memory map (offsets from a 1024-byte aligned base) ------------
constexpr uint32_t RAW_Q = 0, RAW_K = 16384, RAW_V = 32768, RAW_A = 49152;  // TMA tiles [64][128] bf16
constexpr uint32_t OFF_S0T = 65536;   // S^T bf16, 128 x 128, K-major (rows j, K = i)
constexpr uint32_t OFF_QG = 98304;    // Gamma (.) q      [token][channel] tile
constexpr uint32_t OFF_KB = 114688;   // Kbar             [token][channel]
constexpr uint32_t OFF_AG = 131072;   // Gamma (.) a~     [token][channel]; later W
constexpr uint32_t OFF_MT = 147456;   // M                [token][channel]; later U^T (128 x 64)
constexpr uint32_t OFF_F = 163840;    // level factors; later A, T (fp32), T, P (bf16)
constexpr uint32_t OFF_FA = OFF_F;            // 128 rows x 128 ch (32 KB)
constexpr uint32_t OFF_FB = OFF_F + 32768;    // 64 rows x 128 ch (16 KB)
constexpr uint32_t OFF_AF32 = OFF_F;          // A  fp32 [64][65]
constexpr uint32_t OFF_TF32 = OFF_F + 16640;  // T  fp32 [64][65]
constexpr uint32_t OFF_X = OFF_F + 33280;     // 3 x 16 x 16 fp32 scratch of the block solve
constexpr uint32_t OFF_TBF = OFF_F + 36864;   // T bf16 64 x 64 K-major
constexpr uint32_t OFF_PBF = OFF_F + 45056;   // P bf16 64 x 64 K-major
constexpr uint32_t OFF_MISC = OFF_F + 53248;
constexpr uint32_t M_G1 = OFF_MISC, M_G2 = OFF_MISC + 256, M_GAMC = OFF_MISC + 512, M_TOT = OFF_MISC + 1024,
                   M_PDIAG = OFF_MISC + 5120, M_BAR = OFF_MISC + 5376, M_TMEM = OFF_MISC + 5408,
                   M_FLAG = OFF_MISC + 5412;
constexpr uint32_t SMEM_USED = OFF_MISC + 5440;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;  // slack for aligning the base
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// ---- TMEM columns ---------------------------------------------------------
constexpr uint32_t TM_S = 0, TM_U = 128, TM_O = 192, TM_W = 256;
__device__ __forceinline__ uint32_t tm_ap(int p) { return p == 0 ? 384u : (p == 1 ? 448u : 256u); }

constexpr long long WAIT_CYCLES = 4000000000ll;  // ~2 s: only a broken pipeline gets near it

struct ChunkParams {
    CUtensorMap tq, tk, tv, ta;  // [B*T][H][128] bf16, box {128, 1, 64}
    FwdArgs a;
};

// ---- small helpers --------------------------------------------------------
__device__ __forceinline__ void unpack8(const uint4 &u, float *f)
{
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ uint4 pack8(const float *f)
{
    return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
}
// 16-byte chunk kc (8 consecutive K elements) of row `row` in a K-major
// 128B-swizzled tile with `rows` rows: 64-element panels of rows*128 bytes.
__device__ __forceinline__ uint32_t sw_chunk(uint32_t rows, uint32_t row, uint32_t kc)
{
    return (kc >> 3) * (rows * 128u) + row * 128u + ((((kc & 7u) ^ (row & 7u))) << 4);
}
__device__ __forceinline__ uint32_t sw_elem(uint32_t rows, uint32_t row, uint32_t k)
{
    return sw_chunk(rows, row, k >> 3) + (k & 7u) * 2u;
}
// raw TMA tile: row-major [64][128] bf16
__device__ __forceinline__ uint4 raw_row(const uint8_t *sm, uint32_t base, int r, int cg)
{
    return *reinterpret_cast<const uint4 *>(sm + base + r * 256 + cg * 16);
}

// K-major descriptor of a 128B-swizzled tile, K step kk (16 elements)
__device__ __forceinline__ uint64_t dK(uint32_t base, uint32_t rows, int kk)
{
    return make_desc_sw128(base + (uint32_t)(kk >> 2) * rows * 128u + (uint32_t)(kk & 3) * 32u, 16);
}
// MN-major descriptor of a [token][channel] tile (MN = 128 channels in two
// 64-wide panels 8 KB apart, K = tokens), K step kk (16 tokens)
__device__ __forceinline__ uint64_t dMN(uint32_t base, int kk)
{
    return make_desc_sw128(base + (uint32_t)kk * 2048u, 8192);
}

__device__ __forceinline__ float g_scalar(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }

// ---- the kernel -------------------------------------------------------------
__global__ void __launch_bounds__(NT, 1) chunk_fwd_kernel(const __grid_constant__ ChunkParams P)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);
    const FwdArgs &a = P.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;                      // TMEM lane quarter of this warp
    const int H = a.H;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    int b, t0, len;
    if (a.cu_seqlens) { b = 0; t0 = a.cu_seqlens[n]; len = a.cu_seqlens[n + 1] - t0; }
    else { b = n; t0 = 0; len = a.T; }
    const int nchunks = (len + C - 1) / C;

    float *s_g1 = reinterpret_cast<float *>(sm + M_G1);
    float *s_g2 = reinterpret_cast<float *>(sm + M_G2);
    float *s_gamC = reinterpret_cast<float *>(sm + M_GAMC);
    float *s_tot = reinterpret_cast<float *>(sm + M_TOT);   // [8][128]
    float *s_pdiag = reinterpret_cast<float *>(sm + M_PDIAG);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + M_BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + M_TMEM);
    float *Af = reinterpret_cast<float *>(sm + OFF_AF32);
    float *Tf = reinterpret_cast<float *>(sm + OFF_TF32);
    float *Xs = reinterpret_cast<float *>(sm + OFF_X);

    const __nv_bfloat16 *g1p = (const __nv_bfloat16 *)a.g1, *g2p = (const __nv_bfloat16 *)a.g2;
    __nv_bfloat16 *op = (__nv_bfloat16 *)a.o;
    const bool gdn2 = a.variant == GDN2;

    if (warp == 0) tmem_alloc(s_tmem, 512);
    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    uint32_t ph_tma = 0, ph_mma = 0;
    bool ok = true;

    const CUtensorMap *map_q = &P.tq, *map_k = &P.tk, *map_v = &P.tv, *map_a = &P.ta;
    auto issue_tma = [&](int chunk) {
        const int g = b * a.T + t0 + chunk * C;  // token row of the packed [B*T] axis
        mbar_expect_tx(bar_tma, 4 * 16384);
        tma_load_3d(sm + RAW_Q, map_q, bar_tma, 0, h, g);
        tma_load_3d(sm + RAW_K, map_k, bar_tma, 0, h, g);
        tma_load_3d(sm + RAW_V, map_v, bar_tma, 0, h, g);
        tma_load_3d(sm + RAW_A, map_a, bar_tma, 0, h, g);
    };
    // all threads: wait for the MMAs committed so far, then order TMEM reads after them
    auto wait_mma = [&]() {
        if (!mbar_wait_cycles(bar_mma, ph_mma, WAIT_CYCLES)) ok = false;
        ph_mma ^= 1;
        tc_fence_after();
    };
    // all threads: publish shared-memory / TMEM writes to the tensor core, then barrier
    auto publish = [&]() {
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
    };

    if (nchunks > 0 && tid == 0) issue_tma(0);

    // ---- initial state -> TMEM (fp32) and S0^T (bf16) ----------------------
    {
        const size_t soff = ((size_t)n * H + h) * D * D;
        const int j = quarter * 32 + lane;          // value column = TMEM lane
        const int ihalf = warp >> 2;                // key channels [64*ihalf, +64)
        for (int c16 = 0; c16 < 4; ++c16) {
            float v[16];
            const int i0 = ihalf * 64 + c16 * 16;
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = a.s0 ? a.s0[soff + (size_t)(i0 + e) * D + j] : 0.f;
            tmem_st16(tbase + lane_base + TM_S + i0, v);
            *reinterpret_cast<uint4 *>(sm + OFF_S0T + sw_chunk(128, j, i0 >> 3)) = pack8(v);
            *reinterpret_cast<uint4 *>(sm + OFF_S0T + sw_chunk(128, j, (i0 >> 3) + 1)) = pack8(v + 8);
        }
        tmem_wait_st();
    }
    publish();

    for (int ch = 0; ch < nchunks && ok; ++ch) {
        const int tok0 = t0 + ch * C;
        const int nvalid = min(C, len - ch * C);
        const size_t rowbase = (size_t)b * a.T + tok0;   // packed token index of chunk row 0

        // gate scalars (masked to 0 past the sequence end)
        if (tid < C) {
            const bool v = tid < nvalid;
            const size_t tok = (rowbase + tid) * H + h;
            if (!gdn2) {
                s_g1[tid] = v ? g_scalar(g1p, tok) : 0.f;
                s_g2[tid] = v ? (a.variant == KDA ? g_scalar(g1p, tok) : g_scalar(g2p, tok)) : 0.f;
            }
        }
        if (!mbar_wait_cycles(bar_tma, ph_tma, WAIT_CYCLES)) ok = false;
        ph_tma ^= 1;
        __syncthreads();  // gate scalars visible to every thread

        // ===== 1a. block totals of alpha; M; diagonal of P ====================
        if (tid < 128) {
            const int tg = tid >> 4, cg = tid & 15;
            float tot[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) tot[c] = 1.f;
            for (int i = 0; i < 8; ++i) {
                const int r = tg * 8 + i;
                if (r < nvalid) {
                    float al[8];
                    unpack8(raw_row(sm, RAW_A, r, cg), al);
#pragma unroll
                    for (int c = 0; c < 8; ++c) tot[c] *= al[c];
                }
            }
            *reinterpret_cast<float4 *>(s_tot + tg * 128 + cg * 8) = make_float4(tot[0], tot[1], tot[2], tot[3]);
            *reinterpret_cast<float4 *>(s_tot + tg * 128 + cg * 8 + 4) = make_float4(tot[4], tot[5], tot[6], tot[7]);
        } else {
            const int u = tid - 128, tg = u >> 4, cg = u & 15;
            for (int i = 0; i < 8; ++i) {
                const int r = tg * 8 + i;
                float mv[8], vv[8];
                unpack8(raw_row(sm, RAW_V, r, cg), vv);
                if (r < nvalid) {
                    if (gdn2) {
                        float wv[8];
                        unpack8(*reinterpret_cast<const uint4 *>(g2p + ((rowbase + r) * H + h) * D + cg * 8), wv);
#pragma unroll
                        for (int c = 0; c < 8; ++c) mv[c] = wv[c] * vv[c];
                    } else {
                        const float g = s_g2[r];
#pragma unroll
                        for (int c = 0; c < 8; ++c) mv[c] = g * vv[c];
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c) mv[c] = 0.f;
                }
                *reinterpret_cast<uint4 *>(sm + OFF_MT + sw_chunk(64, r, cg)) = pack8(mv);
            }
            // P_{r,r} = q_r . k_r : two threads per row
            const int r = u >> 1, hf = u & 1;
            float acc = 0.f;
            for (int cc = 0; cc < 8; ++cc) {
                float qv[8], kv[8];
                unpack8(raw_row(sm, RAW_Q, r, hf * 8 + cc), qv);
                unpack8(raw_row(sm, RAW_K, r, hf * 8 + cc), kv);
#pragma unroll
                for (int c = 0; c < 8; ++c) acc = fmaf(qv[c], kv[c], acc);
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            if (hf == 0) s_pdiag[r] = (r < nvalid) ? acc : 0.f;
        }
        __syncthreads();

        // ===== 1b. Gamma (.) q, Gamma (.) a~, Kbar, Gamma_C ==================
        if (tid < 128) {
            const int tg = tid >> 4, cg = tid & 15;
            float pre[8], suf[8], run[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) { pre[c] = 1.f; suf[c] = 1.f; run[c] = 1.f; }
            for (int g = 0; g < 8; ++g) {
                float t8[8];
                *reinterpret_cast<float4 *>(t8) = *reinterpret_cast<const float4 *>(s_tot + g * 128 + cg * 8);
                *reinterpret_cast<float4 *>(t8 + 4) = *reinterpret_cast<const float4 *>(s_tot + g * 128 + cg * 8 + 4);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    if (g < tg) pre[c] *= t8[c];
                    if (g > tg) suf[c] *= t8[c];
                }
            }
            for (int i = 0; i < 8; ++i) {
                const int r = tg * 8 + i;
                const bool v = r < nvalid;
                float al[8], qv[8], kv[8], gq[8], ga[8];
                unpack8(raw_row(sm, RAW_A, r, cg), al);
                unpack8(raw_row(sm, RAW_Q, r, cg), qv);
                unpack8(raw_row(sm, RAW_K, r, cg), kv);
                float e[8];
                if (gdn2) {
                    if (v) unpack8(*reinterpret_cast<const uint4 *>(g1p + ((rowbase + r) * H + h) * D + cg * 8), e);
                    else {
#pragma unroll
                        for (int c = 0; c < 8; ++c) e[c] = 0.f;
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c) e[c] = s_g1[r];
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float alc = v ? al[c] : 1.f;
                    run[c] *= alc;
                    const float gam = pre[c] * run[c];
                    gq[c] = v ? gam * qv[c] : 0.f;
                    ga[c] = v ? gam * (e[c] * kv[c]) : 0.f;
                }
                *reinterpret_cast<uint4 *>(sm + OFF_QG + sw_chunk(64, r, cg)) = pack8(gq);
                *reinterpret_cast<uint4 *>(sm + OFF_AG + sw_chunk(64, r, cg)) = pack8(ga);
            }
            // exclusive suffix inside the block, times the later blocks' totals
            float sx[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) sx[c] = 1.f;
            for (int i = 7; i >= 0; --i) {
                const int r = tg * 8 + i;
                const bool v = r < nvalid;
                float al[8], kv[8], kb[8];
                unpack8(raw_row(sm, RAW_A, r, cg), al);
                unpack8(raw_row(sm, RAW_K, r, cg), kv);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    kb[c] = v ? suf[c] * sx[c] * kv[c] : 0.f;
                    sx[c] *= v ? al[c] : 1.f;
                }
                *reinterpret_cast<uint4 *>(sm + OFF_KB + sw_chunk(64, r, cg)) = pack8(kb);
            }
            if (tg == 0) {
                // Gamma_C = product of all block totals = own block total (sx) x later blocks (suf)
#pragma unroll
                for (int c = 0; c < 8; ++c) s_gamC[cg * 8 + c] = sx[c] * suf[c];
            }
        }

        // ===== 2. A and P by anchored levels on the tensor core ===============
        for (int p = 0; p < 3; ++p) {
            // threads 0..127 build level 2p+1, threads 128..255 level 2p+2
            {
                const int lvl = 2 * p + 1 + (tid >> 7);
                const int hh = 32 >> (lvl - 1);
                const int slot = tid >> 7;                 // 0: first level of the pair, 1: second
                const int u = tid & 127, tg = u >> 4, cg = u & 15;
                // carries over whole 8-token blocks (levels 1-3 only)
                float cpre[8], csuf[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) { cpre[c] = 1.f; csuf[c] = 1.f; }
                if (hh >= 8) {
                    const int r0 = tg * 8, pos0 = r0 % (2 * hh);
                    const int gs = (r0 - pos0 + hh) >> 3;       // first block of the second half
                    const int ge = (r0 - pos0 + hh - 1) >> 3;   // last block of the first half
                    for (int g = 0; g < 8; ++g) {
                        const bool in_pre = pos0 >= hh && g >= gs && g < tg;
                        const bool in_suf = pos0 < hh && g > tg && g <= ge;
                        if (in_pre || in_suf) {
                            float t8[8];
                            *reinterpret_cast<float4 *>(t8) = *reinterpret_cast<const float4 *>(s_tot + g * 128 + cg * 8);
                            *reinterpret_cast<float4 *>(t8 + 4) =
                                *reinterpret_cast<const float4 *>(s_tot + g * 128 + cg * 8 + 4);
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                if (in_pre) cpre[c] *= t8[c];
                                if (in_suf) csuf[c] *= t8[c];
                            }
                        }
                    }
                }
                // forward: second-half rows, prefix from the half start
                float run[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) run[c] = cpre[c];
                for (int i = 0; i < 8; ++i) {
                    const int r = tg * 8 + i, pos = r % (2 * hh);
                    if (pos == hh && hh < 8) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) run[c] = 1.f;
                    }
                    if (pos < hh) continue;
                    const bool v = r < nvalid;
                    float al[8], qv[8], kv[8], fa[8], fp[8], e[8];
                    unpack8(raw_row(sm, RAW_A, r, cg), al);
                    unpack8(raw_row(sm, RAW_Q, r, cg), qv);
                    unpack8(raw_row(sm, RAW_K, r, cg), kv);
                    if (gdn2) {
                        if (v) unpack8(*reinterpret_cast<const uint4 *>(g1p + ((rowbase + r) * H + h) * D + cg * 8), e);
                        else {
#pragma unroll
                            for (int c = 0; c < 8; ++c) e[c] = 0.f;
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 8; ++c) e[c] = s_g1[r];
                    }
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        run[c] *= v ? al[c] : 1.f;
                        fa[c] = v ? run[c] * e[c] * kv[c] : 0.f;
                        fp[c] = v ? run[c] * qv[c] : 0.f;
                    }
                    const int idx = (r / (2 * hh)) * hh + (pos - hh);
                    *reinterpret_cast<uint4 *>(sm + OFF_FA + sw_chunk(128, slot * 32 + idx, cg)) = pack8(fa);
                    *reinterpret_cast<uint4 *>(sm + OFF_FA + sw_chunk(128, 64 + slot * 32 + idx, cg)) = pack8(fp);
                }
                // backward: first-half columns, exclusive suffix to the half end
                float sx[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) sx[c] = csuf[c];
                for (int i = 7; i >= 0; --i) {
                    const int r = tg * 8 + i, pos = r % (2 * hh);
                    if (pos == 2 * hh - 1 && hh < 8) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) sx[c] = 1.f;
                    }
                    if (pos >= hh) continue;
                    if (pos == hh - 1 && hh < 8) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) sx[c] = 1.f;
                    }
                    const bool v = r < nvalid;
                    float al[8], kv[8], fc[8];
                    unpack8(raw_row(sm, RAW_A, r, cg), al);
                    unpack8(raw_row(sm, RAW_K, r, cg), kv);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        fc[c] = v ? sx[c] * kv[c] : 0.f;
                        sx[c] *= v ? al[c] : 1.f;
                    }
                    const int idx = (r / (2 * hh)) * hh + pos;
                    *reinterpret_cast<uint4 *>(sm + OFF_FB + sw_chunk(64, slot * 32 + idx, cg)) = pack8(fc);
                }
            }
            publish();
            if (tid == 0) {
                tc_fence_after();
                const uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tbase + tm_ap(p), dK(sb + OFF_FA, 128, kk), dK(sb + OFF_FB, 64, kk), idesc, kk > 0);
                mma_commit(bar_mma);
            }
            wait_mma();
        }
        // raw tiles consumed: prefetch the next chunk
        __syncthreads();
        if (tid == 0 && ch + 1 < nchunks) issue_tma(ch + 1);

        // ===== 2b. read A, P out of TMEM ======================================
        for (int e = tid; e < 64 * 65; e += NT) { Af[e] = 0.f; Tf[e] = 0.f; }
        for (int e = tid; e < 512; e += NT) *reinterpret_cast<uint4 *>(sm + OFF_PBF + e * 16) = make_uint4(0, 0, 0, 0);
        __syncthreads();
        for (int p = (warp >> 2); p < 3; p += 2) {
            const int lvl = 2 * p + 1 + (quarter & 1);
            const int hh = 32 >> (lvl - 1);
            const bool isP = quarter >= 2;
            float v[32];
            tmem_ld32(tbase + lane_base + tm_ap(p) + (quarter & 1) * 32, v);
            tmem_wait_ld();
            const int r = (lane / hh) * 2 * hh + hh + (lane % hh);
            const int c0 = (r / (2 * hh)) * hh;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                if (c >= c0 && c < c0 + hh) {
                    const int s = (c / hh) * 2 * hh + (c % hh);
                    if (!isP) Af[r * 65 + s] = v[c];
                    else *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_PBF + sw_elem(64, r, s)) = __float2bfloat16_rn(v[c]);
                }
            }
        }
        if (tid < C) *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_PBF + sw_elem(64, tid, tid)) =
            __float2bfloat16_rn(s_pdiag[tid]);
        tc_fence_before();
        __syncthreads();

        // ===== 3. T = (I + A)^{-1}: 16x16 diagonal blocks, then block rows ====
        if (tid < 64) {
            const int I = tid >> 4, c = tid & 15;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                if (rr < c) x[rr] = 0.f;
                else if (rr == c) x[rr] = 1.f;
                else {
                    float acc = 0.f;
#pragma unroll
                    for (int ss = 0; ss < rr; ++ss) acc = fmaf(Af[(16 * I + rr) * 65 + 16 * I + ss], x[ss], acc);
                    x[rr] = -acc;
                }
            }
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) Tf[(16 * I + rr) * 65 + 16 * I + c] = x[rr];
        }
        __syncthreads();
        for (int d = 1; d < 4; ++d) {
            const int nel = (4 - d) * 256;
            for (int e = tid; e < nel; e += NT) {
                const int J = e >> 8, I = J + d, rr = (e >> 4) & 15, cc = e & 15;
                float acc = 0.f;
                for (int uu = 16 * J; uu < 16 * I; ++uu)
                    acc = fmaf(Af[(16 * I + rr) * 65 + uu], Tf[uu * 65 + 16 * J + cc], acc);
                Xs[e] = acc;
            }
            __syncthreads();
            for (int e = tid; e < nel; e += NT) {
                const int J = e >> 8, I = J + d, rr = (e >> 4) & 15, cc = e & 15;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    acc = fmaf(Tf[(16 * I + rr) * 65 + 16 * I + m], Xs[(J << 8) + m * 16 + cc], acc);
                Tf[(16 * I + rr) * 65 + 16 * J + cc] = -acc;
            }
            __syncthreads();
        }
        {
            const int r = tid >> 2, kc0 = (tid & 3) * 2;
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                float t8[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) t8[c] = Tf[r * 65 + (kc0 + q2) * 8 + c];
                *reinterpret_cast<uint4 *>(sm + OFF_TBF + sw_chunk(64, r, kc0 + q2)) = pack8(t8);
            }
        }
        publish();

        // ===== 4. W = T (Gamma (.) A~)  and  U^T = M^T T^T ====================
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_w = idesc_bf16(64, 128, false, true);
            const uint32_t id_u = idesc_bf16(128, 64, true, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16(tbase + TM_W, dK(sb + OFF_TBF, 64, kk), dMN(sb + OFF_AG, kk), id_w, kk > 0);
                mma_bf16(tbase + TM_U, dMN(sb + OFF_MT, kk), dK(sb + OFF_TBF, 64, kk), id_u, kk > 0);
            }
            mma_commit(bar_mma);
        }
        wait_mma();
        // W (M = 64 layout: rows 16q..16q+15 in lanes 0..15 of quarter q) -> [token][channel] tile
        {
            const int r = quarter * 16 + (lane & 15);
            const int chalf = warp >> 2;
#pragma unroll
            for (int c32 = 0; c32 < 2; ++c32) {
                float v[32];
                tmem_ld32(tbase + lane_base + TM_W + chalf * 64 + c32 * 32, v);
                tmem_wait_ld();
                if (lane < 16) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int kc = chalf * 8 + c32 * 4 + q4;
                        *reinterpret_cast<uint4 *>(sm + OFF_AG + sw_chunk(64, r, kc)) = pack8(v + q4 * 8);
                    }
                }
            }
        }
        publish();

        // ===== 5. U^T -= S0^T W^T ;  O^T = S0^T (Gamma (.) Q)^T ==============
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_neg = idesc_bf16(128, 64, false, false, true);
            const uint32_t id_pos = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                mma_bf16(tbase + TM_U, dK(sb + OFF_S0T, 128, kk), dK(sb + OFF_AG, 64, kk), id_neg, 1);
                mma_bf16(tbase + TM_O, dK(sb + OFF_S0T, 128, kk), dK(sb + OFF_QG, 64, kk), id_pos, kk > 0);
            }
            mma_commit(bar_mma);
        }
        wait_mma();
        {
            const int j = quarter * 32 + lane, shalf = warp >> 2;
            // U^T row j, tokens [32*shalf, +32) -> bf16 K-major tile (rows j, K = token)
            float v[32];
            tmem_ld32(tbase + lane_base + TM_U + shalf * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4 *>(sm + OFF_MT + sw_chunk(128, j, shalf * 4 + q4)) = pack8(v + q4 * 8);
            // S^T row j, key channels [64*shalf, +64): scale by Gamma_C
#pragma unroll
            for (int c32 = 0; c32 < 2; ++c32) {
                const int i0 = shalf * 64 + c32 * 32;
                float s[32];
                tmem_ld32(tbase + lane_base + TM_S + i0, s);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) s[e] *= s_gamC[i0 + e];
                tmem_st16(tbase + lane_base + TM_S + i0, s);
                tmem_st16(tbase + lane_base + TM_S + i0 + 16, s + 16);
            }
            tmem_wait_st();
        }
        publish();

        // ===== 6. O^T += U^T P^T ;  S^T += U^T Kbar ==========================
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_o = idesc_bf16(128, 64, false, false);
            const uint32_t id_s = idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16(tbase + TM_O, dK(sb + OFF_MT, 128, kk), dK(sb + OFF_PBF, 64, kk), id_o, 1);
                mma_bf16(tbase + TM_S, dK(sb + OFF_MT, 128, kk), dMN(sb + OFF_KB, kk), id_s, 1);
            }
            mma_commit(bar_mma);
        }
        wait_mma();
        {
            const int j = quarter * 32 + lane, shalf = warp >> 2;
            float v[32];
            tmem_ld32(tbase + lane_base + TM_O + shalf * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int r = shalf * 32 + e;
                if (r < nvalid) op[((rowbase + r) * H + h) * D + j] = __float2bfloat16_rn(v[e]);
            }
#pragma unroll
            for (int c32 = 0; c32 < 2; ++c32) {
                const int i0 = shalf * 64 + c32 * 32;
                float s[32];
                tmem_ld32(tbase + lane_base + TM_S + i0, s);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    *reinterpret_cast<uint4 *>(sm + OFF_S0T + sw_chunk(128, j, (i0 >> 3) + q4)) = pack8(s + q4 * 8);
            }
        }
        fence_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;  // every thread leaves the loop together
    }

    // ---- final state (or NaN if an internal wait timed out) ----------------
    tc_fence_after();
    if (a.sf) {
        const size_t soff = ((size_t)n * H + h) * D * D;
        const int j = quarter * 32 + lane, shalf = warp >> 2;
#pragma unroll
        for (int c32 = 0; c32 < 2; ++c32) {
            const int i0 = shalf * 64 + c32 * 32;
            float s[32];
            tmem_ld32(tbase + lane_base + TM_S + i0, s);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) a.sf[soff + (size_t)(i0 + e) * D + j] = ok ? s[e] : __int_as_float(0x7fc00000);
        }
    }
    if (!ok) {
        // drain any TMA still in flight (bounded) before the CTA's shared memory is released
        mbar_wait_cycles(bar_tma, ph_tma, WAIT_CYCLES);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

// ---- host side --------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map(CUtensorMap *m, const void *base, long long rows, int H)
{
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {128, 1, 64}, es[3] = {1, 1, 1};
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunk_fwd_sm100(const FwdArgs &a, cudaStream_t st)
{
    // the dynamic shared-memory opt-in is per device; set it once per device
    static std::mutex mu;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        if (!attr_done[dev]) {
            e = cudaFuncSetAttribute(chunk_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
            if (e != cudaSuccess) return e;
            attr_done[dev] = true;
        }
    }
    ChunkParams p;
    memset(&p, 0, sizeof(p));
    p.a = a;
    const long long rows = (long long)a.B * a.T;
    if (rows > 0) {
        if (!make_map(&p.tq, a.q, rows, a.H) || !make_map(&p.tk, a.k, rows, a.H) ||
            !make_map(&p.tv, a.v, rows, a.H) || !make_map(&p.ta, a.alpha, rows, a.H))
            return cudaErrorInvalidValue;
    }
    const int N = a.cu_seqlens ? a.num_seqs : a.B;
    chunk_fwd_kernel<<<(unsigned)(N * a.H), NT, SMEM_ALLOC, st>>>(p);
    return cudaGetLastError();
}

}  // namespace kda
