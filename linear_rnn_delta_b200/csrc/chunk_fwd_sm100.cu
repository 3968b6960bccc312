// Chunked-parallel forward of the gated delta-rule recurrence on sm_100a
// tensor cores (bf16 inputs, d_k = d_v = 128, chunk C = 64).
//
// Recurrence (update equations on the Raon-1-mini-preview discussion page):
//   S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T,   u_t = m_t - (Diag(alpha_t) S_{t-1})^T a~_t,
//   o_t = S_t^T q_t,
// with (a~, m) = (beta k, beta v) for KDA / Complex KDA, (e k, w v) for RDA and
// (b (.) k, w (.) v) for GDN-2.  Unrolled over a chunk of C tokens that starts
// from state S0 (positions r, s in 0..C-1; every product taken forward):
//   Gamma_r   = prod_{t<=r} alpha_t                 (per key channel)
//   Lam_{r,s} = prod_{s<t<=r} alpha_t
//   A_{r,s}   = sum_c a~_{r,c} Lam_{r,s,c} k_{s,c}   (s < r)
//   P_{r,s}   = sum_c q_{r,c}  Lam_{r,s,c} k_{s,c}   (s <= r)
//   T         = (I + A)^{-1}                        (UT transform)
//   W         = T (Gamma (.) A~),   U = T M - W S0  (WY form)
//   O         = (Gamma (.) Q) S0 + P U
//   S_C       = Diag(Gamma_C) S0 + Kbar^T U,   Kbar_s = Lam_{C-1,s} (.) k_s
//
// Sign-safe decay.  Complex-KDA gates lie in [-1,1], so cumulative products can
// be negative, zero or vanishingly small; no logarithm of alpha is ever taken.
// A and P are formed one of two ways, decided per chunk for the whole CTA:
//  * fast path, when every |alpha| <= 1 and every channel's chunk product
//    satisfies |Gamma_C| >= 2^-110: Lam_{r,s} = (Gamma_r / Gamma_C) Lam_{C-1,s},
//    so [A; P] is ONE tensor-core GEMM of the row operand
//    [Gamma (.) A~ / Gamma_C ; Gamma (.) Q / Gamma_C] with Kbar (K = d_k).  The
//    only division is by Gamma_C, which is bounded away from zero.  The state
//    operand is then the scaled state Diag(Gamma_C) S0, which makes
//    W S0 = (W / Gamma_C)(Gamma_C S0) and (Gamma Q) S0 = (Gamma Q / Gamma_C)(Gamma_C S0).
//  * anchored path otherwise (zero or tiny gates): at level L = 1..6 the chunk
//    is cut into blocks of 2h tokens (h = 32 >> (L-1)); for r in a block's
//    second half and s in its first half, with a = last token of the first half,
//      Lam_{r,s} = (prod_{a<t<=r} alpha_t) (.) (prod_{s<t<=a} alpha_t),
//    a product of forward "row" and "column" factors, so each level's pairs are
//    one dense GEMM.  Six levels cover every pair s < r once; P_{r,r} = q_r . k_r.
//    Nothing is divided, so zeros and signs propagate exactly.
//
// Fused form: one CTA of 384 threads per (sequence, head); the fp32 state
// lives in tensor memory (TMEM) for the whole sequence, transposed (lane =
// value column j, column = key channel i), so every state-dependent GEMM has
// M = d_v = 128.  q, k, v, alpha arrive by TMA; every other operand is built
// on chip in 128-byte swizzled shared-memory tiles.  Per chunk:
//   1. TMA raw tiles -> block totals, Gamma_C, M, Kbar, row operands
//   2. A, P  (one GEMM on the fast path, three on the anchored path)
//   3. T = (I + A)^{-1}: 16x16 diagonal blocks, then two recursive-doubling merges
//   4. tcgen05: W = T (row operand a~ part);  U^T = M^T T^T
//   5. state pass: S^T *= Gamma_C in TMEM and its bf16 copy (scaled or not)
//   6. tcgen05: U^T -= S^T W^T;  O^T = S^T Q^T  (one N = 128 GEMM over [-W; Q'])
//   7. tcgen05: O^T += U^T P^T;  S^T += U^T Kbar;  o -> HBM
// The next chunk's TMA loads start as soon as step 2 has consumed the raw tiles.
// Optional input preparation (gate logits, raw keys) rewrites the raw tiles in
// place before step 1 (a compile-time variant, PREP).
//
// Split form: steps 1-4 do not depend on the state, so a persistent kernel
// (chunk_prep_kernel, which pipelines two items per SM) runs them for every
// (chunk, head) on all SMs and stores each chunk's operand tiles to a
// workspace slot; a chain kernel per (sequence, head) then runs steps 5-7 from
// those slots.  Same arithmetic on every element: the two forms give identical
// bits.
#include <cuda.h>
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {
using namespace sm100;

constexpr int C = 64;    // chunk length
constexpr int D = 128;   // d_k = d_v
constexpr int NT = 384;  // threads per CTA: 4 chain warps + 8 prep warps

// ---- shared memory map (offsets from a 1024-byte aligned base) ------------
constexpr uint32_t RAW_Q = 0, RAW_K = 16384, RAW_A = 49152;  // TMA tiles [64][128] bf16, row-major
constexpr uint32_t OFF_UT = 32768;   // U^T bf16 128 x 64 (chain steps 6-7), then o staging [64][128]
constexpr uint32_t OFF_S0T = 65536;   // state operand bf16, 128 x 128, K-major (rows j, K = i)
constexpr uint32_t OFF_QA = 98304;    // 128-row tile: rows 0-63 a~ operand (later W), rows 64-127 q operand
constexpr uint32_t OFF_KB = 131072;   // Kbar [token][channel]
constexpr uint32_t OFF_MT = 147456;   // M [token][channel]: v by 128B-swizzled TMA (GDN-2: scaled by w in place)
constexpr uint32_t OFF_F = 163840;    // anchored-path level factors | A, T fp32, T, P bf16 | o staging
constexpr uint32_t OFF_LA = OFF_F;            // level row factors: 128 rows x 128 ch
constexpr uint32_t OFF_LB = OFF_F + 32768;    // level column factors: 64 rows x 128 ch
constexpr int TP = 68;                        // pitch (floats) of the fp32 A and T tiles: 16-byte rows
constexpr uint32_t OFF_AF32 = OFF_F;          // A fp32 [64][TP]
constexpr uint32_t OFF_TF32 = OFF_F + 17408;  // T fp32 [64][TP]
constexpr uint32_t OFF_X = OFF_F + 34816;     // 32 x 32 fp32 scratch of the block solve
constexpr uint32_t OFF_TBF = OFF_F + 38912;   // T Diag(e) / T Diag(w) bf16 64 x 64 K-major
constexpr uint32_t OFF_PBF = OFF_F + 47104;   // P bf16 64 x 64 K-major
constexpr uint32_t OFF_MISC = OFF_F + 55296;
constexpr int PBAND = 5;   // P_{r,s} for r-4 <= s <= r computed exactly (SIMT) from the bf16 inputs
constexpr uint32_t M_G1 = OFF_MISC, M_G2 = OFF_MISC + 256, M_GAMC = OFF_MISC + 512, M_TOT = OFF_MISC + 1536,
                   M_PBAND = OFF_MISC + 5632, M_FAST = OFF_MISC + 6912, M_BAR = OFF_MISC + 6920,
                   M_TMEM = OFF_MISC + 6976;
constexpr uint32_t M_G1B = OFF_MISC + 6992, M_G2B = OFF_MISC + 7248;   // gates of the other item parity
constexpr uint32_t SMEM_USED = OFF_MISC + 7504;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;  // slack for aligning the base
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert((OFF_TBF & 1023) == 0 && (OFF_PBF & 1023) == 0 && (OFF_QA & 1023) == 0, "swizzle atoms");

// ---- TMEM columns ---------------------------------------------------------
constexpr uint32_t TM_S = 0, TM_U = 128, TM_O = 192, TM_W = 256, TM_AP = 384;
__device__ __forceinline__ uint32_t tm_lvl(int p) { return p == 0 ? 384u : (p == 1 ? 448u : 256u); }

constexpr long long WAIT_CYCLES = 4000000000ll;  // ~2 s: only a broken pipeline gets near it
constexpr float FAST_MIN_GAMMA = 7.703719777548943e-34f;  // 2^-110

struct ChunkParams {
    CUtensorMap tq, tk, ta;  // [B*T][H][128] bf16, box {128, 1, 64}, no swizzle
    CUtensorMap tv;          // same tensor shape, box {64, 1, 64}, 128-byte swizzle
    FwdArgs a;
    uint8_t *ws;             // split path: chunk operand slots
    int nslots;              // slots per head
    uint32_t epoch;          // split path: tag of this call's slots
    int debug_stall;         // split path, testing aid: stall the chain CTA of (sequence 0, head 0)
};

// ---- split path: per-chunk operand slots in global memory -------------------
// Chunk c of sequence n (first global row R_n) has slot s = n + floor(R_n / C) + c:
// unique, increasing within a sequence, and below N + ceil(rows / C).
// A slot (one per head) holds byte images of the shared-memory operand tiles,
// laid out so the chain kernel loads one contiguous block:
constexpr uint32_t SL_QA = 0;         // [-W'; Q'] 128-row K-major tile (32 KiB)
constexpr uint32_t SL_KB = 32768;     // Kbar (16 KiB)
constexpr uint32_t SL_PBF = 49152;    // P bf16 (8 KiB)
constexpr uint32_t SL_TBF = 57344;    // T Diag(w) bf16 (8 KiB)
constexpr uint32_t SL_META = 65536;   // Gamma_C fp32 [128], status word, epoch tag
constexpr uint32_t SL_META_BYTES = 528;
constexpr uint32_t SL_OPS = 66560;    // bytes the chain kernel loads for every variant
constexpr uint32_t SL_M = 66560;      // GDN-2: M = w (.) v, 128B-swizzled [token][channel] (16 KiB)
constexpr uint32_t SLOT_BYTES = 82944;
constexpr int META_FAST = 1;          // status word bits
constexpr int META_OK = 2;
constexpr int META_EXACT = 4;         // ill-conditioned chunk: the chain runs it token by token

// A chunk is run token by token in fp32 (the exact path below) when the bf16
// WY form would lose too much to cancellation.  Two signs of it, both from
// matrices the preparation has in fp32 anyway:
//  * the UT transform is large: the largest row sum of |T_{r,s}| max(|e_s|,
//    |w_s|) exceeds EXACT_T_NORM.  Runs of strong, barely decaying
//    reflections on correlated keys (erase gates near 2) do this; their exact
//    result is close to an orthogonal map (the 2D rotation of the Complex KDA
//    abstract), and the rounding of T, W and U reaches the state through
//    K^T T (.) with no decay to damp it.
//  * the tokens of the chunk interact strongly: the largest row sum of |A|
//    (A_{r,s} = e_r sum_c k_{r,c} Lam_{r,s,c} k_{s,c}) exceeds EXACT_A_NORM.
//    Aligned keys with little decay (erase gates near 1) make each token
//    overwrite what the previous ones wrote; the readout and the state update
//    then sum many nearly cancelling terms, and every bf16 rounding point
//    (operands, P, U) shows in the result.
// Random chunks of the benchmark recipes stay below 3.1 and 0.9; in emulation
// of the kernel's rounding, adversarial chunks under both bounds stay within
// the bf16 tolerance (worst 0.014 of the 0.02 bound).
constexpr float EXACT_T_NORM = 6.f;
constexpr float EXACT_A_NORM = 3.f;

// Device-side failure word of this library on each device: bits are OR-ed in
// by any CTA whose bounded wait ran out or whose input slot was not prepared,
// and read (and cleared) by kda_device_status.
__device__ unsigned int g_device_status;
constexpr unsigned DEV_WAIT_TIMEOUT = 1u, DEV_SLOT_MISSING = 2u;
__device__ __forceinline__ void report_device_failure(unsigned bits) { atomicOr(&g_device_status, bits); }

// Test-only stall (KDA_FLAG_DEBUG_STALL): the chain CTA of (sequence 0, head 0)
// does not load its first slot and gives up waiting for it after this many
// cycles (~1 ms), so that the bounded-wait expiry path runs on demand.
constexpr long long STALL_WAIT_CYCLES = 1ll << 21;


// One chunk of work for the preparation role.
struct Item {
    int n, h, c, row0, len;   // sequence, head, chunk, first global row of the sequence, its length
    int slot;
    bool valid;
};
// ---- small helpers --------------------------------------------------------
// Elementwise work is done in "items" of 8 tokens x 4 channels (one 8-byte
// half of a 16-byte chunk per row): 256 items cover a 64 x 128 tile.
__device__ __forceinline__ void unpack4(const uint2 &u, float *f)
{
    f[0] = __uint_as_float(u.x << 16);
    f[1] = __uint_as_float(u.x & 0xFFFF0000u);
    f[2] = __uint_as_float(u.y << 16);
    f[3] = __uint_as_float(u.y & 0xFFFF0000u);
}
__device__ __forceinline__ uint2 pack4(const float *f)
{
    return make_uint2(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]));
}
__device__ __forceinline__ void unpack8(const uint4 &u, float *f)
{
    unpack4(make_uint2(u.x, u.y), f);
    unpack4(make_uint2(u.z, u.w), f + 4);
}
__device__ __forceinline__ uint4 pack8(const float *f)
{
    return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
}
__device__ __forceinline__ uint4 pack8_neg(const float *f)   // -f, exact
{
    return make_uint4(pack_bf16(-f[0], -f[1]), pack_bf16(-f[2], -f[3]), pack_bf16(-f[4], -f[5]),
                      pack_bf16(-f[6], -f[7]));
}
// 16-byte chunk kc (8 consecutive K elements) of row `row` in a K-major
// 128B-swizzled tile whose 64-element panels are `pstride` bytes apart.
__device__ __forceinline__ uint32_t sw_chunk(uint32_t pstride, uint32_t row, uint32_t kc)
{
    return (kc >> 3) * pstride + row * 128u + ((((kc & 7u) ^ (row & 7u))) << 4);
}
// 8-byte half-chunk of channel quad cq (channels 4cq .. 4cq+3)
__device__ __forceinline__ uint32_t sw_half(uint32_t pstride, uint32_t row, uint32_t cq)
{
    return sw_chunk(pstride, row, cq >> 1) + (cq & 1u) * 8u;
}
__device__ __forceinline__ uint32_t sw_elem(uint32_t pstride, uint32_t row, uint32_t k)
{
    return sw_chunk(pstride, row, k >> 3) + (k & 7u) * 2u;
}
// raw TMA tile: row-major [64][128] bf16
__device__ __forceinline__ uint4 raw_row(const uint8_t *sm, uint32_t base, int r, int cg)
{
    return *reinterpret_cast<const uint4 *>(sm + base + r * 256 + cg * 16);
}
__device__ __forceinline__ uint2 raw_quad(const uint8_t *sm, uint32_t base, int r, int cq)
{
    return *reinterpret_cast<const uint2 *>(sm + base + r * 256 + cq * 8);
}
// K-major descriptor, K step kk (16 elements), panels `pstride` bytes apart.
// The step only moves the start address (bits 0-13, in 16-byte units; shared
// addresses stay below 2^18 bytes, so the field cannot overflow): the base
// descriptor is computed once and each step adds a constant.
__device__ __forceinline__ uint64_t dK(uint32_t base, uint32_t pstride, int kk)
{
    return make_desc_sw128(base, 16) + (uint64_t)(((uint32_t)(kk >> 2) * pstride + (uint32_t)(kk & 3) * 32u) >> 4);
}
// MN-major descriptor of a [token][channel] tile (channels in two 64-wide
// panels `pstride` bytes apart, K = tokens), K step kk (16 tokens)
__device__ __forceinline__ uint64_t dMN(uint32_t base, uint32_t pstride, int kk)
{
    return make_desc_sw128(base, pstride) + (uint64_t)((uint32_t)kk * (2048u >> 4));
}
__device__ __forceinline__ void load_tot4(const float *s_tot, int g, int cq, float *t4)
{
    *reinterpret_cast<float4 *>(t4) = *reinterpret_cast<const float4 *>(s_tot + g * 128 + cq * 4);
}

struct ChunkCtx {
    uint8_t *sm;
    const float *s_tot, *s_g1;
    const __nv_bfloat16 *g1p;
    size_t rowbase;
    int H, h, nvalid;
    bool gdn2;
    bool logits, ext;   // input preparation: GDN-2's erase vector arrives as logits; extended range
    uint32_t qa, kb, la, lb;   // shared-memory offsets of the row-operand tile, Kbar and the level factors
};

// Channel-wise part of the erase direction of row r for 4 channels (GDN-2:
// the vector b; 1 otherwise, because the scalar erase gate is folded into the
// rows of A and the columns of T instead of into the bf16 operands).
__device__ __forceinline__ void erase_gate4(const ChunkCtx &x, int r, int cq, float *e)
{
    if (x.gdn2 && r < x.nvalid) {
        unpack4(*reinterpret_cast<const uint2 *>(x.g1p + ((x.rowbase + r) * x.H + x.h) * D + cq * 4), e);
        if (x.logits) {
#pragma unroll
            for (int c = 0; c < 4; ++c) e[c] = round_bf16(prep_gate(e[c], x.ext));
        }
    } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) e[c] = 1.f;
    }
}

// Step 6 of the chain: U^T += S^T (-W)^T and O^T = S^T Q^T.  The operand tile
// qa holds [-W; Q'] as 128 K-major rows and U^T, O^T are adjacent in TMEM, so
// after the first K step (U^T accumulates onto U'^T, O^T starts fresh) both
// run as one N = 128 GEMM.
__device__ __forceinline__ void step6_mmas(uint32_t tbase, uint32_t s0t, uint32_t qa)
{
    const uint32_t id64 = idesc_bf16(128, 64, false, false), id128 = idesc_bf16(128, 128, false, false);
    mma_bf16(tbase + TM_U, dK(s0t, 16384, 0), dK(qa, 16384, 0), id64, 1);
    mma_bf16(tbase + TM_O, dK(s0t, 16384, 0), dK(qa + 8192, 16384, 0), id64, 0);
#pragma unroll
    for (int kk = 1; kk < 8; ++kk) mma_bf16(tbase + TM_U, dK(s0t, 16384, kk), dK(qa, 16384, kk), id128, 1);
}

// State snapshot after a chunk: S^T (TMEM lane j = value column j, fp32) ->
// snap[slot][h][i][j] for the key channels of 32-column blocks c32 in
// [c32a, c32a + n32); for a fixed i a warp writes 128 contiguous bytes.
__device__ __forceinline__ void snapshot_state(const FwdArgs &a, uint32_t tlane, int slot, int h, int c32a, int n32,
                                               int jcol)
{
    float *dst = a.snap + ((size_t)slot * a.H + h) * D * D + jcol;
#pragma unroll 1
    for (int c32 = c32a; c32 < c32a + n32; ++c32) {
        float s[32];
        tmem_ld32(tlane + TM_S + c32 * 32, s);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) dst[(size_t)(c32 * 32 + e) * D] = s[e];
    }
}

// Fast path, step 1b for the item (tg, cq): one forward sweep over the item's
// 8 rows.  With sc = Gamma_r / Gamma_C (|sc| >= 1 since every |alpha| <= 1):
//   row operands  Gamma a~ / Gamma_C = sc (.) a~,   Gamma q / Gamma_C = sc (.) q,
//   Kbar_r = Lam_{C-1,r} (.) k_r = k_r / sc   (the divisor is bounded away from zero).
// The band of P, P_{r,r-w} = sum_c (sc q)_{r,c} Kbar_{r-w,c} for w = 0..4, is
// formed from these fp32 values: a window keeps Kbar of the four previous
// rows, and each lane's 4-channel partial sums go to band_part[r][w][lane]
// (summed over the 32 lanes = 128 channels by band_reduce).
// FULL: all 64 rows valid (no masking).  EVEC: channel-wise erase vector
// (GDN-2).  UNROLL: rows per unrolled step (register budget permitting).
// BPRE: the erase vector of the thread's 8 rows was loaded by the caller (raw
// bf16 pairs in bpre; the loop is then unrolled fully) instead of row by row.
template <bool FULL, bool EVEC, int UNROLL, bool BPRE = false>
__device__ __forceinline__ void fast_rows(const ChunkCtx &x, const float *s_tot, const float *gamc,
                                          float *band_part, int tg, int cq, int lane, const uint2 *bpre = nullptr)
{
    static_assert(!BPRE || (EVEC && UNROLL == 8), "prefetched erase vectors: full unroll");
    uint8_t *sm = x.sm;
    const int nvalid = x.nvalid;
    float pre[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        if (g >= tg) break;
        float t4[4];
        load_tot4(s_tot, g, cq, t4);
#pragma unroll
        for (int c = 0; c < 4; ++c) pre[c] *= t4[c];
    }
    const float4 gc4 = *reinterpret_cast<const float4 *>(gamc + cq * 4);
    float sc[4] = {pre[0] / gc4.x, pre[1] / gc4.y, pre[2] / gc4.z, pre[3] / gc4.w};
    float kw[4][4];   // Kbar of rows r-4 .. r-1
    {
        float sb4[4] = {sc[0], sc[1], sc[2], sc[3]};   // Gamma_{8tg-1} / Gamma_C
#pragma unroll
        for (int j = 3; j >= 0; --j) {
            const int rp = tg * 8 - 4 + j;
            if (rp >= 0) {
                float kv[4], av[4];
                unpack4(raw_quad(sm, RAW_K, rp, cq), kv);
                unpack4(raw_quad(sm, RAW_A, rp, cq), av);
                const bool v = FULL || rp < nvalid;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    kw[j][c] = v ? __fdividef(kv[c], sb4[c]) : 0.f;
                    sb4[c] = v ? __fdividef(sb4[c], av[c]) : sb4[c];
                }
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) kw[j][c] = 0.f;
            }
        }
    }
    // channel pairs (0, 1) and (2, 3) on the packed fp32 pipe: the same product per channel
    float2 sc2[2] = {make_float2(sc[0], sc[1]), make_float2(sc[2], sc[3])};
    auto dot4 = [](const float (&u)[4], const float (&w)[4]) {   // (u0 w0 + u2 w2) + (u1 w1 + u3 w3)
        const float2 t = __ffma2_rn(make_float2(u[2], u[3]), make_float2(w[2], w[3]),
                                    __fmul2_rn(make_float2(u[0], u[1]), make_float2(w[0], w[1])));
        return t.x + t.y;
    };
#pragma unroll UNROLL
    for (int i = 0; i < 8; ++i) {
        const int r = tg * 8 + i;
        const bool v = FULL || r < nvalid;
        float al[4], kv[4], qv[4], oa[4], oq[4], kb[4];
        unpack4(raw_quad(sm, RAW_A, r, cq), al);
        unpack4(raw_quad(sm, RAW_K, r, cq), kv);
        unpack4(raw_quad(sm, RAW_Q, r, cq), qv);
        float e[4] = {1.f, 1.f, 1.f, 1.f};
        if (BPRE) {
            unpack4(bpre[i], e);
            if (x.logits) {
#pragma unroll
                for (int c = 0; c < 4; ++c) e[c] = round_bf16(prep_gate(e[c], x.ext));
            }
        } else if (EVEC) {
            erase_gate4(x, r, cq, e);
        }
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
            const int c = 2 * pp;
            sc2[pp] = __fmul2_rn(sc2[pp], v ? make_float2(al[c], al[c + 1]) : make_float2(1.f, 1.f));
            const float2 ek = EVEC ? __fmul2_rn(make_float2(e[c], e[c + 1]), make_float2(kv[c], kv[c + 1]))
                                   : make_float2(kv[c], kv[c + 1]);
            const float2 a2 = __fmul2_rn(sc2[pp], ek), q2 = __fmul2_rn(sc2[pp], make_float2(qv[c], qv[c + 1]));
            oa[c] = v ? a2.x : 0.f;
            oa[c + 1] = v ? a2.y : 0.f;
            oq[c] = v ? q2.x : 0.f;
            oq[c + 1] = v ? q2.y : 0.f;
            kb[c] = v ? __fdividef(kv[c], sc2[pp].x) : 0.f;
            kb[c + 1] = v ? __fdividef(kv[c + 1], sc2[pp].y) : 0.f;
        }
        *reinterpret_cast<uint2 *>(sm + x.qa + sw_half(16384, r, cq)) = pack4(oa);
        *reinterpret_cast<uint2 *>(sm + x.qa + sw_half(16384, 64 + r, cq)) = pack4(oq);
        *reinterpret_cast<uint2 *>(sm + x.kb + sw_half(8192, r, cq)) = pack4(kb);
        float *bp = band_part + r * (PBAND * 32) + lane;
        bp[0] = dot4(oq, kb);
#pragma unroll
        for (int w = 1; w < PBAND; ++w) bp[w * 32] = dot4(oq, kw[4 - w]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            kw[0][c] = kw[1][c]; kw[1][c] = kw[2][c]; kw[2][c] = kw[3][c]; kw[3][c] = kb[c];
        }
    }
}

// Fast path: P_{r,r-w} = sum over the 32 lanes of band_part[r][w][lane] for
// the 64 x PBAND band entries (masked past the valid rows and above row 0).
// Lanes start their eight 16-byte reads at rotated offsets: conflict-free.
__device__ __forceinline__ void band_reduce(const float *band_part, float *s_pband, int nvalid, int ptid, int nthreads)
{
    for (int idx = ptid; idx < C * PBAND; idx += nthreads) {
        const float4 *src = reinterpret_cast<const float4 *>(band_part + idx * 32);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 t = src[(j + idx) & 7];
            acc[j & 3] += (t.x + t.y) + (t.z + t.w);
        }
        const int r = idx / PBAND, w = idx - r * PBAND;
        s_pband[idx] = (r < nvalid && r - w >= 0) ? (acc[0] + acc[1]) + (acc[2] + acc[3]) : 0.f;
    }
}

// Anchored path: row and column factors of one level (block half HH) for the
// 8-token x 4-channel item (tg, cq), into level slot `slot` (0 or 1).
template <int HH>
__device__ __forceinline__ void build_level(const ChunkCtx &x, int slot, int tg, int cq)
{
    constexpr int BS = 2 * HH;
    uint8_t *sm = x.sm;
    float cpre[4], csuf[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) { cpre[c] = 1.f; csuf[c] = 1.f; }
    if (HH >= 8) {  // carries over whole 8-token blocks
        const int r0 = tg * 8, pos0 = r0 % BS;
        const int gs = (r0 - pos0 + HH) >> 3, ge = (r0 - pos0 + HH - 1) >> 3;
        for (int g = 0; g < 8; ++g) {
            const bool in_pre = pos0 >= HH && g >= gs && g < tg;
            const bool in_suf = pos0 < HH && g > tg && g <= ge;
            if (in_pre || in_suf) {
                float t4[4];
                load_tot4(x.s_tot, g, cq, t4);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (in_pre) cpre[c] *= t4[c];
                    if (in_suf) csuf[c] *= t4[c];
                }
            }
        }
    }
    float run[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) run[c] = cpre[c];
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {  // second-half rows: prefix from the half start
        const int r = tg * 8 + i, pos = r % BS;
        if (HH < 8 && pos == HH) {
#pragma unroll
            for (int c = 0; c < 4; ++c) run[c] = 1.f;
        }
        if (pos < HH) continue;
        const bool v = r < x.nvalid;
        float al[4], qv[4], kv[4], e[4], fa[4], fp[4];
        unpack4(raw_quad(sm, RAW_A, r, cq), al);
        unpack4(raw_quad(sm, RAW_Q, r, cq), qv);
        unpack4(raw_quad(sm, RAW_K, r, cq), kv);
        erase_gate4(x, r, cq, e);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            run[c] *= v ? al[c] : 1.f;
            fa[c] = v ? run[c] * e[c] * kv[c] : 0.f;
            fp[c] = v ? run[c] * qv[c] : 0.f;
        }
        const int idx = (r / BS) * HH + (pos - HH);
        *reinterpret_cast<uint2 *>(sm + x.la + sw_half(16384, slot * 32 + idx, cq)) = pack4(fa);
        *reinterpret_cast<uint2 *>(sm + x.la + sw_half(16384, 64 + slot * 32 + idx, cq)) = pack4(fp);
    }
    float sx[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) sx[c] = csuf[c];
#pragma unroll 1
    for (int i = 7; i >= 0; --i) {  // first-half columns: exclusive suffix to the half end
        const int r = tg * 8 + i, pos = r % BS;
        if (pos >= HH) continue;
        if (HH < 8 && pos == HH - 1) {
#pragma unroll
            for (int c = 0; c < 4; ++c) sx[c] = 1.f;
        }
        const bool v = r < x.nvalid;
        float al[4], kv[4], fc[4];
        unpack4(raw_quad(sm, RAW_A, r, cq), al);
        unpack4(raw_quad(sm, RAW_K, r, cq), kv);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            fc[c] = v ? sx[c] * kv[c] : 0.f;
            sx[c] *= v ? al[c] : 1.f;
        }
        const int idx = (r / BS) * HH + pos;
        *reinterpret_cast<uint2 *>(sm + x.lb + sw_half(8192, slot * 32 + idx, cq)) = pack4(fc);
    }
}

// Anchored path: scatter one level's A or P entries from the 32 TMEM columns
// the calling warp loaded (rows of this lane's level list).
template <int HH>
__device__ __forceinline__ void scatter_level(uint8_t *pbf, float *Af, const float *s_e, bool isP, int lane,
                                              const float *v)
{
    constexpr int BS = 2 * HH;
    const int r = (lane / HH) * BS + HH + (lane % HH);
    const int c0 = (r / BS) * HH;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        if (c >= c0 && c < c0 + HH) {
            const int s = (c / HH) * BS + (c % HH);
            if (!isP) Af[r * TP + s] = v[c] * s_e[r];
            else *reinterpret_cast<unsigned short *>(pbf + sw_elem(8192, r, s)) = bf16_bits(v[c]);
        }
    }
}

// ---- exact path for ill-conditioned chunks ------------------------------------
// The raw inputs of one chunk, rows 0 .. nv-1 (64 x 128 bf16 each, row-major),
// copied to shared memory with the input preparation applied as the
// preparation kernel applies it (alpha activated and k normalised, both
// rounded to bf16); rows past nv are not written.  All `nthreads` threads
// from `tid` take part; the caller synchronises afterwards.
__device__ __forceinline__ void stage_exact_inputs(const FwdArgs &a, size_t tok0, int nv, int h, uint8_t *dq,
                                                   uint8_t *dk, uint8_t *da, int tid, int nthreads)
{
    const int H = a.H;
    const uint4 *gq = reinterpret_cast<const uint4 *>(a.q), *gk = reinterpret_cast<const uint4 *>(a.k),
                *ga = reinterpret_cast<const uint4 *>(a.alpha);
    const bool logits = (a.prep & PREP_LOGITS) != 0, l2k = (a.prep & PREP_L2NORM_K) != 0, ext = a.ext != 0;
    // four threads per row (adjacent lanes), 32 channels (four 16-byte pieces) each; every lane of
    // a warp runs the same iterations (nthreads is a multiple of 32), so the row sums can shuffle
    for (int base = 0; base < nv * 4; base += nthreads) {
        const int e = base + tid;
        const bool act = e < nv * 4;
        const int r = e >> 2, part = e & 3;
        const size_t g = ((tok0 + r) * H + h) * (D / 8) + part * 4;
        uint4 qv[4], kv[4], av[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            qv[j] = act ? gq[g + j] : make_uint4(0, 0, 0, 0);
            kv[j] = act ? gk[g + j] : make_uint4(0, 0, 0, 0);
            av[j] = act ? ga[g + j] : make_uint4(0, 0, 0, 0);
        }
        if (logits) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float f[8];
                unpack8(av[j], f);
#pragma unroll
                for (int c = 0; c < 8; ++c) f[c] = prep_alpha(f[c], ext);
                av[j] = pack8(f);
            }
        }
        if (l2k) {
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float f[8];
                unpack8(kv[j], f);
#pragma unroll
                for (int c = 0; c < 8; ++c) ss = fmaf(f[c], f[c], ss);
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);   // the row's four threads are adjacent lanes
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            const float sc = prep_kscale(ss);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float f[8];
                unpack8(kv[j], f);
#pragma unroll
                for (int c = 0; c < 8; ++c) f[c] *= sc;
                kv[j] = pack8(f);
            }
        }
        if (act) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                reinterpret_cast<uint4 *>(dq + r * 256)[part * 4 + j] = qv[j];
                reinterpret_cast<uint4 *>(dk + r * 256)[part * 4 + j] = kv[j];
                reinterpret_cast<uint4 *>(da + r * 256)[part * 4 + j] = av[j];
            }
        }
    }
}

// The recurrence of one chunk token by token, in fp32, on the state in TMEM
// (lane j = value column j, column i = key channel i): per token
//   S' = Diag(alpha) S,  u = m - S'^T a~,  S = S' + k u^T,  o = S^T q = S'^T q + (k . q) u.
// The calling thread owns value column jcol and key channels [i0, i0 + 32 NP)
// at TMEM address `tstate` (its lane, column 0 of S).  With PAIR the other
// channels of the column belong to the thread of the other warp of the same
// TMEM lane quarter; the two add their partial sums through `xch`
// (float4 [2][2][128]) and named barrier `bar_id` (64 threads).  q, k, alpha
// rows come from the staging tiles (row-major [64][128] bf16, prepared);
// v, the gates and GDN-2's erase vector are read from global memory (and
// activated here when they are logits).  o_t,j goes to bf16 element
// ost[t * ost_stride + jcol] (a staging tile or o itself) when `write_o`.
// Every warp of the caller runs the same token loop (the TMEM accesses are
// warp-wide).
template <int NP, bool PAIR>
__device__ __noinline__ void exact_chunk(const FwdArgs &a, uint32_t tstate, int i0, int jcol, int half,
                                         const uint8_t *sq, const uint8_t *sk, const uint8_t *sa, size_t tok0,
                                         int nv, int h, float4 *xch, uint32_t bar_id, unsigned short *ost,
                                         size_t ost_stride, bool write_o)
{
    const int H = a.H;
    const __nv_bfloat16 *g1 = (const __nv_bfloat16 *)a.g1, *g2 = (const __nv_bfloat16 *)a.g2,
                        *vv = (const __nv_bfloat16 *)a.v;
    const bool gdn2 = a.variant == GDN2, logits = (a.prep & PREP_LOGITS) != 0, ext = a.ext != 0;
    auto gate = [&](float x) { return logits ? round_bf16(prep_gate(x, ext)) : x; };
#pragma unroll 1
    for (int t = 0; t < nv; ++t) {
        const size_t tok = (tok0 + t) * H + h;
        float e, m;
        const float vj = __bfloat162float(vv[tok * D + jcol]);
        if (gdn2) {
            e = 1.f;
            m = gate(__bfloat162float(g2[tok * D + jcol])) * vj;
        } else {
            e = gate(__bfloat162float(g1[tok]));
            m = (a.variant == KDA ? e : gate(__bfloat162float(g2[tok]))) * vj;
        }
        const uint4 *qr = reinterpret_cast<const uint4 *>(sq + t * 256);
        const uint4 *kr = reinterpret_cast<const uint4 *>(sk + t * 256);
        const uint4 *ar = reinterpret_cast<const uint4 *>(sa + t * 256);
        const uint4 *br = gdn2 ? reinterpret_cast<const uint4 *>(g1 + tok * D) : nullptr;
        float pk = 0.f, pq = 0.f, pkq = 0.f;
#pragma unroll 1
        for (int p = 0; p < NP; ++p) {
            const int c0 = i0 + 32 * p;
            float s[32];
            tmem_ld32(tstate + c0, s);
            tmem_wait_ld();
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8) {
                float qf[8], kf[8], af[8];
                unpack8(qr[c0 / 8 + j8], qf);
                unpack8(kr[c0 / 8 + j8], kf);
                unpack8(ar[c0 / 8 + j8], af);
                if (gdn2) {   // erase direction b (.) k
                    float bf[8];
                    unpack8(br[c0 / 8 + j8], bf);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float sp = af[c] * s[j8 * 8 + c];
                        pk = fmaf(gate(bf[c]) * kf[c], sp, pk);
                        pq = fmaf(qf[c], sp, pq);
                        pkq = fmaf(qf[c], kf[c], pkq);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float sp = af[c] * s[j8 * 8 + c];
                        pk = fmaf(kf[c], sp, pk);
                        pq = fmaf(qf[c], sp, pq);
                        pkq = fmaf(qf[c], kf[c], pkq);
                    }
                }
            }
        }
        if (PAIR) {
            float4 *mine = xch + (t & 1) * 256;
            mine[half * 128 + jcol] = make_float4(pk, pq, pkq, 0.f);
            group_sync(bar_id, 64);
            const float4 o4 = mine[(half ^ 1) * 128 + jcol];
            pk += o4.x;
            pq += o4.y;
            pkq += o4.z;
        }
        const float u = m - e * pk;
        if (write_o) ost[t * ost_stride + jcol] = bf16_bits(fmaf(pkq, u, pq));
#pragma unroll 1
        for (int p = 0; p < NP; ++p) {
            const int c0 = i0 + 32 * p;
            float s[32];
            tmem_ld32(tstate + c0, s);
            tmem_wait_ld();
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8) {
                float kf[8], af[8];
                unpack8(kr[c0 / 8 + j8], kf);
                unpack8(ar[c0 / 8 + j8], af);
#pragma unroll
                for (int c = 0; c < 8; ++c) s[j8 * 8 + c] = fmaf(kf[c], u, af[c] * s[j8 * 8 + c]);
            }
            tmem_st16(tstate + c0, s);
            tmem_st16(tstate + c0 + 16, s + 16);
        }
        tmem_wait_st();
    }
}

// ---- the kernel -------------------------------------------------------------
// Warp roles.  Warps 0-3 (CHAIN, 128 threads) own the state: for chunk n they
// scale S by Gamma_C and copy it to bf16, run U^T -= S^T W^T, O^T = S^T Q^T,
// read U^T out, run O^T += U^T P^T, S^T += U^T Kbar, and write o.  Warps 4-11
// (PREP, 256 threads) build chunk n+1's operands meanwhile: decay products,
// row operands, Kbar, the band of P, A and P, T = (I+A)^{-1}, W and U'^T.
// Hand-offs go through mbarriers; each buffer the two groups share is
// released by the step that last reads it:
//   ready  : prep(n) -> chain(n)   (QA = [-W'; Q'], Kbar, P, U' in TMEM, Gamma_C)
//   s6     : chain(n) GEMMs of step 6 done -> prep(n+1) may rewrite QA
//   s7     : chain(n) GEMMs of step 7 done -> prep(n+1) may rewrite Kbar, P, levels
//   ufree  : chain(n) has read U^T out of TMEM -> prep(n+1) may write U'^T
constexpr int NCHAIN = 128, NPREP = 256;
constexpr uint32_t BAR_PREP = 1, BAR_CHAIN = 2;

// The fused kernel: one CTA per (sequence, head), both roles.
// PREP: input preparation requested (gate logits and / or raw keys); without
// it the preparation code is compiled out.
template <bool PREP>
__global__ void __launch_bounds__(NT, 1) chunk_fwd_kernel(const __grid_constant__ ChunkParams P)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);
    const FwdArgs &a = P.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;       // TMEM lane quarter of this warp
    const int H = a.H;
    const int n = blockIdx.x / H, h = blockIdx.x % H;   // this CTA's sequence and head
    const int len = seq_len(a, n);
    const int nchunks = (len + C - 1) / C;

    // scalar gates, per item parity (filled one item ahead)
    auto s_g1buf = [&](uint32_t parity) { return reinterpret_cast<float *>(sm + (parity ? M_G1B : M_G1)); };
    auto s_g2buf = [&](uint32_t parity) { return reinterpret_cast<float *>(sm + (parity ? M_G2B : M_G2)); };
    float *s_gamC = reinterpret_cast<float *>(sm + M_GAMC);     // [2][128]: chunk parity
    float *s_tot = reinterpret_cast<float *>(sm + M_TOT);       // [8][128] block totals of alpha
    float *s_pband = reinterpret_cast<float *>(sm + M_PBAND);   // [64][PBAND]: P_{r, r-w}
    int *s_fast = reinterpret_cast<int *>(sm + M_FAST);         // [2]: chunk parity
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + M_BAR);
    uint64_t *bar_tma = bars + 0, *bar_v = bars + 1, *bar_pmma = bars + 2, *bar_ready = bars + 3;
    uint64_t *bar_s6 = bars + 4, *bar_s7 = bars + 5, *bar_ufree = bars + 6;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + M_TMEM);
    float *Af = reinterpret_cast<float *>(sm + OFF_AF32);
    float *Tf = reinterpret_cast<float *>(sm + OFF_TF32);
    float *Xs = reinterpret_cast<float *>(sm + OFF_X);

    const __nv_bfloat16 *g1p = (const __nv_bfloat16 *)a.g1, *g2p = (const __nv_bfloat16 *)a.g2;
    uint8_t *op = (uint8_t *)a.o;
    const bool gdn2 = a.variant == GDN2;
    const bool same_gates = a.variant != RDA;   // erase and write gates coincide: one T copy serves both
    const bool logits = PREP && (a.prep & PREP_LOGITS) != 0, l2k = PREP && (a.prep & PREP_L2NORM_K) != 0;
    const bool ext = a.ext != 0;

    if (warp == 0) tmem_alloc(s_tmem, 512);
    if (tid == 0) {
        for (int i = 0; i < 7; ++i) mbar_init(bars + i, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    bool ok = true;

    if (warp < 4) {
        // =====================================================================
        // CHAIN group
        // =====================================================================
        const int jcol = tid;   // value column j = TMEM lane
        {   // initial state -> TMEM (fp32)
            const size_t soff = ((size_t)n * H + h) * D * D;
#pragma unroll 1
            for (int c16 = 0; c16 < 8; ++c16) {
                float v[16];
                const int i0 = c16 * 16;
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = a.s0 ? a.s0[soff + (size_t)(i0 + e) * D + jcol] : 0.f;
                tmem_st16(tbase + lane_base + TM_S + i0, v);
            }
            tmem_wait_st();
        }
        for (int ch = 0; ch < nchunks && ok; ++ch) {
            const uint32_t par = ch & 1;
            const int nvalid = min(C, len - ch * C);
            const size_t rowbase = (size_t)seq_row0(a, n) + ch * C;
            if (!mbar_wait_cycles(bar_ready, par, WAIT_CYCLES)) ok = false;
            tc_fence_after();
            const int cflags = s_fast[par];
            unsigned short *ost = reinterpret_cast<unsigned short *>(sm + OFF_UT);   // o staging [r][j]
            const bool exact = ok && (cflags & META_EXACT);
            if (exact) {
                // ---- exact path: this chunk token by token in fp32.  None of its prepared operands
                // is read, so they are released at once; q and k are staged in the state-operand
                // tile, alpha in the U^T tile (the chain's own shared memory), and o goes straight
                // to HBM.
                if (tid == 0) {
                    mbar_arrive(bar_s6);
                    mbar_arrive(bar_ufree);
                    mbar_arrive(bar_s7);
                }
                uint8_t *stq = sm + OFF_S0T, *stk = sm + OFF_S0T + 16384, *sta = sm + OFF_UT;
                stage_exact_inputs(a, rowbase, nvalid, h, stq, stk, sta, tid, NCHAIN);
                group_sync(BAR_CHAIN, NCHAIN);
                exact_chunk<4, false>(a, tbase + lane_base + TM_S, 0, jcol, 0, stq, stk, sta, rowbase, nvalid, h,
                                      nullptr, 0, reinterpret_cast<unsigned short *>(op) + (rowbase * H + h) * D,
                                      (size_t)H * D, true);
                tc_fence_before();
                group_sync(BAR_CHAIN, NCHAIN);
                tc_fence_after();
                if (a.snap) snapshot_state(a, tbase + lane_base, slot_base(a, n) + ch, h, 0, 4, jcol);
            } else {
                const bool fast = (cflags & META_FAST) != 0;
                const float *gamC = s_gamC + par * 128;
                // ---- state pass: S^T *= Gamma_C in TMEM; bf16 operand copy (scaled on the fast path)
#pragma unroll 1
                for (int c32 = 0; c32 < 4; ++c32) {
                    const int i0 = c32 * 32;
                    float s[32], t[32];
                    tmem_ld32(tbase + lane_base + TM_S + i0, s);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        t[e] = s[e] * gamC[i0 + e];
                        if (fast) s[e] = t[e];
                    }
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4 *>(sm + OFF_S0T + sw_chunk(16384, jcol, (i0 >> 3) + q4)) = pack8(s + q4 * 8);
                    tmem_st16(tbase + lane_base + TM_S + i0, t);
                    tmem_st16(tbase + lane_base + TM_S + i0 + 16, t + 16);
                }
                tmem_wait_st();
                fence_async_smem();
                tc_fence_before();
                group_sync(BAR_CHAIN, NCHAIN);
                // ---- step 6: U^T -= S^T W^T ; O^T = S^T Q^T
                if (tid == 0) {
                    tc_fence_after();
                    step6_mmas(tbase, sb + OFF_S0T, sb + OFF_QA);
                    mma_commit(bar_s6);
                }
                if (!mbar_wait_cycles(bar_s6, par, WAIT_CYCLES)) ok = false;
                tc_fence_after();
                // ---- U^T row j -> bf16 K-major tile (rows j, K = token); then release TMEM U
#pragma unroll
                for (int c32 = 0; c32 < 2; ++c32) {
                    float v[32];
                    tmem_ld32(tbase + lane_base + TM_U + c32 * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4 *>(sm + OFF_UT + sw_chunk(16384, jcol, c32 * 4 + q4)) = pack8(v + q4 * 8);
                }
                fence_async_smem();
                tc_fence_before();
                group_sync(BAR_CHAIN, NCHAIN);
                // ---- step 7: O^T += U^T P^T ; S^T += U^T Kbar
                if (tid == 0) {
                    mbar_arrive(bar_ufree);
                    tc_fence_after();
                    const uint32_t id_o = idesc_bf16(128, 64, false, false);
                    const uint32_t id_s = idesc_bf16(128, 128, false, true);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        mma_bf16(tbase + TM_O, dK(sb + OFF_UT, 16384, kk), dK(sb + OFF_PBF, 8192, kk), id_o, 1);
                        mma_bf16(tbase + TM_S, dK(sb + OFF_UT, 16384, kk), dMN(sb + OFF_KB, 8192, kk), id_s, 1);
                    }
                    mma_commit(bar_s7);
                }
                if (!mbar_wait_cycles(bar_s7, par, WAIT_CYCLES)) ok = false;
                tc_fence_after();
                if (a.snap) snapshot_state(a, tbase + lane_base, slot_base(a, n) + ch, h, 0, 4, jcol);
                // ---- o: TMEM (lane j, column r) -> bf16 staging [r][j] in the U^T slot -> HBM
#pragma unroll
                for (int c32 = 0; c32 < 2; ++c32) {
                    float v[32];
                    tmem_ld32(tbase + lane_base + TM_O + c32 * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const uint32_t pk = pack_bf16(v[e], v[e + 1]);
                        ost[(c32 * 32 + e) * 128 + jcol] = (unsigned short)(pk & 0xFFFFu);
                        ost[(c32 * 32 + e + 1) * 128 + jcol] = (unsigned short)(pk >> 16);
                    }
                }
            }   // normal (tensor-core) chunk
            tc_fence_before();
            group_sync(BAR_CHAIN, NCHAIN);
            if (!exact) {   // the exact path wrote o itself
                for (int e = tid; e < nvalid * 16; e += NCHAIN) {
                    const int r = e >> 4, cgo = e & 15;
                    *reinterpret_cast<uint4 *>(op + (((rowbase + r) * H + h) * D + cgo * 8) * 2) =
                        *reinterpret_cast<const uint4 *>(sm + OFF_UT + r * 256 + cgo * 16);
                }
            }
            ok = group_sync_and(BAR_CHAIN, NCHAIN, ok);   // staging read before the next U^T write
        }
    } else {
        // =====================================================================
        // PREP group
        // =====================================================================
        const int ptid = tid - NCHAIN, pw = warp - 4;
        const int phalf = pw >> 2;              // the two prep warps of a lane quarter split columns
        const int jrow = quarter * 32 + lane;   // TMEM lane of this thread
        const int tg = ptid >> 5, cq = ptid & 31;   // elementwise item: 8 tokens x 4 channels
        uint32_t ph_tma = 0, ph_v = 0, ph_pmma = 0;

        const CUtensorMap *map_q = &P.tq, *map_k = &P.tk, *map_v = &P.tv, *map_a = &P.ta;
        auto issue_tma = [&](const Item &it) {   // q, k, alpha of a chunk
            const int g = it.row0 + it.c * C;
            mbar_expect_tx(bar_tma, 3 * 16384);
            tma_load_3d(sm + RAW_Q, map_q, bar_tma, 0, it.h, g);
            tma_load_3d(sm + RAW_K, map_k, bar_tma, 0, it.h, g);
            tma_load_3d(sm + RAW_A, map_a, bar_tma, 0, it.h, g);
        };
        auto issue_tma_v = [&](const Item &it) {   // v, straight into its swizzled operand layout
            const int g = it.row0 + it.c * C;
            mbar_expect_tx(bar_v, 16384);
            tma_load_3d(sm + OFF_MT, map_v, bar_v, 0, it.h, g);
            tma_load_3d(sm + OFF_MT + 8192, map_v, bar_v, 64, it.h, g);
        };
        auto wait_pmma = [&]() {
            if (!mbar_wait_cycles(bar_pmma, ph_pmma, WAIT_CYCLES)) ok = false;
            ph_pmma ^= 1;
            tc_fence_after();
        };
        auto publish = [&]() {
            fence_async_smem();
            tc_fence_before();
            group_sync(BAR_PREP, NPREP);
        };
        auto publish_and = [&](bool pred) {   // publish, and the AND of pred over the group
            fence_async_smem();
            tc_fence_before();
            return group_sync_and(BAR_PREP, NPREP, pred);
        };
        // scalar gates of row r of a chunk into the gate arrays of item parity `parity`
        // (0 past the chunk's end; GDN-2 keeps its gates channel-wise: 1 here)
        auto fetch_gates = [&](const Item &it, int r, uint32_t parity) {
            const int nv = min(C, it.len - it.c * C);
            const size_t tok = ((size_t)it.row0 + it.c * C + r) * H + it.h;
            const bool v = r < nv;
            const unsigned short *g1u = reinterpret_cast<const unsigned short *>(g1p);
            const unsigned short *g2u = reinterpret_cast<const unsigned short *>(g2p);
            uint32_t ge, gw;
            if (gdn2) { ge = v ? 0x3F80u : 0u; gw = ge; }   // bf16 1.0 / 0.0
            else {
                ge = v ? (uint32_t)g1u[tok] : 0u;
                gw = v ? (uint32_t)(a.variant == KDA ? g1u[tok] : g2u[tok]) : 0u;
            }
            float fe = __uint_as_float(ge << 16), fw = __uint_as_float(gw << 16);
            if (logits && !gdn2 && v) {
                fe = round_bf16(prep_gate(fe, ext));
                fw = round_bf16(prep_gate(fw, ext));
            }
            s_g1buf(parity)[r] = fe;
            s_g2buf(parity)[r] = fw;
        };
        // the chunks of this CTA's sequence, one after the other
        auto fused_item = [&](int c) {
            Item it{n, h, c, 0, len, 0, c < nchunks};
            it.row0 = seq_row0(a, n);
            return it;
        };
        Item cur = fused_item(0);
        if (cur.valid && ptid == 0) {
            issue_tma(cur);
            issue_tma_v(cur);
        }
        if (ptid < C && cur.valid) fetch_gates(cur, ptid, 0);

        for (int ch = 0; cur.valid && ok; ++ch) {
            const uint32_t par = ch & 1, ppar = (ch - 1) & 1;
            const Item nxt = fused_item(ch + 1);
            const int h = cur.h;
            const int nvalid = min(C, cur.len - cur.c * C);
            const size_t rowbase = (size_t)cur.row0 + cur.c * C;
            float *const s_g1 = s_g1buf(par);
            float *const s_g2 = s_g2buf(par);
            const ChunkCtx x{sm,   s_tot, s_g1,   g1p,    rowbase, H,     h,     nvalid,
                             gdn2, logits, ext, OFF_QA, OFF_KB, OFF_LA, OFF_LB};
            float *gamc = s_gamC + par * 128;

            if (!mbar_wait_cycles(bar_tma, ph_tma, WAIT_CYCLES)) ok = false;
            ph_tma ^= 1;
            if (!mbar_wait_cycles(bar_v, ph_v, WAIT_CYCLES)) ok = false;
            ph_v ^= 1;
            group_sync(BAR_PREP, NPREP);

            // ===== 0. input preparation, in place in the raw tiles (this thread's 8 rows x 4 channels),
            // rounded to bf16 as a separate activation / normalisation pass would have stored them
            if (PREP && logits) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint2 *pa = reinterpret_cast<uint2 *>(sm + RAW_A + (tg * 8 + i) * 256 + cq * 8);
                    float al[4];
                    unpack4(*pa, al);
#pragma unroll
                    for (int c = 0; c < 4; ++c) al[c] = prep_alpha(al[c], ext);
                    *pa = pack4(al);
                }
            }
            if (PREP && l2k) {   // 1 / ||k_r|| of this warp's 8 rows: 4-channel partial sums, reduce-scattered
                float ss[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float kv[4];
                    unpack4(raw_quad(sm, RAW_K, tg * 8 + i, cq), kv);
                    ss[i] = kv[0] * kv[0] + kv[1] * kv[1] + kv[2] * kv[2] + kv[3] * kv[3];
                }
                const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float send = b4 ? ss[i] : ss[i + 4];
                    ss[i] = (b4 ? ss[i + 4] : ss[i]) + __shfl_xor_sync(0xffffffffu, send, 16);
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float send = b3 ? ss[i] : ss[i + 2];
                    ss[i] = (b3 ? ss[i + 2] : ss[i]) + __shfl_xor_sync(0xffffffffu, send, 8);
                }
                {
                    const float send = b2 ? ss[0] : ss[1];
                    ss[0] = (b2 ? ss[1] : ss[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
                }
                ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], 2);
                ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], 1);
                // lane 4 i holds row i's sum (i = 4 b4 + 2 b3 + b2): hand each lane its rows' scales
                const float sc = prep_kscale(ss[0]);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float sci = __shfl_sync(0xffffffffu, sc, ((i & 4) ? 16 : 0) + ((i & 2) ? 8 : 0) + ((i & 1) ? 4 : 0));
                    uint2 *pk = reinterpret_cast<uint2 *>(sm + RAW_K + (tg * 8 + i) * 256 + cq * 8);
                    float kv[4];
                    unpack4(*pk, kv);
#pragma unroll
                    for (int c = 0; c < 4; ++c) kv[c] *= sci;
                    *pk = pack4(kv);
                }
            }

            // ===== 1a. block totals of alpha (and range check) | GDN-2: M = w (.) v
            bool in_range = true;
            {
                float tot[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = tg * 8 + i;
                    if (r < nvalid) {
                        float al[4];
                        unpack4(raw_quad(sm, RAW_A, r, cq), al);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            tot[c] *= al[c];
                            in_range = in_range && (fabsf(al[c]) <= 1.f);
                        }
                    }
                }
                *reinterpret_cast<float4 *>(s_tot + tg * 128 + cq * 4) = make_float4(tot[0], tot[1], tot[2], tot[3]);
            }
            if (gdn2) {   // in place in the swizzled v tile; rows past the end -> 0
#pragma unroll 2
                for (int i = 0; i < 8; ++i) {
                    const int r = tg * 8 + i;
                    uint2 *pv = reinterpret_cast<uint2 *>(sm + OFF_MT + sw_half(8192, r, cq));
                    float mv[4], vv[4], wv[4];
                    unpack4(*pv, vv);
                    if (r < nvalid) {
                        unpack4(*reinterpret_cast<const uint2 *>(g2p + ((rowbase + r) * H + h) * D + cq * 4), wv);
#pragma unroll
                        for (int c = 0; c < 4; ++c) mv[c] = (logits ? round_bf16(prep_gate(wv[c], ext)) : wv[c]) * vv[c];
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c) mv[c] = 0.f;
                    }
                    *pv = pack4(mv);
                }
            }
            in_range = group_sync_and(BAR_PREP, NPREP, in_range);

            // ===== Gamma_C and the per-chunk path decision ========================
            bool gam_ok = true;
            if (ptid < 32) {
                float gc[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    float t4[4];
                    load_tot4(s_tot, g, ptid, t4);
#pragma unroll
                    for (int c = 0; c < 4; ++c) gc[c] *= t4[c];
                }
                *reinterpret_cast<float4 *>(gamc + ptid * 4) = make_float4(gc[0], gc[1], gc[2], gc[3]);
#pragma unroll
                for (int c = 0; c < 4; ++c) gam_ok = gam_ok && (fabsf(gc[c]) >= FAST_MIN_GAMMA);
            }
            const bool fast = group_sync_and(BAR_PREP, NPREP, gam_ok) && in_range;

            // the previous chunk's chain must be done with QA (step 6) and with Kbar / P (step 7)
            if (ch > 0) {
                if (!mbar_wait_cycles(bar_s6, ppar, WAIT_CYCLES)) ok = false;
                if (!mbar_wait_cycles(bar_s7, ppar, WAIT_CYCLES)) ok = false;
            }

            // ===== 1b. row operands, Kbar and the exact band of P ================
            if (fast) {
                // one forward sweep per item; band partials to the F region, reduced after the A/P GEMM issue
                float *band_part = reinterpret_cast<float *>(sm + OFF_F);
                if (nvalid == C) {
                    if (gdn2) fast_rows<true, true, 1>(x, s_tot, gamc, band_part, tg, cq, lane);
                    else fast_rows<true, false, 1>(x, s_tot, gamc, band_part, tg, cq, lane);
                } else {
                    fast_rows<false, true, 1>(x, s_tot, gamc, band_part, tg, cq, lane);
                }
            } else {
            {
                    float pre[4] = {1.f, 1.f, 1.f, 1.f}, suf[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        if (g == tg) continue;
                        float t4[4];
                        load_tot4(s_tot, g, cq, t4);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            if (g < tg) pre[c] *= t4[c];
                            else suf[c] *= t4[c];
                        }
                    }
                    float sc[4];
                    if (fast) {
                        const float4 gc4 = *reinterpret_cast<const float4 *>(gamc + cq * 4);
                        sc[0] = pre[0] / gc4.x; sc[1] = pre[1] / gc4.y; sc[2] = pre[2] / gc4.z; sc[3] = pre[3] / gc4.w;
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c) sc[c] = pre[c];
                    }
#pragma unroll 2
                    for (int i = 0; i < 8; ++i) {   // forward: rows 0-63 Gamma a~, rows 64-127 Gamma q
                        const int r = tg * 8 + i;
                        const bool v = r < nvalid;
                        float al[4], kv[4], qv[4], e[4], oa[4], oq[4];
                        unpack4(raw_quad(sm, RAW_A, r, cq), al);
                        unpack4(raw_quad(sm, RAW_K, r, cq), kv);
                        unpack4(raw_quad(sm, RAW_Q, r, cq), qv);
                        erase_gate4(x, r, cq, e);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            sc[c] *= v ? al[c] : 1.f;
                            oa[c] = v ? sc[c] * (e[c] * kv[c]) : 0.f;
                            oq[c] = v ? sc[c] * qv[c] : 0.f;
                        }
                        *reinterpret_cast<uint2 *>(sm + OFF_QA + sw_half(16384, r, cq)) = pack4(oa);
                        *reinterpret_cast<uint2 *>(sm + OFF_QA + sw_half(16384, 64 + r, cq)) = pack4(oq);
                    }
                    float sx[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) sx[c] = suf[c];
#pragma unroll 2
                    for (int i = 7; i >= 0; --i) {   // backward: Kbar_s = (prod_{s<t<C} alpha_t) (.) k_s
                        const int r = tg * 8 + i;
                        const bool v = r < nvalid;
                        float al[4], kv[4], kb[4];
                        unpack4(raw_quad(sm, RAW_A, r, cq), al);
                        unpack4(raw_quad(sm, RAW_K, r, cq), kv);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            kb[c] = v ? sx[c] * kv[c] : 0.f;
                            sx[c] *= v ? al[c] : 1.f;
                        }
                        *reinterpret_cast<uint2 *>(sm + OFF_KB + sw_half(8192, r, cq)) = pack4(kb);
                    }
                }
                {   // band of P: P_{r,r-w} = sum_c q_rc (alpha_r ... alpha_{r-w+1})_c k_{r-w,c}, w = 0..4,
                    // from the bf16 inputs in fp32: the entries whose bf16 GEMM rounding would hurt most.
                    // Four threads per row (32 channels each), chunk order staggered by row so the loads
                    // are bank-conflict free; rows below w are clamped and masked afterwards.
                    const int r = ptid >> 2, c4 = ptid & 3;
                    float acc[PBAND];
#pragma unroll
                    for (int w = 0; w < PBAND; ++w) acc[w] = 0.f;
#pragma unroll 1
                    for (int j = 0; j < 4; ++j) {
                        const int cgx = c4 * 4 + ((j + r) & 3);
                        float hv[8];
                        unpack8(raw_row(sm, RAW_Q, r, cgx), hv);
#pragma unroll
                        for (int w = 0; w < PBAND; ++w) {
                            float kv[8];
                            unpack8(raw_row(sm, RAW_K, max(r - w, 0), cgx), kv);
#pragma unroll
                            for (int c = 0; c < 8; ++c) acc[w] = fmaf(hv[c], kv[c], acc[w]);
                            if (w + 1 < PBAND) {
                                float av[8];
                                unpack8(raw_row(sm, RAW_A, max(r - w, 0), cgx), av);
#pragma unroll
                                for (int c = 0; c < 8; ++c) hv[c] *= av[c];
                            }
                        }
                    }
#pragma unroll
                    for (int w = 0; w < PBAND; ++w) {
                        float t = acc[w] + __shfl_xor_sync(0xffffffffu, acc[w], 1);
                        t += __shfl_xor_sync(0xffffffffu, t, 2);
                        if (c4 == 0) s_pband[r * PBAND + w] = (r < nvalid && r - w >= 0) ? t : 0.f;
                    }
                }
            }
            group_sync(BAR_PREP, NPREP);   // band and row operands complete before either A/P path reads them

            // ===== 2. A and P ======================================================
            if (fast) {
                publish();
                if (ptid == 0) {
                    tc_fence_after();
                    const uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tbase + TM_AP, dK(sb + OFF_QA, 16384, kk), dK(sb + OFF_KB, 8192, kk), idesc, kk > 0);
                    mma_commit(bar_pmma);
                }
                // band of P while the GEMM runs; the partials' F region is rewritten by the read-out below
                band_reduce(reinterpret_cast<const float *>(sm + OFF_F), s_pband, nvalid, ptid, NPREP);
                group_sync(BAR_PREP, NPREP);
                wait_pmma();
                if (ptid == 0 && nxt.valid) issue_tma(nxt);   // raw tiles consumed
                // rows 0-63: A (strictly lower, scaled by e_r), rows 64-127: P (band exact)
                float v[32];
                tmem_ld32(tbase + lane_base + TM_AP + phalf * 32, v);
                tmem_wait_ld();
                const int rr = jrow & 63;
                if (jrow < 64) {
                    const float er = s_g1[rr];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int s = phalf * 32 + c;
                        v[c] = (s < rr) ? v[c] * er : 0.f;
                    }
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        *reinterpret_cast<float4 *>(Af + rr * TP + phalf * 32 + 4 * q4) =
                            make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int s = phalf * 32 + c;
                        const int w = rr - s;
                        v[c] = (w >= PBAND) ? v[c] : ((w >= 0) ? s_pband[rr * PBAND + w] : 0.f);
                    }
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4 *>(sm + OFF_PBF + sw_chunk(8192, rr, phalf * 4 + q4)) = pack8(v + q4 * 8);
                }
            } else {
                // anchored levels: three GEMMs of two levels each
                for (int p = 0; p < 3; ++p) {
#pragma unroll 1
                    for (int slot = 0; slot < 2; ++slot) {
                        switch (2 * p + 1 + slot) {
                        case 1: build_level<32>(x, slot, tg, cq); break;
                        case 2: build_level<16>(x, slot, tg, cq); break;
                        case 3: build_level<8>(x, slot, tg, cq); break;
                        case 4: build_level<4>(x, slot, tg, cq); break;
                        case 5: build_level<2>(x, slot, tg, cq); break;
                        default: build_level<1>(x, slot, tg, cq); break;
                        }
                    }
                    publish();
                    if (ptid == 0) {
                        tc_fence_after();
                        const uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_bf16(tbase + tm_lvl(p), dK(sb + OFF_LA, 16384, kk), dK(sb + OFF_LB, 8192, kk), idesc,
                                     kk > 0);
                        mma_commit(bar_pmma);
                    }
                    wait_pmma();
                }
                if (ptid == 0 && nxt.valid) issue_tma(nxt);   // raw tiles consumed
                for (int e = ptid; e < 64 * TP; e += NPREP) Af[e] = 0.f;
                for (int e = ptid; e < 512; e += NPREP)
                    *reinterpret_cast<uint4 *>(sm + OFF_PBF + e * 16) = make_uint4(0, 0, 0, 0);
                group_sync(BAR_PREP, NPREP);
                for (int p = phalf; p < 3; p += 2) {   // the two warps of a lane quarter share the pairs
                    const int lvl = 2 * p + 1 + (quarter & 1);
                    const bool isP = quarter >= 2;
                    float v[32];
                    tmem_ld32(tbase + lane_base + tm_lvl(p) + (quarter & 1) * 32, v);
                    tmem_wait_ld();
                    switch (lvl) {
                    case 1: scatter_level<32>(sm + OFF_PBF, Af, s_g1, isP, lane, v); break;
                    case 2: scatter_level<16>(sm + OFF_PBF, Af, s_g1, isP, lane, v); break;
                    case 3: scatter_level<8>(sm + OFF_PBF, Af, s_g1, isP, lane, v); break;
                    case 4: scatter_level<4>(sm + OFF_PBF, Af, s_g1, isP, lane, v); break;
                    case 5: scatter_level<2>(sm + OFF_PBF, Af, s_g1, isP, lane, v); break;
                    default: scatter_level<1>(sm + OFF_PBF, Af, s_g1, isP, lane, v); break;
                    }
                }
                group_sync(BAR_PREP, NPREP);
                if (ptid < C) {
#pragma unroll
                    for (int w = 0; w < PBAND; ++w)
                        if (ptid - w >= 0)
                            *reinterpret_cast<unsigned short *>(sm + OFF_PBF + sw_elem(8192, ptid, ptid - w)) =
                                bf16_bits(s_pband[ptid * PBAND + w]);
                }
            }
            tc_fence_before();
            group_sync(BAR_PREP, NPREP);

            // ===== 3. T = (I + A)^{-1} =============================================
            // 16x16 diagonal blocks by forward substitution (one column per thread), then
            // recursive doubling: T[16(I+1):, 16I:] = -D_{I+1} A_{I+1,I} D_I for I = 0, 2, and
            // T[32:, :32] = -T2 A21 T1.  fp32 throughout; A rows read four at a time.
            if (ptid < 64) {
                const int I = ptid >> 4, c = ptid & 15;
                float xv[16];
#pragma unroll
                for (int r2 = 0; r2 < 16; ++r2) {
                    float arow[16];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<float4 *>(arow + 4 * q4) =
                            *reinterpret_cast<const float4 *>(Af + (16 * I + r2) * TP + 16 * I + 4 * q4);
                    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < r2; ++s2) {
                        if (s2 & 1) acc1 = fmaf(arow[s2], xv[s2], acc1);
                        else acc0 = fmaf(arow[s2], xv[s2], acc0);
                    }
                    xv[r2] = (r2 < c) ? 0.f : ((r2 == c) ? 1.f : -(acc0 + acc1));
                }
#pragma unroll
                for (int r2 = 0; r2 < 16; ++r2) Tf[(16 * I + r2) * TP + 16 * I + c] = xv[r2];
                for (int r2 = 0; r2 < 16 * I; ++r2) Tf[r2 * TP + 16 * I + c] = 0.f;  // above the block
            } else if (ptid < 64 + C) {   // meanwhile: the next item's gates
                if (nxt.valid) fetch_gates(nxt, ptid - 64, par ^ 1u);
            }
            group_sync(BAR_PREP, NPREP);
            {   // X = A_{I+1,I} D_I for I = 0, 2 (two outputs per thread)
                const int r2 = (ptid >> 4) & 15, c2 = ptid & 15;
                float acc[2] = {0.f, 0.f};
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
#pragma unroll
                    for (int blk = 0; blk < 2; ++blk) {
                        const int I = 2 * blk;
                        const float4 av = *reinterpret_cast<const float4 *>(Af + (16 * I + 16 + r2) * TP + 16 * I + 4 * m4);
                        const float *tcol = Tf + (16 * I + 4 * m4) * TP + 16 * I + c2;
                        acc[blk] = fmaf(av.x, tcol[0], acc[blk]);
                        acc[blk] = fmaf(av.y, tcol[TP], acc[blk]);
                        acc[blk] = fmaf(av.z, tcol[2 * TP], acc[blk]);
                        acc[blk] = fmaf(av.w, tcol[3 * TP], acc[blk]);
                    }
                }
                Xs[ptid] = acc[0];
                Xs[256 + ptid] = acc[1];
            }
            group_sync(BAR_PREP, NPREP);
            {   // T_{I+1,I} = -D_{I+1} X
                const int r2 = (ptid >> 4) & 15, c2 = ptid & 15;
                float acc[2] = {0.f, 0.f};
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
#pragma unroll
                    for (int blk = 0; blk < 2; ++blk) {
                        const int I = 2 * blk;
                        const float4 tv = *reinterpret_cast<const float4 *>(Tf + (16 * I + 16 + r2) * TP + 16 * I + 16 + 4 * m4);
                        const float *xcol = Xs + (blk << 8) + (4 * m4) * 16 + c2;
                        acc[blk] = fmaf(tv.x, xcol[0], acc[blk]);
                        acc[blk] = fmaf(tv.y, xcol[16], acc[blk]);
                        acc[blk] = fmaf(tv.z, xcol[32], acc[blk]);
                        acc[blk] = fmaf(tv.w, xcol[48], acc[blk]);
                    }
                }
                Tf[(16 + r2) * TP + c2] = -acc[0];
                Tf[(48 + r2) * TP + 32 + c2] = -acc[1];
            }
            group_sync(BAR_PREP, NPREP);
            {   // X = A21 T1 (rows r0 + 8k, column c2)
                const int r0 = ptid >> 5, c2 = ptid & 31;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m4 = 0; m4 < 8; ++m4) {
                    const float *tcol = Tf + (4 * m4) * TP + c2;
                    const float t0v = tcol[0], t1v = tcol[TP], t2v = tcol[2 * TP], t3v = tcol[3 * TP];
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const float4 av = *reinterpret_cast<const float4 *>(Af + (32 + r0 + 8 * k4) * TP + 4 * m4);
                        acc[k4] = fmaf(av.x, t0v, acc[k4]);
                        acc[k4] = fmaf(av.y, t1v, acc[k4]);
                        acc[k4] = fmaf(av.z, t2v, acc[k4]);
                        acc[k4] = fmaf(av.w, t3v, acc[k4]);
                    }
                }
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) Xs[(r0 + 8 * k4) * 32 + c2] = acc[k4];
            }
            group_sync(BAR_PREP, NPREP);
            {   // T21 = -T2 X
                const int r0 = ptid >> 5, c2 = ptid & 31;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m4 = 0; m4 < 8; ++m4) {
                    const float *xcol = Xs + (4 * m4) * 32 + c2;
                    const float x0 = xcol[0], x1 = xcol[32], x2 = xcol[64], x3 = xcol[96];
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const float4 tv = *reinterpret_cast<const float4 *>(Tf + (32 + r0 + 8 * k4) * TP + 32 + 4 * m4);
                        acc[k4] = fmaf(tv.x, x0, acc[k4]);
                        acc[k4] = fmaf(tv.y, x1, acc[k4]);
                        acc[k4] = fmaf(tv.z, x2, acc[k4]);
                        acc[k4] = fmaf(tv.w, x3, acc[k4]);
                    }
                }
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) Tf[(32 + r0 + 8 * k4) * TP + c2] = -acc[k4];
            }
            group_sync(BAR_PREP, NPREP);

            // ===== 4. W = T Diag(e) (row operand a~ part);  U'^T = M^T (T Diag(w))^T ==
            // T copies go through one bf16 tile: T Diag(e) for W, then (RDA only, whose two
            // gates differ) T Diag(w) for U' once the W GEMM has read the first copy.
            // Also returns whether row r stays within both bounds of the exact path: its sum of
            // |T_{r,s}| max(|e_s|, |w_s|) and its sum of |A_{r,s}| (the four threads of a row are
            // adjacent lanes).
            auto write_t_copy = [&](const float *gate) {
                const int r = ptid >> 2, kc0 = (ptid & 3) * 2;
                float tsum = 0.f, asum = 0.f;
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    float te[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const int s = (kc0 + q2) * 8 + c;
                        const float t = (s <= r) ? Tf[r * TP + s] : 0.f;
                        te[c] = t * gate[s];
                        tsum += fabsf(t) * fmaxf(fabsf(s_g1[s]), fabsf(s_g2[s]));
                        asum += fabsf(Af[r * TP + s]);   // zero on and above the diagonal
                    }
                    *reinterpret_cast<uint4 *>(sm + OFF_TBF + sw_chunk(8192, r, kc0 + q2)) = pack8(te);
                }
#pragma unroll
                for (int m = 1; m <= 2; m <<= 1) {
                    tsum += __shfl_xor_sync(0xffffffffu, tsum, m);
                    asum += __shfl_xor_sync(0xffffffffu, asum, m);
                }
                return tsum <= EXACT_T_NORM && asum <= EXACT_A_NORM;
            };
            // an ill-conditioned chunk is run token by token by the chain instead (exact path)
            const bool exact = !publish_and(write_t_copy(s_g1));
            // U'^T overwrites TMEM U: the chain must have read the previous chunk's U out
            // (the split kernel leaves U' to the chain kernel and stores T Diag(w) instead)
            if (ch > 0 && !mbar_wait_cycles(bar_ufree, ppar, WAIT_CYCLES)) ok = false;
            if (ptid == 0) {
                tc_fence_after();
                const uint32_t id_w = idesc_bf16(64, 128, false, true);
                const uint32_t id_u = idesc_bf16(128, 64, true, false);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    mma_bf16(tbase + TM_W, dK(sb + OFF_TBF, 8192, kk), dMN(sb + OFF_QA, 16384, kk), id_w, kk > 0);
                    if (same_gates)
                        mma_bf16(tbase + TM_U, dMN(sb + OFF_MT, 8192, kk), dK(sb + OFF_TBF, 8192, kk), id_u, kk > 0);
                }
                mma_commit(bar_pmma);
            }
            wait_pmma();
            if (!same_gates) {
                write_t_copy(s_g2);
                publish();
                if (ptid == 0) {
                    tc_fence_after();
                    const uint32_t id_u = idesc_bf16(128, 64, true, false);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tbase + TM_U, dMN(sb + OFF_MT, 8192, kk), dK(sb + OFF_TBF, 8192, kk), id_u, kk > 0);
                    mma_commit(bar_pmma);
                }
                wait_pmma();
            }
            if (ptid == 0 && nxt.valid) issue_tma_v(nxt);   // v consumed by U'^T = M^T T^T
            // W (M = 64 layout: rows 16q..16q+15 in lanes 0..15 of quarter q) -> rows 0-63 of QA
            {
                const int r = quarter * 16 + (lane & 15);
#pragma unroll
                for (int c32 = 0; c32 < 2; ++c32) {
                    float v[32];
                    tmem_ld32(tbase + lane_base + TM_W + phalf * 64 + c32 * 32, v);
                    tmem_wait_ld();
                    if (lane < 16) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            *reinterpret_cast<uint4 *>(sm + OFF_QA + sw_chunk(16384, r, phalf * 8 + c32 * 4 + q4)) =
                                pack8_neg(v + q4 * 8);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            ok = group_sync_and(BAR_PREP, NPREP, ok);
            if (ptid == 0) {   // chunk ch's operands are ready for the chain
                s_fast[par] = (fast ? META_FAST : 0) | (exact ? META_EXACT : 0);
                mbar_arrive(bar_ready);
            }
            cur = nxt;
        }
        if (!ok) {  // drain TMA still in flight (bounded)
            mbar_wait_cycles(bar_tma, ph_tma, WAIT_CYCLES);
            mbar_wait_cycles(bar_v, ph_v, WAIT_CYCLES);
        }
    }

    // ---- final state (NaN if an internal wait timed out; the failure is also recorded in the
    // device status word, where kda_device_status finds it) -------------------------------------
    __syncthreads();
    tc_fence_after();
    ok = __syncthreads_and(ok) != 0;
    if (!ok && tid == 0) report_device_failure(DEV_WAIT_TIMEOUT);
    if (warp < 4 && a.sf) {
        const size_t soff = ((size_t)n * H + h) * D * D;
        const int jcol = tid;
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
            const int i0 = c32 * 32;
            float s[32];
            tmem_ld32(tbase + lane_base + TM_S + i0, s);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e)
                a.sf[soff + (size_t)(i0 + e) * D + jcol] = ok ? s[e] : __int_as_float(0x7fc00000);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

// ---- split form: the preparation kernel, two items in flight per SM --------
// Preparing one (chunk, head) item is a chain of short, latency-bound phases
// (about 15 K cycles per item with one item per SM, most issue slots idle).
// This kernel overlaps two items on each SM:
//   FRONT (warps 0-7) runs steps 0-2 of item j+1: input preparation, block
//     totals, Gamma_C and the path decision, row operands, Kbar and the band
//     of P, the A/P GEMM(s) and their read-out into A (fp32) and P (bf16);
//   BACK (warps 8-11) runs the rest of item j: the UT transform T (solved in
//     place over its copy of A), the exact-path decision, the T Diag(.)
//     copies, the W GEMM and its read-out into -W'.
// Each group bulk-stores its own part of the item's slot (front: Q', Kbar, P,
// GDN-2's M; back: -W', T Diag(w), the meta block).  GDN-2's v arrives in the
// one M tile; M = w (.) v is stored as soon as it is formed, and the next
// item's v is loaded once that store has read the tile.  Two mbarriers hand items
// over: `full` (front -> back: A, the a~' rows of the row-operand tile, the
// gates, Gamma_C and the path flag of item j are ready) and `taken` (back ->
// front: the back has copied them into its own buffers, so the front may
// rewrite them for item j+1).  Items are decoded four ahead by one back
// thread into a ring in shared memory.  Every element is computed by the same
// arithmetic as in the fused kernel (only the thread that computes it
// differs), so the two forms still give identical bits.
constexpr int PF_FRONT = 256, PF_BACK = 128, PF_NT = PF_FRONT + PF_BACK;
constexpr uint32_t BAR_FRONT = 1, BAR_BACK = 2;
// raw TMA tiles [64][128] bf16 at the fused kernel's offsets (the shared helpers read them there)
constexpr uint32_t P2_RAW_Q = RAW_Q, P2_RAW_K = RAW_K, P2_RAW_A = RAW_A;
constexpr uint32_t P2_KB = 32768;     // Kbar [token][channel], between the k and alpha tiles
constexpr uint32_t P2_QA = 65536;     // [a~'; Q'] 128-row K-major tile (A/P GEMM operand)
constexpr uint32_t P2_AT = 98304;     // back: the a~' rows (2 panels x 64 rows), then -W'
constexpr uint32_t P2_FR = 114688;    // front: band partials | level factors; then A fp32 and P bf16
constexpr uint32_t P2_LA = P2_FR, P2_LB = P2_FR + 32768, P2_AF = P2_FR, P2_PBF = P2_FR + 17408;
constexpr uint32_t P2_TB = 163840;    // back: A, then T in place, fp32 [64][TP]
constexpr uint32_t P2_TBF = 181248;   // back: the 32 x 32 scratch of the T solve, then T Diag(.) bf16
constexpr uint32_t P2_X = P2_TBF;
constexpr uint32_t P2_MT = 189440;    // front, GDN-2: v, then M = w (.) v in place
constexpr uint32_t P2_MISC = 205824;
constexpr uint32_t P2_TOT = P2_MISC;                 // float [8][128] block totals of alpha
constexpr uint32_t P2_PBAND = P2_MISC + 4096;        // float [64][PBAND]
constexpr uint32_t P2_GATES = P2_MISC + 5376;        // float [4][2][64]: gates by item index mod 4
constexpr uint32_t P2_GAMC = P2_MISC + 7424;         // float [2][128]: Gamma_C by item parity
constexpr uint32_t P2_META = P2_MISC + 8448;         // back: Gamma_C fp32 [128], status word, epoch tag
constexpr uint32_t P2_RING = P2_MISC + 8992;         // int [8][8]: decoded items
constexpr uint32_t P2_FLAGS = P2_MISC + 9248;        // int [2] path flags by item parity, [1] abort
constexpr uint32_t P2_BAR = P2_MISC + 9264;          // mbarriers: tma (alpha), v, pmma, wmma, full, taken, qk
constexpr uint32_t P2_TMEM = P2_MISC + 9320;
constexpr uint32_t P2_APART = P2_MISC + 9328;        // float [2][2][64]: |A| half-row sums by item parity
constexpr uint32_t P2_ALLOC = P2_MISC + 10352 + 1024;
static_assert(P2_ALLOC <= 232448, "shared memory budget");
static_assert(P2_FR + 40960 <= P2_TB && P2_LB + 16384 <= P2_TB && P2_PBF + 8192 <= P2_TB, "front region");
static_assert(P2_TB + 64 * TP * 4 <= P2_TBF && P2_TBF + 8192 <= P2_MT && P2_MT + 16384 <= P2_MISC, "back region");
static_assert(((P2_QA | P2_KB | P2_AT | P2_PBF | P2_TBF | P2_MT) & 1023) == 0, "swizzle atoms");
static_assert(RAW_Q + 16384 <= RAW_K && RAW_K + 16384 <= P2_KB && P2_KB + 16384 <= RAW_A &&
              RAW_A + 16384 <= P2_QA && P2_QA + 32768 <= P2_AT && P2_AT + 16384 <= P2_FR, "tile map");
static_assert((P2_META & 15) == 0 && (P2_BAR & 7) == 0, "alignment");
// TMEM columns: front A/P at TM_AP, anchored levels below; back W at TM_W
__device__ __forceinline__ uint32_t tm_lvl_split(int p) { return p == 0 ? 384u : (p == 1 ? 448u : 128u); }

// Next valid item at or after work index w (w += gridDim.x), with the sequence
// found by walking forward from n (items of one CTA come in increasing slot order).
__device__ __forceinline__ Item next_item_walk(const FwdArgs &a, int N, int nwork, int &w, int &n)
{
    for (; w < nwork; w += gridDim.x) {
        Item it;
        it.h = w % a.H;
        it.slot = w / a.H;
        while (n + 1 < N && slot_base(a, n + 1) <= it.slot) ++n;
        it.n = n;
        it.row0 = seq_row0(a, n);
        it.len = seq_len(a, n);
        it.c = it.slot - slot_base(a, n);
        it.valid = it.c >= 0 && it.c * C < it.len;
        if (it.valid) return it;
    }
    Item none{};
    none.valid = false;
    return none;
}
__device__ __forceinline__ void ring_put(int *ring, int k, const Item &it)
{
    int *d = ring + (k & 7) * 8;
    d[0] = it.n; d[1] = it.h; d[2] = it.c; d[3] = it.row0; d[4] = it.len; d[5] = it.slot; d[6] = it.valid ? 1 : 0;
}
__device__ __forceinline__ Item ring_get(const int *ring, int k)
{
    const int *d = ring + (k & 7) * 8;
    Item it;
    it.n = d[0]; it.h = d[1]; it.c = d[2]; it.row0 = d[3]; it.len = d[4]; it.slot = d[5]; it.valid = d[6] != 0;
    return it;
}

template <bool PREP>
__global__ void __launch_bounds__(PF_NT, 1) chunk_prep_kernel(const __grid_constant__ ChunkParams P)
{
    // the chain kernel may be scheduled now: it sets itself up on SMs this grid leaves and waits
    // for this grid's completion before it reads a slot
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);
    const FwdArgs &a = P.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;
    const int H = a.H;
    const int N = a.cu_seqlens ? a.num_seqs : a.B;
    const int nwork = P.nslots * H;
    float *s_tot = reinterpret_cast<float *>(sm + P2_TOT);
    float *s_pband = reinterpret_cast<float *>(sm + P2_PBAND);
    float *s_gates = reinterpret_cast<float *>(sm + P2_GATES);
    float *s_gamc = reinterpret_cast<float *>(sm + P2_GAMC);
    int *s_meta = reinterpret_cast<int *>(sm + P2_META);
    int *s_ring = reinterpret_cast<int *>(sm + P2_RING);
    int *s_flags = reinterpret_cast<int *>(sm + P2_FLAGS);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + P2_BAR);
    uint64_t *bar_tma = bars + 0, *bar_v = bars + 1, *bar_pmma = bars + 2, *bar_wmma = bars + 3;
    uint64_t *bar_full = bars + 4, *bar_taken = bars + 5, *bar_qk = bars + 6;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + P2_TMEM);
    const __nv_bfloat16 *g1p = (const __nv_bfloat16 *)a.g1, *g2p = (const __nv_bfloat16 *)a.g2;
    const bool gdn2 = a.variant == GDN2;
    const bool same_gates = a.variant != RDA;
    const bool logits = PREP && (a.prep & PREP_LOGITS) != 0, l2k = PREP && (a.prep & PREP_L2NORM_K) != 0;
    const bool ext = a.ext != 0;
    // the item decoder (one back thread) keeps its cursor across the whole kernel
    const bool decoder = tid == PF_FRONT + 64;
    int wdec = blockIdx.x, ndec = 0;

    if (warp == 0) tmem_alloc(s_tmem, 512);
    if (tid == 0) {
        for (int i = 0; i < 7; ++i) mbar_init(bars + i, 1);
        s_flags[2] = 0;   // abort
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (decoder) {   // the first four items
        for (int k = 0; k < 4; ++k) {
            ring_put(s_ring, k, next_item_walk(a, N, nwork, wdec, ndec));
            wdec += gridDim.x;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    bool ok = true;

    if (tid < PF_FRONT) {
        // =====================================================================
        // FRONT: steps 0-2 of each item
        // =====================================================================
        const int ptid = tid, pw = warp;
        const int phalf = pw >> 2;
        const int jrow = quarter * 32 + lane;
        const int tg = ptid >> 5, cq = ptid & 31;
        uint32_t ph_tma = 0, ph_qk = 0, ph_v = 0, ph_pmma = 0, ph_taken = 0;
        float *Af = reinterpret_cast<float *>(sm + P2_AF);
        float *s_apart = reinterpret_cast<float *>(sm + P2_APART);
        // alpha first, on its own barrier: steps 0-1a need alpha only (and k, when keys are
        // normalised in place), so q and k may still be in flight while they run
        auto issue_tma = [&](const Item &it) {
            const int g = it.row0 + it.c * C;
            mbar_expect_tx(bar_tma, 16384);
            tma_load_3d(sm + P2_RAW_A, &P.ta, bar_tma, 0, it.h, g);
            mbar_expect_tx(bar_qk, 2 * 16384);
            tma_load_3d(sm + P2_RAW_Q, &P.tq, bar_qk, 0, it.h, g);
            tma_load_3d(sm + P2_RAW_K, &P.tk, bar_qk, 0, it.h, g);
        };
        auto wait_qk = [&]() {
            if (!mbar_wait_cycles(bar_qk, ph_qk, WAIT_CYCLES)) ok = false;
            ph_qk ^= 1;
        };
        auto issue_tma_v = [&](const Item &it) {   // GDN-2: v into the M tile
            const int g = it.row0 + it.c * C;
            mbar_expect_tx(bar_v, 16384);
            tma_load_3d(sm + P2_MT, &P.tv, bar_v, 0, it.h, g);
            tma_load_3d(sm + P2_MT + 8192, &P.tv, bar_v, 64, it.h, g);
        };
        auto wait_pmma = [&]() {
            if (!mbar_wait_cycles(bar_pmma, ph_pmma, WAIT_CYCLES)) ok = false;
            ph_pmma ^= 1;
            tc_fence_after();
        };
        auto publish = [&]() {
            fence_async_smem();
            tc_fence_before();
            group_sync(BAR_FRONT, PF_FRONT);
        };
        auto gates_of = [&](int k) { return s_gates + (k & 3) * 128; };   // g1 [64], then g2 [64]
        // scalar gates of row r of an item: loaded early (raw bf16 bits), stored later, so that
        // the global-load latency is not on any barrier's critical path
        auto load_gates = [&](const Item &it, int r, uint32_t &ge, uint32_t &gw) {
            const int nv = min(C, it.len - it.c * C);
            const size_t tok = ((size_t)it.row0 + it.c * C + r) * H + it.h;
            const bool v = it.valid && r < nv;
            const unsigned short *g1u = reinterpret_cast<const unsigned short *>(g1p);
            const unsigned short *g2u = reinterpret_cast<const unsigned short *>(g2p);
            if (gdn2) { ge = v ? 0x3F80u : 0u; gw = ge; }   // GDN-2 keeps its gates channel-wise: 1 here
            else {
                ge = v ? (uint32_t)g1u[tok] : 0u;
                gw = v ? (uint32_t)(a.variant == KDA ? g1u[tok] : g2u[tok]) : 0u;
            }
        };
        auto store_gates = [&](int r, uint32_t ge, uint32_t gw, bool valid_row, float *dst) {
            float fe = __uint_as_float(ge << 16), fw = __uint_as_float(gw << 16);
            if (logits && !gdn2 && valid_row) {
                fe = round_bf16(prep_gate(fe, ext));
                fw = round_bf16(prep_gate(fw, ext));
            }
            dst[r] = fe;
            dst[64 + r] = fw;
        };
        auto row_valid = [&](const Item &it, int r) { return it.valid && r < min(C, it.len - it.c * C); };

        Item cur = ring_get(s_ring, 0);
        if (cur.valid && ptid == 0) {
            issue_tma(cur);
            if (gdn2) issue_tma_v(cur);
        }
        if (ptid < C && cur.valid) {
            uint32_t ge, gw;
            load_gates(cur, ptid, ge, gw);
            store_gates(ptid, ge, gw, row_valid(cur, ptid), gates_of(0));
        }
        int j = 0;
        for (; cur.valid && ok; ++j) {
            const uint32_t par = j & 1;
            const Item nxt = ring_get(s_ring, j + 1);
            const int h = cur.h;
            const int nvalid = min(C, cur.len - cur.c * C);
            const size_t rowbase = (size_t)cur.row0 + cur.c * C;
            float *const s_g1 = gates_of(j);
            const ChunkCtx x{sm,   s_tot, s_g1,  g1p,   rowbase, H,     h,     nvalid,
                             gdn2, logits, ext, P2_QA, P2_KB,   P2_LA, P2_LB};
            float *gamc = s_gamc + par * 128;
            uint8_t *slot = P.ws + ((size_t)cur.slot * H + h) * SLOT_BYTES;
            // the next item's gates (threads 64..127) and, for GDN-2, this item's write vector w
            // (every thread: its 8 rows x 4 channels) are put in flight first
            uint32_t nge = 0, ngw = 0;
            if (ptid >= 64 && ptid < 64 + C) load_gates(nxt, ptid - 64, nge, ngw);
            uint2 wraw[8], braw[8];   // GDN-2: write and erase vectors of the thread's rows
            if (gdn2) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = tg * 8 + i;
                    const size_t off = ((rowbase + r) * H + h) * D + cq * 4;
                    wraw[i] = r < nvalid ? *reinterpret_cast<const uint2 *>(g2p + off) : make_uint2(0u, 0u);
                }
            }

            if (!mbar_wait_cycles(bar_tma, ph_tma, WAIT_CYCLES)) ok = false;
            ph_tma ^= 1;
            if (PREP && l2k) wait_qk();   // pass 0 rewrites k
            if (gdn2) {
                if (!mbar_wait_cycles(bar_v, ph_v, WAIT_CYCLES)) ok = false;
                ph_v ^= 1;
            }
            group_sync(BAR_FRONT, PF_FRONT);

            // ===== 0. input preparation, in place in the raw tiles
            if (PREP && logits) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint2 *pa = reinterpret_cast<uint2 *>(sm + P2_RAW_A + (tg * 8 + i) * 256 + cq * 8);
                    float al[4];
                    unpack4(*pa, al);
#pragma unroll
                    for (int c = 0; c < 4; ++c) al[c] = prep_alpha(al[c], ext);
                    *pa = pack4(al);
                }
            }
            if (PREP && l2k) {
                float ss[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float kv[4];
                    unpack4(raw_quad(sm, P2_RAW_K, tg * 8 + i, cq), kv);
                    ss[i] = kv[0] * kv[0] + kv[1] * kv[1] + kv[2] * kv[2] + kv[3] * kv[3];
                }
                const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float send = b4 ? ss[i] : ss[i + 4];
                    ss[i] = (b4 ? ss[i + 4] : ss[i]) + __shfl_xor_sync(0xffffffffu, send, 16);
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float send = b3 ? ss[i] : ss[i + 2];
                    ss[i] = (b3 ? ss[i + 2] : ss[i]) + __shfl_xor_sync(0xffffffffu, send, 8);
                }
                {
                    const float send = b2 ? ss[0] : ss[1];
                    ss[0] = (b2 ? ss[1] : ss[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
                }
                ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], 2);
                ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], 1);
                const float sc = prep_kscale(ss[0]);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float sci = __shfl_sync(0xffffffffu, sc, ((i & 4) ? 16 : 0) + ((i & 2) ? 8 : 0) + ((i & 1) ? 4 : 0));
                    uint2 *pk = reinterpret_cast<uint2 *>(sm + P2_RAW_K + (tg * 8 + i) * 256 + cq * 8);
                    float kv[4];
                    unpack4(*pk, kv);
#pragma unroll
                    for (int c = 0; c < 4; ++c) kv[c] *= sci;
                    *pk = pack4(kv);
                }
            }

            // ===== 1a. block totals of alpha (and range check) | GDN-2: M = w (.) v
            bool in_range = true;
            {
                float tot[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = tg * 8 + i;
                    if (r < nvalid) {
                        float al[4];
                        unpack4(raw_quad(sm, P2_RAW_A, r, cq), al);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            tot[c] *= al[c];
                            in_range = in_range && (fabsf(al[c]) <= 1.f);
                        }
                    }
                }
                *reinterpret_cast<float4 *>(s_tot + tg * 128 + cq * 4) = make_float4(tot[0], tot[1], tot[2], tot[3]);
            }
            if (gdn2) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = tg * 8 + i;
                    uint2 *pv = reinterpret_cast<uint2 *>(sm + P2_MT + sw_half(8192, r, cq));
                    float mv[4], vv[4], wv[4];
                    unpack4(*pv, vv);
                    if (r < nvalid) {
                        unpack4(wraw[i], wv);
#pragma unroll
                        for (int c = 0; c < 4; ++c) mv[c] = (logits ? round_bf16(prep_gate(wv[c], ext)) : wv[c]) * vv[c];
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c) mv[c] = 0.f;
                    }
                    *pv = pack4(mv);
                }
            }
            if (gdn2) {   // the erase vectors, read by the row sweep (w is consumed: its registers are free)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = tg * 8 + i;
                    braw[i] = r < nvalid ? *reinterpret_cast<const uint2 *>(g1p + ((rowbase + r) * H + h) * D + cq * 4)
                                         : make_uint2(0u, 0u);
                }
            }
            if (lane == 0) bulk_wait_read();   // this group's stores of the previous item have read their tiles
            fence_async_smem();
            in_range = group_sync_and(BAR_FRONT, PF_FRONT, in_range);
            if (gdn2 && ptid == 128 && ok) {   // M is final: to the slot now; the next v may then follow
                bulk_store(slot + SL_M, sm + P2_MT, 16384);
                bulk_commit();
            }

            // ===== Gamma_C and the path decision; meanwhile the next item's gates
            bool gam_ok = true;
            if (ptid < 32) {
                float gc[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    float t4[4];
                    load_tot4(s_tot, g, ptid, t4);
#pragma unroll
                    for (int c = 0; c < 4; ++c) gc[c] *= t4[c];
                }
                *reinterpret_cast<float4 *>(gamc + ptid * 4) = make_float4(gc[0], gc[1], gc[2], gc[3]);
#pragma unroll
                for (int c = 0; c < 4; ++c) gam_ok = gam_ok && (fabsf(gc[c]) >= FAST_MIN_GAMMA);
            } else if (ptid >= 64 && ptid < 64 + C) {
                store_gates(ptid - 64, nge, ngw, row_valid(nxt, ptid - 64), gates_of(j + 1));
            }
            const bool fast = group_sync_and(BAR_FRONT, PF_FRONT, gam_ok) && in_range;

            // the back must have taken the previous item's A, a~' rows, gates and Gamma_C
            if (j > 0) {
                if (!mbar_wait_cycles(bar_taken, ph_taken, WAIT_CYCLES)) ok = false;
                ph_taken ^= 1;
            }
            if (!(PREP && l2k)) wait_qk();   // q and k, read from here on

            // ===== 1b. row operands, Kbar and the exact band of P
            if (fast) {
                float *band_part = reinterpret_cast<float *>(sm + P2_FR);
                if (nvalid == C) {
                    if (gdn2) fast_rows<true, true, 8, true>(x, s_tot, gamc, band_part, tg, cq, lane, braw);
                    else fast_rows<true, false, 4>(x, s_tot, gamc, band_part, tg, cq, lane);
                } else {
                    fast_rows<false, true, 1>(x, s_tot, gamc, band_part, tg, cq, lane);
                }
            } else {
                {
                    float pre[4] = {1.f, 1.f, 1.f, 1.f}, suf[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        if (g == tg) continue;
                        float t4[4];
                        load_tot4(s_tot, g, cq, t4);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            if (g < tg) pre[c] *= t4[c];
                            else suf[c] *= t4[c];
                        }
                    }
                    float sc[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) sc[c] = pre[c];
#pragma unroll 2
                    for (int i = 0; i < 8; ++i) {
                        const int r = tg * 8 + i;
                        const bool v = r < nvalid;
                        float al[4], kv[4], qv[4], e[4], oa[4], oq[4];
                        unpack4(raw_quad(sm, P2_RAW_A, r, cq), al);
                        unpack4(raw_quad(sm, P2_RAW_K, r, cq), kv);
                        unpack4(raw_quad(sm, P2_RAW_Q, r, cq), qv);
                        erase_gate4(x, r, cq, e);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            sc[c] *= v ? al[c] : 1.f;
                            oa[c] = v ? sc[c] * (e[c] * kv[c]) : 0.f;
                            oq[c] = v ? sc[c] * qv[c] : 0.f;
                        }
                        *reinterpret_cast<uint2 *>(sm + P2_QA + sw_half(16384, r, cq)) = pack4(oa);
                        *reinterpret_cast<uint2 *>(sm + P2_QA + sw_half(16384, 64 + r, cq)) = pack4(oq);
                    }
                    float sx[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) sx[c] = suf[c];
#pragma unroll 2
                    for (int i = 7; i >= 0; --i) {
                        const int r = tg * 8 + i;
                        const bool v = r < nvalid;
                        float al[4], kv[4], kb[4];
                        unpack4(raw_quad(sm, P2_RAW_A, r, cq), al);
                        unpack4(raw_quad(sm, P2_RAW_K, r, cq), kv);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            kb[c] = v ? sx[c] * kv[c] : 0.f;
                            sx[c] *= v ? al[c] : 1.f;
                        }
                        *reinterpret_cast<uint2 *>(sm + P2_KB + sw_half(8192, r, cq)) = pack4(kb);
                    }
                }
                {   // exact band of P from the bf16 inputs (four threads per row)
                    const int r = ptid >> 2, c4 = ptid & 3;
                    float acc[PBAND];
#pragma unroll
                    for (int w = 0; w < PBAND; ++w) acc[w] = 0.f;
#pragma unroll 1
                    for (int jj = 0; jj < 4; ++jj) {
                        const int cgx = c4 * 4 + ((jj + r) & 3);
                        float hv[8];
                        unpack8(raw_row(sm, P2_RAW_Q, r, cgx), hv);
#pragma unroll
                        for (int w = 0; w < PBAND; ++w) {
                            float kv[8];
                            unpack8(raw_row(sm, P2_RAW_K, max(r - w, 0), cgx), kv);
#pragma unroll
                            for (int c = 0; c < 8; ++c) acc[w] = fmaf(hv[c], kv[c], acc[w]);
                            if (w + 1 < PBAND) {
                                float av[8];
                                unpack8(raw_row(sm, P2_RAW_A, max(r - w, 0), cgx), av);
#pragma unroll
                                for (int c = 0; c < 8; ++c) hv[c] *= av[c];
                            }
                        }
                    }
#pragma unroll
                    for (int w = 0; w < PBAND; ++w) {
                        float t = acc[w] + __shfl_xor_sync(0xffffffffu, acc[w], 1);
                        t += __shfl_xor_sync(0xffffffffu, t, 2);
                        if (c4 == 0) s_pband[r * PBAND + w] = (r < nvalid && r - w >= 0) ? t : 0.f;
                    }
                }
            }
            fence_async_smem();   // Q' and Kbar are final: to the slot now, read by the bulk copies
            group_sync(BAR_FRONT, PF_FRONT);
            if (ok && lane == 0 && (pw == 5 || pw == 6 || pw == 7)) {
                if (pw == 5) bulk_store(slot + SL_QA + 8192, sm + P2_QA + 8192, 8192);          // Q', panel 0
                else if (pw == 6) bulk_store(slot + SL_QA + 24576, sm + P2_QA + 24576, 8192);   // Q', panel 1
                else bulk_store(slot + SL_KB, sm + P2_KB, 16384);
                bulk_commit();
            }
            if (gdn2 && ptid == 128 && nxt.valid) {   // the M store has read its tile: the next item's v
                bulk_wait_read();
                issue_tma_v(nxt);
            }
            // fast path: nothing reads the raw tiles after step 1b -- the next item's may come in now
            if (fast && ptid == 0 && nxt.valid) issue_tma(nxt);

            // ===== 2. A and P
            if (fast) {
                publish();
                if (ptid == 0) {
                    tc_fence_after();
                    const uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tbase + TM_AP, dK(sb + P2_QA, 16384, kk), dK(sb + P2_KB, 8192, kk), idesc, kk > 0);
                    mma_commit(bar_pmma);
                }
                band_reduce(reinterpret_cast<const float *>(sm + P2_FR), s_pband, nvalid, ptid, PF_FRONT);
                group_sync(BAR_FRONT, PF_FRONT);
                wait_pmma();
                float v[32];
                tmem_ld32(tbase + lane_base + TM_AP + phalf * 32, v);
                tmem_wait_ld();
                const int rr = jrow & 63;
                if (jrow < 64) {
                    const float er = s_g1[rr];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int s = phalf * 32 + c;
                        v[c] = (s < rr) ? v[c] * er : 0.f;
                    }
                    // |A| over this half row, as two 16-column sums (the order the fused kernel adds them in)
                    float g0 = 0.f, g1s = 0.f;
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        g0 += fabsf(v[c]);
                        g1s += fabsf(v[16 + c]);
                    }
                    s_apart[(par * 2 + phalf) * 64 + rr] = g0 + g1s;
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        *reinterpret_cast<float4 *>(Af + rr * TP + phalf * 32 + 4 * q4) =
                            make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int s = phalf * 32 + c;
                        const int w = rr - s;
                        v[c] = (w >= PBAND) ? v[c] : ((w >= 0) ? s_pband[rr * PBAND + w] : 0.f);
                    }
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4 *>(sm + P2_PBF + sw_chunk(8192, rr, phalf * 4 + q4)) = pack8(v + q4 * 8);
                }
            } else {
                for (int p = 0; p < 3; ++p) {
#pragma unroll 1
                    for (int sl = 0; sl < 2; ++sl) {
                        switch (2 * p + 1 + sl) {
                        case 1: build_level<32>(x, sl, tg, cq); break;
                        case 2: build_level<16>(x, sl, tg, cq); break;
                        case 3: build_level<8>(x, sl, tg, cq); break;
                        case 4: build_level<4>(x, sl, tg, cq); break;
                        case 5: build_level<2>(x, sl, tg, cq); break;
                        default: build_level<1>(x, sl, tg, cq); break;
                        }
                    }
                    publish();
                    if (ptid == 0) {
                        tc_fence_after();
                        const uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_bf16(tbase + tm_lvl_split(p), dK(sb + P2_LA, 16384, kk), dK(sb + P2_LB, 8192, kk),
                                     idesc, kk > 0);
                        mma_commit(bar_pmma);
                    }
                    wait_pmma();
                }
                if (ptid == 0 && nxt.valid) issue_tma(nxt);   // raw tiles consumed
                for (int e = ptid; e < 64 * TP; e += PF_FRONT) Af[e] = 0.f;
                for (int e = ptid; e < 512; e += PF_FRONT)
                    *reinterpret_cast<uint4 *>(sm + P2_PBF + e * 16) = make_uint4(0, 0, 0, 0);
                group_sync(BAR_FRONT, PF_FRONT);
                for (int p = phalf; p < 3; p += 2) {
                    const int lvl = 2 * p + 1 + (quarter & 1);
                    const bool isP = quarter >= 2;
                    float v[32];
                    tmem_ld32(tbase + lane_base + tm_lvl_split(p) + (quarter & 1) * 32, v);
                    tmem_wait_ld();
                    uint8_t *pbf = sm + P2_PBF;
                    switch (lvl) {
                    case 1: scatter_level<32>(pbf, Af, s_g1, isP, lane, v); break;
                    case 2: scatter_level<16>(pbf, Af, s_g1, isP, lane, v); break;
                    case 3: scatter_level<8>(pbf, Af, s_g1, isP, lane, v); break;
                    case 4: scatter_level<4>(pbf, Af, s_g1, isP, lane, v); break;
                    case 5: scatter_level<2>(pbf, Af, s_g1, isP, lane, v); break;
                    default: scatter_level<1>(pbf, Af, s_g1, isP, lane, v); break;
                    }
                }
                group_sync(BAR_FRONT, PF_FRONT);
                if (ptid < C) {
#pragma unroll
                    for (int w = 0; w < PBAND; ++w)
                        if (ptid - w >= 0)
                            *reinterpret_cast<unsigned short *>(sm + P2_PBF + sw_elem(8192, ptid, ptid - w)) =
                                bf16_bits(s_pband[ptid * PBAND + w]);
                }
                {   // |A| half-row sums: four threads per row, 16 columns each, adjacent lanes paired
                    const int r = ptid >> 2, m = ptid & 3;
                    float g = 0.f;
#pragma unroll
                    for (int c = 0; c < 16; ++c) g += fabsf(Af[r * TP + 16 * m + c]);
                    g += __shfl_xor_sync(0xffffffffu, g, 1);
                    if (!(m & 1)) s_apart[(par * 2 + (m >> 1)) * 64 + r] = g;
                }
            }
            fence_async_smem();
            tc_fence_before();
            ok = group_sync_and(BAR_FRONT, PF_FRONT, ok);

            // ===== P to the slot (Q', Kbar and GDN-2's M left earlier); then hand the item over
            if (ok && lane == 0 && pw == 3) {
                bulk_store(slot + SL_PBF, sm + P2_PBF, 8192);
                bulk_commit();
            }
            if (ptid == 0) {
                s_flags[par] = fast ? META_FAST : 0;
                mbar_arrive(bar_full);
            }
            cur = nxt;
        }
        // no item j for the back: the ring says so (or the abort flag, after a failure).  The back
        // must have waited for item j-1 first: `full` may run at most one phase ahead of its
        // waits (a parity wait cannot tell two completed phases from none)
        if (j > 0) {
            if (!mbar_wait_cycles(bar_taken, ph_taken, WAIT_CYCLES)) ok = false;
            ph_taken ^= 1;
        }
        if (ptid == 0) {
            if (!ok) s_flags[2] = 1;
            mbar_arrive(bar_full);
        }
        if (!ok) {   // drain TMA still in flight (bounded)
            mbar_wait_cycles(bar_tma, ph_tma, WAIT_CYCLES);
            mbar_wait_cycles(bar_qk, ph_qk, WAIT_CYCLES);
            if (gdn2) mbar_wait_cycles(bar_v, ph_v, WAIT_CYCLES);
        }
        if (lane == 0) bulk_wait_all();
    } else {
        // =====================================================================
        // BACK: T, the exact-path decision, W, and the rest of the slot
        // =====================================================================
        const int btid = tid - PF_FRONT, bw = warp - PF_FRONT / 32;
        uint32_t ph_full = 0, ph_wmma = 0;
        float *TB = reinterpret_cast<float *>(sm + P2_TB);
        float *Xs = reinterpret_cast<float *>(sm + P2_X);
        auto publish_and = [&](bool pred) {
            fence_async_smem();
            tc_fence_before();
            return group_sync_and(BAR_BACK, PF_BACK, pred);
        };
        // T Diag(gate) -> TBF (bf16, K-major); two passes cover the 64 rows with the fused
        // kernel's thread mapping (row ptid'/4, 16 columns).  Returns whether both of this
        // thread's rows stay within the exact path's |T| bound.
        auto write_t_copy = [&](const float *gate, const float *s_bg1, const float *s_bg2) {
            bool well = true;
#pragma unroll 1
            for (int pp = 0; pp < 2; ++pp) {
                const int pt = btid + PF_BACK * pp;
                const int r = pt >> 2, kc0 = (pt & 3) * 2;
                float tsum = 0.f;
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    float te[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const int s = (kc0 + q2) * 8 + c;
                        const float t = (s <= r) ? TB[r * TP + s] : 0.f;
                        te[c] = t * gate[s];
                        tsum += fabsf(t) * fmaxf(fabsf(s_bg1[s]), fabsf(s_bg2[s]));
                    }
                    *reinterpret_cast<uint4 *>(sm + P2_TBF + sw_chunk(8192, r, kc0 + q2)) = pack8(te);
                }
#pragma unroll
                for (int m = 1; m <= 2; m <<= 1) tsum += __shfl_xor_sync(0xffffffffu, tsum, m);
                well = well && tsum <= EXACT_T_NORM;
            }
            return well;
        };

        for (int j = 0; ok; ++j) {
            if (!mbar_wait_cycles(bar_full, ph_full, WAIT_CYCLES)) {
                ok = false;
                break;
            }
            ph_full ^= 1;
            const Item it = ring_get(s_ring, j);
            if (!it.valid || s_flags[2]) break;
            const uint32_t par = j & 1;
            if (lane == 0) bulk_wait_read();   // this group's stores of item j-1 have read AT, TBF, meta
            group_sync(BAR_BACK, PF_BACK);
            // ---- take item j: A, the a~' rows, gates, Gamma_C, path flag
            {
                // all loads of a batch are issued before its stores
                constexpr int NA = 64 * TP / 4;   // 16-byte pieces of A (1088 = 8.5 per thread)
                const uint4 *src = reinterpret_cast<const uint4 *>(sm + P2_AF);
                uint4 *dst = reinterpret_cast<uint4 *>(sm + P2_TB);
                uint4 buf[9];
#pragma unroll
                for (int i = 0; i < 9; ++i) {
                    const int e = btid + PF_BACK * i;
                    if (e < NA) buf[i] = src[e];
                }
#pragma unroll
                for (int i = 0; i < 9; ++i) {
                    const int e = btid + PF_BACK * i;
                    if (e < NA) dst[e] = buf[i];
                }
                uint4 qb[8];   // the a~' rows: 2 panels x 512 pieces
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int e = btid + PF_BACK * i, pnl = e >> 9;
                    qb[i] = reinterpret_cast<const uint4 *>(sm + P2_QA + pnl * 16384)[e & 511];
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int e = btid + PF_BACK * i, pnl = e >> 9;
                    reinterpret_cast<uint4 *>(sm + P2_AT + pnl * 8192)[e & 511] = qb[i];
                }
                reinterpret_cast<float *>(s_meta)[btid] = s_gamc[par * 128 + btid];
            }
            const bool fast = s_flags[par] != 0;
            // the gates stay where the front put them: their buffer (item index mod 4) is not
            // rewritten before this item is done
            const float *s_bg1 = s_gates + (j & 3) * 128, *s_bg2 = s_bg1 + 64;
            group_sync(BAR_BACK, PF_BACK);
            if (btid == 0) mbar_arrive(bar_taken);
            uint8_t *slot = P.ws + ((size_t)it.slot * H + it.h) * SLOT_BYTES;

            // ---- |A| row sums (the exact path's second bound), from the front's half-row sums
            bool well_a = true;
            {
                const float *ap = reinterpret_cast<const float *>(sm + P2_APART) + par * 128;
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {
                    const int r = (btid + PF_BACK * pp) >> 2;
                    well_a = well_a && (ap[r] + ap[64 + r]) <= EXACT_A_NORM;
                }
            }

            // ===== 3. T = (I + A)^{-1}, in place: 16x16 diagonal blocks, then recursive doubling
            {
                float xv[16];
                const int I = btid >> 4, c = btid & 15;
                if (btid < 64) {
#pragma unroll
                    for (int r2 = 0; r2 < 16; ++r2) {
                        float arow[16];
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            *reinterpret_cast<float4 *>(arow + 4 * q4) =
                                *reinterpret_cast<const float4 *>(TB + (16 * I + r2) * TP + 16 * I + 4 * q4);
                        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                        for (int s2 = 0; s2 < r2; ++s2) {
                            if (s2 & 1) acc1 = fmaf(arow[s2], xv[s2], acc1);
                            else acc0 = fmaf(arow[s2], xv[s2], acc0);
                        }
                        xv[r2] = (r2 < c) ? 0.f : ((r2 == c) ? 1.f : -(acc0 + acc1));
                    }
                } else if (decoder) {   // meanwhile: the item four ahead
                    ring_put(s_ring, j + 4, next_item_walk(a, N, nwork, wdec, ndec));
                    wdec += gridDim.x;
                }
                group_sync(BAR_BACK, PF_BACK);   // every read of the diagonal blocks of A is done
                if (btid < 64) {
#pragma unroll
                    for (int r2 = 0; r2 < 16; ++r2) TB[(16 * I + r2) * TP + 16 * I + c] = xv[r2];
                }
            }
            group_sync(BAR_BACK, PF_BACK);
            // The merges give every output the fused kernel's multiply-add chain (same terms,
            // same order); a thread owns two adjacent columns and runs both chains at once on
            // the packed fp32 pipe.
            {   // X = A_{I+1,I} D_I for I = 0, 2: thread (row r2, columns c2, c2 + 1) of both blocks
                const int r2 = btid >> 3, c2 = (btid & 7) * 2;
                float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
#pragma unroll
                    for (int blk = 0; blk < 2; ++blk) {
                        const int I = 2 * blk;
                        const float4 av = *reinterpret_cast<const float4 *>(TB + (16 * I + 16 + r2) * TP + 16 * I + 4 * m4);
                        const float *tcol = TB + (16 * I + 4 * m4) * TP + 16 * I + c2;
                        acc[blk] = __ffma2_rn(make_float2(av.x, av.x), *reinterpret_cast<const float2 *>(tcol), acc[blk]);
                        acc[blk] = __ffma2_rn(make_float2(av.y, av.y), *reinterpret_cast<const float2 *>(tcol + TP), acc[blk]);
                        acc[blk] = __ffma2_rn(make_float2(av.z, av.z), *reinterpret_cast<const float2 *>(tcol + 2 * TP), acc[blk]);
                        acc[blk] = __ffma2_rn(make_float2(av.w, av.w), *reinterpret_cast<const float2 *>(tcol + 3 * TP), acc[blk]);
                    }
                }
                *reinterpret_cast<float2 *>(Xs + r2 * 16 + c2) = acc[0];
                *reinterpret_cast<float2 *>(Xs + 256 + r2 * 16 + c2) = acc[1];
            }
            group_sync(BAR_BACK, PF_BACK);
            {   // T_{I+1,I} = -D_{I+1} X, over A_{I+1,I}
                const int r2 = btid >> 3, c2 = (btid & 7) * 2;
                float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
#pragma unroll
                    for (int blk = 0; blk < 2; ++blk) {
                        const int I = 2 * blk;
                        const float4 tv = *reinterpret_cast<const float4 *>(TB + (16 * I + 16 + r2) * TP + 16 * I + 16 + 4 * m4);
                        const float *xcol = Xs + (blk << 8) + (4 * m4) * 16 + c2;
                        acc[blk] = __ffma2_rn(make_float2(tv.x, tv.x), *reinterpret_cast<const float2 *>(xcol), acc[blk]);
                        acc[blk] = __ffma2_rn(make_float2(tv.y, tv.y), *reinterpret_cast<const float2 *>(xcol + 16), acc[blk]);
                        acc[blk] = __ffma2_rn(make_float2(tv.z, tv.z), *reinterpret_cast<const float2 *>(xcol + 32), acc[blk]);
                        acc[blk] = __ffma2_rn(make_float2(tv.w, tv.w), *reinterpret_cast<const float2 *>(xcol + 48), acc[blk]);
                    }
                }
                *reinterpret_cast<float2 *>(TB + (16 + r2) * TP + c2) = make_float2(-acc[0].x, -acc[0].y);
                *reinterpret_cast<float2 *>(TB + (48 + r2) * TP + 32 + c2) = make_float2(-acc[1].x, -acc[1].y);
            }
            group_sync(BAR_BACK, PF_BACK);
            // level 32: warp bw takes rows bw + 4i, half-warp h the i in [4h, 4h + 4), lane pair
            // columns c2, c2 + 1; a column pair of T1 (or X) serves the thread's four rows
            const int hh = lane >> 4, cp = (lane & 15) * 2;
            {   // X = A21 T1
                float2 acc[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
                for (int m4 = 0; m4 < 8; ++m4) {
                    const float *tcol = TB + (4 * m4) * TP + cp;
                    const float2 t0 = *reinterpret_cast<const float2 *>(tcol);
                    const float2 t1 = *reinterpret_cast<const float2 *>(tcol + TP);
                    const float2 t2 = *reinterpret_cast<const float2 *>(tcol + 2 * TP);
                    const float2 t3 = *reinterpret_cast<const float2 *>(tcol + 3 * TP);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int row = bw + 4 * (4 * hh + i);
                        const float4 av = *reinterpret_cast<const float4 *>(TB + (32 + row) * TP + 4 * m4);
                        acc[i] = __ffma2_rn(make_float2(av.x, av.x), t0, acc[i]);
                        acc[i] = __ffma2_rn(make_float2(av.y, av.y), t1, acc[i]);
                        acc[i] = __ffma2_rn(make_float2(av.z, av.z), t2, acc[i]);
                        acc[i] = __ffma2_rn(make_float2(av.w, av.w), t3, acc[i]);
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) *reinterpret_cast<float2 *>(Xs + (bw + 4 * (4 * hh + i)) * 32 + cp) = acc[i];
            }
            group_sync(BAR_BACK, PF_BACK);
            {   // T21 = -T2 X, over A21 (read by the previous phase); same split
                float2 acc[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
                for (int m4 = 0; m4 < 8; ++m4) {
                    const float *xcol = Xs + (4 * m4) * 32 + cp;
                    const float2 x0 = *reinterpret_cast<const float2 *>(xcol);
                    const float2 x1 = *reinterpret_cast<const float2 *>(xcol + 32);
                    const float2 x2 = *reinterpret_cast<const float2 *>(xcol + 64);
                    const float2 x3 = *reinterpret_cast<const float2 *>(xcol + 96);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int row = bw + 4 * (4 * hh + i);
                        const float4 tv = *reinterpret_cast<const float4 *>(TB + (32 + row) * TP + 32 + 4 * m4);
                        acc[i] = __ffma2_rn(make_float2(tv.x, tv.x), x0, acc[i]);
                        acc[i] = __ffma2_rn(make_float2(tv.y, tv.y), x1, acc[i]);
                        acc[i] = __ffma2_rn(make_float2(tv.z, tv.z), x2, acc[i]);
                        acc[i] = __ffma2_rn(make_float2(tv.w, tv.w), x3, acc[i]);
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    *reinterpret_cast<float2 *>(TB + (32 + bw + 4 * (4 * hh + i)) * TP + cp) = make_float2(-acc[i].x, -acc[i].y);
            }
            group_sync(BAR_BACK, PF_BACK);

            // ===== 4. T Diag(e) -> W = T Diag(e) a~'; the exact-path decision; T Diag(w) for the slot
            const bool exact = !publish_and(write_t_copy(s_bg1, s_bg1, s_bg2) && well_a);
            if (btid == 0) {
                tc_fence_after();
                const uint32_t id_w = idesc_bf16(64, 128, false, true);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tbase + TM_W, dK(sb + P2_TBF, 8192, kk), dMN(sb + P2_AT, 8192, kk), id_w, kk > 0);
                mma_commit(bar_wmma);
            }
            if (!mbar_wait_cycles(bar_wmma, ph_wmma, WAIT_CYCLES)) ok = false;
            ph_wmma ^= 1;
            tc_fence_after();
            if (!same_gates) {
                write_t_copy(s_bg2, s_bg1, s_bg2);
                fence_async_smem();
                group_sync(BAR_BACK, PF_BACK);
            }
            // W (M = 64 layout: rows 16q..16q+15 in lanes 0..15 of quarter q) -> -W' in AT
            {
                const int r = quarter * 16 + (lane & 15);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    float v[32];
                    tmem_ld32(tbase + lane_base + TM_W + c4 * 32, v);
                    tmem_wait_ld();
                    if (lane < 16) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            *reinterpret_cast<uint4 *>(sm + P2_AT + sw_chunk(8192, r, c4 * 4 + q4)) =
                                pack8_neg(v + q4 * 8);
                    }
                }
            }
            if (btid == 0) {   // status word and epoch tag of the slot
                s_meta[128] = META_OK | (fast ? META_FAST : 0) | (exact ? META_EXACT : 0);
                s_meta[129] = (int)P.epoch;
            }
            fence_async_smem();
            tc_fence_before();
            ok = group_sync_and(BAR_BACK, PF_BACK, ok);
            if (ok && lane == 0) {
                if (bw == 0) bulk_store(slot + SL_QA, sm + P2_AT, 8192);                 // -W', panel 0
                else if (bw == 1) bulk_store(slot + SL_QA + 16384, sm + P2_AT + 8192, 8192);   // -W', panel 1
                else if (bw == 2) bulk_store(slot + SL_TBF, sm + P2_TBF, 8192);
                else bulk_store(slot + SL_META, sm + P2_META, SL_META_BYTES);
                bulk_commit();
            }
        }
        if (lane == 0) bulk_wait_all();
    }

    __syncthreads();
    tc_fence_after();
    ok = __syncthreads_and(ok) != 0;
    if (!ok && tid == 0) report_device_failure(DEV_WAIT_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

// ---- chain kernel (split path) ----------------------------------------------
// One CTA of 256 threads per (sequence, head) runs steps 5-7 over the chunks
// whose operands the preparation kernel stored in their slots: two slot
// buffers in shared memory, the next-but-one chunk loading while a chunk is
// processed.  Warps w and w + 4 share TMEM lane quarter w (value columns
// 32w .. 32w+31) and split the TMEM columns of every tile between them.
// Chunk c's o is staged in shared memory after its step-7 GEMMs and goes to
// HBM while the step-6 GEMMs of chunk c + 1 run (global stores, no tensor
// memory traffic next to the GEMMs).
constexpr int CK_NT = 256;
constexpr uint32_t CK_BUF = SLOT_BYTES;        // a slot image; M (or v) at SL_M
constexpr uint32_t CK_S0T = 2 * CK_BUF;         // state operand bf16 128 x 128, K-major
constexpr uint32_t CK_UT = CK_S0T + 32768;      // U^T bf16 128 x 64, then o staging
constexpr uint32_t CK_BAR = CK_UT + 16384;      // mbarriers: load[2], mma
constexpr uint32_t CK_TMEM = CK_BAR + 32;
constexpr uint32_t CK_ALLOC = CK_BAR + 64 + 1024;
constexpr uint32_t CK_TMEM_COLS = 256;   // S^T [0,128), U^T [128,192), O^T [192,256)
static_assert(CK_ALLOC <= 232448, "shared memory budget");
static_assert((CK_BUF & 1023) == 0 && (CK_S0T & 1023) == 0 && (CK_UT & 1023) == 0, "swizzle atoms");

// SNAP: state snapshots requested (compiled out otherwise)
template <bool SNAP>
__global__ void __launch_bounds__(CK_NT, 1) chunk_chain_kernel(const __grid_constant__ ChunkParams P)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);
    const FwdArgs &a = P.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int half = warp >> 2;   // which half of a tile's TMEM columns this warp handles
    const int H = a.H;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    const int row0 = seq_row0(a, n), len = seq_len(a, n), sbase = slot_base(a, n);
    const int nchunks = (len + C - 1) / C;
    const bool gdn2 = a.variant == GDN2;
    uint64_t *bar_load = reinterpret_cast<uint64_t *>(sm + CK_BAR), *bar_mma = bar_load + 2;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + CK_TMEM);
    uint8_t *op = (uint8_t *)a.o;

    if (warp == 0) tmem_alloc(s_tmem, CK_TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(bar_load + i, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int jcol = (warp & 3) * 32 + lane;   // value column j = TMEM lane
    bool ok = true;

    // chunk c's slot (operands, meta, GDN-2 M) and, except for GDN-2, its v tile
    auto issue_load = [&](int c, int buf) {
        uint8_t *dst = sm + buf * CK_BUF;
        const uint8_t *slot = P.ws + ((size_t)(sbase + c) * H + h) * SLOT_BYTES;
        mbar_expect_tx(bar_load + buf, SL_OPS + 16384);
        bulk_load(dst, slot, SL_OPS, bar_load + buf);
        if (gdn2) {
            bulk_load(dst + SL_M, slot + SL_M, 16384, bar_load + buf);
        } else {
            const int g = row0 + c * C;
            tma_load_3d(dst + SL_M, &P.tv, bar_load + buf, 0, h, g);
            tma_load_3d(dst + SL_M + 8192, &P.tv, bar_load + buf, 64, h, g);
        }
    };
    // o of chunk c: TMEM O^T -> bf16 staging [token][j] in the U^T tile (free once the step-7
    // GEMMs have read it), then 16-byte rows to HBM
    unsigned short *ost = reinterpret_cast<unsigned short *>(sm + CK_UT);
    auto stage_o = [&]() {
        float v[32];
        tmem_ld32(tbase + lane_base + TM_O + half * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const uint32_t pk = pack_bf16(v[e], v[e + 1]);
            ost[(half * 32 + e) * 128 + jcol] = (unsigned short)(pk & 0xFFFFu);
            ost[(half * 32 + e + 1) * 128 + jcol] = (unsigned short)(pk >> 16);
        }
    };
    auto store_o = [&](int c) {
        const int nv = min(C, len - c * C);
        const size_t rb = (size_t)row0 + c * C;
        for (int e = tid; e < nv * 16; e += CK_NT) {
            const int r = e >> 4, cgo = e & 15;
            *reinterpret_cast<uint4 *>(op + (((rb + r) * H + h) * D + cgo * 8) * 2) =
                *reinterpret_cast<const uint4 *>(sm + CK_UT + r * 256 + cgo * 16);
        }
    };
    // testing aid: this CTA never loads its first slot, so that waiting for it runs out
    const bool stall = P.debug_stall && blockIdx.x == 0;
    if (tid == 0) {
        // launched as a programmatic dependent of the preparation kernel: the slots are complete
        // and visible once this returns (at once when launched plainly).  Nothing else this
        // kernel reads before its first slot is written by the preparation kernel.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (nchunks > 0 && !stall) issue_load(0, 0);
        if (nchunks > 1) issue_load(1, 1);
    }
    {   // initial state -> TMEM (fp32), key channels 64 half .. 64 half + 63
        const size_t soff = ((size_t)n * H + h) * D * D;
#pragma unroll 1
        for (int c16 = 0; c16 < 4; ++c16) {
            float v[16];
            const int i0 = half * 64 + c16 * 16;
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = a.s0 ? a.s0[soff + (size_t)(i0 + e) * D + jcol] : 0.f;
            tmem_st16(tbase + lane_base + TM_S + i0, v);
        }
        tmem_wait_st();
    }
    uint32_t ph_mma = 0;
    bool mma_pending = false;   // thread 0: GEMMs issued but not yet committed and waited for
    bool timed_out = false, slot_missing = false;   // this thread's view of a failure
    int ch = 0;
    for (; ch < nchunks && ok; ++ch) {
        const int buf = ch & 1;
        const uint32_t bufa = sb + buf * CK_BUF;
        if (!mbar_wait_cycles(bar_load + buf, (ch >> 1) & 1, (stall && ch == 0) ? STALL_WAIT_CYCLES : WAIT_CYCLES))
            ok = false, timed_out = true;
        tc_fence_after();
        const int *meta = reinterpret_cast<const int *>(sm + buf * CK_BUF + SL_META);
        const float *gamC = reinterpret_cast<const float *>(meta);
        if (tid == 0 && ok && !(meta[128] & META_EXACT)) {   // U'^T = M^T (T Diag(w))^T: independent of the state
            const uint32_t id_u = idesc_bf16(128, 64, true, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tbase + TM_U, dMN(bufa + SL_M, 8192, kk), dK(bufa + SL_TBF, 8192, kk), id_u, kk > 0);
            mma_pending = true;   // completed by the step-6 commit
        }
        // a slot this call's preparation kernel did not complete reads as a failure
        const bool slot_ok = (meta[128] & META_OK) && meta[129] == (int)P.epoch;
        if (ok && !slot_ok) slot_missing = true;
        ok = __syncthreads_and(ok && slot_ok) != 0;
        if (!ok) break;
        if (meta[128] & META_EXACT) {
            // ---- exact path: this chunk token by token in fp32 from its raw inputs, staged in the
            // slot buffer (its prepared operands are not needed); o goes to the staging tile once the
            // previous chunk's o has left it
            const int nv = min(C, len - ch * C);
            if (ch > 0) store_o(ch - 1);
            __syncthreads();
            uint8_t *stq = sm + buf * CK_BUF, *stk = stq + 16384, *sta = stq + 32768;
            stage_exact_inputs(a, (size_t)row0 + ch * C, nv, h, stq, stk, sta, tid, CK_NT);
            __syncthreads();
            exact_chunk<2, true>(a, tbase + lane_base + TM_S, half * 64, jcol, half, stq, stk, sta,
                                 (size_t)row0 + ch * C, nv, h, reinterpret_cast<float4 *>(sm + CK_S0T),
                                 1 + (warp & 3), ost, 128, half == 0);
            fence_async_smem();   // the staging writes precede the next bulk load into this buffer
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (SNAP) snapshot_state(a, tbase + lane_base, sbase + ch, h, half * 2, 2, jcol);
            if (tid == 0 && ok && ch + 2 < nchunks) issue_load(ch + 2, buf);
            tc_fence_before();
            ok = __syncthreads_and(ok) != 0;
            continue;
        }
        const bool fast = (meta[128] & META_FAST) != 0;
        // ---- state pass: S^T *= Gamma_C in TMEM; bf16 operand copy (scaled on the fast path)
        {
            float s[64];
            tmem_ld32(tbase + lane_base + TM_S + half * 64, s);
            tmem_ld32(tbase + lane_base + TM_S + half * 64 + 32, s + 32);
            tmem_wait_ld();
#pragma unroll
            for (int c32 = 0; c32 < 2; ++c32) {
                const int i0 = half * 64 + c32 * 32;
                float *sv = s + c32 * 32;
                float t[32];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {   // column pairs on the packed fp32 pipe
                    const float2 t2 = __fmul2_rn(make_float2(sv[e], sv[e + 1]),
                                                 *reinterpret_cast<const float2 *>(gamC + i0 + e));
                    t[e] = t2.x;
                    t[e + 1] = t2.y;
                    if (fast) {
                        sv[e] = t2.x;
                        sv[e + 1] = t2.y;
                    }
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    *reinterpret_cast<uint4 *>(sm + CK_S0T + sw_chunk(16384, jcol, (i0 >> 3) + q4)) =
                        pack8(sv + q4 * 8);
                tmem_st16(tbase + lane_base + TM_S + i0, t);
                tmem_st16(tbase + lane_base + TM_S + i0 + 16, t + 16);
            }
        }
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- step 6: U^T -= S^T W^T ; O^T = S^T Q^T
        if (tid == 0) {
            tc_fence_after();
            step6_mmas(tbase, sb + CK_S0T, bufa + SL_QA);
            mma_commit(bar_mma);
        }
        // ---- o of the previous chunk, staged in the U^T tile, to HBM while the step-6 GEMMs run
        if (ch > 0) store_o(ch - 1);
        if (!mbar_wait_cycles(bar_mma, ph_mma, WAIT_CYCLES)) ok = false, timed_out = true;
        ph_mma ^= 1;
        mma_pending = false;
        tc_fence_after();
        __syncthreads();   // staging read before the U^T tile is rewritten
        // ---- U^T row j -> bf16 K-major tile (rows j, K = token); tokens 32 half .. 32 half + 31
        {
            float v[32];
            tmem_ld32(tbase + lane_base + TM_U + half * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4 *>(sm + CK_UT + sw_chunk(16384, jcol, half * 4 + q4)) = pack8(v + q4 * 8);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- step 7: O^T += U^T P^T ; S^T += U^T Kbar
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_o = idesc_bf16(128, 64, false, false);
            const uint32_t id_s = idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16(tbase + TM_O, dK(sb + CK_UT, 16384, kk), dK(bufa + SL_PBF, 8192, kk), id_o, 1);
                mma_bf16(tbase + TM_S, dK(sb + CK_UT, 16384, kk), dMN(bufa + SL_KB, 8192, kk), id_s, 1);
            }
            mma_commit(bar_mma);
        }
        if (!mbar_wait_cycles(bar_mma, ph_mma, WAIT_CYCLES)) ok = false, timed_out = true;
        ph_mma ^= 1;
        tc_fence_after();
        if (SNAP) snapshot_state(a, tbase + lane_base, sbase + ch, h, half * 2, 2, jcol);
        // every read of this buffer is done: load chunk ch + 2 into it
        if (tid == 0 && ok && ch + 2 < nchunks) issue_load(ch + 2, buf);
        stage_o();   // the U^T tile is free: the step-7 GEMMs are done
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;
    }
    if (ok && nchunks > 0) store_o(nchunks - 1);
    if (timed_out || slot_missing) report_device_failure((timed_out ? DEV_WAIT_TIMEOUT : 0u) |
                                                         (slot_missing ? DEV_SLOT_MISSING : 0u));
    if (!ok && tid == 0) {   // drain loads (those issued) and an uncommitted GEMM still in flight (bounded)
        for (int c = ch; c < nchunks && c < ch + 2; ++c)
            if (!(stall && c == 0)) mbar_wait_cycles(bar_load + (c & 1), (c >> 1) & 1, WAIT_CYCLES);
        if (mma_pending) {
            mma_commit(bar_mma);
            mbar_wait_cycles(bar_mma, ph_mma, WAIT_CYCLES);
        }
    }
    // ---- final state (NaN if a wait timed out or a slot was missing)
    __syncthreads();
    tc_fence_after();
    if (a.sf) {
        const size_t soff = ((size_t)n * H + h) * D * D;
#pragma unroll 1
        for (int c32 = 0; c32 < 2; ++c32) {
            const int i0 = half * 64 + c32 * 32;
            float s[32];
            tmem_ld32(tbase + lane_base + TM_S + i0, s);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e)
                a.sf[soff + (size_t)(i0 + e) * D + jcol] = ok ? s[e] : __int_as_float(0x7fc00000);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, CK_TMEM_COLS);
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

// [rows = B*T][H][128] bf16; box {inner, 1, 64}; inner 128 without swizzle (row-major
// tile) or 64 with the 128-byte swizzle (one K-major / MN-major operand panel)
bool make_map(CUtensorMap *m, const void *base, long long rows, int H, bool swizzle)
{
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {swizzle ? 64u : 128u, 1, 64}, es[3] = {1, 1, 1};
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace {
// Per-device one-time set-up: dynamic shared-memory opt-ins and the SM count.
cudaError_t device_setup(int &num_sms)
{
    static std::mutex mu;
    static int sms[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!sms[dev]) {
        if ((e = cudaFuncSetAttribute(chunk_fwd_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      SMEM_ALLOC)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(chunk_fwd_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      SMEM_ALLOC)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(chunk_prep_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      P2_ALLOC)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(chunk_prep_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      P2_ALLOC)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(chunk_chain_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      CK_ALLOC)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(chunk_chain_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      CK_ALLOC)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return e;
    }
    num_sms = sms[dev];
    return cudaSuccess;
}

cudaError_t make_params(ChunkParams &p, const FwdArgs &a)
{
    memset(&p, 0, sizeof(p));
    p.a = a;
    const long long rows = (long long)a.B * a.T;
    if (rows > 0) {
        if (!make_map(&p.tq, a.q, rows, a.H, false) || !make_map(&p.tk, a.k, rows, a.H, false) ||
            !make_map(&p.tv, a.v, rows, a.H, true) || !make_map(&p.ta, a.alpha, rows, a.H, false))
            return cudaErrorInvalidValue;
    }
    return cudaSuccess;
}
}  // namespace

namespace {
__device__ unsigned int g_status_taken;
__global__ void take_status_kernel() { g_status_taken = atomicExch(&g_device_status, 0u); }
}  // namespace

cudaError_t take_device_status(cudaStream_t st, unsigned *bits)
{
    static std::mutex mu;   // one reader of the staging word at a time
    std::lock_guard<std::mutex> lock(mu);
    take_status_kernel<<<1, 1, 0, st>>>();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    unsigned w = 0;
    if ((e = cudaMemcpyFromSymbolAsync(&w, g_status_taken, sizeof(w), 0, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        return e;
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
    *bits = w;
    return cudaSuccess;
}

cudaError_t launch_chunk_fwd_sm100(const FwdArgs &a, cudaStream_t st)
{
    int num_sms = 0;
    cudaError_t e = device_setup(num_sms);
    if (e != cudaSuccess) return e;
    ChunkParams p;
    if ((e = make_params(p, a)) != cudaSuccess) return e;
    const int N = a.cu_seqlens ? a.num_seqs : a.B;
    if (a.prep) chunk_fwd_kernel<true><<<(unsigned)(N * a.H), NT, SMEM_ALLOC, st>>>(p);
    else chunk_fwd_kernel<false><<<(unsigned)(N * a.H), NT, SMEM_ALLOC, st>>>(p);
    return cudaGetLastError();
}

bool chunk_prefer_split(const FwdArgs &a)
{
    // Cost model from measured kernel times on B200 (thousands of SM cycles per chunk):
    // preparation of one (chunk, head) by the two-group split kernel ~12.0, the split chain
    // ~4.4, the fused kernel's critical path ~16.3.  With U = N*H units on S SMs and
    // W = ceil(U / S) waves of the per-unit kernels:  fused ~ W * 16.3,
    // split ~ (U / S) * 12.0 + W * 4.4  (per chunk).
    // Packed (varlen) batches take the split form: the fused kernel's time is that of the
    // longest sequence per CTA, while the preparation kernel balances chunks over all SMs.
    int num_sms = 0;
    if (device_setup(num_sms) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    if (a.cu_seqlens) return true;
    const double U = (double)a.B * a.H, S = num_sms;
    const double W = std::ceil(U / S);
    return (U / S) * 12.0 + W * 4.4 < W * 16.3;
}

size_t chunk_split_workspace_bytes(const FwdArgs &a)
{
    const long long N = a.cu_seqlens ? a.num_seqs : a.B;
    const long long rows = (long long)a.B * a.T;
    return (size_t)(N + (rows + C - 1) / C) * a.H * SLOT_BYTES;
}

cudaError_t launch_chunk_split_sm100(const FwdArgs &a, void *ws, cudaStream_t st)
{
    int num_sms = 0;
    cudaError_t e = device_setup(num_sms);
    if (e != cudaSuccess) return e;
    ChunkParams p;
    if ((e = make_params(p, a)) != cudaSuccess) return e;
    static std::atomic<uint32_t> epoch{0};
    const int N = a.cu_seqlens ? a.num_seqs : a.B;
    const long long rows = (long long)a.B * a.T;
    p.ws = static_cast<uint8_t *>(ws);
    p.nslots = (int)(N + (rows + C - 1) / C);
    p.epoch = epoch.fetch_add(1) + 1;   // a 32-bit tag: it repeats only after 2^32 split-form calls
    p.debug_stall = a.debug_stall;
    const long long nwork = (long long)p.nslots * a.H;
    const bool prep = rows > 0 && nwork > 0;
    if (prep) {
        const unsigned grid = (unsigned)std::min<long long>(nwork, num_sms);
        if (a.prep) chunk_prep_kernel<true><<<grid, PF_NT, P2_ALLOC, st>>>(p);
        else chunk_prep_kernel<false><<<grid, PF_NT, P2_ALLOC, st>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // The chain kernel is a programmatic dependent of the preparation kernel (it may start its
    // set-up while the preparation grid drains; its slot reads wait for that grid).  Only then:
    // behind any other kernel its initial-state reads would not wait.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(N * a.H));
    cfg.blockDim = dim3(CK_NT);
    cfg.dynamicSmemBytes = CK_ALLOC;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = prep ? 1 : 0;
    if (a.snap) e = cudaLaunchKernelEx(&cfg, chunk_chain_kernel<true>, p);
    else e = cudaLaunchKernelEx(&cfg, chunk_chain_kernel<false>, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace kda
