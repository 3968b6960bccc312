// C ABI of the kda library: host-side argument checks and kernel dispatch.
// Declarations, layouts and error semantics: include/kda.h.
#include <cstdarg>
#include <cstdio>
#include <cstdint>

#include "../../include/kda.h"
#include "scan_bwd.cuh"
#include "rank2.cuh"

namespace {

thread_local char g_detail[512] = "";

int fail(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *where)
{
    return fail(KDA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Input-preparation flags and their kernel-side bits.
constexpr unsigned PREP_FLAGS = KDA_FLAG_GATE_LOGITS | KDA_FLAG_L2NORM_K;
unsigned prep_bits(unsigned flags)
{
    return ((flags & KDA_FLAG_GATE_LOGITS) ? kda::PREP_LOGITS : 0u) |
           ((flags & KDA_FLAG_L2NORM_K) ? kda::PREP_L2NORM_K : 0u);
}
bool head_dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool chunk_ok(int c) { return c == 16 || c == 32 || c == 64 || c == 128; }

// Checks shared by the forward and decode calls: enums, head dims, pointers.
int check_common(int variant, int gate_range, int dtype, int d_k, int d_v,
                 const void *q, const void *k, const void *v, const void *alpha,
                 const void *g1, const void *g2, const void *o, bool need_data)
{
    if (variant < KDA_VARIANT_KDA || variant > KDA_VARIANT_GDN2)
        return fail(KDA_ERR_INVALID_ARG, "variant %d is not KDA(0), RDA(1) or GDN2(2)", variant);
    if (gate_range != KDA_RANGE_STANDARD && gate_range != KDA_RANGE_EXTENDED)
        return fail(KDA_ERR_INVALID_ARG, "gate_range %d is not STANDARD(0) or EXTENDED(1)", gate_range);
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_F32)
        return fail(KDA_ERR_INVALID_ARG, "dtype %d is not BF16(0) or F32(1)", dtype);
    if (d_k < 1 || d_v < 1) return fail(KDA_ERR_INVALID_ARG, "head dims must be positive (d_k=%d, d_v=%d)", d_k, d_v);
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "head dims d_k=%d, d_v=%d: supported are 16, 32, 64, 128", d_k, d_v);
    if (!need_data) return KDA_OK;
    const void *ptrs[] = {q, k, v, alpha, g1, o};
    const char *names[] = {"q", "k", "v", "alpha", "g1", "o"};
    for (int i = 0; i < 6; ++i) {
        if (!ptrs[i]) return fail(KDA_ERR_INVALID_ARG, "%s is NULL", names[i]);
        if (!aligned16(ptrs[i])) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
    }
    if (variant != KDA_VARIANT_KDA) {
        if (!g2) return fail(KDA_ERR_INVALID_ARG, "g2 (write gate) is NULL for RDA/GDN2");
        if (!aligned16(g2)) return fail(KDA_ERR_INVALID_ARG, "g2 is not 16-byte aligned");
    }
    return KDA_OK;
}

// Form of the tensor-core path: the fused kernel (no workspace) or the split
// preparation + chain kernels; by shape unless a flag forces one.
bool use_split(const kda::FwdArgs &a, unsigned flags)
{
    if (flags & KDA_FLAG_FORCE_FUSED) return false;
    if (flags & KDA_FLAG_FORCE_SPLIT) return true;
#ifdef KDA_WITH_SM100_CHUNK
    return kda::chunk_prefer_split(a);
#else
    (void)a;
    return false;
#endif
}

// Validated forward arguments; returns KDA_OK or the error code (detail set).
int chunk_args(kda::FwdArgs &a, int variant, int gate_range, int dtype, int B, int T, int H, int d_k, int d_v,
               const void *q, const void *k, const void *v, const void *alpha, const void *g1, const void *g2,
               const int32_t *cu_seqlens, int num_seqs, const float *initial_state, float *final_state, void *o,
               int chunk_size, unsigned flags)
{
    if (B < 1 || T < 0 || H < 1)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d T=%d H=%d (need B>=1, T>=0, H>=1)", B, T, H);
    if ((unsigned long long)B * (unsigned long long)T * H * 128ull > (1ull << 46))
        return fail(KDA_ERR_INVALID_ARG, "problem too large (B*T*H=%llu)", (unsigned long long)B * T * H);
    int rc = check_common(variant, gate_range, dtype, d_k, d_v, q, k, v, alpha, g1, g2, o, T > 0);
    if (rc != KDA_OK) return rc;
    if (!chunk_ok(chunk_size))
        return fail(KDA_ERR_UNSUPPORTED, "chunk_size %d: supported are 16, 32, 64, 128", chunk_size);
    if (flags & ~(KDA_FLAG_VALIDATE_RANGE | KDA_FLAG_FORCE_SCAN | KDA_FLAG_FORCE_FUSED | KDA_FLAG_FORCE_SPLIT |
                  PREP_FLAGS | KDA_FLAG_DEBUG_STALL))
        return fail(KDA_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
    if ((flags & KDA_FLAG_FORCE_FUSED) && (flags & KDA_FLAG_FORCE_SPLIT))
        return fail(KDA_ERR_INVALID_ARG, "KDA_FLAG_FORCE_FUSED and KDA_FLAG_FORCE_SPLIT exclude each other");
    if ((flags & KDA_FLAG_DEBUG_STALL) && !(flags & KDA_FLAG_FORCE_SPLIT))
        return fail(KDA_ERR_INVALID_ARG, "KDA_FLAG_DEBUG_STALL needs KDA_FLAG_FORCE_SPLIT");
    int N = B;
    if (cu_seqlens) {
        if (B != 1) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens requires B == 1 (got B=%d)", B);
        if (num_seqs < 1) return fail(KDA_ERR_INVALID_ARG, "num_seqs must be >= 1 with cu_seqlens (got %d)", num_seqs);
        if (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)
            return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
        N = num_seqs;
    }
    if (initial_state && !aligned16(initial_state))
        return fail(KDA_ERR_INVALID_ARG, "initial_state is not 16-byte aligned");
    if (final_state && !aligned16(final_state))
        return fail(KDA_ERR_INVALID_ARG, "final_state is not 16-byte aligned");
    a = kda::FwdArgs{variant, B, T, H, d_k, d_v, q, k, v, alpha, g1, g2, cu_seqlens, N,
                     initial_state, final_state, o, prep_bits(flags), gate_range == KDA_RANGE_EXTENDED};
    a.debug_stall = (flags & KDA_FLAG_DEBUG_STALL) ? 1 : 0;
    return KDA_OK;
}

// KDA_FLAG_VALIDATE_RANGE: check the gates against the declared range and
// cu_seqlens against its contract on the device, wait for the outcome, and
// refuse the call (nothing launched) on a violation.  Gate logits are not
// gates yet: with KDA_FLAG_GATE_LOGITS only cu_seqlens is checked.
int validate(const kda::FwdArgs &a, int gate_range, int dtype, unsigned flags, cudaStream_t st)
{
    if (!(flags & KDA_FLAG_VALIDATE_RANGE)) return KDA_OK;
    const long long n_tok = (flags & KDA_FLAG_GATE_LOGITS) ? 0 : (long long)a.B * a.T * a.H;
    int bad_gates = 0, bad_seqlens = 0;
    const cudaError_t e = kda::validate_inputs(a.variant, gate_range, dtype == KDA_DTYPE_BF16, n_tok, a.dk, a.alpha,
                                               a.g1, a.cu_seqlens, a.num_seqs, (long long)a.B * a.T, st, &bad_gates,
                                               &bad_seqlens);
    if (e != cudaSuccess) return cuda_fail(e, "input validation");
    if (bad_seqlens)
        return fail(KDA_ERR_INVALID_ARG, "cu_seqlens violates cu[0] = 0, cu[n] <= cu[n+1], cu[N] = %lld "
                                         "(%d violations)", (long long)a.B * a.T, bad_seqlens);
    if (bad_gates)
        return fail(KDA_ERR_RANGE, "%d gate values outside the declared range (or NaN)", bad_gates);
    return KDA_OK;
}

bool tensor_core_path(const kda::FwdArgs &a, int dtype, int chunk_size, unsigned flags)
{
#ifdef KDA_WITH_SM100_CHUNK
    return dtype == KDA_DTYPE_BF16 && a.dk == 128 && a.dv == 128 && chunk_size == 64 &&
           !(flags & KDA_FLAG_FORCE_SCAN);
#else
    (void)a; (void)dtype; (void)chunk_size; (void)flags;
    return false;
#endif
}

// Launches the chosen path; `ws` (may be NULL) holds `ws_bytes` bytes.
int chunk_launch(const kda::FwdArgs &a, int dtype, int chunk_size, unsigned flags, void *ws, size_t ws_bytes,
                 cudaStream_t st)
{
    cudaError_t e = cudaSuccess;
    if (tensor_core_path(a, dtype, chunk_size, flags)) {
#ifdef KDA_WITH_SM100_CHUNK
        if (use_split(a, flags) && ws && ws_bytes >= kda::chunk_split_workspace_bytes(a))
            e = kda::launch_chunk_split_sm100(a, ws, st);
        else
            e = kda::launch_chunk_fwd_sm100(a, st);
#endif
    } else {
        e = kda::launch_scan_fwd(a, dtype == KDA_DTYPE_BF16, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd launch");
    return KDA_OK;
}

}  // namespace

extern "C" size_t kda_chunk_fwd_workspace_size(int dtype, int B, int T, int H, int d_k, int d_v,
                                               int has_cu_seqlens, int num_seqs, int chunk_size, unsigned flags)
{
    if (B < 1 || T < 0 || H < 1 || (has_cu_seqlens && (B != 1 || num_seqs < 1))) return 0;
    if ((unsigned long long)B * (unsigned long long)T * H * 128ull > (1ull << 46)) return 0;
    if ((flags & KDA_FLAG_FORCE_FUSED) && (flags & KDA_FLAG_FORCE_SPLIT)) return 0;
    kda::FwdArgs a{};
    a.B = B; a.T = T; a.H = H; a.dk = d_k; a.dv = d_v;
    a.num_seqs = has_cu_seqlens ? num_seqs : B;
    a.cu_seqlens = has_cu_seqlens ? reinterpret_cast<const int32_t *>(16) : nullptr;  // presence only
    if (!tensor_core_path(a, dtype, chunk_size, flags) || !use_split(a, flags)) return 0;
#ifdef KDA_WITH_SM100_CHUNK
    return kda::chunk_split_workspace_bytes(a);
#else
    return 0;
#endif
}

extern "C" int kda_chunk_fwd_ws(int variant, int gate_range, int dtype,
                                int B, int T, int H, int d_k, int d_v,
                                const void *q, const void *k, const void *v, const void *alpha,
                                const void *g1, const void *g2,
                                const int32_t *cu_seqlens, int num_seqs,
                                const float *initial_state, float *final_state, float *chunk_states,
                                void *o, int chunk_size, void *workspace, size_t workspace_bytes,
                                unsigned flags, void *stream)
{
    kda::FwdArgs a;
    int rc = chunk_args(a, variant, gate_range, dtype, B, T, H, d_k, d_v, q, k, v, alpha, g1, g2, cu_seqlens,
                        num_seqs, initial_state, final_state, o, chunk_size, flags);
    if (rc != KDA_OK) return rc;
    if (chunk_states && !aligned16(chunk_states))
        return fail(KDA_ERR_INVALID_ARG, "chunk_states is not 16-byte aligned");
    a.snap = chunk_states;
    if (workspace && !aligned16(workspace)) return fail(KDA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    if ((flags & KDA_FLAG_DEBUG_STALL) && !tensor_core_path(a, dtype, chunk_size, flags))
        return fail(KDA_ERR_INVALID_ARG, "KDA_FLAG_DEBUG_STALL needs the tensor-core split form");
    if ((flags & KDA_FLAG_FORCE_SPLIT) && tensor_core_path(a, dtype, chunk_size, flags)) {
        size_t need = 0;
#ifdef KDA_WITH_SM100_CHUNK
        need = kda::chunk_split_workspace_bytes(a);
#endif
        if (!workspace || workspace_bytes < need)
            return fail(KDA_ERR_INVALID_ARG, "KDA_FLAG_FORCE_SPLIT needs a workspace of %zu bytes (got %zu)", need,
                        workspace ? workspace_bytes : (size_t)0);
    }
    if ((rc = validate(a, gate_range, dtype, flags, static_cast<cudaStream_t>(stream))) != KDA_OK) return rc;
    return chunk_launch(a, dtype, chunk_size, flags, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" int kda_chunk_fwd(int variant, int gate_range, int dtype,
                             int B, int T, int H, int d_k, int d_v,
                             const void *q, const void *k, const void *v, const void *alpha,
                             const void *g1, const void *g2,
                             const int32_t *cu_seqlens, int num_seqs,
                             const float *initial_state, float *final_state,
                             void *o, int chunk_size, unsigned flags, void *stream)
{
    kda::FwdArgs a;
    int rc = chunk_args(a, variant, gate_range, dtype, B, T, H, d_k, d_v, q, k, v, alpha, g1, g2, cu_seqlens,
                        num_seqs, initial_state, final_state, o, chunk_size, flags);
    if (rc != KDA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((flags & KDA_FLAG_DEBUG_STALL) && !tensor_core_path(a, dtype, chunk_size, flags))
        return fail(KDA_ERR_INVALID_ARG, "KDA_FLAG_DEBUG_STALL needs the tensor-core split form");
    if ((rc = validate(a, gate_range, dtype, flags, st)) != KDA_OK) return rc;
    void *ws = nullptr;
    size_t ws_bytes = 0;
#ifdef KDA_WITH_SM100_CHUNK
    if (tensor_core_path(a, dtype, chunk_size, flags) && use_split(a, flags)) {
        // stream-ordered workspace; without it the fused kernel runs
        ws_bytes = kda::chunk_split_workspace_bytes(a);
        if (cudaMallocAsync(&ws, ws_bytes, st) != cudaSuccess) {
            (void)cudaGetLastError();
            ws = nullptr;
            ws_bytes = 0;
        }
    }
#endif
    if ((flags & KDA_FLAG_FORCE_SPLIT) && !ws && tensor_core_path(a, dtype, chunk_size, flags) &&
        (flags & KDA_FLAG_DEBUG_STALL))
        return fail(KDA_ERR_CUDA, "KDA_FLAG_DEBUG_STALL: the split form's workspace could not be allocated");
    rc = chunk_launch(a, dtype, chunk_size, flags, ws, ws_bytes, st);
    if (ws) {
        const cudaError_t ef = cudaFreeAsync(ws, st);
        if (rc == KDA_OK && ef != cudaSuccess) rc = cuda_fail(ef, "kda_chunk_fwd workspace release");
    }
    return rc;
}

extern "C" int kda_chunk_fwd_noalloc(int variant, int gate_range, int dtype,
                                     int B, int T, int H, int d_k, int d_v,
                                     const void *q, const void *k, const void *v, const void *alpha,
                                     const void *g1, const void *g2,
                                     const int32_t *cu_seqlens, int num_seqs,
                                     const float *initial_state, float *final_state,
                                     void *o, unsigned flags, void *stream)
{
    kda::FwdArgs a;
    int rc = chunk_args(a, variant, gate_range, dtype, B, T, H, d_k, d_v, q, k, v, alpha, g1, g2, cu_seqlens,
                        num_seqs, initial_state, final_state, o, 64, 0u);
    if (rc != KDA_OK) return rc;
    if (flags != 0) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_noalloc takes no flags (got 0x%x)", flags);
#ifdef KDA_WITH_SM100_CHUNK
    if (!tensor_core_path(a, dtype, 64, 0u))
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd_noalloc serves bf16 with d_k = d_v = 128 only "
                                         "(got dtype %d, d_k %d, d_v %d)", dtype, d_k, d_v);
    const size_t need = kda::chunk_split_workspace_bytes(a), cap = kda::chunk_noalloc_capacity();
    if (need > cap)
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd_noalloc: this problem needs %zu bytes of scratch, "
                                         "the fixed array holds %zu ((N + ceil(B*T/64)) * H must be <= %zu)",
                    need, cap, cap / 82944);
    const cudaError_t e = kda::launch_chunk_split_noalloc(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_noalloc launch");
    return KDA_OK;
#else
    return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd_noalloc: built without the sm_100a chunked kernels");
#endif
}

namespace {

// Backward workspace: the forward's state snapshots (chunk slots), u_t of
// every token, and each CTA's per-chunk states, in that order.
size_t bwd_snap_bytes(const kda::FwdArgs &a)
{
    const long long N = a.cu_seqlens ? a.num_seqs : a.B;
    const long long slots = N + ((long long)a.B * a.T + 63) / 64;
    return (size_t)slots * a.H * a.dk * a.dv * sizeof(float);
}
size_t bwd_u_bytes(const kda::FwdArgs &a) { return (size_t)a.B * a.T * a.H * a.dv * sizeof(float); }
size_t bwd_workspace_bytes(const kda::FwdArgs &a)
{
    return bwd_snap_bytes(a) + bwd_u_bytes(a) + kda::scan_bwd_scratch_bytes(a);
}

}  // namespace

extern "C" size_t kda_chunk_bwd_workspace_size(int dtype, int B, int T, int H, int d_k, int d_v,
                                               int has_cu_seqlens, int num_seqs)
{
    if (B < 1 || T < 0 || H < 1 || (has_cu_seqlens && (B != 1 || num_seqs < 1))) return 0;
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_F32) return 0;
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v)) return 0;
    if ((unsigned long long)B * (unsigned long long)T * H * 128ull > (1ull << 46)) return 0;
    kda::FwdArgs a{};
    a.B = B; a.T = T; a.H = H; a.dk = d_k; a.dv = d_v;
    a.num_seqs = has_cu_seqlens ? num_seqs : B;
    a.cu_seqlens = has_cu_seqlens ? reinterpret_cast<const int32_t *>(16) : nullptr;   // presence only
    return bwd_workspace_bytes(a);
}

extern "C" int kda_chunk_bwd(int variant, int gate_range, int dtype,
                             int B, int T, int H, int d_k, int d_v,
                             const void *q, const void *k, const void *v, const void *alpha,
                             const void *g1, const void *g2,
                             const int32_t *cu_seqlens, int num_seqs, const float *initial_state,
                             const void *d_o, const float *d_final_state,
                             float *dq, float *dk, float *dv, float *dalpha, float *dg1, float *dg2,
                             float *d_initial_state, void *workspace, size_t workspace_bytes,
                             unsigned flags, void *stream)
{
    if (flags) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd takes no flags (got 0x%x)", flags);
    if (T > 0 && !d_o) return fail(KDA_ERR_INVALID_ARG, "d_o is NULL");
    // d_o has o's layout and dtype: the forward's checks cover it in o's place
    kda::FwdArgs a;
    int rc = chunk_args(a, variant, gate_range, dtype, B, T, H, d_k, d_v, q, k, v, alpha, g1, g2, cu_seqlens,
                        num_seqs, initial_state, nullptr, const_cast<void *>(d_o), 64, 0u);
    if (rc != KDA_OK) return rc;
    if (T > 0) {
        const void *need[] = {d_o, dq, dk, dv, dalpha, dg1};
        const char *names[] = {"d_o", "dq", "dk", "dv", "dalpha", "dg1"};
        for (int i = 0; i < 6; ++i) {
            if (!need[i]) return fail(KDA_ERR_INVALID_ARG, "%s is NULL", names[i]);
            if (!aligned16(need[i])) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
        }
        if (variant != KDA_VARIANT_KDA && (!dg2 || !aligned16(dg2)))
            return fail(KDA_ERR_INVALID_ARG, "dg2 is NULL or misaligned (RDA and GDN-2 have a write gate)");
    }
    if ((d_final_state && !aligned16(d_final_state)) || (d_initial_state && !aligned16(d_initial_state)))
        return fail(KDA_ERR_INVALID_ARG, "d_final_state / d_initial_state is not 16-byte aligned");
    const size_t need_ws = bwd_workspace_bytes(a);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need_ws)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd needs a 16-byte aligned workspace of %zu bytes", need_ws);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == KDA_DTYPE_BF16;
    // 1. forward scan in fp32, keeping only the state after every 64 tokens (the checkpoints)
    //    and u_t of every token
    a.o = nullptr;
    a.sf = nullptr;
    a.snap = static_cast<float *>(workspace);
    float *u_save = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + bwd_snap_bytes(a));
    cudaError_t e = kda::launch_scan_checkpoints(a, u_save, bf16, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_bwd forward replay");
    // 2. adjoint scan
    kda::BwdArgs g{d_o, d_final_state, dq, dk, dv, dalpha, dg1, dg2, d_initial_state,
                   reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + bwd_snap_bytes(a) + bwd_u_bytes(a)),
                   u_save};
    e = kda::launch_scan_bwd(a, g, bf16, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_bwd launch");
    return KDA_OK;
}

namespace {

// Rank-2 steps: workspace regions (256-byte aligned) for the sub-token problem
// of B x 2T tokens: q2, alpha2 [B,2T,H,d_k], o2 [B,2T,H,d_v], doubled
// cu_seqlens, then the chunked path's own workspace.
struct Rank2Layout {
    size_t q2, a2, o2, cu2, chunk, chunk_bytes, total;
};

Rank2Layout rank2_layout(int dtype, int B, int T, int H, int d_k, int d_v, int has_cu, int num_seqs, int chunk_size,
                         unsigned flags)
{
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    const size_t tok2 = (size_t)B * 2 * (size_t)T * H;
    Rank2Layout L;
    L.q2 = 0;
    L.a2 = up(tok2 * d_k * es);
    L.o2 = L.a2 + up(tok2 * d_k * es);
    L.cu2 = L.o2 + up(tok2 * d_v * es);
    L.chunk = L.cu2 + up(has_cu ? (size_t)(num_seqs + 1) * 4 : 0);
    L.chunk_bytes = kda_chunk_fwd_workspace_size(dtype, B, 2 * T, H, d_k, d_v, has_cu, num_seqs, chunk_size, flags);
    L.total = L.chunk + up(L.chunk_bytes);
    return L;
}

bool rank2_sizes_ok(int dtype, int B, int T, int H, int d_k, int d_v, int has_cu, int num_seqs)
{
    if (B < 1 || T < 0 || T > (1 << 29) || H < 1 || (has_cu && (B != 1 || num_seqs < 1))) return false;
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_F32) return false;
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v)) return false;
    return (unsigned long long)B * (2ull * (unsigned long long)T) * H * 128ull <= (1ull << 46);
}

}  // namespace

extern "C" size_t kda_chunk_fwd_rank2_workspace_size(int dtype, int B, int T, int H, int d_k, int d_v,
                                                     int has_cu_seqlens, int num_seqs, int chunk_size, unsigned flags)
{
    if (!rank2_sizes_ok(dtype, B, T, H, d_k, d_v, has_cu_seqlens, num_seqs)) return 0;
    if ((flags & KDA_FLAG_FORCE_FUSED) && (flags & KDA_FLAG_FORCE_SPLIT)) return 0;
    return rank2_layout(dtype, B, T, H, d_k, d_v, has_cu_seqlens, num_seqs, chunk_size, flags).total;
}

extern "C" int kda_chunk_fwd_rank2(int variant, int gate_range, int dtype,
                                   int B, int T, int H, int d_k, int d_v,
                                   const void *q, const void *k, const void *v, const void *alpha,
                                   const void *g1, const void *g2,
                                   const int32_t *cu_seqlens, int num_seqs,
                                   const float *initial_state, float *final_state,
                                   void *o, int chunk_size, void *workspace, size_t workspace_bytes,
                                   unsigned flags, void *stream)
{
    if (flags & KDA_FLAG_GATE_LOGITS)
        return fail(KDA_ERR_UNSUPPORTED, "rank-2 steps take gate values, not logits "
                                         "(the second sub-step's alpha = 1 has no finite logit)");
    if (flags & (KDA_FLAG_VALIDATE_RANGE | KDA_FLAG_DEBUG_STALL))
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd_rank2 takes neither KDA_FLAG_VALIDATE_RANGE nor "
                                         "KDA_FLAG_DEBUG_STALL (check the gates with kda_check_gates)");
    if (B < 1 || T < 0 || H < 1 || T > (1 << 29))
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d T=%d H=%d (need B>=1, 0<=T<=2^29, H>=1)", B, T, H);
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_F32) return fail(KDA_ERR_INVALID_ARG, "bad dtype %d", dtype);
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "head dims d_k=%d d_v=%d: supported are 16, 32, 64, 128", d_k, d_v);
    if (!rank2_sizes_ok(dtype, B, T, H, d_k, d_v, cu_seqlens != nullptr, num_seqs))
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d T=%d H=%d num_seqs=%d (cu_seqlens needs B == 1)", B, T, H,
                    num_seqs);
    if (T > 0) {
        const void *need[] = {q, alpha, o};
        const char *names[] = {"q", "alpha", "o"};
        for (int i = 0; i < 3; ++i) {
            if (!need[i]) return fail(KDA_ERR_INVALID_ARG, "%s is NULL", names[i]);
            if (!aligned16(need[i])) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
        }
    }
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
    const Rank2Layout L = rank2_layout(dtype, B, T, H, d_k, d_v, cu_seqlens != nullptr, num_seqs, chunk_size, flags);
    if (!workspace || !aligned16(workspace) || workspace_bytes < L.total)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_rank2 needs a 16-byte aligned workspace of %zu bytes",
                    L.total);
    uint8_t *w = static_cast<uint8_t *>(workspace);
    int32_t *cu2 = cu_seqlens ? reinterpret_cast<int32_t *>(w + L.cu2) : nullptr;
    // the sub-token problem: k, v and the gates are already [B,2T,H,.]; q, alpha and o live in the workspace
    kda::FwdArgs a;
    int rc = chunk_args(a, variant, gate_range, dtype, B, 2 * T, H, d_k, d_v, w + L.q2, k, v, w + L.a2, g1, g2,
                        cu2, num_seqs, initial_state, final_state, w + L.o2, chunk_size, flags);
    if (rc != KDA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == KDA_DTYPE_BF16;
    const long long tokens = (long long)B * T;
    cudaError_t e = kda::launch_rank2_expand(bf16, q, alpha, w + L.q2, w + L.a2, tokens, H * d_k, cu_seqlens, cu2,
                                             cu_seqlens ? num_seqs + 1 : 0, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_rank2 expand");
    rc = chunk_launch(a, dtype, chunk_size, flags, w + L.chunk, L.chunk_bytes, st);
    if (rc != KDA_OK) return rc;
    e = kda::launch_rank2_gather(bf16, w + L.o2, o, tokens, H * d_v, 1, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_rank2 gather");
    return KDA_OK;
}

namespace {

// Gradient of rank-2 steps: workspace regions (256-byte aligned) for the
// sub-token problem of B x 2T tokens: q2, alpha2 [B,2T,H,d_k] and d_o2
// [B,2T,H,d_v] in the input dtype, dq2 and dalpha2 [B,2T,H,d_k] fp32, the
// doubled cu_seqlens, then the rank-1 backward's own workspace.
struct Rank2BwdLayout {
    size_t q2, a2, do2, dq2, da2, cu2, bwd, bwd_bytes, total;
};

Rank2BwdLayout rank2_bwd_layout(int dtype, int B, int T, int H, int d_k, int d_v, int has_cu, int num_seqs)
{
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    const size_t tok2 = (size_t)B * 2 * (size_t)T * H;
    Rank2BwdLayout L;
    L.q2 = 0;
    L.a2 = up(tok2 * d_k * es);
    L.do2 = L.a2 + up(tok2 * d_k * es);
    L.dq2 = L.do2 + up(tok2 * d_v * es);
    L.da2 = L.dq2 + up(tok2 * d_k * 4);
    L.cu2 = L.da2 + up(tok2 * d_k * 4);
    L.bwd = L.cu2 + up(has_cu ? (size_t)(num_seqs + 1) * 4 : 0);
    L.bwd_bytes = kda_chunk_bwd_workspace_size(dtype, B, 2 * T, H, d_k, d_v, has_cu, num_seqs);
    L.total = L.bwd + up(L.bwd_bytes);
    return L;
}

}  // namespace

extern "C" size_t kda_chunk_bwd_rank2_workspace_size(int dtype, int B, int T, int H, int d_k, int d_v,
                                                     int has_cu_seqlens, int num_seqs)
{
    if (!rank2_sizes_ok(dtype, B, T, H, d_k, d_v, has_cu_seqlens, num_seqs)) return 0;
    return rank2_bwd_layout(dtype, B, T, H, d_k, d_v, has_cu_seqlens, num_seqs).total;
}

extern "C" int kda_chunk_bwd_rank2(int variant, int gate_range, int dtype,
                                   int B, int T, int H, int d_k, int d_v,
                                   const void *q, const void *k, const void *v, const void *alpha,
                                   const void *g1, const void *g2,
                                   const int32_t *cu_seqlens, int num_seqs, const float *initial_state,
                                   const void *d_o, const float *d_final_state,
                                   float *dq, float *dk, float *dv, float *dalpha, float *dg1, float *dg2,
                                   float *d_initial_state, void *workspace, size_t workspace_bytes,
                                   unsigned flags, void *stream)
{
    if (flags) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_rank2 takes no flags (got 0x%x)", flags);
    if (B < 1 || T < 0 || H < 1 || T > (1 << 29))
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d T=%d H=%d (need B>=1, 0<=T<=2^29, H>=1)", B, T, H);
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_F32) return fail(KDA_ERR_INVALID_ARG, "bad dtype %d", dtype);
    if (!head_dim_ok(d_k) || !head_dim_ok(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "head dims d_k=%d d_v=%d: supported are 16, 32, 64, 128", d_k, d_v);
    if (!rank2_sizes_ok(dtype, B, T, H, d_k, d_v, cu_seqlens != nullptr, num_seqs))
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d T=%d H=%d num_seqs=%d (cu_seqlens needs B == 1)", B, T, H,
                    num_seqs);
    if (T > 0) {
        const void *need[] = {q, alpha, d_o, dq, dalpha, dk, dv, dg1};
        const char *names[] = {"q", "alpha", "d_o", "dq", "dalpha", "dk", "dv", "dg1"};
        for (int i = 0; i < 8; ++i) {
            if (!need[i]) return fail(KDA_ERR_INVALID_ARG, "%s is NULL", names[i]);
            if (!aligned16(need[i])) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
        }
        if (variant != KDA_VARIANT_KDA && (!dg2 || !aligned16(dg2)))
            return fail(KDA_ERR_INVALID_ARG, "dg2 is NULL or misaligned (RDA and GDN-2 have a write gate)");
    }
    if ((d_final_state && !aligned16(d_final_state)) || (d_initial_state && !aligned16(d_initial_state)))
        return fail(KDA_ERR_INVALID_ARG, "d_final_state / d_initial_state is not 16-byte aligned");
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
    const Rank2BwdLayout L = rank2_bwd_layout(dtype, B, T, H, d_k, d_v, cu_seqlens != nullptr, num_seqs);
    if (!workspace || !aligned16(workspace) || workspace_bytes < L.total)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_rank2 needs a 16-byte aligned workspace of %zu bytes",
                    L.total);
    uint8_t *w = static_cast<uint8_t *>(workspace);
    int32_t *cu2 = cu_seqlens ? reinterpret_cast<int32_t *>(w + L.cu2) : nullptr;
    // the sub-token problem's own checks (k, v, gates; variant, range, sizes) before anything is launched
    kda::FwdArgs chk;
    int rc = chunk_args(chk, variant, gate_range, dtype, B, 2 * T, H, d_k, d_v, w + L.q2, k, v, w + L.a2, g1, g2,
                        cu2, num_seqs, initial_state, nullptr, w + L.do2, 64, 0u);
    if (rc != KDA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == KDA_DTYPE_BF16;
    const long long tokens = (long long)B * T;
    cudaError_t e = kda::launch_rank2_expand(bf16, q, alpha, w + L.q2, w + L.a2, tokens, H * d_k, cu_seqlens, cu2,
                                             cu_seqlens ? num_seqs + 1 : 0, st);
    if (e == cudaSuccess) e = kda::launch_rank2_spread(bf16, d_o, w + L.do2, tokens, H * d_v, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_bwd_rank2 expand");
    // k, v and the gates (and their gradients) are already in the sub-token layout [B,2T,H,.]
    rc = kda_chunk_bwd(variant, gate_range, dtype, B, 2 * T, H, d_k, d_v, w + L.q2, k, v, w + L.a2, g1, g2, cu2,
                       num_seqs, initial_state, w + L.do2, d_final_state, reinterpret_cast<float *>(w + L.dq2), dk,
                       dv, reinterpret_cast<float *>(w + L.da2), dg1, dg2, d_initial_state, w + L.bwd, L.bwd_bytes,
                       0u, stream);
    if (rc != KDA_OK) return rc;
    e = kda::launch_rank2_gather(false, w + L.dq2, dq, tokens, H * d_k, 1, st);   // q enters the second sub-token
    if (e == cudaSuccess) e = kda::launch_rank2_gather(false, w + L.da2, dalpha, tokens, H * d_k, 0, st);   // alpha the first
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_bwd_rank2 gather");
    return KDA_OK;
}

extern "C" int kda_decode_step(int variant, int gate_range, int dtype,
                               int N, int H, int d_k, int d_v,
                               const void *q, const void *k, const void *v, const void *alpha,
                               const void *g1, const void *g2,
                               float *state, void *o, unsigned flags, void *stream)
{
    if (N < 1 || H < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes N=%d H=%d (need >= 1)", N, H);
    int rc = check_common(variant, gate_range, dtype, d_k, d_v, q, k, v, alpha, g1, g2, o, true);
    if (rc != KDA_OK) return rc;
    if (!state) return fail(KDA_ERR_INVALID_ARG, "state is NULL");
    if (!aligned16(state)) return fail(KDA_ERR_INVALID_ARG, "state is not 16-byte aligned");
    if (flags & ~(PREP_FLAGS | KDA_FLAG_VALIDATE_RANGE))
        return fail(KDA_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
    if ((unsigned long long)N * H > (1ull << 31) - 1)
        return fail(KDA_ERR_INVALID_ARG, "N*H too large for one launch");
    kda::FwdArgs a{variant, N, 1, H, d_k, d_v, q, k, v, alpha, g1, g2, nullptr, N, state, state, o,
                   prep_bits(flags), gate_range == KDA_RANGE_EXTENDED};
    if ((rc = validate(a, gate_range, dtype, flags, static_cast<cudaStream_t>(stream))) != KDA_OK) return rc;
    cudaError_t e = kda::launch_decode_step(a, dtype == KDA_DTYPE_BF16, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kda_decode_step launch");
    return KDA_OK;
}

extern "C" int kda_check_gates(int variant, int gate_range, int dtype, long long n_tok, int d_k,
                               const void *alpha, const void *g1, int *d_count, void *stream)
{
    if (variant < KDA_VARIANT_KDA || variant > KDA_VARIANT_GDN2)
        return fail(KDA_ERR_INVALID_ARG, "variant %d is not KDA(0), RDA(1) or GDN2(2)", variant);
    if (gate_range != KDA_RANGE_STANDARD && gate_range != KDA_RANGE_EXTENDED)
        return fail(KDA_ERR_INVALID_ARG, "gate_range %d is not STANDARD(0) or EXTENDED(1)", gate_range);
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_F32)
        return fail(KDA_ERR_INVALID_ARG, "dtype %d is not BF16(0) or F32(1)", dtype);
    if (n_tok < 0 || d_k < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes n_tok=%lld d_k=%d", n_tok, d_k);
    if (!d_count) return fail(KDA_ERR_INVALID_ARG, "d_count is NULL");
    if (n_tok > 0 && (!alpha || !g1)) return fail(KDA_ERR_INVALID_ARG, "alpha or g1 is NULL");
    cudaError_t e = kda::launch_check_gates(variant, gate_range, dtype == KDA_DTYPE_BF16, n_tok, d_k,
                                            alpha, g1, d_count, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kda_check_gates launch");
    return KDA_OK;
}

extern "C" int kda_check_seqlens(const int32_t *cu_seqlens, int num_seqs, long long total_tokens, int *d_count,
                                 void *stream)
{
    if (num_seqs < 1 || total_tokens < 0)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes num_seqs=%d total_tokens=%lld", num_seqs, total_tokens);
    if (!cu_seqlens || !d_count) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens or d_count is NULL");
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(d_count) & 3u))
        return fail(KDA_ERR_INVALID_ARG, "cu_seqlens or d_count is not 4-byte aligned");
    const cudaError_t e = kda::launch_check_seqlens(cu_seqlens, num_seqs, total_tokens, d_count,
                                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kda_check_seqlens launch");
    return KDA_OK;
}

extern "C" int kda_device_status(void *stream, unsigned *bits)
{
    unsigned w = 0;
    const cudaError_t e = kda::take_device_status(static_cast<cudaStream_t>(stream), &w);
    if (e != cudaSuccess) return cuda_fail(e, "kda_device_status");
    if (bits) *bits = w;
    if (w) return fail(KDA_ERR_DEVICE_TIMEOUT, "device failure bits 0x%x (%s%s)", w,
                       (w & KDA_DEVICE_WAIT_TIMEOUT) ? "a bounded wait ran out " : "",
                       (w & KDA_DEVICE_SLOT_MISSING) ? "a chunk slot was not prepared" : "");
    return KDA_OK;
}

extern "C" const char *kda_error_string(int code)
{
    switch (code) {
    case KDA_OK: return "KDA_OK: success";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: valid but unsupported size or option";
    case KDA_ERR_RANGE: return "KDA_ERR_RANGE: gate outside the declared range";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA runtime or launch failure";
    case KDA_ERR_DEVICE_TIMEOUT:
        return "KDA_ERR_DEVICE_TIMEOUT: a kernel gave up a bounded wait or found its input missing";
    }
    return "unknown kda status code";
}

extern "C" const char *kda_last_error_detail(void) { return g_detail; }

extern "C" int kda_version(void) { return 200; }
