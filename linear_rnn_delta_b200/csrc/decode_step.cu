// Single-token decode step: stream the fp32 state once, in place.
//
// The decode state is fixed-size in the sequence length (openarchlab page on
// GDN/KDA state updates, sec. 1 and 3), so a step is one read and one write
// of N*H*d_k*d_v fp32 values plus a few vectors per head: HBM-bound.  The
// delta rule's error-correcting write needs the prediction S'^T a~ before the
// update, and the readout needs S_t^T q; both reductions over d_k are taken
// in the SAME pass over the decayed state S' = Diag(alpha) S, because
//   o = S_t^T q = S'^T q + (k.q) u,   u = m - S'^T a~,
// so the state is read once and written once.
//
// One CTA per (sequence, head).  Thread layout for d_v = 128: each warp owns
// a block of rows, lane l owns columns 4l..4l+3 (one 16-byte load per row,
// a full 512-byte row per warp instruction).  Each thread keeps its slice of
// S in registers between the read and the write.  Partial sums of the two
// reductions go through shared memory across warps.
#include "common.cuh"

namespace kda {
namespace {

template <int DK, int DV>
struct DecodeShape {
    static constexpr int THREADS = (DK * DV / 4 >= 256) ? 256 : DK * DV / 4;
    static constexpr int CT = DV / 4;          // threads per row (one float4 each)
    static constexpr int RP = THREADS / CT;    // rows covered per pass
    static constexpr int RPT = DK / RP;        // rows per thread
    static_assert(RPT * RP == DK, "rows must divide evenly");
};

// PREP: input preparation requested; without it that code is compiled out.
template <int DK, int DV, typename TIn, bool PREP>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::THREADS)
decode_step_kernel(FwdArgs a)
{
    using Sh = DecodeShape<DK, DV>;
    constexpr int RP = Sh::RP, RPT = Sh::RPT, CT = Sh::CT;
    __shared__ __align__(16) float s_q[DK], s_k[DK], s_al[DK], s_at[DK], s_m[DV];
    __shared__ __align__(16) float s_red[2][RP][DV];
    __shared__ float s_u[DV], s_p[DV], s_kq, s_ksc;

    const int nh = blockIdx.x;
    const int tid = threadIdx.x;
    const int c4 = tid % CT, rg = tid / CT;
    float4 *S4 = reinterpret_cast<float4 *>(a.sf) + (size_t)nh * (DK * DV / 4);

    // 1. put the whole state slice in flight first
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) s[r] = __ldcs(S4 + (size_t)(rg + r * RP) * CT + c4);

    // 2. token vectors -> shared (fp32)
    const TIn *q = (const TIn *)a.q + (size_t)nh * DK, *k = (const TIn *)a.k + (size_t)nh * DK;
    const TIn *al = (const TIn *)a.alpha + (size_t)nh * DK, *v = (const TIn *)a.v + (size_t)nh * DV;
    const TIn *g1 = (const TIn *)a.g1, *g2 = (const TIn *)a.g2;
    const bool logits = PREP && (a.prep & PREP_LOGITS), l2k = PREP && (a.prep & PREP_L2NORM_K), ext = a.ext != 0;
    auto erase_gate = [&](int i) {   // beta / e, or GDN-2's b_i (activated from its logit on request)
        const float g = (a.variant == GDN2) ? ld_f32(g1 + (size_t)nh * DK + i) : ld_f32(g1 + nh);
        return logits ? round_to<TIn>(prep_gate(g, ext)) : g;
    };
    for (int i = tid; i < DK; i += Sh::THREADS) {
        const float kk = ld_f32(k + i);
        float ai = ld_f32(al + i);
        if (logits) ai = round_to<TIn>(prep_alpha(ai, ext));
        s_q[i] = ld_f32(q + i);
        s_k[i] = kk;
        s_al[i] = ai;
        s_at[i] = erase_gate(i) * kk;
    }
    for (int j = tid; j < DV; j += Sh::THREADS) {
        float g;
        if (a.variant == KDA) g = ld_f32(g1 + nh);
        else if (a.variant == RDA) g = ld_f32(g2 + nh);
        else g = ld_f32(g2 + (size_t)nh * DV + j);
        if (logits) g = round_to<TIn>(prep_gate(g, ext));
        s_m[j] = g * ld_f32(v + j);
    }
    __syncthreads();
    if (l2k) {   // k / ||k|| (rounded to the input dtype); a~ = g (.) k with the normalised k
        if (tid < 32) {
            float ss = 0.f;
            for (int i = tid; i < DK; i += 32) ss = fmaf(s_k[i], s_k[i], ss);
#pragma unroll
            for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            if (tid == 0) s_ksc = prep_kscale(ss);
        }
        __syncthreads();
        for (int i = tid; i < DK; i += Sh::THREADS) {
            const float kn = round_to<TIn>(s_k[i] * s_ksc);
            s_k[i] = kn;
            s_at[i] = erase_gate(i) * kn;
        }
        __syncthreads();
    }

    // 3. decay in registers; partial S'^T a~ and S'^T q over this thread's rows
    float pu[4] = {0.f, 0.f, 0.f, 0.f}, pp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg + r * RP;
        const float ai = s_al[i], ti = s_at[i], qi = s_q[i];
        s[r].x *= ai; s[r].y *= ai; s[r].z *= ai; s[r].w *= ai;
        pu[0] = fmaf(s[r].x, ti, pu[0]); pu[1] = fmaf(s[r].y, ti, pu[1]);
        pu[2] = fmaf(s[r].z, ti, pu[2]); pu[3] = fmaf(s[r].w, ti, pu[3]);
        pp[0] = fmaf(s[r].x, qi, pp[0]); pp[1] = fmaf(s[r].y, qi, pp[1]);
        pp[2] = fmaf(s[r].z, qi, pp[2]); pp[3] = fmaf(s[r].w, qi, pp[3]);
    }
    *reinterpret_cast<float4 *>(&s_red[0][rg][4 * c4]) = make_float4(pu[0], pu[1], pu[2], pu[3]);
    *reinterpret_cast<float4 *>(&s_red[1][rg][4 * c4]) = make_float4(pp[0], pp[1], pp[2], pp[3]);
    if (tid < 32) {  // k.q by warp 0
        float kq = 0.f;
        for (int i = tid; i < DK; i += 32) kq = fmaf(s_k[i], s_q[i], kq);
#pragma unroll
        for (int off = 16; off; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (tid == 0) s_kq = kq;
    }
    __syncthreads();

    // 4. finish the two reductions: u = m - S'^T a~,  p = S'^T q
    for (int e = tid; e < 2 * DV; e += Sh::THREADS) {
        const int which = e / DV, j = e % DV;
        float acc = 0.f;
#pragma unroll 8
        for (int g = 0; g < RP; ++g) acc += s_red[which][g][j];
        if (which == 0) s_u[j] = s_m[j] - acc;
        else s_p[j] = acc;
    }
    __syncthreads();

    // 5. S = S' + k u^T, written back in place; o = p + (k.q) u
    const float4 u4 = *reinterpret_cast<const float4 *>(&s_u[4 * c4]);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg + r * RP;
        const float ki = s_k[i];
        float4 x = s[r];
        x.x = fmaf(ki, u4.x, x.x); x.y = fmaf(ki, u4.y, x.y);
        x.z = fmaf(ki, u4.z, x.z); x.w = fmaf(ki, u4.w, x.w);
        __stcs(S4 + (size_t)i * CT + c4, x);
    }
    for (int j = tid; j < DV; j += Sh::THREADS)
        st_out((TIn *)a.o + (size_t)nh * DV + j, fmaf(s_kq, s_u[j], s_p[j]));
}

template <int DK, int DV>
cudaError_t launch_dims(const FwdArgs &a, bool bf16, cudaStream_t st)
{
    dim3 grid((unsigned)(a.B * a.H)), block(DecodeShape<DK, DV>::THREADS);
    if (bf16) {
        if (a.prep) decode_step_kernel<DK, DV, __nv_bfloat16, true><<<grid, block, 0, st>>>(a);
        else decode_step_kernel<DK, DV, __nv_bfloat16, false><<<grid, block, 0, st>>>(a);
    } else {
        if (a.prep) decode_step_kernel<DK, DV, float, true><<<grid, block, 0, st>>>(a);
        else decode_step_kernel<DK, DV, float, false><<<grid, block, 0, st>>>(a);
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

// a.B carries N (sequences in the step); a.sf is the in-place state.
cudaError_t launch_decode_step(const FwdArgs &a, bool bf16, cudaStream_t st)
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
