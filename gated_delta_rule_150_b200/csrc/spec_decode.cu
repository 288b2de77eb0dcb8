// spec_decode.cu -- draft decode with per-token state retention, and rollback.
//
// "Modele hybrydowe: co Gated DeltaNet zastępuje w cache KV", section "Co stan
// rekurencyjny zmienia przy serwowaniu", point 2: a KV cache drops the
// entries of rejected draft tokens, but a recurrent state has already
// absorbed them, so speculative decoding needs the state from before the
// rejected tokens back.  The draft kernel runs K decode tokens per sequence
// from a read-only state and stores the state after every token; the accept
// kernel then copies, per sequence, the state after its last accepted token
// into the live state (or leaves it alone when nothing was accepted).
//
// Each token is the decode update of the KDA step ("kda-graft", section
// "2. Decode: O(1) против O(L)"), per state row j (value channel):
//     s' = s * a,  p = s' . k,  c = s' . (scale q),  d = beta (v_j - p)
//     s  = s' + d k,  o_j = c + d (k . scale q)
// The state rows stay in registers across the K tokens: the kernel reads the
// state once and writes it K times, so it is HBM-bound on
// (1 + K) * 4 d_v d_k bytes per head-state plus the tokens' inputs.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace gdr {
namespace {

constexpr int kThreads = 256;
constexpr int kTPR = 16;                      // threads per state row
constexpr int kRowsPerPass = kThreads / kTPR; // 16 rows at a time

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float sum16(float x) {
#pragma unroll
    for (int m = 8; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

// Four consecutive elements as loaded (16-byte aligned for fp32, 8 for
// bf16), converted where they are used: the next token's loads are issued
// before this token is computed, and a conversion right after a load would
// wait for it there (5 % faster draft than converting at the load).
template <typename T> struct Raw4;
template <> struct Raw4<float> {
    float4 u;
    __device__ __forceinline__ void load(const float* p) { u = __ldg(reinterpret_cast<const float4*>(p)); }
    __device__ __forceinline__ float4 get() const { return u; }
};
template <> struct Raw4<__nv_bfloat16> {
    uint2 u;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint2*>(p)); }
    __device__ __forceinline__ float4 get() const {
        const float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y);
        return make_float4(a.x, a.y, b.x, b.y);
    }
};

// One token's inputs as seen by one thread, as loaded: its float4 columns of
// k, q and log a (a scalar gate: la[0].x), the v entries of its rows (PASSES
// rows from row0, 16 apart), and beta.
template <typename T, int DK, int DV, int PASSES, bool SCALAR>
struct TokenIn {
    static constexpr int NV = DK / (4 * kTPR);
    Raw4<T> k[NV], q[NV];
    float4 la[NV];
    T v[PASSES];
    float beta;
    __device__ __forceinline__ float4 decay(int i) const {
        const float4 x = SCALAR ? make_float4(la[0].x, la[0].x, la[0].x, la[0].x) : la[i];
        return make_float4(expf(x.x), expf(x.y), expf(x.z), expf(x.w));
    }

    __device__ __forceinline__ void load(const T* __restrict__ q_, const T* __restrict__ k_,
                                         const T* __restrict__ v_, const float* __restrict__ beta_,
                                         const float* __restrict__ log_a_, size_t tok, int lane16,
                                         int row0) {
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int c = 4 * (lane16 + kTPR * i);
            k[i].load(k_ + tok * DK + c);
            q[i].load(q_ + tok * DK + c);
            if (!SCALAR) la[i] = __ldg(reinterpret_cast<const float4*>(log_a_ + tok * DK + c));
        }
        if (SCALAR) la[0].x = __ldg(log_a_ + tok);
#pragma unroll
        for (int p = 0; p < PASSES; ++p) v[p] = v_[tok * DV + row0 + kRowsPerPass * p];
        beta = __ldg(beta_ + tok);
    }
};

// RS CTAs per (sequence b, head h), CTA part j owning the state rows
// [j DV / RS, (j + 1) DV / RS) (rows are independent given the token).  Thread
// t owns rows row0 + t / 16 + 16 p and the float4 columns {t % 16 + 16 i} of
// the state for all K tokens.  Token t of sequence b is input row
// (b K + t) H + h of q, k, v, beta, log a, o and token_states; the next
// token's inputs are loaded while this one computes.
// At d 64 the kernel is capped at 64 registers so that four CTAs fit on an SM
// (7 % faster on B200 than three CTAs at 78 registers; the fp32 per-channel
// case spills 68 bytes); wider states keep their registers.
template <int DK, int DV>
constexpr int draft_min_ctas() { return (DK == 64 && DV == 64) ? 4 : 1; }

template <typename T, int DK, int DV, bool SCALAR, int RS>
__global__ void __launch_bounds__(kThreads, draft_min_ctas<DK, DV>())
decode_draft_kernel(int H, int K, const T* __restrict__ q, const T* __restrict__ k,
                    const T* __restrict__ v, const float* __restrict__ beta,
                    const float* __restrict__ log_a, float scale, const float* __restrict__ state,
                    float* __restrict__ o, float* __restrict__ token_states) {
    constexpr int PASSES = DV / (RS * kRowsPerPass);
    static_assert(PASSES >= 1 && PASSES * RS * kRowsPerPass == DV, "row split");
    pdl_launch_dependents();
    pdl_wait();                                // the previous kernel's writes are visible
    using Tok = TokenIn<T, DK, DV, PASSES, SCALAR>;
    constexpr int NV = Tok::NV;
    const int bh = blockIdx.x / RS;
    const int part = blockIdx.x - bh * RS;
    const int b = bh / H;
    const int h = bh - b * H;
    const int lane16 = threadIdx.x % kTPR;
    const int row0 = part * (DV / RS) + threadIdx.x / kTPR;

    const size_t tok0 = (size_t)b * K * H + h;
    Tok nxt;
    nxt.load(q, k, v, beta, log_a, tok0, lane16, row0);

    const float* S0 = state + (size_t)bh * DV * DK;
    float4 s[PASSES][NV];
#pragma unroll
    for (int p = 0; p < PASSES; ++p)
#pragma unroll
        for (int i = 0; i < NV; ++i)
            s[p][i] = __ldg(reinterpret_cast<const float4*>(
                S0 + (size_t)(row0 + kRowsPerPass * p) * DK + 4 * (lane16 + kTPR * i)));

#pragma unroll 1
    for (int t = 0; t < K; ++t) {
        const Tok cur = nxt;
        const size_t tok = tok0 + (size_t)t * H;
        if (t + 1 < K) nxt.load(q, k, v, beta, log_a, tok + H, lane16, row0);

        float4 aa[NV], qq[NV], kk[NV];
        float kq_part = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            aa[i] = cur.decay(i);
            const float4 qv = cur.q[i].get();
            kk[i] = cur.k[i].get();
            qq[i] = make_float4(qv.x * scale, qv.y * scale, qv.z * scale, qv.w * scale);
            kq_part += kk[i].x * qq[i].x + kk[i].y * qq[i].y + kk[i].z * qq[i].z + kk[i].w * qq[i].w;
        }
        const float kq = sum16(kq_part);

        float* St = token_states + tok * DV * DK;
#pragma unroll
        for (int p = 0; p < PASSES; ++p) {
            const int row = row0 + kRowsPerPass * p;
            // column pairs on packed fp32 (__fmul2_rn, __ffma2_rn; the k and q
            // dot products summed as two interleaved halves): 1 % faster
            float2 pk2 = make_float2(0.f, 0.f), pq2 = make_float2(0.f, 0.f);
            float2 xl[NV], xh[NV];
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const float4 x = s[p][i];
                xl[i] = __fmul2_rn(make_float2(x.x, x.y), make_float2(aa[i].x, aa[i].y));
                xh[i] = __fmul2_rn(make_float2(x.z, x.w), make_float2(aa[i].z, aa[i].w));
                pk2 = __ffma2_rn(xl[i], make_float2(kk[i].x, kk[i].y), pk2);
                pk2 = __ffma2_rn(xh[i], make_float2(kk[i].z, kk[i].w), pk2);
                pq2 = __ffma2_rn(xl[i], make_float2(qq[i].x, qq[i].y), pq2);
                pq2 = __ffma2_rn(xh[i], make_float2(qq[i].z, qq[i].w), pq2);
            }
            const float pk = sum16(pk2.x + pk2.y);
            const float pq = sum16(pq2.x + pq2.y);
            const float d = cur.beta * (to_f<T>(cur.v[p]) - pk);
            const float2 d2 = make_float2(d, d);
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const float2 lo = __ffma2_rn(d2, make_float2(kk[i].x, kk[i].y), xl[i]);
                const float2 hi = __ffma2_rn(d2, make_float2(kk[i].z, kk[i].w), xh[i]);
                s[p][i] = make_float4(lo.x, lo.y, hi.x, hi.y);
                // kept states are written once and mostly never read again
                __stcs(reinterpret_cast<float4*>(St + (size_t)row * DK + 4 * (lane16 + kTPR * i)), s[p][i]);
            }
            if (lane16 == 0) o[tok * DV + row] = pq + d * kq;
        }
    }
}

// One CTA per (sequence b, head h): state[b, h] = token_states[b, n - 1, h]
// with n = n_accept[b] clamped to [0, K]; nothing happens for n = 0.
__global__ void __launch_bounds__(kThreads)
decode_accept_kernel(int H, int K, int n4, const int32_t* __restrict__ n_accept,
                     const float* __restrict__ token_states, float* __restrict__ state) {
    pdl_launch_dependents();
    pdl_wait();                                // the draft's kept states are visible
    const int bh = blockIdx.x;
    const int b = bh / H;
    const int h = bh - b * H;
    int n = __ldg(n_accept + b);
    n = n < 0 ? 0 : (n > K ? K : n);
    if (n == 0) return;
    const float4* src = reinterpret_cast<const float4*>(token_states) +
                        (((size_t)b * K + (n - 1)) * H + h) * (size_t)n4;
    float4* dst = reinterpret_cast<float4*>(state) + (size_t)bh * n4;
    constexpr int kUnroll = 4;
    for (int base = threadIdx.x; base < n4; base += kThreads * kUnroll) {
        float4 x[kUnroll];
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            const int i = base + j * kThreads;
            if (i < n4) x[j] = __ldcs(src + i);
        }
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            const int i = base + j * kThreads;
            if (i < n4) dst[i] = x[j];
        }
    }
}

// CTAs per head-state of the draft kernel (splitting the rows over 2 or 4
// CTAs measured 8 % and 47 % slower at d 64: each CTA repeats the token's
// inputs and k . q).
constexpr int kRowSplit = 1;

template <typename T, int DK, int DV>
cudaError_t draft_typed(int B, int K, int H, const void* q, const void* k, const void* v,
                        const float* beta, const float* log_a, int scalar, float scale,
                        const float* state, float* o, float* ts, cudaStream_t st) {
    const dim3 grid((unsigned)((int64_t)B * H * kRowSplit));
    if (scalar)
        return launch_pdl(true, decode_draft_kernel<T, DK, DV, true, kRowSplit>, grid, dim3(kThreads), 0,
                          st, H, K, (const T*)q, (const T*)k, (const T*)v, beta, log_a, scale, state, o, ts);
    return launch_pdl(true, decode_draft_kernel<T, DK, DV, false, kRowSplit>, grid, dim3(kThreads), 0, st,
                      H, K, (const T*)q, (const T*)k, (const T*)v, beta, log_a, scale, state, o, ts);
}

template <typename T>
cudaError_t draft_dims(int B, int K, int H, int dk, int dv, const void* q, const void* k,
                       const void* v, const float* beta, const float* log_a, int scalar,
                       float scale, const float* state, float* o, float* ts, cudaStream_t st) {
    if (dk == 64 && dv == 64)
        return draft_typed<T, 64, 64>(B, K, H, q, k, v, beta, log_a, scalar, scale, state, o, ts, st);
    if (dk == 64 && dv == 128)
        return draft_typed<T, 64, 128>(B, K, H, q, k, v, beta, log_a, scalar, scale, state, o, ts, st);
    if (dk == 128 && dv == 64)
        return draft_typed<T, 128, 64>(B, K, H, q, k, v, beta, log_a, scalar, scale, state, o, ts, st);
    return draft_typed<T, 128, 128>(B, K, H, q, k, v, beta, log_a, scalar, scale, state, o, ts, st);
}

}  // namespace

cudaError_t launch_decode_draft(int B, int K, int H, int dk, int dv, gdr_dtype dt, const void* q,
                                const void* k, const void* v, const float* beta,
                                const float* log_a, int scalar, float scale, const float* state,
                                float* o, float* token_states, cudaStream_t st) {
    if (dt == GDR_BF16)
        return draft_dims<__nv_bfloat16>(B, K, H, dk, dv, q, k, v, beta, log_a, scalar, scale,
                                         state, o, token_states, st);
    return draft_dims<float>(B, K, H, dk, dv, q, k, v, beta, log_a, scalar, scale, state, o,
                             token_states, st);
}

cudaError_t launch_decode_accept(int B, int K, int H, int dk, int dv, const int32_t* n_accept,
                                 const float* token_states, float* state, cudaStream_t st) {
    return launch_pdl(true, decode_accept_kernel, dim3((unsigned)(B * H)), dim3(kThreads), 0, st, H, K,
                      dk * dv / 4, n_accept, token_states, state);
}

}  // namespace gdr
