// preprocess.cu -- the recurrence's inputs from raw per-head projections, in
// one pass: width-4 causal depthwise conv on q, k and v, L2 norm of q and k,
// beta = sigmoid(beta_raw), log a = log_sigmoid(a_raw + a_bias).
//
// "kda-graft: Qwen2.5-0.5B с трансплантированным KDA", section "Идея и
// архитектура": the graft adds a width-4 convolution (initialised as an
// identity tap), the alpha gate with bias +5 and the write strength beta
// around the q/k/v projections.  Readings: no activation after the conv, q and
// k normalised per (token, head) after it as y / max(||y||, 1e-12), the conv
// restarting from zero history at every sequence start.
//
// Layout of the work: one warp per (head, span of kSpan tokens).  Lane l
// owns channels [l C, l C + C) of the head, C = D / 32 (2 at d 64, 4 at
// d 128), so a warp's access to one (token, head) row of x_q, x_k, x_v, q, k,
// v or log a is one contiguous, coalesced row.  The lane keeps its channels'
// conv taps in registers and walks the span's tokens in order with the last
// three raw rows of x_q, x_k and x_v in a register window, so every raw row
// is read from memory once (plus a three-row halo per span); the window is
// cleared at every sequence start.  Loads run kPref tokens ahead of the
// arithmetic.  L2 norms are warp sums.  The HBM traffic is x_q, x_k, x_v,
// beta_raw and a_raw read and q, k, v, beta, log a written, once each.
#include <cuda_bf16.h>

#include "internal.h"

namespace gdr {
namespace {

constexpr int kThreads = 256;

constexpr int kSpan = 32;          // tokens per warp
constexpr int kPref = 4;           // tokens of loads in flight ahead of the arithmetic

// C consecutive channels of one row, as loaded (bf16 or fp32).
template <typename T, int C> struct RowC;
template <> struct RowC<__nv_bfloat16, 2> {
    uint32_t u;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint32_t*>(p)); }
    __device__ __forceinline__ void get(float* x) const {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
        x[0] = f.x; x[1] = f.y;
    }
};
template <> struct RowC<__nv_bfloat16, 4> {
    uint2 u;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint2*>(p)); }
    __device__ __forceinline__ void get(float* x) const {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    }
};
template <> struct RowC<float, 2> {
    float2 u;
    __device__ __forceinline__ void load(const float* p) { u = __ldg(reinterpret_cast<const float2*>(p)); }
    __device__ __forceinline__ void get(float* x) const { x[0] = u.x; x[1] = u.y; }
};
template <> struct RowC<float, 4> {
    float4 u;
    __device__ __forceinline__ void load(const float* p) { u = __ldg(reinterpret_cast<const float4*>(p)); }
    __device__ __forceinline__ void get(float* x) const { x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w; }
};

template <int C> __device__ __forceinline__ void storeC(float* p, const float* x);
template <> __device__ __forceinline__ void storeC<2>(float* p, const float* x) {
    *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
}
template <> __device__ __forceinline__ void storeC<4>(float* p, const float* x) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
template <int C> __device__ __forceinline__ void storeC(__nv_bfloat16* p, const float* x);
template <> __device__ __forceinline__ void storeC<2>(__nv_bfloat16* p, const float* x) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(x[0], x[1]);
    *reinterpret_cast<__nv_bfloat162*>(p) = b;
}
template <> __device__ __forceinline__ void storeC<4>(__nv_bfloat16* p, const float* x) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&a);
    u.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

__device__ __forceinline__ float log_sigmoid(float z) {
    return fminf(z, 0.f) - log1pf(expf(-fabsf(z)));
}

__device__ __forceinline__ float sigmoid(float z) {
    const float e = expf(-fabsf(z));
    return z >= 0.f ? 1.0f / (1.0f + e) : e / (1.0f + e);
}

// Inputs of one token for one lane, as loaded.
template <typename T, int C, bool SCALAR>
struct TokenIn {
    RowC<T, C> xq, xk, xv;
    RowC<float, C> a;          // a_raw (per-channel gate)
    float a_s, b;              // a_raw (scalar gate), beta_raw
    __device__ __forceinline__ void load(const T* xq_, const T* xk_, const T* xv_,
                                         const float* a_raw, const float* beta_raw, int64_t t,
                                         int H, int h, int c0) {
        const size_t off = ((size_t)t * H + h) * (C * 32) + c0;
        xq.load(xq_ + off);
        xk.load(xk_ + off);
        xv.load(xv_ + off);
        if (SCALAR) a_s = __ldg(a_raw + (size_t)t * H + h);
        else a.load(a_raw + off);
        b = __ldg(beta_raw + (size_t)t * H + h);
    }
};

// Causal width-4 conv of one lane's channels with a window of the three
// previous raw rows (w0 = oldest): y = w[0] x_{t-3} + w[1] x_{t-2} +
// w[2] x_{t-1} + w[3] x_t, then the window advances.
template <int C>
__device__ __forceinline__ void conv_step(const float (&w)[C][4], float (&win)[3][C],
                                          const float* x, float* y) {
#pragma unroll
    for (int e = 0; e < C; ++e) {
        float acc = w[e][3] * x[e];
        acc = fmaf(w[e][2], win[2][e], acc);
        acc = fmaf(w[e][1], win[1][e], acc);
        acc = fmaf(w[e][0], win[0][e], acc);
        y[e] = acc;
        win[0][e] = win[1][e];
        win[1][e] = win[2][e];
        win[2][e] = x[e];
    }
}

template <typename T, int D, bool SCALAR>
__global__ void __launch_bounds__(kThreads)
preprocess_kernel(int n_seqs, int H, int64_t T_tot, int64_t n_units, const int32_t* __restrict__ cu,
                  const T* __restrict__ xq, const T* __restrict__ xk, const T* __restrict__ xv,
                  const float* __restrict__ wq, const float* __restrict__ wk,
                  const float* __restrict__ wv, const float* __restrict__ beta_raw,
                  const float* __restrict__ a_raw, const float* __restrict__ a_bias,
                  T* __restrict__ q, T* __restrict__ k, T* __restrict__ v,
                  float* __restrict__ beta, float* __restrict__ log_a) {
    constexpr int C = D / 32;                  // channels per lane
    const int lane = threadIdx.x & 31;
    const int64_t unit = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / 32;
    if (unit >= n_units) return;               // whole warps leave together
    const int h = (int)(unit % H);
    const int64_t t0 = (unit / H) * kSpan;
    const int64_t t1 = t0 + kSpan < T_tot ? t0 + kSpan : T_tot;
    const int c0 = C * lane;

    // this lane's taps and gate bias
    float tq[C][4], tk[C][4], tv[C][4], bias[C];
#pragma unroll
    for (int e = 0; e < C; ++e) {
        const size_t r = ((size_t)h * D + c0 + e) * 4;
        const float4 fq = __ldg(reinterpret_cast<const float4*>(wq + r));
        const float4 fk = __ldg(reinterpret_cast<const float4*>(wk + r));
        const float4 fv = __ldg(reinterpret_cast<const float4*>(wv + r));
        tq[e][0] = fq.x; tq[e][1] = fq.y; tq[e][2] = fq.z; tq[e][3] = fq.w;
        tk[e][0] = fk.x; tk[e][1] = fk.y; tk[e][2] = fk.z; tk[e][3] = fk.w;
        tv[e][0] = fv.x; tv[e][1] = fv.y; tv[e][2] = fv.z; tv[e][3] = fv.w;
        bias[e] = SCALAR ? 0.f : __ldg(a_bias + (size_t)h * D + c0 + e);
    }
    const float bias_s = SCALAR ? __ldg(a_bias + h) : 0.f;

    // the sequence holding t0: the largest n with cu[n] <= t0
    int n = 0;
    {
        int lo = 0, hi = n_seqs - 1;
        while (lo <= hi) {
            const int mid = (lo + hi) >> 1;
            if ((int64_t)__ldg(cu + mid) <= t0) { n = mid; lo = mid + 1; } else { hi = mid - 1; }
        }
    }
    const int64_t s = __ldg(cu + n);
    int64_t next = __ldg(cu + n + 1);          // start of the next sequence

    // window: the three raw rows before t0 that belong to t0's sequence
    float wq_[3][C], wk_[3][C], wv_[3][C];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int64_t tt = t0 - 3 + j;
        if (tt >= s) {
            RowC<T, C> a, b, c;
            const size_t off = ((size_t)tt * H + h) * D + c0;
            a.load(xq + off); b.load(xk + off); c.load(xv + off);
            a.get(wq_[j]); b.get(wk_[j]); c.get(wv_[j]);
        } else {
#pragma unroll
            for (int e = 0; e < C; ++e) wq_[j][e] = wk_[j][e] = wv_[j][e] = 0.f;
        }
    }

    // loads kPref tokens ahead (ring of kPref slots, index t % kPref)
    TokenIn<T, C, SCALAR> ring[kPref];
#pragma unroll
    for (int i = 0; i < kPref; ++i)
        if (t0 + i < t1) ring[i].load(xq, xk, xv, a_raw, beta_raw, t0 + i, H, h, c0);

    for (int64_t tb = t0; tb < t1; tb += kPref) {
#pragma unroll
        for (int i = 0; i < kPref; ++i) {
            const int64_t t = tb + i;
            if (t >= t1) break;
            const TokenIn<T, C, SCALAR> in = ring[i];
            if (t + kPref < t1) ring[i].load(xq, xk, xv, a_raw, beta_raw, t + kPref, H, h, c0);
            if (t == next) {                   // a sequence starts here: clear the window
                while (n + 1 < n_seqs && (int64_t)__ldg(cu + n + 1) <= t) ++n;
                next = __ldg(cu + n + 1);
#pragma unroll
                for (int j = 0; j < 3; ++j)
#pragma unroll
                    for (int e = 0; e < C; ++e) wq_[j][e] = wk_[j][e] = wv_[j][e] = 0.f;
            }
            float x[C], yq[C], yk[C], yv[C];
            in.xq.get(x); conv_step<C>(tq, wq_, x, yq);
            in.xk.get(x); conv_step<C>(tk, wk_, x, yk);
            in.xv.get(x); conv_step<C>(tv, wv_, x, yv);
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int e = 0; e < C; ++e) { sq = fmaf(yq[e], yq[e], sq); sk = fmaf(yk[e], yk[e], sk); }
            sq = warp_sum(sq);
            sk = warp_sum(sk);
            const float iq = 1.0f / fmaxf(sqrtf(sq), 1e-12f), ik = 1.0f / fmaxf(sqrtf(sk), 1e-12f);
#pragma unroll
            for (int e = 0; e < C; ++e) { yq[e] *= iq; yk[e] *= ik; }
            const size_t row = ((size_t)t * H + h) * D + c0;
            storeC<C>(q + row, yq);
            storeC<C>(k + row, yk);
            storeC<C>(v + row, yv);
            if (SCALAR) {
                if (lane == 0) log_a[(size_t)t * H + h] = log_sigmoid(in.a_s + bias_s);
            } else {
                float z[C];
                in.a.get(z);
#pragma unroll
                for (int e = 0; e < C; ++e) z[e] = log_sigmoid(z[e] + bias[e]);
                storeC<C>(log_a + row, z);
            }
            if (lane == 1) beta[(size_t)t * H + h] = sigmoid(in.b);
        }
    }
}

template <typename T, int D>
cudaError_t launch_typed(const gdr_preprocess_args& a, cudaStream_t st) {
    const int64_t spans = (a.total_tokens + kSpan - 1) / kSpan;
    const int64_t n_units = spans * a.n_heads;             // one warp each
    const int64_t blocks = (n_units + kThreads / 32 - 1) / (kThreads / 32);
    if (blocks > (int64_t)INT32_MAX) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)blocks);
    auto* xq = static_cast<const T*>(a.xq);
    auto* xk = static_cast<const T*>(a.xk);
    auto* xv = static_cast<const T*>(a.xv);
    auto* q = static_cast<T*>(a.q);
    auto* k = static_cast<T*>(a.k);
    auto* v = static_cast<T*>(a.v);
    if (a.scalar_decay)
        preprocess_kernel<T, D, true><<<grid, kThreads, 0, st>>>(
            a.n_seqs, a.n_heads, a.total_tokens, n_units, a.cu_seqlens, xq, xk, xv, a.conv_q,
            a.conv_k, a.conv_v, a.beta_raw, a.a_raw, a.a_bias, q, k, v, a.beta, a.log_a);
    else
        preprocess_kernel<T, D, false><<<grid, kThreads, 0, st>>>(
            a.n_seqs, a.n_heads, a.total_tokens, n_units, a.cu_seqlens, xq, xk, xv, a.conv_q,
            a.conv_k, a.conv_v, a.beta_raw, a.a_raw, a.a_bias, q, k, v, a.beta, a.log_a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_preprocess(const gdr_preprocess_args& a, cudaStream_t st) {
    if (a.io_dtype == GDR_BF16)
        return a.d == 64 ? launch_typed<__nv_bfloat16, 64>(a, st)
                         : launch_typed<__nv_bfloat16, 128>(a, st);
    return a.d == 64 ? launch_typed<float, 64>(a, st) : launch_typed<float, 128>(a, st);
}

}  // namespace gdr
