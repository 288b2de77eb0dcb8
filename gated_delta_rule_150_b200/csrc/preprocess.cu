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
// Layout of the work: D / 8 consecutive threads own one (token, head) and
// eight consecutive channels each, so a warp reads and writes whole
// contiguous rows of [T, H, D].  Each thread reads its channels of the
// current token and up to three earlier ones of the same sequence (the
// earlier rows were just read by neighbouring warps and come from L1/L2, so
// HBM sees each row about once).  The tap loads are unconditional (a tap
// before the sequence start reads the current row and is then skipped), so
// all twelve are in flight together instead of one after another.  The L2
// norms are shuffle sums over the D / 8 lanes of a (token, head).  The HBM
// traffic is x_q, x_k, x_v, beta_raw, a_raw read and q, k, v, beta, log a
// written, once each; the conv taps' per-thread loads (eight 16-byte loads
// whose lanes sit 128 bytes apart) cost more L1 wavefronts than that traffic
// takes in HBM time, so the kernel is L1-bound at d 64.
#include <cuda_bf16.h>

#include "internal.h"

namespace gdr {
namespace {

constexpr int kThreads = 256;

// Eight consecutive fp32 values from p (16-byte aligned).
__device__ __forceinline__ void load8(const float* p, float* x) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void store8(float* p, const float* x) {
    reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* x) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// First token of the sequence holding token t: cu[n] for the largest n with
// cu[n] <= t (empty sequences share their start with the next one).
__device__ __forceinline__ int64_t seq_start(const int32_t* __restrict__ cu, int n_seqs,
                                             int64_t t) {
    int lo = 0, hi = n_seqs - 1, found = 0;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        if ((int64_t)__ldg(cu + mid) <= t) { found = mid; lo = mid + 1; } else { hi = mid - 1; }
    }
    return __ldg(cu + found);
}

// Eight consecutive raw values of x_q / x_k / x_v, held as loaded (16 bytes
// of bf16 or 32 bytes of fp32) until the conv uses them.
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) {
        u = __ldg(reinterpret_cast<const uint4*>(p));
    }
    __device__ __forceinline__ void to_f32(float* x) const {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
        }
    }
};
template <>
struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = __ldg(reinterpret_cast<const float4*>(p));
        b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void to_f32(float* x) const {
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};

// y[0..7] = sum over the taps j = 0..3 with t - 3 + j >= s of
// w[c][j] * x[t - 3 + j][c], c = c0 .. c0 + 7 (w row-major [H D, 4]); r[j]
// holds tap j's values (any row when the tap is before the sequence start).
template <typename T, int D>
__device__ __forceinline__ void conv4(const Raw8<T> (&r)[4], const float* __restrict__ w,
                                      int64_t t, int64_t s, int h, int c0, float* y) {
    float wt[8][4];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(w + ((size_t)h * D + c0 + e) * 4));
        wt[e][0] = f.x; wt[e][1] = f.y; wt[e][2] = f.z; wt[e][3] = f.w;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (t - 3 + j >= s) {
            float x[8];
            r[j].to_f32(x);
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = fmaf(wt[e][j], x[e], y[e]);
        }
    }
}

// Sum over the G = D / 8 lanes of this (token, head) group (G divides 32 and
// groups are G-aligned, so xor offsets below G stay inside the group).
template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int m = G / 2; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

template <int G>
__device__ __forceinline__ void l2_normalise(float* y) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(y[e], y[e], ss);
    ss = group_sum<G>(ss);
    const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] *= inv;
}

__device__ __forceinline__ float log_sigmoid(float z) {
    return fminf(z, 0.f) - log1pf(expf(-fabsf(z)));
}

__device__ __forceinline__ float sigmoid(float z) {
    const float e = expf(-fabsf(z));
    return z >= 0.f ? 1.0f / (1.0f + e) : e / (1.0f + e);
}

// Grid-stride over (token, head) units, warp-uniform: every lane of a warp
// runs the same iterations; lanes past the end work on the last unit (so
// every address is valid), join the shuffles and store nothing.  All global
// loads of an iteration are issued before any of them is used.
template <typename T, int D, bool SCALAR>
__global__ void __launch_bounds__(kThreads, 2)
preprocess_kernel(int n_seqs, int H, int64_t units, const int32_t* __restrict__ cu,
                  const T* __restrict__ xq, const T* __restrict__ xk, const T* __restrict__ xv,
                  const float* __restrict__ wq, const float* __restrict__ wk,
                  const float* __restrict__ wv, const float* __restrict__ beta_raw,
                  const float* __restrict__ a_raw, const float* __restrict__ a_bias,
                  T* __restrict__ q, T* __restrict__ k, T* __restrict__ v,
                  float* __restrict__ beta, float* __restrict__ log_a) {
    constexpr int G = D / 8;                   // threads per (token, head)
    constexpr int kUnitsPerWarp = 32 / G;
    const int lane = threadIdx.x & 31;
    const int sub = lane % G;                  // channel group: channels 8 sub .. 8 sub + 7
    const int c0 = 8 * sub;
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / 32;
    const int64_t n_warps = (int64_t)gridDim.x * kThreads / 32;
    for (int64_t base = warp * kUnitsPerWarp; base < units; base += n_warps * kUnitsPerWarp) {
        const int64_t u0 = base + lane / G;
        const bool valid = u0 < units;
        const int64_t u = valid ? u0 : units - 1;
        const int64_t t = u / H;
        const int h = (int)(u - t * H);
        const int64_t s = seq_start(cu, n_seqs, t);

        Raw8<T> rq[4], rk[4], rv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t tt = (t - 3 + j >= s) ? t - 3 + j : t;   // a valid row either way
            const size_t off = ((size_t)tt * H + h) * D + c0;
            rq[j].load(xq + off);
            rk[j].load(xk + off);
            rv[j].load(xv + off);
        }
        const size_t row = (size_t)u * D + c0;
        float z[8];
        if (SCALAR) {
            z[0] = __ldg(a_raw + u) + __ldg(a_bias + h);
        } else {
            float bz[8];
            load8(a_raw + row, z);
            load8(a_bias + (size_t)h * D + c0, bz);
#pragma unroll
            for (int e = 0; e < 8; ++e) z[e] += bz[e];
        }
        const float br = __ldg(beta_raw + u);

        float yq[8], yk[8], yv[8];
        conv4<T, D>(rq, wq, t, s, h, c0, yq);
        conv4<T, D>(rk, wk, t, s, h, c0, yk);
        conv4<T, D>(rv, wv, t, s, h, c0, yv);
        l2_normalise<G>(yq);
        l2_normalise<G>(yk);
        if (!valid) continue;
        store8(q + row, yq);
        store8(k + row, yk);
        store8(v + row, yv);
        if (SCALAR) {
            if (sub == 0) log_a[u] = log_sigmoid(z[0]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) z[e] = log_sigmoid(z[e]);
            store8(log_a + row, z);
        }
        if (sub == 0) beta[u] = sigmoid(br);
    }
}

template <typename T, int D>
cudaError_t launch_typed(const gdr_preprocess_args& a, cudaStream_t st) {
    const int64_t units = a.total_tokens * a.n_heads;
    constexpr int G = D / 8;
    const int64_t warps = (units * G + 31) / 32;
    int64_t blocks = (warps + kThreads / 32 - 1) / (kThreads / 32);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = (int64_t)sms * 8;      // eight 256-thread CTAs per SM
    if (blocks > cap) blocks = cap;
    const dim3 grid((unsigned)blocks);
    auto* xq = static_cast<const T*>(a.xq);
    auto* xk = static_cast<const T*>(a.xk);
    auto* xv = static_cast<const T*>(a.xv);
    auto* q = static_cast<T*>(a.q);
    auto* k = static_cast<T*>(a.k);
    auto* v = static_cast<T*>(a.v);
    if (a.scalar_decay)
        preprocess_kernel<T, D, true><<<grid, kThreads, 0, st>>>(
            a.n_seqs, a.n_heads, units, a.cu_seqlens, xq, xk, xv, a.conv_q, a.conv_k, a.conv_v,
            a.beta_raw, a.a_raw, a.a_bias, q, k, v, a.beta, a.log_a);
    else
        preprocess_kernel<T, D, false><<<grid, kThreads, 0, st>>>(
            a.n_seqs, a.n_heads, units, a.cu_seqlens, xq, xk, xv, a.conv_q, a.conv_k, a.conv_v,
            a.beta_raw, a.a_raw, a.a_bias, q, k, v, a.beta, a.log_a);
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
