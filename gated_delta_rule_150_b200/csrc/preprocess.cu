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
// Layout of the work: one CTA per (head, block of kTok tokens), heads
// fastest in the launch order, so that the CTAs resident at one time read
// every head of the same tokens: contiguous runs of H * D elements per
// token instead of one head's D elements every H * D (measured 7 % faster at
// d 64 and 5 % at d 128 than token blocks fastest, the difference being DRAM
// page locality).  It first
// stages, by 16-byte cp.async from every thread, the raw rows of x_q, x_k and
// x_v for tokens [t0 - 3, t0 + kTok) (the three before the block for the
// conv), the block's a_raw rows, beta_raw and the head's conv taps and gate
// bias: about 25 KB per CTA at d 64, all in flight at once, so the kernel
// keeps enough bytes moving to stream at HBM speed, in four commit groups
// (x_q, x_k, x_v, the gates) so that each tensor is computed as soon as its
// rows have landed (11 % faster at d 128, 2 % at d 64).  Then D / 8 threads own
// a token (eight channels each; at d 128 two consecutive tokens) and compute
// its outputs from shared memory, one tensor after another; a tap that
// reaches before the token's sequence start is skipped.  L2 norms
// are shuffle sums over the token's D / 8 lanes.  Outputs go straight to
// global memory, each token row written by D / 8 neighbouring threads.  HBM
// traffic: x_q, x_k, x_v, beta_raw and a_raw read (plus a three-row halo per
// block), q, k, v, beta and log a written.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace gdr {
namespace {

constexpr int kThreads = 256;
constexpr int kTok = 32;            // tokens per CTA (32 measured faster than 64)
// Consecutive tokens per thread: at d 128 a thread takes two, so each staged
// raw row is unpacked for both (1.34 against 1.39 ms on 8 varlen sequences x
// 32 heads); at d 64 one (two tokens per thread took twice the registers
// there for no gain).
template <int D>
__host__ __device__ constexpr int run_for() { return D == 128 ? 2 : 1; }

template <typename T, int D, bool SCALAR>
struct PreLayout {
    static constexpr uint32_t kRows = kTok + 3;                    // staged raw rows
    static constexpr uint32_t X = 0;                               // [3][kRows][D] raw x
    static constexpr uint32_t A = X + 3u * kRows * D * sizeof(T);  // [kTok][D] a_raw (or [kTok])
    static constexpr uint32_t a_bytes = SCALAR ? 4u * kTok : 4u * kTok * D;
    static constexpr uint32_t B = A + ((a_bytes + 15u) & ~15u);    // [kTok] beta_raw
    static constexpr uint32_t W = B + 4u * kTok;                   // [3][4][D] taps, tap-major
    static constexpr uint32_t Bias = W + 3u * D * 16u;             // [D] (or [1]) gate bias
    static constexpr uint32_t bytes = Bias + 4u * D;
};

// log(1 + e) with the fast log: e = exp(-|z|) is in (0, 1], so 1 + e is in
// (1, 2], where __logf's absolute error is documented below 2^-21.4 (about
// 4e-7), inside the 2e-6 absolute bound the outputs are held to (measured
// 4-6 % faster than log1pf)
__device__ __forceinline__ float log_sigmoid(float z) {
    return fminf(z, 0.f) - __logf(1.f + __expf(-fabsf(z)));
}

__device__ __forceinline__ float sigmoid(float z) {
    const float e = expf(-fabsf(z));
    return z >= 0.f ? 1.0f / (1.0f + e) : e / (1.0f + e);
}

// Eight channels of a row as four channel pairs (2p, 2p + 1): the arithmetic
// below runs on pairs with sm_100's packed fp32 instructions (__ffma2_rn,
// __fmul2_rn, __fadd2_rn: two fp32 operations per instruction, each rounded
// like its scalar form; measured 1-2 % faster than scalar fp32 here)
template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load2(const __nv_bfloat16* p, float2 (&x)[4]) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        x[0] = unpack_bf16(u.x); x[1] = unpack_bf16(u.y); x[2] = unpack_bf16(u.z); x[3] = unpack_bf16(u.w);
    }
    static __device__ __forceinline__ void store2(__nv_bfloat16* p, const float2 (&x)[4]) {
        uint4 u;
        u.x = pack_bf16(x[0].x, x[0].y); u.y = pack_bf16(x[1].x, x[1].y);
        u.z = pack_bf16(x[2].x, x[2].y); u.w = pack_bf16(x[3].x, x[3].y);
        *reinterpret_cast<uint4*>(p) = u;
    }
};
template <> struct Vec8<float> {
    static __device__ __forceinline__ void load2(const float* p, float2 (&x)[4]) {
        const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
        x[0] = make_float2(a.x, a.y); x[1] = make_float2(a.z, a.w);
        x[2] = make_float2(b.x, b.y); x[3] = make_float2(b.z, b.w);
    }
    static __device__ __forceinline__ void store2(float* p, const float2 (&x)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0].x, x[0].y, x[1].x, x[1].y);
        *reinterpret_cast<float4*>(p + 4) = make_float4(x[2].x, x[2].y, x[3].x, x[3].y);
    }
};

// The fp32 rows in shared memory (taps, a_raw, gate bias) store 16-byte word
// w (channels 4w .. 4w + 3) at word w ^ ((w >> 3) & 1).  A thread reads
// words 2 cg and 2 cg + 1 (its channels 8 cg .. 8 cg + 7); in the plain order
// the eight lanes of a quarter-warp would hit every bank group twice (words
// 32 bytes apart), swizzled they hit each once, and eight consecutive words
// written by consecutive lanes stay in distinct bank groups too.
__device__ __forceinline__ int swz_word(int w) { return w ^ ((w >> 3) & 1); }

__device__ __forceinline__ void load8_swz2(const float* row, int cg, float2 (&x)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(row + 4 * swz_word(2 * cg));
    const float4 b = *reinterpret_cast<const float4*>(row + 4 * swz_word(2 * cg + 1));
    x[0] = make_float2(a.x, a.y); x[1] = make_float2(a.z, a.w);
    x[2] = make_float2(b.x, b.y); x[3] = make_float2(b.z, b.w);
}

// Sum over the G = D / 8 lanes of a token (G divides 32; groups are G-aligned).
// The shuffles name only the token's own lanes: in a ragged last block the
// lanes of tokens past its end have left the token loop.
template <int G>
__device__ __forceinline__ float group_sum(float v) {
    const unsigned lane = threadIdx.x & 31u;
    const unsigned mask = G == 32 ? 0xffffffffu : ((1u << G) - 1u) << (lane & ~(unsigned)(G - 1));
#pragma unroll
    for (int m = G / 2; m >= 1; m >>= 1) v += __shfl_xor_sync(mask, v, m);
    return v;
}

template <typename T, int D, bool SCALAR>
__global__ void __launch_bounds__(kThreads)
preprocess_kernel(int n_seqs, int H, int64_t T_tot, const int32_t* __restrict__ cu,
                  const T* __restrict__ xq, const T* __restrict__ xk, const T* __restrict__ xv,
                  const float* __restrict__ wq, const float* __restrict__ wk,
                  const float* __restrict__ wv, const float* __restrict__ beta_raw,
                  const float* __restrict__ a_raw, const float* __restrict__ a_bias,
                  T* __restrict__ q, T* __restrict__ k, T* __restrict__ v,
                  float* __restrict__ beta, float* __restrict__ log_a) {
    using L = PreLayout<T, D, SCALAR>;
    constexpr int G = D / 8;                       // threads per token
    constexpr int kRun = run_for<D>();
    constexpr int TPP = kThreads / G * kRun;       // tokens per pass
    constexpr int kPer = D * (int)sizeof(T) / 16;  // 16-byte pieces per raw row
    extern __shared__ __align__(16) uint8_t sm[];
    const int tid = threadIdx.x;
    pdl_launch_dependents();
    pdl_wait();                                    // the previous kernel's writes are visible
    const int h = (int)(blockIdx.x % (unsigned)H);
    const int64_t t0 = (int64_t)(blockIdx.x / (unsigned)H) * kTok;
    const int ntok = (int)(T_tot - t0 < kTok ? T_tot - t0 : kTok);

    // ---- stage everything the block reads, in four commit groups -----------------
    // (x_q with the taps, x_k, x_v, then a_raw, beta_raw and the bias), so
    // that q is computed while x_k, x_v and the gates are still arriving
    auto stage_x = [&](int tsr) {
        const T* x = tsr == 0 ? xq : (tsr == 1 ? xk : xv);
        for (int i = tid; i < (kTok + 3) * kPer; i += kThreads) {
            const int row = i / kPer, piece = i % kPer;
            const int64_t tok = t0 - 3 + row;
            const bool in = tok >= 0 && tok < T_tot;
            const T* src = x + ((in ? tok : 0) * H + h) * (int64_t)D;
            cp_async16(sm + L::X + ((size_t)(tsr * (kTok + 3) + row) * D) * sizeof(T) + 16 * piece,
                       reinterpret_cast<const uint8_t*>(src) + 16 * piece, in ? 16u : 0u);
        }
    };
    stage_x(0);
    // taps transposed to [tensor][tap][channel] (16-byte words swizzled as
    // above), so that a thread's eight channels of one tap are two 16-byte
    // words; copied element by element by 4-byte cp.async, in flight with the
    // rows (5 % faster at d 64 than loading them into registers and storing)
    for (int i = tid; i < 3 * 4 * D; i += kThreads) {
        const int tsr = i / (4 * D), j = (i / D) % 4, c = i % D;
        const float* w = tsr == 0 ? wq : (tsr == 1 ? wk : wv);
        cp_async4(sm + L::W + 4 * ((tsr * 4 + j) * D + 4 * swz_word(c / 4) + c % 4),
                  w + ((size_t)h * D + c) * 4 + j, 4u);
    }
    cp_async_commit();
    stage_x(1);
    cp_async_commit();
    stage_x(2);
    cp_async_commit();
    if (SCALAR) {
        for (int i = tid; i < kTok; i += kThreads)
            cp_async4(sm + L::A + 4 * i, a_raw + ((i < ntok ? t0 + i : 0) * H + h), i < ntok ? 4u : 0u);
    } else {
        for (int i = tid; i < kTok * D / 4; i += kThreads) {
            const int row = i / (D / 4), piece = i % (D / 4);
            const bool in = row < ntok;
            cp_async16(sm + L::A + 4 * (row * D + 4 * swz_word(piece)),
                       a_raw + ((in ? t0 + row : 0) * H + h) * (int64_t)D + 4 * piece, in ? 16u : 0u);
        }
    }
    for (int i = tid; i < kTok; i += kThreads)
        cp_async4(sm + L::B + 4 * i, beta_raw + ((i < ntok ? t0 + i : 0) * H + h), i < ntok ? 4u : 0u);
    if (SCALAR) {
        if (tid == 0) cp_async4(sm + L::Bias, a_bias + h, 4u);
    } else {
        for (int i = tid; i < D / 4; i += kThreads)
            cp_async16(sm + L::Bias + 16 * swz_word(i), a_bias + (size_t)h * D + 4 * i, 16u);
    }
    cp_async_commit();

    // ---- outputs: thread (tokens r0 .. r0 + kRun - 1, channels c0 .. c0 + 7) ----------
    static_assert(TPP == kTok, "one pass over the block's tokens");
    const int cg = tid % G, c0 = 8 * cg;
    const T* X = reinterpret_cast<const T*>(sm + L::X);
    const float* Wt = reinterpret_cast<const float*>(sm + L::W);
    const float* Av = reinterpret_cast<const float*>(sm + L::A);
    const float* Bv = reinterpret_cast<const float*>(sm + L::B);
    const float* Bias = reinterpret_cast<const float*>(sm + L::Bias);
    const int r0 = (tid / G) * kRun;
    const bool act = r0 < ntok;                    // uniform over the run's lanes
    const int64_t t = t0 + r0;
    int64_t su[kRun];
    if (act) {
        // first token of t's sequence: cu[n] for the largest n with cu[n] <= t;
        // a later token of the run starts a new sequence where cu[n + 1] is it
        int lo = 0, hi = n_seqs - 1, n = 0;
        while (lo <= hi) {
            const int mid = (lo + hi) >> 1;
            if ((int64_t)__ldg(cu + mid) <= t) { n = mid; lo = mid + 1; } else { hi = mid - 1; }
        }
        su[0] = __ldg(cu + n);
        const int64_t nxt = __ldg(cu + n + 1);
#pragma unroll
        for (int u = 1; u < kRun; ++u) su[u] = nxt <= t + u ? nxt : su[u - 1];
    }
    // one tensor at a time, each as soon as its rows have landed: conv of the
    // run's tokens, L2 norm (q, k), store
#pragma unroll
    for (int tsr = 0; tsr < 3; ++tsr) {
        if (tsr == 0) cp_async_wait_group<3>();
        else if (tsr == 1) cp_async_wait_group<2>();
        else cp_async_wait_group<1>();
        __syncthreads();
        if (!act) continue;
        float2 y[kRun][4];
        // the run's raw rows, each unpacked once: staged row r0 + i is token t - 3 + i
        float2 x[kRun + 3][4];
#pragma unroll
        for (int i = 0; i < kRun + 3; ++i)
            Vec8<T>::load2(X + ((size_t)(tsr * (kTok + 3) + r0 + i)) * D + c0, x[i]);
        // taps 3 .. 0 on rows t + u, ..., t + u - 3
#pragma unroll
        for (int j = 3; j >= 0; --j) {
            float2 w[4];
            load8_swz2(Wt + (size_t)(tsr * 4 + j) * D, cg, w);
#pragma unroll
            for (int u = 0; u < kRun; ++u) {
                if (j < 3 && t + u - 3 + j < su[u]) continue;
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    y[u][p] = (j == 3) ? __fmul2_rn(w[p], x[u + j][p])
                                       : __ffma2_rn(w[p], x[u + j][p], y[u][p]);
            }
        }
        if (tsr < 2) {
#pragma unroll
            for (int u = 0; u < kRun; ++u) {
                float2 s2 = __fmul2_rn(y[u][0], y[u][0]);
#pragma unroll
                for (int p = 1; p < 4; ++p) s2 = __ffma2_rn(y[u][p], y[u][p], s2);
                const float ss = group_sum<G>(s2.x + s2.y);
                const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
                const float2 inv2 = make_float2(inv, inv);
#pragma unroll
                for (int p = 0; p < 4; ++p) y[u][p] = __fmul2_rn(y[u][p], inv2);
            }
        }
        T* dst = tsr == 0 ? q : (tsr == 1 ? k : v);
#pragma unroll
        for (int u = 0; u < kRun; ++u)
            if (r0 + u < ntok) Vec8<T>::store2(dst + ((size_t)(t + u) * H + h) * D + c0, y[u]);
    }
    cp_async_wait_group<0>();
    __syncthreads();
    if (!act) return;
#pragma unroll
    for (int u = 0; u < kRun; ++u) {
        const int r = r0 + u;
        if (r >= ntok) break;
        const size_t row = ((size_t)(t + u) * H + h) * D + c0;
        if (SCALAR) {
            if (cg == 0) log_a[(size_t)(t + u) * H + h] = log_sigmoid(Av[r] + Bias[0]);
        } else {
            float2 z[4], bz[4];
            load8_swz2(Av + (size_t)r * D, cg, z);
            load8_swz2(Bias, cg, bz);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float2 zb = __fadd2_rn(z[p], bz[p]);
                z[p] = make_float2(log_sigmoid(zb.x), log_sigmoid(zb.y));
            }
            Vec8<float>::store2(log_a + row, z);
        }
        if (cg == 0) beta[(size_t)(t + u) * H + h] = sigmoid(Bv[r]);
    }
}

template <typename T, int D, bool SCALAR>
cudaError_t launch_kernel(const gdr_preprocess_args& a, cudaStream_t st) {
    auto kern = preprocess_kernel<T, D, SCALAR>;
    constexpr uint32_t smem = PreLayout<T, D, SCALAR>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // one CTA per (token block, head), heads fastest
    const int64_t ctas = (a.total_tokens + kTok - 1) / kTok * (int64_t)a.n_heads;
    if (ctas == 0) return cudaSuccess;
    if (ctas > (int64_t)INT32_MAX) return cudaErrorInvalidValue;
    // early launch: the CTAs take the SMs the previous kernel's last CTAs leave
    return launch_pdl(true, kern, dim3((unsigned)ctas), dim3(kThreads), smem, st, a.n_seqs, a.n_heads,
                      a.total_tokens, a.cu_seqlens, static_cast<const T*>(a.xq),
                      static_cast<const T*>(a.xk), static_cast<const T*>(a.xv), a.conv_q, a.conv_k,
                      a.conv_v, a.beta_raw, a.a_raw, a.a_bias, static_cast<T*>(a.q),
                      static_cast<T*>(a.k), static_cast<T*>(a.v), a.beta, a.log_a);
}

template <typename T, int D>
cudaError_t launch_typed(const gdr_preprocess_args& a, cudaStream_t st) {
    return a.scalar_decay ? launch_kernel<T, D, true>(a, st) : launch_kernel<T, D, false>(a, st);
}

}  // namespace

cudaError_t launch_preprocess(const gdr_preprocess_args& a, cudaStream_t st) {
    if (a.io_dtype == GDR_BF16)
        return a.d == 64 ? launch_typed<__nv_bfloat16, 64>(a, st)
                         : launch_typed<__nv_bfloat16, 128>(a, st);
    return a.d == 64 ? launch_typed<float, 64>(a, st) : launch_typed<float, 128>(a, st);
}

}  // namespace gdr
