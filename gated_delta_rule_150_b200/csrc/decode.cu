// decode.cu -- one O(1)-state decode step of the gated delta rule.
//
// "kda-graft", section "2. Decode: O(1) против O(L)": a decode step of the
// KDA layer reads and writes a fixed-size state, so its cost does not depend
// on the context length.  Per (sequence, head) and per state row j (value
// channel), with s the row of S and a = exp(log_a):
//     s' = s * a                      (S Diag(a); "Gated DeltaNet: dodaj zanik")
//     p  = s' . k,  c = s' . (scale q)
//     d  = beta (v_j - p)             ("Reguła delta: zapisz poprawkę, nie sumę")
//     s  = s' + d k
//     o_j = s . (scale q) = c + d (k . scale q)   (read after the update)
// Rows are independent given (k, beta, a), so the kernel streams the state
// once: each row is read and written exactly once with 128-bit accesses.
//
// Memory roofline: per head-state 2 * 4 * d_v * d_k bytes of state plus the
// token's inputs and the output row; no reuse, so the kernel is HBM-bound.
// Launched with programmatic stream serialization: back-to-back steps (the
// layers of a decode pass) schedule their CTAs while the previous step's last
// wave drains, each waiting for that step's memory before its first access.
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

// Output epilogue ("kda-graft", section "Идея и архитектура": each KDA layer
// of the graft ends in an RMSNorm and an output gate): over the d_v outputs
// of a (sequence, head), o = x / sqrt(mean x^2 + eps) * w * sigmoid(gate_raw).
template <typename T>
struct DecodeGate {
    const T* gate;           // [B, H, d_v]
    const float* weight;     // [d_v]
    float eps;
};

// Four consecutive elements as loaded (16-byte aligned for fp32, 8 for
// bf16), converted only where they are used, so that every load of a step is
// issued before the first of them is waited for.
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

// Everything one thread reads for one (sequence, head): its state rows
// (row group rgrp, float4 columns lane16 + 16 i) and the token's inputs,
// all requested at once (the state rows no longer wait behind the inputs'
// round trip and the decay's exponentials: 2.5 % more state bandwidth at
// d 128, the same at d 64).
template <typename T, int DK, int DV, bool SCALAR>
struct StepLoads {
    static constexpr int NV = DK / (4 * kTPR);        // float4 per thread per row: 1 or 2
    static constexpr int PASSES = DV / kRowsPerPass;  // 4 or 8
    Raw4<T> k[NV], q[NV];
    float4 la[NV];                                    // log a (scalar gate: la[0].x)
    T v[PASSES];
    float beta;
    float4 s[PASSES][NV];
    __device__ __forceinline__ void issue(int bh, const T* __restrict__ q_, const T* __restrict__ k_,
                                          const T* __restrict__ v_, const float* __restrict__ beta_,
                                          const float* __restrict__ log_a_, const float* state,
                                          int lane16, int rgrp) {
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int c = 4 * (lane16 + kTPR * i);
            k[i].load(k_ + (size_t)bh * DK + c);
            q[i].load(q_ + (size_t)bh * DK + c);
            if (!SCALAR) la[i] = __ldg(reinterpret_cast<const float4*>(log_a_ + (size_t)bh * DK + c));
        }
        if (SCALAR) la[0].x = __ldg(log_a_ + bh);
        beta = __ldg(beta_ + bh);
        const float* S = state + (size_t)bh * DV * DK;
#pragma unroll
        for (int p = 0; p < PASSES; ++p)
#pragma unroll
            for (int i = 0; i < NV; ++i)
                s[p][i] = *reinterpret_cast<const float4*>(S + (size_t)(rgrp + kRowsPerPass * p) * DK +
                                                           4 * (lane16 + kTPR * i));
#pragma unroll
        for (int p = 0; p < PASSES; ++p) v[p] = v_[(size_t)bh * DV + rgrp + kRowsPerPass * p];
    }
};

// The step of one (sequence, head) from its loads: state rows updated and
// written back, outputs (with the gate epilogue) stored.
template <typename T, int DK, int DV, bool SCALAR, bool GATED>
__device__ __forceinline__ void step_one(const StepLoads<T, DK, DV, SCALAR>& in, int bh, float scale,
                                         float* __restrict__ state, float* __restrict__ o,
                                         const DecodeGate<T>& og, int lane16, int rgrp) {
    constexpr int NV = StepLoads<T, DK, DV, SCALAR>::NV;
    constexpr int PASSES = StepLoads<T, DK, DV, SCALAR>::PASSES;
    float4 kk[NV], qq[NV], aa[NV];
    float kq_part = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        kk[i] = in.k[i].get();
        const float4 qv = in.q[i].get();
        qq[i] = make_float4(qv.x * scale, qv.y * scale, qv.z * scale, qv.w * scale);
        if (SCALAR) {
            const float a = expf(in.la[0].x);
            aa[i] = make_float4(a, a, a, a);
        } else {
            const float4 la = in.la[i];
            aa[i] = make_float4(expf(la.x), expf(la.y), expf(la.z), expf(la.w));
        }
        kq_part += kk[i].x * qq[i].x + kk[i].y * qq[i].y + kk[i].z * qq[i].z + kk[i].w * qq[i].w;
    }
    const float kq = sum16(kq_part);
    float* S = state + (size_t)bh * DV * DK;
    float ov[PASSES];                          // this row group's outputs (epilogue)
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int row = rgrp + kRowsPerPass * p;
        float pk = 0.f, pq = 0.f;
        float4 s[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            float4 x = in.s[p][i];
            x.x *= aa[i].x; x.y *= aa[i].y; x.z *= aa[i].z; x.w *= aa[i].w;
            pk += x.x * kk[i].x + x.y * kk[i].y + x.z * kk[i].z + x.w * kk[i].w;
            pq += x.x * qq[i].x + x.y * qq[i].y + x.z * qq[i].z + x.w * qq[i].w;
            s[i] = x;
        }
        pk = sum16(pk);
        pq = sum16(pq);
        const float d = in.beta * (to_f<T>(in.v[p]) - pk);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            float4& x = s[i];
            x.x += d * kk[i].x; x.y += d * kk[i].y; x.z += d * kk[i].z; x.w += d * kk[i].w;
            *reinterpret_cast<float4*>(S + (size_t)row * DK + 4 * (lane16 + kTPR * i)) = x;
        }
        if (GATED) ov[p] = pq + d * kq;
        else if (lane16 == 0) o[(size_t)bh * DV + row] = pq + d * kq;
    }
    if (GATED) {
        // mean square over the d_v outputs: one partial per row group
        __shared__ float part[kRowsPerPass];
        float ss = 0.f;
#pragma unroll
        for (int p = 0; p < PASSES; ++p) ss = fmaf(ov[p], ov[p], ss);
        if (lane16 == 0) part[rgrp] = ss;
        __syncthreads();
        float tot = 0.f;
#pragma unroll
        for (int r = 0; r < kRowsPerPass; ++r) tot += part[r];
        const float rstd = rsqrtf(tot * (1.f / DV) + og.eps);
#pragma unroll
        for (int p = 0; p < PASSES; ++p) {
            if (lane16 != p) continue;             // pass p's row is stored by lane p
            const int row = rgrp + kRowsPerPass * p;
            const float g = to_f<T>(og.gate[(size_t)bh * DV + row]);
            const float sig = __fdividef(1.f, 1.f + __expf(-g));
            o[(size_t)bh * DV + row] = ov[p] * rstd * __ldg(og.weight + row) * sig;
        }
    }
}

// One CTA per (sequence, head).  The explicit minimum of one CTA per SM
// leaves the register allocation free to keep every load in flight (128
// registers at d 128, 53 at d 64; measured 2.5 % faster at d 128 than the
// tighter default allocation of 114, and no slower at d 64 with 4 CTAs per SM
// instead of 6).
template <typename T, int DK, int DV, bool SCALAR, bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const float* __restrict__ beta, const float* __restrict__ log_a, float scale,
                   float* __restrict__ state, float* __restrict__ o, const DecodeGate<T> og) {
    pdl_launch_dependents();
    pdl_wait();                                // the previous kernel's writes are visible
    const int lane16 = threadIdx.x % kTPR;
    const int rgrp = threadIdx.x / kTPR;
    const int bh = blockIdx.x;
    StepLoads<T, DK, DV, SCALAR> in;
    in.issue(bh, q, k, v, beta, log_a, state, lane16, rgrp);
    step_one<T, DK, DV, SCALAR, GATED>(in, bh, scale, state, o, og, lane16, rgrp);
}

template <typename T, int DK, int DV, bool GATED>
cudaError_t launch_typed(int B, int H, const void* q, const void* k, const void* v,
                         const float* beta, const float* log_a, int scalar, float scale,
                         float* state, float* o, const DecodeGate<T>& og, cudaStream_t st) {
    const dim3 grid((unsigned)(B * H));
    if (scalar)
        return launch_pdl(true, decode_step_kernel<T, DK, DV, true, GATED>, grid, dim3(kThreads), 0, st,
                          (const T*)q, (const T*)k, (const T*)v, beta, log_a, scale, state, o, og);
    return launch_pdl(true, decode_step_kernel<T, DK, DV, false, GATED>, grid, dim3(kThreads), 0, st,
                      (const T*)q, (const T*)k, (const T*)v, beta, log_a, scale, state, o, og);
}

template <typename T, bool GATED>
cudaError_t launch_dims(int B, int H, int dk, int dv, const void* q, const void* k,
                        const void* v, const float* beta, const float* log_a, int scalar,
                        float scale, float* state, float* o, const DecodeGate<T>& og,
                        cudaStream_t st) {
    if (dk == 64 && dv == 64)
        return launch_typed<T, 64, 64, GATED>(B, H, q, k, v, beta, log_a, scalar, scale, state, o, og, st);
    if (dk == 64 && dv == 128)
        return launch_typed<T, 64, 128, GATED>(B, H, q, k, v, beta, log_a, scalar, scale, state, o, og, st);
    if (dk == 128 && dv == 64)
        return launch_typed<T, 128, 64, GATED>(B, H, q, k, v, beta, log_a, scalar, scale, state, o, og, st);
    return launch_typed<T, 128, 128, GATED>(B, H, q, k, v, beta, log_a, scalar, scale, state, o, og, st);
}

}  // namespace

cudaError_t launch_decode(int B, int H, int dk, int dv, gdr_dtype dt, const void* q,
                          const void* k, const void* v, const float* beta,
                          const float* log_a, int scalar, float scale, float* state,
                          float* o, cudaStream_t st) {
    if (dt == GDR_BF16)
        return launch_dims<__nv_bfloat16, false>(B, H, dk, dv, q, k, v, beta, log_a, scalar, scale,
                                                 state, o, DecodeGate<__nv_bfloat16>{}, st);
    return launch_dims<float, false>(B, H, dk, dv, q, k, v, beta, log_a, scalar, scale, state, o,
                                     DecodeGate<float>{}, st);
}

cudaError_t launch_decode_gated(int B, int H, int dk, int dv, gdr_dtype dt, const void* q,
                                const void* k, const void* v, const float* beta,
                                const float* log_a, int scalar, float scale, float* state,
                                const void* gate_raw, const float* norm_weight, float norm_eps,
                                float* o, cudaStream_t st) {
    if (dt == GDR_BF16)
        return launch_dims<__nv_bfloat16, true>(
            B, H, dk, dv, q, k, v, beta, log_a, scalar, scale, state, o,
            DecodeGate<__nv_bfloat16>{static_cast<const __nv_bfloat16*>(gate_raw), norm_weight, norm_eps}, st);
    return launch_dims<float, true>(B, H, dk, dv, q, k, v, beta, log_a, scalar, scale, state, o,
                                    DecodeGate<float>{static_cast<const float*>(gate_raw), norm_weight,
                                                      norm_eps}, st);
}

}  // namespace gdr
