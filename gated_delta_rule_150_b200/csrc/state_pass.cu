// state_pass.cu -- sequential inter-chunk pass of the chunked prefill.
//
// "Modele hybrydowe: co Gated DeltaNet zastępuje w cache KV", closing
// paragraph of "Co stan rekurencyjny zmienia przy serwowaniu": inside a chunk
// the updates are dense matrix products; only the step from one chunk to the
// next is sequential.  This kernel is that sequential step.  For a chunk with
// start state S0 (d_v x d_k, fp32) and the factors the intra-chunk kernel
// stored (W, U, Qg, P, Kd, gamma), it computes
//     Delta^T = U^T - S0 W^T                        (d_v x 64)
//     O^T     = S0 Qg^T + Delta^T P^T                (d_v x 64)  -> o
//     S_next  = S0 Diag(gamma) + Delta^T Kd          (d_v x d_k)
// which is the token recurrence S_t = S_{t-1} Diag(a_t)(I - b_t k_t k_t^T) +
// b_t v_t k_t^T, o_t = S_t q_t unrolled over the chunk.
//
// One CTA per (sequence, head) walks the sequence's chunks in order.  The fp32
// master state stays in registers (thread = state row) for the whole
// sequence; its bf16 copy in shared memory is the A operand of the tensor-core
// products.  Each chunk's record arrives with one bulk (TMA) copy, prefetched
// one chunk ahead into a second stage.  The four products run as tcgen05 MMAs
// (bf16 in, fp32 accumulate in tensor memory):
//     group 1:  X = S0 W^T  (M=d_v, N=64, K=d_k)   Y = S0 Qg^T (M=d_v, N=64, K=d_k)
//     group 2:  Y += Delta^T P^T (K=64)              Z = Delta^T Kd (M=d_v, N=d_k, K=64)
// Snapshots of the state are written at every snap_interval boundary
// (section "Co stan rekurencyjny...", point 1: prefix reuse needs the state at
// that position).
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace gdr {
namespace {

constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 256;   // X: [0,64)  Y: [64,128)  Z: [128,128+D)

template <typename T> __device__ __forceinline__ void store_out(T* p, float x);
template <> __device__ __forceinline__ void store_out<float>(float* p, float x) { *p = x; }
template <> __device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
}

template <int D>
struct PassSmem {
    static constexpr RecordLayout R = record_layout(D);
    static constexpr uint32_t stage0 = 0;
    static constexpr uint32_t stage1 = R.bytes;
    static constexpr uint32_t S = 2 * R.bytes;               // bf16 [D x D] operand
    static constexpr uint32_t Dt = S + D * D * 2;            // bf16 [D x 64] Delta^T
    static constexpr uint32_t bytes = Dt + D * 128;
    static constexpr uint32_t dyn_bytes = bytes + 1024;      // + alignment slack
};

// Bounded drain used on the error path only: wait for the copies this CTA
// issued, so no bulk copy lands after the CTA has exited.
__device__ void drain_copies(uint64_t* full, const uint32_t* issued, const uint32_t* done) {
    for (int s = 0; s < 2; ++s)
        for (uint32_t u = done[s]; u < issued[s]; ++u) mbar_wait(&full[s], u & 1);
}

template <int D, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
state_pass_kernel(const int32_t* __restrict__ cu, int n_seqs, int H,
                  const uint8_t* __restrict__ records, const float* init_state,
                  OutT* __restrict__ o, float* final_state, int snap_interval,
                  float* __restrict__ snapshots, uint32_t* err) {
    using L = PassSmem<D>;
    constexpr RecordLayout R = record_layout(D);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t full[2];
    __shared__ uint64_t mma_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int64_t snap_base_s;
    __shared__ uint32_t issued_s[2], done_s[2];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    const int row = (D == 128) ? (32 * warp + lane) : (16 * warp + lane);
    const bool active = (D == 128) || (lane < 16);
    const int s0 = __ldg(cu + n), s1 = __ldg(cu + n + 1);
    const int len_seq = s1 - s0;
    const int nchunks = (len_seq + kChunk - 1) / kChunk;

    uint8_t* stage[2] = {sm + L::stage0, sm + L::stage1};
    uint8_t* sS = sm + L::S;
    uint8_t* sDt = sm + L::Dt;

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&mma_bar, 1);
        fence_mbar_init();
        issued_s[0] = issued_s[1] = done_s[0] = done_s[1] = 0;
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, kTmemCols);
        // snapshot slot base: full intervals of all earlier sequences
        int64_t acc = 0;
        if (snap_interval > 0)
            for (int m = lane; m < n; m += 32) acc += (__ldg(cu + m + 1) - __ldg(cu + m)) / snap_interval;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) snap_base_s = acc;
    }

    // Load the initial state row (fp32) and its bf16 operand copy.
    float S[D];
    const size_t state_off = ((size_t)n * H + h) * D * D + (size_t)row * D;
#pragma unroll
    for (int c = 0; c < D; c += 4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (active && init_state) x = *reinterpret_cast<const float4*>(init_state + state_off + c);
        S[c] = x.x; S[c + 1] = x.y; S[c + 2] = x.z; S[c + 3] = x.w;
    }
    if (active) {
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
            uint4 u;
            u.x = pack_bf16(S[8 * j + 0], S[8 * j + 1]);
            u.y = pack_bf16(S[8 * j + 2], S[8 * j + 3]);
            u.z = pack_bf16(S[8 * j + 4], S[8 * j + 5]);
            u.w = pack_bf16(S[8 * j + 6], S[8 * j + 7]);
            *reinterpret_cast<uint4*>(sS + sw128_chunk(D, row, j)) = u;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_slot;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const int64_t snap_base = snap_base_s;

    auto record_of = [&](int k) -> const uint8_t* {
        const int64_t slot = (int64_t)(s0 / kChunk) + k + n;
        return records + ((size_t)slot * H + h) * R.bytes;
    };
    if (tid == 0 && nchunks > 0) {
        mbar_arrive_expect_tx(&full[0], R.bytes);
        bulk_g2s(stage[0], record_of(0), R.bytes, &full[0]);
        issued_s[0] = 1;
    }

    uint32_t mma_phase = 0;
    bool failed = false;
    const uint32_t id_y = idesc_bf16_f32(D, 64);
    const uint32_t id_z = idesc_bf16_f32(D, D);
    const uint32_t aS = smem_u32(sS), aDt = smem_u32(sDt);

    for (int k = 0; k < nchunks; ++k) {
        const int st = k & 1;
        uint8_t* rec = stage[st];
        const int t0 = s0 + k * kChunk;
        const int len = min(kChunk, s1 - t0);
        if (tid == 0 && k + 1 < nchunks) {
            const int ns = (k + 1) & 1;
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&full[ns], R.bytes);
            bulk_g2s(stage[ns], record_of(k + 1), R.bytes, &full[ns]);
            issued_s[ns] += 1;
        }
        if (!mbar_wait(&full[st], (uint32_t)(k >> 1) & 1)) failed = true;
        if (tid == 0) done_s[st] += 1;

        // group 1: X = S0 W^T, Y = S0 Qg^T
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t aW = smem_u32(rec + R.W), aQ = smem_u32(rec + R.Qg);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t da = sw128_desc(aS, D, 0, 16 * kk);
                mma_bf16(tmem + 0, da, sw128_desc(aW, 64, 0, 16 * kk), id_y, kk > 0);
                mma_bf16(tmem + 64, da, sw128_desc(aQ, 64, 0, 16 * kk), id_y, kk > 0);
            }
            mma_commit(&mma_bar);
        }
        if (!mbar_wait(&mma_bar, mma_phase)) failed = true;
        mma_phase ^= 1;
        tc_fence_after_sync();

        // Delta^T row = U^T row - X row, stored as the bf16 A operand of group 2
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float x[32];
            tmem_ld32(tmem + lane_base + 32 * half, x);
            tmem_ld_wait();
            if (active) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int chunk = 4 * half + j;
                    const uint4 u = *reinterpret_cast<const uint4*>(rec + R.Ut + sw128_chunk(D, row, chunk));
                    const float2 u0 = unpack_bf16(u.x), u1 = unpack_bf16(u.y);
                    const float2 u2 = unpack_bf16(u.z), u3 = unpack_bf16(u.w);
                    uint4 d;
                    d.x = pack_bf16(u0.x - x[8 * j + 0], u0.y - x[8 * j + 1]);
                    d.y = pack_bf16(u1.x - x[8 * j + 2], u1.y - x[8 * j + 3]);
                    d.z = pack_bf16(u2.x - x[8 * j + 4], u2.y - x[8 * j + 5]);
                    d.w = pack_bf16(u3.x - x[8 * j + 6], u3.y - x[8 * j + 7]);
                    *reinterpret_cast<uint4*>(sDt + sw128_chunk(D, row, chunk)) = d;
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        if (__syncthreads_or(failed)) break;

        // group 2: Y += Delta^T P^T, Z = Delta^T Kd
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t aP = smem_u32(rec + R.P), aK = smem_u32(rec + R.Kt);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t da = sw128_desc(aDt, D, 0, 16 * kk);
                mma_bf16(tmem + 64, da, sw128_desc(aP, 64, 0, 16 * kk), id_y, 1);
                mma_bf16(tmem + 128, da, sw128_desc(aK, D, 0, 16 * kk), id_z, kk > 0);
            }
            mma_commit(&mma_bar);
        }
        if (!mbar_wait(&mma_bar, mma_phase)) failed = true;
        mma_phase ^= 1;
        tc_fence_after_sync();

        // o rows of this chunk (column r of O^T = output token t0 + r)
        OutT* orow = o + (size_t)t0 * H * D + (size_t)h * D + row;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float y[32];
            tmem_ld32(tmem + lane_base + 64 + 32 * half, y);
            tmem_ld_wait();
            if (active) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (32 * half + j < len) store_out<OutT>(orow + (size_t)(32 * half + j) * H * D, y[j]);
            }
        }
        // S <- S Diag(gamma) + Z, and refresh the bf16 operand copy
        const float* gam = reinterpret_cast<const float*>(rec + R.gamma);
#pragma unroll
        for (int piece = 0; piece < D / 32; ++piece) {
            float z[32];
            tmem_ld32(tmem + lane_base + 128 + 32 * piece, z);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) S[32 * piece + j] = fmaf(S[32 * piece + j], gam[32 * piece + j], z[j]);
            if (active) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c = 32 * piece + 8 * j;
                    uint4 u;
                    u.x = pack_bf16(S[c + 0], S[c + 1]);
                    u.y = pack_bf16(S[c + 2], S[c + 3]);
                    u.z = pack_bf16(S[c + 4], S[c + 5]);
                    u.w = pack_bf16(S[c + 6], S[c + 7]);
                    *reinterpret_cast<uint4*>(sS + sw128_chunk(D, row, 4 * piece + j)) = u;
                }
            }
        }
        if (snap_interval > 0 && len == kChunk && ((k + 1) * kChunk) % snap_interval == 0 && active) {
            const int64_t slot = snap_base + ((int64_t)(k + 1) * kChunk) / snap_interval - 1;
            float* dst = snapshots + ((size_t)slot * H + h) * D * D + (size_t)row * D;
#pragma unroll
            for (int c = 0; c < D; c += 4)
                *reinterpret_cast<float4*>(dst + c) = make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        if (__syncthreads_or(failed)) break;
        tc_fence_after_sync();
    }

    if (failed) {
        if (tid == 0) {
            atomicOr(err, 1u);
            drain_copies(full, issued_s, done_s);
        }
    } else if (active) {
        float* dst = final_state + state_off;
#pragma unroll
        for (int c = 0; c < D; c += 4)
            *reinterpret_cast<float4*>(dst + c) = make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

template <int D, typename OutT>
cudaError_t launch_typed(const gdr_prefill_args& a, const uint8_t* records, uint32_t* err,
                         cudaStream_t st) {
    auto kern = state_pass_kernel<D, OutT>;
    const uint32_t smem = PassSmem<D>::dyn_bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)a.n_seqs * (unsigned)a.n_heads;
    kern<<<grid, kThreads, smem, st>>>(a.cu_seqlens, a.n_seqs, a.n_heads, records, a.init_state,
                                       static_cast<OutT*>(a.o), a.final_state, a.snap_interval,
                                       a.snapshots, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_pass(const gdr_prefill_args& a, const uint8_t* records, uint32_t* err,
                              cudaStream_t st) {
    if ((int64_t)a.n_seqs * a.n_heads == 0) return cudaSuccess;
    if (a.d_k == 64)
        return a.qkv_dtype == GDR_BF16 ? launch_typed<64, __nv_bfloat16>(a, records, err, st)
                                       : launch_typed<64, float>(a, records, err, st);
    return a.qkv_dtype == GDR_BF16 ? launch_typed<128, __nv_bfloat16>(a, records, err, st)
                                   : launch_typed<128, float>(a, records, err, st);
}

}  // namespace gdr
