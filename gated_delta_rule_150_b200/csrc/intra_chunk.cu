// intra_chunk.cu -- the parallel part of the chunked prefill.
//
// "Modele hybrydowe: co Gated DeltaNet zastępuje w cache KV", closing
// paragraph of "Co stan rekurencyjny zmienia przy serwowaniu": inside a chunk
// of tokens the updates are dense matrix products.  Unrolling the recurrence
// S_t = S_{t-1} Diag(a_t)(I - b_t k_t k_t^T) + b_t v_t k_t^T over one chunk of
// C = 64 tokens with start state S0 gives (g = chunk-local cumulative log
// decay, Gamma_r = exp(g_r), all products per key channel c):
//     A[r,i] = b_r sum_c k[r,c] k[i,c] exp(g[r,c] - g[i,c])      i < r
//     P[r,i] = scale sum_c q[r,c] k[i,c] exp(g[r,c] - g[i,c])    i <= r
//     T      = (I + A)^-1                  (forward substitution, fp32)
//     W      = T diag(b) (K * Gamma)       U = T diag(b) V
//     Qg     = scale Q * Gamma             Kd = K * exp(g_last - g)
//     gamma  = exp(g_last)
// Nothing here depends on S0, so every (chunk, head) is independent: one CTA
// each, all in parallel.  The sequential pass (state_pass.cu) then needs only
// Delta = U - W S0^T, O = Qg S0^T + P Delta, S = S0 Diag(gamma) + Delta^T Kd.
//
// Tensor cores.  A and P are decay-weighted K K^T / Q K^T products.  With a
// per-channel decay (KDA) the weight exp(g[r,c] - g[i,c]) does not factor into
// a bounded row term times a bounded column term over a whole chunk (g can
// fall by hundreds over 64 tokens), so the chunk is cut into four 16-token
// blocks, each with a reference point m_b = g at the middle of block b:
//     exp(g_r - g_i) = exp(g_r - m_b(r)) * exp(m_b(r) - m_b(i)) * exp(m_b(i) - g_i)
// The outer factors are bounded by exp(half a block's decay); the middle one
// is <= 1 and is folded into the key operand of query block b(r).  One
// tcgen05 MMA per query block b (M = 128 rows: the 64 scaled queries stacked
// on the 64 scaled keys, N = 16(b+1) keys, K = d_k) yields P and A together.
// A chunk whose half-block decay exceeds exp(80) in some channel (log decay
// below about -10 per token) would overflow fp32 in that form; it takes an
// exact elementwise path instead.  With a scalar decay (Gated DeltaNet) the
// weight is exp(g_r - g_i) for the whole row and is applied after one plain
// Q K^T / K K^T MMA.  W and U come from one more MMA, W^T | U^T =
// [diag(b)(K*Gamma) | diag(b)V]^T T^T, with T rounded to bf16.
//
// Outputs go to the chunk-head record of the workspace in tensor-core operand
// layout (internal.h), ready for the state pass to load with one bulk copy.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace gdr {
namespace {

constexpr int kThreads = 128;
constexpr float kMaxFactorExp = 80.f;
constexpr uint32_t kTmemCols = 256;

__host__ __device__ constexpr uint32_t al1024(uint32_t x) { return (x + 1023u) & ~1023u; }
__host__ __device__ constexpr uint32_t umax(uint32_t a, uint32_t b) { return a > b ? a : b; }

template <int D, bool SCALAR>
struct IntraSmem {
    static constexpr uint32_t XA = 0;                         // bf16 [128 x D] scaled [Q; K]
    static constexpr uint32_t KT0 = 256 * D;                  // key tiles, 16(b+1) rows each
    static constexpr uint32_t op_bytes = SCALAR ? 256 * D : 256 * D + 320 * D;
    static constexpr uint32_t Pf = 0;                         // fp32 [64][65], after MMA 1
    static constexpr uint32_t Wst = 17408;                    // bf16 W image [64 x D]
    static constexpr uint32_t region0 = al1024(umax(op_bytes, Wst + 128 * D));
    static constexpr uint32_t Bt = region0;                   // bf16 [2D x 64]
    static constexpr uint32_t Tb = Bt + 256 * D;              // bf16 [64 x 64]
    static constexpr uint32_t As = Tb + 8192;                 // fp32 [64][65]
    static constexpr uint32_t Ts = As + 16896;                // fp32 [64][65]
    static constexpr uint32_t Yt = Ts + 16896;                // fp32 [3][16][16]
    static constexpr uint32_t Gl = Yt + 3072;                 // fp32 [D] g_last
    static constexpr uint32_t Bs = Gl + 4 * D;                // fp32 [64] beta
    static constexpr uint32_t Gs = Bs + 256;                  // fp32 [64] g (scalar decay)
    static constexpr uint32_t bytes = Gs + 256;
    static constexpr uint32_t dyn_bytes = bytes + 1024;
    __host__ __device__ static constexpr uint32_t kt_off(int b) { return KT0 + 32u * D * (uint32_t)(b * (b + 1) / 2); }
};

__host__ __device__ constexpr uint32_t ap_col(int b) { return (uint32_t)(8 * b * (b + 1)); }

template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[8]) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), c = unpack_bf16(u.z), d = unpack_bf16(u.w);
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y; x[4] = c.x; x[5] = c.y; x[6] = d.x; x[7] = d.y;
    }
};
template <> struct Vec8<float> {
    static __device__ __forceinline__ void load(const float* p, float (&x)[8]) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p));
        const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};

__device__ __forceinline__ void load8f(const float* p, float (&x)[8]) { Vec8<float>::load(p, x); }

__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
    uint4 u;
    u.x = pack_bf16(x[0], x[1]); u.y = pack_bf16(x[2], x[3]);
    u.z = pack_bf16(x[4], x[5]); u.w = pack_bf16(x[6], x[7]);
    return u;
}

template <int D, typename InT, bool SCALAR>
__global__ void __launch_bounds__(kThreads)
intra_chunk_kernel(const int32_t* __restrict__ cu, int n_seqs, int H,
                   const InT* __restrict__ q, const InT* __restrict__ k, const InT* __restrict__ v,
                   const float* __restrict__ beta, const float* __restrict__ g, float scale,
                   uint8_t* __restrict__ records, uint32_t* err) {
    using L = IntraSmem<D, SCALAR>;
    constexpr RecordLayout R = record_layout(D);
    constexpr int CG = D / 8;              // channel groups of 8
    constexpr int RG = kThreads / CG;      // row groups
    constexpr int RPT = 64 / RG;           // rows per thread: 4 (D=64) or 8 (D=128)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t mma_bar;
    __shared__ uint32_t tmem_slot;

    int seq, start, len;
    if (!slot_to_chunk(cu, n_seqs, blockIdx.x, &seq, &start, &len)) return;
    const int h = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* rec = records + ((size_t)blockIdx.x * H + h) * R.bytes;

    float* As = reinterpret_cast<float*>(sm + L::As);
    float* Ts = reinterpret_cast<float*>(sm + L::Ts);
    float* Pf = reinterpret_cast<float*>(sm + L::Pf);
    float* Yt = reinterpret_cast<float*>(sm + L::Yt);
    float* Gl = reinterpret_cast<float*>(sm + L::Gl);
    float* Bs = reinterpret_cast<float*>(sm + L::Bs);
    float* Gs = reinterpret_cast<float*>(sm + L::Gs);

    if (tid == 0) {
        mbar_init(&mma_bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&tmem_slot, kTmemCols);

    const int cg = tid % CG, rg = tid / CG, c0 = 8 * cg;
    const int r0 = rg * RPT;
    const int jb = r0 / 16;                                   // this thread's 16-row block
    const size_t tok_stride = (size_t)H * D;
    const InT* qh = q + (size_t)start * tok_stride + (size_t)h * D + c0;
    const InT* kh = k + (size_t)start * tok_stride + (size_t)h * D + c0;
    const InT* vh = v + (size_t)start * tok_stride + (size_t)h * D + c0;

    // ---- phase 1: reference points and the overflow check -------------------
    float gl[8], mj[8];                       // g_last and m_{jb} for this thread's channels
    float ecross[4][8];                       // exp(m_b - m_jb) for b > jb (per-channel)
    bool bad = false;
    if (!SCALAR) {
        const float* gh = g + (size_t)start * tok_stride + (size_t)h * D + c0;
        load8f(gh + (size_t)(len - 1) * tok_stride, gl);
        load8f(gh + (size_t)min(16 * jb + 8, len - 1) * tok_stride, mj);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            if (b > jb) {
                float mb[8];
                load8f(gh + (size_t)min(16 * b + 8, len - 1) * tok_stride, mb);
#pragma unroll
                for (int e = 0; e < 8; ++e) ecross[b][e] = expf(mb[e] - mj[e]);
            }
        }
#pragma unroll
        for (int u = 0; u < RPT; ++u) {
            const int r = r0 + u;
            float gr[8];
            if (r < len) load8f(gh + (size_t)r * tok_stride, gr);
            else {
#pragma unroll
                for (int e = 0; e < 8; ++e) gr[e] = gl[e];
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) bad |= fabsf(gr[e] - mj[e]) > kMaxFactorExp;
        }
        if (rg == 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e) Gl[c0 + e] = gl[e];
        }
    } else {
        const float glast = __ldg(g + (size_t)(start + len - 1) * H + h);
#pragma unroll
        for (int e = 0; e < 8; ++e) gl[e] = glast;
        if (tid < 64) Gs[tid] = tid < len ? __ldg(g + (size_t)(start + tid) * H + h) : glast;
        if (tid < D) Gl[tid] = glast;
    }
    if (tid < 64) Bs[tid] = tid < len ? __ldg(beta + (size_t)(start + tid) * H + h) : 0.f;
    const bool bad_chunk = __syncthreads_or(bad);

    // ---- phase 2: operands and the elementwise outputs ----------------------
    uint8_t* XA = sm + L::XA;
    uint8_t* Bt = sm + L::Bt;
    float em[8], eld[8];        // exp(m_jb), exp(g_last - m_jb)
    if (!SCALAR) {
#pragma unroll
        for (int e = 0; e < 8; ++e) { em[e] = expf(mj[e]); eld[e] = expf(gl[e] - mj[e]); }
    }
    uint32_t pb1[8][RPT / 2], pb2[8][RPT / 2], pkd[8][RPT / 2];   // transposed bf16 pairs
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
        const int r = r0 + u;
        const bool valid = r < len;
        float qv[8], kv[8], vv[8], gr[8];
        const float br = Bs[r];
        if (valid) {
            Vec8<InT>::load(qh + (size_t)r * tok_stride, qv);
            Vec8<InT>::load(kh + (size_t)r * tok_stride, kv);
            Vec8<InT>::load(vh + (size_t)r * tok_stride, vv);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) qv[e] = kv[e] = vv[e] = 0.f;
        }
        if (!SCALAR) {
            if (valid) load8f(g + (size_t)(start + r) * tok_stride + (size_t)h * D + c0, gr);
            else {
#pragma unroll
                for (int e = 0; e < 8; ++e) gr[e] = gl[e];
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) gr[e] = Gs[r];
        }
        float xq[8], xk[8], kk0[8], b1[8], qg[8], kd[8];
        if (!SCALAR && !bad_chunk) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float d = gr[e] - mj[e];
                const float F = expf(d), Fi = expf(-d);
                xq[e] = scale * qv[e] * F;
                xk[e] = kv[e] * F;
                kk0[e] = kv[e] * Fi;
                b1[e] = br * xk[e] * em[e];
                qg[e] = xq[e] * em[e];
                kd[e] = kk0[e] * eld[e];
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float G = expf(gr[e]);
                xq[e] = SCALAR ? scale * qv[e] : 0.f;
                xk[e] = SCALAR ? kv[e] : 0.f;
                kk0[e] = 0.f;
                b1[e] = br * kv[e] * G;
                qg[e] = scale * qv[e] * G;
                kd[e] = kv[e] * expf(gl[e] - gr[e]);
            }
        }
        // A-side operand rows r (queries) and 64 + r (keys)
        *reinterpret_cast<uint4*>(XA + sw128_chunk(128, r, cg)) = pack8(xq);
        *reinterpret_cast<uint4*>(XA + sw128_chunk(128, 64 + r, cg)) = pack8(xk);
        if (!SCALAR) {
            // key operand of every query block b >= jb (row r of tile b)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                if (b < jb) continue;
                float kb[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) kb[e] = (b == jb) ? kk0[e] : kk0[e] * ecross[b][e];
                *reinterpret_cast<uint4*>(sm + L::kt_off(b) + sw128_chunk(16 * (b + 1), r, cg)) = pack8(kb);
            }
        }
        // Qg image row r (global record)
        *reinterpret_cast<uint4*>(rec + R.Qg + sw128_chunk(64, r, cg)) = pack8(qg);
        // transposed operands: collect pairs of rows per channel
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float bv = br * vv[e];
            if ((u & 1) == 0) {
                pb1[e][u / 2] = pack_bf16(b1[e], 0.f);
                pb2[e][u / 2] = pack_bf16(bv, 0.f);
                pkd[e][u / 2] = pack_bf16(kd[e], 0.f);
            } else {
                pb1[e][u / 2] = (pb1[e][u / 2] & 0xFFFFu) | (pack_bf16(0.f, b1[e]) & 0xFFFF0000u);
                pb2[e][u / 2] = (pb2[e][u / 2] & 0xFFFFu) | (pack_bf16(0.f, bv) & 0xFFFF0000u);
                pkd[e][u / 2] = (pkd[e][u / 2] & 0xFFFFu) | (pack_bf16(0.f, kd[e]) & 0xFFFF0000u);
            }
        }
    }
    // B1^T rows c (token columns r0..r0+RPT-1), B2^T rows D + c, Kd^T image rows c
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int c = c0 + e;
        const uint32_t o1 = sw128_chunk(2 * D, c, r0 / 8) + (r0 % 8) * 2;
        const uint32_t o2 = sw128_chunk(2 * D, D + c, r0 / 8) + (r0 % 8) * 2;
        const uint32_t o3 = sw128_chunk(D, c, r0 / 8) + (r0 % 8) * 2;
        if (RPT == 8) {
            *reinterpret_cast<uint4*>(Bt + o1) = make_uint4(pb1[e][0], pb1[e][1], pb1[e][2 % (RPT / 2)], pb1[e][3 % (RPT / 2)]);
            *reinterpret_cast<uint4*>(Bt + o2) = make_uint4(pb2[e][0], pb2[e][1], pb2[e][2 % (RPT / 2)], pb2[e][3 % (RPT / 2)]);
            *reinterpret_cast<uint4*>(rec + R.Kt + o3) = make_uint4(pkd[e][0], pkd[e][1], pkd[e][2 % (RPT / 2)], pkd[e][3 % (RPT / 2)]);
        } else {
            *reinterpret_cast<uint2*>(Bt + o1) = make_uint2(pb1[e][0], pb1[e][1 % (RPT / 2)]);
            *reinterpret_cast<uint2*>(Bt + o2) = make_uint2(pb2[e][0], pb2[e][1 % (RPT / 2)]);
            *reinterpret_cast<uint2*>(rec + R.Kt + o3) = make_uint2(pkd[e][0], pkd[e][1 % (RPT / 2)]);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_slot;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;

    // ---- phase 3: decay-weighted Q K^T and K K^T on the tensor cores --------
    if (tid == 0) {
        const uint32_t aXA = smem_u32(XA);
        if (!SCALAR) {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t id = idesc_bf16_f32(128, 16 * (b + 1));
                const uint32_t aK = smem_u32(sm + L::kt_off(b));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_bf16(tmem + ap_col(b), sw128_desc(aXA, 128, 0, 16 * kk),
                             sw128_desc(aK, 16 * (b + 1), 0, 16 * kk), id, kk > 0);
            }
        } else {
            const uint32_t id = idesc_bf16_f32(128, 64);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_bf16(tmem, sw128_desc(aXA, 128, 0, 16 * kk), sw128_desc(aXA, 128, 64, 16 * kk), id, kk > 0);
        }
        mma_commit(&mma_bar);
    }
    bool failed = !mbar_wait(&mma_bar, 0);
    tc_fence_after_sync();

    // ---- phase 4: P (masked) and A (masked, times beta) into fp32 smem ------
    {
        const bool is_p = warp < 2;
        const int rr = 32 * (warp & 1) + lane;                // chunk row
        float* dst = is_p ? Pf : As;
        const float scl = is_p ? 1.f : Bs[rr];
#pragma unroll 4
        for (int i = 0; i < 64; ++i) dst[rr * 65 + i] = 0.f;
        if (!SCALAR) {
            const int b = rr >> 4;
            const int off = (int)ap_col(b), width = 16 * (b + 1);
            const int lim = is_p ? rr : rr - 1;               // last valid key index
#pragma unroll
            for (int p = 0; p < 5; ++p) {
                float x[32];
                tmem_ld32(tmem + lane_base + 32 * p, x);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int i = 32 * p + j - off;
                    if (i >= 0 && i < width && i <= lim) dst[rr * 65 + i] = scl * x[j];
                }
            }
        } else {
            const float gr = Gs[rr];
            const int lim = is_p ? rr : rr - 1;
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float x[32];
                tmem_ld32(tmem + lane_base + 32 * p, x);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int i = 32 * p + j;
                    if (i <= lim) dst[rr * 65 + i] = scl * x[j] * expf(gr - Gs[i]);
                }
            }
        }
        if (!SCALAR && bad_chunk) {
            // exact path: every term with its own exp (chunks with extreme decay only)
            const int lim = is_p ? rr : rr - 1;
            const bool vr = rr < len;
            for (int i = 0; i <= lim && vr; ++i) {
                float acc = 0.f;
                for (int c = 0; c < D; ++c) {
                    const size_t tr = (size_t)(start + rr) * tok_stride + (size_t)h * D + c;
                    const size_t ti = (size_t)(start + i) * tok_stride + (size_t)h * D + c;
                    const float xr = is_p ? scale * (float)q[tr] : (float)k[tr];
                    acc += xr * (float)k[ti] * expf(g[tr] - g[ti]);
                }
                dst[rr * 65 + i] = scl * acc;
            }
        }
    }
    __syncthreads();

    // ---- phase 5: T = (I + A)^-1 by blocked forward substitution (fp32) ----
    if (tid < 64) {
        // diagonal 16x16 blocks, one column per thread
        const int b = tid >> 4, cc = tid & 15, o = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i)
                if (i >= cc) acc -= As[(o + r) * 65 + o + i] * x[i];
            x[r] = (r >= cc) ? acc : 0.f;
            Ts[(o + r) * 65 + o + cc] = x[r];
        }
    } else {
        // meanwhile: P image -> record (8 chunks of 8 per row)
        for (int qd = tid - 64; qd < 512; qd += 64) {
            const int r = qd >> 3, jj = qd & 7;
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = Pf[r * 65 + 8 * jj + e];
            *reinterpret_cast<uint4*>(rec + R.P + sw128_chunk(64, r, jj)) = pack8(x);
        }
    }
    __syncthreads();
#pragma unroll
    for (int d = 1; d <= 3; ++d) {
        // Y_bj = sum_{l=j}^{b-1} A_bl T_lj for all pairs (b, j = b - d)
        for (int e = tid; e < (4 - d) * 256; e += kThreads) {
            const int p = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            const int b = d + p, j = p;
            float acc = 0.f;
            for (int l = j; l < b; ++l)
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    acc += As[(16 * b + rr) * 65 + 16 * l + m] * Ts[(16 * l + m) * 65 + 16 * j + cc];
            Yt[p * 256 + rr * 16 + cc] = acc;
        }
        __syncthreads();
        // T_bj = -T_bb Y_bj
        for (int e = tid; e < (4 - d) * 256; e += kThreads) {
            const int p = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            const int b = d + p, j = p;
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m)
                if (m <= rr) acc += Ts[(16 * b + rr) * 65 + 16 * b + m] * Yt[p * 256 + m * 16 + cc];
            Ts[(16 * b + rr) * 65 + 16 * j + cc] = -acc;
        }
        __syncthreads();
    }
    // T -> bf16 operand tile [64 r][64 i] (zero above the diagonal)
    for (int qd = tid; qd < 512; qd += kThreads) {
        const int r = qd >> 3, jj = qd & 7;
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = (8 * jj + e <= r) ? Ts[r * 65 + 8 * jj + e] : 0.f;
        *reinterpret_cast<uint4*>(sm + L::Tb + sw128_chunk(64, r, jj)) = pack8(x);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    failed = __syncthreads_or(failed);
    tc_fence_after_sync();

    // ---- phase 6: [W | U]^T = [diag(b)(K*Gamma) | diag(b)V]^T T^T ----------
    if (tid == 0 && !failed) {
        const uint32_t id = idesc_bf16_f32(128, 64);
        const uint32_t aB = smem_u32(Bt), aT = smem_u32(sm + L::Tb);
#pragma unroll
        for (int half = 0; half < 2 * D / 128; ++half)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + 64 * half, sw128_desc(aB, 2 * D, 128 * half, 16 * kk),
                         sw128_desc(aT, 64, 0, 16 * kk), id, kk > 0);
        mma_commit(&mma_bar);
    }
    if (!failed && !mbar_wait(&mma_bar, 1)) failed = true;
    tc_fence_after_sync();

    // ---- phase 7: W image (staged, transposed) and U^T image ----------------
    {
        uint8_t* Wst = sm + L::Wst;
        // lanes 0..D-1 hold W^T rows; U^T rows are lanes D..2D-1 (D = 64) or
        // columns 64..127 of the same lanes (D = 128)
        const int lrow = 32 * warp + lane;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const bool wpart = (D == 64) ? (lrow < 64) : (part == 0);
            const int row = (D == 64) ? (lrow & 63) : lrow;
            if (D == 64 && part == 1) break;
            const uint32_t col0 = (D == 64) ? 0u : 64u * part;
#pragma unroll
            for (int piece = 0; piece < 2; ++piece) {
                float x[32];
                tmem_ld32(tmem + lane_base + col0 + 32 * piece, x);
                tmem_ld_wait();
                if (wpart) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        *reinterpret_cast<__nv_bfloat16*>(Wst + sw128_offset(64, 32 * piece + j, row)) =
                            __float2bfloat16_rn(x[j]);
                } else {
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = x[8 * jj + e];
                        *reinterpret_cast<uint4*>(rec + R.Ut + sw128_chunk(D, row, 4 * piece + jj)) = pack8(y);
                    }
                }
            }
        }
        if (tid < D) reinterpret_cast<float*>(rec + R.gamma)[tid] = expf(Gl[tid]);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        bulk_s2g(rec + R.W, sm + L::Wst, (uint32_t)(D * 128));
        bulk_commit_group();
        bulk_wait_group_read0();
        if (failed) atomicOr(err, 1u);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Unpack records into plain fp32 arrays (inspection / tests only).
template <int D>
__global__ void unpack_kernel(const int32_t* __restrict__ cu, int n_seqs, int H,
                              const uint8_t* __restrict__ records, float* W, float* U, float* P,
                              float* Qg, float* Kd, float* gamma) {
    constexpr RecordLayout R = record_layout(D);
    int seq, start, len;
    if (!slot_to_chunk(cu, n_seqs, blockIdx.x, &seq, &start, &len)) return;
    const size_t sh = (size_t)blockIdx.x * H + blockIdx.y;
    const uint8_t* rec = records + sh * R.bytes;
    auto bf = [&](uint32_t off) {
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(rec + off));
    };
    for (int e = threadIdx.x; e < 64 * D; e += blockDim.x) {
        const int r = e / D, c = e % D;
        W[sh * 64 * D + e] = bf(R.W + sw128_offset(64, r, c));
        Qg[sh * 64 * D + e] = bf(R.Qg + sw128_offset(64, r, c));
        U[sh * 64 * D + e] = bf(R.Ut + sw128_offset(D, c, r));
        Kd[sh * 64 * D + e] = bf(R.Kt + sw128_offset(D, c, r));
    }
    for (int e = threadIdx.x; e < 64 * 64; e += blockDim.x)
        P[sh * 4096 + e] = bf(R.P + sw128_offset(64, e / 64, e % 64));
    for (int c = threadIdx.x; c < D; c += blockDim.x)
        gamma[sh * D + c] = reinterpret_cast<const float*>(rec + R.gamma)[c];
}

template <int D, typename InT, bool SCALAR>
cudaError_t launch_typed(const gdr_prefill_args& a, const float* g, uint8_t* records,
                         uint32_t* err, cudaStream_t st) {
    auto kern = intra_chunk_kernel<D, InT, SCALAR>;
    const uint32_t smem = IntraSmem<D, SCALAR>::dyn_bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)n_chunk_slots(a.total_tokens, a.n_seqs), (unsigned)a.n_heads);
    kern<<<grid, kThreads, smem, st>>>(a.cu_seqlens, a.n_seqs, a.n_heads, (const InT*)a.q,
                                       (const InT*)a.k, (const InT*)a.v, a.beta, g, a.scale,
                                       records, err);
    return cudaGetLastError();
}

template <int D, typename InT>
cudaError_t launch_decay(const gdr_prefill_args& a, const float* g, uint8_t* records,
                         uint32_t* err, cudaStream_t st) {
    return a.scalar_decay ? launch_typed<D, InT, true>(a, g, records, err, st)
                          : launch_typed<D, InT, false>(a, g, records, err, st);
}

}  // namespace

cudaError_t launch_intra_chunk(const gdr_prefill_args& a, const float* g, uint8_t* records,
                               uint32_t* err, cudaStream_t st) {
    if (n_chunk_slots(a.total_tokens, a.n_seqs) == 0) return cudaSuccess;
    if (a.d_k == 64)
        return a.qkv_dtype == GDR_BF16 ? launch_decay<64, __nv_bfloat16>(a, g, records, err, st)
                                       : launch_decay<64, float>(a, g, records, err, st);
    return a.qkv_dtype == GDR_BF16 ? launch_decay<128, __nv_bfloat16>(a, g, records, err, st)
                                   : launch_decay<128, float>(a, g, records, err, st);
}

cudaError_t launch_unpack_records(const gdr_prefill_args& a, const uint8_t* records, float* W,
                                  float* U, float* P, float* Qg, float* Kd, float* gamma,
                                  cudaStream_t st) {
    const int64_t slots = n_chunk_slots(a.total_tokens, a.n_seqs);
    if (slots == 0) return cudaSuccess;
    const dim3 grid((unsigned)slots, (unsigned)a.n_heads);
    if (a.d_k == 64)
        unpack_kernel<64><<<grid, 256, 0, st>>>(a.cu_seqlens, a.n_seqs, a.n_heads, records, W, U, P, Qg, Kd, gamma);
    else
        unpack_kernel<128><<<grid, 256, 0, st>>>(a.cu_seqlens, a.n_seqs, a.n_heads, records, W, U, P, Qg, Kd, gamma);
    return cudaGetLastError();
}

}  // namespace gdr
