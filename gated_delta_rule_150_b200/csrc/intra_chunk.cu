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
// so that Delta = U - W S0^T, O = Qg S0^T + P Delta and
// S_next = S0 Diag(gamma) + Delta^T Kd with gamma = exp(g_last).  The chunk's
// effect is affine in S0, and this kernel also forms the four S0-free
// matrices of that map,
//     Qt = Qg - P W,  PU = P U,  BS = -Kd^T W,  NC = U^T Kd,
// so that the sequential pass (state_pass.cu) is left with
//     S_next = S0 Diag(gamma) + S0 BS^T + NC,   O = Qt S0^T + PU,
// one tensor-core product per chunk on its critical path.  Nothing here
// depends on S0: every (chunk, head) item is independent.
//
// Structure.  A persistent kernel: as many CTAs as fit (two per SM at d 64,
// one at d 128) take the items round-robin.  A loader warp requests the next
// item's q, k, v and log a by 2-D TMA as soon as the current item's operand
// build has read its own (while the A/P MMA runs);
// the chunk-local cumulative decay (the standalone cumdecay kernel's
// quantity) is summed in shared memory, for per-channel decay by warps 4-7
// during the previous item's triangular solve; the record leaves by two bulk
// stores that drain behind the next item's first phases.
//
// Tensor cores.  A and P are decay-weighted K K^T / Q K^T products.  With a
// per-channel decay (KDA) exp(g[r,c] - g[i,c]) does not factor into a bounded
// row term times a bounded column term over a whole chunk (g can fall by
// hundreds over 64 tokens), so the chunk is cut into four 16-token blocks with
// reference points m_b = g at the middle of block b:
//     exp(g_r - g_i) = exp(g_r - m_b(r)) * exp(m_b(r) - m_b(i)) * exp(m_b(i) - g_i)
// The outer factors are bounded by exp(half a block's decay) and the middle
// one is <= 1; it is folded into the key operand of query block b(r).  The
// four key operands (16(b+1) keys each) are stacked into one of 160 rows, and
// one tcgen05 MMA chain (M = 128: the 64 scaled queries stacked on the 64
// scaled keys, N = 160, K = d_k) yields P and A together, query block b
// reading its columns.  A chunk
// whose half-block decay exceeds exp(80) in some channel (log decay below
// about -10 per token) would overflow fp32 in that form; it takes an exact
// elementwise path instead.  With a scalar decay (Gated DeltaNet) the weight
// exp(g_r - g_i) is applied after one plain Q K^T / K K^T MMA.  W and U come
// from [W | U]^T = [diag(b)(K*Gamma) | diag(b)V]^T T^T with T rounded to
// bf16; P [W | U], Kd^T W and U^T Kd are three more MMAs.
#include <cuda_bf16.h>

#include <cstring>
#include <cuda.h>      // CUtensorMap and its enums; the encoder is looked up at run time

#include "internal.h"
#include "sm100.cuh"

namespace gdr {
namespace {

// Threads per CTA: 8 warps (two CTAs per SM at d 64); 16 for the scalar
// decay at d 128 (one CTA per SM, whose phases then run twice as wide; the
// per-channel kernel measured slower that way, its phases being bound by
// shared memory rather than by issue).
template <int D, bool SCALAR>
__host__ __device__ constexpr int threads_for() { return (D == 128 && SCALAR) ? 512 : 256; }
constexpr float kMaxFactorExp = 80.f;
constexpr int kLd = 68;                       // row stride (floats) of the fp32 64x64 tiles

__host__ __device__ constexpr uint32_t al1024(uint32_t x) { return (x + 1023u) & ~1023u; }
__host__ __device__ constexpr uint32_t umax(uint32_t a, uint32_t b) { return a > b ? a : b; }

// Gate activations of the fused input path (raw projections).
// log(1 + e) with the fast log: e = exp(-|z|) is in (0, 1], so 1 + e is in
// (1, 2] where __logf's absolute error is a few 1e-8 -- far inside what the
// bf16 operands built from log a resolve
__device__ __forceinline__ float log_sigmoid_f(float z) {
    return fminf(z, 0.f) - __logf(1.f + __expf(-fabsf(z)));
}

__device__ __forceinline__ float sigmoid_f(float z) {
    const float e = __expf(-fabsf(z));
    return z >= 0.f ? 1.0f / (1.0f + e) : e / (1.0f + e);
}

template <int D, typename InT, bool SCALAR, bool RAW = false>
struct IntraLayout {
    static constexpr uint32_t elem = sizeof(InT);
    // fp32 q/k/v at d 128 do not fit next to everything else: read from global
    static constexpr bool kStageQKV = !(elem == 4 && D == 128);
    // region 1: the staged inputs of one chunk.  Free once the A/P products
    // are read out, when it is refilled with the next chunk's inputs.
    static constexpr uint32_t sQ = 0;
    static constexpr uint32_t sK = sQ + (kStageQKV ? 64u * D * elem : 0u);
    static constexpr uint32_t sV = sK + (kStageQKV ? 64u * D * elem : 0u);
    static constexpr uint32_t sG = sV + (kStageQKV ? 64u * D * elem : 0u);
    static constexpr uint32_t in_bytes = sG + (SCALAR ? 0u : 64u * D * 4u);
    static constexpr uint32_t r1 = al1024(in_bytes);
    // region 2: A/P operands; then As (A, overwritten by T), Pt, Tb, Yt;
    // finally the record, staged for its bulk store (reaching into Bt, Kdt)
    static constexpr uint32_t XA = r1;                        // bf16 [128][D]
    // key tiles of query blocks b = 0..3 (16(b+1) rows each), stacked as one
    // bf16 [160][D] operand, tile b from row ap_col(b)
    static constexpr uint32_t KT0 = XA + 256u * D;
    static constexpr uint32_t op_bytes = SCALAR ? 256u * D : 576u * D;
    static constexpr uint32_t As = r1;                        // fp32 [64][kLd]
    static constexpr uint32_t Pt = As + 64u * kLd * 4u;       // bf16 [64][64]
    static constexpr uint32_t Tb = Pt + 8192u;                // bf16 [64][64]
    static constexpr uint32_t Yt = Tb + 8192u;                // fp32 [32][32] scratch
    static constexpr uint32_t solve_bytes = 64u * kLd * 4u + 16384u + 4096u;
    static constexpr uint32_t Rec = r1;                       // record staging
    static constexpr uint32_t rec_bytes = record_layout(D).bytes;
    static constexpr uint32_t r2 = al1024(umax(umax(op_bytes, solve_bytes),
                                               rec_bytes > 384u * D ? rec_bytes - 384u * D : 0u));
    // region 3: live through the chunk
    static constexpr uint32_t Bt = r1 + r2;                   // bf16 [2D][64]; then [W | U]^T
    static constexpr uint32_t WUt = Bt;
    static constexpr uint32_t Kdt = Bt + 256u * D;            // bf16 [D][64]
    static constexpr uint32_t Qgs = Kdt + 128u * D;           // bf16 [64][D]
    static constexpr uint32_t Gl = Qgs + 128u * D;            // fp32 [D] g_last
    static constexpr uint32_t Bs = Gl + 4u * D;               // fp32 [64] beta
    static constexpr uint32_t Gs = Bs + 256u;                 // fp32 [64] g (scalar decay)
    // fp32 partials of the per-channel scan [1024 B]: that scan runs only for
    // a CTA's first item (later items are scanned during the previous item's
    // solve, without partials), when nothing else is in region 2
    static constexpr uint32_t kPtotBytes = 4u * threads_for<D, SCALAR>();
    static constexpr uint32_t Ptot = r1;
    // raw projections (fused input activations): the item's conv taps
    // [3 tensors][4 taps][D] fp32 and the three raw rows before the chunk of x_q,
    // x_k, x_v [3][3][D], fetched at the item start into the Qg tile (dead
    // from the previous item's map MMAs on, outside its record staging, and
    // written only by this item's operand build, after their last use)
    static constexpr uint32_t Taps = Qgs;
    static constexpr uint32_t Halo = Taps + 3u * D * 16u;
    static constexpr uint32_t halo_bytes = RAW ? 9u * D * elem : 0u;
    static constexpr uint32_t bytes = Gs + 256u;
    // at d 128 the 512 TMEM columns of a CTA allow one CTA per SM: request
    // enough shared memory that a second one is never scheduled
    static constexpr uint32_t dyn_bytes = (D == 128) ? umax(bytes + 1024u, 118784u) : bytes + 1024u;
    static_assert(dyn_bytes + 256u <= 232448u, "shared memory budget (with the kernel's static variables)");
    static_assert(kPtotBytes <= r2, "scan partials fit in region 2");
    static_assert(!RAW || kStageQKV, "raw projections are staged");
    static_assert(!RAW || (Halo + halo_bytes <= Qgs + 128u * D && Taps >= Rec + rec_bytes),
                  "taps and halo fit in the Qg tile, outside the record staging");
    static_assert((64u * kLd * 4u) % 1024u == 0u, "Pt alignment");
    static_assert(Rec + rec_bytes <= Qgs, "record staging stays below Qgs");
    static_assert(!(SCALAR && D == 128) || XA + op_bytes <= Rec + record_layout(D).Qt,
                  "scalar d 128: the operand build writes only what the first record store reads");
    // TMEM is allocated once per persistent CTA: never more CTAs on an SM
    // than its 512 columns hold (2 x 256 at d 64, 1 x 512 at d 128)
    static_assert(3u * (dyn_bytes + 1088u) > 233472u, "at most two CTAs per SM");
    static_assert(!(D == 64 && elem == 2) || dyn_bytes + 1088u <= 114688u, "two CTAs per SM at d 64");
    static_assert(D != 128 || 2u * (dyn_bytes + 1088u) > 233472u, "one CTA per SM at d 128");
};

// TMEM column of query block b's A/P product (16(b+1) columns each).
__host__ __device__ constexpr uint32_t ap_col(int b) { return (uint32_t)(8 * b * (b + 1)); }

template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load_reg(const uint4 u, float (&x)[8]) {
        float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), c = unpack_bf16(u.z), d = unpack_bf16(u.w);
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y; x[4] = c.x; x[5] = c.y; x[6] = d.x; x[7] = d.y;
    }
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[8]) {
        load_reg(*reinterpret_cast<const uint4*>(p), x);
    }
};
template <> struct Vec8<float> {
    static __device__ __forceinline__ void load_reg(const uint4, float (&x)[8]) {   // not used for fp32
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 0.f;
    }
    static __device__ __forceinline__ void load(const float* p, float (&x)[8]) {
        const float4 a = *reinterpret_cast<const float4*>(p);
        const float4 b = *reinterpret_cast<const float4*>(p + 4);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};

__device__ __forceinline__ void load8f(const float* p, float (&x)[8]) { Vec8<float>::load(p, x); }

// The conv taps of the raw path keep channel c in column g_col(c) of their
// rows: the 16-byte words of a row are swizzled, word w at w ^ bit 3 of w (an
// involution), so that the eight lanes of a quarter-warp reading a thread's
// two words (channels 8 cg .. 8 cg + 7) hit each bank group once.
__device__ __forceinline__ int swz_word(int w) { return w ^ ((w >> 3) & 1); }
__device__ __forceinline__ int g_col(int c) { return 4 * swz_word(c >> 2) + (c & 3); }

// Channels c0 .. c0 + 7 (c0 a multiple of 8) of a swizzled row.
__device__ __forceinline__ void load8g(const float* row, int c0, float (&x)[8]) {
    const int w = c0 >> 2;
    const float4 a = *reinterpret_cast<const float4*>(row + 4 * swz_word(w));
    const float4 b = *reinterpret_cast<const float4*>(row + 4 * swz_word(w + 1));
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
    uint4 u;
    u.x = pack_bf16(x[0], x[1]); u.y = pack_bf16(x[2], x[3]);
    u.z = pack_bf16(x[4], x[5]); u.w = pack_bf16(x[6], x[7]);
    return u;
}

__device__ __forceinline__ float4 f4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// acc[2][4] += X[xr, xr+1][xk .. xk+16) * Y[yk .. yk+16)[yc .. yc+4): one
// 16-deep step of a 2 x 4 output tile (fp32, shared-memory operands; X has
// row stride kLd, Y row stride LDY).
template <int LDY>
__device__ __forceinline__ void tile16(const float* X, int xr, int xk, const float* Y, int yk, int yc,
                                       float (&a0)[4], float (&a1)[4]) {
#pragma unroll
    for (int m4 = 0; m4 < 4; ++m4) {
        const float4 x0 = f4(X + xr * kLd + xk + 4 * m4), x1 = f4(X + (xr + 1) * kLd + xk + 4 * m4);
        const float x0v[4] = {x0.x, x0.y, x0.z, x0.w}, x1v[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const float4 yv = f4(Y + (yk + 4 * m4 + qq) * LDY + yc);
            a0[0] = fmaf(x0v[qq], yv.x, a0[0]); a0[1] = fmaf(x0v[qq], yv.y, a0[1]);
            a0[2] = fmaf(x0v[qq], yv.z, a0[2]); a0[3] = fmaf(x0v[qq], yv.w, a0[3]);
            a1[0] = fmaf(x1v[qq], yv.x, a1[0]); a1[1] = fmaf(x1v[qq], yv.y, a1[1]);
            a1[2] = fmaf(x1v[qq], yv.z, a1[2]); a1[3] = fmaf(x1v[qq], yv.w, a1[3]);
        }
    }
}

// Store -z (a 2 x 4 block of T at rows r, r+1, columns c .. c+3) to the fp32
// tile Ts (row stride kLd) and to the bf16 operand tile Tb.
__device__ __forceinline__ void store_t_tile(float* Ts, uint8_t* Tb, int r, int c,
                                             const float (&z0)[4], const float (&z1)[4]) {
    *reinterpret_cast<float4*>(Ts + r * kLd + c) = make_float4(-z0[0], -z0[1], -z0[2], -z0[3]);
    *reinterpret_cast<float4*>(Ts + (r + 1) * kLd + c) = make_float4(-z1[0], -z1[1], -z1[2], -z1[3]);
    *reinterpret_cast<uint2*>(Tb + sw128_offset(64, r, c)) =
        make_uint2(pack_bf16(-z0[0], -z0[1]), pack_bf16(-z0[2], -z0[3]));
    *reinterpret_cast<uint2*>(Tb + sw128_offset(64, r + 1, c)) =
        make_uint2(pack_bf16(-z1[0], -z1[1]), pack_bf16(-z1[2], -z1[3]));
}

// a[e] <- a[e ^ s] for e < 8, by three conditional swap stages (s < 8).
template <int N>
__device__ __forceinline__ void xor_permute(uint32_t (&a)[8][N], int s) {
#pragma unroll
    for (int bit = 1; bit < 8; bit <<= 1) {
        const bool sw = (s & bit) != 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (e & bit) continue;
#pragma unroll
            for (int n = 0; n < N; ++n) {
                const uint32_t x = a[e][n], y = a[e ^ bit][n];
                a[e][n] = sw ? y : x;
                a[e ^ bit][n] = sw ? x : y;
            }
        }
    }
}

// Barrier among the first `count` threads of the CTA (named barrier `id`).
__device__ __forceinline__ void named_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void solve_bar() { named_bar(1, 128); }

// OR of `pred` over the `count` threads that reach named barrier `id`.
__device__ __forceinline__ bool bar_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r) : "r"((uint32_t)pred), "r"(id), "r"(count) : "memory");
    return r != 0;
}

// Chunk-local cumulative log decay of one chunk in place (sG: [64 x D] fp32),
// by NS threads (t = 0 .. NS-1): 128 / D row parts per channel, the parts
// joined by a shuffle.  Rows past len add 0.  Returns whether this thread saw
// a log a below -kMaxFactorExp / 8.
template <int D, int NS, bool RAW>
__device__ __forceinline__ bool scan_channels(float* sG, int len, int t,
                                              const float* __restrict__ bias) {
    static_assert(NS == 128 && (D == 64 || D == 128), "two parts of 32 rows (d 64) or one of 64");
    constexpr int P = NS / D, RP = 64 / P;
    // D = 64: channel c = 16 (t / 32) + (t % 32) / 2, part = t % 2; D = 128: c = t
    const int c = (P == 1) ? t : 16 * (t >> 5) + ((t & 31) >> 1);
    const int part = (P == 1) ? 0 : (t & 1);
    bool bad = false;
    float run = 0.f;
    const float bc = RAW ? __ldg(bias + c) : 0.f;
#pragma unroll 4
    for (int r = part * RP; r < (part + 1) * RP; ++r) {
        // raw projections: log a = log_sigmoid(a_raw + bias) on the fly
        const float la = r < len ? (RAW ? log_sigmoid_f(sG[r * D + c] + bc) : sG[r * D + c]) : 0.f;
        bad |= la < -kMaxFactorExp / 8.f;
        run += la;
        sG[r * D + c] = run;
    }
    if (P == 2) {
        const float tot0 = __shfl_xor_sync(0xffffffffu, run, 1);    // part 0's total
        if (part == 1) {
#pragma unroll 4
            for (int r = RP; r < 64; ++r) sG[r * D + c] += tot0;
        }
    }
    return bad;
}

// Reference points of this thread's channels c0 .. c0 + 7: g_last, the
// midpoint m_jb of its 16-row block and exp(m_b - m_jb) for later blocks b
// (per-channel decay; with a scalar decay g_last only); g_last also goes to Gl.
template <int D, bool SCALAR>
__device__ __forceinline__ void reference_points(const float* sG, const float* Gs, float* Gl,
                                                 int len, int jb, int c0, int rg, int tid,
                                                 float (&gl)[8], float (&mj)[8],
                                                 float (&ecross)[4][8]) {
    if (!SCALAR) {
        load8f(sG + (size_t)(len - 1) * D + c0, gl);
        load8f(sG + (size_t)min(16 * jb + 8, len - 1) * D + c0, mj);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            if (b > jb) {
                float mb[8];
                load8f(sG + (size_t)min(16 * b + 8, len - 1) * D + c0, mb);
#pragma unroll
                for (int e = 0; e < 8; ++e) ecross[b][e] = __expf(mb[e] - mj[e]);
            }
        }
        if (rg == 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e) Gl[c0 + e] = gl[e];
        }
    } else {
        const float glast = Gs[len - 1];
#pragma unroll
        for (int e = 0; e < 8; ++e) gl[e] = glast;
        if (tid < D) Gl[tid] = glast;
    }
}

// One unit of work: chunk slot idx / H of head idx % H (idx < 0: none).
struct Item {
    int64_t idx;
    int h, start, len;
    int sstart;                 // first token of the chunk's sequence
};

// The first item at or after `from`, stepping by the grid size, whose chunk
// slot holds a chunk (the slot map leaves one unused slot per sequence).
__device__ __forceinline__ Item find_item(const int32_t* __restrict__ cu, int n_seqs, int H,
                                          int64_t n_items, int64_t from) {
    Item it{-1, 0, 0, 0, 0};
    for (int64_t i = from; i < n_items; i += gridDim.x) {
        int seq, start, len;
        if (slot_to_chunk(cu, n_seqs, i / H, &seq, &start, &len)) {
            it.idx = i;
            it.h = (int)(i % H);
            it.start = start;
            it.len = len;
            it.sstart = __ldg(cu + seq);
            break;
        }
    }
    return it;
}

// Tensor maps of the token-major inputs: q, k, v and log a, each a 2-D view
// [tokens][H * D] read in boxes of 64 tokens x D channels (rows past the
// tensor end are zero-filled; rows past a sequence end are masked by their
// consumers).
struct InputMaps {
    CUtensorMap q, k, v, g;
};

// Fused input activations ("kda-graft", section "Идея и архитектура": a
// width-4 conv initialised as an identity tap, the alpha gate with bias +5,
// beta): the maps above then read the raw projections x_q, x_k, x_v and
// a_raw, beta comes from beta_raw, and these are the per-head parameters.
struct RawParams {
    const float* wq;            // [H D, 4] conv taps (tap 3 = current token)
    const float* wk;
    const float* wv;
    const float* a_bias;        // [H, D], or [H] with a scalar gate
};


// Issue the copies of one item's inputs, from one warp: lane 0 starts the
// tiled TMA loads of log a (completing on bar_g) and of q, k, v (on bar_qkv);
// beta and the scalar log a go by 4-byte cp.async with zero fill.
// The inputs of item `it`: with `tiles`, the per-channel decay tile and q,
// k, v (region 1) by 2-D TMA from lane 0; always beta (and a scalar log a)
// by cp.async from every lane.
template <int D, typename InT, bool SCALAR, bool RAW, typename L>
__device__ __forceinline__ void issue_inputs(uint8_t* sm, uint64_t* bar_g, uint64_t* bar_qkv,
                                             const InputMaps& maps, const float* __restrict__ beta,
                                             const float* __restrict__ log_a, int H, const Item& it,
                                             int lane, bool hint, bool tiles) {
    if (lane == 0 && tiles) {
        const int x = it.h * D;
        const uint64_t pol = l2_policy_evict_first();             // inputs are read once
        if (!SCALAR) {
            mbar_arrive_expect_tx(bar_g, 64u * D * 4u);
            if (hint) tma_load_2d_hint(sm + L::sG, &maps.g, x, it.start, bar_g, pol);
            else tma_load_2d(sm + L::sG, &maps.g, x, it.start, bar_g);
        }
        if (L::kStageQKV) {
            mbar_arrive_expect_tx(bar_qkv, 3u * 64u * D * (uint32_t)sizeof(InT));
            if (hint) tma_load_2d_hint(sm + L::sQ, &maps.q, x, it.start, bar_qkv, pol);
            else tma_load_2d(sm + L::sQ, &maps.q, x, it.start, bar_qkv);
            if (hint) tma_load_2d_hint(sm + L::sK, &maps.k, x, it.start, bar_qkv, pol);
            else tma_load_2d(sm + L::sK, &maps.k, x, it.start, bar_qkv);
            if (hint) tma_load_2d_hint(sm + L::sV, &maps.v, x, it.start, bar_qkv, pol);
            else tma_load_2d(sm + L::sV, &maps.v, x, it.start, bar_qkv);
        }
    }
    for (int t = lane; t < 64; t += 32) {
        const int tc = t < it.len ? t : it.len - 1;
        const size_t o = (size_t)(it.start + tc) * H + it.h;
        const uint32_t n = t < it.len ? 4u : 0u;
        cp_async4(sm + L::Bs + 4 * t, beta + o, n);
        if (SCALAR) cp_async4(sm + L::Gs + 4 * t, log_a + o, n);
    }
    cp_async_commit();
}

// Read the A/P products of this thread's row from TMEM (per-channel decay).
// Lanes of warp parity `par` own rows 32 par .. 32 par + 31, i.e. query
// blocks 2 par and 2 par + 1, whose columns are loaded together.
template <int PAR>
__device__ __forceinline__ void load_ap_row(uint32_t taddr, int b, float (&v)[64]) {
    constexpr int blo = 2 * PAR;
    constexpr int wlo = 16 * (blo + 1);
    constexpr int c0 = (int)ap_col(blo);
    constexpr int ncol = 16 * (blo + 1) + 16 * (blo + 2);     // 48 or 112
    float u[ncol];
    if (PAR == 0) {
        float* a = u;
        tmem_ld32(taddr + 0, *reinterpret_cast<float(*)[32]>(a));
        tmem_ld16(taddr + 32, *reinterpret_cast<float(*)[16]>(a + 32));
    } else {
        float* a = u;
        tmem_ld16(taddr + 48, *reinterpret_cast<float(*)[16]>(a));
        tmem_ld32(taddr + 64, *reinterpret_cast<float(*)[32]>(a + 16));
        tmem_ld32(taddr + 96, *reinterpret_cast<float(*)[32]>(a + 48));
        tmem_ld32(taddr + 128, *reinterpret_cast<float(*)[32]>(a + 80));
    }
    (void)c0;
    tmem_ld_wait();
    const bool lo = (b == blo);
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const float x_lo = (i < wlo) ? u[i] : 0.f;
        const float x_hi = (wlo + i < ncol) ? u[(wlo + i < ncol) ? wlo + i : 0] : 0.f;
        v[i] = lo ? x_lo : x_hi;
    }
}

// RAW: q, k, v, beta and log_a are the raw projections x_q, x_k, x_v,
// beta_raw and a_raw; the input activations are applied on the fly (`rp`).
template <int D, typename InT, bool SCALAR, bool RAW>
__global__ void __launch_bounds__(threads_for<D, SCALAR>(), (D == 64) ? 2 : 1)
intra_chunk_kernel(const int32_t* __restrict__ cu, int n_seqs, int H,
                   const InT* __restrict__ q, const InT* __restrict__ k, const InT* __restrict__ v,
                   const float* __restrict__ beta, const float* __restrict__ log_a, float scale,
                   int64_t n_items, uint8_t* __restrict__ records, uint32_t* err,
                   const __grid_constant__ InputMaps maps, int keep_records,
                   const __grid_constant__ RawParams rp) {
    using L = IntraLayout<D, InT, SCALAR, RAW>;
    constexpr RecordLayout R = record_layout(D);
    constexpr int CG = D / 8;              // channel groups of 8
    constexpr int NT = threads_for<D, SCALAR>();
    constexpr int NG = NT / 128;           // warp groups; warps w, w + 4, ... share TMEM lanes
    constexpr int RG = NT / CG;            // row groups
    constexpr int RPT = 64 / RG;           // rows per thread: 2 (D=64) or 4 (D=128)
    constexpr uint32_t kTmemCols = (D == 64) ? 256u : 512u;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align_smem<1024>(smem_raw);
    __shared__ uint64_t mma_bar;
    __shared__ uint64_t in_bar[2];          // inputs landed: log a, q/k/v
    __shared__ uint32_t tmem_slot;
    __shared__ Item s_item[2];              // the next two items, by iteration parity
    __shared__ int s_bad_next;              // the scanned next item has a log a < -10

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t tok_stride = (size_t)H * D;

    float* As = reinterpret_cast<float*>(sm + L::As);
    float* Yt = reinterpret_cast<float*>(sm + L::Yt);
    float* Gl = reinterpret_cast<float*>(sm + L::Gl);
    float* Bs = reinterpret_cast<float*>(sm + L::Bs);
    float* Gs = reinterpret_cast<float*>(sm + L::Gs);
    float* sG = reinterpret_cast<float*>(sm + L::sG);

    constexpr int kLoadWarp = NT / 32 - 1;                    // issues the input copies
    if (tid == 0) {
        mbar_init(&mma_bar, 1);
        mbar_init(&in_bar[0], 1);
        mbar_init(&in_bar[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&tmem_slot, kTmemCols);
    pdl_wait();                               // the previous kernel's memory is final

    // Persistent CTA: items blockIdx.x, blockIdx.x + gridDim.x, ...  The next
    // item's inputs are staged while the current one is finished, and each
    // record's bulk store drains while the next item starts.
    Item cur = find_item(cu, n_seqs, H, n_items, blockIdx.x);
    if (tid == 0) {
        s_item[1] = cur.idx >= 0 ? find_item(cu, n_seqs, H, n_items, cur.idx + gridDim.x) : cur;
        s_item[0] = s_item[1];
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    // requests of decay tiles and of the other inputs (load warp) and MMA
    // commits (thread 0) so far: on a timed-out wait the last of each is
    // drained before the CTA exits
    uint32_t tiles_issued = 0, mma_commits = 0;
    if (cur.idx >= 0 && warp == kLoadWarp) {
        issue_inputs<D, InT, SCALAR, RAW, L>(sm, &in_bar[0], &in_bar[1], maps, beta, log_a, H, cur,
                                             lane, keep_records != 0, true);
        ++tiles_issued;
    }
    const uint32_t tmem = tmem_slot;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int wgrp = warp >> 2;                               // warp group (0 .. NG - 1)
    uint32_t phase = 0;                                       // parity of the next MMA commit
    uint32_t in_phase = 0;                                    // parity of the inputs' barriers
    int iter = 0;                                             // item n: s_item[(n+1)&1] = item n+1
    // per-channel decay at 8 warps: the next item's scan runs on warps 4-7
    // while warps 0-3 do the triangular solve
    constexpr bool kEarlyScan = !SCALAR && NT == 256;
    // (see the wait for the previous record's stores at the operand build)
    constexpr bool kLateRecWait = SCALAR && D == 128;
    bool pre_scanned = false;                                 // this item's g is already in sG
    bool failed = false;

    while (cur.idx >= 0) {
    const int h = cur.h, start = cur.start, len = cur.len;
    uint8_t* rec = records + (size_t)cur.idx * R.bytes;       // item = slot * H + h
    const size_t base = (size_t)start * tok_stride + (size_t)h * D;

    // raw projections: the CTA fetches this head's conv taps and the first row
    // group the three raw rows before the chunk (x_q, x_k, x_v; zeros before
    // the sequence start) by cp.async now, so that the copies are in flight
    // during the waits below
    constexpr int kTapsPer = RAW ? (3 * 4 * D + NT - 1) / NT : 1;
    float taps[kTapsPer];                     // this thread's share, stored tap-major below
    if constexpr (RAW) {
#pragma unroll
        for (int u = 0; u < kTapsPer; ++u) {
            const int i = tid + u * NT;
            if (i < 3 * 4 * D) {
                const int tsr = i / (4 * D), j = (i / D) % 4, c = i % D;
                const float* wsrc = tsr == 0 ? rp.wq : (tsr == 1 ? rp.wk : rp.wv);
                taps[u] = __ldg(wsrc + ((size_t)h * D + c) * 4 + j);
            }
        }
        if (tid < CG) {
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const int tok = start - 3 + j;
                const bool in = tok >= cur.sstart;
                const size_t off = ((size_t)(in ? tok : start) * H + h) * D + 8 * tid;
#pragma unroll
                for (int tsr = 0; tsr < 3; ++tsr) {
                    const InT* src = tsr == 0 ? q : (tsr == 1 ? k : v);
                    cp_async16(sm + L::Halo + ((size_t)(tsr * 3 + j) * D + 8 * tid) * sizeof(InT), src + off,
                               in ? 16u : 0u);
                }
            }
        }
        cp_async_commit();
    }

    // ---- this item's log a and beta have landed --------------------------------
    {
        const bool ok = SCALAR || mbar_wait(&in_bar[0], in_phase);
        if (warp == kLoadWarp) cp_async_wait_all();
        failed = __syncthreads_or(!ok);
        if (failed) {
            if (tid == 0) atomicOr(err, 1u);
            break;
        }
    }

    // ---- chunk-local cumulative log decay, g[r] = sum_{i <= r} log a_i -------
    // (the same quantity gdr_cumdecay computes; padded rows add 0, so past the
    // chunk end g stays at g_last).  The factored per-channel products below
    // need |g_r - m_b| <= kMaxFactorExp inside each 16-row block, which holds
    // whenever every log a >= -kMaxFactorExp / 8; a chunk with a smaller log a
    // in some channel takes the exact path.
    bool bad = false;
    bool bad_chunk;
    if (kEarlyScan && pre_scanned) {
        bad_chunk = s_bad_next != 0;          // scanned during the previous item's solve
    } else {
    if (!SCALAR) {
        constexpr int P = NT / D, RP = 64 / P;                // row parts per channel
        float* Ptot = reinterpret_cast<float*>(sm + L::Ptot);
        const int c = tid % D, part = tid / D;
        const float bc = RAW ? __ldg(rp.a_bias + (size_t)h * D + c) : 0.f;
        float run = 0.f;
#pragma unroll 4
        for (int r = part * RP; r < (part + 1) * RP; ++r) {
            // rows past the end add 0; raw projections: log a = log_sigmoid(a_raw + bias)
            const float la = r < len ? (RAW ? log_sigmoid_f(sG[r * D + c] + bc) : sG[r * D + c]) : 0.f;
            bad |= la < -kMaxFactorExp / 8.f;
            run += la;
            sG[r * D + c] = run;
        }
        Ptot[part * D + c] = run;
        __syncthreads();
        if (part > 0) {
            float off = 0.f;
            for (int p2 = 0; p2 < part; ++p2) off += Ptot[p2 * D + c];
#pragma unroll 4
            for (int r = part * RP; r < (part + 1) * RP; ++r) sG[r * D + c] += off;
        }
    } else if (warp == 0) {
        float x0 = Gs[2 * lane], x1 = Gs[2 * lane + 1];
        if (RAW) {
            const float bh = __ldg(rp.a_bias + h);
            x0 = 2 * lane < len ? log_sigmoid_f(x0 + bh) : 0.f;
            x1 = 2 * lane + 1 < len ? log_sigmoid_f(x1 + bh) : 0.f;
        }
        const float pair = x0 + x1;
        float incl = pair;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, m);
            if (lane >= m) incl += y;
        }
        const float excl = incl - pair;
        Gs[2 * lane] = excl + x0;
        Gs[2 * lane + 1] = excl + pair;
    }
    bad_chunk = __syncthreads_or(bad);
    }

    const int cg = tid % CG, rg = tid / CG, c0 = 8 * cg;
    const int r0 = rg * RPT;
    const int jb = r0 / 16;                                   // this thread's 16-row block

    // ---- reference points: g_last, block midpoints m_b -------------------------
    // (with raw projections computed after the input activations, so that
    // these registers are not live through them)
    float gl[8], mj[8];
    float ecross[4][8];                       // exp(m_b - m_jb) for b > jb (per-channel)
    if (!RAW) reference_points<D, SCALAR>(sG, Gs, Gl, len, jb, c0, rg, tid, gl, mj, ecross);
    // q, k, v have landed and the previous record's bulk store has finished
    // reading the region the operands go to
    {
        const bool ok = !L::kStageQKV || mbar_wait(&in_bar[1], in_phase);
        in_phase ^= 1u;
        // the previous record's bulk stores have read the staging area the
        // operands go to.  With the scalar gate at d 128 the operand build
        // writes only the part of region 2 the first store read (BS, NC); the
        // second store (Qt, PU, gamma) reaches into Bt and Kdt, written after
        // the barrier below, so it is waited for just before that barrier.
        if (tid == 0) {
            if constexpr (kLateRecWait) bulk_wait_group_read<1>();
            else bulk_wait_group_read0();
        }
        if constexpr (RAW) {
            cp_async_wait_all();                       // the halo rows
#pragma unroll
            for (int u = 0; u < kTapsPer; ++u)         // the taps, tap-major
                if (tid + u * NT < 3 * 4 * D) {
                    const int i = tid + u * NT;     // (tensor, tap) row i / D, channel i % D
                    reinterpret_cast<float*>(sm + L::Taps)[i - i % D + g_col(i % D)] = taps[u];
                }
        }
        failed = __syncthreads_or(!ok);
        if (failed) {
            if (tid == 0) atomicOr(err, 1u);
            break;
        }
    }

    // ---- raw projections: conv-4, L2 norm of q and k, beta ----------------------
    // (the input activations, "kda-graft", section "Идея и архитектура").  Row
    // r of the chunk reads raw rows r-3 .. r (the three before the chunk from
    // the halo, zero before the sequence start); tap 3 is the current token.
    // The staged q, k, v rows are replaced by their activated values once
    // every thread has read the raw rows it needs.  Each thread keeps the rows
    // and channels it builds the operands from below.
    if constexpr (RAW) {
        if (tid < len) Bs[tid] = sigmoid_f(Bs[tid]);
        uint4 y[3][RPT];                      // activated rows, as bf16 (how they are stored)
#pragma unroll
        for (int tsr = 0; tsr < 3; ++tsr) {
            const InT* stg = reinterpret_cast<const InT*>(sm + (tsr == 0 ? L::sQ : (tsr == 1 ? L::sK : L::sV)));
            const float* wsm = reinterpret_cast<const float*>(sm + L::Taps) + (size_t)tsr * 4 * D;
            float2 w[4][4];                       // [tap][channel pair]
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float t8[8];
                load8g(wsm + (size_t)j * D, c0, t8);
#pragma unroll
                for (int p = 0; p < 4; ++p) w[j][p] = make_float2(t8[2 * p], t8[2 * p + 1]);
            }
            // the RPT + 3 raw rows r0 - 3 .. r0 + RPT - 1 this thread's rows read,
            // each loaded once
            const InT* hal = reinterpret_cast<const InT*>(sm + L::Halo) + (size_t)tsr * 3 * D;
            uint4 xr[RPT + 3];                    // as stored (bf16): raw projections are bf16
#pragma unroll
            for (int i = 0; i < RPT + 3; ++i) {
                const int rr = r0 - 3 + i;
                xr[i] = *reinterpret_cast<const uint4*>(rr >= 0 ? stg + (size_t)rr * D + c0 : hal + (size_t)(rr + 3) * D + c0);
            }
#pragma unroll
            for (int u = 0; u < RPT; ++u) {
                // x of tap j: raw row r0 + u - 3 + j, as channel pairs, on
                // packed fp32 FMAs (__ffma2_rn: two fmaf per instruction)
                float2 acc[4];
#pragma unroll
                for (int j = 3; j >= 0; --j) {
                    const uint4 q4 = xr[u + j];
                    const float2 x2[4] = {unpack_bf16(q4.x), unpack_bf16(q4.y), unpack_bf16(q4.z), unpack_bf16(q4.w)};
#pragma unroll
                    for (int p = 0; p < 4; ++p)
                        acc[p] = (j == 3) ? __fmul2_rn(w[3][p], x2[p]) : __ffma2_rn(w[j][p], x2[p], acc[p]);
                }
                if (tsr < 2) {
                    // L2 norm over the row's D channels: CG consecutive lanes
                    float2 s2 = __fmul2_rn(acc[0], acc[0]);
#pragma unroll
                    for (int p = 1; p < 4; ++p) s2 = __ffma2_rn(acc[p], acc[p], s2);
                    float ss = s2.x + s2.y;
#pragma unroll
                    for (int m = 1; m < CG; m <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                    const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
                    const float2 inv2 = make_float2(inv, inv);
#pragma unroll
                    for (int p = 0; p < 4; ++p) acc[p] = __fmul2_rn(acc[p], inv2);
                }
                y[tsr][u] = make_uint4(pack_bf16(acc[0].x, acc[0].y), pack_bf16(acc[1].x, acc[1].y),
                                       pack_bf16(acc[2].x, acc[2].y), pack_bf16(acc[3].x, acc[3].y));
            }
        }
        __syncthreads();                      // every raw row has been read
#pragma unroll
        for (int tsr = 0; tsr < 3; ++tsr) {
            uint8_t* stg = sm + (tsr == 0 ? L::sQ : (tsr == 1 ? L::sK : L::sV));
#pragma unroll
            for (int u = 0; u < RPT; ++u)
                *reinterpret_cast<uint4*>(stg + ((size_t)(r0 + u) * D + c0) * sizeof(InT)) = y[tsr][u];
        }
        // the operand passes below read only this thread's rows and channels;
        // beta and other threads' rows are read after the next barrier
        reference_points<D, SCALAR>(sG, Gs, Gl, len, jb, c0, rg, tid, gl, mj, ecross);
    }

    // ---- operands and per-token outputs -------------------------------------
    uint8_t* XA = sm + L::XA;
    uint8_t* Bt = sm + L::Bt;
    uint8_t* Kdt = sm + L::Kdt;
    uint8_t* Qgs = sm + L::Qgs;
    float em[8], eld[8];        // exp(m_jb), exp(g_last - m_jb)
    if (!SCALAR) {
#pragma unroll
        for (int e = 0; e < 8; ++e) { em[e] = __expf(mj[e]); eld[e] = __expf(gl[e] - mj[e]); }
    }
    uint32_t pb1[8][RPT / 2], pb2[8][RPT / 2], pkd[8][RPT / 2];   // transposed bf16 pairs
    float p_b1[8], p_bv[8], p_kd[8];                               // even row of the pair
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
        const int r = r0 + u;
        const bool valid = r < len;
        float qv[8], kv[8], vv[8], gr[8];
        const float br = Bs[r];
        if (valid && L::kStageQKV) {
            Vec8<InT>::load(reinterpret_cast<const InT*>(sm + L::sQ) + (size_t)r * D + c0, qv);
            Vec8<InT>::load(reinterpret_cast<const InT*>(sm + L::sK) + (size_t)r * D + c0, kv);
            Vec8<InT>::load(reinterpret_cast<const InT*>(sm + L::sV) + (size_t)r * D + c0, vv);
        } else if (valid) {
            Vec8<InT>::load(q + base + (size_t)r * tok_stride + c0, qv);
            Vec8<InT>::load(k + base + (size_t)r * tok_stride + c0, kv);
            Vec8<InT>::load(v + base + (size_t)r * tok_stride + c0, vv);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) qv[e] = kv[e] = vv[e] = 0.f;
        }
        if (!SCALAR) {
            if (valid) load8f(sG + (size_t)r * D + c0, gr);
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
            // channel pairs on sm_100's packed fp32 multiply (__fmul2_rn, each
            // lane rounded like fmul: the same values as scalar code, 2.4 %
            // less intra time at d 128)
            const float2 sc2 = make_float2(scale, scale), br2 = make_float2(br, br);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const int e = 2 * p;
                const float d0 = gr[e] - mj[e], d1 = gr[e + 1] - mj[e + 1];
                const float2 F = make_float2(__expf(d0), __expf(d1)), Fi = make_float2(__expf(-d0), __expf(-d1));
                const float2 q2 = make_float2(qv[e], qv[e + 1]), k2 = make_float2(kv[e], kv[e + 1]);
                const float2 em2 = make_float2(em[e], em[e + 1]), eld2 = make_float2(eld[e], eld[e + 1]);
                const float2 xq2 = __fmul2_rn(__fmul2_rn(sc2, q2), F);
                const float2 xk2 = __fmul2_rn(k2, F);
                const float2 kk2 = __fmul2_rn(k2, Fi);
                const float2 b12 = __fmul2_rn(__fmul2_rn(br2, xk2), em2);
                const float2 qg2 = __fmul2_rn(xq2, em2);
                const float2 kd2 = __fmul2_rn(kk2, eld2);
                xq[e] = xq2.x; xq[e + 1] = xq2.y; xk[e] = xk2.x; xk[e + 1] = xk2.y;
                kk0[e] = kk2.x; kk0[e + 1] = kk2.y; b1[e] = b12.x; b1[e + 1] = b12.y;
                qg[e] = qg2.x; qg[e + 1] = qg2.y; kd[e] = kd2.x; kd[e + 1] = kd2.y;
            }
        } else if (SCALAR) {
            const float G = __expf(gr[0]), Ed = __expf(gl[0] - gr[0]);   // one gate per row
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                xq[e] = scale * qv[e];
                xk[e] = kv[e];
                kk0[e] = 0.f;
                b1[e] = br * kv[e] * G;
                qg[e] = scale * qv[e] * G;
                kd[e] = kv[e] * Ed;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float G = __expf(gr[e]);
                xq[e] = 0.f;
                xk[e] = 0.f;
                kk0[e] = 0.f;
                b1[e] = br * kv[e] * G;
                qg[e] = scale * qv[e] * G;
                kd[e] = kv[e] * __expf(gl[e] - gr[e]);
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
                for (int p = 0; p < 4; ++p) {
                    const float2 r2 = (b == jb) ? make_float2(kk0[2 * p], kk0[2 * p + 1])
                                                : __fmul2_rn(make_float2(kk0[2 * p], kk0[2 * p + 1]),
                                                             make_float2(ecross[b][2 * p], ecross[b][2 * p + 1]));
                    kb[2 * p] = r2.x; kb[2 * p + 1] = r2.y;
                }
                *reinterpret_cast<uint4*>(sm + L::KT0 + sw128_chunk(160, (int)ap_col(b) + r, cg)) = pack8(kb);
            }
        }
        *reinterpret_cast<uint4*>(Qgs + sw128_chunk(64, r, cg)) = pack8(qg);
        // transposed operands: pack pairs of rows (u-1, u) per channel
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float bv = br * vv[e];
            if ((u & 1) == 0) {
                p_b1[e] = b1[e];
                p_bv[e] = bv;
                p_kd[e] = kd[e];
            } else {
                pb1[e][u / 2] = pack_bf16(p_b1[e], b1[e]);
                pb2[e][u / 2] = pack_bf16(p_bv[e], bv);
                pkd[e][u / 2] = pack_bf16(p_kd[e], kd[e]);
            }
        }
    }
    // B1^T rows c, B2^T rows D + c, Kd^T rows c (token columns r0 .. r0 + RPT - 1):
    // stored here at d 64; at d 128 while the A/P MMA runs (measured 4 % faster there,
    // no gain at d 64, where keeping the pairs live across the MMA issue spills)
    if constexpr (D == 64) {
    // B1^T rows c, B2^T rows D + c, Kd^T rows c; token columns r0 .. r0 + RPT - 1.
    // Step e of lane group cg writes channel c0 + (e ^ s), s = cg mod 8, so the
    // lanes of a warp hit 8 different swizzle positions instead of one.
    const int s8 = cg & 7;
    xor_permute(pb1, s8);
    xor_permute(pb2, s8);
    xor_permute(pkd, s8);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int c = c0 + (e ^ s8);
        const uint32_t o1 = sw128_chunk(2 * D, c, r0 / 8) + (r0 % 8) * 2;
        const uint32_t o2 = sw128_chunk(2 * D, D + c, r0 / 8) + (r0 % 8) * 2;
        const uint32_t o3 = sw128_chunk(D, c, r0 / 8) + (r0 % 8) * 2;
        if constexpr (RPT == 4) {
            *reinterpret_cast<uint2*>(Bt + o1) = make_uint2(pb1[e][0], pb1[e][RPT / 2 - 1]);
            *reinterpret_cast<uint2*>(Bt + o2) = make_uint2(pb2[e][0], pb2[e][RPT / 2 - 1]);
            *reinterpret_cast<uint2*>(Kdt + o3) = make_uint2(pkd[e][0], pkd[e][RPT / 2 - 1]);
        } else {
            *reinterpret_cast<uint32_t*>(Bt + o1) = pb1[e][0];
            *reinterpret_cast<uint32_t*>(Bt + o2) = pb2[e][0];
            *reinterpret_cast<uint32_t*>(Kdt + o3) = pkd[e][0];
        }
    }
    }
    if constexpr (kLateRecWait) {
        if (tid == 0) bulk_wait_group_read0();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    // ---- the next item's decay tile and q, k, v -------------------------------
    // This item read region 1 (g, q, k, v) in the operand build above; only a
    // chunk with extreme decay reads it again (the exact path of the A/P
    // readout), and there the tiles keep the late request with beta (which
    // the readout reads).  Otherwise they are requested now, so that the
    // decay tile has landed when warps 4-7 scan it during the solve.
    const bool tiles_early = SCALAR || !bad_chunk;
    if (tiles_early && warp == kLoadWarp) {
        const Item nxt = s_item[(iter + 1) & 1];
        if (nxt.idx >= 0) {
            fence_proxy_async_smem();             // the operand build's reads of region 1 come first
            if (lane == 0) {
                const int x = nxt.h * D;
                const uint64_t pol = l2_policy_evict_first();
                const bool hint = keep_records != 0;
                if (!SCALAR) {
                    mbar_arrive_expect_tx(&in_bar[0], 64u * D * 4u);
                    if (hint) tma_load_2d_hint(sm + L::sG, &maps.g, x, nxt.start, &in_bar[0], pol);
                    else tma_load_2d(sm + L::sG, &maps.g, x, nxt.start, &in_bar[0]);
                }
                if (L::kStageQKV) {
                    mbar_arrive_expect_tx(&in_bar[1], 3u * 64u * D * (uint32_t)sizeof(InT));
                    if (hint) {
                        tma_load_2d_hint(sm + L::sQ, &maps.q, x, nxt.start, &in_bar[1], pol);
                        tma_load_2d_hint(sm + L::sK, &maps.k, x, nxt.start, &in_bar[1], pol);
                        tma_load_2d_hint(sm + L::sV, &maps.v, x, nxt.start, &in_bar[1], pol);
                    } else {
                        tma_load_2d(sm + L::sQ, &maps.q, x, nxt.start, &in_bar[1]);
                        tma_load_2d(sm + L::sK, &maps.k, x, nxt.start, &in_bar[1]);
                        tma_load_2d(sm + L::sV, &maps.v, x, nxt.start, &in_bar[1]);
                    }
                }
            }
            ++tiles_issued;
        }
    }

    // ---- decay-weighted Q K^T and K K^T on the tensor cores ------------------
    if (tid == 0) {
        const uint32_t aXA = smem_u32(XA);
        if (!SCALAR) {
            // the four key tiles stacked as one B operand of 160 rows (tile b at
            // row ap_col(b), which is also its TMEM column): one MMA of N = 160
            // per K step instead of four of N = 16(b+1) (d 128: 4.8 % less time
            // for this kernel, the A/P MMA phase being bound by its instruction
            // count, not its work)
            const uint32_t id = idesc_bf16_f32(128, 160);
            const uint32_t aK = smem_u32(sm + L::KT0);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_bf16(tmem, sw128_desc(aXA, 128, 0, 16 * kk), sw128_desc(aK, 160, 0, 16 * kk), id, kk > 0);
        } else {
            const uint32_t id = idesc_bf16_f32(128, 64);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_bf16(tmem, sw128_desc(aXA, 128, 0, 16 * kk), sw128_desc(aXA, 128, 64, 16 * kk), id, kk > 0);
        }
        mma_commit(&mma_bar);
        ++mma_commits;
    }
    if constexpr (D != 64) {
    // B1^T rows c, B2^T rows D + c, Kd^T rows c; token columns r0 .. r0 + RPT - 1.
    // Step e of lane group cg writes channel c0 + (e ^ s), s = cg mod 8, so the
    // lanes of a warp hit 8 different swizzle positions instead of one.
    const int s8 = cg & 7;
    xor_permute(pb1, s8);
    xor_permute(pb2, s8);
    xor_permute(pkd, s8);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int c = c0 + (e ^ s8);
        const uint32_t o1 = sw128_chunk(2 * D, c, r0 / 8) + (r0 % 8) * 2;
        const uint32_t o2 = sw128_chunk(2 * D, D + c, r0 / 8) + (r0 % 8) * 2;
        const uint32_t o3 = sw128_chunk(D, c, r0 / 8) + (r0 % 8) * 2;
        if constexpr (RPT == 4) {
            *reinterpret_cast<uint2*>(Bt + o1) = make_uint2(pb1[e][0], pb1[e][RPT / 2 - 1]);
            *reinterpret_cast<uint2*>(Bt + o2) = make_uint2(pb2[e][0], pb2[e][RPT / 2 - 1]);
            *reinterpret_cast<uint2*>(Kdt + o3) = make_uint2(pkd[e][0], pkd[e][RPT / 2 - 1]);
        } else {
            *reinterpret_cast<uint32_t*>(Bt + o1) = pb1[e][0];
            *reinterpret_cast<uint32_t*>(Bt + o2) = pb2[e][0];
            *reinterpret_cast<uint32_t*>(Kdt + o3) = pkd[e][0];
        }
    }
        fence_proxy_async_smem();     // read by later MMAs, after the next barrier
    }
    failed = !mbar_wait(&mma_bar, phase);
    phase ^= 1u;
    tc_fence_after_sync();

    // ---- P (masked, bf16 operand) and A (masked, times beta, fp32) ----------
    // the NG warps on the same TMEM lanes read the same rows; each writes
    // 64 / NG of the columns
    {
        constexpr int CWc = 64 / NG;                          // columns per warp group
        const int sub = warp & 3;
        const bool is_p = sub < 2;
        const int rr = 32 * (sub & 1) + lane;                 // chunk row
        const int lim = is_p ? rr : rr - 1;                   // last valid key index
        const int i0 = CWc * wgrp;                            // first column of this group
        float v32[CWc];
        if (!SCALAR) {
            float vrow[64];
            if ((sub & 1) == 0) load_ap_row<0>(tmem + lane_base, rr >> 4, vrow);
            else load_ap_row<1>(tmem + lane_base, rr >> 4, vrow);
#pragma unroll
            for (int il = 0; il < CWc; ++il) {
                float x = vrow[il];
#pragma unroll
                for (int g = 1; g < NG; ++g) x = (wgrp == g) ? vrow[CWc * g + il] : x;
                v32[il] = x;
            }
        } else {
            if constexpr (CWc == 32) tmem_ld32(tmem + lane_base + (uint32_t)i0, v32);
            else tmem_ld16(tmem + lane_base + (uint32_t)i0, v32);
            tmem_ld_wait();
            const float gr = Gs[rr];
#pragma unroll
            for (int il = 0; il < CWc; ++il)
                v32[il] = (i0 + il <= lim) ? v32[il] * __expf(gr - Gs[i0 + il]) : 0.f;
        }
        if (!SCALAR && bad_chunk) {
            // exact path: every term with its own exp (chunks with extreme decay only)
#pragma unroll
            for (int il = 0; il < CWc; ++il) {
                const int i = i0 + il;
                float acc = 0.f;
                if (i <= lim && rr < len) {
                    for (int c = 0; c < D; ++c) {
                        // q and k as staged (the same values as in memory; with
                        // raw projections, the activated ones)
                        float qr, kr, ki;
                        if (L::kStageQKV) {
                            const InT* sq = reinterpret_cast<const InT*>(sm + L::sQ);
                            const InT* sk = reinterpret_cast<const InT*>(sm + L::sK);
                            qr = (float)sq[rr * D + c];
                            kr = (float)sk[rr * D + c];
                            ki = (float)sk[i * D + c];
                        } else {
                            qr = (float)q[base + (size_t)rr * tok_stride + c];
                            kr = (float)k[base + (size_t)rr * tok_stride + c];
                            ki = (float)k[base + (size_t)i * tok_stride + c];
                        }
                        const float xr = is_p ? scale * qr : kr;
                        acc += xr * ki * expf(sG[rr * D + c] - sG[i * D + c]);
                    }
                }
                v32[il] = acc;
            }
        }
        if (is_p) {
#pragma unroll
            for (int jj = 0; jj < CWc / 8; ++jj) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = (i0 + 8 * jj + e <= lim) ? v32[8 * jj + e] : 0.f;
                *reinterpret_cast<uint4*>(sm + L::Pt + sw128_chunk(64, rr, i0 / 8 + jj)) = pack8(x);
            }
        } else {
            const float br = Bs[rr];
#pragma unroll
            for (int i4 = 0; i4 < CWc / 4; ++i4) {
                const int i = i0 + 4 * i4;
                float4 x;
                x.x = (i + 0 <= lim) ? br * v32[4 * i4 + 0] : 0.f;
                x.y = (i + 1 <= lim) ? br * v32[4 * i4 + 1] : 0.f;
                x.z = (i + 2 <= lim) ? br * v32[4 * i4 + 2] : 0.f;
                x.w = (i + 3 <= lim) ? br * v32[4 * i4 + 3] : 0.f;
                *reinterpret_cast<float4*>(As + rr * kLd + i) = x;
            }
        }
    }
    __syncthreads();

    // region 1 and beta are free: stage the next item's beta (and its tiles
    // if they were not requested during the A/P MMA) and, except with raw
    // projections (below), look up the item after it (read by every thread at
    // this item's end)
    if (warp == kLoadWarp) {
        const Item nxt = s_item[(iter + 1) & 1];
        fence_proxy_async_smem();             // this item's reads of region 1 come first
        if (nxt.idx >= 0) {
            issue_inputs<D, InT, SCALAR, RAW, L>(sm, &in_bar[0], &in_bar[1], maps, beta, log_a, H, nxt,
                                                 lane, keep_records != 0, !tiles_early);
            if (!tiles_early) ++tiles_issued;
        }
        if (!RAW && lane == 0)
            s_item[iter & 1] = nxt.idx >= 0 ? find_item(cu, n_seqs, H, n_items, nxt.idx + gridDim.x) : nxt;
    }

    // ---- T = (I + A)^-1: 16x16 diagonal blocks, then block merges -----------
    // T overwrites A in As block by block, each block once the phases that
    // still read it have passed a barrier.  Every phase also writes its bf16
    // copy straight into the operand tile Tb, whose blocks above the
    // diagonal are zeroed here.
    // Warps 0-3 solve (named barrier 1); warps 4-7 meanwhile scan the next
    // item's log a, which the loader warp has just requested.
    uint8_t* Tb = sm + L::Tb;
    if (tid < 128) {
        // with raw projections the item after the next one (a chain of
        // dependent loads of cu_seqlens) is looked up by warp 2, idle while
        // warps 0-1 solve the diagonal blocks, instead of by the loader warp:
        // there the next item's decay scan (with its log_sigmoid) outlasts the
        // solve, and the loader warp's share of it would finish last (1-2.5 %
        // faster); with ready inputs the scan ends first and the lookup on
        // warp 2 would only delay the solve (1 % slower)
        if (RAW && tid == 64) {
            const Item nxt = s_item[(iter + 1) & 1];
            s_item[iter & 1] = nxt.idx >= 0 ? find_item(cu, n_seqs, H, n_items, nxt.idx + gridDim.x) : nxt;
        }
        if (tid >= 64) {
            // (row, chunk) pairs of the zero blocks (b, j > b): 96 + 64 + 32
#pragma unroll
            for (int z = tid - 64; z < 192; z += 64) {
                int r, jj;
                if (z < 96) { r = z / 6; jj = 2 + z % 6; }
                else if (z < 160) { r = 16 + (z - 96) / 4; jj = 4 + (z - 96) % 4; }
                else { r = 32 + (z - 160) / 2; jj = 6 + (z - 160) % 2; }
                *reinterpret_cast<uint4*>(Tb + sw128_chunk(64, r, jj)) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        if (tid < 64) {
            // column cc of T_bb, right-looking: once x_j is known it is folded
            // into every later row's running sum, so each step waits on one FMA
            const int b = tid >> 4, cc = tid & 15, o = 16 * b;
            float x[16], acc[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) acc[r] = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                x[j] = (j < cc) ? 0.f : ((j == cc) ? 1.f : -acc[j]);
#pragma unroll
                for (int r = j + 1; r < 16; ++r) acc[r] = fmaf(As[(o + r) * kLd + o + j], x[j], acc[r]);
            }
            __syncwarp();          // every lane has read A_bb before T_bb overwrites it
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                As[(o + r) * kLd + o + cc] = x[r];
                *reinterpret_cast<__nv_bfloat16*>(Tb + sw128_offset(64, o + r, o + cc)) = __float2bfloat16_rn(x[r]);
            }
        }
        solve_bar();
        // first-level merges inside each 32-row half: T_10 = -T_11 A_10 T_00 and
        // T_32 = -T_33 A_32 T_22 (a 2 x 4 tile per thread, 64 threads)
        const int t32 = tid & 31, rr0 = 2 * (t32 >> 2), c4 = 4 * (t32 & 3);
        if (tid < 64) {
            const int p = tid >> 5, b = 2 * p + 1, j = 2 * p;
            float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
            tile16<kLd>(As, 16 * b + rr0, 16 * j, As, 16 * j, 16 * j + c4, y0, y1);
            *reinterpret_cast<float4*>(Yt + p * 256 + rr0 * 16 + c4) = make_float4(y0[0], y0[1], y0[2], y0[3]);
            *reinterpret_cast<float4*>(Yt + p * 256 + (rr0 + 1) * 16 + c4) = make_float4(y1[0], y1[1], y1[2], y1[3]);
        }
        solve_bar();
        if (tid < 64) {
            const int p = tid >> 5, b = 2 * p + 1, j = 2 * p;
            float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
            tile16<16>(As, 16 * b + rr0, 16 * b, Yt + p * 256, 0, c4, z0, z1);
            store_t_tile(As, Tb, 16 * b + rr0, 16 * j + c4, z0, z1);
        }
        solve_bar();
        // bottom-left 32 x 32 block, blocks (b, j) with b in {2, 3}, j in {0, 1}:
        //   Y_bj = sum_{l=j}^{1} A_bl T_lj        T_bj = -sum_{l=2}^{b} T_bl Y_lj
        {
            const int q = (tid >> 5) & 3, b = 2 + (q >> 1), j = q & 1;
            if (tid < 128) {
                float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
                for (int l = j; l <= 1; ++l)
                    tile16<kLd>(As, 16 * b + rr0, 16 * l, As, 16 * l, 16 * j + c4, y0, y1);
                *reinterpret_cast<float4*>(Yt + (16 * (b - 2) + rr0) * 32 + 16 * j + c4) = make_float4(y0[0], y0[1], y0[2], y0[3]);
                *reinterpret_cast<float4*>(Yt + (16 * (b - 2) + rr0 + 1) * 32 + 16 * j + c4) = make_float4(y1[0], y1[1], y1[2], y1[3]);
            }
            solve_bar();
            if (tid < 128) {
                float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
                for (int l = 2; l <= b; ++l)
                    tile16<32>(As, 16 * b + rr0, 16 * l, Yt, 16 * (l - 2), 16 * j + c4, z0, z1);
                store_t_tile(As, Tb, 16 * b + rr0, 16 * j + c4, z0, z1);
            }
        }
    } else if (kEarlyScan && tid < 256) {
        // the next item's chunk-local cumulative decay (see the item start)
        const Item nx = s_item[(iter + 1) & 1];
        bool nbad = false;
        if (nx.idx >= 0) {
            if (!mbar_wait(&in_bar[0], in_phase)) failed = true;
            nbad = scan_channels<D, 128, RAW>(sG, nx.len, tid - 128,
                                              RAW ? rp.a_bias + (size_t)nx.h * D : nullptr);
        }
        nbad = bar_or(2, 128, nbad);
        if (tid == 128) s_bad_next = nbad ? 1 : 0;
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    failed = __syncthreads_or(failed);
    tc_fence_after_sync();

    // ---- [W | U]^T = [diag(b)(K*Gamma) | diag(b)V]^T T^T ---------------------
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
        ++mma_commits;
        ++mma_commits;
    }
    if (!failed && !mbar_wait(&mma_bar, phase)) failed = true;
    phase ^= 1u;
    tc_fence_after_sync();

    // W^T rows c and U^T rows v -> one bf16 tile [2D][64] (row D + v for U^T)
    {
        uint8_t* WUt = sm + L::WUt;
        const int lrow = 32 * (warp & 3) + lane;
        // (part, piece) = (128-row part, 32-column piece), dealt round-robin
        // to the warp groups
#pragma unroll
        for (int part = 0; part < 2 * D / 128; ++part) {
            const int row = lrow + 128 * part;
#pragma unroll
            for (int piece = 0; piece < 2; ++piece) {
                if ((2 * part + piece) % NG != wgrp) continue;
                float x[32];
                tmem_ld32(tmem + lane_base + 64 * part + 32 * piece, x);
                tmem_ld_wait();
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = x[8 * jj + e];
                    *reinterpret_cast<uint4*>(WUt + sw128_chunk(2 * D, row, 4 * piece + jj)) = pack8(y);
                }
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    failed = __syncthreads_or(failed);
    tc_fence_after_sync();

    // ---- P [W | U], Kd^T W, U^T Kd --------------------------------------------
    if (tid == 0 && !failed) {
        const uint32_t aP = smem_u32(sm + L::Pt), aWU = smem_u32(sm + L::WUt), aKd = smem_u32(Kdt);
        const uint32_t id_pwu = idesc_bf16_f32(64, 2 * D);
        const uint32_t id_dd = idesc_bf16_f32(D, D);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            mma_bf16(tmem, sw128_desc(aP, 64, 0, 16 * kk), sw128_desc(aWU, 2 * D, 0, 16 * kk), id_pwu, kk > 0);
            mma_bf16(tmem + 2 * D, sw128_desc(aKd, D, 0, 16 * kk), sw128_desc(aWU, 2 * D, 0, 16 * kk), id_dd, kk > 0);
            mma_bf16(tmem + 3 * D, sw128_desc(aWU, 2 * D, D, 16 * kk), sw128_desc(aKd, D, 0, 16 * kk), id_dd, kk > 0);
        }
        mma_commit(&mma_bar);
        ++mma_commits;
    }
    if (!failed && !mbar_wait(&mma_bar, phase)) failed = true;
    phase ^= 1u;
    tc_fence_after_sync();

    // ---- record: Qt = Qg - P W, PU, BS = -Kd^T W, NC = U^T Kd, gamma ----------
    // assembled in region 2 and the dead Bt, Kdt (everything there is dead
    // once the MMAs above have completed) and written with two bulk stores,
    // the second of which drains while the next item starts
    uint8_t* srec = sm + L::Rec;
    // rows of the M = 64 products live in lanes 16 w + l (l < 16)
    const int r64 = 16 * (warp & 3) + lane;
    const bool act64 = lane < 16;
    {
        const int rD = (D == 128) ? (32 * (warp & 3) + lane) : r64;
        const bool actD = (D == 128) || act64;
#pragma unroll
        for (int piece = 0; piece < D / 32; ++piece) {
            if (piece % NG != wgrp) continue;
            float bs[32], nc[32];
            tmem_ld32(tmem + lane_base + 2 * D + 32 * piece, bs);
            tmem_ld32(tmem + lane_base + 3 * D + 32 * piece, nc);
            tmem_ld_wait();
            if (actD) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int chunk = 4 * piece + jj;
                    float a[8], b[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) { a[e] = -bs[8 * jj + e]; b[e] = nc[8 * jj + e]; }
                    *reinterpret_cast<uint4*>(srec + R.BS + sw128_chunk(D, rD, chunk)) = pack8(a);
                    *reinterpret_cast<uint4*>(srec + R.NC + sw128_chunk(D, rD, chunk)) = pack8(b);
                }
            }
        }
    }
    // BS and NC (the larger part) go out first; their bulk store drains while
    // Qt, PU and gamma are assembled
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        if (keep_records) bulk_s2g_hint(rec + R.BS, srec + R.BS, 4u * D * D, l2_policy_evict_last());
        else bulk_s2g(rec + R.BS, srec + R.BS, 4u * D * D);
        bulk_commit_group();
    }
    {
#pragma unroll
        for (int piece = 0; piece < D / 32; ++piece) {
            if (piece % NG != wgrp) continue;
            float pw[32], pu[32];
            tmem_ld32(tmem + lane_base + 32 * piece, pw);
            tmem_ld32(tmem + lane_base + D + 32 * piece, pu);
            tmem_ld_wait();
            if (act64) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int chunk = 4 * piece + jj;
                    float qgv[8];
                    Vec8<__nv_bfloat16>::load(reinterpret_cast<const __nv_bfloat16*>(Qgs + sw128_chunk(64, r64, chunk)), qgv);
                    float a[8], b[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) { a[e] = qgv[e] - pw[8 * jj + e]; b[e] = pu[8 * jj + e]; }
                    *reinterpret_cast<uint4*>(srec + R.Qt + sw128_chunk(64, r64, chunk)) = pack8(a);
                    *reinterpret_cast<uint4*>(srec + R.PU + sw128_chunk(64, r64, chunk)) = pack8(b);
                }
            }
        }
        if (tid < D) reinterpret_cast<float*>(srec + R.gamma)[tid] = expf(Gl[tid]);
    }
    const Item nxt = s_item[(iter + 1) & 1];  // read before the loader may overwrite it
    fence_proxy_async_smem();
    tc_fence_before_sync();
    failed = __syncthreads_or(failed);
    tc_fence_after_sync();
    if (tid == 0) {
        if (keep_records) bulk_s2g_hint(rec + R.Qt, srec + R.Qt, R.bytes - 4u * D * D, l2_policy_evict_last());
        else bulk_s2g(rec + R.Qt, srec + R.Qt, R.bytes - 4u * D * D);
        bulk_commit_group();
        if (failed) atomicOr(err, 1u);
    }
    if (failed) break;                        // a timed-out MMA: stop issuing work
    cur = nxt;
    ++iter;
    pre_scanned = kEarlyScan;
    }

    pdl_launch_dependents();
    if (failed) {
        // a wait gave up: nothing this CTA started may still be running when it
        // releases its tensor memory and exits -- the last committed MMA and
        // the last requested inputs (at most one of each is outstanding; these
        // waits are bounded too)
        if (tid == 0 && mma_commits > 0) (void)mbar_wait(&mma_bar, (mma_commits - 1u) & 1u);
        if (warp == kLoadWarp && lane == 0 && tiles_issued > 0) {
            if (!SCALAR) (void)mbar_wait(&in_bar[0], (tiles_issued - 1u) & 1u);
            if (L::kStageQKV) (void)mbar_wait(&in_bar[1], (tiles_issued - 1u) & 1u);
        }
    }
    cp_async_wait_all();
    if (tid == 0) bulk_wait_group0();
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Unpack records into plain fp32 arrays (inspection / tests only).
template <int D>
__global__ void unpack_kernel(const int32_t* __restrict__ cu, int n_seqs, int H,
                              const uint8_t* __restrict__ records, float* Qt, float* PU, float* BS,
                              float* NC, float* gamma) {
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
        Qt[sh * 64 * D + e] = bf(R.Qt + sw128_offset(64, r, c));
        PU[sh * 64 * D + e] = bf(R.PU + sw128_offset(64, r, c));
    }
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
        const int r = e / D, c = e % D;
        BS[sh * D * D + e] = bf(R.BS + sw128_offset(D, r, c));
        NC[sh * D * D + e] = bf(R.NC + sw128_offset(D, r, c));
    }
    for (int c = threadIdx.x; c < D; c += blockDim.x)
        gamma[sh * D + c] = reinterpret_cast<const float*>(rec + R.gamma)[c];
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, fetched through the runtime once.
cudaError_t tensor_map_encoder(EncodeTiledFn* fn) {
    static EncodeTiledFn cached = nullptr;
    if (!cached) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || p == nullptr) return cudaErrorSymbolNotFound;
        cached = reinterpret_cast<EncodeTiledFn>(p);
    }
    *fn = cached;
    return cudaSuccess;
}

// Map of a token-major [T][H][D] tensor as [T][H * D], box 64 tokens x D.
cudaError_t token_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, CUtensorMapDataType dt,
                      uint32_t elem, int64_t T, int H, int D) {
    const cuuint64_t dims[2] = {(cuuint64_t)H * D, (cuuint64_t)T};
    const cuuint64_t strides[1] = {(cuuint64_t)H * D * elem};
    const cuuint32_t box[2] = {(cuuint32_t)D, 64u};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D, typename InT, bool SCALAR, bool RAW>
cudaError_t launch_typed(const gdr_prefill_args& a, const RawParams& rp, uint8_t* records,
                         uint32_t* err, cudaStream_t st) {
    auto kern = intra_chunk_kernel<D, InT, SCALAR, RAW>;
    using Lay = IntraLayout<D, InT, SCALAR, RAW>;
    const uint32_t smem = Lay::dyn_bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // all of the unified L1 / shared memory as shared memory, so that the
    // occupancy below (two CTAs per SM at d 64) is what the launch gets
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    // persistent grid: every CTA that fits on the device at once, items
    // (chunk slot, head) handed out round-robin
    static thread_local int cached_dev = -1, resident = 0;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev != cached_dev) {
        // CTAs per SM from the kernel's registers and shared memory (the
        // occupancy calculator under-reports the two CTAs per SM that fit at
        // d 64); at most two, which is what the TMEM columns allow
        int sms = 0, smem_sm = 0, rsv = 0;
        cudaFuncAttributes fa;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess)
            return e;
        if ((e = cudaDeviceGetAttribute(&rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess) return e;
        if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
        const int cta_smem = ((int)(smem + fa.sharedSizeBytes) + rsv + 127) & ~127;
        const int cta_regs = ((fa.numRegs + 7) & ~7) * threads_for<D, SCALAR>();
        int per_sm = smem_sm / cta_smem;
        per_sm = per_sm < 65536 / cta_regs ? per_sm : 65536 / cta_regs;
        per_sm = per_sm < 2 ? per_sm : 2;
        resident = sms * (per_sm > 0 ? per_sm : 1);
        cached_dev = dev;
    }
    const int64_t n_items = n_chunk_slots(a.total_tokens, a.n_seqs) * (int64_t)a.n_heads;
    EncodeTiledFn enc = nullptr;
    if ((e = tensor_map_encoder(&enc)) != cudaSuccess) return e;
    InputMaps maps;
    memset(&maps, 0, sizeof(maps));
    const CUtensorMapDataType dt = sizeof(InT) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    if (Lay::kStageQKV) {
        if ((e = token_map(enc, &maps.q, a.q, dt, sizeof(InT), a.total_tokens, a.n_heads, D)) != cudaSuccess) return e;
        if ((e = token_map(enc, &maps.k, a.k, dt, sizeof(InT), a.total_tokens, a.n_heads, D)) != cudaSuccess) return e;
        if ((e = token_map(enc, &maps.v, a.v, dt, sizeof(InT), a.total_tokens, a.n_heads, D)) != cudaSuccess) return e;
    }
    if (!SCALAR &&
        (e = token_map(enc, &maps.g, a.log_a, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.total_tokens, a.n_heads, D)) != cudaSuccess)
        return e;
    const unsigned grid = (unsigned)(n_items < resident ? n_items : resident);
    return launch_pdl(true, kern, dim3(grid), dim3(threads_for<D, SCALAR>()), smem, st, a.cu_seqlens,
                      a.n_seqs, a.n_heads, (const InT*)a.q, (const InT*)a.k, (const InT*)a.v, a.beta,
                      a.log_a, a.scale, n_items, records, err, maps,
                      records_fit_l2(n_chunk_slots(a.total_tokens, a.n_seqs), a.n_heads, D) ? 1 : 0, rp);
}

template <int D, typename InT, bool RAW>
cudaError_t launch_decay(const gdr_prefill_args& a, const RawParams& rp, uint8_t* records,
                         uint32_t* err, cudaStream_t st) {
    return a.scalar_decay ? launch_typed<D, InT, true, RAW>(a, rp, records, err, st)
                          : launch_typed<D, InT, false, RAW>(a, rp, records, err, st);
}

}  // namespace

cudaError_t launch_intra_chunk(const gdr_prefill_args& a, uint8_t* records, uint32_t* err,
                               cudaStream_t st) {
    if (n_chunk_slots(a.total_tokens, a.n_seqs) == 0) return cudaSuccess;
    const RawParams none{};
    if (a.d_k == 64)
        return a.qkv_dtype == GDR_BF16 ? launch_decay<64, __nv_bfloat16, false>(a, none, records, err, st)
                                       : launch_decay<64, float, false>(a, none, records, err, st);
    return a.qkv_dtype == GDR_BF16 ? launch_decay<128, __nv_bfloat16, false>(a, none, records, err, st)
                                   : launch_decay<128, float, false>(a, none, records, err, st);
}

// The same stage from raw projections (bf16 only): a's q, k, v, beta and
// log_a are x_q, x_k, x_v, beta_raw and a_raw.
cudaError_t launch_intra_chunk_raw(const gdr_prefill_args& a, const float* wq, const float* wk,
                                   const float* wv, const float* a_bias, uint8_t* records,
                                   uint32_t* err, cudaStream_t st) {
    if (n_chunk_slots(a.total_tokens, a.n_seqs) == 0) return cudaSuccess;
    if (a.qkv_dtype != GDR_BF16) return cudaErrorInvalidValue;
    const RawParams rp{wq, wk, wv, a_bias};
    return a.d_k == 64 ? launch_decay<64, __nv_bfloat16, true>(a, rp, records, err, st)
                       : launch_decay<128, __nv_bfloat16, true>(a, rp, records, err, st);
}

cudaError_t launch_unpack_records(const gdr_prefill_args& a, const uint8_t* records, float* Qt,
                                  float* PU, float* BS, float* NC, float* gamma, cudaStream_t st) {
    const int64_t slots = n_chunk_slots(a.total_tokens, a.n_seqs);
    if (slots == 0) return cudaSuccess;
    const dim3 grid((unsigned)slots, (unsigned)a.n_heads);
    if (a.d_k == 64)
        unpack_kernel<64><<<grid, 256, 0, st>>>(a.cu_seqlens, a.n_seqs, a.n_heads, records, Qt, PU, BS, NC, gamma);
    else
        unpack_kernel<128><<<grid, 256, 0, st>>>(a.cu_seqlens, a.n_seqs, a.n_heads, records, Qt, PU, BS, NC, gamma);
    return cudaGetLastError();
}

}  // namespace gdr
