// state_pass.cu -- sequential inter-chunk pass of the chunked prefill.
//
// "Modele hybrydowe: co Gated DeltaNet zastępuje w cache KV", closing
// paragraph of "Co stan rekurencyjny zmienia przy serwowaniu": inside a chunk
// the updates are dense matrix products; only the step from one chunk to the
// next is sequential.  This file is that sequential step.  The intra-chunk
// kernel has reduced each chunk to an affine map of its start state S0
// (d_v x d_k, fp32):
//     S_next = S0 Diag(gamma) + S0 BS^T + NC          O = Qt S0^T + PU
// (record layout in internal.h).  Per chunk, two tcgen05 MMAs read the bf16
// copy of S0 from shared memory:
//     Z = S0 BS^T  (M = d_v, N = d_k, K = d_k)   -> the state, on the critical path
//     O = Qt S0^T  (M = 64,  N = d_v, K = d_k)   -> the outputs, off it
// The fp32 master state stays in registers for the whole run (8 warps; a
// thread owns half of a state row); S = S * gamma + Z + NC is done in fp32.
// The outputs of chunk k are read from tensor memory before chunk k+1's MMAs
// are issued, then added to PU and stored while those run.  Each record
// arrives by one bulk (TMA) copy, prefetched up to kStages chunks ahead, and
// every kernel of the pass is launched early (programmatic dependent launch).
// Snapshots of the state
// are written at every snap_interval boundary (section "Co stan
// rekurencyjny...", point 1: prefix reuse needs the state at that position).
//
// Long sequences with few heads are cut into segments (internal.h): kLocal
// runs each segment from a zero state and from the identity at once, giving
// the segment's affine map (N, M); combine_kernel chains the maps into each
// segment's true start state E in fp32; kApply replays each segment from E to
// produce its outputs, snapshots and, for the last segment, the final state.
// kFull is the single pass over whole sequences.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace gdr {
namespace {

constexpr int kThreads = 256;
enum Mode { kFull = 0, kLocal = 1, kApply = 2 };

template <typename T> struct Out8;
template <> struct Out8<float> {
    static __device__ __forceinline__ void store(float* p, const float (&x)[8]) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
        *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
    }
};
template <> struct Out8<__nv_bfloat16> {
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&x)[8]) {
        uint4 u;
        u.x = pack_bf16(x[0], x[1]); u.y = pack_bf16(x[2], x[3]);
        u.z = pack_bf16(x[4], x[5]); u.w = pack_bf16(x[6], x[7]);
        *reinterpret_cast<uint4*>(p) = u;
    }
};

// Barrier of warps w and w + 4 (w = sub in 0..3) on named barrier 1 + w.
template <int ID>
__device__ __forceinline__ void pair_bar_id() {
    asm volatile("bar.sync %0, 64;" ::"n"(ID) : "memory");
}
__device__ __forceinline__ void pair_bar(int sub) {
    if (sub == 0) pair_bar_id<1>();
    else if (sub == 1) pair_bar_id<2>();
    else if (sub == 2) pair_bar_id<3>();
    else pair_bar_id<4>();
}

template <typename T> struct In8;
template <> struct In8<float> {
    static __device__ __forceinline__ void load(const float* p, float (&x)[8]) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p));
        const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};
template <> struct In8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[8]) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), c = unpack_bf16(u.z), d = unpack_bf16(u.w);
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y; x[4] = c.x; x[5] = c.y; x[6] = d.x; x[7] = d.y;
    }
};

// Output epilogue of the mixer ("kda-graft", section "Идея и архитектура":
// every KDA layer of the graft ends in an RMSNorm and an output gate):
//     y = o / sqrt(mean_c o_c^2 + eps) * w * sigmoid(gate_raw)
// over the d_v channels of each (token, head), w [d_v] shared by the heads.
struct OutputGate {
    const void* gate;        // [T, H, d_v], the outputs' dtype; NULL: no epilogue
    const float* weight;     // [d_v]
    float eps;
};

template <int D, int MODE>
struct PassLayout {
    static constexpr RecordLayout R = record_layout(D);
    static constexpr bool kOut = MODE != kLocal;
    static constexpr int kStages = (D == 64) ? 3 : 2;
    // rows of the bf16 state operand: S (and the identity-started X rows in kLocal)
    static constexpr int kRows = (MODE == kLocal) ? 2 * D : D;
    static constexpr uint32_t S = 0;                                        // bf16 [kRows x D]
    // kStages record images, 1024-byte aligned, at the record's own offsets:
    // the whole record with outputs (one bulk copy); BS, NC and then gamma
    // (two copies) without
    static constexpr uint32_t Rec0 = S + 2u * kRows * D;
    static constexpr uint32_t kGamma = kOut ? R.gamma : 4u * D * D;         // gamma in a stage
    static constexpr uint32_t kStride = kOut ? R.bytes : 4u * D * D + 1024u;
    static constexpr uint32_t bytes = Rec0 + (kStages - 1) * kStride + kGamma + 4u * D;
    static constexpr uint32_t dyn_bytes = bytes + 1024u;
    // record parts (see the kernel): split at d 128 only
    static constexpr bool kSplit = (D == 128);
    static constexpr uint32_t tx_whole = kOut ? R.used : 4u * D * D + 4u * D;
    static constexpr uint32_t tx_a = kSplit ? 2u * D * D + (kOut ? 128u * D : 0u) : tx_whole;   // BS (Qt)
    static constexpr uint32_t tx_b = 2u * D * D + (kOut ? R.used - R.PU : 4u * D);              // NC, (PU,) gamma
    static_assert(kStride % 1024u == 0u && Rec0 % 1024u == 0u, "tile alignment");
    static_assert(dyn_bytes + 128u <= 232448u, "shared memory budget");
};

// GATED: the output epilogue is applied (og.gate is set); a template
// parameter so that the plain kernels keep their register allocation.
template <int D, typename OutT, int MODE, bool GATED>
__global__ void __launch_bounds__(kThreads, (D == 64) ? 2 : 1)
state_pass_kernel(const int32_t* __restrict__ cu, int n_seqs, int H,
                  const uint8_t* __restrict__ records, const float* init_state,
                  OutT* __restrict__ o, float* final_state, int snap_interval,
                  float* __restrict__ snapshots, const int64_t* __restrict__ snap_offsets,
                  int seg_chunks, float* seg_ws, uint32_t* err, int keep_records,
                  const __grid_constant__ OutputGate og, int dk, int dv) {
    using L = PassLayout<D, MODE>;
    constexpr RecordLayout R = record_layout(D);
    constexpr int ST = L::kStages;
    constexpr bool kOut = L::kOut;
    constexpr bool kSplit = L::kSplit;
    // M of the state product: D rows (kLocal, D = 64: S and X stacked, 128 rows;
    // kLocal, D = 128: two products of 128 rows)
    constexpr int kMS = (MODE == kLocal && D == 64) ? 128 : D;
    constexpr int kNT = (MODE == kLocal && D == 128) ? 2 : 1;      // state products
    constexpr uint32_t kTmemCols = (D == 64) ? 256u : 512u;
    constexpr int CW = D / 2;                                       // columns per thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align_smem<1024>(smem_raw);
    // record parts of each stage: A = the MMA's operands (BS, and Qt with
    // outputs), B = the rest (NC, gamma, and PU with outputs)
    __shared__ uint64_t full_a[ST], full_b[ST];
    __shared__ uint64_t mma_bar;
#ifdef GDR_TEST_WAIT_LIMIT_NS
    // test builds only: a barrier nothing arrives on, waited for with a short
    // limit at the second chunk, so that the timeout path runs on demand
    __shared__ uint64_t never_bar;
#endif
    __shared__ uint32_t tmem_slot;
    __shared__ int64_t snap_base_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sub = warp & 3, half = warp >> 2;
    pdl_wait();                               // the previous kernel's memory is final
    int n, h, s0, s1, seg_start;
    if (MODE == kFull) {
        n = blockIdx.x / H;
        h = blockIdx.x % H;
        s0 = __ldg(cu + n);
        s1 = __ldg(cu + n + 1);
        seg_start = s0;
    } else {
        int len_span;
        if (!slot_to_span(cu, n_seqs, blockIdx.x, kChunk * seg_chunks, &n, &s0, &len_span)) return;
        h = blockIdx.y;
        seg_start = __ldg(cu + n);
        s1 = s0 + len_span;
    }
    const int chunk0 = (s0 - seg_start) / kChunk;             // absolute chunk index of chunk 0
    const int nchunks = (s1 - s0 + kChunk - 1) / kChunk;
    float* seg_base = seg_ws ? seg_ws + ((size_t)blockIdx.x * H + h) * 3u * D * D : nullptr;

    // thread -> state row (tensor-memory lane layout of the M = kMS product)
    const int row = (kMS == 128) ? (32 * sub + lane) : (16 * sub + lane);
    const bool active = (kMS == 128) || (lane < 16);
    const bool is_x = (MODE == kLocal && D == 64) && row >= D;     // identity-started rows
    const int srow = is_x ? row - D : row;                          // row within S or X
    const int cb = half * CW;                                       // first column
    // thread -> output row (lane layout of an M = 64 product), columns [cb, cb + CW)
    const int orow = 16 * sub + lane;
    const bool oactive = lane < 16;

    auto record_of = [&](int c) -> const uint8_t* {
        const int64_t slot = (int64_t)(seg_start / kChunk) + chunk0 + c + n;
        return records + ((size_t)slot * H + h) * R.bytes;
    };
    auto stage = [&](int s) { return sm + L::Rec0 + (uint32_t)s * L::kStride; };
    // At d 128 (two stages) each record comes in two parts with a barrier
    // each, so that a stage's operand part can be refilled as soon as the MMA
    // that read it has completed, a whole chunk earlier than the rest, whose
    // last reader is the chunk's output step: part A = BS (and Qt), part B =
    // NC, gamma (and PU) -- 15 % off the single pass at d 128.  At d 64 three
    // stages hide the copies already and one copy per record (part A is the
    // whole record, no part B) measured faster.  A CTA's bulk copies are served
    // one after another.  Thread 0 only.
    auto policy = [&]() {
        // a record set that fits in L2: the state-only pass leaves it there
        // for the replay, the passes with outputs read it for the last time
        return (MODE == kLocal) ? l2_policy_evict_last() : l2_policy_evict_first();
    };
    auto copy = [&](uint8_t* dst, const uint8_t* src, uint32_t n, uint64_t* bar) {
        if (keep_records) bulk_g2s_hint(dst, src, n, bar, policy());
        else bulk_g2s(dst, src, n, bar);
    };
    auto issue_a = [&](int c) {
        const int s = c % ST;
        const uint8_t* r = record_of(c);
        mbar_arrive_expect_tx(&full_a[s], L::tx_a);
        if (!kSplit && kOut) {
            copy(stage(s), r, R.used, &full_a[s]);                               // the whole record
        } else if (!kSplit) {
            copy(stage(s) + R.BS, r + R.BS, 4u * D * D, &full_a[s]);              // BS and NC
            copy(stage(s) + L::kGamma, r + R.gamma, 4u * D, &full_a[s]);
        } else {
            copy(stage(s) + R.BS, r + R.BS, 2u * D * D, &full_a[s]);
            if (kOut) copy(stage(s) + R.Qt, r + R.Qt, 128u * D, &full_a[s]);
        }
    };
    auto issue_b = [&](int c) {
        const int s = c % ST;
        const uint8_t* r = record_of(c);
        mbar_arrive_expect_tx(&full_b[s], L::tx_b);
        copy(stage(s) + R.NC, r + R.NC, 2u * D * D, &full_b[s]);
        if (kOut) copy(stage(s) + R.PU, r + R.PU, R.used - R.PU, &full_b[s]);        // PU and gamma
        else copy(stage(s) + L::kGamma, r + R.gamma, 4u * D, &full_b[s]);
    };

    int a_issued = 0, b_issued = 0;                                 // thread 0's bookkeeping
    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full_a[s], 1);
            mbar_init(&full_b[s], 1);
        }
        mbar_init(&mma_bar, 1);
#ifdef GDR_TEST_WAIT_LIMIT_NS
        mbar_init(&never_bar, 1);
#endif
        fence_mbar_init();
        // the first records start arriving while the initial state is loaded
        for (int c = 0; c < ST && c < nchunks; ++c) {
            issue_a(c);
            if (kSplit) issue_b(c);
        }
        a_issued = min(ST, nchunks);
        b_issued = kSplit ? a_issued : 0;
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, kTmemCols);
        // first snapshot slot of sequence n: the caller's offsets, or the sum
        // of the earlier sequences' snapshot counts
        int64_t acc = 0;
        if (kOut && snap_interval > 0 && !snap_offsets)
            for (int m = lane; m < n; m += 32) acc += (__ldg(cu + m + 1) - __ldg(cu + m)) / snap_interval;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (kOut && snap_interval > 0 && snap_offsets) acc = __ldg(snap_offsets + n);
        if (lane == 0) snap_base_s = acc;
    }

    // ---- initial state --------------------------------------------------------
    // S[t][j]: tile t (0 = S, 1 = X for kLocal with two products), column cb + j.
    // The caller's states are d_v x d_k; with d_k != d_v the kernel works on
    // D x D (D = max) and the extra rows / columns stay zero.
    float S[kNT][CW];
    const size_t state_off = ((size_t)n * H + h) * dv * dk;     // caller's layout
    const float* src = nullptr;
    bool src_user = true;                                         // caller's layout or E
    if (MODE == kFull) src = init_state;
    if (MODE == kApply) {
        if (s0 == seg_start) src = init_state;
        else { src = seg_base + 2u * D * D; src_user = false; }  // E: this segment's start state
    }
    const bool row_in = srow < dv;                                // a row of the caller's state
#pragma unroll
    for (int t = 0; t < kNT; ++t) {
        const bool x_tile = (MODE == kLocal) && (t == 1 || is_x);
#pragma unroll
        for (int j = 0; j < CW; j += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (MODE != kLocal && active && src) {
                if (!src_user)
                    x = *reinterpret_cast<const float4*>(src + (size_t)srow * D + cb + j);
                else if (row_in && cb + j < dk)
                    x = *reinterpret_cast<const float4*>(src + state_off + (size_t)srow * dk + cb + j);
            }
            if (x_tile) {
                const int c = cb + j;
                x = make_float4(c + 0 == srow ? 1.f : 0.f, c + 1 == srow ? 1.f : 0.f,
                                c + 2 == srow ? 1.f : 0.f, c + 3 == srow ? 1.f : 0.f);
            }
            S[t][j] = x.x; S[t][j + 1] = x.y; S[t][j + 2] = x.z; S[t][j + 3] = x.w;
        }
    }
    uint8_t* sS = sm + L::S;
    auto write_operand = [&](int t, int j0) {   // bf16 copy of columns cb + j0 .. + 8
        const int orow_t = (MODE == kLocal && D == 128) ? row + t * D : row;
        uint4 u;
        u.x = pack_bf16(S[t][j0 + 0], S[t][j0 + 1]);
        u.y = pack_bf16(S[t][j0 + 2], S[t][j0 + 3]);
        u.z = pack_bf16(S[t][j0 + 4], S[t][j0 + 5]);
        u.w = pack_bf16(S[t][j0 + 6], S[t][j0 + 7]);
        *reinterpret_cast<uint4*>(sS + sw128_chunk(L::kRows, orow_t, (cb + j0) / 8)) = u;
    };
    if (active) {
#pragma unroll
        for (int t = 0; t < kNT; ++t)
#pragma unroll
            for (int j = 0; j < CW; j += 8) write_operand(t, j);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_slot;
    const uint32_t lane_base = (uint32_t)(32 * sub) << 16;
    const int64_t snap_base = snap_base_s;

    const uint32_t id_z = idesc_bf16_f32(kMS, D);
    const uint32_t id_o = idesc_bf16_f32(64, D);
    const uint32_t aS = smem_u32(sS);
    auto issue_mma = [&](int c) {        // thread 0 only; operands of chunk c are resident
        const int s = c % ST;
        const uint32_t aBS = smem_u32(stage(s) + R.BS);
        tc_fence_after_sync();
#pragma unroll
        for (int t = 0; t < kNT; ++t)
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_bf16(tmem + (uint32_t)(t * 128), sw128_desc(aS, L::kRows, t * 128, 16 * kk),
                         sw128_desc(aBS, D, 0, 16 * kk), id_z, kk > 0);
        if (kOut) {
            const uint32_t aQt = smem_u32(stage(s) + R.Qt);
            const uint32_t o_col = (uint32_t)D * (1 + (c & 1));
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_bf16(tmem + o_col, sw128_desc(aQt, 64, 0, 16 * kk), sw128_desc(aS, D, 0, 16 * kk),
                         id_o, kk > 0);
        }
        mma_commit(&mma_bar);
    };

    bool failed = false;
    int a_waited = 0, b_waited = 0, mmas_issued = 0;                // thread 0's bookkeeping
    if (tid == 0 && nchunks > 0) {
        if (!mbar_wait(&full_a[0], 0)) failed = true;
        a_waited = 1;
        issue_mma(0);
        mmas_issued = 1;
    }
    int mmas_waited = 0;

    // output epilogue with bf16 outputs: this chunk's raw gate values are
    // loaded at the top of its iteration, so that the loads complete during
    // the waits and the state update instead of on the output path
    constexpr bool kGatePre = GATED && kOut && sizeof(OutT) == 2;
    constexpr int kGateVec = kGatePre ? CW / 8 : 1;
    for (int k = 0; k < nchunks; ++k) {
        const int st = k % ST;
        const int t0 = s0 + k * kChunk;
        const int len = min(kChunk, s1 - t0);
        uint4 gpre[kGateVec];
        if (kGatePre && GATED && oactive && orow < len && cb < dv) {
            const uint4* g = reinterpret_cast<const uint4*>(static_cast<const OutT*>(og.gate) +
                                                            ((size_t)(t0 + orow) * H + h) * dv + cb);
#pragma unroll
            for (int i = 0; i < kGateVec; ++i) gpre[i] = __ldg(g + i);
        }
        if (!mbar_wait(kSplit ? &full_b[st] : &full_a[st], (uint32_t)(k / ST) & 1)) failed = true;
        if (tid == 0 && kSplit) b_waited = k + 1;
#ifdef GDR_TEST_WAIT_LIMIT_NS
        if (k == 1 && !mbar_wait_for(&never_bar, 0u, (uint64_t)GDR_TEST_WAIT_LIMIT_NS)) failed = true;
#endif
        const float* gam = reinterpret_cast<const float*>(stage(st) + L::kGamma);
        const uint8_t* nc = stage(st) + R.NC;
        // gamma and this row's NC, read while the MMAs of chunk k finish
        // (at d 64 with outputs the registers go to the early output read)
        constexpr bool kPre = (kNT == 1) && !(kOut && D == 64);
        float gv[kPre ? CW : 1];
        uint32_t nvp[kPre ? CW / 2 : 1];
        if (kPre && active) {
#pragma unroll
            for (int j = 0; j < CW; j += 4) {
                const float4 g4 = *reinterpret_cast<const float4*>(gam + cb + j);
                gv[j] = g4.x; gv[j + 1] = g4.y; gv[j + 2] = g4.z; gv[j + 3] = g4.w;
            }
            if (!is_x) {
#pragma unroll
                for (int j = 0; j < CW; j += 8) {
                    const uint4 u = *reinterpret_cast<const uint4*>(nc + sw128_chunk(D, srow, (cb + j) / 8));
                    nvp[j / 2] = u.x; nvp[j / 2 + 1] = u.y; nvp[j / 2 + 2] = u.z; nvp[j / 2 + 3] = u.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < CW / 2; ++j) nvp[j] = 0u;
            }
        }
        if (!mbar_wait(&mma_bar, (uint32_t)k & 1)) failed = true;
        mmas_waited = k + 1;
        tc_fence_after_sync();
        // the MMAs of chunk k have read this stage's part A: refill it
        if (kSplit && tid == 0 && !failed && k + ST < nchunks) {
            issue_a(k + ST);
            a_issued = k + ST + 1;
        }

        // ---- state: S = S * gamma + Z (+ NC for S rows), critical path ----------
#pragma unroll
        for (int t = 0; t < kNT; ++t) {
            const bool x_tile = (MODE == kLocal) && (t == 1 || is_x);
#pragma unroll
            for (int p = 0; p < CW / 32; ++p) {
                float z[32];
                tmem_ld16(tmem + lane_base + (uint32_t)(t * 128) + cb + 32 * p, *reinterpret_cast<float(*)[16]>(z));
                tmem_ld16(tmem + lane_base + (uint32_t)(t * 128) + cb + 32 * p + 16, *reinterpret_cast<float(*)[16]>(z + 16));
                tmem_ld_wait();
                if (active) {
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = 32 * p + 8 * jj, c = cb + j;
                        float g8[8], n8[8];
                        if (kPre) {
#pragma unroll
                            for (int e2 = 0; e2 < 4; ++e2) {
                                const float2 f = unpack_bf16(nvp[(j + 2 * e2) / 2]);
                                n8[2 * e2] = f.x; n8[2 * e2 + 1] = f.y;
                            }
#pragma unroll
                            for (int e = 0; e < 8; ++e) g8[e] = gv[j + e];
                        } else {
                            const float4 g0 = *reinterpret_cast<const float4*>(gam + c);
                            const float4 g1 = *reinterpret_cast<const float4*>(gam + c + 4);
                            g8[0] = g0.x; g8[1] = g0.y; g8[2] = g0.z; g8[3] = g0.w;
                            g8[4] = g1.x; g8[5] = g1.y; g8[6] = g1.z; g8[7] = g1.w;
#pragma unroll
                            for (int e = 0; e < 8; ++e) n8[e] = 0.f;
                            if (!x_tile) {
                                const uint4 u = *reinterpret_cast<const uint4*>(nc + sw128_chunk(D, srow, c / 8));
                                const float2 n0 = unpack_bf16(u.x), n1 = unpack_bf16(u.y);
                                const float2 n2 = unpack_bf16(u.z), n3 = unpack_bf16(u.w);
                                n8[0] = n0.x; n8[1] = n0.y; n8[2] = n1.x; n8[3] = n1.y;
                                n8[4] = n2.x; n8[5] = n2.y; n8[6] = n3.x; n8[7] = n3.y;
                            }
                        }
                        // channel pairs on packed fp32 (__fadd2_rn, __ffma2_rn:
                        // each lane rounded like its scalar form; 1 % faster)
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const float2 zn = __fadd2_rn(make_float2(z[8 * jj + e], z[8 * jj + e + 1]),
                                                         make_float2(n8[e], n8[e + 1]));
                            const float2 r = __ffma2_rn(make_float2(S[t][j + e], S[t][j + e + 1]),
                                                        make_float2(g8[e], g8[e + 1]), zn);
                            S[t][j + e] = r.x;
                            S[t][j + e + 1] = r.y;
                        }
                        write_operand(t, j);
                    }
                }
            }
        }
        // this chunk's outputs Qt S0^T, read before the next chunk's MMAs are
        // issued: a tensor-memory load behind running MMAs waits for them
        constexpr bool kOEarly = kOut;
        float ov[kOut ? CW : 1];
        if (kOEarly) {
            const uint32_t o_col = (uint32_t)D * (1 + (k & 1));
#pragma unroll
            for (int p = 0; p < CW / 16; ++p)
                tmem_ld16(tmem + lane_base + o_col + cb + 16 * p, *reinterpret_cast<float(*)[16]>(ov + 16 * p));
            tmem_ld_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        if (__syncthreads_or(failed)) { failed = true; break; }
        tc_fence_after_sync();
        if (tid == 0 && k + 1 < nchunks) {
            if (!mbar_wait(&full_a[(k + 1) % ST], (uint32_t)((k + 1) / ST) & 1)) failed = true;
            a_waited = k + 2;
            issue_mma(k + 1);
            mmas_issued = k + 2;
        }
        // with three or more stages, chunk k-1's stage (free since the last
        // barrier, its reads fenced before it) takes record k-1+ST now, under
        // the MMAs just issued
        if (ST >= 3 && tid == 0 && k >= 1 && k - 1 + ST < nchunks) {
            if (kSplit) {
                issue_b(k - 1 + ST);
                b_issued = k + ST;
            } else {
                issue_a(k - 1 + ST);
                a_issued = k + ST;
            }
        }

        if (kOut) {
            // ---- snapshot and outputs of chunk k (overlap chunk k+1's MMAs) -------
            const int kabs = chunk0 + k;
            if (snap_interval > 0 && len == kChunk && ((kabs + 1) * kChunk) % snap_interval == 0 && active) {
                const int64_t slot = snap_base + ((int64_t)(kabs + 1) * kChunk) / snap_interval - 1;
                float* dst = snapshots + ((size_t)slot * H + h) * dv * dk + (size_t)srow * dk + cb;
#pragma unroll
                for (int j = 0; j < CW; j += 4)
                    if (row_in && cb + j < dk)
                        *reinterpret_cast<float4*>(dst + j) = make_float4(S[0][j], S[0][j + 1], S[0][j + 2], S[0][j + 3]);
            }
            const uint8_t* pu = stage(st) + R.PU;
            OutT* orow_ptr = o + ((size_t)(t0 + orow) * H + h) * dv + cb;
            if (GATED) {
                // o = Qt S0^T + PU in place, then the row's RMS: the two halves
                // of a row (warps w and w + 4, same lane) swap their partial sums
                // of squares through shared memory behind a barrier of the pair
                float ss = 0.f;
#pragma unroll
                for (int j = 0; j < CW; j += 8) {
                    const uint4 u = *reinterpret_cast<const uint4*>(pu + sw128_chunk(64, orow & 63, (cb + j) / 8));
                    const float2 p0 = unpack_bf16(u.x), p1 = unpack_bf16(u.y);
                    const float2 p2 = unpack_bf16(u.z), p3 = unpack_bf16(u.w);
                    ov[j + 0] += p0.x; ov[j + 1] += p0.y; ov[j + 2] += p1.x; ov[j + 3] += p1.y;
                    ov[j + 4] += p2.x; ov[j + 5] += p2.y; ov[j + 6] += p3.x; ov[j + 7] += p3.y;
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(ov[j + e], ov[j + e], ss);
                }
                // [half][row] partial sums, in this stage's NC part: the state
                // update that read it is done (barrier above), and part B is
                // refilled only after a later barrier (shared memory is full
                // at d 128; part A may already be refilling)
                float* ssq = reinterpret_cast<float*>(stage(st) + R.NC);
                if (oactive) ssq[half * 64 + orow] = ss;
                pair_bar(sub);
                const float tot = ss + (oactive ? ssq[(half ^ 1) * 64 + orow] : 0.f);
                const float rstd = rsqrtf(tot / (float)dv + og.eps);
                if (oactive && orow < len) {
                    const OutT* g = static_cast<const OutT*>(og.gate) + ((size_t)(t0 + orow) * H + h) * dv + cb;
#pragma unroll
                    for (int j = 0; j < CW; j += 8) {
                        if (cb + j >= dv) continue;
                        float gv[8], wv[8], x[8];
                        if (kGatePre) {
                            const uint4 u = gpre[j / 8];
                            const float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y);
                            const float2 c = unpack_bf16(u.z), d = unpack_bf16(u.w);
                            gv[0] = a.x; gv[1] = a.y; gv[2] = b.x; gv[3] = b.y;
                            gv[4] = c.x; gv[5] = c.y; gv[6] = d.x; gv[7] = d.y;
                        } else {
                            In8<OutT>::load(g + j, gv);
                        }
                        In8<float>::load(og.weight + cb + j, wv);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float sig = __fdividef(1.f, 1.f + __expf(-gv[e]));
                            x[e] = ov[j + e] * rstd * wv[e] * sig;
                        }
                        Out8<OutT>::store(orow_ptr + j, x);
                    }
                }
            } else {
#pragma unroll
            for (int p = 0; p < CW / 16; ++p) {
                const float* y = ov + 16 * p;
                if (!kOEarly) {
                    tmem_ld16(tmem + lane_base + (uint32_t)D * (1 + (k & 1)) + cb + 16 * p,
                              *reinterpret_cast<float(*)[16]>(ov + 16 * p));
                    tmem_ld_wait();
                }
                if (oactive && orow < len && cb + 16 * p < dv) {
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int j = 16 * p + 8 * jj;
                        const uint4 u = *reinterpret_cast<const uint4*>(pu + sw128_chunk(64, orow, (cb + j) / 8));
                        const float2 p0 = unpack_bf16(u.x), p1 = unpack_bf16(u.y);
                        const float2 p2 = unpack_bf16(u.z), p3 = unpack_bf16(u.w);
                        const float x[8] = {y[8 * jj + 0] + p0.x, y[8 * jj + 1] + p0.y,
                                            y[8 * jj + 2] + p1.x, y[8 * jj + 3] + p1.y,
                                            y[8 * jj + 4] + p2.x, y[8 * jj + 5] + p2.y,
                                            y[8 * jj + 6] + p3.x, y[8 * jj + 7] + p3.y};
                        Out8<OutT>::store(orow_ptr + j, x);
                    }
                }
            }
            }
        }
        // With two stages this chunk's stage is refilled now, once every
        // thread has read its PU.  With three or more the refill comes after
        // the next chunk's first barrier, which orders those reads already,
        // and no second barrier is needed.
        if (ST < 3) {
            fence_proxy_async_smem();         // reads of this stage, then its refill
            tc_fence_before_sync();
            if (__syncthreads_or(failed)) { failed = true; break; }
            if (tid == 0 && k + ST < nchunks) {
                if (kSplit) {
                    issue_b(k + ST);
                    b_issued = k + ST + 1;
                } else {
                    issue_a(k + ST);
                    a_issued = k + ST + 1;
                }
            }
        }
    }

    pdl_launch_dependents();
    if (failed) {
        if (tid == 0) atomicOr(err, 1u);
    } else if (active) {
        auto store_row = [&](float* dst, int t, int ncols) {
#pragma unroll
            for (int j = 0; j < CW; j += 4)
                if (cb + j < ncols)
                    *reinterpret_cast<float4*>(dst + j) = make_float4(S[t][j], S[t][j + 1], S[t][j + 2], S[t][j + 3]);
        };
        if ((MODE == kFull || (MODE == kApply && s1 == __ldg(cu + n + 1))) && row_in)
            store_row(final_state + state_off + (size_t)srow * dk + cb, 0, dk);
        if (MODE == kLocal) {
            // N (rows of S) then M (rows of X) of this segment's affine map
            store_row(seg_base + (is_x ? (size_t)D * D : 0) + (size_t)srow * D + cb, 0, D);
            if (kNT == 2) store_row(seg_base + (size_t)D * D + (size_t)srow * D + cb, kNT - 1, D);
        }
    }
    // error path: no copy or MMA of this CTA may still be in flight when it
    // exits (each of these waits is bounded too)
    if (tid == 0 && failed) {
        for (int c = mmas_waited; c < mmas_issued; ++c) mbar_wait(&mma_bar, (uint32_t)c & 1);
        for (int c = a_waited; c < a_issued; ++c) mbar_wait(&full_a[c % ST], (uint32_t)(c / ST) & 1);
        for (int c = b_waited; c < b_issued; ++c) mbar_wait(&full_b[c % ST], (uint32_t)(c / ST) & 1);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Chains the segments' affine maps into each segment's start state:
//     E_0 = init,   E_{s+1} = E_s M_s + N_s       (fp32, in the chain's order)
// Rows of the state are independent, so a CTA owns kCombineRows state rows of
// one (sequence, head).  Warp w owns the column slab [w D/8, (w+1) D/8) for
// all of the CTA's rows, so each step reads M_s from shared memory once per
// CTA: lane (j = lane % 8, kq = lane / 8) sums row j over the inner indices
// k = 4i + kq, and the four partial sums meet by a shuffle reduce-scatter.  Each step's M_s
// (rows padded so the four k of one load fall in different banks) and the
// CTA's rows of N_s are fetched kCombineBufs - 1 steps ahead by 16-byte
// cp.async from every thread (a CTA's bulk copies would be served one after
// another, one chain step each); E is double buffered, so a step needs one
// barrier.  E_s goes to the workspace of segment s (its start state); the
// last segment's own map is not needed (replaying that segment produces the
// final state).  An empty sequence has no segment: its final state is its
// initial state.
constexpr int kCombineRows = 8;
constexpr int kCombineThreads = 256;

// steps in flight: the chain step is short next to an L2 round trip
template <int D>
__host__ __device__ constexpr int combine_bufs() { return D == 64 ? 6 : 3; }

template <int D>
struct CombineLayout {
    static constexpr int kCombineBufs = combine_bufs<D>();
    static constexpr int kLdM = D + 4;                                  // padded M rows
    static constexpr int kLdE = D + 4;                                  // padded E rows
    static constexpr uint32_t M0 = 0;                                   // bufs x [D x kLdM] fp32
    static constexpr uint32_t N0 = kCombineBufs * D * kLdM * 4u;        // bufs x [rows x D] fp32
    static constexpr uint32_t E = N0 + kCombineBufs * kCombineRows * D * 4u;   // 2 x [rows x kLdE]
    static constexpr uint32_t bytes = E + 2u * kCombineRows * kLdE * 4u;
    static constexpr uint32_t dyn_bytes = bytes + 128u;
    static_assert(dyn_bytes <= 232448u, "shared memory budget");
};

template <int D>
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const int32_t* __restrict__ cu, int H, int seg_chunks, const float* init_state,
               float* final_state, float* seg_ws, uint32_t* err, int dk, int dv) {
    using L = CombineLayout<D>;
    constexpr int RB = kCombineRows;
    constexpr int NT = kCombineThreads;
    constexpr int NB = L::kCombineBufs;
    constexpr int CW = D / 8;                                           // columns per warp
    static_assert(RB == 8 && NT == 256, "8 rows x 4 inner-index phases per warp, 8 warps");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align_smem<128>(smem_raw);
    pdl_wait();                               // the previous kernel's memory is final
    const int pair = blockIdx.x, rb = blockIdx.y;
    const int n = pair / H, h = pair % H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int j = lane & 7, kq = lane >> 3, c0 = CW * warp;
    const int s0 = __ldg(cu + n), s1 = __ldg(cu + n + 1);
    const int span = kChunk * seg_chunks;
    const int nseg = (s1 - s0 + span - 1) / span;
    // the caller's states are d_v x d_k; the maps and E are D x D (D = max)
    const size_t state_off = ((size_t)n * H + h) * dv * dk;
    const size_t row_off = (size_t)(rb * RB + j) * dk + c0;             // this lane's row, slab start
    (void)err;
    if (nseg == 0) {
        if (kq == 0 && rb * RB + j < dv) {
#pragma unroll
            for (int c = 0; c < CW; c += 4) {
                if (c0 + c >= dk) continue;
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (init_state) x = *reinterpret_cast<const float4*>(init_state + state_off + row_off + c);
                *reinterpret_cast<float4*>(final_state + state_off + row_off + c) = x;
            }
        }
        return;
    }
    if (nseg == 1) return;
    const int64_t slot0 = (int64_t)(s0 / span) + n;
    float* e = reinterpret_cast<float*>(sm + L::E);
    auto seg_ptr = [&](int s) { return seg_ws + ((size_t)(slot0 + s) * H + h) * 3u * D * D; };
    auto issue = [&](int s) {      // every thread: its share of M_s and of this CTA's rows of N_s
        const int b = s % NB;
        const uint8_t* msrc = reinterpret_cast<const uint8_t*>(seg_ptr(s) + (size_t)D * D);
        const uint8_t* nsrc = reinterpret_cast<const uint8_t*>(seg_ptr(s) + (size_t)rb * RB * D);
        float* mdst = reinterpret_cast<float*>(sm + L::M0 + b * D * L::kLdM * 4u);
        uint8_t* ndst = sm + L::N0 + b * RB * D * 4u;
#pragma unroll
        for (int c = tid; c < D * D / 4; c += NT)
            cp_async16(mdst + (c / (D / 4)) * L::kLdM + 4 * (c % (D / 4)), msrc + 16 * c, 16u);
#pragma unroll
        for (int c = tid; c < RB * D / 4; c += NT) cp_async16(ndst + 16 * c, nsrc + 16 * c, 16u);
    };
    for (int c = tid; c < RB * D; c += NT) {
        const int r = c / D, col = c % D;
        const bool in = init_state && rb * RB + r < dv && col < dk;
        e[r * L::kLdE + col] = in ? init_state[state_off + (size_t)(rb * RB + r) * dk + col] : 0.f;
    }
    // steps 0 .. NB-2 in flight (one commit group per step, empty past the end)
#pragma unroll
    for (int s = 0; s < NB - 1; ++s) {
        if (s <= nseg - 2) issue(s);
        cp_async_commit();
    }
    for (int s = 0; s + 1 < nseg; ++s) {
        cp_async_wait_group<NB - 2>();             // this thread's copies of step s
        __syncthreads();                           // everyone's copies, E_s, buffer (s-1) free
        if (s + NB - 1 <= nseg - 2) issue(s + NB - 1);
        cp_async_commit();
        const int b = s % NB;
        const float* Mm = reinterpret_cast<const float*>(sm + L::M0 + b * D * L::kLdM * 4u);
        const float* Nm = reinterpret_cast<const float*>(sm + L::N0 + b * RB * D * 4u);
        const float* ec = e + (s & 1) * RB * L::kLdE + j * L::kLdE;
        float acc[CW];
#pragma unroll
        for (int c = 0; c < CW; ++c) acc[c] = 0.f;
        // inner indices in groups of 16: the loads of a group are issued
        // before its FMAs
#pragma unroll
        for (int i0 = 0; i0 < D / 4; i0 += 16) {
            float ek[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) ek[i] = ec[4 * (i0 + i) + kq];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float* mrow = Mm + (4 * (i0 + i) + kq) * L::kLdM + c0;
#pragma unroll
                for (int c = 0; c < CW; c += 4) {
                    const float4 m = *reinterpret_cast<const float4*>(mrow + c);
                    acc[c] = fmaf(ek[i], m.x, acc[c]);
                    acc[c + 1] = fmaf(ek[i], m.y, acc[c + 1]);
                    acc[c + 2] = fmaf(ek[i], m.z, acc[c + 2]);
                    acc[c + 3] = fmaf(ek[i], m.w, acc[c + 3]);
                }
            }
        }
        // reduce-scatter over the four inner-index phases: after two shuffle
        // rounds lane kq holds the full sums of columns c0 + kq * CW/4 ...
        constexpr int CH = CW / 2, CQ = CW / 4;
        const bool hi16 = (kq & 2) != 0, hi8 = (kq & 1) != 0;
        float h[CH];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const float send = hi16 ? acc[c] : acc[CH + c];
            const float keep = hi16 ? acc[CH + c] : acc[c];
            h[c] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
        float qv[CQ];
#pragma unroll
        for (int c = 0; c < CQ; ++c) {
            const float send = hi8 ? h[c] : h[CQ + c];
            const float keep = hi8 ? h[CQ + c] : h[c];
            qv[c] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
        {
            const int cq = c0 + (hi16 ? CH : 0) + (hi8 ? CQ : 0);     // this lane's columns
            float* en = e + ((s + 1) & 1) * RB * L::kLdE + j * L::kLdE + cq;
            float* eg = seg_ptr(s + 1) + 2u * D * D + (size_t)(rb * RB + j) * D + cq;
            const float* nr = Nm + j * D + cq;
#pragma unroll
            for (int c = 0; c < CQ; c += 2) {
                const float2 nv = *reinterpret_cast<const float2*>(nr + c);
                const float2 x = make_float2(qv[c] + nv.x, qv[c + 1] + nv.y);
                *reinterpret_cast<float2*>(en + c) = x;
                *reinterpret_cast<float2*>(eg + c) = x;
            }
        }
    }
    pdl_launch_dependents();
    cp_async_wait_all();
}

template <int D, typename OutT, int MODE, bool GATED>
cudaError_t launch_gated(const gdr_prefill_args& a, const uint8_t* records,
                         const WorkspaceLayout& lay, float* seg_ws, uint32_t* err, cudaStream_t st) {
    auto kern = state_pass_kernel<D, OutT, MODE, GATED>;
    const uint32_t smem = PassLayout<D, MODE>::dyn_bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid;
    if (MODE == kFull) grid = dim3((unsigned)a.n_seqs * (unsigned)a.n_heads);
    else grid = dim3((unsigned)lay.n_seg_slots, (unsigned)a.n_heads);
    // early launch (programmatic dependent launch): the kernel's CTAs take the
    // SMs the previous kernel's last CTAs leave and wait there for its memory
    // (3.7 % off the graft layer's segmented step)
    return launch_pdl(true, kern, grid, dim3(kThreads), smem, st, a.cu_seqlens, a.n_seqs, a.n_heads,
                      records, a.init_state, static_cast<OutT*>(a.o), a.final_state,
                      a.snap_interval, a.snapshots, a.snap_offsets, lay.seg_chunks, seg_ws, err,
                      records_fit_l2(lay.n_slots, a.n_heads, D) ? 1 : 0,
                      OutputGate{a.gate_raw, a.norm_weight, a.norm_eps}, a.d_k, a.d_v);
}

template <int D, typename OutT, int MODE>
cudaError_t launch_mode(const gdr_prefill_args& a, const uint8_t* records,
                        const WorkspaceLayout& lay, float* seg_ws, uint32_t* err, cudaStream_t st) {
    // the zero-state pass writes no outputs: never gated
    if constexpr (MODE != kLocal) {
        if (a.gate_raw) return launch_gated<D, OutT, MODE, true>(a, records, lay, seg_ws, err, st);
    }
    return launch_gated<D, OutT, MODE, false>(a, records, lay, seg_ws, err, st);
}

template <int D, typename OutT>
cudaError_t launch_typed(const gdr_prefill_args& a, const uint8_t* records,
                         const WorkspaceLayout& lay, uint8_t* ws, uint32_t* err, cudaStream_t st) {
    if (lay.seg_chunks <= 0) return launch_mode<D, OutT, kFull>(a, records, lay, nullptr, err, st);
    float* seg_ws = reinterpret_cast<float*>(ws + lay.seg_off);
    cudaError_t e = launch_mode<D, OutT, kLocal>(a, records, lay, seg_ws, err, st);
    if (e != cudaSuccess) return e;
    auto ck = combine_kernel<D>;
    e = cudaFuncSetAttribute(ck, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)CombineLayout<D>::dyn_bytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(true, ck, dim3((unsigned)a.n_seqs * (unsigned)a.n_heads, D / kCombineRows),
                   dim3(kCombineThreads), CombineLayout<D>::dyn_bytes, st, a.cu_seqlens,
                   a.n_heads, lay.seg_chunks, a.init_state, a.final_state, seg_ws, err, a.d_k,
                   a.d_v);
    if (e != cudaSuccess) return e;
    return launch_mode<D, OutT, kApply>(a, records, lay, seg_ws, err, st);
}

}  // namespace

cudaError_t launch_state_pass(const gdr_prefill_args& a, const uint8_t* records,
                              const WorkspaceLayout& lay, uint8_t* ws, uint32_t* err,
                              cudaStream_t st) {
    if ((int64_t)a.n_seqs * a.n_heads == 0) return cudaSuccess;
    if (a.d_k == 64 && a.d_v == 64)       // else D = 128 (d_k, d_v in {64, 128})
        return a.qkv_dtype == GDR_BF16 ? launch_typed<64, __nv_bfloat16>(a, records, lay, ws, err, st)
                                       : launch_typed<64, float>(a, records, lay, ws, err, st);
    return a.qkv_dtype == GDR_BF16 ? launch_typed<128, __nv_bfloat16>(a, records, lay, ws, err, st)
                                   : launch_typed<128, float>(a, records, lay, ws, err, st);
}

}  // namespace gdr
