// internal.h -- launch helpers and the prefill workspace layout shared by the
// host API (gdr_api.cu) and the kernels.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "gdr.h"

namespace gdr {

constexpr int kChunk = 64;          // tokens per chunk (C)

// Number of chunk slots for a packed batch: chunk j of sequence n lives in slot
// floor((cu[n] + 64 j) / 64) + n.  Slots of different chunks never collide and
// all are below floor(T / 64) + N.
inline int64_t n_chunk_slots(int64_t total_tokens, int n_seqs) {
    return total_tokens / kChunk + n_seqs;
}

// One chunk-head record of the workspace, written by the intra-chunk kernel
// and read by the state-pass kernel.  With S0 the chunk's start state
// (d_v x d_k), the chunk's effect is affine in S0:
//     S_next = S0 Diag(gamma) + S0 BS^T + NC        O = Qt S0^T + PU
// so the sequential pass needs one product per chunk for the state.
// Qt and BS are tensor-core operand tiles (K-major, 128-byte swizzle, see
// sm100.cuh); PU and NC are read row by row by threads (same swizzle of their
// 16-byte chunks, so rows read without bank conflicts).
// The parts the state-only pass needs (BS, NC) come first and everything the
// pass reads is one contiguous span (`used` bytes), fetched by one bulk copy:
// a CTA's bulk copies are served one after another, so their number, not
// their size, sets the fetch time of a small record.
struct RecordLayout {
    uint32_t BS;      // [D x D]   row c': -(Kd^T W)[c', :]                    (bf16)
    uint32_t NC;      // [D x D]   row v: (U^T Kd)[v, :]                       (bf16)
    uint32_t Qt;      // [64 x D]  row r: scale q_r exp(g_r) - (P W)_r        (bf16)
    uint32_t PU;      // [64 x D]  row r: (P U)_r                              (bf16)
    uint32_t gamma;   // [D]       exp(g_last)                                 (fp32)
    uint32_t used;    // bytes up to the end of gamma (a multiple of 16)
    uint32_t bytes;   // slot size, a multiple of 1024 (tile alignment)
};

__host__ __device__ constexpr RecordLayout record_layout(int D) {
    return RecordLayout{0u,
                        (uint32_t)(2 * D * D),
                        (uint32_t)(4 * D * D),
                        (uint32_t)(4 * D * D + 128 * D),
                        (uint32_t)(4 * D * D + 256 * D),
                        (uint32_t)(4 * D * D + 256 * D + 4 * D),
                        (uint32_t)(((4 * D * D + 256 * D + 4 * D) + 1023) / 1024 * 1024)};
}

// Launch, with programmatic stream serialization when `early`: the kernel's
// CTAs may then be scheduled while the previous kernel in the stream drains,
// hiding the launch gap.  Every kernel launched here calls pdl_wait()
// (sm100.cuh) before its first global memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(bool early, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = early ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Records small enough to stay in L2 (126 MB) between the two stages are
// written and first read with an evict-last hint (and the inputs read with
// evict-first); larger sets use the default cache policy.
inline bool records_fit_l2(int64_t n_slots, int H, int D) {
    return (double)n_slots * H * record_layout(D).bytes <= 96.0 * 1024 * 1024;
}

// Sequence segmentation of the sequential pass.  With few (sequence, head)
// pairs the chunk-to-chunk chain leaves most SMs idle, so each sequence is cut
// into segments of seg_chunks chunks: every segment first runs from a zero
// state while also carrying the identity (its chunks' composed affine map
// S_end = S_start M + N), a short fp32 chain combines the maps into each
// segment's true start state, and every segment then replays its chunks from
// that state to produce its outputs.  seg_chunks == 0 means one pass.
inline int segment_chunks(int n_seqs, int H, int64_t T, int D) {
    if (n_seqs <= 0 || T <= 0) return 0;
    const int64_t pairs = (int64_t)n_seqs * H;
    // about two CTAs per SM (the state-pass kernels fit two per SM at d = 64;
    // at d = 128 two waves of shorter segments beat one wave of longer ones),
    // never more: a CTA past the last full wave costs a whole segment's time
    // (16 heads at d 128: 19 segments = 304 CTAs, 8 of them in a third wave)
    (void)D;
    const int64_t target_ctas = 2 * 148;
    int64_t segs = target_ctas / pairs;
    if (segs <= 1) return 0;                  // enough pairs for one pass
    if (segs > 32) segs = 32;
    const int64_t avg_chunks = (T / n_seqs + kChunk - 1) / kChunk;
    int64_t sc = (avg_chunks + segs - 1) / segs;
    if (sc < 7) sc = 7;
    if (segs <= 1 || sc >= avg_chunks) return 0;
    return (int)sc;
}

// Segment slot of segment j of sequence n: floor(cu[n] / span) + j + n with
// span = 64 seg_chunks tokens (same collision-free scheme as chunk slots).
inline int64_t n_segment_slots(int64_t total_tokens, int n_seqs, int seg_chunks) {
    return seg_chunks > 0 ? total_tokens / ((int64_t)kChunk * seg_chunks) + n_seqs : 0;
}

struct WorkspaceLayout {
    size_t err_off;     // uint32 error word (0 = ok)
    size_t rec_off;     // chunk-head records
    size_t seg_off;     // per (segment slot, head): N, M, E, each [D x D] fp32
    int64_t n_slots;
    int64_t n_seg_slots;
    int seg_chunks;
    size_t rec_bytes;
    // d_k != d_v: the narrower side's inputs widened to D = max(d_k, d_v)
    // (zero channels), each [T, H, D] with 4 bytes per element reserved
    size_t wq_off, wk_off, wg_off, wv_off;   // 0 when not used
    size_t total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WorkspaceLayout workspace_layout(int n_seqs, int H, int D, int64_t T, int scalar) {
    WorkspaceLayout w{};
    (void)scalar;
    w.err_off = 0;
    w.rec_off = 1024;
    w.n_slots = n_chunk_slots(T, n_seqs);
    w.rec_bytes = record_layout(D).bytes;
    w.seg_off = align_up(w.rec_off + (size_t)w.n_slots * (size_t)H * w.rec_bytes, 1024);
    w.seg_chunks = segment_chunks(n_seqs, H, T, D);
    w.n_seg_slots = n_segment_slots(T, n_seqs, w.seg_chunks);
    w.total = w.seg_off + (size_t)w.n_seg_slots * (size_t)H * 3u * (size_t)D * D * sizeof(float);
    w.wq_off = w.wk_off = w.wg_off = w.wv_off = 0;
    return w;
}

// Workspace of a prefill with key width dk and value width dv: the square
// layout for D = max(dk, dv), then (dk != dv) the widened inputs.
inline WorkspaceLayout workspace_layout_dims(int n_seqs, int H, int dk, int dv, int64_t T,
                                             int scalar) {
    const int D = dk > dv ? dk : dv;
    WorkspaceLayout w = workspace_layout(n_seqs, H, D, T, scalar);
    if (dk == dv) return w;
    const size_t arr = align_up((size_t)T * (size_t)H * (size_t)D * 4u, 1024);
    size_t off = align_up(w.total, 1024);
    if (dk < D) {
        w.wq_off = off; off += arr;
        w.wk_off = off; off += arr;
        if (!scalar) { w.wg_off = off; off += arr; }
    } else {
        w.wv_off = off; off += arr;
    }
    w.total = off;
    return w;
}

// Kernel launchers (each returns the launch's cudaError_t).
cudaError_t launch_cumdecay(int n_seqs, int H, int D, int64_t T, const int32_t* cu,
                            const float* log_a, int scalar, float* g, cudaStream_t st);

cudaError_t launch_intra_chunk(const gdr_prefill_args& a, uint8_t* records, uint32_t* err,
                               cudaStream_t st);

cudaError_t launch_intra_chunk_raw(const gdr_prefill_args& a, const float* wq, const float* wk,
                                   const float* wv, const float* a_bias, uint8_t* records,
                                   uint32_t* err, cudaStream_t st);

cudaError_t launch_state_pass(const gdr_prefill_args& a, const uint8_t* records,
                              const WorkspaceLayout& lay, uint8_t* ws, uint32_t* err,
                              cudaStream_t st);

cudaError_t launch_unpack_records(const gdr_prefill_args& a, const uint8_t* records,
                                  float* Qt, float* PU, float* BS, float* NC, float* gamma,
                                  cudaStream_t st);

cudaError_t launch_decode(int B, int H, int dk, int dv, gdr_dtype dt, const void* q,
                          const void* k, const void* v, const float* beta,
                          const float* log_a, int scalar, float scale, float* state,
                          float* o, cudaStream_t st);

cudaError_t launch_decode_gated(int B, int H, int dk, int dv, gdr_dtype dt, const void* q,
                                const void* k, const void* v, const float* beta,
                                const float* log_a, int scalar, float scale, float* state,
                                const void* gate_raw, const float* norm_weight, float norm_eps,
                                float* o, cudaStream_t st);

cudaError_t launch_preprocess(const gdr_preprocess_args& a, cudaStream_t st);

// Copy rows of width w of a [rows, w] array into [rows, D] with zeros past w
// (elem = 2 or 4 bytes; w and D multiples of 64).
cudaError_t launch_widen(const void* src, void* dst, int64_t rows, int w, int D, int elem,
                         cudaStream_t st);

cudaError_t launch_decode_draft(int B, int K, int H, int dk, int dv, gdr_dtype dt, const void* q,
                                const void* k, const void* v, const float* beta,
                                const float* log_a, int scalar, float scale, const float* state,
                                float* o, float* token_states, cudaStream_t st);

cudaError_t launch_decode_accept(int B, int K, int H, int dk, int dv, const int32_t* n_accept,
                                 const float* token_states, float* state, cudaStream_t st);

// Device helper: slot -> (sequence, chunk index).  f(n) = floor(cu[n]/64) + n is
// strictly increasing, so the owner of slot j is the largest n with f(n) <= j.
// Returns false if the slot holds no chunk.
__device__ __forceinline__ bool slot_to_span(const int32_t* __restrict__ cu, int n_seqs,
                                             int64_t slot, int span, int* seq, int* start,
                                             int* len) {
    int lo = 0, hi = n_seqs - 1, found = -1;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const int64_t f = (int64_t)(__ldg(cu + mid) / span) + mid;
        if (f <= slot) { found = mid; lo = mid + 1; } else { hi = mid - 1; }
    }
    if (found < 0) return false;
    const int s0 = __ldg(cu + found), s1 = __ldg(cu + found + 1);
    const int64_t c = slot - ((int64_t)(s0 / span) + found);
    const int64_t st = (int64_t)s0 + c * span;
    if (st >= s1) return false;
    *seq = found;
    *start = (int)st;
    *len = (int)((s1 - st) < span ? (s1 - st) : span);
    return true;
}

__device__ __forceinline__ bool slot_to_chunk(const int32_t* __restrict__ cu, int n_seqs,
                                              int64_t slot, int* seq, int* start, int* len) {
    return slot_to_span(cu, n_seqs, slot, kChunk, seq, start, len);
}

__host__ __device__ inline int64_t chunk_slot(int32_t seq_start, int seq, int chunk_idx) {
    return (int64_t)((seq_start + (int64_t)chunk_idx * kChunk) / kChunk) + seq;
}

}  // namespace gdr
