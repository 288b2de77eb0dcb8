// internal.h -- launch helpers and the prefill workspace layout shared by the
// host API (gdr_api.cu) and the kernels.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
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
// and read whole (one bulk copy) by the state-pass kernel.  Every image is a
// tensor-core operand tile in the K-major 128-byte-swizzle layout (sm100.cuh),
// so the bytes land in shared memory ready to use.
struct RecordLayout {
    uint32_t W;       // [64 x D]  rows = token r, cols = key channel   (W)
    uint32_t Qg;      // [64 x D]  rows = token r, cols = key channel   (scale q exp(g))
    uint32_t Kt;      // [D x 64]  rows = key channel, cols = token i   (Kd transposed)
    uint32_t Ut;      // [D x 64]  rows = value channel, cols = token i (U transposed)
    uint32_t P;       // [64 x 64] rows = token r, cols = token i       (masked Q K^T decay)
    uint32_t gamma;   // [D] fp32  exp(g_last)
    uint32_t bytes;   // total, a multiple of 1024
};

__host__ __device__ constexpr RecordLayout record_layout(int D) {
    return RecordLayout{0u,
                        (uint32_t)(D * 128),
                        (uint32_t)(2 * D * 128),
                        (uint32_t)(3 * D * 128),
                        (uint32_t)(4 * D * 128),
                        (uint32_t)(4 * D * 128 + 8192),
                        (uint32_t)(4 * D * 128 + 8192 + 1024)};
}

struct WorkspaceLayout {
    size_t err_off;     // uint32 error word (0 = ok)
    size_t g_off;       // fp32 cumulative log decay, same layout as log_a
    size_t rec_off;     // chunk-head records
    int64_t n_slots;
    size_t rec_bytes;
    size_t total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WorkspaceLayout workspace_layout(int n_seqs, int H, int D, int64_t T, int scalar) {
    WorkspaceLayout w{};
    w.err_off = 0;
    w.g_off = 1024;
    const size_t g_elems = (size_t)T * (size_t)H * (scalar ? 1 : (size_t)D);
    w.rec_off = align_up(w.g_off + g_elems * sizeof(float), 1024);
    w.n_slots = n_chunk_slots(T, n_seqs);
    w.rec_bytes = record_layout(D).bytes;
    w.total = w.rec_off + (size_t)w.n_slots * (size_t)H * w.rec_bytes;
    return w;
}

// Kernel launchers (each returns the launch's cudaError_t).
cudaError_t launch_cumdecay(int n_seqs, int H, int D, int64_t T, const int32_t* cu,
                            const float* log_a, int scalar, float* g, cudaStream_t st);

cudaError_t launch_intra_chunk(const gdr_prefill_args& a, const float* g, uint8_t* records,
                               uint32_t* err, cudaStream_t st);

cudaError_t launch_state_pass(const gdr_prefill_args& a, const uint8_t* records,
                              uint32_t* err, cudaStream_t st);

cudaError_t launch_unpack_records(const gdr_prefill_args& a, const uint8_t* records,
                                  float* W, float* U, float* P, float* Qg, float* Kd,
                                  float* gamma, cudaStream_t st);

cudaError_t launch_decode(int B, int H, int dk, int dv, gdr_dtype dt, const void* q,
                          const void* k, const void* v, const float* beta,
                          const float* log_a, int scalar, float scale, float* state,
                          float* o, cudaStream_t st);

// Device helper: slot -> (sequence, chunk index).  f(n) = floor(cu[n]/64) + n is
// strictly increasing, so the owner of slot j is the largest n with f(n) <= j.
// Returns false if the slot holds no chunk.
__device__ __forceinline__ bool slot_to_chunk(const int32_t* __restrict__ cu, int n_seqs,
                                              int64_t slot, int* seq, int* start, int* len) {
    int lo = 0, hi = n_seqs - 1, found = -1;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const int64_t f = (int64_t)(__ldg(cu + mid) / kChunk) + mid;
        if (f <= slot) { found = mid; lo = mid + 1; } else { hi = mid - 1; }
    }
    if (found < 0) return false;
    const int s0 = __ldg(cu + found), s1 = __ldg(cu + found + 1);
    const int64_t c = slot - ((int64_t)(s0 / kChunk) + found);
    const int64_t st = (int64_t)s0 + c * kChunk;
    if (st >= s1) return false;
    *seq = found;
    *start = (int)st;
    *len = (int)((s1 - st) < kChunk ? (s1 - st) : kChunk);
    return true;
}

__host__ __device__ inline int64_t chunk_slot(int32_t seq_start, int seq, int chunk_idx) {
    return (int64_t)((seq_start + (int64_t)chunk_idx * kChunk) / kChunk) + seq;
}

}  // namespace gdr
