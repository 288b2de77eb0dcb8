// cumdecay.cu -- chunk-local cumulative log decay.
//
// "Modele hybrydowe: co Gated DeltaNet zastępuje w cache KV", closing
// paragraph of "Co stan rekurencyjny zmienia przy serwowaniu": prefill runs
// chunk by chunk.  Inside a chunk every token's decay relative to the chunk
// start is the running sum of log a:
//     g[t] = sum_{chunk start <= i <= t} log_a[i]        (per key channel)
// Chunks are 64 tokens and restart at every sequence start; the last chunk of a
// sequence may be shorter.  The sum is kept in fp32 in the order of the tokens.
//
// One CTA per (chunk slot, head); per-channel decay uses one thread per key
// channel (coalesced across channels), scalar decay one warp per (slot, head)
// with a warp scan over the chunk's tokens.  HBM-bound: 4 bytes read and
// 4 bytes written per element.
#include "internal.h"

namespace gdr {
namespace {

// Per-channel: blockDim.x == D, grid (n_slots, H).
__global__ void cumdecay_channel_kernel(const int32_t* __restrict__ cu, int n_seqs, int H, int D,
                                        const float* __restrict__ log_a, float* __restrict__ g) {
    int seq, start, len;
    if (!slot_to_chunk(cu, n_seqs, blockIdx.x, &seq, &start, &len)) return;
    const int h = blockIdx.y, c = threadIdx.x;
    const size_t stride = (size_t)H * D;
    const float* src = log_a + (size_t)start * stride + (size_t)h * D + c;
    float* dst = g + (size_t)start * stride + (size_t)h * D + c;
    float acc = 0.f;
    int t = 0;
    for (; t + 8 <= len; t += 8) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = __ldg(src + (size_t)(t + u) * stride);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            acc += x[u];
            dst[(size_t)(t + u) * stride] = acc;
        }
    }
    for (; t < len; ++t) {
        acc += __ldg(src + (size_t)t * stride);
        dst[(size_t)t * stride] = acc;
    }
}

// Scalar: one warp per (slot, head); lane l owns tokens 2l and 2l+1.
__global__ void cumdecay_scalar_kernel(const int32_t* __restrict__ cu, int n_seqs, int H,
                                       const float* __restrict__ log_a, float* __restrict__ g) {
    int seq, start, len;
    if (!slot_to_chunk(cu, n_seqs, blockIdx.x, &seq, &start, &len)) return;
    const int h = blockIdx.y, l = threadIdx.x;
    const int t0 = 2 * l, t1 = 2 * l + 1;
    const float x0 = t0 < len ? __ldg(log_a + (size_t)(start + t0) * H + h) : 0.f;
    const float x1 = t1 < len ? __ldg(log_a + (size_t)(start + t1) * H + h) : 0.f;
    // Sequential order inside the pair, then an inclusive scan over pairs.
    // (Addition order differs from a strict left-to-right sum only by
    // associativity; every partial sum is a sum of the same terms.)
    const float pair = x0 + x1;
    float incl = pair;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, m);
        if (l >= m) incl += y;
    }
    const float excl = incl - pair;
    if (t0 < len) g[(size_t)(start + t0) * H + h] = excl + x0;
    if (t1 < len) g[(size_t)(start + t1) * H + h] = excl + pair;
}

}  // namespace

cudaError_t launch_cumdecay(int n_seqs, int H, int D, int64_t T, const int32_t* cu,
                            const float* log_a, int scalar, float* g, cudaStream_t st) {
    const int64_t slots = n_chunk_slots(T, n_seqs);
    if (slots == 0) return cudaSuccess;
    const dim3 grid((unsigned)slots, (unsigned)H);
    if (scalar)
        cumdecay_scalar_kernel<<<grid, 32, 0, st>>>(cu, n_seqs, H, log_a, g);
    else
        cumdecay_channel_kernel<<<grid, D, 0, st>>>(cu, n_seqs, H, D, log_a, g);
    return cudaGetLastError();
}

}  // namespace gdr
