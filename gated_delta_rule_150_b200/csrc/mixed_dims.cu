// mixed_dims.cu -- inputs of a prefill whose key and value widths differ.
//
// The prefill kernels work on square D x D states, D = max(d_k, d_v).  The
// narrower side is widened with zero channels, which changes nothing in the
// caller's channels of the recurrence
//     S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t:
//   * extra key channels (q = k = 0, log a = 0): every product S k, S q and
//     k k^T ignores those columns of S, and the update adds delta k^T = 0 to
//     them, so they stay at their zero start and the caller's columns evolve
//     exactly as without them;
//   * extra value channels (v = 0): rows of S evolve independently given
//     (k, beta, a), so the caller's rows are unchanged, and an extra row that
//     starts at zero keeps delta = beta (0 - 0) = 0 and stays zero.
// The state pass reads and writes the caller's d_v x d_k states and o of
// width d_v directly (extra rows and columns are neither read nor written);
// only q, k and log a (d_k < d_v) or v (d_v < d_k) are copied here into
// workspace arrays of width D.
#include <cuda_bf16.h>

#include "internal.h"

namespace gdr {
namespace {

// 16-byte vectors; w and D are multiples of 64 elements, so a vector never
// straddles the edge of the caller's width.
__global__ void widen_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t rows,
                             int w_vec, int d_vec) {
    const int64_t n = rows * d_vec;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / d_vec;
        const int c = (int)(i - r * d_vec);
        dst[i] = c < w_vec ? __ldg(src + r * w_vec + c) : make_uint4(0u, 0u, 0u, 0u);
    }
}

}  // namespace

cudaError_t launch_widen(const void* src, void* dst, int64_t rows, int w, int D, int elem,
                         cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const int per = 16 / elem;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t n = rows * (D / per);
    const int64_t blocks = (n + 255) / 256;
    const unsigned grid = (unsigned)(blocks < 8LL * sms ? blocks : 8LL * sms);
    widen_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                       rows, w / per, D / per);
    return cudaGetLastError();
}

}  // namespace gdr
