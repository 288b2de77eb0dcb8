// gdr_api.cu -- the C ABI declared in include/gdr.h: argument checks, the
// prefill workspace layout and the kernel launches, all on the caller's
// stream.  Nothing here allocates, frees or synchronises (except
// gdr_prefill_status, which reads one word back by design).
#include <cstring>

#include "internal.h"

namespace {

using gdr::WorkspaceLayout;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned_elem(const void* p, gdr_dtype dt) {
    return (reinterpret_cast<uintptr_t>(p) & (dt == GDR_BF16 ? 1u : 3u)) == 0;
}

// A failed launch also leaves the runtime's last-error state set; it is
// cleared here so that the next call's launch check does not report it again.
gdr_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return GDR_OK;
    (void)cudaGetLastError();
    return GDR_ERR_CUDA;
}

bool supported_width(int d) { return d == 64 || d == 128; }

// Shared checks of the prefill arguments that do not depend on outputs.
gdr_status check_prefill_inputs(const gdr_prefill_args* a) {
    if (!a) return GDR_ERR_INVALID_ARG;
    if (a->n_seqs < 0 || a->n_heads <= 0 || a->d_k <= 0 || a->d_v <= 0 || a->total_tokens < 0)
        return GDR_ERR_INVALID_ARG;
    if (a->total_tokens > (int64_t)INT32_MAX) return GDR_ERR_INVALID_ARG;
    if (a->qkv_dtype != GDR_BF16 && a->qkv_dtype != GDR_F32) return GDR_ERR_INVALID_ARG;
    if (!supported_width(a->d_k) || !supported_width(a->d_v)) return GDR_ERR_UNSUPPORTED;
    if (!a->cu_seqlens || !aligned4(a->cu_seqlens)) return GDR_ERR_INVALID_ARG;
    if (a->total_tokens > 0) {
        const void* vec[] = {a->q, a->k, a->v};
        for (const void* p : vec)
            if (!p || !aligned16(p)) return GDR_ERR_INVALID_ARG;
        if (!a->beta || !aligned4(a->beta)) return GDR_ERR_INVALID_ARG;
        if (!a->log_a || !(a->scalar_decay ? aligned4(a->log_a) : aligned16(a->log_a)))
            return GDR_ERR_INVALID_ARG;
    }
    if (a->snap_interval < 0 || a->snap_interval % gdr::kChunk != 0) return GDR_ERR_INVALID_ARG;
    return GDR_OK;
}

// The address kernels use for `p`: a device (or managed) pointer as it is, a
// page-locked host pointer as its mapped device address (the same value under
// unified addressing).  Pageable host memory is rejected.
gdr_status kernel_address(void* p, void** out) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return GDR_ERR_INVALID_ARG;
    }
    if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) {
        *out = p;
        return GDR_OK;
    }
    if (at.type == cudaMemoryTypeHost && at.devicePointer) {
        *out = at.devicePointer;
        return aligned16(*out) ? GDR_OK : GDR_ERR_INVALID_ARG;
    }
    return GDR_ERR_INVALID_ARG;
}

gdr_status check_workspace(const gdr_prefill_args* a, WorkspaceLayout* lay) {
    *lay = gdr::workspace_layout_dims(a->n_seqs, a->n_heads, a->d_k, a->d_v, a->total_tokens,
                                      a->scalar_decay);
    if (!a->workspace || (reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
        return GDR_ERR_WORKSPACE;
    if (a->workspace_bytes < lay->total) return GDR_ERR_WORKSPACE;
    return GDR_OK;
}

// Checks of the prefill's outputs and options (not of its inputs).
gdr_status check_prefill_outputs(const gdr_prefill_args* a) {
    if (!a->final_state || !aligned16(a->final_state)) return GDR_ERR_INVALID_ARG;
    if (a->total_tokens > 0 && (!a->o || !aligned_elem(a->o, a->qkv_dtype))) return GDR_ERR_INVALID_ARG;
    if (a->init_state && !aligned16(a->init_state)) return GDR_ERR_INVALID_ARG;
    if (a->snap_interval > 0 && (!a->snapshots || !aligned16(a->snapshots)))
        return GDR_ERR_INVALID_ARG;
    if (a->snap_offsets && (reinterpret_cast<uintptr_t>(a->snap_offsets) & 7u) != 0)
        return GDR_ERR_INVALID_ARG;
    if (a->gate_raw) {
        if (!aligned16(a->gate_raw) || !a->norm_weight || !aligned16(a->norm_weight))
            return GDR_ERR_INVALID_ARG;
        if (!(a->norm_eps >= 0.f) || a->norm_eps > 3.0e38f) return GDR_ERR_INVALID_ARG;
    }
    return GDR_OK;
}

}  // namespace

extern "C" {

const char* gdr_status_string(gdr_status s) {
    switch (s) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_INVALID_ARG: return "GDR_ERR_INVALID_ARG";
        case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED";
        case GDR_ERR_WORKSPACE: return "GDR_ERR_WORKSPACE";
        case GDR_ERR_CUDA: return "GDR_ERR_CUDA";
        case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT";
    }
    return "GDR_ERR_UNKNOWN";
}

int gdr_version(void) { return 100; }

size_t gdr_prefill_workspace_size(int n_seqs, int n_heads, int d_k, int d_v,
                                  int64_t total_tokens, int scalar_decay) {
    if (n_seqs < 0 || n_heads <= 0 || total_tokens < 0) return 0;
    if (!supported_width(d_k) || !supported_width(d_v)) return 0;
    return gdr::workspace_layout_dims(n_seqs, n_heads, d_k, d_v, total_tokens, scalar_decay).total;
}

int gdr_prefill_kernel_count(int n_seqs, int n_heads, int d_k, int d_v, int64_t total_tokens,
                             int scalar_decay) {
    if (gdr_prefill_workspace_size(n_seqs, n_heads, d_k, d_v, total_tokens, scalar_decay) == 0)
        return 0;
    if (n_seqs == 0) return 0;
    const int D = d_k > d_v ? d_k : d_v;
    const int intra = total_tokens > 0 ? 1 : 0;
    // widening of the narrower side's inputs (d_k != d_v)
    const int widen = (total_tokens > 0 && d_k != d_v) ? (d_k < d_v ? (scalar_decay ? 2 : 3) : 1) : 0;
    return widen + intra + (gdr::segment_chunks(n_seqs, n_heads, total_tokens, D) > 0 ? 3 : 1);
}

int64_t gdr_snapshot_count(const int32_t* host_cu, int n_seqs, int snap_interval) {
    if (!host_cu || n_seqs < 0 || snap_interval < 0) return -1;
    if (snap_interval == 0) return 0;
    int64_t total = 0;
    for (int n = 0; n < n_seqs; ++n) {
        const int32_t len = host_cu[n + 1] - host_cu[n];
        if (len < 0) return -1;
        total += len / snap_interval;
    }
    return total;
}

gdr_status gdr_snapshot_offsets(const int32_t* host_cu, int n_seqs, int snap_interval,
                                int64_t* out) {
    if (!host_cu || !out || n_seqs < 0 || snap_interval <= 0) return GDR_ERR_INVALID_ARG;
    int64_t total = 0;
    for (int n = 0; n < n_seqs; ++n) {
        out[n] = total;
        const int32_t len = host_cu[n + 1] - host_cu[n];
        if (len < 0) return GDR_ERR_INVALID_ARG;
        total += len / snap_interval;
    }
    out[n_seqs] = total;
    return GDR_OK;
}

namespace {

// The activations gdr_prefill_from_projections stages in the workspace when
// it runs them as their own kernel: only at d 128 with a per-channel gate,
// where that chain measured faster than the fused first stage.
bool staged_activations(int d, int scalar_decay) { return d == 128 && !scalar_decay; }

size_t align256(size_t x) { return (x + 255u) & ~(size_t)255u; }

// [q | k | v] bf16, beta fp32, log a fp32, each 256-byte aligned
size_t activation_bytes(int n_heads, int d, int64_t total_tokens) {
    const size_t th = (size_t)total_tokens * (size_t)n_heads;
    return 3 * align256(th * d * 2) + align256(th * 4) + align256(th * d * 4);
}

}  // namespace

size_t gdr_prefill_from_projections_workspace_size(int n_seqs, int n_heads, int d,
                                                   int64_t total_tokens, int scalar_decay) {
    const size_t base = gdr_prefill_workspace_size(n_seqs, n_heads, d, d, total_tokens, scalar_decay);
    if (base == 0 || !staged_activations(d, scalar_decay)) return base;
    return align256(base) + activation_bytes(n_heads, d, total_tokens);
}

gdr_status gdr_prefill_from_projections(const gdr_prefill_args* a, const gdr_projections* p,
                                        void* stream) {
    if (!a || !p) return GDR_ERR_INVALID_ARG;
    // the raw tensors take the places of q, k, v, beta and log a
    gdr_prefill_args r = *a;
    r.q = p->xq;
    r.k = p->xk;
    r.v = p->xv;
    r.beta = p->beta_raw;
    r.log_a = p->a_raw;
    gdr_status s = check_prefill_inputs(&r);
    if (s != GDR_OK) return s;
    if (r.qkv_dtype != GDR_BF16 || r.d_k != r.d_v) return GDR_ERR_UNSUPPORTED;
    if (r.total_tokens > 0) {
        const void* taps[] = {p->conv_q, p->conv_k, p->conv_v};
        for (const void* t : taps)
            if (!t || !aligned16(t)) return GDR_ERR_INVALID_ARG;
        if (!p->a_bias || !(r.scalar_decay ? aligned4(p->a_bias) : aligned16(p->a_bias)))
            return GDR_ERR_INVALID_ARG;
    }
    s = check_prefill_outputs(&r);
    if (s != GDR_OK) return s;
    WorkspaceLayout lay;
    s = check_workspace(&r, &lay);
    if (s != GDR_OK) return s;
    if (r.n_seqs == 0) return GDR_OK;
    // with room for the activations (d 128, per-channel gate): gdr_preprocess
    // into the workspace's tail, then gdr_prefill from there
    if (staged_activations(r.d_k, r.scalar_decay) && r.total_tokens > 0 &&
        r.workspace_bytes >= gdr_prefill_from_projections_workspace_size(
                                 r.n_seqs, r.n_heads, r.d_k, r.total_tokens, r.scalar_decay)) {
        const size_t th = (size_t)r.total_tokens * (size_t)r.n_heads;
        uint8_t* act = static_cast<uint8_t*>(r.workspace) + align256(lay.total);
        gdr_preprocess_args pa;
        memset(&pa, 0, sizeof(pa));
        pa.n_seqs = r.n_seqs;
        pa.n_heads = r.n_heads;
        pa.d = r.d_k;
        pa.total_tokens = r.total_tokens;
        pa.cu_seqlens = r.cu_seqlens;
        pa.io_dtype = GDR_BF16;
        pa.xq = p->xq;
        pa.xk = p->xk;
        pa.xv = p->xv;
        pa.conv_q = p->conv_q;
        pa.conv_k = p->conv_k;
        pa.conv_v = p->conv_v;
        pa.beta_raw = p->beta_raw;
        pa.a_raw = p->a_raw;
        pa.a_bias = p->a_bias;
        pa.scalar_decay = r.scalar_decay;
        const size_t qkv = align256(th * r.d_k * 2);
        pa.q = act;
        pa.k = act + qkv;
        pa.v = act + 2 * qkv;
        pa.beta = reinterpret_cast<float*>(act + 3 * qkv);
        pa.log_a = reinterpret_cast<float*>(act + 3 * qkv + align256(th * 4));
        s = gdr_preprocess(&pa, stream);
        if (s != GDR_OK) return s;
        gdr_prefill_args c = *a;
        c.q = pa.q;
        c.k = pa.k;
        c.v = pa.v;
        c.beta = pa.beta;
        c.log_a = pa.log_a;
        return gdr_prefill(&c, stream);
    }
    if (r.snap_interval > 0) {
        s = kernel_address(a->snapshots, reinterpret_cast<void**>(&r.snapshots));
        if (s != GDR_OK) return s;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(r.workspace);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws + lay.err_off);
    uint8_t* rec = ws + lay.rec_off;
    if (cudaMemsetAsync(err, 0, sizeof(uint32_t), st) != cudaSuccess) return from_cuda(cudaErrorUnknown);
    if (r.total_tokens > 0) {
        s = from_cuda(gdr::launch_intra_chunk_raw(r, p->conv_q, p->conv_k, p->conv_v, p->a_bias, rec,
                                                  err, st));
        if (s != GDR_OK) return s;
    }
    return from_cuda(gdr::launch_state_pass(r, rec, lay, ws, err, st));
}

gdr_status gdr_prefill_stages(const gdr_prefill_args* a, int first, int last, void* stream) {
    if (first < 0 || last > 1 || first > last) return GDR_ERR_INVALID_ARG;
    gdr_status s = check_prefill_inputs(a);
    if (s != GDR_OK) return s;
    if (!a->final_state || !aligned16(a->final_state)) return GDR_ERR_INVALID_ARG;
    if (a->total_tokens > 0 && (!a->o || !aligned_elem(a->o, a->qkv_dtype))) return GDR_ERR_INVALID_ARG;
    if (a->init_state && !aligned16(a->init_state)) return GDR_ERR_INVALID_ARG;
    if (a->snap_interval > 0 && (!a->snapshots || !aligned16(a->snapshots)))
        return GDR_ERR_INVALID_ARG;
    if (a->snap_offsets && (reinterpret_cast<uintptr_t>(a->snap_offsets) & 7u) != 0)
        return GDR_ERR_INVALID_ARG;
    if (a->gate_raw) {
        if (!aligned16(a->gate_raw) || !a->norm_weight || !aligned16(a->norm_weight))
            return GDR_ERR_INVALID_ARG;
        if (!(a->norm_eps >= 0.f) || a->norm_eps > 3.0e38f) return GDR_ERR_INVALID_ARG;
    }
    WorkspaceLayout lay;
    s = check_workspace(a, &lay);
    if (s != GDR_OK) return s;
    if (a->n_seqs == 0) return GDR_OK;
    gdr_prefill_args args = *a;
    if (last >= 1 && a->snap_interval > 0) {
        s = kernel_address(a->snapshots, reinterpret_cast<void**>(&args.snapshots));
        if (s != GDR_OK) return s;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(args.workspace);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws + lay.err_off);
    uint8_t* rec = ws + lay.rec_off;
    if (first == 0 && cudaMemsetAsync(err, 0, sizeof(uint32_t), st) != cudaSuccess)
        return GDR_ERR_CUDA;
    if (first == 0 && args.total_tokens > 0) {
        // d_k != d_v: the intra-chunk kernel reads inputs widened to D = max
        gdr_prefill_args sq = args;
        if (a->d_k != a->d_v) {
            const int D = a->d_k > a->d_v ? a->d_k : a->d_v;
            const int elem = a->qkv_dtype == GDR_BF16 ? 2 : 4;
            const int64_t rows = a->total_tokens * a->n_heads;
            if (a->d_k < D) {
                s = from_cuda(gdr::launch_widen(a->q, ws + lay.wq_off, rows, a->d_k, D, elem, st));
                if (s == GDR_OK)
                    s = from_cuda(gdr::launch_widen(a->k, ws + lay.wk_off, rows, a->d_k, D, elem, st));
                if (s == GDR_OK && !a->scalar_decay)
                    s = from_cuda(gdr::launch_widen(a->log_a, ws + lay.wg_off, rows, a->d_k, D, 4, st));
                sq.q = ws + lay.wq_off;
                sq.k = ws + lay.wk_off;
                if (!a->scalar_decay) sq.log_a = reinterpret_cast<const float*>(ws + lay.wg_off);
            } else {
                s = from_cuda(gdr::launch_widen(a->v, ws + lay.wv_off, rows, a->d_v, D, elem, st));
                sq.v = ws + lay.wv_off;
            }
            if (s != GDR_OK) return s;
            sq.d_k = sq.d_v = D;
        }
        s = from_cuda(gdr::launch_intra_chunk(sq, rec, err, st));
        if (s != GDR_OK) return s;
    }
    if (last >= 1) return from_cuda(gdr::launch_state_pass(args, rec, lay, ws, err, st));
    return GDR_OK;
}

gdr_status gdr_prefill(const gdr_prefill_args* a, void* stream) {
    return gdr_prefill_stages(a, 0, 1, stream);
}

gdr_status gdr_snapshot_offload(const float* dev_snapshots, float* host_snapshots, size_t bytes,
                                void* compute_stream, void* copy_stream, void* event) {
    if (!event || compute_stream == copy_stream) return GDR_ERR_INVALID_ARG;
    if (bytes > 0 && (!dev_snapshots || !host_snapshots || !aligned16(dev_snapshots) ||
                      !aligned16(host_snapshots)))
        return GDR_ERR_INVALID_ARG;
    cudaEvent_t ev = static_cast<cudaEvent_t>(event);
    cudaStream_t cs = static_cast<cudaStream_t>(compute_stream);
    cudaStream_t xs = static_cast<cudaStream_t>(copy_stream);
    gdr_status s = from_cuda(cudaEventRecord(ev, cs));
    if (s != GDR_OK || bytes == 0) return s;
    s = from_cuda(cudaStreamWaitEvent(xs, ev, 0));
    if (s != GDR_OK) return s;
    return from_cuda(cudaMemcpyAsync(host_snapshots, dev_snapshots, bytes, cudaMemcpyDeviceToHost, xs));
}

gdr_status gdr_prefill_status(const void* workspace, void* stream) {
    if (!workspace) return GDR_ERR_INVALID_ARG;
    uint32_t word = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return GDR_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GDR_ERR_CUDA;
    return word == 0 ? GDR_OK : GDR_ERR_TIMEOUT;
}

gdr_status gdr_cumdecay(int n_seqs, int n_heads, int d_k, int64_t total_tokens,
                        const int32_t* cu_seqlens, const float* log_a, int scalar_decay,
                        float* g, void* stream) {
    if (n_seqs < 0 || n_heads <= 0 || total_tokens < 0 || total_tokens > (int64_t)INT32_MAX)
        return GDR_ERR_INVALID_ARG;
    if (!supported_width(d_k)) return GDR_ERR_UNSUPPORTED;
    if (!cu_seqlens || !aligned4(cu_seqlens)) return GDR_ERR_INVALID_ARG;
    if (total_tokens == 0 || n_seqs == 0) return GDR_OK;
    if (!log_a || !g || !aligned4(log_a) || !aligned4(g)) return GDR_ERR_INVALID_ARG;
    return from_cuda(gdr::launch_cumdecay(n_seqs, n_heads, d_k, total_tokens, cu_seqlens, log_a,
                                          scalar_decay, g, static_cast<cudaStream_t>(stream)));
}

gdr_status gdr_chunk_factors(const gdr_prefill_args* a, float* Qt, float* PU, float* BS,
                             float* NC, float* gamma, void* stream) {
    gdr_status s = check_prefill_inputs(a);
    if (s != GDR_OK) return s;
    if (a->d_k != a->d_v) return GDR_ERR_UNSUPPORTED;
    WorkspaceLayout lay;
    s = check_workspace(a, &lay);
    if (s != GDR_OK) return s;
    if (a->n_seqs == 0 || a->total_tokens == 0) return GDR_OK;
    const void* outs[] = {Qt, PU, BS, NC, gamma};
    for (const void* p : outs)
        if (!p || !aligned16(p)) return GDR_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(a->workspace);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws + lay.err_off);
    uint8_t* rec = ws + lay.rec_off;
    if (cudaMemsetAsync(err, 0, sizeof(uint32_t), st) != cudaSuccess) return GDR_ERR_CUDA;
    s = from_cuda(gdr::launch_intra_chunk(*a, rec, err, st));
    if (s != GDR_OK) return s;
    return from_cuda(gdr::launch_unpack_records(*a, rec, Qt, PU, BS, NC, gamma, st));
}

gdr_status gdr_decode_step(int batch, int n_heads, int d_k, int d_v, gdr_dtype qkv_dtype,
                           const void* q, const void* k, const void* v, const float* beta,
                           const float* log_a, int scalar_decay, float scale, float* state,
                           float* o, void* stream) {
    if (batch < 0 || n_heads <= 0 || d_k <= 0 || d_v <= 0) return GDR_ERR_INVALID_ARG;
    if (qkv_dtype != GDR_BF16 && qkv_dtype != GDR_F32) return GDR_ERR_INVALID_ARG;
    if (!supported_width(d_k) || !supported_width(d_v)) return GDR_ERR_UNSUPPORTED;
    if ((int64_t)batch * n_heads > (int64_t)INT32_MAX) return GDR_ERR_INVALID_ARG;
    if (batch == 0) return GDR_OK;
    const void* vec[] = {q, k, state};
    for (const void* p : vec)
        if (!p || !aligned16(p)) return GDR_ERR_INVALID_ARG;
    if (!v || !aligned_elem(v, qkv_dtype) || !beta || !aligned4(beta) || !o || !aligned4(o))
        return GDR_ERR_INVALID_ARG;
    if (!log_a || !(scalar_decay ? aligned4(log_a) : aligned16(log_a))) return GDR_ERR_INVALID_ARG;
    return from_cuda(gdr::launch_decode(batch, n_heads, d_k, d_v, qkv_dtype, q, k, v, beta, log_a,
                                        scalar_decay, scale, state, o,
                                        static_cast<cudaStream_t>(stream)));
}

gdr_status gdr_decode_step_gated(int batch, int n_heads, int d_k, int d_v, gdr_dtype qkv_dtype,
                                 const void* q, const void* k, const void* v, const float* beta,
                                 const float* log_a, int scalar_decay, float scale, float* state,
                                 const void* gate_raw, const float* norm_weight, float norm_eps,
                                 float* o, void* stream) {
    if (batch < 0 || n_heads <= 0 || d_k <= 0 || d_v <= 0) return GDR_ERR_INVALID_ARG;
    if (qkv_dtype != GDR_BF16 && qkv_dtype != GDR_F32) return GDR_ERR_INVALID_ARG;
    if (!supported_width(d_k) || !supported_width(d_v)) return GDR_ERR_UNSUPPORTED;
    if ((int64_t)batch * n_heads > (int64_t)INT32_MAX) return GDR_ERR_INVALID_ARG;
    if (batch == 0) return GDR_OK;
    const void* vec[] = {q, k, state, norm_weight};
    for (const void* p : vec)
        if (!p || !aligned16(p)) return GDR_ERR_INVALID_ARG;
    if (!v || !aligned_elem(v, qkv_dtype) || !beta || !aligned4(beta) || !o || !aligned4(o))
        return GDR_ERR_INVALID_ARG;
    if (!gate_raw || !aligned_elem(gate_raw, qkv_dtype)) return GDR_ERR_INVALID_ARG;
    if (!(norm_eps >= 0.f) || norm_eps > 3.0e38f) return GDR_ERR_INVALID_ARG;
    if (!log_a || !(scalar_decay ? aligned4(log_a) : aligned16(log_a))) return GDR_ERR_INVALID_ARG;
    return from_cuda(gdr::launch_decode_gated(batch, n_heads, d_k, d_v, qkv_dtype, q, k, v, beta,
                                              log_a, scalar_decay, scale, state, gate_raw,
                                              norm_weight, norm_eps, o,
                                              static_cast<cudaStream_t>(stream)));
}

gdr_status gdr_preprocess(const gdr_preprocess_args* a, void* stream) {
    if (!a) return GDR_ERR_INVALID_ARG;
    if (a->n_seqs < 0 || a->n_heads <= 0 || a->d <= 0 || a->total_tokens < 0 ||
        a->total_tokens > (int64_t)INT32_MAX)
        return GDR_ERR_INVALID_ARG;
    // one CTA per (32-token block, head)
    if ((a->total_tokens + 31) / 32 * (int64_t)a->n_heads > (int64_t)INT32_MAX) return GDR_ERR_INVALID_ARG;
    if (a->io_dtype != GDR_BF16 && a->io_dtype != GDR_F32) return GDR_ERR_INVALID_ARG;
    if (!supported_width(a->d)) return GDR_ERR_UNSUPPORTED;
    if (a->total_tokens == 0) return GDR_OK;
    if (a->n_seqs == 0 || !a->cu_seqlens || !aligned4(a->cu_seqlens)) return GDR_ERR_INVALID_ARG;
    const void* v16[] = {a->xq, a->xk, a->xv, a->conv_q, a->conv_k, a->conv_v, a->q, a->k, a->v};
    for (const void* p : v16)
        if (!p || !aligned16(p)) return GDR_ERR_INVALID_ARG;
    const void* gate[] = {a->a_raw, a->a_bias, a->log_a};
    for (const void* p : gate)
        if (!p || !(a->scalar_decay ? aligned4(p) : aligned16(p))) return GDR_ERR_INVALID_ARG;
    if (!a->beta_raw || !aligned4(a->beta_raw) || !a->beta || !aligned4(a->beta))
        return GDR_ERR_INVALID_ARG;
    return from_cuda(gdr::launch_preprocess(*a, static_cast<cudaStream_t>(stream)));
}

gdr_status gdr_decode_draft(int batch, int n_tokens, int n_heads, int d_k, int d_v,
                            gdr_dtype qkv_dtype, const void* q, const void* k, const void* v,
                            const float* beta, const float* log_a, int scalar_decay, float scale,
                            const float* state, float* o, float* token_states, void* stream) {
    if (batch < 0 || n_tokens < 0 || n_heads <= 0 || d_k <= 0 || d_v <= 0)
        return GDR_ERR_INVALID_ARG;
    if (qkv_dtype != GDR_BF16 && qkv_dtype != GDR_F32) return GDR_ERR_INVALID_ARG;
    if (!supported_width(d_k) || !supported_width(d_v)) return GDR_ERR_UNSUPPORTED;
    // the draft kernel runs up to four CTAs per (sequence, head)
    if ((int64_t)batch * n_heads > (int64_t)INT32_MAX / 4) return GDR_ERR_INVALID_ARG;
    if (batch == 0 || n_tokens == 0) return GDR_OK;
    const void* vec[] = {q, k, state, token_states};
    for (const void* p : vec)
        if (!p || !aligned16(p)) return GDR_ERR_INVALID_ARG;
    if (!v || !aligned_elem(v, qkv_dtype) || !beta || !aligned4(beta) || !o || !aligned4(o))
        return GDR_ERR_INVALID_ARG;
    if (!log_a || !(scalar_decay ? aligned4(log_a) : aligned16(log_a))) return GDR_ERR_INVALID_ARG;
    return from_cuda(gdr::launch_decode_draft(batch, n_tokens, n_heads, d_k, d_v, qkv_dtype, q, k,
                                              v, beta, log_a, scalar_decay, scale, state, o,
                                              token_states, static_cast<cudaStream_t>(stream)));
}

gdr_status gdr_decode_accept(int batch, int n_tokens, int n_heads, int d_k, int d_v,
                             const int32_t* n_accept, const float* token_states, float* state,
                             void* stream) {
    if (batch < 0 || n_tokens < 0 || n_heads <= 0 || d_k <= 0 || d_v <= 0)
        return GDR_ERR_INVALID_ARG;
    if (!supported_width(d_k) || !supported_width(d_v)) return GDR_ERR_UNSUPPORTED;
    if ((int64_t)batch * n_heads > (int64_t)INT32_MAX) return GDR_ERR_INVALID_ARG;
    if (batch == 0 || n_tokens == 0) return GDR_OK;
    if (!n_accept || !aligned4(n_accept)) return GDR_ERR_INVALID_ARG;
    if (!token_states || !aligned16(token_states) || !state || !aligned16(state))
        return GDR_ERR_INVALID_ARG;
    return from_cuda(gdr::launch_decode_accept(batch, n_tokens, n_heads, d_k, d_v, n_accept,
                                               token_states, state,
                                               static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
