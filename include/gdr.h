/*
 * gdr.h -- C ABI of the gated delta-rule library (B200, sm_100a).
 *
 * The operation.  For every sequence and head, with a state S of d_v x d_k
 * values (row = value channel, column = key channel):
 *
 *     S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t (scale * q_t)
 *
 * Sources (the pages this library implements):
 *   - "Modele hybrydowe: co Gated DeltaNet zastępuje w cache KV" (trefon.com):
 *       section "Atencja liniowa: stan o stałym rozmiarze" -- a fixed
 *       d_v x d_k state per head and o_t = S_t q_t;
 *       section "Reguła delta: zapisz poprawkę, nie sumę" -- the delta write;
 *       section "Gated DeltaNet: dodaj zanik" -- the decay alpha_t applied to
 *       the old state before the delta read;
 *       section "Co stan rekurencyjny zmienia przy serwowaniu" -- point 1
 *       (prefix snapshots), and the closing paragraph: chunked prefill, dense
 *       products inside a chunk, sequential only from chunk to chunk.
 *   - "kda-graft: Qwen2.5-0.5B с трансплантированным KDA" (ailist.pro):
 *       section "Идея и архитектура" -- KDA (Kimi Delta Attention / gated
 *       delta rule), whose decay is one gate per key channel, a_t in (0,1]^d_k;
 *       section "Быстрый старт" -- the state is kept in fp32;
 *       section "2. Decode: O(1) против O(L)" -- the decode step reads and
 *       writes a state whose size does not depend on the context length.
 *
 * Conventions for every call below.
 *   - Pointers marked "device" are CUDA device pointers (cudaMalloc'd or from
 *     any allocator of the same context); "host" pointers are ordinary memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued on it; nothing synchronises the host.
 *   - The library never allocates, frees or synchronises.  The caller owns
 *     every buffer, including the prefill workspace.
 *   - Tensors are dense, row-major, in the layouts stated per argument.
 *     q, k, v (prefill), per-channel log_a, states, snapshots and the
 *     workspace pointers must be 16-byte aligned (the workspace 256-byte);
 *     beta, scalar log_a, o and the decode v need only their element
 *     alignment.
 *   - Arguments are checked on the host before anything is launched; a failed
 *     check returns an error status and enqueues nothing.  A launch failure
 *     returns GDR_ERR_CUDA.
 *   - Stream order holds as for ordinary launches.  Some prefill kernels are
 *     launched with programmatic stream serialization, so their CTAs may be
 *     scheduled while the previous kernel on the stream finishes; they touch
 *     no global memory before that kernel has completed.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, bad cu_seqlens */
    GDR_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement */
    GDR_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
    GDR_ERR_CUDA = 4,          /* a CUDA launch or device query failed */
    GDR_ERR_TIMEOUT = 5        /* a kernel gave up a bounded wait (see gdr_prefill_status) */
} gdr_status;

typedef enum {
    GDR_BF16 = 0,              /* bfloat16 q, k, v (and o for prefill) */
    GDR_F32 = 1                /* float32 q, k, v (and o for prefill) */
} gdr_dtype;

/* Human-readable name of a status; never NULL. */
const char* gdr_status_string(gdr_status s);

/* Library version: major * 10000 + minor * 100 + patch. */
int gdr_version(void);

/* ------------------------------------------------------------------------
 * Prefill: chunked-parallel evaluation of the recurrence over a packed batch
 * of sequences ("Modele hybrydowe", closing paragraph of "Co stan rekurencyjny
 * zmienia przy serwowaniu": chunks of C = 64 tokens, dense products inside a
 * chunk, a sequential pass from chunk to chunk).  Chunks restart at every
 * sequence start; the last chunk of a sequence may be partial.
 * ---------------------------------------------------------------------- */
typedef struct {
    int n_seqs;                 /* N >= 0 sequences packed by cu_seqlens */
    int n_heads;                /* H >= 1 */
    int d_k;                    /* key/query width: 64 or 128 */
    int d_v;                    /* value width: 64 or 128, any pairing with d_k.  With
                                   d_k != d_v the kernels run at D = max(d_k, d_v) on
                                   inputs whose narrower side is copied, widened with
                                   zero channels, into the workspace (exact: zero key
                                   channels leave the other columns of S untouched and
                                   stay zero; rows of S evolve independently, and a
                                   zero value row stays zero); states and o keep the
                                   caller's d_v x d_k and d_v layouts. */
    int64_t total_tokens;       /* T_tot = cu_seqlens[N]; host copy of the device value */
    const int32_t* cu_seqlens;  /* device [N+1]: 0 = cu[0] <= cu[1] <= ... <= cu[N] = T_tot */
    gdr_dtype qkv_dtype;        /* dtype of q, k, v and o */
    const void* q;              /* device [T_tot, H, d_k] */
    const void* k;              /* device [T_tot, H, d_k] */
    const void* v;              /* device [T_tot, H, d_v] */
    const float* beta;          /* device [T_tot, H], write strength in (0, 1) */
    const float* log_a;         /* device [T_tot, H, d_k] (KDA), or [T_tot, H] when
                                   scalar_decay != 0 (Gated DeltaNet); log a_t <= 0 */
    int scalar_decay;           /* 0: per-key-channel decay, 1: one decay per head-token */
    float scale;                /* multiplies q; the pages use none: pass 1.0f */
    const float* init_state;    /* device [N, H, d_v, d_k] or NULL for zero states.
                                   May alias final_state. */
    void* o;                    /* device [T_tot, H, d_v], dtype qkv_dtype (output) */
    float* final_state;         /* device [N, H, d_v, d_k] (output) */
    int snap_interval;          /* 0: no snapshots; else a multiple of 64 */
    float* snapshots;           /* device [gdr_snapshot_count(...), H, d_v, d_k] (output):
                                   the state after tokens [0, m*snap_interval) of each
                                   sequence, m = 1 .. floor(L_n / snap_interval),
                                   sequences in order ("Co stan rekurencyjny zmienia przy
                                   serwowaniu", point 1: a prefix is reused from the
                                   snapshot taken at its end).  May be pinned host
                                   memory (see "Snapshot offload" below). */
    const int64_t* snap_offsets;/* device [N+1] or NULL: first snapshot slot of each
                                   sequence, as gdr_snapshot_offsets returns it
                                   (NULL: the kernels sum the sequence lengths) */
    const void* gate_raw;       /* device [T_tot, H, d_v], dtype qkv_dtype, or NULL.  When
                                   given, o receives the mixer's output after its RMSNorm
                                   and output gate ("kda-graft", section "Идея и
                                   архитектура": each KDA layer ends in both), per token
                                   and head over the d_v channels:
                                     o = x / sqrt(mean_c x_c^2 + norm_eps) * norm_weight
                                           * sigmoid(gate_raw),   x = S_t (scale q_t) */
    const float* norm_weight;   /* device [d_v] fp32, shared by the heads (with gate_raw) */
    float norm_eps;             /* RMSNorm epsilon >= 0 (with gate_raw), e.g. 1e-6f */
    void* workspace;            /* device scratch, >= gdr_prefill_workspace_size(...) bytes,
                                   256-byte aligned; contents on entry do not matter */
    size_t workspace_bytes;
} gdr_prefill_args;

/* Bytes of device workspace gdr_prefill needs for these sizes (0 on bad sizes). */
size_t gdr_prefill_workspace_size(int n_seqs, int n_heads, int d_k, int d_v,
                                  int64_t total_tokens, int scalar_decay);

/*
 * Number of kernel launches gdr_prefill enqueues for these sizes (0 on bad
 * sizes): the intra-chunk kernel plus one state pass, or three (zero-state
 * pass, chaining of segment maps, replay) when long sequences with few
 * (sequence, head) pairs are cut into segments; with d_k != d_v, plus one
 * widening copy per widened input (q, k and a per-channel log_a, or v).
 */
int gdr_prefill_kernel_count(int n_seqs, int n_heads, int d_k, int d_v, int64_t total_tokens,
                             int scalar_decay);

/* Number of snapshot slots for host-side cu_seqlens [N+1] (-1 on bad input). */
int64_t gdr_snapshot_count(const int32_t* host_cu_seqlens, int n_seqs, int snap_interval);

/*
 * Where each sequence's snapshots start ("Co stan rekurencyjny zmienia przy
 * serwowaniu", point 1: a request whose prompt extends a stored prefix resumes
 * from the snapshot at the prefix's end, so a caller must find sequence n's
 * m-th snapshot).  host_cu_seqlens [N+1] and host_offsets_out [N+1] are host
 * memory.  On return host_offsets_out[n] = sum over sequences m < n of
 * floor(L_m / snap_interval); sequence n's m-th snapshot (m = 1 .. floor(L_n /
 * snap_interval), the state after its first m * snap_interval tokens) is slot
 * host_offsets_out[n] + m - 1 of gdr_prefill_args.snapshots, and
 * host_offsets_out[N] is the slot count.  A copy of the array on the device
 * may be passed as gdr_prefill_args.snap_offsets.  Errors: GDR_ERR_INVALID_ARG
 * for a null pointer, n_seqs < 0, snap_interval <= 0 or a decreasing
 * cu_seqlens (host_offsets_out is then left unspecified).
 */
gdr_status gdr_snapshot_offsets(const int32_t* host_cu_seqlens, int n_seqs, int snap_interval,
                                int64_t* host_offsets_out);

/*
 * Snapshot offload.  A serving engine keeps prefix snapshots in host memory
 * ("Co stan rekurencyjny zmienia przy serwowaniu", point 1: dozens of
 * checkpoints of ~149 MiB each; saving them was made asynchronous so that it
 * stops stalling prefill).  Two ways:
 *   - gdr_snapshot_offload (below): the prefill writes its snapshots to
 *     device memory and a copy engine moves them to page-locked host memory
 *     on a second stream while the next prefill computes -- the prefill runs
 *     at full speed;
 *   - gdr_prefill_args.snapshots may point to page-locked host memory
 *     (cudaHostAlloc / cudaMallocHost, or cudaHostRegister with
 *     cudaHostRegisterMapped): the state-pass kernel then writes each
 *     snapshot straight over the host link as soon as it is known, with no
 *     device buffer, but those stores go at the link's pace and hold up the
 *     state pass (measured: +51 % on a 65 536-token, 16-head, d 128 prefill
 *     writing 16 MiB of snapshots).
 * Pageable host memory is rejected with GDR_ERR_INVALID_ARG.
 */

/*
 * Snapshot offload on a copy stream: copy `bytes` of snapshots from device
 * memory to page-locked host memory on `copy_stream`, ordered after
 * everything enqueued so far on `compute_stream` (the prefill that wrote
 * them) by `event`, which this call records on compute_stream.  Prefills
 * enqueued later on compute_stream do not wait for the copy; the caller must
 * not let a later prefill overwrite dev_snapshots before the copy has read
 * them (use separate snapshot buffers, or make compute_stream wait for
 * copy_stream).  `event` is created by the caller (cudaEventCreateWithFlags;
 * timing may be disabled) and passed as void*.  Nothing is allocated.
 * Errors: GDR_ERR_INVALID_ARG (null pointer, compute_stream == copy_stream,
 * buffers not 16-byte aligned), GDR_ERR_CUDA if a runtime call fails.
 * bytes == 0 only records the event.
 */
gdr_status gdr_snapshot_offload(const float* dev_snapshots, float* host_snapshots, size_t bytes,
                                void* compute_stream, void* copy_stream, void* event);

/*
 * Enqueue a prefill.  Outputs: o, final_state and (if snap_interval > 0)
 * snapshots.  Zero-length sequences are legal: their final state is their
 * initial state.  Errors: GDR_ERR_INVALID_ARG / GDR_ERR_UNSUPPORTED /
 * GDR_ERR_WORKSPACE before launch, GDR_ERR_CUDA on a failed launch.
 */
gdr_status gdr_prefill(const gdr_prefill_args* args, void* stream);

/*
 * Enqueue only stages first..last (inclusive) of a prefill: 0 = intra-chunk
 * factors (the chunk-local cumulative decay of gdr_cumdecay is computed inside
 * this stage, so g never goes through memory), 1 = sequential inter-chunk
 * pass.  gdr_prefill(a) is gdr_prefill_stages(a, 0, 1).  A later stage reads what the
 * earlier stages left in the workspace, so a range starting after 0 must
 * follow a call that ran the stages before it with the same arguments.  Used
 * to time the kernels one by one.  Errors as for gdr_prefill, plus
 * GDR_ERR_INVALID_ARG for a bad stage range.
 */
gdr_status gdr_prefill_stages(const gdr_prefill_args* args, int first, int last, void* stream);

/*
 * gdr_prefill without a caller-provided workspace, for callers that cannot
 * allocate device memory: code running under CUDA graph capture (cudaMalloc
 * cannot be captured), plugins whose host framework owns all allocation, and
 * serving paths where allocating is not allowed.  The pages have no
 * counterpart; this is a property of the library, not of the method.
 *
 * The workspace is a fixed GDR_STATIC_WORKSPACE_BYTES array in the library's
 * own device memory (held by every GPU that loads the library until the
 * process exits).  args->workspace and args->workspace_bytes are ignored; every
 * other field means what it means for gdr_prefill, and the results are the
 * same.  A request whose workspace (gdr_prefill_workspace_size) exceeds
 * GDR_STATIC_WORKSPACE_BYTES returns GDR_ERR_WORKSPACE and enqueues nothing.
 * Nothing is allocated or freed.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture.  All calls share the one
 * array: calls that may overlap on the GPU (other streams, other host threads)
 * race and must be serialised by the caller.  Use gdr_prefill_static_status
 * (not gdr_prefill_status) to learn whether the call's kernels completed.
 *
 * Size limit: gdr_prefill_workspace_size(...) <= GDR_STATIC_WORKSPACE_BYTES,
 * where the workspace is 1 KiB + (floor(T/64) + N) * H * R(d) bytes of chunk
 * records, R(64) = 33 792 and R(128) = 99 328, plus, when long sequences with
 * few (sequence, head) pairs are cut into segments, 12 d^2 bytes per segment
 * slot and head.  For one sequence that is up to 7 424 tokens at 14 heads and
 * d 64 (the 8 192-token Qwen2.5-0.5B graft layer does not fit), 60 480 tokens
 * at 2 heads and d 64, and 1 984 tokens at 16 heads and d 128.
 *
 * The device address of the array is looked up again (cudaGetSymbolAddress)
 * on every call made while `stream` is not capturing, so a context re-created
 * after cudaDeviceReset is handled; while capturing, the address from the last
 * call on that device outside capture is used.
 */
#define GDR_STATIC_WORKSPACE_BYTES (64u << 20)
gdr_status gdr_prefill_static_workspace(const gdr_prefill_args* args, void* stream);

/*
 * Status the device side of the most recent gdr_prefill_static_workspace call
 * on the current device recorded: GDR_OK, or GDR_ERR_TIMEOUT if one of its
 * kernels abandoned a bounded wait (the outputs of that call are then
 * undefined).  Reads one word of the library's array (no allocation) and
 * synchronises `stream`, so it cannot be called while `stream` is capturing;
 * GDR_ERR_CUDA if the read fails.
 */
gdr_status gdr_prefill_static_status(void* stream);

/*
 * Status the device side of the most recent gdr_prefill on this workspace
 * recorded: GDR_OK, or GDR_ERR_TIMEOUT if a kernel abandoned a bounded wait
 * (its outputs are then undefined).  Synchronises `stream`.
 */
gdr_status gdr_prefill_status(const void* workspace, void* stream);

/*
 * The chunk-local cumulative log decay on its own: g[t] = sum of log_a over
 * the tokens of t's chunk up to and including t, chunks as in gdr_prefill.
 * (gdr_prefill computes the same sums inside its intra-chunk stage.)  log_a and g share the layout
 * [T_tot, H, d_k] (or [T_tot, H] when scalar_decay != 0), fp32, device.
 */
gdr_status gdr_cumdecay(int n_seqs, int n_heads, int d_k, int64_t total_tokens,
                        const int32_t* cu_seqlens, const float* log_a, int scalar_decay,
                        float* g, void* stream);

/*
 * The intra-chunk factors on their own (the prefill's first stage), unpacked
 * to plain fp32 arrays for inspection.  With
 * n_slots = floor(T_tot / 64) + N chunk slots, chunk j of sequence n lives in
 * slot floor(cu[n] / 64) + j + n; unused slots are left untouched.  For a
 * chunk with start state S0, its effect on the state and outputs is
 *     S_next = S0 Diag(gamma) + S0 BS^T + NC        O = Qt S0^T + PU
 * where, with g the chunk-local cumulative log decay, Gamma = exp(g),
 * A[r,i] = beta_r sum_c k[r,c] k[i,c] exp(g[r,c] - g[i,c]) (i < r),
 * P[r,i] = scale sum_c q[r,c] k[i,c] exp(g[r,c] - g[i,c]) (i <= r),
 * T = (I + A)^-1, W = T diag(beta)(K * Gamma), U = T diag(beta) V,
 * Qg = scale Q * Gamma and Kd = K * exp(g_last - g):
 *   Qt    [n_slots, H, 64, d_k]  = Qg - P W
 *   PU    [n_slots, H, 64, d_v]  = P U
 *   BS    [n_slots, H, d_k, d_k] = -Kd^T W
 *   NC    [n_slots, H, d_v, d_k] = U^T Kd
 *   gamma [n_slots, H, d_k]      = exp(g_last)
 * Rows past the end of a partial chunk are zero.  `workspace` as for
 * gdr_prefill with the same arguments; q, k, v, beta, log_a, cu_seqlens,
 * scalar_decay and scale are read from `args`, its outputs are ignored.
 * d_k must equal d_v here (GDR_ERR_UNSUPPORTED otherwise).
 */
gdr_status gdr_chunk_factors(const gdr_prefill_args* args, float* Qt, float* PU, float* BS,
                             float* NC, float* gamma, void* stream);

/* ------------------------------------------------------------------------
 * Decode: one token per sequence, state updated in place ("kda-graft",
 * section "2. Decode: O(1) против O(L)": the step streams a fixed-size fp32
 * state, independent of the context length).
 *   q, k   device [B, H, d_k], dtype qkv_dtype
 *   v      device [B, H, d_v], dtype qkv_dtype
 *   beta   device [B, H] fp32
 *   log_a  device [B, H, d_k] fp32, or [B, H] when scalar_decay != 0
 *   state  device [B, H, d_v, d_k] fp32, read and overwritten
 *   o      device [B, H, d_v] fp32 (output), o = S_new (scale * q)
 * d_k in {64, 128}; d_v in {64, 128}.  B == 0 is a no-op.
 * ---------------------------------------------------------------------- */
gdr_status gdr_decode_step(int batch, int n_heads, int d_k, int d_v, gdr_dtype qkv_dtype,
                           const void* q, const void* k, const void* v, const float* beta,
                           const float* log_a, int scalar_decay, float scale, float* state,
                           float* o, void* stream);

/*
 * gdr_decode_step followed by the output epilogue of gdr_prefill_args.gate_raw
 * (RMSNorm over the d_v channels of each (sequence, head), weight shared by
 * the heads, then the sigmoid output gate):
 *   gate_raw     device [B, H, d_v], dtype qkv_dtype
 *   norm_weight  device [d_v] fp32
 *   norm_eps     >= 0
 *   o            device [B, H, d_v] fp32 (output): the gated, normalised output
 * Other arguments, results and errors as for gdr_decode_step.
 */
gdr_status gdr_decode_step_gated(int batch, int n_heads, int d_k, int d_v, gdr_dtype qkv_dtype,
                                 const void* q, const void* k, const void* v, const float* beta,
                                 const float* log_a, int scalar_decay, float scale, float* state,
                                 const void* gate_raw, const float* norm_weight, float norm_eps,
                                 float* o, void* stream);

/* ------------------------------------------------------------------------
 * Input activations: the recurrence's q, k, v, beta and log a from raw
 * per-head projections in one pass ("kda-graft", section "Идея и
 * архитектура": the graft adds a width-4 convolution initialised as an
 * identity tap, the alpha gate with bias +5 and the write strength beta).
 * For token t of a sequence starting at s, head h, channel c:
 *     conv(x)[t] = sum_{j=0..3, t-3+j >= s} w[h d + c][j] x[t-3+j]
 *     q = conv(x_q) / max(||conv(x_q)||, 1e-12)   (norm over the head's d channels)
 *     k = conv(x_k) / max(||conv(x_k)||, 1e-12)
 *     v = conv(x_v)
 *     beta = sigmoid(beta_raw),  log_a = log_sigmoid(a_raw + a_bias)
 * The conv restarts from zero history at every sequence start; tap 3 is the
 * current token.  The outputs are gdr_prefill's inputs, in its layouts.
 * ---------------------------------------------------------------------- */
typedef struct {
    int n_seqs;                 /* N >= 0 sequences packed by cu_seqlens */
    int n_heads;                /* H >= 1 */
    int d;                      /* d_k = d_v: 64 or 128 */
    int64_t total_tokens;       /* T_tot = cu_seqlens[N] (host copy) */
    const int32_t* cu_seqlens;  /* device [N+1], as for gdr_prefill */
    gdr_dtype io_dtype;         /* dtype of x_q, x_k, x_v and of q, k, v */
    const void* xq;             /* device [T_tot, H, d] raw projections */
    const void* xk;             /* device [T_tot, H, d] */
    const void* xv;             /* device [T_tot, H, d] */
    const float* conv_q;        /* device [H d, 4] fp32 taps per channel (row h d + c) */
    const float* conv_k;        /* device [H d, 4] */
    const float* conv_v;        /* device [H d, 4] */
    const float* beta_raw;      /* device [T_tot, H] */
    const float* a_raw;         /* device [T_tot, H, d], or [T_tot, H] if scalar_decay */
    const float* a_bias;        /* device [H, d], or [H] if scalar_decay */
    int scalar_decay;           /* 0: per-key-channel gate, 1: one gate per head-token */
    void* q;                    /* device [T_tot, H, d], io_dtype (output) */
    void* k;                    /* device [T_tot, H, d], io_dtype (output) */
    void* v;                    /* device [T_tot, H, d], io_dtype (output) */
    float* beta;                /* device [T_tot, H] (output) */
    float* log_a;               /* device [T_tot, H, d] or [T_tot, H] (output) */
} gdr_preprocess_args;

/*
 * Enqueue the input activations.  Outputs must not overlap the inputs.
 * Errors: GDR_ERR_INVALID_ARG (null or misaligned pointer -- xq, xk, xv, the
 * conv taps, q, k, v and, with a per-channel gate, a_raw, a_bias and log_a
 * need 16-byte alignment -- or bad sizes, including ceil(T_tot / 32) * H
 * above 2^31 - 1), GDR_ERR_UNSUPPORTED (d not 64 or 128), GDR_ERR_CUDA on a
 * failed launch.  T_tot == 0 is a no-op.
 */
gdr_status gdr_preprocess(const gdr_preprocess_args* args, void* stream);

/* ------------------------------------------------------------------------
 * Prefill from raw projections: gdr_preprocess's input activations (width-4
 * conv, L2 norm of q and k, beta = sigmoid(beta_raw), log a =
 * log_sigmoid(a_raw + a_bias)) applied inside the prefill's first stage, so
 * that q, k, v, beta and log a are never written to memory ("kda-graft",
 * section "Идея и архитектура": the activations sit right before the
 * recurrence).  The results equal gdr_preprocess followed by gdr_prefill up
 * to the summation order of the L2 norms.
 * ---------------------------------------------------------------------- */
typedef struct {
    const void* xq;             /* device [T_tot, H, d] raw projections, bf16 */
    const void* xk;             /* device [T_tot, H, d] */
    const void* xv;             /* device [T_tot, H, d] */
    const float* conv_q;        /* device [H d, 4] fp32 taps (row h d + c; tap 3 = current token) */
    const float* conv_k;        /* device [H d, 4] */
    const float* conv_v;        /* device [H d, 4] */
    const float* beta_raw;      /* device [T_tot, H] */
    const float* a_raw;         /* device [T_tot, H, d], or [T_tot, H] if args->scalar_decay */
    const float* a_bias;        /* device [H, d], or [H] if args->scalar_decay */
} gdr_projections;

/*
 * Enqueue a prefill whose inputs are raw projections.  `args` as for
 * gdr_prefill, with its q, k, v, beta and log_a ignored (may be NULL);
 * qkv_dtype must be GDR_BF16 and d_k == d_v (64 or 128), else
 * GDR_ERR_UNSUPPORTED.  xq, xk, xv, the conv taps and (per-channel gate)
 * a_raw and a_bias must be 16-byte aligned.  Outputs and errors as for
 * gdr_prefill.  Workspace: at least gdr_prefill_workspace_size(...) bytes,
 * with which the activations are applied inside the prefill's first kernel.
 * At d 128 with a per-channel gate that first stage is bound by its
 * per-chunk latency and the activations lengthen it more than an HBM round
 * trip of them costs: given gdr_prefill_from_projections_workspace_size(...)
 * bytes, the call runs gdr_preprocess into the workspace's tail and then
 * gdr_prefill (about 12 % faster on a B200; 1284 more bytes of workspace
 * per token and head).  At d 64, or with a scalar gate, both sizes are the
 * same and the fused first stage runs (about 8 % faster than the two calls
 * at d 64).
 */
gdr_status gdr_prefill_from_projections(const gdr_prefill_args* args, const gdr_projections* proj,
                                        void* stream);

/*
 * Workspace bytes with which gdr_prefill_from_projections stages the
 * activations (see above): gdr_prefill_workspace_size(n_seqs, n_heads, d, d,
 * total_tokens, scalar_decay), plus, at d == 128 with scalar_decay == 0,
 * room for q, k, v (bf16), beta and log a (fp32) of every token and head.
 * 0 for invalid sizes, as gdr_prefill_workspace_size.
 */
size_t gdr_prefill_from_projections_workspace_size(int n_seqs, int n_heads, int d,
                                                   int64_t total_tokens, int scalar_decay);

/* ------------------------------------------------------------------------
 * Speculative decoding with rollback ("Modele hybrydowe", section "Co stan
 * rekurencyjny zmienia przy serwowaniu", point 2: a KV cache drops rejected
 * draft tokens, but the recurrent state has already absorbed them, so the
 * engine needs the state from before them back).  A draft runs K tokens per
 * sequence from a state it does not modify and keeps the state after every
 * token; after verification, gdr_decode_accept makes each sequence's state
 * the one kept after its last accepted token.  Each token is the decode step
 * above.
 * ---------------------------------------------------------------------- */

/*
 * Draft: n_tokens = K >= 0 tokens per sequence.  Token t of sequence b is
 * row (b K + t) of the [B K, ...] arrays below (sequence-major, then token):
 *   q, k          device [B, K, H, d_k], dtype qkv_dtype
 *   v             device [B, K, H, d_v], dtype qkv_dtype
 *   beta          device [B, K, H] fp32
 *   log_a         device [B, K, H, d_k] fp32, or [B, K, H] when scalar_decay != 0
 *   state         device [B, H, d_v, d_k] fp32, read only
 *   o             device [B, K, H, d_v] fp32 (output): o of token t, read from
 *                 the state after token t
 *   token_states  device [B, K, H, d_v, d_k] fp32 (output): the state after
 *                 token t of sequence b; must not overlap `state`
 * d_k, d_v in {64, 128}.  B == 0 or K == 0 is a no-op.  Errors as for
 * gdr_decode_step.
 */
gdr_status gdr_decode_draft(int batch, int n_tokens, int n_heads, int d_k, int d_v,
                            gdr_dtype qkv_dtype, const void* q, const void* k, const void* v,
                            const float* beta, const float* log_a, int scalar_decay, float scale,
                            const float* state, float* o, float* token_states, void* stream);

/*
 * Accept (rollback): for every sequence b, with n = n_accept[b] clamped to
 * [0, K], state[b] = token_states[b, n - 1] if n >= 1; for n == 0 state[b] is
 * left as it was (every draft token rejected).
 *   n_accept      device [B] int32 (read on the device, so it may be written
 *                 by an earlier kernel on the stream)
 *   token_states  device [B, K, H, d_v, d_k] fp32, from gdr_decode_draft
 *   state         device [B, H, d_v, d_k] fp32, overwritten where n >= 1;
 *                 must not overlap token_states
 * B == 0 or K == 0 is a no-op.
 */
gdr_status gdr_decode_accept(int batch, int n_tokens, int n_heads, int d_k, int d_v,
                             const int32_t* n_accept, const float* token_states, float* state,
                             void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
