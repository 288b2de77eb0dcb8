/*
 * gdr_oracle.c -- plain fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only tests/, __graft_entry__.smoke() and the cpu_baseline
 * / reference legs of bench.py use it.  It shares no code, header or constant
 * with the CUDA library in gated_delta_rule_150_b200/.
 *
 * What it computes, token by token, for every sequence n and head h on its
 * own (no chunking, no blocking, no reordering):
 *
 *   S   <- S * Diag(a_t)                     a_t = exp(log_a_t), per key channel
 *   d   <- beta_t * (v_t - S k_t)            the delta rule reads the decayed state
 *   S   <- S + d k_t^T
 *   o_t <- S (scale * q_t)                   output read from the updated state
 *
 * which is S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
 *
 * Passages followed ("Modele hybrydowe: co Gated DeltaNet zastępuje w cache
 * KV", trefon.com):
 *   - section "Atencja liniowa: stan o stałym rozmiarze": the state is a
 *     d_v x d_k matrix per head and the output is o_t = S_t q_t, read after the
 *     update;
 *   - section "Reguła delta: zapisz poprawkę, nie sumę": the write is the
 *     error beta_t (v_t - S k_t) along k_t;
 *   - section "Gated DeltaNet: dodaj zanik": S_t = alpha_t S_{t-1}
 *     (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, i.e. the decay multiplies the
 *     old state before the delta read;
 *   - the per-key-channel decay of KDA ("kda-graft" page, section "Идея и
 *     архитектура": the mixer is Kimi Delta Attention / gated delta rule with an
 *     alpha gate per channel) replaces alpha_t by Diag(a_t) acting on the key
 *     columns; a scalar gate is the special case a_t = alpha_t * 1;
 *   - "kda-graft", section "Быстрый старт": the state is kept in fp32 on the
 *     GPU; here it is fp64.
 *   - section "Co stan rekurencyjny zmienia przy serwowaniu", point 1: a prefix
 *     can only be reused from a snapshot of the state taken at that position,
 *     so the state after every full snap_interval tokens of a sequence is
 *     copied out;
 *   - the same section, point 2: speculative decoding needs a real rollback,
 *     because the state has already absorbed the rejected draft tokens, so a
 *     draft of K tokens keeps the state after each of them and accepting n of
 *     them restores the state kept after token n.
 *
 * Layouts (row-major, token-major, sequences packed by cu_seqlens):
 *   q, k [T, H, dk]  v [T, H, dv]  beta [T, H]  log_a [T, H, dk] or [T, H]
 *   o [T, H, dv]  init_state / final_state [N, H, dv, dk]
 *   snapshots [sum_n floor(L_n / snap_interval), H, dv, dk], sequence-major.
 *
 * Draft decode: q, k [B, K, H, dk]  v [B, K, H, dv]  beta [B, K, H]
 *   log_a [B, K, H, dk] or [B, K, H]  o [B, K, H, dv]
 *   token_states [B, K, H, dv, dk]: the state after token t of sequence b.
 *
 * GDR_ORACLE_MUTANT (compile-time, default 0) plants one deliberate mistake;
 * it exists only so that the pin tests can show that each plausible mistake
 * is caught.  The default build has none.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef GDR_ORACLE_MUTANT
#define GDR_ORACLE_MUTANT 0
#endif

/* One token of the recurrence on one head's state S[dv][dk]. */
static void oracle_step(int dk, int dv, double* S, const double* q, const double* k,
                        const double* v, double beta, const double* a, double scale,
                        double* o, double* tmp)
{
    int j, c;
#if GDR_ORACLE_MUTANT == 2
    /* mutant: the delta read uses the state before the decay */
    for (j = 0; j < dv; ++j) {
        double p = 0.0;
        for (c = 0; c < dk; ++c) p += S[j * dk + c] * k[c];
        tmp[j] = beta * (v[j] - p);
    }
    for (j = 0; j < dv; ++j)
        for (c = 0; c < dk; ++c) S[j * dk + c] *= a[c];
    for (j = 0; j < dv; ++j)
        for (c = 0; c < dk; ++c) S[j * dk + c] += tmp[j] * k[c];
#else
    (void)tmp;
#if GDR_ORACLE_MUTANT != 7
    /* S <- S Diag(a): column c (key channel) is scaled by a_c */
    for (j = 0; j < dv; ++j)
        for (c = 0; c < dk; ++c)
#if GDR_ORACLE_MUTANT == 3
            S[j * dk + c] *= a[j % dk];          /* mutant: decay on the value rows */
#else
            S[j * dk + c] *= a[c];
#endif
#endif
#if GDR_ORACLE_MUTANT == 1
    /* mutant: output read from the state before the update */
    for (j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (c = 0; c < dk; ++c) acc += S[j * dk + c] * scale * q[c];
        o[j] = acc;
    }
#endif
    for (j = 0; j < dv; ++j) {
        double p = 0.0, d;
        for (c = 0; c < dk; ++c) p += S[j * dk + c] * k[c];
#if GDR_ORACLE_MUTANT == 4
        d = beta * (v[j] + p);                   /* mutant: sign of the erase term */
#elif GDR_ORACLE_MUTANT == 5
        d = (v[j] - p);                          /* mutant: write strength dropped */
#else
        d = beta * (v[j] - p);
#endif
        for (c = 0; c < dk; ++c) S[j * dk + c] += d * k[c];
    }
#if GDR_ORACLE_MUTANT == 7
    for (j = 0; j < dv; ++j)                     /* mutant: decay after the update */
        for (c = 0; c < dk; ++c) S[j * dk + c] *= a[c];
#endif
#endif
#if GDR_ORACLE_MUTANT != 1
    for (j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (c = 0; c < dk; ++c)
#if GDR_ORACLE_MUTANT == 6
            acc += S[j * dk + c] * scale * k[c]; /* mutant: reads with k instead of q */
#else
            acc += S[j * dk + c] * scale * q[c];
#endif
        o[j] = acc;
    }
#endif
}

/* Number of snapshot slots for the packed batch (one per full interval). */
int64_t gdr_oracle_snapshot_count(int n_seqs, const int32_t* cu, int snap_interval)
{
    int64_t total = 0;
    int n;
    if (snap_interval <= 0) return 0;
    for (n = 0; n < n_seqs; ++n) total += (int64_t)((cu[n + 1] - cu[n]) / snap_interval);
    return total;
}

/*
 * Prefill over a packed batch.  Returns 0 on success, -1 on bad arguments.
 * init_state may be NULL (zero state); snapshots may be NULL when
 * snap_interval == 0.
 */
int gdr_oracle_prefill(int n_seqs, int H, int dk, int dv, const int32_t* cu,
                       const double* q, const double* k, const double* v,
                       const double* beta, const double* log_a, int scalar_decay,
                       double scale, const double* init_state, double* o,
                       double* final_state, int snap_interval, double* snapshots)
{
    int64_t* snap_base;
    int n, pair;
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu) return -1;
    for (n = 0; n < n_seqs; ++n)
        if (cu[n + 1] < cu[n]) return -1;
    if (snap_interval > 0 && !snapshots) return -1;
    snap_base = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_seqs + 1));
    if (!snap_base) return -1;
    snap_base[0] = 0;
    for (n = 0; n < n_seqs; ++n)
        snap_base[n + 1] = snap_base[n] +
            (snap_interval > 0 ? (cu[n + 1] - cu[n]) / snap_interval : 0);

#pragma omp parallel for schedule(dynamic, 1)
    for (pair = 0; pair < n_seqs * H; ++pair) {
        int sn = pair / H, h = pair % H;
        size_t sz = (size_t)dv * (size_t)dk;
        double* S = (double*)malloc(sizeof(double) * sz);
        double* a = (double*)malloc(sizeof(double) * (size_t)dk);
        double* tmp = (double*)malloc(sizeof(double) * (size_t)dv);
        int64_t t, slot = snap_base[sn];
        int c;
        if (init_state)
            memcpy(S, init_state + ((size_t)sn * H + h) * sz, sizeof(double) * sz);
        else
            memset(S, 0, sizeof(double) * sz);
        for (t = cu[sn]; t < cu[sn + 1]; ++t) {
            size_t th = (size_t)t * H + h;
#if GDR_ORACLE_MUTANT == 9
            size_t th_gate = (size_t)t * H + (h + 1) % H;   /* mutant: gate of the next head */
#else
            size_t th_gate = th;
#endif
            for (c = 0; c < dk; ++c)
                a[c] = exp(scalar_decay ? log_a[th_gate] : log_a[th_gate * dk + c]);
            oracle_step(dk, dv, S, q + th * dk, k + th * dk, v + th * dv, beta[th], a,
                        scale, o + th * dv, tmp);
#if GDR_ORACLE_MUTANT == 8
            if (snap_interval > 0 && (t - cu[sn]) % snap_interval == 0 && t > cu[sn] &&
                slot < snap_base[sn + 1]) {            /* mutant: snapshot one token late */
#else
            if (snap_interval > 0 && (t + 1 - cu[sn]) % snap_interval == 0) {
#endif
                memcpy(snapshots + ((size_t)slot * H + h) * sz, S, sizeof(double) * sz);
                ++slot;
            }
        }
#if GDR_ORACLE_MUTANT == 10
        {   /* mutant: final state written transposed (square heads only) */
            int j;
            for (j = 0; j < dv; ++j)
                for (c = 0; c < dk; ++c)
                    final_state[((size_t)sn * H + h) * sz + (size_t)c * dv + j] = S[(size_t)j * dk + c];
        }
#else
        memcpy(final_state + ((size_t)sn * H + h) * sz, S, sizeof(double) * sz);
#endif
        free(S);
        free(a);
        free(tmp);
    }
    free(snap_base);
    return 0;
}

/*
 * One decode step for a batch of independent sequences: the same token update
 * as above with T = 1, state updated in place.  state [B, H, dv, dk],
 * q, k [B, H, dk], v [B, H, dv], beta [B, H], log_a [B, H, dk] or [B, H],
 * o [B, H, dv].
 */
int gdr_oracle_decode_step(int B, int H, int dk, int dv, const double* q, const double* k,
                           const double* v, const double* beta, const double* log_a,
                           int scalar_decay, double scale, double* state, double* o)
{
    int pair;
    if (B < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (pair = 0; pair < B * H; ++pair) {
        size_t sz = (size_t)dv * (size_t)dk;
        double* a = (double*)malloc(sizeof(double) * (size_t)dk);
        double* tmp = (double*)malloc(sizeof(double) * (size_t)dv);
        int c;
        for (c = 0; c < dk; ++c)
            a[c] = exp(scalar_decay ? log_a[pair] : log_a[(size_t)pair * dk + c]);
        oracle_step(dk, dv, state + (size_t)pair * sz, q + (size_t)pair * dk,
                    k + (size_t)pair * dk, v + (size_t)pair * dv, beta[pair], a, scale,
                    o + (size_t)pair * dv, tmp);
        free(a);
        free(tmp);
    }
    return 0;
}

/*
 * Draft decode for speculative decoding: K tokens per sequence from `state`
 * (not modified), keeping the state after every token in token_states.
 * Each token is the same update as above.
 */
int gdr_oracle_decode_draft(int B, int K, int H, int dk, int dv, const double* q,
                            const double* k, const double* v, const double* beta,
                            const double* log_a, int scalar_decay, double scale,
                            const double* state, double* o, double* token_states)
{
    int pair;
    if (B < 0 || K < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (pair = 0; pair < B * H; ++pair) {
        int b = pair / H, h = pair % H, t, c;
        size_t sz = (size_t)dv * (size_t)dk;
        double* S = (double*)malloc(sizeof(double) * sz);
        double* a = (double*)malloc(sizeof(double) * (size_t)dk);
        double* tmp = (double*)malloc(sizeof(double) * (size_t)dv);
        memcpy(S, state + (size_t)pair * sz, sizeof(double) * sz);
        for (t = 0; t < K; ++t) {
            size_t th = ((size_t)b * K + t) * H + h;     /* token t of sequence b, head h */
            for (c = 0; c < dk; ++c)
                a[c] = exp(scalar_decay ? log_a[th] : log_a[th * dk + c]);
#if GDR_ORACLE_MUTANT == 11
            /* mutant: keeps the state from before the token */
            memcpy(token_states + th * sz, S, sizeof(double) * sz);
#endif
            oracle_step(dk, dv, S, q + th * dk, k + th * dk, v + th * dv, beta[th], a, scale,
                        o + th * dv, tmp);
#if GDR_ORACLE_MUTANT != 11
            memcpy(token_states + th * sz, S, sizeof(double) * sz);
#endif
        }
        free(S);
        free(a);
        free(tmp);
    }
    return 0;
}

/*
 * Accept n_accept[b] of the K draft tokens of sequence b: its state becomes
 * the state kept after token n (n = 1 .. K) and stays as it is for n = 0.
 * n_accept is clamped to [0, K].
 */
int gdr_oracle_decode_accept(int B, int K, int H, int dk, int dv, const int32_t* n_accept,
                             const double* token_states, double* state)
{
    int b, h;
    size_t sz = (size_t)dv * (size_t)dk;
    if (B < 0 || K < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    for (b = 0; b < B; ++b) {
        int n = n_accept[b] < 0 ? 0 : (n_accept[b] > K ? K : n_accept[b]);
#if GDR_ORACLE_MUTANT == 12
        int pick = n < K ? n : K - 1;                /* mutant: one token too far */
#else
        int pick = n - 1;
#endif
        if (n == 0) continue;
        for (h = 0; h < H; ++h)
            memcpy(state + ((size_t)b * H + h) * sz,
                   token_states + (((size_t)b * K + pick) * H + h) * sz, sizeof(double) * sz);
    }
    return 0;
}
