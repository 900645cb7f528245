/*
 * DeltaNet forward oracle: the token recurrence in float64, on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library.  It shares no
 * code, header or table with the CUDA path.
 *
 * What it computes ("Linear Attention, Visualized", section "DeltaNet:
 * correcting memory collisions", subsection "Recurrent form"), in the row-vector
 * convention of that page, with S a d_k x d_v matrix per (sequence, head):
 *
 *     vhat_t = k_t S_{t-1}              prediction read at the current key
 *     u_t    = beta_t (v_t - vhat_t)    scaled correction
 *     S_t    = S_{t-1} + k_t^T u_t      rank-one write
 *     o_t    = q_t S_t                  readout after the write
 *
 * This is the column-convention recurrence S_t = S_{t-1}(I - b k k^T) + b v k^T,
 * o_t = S_t q_t of "Context Parallelism for DeltaNet" (section 2) transposed.
 * Gated DeltaNet (same page, section "Gated DeltaNet (GDN)") multiplies the
 * whole transition by a per-token scalar decay a_t,
 *     S_t = a_t (I - beta_t k_t^T k_t) S_{t-1} + beta_t k_t^T v_t,
 * so with a gate the loop first decays the state, S <- a_t S_{t-1}, and then
 * makes the same prediction, correction and write from the decayed state.
 * The gate arrives as g_t = ln a_t (fp32 [B, T, H]); a_t = exp(g_t) in float64.
 *
 * Gated Delta Product (same page, section "Gated Delta Product (GDP)") makes
 * n_sub delta-rule writes per token, each with its own key, value and beta,
 * after one decay of the state and before the token's readout:
 *     S_{t,0} = a_t S_{t-1};  S_{t,j} = (I - b_{t,j} k_{t,j}^T k_{t,j}) S_{t,j-1}
 *     + b_{t,j} k_{t,j}^T v_{t,j} for j = 1..n_sub;  S_t = S_{t,n_sub};  o_t = q_t S_t.
 * k, v and beta then hold n_sub rows per token, substep-major within the token
 * (row t * n_sub + j - 1, i.e. [B, T * n_sub, H, .]); q, gate and out keep one
 * row per token.  n_sub = 1 is (Gated) DeltaNet.
 *
 * Kimi Delta Attention (same page, section "Kimi Delta Attention (KDA)") decays
 * every key channel of the state at its own rate before the delta correction:
 *     S_t = Diag(a_t) S_{t-1} + beta_t k_t^T (v_t - k_t Diag(a_t) S_{t-1}),
 * with a_t in (0, 1]^{d_k} scaling row c of S by a_{t,c}.  Its gate arrives as
 * g [B, T, H, dk] (gate_per_key = 1); the loop scales row c by exp(g_{t,c})
 * and then runs the same prediction, correction and write.
 * S starts from the caller's initial state (or zero) at the first token of each
 * sequence.  No query scaling is applied.  Inputs stored as bf16 are widened
 * exactly to float64; every sum is accumulated in float64.
 *
 * Layouts (contiguous, row-major):
 *   q [B, T, H, dk]  out [B, T, H, dv]  gate [B, T, H] or [B, T, H, dk] (fp32)
 *   k [B, T n_sub, H, dk]  v [B, T n_sub, H, dv]  beta [B, T n_sub, H] (fp32)
 *   init_state, final_state [N, H, dk, dv]
 * With cu_seqlens (host int32 [N+1]) B must be 1 and sequence n covers tokens
 * cu[n] .. cu[n+1]-1; without it N = B and sequence n is batch row n.
 * Only heads h_begin .. h_end-1 are computed; other heads' outputs are left
 * untouched.  out may be NULL (state only).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

static double load_elt(const void* base, int dtype, int64_t i) {
    if (dtype == OR_BF16) {
        uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    if (dtype == OR_F64) return ((const double*)base)[i];
    return (double)((const float*)base)[i];
}

typedef struct {
    const void *q, *k, *v;
    int in_dtype;
    const float* beta;
    const float* gate;          /* g = ln a, or NULL (no decay) */
    const double* init_state;   /* float64 copy or NULL */
    const int32_t* cu;
    int64_t n_seq, B, T, H, dk, dv, h_begin, h_end;
    int64_t n_sub;              /* delta-rule writes per token (1 for DeltaNet / GDN) */
    int gate_per_key;           /* 1: gate holds one log decay per key channel (KDA) */
    void* out;
    int out_dtype;
    double* final_state;        /* may be NULL */
    int64_t n_jobs;
    int64_t next_job;           /* shared counter, guarded by lock */
    pthread_mutex_t lock;
} oracle_ctx;

static void run_job(oracle_ctx* c, int64_t job, double* S, double* kt, double* qt, double* u) {
    const int64_t n_heads = c->h_end - c->h_begin;
    const int64_t n = job / n_heads;
    const int64_t h = c->h_begin + job % n_heads;
    const int64_t dk = c->dk, dv = c->dv, H = c->H;
    int64_t row0, len;
    if (c->cu) {
        row0 = c->cu[n];
        len = (int64_t)c->cu[n + 1] - c->cu[n];
    } else {
        row0 = n * c->T;
        len = c->T;
    }
    const int64_t sidx = (n * H + h) * dk * dv;
    if (c->init_state) memcpy(S, c->init_state + sidx, sizeof(double) * dk * dv);
    else memset(S, 0, sizeof(double) * dk * dv);

    for (int64_t t = 0; t < len; ++t) {
        const int64_t tok = row0 + t;                 /* flattened (b, t) row */
        const int64_t q_off = (tok * H + h) * dk;
        const int64_t o_off = (tok * H + h) * dv;
        if (c->gate && c->gate_per_key) {
            /* channelwise decay first: row a of S by exp(g_{t,a}) */
            const float* ga = c->gate + (tok * H + h) * dk;
            for (int64_t a = 0; a < dk; ++a) {
                const double f = exp((double)ga[a]);
                for (int64_t j = 0; j < dv; ++j) S[a * dv + j] *= f;
            }
        } else if (c->gate) {
            /* decay first: the prediction below reads a_t S_{t-1} */
            const double a = exp((double)c->gate[tok * H + h]);
            for (int64_t e = 0; e < dk * dv; ++e) S[e] *= a;
        }
        for (int64_t sub = 0; sub < c->n_sub; ++sub) {
            const int64_t row = tok * c->n_sub + sub;  /* this write's k, v, beta row */
            const int64_t k_off = (row * H + h) * dk;
            const int64_t v_off = (row * H + h) * dv;
            const double b = (double)c->beta[row * H + h];
            for (int64_t a = 0; a < dk; ++a) kt[a] = load_elt(c->k, c->in_dtype, k_off + a);
            /* vhat = k S ; u = beta (v - vhat) */
            for (int64_t j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int64_t a = 0; a < dk; ++a) acc += kt[a] * S[a * dv + j];
                u[j] = b * (load_elt(c->v, c->in_dtype, v_off + j) - acc);
            }
            /* S += k^T u */
            for (int64_t a = 0; a < dk; ++a)
                for (int64_t j = 0; j < dv; ++j) S[a * dv + j] += kt[a] * u[j];
        }
        /* o = q S (after the writes) */
        if (c->out) {
            for (int64_t a = 0; a < dk; ++a) qt[a] = load_elt(c->q, c->in_dtype, q_off + a);
            for (int64_t j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int64_t a = 0; a < dk; ++a) acc += qt[a] * S[a * dv + j];
                if (c->out_dtype == OR_F64) ((double*)c->out)[o_off + j] = acc;
                else ((float*)c->out)[o_off + j] = (float)acc;
            }
        }
    }
    if (c->final_state) memcpy(c->final_state + sidx, S, sizeof(double) * dk * dv);
}

static void* worker(void* arg) {
    oracle_ctx* c = (oracle_ctx*)arg;
    double* S = (double*)malloc(sizeof(double) * c->dk * c->dv);
    double* kt = (double*)malloc(sizeof(double) * c->dk);
    double* qt = (double*)malloc(sizeof(double) * c->dk);
    double* u = (double*)malloc(sizeof(double) * c->dv);
    for (;;) {
        pthread_mutex_lock(&c->lock);
        int64_t job = c->next_job++;
        pthread_mutex_unlock(&c->lock);
        if (job >= c->n_jobs) break;
        run_job(c, job, S, kt, qt, u);
    }
    free(S); free(kt); free(qt); free(u);
    return NULL;
}

/* Returns 0 on success, -1 on a bad argument, -2 on allocation failure.
 * gate may be NULL (no decay), one log decay per (token, head) (gate_per_key 0)
 * or one per key channel (gate_per_key 1); n_sub >= 1 writes per token (T counts
 * tokens, cu_seqlens token offsets). */
int delta_oracle_fwd(const void* q, const void* k, const void* v, int in_dtype,
                     const float* beta, const float* gate, int gate_per_key,
                     const double* init_state, const int32_t* cu_seqlens, int64_t n_seq,
                     int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t n_sub,
                     int64_t h_begin, int64_t h_end,
                     void* out, int out_dtype, double* final_state, int n_threads) {
    if ((B * T > 0) && (!q || !k || !v || !beta)) return -1;
    if (n_sub < 1) return -1;
    if (in_dtype != OR_F32 && in_dtype != OR_BF16 && in_dtype != OR_F64) return -1;
    if (out_dtype != OR_F32 && out_dtype != OR_F64) return -1;
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    if (h_begin < 0 || h_end > H || h_begin >= h_end) return -1;
    if (cu_seqlens) {
        if (B != 1 || n_seq < 0 || cu_seqlens[0] != 0 || cu_seqlens[n_seq] != T) return -1;
        for (int64_t i = 0; i < n_seq; ++i)
            if (cu_seqlens[i + 1] < cu_seqlens[i]) return -1;
    } else {
        n_seq = B;
    }
    oracle_ctx c;
    memset(&c, 0, sizeof c);
    c.q = q; c.k = k; c.v = v; c.in_dtype = in_dtype; c.beta = beta; c.gate = gate;
    c.init_state = init_state; c.cu = cu_seqlens; c.n_seq = n_seq;
    c.B = B; c.T = T; c.H = H; c.dk = dk; c.dv = dv;
    c.h_begin = h_begin; c.h_end = h_end; c.n_sub = n_sub; c.gate_per_key = gate_per_key != 0;
    c.out = out; c.out_dtype = out_dtype; c.final_state = final_state;
    c.n_jobs = n_seq * (h_end - h_begin);
    c.next_job = 0;
    pthread_mutex_init(&c.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > c.n_jobs) n_threads = (int)(c.n_jobs > 0 ? c.n_jobs : 1);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!th) return -2;
    int started = 0;
    for (int i = 0; i < n_threads; ++i) {
        if (pthread_create(&th[i], NULL, worker, &c) == 0) ++started;
        else break;
    }
    if (started == 0) worker(&c);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&c.lock);
    return 0;
}

/* Gated Delta Product with a scalar gate per token. */
int gdp_oracle_fwd(const void* q, const void* k, const void* v, int in_dtype,
                   const float* beta, const float* gate, const double* init_state,
                   const int32_t* cu_seqlens, int64_t n_seq,
                   int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t n_sub,
                   int64_t h_begin, int64_t h_end,
                   void* out, int out_dtype, double* final_state, int n_threads) {
    return delta_oracle_fwd(q, k, v, in_dtype, beta, gate, 0, init_state, cu_seqlens, n_seq, B,
                            T, H, dk, dv, n_sub, h_begin, h_end, out, out_dtype, final_state,
                            n_threads);
}

/* Gated DeltaNet: one write per token (gate may be NULL: plain DeltaNet). */
int gdn_oracle_fwd(const void* q, const void* k, const void* v, int in_dtype,
                   const float* beta, const float* gate, const double* init_state,
                   const int32_t* cu_seqlens, int64_t n_seq,
                   int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                   int64_t h_begin, int64_t h_end,
                   void* out, int out_dtype, double* final_state, int n_threads) {
    return gdp_oracle_fwd(q, k, v, in_dtype, beta, gate, init_state, cu_seqlens, n_seq, B, T, H,
                          dk, dv, 1, h_begin, h_end, out, out_dtype, final_state, n_threads);
}

/* Plain DeltaNet: the gated loop with every a_t = 1 (no decay step at all). */
int dn_oracle_fwd(const void* q, const void* k, const void* v, int in_dtype,
                  const float* beta, const double* init_state,
                  const int32_t* cu_seqlens, int64_t n_seq,
                  int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                  int64_t h_begin, int64_t h_end,
                  void* out, int out_dtype, double* final_state, int n_threads) {
    return gdn_oracle_fwd(q, k, v, in_dtype, beta, NULL, init_state, cu_seqlens, n_seq, B, T, H,
                          dk, dv, h_begin, h_end, out, out_dtype, final_state, n_threads);
}
