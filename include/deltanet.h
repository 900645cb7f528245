/*
 * deltanet.h -- C ABI of the B200 (sm_100a) chunkwise DeltaNet forward pass.
 *
 * The operation ("Linear Attention, Visualized", section "DeltaNet: correcting
 * memory collisions"; "Context Parallelism for DeltaNet", section 2): for every
 * sequence n and head h, starting from S = initial_state[n, h] (or zero),
 *
 *     vhat_t = k_t S,  u_t = beta_t (v_t - vhat_t),  S <- S + k_t^T u_t,  o_t = q_t S
 *
 * in the row-vector convention, S being d_k x d_v ("Recurrent form").  This is
 * S_t = S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t with the
 * state transposed.  The library evaluates it chunk by chunk (chunk C = 64)
 * through the WY/UT factors of the "Complete per-chunk algorithm"
 * (L = (K K^T) o M^-, (I + B L) T = B, W = T K, U = T V, Z = U - W S,
 * O = Q S + (Q K^T o M) Z, S' = S + K^T Z), and splits each sequence's chain of
 * chunk states across the GPU's SMs by composing the affine maps
 * S_end = P S_start + H of runs of chunks ("One chunk as an affine recurrence";
 * "Context Parallelism for DeltaNet", section 3).  No query scaling is applied.
 *
 * Tensors are passed as descriptors of device memory (dn_tensor).  Strides are
 * in ELEMENTS.  Every call is asynchronous on the given CUDA stream.
 */
#ifndef DELTANET_H_
#define DELTANET_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DN_OK = 0,
    DN_ERR_INVALID_ARG = 1,   /* bad shape, dtype, stride, alignment or NULL pointer */
    DN_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement (chunk size,
                                 head dims, device other than sm_100) */
    DN_ERR_ALIAS = 3,         /* an output overlaps an input or another output */
    DN_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    DN_ERR_WORKSPACE = 5,     /* workspace allocation failed */
    DN_ERR_SEQLENS = 6,       /* cu_seqlens content invalid (reported by deltanet_get_error) */
    DN_ERR_TIMEOUT = 7        /* a bounded device-side wait gave up (reported by deltanet_get_error) */
} dn_status;

typedef enum { DN_F32 = 0, DN_BF16 = 1, DN_I32 = 2 } dn_dtype;

/* A strided view of device memory.  shape/stride entries beyond ndim are ignored. */
typedef struct {
    void* data;
    int32_t dtype;        /* dn_dtype */
    int32_t ndim;
    int64_t shape[4];
    int64_t stride[4];    /* in elements */
} dn_tensor;

/*
 * deltanet_fwd -- DeltaNet forward pass over a batch.
 *
 *   q, k          [B, T, H, d_k]   bf16 or fp32 (the same dtype for q, k, v, out)
 *   v             [B, T, H, d_v]
 *   beta          [B, T, H]        fp32, any finite values (the pages use 0 < beta <= 1)
 *   initial_state [N, H, d_k, d_v] fp32, or NULL for zeros
 *   cu_seqlens    int32 [N + 1] device array, or NULL.  With it, B must be 1 and
 *                 sequence n covers tokens cu[n] .. cu[n+1]-1 (cu[0] = 0,
 *                 cu[N] = T, non-decreasing; zero-length sequences allowed).
 *                 Without it N = B and each batch row is one sequence.
 *   chunk_size    must be 64 (others: DN_ERR_UNSUPPORTED)
 *   out           [B, T, H, d_v], dtype of q; fully overwritten (bf16 rounded to
 *                 nearest-even from the fp32 accumulator)
 *   final_state   [N, H, d_k, d_v] fp32, or NULL (not produced)
 *   stream        cudaStream_t (NULL = legacy default stream)
 *
 * Supported head dims: bf16 d_k, d_v in {64, 128}; fp32 d_k = d_v = 64.
 * Layout rules: the last dimension of every tensor has stride 1; q/k/v/out base
 * addresses and their B/T/H strides are multiples of 16 bytes; states have
 * stride[3] = 1 and stride[2] = d_v, with 16-byte aligned N/H strides and base.
 * The caller owns every buffer; the library only reads the inputs.  Any byte
 * overlap between an output and an input or the other output returns
 * DN_ERR_ALIAS (final_state may not alias initial_state).
 *
 * Returns DN_OK once all kernels are enqueued on `stream`.  Argument errors are
 * reported synchronously and nothing is launched.  Errors found on the device
 * (invalid cu_seqlens contents, a bounded wait that ran out) are recorded in a
 * per-stream flag read by deltanet_get_error; in that case out/final_state are
 * unspecified.  Reentrant: calls on different streams use separate workspaces.
 */
dn_status deltanet_fwd(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                       const dn_tensor* beta, const dn_tensor* initial_state,
                       const dn_tensor* cu_seqlens, int chunk_size,
                       dn_tensor* out, dn_tensor* final_state, void* stream);

/*
 * deltanet_fwd_ex -- deltanet_fwd with a scheduling override.
 * seg_chunks > 0 forces every sequence to be split into runs of
 * (seg_chunks & 0xffff) chunks (the last run of each sequence may be shorter),
 * each run on its own CTA, composed through the segment maps; 0 lets the
 * library choose.  For dense batches, bits 16-30 may force a different length
 * of the first run ((seg_chunks >> 16): its chunks, 1 .. the run length; 0:
 * the same length).  The result is the same up to rounding for every value
 * (the composition is exact), which the tests exercise.  Returns
 * DN_ERR_WORKSPACE if the forced split needs more segment slots than the
 * library's limit (4096), DN_ERR_INVALID_ARG for a first run longer than the
 * others.
 */
dn_status deltanet_fwd_ex(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                          const dn_tensor* beta, const dn_tensor* initial_state,
                          const dn_tensor* cu_seqlens, int chunk_size,
                          dn_tensor* out, dn_tensor* final_state, void* stream,
                          int seg_chunks);

/*
 * gated_deltanet_fwd -- Gated DeltaNet forward pass ("Linear Attention,
 * Visualized", section "Gated DeltaNet (GDN)"): the same recurrence with a
 * per-token scalar decay a_t on the whole transition,
 *
 *     S_t = a_t (I - beta_t k_t^T k_t) S_{t-1} + beta_t k_t^T v_t,   o_t = q_t S_t,
 *
 * i.e. S <- a_t S first, then the DeltaNet prediction, correction and write
 * from the decayed state.  It is evaluated with that section's "Complete
 * per-chunk algorithm" (decay products lambda[i:j] inside a chunk, the mask
 * Gamma[l][i] = lambda[i+1:l], left-decayed q, k and right-decayed k) and the
 * same split of each chain across SMs (a chunk is still an affine map of the
 * state, S' = (lambda[1:C] I - K->^T W<-) S + K->^T U).
 *
 *   g             [B, T, H] fp32, the decay as its natural log: g_t = ln a_t
 *                 (finite; the pages use 0 < a_t <= 1, i.e. g_t <= 0).  Decay
 *                 products are formed as exp of differences of the chunk's
 *                 running fp32 sum of g, so their relative error grows with
 *                 |sum of g over a chunk| times 2^-24.
 *   other arguments, layouts, ownership, aliasing (g is an input) and errors
 *   as deltanet_fwd; g == NULL returns DN_ERR_INVALID_ARG.
 *
 * bf16 with d_k = d_v = 128 runs on the tensor-core (tcgen05) kernels' gated
 * instances: a pre-pass that also writes T diag(lambda), the decayed queries and
 * the row factors per (chunk, head), then the summary and boundary passes.  The
 * other supported shapes run on the mma.sync chain kernels.
 */
dn_status gated_deltanet_fwd(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                             const dn_tensor* beta, const dn_tensor* g,
                             const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                             int chunk_size, dn_tensor* out, dn_tensor* final_state,
                             void* stream);

/* gated_deltanet_fwd with the seg_chunks override of deltanet_fwd_ex. */
dn_status gated_deltanet_fwd_ex(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                                const dn_tensor* beta, const dn_tensor* g,
                                const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                                int chunk_size, dn_tensor* out, dn_tensor* final_state,
                                void* stream, int seg_chunks);

/*
 * deltanet_fwd_states -- the forward pass that also keeps the state entering
 * every chunk, the chunk-boundary states S_[r] that a backward pass reuses
 * ("Linear Attention, Visualized", section "Chunkwise algorithm": the chunk
 * states are the only quantities carried between chunks).
 *
 *   g             NULL for DeltaNet, or Gated DeltaNet's log decay [B, T, H] fp32
 *   chunk_states  [rows, H, d_k, d_v] fp32 (state layout rules): row = global
 *                 chunk index, chunks numbered per sequence in input order
 *                 (dense: b * ceil(T / 64) + r; packed: the chunks of earlier
 *                 sequences first, ceil(L_n / 64) per sequence).  Dense batches
 *                 need rows == B * ceil(T / 64); packed input rows >=
 *                 ceil(T / 64) + N (rows past the total are not written).  Row r
 *                 holds the state before chunk r's tokens (row 0 of a sequence is
 *                 its initial state).
 *   seg_chunks    as deltanet_fwd_ex (0: the library chooses)
 *   other arguments, layouts, ownership and errors as deltanet_fwd /
 *   gated_deltanet_fwd; chunk_states may not overlap any other tensor.
 *
 * bf16 with d_k = d_v = 128 runs on the tensor-core kernels, whose boundary
 * pass stores the state from tensor memory at every chunk start; the other
 * supported shapes run on the mma.sync chain kernels, which keep the state in
 * registers and store it likewise.
 */
dn_status deltanet_fwd_states(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                              const dn_tensor* beta, const dn_tensor* g,
                              const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                              int chunk_size, dn_tensor* out, dn_tensor* final_state,
                              dn_tensor* chunk_states, void* stream, int seg_chunks);

/*
 * gated_deltaproduct_fwd -- Gated Delta Product forward pass ("Linear
 * Attention, Visualized", section "Gated Delta Product (GDP)"): each token makes
 * n_h delta-rule writes, each with its own key, value and beta, after one decay
 * of the state and before the token's readout:
 *
 *     S_{t,0} = a_t S_{t-1},
 *     S_{t,j} = (I - beta_{t,j} k_{t,j}^T k_{t,j}) S_{t,j-1} + beta_{t,j} k_{t,j}^T v_{t,j}
 *               for j = 1 .. n_h,
 *     S_t = S_{t,n_h},  o_t = q_t S_t.
 *
 * Evaluated as that section's "GDP as GDN over a virtual sequence": the writes
 * are the steps m = n_h (t - 1) + j of a sequence n_h times longer, with the
 * decay on each token's first step and the query on its last; the kernels read
 * the query, the decay and write the output through that index map, so nothing
 * of the virtual sequence is materialised.
 *
 *   q             [B, T, H, d_k]        one row per token
 *   k             [B, T * n_h, H, d_k]  n_h rows per token, substep-major: row
 *                                       (t * n_h + j - 1) is write j of token t
 *                                       (the [B, T, n_h, H, d] layout, flattened)
 *   v             [B, T * n_h, H, d_v]
 *   beta          [B, T * n_h, H] fp32
 *   g             [B, T, H] fp32        ln a_t, one per token (as gated_deltanet_fwd)
 *   cu_seqlens    token offsets (not write offsets), or NULL
 *   n_h           writes per token, 1 .. 1024 (1 is gated_deltanet_fwd)
 *   out           [B, T, H, d_v]        one row per token
 *   other arguments, layouts, ownership, aliasing and errors as gated_deltanet_fwd;
 *   B * T * n_h must stay below 2^31.
 * bf16 with d_k = d_v = 128 runs on the tensor-core kernels' gated instances for
 * several steps per token; the other supported shapes on the mma.sync chain kernels.
 */
dn_status gated_deltaproduct_fwd(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                                 const dn_tensor* beta, const dn_tensor* g,
                                 const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                                 int n_h, int chunk_size, dn_tensor* out,
                                 dn_tensor* final_state, void* stream);

/* gated_deltaproduct_fwd with the seg_chunks override of deltanet_fwd_ex (runs
 * count chunks of the virtual sequence). */
dn_status gated_deltaproduct_fwd_ex(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                                    const dn_tensor* beta, const dn_tensor* g,
                                    const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                                    int n_h, int chunk_size, dn_tensor* out,
                                    dn_tensor* final_state, void* stream, int seg_chunks);

/*
 * kda_fwd -- Kimi Delta Attention forward ("Linear Attention, Visualized",
 * section "Kimi Delta Attention (KDA)"): every key channel c decays by its own
 * a_t[c] before the delta-rule correction,
 *   S_t = (I - beta_t k_t^T k_t) Diag(a_t) S_{t-1} + beta_t k_t^T v_t,  o_t = q_t S_t,
 * evaluated with the section's complete per-chunk algorithm (decayed K<- / K->
 * / Q<- rows, channel-decayed L and A, S' = Diag(lambda[1:C]) S + K->^T Z).
 *
 * Arguments as gated_deltanet_fwd, except
 *   g   [B, T, H, d_k] fp32, g[b, t, h, c] = ln a_t[c] for head h (channel c of
 *       the key), last dim contiguous, 16-byte aligned rows and strides (it is
 *       read in 16-byte pieces); finite, and |g| < 5.8 per token and channel
 *       (within a chunk the kernel forms decay ratios over up to 15 tokens from
 *       running sums of g, which stay in range under that bound).
 * Supported: bf16 q/k/v/out with d_k, d_v in {64, 128}, dense or packed
 * (cu_seqlens), split across SMs like deltanet_fwd.  A dense batch with
 * d_k = d_v = 128 whose chains the schedule does not split runs on the tensor
 * cores: a KDA pre-pass writes T, P, the decayed Q<-, K<-, K-> and lambda[1:C]
 * per (chunk, head) (66,560 bytes of workspace each), then the boundary kernel's
 * KDA instance runs the chains.  Split chains, packed input and d = 64 run on
 * the mma.sync chain kernels.  Pad rows of a last partial chunk carry g = 0
 * (identity steps).
 * Returns DN_ERR_UNSUPPORTED for fp32 inputs or other head sizes.
 */
dn_status kda_fwd(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v, const dn_tensor* beta,
                  const dn_tensor* g, const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                  int chunk_size, dn_tensor* out, dn_tensor* final_state, void* stream);

/* kda_fwd with the seg_chunks override of deltanet_fwd_ex. */
dn_status kda_fwd_ex(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v, const dn_tensor* beta,
                     const dn_tensor* g, const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                     int chunk_size, dn_tensor* out, dn_tensor* final_state, void* stream,
                     int seg_chunks);

/*
 * deltanet_fwd_noalloc -- the forward pass without any device allocation.
 * (No counterpart on the pages: this is a deployment variant of deltanet_fwd.)
 *
 * For callers that cannot call cudaMalloc: code running where the allocator
 * must not be entered (host callbacks, plugins inside another runtime's
 * allocator, graph-recording runtimes that forbid allocation) or processes
 * whose device memory is capped and owned by someone else.  deltanet_fwd may
 * grow a cached workspace with cudaMallocAsync; this call never allocates.
 * Its scratch (the per-chunk UT factors and an error word) is one fixed
 * 48 MiB + 256 B __device__ array that every GPU loading the library holds
 * until the process exits.
 *
 * Arguments as deltanet_fwd, without cu_seqlens.  Supported: dense batches,
 * bf16 q/k/v/out, d_k = d_v = 128, chunk_size 64, and
 * B * ceil(T / 64) * H <= 3072 (chunk, head) pairs; larger problems return
 * DN_ERR_WORKSPACE, other shapes or dtypes DN_ERR_UNSUPPORTED / _INVALID_ARG.
 * Aliasing as deltanet_fwd: an output that overlaps an input or the other
 * output (final_state == initial_state included) returns DN_ERR_ALIAS.  Each
 * (sequence, head) runs as one run of chunks (no split across SMs).
 * Device-side errors (DN_ERR_TIMEOUT) go to the array's error word, which
 * each call clears when it starts; deltanet_get_error(stream), called with
 * the stream of the call, reads and clears it.
 * The first call on a device looks up the array's device address and sets
 * kernel attributes; make it before any stream capture.  All calls share the
 * array, which keeps the last call's contents, so calls that overlap on the
 * GPU race with each other; serialise them (one stream, or events).
 */
dn_status deltanet_fwd_noalloc(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                               const dn_tensor* beta, const dn_tensor* initial_state,
                               int chunk_size, dn_tensor* out, dn_tensor* final_state,
                               void* stream);

/* Human-readable name of a status code (static storage; never NULL). */
const char* deltanet_status_string(dn_status status);

/*
 * deltanet_get_error -- synchronises `stream`, then returns and clears the
 * device-side error flag of the calls made on it (DN_OK, DN_ERR_SEQLENS or
 * DN_ERR_TIMEOUT), or DN_ERR_CUDA if the stream itself reports an error.
 * It also reads and clears the error word of deltanet_fwd_noalloc's scratch
 * on the current device (one per device, shared by all streams).
 */
dn_status deltanet_get_error(void* stream);

/*
 * deltanet_test_set_wait -- test hook for the time-out path of the bounded
 * device waits, for the calls made after it on this host thread.
 * wait_ns: time after which a device wait gives up and the call reports
 * DN_ERR_TIMEOUT through deltanet_get_error (0 restores the default, 2 s).
 * stall_chunk > 0: in the tensor-core boundary kernel (bf16, d_k = d_v = 128),
 * the thread that issues the state-chain products waits, at chunk
 * stall_chunk - 1 of every run, on a barrier that nothing completes, so that
 * the wait runs out: the kernel then gives up, waits for its copies and
 * products in flight, frees its tensor memory, exits and reports the
 * time-out.  The outputs of such a call are unspecified.  0 (the default):
 * no stall.  deltanet_test_set_wait(0, 0) restores normal calls.
 */
void deltanet_test_set_wait(unsigned long long wait_ns, int stall_chunk);

/* Frees every cached workspace (synchronises the device first). */
void deltanet_release_workspace(void);

/*
 * deltanet_last_schedule -- the segmentation chosen by the last successful
 * call on this thread for dense (cu_seqlens == NULL) batches: segments per
 * sequence-head chain, chunks per segment, and chunks of the first segment
 * (which may be shorter: on the tensor-core path it runs next to the summary
 * pass, which costs less per chunk).  Any pointer may be NULL.  Varlen batches
 * are scheduled on the device and report -1 for all three.  For tests and
 * benchmarks.
 */
void deltanet_last_schedule(int* segments_per_chain, int* chunks_per_segment,
                            int* chunks_first_segment);

/* Number of kernels the last successful call on this thread enqueued. */
int deltanet_last_launches(void);

/*
 * deltanet_set_kernel_events -- profiling hook.  While set (non-NULL), every
 * deltanet_fwd / gated_deltanet_fwd / gated_deltaproduct_fwd (and _ex) /
 * deltanet_fwd_states call on this thread records start_event on
 * its stream right before launching the boundary-pass kernel (the output
 * kernel, which dominates the call) and stop_event right after it, so that
 * cudaEventElapsedTime gives that kernel's device time.  The caller owns the
 * events (cudaEvent_t, created with timing enabled); pass NULL, NULL to stop.
 */
void deltanet_set_kernel_events(void* start_event, void* stop_event);

#ifdef __cplusplus
}
#endif

#endif /* DELTANET_H_ */
