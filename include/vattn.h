/*
 * vattn — verified sparse attention (vAttention) for one decode step, on
 * B200 (sm_100a).
 *
 * The operation (from "vAttention: A New Approach to Sparse Attention with
 * Guaranteed Accuracy", section "How vAttention Works", and the paragraph
 * after it on the denominator): for every sequence b and KV head h of a
 * decode step, attention over the cached keys is approximated by
 *   - a deterministic index set I_f: the first `sinks` positions (attention
 *     sinks), the last `window` positions (sliding window) and the top-k of
 *     the remaining middle positions under a ranking score (predicted top-k);
 *   - a uniform random sample, with replacement, of the remaining tail T,
 *     |T| = N_tail, whose size b is set from a pilot sample by the Central
 *     Limit Theorem: n >= (z_{1-delta/2} * N_tail * sigma / (eps * D))^2, so
 *     that the softmax denominator D has relative error <= eps with
 *     probability about 1 - delta;
 *   - output o = (A_f + (N_tail/b) A_s) / (L_f + (N_tail/b) L_s), where A and
 *     L are the exp-weighted value sums and exp sums over I_f and the sample.
 * The same page calls the denominator-only bound a relaxation of bounding the
 * attention output. With vattn_params.guarantee = VATTN_GUARANTEE_OUTPUT the
 * budget also bounds the numerator vector Nv = sum_j x_j v_j (x_j =
 * exp(s_j - m)) by the same CLT condition (a reading; the pages give no
 * formula): n >= (z * N_tail / (eps * |Nv|))^2 * tr(Sigma), with tr(Sigma)
 * the sum over dimensions of the pilot's unbiased variance of x v, and |Nv|^2
 * replaced by a one-sided lower confidence bound from the pilot: with
 * R = N_tail^2 tr(Sigma) / p the noise energy of the pilot mean and
 * U = |Nv_hat|^2 - R, L = U - z sqrt(4 max(U, 0) R + 2 R^2) (not positive:
 * the whole tail). Computed in double in a fixed order (items in
 * list order, then dimensions ascending), so it is reproducible bit for bit.
 * The ranking score is exact (q . k), a SparQ-style proxy over the r largest
 * query components ("SparQ Attention: Bandwidth-Efficient LLM Inference",
 * abstract), or a Loki-style score in a stored low-rank key space ("Loki:
 * Low-rank Keys for Efficient Sparse Attention", abstract).
 *
 * Memory: every array argument is caller-owned DEVICE memory unless stated;
 * the context owns only its workspace, allocated once in vattn_create.
 * vattn_decode allocates no device memory, encodes two row maps of the K and
 * V caches on the host (tensor-map descriptors, passed to the gathers by
 * value), never synchronises the host, and enqueues all its work on
 * `stream`, so it may be captured in a CUDA graph (score-pass timing, when
 * enabled, adds event records on `stream`).
 *
 * Layouts (row-major, innermost last; Hq query heads, Hkv KV heads, d head
 * dim, G = Hq/Hkv, query head hq belongs to KV head hq / G):
 *   q          [batch][Hq][d]                       dtype
 *   k_cache    [num_pages][Hkv][page_size][d]       dtype
 *   v_cache    [num_pages][Hkv][page_size][d]       dtype
 *   page_table [batch][pages_per_seq] int32, pages_per_seq = ceil(max_ctx/page_size);
 *              entries for positions < seq_lens[b] must lie in [0, num_pages)
 *   seq_lens   [batch] int32, 0 <= seq_lens[b] <= max_ctx
 *   out        [batch][Hq][d] float32
 *   sel_idx    [batch][Hkv][max_ctx] int32: I_f ascending, then the b sample
 *              positions in draw order (repeats kept), or, when the sample
 *              would cover the tail (b >= N_tail), the whole tail ascending
 *   sel_count  [batch][Hkv] int32: |I_f| + b (or + N_tail)
 *   budgets    [batch][Hkv] int32: b (N_tail when the tail was taken whole,
 *              0 when there is no tail)
 *   head_need  [batch][Hq] int32: n_h, the CLT size required by query head
 *              hq (N_tail when the tail was taken whole before any pilot); with
 *              the output guarantee, the larger of the denominator's and the
 *              numerator's sizes
 * A contiguous cache is one page per sequence: page_size >= max_ctx (a
 * multiple of 16) and page_table[b][0] = b.
 *
 * Return codes: VATTN_OK, or a negative VATTN_E* code for bad host arguments
 * (nothing is launched) or a CUDA launch failure. Device-side violations (a
 * page id out of range, a sequence length outside [0, max_ctx]) never trap:
 * the kernel treats that sequence as empty (zero output, empty selection)
 * and sets a bit in the context's device error word, read by
 * vattn_last_error.
 */
#ifndef VATTN_H
#define VATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { VATTN_FP32 = 0, VATTN_BF16 = 1 };
enum { VATTN_EXACT = 0, VATTN_SPARQ = 1, VATTN_LOKI = 2 };
/* where the K and V caches live (vattn_config.kv_location) */
enum { VATTN_KV_DEVICE = 0, VATTN_KV_HOST = 1 };
/* what the sample size bounds: the softmax denominator alone (the pages'
   practical form), or the denominator and the numerator vector (output) */
enum { VATTN_GUARANTEE_DENOMINATOR = 0, VATTN_GUARANTEE_OUTPUT = 1 };

enum {
  VATTN_OK = 0,
  VATTN_EINVAL = -1, /* a host argument is out of range or a required pointer is NULL */
  VATTN_ENOMEM = -2, /* workspace allocation failed in vattn_create                 */
  VATTN_ECUDA = -3,  /* a CUDA call or kernel launch failed                          */
  VATTN_ESCRATCH = -4 /* vattn_dense_decode_static: the call needs more scratch than
                         its fixed device array holds                              */
};

/* bits of the device error word; VATTN_DEV_TIMEOUT: a kernel's bounded wait
   for its own copies ran out, so the call's outputs are not valid */
enum { VATTN_DEV_BAD_SEQLEN = 1, VATTN_DEV_BAD_PAGE = 2, VATTN_DEV_TIMEOUT = 4 };

typedef struct vattn_ctx vattn_ctx;

/* Fixed for the life of a context. */
typedef struct {
  int num_q_heads;  /* Hq, a multiple of num_kv_heads with Hq/Hkv in {1,2,4,8} */
  int num_kv_heads; /* Hkv >= 1                                                  */
  int head_dim;     /* d in {64, 128}                                            */
  int dtype;        /* VATTN_FP32 or VATTN_BF16, for q and every cache          */
  int page_size;    /* rows per page, a multiple of 16 (contiguous cache: max_ctx */
                    /* rounded up to a multiple of 16)                            */
  int max_batch;    /* upper bound on `batch` in every call                      */
  int max_ctx;      /* upper bound on seq_lens[b]; 1 <= max_ctx <= 2^24          */
  int proxy;        /* VATTN_EXACT, VATTN_SPARQ or VATTN_LOKI                    */
  int proxy_rank;   /* SparQ: r in [1, d]; Loki: the stored rank, 32             */
  /* VATTN_KV_DEVICE: k_cache and v_cache are device memory. VATTN_KV_HOST: they
     are page-locked host memory (cudaHostAlloc / cudaMallocHost, or
     cudaHostRegister with cudaHostRegisterMapped), passed by their host
     address; the library maps each call's pointers to their device addresses
     and reads only the rows it selects (and, in exact mode, the whole of K for
     the ranking pass) over the host link ("vAttention: A New Approach to
     Sparse Attention with Guaranteed Accuracy", section "Performance and
     Efficiency": speedups when the KV cache is hosted on the CPU). Every other
     array, the SparQ and Loki proxy caches included, stays in device memory.
     A cache pointer that is not page-locked host memory returns VATTN_EINVAL. */
  int kv_location;
} vattn_config;

/* Per call. */
typedef struct {
  int sinks, window; /* >= 0                                                      */
  /* top-k size for a sequence of length N: topk_abs if topk_den == 0, else
     floor(N * topk_num / topk_den); then capped by the middle's length        */
  int topk_abs, topk_num, topk_den;
  /* pilot size: pilot_min if pilot_den == 0, else
     max(pilot_min, ceil(N * pilot_num / pilot_den)); pilot_min >= 2           */
  int pilot_min, pilot_num, pilot_den;
  float eps;         /* > 0: relative error target on the softmax denominator   */
                     /* (and on |Nv| with the output guarantee)                  */
  float delta;       /* in (0, 1): allowed failure probability                  */
  uint64_t seed;     /* Philox4x32-10 key of the tail sampler                   */
  int num_pages;     /* pages in the caches (bound for page_table entries);     */
                     /* num_pages * Hkv * page_size must stay below 2^31        */
  const void* k_t_cache;    /* SparQ: dim-major K [num_pages][Hkv][d][page_size], else NULL  */
  const void* k_proj_cache; /* Loki: projected K [num_pages][Hkv][page_size][rank], else NULL */
  const float* proj_basis;  /* Loki: basis fp32 [Hkv][d][rank], else NULL                     */
  int guarantee;     /* VATTN_GUARANTEE_DENOMINATOR (0) or VATTN_GUARANTEE_OUTPUT;  */
                     /* OUTPUT adds one kernel that reads the V rows of I_f and the */
                     /* pilot once more; anything else: VATTN_EINVAL                */
  /* Top-p selection (the pages name top-k "(or top-p)" selection as the
     predictor of the deterministic set; "vAttention: A New Approach to Sparse
     Attention with Guaranteed Accuracy", third paragraph). topp_den > 0
     replaces the fixed top-k (topk_* are then ignored): the predicted set is
     the smallest number of the highest-ranked middle positions (ranking order,
     ties to the lower position) whose share of the middle's softmax mass under
     the scaled ranking scores reaches p = topp_num / topp_den, the mass taken
     in 2^-32 fixed point (w_j = rint(exp(r_j/sqrt(d) - max) * 2^32), exp the
     budget's fixed-order exp) so that the cut is the exact integer test
     prefix * den >= num * S. 0 <= topp_num <= topp_den; topp_den = 0: off. */
  int topp_num, topp_den;
  /* Sharded runs: when this call decodes a slice of a larger batch (a range of
     sequences, or a range of KV heads with their query heads), the index of its
     first sequence and first KV head in the whole batch. The sampler's draw
     counter names the sequence and KV head in the whole batch, (batch_offset + b,
     head_offset + h), so the shards together draw exactly what one call over the
     whole batch would. 0 for an unsharded call; both >= 0. */
  int batch_offset, head_offset;
} vattn_params;

/* Create a context on the current CUDA device and allocate its workspace.
   Returns VATTN_OK and sets *out, or VATTN_EINVAL / VATTN_ENOMEM. */
int vattn_create(vattn_ctx** out, const vattn_config* cfg);

/* One sparse decode step (the operation described above) for `batch`
   sequences, enqueued on `stream` (a cudaStream_t; NULL = legacy default). */
int vattn_decode(vattn_ctx* ctx, const void* q, const void* k_cache, const void* v_cache,
                 const int32_t* page_table, const int32_t* seq_lens, int batch,
                 const vattn_params* params, float* out, int32_t* sel_idx, int32_t* sel_count,
                 int32_t* budgets, int32_t* head_need, void* stream);

/* Dense decode attention over all seq_lens[b] positions, same layouts: the
   comparison baseline for vattn_decode (softmax(q K^T / sqrt(d)) V). */
int vattn_dense_decode(vattn_ctx* ctx, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* page_table, const int32_t* seq_lens, int batch,
                       int num_pages, float* out, void* stream);

/* Dense decode attention, as vattn_dense_decode, without a context and
   without allocating anything. The paper has no counterpart: this entry point
   serves callers that cannot allocate device memory when they call, e.g. a
   server that has given all free memory to its KV-cache pool (an allocation
   would fail), code that must not risk the device-wide wait that freeing
   memory can cause, or a plug-in that cannot keep a context between calls.
   `cfg` gives the shapes (proxy and proxy_rank are ignored); the other
   arguments are those of vattn_dense_decode, on the current device.

   Scratch: a fixed array of 8 MiB per device, defined in the library. A call
   needs batch * Hq * (head_dim + 2) * 4 bytes of it at least; a larger call
   returns VATTN_ESCRATCH before touching the device. The first call made
   under a CUDA context looks up that device's copy of the array (and its SM
   count); a call under a different context on the same device (after
   cudaDeviceReset, or with a driver-API context current) looks it up again,
   since the old address belongs to the old context. Make the first call of
   each context before any stream capture begins. Every later
   call on the device shares the same array: it keeps the last call's partial
   results, nothing in it needs to start at zero (a call writes every part it
   reads), and calls that overlap in time on one device race and corrupt
   each other's output, so order them (one stream, or events). Device-side
   violations (a page id out of range, a bad sequence length) give a zero
   output for that sequence; there is no error word to read. */
int vattn_dense_decode_static(const vattn_config* cfg, const void* q, const void* k_cache,
                              const void* v_cache, const int32_t* page_table,
                              const int32_t* seq_lens, int batch, int num_pages, float* out,
                              void* stream);

/* sync != 0: wait for the device, then return and clear the device error
   word (VATTN_DEV_* bits). sync == 0: return the host status of the last
   call on this context, without touching the device. */
int vattn_last_error(vattn_ctx* ctx, int sync);

/* Self-check of the device error path: launches one warp on `stream` that
   waits, with a limit of `tries` tries (1 .. 2^20), on a barrier that no copy
   ever completes, exactly as the kernels' copy rings wait for their copies,
   and sets VATTN_DEV_TIMEOUT in the context's error word when the limit runs
   out (it always does). The kernel then returns normally; nothing is left in
   flight, and the context stays usable. vattn_last_error(ctx, 1) reports and
   clears the bit. Returns VATTN_EINVAL for a bad argument. (No counterpart in
   the pages: it exists so that the timeout path can be tested without a
   fault.) */
int vattn_check_bounded_wait(vattn_ctx* ctx, int tries, void* stream);

/* Bytes of device workspace the context holds. */
size_t vattn_workspace_bytes(const vattn_ctx* ctx);

/* Per-call kernel timing: with period >= 1, every period-th vattn_decode call
   records a CUDA event pair around its dominant kernel (the ranking-score
   pass) on `stream` (0 turns it off; the event pair breaks the overlap of
   that kernel with its neighbours, so sampling keeps the other calls
   undisturbed); vattn_score_pass_ms returns the summed elapsed time in
   milliseconds since the last reset and how many passes it covers. Calls
   synchronise on the recorded events (host wait). */
int vattn_set_timing(vattn_ctx* ctx, int period);
int vattn_score_pass_ms(vattn_ctx* ctx, double* total_ms, int* count, int reset);

/* Number of kernel launches the last vattn_decode / vattn_dense_decode call
   enqueued. */
int vattn_last_launch_count(const vattn_ctx* ctx);

/* Text for a return code. */
const char* vattn_strerror(int code);

/* Release the workspace and the context. NULL is allowed. */
void vattn_destroy(vattn_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* VATTN_H */
