/*
 * jolt.h -- C ABI of the JoLT / FlashJoLT KV-cache compressor for NVIDIA B200 (sm_100a).
 *
 * What it computes (sources: "A JoLT for the KV cache: Near-Lossless KV Cache Compression
 * via Joint Rank-bit Allocation", abstract; "A JoLT for the KV Cache: Near-Lossless KV
 * Cache Compression via Joint Tucker and JL-Residual Allocation for LLMs", introduction):
 * per layer group and separately for keys and values, the grouped prefill cache
 * X[l, h, t, d] (layers x heads x tokens x features) is factored by a partial Tucker
 * decomposition on the token and feature modes only, X[l,h] ~ U C[l,h] W^T; the
 * truncation residual is rotated by a random orthogonal (Johnson-Lindenstrauss) rotation
 * and quantised to b bits; one Lagrangian dual picks (token rank, feature rank, bits)
 * for every unit under one global byte budget.  JoLT takes the token factor from an
 * exact eigen-decomposition; FlashJoLT from a randomized SVD sketch Y = X_(T) Omega.
 *
 * Readings of what the pages leave open (all fixed here):
 *   - unit u = 2*g + kv: layer group g (layers_per_group consecutive layers), kv 0 = K, 1 = V;
 *     S = layers_per_group * n_heads slices per unit, M = S * head_dim;
 *   - rotation along the features of every row: rho = r diag(sigma) H_D / sqrt(D), H_D the
 *     Sylvester Hadamard matrix, sigma from splitmix64 (seed, stream 2<<32 | u, index d);
 *   - quantiser: blocks of 16 consecutive rotated features, lo = fp16 round-down(min),
 *     step = fp16 round-up((max - lo)/(2^b - 1)), code = round-half-even((rho - lo)/step);
 *   - stored factors U (T x r_T), W (D x r_D), core (S x r_T x r_D) in bf16; the decoder
 *     forms U P' with P' = bf16((C W^T) diag(sigma) H_D / sqrt(D)) and un-rotates the sum
 *     of that and the dequantised residual;
 *   - budget = total blob bytes including the 64-byte global header and 64 bytes per unit.
 *
 * Conventions for every call:
 *   - every pointer named *_dev is device memory the caller owns; the library keeps no
 *     pointer after the call returns and takes no workspace from cudaMalloc.  It does own
 *     these per-thread resources, created on first use and kept until jolt_release() or
 *     thread exit: a cuSOLVER handle and parameter object for each of two streams (eigen
 *     solves that are not the library's own kernels), one auxiliary non-blocking stream with
 *     two events (the feature factor runs on it beside the token factor), one capture stream
 *     and up to 8 instantiated CUDA graphs of compress calls (see jolt_set_graphs), and the
 *     CUDA events of stage timing (jolt_profile_begin/end).  The compiled-in 64 KiB array of
 *     jolt_frobenius_noalloc is held by every device that loads the library;
 *   - calls are stream-ordered on `stream` (a cudaStream_t, NULL = legacy default stream)
 *     and return before the GPU work finishes, except where a call says it synchronises;
 *   - argument errors are detected on the host and returned before anything is launched;
 *     errors found on the device (non-finite input, infeasible budget, factorisation
 *     breakdown) are written to the blob's header status word and returned by the next
 *     call that synchronises (jolt_read_header, jolt_decompress);
 *   - on any non-OK return, jolt_last_error() gives a one-line message (thread-local).
 */
#ifndef JOLT_H_
#define JOLT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  JOLT_OK = 0,
  JOLT_ERR_INVALID_ARG = 1,        /* null pointer, bad enum, bad candidate list */
  JOLT_ERR_UNSUPPORTED_SHAPE = 2,  /* head_dim not in {16,32,64,128}, n_tokens % 16, ... */
  JOLT_ERR_WORKSPACE_TOO_SMALL = 3,
  JOLT_ERR_OUTPUT_TOO_SMALL = 4,   /* blob capacity below the budget */
  JOLT_ERR_BUDGET_INFEASIBLE = 5,  /* budget below every unit's fewest-bytes choice */
  JOLT_ERR_NUMERIC = 6,            /* NaN/Inf in the cache, or an eigen/Cholesky breakdown */
  JOLT_ERR_TIMEOUT = 7,            /* a bounded device-side wait (tensor-core pipeline) gave up */
  JOLT_ERR_CUDA = 8,               /* a CUDA runtime or cuSOLVER call failed */
  JOLT_ERR_BAD_BLOB = 9            /* blob header failed validation */
} jolt_status;

typedef enum { JOLT_BF16 = 0, JOLT_F32 = 1 } jolt_dtype;
typedef enum { JOLT_EXACT = 0, JOLT_RANDOMIZED = 1 } jolt_method;

/* Shape of ONE of the two cache tensors K and V, both [n_layers, n_heads, n_tokens, head_dim],
 * row-major, element type `dtype`.  n_layers % layers_per_group == 0. */
typedef struct {
  int32_t n_layers;
  int32_t n_heads;
  int32_t n_tokens;
  int32_t head_dim;
  int32_t layers_per_group;
  int32_t dtype; /* jolt_dtype */
} jolt_shape;

#define JOLT_MAX_CANDIDATES 8

/* Candidate sets of the allocation (ascending, no repeats) and the token-factor method.
 * Choice index c = (i_T * n_feature_ranks + i_D) * n_bits + i_b. */
typedef struct {
  int32_t n_token_ranks;
  int32_t token_ranks[JOLT_MAX_CANDIDATES];   /* 1 <= r_T <= n_tokens (and <= M) */
  int32_t n_feature_ranks;
  int32_t feature_ranks[JOLT_MAX_CANDIDATES]; /* 1 <= r_D <= head_dim */
  int32_t n_bits;
  int32_t bits[JOLT_MAX_CANDIDATES];          /* 0 <= b <= 8; 0 = no residual */
  int32_t method;                             /* jolt_method */
  int32_t oversample;                         /* FlashJoLT sketch width = max r_T + oversample */
  int32_t power_iters;                        /* FlashJoLT power iterations */
  int32_t unit_offset;                        /* global index of this cache's first unit, 0 for a whole
                                                 cache; a shard holding layer groups g0.. of a larger
                                                 cache passes 2 * g0, so the rotation signs and the
                                                 sketch of its units are those of the whole cache
                                                 (recorded in the blob header for the decoder) */
} jolt_options;

/* Per-unit record of a compressed blob, as returned by jolt_read_header. */
typedef struct {
  int32_t r_T, r_D, bits, choice;
  uint64_t off_U, off_W, off_C, off_codes, off_scales; /* byte offsets inside the blob */
  double distortion;  /* table value || X_u - decode(encode(X_u)) ||_F^2 of the choice */
} jolt_unit_record;

/* Library version string. */
const char* jolt_version(void);

/* Message of the last non-OK status returned on this thread. */
const char* jolt_last_error(void);

/* Sizes the caller must provide.
 *   ws_bytes   : device workspace for jolt_compress / jolt_factor / jolt_table / jolt_encode
 *   blob_bytes : the largest blob any budget can produce (every unit at its largest choice)
 *   dws_bytes  : device workspace for jolt_decompress
 * Returns INVALID_ARG / UNSUPPORTED_SHAPE for shapes or options the library rejects. */
jolt_status jolt_workspace_size(const jolt_shape* shape, const jolt_options* opts, size_t* ws_bytes,
                                size_t* blob_bytes, size_t* dws_bytes);

/* Number of units (2 * n_layers / layers_per_group) and of choices per unit. */
jolt_status jolt_counts(const jolt_shape* shape, const jolt_options* opts, int32_t* n_units,
                        int32_t* n_choices);

/* Payload bytes of every choice (identical for all units), n_choices uint64 on the HOST.
 * Formula: pad16(2 T r_T) + pad16(2 D r_D) + pad16(2 S r_T r_D)
 *        + [b > 0] (pad16(nblk * 2b) + pad16(nblk * 4)),  nblk = S T D / 16.
 * (The abstract of "A JoLT for the KV cache ... Joint Rank-bit Allocation" sets one global
 * byte limit over all groups; this is the byte count each choice is charged.) */
jolt_status jolt_choice_bytes(const jolt_shape* shape, const jolt_options* opts, uint64_t* bytes_host);

/* Whole compress (abstract of "A JoLT for the KV cache ... Joint Rank-bit Allocation": the
 * grouped cache is a fourth-order tensor factored on its token and feature modes; a
 * rotated few-bit quantiser stores the truncation residual; one Lagrangian dual sets the
 * ranks and bit-widths of every group under a single global byte limit).
 *   k_dev, v_dev : input caches (read only), shape/dtype as `shape`
 *   budget_bytes : total blob bytes allowed (headers included)
 *   seed         : seeds the rotation signs and the FlashJoLT sketch
 *   blob_dev     : output, capacity blob_cap >= budget_bytes; layout: 64-byte header,
 *                  64 bytes per unit, then per unit U, W, core, codes, scales (16-B aligned)
 *   ws_dev       : workspace of ws_bytes >= jolt_workspace_size().ws_bytes
 * Asynchronous.  Infeasible budget / non-finite input are reported in the blob header. */
jolt_status jolt_compress(const jolt_shape* shape, const void* k_dev, const void* v_dev, const jolt_options* opts,
                          uint64_t budget_bytes, uint64_t seed, void* blob_dev, size_t blob_cap, void* ws_dev,
                          size_t ws_bytes, void* stream);

/* Stage 1: token and feature factors of every unit (partial Tucker on the token and feature
 * modes; FlashJoLT swaps the exact token-mode SVD for a randomized one, abstract).
 *   u_dev : [n_units][n_tokens][ld_u] fp32, unrounded token factor (leading max r_T columns)
 *   w_dev : [n_units][head_dim][ld_w] fp32, unrounded feature factor (leading max r_D columns)
 *   ld_u >= max r_T and a multiple of 8, ld_w >= max r_D.  Columns ordered by descending singular value, the
 *   entry of largest magnitude of every column positive.  Asynchronous. */
jolt_status jolt_factor(const jolt_shape* shape, const void* k_dev, const void* v_dev, const jolt_options* opts,
                        uint64_t seed, float* u_dev, int64_t ld_u, float* w_dev, int64_t ld_w, void* ws_dev,
                        size_t ws_bytes, void* stream);

/* Stage 2: stored core and distortion table from given bf16 factors.
 *   u_bf16_dev : [n_units][n_tokens][ld_u] bf16 (leading max r_T columns used)
 *   w_bf16_dev : [n_units][head_dim][ld_w] bf16 (leading max r_D columns used)
 *   core_dev   : out [n_units][S][max r_T][max r_D] bf16, C = bf16(U^T bf16(X W)) per slice
 *   table_dev  : out [n_units][n_choices] fp64, || X - decode(encode_c(X)) ||_F^2
 * Asynchronous. */
jolt_status jolt_table(const jolt_shape* shape, const void* k_dev, const void* v_dev, const jolt_options* opts,
                       uint64_t seed, const void* u_bf16_dev, int64_t ld_u, const void* w_bf16_dev, int64_t ld_w,
                       void* core_dev, double* table_dev, void* ws_dev, size_t ws_bytes, void* stream);

/* Stage 2b: the rotated reconstruction operators the table, encoder and decoder use
 * (the residual is rotated before quantisation, introduction of "... Joint Tucker and
 * JL-Residual Allocation for LLMs"; folding the rotation into the operator is this
 * library's form of it):
 *   P'[i_D][u][s] = bf16( (C[u][s][:, :r_D] W[u][:, :r_D]^T) diag(sigma_u) H_D / sqrt(D) )
 *   core_dev   : [n_units][S][max r_T][max r_D] bf16 (as written by jolt_table)
 *   w_bf16_dev : [n_units][head_dim][ld_w] bf16
 *   p_dev      : out [n_feature_ranks][n_units][S][max r_T][head_dim] bf16
 * Asynchronous. */
jolt_status jolt_recon_operator(const jolt_shape* shape, const jolt_options* opts, uint64_t seed,
                                const void* core_dev, const void* w_bf16_dev, int64_t ld_w, void* p_dev, void* ws_dev,
                                size_t ws_bytes, void* stream);

/* Stage 3: the single Lagrangian dual (abstract of "A JoLT for the KV cache ... Joint Rank-bit
 * Allocation"; introduction of "... Joint Tucker and JL-Residual Allocation for LLMs": ranks
 * and bit-widths are set per layer group, for keys and values separately, against one
 * shared byte budget).
 *   dist_dev [n_units][n_choices] fp64, bytes_dev [n_units][n_choices] uint64 (device),
 *   budget_bytes: payload bytes available (headers NOT included here).
 *   choice_dev [n_units] int32 out, lambda_dev [1] fp64 out (+inf when infeasible),
 *   status_dev [1] uint32 out: 0 ok, 4 infeasible.
 * Rule: lambda = 0 if the distortion-minimising choices fit; else lo = 0, hi = 1 doubled
 * until the choices fit, then 200 bisection halvings; answer = choices at hi.  Per unit,
 * argmin D + lambda*B in fp64 (no fused multiply-add), ties to fewer bytes then lower index.
 * Asynchronous; one CTA. */
jolt_status jolt_allocate(const double* dist_dev, const uint64_t* bytes_dev, int32_t n_units, int32_t n_choices,
                          uint64_t budget_bytes, int32_t* choice_dev, double* lambda_dev, uint32_t* status_dev,
                          void* stream);

/* Stage 4: write the blob for given factors, core and choices (choice_dev [n_units] int32,
 * dist_dev [n_units][n_choices] fp64 recorded in the unit headers).  Same factor layouts as
 * jolt_table.  Asynchronous. */
jolt_status jolt_encode(const jolt_shape* shape, const void* k_dev, const void* v_dev, const jolt_options* opts,
                        uint64_t seed, const void* u_bf16_dev, int64_t ld_u, const void* w_bf16_dev, int64_t ld_w,
                        const void* core_dev, const int32_t* choice_dev, const double* dist_dev, void* blob_dev,
                        size_t blob_cap, void* ws_dev, size_t ws_bytes, void* stream);

/* Read and validate a blob's headers (SYNCHRONISES the stream).  records: n_units entries
 * (capacity `cap`).  Returns the device-side status recorded in the header
 * (BUDGET_INFEASIBLE, NUMERIC, OUTPUT_TOO_SMALL) or BAD_BLOB for a corrupt header. */
jolt_status jolt_read_header(const void* blob_dev, jolt_shape* shape_out, uint64_t* total_bytes,
                             jolt_unit_record* records, int32_t cap, void* stream);

/* Decompress: the dense reconstruction from the stored factors (the abstract's decode kernel
 * reads the same factors; this call materialises them):
 * X_hat = (U P' + dequant(codes)) diag(sigma) H_D / sqrt(D) per unit.
 *   out_dtype: JOLT_BF16 or JOLT_F32; k_out_dev, v_out_dev: [n_layers, H, T, D].
 * Reads the headers first (SYNCHRONISES once), then runs asynchronously. */
jolt_status jolt_decompress(const void* blob_dev, int32_t out_dtype, void* k_out_dev, void* v_out_dev, void* ws_dev,
                            size_t ws_bytes, void* stream);

/* Decode-side attention over the stored factors (abstract of "A JoLT for the KV cache ...
 * Joint Rank-bit Allocation": the decode path evaluates attention directly over the stored
 * factors, without forming dense K and V).  One decode step of n_q_heads query heads against
 * every token of one layer: query head j reads KV head j / (n_q_heads / n_heads), scores
 * s_t = k_hat_t . q / sqrt(head_dim) with k_hat the decoder's reconstruction of the stored K,
 * weights p = softmax(s), output p^T v_hat.  Computed as U_K (P'_K q') + rho_hat_K . q' and
 * ((p^T U_V) P'_V + p^T rho_hat_V) Phi_V^T with q' = Phi_K^T q: the stored token factors,
 * codes and scales are read, no dense K or V row is formed.  fp32 arithmetic.
 *
 * jolt_attend_prepare: the aligned token factors and the rotated operators P' of every unit
 *   into ws_dev (the workspace of jolt_decompress, dws_bytes of jolt_workspace_size for the
 *   blob's shape and candidate sets); reads the blob's headers (SYNCHRONISES once).  Call it
 *   once per blob; any number of jolt_attend calls then read the prepared workspace.
 * jolt_attend_scratch_size: bytes of the per-call scratch for n_q_heads query heads when the
 *   stored token ranks are at most max_token_rank.
 * jolt_attend: q_dev [n_q_heads][head_dim] fp32 (read only), out_dev [n_q_heads][head_dim]
 *   fp32; layer in [0, n_layers); n_q_heads a multiple of n_heads with at most 8 query heads
 *   per KV head; stored token ranks at most 1024.  Reads the blob's header (SYNCHRONISES once),
 *   then runs asynchronously.  Errors: INVALID_ARG (layer, heads, null pointers),
 *   WORKSPACE_TOO_SMALL (ws or scratch), BAD_BLOB. */
jolt_status jolt_attend_prepare(const void* blob_dev, void* ws_dev, size_t ws_bytes, void* stream);
jolt_status jolt_attend_scratch_size(const jolt_shape* shape, int32_t max_token_rank, int32_t n_q_heads,
                                     size_t* bytes);
jolt_status jolt_attend(const void* blob_dev, const void* ws_dev, size_t ws_bytes, int32_t layer, const float* q_dev,
                        int32_t n_q_heads, float* out_dev, void* scratch_dev, size_t scratch_bytes, void* stream);

/* Per-block b-bit quantisation of the caches themselves, without factors or rotation: the
 * plain quantisation baseline of the introduction of "A JoLT for the KV Cache ... Joint Tucker
 * and JL-Residual Allocation for LLMs" (JoLT's error is roughly an order of magnitude below it
 * and below cross-layer SVD; the cross-layer SVD baseline is jolt_compress with the feature
 * ranks {head_dim} and the bit-widths {0}).  The quantiser of the residual: 16 consecutive
 * features per block, fp16 lo = round-down(min), step = round-up((max - lo)/(2^b - 1)).
 *   bits: 1..8; sq_dev [n_units][2] fp64 out: ||X_u||^2 and ||X_u - Q(X_u)||^2 (+inf if a
 *   block's scale overflows fp16); codes_dev (2b bytes per block) and scales_dev (fp16 pairs)
 *   optional (both or neither), blocks of unit u after those of units < u, 16-byte aligned;
 *   ws_dev: 148 * 16 bytes per unit.  The stored form takes 2b + 4 bytes per 16 values.
 *   Asynchronous. */
jolt_status jolt_quant_baseline(const jolt_shape* shape, const void* k_dev, const void* v_dev, int32_t bits,
                                void* codes_dev, void* scales_dev, double* sq_dev, void* ws_dev, size_t ws_bytes,
                                void* stream);

/* Per-unit sums of squares (the introduction reports the relative Frobenius error of K and
 * of V separately): sq_dev[2*u] = ||X_u||^2, sq_dev[2*u+1] = ||X_u - Y_u||^2
 * (fp64), X and Y of the same shape; y may be NULL (then only ||X_u||^2).  ydtype is Y's
 * element type.  Asynchronous. */
jolt_status jolt_frobenius(const jolt_shape* shape, const void* k_dev, const void* v_dev, const void* ky_dev,
                           const void* vy_dev, int32_t ydtype, double* sq_dev, void* ws_dev, size_t ws_bytes,
                           void* stream);

/* jolt_frobenius without a workspace argument (the paper has no counterpart: this is a
 * convenience of the library).  For callers that cannot allocate device memory themselves,
 * e.g. a host program whose device memory is entirely owned by another allocator: the
 * partial sums go to a 64 KiB array compiled into the library, which every device that loads
 * the library holds until the process exits.  Same arguments and results as jolt_frobenius.
 *   - at most 64 units (2 * n_layers / layers_per_group <= 64); more returns
 *     JOLT_ERR_WORKSPACE_TOO_SMALL with a message naming the limit;
 *   - the first call on each device looks up the array's device address with that device
 *     current (a one-time set-up); make that first call before any stream capture.  The
 *     looked-up address is kept for the process: after cudaDeviceReset the device's module
 *     is loaded again and the array may move, so do not call this entry point on a device
 *     that has been reset since its first call;
 *   - all calls share the one array: two calls whose GPU work overlaps (different streams or
 *     threads without ordering between them) race on it and may return wrong sums;
 *   - allocates nothing.  Asynchronous. */
jolt_status jolt_frobenius_noalloc(const jolt_shape* shape, const void* k_dev, const void* v_dev, const void* ky_dev,
                                   const void* vy_dev, int32_t ydtype, double* sq_dev, void* stream);

/* CUDA graphs of compress calls (no counterpart on the pages; on by default).  With graphs
 * on, jolt_compress captures its stages once per distinct argument set (shape, options,
 * every pointer and size, budget, seed, device; up to 8 per host thread, least recently used
 * dropped) on a private stream and afterwards replays the captured graph on the caller's
 * stream: the same kernels on the same buffers, with one launch.  The captured graph reads
 * the caller's buffers at replay time, so changing their contents between calls is fine;
 * freeing a buffer and passing a new one at the same address with the same size is also
 * fine.  Calls made while stage timing is on, or on a stream that is itself being
 * captured, run directly.  jolt_set_graphs(0) turns graphs off for this thread and drops
 * its cached graphs. */
void jolt_set_graphs(int32_t enable);

/* Stage timing for measurement (no counterpart on the pages).  jolt_profile_begin starts
 * recording CUDA events around every internal stage launched by this thread (on the call's
 * stream); jolt_profile_end stops, SYNCHRONISES on the recorded events and writes one line
 * per stage, "name total_ms launches units\n", into buf (capacity cap, NUL-terminated).
 * Recording adds two event records per stage and changes no result. */
jolt_status jolt_profile_begin(void);
/* Number of kernels this library has launched in the process so far (its own kernels; work
 * launched inside cuSOLVER is not counted). */
uint64_t jolt_launch_count(void);
jolt_status jolt_profile_end(char* buf, size_t cap);

/* Release this thread's library-owned resources (no counterpart on the pages): the cached
 * CUDA graphs and their capture stream, the auxiliary stream and its events, the cuSOLVER
 * handles and the stage-timing events.  Call it after this thread's library work has
 * finished (for example after synchronising its streams); later calls recreate what they
 * need.  Returns JOLT_ERR_CUDA if a stream could not be destroyed. */
jolt_status jolt_release(void);

/* FP32-pipe rate probe for the roofline of the ALU-bound kernels (no counterpart on the
 * pages; measurement only).  Launches 8 CTAs of 256 threads per SM; every thread runs
 * `iters` rounds of 8 independent fused multiply-add chains, scalar (packed = 0) or on
 * packed pairs (packed != 0, two FMAs per instruction).  *fma_ops receives the number of
 * FMAs the launch performs (each counted as one operation); time the launch with events on
 * `stream`.  sink_dev: 8 * 256 * SMs floats the kernel may write (it never does in
 * practice).  Asynchronous. */
jolt_status jolt_fp32_rate_probe(int32_t packed, int32_t iters, float* sink_dev, uint64_t* fma_ops, void* stream);

/* Self-test of the bounded device wait the tensor-core pipeline uses (no counterpart on the
 * pages; failure-detection check).  One thread initialises an mbarrier for one arrival,
 * arrives on it only if `arrive` != 0, and waits for it with a limit of limit_us
 * microseconds (1 .. 5e6).  With no arrival the wait gives up, the kernel sets the timeout
 * bit in *status_dev and returns normally, and this call returns JOLT_ERR_TIMEOUT; with the
 * arrival it returns JOLT_OK.  status_dev: one uint32 of device memory.  SYNCHRONISES the
 * stream. */
jolt_status jolt_wait_selftest(int32_t arrive, uint32_t limit_us, uint32_t* status_dev, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* JOLT_H_ */
