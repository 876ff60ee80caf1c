/*
 * sol_attn.h -- C ABI of the B200 (sm_100a) Sol-Attn / Sol-Attn2 forward library.
 *
 * Operation (what the entry points compute), from the pages:
 *   "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention Sparsification"
 *   (arXiv 2607.24027): section 3.1 (query-dependent threshold, Eqs. (4)-(5)), section 3.2
 *   (chunk-wise on-the-fly thresholding, proxy-score reuse as approximate correction,
 *   hardware-aligned nested-loop kernel, Fig. 4); the Sol-Attn README (NVlabs/Sana
 *   sparse_backends), "Core API" and "Exact KV sink"; the stable-diffusion.cpp Sol-Attn
 *   documentation (adjacent blocks remain exact, K means and V sums); and
 *   "Sol-Attn2: Sparse Attention with Complementary Approximation", Method, "Routing and
 *   complementary approximation".
 *
 * Common conventions for every entry point
 *   - q, k, v, out: DEVICE pointers to contiguous BF16 tensors in BTHD layout [B, N, H, 128]:
 *     element (b, t, h, c) sits at ((b*N + t)*H + h)*128 + c.  Head dimension is fixed at 128,
 *     attention is non-causal and unmasked, Q/K/V share N and H (self-attention).  Pointers must
 *     be 16-byte aligned; `out` must not overlap q, k or v.  The caller owns all four buffers.
 *   - Blocks: 64-token key/query blocks, Nb = ceil(N / 64); the last block may be partial.
 *   - tau: the threshold coefficient beta of tau_i = mu_i + beta * sigma_i (higher selects fewer
 *     blocks).  Must be finite; 0 does not mean dense.
 *   - Sink: sink_tokens <= 0 means no sink.  sink_start >= 0 makes [sink_start,
 *     sink_start + sink_tokens) exact (clipped to N); sink_start < 0 makes the suffix
 *     [N - sink_tokens, N) exact.  sink_start >= N is an error.  Every key block overlapping the
 *     range is exact for every query.
 *   - stream: a cudaStream_t passed as void*.  NULL is the legacy default stream.  All work is
 *     enqueued on it; the call returns after enqueueing (no host synchronisation), except that a
 *     call may synchronise the device once to grow the library's workspace.
 *   - Workspace: the library owns a per-device workspace that grows on demand and is reused.
 *     Calls on different streams of the same device are ordered by the library (each call waits
 *     for the previous one through an event), so they never race on the workspace.
 *   - Return value: SOL_OK (0) or a negative sol_status.  Argument errors are detected on the host
 *     before anything is launched.  sol_attn_last_error() gives a message for the calling thread.
 *   - Device-side faults never trap: every wait inside a kernel is bounded (about one second)
 *     and a wait that runs out records SOL_ERR_TIMEOUT in a device status word that
 *     sol_attn_get_device_status() reads.
 */
#ifndef SOL_ATTN_H_
#define SOL_ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SOL_OK = 0,
  SOL_ERR_NULL = -1,    /* a required pointer is NULL */
  SOL_ERR_SHAPE = -2,   /* B, N or H <= 0, or sizes overflow the supported range */
  SOL_ERR_TAU = -3,     /* tau is not finite */
  SOL_ERR_SINK = -4,    /* sink_start >= N */
  SOL_ERR_ALIGN = -5,   /* a tensor pointer is not 16-byte aligned, or out overlaps an input */
  SOL_ERR_ALLOC = -6,   /* workspace allocation failed */
  SOL_ERR_LAUNCH = -7,  /* a CUDA launch or runtime call failed */
  SOL_ERR_DEVICE = -8,  /* no usable sm_100 device */
  SOL_ERR_TIMEOUT = -9, /* a bounded wait inside a kernel ran out (see sol_attn_get_device_status) */
  SOL_ERR_OPTION = -10  /* an option value is out of range or a reserved field is nonzero */
} sol_status;

/* Threshold estimators ("Sol-Attn" paper: Eq. (5) and appendix "Diagonal threshold estimator"). */
typedef enum {
  SOL_THRESH_EXACT = 0, /* full-covariance sigma_i (the Sol-Attn README default, thresh_type="exact") */
  SOL_THRESH_DIAG = 1   /* sigma_i^2 = (Qbar_i * Qbar_i) . v_K with v_K the per-channel variance of Kbar */
} sol_thresh_type;

#define SOL_MAX_EXTRA_SINKS 4
#define SOL_MAX_KV_SPLITS 8

/* Arithmetic of the attention products (sol_attn_options.precision). */
typedef enum {
  SOL_PRECISION_BF16 = 0, /* BF16 operands, FP32 accumulation and exponentials (the default) */
  SOL_PRECISION_FP8 = 1   /* E4M3 operands and ExpCast weights, as sol_attn_fwd_fp8 / sol_attn2_fwd_fp8 */
} sol_precision;

/*
 * Options of the _ex entry points.  A NULL pointer means all defaults (an all-zero struct is the
 * default too); reserved fields must be 0.
 *   thresh_type        sol_thresh_type.
 *   n_extra_sinks      0 .. SOL_MAX_EXTRA_SINKS further exact key ranges, in addition to the
 *                      sink_start / sink_tokens range (for inputs with several text segments, e.g.
 *                      joint attention over interleaved text and video tokens).  Range e covers
 *                      tokens [extra_sink_start[e], extra_sink_start[e] + extra_sink_tokens[e]),
 *                      clipped to N; it needs 0 <= start < N and tokens > 0.  Like the main sink,
 *                      every key block overlapping a range is exact for every query.
 *   kv_splits          0 or 1: one CTA per 128-row query tile.  2 .. SOL_MAX_KV_SPLITS: split-KV
 *                      (the Sol-Attn README's kv_splits, "Long-sequence tuning on H100"): each
 *                      query tile's key tiles are divided into kv_splits contiguous shares, one CTA
 *                      each, and a combine kernel merges the partial softmax states exactly
 *                      (o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s).  Results equal the
 *                      unsplit call up to FP32 rounding.  Raises parallelism when there are few
 *                      query tiles; the workspace grows by kv_splits * B*H*ceil(N/128)*128 * 520
 *                      bytes.  Sol-Attn only: sol_attn2_fwd_ex rejects kv_splits > 1.
 *   precision          sol_precision.  SOL_PRECISION_FP8 makes sol_attn_fwd_ex, sol_attn2_fwd_ex and
 *                      sol_attn_fwd_varlen run the FP8 path of sol_attn_fwd_fp8 / sol_attn2_fwd_fp8;
 *                      it cannot be combined with kv_splits > 1.  The routing (and so
 *                      sol_attn_debug_route_ex) is the same for both.
 *   m_tile             query rows per work unit of the fused kernel: 0 or 128 (default), two
 *                      adjacent 64-token query blocks per unit, which walk the union of their exact
 *                      sets (a key block exact for only one of them is computed for both rows and
 *                      masked for the other: the union-tile waste); 64, one query block per unit,
 *                      which walks only its own exact set (no union waste) at the same tensor cost
 *                      per tile as two blocks, so it pays only where the union waste exceeds one
 *                      half (the tensor-core tile stays M = 128; its second half is idle).  The
 *                      Sol-Attn README's per-shape tuning knobs ("Long-sequence tuning on H100")
 *                      motivate it.  Results equal the default up to FP32 rounding.  BF16 path
 *                      only: an FP8 precision with m_tile 64 returns SOL_ERR_OPTION.
 */
typedef struct {
  int thresh_type;
  int n_extra_sinks;
  int extra_sink_start[SOL_MAX_EXTRA_SINKS];
  int extra_sink_tokens[SOL_MAX_EXTRA_SINKS];
  int kv_splits;
  int precision;
  int m_tile;
  int reserved[3];
} sol_attn_options;

/*
 * Sol-Attn forward (arXiv 2607.24027, sections 3.1-3.2).  For each (b, h) and 64-token query
 * block i: block means Qbar_i, Kbar_j; proxies s_ij = Qbar_i . Kbar_j / sqrt(128); threshold
 * tau_i = mu_i + tau * sigma_i with mu_i, sigma_i the mean and standard deviation of row i of the
 * proxy map (full covariance form, Eq. (5)); key block j is exact iff s_ij > tau_i, |i - j| <= 1,
 * or j overlaps the sink.  Each query token attends exactly to the tokens of its exact blocks and
 * approximately to every other block through the surrogate (logit q.Kbar_j / sqrt(128), mass
 * n_j, value sum Vhat_j); both share one softmax normaliser.  Result rounded to BF16 in `out`.
 */
int sol_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                 int sink_start, int sink_tokens, void* stream);

/*
 * Sol-Attn2 complementary-tail forward ("Sol-Attn2", Method, "Routing and complementary
 * approximation").  Same exact sets E_i as sol_attn_fwd.  Each key block is split into two groups
 * by its keys' projection on the mean-query direction u (the mean of all queries of the (b, h)):
 * group 1 holds keys with k.u above the block mean's projection.  For each 32-token anchor a with
 * mean query qbar_a, over the groups of the blocks outside E of its query block:
 * w_ag = n_g exp(qbar_a . kbar_g / sqrt(128)), Z_a = sum w, (mu_a, nu_a) = sum w (kbar_g, vbar_g) / Z_a.
 * Query i of the anchor gets Zhat_i = Z_a exp((q_i - qbar_a) . mu_a / sqrt(128)) and
 * o_i = (sum_{E_i} e^{z} v + Zhat_i nu_a) / (sum_{E_i} e^{z} + Zhat_i).  Same arguments as
 * sol_attn_fwd.
 */
int sol_attn2_fwd(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                  int sink_start, int sink_tokens, void* stream);

/*
 * sol_attn_fwd / sol_attn2_fwd / sol_attn_debug_route with options (`opts` may be NULL).  With
 * SOL_THRESH_DIAG the threshold's variance keeps only the diagonal of the key-block-mean covariance
 * (the mean mu_i stays exact); extra sink ranges add exact key blocks as described at
 * sol_attn_options; everything else is as in the plain entry points.  An invalid option returns
 * SOL_ERR_OPTION before anything is launched.
 */
int sol_attn_fwd_ex(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                    int sink_start, int sink_tokens, const sol_attn_options* opts, void* stream);
int sol_attn2_fwd_ex(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                     int sink_start, int sink_tokens, const sol_attn_options* opts, void* stream);
int sol_attn_debug_route_ex(const void* q, const void* k, int B, int N, int H, float tau, int sink_start,
                            int sink_tokens, const sol_attn_options* opts, unsigned char* mask, float* thresh,
                            void* stream);

/* Message for the last error returned on the calling thread ("" if none).  Owned by the library. */
const char* sol_attn_last_error(void);

/*
 * Synchronises `stream`, then reads and clears this device's status word.  Returns SOL_OK, or
 * SOL_ERR_TIMEOUT if a bounded wait inside a kernel ran out since the last read, or
 * SOL_ERR_LAUNCH if the synchronisation itself failed, a kernel found its shared-memory window
 * misaligned (it then returned without running), or a bounds check of the debug build
 * (libsolattn_debug.so) failed and the access was skipped.
 */
int sol_attn_get_device_status(void* stream);

/*
 * Routing only (test and bench introspection): runs the block-summary, threshold and routing
 * kernels of sol_attn_fwd and expands the exact-block bitmask.
 *   mask   : DEVICE uint8 [B, H, Nb, Nb], 1 where key block j is exact for query block i.
 *   thresh : DEVICE float [B, H, Nb] thresholds tau_i, or NULL.
 * Same argument rules as sol_attn_fwd; q and k only.
 */
int sol_attn_debug_route(const void* q, const void* k, int B, int N, int H, float tau, int sink_start,
                         int sink_tokens, unsigned char* mask, float* thresh, void* stream);

/*
 * Realised routing statistics of the most recent sol_attn_fwd / sol_attn2_fwd /
 * sol_attn_debug_route on this device: number of exact (query-block, key-block) pairs, number of
 * pairs in total, and the smallest and largest number of exact blocks in one query-block row.
 * Synchronises the stream of that call.  Any output pointer may be NULL.
 */
int sol_attn_last_stats(long long* exact_pairs, long long* total_pairs, int* min_row, int* max_row);

/*
 * Kernel timing for measurement: when enabled (nonzero), each forward call records a pair of CUDA
 * events on its stream around the fused attention kernel (and, with kv_splits > 1, the combine
 * kernel that follows it), in a ring of 256 pairs per device that
 * enabling resets.  sol_attn_last_kernel_ms() synchronises on the most recent closing event and
 * returns that launch's duration in milliseconds; sol_attn_kernel_ms_sum(n) returns the summed
 * duration of the last n timed launches (n <= 256).  Both return a negative value if unavailable.
 */
int sol_attn_set_kernel_timing(int enable);
float sol_attn_last_kernel_ms(void);
float sol_attn_kernel_ms_sum(int n);

/*
 * Per-CTA timing of the fused attention kernel (measurement only; the pages have no counterpart).
 * With sol_attn_set_unit_timing(1), every later BF16 forward call records, for each CTA (work unit:
 * one 128-row query tile, or one split-KV share of it) of its fused launch, the %globaltimer value
 * at its start and at its end (nanoseconds) and the SM it ran on.  sol_attn_last_unit_times
 * synchronises the last call's stream and copies min(max_units, CTAs) records of three unsigned
 * 64-bit values (start, end, SM id), in CTA order, to the HOST array `host`; *units receives the
 * CTA count.  The first enabled call allocates a device buffer (library-owned, kept until the
 * process exits).  Off by default; costs two stores per CTA when on.  The FP8 entry points do not
 * record.  Errors: SOL_ERR_NULL for NULL pointers, SOL_ERR_LAUNCH when no timed
 * launch ran.
 */
int sol_attn_set_unit_timing(int enable);
int sol_attn_last_unit_times(unsigned long long* host, int max_units, int* units);

/* Number of kernels the most recent forward call launched. */
int sol_attn_last_launch_count(void);

/* Frees this process's workspaces on every device (synchronises each device first). */
void sol_attn_release_workspace(void);

/*
 * Allocation-free variant of sol_attn_fwd (the pages have no counterpart: this serves callers that
 * cannot allocate device memory during the call, e.g. code running inside a memory pool that
 * forbids outside allocations or a runtime that reserved all device memory up front).
 *   - Same arguments, layout, results and argument errors as sol_attn_fwd.
 *   - Its scratch is a fixed 64 MiB region declared at file scope in the library (plus two small
 *     status / statistics words); every GPU that loads the library holds it until the process
 *     exits.  The call never calls cudaMalloc / cudaFree or any allocating routine.  A shape whose
 *     scratch exceeds 64 MiB (for example B*H = 32 at N > ~38K tokens) returns SOL_ERR_SHAPE with a
 *     message; use sol_attn_fwd for those.
 *   - The first call on a device (with that device current) looks up the scratch region's device
 *     address.  Under CUDA's default lazy module loading that lookup is also when the driver
 *     loads this part of the library on the device and reserves the 64 MiB, so make that first
 *     call (or sol_attn_noalloc_get_device_status) early: before reserving the rest of the
 *     device's memory and before any stream capture on the device.
 *   - All calls share the one region: calls that overlap on the GPU (different streams, or several
 *     host threads) race and must be serialised by the caller.  The region keeps the last call's
 *     contents; everything a call needs zeroed it clears itself.
 *   - Device-side failures (a bounded wait that ran out) are reported by
 *     sol_attn_noalloc_get_device_status, not by sol_attn_get_device_status; sol_attn_last_stats
 *     and kernel timing report the pooled-workspace entry points only.
 */
int sol_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                         int sink_start, int sink_tokens, void* stream);

/*
 * Status of the allocation-free calls on the current device (the pages have no counterpart).
 * Synchronises `stream`, then reads and clears the status word that sol_attn_fwd_noalloc's kernels
 * write: SOL_OK, SOL_ERR_TIMEOUT (a bounded wait inside a kernel ran out: that call's `out` is not
 * valid) or SOL_ERR_LAUNCH (a kernel found its shared memory misaligned and did not run).  Reads
 * four bytes into a host variable and clears them with cudaMemset: it allocates nothing.
 */
int sol_attn_noalloc_get_device_status(void* stream);

/*
 * Variable-length batch (packed sequences, as the pages' integrations pass them): sequence s holds
 * the tokens [cu_seqlens[s], cu_seqlens[s + 1]) of the packed tensors q, k, v, out, each laid out
 * [total_tokens, H, 128] (BTHD with B = 1 per sequence).  Every sequence is an independent
 * sol_attn_fwd_ex call on its own tokens (its own blocks, thresholds and routing; the sink range
 * and extra sinks are relative to each sequence's first token), issued in order on `stream`.
 *   cu_seqlens : HOST int array of nseq + 1 non-decreasing offsets, cu_seqlens[0] = 0; empty
 *                sequences are skipped.  Pointers and options follow sol_attn_fwd_ex.
 *   Errors: SOL_ERR_NULL / SOL_ERR_SHAPE for a bad cu_seqlens, SOL_ERR_SINK when sink_start is not
 *   inside every non-empty sequence; otherwise the first failing sequence's status (earlier
 *   sequences are already enqueued).  sol_attn_last_stats then reports the last sequence.
 */
int sol_attn_fwd_varlen(const void* q, const void* k, const void* v, void* out, const int* cu_seqlens, int nseq,
                        int H, float tau, int sink_start, int sink_tokens, const sol_attn_options* opts, void* stream);

/*
 * Dense companion call for text query rows in joint (MMDiT) attention.  The Sol-Attn README,
 * "Exact KV sink": a sink keeps the text KEY blocks exact for every query but does not make the
 * text QUERY rows dense; an integration should use dense attention for the valid text queries and
 * Sol-Attn for the image/video queries.  This entry point computes exact softmax attention of the
 * query tokens [q_start, q_start + q_tokens) (clipped to N) over all N keys,
 * o_r = sum_t exp(q_r.k_t / sqrt(128)) v_t / sum_t exp(q_r.k_t / sqrt(128)), rounded to BF16, and
 * writes only those rows of `out`; every other row of `out` is left as it was.  Call it after
 * sol_attn_fwd / sol_attn2_fwd on the same `out` to give the text rows dense attention.
 *   - q_start < 0 means the suffix [N - q_tokens, N); q_tokens <= 0 is a no-op (SOL_OK).
 *   - q_start >= N (with q_tokens > 0) returns SOL_ERR_SINK; the other argument rules are those
 *     of sol_attn_fwd (tau and the sink do not apply).
 */
int sol_attn_dense_rows(const void* q, const void* k, const void* v, void* out, int B, int N, int H, int q_start,
                        int q_tokens, void* stream);

/*
 * Caps the workspace the library may hold on each device at `bytes` (0 removes the cap; applies to
 * later calls).  A call that would need more returns SOL_ERR_ALLOC with a message and launches
 * nothing; an existing larger workspace is kept until sol_attn_release_workspace().  No counterpart
 * on the pages: it bounds the library's memory next to other users of the GPU and makes the
 * allocation-failure path testable.
 */
void sol_attn_set_workspace_limit(size_t bytes);

/*
 * Self-test of the device-side failure path (no counterpart on the pages; for tests and health
 * checks).  Enqueues on `stream` one tiny kernel whose single bounded wait can never be satisfied,
 * so it runs out after about one second and records a timeout in the device status word, as a
 * stalled pipeline stage in the attention kernels would.  Nothing traps or faults; the next
 * sol_attn_get_device_status(stream) returns SOL_ERR_TIMEOUT (and clears the word), after which
 * the library works as before.  Returns SOL_OK once enqueued, or SOL_ERR_DEVICE without a usable
 * device.
 */
int sol_attn_selftest_wait_timeout(void* stream);

/*
 * Host-buffer entry points (the Sol-Attn README's sol_attn call takes and returns tensors; these
 * take them in host memory).  q, k, v and out are HOST pointers to [B, N, H, 128] BF16 arrays (BTHD,
 * contiguous; no alignment needed); the computation is sol_attn_fwd_ex / sol_attn2_fwd_ex (`opts`
 * may be NULL) and the call blocks until `out` holds the result.
 *   - Heads are independent problems, so the call splits the work into (b, head-chunk) slices of
 *     heads_per_chunk heads (0: ceil(H / 16)) and pipelines them on three internal streams of the
 *     current device: the strided copy of slice c + 1 into device memory, the attention of slice c
 *     and the copy of slice c - 1 back to the host overlap.  Overlap needs page-locked host memory
 *     (cudaHostAlloc / cudaHostRegister); pageable buffers give the same result without it.
 *   - Each slice is a separate call (its own routing, launches and statistics): the result equals
 *     sol_attn_fwd_ex on device copies of the tensors bit for bit.
 *   - The library keeps two sets of device staging buffers (4 x N x heads_per_chunk x 256 bytes
 *     each) besides its workspace, until sol_attn_release_workspace.  Calls are serialised.
 *   - Errors: SOL_ERR_NULL / SOL_ERR_SHAPE for bad arguments, SOL_ERR_ALLOC when staging buffers
 *     cannot be allocated, SOL_ERR_LAUNCH when a copy fails, otherwise the first failing slice's
 *     status (nothing is left in flight).
 */
int sol_attn_fwd_host(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                      int sink_start, int sink_tokens, const sol_attn_options* opts, int heads_per_chunk);
int sol_attn2_fwd_host(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                       int sink_start, int sink_tokens, const sol_attn_options* opts, int heads_per_chunk);

/*
 * FP8 (E4M3) + ExpCast forward ("Sol-Attn2" draft, section "FP8 quantization and ExpCast").  Same
 * arguments, routing and exact sets as sol_attn_fwd_ex / sol_attn2_fwd_ex (BF16 inputs and output;
 * the routing is computed from the BF16 inputs exactly as there).  The attention products then run
 * on E4M3 operands with FP32 accumulation:
 *   - Q and K are quantised with one scale per (b, h, 64-token block), V with one per (b, h):
 *     s = max |X| / 448 (1 for an all-zero block), X8 = E4M3(X / s), round to nearest even,
 *     saturating.  sol_attn_fwd_fp8's surrogate keys Kbar_j take one scale per 64 consecutive key
 *     blocks of a (b, h), its value means Vbar_j = Vhat_j / n_j the head's V scale; a surrogate
 *     block's logit is q8 . Kbar8_j / sqrt(128) + ln n_j.
 *   - Every softmax weight is an ExpCast byte: with u the base-2 score minus the row's pivot,
 *     c(u) = clip_[0,120](RNE(8u + 55.65)), weight decode_E4M3(c) ~= 2^u (within 7.5 %).  The pivot is
 *     an integer that moves only when the running maximum exceeds it by more than 8, to
 *     ceil(max) - 8.  The same decoded weights enter the P V product and the denominator.
 *   - sol_attn2_fwd_fp8: the exact branch as above; the complementary tail (Z_a, mu_a, nu_a) as in
 *     sol_attn2_fwd from the BF16 inputs, with delta_i taken from the dequantised query, merged
 *     into the denominator with its exact exponential.
 * Results differ from the BF16 entry points by the E4M3 and ExpCast roundings (about 5 % relative
 * L2 on unit-variance inputs).  kv_splits > 1 returns SOL_ERR_OPTION.  The workspace grows by
 * 3 * B*N*H*128 bytes (E4M3 copies of Q, K, V) plus the compressed operands and scales.
 * Kernel timing (sol_attn_set_kernel_timing) covers the fused kernel only; the quantisation
 * kernels run before it, after the routing.
 */
int sol_attn_fwd_fp8(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                     int sink_start, int sink_tokens, const sol_attn_options* opts, void* stream);
int sol_attn2_fwd_fp8(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                      int sink_start, int sink_tokens, const sol_attn_options* opts, void* stream);

/*
 * Host evaluation of the FP8 kernels' ExpCast encoder (the same inline function the softmax runs;
 * for checking it against a reference without a GPU).  For n scores x (HOST floats, n a multiple
 * of 4), base-2 multiplier fs > 0 and integer pivot: code_i = the E4M3 byte of
 * u_i = x_i * fs - pivot computed as max(fma(x_i, 8 fs, 55.65 - 8 pivot), 0) rounded to the nearest
 * integer (ties to even); words[i / 4] holds codes i .. i + 3, the first in the low byte (the
 * layout of a P operand column in tensor memory).  The clip at 120 is the caller's invariant
 * u <= 8 (the kernels' pivot rule keeps it).  Returns SOL_ERR_NULL, SOL_ERR_SHAPE (n) or
 * SOL_ERR_OPTION (fs, pivot) without writing.
 */
int sol_attn_expcast_host(const float* x, int n, float fs, float pivot, unsigned int* words);

/*
 * Host evaluation of the FP8 quantisers' scaled value X / s, s = m / 448 ([Sol2] "FP8 quantization
 * and ExpCast": scale = max |X| / 448 of the block or head), as the GPU computes it before the
 * E4M3 rounding (the same inline function; for checking it without a GPU).  The kernels evaluate
 * RN(RN(x * 448) / m) without a division per element (a reciprocal per block and one FMA
 * correction step); this entry point lets a test compare that against the IEEE division.  For n
 * HOST floats x and 0 < m < inf, q_i = the kernels' value for x_i.  Returns SOL_ERR_NULL,
 * SOL_ERR_SHAPE (n < 0) or SOL_ERR_OPTION (m) without writing.
 */
int sol_attn_quot448_host(const float* x, int n, float m, float* q);

#ifdef __cplusplus
}
#endif

#endif /* SOL_ATTN_H_ */
