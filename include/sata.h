/*
 * sata.h - C ABI of libsata: causal symmetry-aware Taylor (SATA) attention on
 * NVIDIA B200 (sm_100a).
 *
 * The method (sources cited by page title and section):
 *   [CC-TAYLOR] "Self-attention at constant cost per token via symmetry-aware
 *               Taylor approximation" (blog.hotdry.top, 2026-02-05)
 *   [CC-HW]     "Constant-cost attention: hardware optimization" (same blog)
 *
 *   exp(q.k / c) ~= sum_{p=0}^{P-1} alpha_p <phi_p(q), phi_p(k)>_{C_p},
 *   alpha_p = 1 / (p! c^p),  c = sqrt(d_K)          ([CC-TAYLOR] "The Taylor
 *                                                     approximation", "Feature
 *                                                     maps and linear attention")
 *   phi_p(x)[r] = prod_m x[M_p[r][m]] over the nondecreasing index tuples M_p,
 *   C_p[r] = number of times tuple r's monomial occurs in (q.k)^p.
 *   Z_p = sum_t phi_p(k_t),  S_p = sum_t phi_p(k_t) v_t^T            (states)
 *   y_T = sum_p alpha_p phi_p(q_T)^T C_p S_p / sum_p alpha_p <phi_p(q_T), Z_p>_C
 *                                            ([CC-TAYLOR] "Feature maps and
 *                                             linear attention")
 *
 * Conventions shared by every entry point:
 *   - P is the number of Taylor terms (degrees 0..P-1).  F = binom(d_K+P-1, P-1)
 *     features per head, concatenated p = 0..P-1, lexicographic within a degree.
 *   - The causal range is inclusive: token t's output sees tokens 0..t; a decode
 *     step adds (k, v) to the state before reading it.
 *   - Attention inputs q, k, v are bf16, row-major [B][H][N][d] (prefill) or
 *     [B][H][d] (decode); outputs are fp32 [B][H][N][d_V] / [B][H][d_V].
 *   - The state is fp32, unweighted (alpha_p and C_p are applied on the query
 *     side): S [B][H][F][d_V], Z [B][H][F], features in the order above.
 *   - All device pointers must be 16-byte aligned.  Buffers are owned by the
 *     caller; the library owns only its cached basis tables and internal
 *     workspaces (freed by sata_shutdown).
 *   - Every call returns SATA_OK (0) or a negative status; none throws.  Work is
 *     enqueued asynchronously on a CUDA stream; argument checks happen before any
 *     launch.  Launch failures return SATA_ECUDA (sata_last_cuda_error() gives
 *     the cudaError_t).  Device-side conditions (a bounded wait that gave up, an
 *     input outside the prefill's operand range) set a per-device flag that
 *     sata_sync_status() reports.
 *   - Supported: 1 <= d_K <= 128, d_V in {4, 8, 16, 32, 64, 128}, 1 <= P <= 8
 *     (P is a tunable hyperparameter: [CC-TAYLOR] "Precision and efficiency
 *     trade-off" (精度与效率的权衡); [CC-HW] "Taylor-expansion trade-off between
 *     precision and efficiency" (精度与效率的泰勒展开权衡) weighs P = 8).  The
 *     tensor-core prefill serves P <= 4 with (d_K, d_V) one of (16|32, 16|32|64),
 *     (64, 16|32|64|128) and (128, 64|128); every other supported shape runs on
 *     the CUDA-core prefill (fp32).  sata_decode_step_static takes P <= 4.  Other
 *     values return SATA_EUNSUPPORTED.  There is no CPU fallback.
 *   - The tensor-core prefill scales each head's rows by powers of two before its
 *     fp16 operands are formed (exact), so every finite bf16 input is in range;
 *     only a non-finite input, or an output beyond the fp32 range, sets the
 *     range flag (SATA_ERANGE at the next sata_sync_status).
 *   - The library-owned workspaces are shared by all calls on a device: calls
 *     that may overlap on different streams must pass their own workspace
 *     (sata_prefill_ex) or be ordered by the caller.  That includes calls made
 *     from different host threads: the library serialises the sizing and
 *     allocation of a workspace, not the kernels that use it.
 *   - The first call for a given (device, d_K, P) uploads the basis tables with
 *     synchronous copies; make it before capturing a CUDA graph.
 */
#ifndef SATA_H
#define SATA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SATA_API __attribute__((visibility("default")))
#else
#define SATA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum sata_status {
    SATA_OK = 0,
    SATA_EINVAL = -1,        /* invalid argument (null, negative size, state mismatch) */
    SATA_EUNSUPPORTED = -2,  /* valid, but d_K / d_V / P outside the supported set */
    SATA_ECUDA = -3,         /* CUDA runtime or launch error; see sata_last_cuda_error() */
    SATA_ETIMEOUT = -4,      /* a bounded device-side wait expired (reported at sync) */
    SATA_ENOMEM = -5,        /* internal workspace allocation failed, or too small */
    SATA_ERANGE = -6,        /* tensor-core prefill: a non-finite input or output (at sync) */
    SATA_EALIGN = -7         /* a device pointer is not 16-byte aligned */
};

/* Per-sequence recurrent state: caller-allocated struct and device buffers. */
typedef struct sata_state {
    int32_t B, H, d_K, d_V, P;
    int64_t F;        /* features per head */
    float *S;         /* device [B][H][F][d_V] fp32 */
    float *Z;         /* device [B][H][F] fp32 */
    void *stream;     /* cudaStream_t used by sata_decode_step (NULL: legacy stream) */
    int64_t tokens;   /* tokens absorbed so far (prefill + decode) */
} sata_state;

/* Human-readable name of a status code (static string). */
SATA_API const char *sata_status_string(int status);
/* cudaError_t of the last failed CUDA call made by this library on this thread. */
SATA_API int sata_last_cuda_error(void);
/* Library version: major * 10000 + minor * 100 + patch. */
SATA_API int sata_version(void);

/* F = binom(d_K+P-1, P-1): number of features of the truncated basis
 * ([CC-TAYLOR] "Hidden-state size and FLOPs").  Host only. */
SATA_API int sata_num_features(int d_K, int P, int64_t *F_out);

/*
 * Minimal symmetric basis ([CC-TAYLOR] "The Taylor approximation": keep one
 * representative of each monomial, the upper-triangular / nondecreasing index
 * tuples, binom(d_K+p-1, p) of them; "Feature maps and linear attention": C_p
 * counts each monomial's occurrences; [CC-HW] "Compute density":
 * phi = x[..., M].prod(-1)).  Host only, deterministic, bit-exact.
 *   M       [F][max(P-1,1)] uint8: row r holds the p indices of feature r
 *           (nondecreasing) followed by 0xFF padding; NULL to skip.
 *   C       [F] uint32 multiplicities p!/prod(mult!); NULL to skip.
 *   offsets [P+1]: first feature of degree p, offsets[P] = F; NULL to skip.
 *   F_out   receives F; NULL to skip.  All NULL: size query.
 * Requires d_K <= 255 (indices fit a byte).
 */
SATA_API int sata_build_basis(int d_K, int P, uint8_t *M, uint32_t *C, int64_t *offsets, int64_t *F_out);

/* Stream used by sata_prefill (the plain form); default: the legacy stream.
 * Process-wide; set it before launching from another stream. */
SATA_API int sata_set_stream(void *stream);

/* Synchronise `stream` and report device-side conditions raised since the last
 * call on this device: SATA_ETIMEOUT, SATA_ERANGE, or SATA_OK.  Clears them. */
SATA_API int sata_sync_status(void *stream);

/* Free the library's cached device tables and workspaces on every device. */
SATA_API void sata_shutdown(void);

/* Bytes of S and Z for a state of this shape ([CC-TAYLOR] "Hidden-state size
 * and FLOPs": (d_V + 1) binom(d_K+P-1, P-1) values per head). */
SATA_API int sata_state_bytes(int B, int H, int d_K, int d_V, int P, size_t *S_bytes, size_t *Z_bytes);

/* Fill *st for caller-owned device buffers S, Z (sizes from sata_state_bytes)
 * and zero them on `stream`: the empty context, Z_0 = 0 and S_0 = 0, from which
 * the recurrence of [CC-TAYLOR] "Feature maps and linear attention"
 * (特征映射与线性注意力) accumulates phi(k_t) and phi(k_t) v_t^T.  tokens = 0. */
SATA_API int sata_state_init(sata_state *st, int B, int H, int d_K, int d_V, int P,
                    float *S, float *Z, void *stream);

/*
 * Absorb another token segment's state into st: st->S += S, st->Z += Z
 * (elementwise), st->tokens += tokens, on st->stream.  S and Z are device
 * buffers of st's shape ([B][H][F][d_V] and [B][H][F] fp32), e.g. the state a
 * prefill of the segment left in a fresh sata_state.  The states are sums over
 * tokens, so the state after a concatenation of segments is the sum of the
 * segments' states ([CC-TAYLOR] "Feature maps and linear attention": the
 * recurrence may be evaluated as a parallel prefix scan).  This is the
 * combining step of a prefill split by sequence across GPUs: after an
 * all-gather of the segment states, each rank adds those of the segments
 * before its own, then prefills its segment from the sum.
 * Errors: SATA_EINVAL (null, negative tokens, st inconsistent), SATA_EALIGN.
 */
SATA_API int sata_state_accumulate(sata_state *st, const float *S, const float *Z, int64_t tokens);

/* Workspace bytes sata_prefill_ex needs for this shape: the larger of the
 * fresh-state and carried-state needs, so one size serves calls with or
 * without a sata_state (under the options in force at the query). */
SATA_API int sata_workspace_bytes(int B, int H, int64_t N, int d_K, int d_V, int P, size_t *bytes);

/*
 * Causal SATA prefill over N tokens of B*H independent heads, fresh (zero)
 * state, on the stream set by sata_set_stream, library-owned workspace.
 *   q, k: bf16 [B][H][N][d_K];  v: bf16 [B][H][N][d_V];  out: fp32 [B][H][N][d_V].
 * Output y_t for every token: the chunked form of the state recurrence
 * ([CC-TAYLOR] "Feature maps and linear attention": the recurrence may be
 * evaluated sequentially or as a parallel prefix scan).  N = 0 is a no-op.
 */
SATA_API int sata_prefill(const void *q, const void *k, const void *v, float *out,
                 int B, int H, int64_t N, int d_K, int d_V, int P);

/*
 * As sata_prefill, with explicit state, workspace and stream.
 *   st:        NULL (fresh state, final state discarded) or a state of the same
 *              (B, H, d_K, d_V, P): the prefill continues from it and leaves the
 *              final state there; st->tokens += N.
 *   workspace: NULL (library-owned) or a device buffer of ws_bytes >=
 *              sata_workspace_bytes(...), used only while the enqueued work runs.
 *   stream:    cudaStream_t (NULL: legacy stream).
 */
SATA_API int sata_prefill_ex(const void *q, const void *k, const void *v, float *out,
                    int B, int H, int64_t N, int d_K, int d_V, int P,
                    sata_state *st, void *workspace, size_t ws_bytes, void *stream);

/*
 * As sata_prefill_ex with fp32 q, k, v (same layouts) and a library-owned
 * workspace: the inputs are used as given, with no rounding to bf16.  Runs on
 * the CUDA-core prefill (fp32 arithmetic throughout) for every supported shape,
 * the same chunked form of the recurrence ([CC-TAYLOR] "Feature maps and linear
 * attention").  For inputs that are specified in fp32 (the tiny d = 8 case);
 * bf16 inputs should use sata_prefill_ex, whose tensor-core path is much faster.
 *   q, k, v, out: device pointers, 16-byte aligned, owned by the caller.
 *   st, stream:   as in sata_prefill_ex.
 * Errors as sata_prefill_ex.
 */
SATA_API int sata_prefill_f32(const float *q, const float *k, const float *v, float *out,
                    int B, int H, int64_t N, int d_K, int d_V, int P,
                    sata_state *st, void *stream);

/*
 * As sata_prefill_ex, with q, k, v and out in HOST memory (same layouts and
 * dtypes) and a library-owned workspace.  The same computation as
 * sata_prefill_ex, so the output is the same; the difference is the transfers:
 * the call copies the inputs to the device in token segments (at least four
 * for the tensor-core path) on a library copy stream, starts each segment as
 * soon as its rows have landed, and copies each segment's output back on a
 * second copy stream while later segments compute.  Everything is enqueued
 * behind the work already on `stream`, and `stream` completes only after the
 * last output row is in host memory.
 *   q, k, v, out: host pointers, owned by the caller, valid and unmodified
 *                 until `stream` completes.  Page-locked (pinned) memory lets
 *                 the copies overlap the kernels; pageable memory works, but
 *                 the CUDA runtime then stages the copies synchronously.
 *   st, stream:   as in sata_prefill_ex (st, when given, is device memory).
 * Device memory: the library keeps device copies of the inputs and the output
 * (reused by later calls) besides the usual workspace; SATA_ENOMEM if they
 * cannot be allocated.  Errors otherwise as sata_prefill_ex (no SATA_EALIGN for
 * the host pointers).
 */
SATA_API int sata_prefill_host(const void *q, const void *k, const void *v, float *out,
                    int B, int H, int64_t N, int d_K, int d_V, int P,
                    sata_state *st, void *stream);

/*
 * Backward pass of a fresh-state prefill: the gradients of a loss L with
 * respect to q, k and v, given dy = dL/dy for every output of sata_prefill on
 * the same inputs.  The method's pages define no backward pass (they expect the
 * attention to be trained in ordinary Transformer pipelines: [CC-TAYLOR]
 * "Comparison with other methods", "Future directions"); this is the exact
 * gradient of the forward as defined in [CC-TAYLOR] "Feature maps and linear
 * attention", y_t = num_t / den_t, computed in the same chunked feature form
 * (fixed cost per token).  With w_ts = T_P(q_t . k_s / c), T_P(x) = sum_{p<P}
 * x^p / p!, and r_t = [dy_t / den_t | -(dy_t . y_t) / den_t]:
 *   dq_t = 1/c sum_{s<=t} (r_t . [v_s|1]) T_{P-1}(x_ts) k_s,
 *   dk_s = 1/c sum_{t>=s} (r_t . [v_s|1]) T_{P-1}(x_ts) q_t,
 *   dv_s = sum_{t>=s} w_ts dy_t / den_t  (T_P' = T_{P-1}).
 * The forward is recomputed on the prefill's path (keeping den).  Where that
 * path is the tensor-core one and SATA_OPT_DETERMINISTIC is 0, the three sums
 * are tensor-core scans: dq and dk over the features of T_{P-1} with d_K-wide
 * values, dv the prefill's scan on the time-reversed sequence (fp16 operands
 * after per-head power-of-two scales, fp32 accumulation, sums added with fp32
 * atomics, so not bitwise repeatable).  Otherwise one CUDA-core pass forward
 * with S gives dq and one backward with G = sum_t phi(q_t) r_t^T gives dk and
 * dv, their contractions on tensor cores with tf32 operands split into high and
 * low parts (fp32-level accuracy), partial sums added in a fixed order: bitwise
 * reproducible when the forward is (SATA_OPT_DETERMINISTIC = 1, or the CUDA-core
 * path).
 *   q, k: bf16 [B][H][N][d_K];  v: bf16 [B][H][N][d_V]  (the forward's inputs)
 *   dy:   fp32 [B][H][N][d_V]
 *   dq, dk: fp32 [B][H][N][d_K];  dv: fp32 [B][H][N][d_V]  (overwritten)
 *   workspace: NULL (library-owned) or a device buffer of ws_bytes >=
 *              sata_backward_workspace_bytes(...).
 *   stream: cudaStream_t (NULL: legacy stream).
 * N = 0 is a no-op.  Errors as sata_prefill_ex.
 */
SATA_API int sata_backward_workspace_bytes(int B, int H, int64_t N, int d_K, int d_V, int P, size_t *bytes);
SATA_API int sata_prefill_backward(const void *q, const void *k, const void *v, const float *dy,
                    float *dq, float *dk, float *dv, int B, int H, int64_t N, int d_K, int d_V, int P,
                    void *workspace, size_t ws_bytes, void *stream);

/*
 * One decode step for every head of `st`, on st->stream: the state absorbs
 * (k, v) and the output is read with q ([CC-TAYLOR] "Feature maps and linear
 * attention": Z_T = Z_{T-1} + phi(k_T), S_T = S_{T-1} + phi(k_T) v_T^T, then
 * y_T; [CC-HW] "Fixed-size hidden state": constant cost per token).
 *   q, k: bf16 [B][H][d_K];  v: bf16 [B][H][d_V];  out: fp32 [B][H][d_V].
 * The state streams through HBM once (read and write).  st->tokens += 1.
 */
SATA_API int sata_decode_step(sata_state *st, const void *q, const void *k, const void *v, float *out);

/*
 * sata_decode_step_static: the same decode step as sata_decode_step, for
 * callers that may not allocate device memory.  The method's pages have no
 * counterpart; this is a deployment variant.
 *
 * Some callers must not call cudaMalloc: a serving runtime that owns every
 * byte of the GPU through a pre-allocated arena, a plugin inside a host
 * application with its own allocator, or a process held to a memory budget.
 * cudaMalloc allocates outside their accounting and can also synchronise the
 * device.  sata_decode_step allocates on first use (its partial-sum workspace
 * and basis tables).  This entry point allocates nothing: the caller passes the
 * state, inputs and outputs, as above.  Its partial sums live in a 4 MiB static
 * device array compiled into the library, and it derives the basis
 * arithmetically instead of from tables.
 *   Limit: B*H*ceil(F/1024)*(d_V+1) <= 1,048,576 fp32 values: about 4500 heads
 *   at d_K = d_V = 32 (7 x 33 values a head), about 340 at d_K = d_V = 64
 *   (47 x 65).  Beyond that it returns SATA_ENOMEM without launching.
 *   The first call in each device context looks up the array's device address
 *   (a context that replaces it, after cudaDeviceReset, looks it up again);
 *   make that call before any stream capture.  All calls share the array, from
 *   every host thread: calls that overlap on the GPU race.  Nothing in it needs
 *   clearing between calls.  Same kernels as sata_decode_step, so the two give
 *   the same result.
 * Returns SATA_OK or a negative status as sata_decode_step; st->tokens += 1.
 */
SATA_API int sata_decode_step_static(sata_state *st, const void *q, const void *k, const void *v, float *out);

/* Tuning and test options (process-wide).  Keys: */
enum sata_option {
    SATA_OPT_PREFILL_PATH = 1,   /* 0 auto, 1 CUDA-core path, 2 tensor-core path */
    SATA_OPT_WAIT_LIMIT = 2,     /* bounded-wait iteration limit (0 = default) */
    SATA_OPT_TEST_STALL = 3,     /* 1: the next tensor-core prefill launch withholds
                                    one producer signal, so its bounded wait expires
                                    (tests the SATA_ETIMEOUT path); auto-resets */
    SATA_OPT_TIME_KERNELS = 4,   /* 1: bracket every kernel launch with CUDA events on
                                    its own stream (read with sata_kernel_stats) */
    SATA_OPT_DETERMINISTIC = 5   /* tensor-core prefill: 0 (default) adds each feature
                                    group's inter-chunk partial sums into one fp32 buffer
                                    with atomic adds (resolved in L2; the order of the
                                    additions, and so the last bits of the output, can
                                    differ between runs); 1 writes every group's partial
                                    and sums them in a fixed order (bitwise reproducible,
                                    one more pass over the partials through HBM).  The
                                    CUDA-core paths and the decode are always reproducible. */
};
SATA_API int sata_set_option(int key, int64_t value);
SATA_API int sata_get_option(int key, int64_t *value);

/* Per-kernel launch statistics since the last reset: launches are always
 * counted; device time (ms, from the events) only while SATA_OPT_TIME_KERNELS
 * is on.  Reading synchronises the recorded events.  Entries: one per kernel
 * that launched at least once; *n_out receives the count (<= max_entries). */
typedef struct sata_kernel_stat {
    char name[40];
    int64_t launches;
    double ms;
} sata_kernel_stat;
SATA_API int sata_kernel_stats(sata_kernel_stat *out, int max_entries, int *n_out);
SATA_API int sata_reset_kernel_stats(void);

#ifdef __cplusplus
}
#endif

#endif /* SATA_H */
