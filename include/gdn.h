/*
 * gdn.h -- C ABI of the B200 (sm_100a) gated delta rule chunked-prefill library.
 *
 * The operation (per sequence n and value head h, qk head hq = h / (Hv/Hq)):
 *
 *   S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *   o_t = scale * S_t q_t                      state S in R^{V x K}
 *
 * computed chunk-parallel (64-token chunks, WY form of the delta rule). The
 * entry points follow the FlashQLA write-up's statement of the problem:
 *   - gdn_chunk_fwd mirrors chunk_gated_delta_rule / chunk_gated_delta_rule_fwd
 *     (page 1, "高级 API 示例" and "底层 API": q, k, v, g, beta, scale,
 *     initial_state, output_final_state, cu_seqlens -> o, final_state, plus
 *     the in-chunk cumulative gate "g" and the chunk matrix "A" it returns);
 *   - gdn_chunk_bwd mirrors chunk_gated_delta_rule_bwd (page 1, "底层 API":
 *     q, k, v, g, beta, A, do, dht, scale, initial_state, cu_seqlens ->
 *     dq, dk, dv, db, dg, dh0);
 *   - the automatic intra-GPU sequence split inside gdn_chunk_fwd is the
 *     "gate-driven automatic intra-card context parallelism" of page 2
 *     ("三大关键特性" table, first row), realised exactly (no truncation);
 *     gdn_chunk_bwd splits its reverse state-gradient scan the same way, with
 *     the same segment count for the same problem.
 *
 * Layouts (contiguous, row-major, device memory unless stated):
 *   q, k        [B, T, Hq, K]   dtype (GDN_DTYPE_F32 or GDN_DTYPE_BF16)
 *   v, o, do    [B, T, Hv, V]   dtype
 *   g, beta     [B, T, Hv]      fp32. g is the per-token LOG decay (<= 0 in
 *                               practice; any finite value is accepted),
 *                               beta the delta-rule write strength.
 *   h0, final_state, dht, dh0
 *               [N, Hv, K, V]   fp32, h = S^T (row index over K, column over V).
 *                               N = B, or num_seqs with cu_seqlens.
 *   cu_seqlens  int32 [num_seqs + 1]: cu[0] = 0, non-decreasing, cu[N] = T,
 *               B must be 1. Sequences are packed along T; each starts from
 *               its own h0[n] and ends in its own final_state[n]. A
 *               zero-length sequence gives final_state[n] = h0[n].
 *   dq, dk      [B, T, Hq, K]   dtype; each sums the value heads of its group.
 *   dv          [B, T, Hv, V]   dtype.
 *   dg, dbeta   [B, T, Hv]      fp32; dg is w.r.t. the raw per-token g.
 *
 * Supported sizes: K, V in {64, 128}; Hv a multiple of Hq; T >= 0; B >= 1.
 *
 * Ownership and synchronisation: every pointer is caller-owned; the problem
 * description and cu_seqlens_host are host memory, everything else is device
 * memory on the current device (a host pointer there is not detected and
 * faults the kernels, so bindings must check it). The library
 * never allocates, frees or synchronises (except gdn_get_device_status); it
 * enqueues its kernels on the caller's stream and keeps no state between
 * calls other than the device status word. Scratch memory comes from the
 * caller's workspace (sizes from the *_workspace_size queries, 256-byte
 * aligned pointer required). All pointers must be 16-byte aligned.
 *
 * Errors: arguments are validated on the host before anything is enqueued;
 * a rejected call enqueues nothing. Device-side problems (an inconsistent
 * device copy of cu_seqlens, a bounded wait that expired) are recorded in a
 * per-device status word read by gdn_get_device_status; the kernels then do
 * no further work for that call and return, they never trap.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,  /* null pointer, bad size, Hv % Hq != 0, bad cu_seqlens, ... */
    GDN_ERR_UNSUPPORTED = 2,  /* K or V not in {64,128}, unknown dtype                     */
    GDN_ERR_WORKSPACE = 3,    /* workspace too small or misaligned                          */
    GDN_ERR_CUDA = 4,         /* a CUDA launch or query failed                              */
    GDN_ERR_TIMEOUT = 5,      /* a bounded device-side wait expired (status word)           */
    GDN_ERR_DEVICE_ARG = 6    /* device copy of cu_seqlens disagrees with the host copy     */
} gdn_status;

typedef enum { GDN_DTYPE_F32 = 0, GDN_DTYPE_BF16 = 1 } gdn_dtype;

typedef struct {
    int B, T, Hq, Hv, K, V;
    int num_seqs;                   /* 0: no packing (N = B); else B == 1 and cu_seqlens given */
    const int32_t *cu_seqlens;      /* device, [num_seqs + 1], or NULL when num_seqs == 0       */
    const int32_t *cu_seqlens_host; /* the same values in host memory (planning without a sync) */
    int dtype;                      /* gdn_dtype of q, k, v, o, do, dq, dk, dv                  */
    float scale;                    /* any finite value; 1/sqrt(K) is the usual choice          */
} gdn_problem;

/* Bytes of caller-provided scratch that gdn_chunk_fwd / gdn_chunk_bwd need
 * for this problem (0 if the problem is invalid). */
size_t gdn_fwd_workspace_size(const gdn_problem *p);
size_t gdn_bwd_workspace_size(const gdn_problem *p);

/* Bytes of the "saved" buffer: the in-chunk cumulative gate gamma (fp32
 * [B*T, Hv]) followed by Ainv = (I + A)^-1 of every 64-token chunk
 * ([num_chunks, Hv, 64, 64], fp32 for GDN_DTYPE_F32 problems, bf16 for
 * GDN_DTYPE_BF16), i.e. the "g, A" that page 1's low-level forward returns
 * and its backward takes back ("底层 API" section of the FlashQLA write-up).
 * For bf16 problems with K = V = 128 the buffer continues with what the
 * tensor-core backward needs from the forward: w = Ainv diag(beta e^gamma) K
 * (bf16 [B*T, Hv, K]), u = Ainv diag(beta) V (fp32 [B*T, Hv, V]), the
 * decay-masked P = M o Q K^T of every chunk (bf16 [num_chunks, Hv, 64, 64]),
 * and every chunk's entry state (bf16, num_chunks * Hv * K * V elements) and
 * Delta (bf16, num_chunks * 64 * Hv * V elements) -- the per-chunk states h
 * that page 1's low-level forward also returns -- so that a backward given
 * `saved` runs neither the chunk prep nor a recompute of the states. The
 * states and Delta are stored in a blocked layout private to this library
 * (one block per chunk, value head and 32-column slice). Each part 256-byte
 * aligned. */
size_t gdn_saved_size(const gdn_problem *p);

/* Forward. h0 may be NULL (zero initial state); final_state may be NULL (not
 * written); saved may be NULL (not written). o must not be NULL.
 * Packed sequences stay independent even for non-finite values: the rows past
 * the end of a sequence's last (ragged) chunk are zeroed or selected out
 * before any product, so a NaN or Inf in one packed sequence cannot reach the
 * outputs or final state of another. */
int gdn_chunk_fwd(const gdn_problem *p, const void *q, const void *k, const void *v,
                  const float *g, const float *beta, const float *h0, void *o,
                  float *final_state, void *saved, void *workspace, size_t workspace_bytes,
                  void *stream /* cudaStream_t */);

/* Backward. h0 and dht may be NULL (zero); saved may be NULL (gamma and Ainv
 * are then recomputed) or the buffer a gdn_chunk_fwd call with the same
 * problem and inputs filled; dh0 may be NULL (not written). The other
 * outputs must not be NULL.
 * As in the forward, packed sequences stay independent for non-finite values:
 * the rows past the end of a sequence's last chunk are zeroed or selected out
 * before any product, so a NaN or Inf in one packed sequence cannot reach the
 * gradients of another. */
int gdn_chunk_bwd(const gdn_problem *p, const void *q, const void *k, const void *v,
                  const float *g, const float *beta, const float *h0, const void *saved,
                  const void *d_o, const float *dht, void *dq, void *dk, void *dv, float *dg,
                  float *dbeta, float *dh0, void *workspace, size_t workspace_bytes,
                  void *stream /* cudaStream_t */);

/* Forward that allocates nothing and needs no workspace.
 *
 * For callers that cannot allocate device memory at all: a plugin hosted by
 * an engine that owns every device allocation and hands out only inputs and
 * outputs, or a latency-critical path that must not call cudaMalloc/cudaFree
 * (either can synchronise the whole device). It runs the same forward as
 * gdn_chunk_fwd with saved = NULL, but its scratch is a fixed static device
 * array of GDN_NOALLOC_SCRATCH_BYTES (16 MiB) inside this library, which every
 * GPU that loads the library holds until the process exits. It calls no
 * cudaMalloc, cudaFree or other allocating routine. The caller still passes
 * inputs and outputs, as for gdn_chunk_fwd.
 *   - A problem whose forward scratch (gdn_fwd_workspace_size) is larger than
 *     GDN_NOALLOC_SCRATCH_BYTES is rejected with GDN_ERR_WORKSPACE before
 *     anything is enqueued.
 *   - The first call on each device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   - Every call shares the one array and it keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other host threads on the
 *     same device) race on it and corrupt each other's results, so serialise
 *     them. Nothing in it has to start at zero: each call writes every byte it
 *     reads before reading it.
 * The FlashQLA pages have no counterpart to this entry point. */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int gdn_chunk_fwd_noalloc(const gdn_problem *p, const void *q, const void *k, const void *v,
                          const float *g, const float *beta, const float *h0, void *o,
                          float *final_state, void *stream /* cudaStream_t */);

/* Token-by-token (decode) step of the same recurrence, for a few tokens per
 * sequence: o_t = scale S_t q_t with S_t = exp(g_t) S_{t-1} (I - beta_t k_t
 * k_t^T) + beta_t v_t k_t^T, taken one token after another from h0 (NULL:
 * zero) to final_state (NULL: not written). The state of every (sequence,
 * value head) is read once and written once per call, so a decode loop calls
 * this once per generated token. Same problem description, layouts, sizes and
 * dtypes as gdn_chunk_fwd; no workspace. final_state may be the same buffer as
 * h0 (the update is in place). Each sequence's tokens are read from the device
 * copy of cu_seqlens; an inconsistent one is recorded as GDN_ERR_DEVICE_ARG in
 * the status word and that sequence is left untouched. The chunked forward is
 * the faster choice once a call covers more than a few dozen tokens per
 * sequence. This is the gated delta rule exactly as the pages state it for
 * the GDN layers (page 1, "什么是 FlashQLA"), taken without chunks: the pages'
 * kernels are the prefill of this recurrence and give no decode kernel. */
int gdn_recurrent_fwd(const gdn_problem *p, const void *q, const void *k, const void *v,
                      const float *g, const float *beta, const float *h0, void *o,
                      float *final_state, void *stream /* cudaStream_t */);

/* Synchronises `stream`, then returns and clears the current device's status
 * word (GDN_OK if no kernel recorded a problem since the last call). */
int gdn_get_device_status(void *stream /* cudaStream_t */);

/* Kernel timing (tracing). While enabled (on != 0), every kernel launch the
 * library makes is bracketed by a pair of CUDA events recorded on the launch
 * stream. gdn_timing_report synchronises the device, then writes into buf a
 * JSON object {"<kernel>": [launches, total_ms], ...} covering every launch
 * since the last enable/reset, and returns the number of bytes needed
 * (excluding the terminating NUL; the output is truncated if buf_len is too
 * small), or minus a gdn_status code on failure. Enabling clears earlier
 * records. The events come from a pool the library creates on first use; it
 * holds no device memory. Timing changes nothing in the results; it adds a few
 * microseconds per launch. */
int gdn_timing_enable(int on);
int gdn_timing_report(char *buf, size_t buf_len);

/* Self-test of the device-side failure detection. Every wait inside this
 * library's kernels (on a TMA or tensor-core completion, or on another warp's
 * hand-over) is bounded: after a limit it gives up, records GDN_ERR_TIMEOUT in
 * the status word and lets the kernel wind down instead of hanging the GPU.
 * This entry point enqueues one small kernel whose two waits can never be
 * satisfied -- an mbarrier phase that nothing completes and a hand-over
 * counter that nothing publishes -- with limit_ns of wall-clock time each
 * (0: the limit the kernels use, 2 s). Nothing else is in flight in it, so it
 * always ends normally. elapsed_ns: device memory, 2 entries (16-byte
 * aligned), receiving the time each wait took before giving up (all ones if
 * a wait was, impossibly, satisfied). Afterwards gdn_get_device_status reports
 * GDN_ERR_TIMEOUT. The FlashQLA pages have no counterpart to this entry
 * point; it serves the failure-detection tests. Returns GDN_ERR_INVALID_ARG
 * for a null or misaligned elapsed_ns, GDN_ERR_CUDA if the launch fails. */
int gdn_selftest_wait_timeout(unsigned long long limit_ns, unsigned long long *elapsed_ns,
                              void *stream /* cudaStream_t */);

/* Static, human-readable name of a status code. */
const char *gdn_status_string(int status);

/* Library build identifier (sm_100a kernels compiled in). */
const char *gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
