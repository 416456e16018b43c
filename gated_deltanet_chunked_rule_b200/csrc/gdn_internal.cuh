// gdn_internal.cuh -- declarations shared by the library's translation units.
//
// Notation (one 64-token chunk, rows r, s; qk head hq, value head h):
//   gamma_r = sum_{j<=r} g_j                  (in-chunk cumulative log decay)
//   A_rs    = beta_r exp(gamma_r - gamma_s) k_r.k_s   (s < r, else 0)
//   Ainv    = (I + A)^-1                      (unit lower triangular)
//   w       = Ainv diag(beta exp(gamma)) K    u = Ainv diag(beta) V
//   Delta   = u - w h                          (h = S^T: chunk-entry state, K x V)
//   o       = scale (diag(exp(gamma)) Q h + (M o Q K^T) Delta),  M_rs = exp(gamma_r - gamma_s), s <= r
//   h'      = exp(gamma_C) h + Ktil^T Delta,  Ktil = diag(exp(gamma_C - gamma)) K
// which is the gated delta rule S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
// o_t = scale S_t q_t of the FlashQLA pages, regrouped per chunk (WY form); every
// exponent that appears is a difference gamma_r - gamma_s with s <= r.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

constexpr int kChunk = 64;

// Sequence table (device, in the workspace) for packed variable-length input:
//   info[0 .. N)        first token of sequence n
//   info[N .. 2N)       length of sequence n
//   info[2N .. 3N]      first global chunk of sequence n (info[3N] = total chunks)
//   info[3N+1 .. 4N]    sequences by decreasing chunk count (ties by index)
// With no packing the table is not built (seq_info == nullptr): sequence n is
// batch row n, tokens [n*T, (n+1)*T), chunks [n*ceil(T/64), (n+1)*ceil(T/64)).
struct Dims {
    int B, T, Hq, Hv, K, V;
    int N;           // number of sequences
    int NC;          // total number of chunks
    int T_total;     // B*T tokens along the flattened token axis
    const int *seq_info;
    float scale;
};

struct SeqRange {
    int start, len, chunk0;
};

__device__ __forceinline__ SeqRange seq_range(const Dims &d, int n) {
    SeqRange r;
    if (d.seq_info) {
        r.start = d.seq_info[n];
        r.len = d.seq_info[d.N + n];
        r.chunk0 = d.seq_info[2 * d.N + n];
    } else {
        const int per = (d.T + kChunk - 1) / kChunk;
        r.start = n * d.T;
        r.len = d.T;
        r.chunk0 = n * per;
    }
    return r;
}

// The k-th sequence in longest-first order (identity without packing).
__device__ __forceinline__ int seq_by_length(const Dims &d, int k) {
    return d.seq_info ? d.seq_info[3 * d.N + 1 + k] : k;
}

// Sequence that owns global chunk c (binary search in the chunk offsets); -1 if none.
__device__ __forceinline__ int chunk_owner(const Dims &d, int c) {
    if (!d.seq_info) {
        const int per = (d.T + kChunk - 1) / kChunk;
        if (per == 0) return -1;
        const int n = c / per;
        return n < d.N ? n : -1;
    }
    const int *off = d.seq_info + 2 * d.N;
    if (c < 0 || c >= off[d.N]) return -1;
    int lo = 0, hi = d.N - 1;  // find last n with off[n] <= c
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= c) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Records the first problem a kernel meets in the per-device status word.
__device__ __forceinline__ void set_status(unsigned *status, unsigned code) {
    if (status) atomicCAS(status, 0u, code);
}

// ----------------------------------------------------------- host-side glue

// Pointers of one forward call after workspace carving.
struct FwdArgs {
    Dims d;
    int dtype;
    const void *q, *k, *v;
    const float *g, *beta, *h0;
    void *o;
    float *final_state;
    float *gamma;    // [T_total, Hv] fp32
    void *ainv;      // [NC, Hv, 64, 64], fp32 (F32 problems) or bf16 (BF16 problems); may be null
                     // for the tensor-core forward when nothing is saved
    void *wy;        // [NC, Hv, 2, 64, 64] bf16: Ainv diag(beta), Ainv diag(beta e^gamma) (optional prep output)
    // Chunk-prep outputs of the tensor-core path (bf16, K = V = 128):
    void *w16;       // [T_total, Hv, K] bf16  w = Ainv diag(beta e^gamma) K
    float *u32;      // [T_total, Hv, V] fp32  u = Ainv diag(beta) V
    void *p16;       // [NC, Hv, 64, 64] bf16  P = M o Q K^T
    unsigned *status;
    cudaStream_t stream;
    // Per-chunk entry states and Delta for the backward's recompute (nullable).
    float *h_chunks;  // [NC, Hv, K, V]
    float *delta;     // [T_total, Hv, V]
    // The same for the tensor-core backward, in bf16 (nullable).
    void *h_chunks16, *delta16;
    int nseg;         // sequence-split segments per sequence (1 = no split)
    int fwd_mode;     // 0: whole sequences; 1: segment pass (c, P); 2: segment output pass
    const float *seg_h0;     // [N * nseg, Hv, K, V] composed start state of every segment
    float *seg_c, *seg_P;    // [N * nseg, Hv, K, V] / [.., K, K] segment end state from zero, operator
};

// Token-by-token (decode) step: q, k [T, Hq, K], v, o [T, Hv, V] (T = B*T or the
// packed length), g, beta [T, Hv], h0 / final_state [N, Hv, K, V] fp32 (may alias).
// cu: the device copy of cu_seqlens, or null for B sequences of T tokens.
struct RecurrentArgs {
    Dims d;
    int dtype;
    const int *cu;
    const void *q, *k, *v;
    const float *g, *beta, *h0;
    void *o;
    float *final_state;
    unsigned *status;
    cudaStream_t stream;
};
cudaError_t launch_recurrent(const RecurrentArgs &a);
// Self-test of the bounded waits (gdn_selftest.cu).
cudaError_t launch_wait_selftest(uint64_t limit_ns, unsigned long long *elapsed, unsigned *status,
                                 cudaStream_t stream);

struct BwdArgs {
    Dims d;
    int dtype;
    const void *q, *k, *v, *d_o;
    const float *g, *beta, *h0, *dht;
    const float *gamma;
    const void *ainv;
    const float *h_chunks, *delta;   // from the recompute
    float *dh_chunks;                // [NC, Hv, K, V]  gradient w.r.t. each chunk's exit state
    float *ddelta;                   // [T_total, Hv, V]
    void *dq, *dk, *dv;
    float *dg, *dbeta, *dh0;
    unsigned *status;
    cudaStream_t stream;
};

// Launchers (return a cudaError_t of the launch).
cudaError_t launch_prep_simt(const FwdArgs &a);
cudaError_t launch_fwd_simt(const FwdArgs &a);
cudaError_t launch_bwd_simt(const BwdArgs &a, float *dq_part, float *dk_part);
bool prep_tc_supported(const FwdArgs &a);
cudaError_t launch_prep_tc(const FwdArgs &a);
cudaError_t launch_fwd3(const FwdArgs &a);
// Chunk prep of the tensor-core path: gamma, Ainv (optional), w, u, P.
bool prep3_supported(const FwdArgs &a);
cudaError_t launch_prep3(const FwdArgs &a);
// Sequence split: start state of every segment from h0 and the segments' (c, P).
cudaError_t launch_split_compose(const FwdArgs &a);
// Tensor-core backward (bf16, K = V = 128): reverse dh scan, then the per-chunk
// gradients, which sum dq and dk over each qk head's group of value heads.
bool tc_bwd_supported(const Dims &d, int dtype);
// Sequence split of the reverse scan (mode 0: whole sequences; 1: segment pass
// writing each segment's r, Q; 2: output pass from each segment's composed
// end gradient seg_dh).
struct BwdSplit {
    int nseg = 1, mode = 0;
    const float *seg_dh = nullptr;
    float *seg_r = nullptr, *seg_Q = nullptr;
};
cudaError_t launch_bwd_dh_tc(const BwdArgs &a, const void *w16, const void *p16, void *dh_chunks16, void *ddelta16,
                             const BwdSplit &sp = BwdSplit());
// Composition of the backward split: seg_dh[nseg-1] = dht, seg_dh[s-1] = Q_s seg_dh[s] + r_s.
cudaError_t launch_split_compose_bwd(const Dims &d, int nseg, const float *dht, const float *seg_r,
                                     const float *seg_Q, float *seg_dh, unsigned *status, cudaStream_t stream);
cudaError_t launch_bwd_grad_tc(const BwdArgs &a, const void *h_chunks16, const void *dh_chunks16,
                               const void *delta16, const void *ddelta16);

}  // namespace gdn
