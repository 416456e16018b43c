// gdn_api.cu -- C ABI of the chunked gated delta rule library (see include/gdn.h).
//
// Host side only plans and launches: it validates the problem, lays the
// caller's workspace out, builds (on the device, without a host sync) the
// sequence table for packed variable-length input, and enqueues the kernels
// on the caller's stream. It never allocates device memory.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "gdn_internal.cuh"

namespace gdn {

// Per-device status word: kernels record the first problem they meet here.
__device__ unsigned g_status_word = 0;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_status_mutex;
unsigned *g_status_ptr[kMaxDevices] = {};

unsigned *status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_status_mutex);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = (unsigned *)p;
    }
    return g_status_ptr[dev];
}

// ------------------------------------------------------------ kernel timing
// While enabled, each launch is bracketed by two events on its stream.
struct TimingRec {
    const char *name;
    cudaEvent_t a, b;
};
std::mutex g_tmu;
bool g_timing = false;
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {  // caller holds g_tmu
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

struct TimedLaunch {
    const char *name;
    cudaStream_t st;
    cudaEvent_t a = nullptr;
    TimedLaunch(const char *n, cudaStream_t s) : name(n), st(s) {
        std::lock_guard<std::mutex> lock(g_tmu);
        if (!g_timing) return;
        a = take_event();
        if (a) cudaEventRecord(a, st);
    }
    ~TimedLaunch() {
        if (!a) return;
        std::lock_guard<std::mutex> lock(g_tmu);
        cudaEvent_t b = take_event();
        if (!b) return;
        cudaEventRecord(b, st);
        g_recs.push_back({name, a, b});
    }
};

size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Validated problem summary computed on the host.
struct Plan {
    Dims d;
    int dtype;
    bool varlen;
    size_t gamma_bytes, ainv_bytes, saved_bytes, seq_info_bytes;
    bool tc_ok;       // bf16 with K = V = 128: the tensor-core path
    size_t w_bytes, u_bytes, p_bytes;  // its chunk-prep outputs w (bf16), u (fp32), P (bf16)
    size_t hs_bytes, ds_bytes;         // per-chunk entry states, Delta (bf16): saved for the backward
    size_t core_bytes;                 // gamma | Ainv | w | u | P (what the forward itself needs)
    int max_chunks;   // chunks of the longest sequence
    int nseg;         // forward sequence split: segments per sequence (1 = none)
    size_t seg_bytes; // split scratch: c, P, start states of every segment
};

// Forward sequence split (the pages' gate-driven intra-card context
// parallelism). With u = N * Hv * V/32 chain units and the longest sequence
// of C chunks, an unsplit forward takes ceil(u / SMs) waves of C chunk steps;
// split into S segments it takes ceil(2 u S / SMs) waves of the segment pass
// (state and operator columns) plus ceil(u S / SMs) waves of the output pass,
// each ceil(C / S) steps long, plus S small composition steps. S minimises
// that estimate (segments of at least 8 chunks); GDN_NSEG overrides it.
int choose_nseg(const Plan &P) {
    const Dims &d = P.d;
    if (!P.tc_ok || P.max_chunks < 2) return 1;
    if (const char *e = getenv("GDN_NSEG")) {
        const int v = atoi(e);
        return v < 1 ? 1 : (v > P.max_chunks ? P.max_chunks : v);
    }
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) sms = v;
    }
    const long long units = (long long)d.N * d.Hv * (d.V / 32);
    auto waves = [&](long long ctas) { return (ctas + sms - 1) / sms; };
    const double step_compose = 1.5;  // one composition step, in chunk steps
    double best = (double)waves(units) * P.max_chunks;
    int best_s = 1;
    for (int S = 2; S <= 64 && S * 8 <= P.max_chunks; ++S) {
        const long long per = (P.max_chunks + S - 1) / S;
        const double cost = (double)(waves(2 * units * S) + waves(units * S)) * per + step_compose * S;
        if (cost < 0.9 * best) best = cost, best_s = S;
    }
    return best_s;
}

int make_plan(const gdn_problem *p, Plan *out) {
    if (!p) return GDN_ERR_INVALID_ARG;
    if (p->dtype != GDN_DTYPE_F32 && p->dtype != GDN_DTYPE_BF16) return GDN_ERR_UNSUPPORTED;
    if (p->B < 1 || p->T < 0 || p->Hq < 1 || p->Hv < 1 || p->K < 1 || p->V < 1)
        return GDN_ERR_INVALID_ARG;
    if (p->Hv % p->Hq) return GDN_ERR_INVALID_ARG;
    if ((p->K != 64 && p->K != 128) || (p->V != 64 && p->V != 128)) return GDN_ERR_UNSUPPORTED;
    if (!isfinite(p->scale)) return GDN_ERR_INVALID_ARG;
    if (p->num_seqs < 0) return GDN_ERR_INVALID_ARG;
    const long long ntok = (long long)p->B * p->T;
    if (ntok > (1ll << 30)) return GDN_ERR_INVALID_ARG;  // token indices stay in int
    Plan P;
    memset(&P, 0, sizeof(P));
    P.dtype = p->dtype;
    P.varlen = p->num_seqs > 0;
    Dims &d = P.d;
    d.B = p->B; d.T = p->T; d.Hq = p->Hq; d.Hv = p->Hv; d.K = p->K; d.V = p->V;
    d.T_total = (int)ntok;
    d.scale = p->scale;
    d.seq_info = nullptr;
    if (P.varlen) {
        if (p->B != 1 || !p->cu_seqlens || !p->cu_seqlens_host) return GDN_ERR_INVALID_ARG;
        const int32_t *cu = p->cu_seqlens_host;
        if (cu[0] != 0 || cu[p->num_seqs] != p->T) return GDN_ERR_INVALID_ARG;
        long long nc = 0;
        for (int n = 0; n < p->num_seqs; ++n) {
            if (cu[n + 1] < cu[n]) return GDN_ERR_INVALID_ARG;
            nc += (cu[n + 1] - cu[n] + kChunk - 1) / kChunk;
        }
        d.N = p->num_seqs;
        d.NC = (int)nc;
        P.seq_info_bytes = align_up(sizeof(int) * (4 * (size_t)d.N + 1));
    } else {
        d.N = p->B;
        d.NC = p->B * ((p->T + kChunk - 1) / kChunk);
    }
    P.gamma_bytes = align_up(sizeof(float) * (size_t)d.T_total * d.Hv);
    P.ainv_bytes = align_up((size_t)d.NC * d.Hv * kChunk * kChunk *
                            (p->dtype == GDN_DTYPE_F32 ? sizeof(float) : sizeof(__nv_bfloat16)));
    P.tc_ok = p->dtype == GDN_DTYPE_BF16 && p->K == 128 && p->V == 128;
    if (P.tc_ok) {
        P.w_bytes = align_up(sizeof(__nv_bfloat16) * (size_t)d.T_total * d.Hv * d.K);
        P.u_bytes = align_up(sizeof(float) * (size_t)d.T_total * d.Hv * d.V);
        P.p_bytes = align_up(sizeof(__nv_bfloat16) * (size_t)d.NC * d.Hv * kChunk * kChunk);
    }
    // saved = gamma | Ainv | (bf16 K = V = 128) w, u, P | every chunk's entry state
    // and Delta, so that a backward given `saved` runs neither the chunk prep nor
    // the recompute of the states
    if (P.tc_ok) {
        P.hs_bytes = align_up(sizeof(__nv_bfloat16) * (size_t)d.NC * d.Hv * d.K * d.V);
        P.ds_bytes = align_up(sizeof(__nv_bfloat16) * (size_t)d.NC * kChunk * d.Hv * d.V);  // per chunk, blocked
    }
    P.core_bytes = P.gamma_bytes + P.ainv_bytes + P.w_bytes + P.u_bytes + P.p_bytes;
    P.saved_bytes = P.core_bytes + P.hs_bytes + P.ds_bytes;
    if (P.varlen) {
        for (int n = 0; n < p->num_seqs; ++n)
            P.max_chunks = std::max(P.max_chunks, (p->cu_seqlens_host[n + 1] - p->cu_seqlens_host[n] + kChunk - 1) / kChunk);
    } else {
        P.max_chunks = (p->T + kChunk - 1) / kChunk;
    }
    P.nseg = choose_nseg(P);
    P.seg_bytes = P.nseg > 1 ? align_up(sizeof(float) * (size_t)d.N * P.nseg * d.Hv * d.K * (2 * d.V + d.K)) : 0;
    *out = P;
    return GDN_OK;
}

// Forward workspace: sequence table | gamma, Ainv, w, u, P (used when the caller
// passes no `saved`) | sequence-split scratch. The size and the offsets come
// from this one function.
struct FwdLayout {
    size_t seq, core, seg, total;
};

FwdLayout fwd_layout(const Plan &P) {
    FwdLayout L;
    L.seq = 0;
    L.core = L.seq + P.seq_info_bytes;
    L.seg = L.core + P.core_bytes;
    L.total = L.seg + P.seg_bytes;
    return L;
}

size_t fwd_ws_bytes(const Plan &P) { return fwd_layout(P).total; }

// Backward workspace: sequence table | gamma, Ainv (when no `saved`) | per-chunk
// entry states h | per-chunk exit-state gradients dh' | Delta | dDelta |
// per-value-head fp32 partials of dq and dk.
struct BwdLayout {
    size_t seq, saved, hc, dhc, delta, ddelta, dqp, dkp, total;
};

BwdLayout bwd_layout(const Plan &P) {
    const Dims &d = P.d;
    BwdLayout L;
    const size_t hc = align_up(sizeof(float) * (size_t)d.NC * d.Hv * d.K * d.V);
    const size_t dl = align_up(sizeof(float) * (size_t)d.T_total * d.Hv * d.V);
    const size_t qp = align_up(sizeof(float) * (size_t)d.T_total * d.Hv * d.K);
    L.seq = 0;
    L.saved = L.seq + P.seq_info_bytes;
    L.hc = L.saved + P.core_bytes;
    L.dhc = L.hc + hc;
    L.delta = L.dhc + hc;
    L.ddelta = L.delta + dl;
    L.dqp = L.ddelta + dl;
    L.dkp = L.dqp + qp;
    L.total = L.dkp + qp;
    return L;
}

// Tensor-core backward (bf16, K = V = 128) workspace: sequence table | gamma, Ainv,
// scaled inverses (when no `saved`) |
// bf16 per-chunk entry states and exit-state gradients | bf16 Delta and dDelta (blocked) |
// sequence-split scratch (r, Q, end gradients of every segment).
struct TcBwdLayout {
    size_t seq, saved, hc, dhc, delta, ddelta, seg, total;
};

TcBwdLayout tc_bwd_layout(const Plan &P) {
    const Dims &d = P.d;
    TcBwdLayout L;
    const size_t hc = align_up(sizeof(__nv_bfloat16) * (size_t)d.NC * d.Hv * d.K * d.V);
    const size_t dlb = align_up(sizeof(__nv_bfloat16) * (size_t)d.NC * kChunk * d.Hv * d.V);  // blocked per chunk
    L.seq = 0;
    L.saved = L.seq + P.seq_info_bytes;
    L.hc = L.saved + P.core_bytes;
    L.dhc = L.hc + hc;
    L.delta = L.dhc + hc;
    L.ddelta = L.delta + dlb;
    L.seg = L.ddelta + dlb;
    L.total = L.seg + P.seg_bytes;
    return L;
}

bool tc_bwd_path(const Plan &P) {
    return !(P.dtype == GDN_DTYPE_F32 || (getenv("GDN_IMPL") && strcmp(getenv("GDN_IMPL"), "simt") == 0)) &&
           tc_bwd_supported(P.d, P.dtype) && P.tc_ok;
}

// Pointers into a saved buffer (or the workspace's copy of its core): gamma | Ainv |
// w | u | P [| chunk entry states | Delta, only in a caller's saved buffer].
void set_saved_ptrs(FwdArgs &a, char *sv, const Plan &P, bool with_states) {
    a.gamma = (float *)sv;
    a.ainv = sv + P.gamma_bytes;
    if (P.tc_ok) {
        char *x = sv + P.gamma_bytes + P.ainv_bytes;
        a.w16 = x;
        a.u32 = (float *)(x + P.w_bytes);
        a.p16 = x + P.w_bytes + P.u_bytes;
        if (with_states) {
            a.h_chunks16 = sv + P.core_bytes;
            a.delta16 = sv + P.core_bytes + P.hs_bytes;
        }
    }
}

// The size reported to callers is that of the path the call takes: the
// tensor-core layout (bf16 states) for bf16 K = V = 128, the CUDA-core layout
// (fp32 states and partials, about twice as large) otherwise or under
// GDN_IMPL=simt. A call whose workspace is smaller than its path needs is
// refused with GDN_ERR_WORKSPACE before anything is enqueued.
size_t bwd_ws_bytes(const Plan &P) { return tc_bwd_path(P) ? tc_bwd_layout(P).total : bwd_layout(P).total; }

// Builds the sequence table from the device copy of cu_seqlens and checks it
// against the host plan (total tokens, total chunks). On any disagreement it
// writes an empty table (no sequence has tokens, so later kernels do nothing)
// and records GDN_ERR_DEVICE_ARG in the status word.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t *__restrict__ cu, int N, int T_total,
                                                    int NC_expected, int *__restrict__ info,
                                                    unsigned *status) {
    __shared__ int ok;
    __shared__ int carry;
    __shared__ int warp_sums[32];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) {
        ok = (cu[0] == 0 && cu[N] == T_total) ? 1 : 0;
        carry = 0;
    }
    __syncthreads();
    for (int base = 0; base < N; base += 1024) {
        const int n = base + tid;
        int nch = 0;
        if (n < N) {
            const int a = cu[n], b = cu[n + 1];
            if (b < a || a < 0 || b > T_total) ok = 0;
            const int len = b > a ? b - a : 0;
            nch = (len + kChunk - 1) / kChunk;
            info[n] = a;
            info[N + n] = len;
        }
        // block-wide inclusive scan of nch
        int x = nch;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sums[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int s = warp_sums[lane];
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            warp_sums[lane] = s;
        }
        __syncthreads();
        const int incl = x + (wid > 0 ? warp_sums[wid - 1] : 0);
        if (n < N) info[2 * N + n] = carry + incl - nch;
        __syncthreads();
        if (tid == 1023) carry += incl;
        __syncthreads();
    }
    if (tid == 0) {
        info[3 * N] = carry;
        if (carry != NC_expected) ok = 0;
    }
    __syncthreads();
    // longest first: order[rank] = n, rank = number of sequences with more chunks
    // (ties by index), so that chain kernels start their longest work first; a
    // batch of more than 1024 sequences keeps its own order (the quadratic ranking
    // would cost more than it saves)
    for (int n = tid; n < N; n += 1024) {
        int rank = n;
        if (N <= 1024) {
            const int cn = info[2 * N + n + 1] - info[2 * N + n];
            rank = 0;
            for (int m = 0; m < N; ++m) {
                const int cm = info[2 * N + m + 1] - info[2 * N + m];
                rank += (cm > cn) || (cm == cn && m < n);
            }
        }
        info[3 * N + 1 + rank] = n;
    }
    __syncthreads();
    if (!ok) {
        for (int e = tid; e < 4 * N + 1; e += 1024) info[e] = e >= 3 * N + 1 ? e - (3 * N + 1) : 0;
        if (tid == 0) set_status(status, GDN_ERR_DEVICE_ARG);
    }
}

bool use_simt(int dtype) {
    if (dtype == GDN_DTYPE_F32) return true;
    const char *e = getenv("GDN_IMPL");
    return e && strcmp(e, "simt") == 0;
}

// Chunk prep: tensor-core Gram + blocked inverse for bf16 K=128, CUDA cores otherwise.
int launch_prep(const FwdArgs &a, const char *tc_name = "prep_tc", const char *simt_name = "prep_simt") {
    if (!use_simt(a.dtype) && prep_tc_supported(a)) {
        TimedLaunch t(tc_name, a.stream);
        return launch_prep_tc(a) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
    }
    TimedLaunch t(simt_name, a.stream);
    return launch_prep_simt(a) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// State chain + output of the tensor-core forward.
cudaError_t launch_chain(const FwdArgs &a) { return launch_fwd3(a); }

int launch_plan(const gdn_problem *p, Plan &P, char *ws, unsigned *status, cudaStream_t st) {
    if (!P.varlen) return GDN_OK;
    int *info = (int *)ws;
    TimedLaunch t("plan", st);
    plan_kernel<<<1, 1024, 0, st>>>(p->cu_seqlens, P.d.N, P.d.T_total, P.d.NC, info, status);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    P.d.seq_info = info;
    return GDN_OK;
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" {

size_t gdn_fwd_workspace_size(const gdn_problem *p) {
    Plan P;
    return make_plan(p, &P) == GDN_OK ? fwd_ws_bytes(P) : 0;
}

size_t gdn_bwd_workspace_size(const gdn_problem *p) {
    Plan P;
    return make_plan(p, &P) == GDN_OK ? bwd_ws_bytes(P) : 0;
}

size_t gdn_saved_size(const gdn_problem *p) {
    Plan P;
    return make_plan(p, &P) == GDN_OK ? P.saved_bytes : 0;
}

int gdn_chunk_fwd(const gdn_problem *p, const void *q, const void *k, const void *v,
                  const float *g, const float *beta, const float *h0, void *o,
                  float *final_state, void *saved, void *workspace, size_t workspace_bytes,
                  void *stream) {
    Plan P;
    int rc = make_plan(p, &P);
    if (rc != GDN_OK) return rc;
    const bool has_tokens = P.d.T_total > 0;
    if (has_tokens && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, h0, o, final_state, saved};
    for (const void *x : ptrs)
        if (x && !aligned16(x)) return GDN_ERR_INVALID_ARG;
    const size_t need = fwd_ws_bytes(P);
    if (workspace_bytes < need || (need && !workspace) || ((uintptr_t)workspace & 255u))
        return GDN_ERR_WORKSPACE;
    if (saved && ((uintptr_t)saved & 255u)) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned *status = status_ptr();
    if (!status) return GDN_ERR_CUDA;
    char *ws = (char *)workspace;
    if ((rc = launch_plan(p, P, ws, status, st)) != GDN_OK) return rc;
    char *sv = saved ? (char *)saved : ws + fwd_layout(P).core;

    FwdArgs a;
    memset(&a, 0, sizeof(a));
    a.d = P.d;
    a.dtype = P.dtype;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.h0 = h0;
    a.o = o; a.final_state = final_state;
    set_saved_ptrs(a, sv, P, saved != nullptr);
    a.status = status;
    a.stream = st;
    a.nseg = 1;
    // bf16 with K = V = 128: the tensor-core kernels (chunk prep, then the state
    // chain with the output); otherwise the fp32 CUDA-core kernels
    const bool hybrid = !use_simt(P.dtype) && P.tc_ok &&
                        (long long)P.d.NC * P.d.Hv * kChunk < (1ll << 31);
    if (hybrid) {
        if (!saved) a.ainv = nullptr;  // the hybrid forward reads w, u, P; Ainv only for `saved`
        TimedLaunch t("prep3", st);
        if (launch_prep3(a) != cudaSuccess) return GDN_ERR_CUDA;
    } else {
        if ((rc = launch_prep(a)) != GDN_OK) return rc;
        if (saved && P.tc_ok) {  // keep `saved` complete for a tensor-core backward
            TimedLaunch t("prep3", st);
            if (launch_prep3(a) != cudaSuccess) return GDN_ERR_CUDA;
        }
    }
    if (hybrid && P.nseg > 1) {
        // sequence split: segment pass (c, P) -> composition of start states -> output pass
        float *seg = (float *)(ws + fwd_layout(P).seg);
        const size_t per = (size_t)P.d.N * P.nseg * P.d.Hv * P.d.K;
        a.nseg = P.nseg;
        a.seg_c = seg;
        a.seg_P = seg + per * P.d.V;
        a.seg_h0 = seg + per * (P.d.V + P.d.K);
        FwdArgs s1 = a;
        s1.o = nullptr;
        s1.final_state = nullptr;
        s1.h_chunks16 = s1.delta16 = nullptr;  // the output pass stores the true states
        s1.fwd_mode = 1;
        {
            TimedLaunch t("fwd_split_seg", st);
            if (launch_chain(s1) != cudaSuccess) return GDN_ERR_CUDA;
        }
        {
            TimedLaunch t("fwd_split_compose", st);
            if (launch_split_compose(a) != cudaSuccess) return GDN_ERR_CUDA;
        }
        a.fwd_mode = 2;
        TimedLaunch t("fwd_hybrid", st);
        if (launch_chain(a) != cudaSuccess) return GDN_ERR_CUDA;
    } else if (hybrid) {
        TimedLaunch t("fwd_hybrid", st);
        if (launch_chain(a) != cudaSuccess) return GDN_ERR_CUDA;
    } else {
        TimedLaunch t("fwd_simt", st);
        if (launch_fwd_simt(a) != cudaSuccess) return GDN_ERR_CUDA;
    }
    if (saved && P.tc_ok && !hybrid) {
        // keep `saved` complete for a tensor-core backward: the chunk states and Delta
        FwdArgs r = a;
        r.o = nullptr;
        r.final_state = nullptr;
        r.nseg = 1;
        r.fwd_mode = 0;
        TimedLaunch t("fwd_states", st);
        if (launch_chain(r) != cudaSuccess) return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

int gdn_chunk_bwd(const gdn_problem *p, const void *q, const void *k, const void *v,
                  const float *g, const float *beta, const float *h0, const void *saved,
                  const void *d_o, const float *dht, void *dq, void *dk, void *dv, float *dg,
                  float *dbeta, float *dh0, void *workspace, size_t workspace_bytes,
                  void *stream) {
    Plan P;
    int rc = make_plan(p, &P);
    if (rc != GDN_OK) return rc;
    const bool has_tokens = P.d.T_total > 0;
    if (has_tokens && (!q || !k || !v || !g || !beta || !d_o || !dq || !dk || !dv || !dg || !dbeta))
        return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, h0, saved, d_o, dht, dq, dk, dv, dg, dbeta, dh0};
    for (const void *x : ptrs)
        if (x && !aligned16(x)) return GDN_ERR_INVALID_ARG;
    const BwdLayout L = bwd_layout(P);
    const size_t need = bwd_ws_bytes(P);
    if (workspace_bytes < need || (need && !workspace) || ((uintptr_t)workspace & 255u))
        return GDN_ERR_WORKSPACE;
    if (saved && ((uintptr_t)saved & 255u)) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned *status = status_ptr();
    if (!status) return GDN_ERR_CUDA;
    char *ws = (char *)workspace;
    if ((rc = launch_plan(p, P, ws, status, st)) != GDN_OK) return rc;

    if (tc_bwd_path(P)) {
        // tensor-core path: prep (gamma, Ainv when not saved, scaled inverses) ->
        // recompute of h, Delta (bf16) -> reverse dh scan -> per-chunk gradients (which
        // also sum dq, dk over each qk head's group of value heads)
        const TcBwdLayout T = tc_bwd_layout(P);
        FwdArgs f;
        memset(&f, 0, sizeof(f));
        f.d = P.d;
        f.dtype = P.dtype;
        f.q = q; f.k = k; f.v = v; f.g = g; f.beta = beta; f.h0 = h0;
        f.status = status;
        f.stream = st;
        f.nseg = 1;
        // gamma | Ainv | w | u | P: from the forward's `saved`, else made here
        char *sv = saved ? (char *)saved : ws + T.saved;
        set_saved_ptrs(f, sv, P, saved != nullptr);
        const void *ainv = f.ainv;
        if (!saved) {
            // no saved forward: chunk prep, then the recompute of every chunk's entry
            // state and Delta
            {
                TimedLaunch t("bwd_prep3", st);
                if (launch_prep3(f) != cudaSuccess) return GDN_ERR_CUDA;
            }
            f.o = nullptr;
            f.final_state = nullptr;
            f.h_chunks16 = ws + T.hc;
            f.delta16 = ws + T.delta;
            TimedLaunch t("bwd_recompute", st);
            if (launch_chain(f) != cudaSuccess) return GDN_ERR_CUDA;
        }
        char *hcs = (char *)f.h_chunks16, *dls = (char *)f.delta16;
        BwdArgs b;
        memset(&b, 0, sizeof(b));
        b.d = P.d;
        b.dtype = P.dtype;
        b.q = q; b.k = k; b.v = v; b.d_o = d_o;
        b.g = g; b.beta = beta; b.h0 = h0; b.dht = dht;
        b.gamma = f.gamma;
        b.ainv = ainv;
        b.dq = dq; b.dk = dk; b.dv = dv; b.dg = dg; b.dbeta = dbeta; b.dh0 = dh0;
        b.status = status;
        b.stream = st;
        if (P.nseg > 1) {
            // sequence split of the reverse scan: segment pass (r, Q) -> composition of the
            // segments' end gradients from dht -> output pass
            float *seg = (float *)(ws + T.seg);
            const size_t per = (size_t)P.d.N * P.nseg * P.d.Hv * P.d.K;
            BwdSplit sp;
            sp.nseg = P.nseg;
            sp.seg_r = seg;
            sp.seg_Q = seg + per * P.d.V;
            sp.seg_dh = seg + per * (P.d.V + P.d.K);
            sp.mode = 1;
            {
                TimedLaunch t("bwd_split_seg", st);
                if (launch_bwd_dh_tc(b, f.w16, f.p16, ws + T.dhc, ws + T.ddelta, sp) != cudaSuccess) return GDN_ERR_CUDA;
            }
            {
                TimedLaunch t("bwd_split_compose", st);
                if (launch_split_compose_bwd(P.d, P.nseg, dht, sp.seg_r, sp.seg_Q, seg + per * (P.d.V + P.d.K), b.status, st) !=
                    cudaSuccess)
                    return GDN_ERR_CUDA;
            }
            sp.mode = 2;
            TimedLaunch t("bwd_dh", st);
            if (launch_bwd_dh_tc(b, f.w16, f.p16, ws + T.dhc, ws + T.ddelta, sp) != cudaSuccess) return GDN_ERR_CUDA;
        } else {
            TimedLaunch t("bwd_dh", st);
            if (launch_bwd_dh_tc(b, f.w16, f.p16, ws + T.dhc, ws + T.ddelta) != cudaSuccess) return GDN_ERR_CUDA;
        }
        {
            TimedLaunch t("bwd_grad", st);
            if (launch_bwd_grad_tc(b, hcs, ws + T.dhc, dls, ws + T.ddelta) != cudaSuccess) return GDN_ERR_CUDA;
        }
        return GDN_OK;
    }

    FwdArgs f;
    memset(&f, 0, sizeof(f));
    f.d = P.d;
    f.dtype = P.dtype;
    f.q = q; f.k = k; f.v = v; f.g = g; f.beta = beta; f.h0 = h0;
    f.status = status;
    f.stream = st;
    f.nseg = 1;
    char *sv = saved ? (char *)saved : ws + L.saved;
    f.gamma = (float *)sv;
    f.ainv = sv + P.gamma_bytes;
    f.h_chunks = (float *)(ws + L.hc);
    f.delta = (float *)(ws + L.delta);
    if (!saved && (rc = launch_prep(f, "bwd_prep_tc", "bwd_prep_simt")) != GDN_OK) return rc;
    {
        TimedLaunch t("bwd_recompute_simt", st);
        if (launch_fwd_simt(f) != cudaSuccess) return GDN_ERR_CUDA;
    }
    BwdArgs b;
    memset(&b, 0, sizeof(b));
    b.d = P.d;
    b.dtype = P.dtype;
    b.q = q; b.k = k; b.v = v; b.d_o = d_o;
    b.g = g; b.beta = beta; b.h0 = h0; b.dht = dht;
    b.gamma = f.gamma;
    b.ainv = f.ainv;
    b.h_chunks = f.h_chunks;
    b.delta = f.delta;
    b.dh_chunks = (float *)(ws + L.dhc);
    b.ddelta = (float *)(ws + L.ddelta);
    b.dq = dq; b.dk = dk; b.dv = dv; b.dg = dg; b.dbeta = dbeta; b.dh0 = dh0;
    b.status = status;
    b.stream = st;
    {
        TimedLaunch t("bwd_simt", st);
        if (launch_bwd_simt(b, (float *)(ws + L.dqp), (float *)(ws + L.dkp)) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

}  // extern "C"

// ----------------------------------------------------- no-allocation forward
// Static scratch for gdn_chunk_fwd_noalloc. In host code the array's name is
// only a host-side stand-in; its device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
namespace gdn {
namespace {
static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];
std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kMaxDevices] = {};

void *noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return nullptr;
        g_noalloc_ptr[dev] = ptr;
    }
    return g_noalloc_ptr[dev];
}
}  // namespace
}  // namespace gdn

extern "C" {

int gdn_chunk_fwd_noalloc(const gdn_problem *p, const void *q, const void *k, const void *v,
                          const float *g, const float *beta, const float *h0, void *o,
                          float *final_state, void *stream) {
    Plan P;
    int rc = make_plan(p, &P);
    if (rc != GDN_OK) return rc;
    if (fwd_ws_bytes(P) > GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_WORKSPACE;
    void *scratch = noalloc_scratch();
    if (!scratch) return GDN_ERR_CUDA;
    return gdn_chunk_fwd(p, q, k, v, g, beta, h0, o, final_state, nullptr, scratch,
                         GDN_NOALLOC_SCRATCH_BYTES, stream);
}

int gdn_recurrent_fwd(const gdn_problem *p, const void *q, const void *k, const void *v,
                      const float *g, const float *beta, const float *h0, void *o,
                      float *final_state, void *stream) {
    Plan P;
    int rc = make_plan(p, &P);
    if (rc != GDN_OK) return rc;
    if (P.d.T_total > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, h0, o, final_state};
    for (const void *x : ptrs)
        if (x && !aligned16(x)) return GDN_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return GDN_ERR_CUDA;
    RecurrentArgs a;
    memset(&a, 0, sizeof(a));
    a.d = P.d;
    a.dtype = P.dtype;
    a.cu = p->num_seqs > 0 ? p->cu_seqlens : nullptr;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.h0 = h0;
    a.o = o; a.final_state = final_state;
    a.status = status;
    a.stream = (cudaStream_t)stream;
    TimedLaunch t("recurrent", a.stream);
    return launch_recurrent(a) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_get_device_status(void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GDN_ERR_CUDA;
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(v)) != cudaSuccess) return GDN_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero)) != cudaSuccess)
        return GDN_ERR_CUDA;
    return (int)v;
}

int gdn_selftest_wait_timeout(unsigned long long limit_ns, unsigned long long *elapsed_ns, void *stream) {
    if (!elapsed_ns || !aligned16(elapsed_ns)) return GDN_ERR_INVALID_ARG;
    unsigned *status = status_ptr();
    if (!status) return GDN_ERR_CUDA;
    TimedLaunch t("selftest_wait", (cudaStream_t)stream);
    return launch_wait_selftest(limit_ns, elapsed_ns, status, (cudaStream_t)stream) == cudaSuccess ? GDN_OK
                                                                                                   : GDN_ERR_CUDA;
}

int gdn_timing_enable(int on) {
    std::lock_guard<std::mutex> lock(g_tmu);
    for (auto &r : g_recs) {
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_recs.clear();
    g_timing = on != 0;
    return GDN_OK;
}

int gdn_timing_report(char *buf, size_t buf_len) {
    std::lock_guard<std::mutex> lock(g_tmu);
    std::vector<std::pair<std::string, std::pair<int, double>>> agg;
    for (auto &r : g_recs) {
        if (cudaEventSynchronize(r.b) != cudaSuccess) return -GDN_ERR_CUDA;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return -GDN_ERR_CUDA;
        size_t i = 0;
        while (i < agg.size() && agg[i].first != r.name) ++i;
        if (i == agg.size()) agg.push_back({r.name, {0, 0.0}});
        agg[i].second.first += 1;
        agg[i].second.second += ms;
    }
    std::string out = "{";
    for (size_t i = 0; i < agg.size(); ++i) {
        char item[256];
        snprintf(item, sizeof(item), "%s\"%s\": [%d, %.6f]", i ? ", " : "", agg[i].first.c_str(),
                 agg[i].second.first, agg[i].second.second);
        out += item;
    }
    out += "}";
    if (buf && buf_len) {
        const size_t n = out.size() < buf_len - 1 ? out.size() : buf_len - 1;
        memcpy(buf, out.data(), n);
        buf[n] = 0;
    }
    return (int)out.size();
}

const char *gdn_status_string(int s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
        case GDN_ERR_DEVICE_ARG: return "GDN_ERR_DEVICE_ARG";
        default: return "GDN_ERR_UNKNOWN";
    }
}

const char *gdn_version(void) { return "gdn-b200 0.1 (sm_100a)"; }

}  // extern "C"
