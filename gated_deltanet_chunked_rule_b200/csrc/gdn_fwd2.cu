// gdn_fwd2.cu -- warp-specialised chunked forward (bf16, K = V = 128): the
// state chain and the output on warp-level tensor-core MMAs, the bulk chunk
// products on tcgen05.
//
// One CTA per (sequence, value head, 32-column slice of V). Per 64-token chunk
// (notation of gdn_internal.cuh; Au = Ainv diag(beta), Aw = Ainv diag(beta e^gamma)
// come ready-made from the chunk-prep kernel):
//
//   tcgen05, TMEM accumulators:
//     S = Q K^T,   W = Aw K,   U = Au V          (independent of h, one chunk ahead)
//     DQ = Q h,    DP = P Delta                  (output, one chunk behind the chain)
//     o = scale (e^gamma o DQ + DP),  P = causal decay mask o S
//   mma.sync, fp32 state in registers (the chain):
//     Delta = U + (-w) h,   h <- e^{gamma_C} h + K^T (e^{gamma_C - gamma} o Delta)
//
// Why this split (measured on B200): a tcgen05 MMA takes ~450 cycles from
// issue to a completed mbarrier, twice per chunk on the chain, whereas a
// dependent mma.sync costs ~20 cycles, so the chain runs on mma.sync. The
// output products stay on tcgen05 because there they read their operands once
// from shared memory, whereas warp-level MMAs split across warps re-read them
// and the shared-memory bandwidth (128 B/clk) is the next limit. The chain
// publishes Delta_j and h_{j+1} together behind one generic-to-async proxy
// fence per chunk.
//
// Warp roles (576 threads, two warps of each CUDA-core role per SM sub-partition):
//   warps 0-7   chain: h (128 x 32 fp32) in mma fragments, warp w holding
//               state rows 32 (w % 4) .. +31 and columns 16 (w / 4) .. +15.
//   warps 8-15  aux: -w and u from TMEM into shared memory for the chain, P
//               from S into shared memory, and o of the previous chunk from
//               DQ/DP; warp 8 + w reads TMEM lanes 32 (w % 4) .. +31 and
//               handles half (w / 4) of the columns.
//   warp 16     MMA issuer A: TMA prologue, S/W/U MMAs.
//   warp 17     MMA issuer B: DQ/DP MMAs, refills of the 3-deep TMA ring.
// Roles hand over through monotonically increasing shared-memory counters
// (release/acquire), which cannot alias the way mbarrier phase parities can
// when a producer runs two phases ahead of a consumer. mbarriers are used only
// where the hardware requires them: TMA completion (full[]) and tcgen05.commit
// (mmaA[] for the aux warps, mmaO for issuer B), each with a single consumer
// that its producer cannot lap. Every wait is
// bounded in time; a wait that expires records GDN_ERR_TIMEOUT and winds the
// CTA down.
#include <cudaTypedefs.h>

#include <cstddef>

#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kThreads = 576;  // 8 chain + 8 aux + 2 TMA/MMA warps
constexpr int kRole = 256;     // threads per CUDA-core role
constexpr int kBV = 32;
constexpr int kStages = 3;

// ---- shared memory (bytes from a 1024-aligned base)
constexpr int kHb = 0;          // 2 x 8192   h (bf16): (n/8)*2048 + (k/8)*128 + (k%8)*16 (k = state row)
constexpr int kDb = 16384;      // 3 x 4096   Delta (bf16), same layout with k = token
constexpr int kDt = 28672;      // 4096       e^{gamma_C - gamma} Delta, chain only
constexpr int kP = 32768;       // 8192       P, K-major SW128 (A of DP)
constexpr int kWn = 40960;      // 16384      -w (bf16), row-major 256 B rows, 16-B chunks XOR (row % 8)
constexpr int kU = 57344;       // 9216       u (fp32), row stride 36 floats
constexpr int kStage0 = 66560;  // TMA ring
constexpr int kQ = 0, kK = 16384, kAu = 32768, kAwS = 40960, kVt = 49152, kStageBytes = 53248;
constexpr int kTxBytes = 16384 + 16384 + 8192 + 8192 + 4096;
constexpr int kSmall = kStage0 + kStages * kStageBytes;
constexpr int kSmemBytes = kSmall + 2560 + 1024;
static_assert(kStage0 % 1024 == 0 && kStageBytes % 1024 == 0 && kSmemBytes <= 232448, "shared memory layout");

// S, W, U double-buffered in tensor memory (buffer b at column 224 b); DQ, DP single.
constexpr uint32_t kColS = 0, kColW = 64, kColU = 192, kABuf = 224, kColQ = 448, kColP = 480, kTmemCols = 512;

struct __align__(16) Gates {
    float gam[64], egam[64];
};

// Hand-over counters: each holds the number of chunks (or states) its producer
// has finished; consumers wait until it reaches the count they need.
enum Ctr { kTmemA, kReady, kPReady, kWnFree, kDelta, kH, kStage, kODone, kTmemO, kNumCtr };

struct Small {
    uint64_t full[kStages];
    uint64_t mmaA[2], mmaO;
    uint32_t ctr[kNumCtr];
    int loads_issued, loads_landed;  // TMA chunk loads issued / observed complete
    uint32_t tmem_base;
    int abort_flag;
    Gates gates[3];
};
static_assert(sizeof(Small) <= 2560, "small area");
static_assert(kSmall % 16 == 0 && offsetof(Small, gates) % 16 == 0, "small area alignment");

template <int N = kRole>
__device__ __forceinline__ bool role_sync_and(int id, bool pred) {
    return warp::role_sync_and<N>(id, pred);
}

// kWhole: one CTA column per sequence, from h0.
// kSegPass: per segment, the chain on [c | P] with c from zero (V columns, u as
//   input) and P from the identity (K more columns, whose v tile is read out of
//   range and so is zero): the segment maps a start state h to P h + c.
// kSegOut: per segment, the chain and the output from the composed start state.
enum Fwd2Mode { kWhole = 0, kSegPass = 1, kSegOut = 2 };

struct Fwd2Params {
    Dims d;
    const float *gamma;   // [T_total, Hv]
    const float *h0;      // [N, Hv, K, V] or null
    __nv_bfloat16 *o;     // [T_total, Hv, V], or null: no output products (the backward's recompute)
    float *final_state;   // [N, Hv, K, V] or null
    __nv_bfloat16 *h_chunks;  // [NC, Hv, K, V] entry state of every chunk (bf16, as the products read it) or null
    __nv_bfloat16 *delta;     // [T_total, Hv, V] Delta (bf16) or null
    // Sequence split: blockIdx.x = sequence * nseg + segment; a segment is a
    // contiguous run of ceil(chunks / nseg) chunks of its sequence.
    int nseg;
    int mode;             // kWhole, kSegPass or kSegOut
    const float *seg_h0;  // kSegOut: [N * nseg, Hv, K, V] start state of every segment
    float *seg_c;         // kSegPass: [N * nseg, Hv, K, V] end state from a zero start
    float *seg_P;         // kSegPass: [N * nseg, Hv, K, K] transition operator of the segment
    unsigned *status;
};

__global__ void __launch_bounds__(kThreads, 1)
fwd2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_wy,
            const Fwd2Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    Small *sm = reinterpret_cast<Small *>(smem + kSmall);
    volatile int *abort_flag = &sm->abort_flag;
    const uint32_t sb = smem_u32(smem);

    const Dims &d = prm.d;
    const int nseg = prm.nseg;
    const int n = blockIdx.x / nseg, sseg = blockIdx.x % nseg, h = blockIdx.y, c0 = blockIdx.z * kBV;
    const int hq = h / (d.Hv / d.Hq);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int K = 128, V = 128;
    // this CTA's chunks [j0, j1) of the sequence, seen as a sequence of their own
    const SeqRange seq = seq_range(d, n);
    const int nch_seq = (seq.len + kChunk - 1) / kChunk;
    const int per_seg = (nch_seq + nseg - 1) / nseg;
    const int j0 = min(sseg * per_seg, nch_seq), j1 = min(j0 + per_seg, nch_seq);
    SeqRange sr;
    sr.start = seq.start + j0 * kChunk;
    sr.chunk0 = seq.chunk0 + j0;
    sr.len = j1 > j0 ? min(seq.len - j0 * kChunk, (j1 - j0) * kChunk) : 0;
    const int nch = j1 - j0;
    const size_t seg_idx = (size_t)n * nseg + sseg;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&sm->full[s], 1);
        mbar_init(&sm->mmaA[0], 1);
        mbar_init(&sm->mmaA[1], 1);
        mbar_init(&sm->mmaO, 1);
        for (int c = 0; c < kNumCtr; ++c) sm->ctr[c] = 0;
        sm->loads_issued = sm->loads_landed = 0;
        sm->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 16) {
        tmem_alloc(&sm->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;
    uint32_t *ctr = sm->ctr;

    auto issue_loads = [&](int ci) {
        const int s = ci % kStages;
        uint8_t *st = smem + kStage0 + s * kStageBytes;
        const int t0 = sr.start + ci * kChunk;
        const int cg = sr.chunk0 + ci;
        mbar_arrive_expect_tx(&sm->full[s], kTxBytes);
        atomicAdd(&sm->loads_issued, 1);
        tma_load_3d(st + kQ, &tm_q, &sm->full[s], 0, hq, t0);
        tma_load_3d(st + kQ + 8192, &tm_q, &sm->full[s], 64, hq, t0);
        tma_load_3d(st + kK, &tm_k, &sm->full[s], 0, hq, t0);
        tma_load_3d(st + kK + 8192, &tm_k, &sm->full[s], 64, hq, t0);
        tma_load_2d(st + kAu, &tm_wy, &sm->full[s], 0, ((cg * d.Hv + h) * 2) * kChunk);
        tma_load_2d(st + kAwS, &tm_wy, &sm->full[s], 0, ((cg * d.Hv + h) * 2 + 1) * kChunk);
        tma_load_3d(st + kVt, &tm_v, &sm->full[s], c0, h, t0);
    };

    if (warp < 8) {
        // =========================================================== chain
        const int p = warp & 3, cb = (warp >> 2) * 2;  // state rows 32p.., n-tiles cb, cb+1 (16 columns)
        const int g = lane >> 2, c4 = lane & 3;
        float hf[2][2][4];  // [m-tile][n-tile][frag]: rows 32p+16mt+g(+8), cols 8(cb+nt)+2c4(+1)
        {
            const float *src = prm.mode == kWhole ? (prm.h0 ? prm.h0 + ((size_t)n * d.Hv + h) * K * V : nullptr)
                               : prm.mode == kSegOut ? prm.seg_h0 + (seg_idx * d.Hv + h) * K * V
                                                     : nullptr;
            const bool ident = prm.mode == kSegPass && c0 >= V;  // operator columns start as I
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int dim = 32 * p + 16 * mt + g + ((q >> 1) << 3);
                        const int col = 8 * (cb + nt) + 2 * c4 + (q & 1);
                        hf[mt][nt][q] = src ? src[(size_t)dim * V + c0 + col] : (ident && dim == c0 - V + col ? 1.f : 0.f);
                    }
        }
        auto write_hb = [&](int buf) {
            const uint32_t base = sb + kHb + buf * 8192 + c4 * 4;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int dim = 32 * p + 16 * mt + g + half * 8;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
                        st_shared_b32(base + (cb + nt) * 2048 + (dim >> 3) * 128 + (dim & 7) * 16,
                                      pack_bf16(hf[mt][nt][2 * half], hf[mt][nt][2 * half + 1]));
                }
        };
        write_hb(0);
        fence_proxy_async();
        bool ok = role_sync_and(1, true);
        if (tid == 0) publish(&ctr[kH], 1);  // h_0

        for (int j = 0; j < nch && ok; ++j) {
            const int len = min(kChunk, sr.len - j * kChunk);
            ok = role_sync_and(1, wait_ge(&ctr[kReady], j + 1, abort_flag));
            if (!ok) break;
            // gate scalars of chunk j (its slot is refilled only after this chunk's -w is consumed)
            const Gates &G = sm->gates[j % 3];
            const float gl = G.gam[63];
            if (prm.h_chunks) {  // entry state of chunk j, rounded as the products read it
                __nv_bfloat16 *hc = prm.h_chunks + ((size_t)(sr.chunk0 + j) * d.Hv + h) * K * V + c0;
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int dim = 32 * p + 16 * mt + g + half * 8;
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
                            *reinterpret_cast<uint32_t *>(hc + (size_t)dim * V + 8 * (cb + nt) + 2 * c4) =
                                pack_bf16(hf[mt][nt][2 * half], hf[mt][nt][2 * half + 1]);
                    }
            }
            const float gtok[2] = {G.gam[16 * p + g], G.gam[16 * p + g + 8]};
            // ---- Delta = u + (-w) h : tokens 16p..16p+15, columns of n-tiles cb, cb+1
            float acc[2][4];
            {
                const float *U = reinterpret_cast<const float *>(smem + kU);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int r0 = 16 * p + g, col = 8 * (cb + nt) + 2 * c4;
                    const float2 a = *reinterpret_cast<const float2 *>(U + r0 * 36 + col);
                    const float2 b = *reinterpret_cast<const float2 *>(U + (r0 + 8) * 36 + col);
                    acc[nt][0] = a.x; acc[nt][1] = a.y; acc[nt][2] = b.x; acc[nt][3] = b.y;
                }
                const uint32_t hb = sb + kHb + (j & 1) * 8192;
                const int arow = 16 * p + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int mi = lane >> 3;  // (kg, nb): (2ks,cb) (2ks+1,cb) (2ks,cb+1) (2ks+1,cb+1)
                uint32_t a[2][4], b[2][4];
                auto load = [&](int ks, int buf) {
                    const int ch = 2 * ks + (lane >> 4);
                    ldsm_x4(a[buf], sb + kWn + arow * 256 + ((ch ^ (arow & 7)) << 4));
                    ldsm_x4_t(b[buf], hb + (cb + (mi >> 1)) * 2048 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
                };
                load(0, 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    if (ks + 1 < 8) load(ks + 1, (ks + 1) & 1);
                    hmma(acc[0], a[ks & 1], b[ks & 1][0], b[ks & 1][1]);
                    hmma(acc[1], a[ks & 1], b[ks & 1][2], b[ks & 1][3]);
                }
            }
            role_sync_and(1, true);
            if (tid == 0) publish(&ctr[kWnFree], j + 1);
            // ---- Delta -> Db[j%3] (read by the output) ; e^{gamma_C - gamma} Delta -> Dt
            ok = role_sync_and(1, j < 3 || wait_ge(&ctr[kODone], j - 2, abort_flag));  // DP of j-3 read Db[j%3]
            if (!ok) break;
            {
                const uint32_t db = sb + kDb + (j % 3) * 4096 + c4 * 4, dt = sb + kDt + c4 * 4;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int tok = 16 * p + g + half * 8;
                    const bool live = tok < len;
                    const float sc = __expf(gl - gtok[half]);
                    const uint32_t off = (tok >> 3) * 128 + (tok & 7) * 16;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const float x0 = live ? acc[nt][2 * half] : 0.f, x1 = live ? acc[nt][2 * half + 1] : 0.f;
                        st_shared_b32(db + (cb + nt) * 1024 + off, pack_bf16(x0, x1));
                        st_shared_b32(dt + (cb + nt) * 1024 + off, pack_bf16(sc * x0, sc * x1));
                        if (prm.delta && live)
                            *reinterpret_cast<uint32_t *>(prm.delta + ((size_t)(sr.start + j * kChunk + tok) * d.Hv + h) * V +
                                                          c0 + 8 * (cb + nt) + 2 * c4) = pack_bf16(x0, x1);
                    }
                }
            }
            role_sync_and(1, true);  // every warp reads all 64 tokens of Dt below
            // ---- h <- e^{gamma_C} h + K^T Dt : rows 32p..32p+31, 16 columns, K = 64 tokens
            {
                const float eC = __expf(gl);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int q = 0; q < 4; ++q) hf[mt][nt][q] *= eC;
                const uint32_t kt = sb + kStage0 + (j % kStages) * kStageBytes + kK;
                const int mi = lane >> 3;
                uint32_t b[2][4], a[2][2][4];
                auto load = [&](int ks, int buf) {
                    ldsm_x4_t(b[buf], sb + kDt + (cb + (mi >> 1)) * 1024 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        // A = K^T rows (state rows) 32p+16mt.., cols (tokens) 16ks..: 8x8
                        // blocks of the token-major, 128-byte-swizzled k tile read transposed
                        const int tt = 16 * ks + (lane & 7) + ((mi >> 1) & 1) * 8;
                        const int dd = 32 * p + 16 * mt + (mi & 1) * 8;
                        ldsm_x4_t(a[buf][mt], kt + (dd >> 6) * 8192 + tt * 128 + ((((dd & 63) >> 3) ^ (tt & 7)) << 4));
                    }
                };
                load(0, 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    if (ks + 1 < 4) load(ks + 1, (ks + 1) & 1);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        hmma(hf[mt][0], a[ks & 1][mt], b[ks & 1][0], b[ks & 1][1]);
                        hmma(hf[mt][1], a[ks & 1][mt], b[ks & 1][2], b[ks & 1][3]);
                    }
                }
            }
            role_sync_and(1, true);
            if (tid == 0) publish(&ctr[kStage], j + 1);
            // ---- h_{j+1} -> Hb[(j+1)%2] once DQ of chunk j-1 (which read it) is done; then
            //      Delta_j and h_{j+1} go to the output MMAs behind one proxy fence
            ok = role_sync_and(1, j < 1 || wait_ge(&ctr[kODone], j, abort_flag));
            if (!ok) break;
            write_hb((j + 1) & 1);
            fence_proxy_async();
            role_sync_and(1, true);
            if (tid == 0) {
                publish(&ctr[kDelta], j + 1);
                publish(&ctr[kH], j + 2);
            }
        }
        if (!ok) {
            if (tid == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        } else {
            // end state: the sequence's final state (from the CTA holding its last chunk),
            // or the segment's c / P columns
            float *dst = nullptr;
            int ld = V;
            if (prm.mode == kSegPass) {
                if (c0 < V) dst = prm.seg_c + (seg_idx * d.Hv + h) * K * V + c0;
                else dst = prm.seg_P + (seg_idx * d.Hv + h) * K * K + (c0 - V), ld = K;
            } else if (prm.final_state && j1 == nch_seq && (j0 < j1 || sseg == 0)) {
                dst = prm.final_state + ((size_t)n * d.Hv + h) * K * V + c0;
            }
            if (dst) {
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const int dim = 32 * p + 16 * mt + g + half * 8;
                            *reinterpret_cast<float2 *>(dst + (size_t)dim * ld + 8 * (cb + nt) + 2 * c4) =
                                make_float2(hf[mt][nt][2 * half], hf[mt][nt][2 * half + 1]);
                        }
            }
        }
    } else if (warp < 16) {
        // ============================================================= aux
        const int atid = tid - kRole, aw = warp - 8;
        const int ap = aw & 3, ah = aw >> 2;  // TMEM sub-partition (rows 16ap..), output column half
        const uint32_t lane_base = (uint32_t)(ap * 32) << 16;
        const int ag = lane >> 2, ac = lane & 3;
        const int ar0 = ap * 16 + ag, ar1 = ar0 + 8;  // rows of M=64 results this thread holds
        bool ok = true;
        const bool want_o = prm.o != nullptr;
        auto output = [&](int jo) -> bool {  // o of chunk jo from DQ, DP (16 columns per warp)
            if (!wait_ge(&ctr[kODone], jo + 1, abort_flag)) return false;
            if (!want_o) return true;
            tc_fence_after();
            const Gates &G = sm->gates[jo % 3];
            const int len = min(kChunk, sr.len - jo * kChunk);
            const int t0 = sr.start + jo * kChunk;
            float dq[8], dp[8];
            tmem_ld16x256_x2(tmem + lane_base + kColQ + 16 * ah, dq);
            tmem_ld16x256_x2(tmem + lane_base + kColP + 16 * ah, dp);
            tc_fence_before();
            const float scl = d.scale;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = half ? ar1 : ar0;
                if (r < len) {
                    const float er = G.egam[r];
                    __nv_bfloat16 *dst = prm.o + ((size_t)(t0 + r) * d.Hv + h) * V + c0 + 16 * ah + 2 * ac;
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int k = 4 * i + 2 * half;
                        *reinterpret_cast<uint32_t *>(dst + 8 * i) =
                            pack_bf16(scl * fmaf(er, dq[k], dp[k]), scl * fmaf(er, dq[k + 1], dp[k + 1]));
                    }
                }
            }
            return true;
        };
        float pg = 0.f;
        auto fetch_gate = [&](int jj) {  // gamma of chunk jj, one value per thread < 64
            if (atid < kChunk && jj < nch) {
                const int t0 = sr.start + jj * kChunk, len = min(kChunk, sr.len - jj * kChunk);
                pg = prm.gamma[(size_t)(t0 + min(atid, len - 1)) * d.Hv + h];
            }
        };
        auto store_gate = [&](int jj) {
            if (atid < kChunk) {
                sm->gates[jj % 3].gam[atid] = pg;
                sm->gates[jj % 3].egam[atid] = __expf(pg);
            }
        };
        if (nch > 0) {
            fetch_gate(0);
            store_gate(0);
            fetch_gate(1);
        }
        for (int j = 0; j < nch && ok; ++j) {
            const int len = min(kChunk, sr.len - j * kChunk);
            const uint32_t abuf = (j & 1) * kABuf;
            // ---- S, W, U of chunk j have landed (the S/W/U MMAs also saw the stage land)
            ok = role_sync_and(2, wait_bar(&sm->mmaA[j & 1], (j >> 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            if (atid == 0) sm->loads_landed = j + 1;
            if (j + 1 < nch) {  // gates of chunk j+1 into their slot (chunk j-2 is fully done with it)
                store_gate(j + 1);
                fetch_gate(j + 2);
            }
            // ---- W, U -> -w and u for the chain, once it is done with chunk j-1's
            ok = role_sync_and(2, wait_ge(&ctr[kWnFree], j, abort_flag));
            if (!ok) break;
            {
                float v[32];
                tmem_ld16x256_x8(tmem + lane_base + abuf + kColW + ah * 64, v);  // columns 64 ah .. +63 of -w
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int r = half ? ar1 : ar0;
                    const uint32_t rowb = sb + kWn + r * 256 + 4 * ac;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int ch = 8 * ah + i;
                        st_shared_b32(rowb + ((ch ^ (r & 7)) << 4), pack_bf16(-v[4 * i + 2 * half], -v[4 * i + 2 * half + 1]));
                    }
                }
                float u[8];
                tmem_ld16x256_x2(tmem + lane_base + abuf + kColU + 16 * ah, u);  // columns 16 ah .. +15 of u
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int r = half ? ar1 : ar0;
                    const bool live = r < len;
#pragma unroll
                    for (int i = 0; i < 2; ++i)
                        st_shared_v2f(sb + kU + (r * 36 + 16 * ah + 8 * i + 2 * ac) * 4, live ? u[4 * i + 2 * half] : 0.f,
                                      live ? u[4 * i + 2 * half + 1] : 0.f);
                }
            }
            role_sync_and(2, true);
            if (atid == 0) publish(&ctr[kReady], j + 1);
            // ---- P = causal decay mask o S -> SW128 tile for DP, once DP of chunk j-1 is done with it
            ok = role_sync_and(2, j < 1 || wait_ge(&ctr[kODone], j, abort_flag));
            if (!ok) break;
            if (want_o) {
                const Gates &G = sm->gates[j % 3];
                float v[16];
                tmem_ld16x256_x4(tmem + lane_base + abuf + kColS + 32 * ah, v);  // key columns 32 ah .. +31
                const float gr0 = G.gam[ar0], gr1 = G.gam[ar1];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int s0 = 32 * ah + 8 * i + 2 * ac;
                    const float2 gs = *reinterpret_cast<const float2 *>(&G.gam[s0]);
                    const float x00 = s0 <= ar0 ? __expf(gr0 - gs.x) * v[4 * i] : 0.f;
                    const float x01 = s0 + 1 <= ar0 ? __expf(gr0 - gs.y) * v[4 * i + 1] : 0.f;
                    const float x10 = s0 <= ar1 ? __expf(gr1 - gs.x) * v[4 * i + 2] : 0.f;
                    const float x11 = s0 + 1 <= ar1 ? __expf(gr1 - gs.y) * v[4 * i + 3] : 0.f;
                    const int ch = 4 * ah + i;
                    st_shared_b32(sb + kP + (ar0 >> 3) * 1024 + (ar0 & 7) * 128 + ((ch ^ (ar0 & 7)) << 4) + 4 * ac,
                                  pack_bf16(x00, x01));
                    st_shared_b32(sb + kP + (ar1 >> 3) * 1024 + (ar1 & 7) * 128 + ((ch ^ (ar1 & 7)) << 4) + 4 * ac,
                                  pack_bf16(x10, x11));
                }
            }
            fence_proxy_async();
            tc_fence_before();
            role_sync_and(2, true);
            if (atid == 0) {
                publish(&ctr[kPReady], j + 1);
                publish(&ctr[kTmemA], j + 1);
            }
            // ---- output of the previous chunk
            if (j >= 1) {
                ok = role_sync_and(2, output(j - 1));
                if (!ok) break;
                if (atid == 0) publish(&ctr[kTmemO], j);
            }
        }
        if (ok && nch > 0) {
            ok = role_sync_and(2, output(nch - 1));
            if (ok && atid == 0) publish(&ctr[kTmemO], nch);
        }
        if (!ok) {
            if (atid == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        }
    } else if (warp == 16) {
        // ==================================================== MMA issuer
        if (lane == 0) {
            bool ok = true;
            for (int c = 0; c < kStages && c < nch; ++c) issue_loads(c);
            const uint32_t id_S = idesc_bf16(64, 64, false, false);
            const uint32_t id_W = idesc_bf16(64, 128, false, true);
            const uint32_t id_U = idesc_bf16(64, 32, false, true);
            for (int j = 0; j < nch && ok; ++j) {
                const uint32_t st = sb + kStage0 + (j % kStages) * kStageBytes;
                // stage landed; accumulator buffer j%2 was last read (by the aux warps) for chunk j-2
                ok = wait_bar(&sm->full[j % kStages], (j / kStages) & 1, abort_flag) &&
                     wait_ge(&ctr[kTmemA], j >= 1 ? j - 1 : 0, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t tb = tmem + (j & 1) * kABuf;
                for (int ks = 0; ks < 4; ++ks) {
                    mma_bf16(tb + kColW, smem_desc(st + kAwS + ks * 32, 16, 1024, kSw128),
                             smem_desc(st + kK + ks * 2048, 8192, 1024, kSw128), id_W, ks > 0);
                    mma_bf16(tb + kColU, smem_desc(st + kAu + ks * 32, 16, 1024, kSw128),
                             smem_desc(st + kVt + ks * 1024, 4096, 512, kSw64), id_U, ks > 0);
                }
                for (int ks = 0; ks < 8 && prm.o; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_bf16(tb + kColS, smem_desc(st + kQ + off, 16, 1024, kSw128),
                             smem_desc(st + kK + off, 16, 1024, kSw128), id_S, ks > 0);
                }
                mma_commit(&sm->mmaA[j & 1]);
            }
            if (!ok) {
                set_status(prm.status, GDN_ERR_TIMEOUT);
                *abort_flag = 1;
            }
        }
        __syncwarp();
    } else {
        // ================================================== MMA issuer B
        if (lane == 0) {
            bool ok = true;
            const uint32_t id_O = idesc_bf16(64, 32, false, true);
            int issued = min(kStages, nch);
            for (int j = 0; j < nch && ok; ++j) {
                const uint32_t st = sb + kStage0 + (j % kStages) * kStageBytes;
                ok = wait_ge(&ctr[kH], j + 1, abort_flag) && wait_ge(&ctr[kDelta], j + 1, abort_flag) &&
                     wait_ge(&ctr[kPReady], j + 1, abort_flag) && wait_ge(&ctr[kTmemO], j, abort_flag);
                if (!ok) break;
                if (!prm.o) {  // recompute for the backward: no output products
                    publish(&ctr[kODone], j + 1);
                } else {
                tc_fence_after();
                const uint32_t hb = sb + kHb + (j & 1) * 8192, db = sb + kDb + (j % 3) * 4096;
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t aoff = (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_bf16(tmem + kColQ, smem_desc(st + kQ + aoff, 16, 1024, kSw128),
                             smem_desc(hb + ks * 256, 128, 2048, kSwNone), id_O, ks > 0);
                }
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + kColP, smem_desc(sb + kP + ks * 32, 16, 1024, kSw128),
                             smem_desc(db + ks * 256, 128, 1024, kSwNone), id_O, ks > 0);
                mma_commit(&sm->mmaO);
                ok = wait_bar(&sm->mmaO, j & 1, abort_flag);
                if (!ok) break;
                tc_fence_before();
                publish(&ctr[kODone], j + 1);
                }
                // refill the stage of chunk j with chunk j + 3 once the chain is done with its k tile
                if (issued < nch) {
                    ok = wait_ge(&ctr[kStage], j + 1, abort_flag);
                    if (!ok) break;
                    issue_loads(issued);
                    ++issued;
                }
            }
            if (!ok) {
                set_status(prm.status, GDN_ERR_TIMEOUT);
                *abort_flag = 1;
            }
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        // let every TMA load still in flight land (bounded) before the CTA exits
        const uint64_t t0 = globaltimer();
        for (int c = sm->loads_landed; c < sm->loads_issued; ++c)
            while (!mbar_try_wait(smem_u32(&sm->full[c % kStages]), (c / kStages) & 1) &&
                   globaltimer() - t0 < 2000000000ull) {
            }
    }
    __syncthreads();
    if (warp == 16) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side
bool make_map(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
              const cuuint32_t *box, CUtensorMapSwizzle sw) {
    return warp::make_bf16_map(m, base, rank, dims, strides, box, sw);
}

}  // namespace

cudaError_t launch_fwd2(const FwdArgs &a) {
    const Dims &d = a.d;
    if (d.N == 0) return cudaSuccess;
    if (!a.wy) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mw;
    const cuuint64_t dq[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hq, (cuuint64_t)(d.T_total > 0 ? d.T_total : 1)};
    const cuuint64_t sq[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hq * d.K * 2};
    const cuuint32_t bq[3] = {64, 1, 64};
    const cuuint64_t dv[3] = {(cuuint64_t)d.V, (cuuint64_t)d.Hv, (cuuint64_t)(d.T_total > 0 ? d.T_total : 1)};
    const cuuint64_t sv[2] = {(cuuint64_t)d.V * 2, (cuuint64_t)d.Hv * d.V * 2};
    const cuuint32_t bv[3] = {kBV, 1, 64};
    const cuuint64_t dw[2] = {64, (cuuint64_t)(d.NC > 0 ? d.NC : 1) * d.Hv * 2 * 64};
    const cuuint64_t sw[1] = {128};
    const cuuint32_t bw[2] = {64, 64};
    if (!make_map(&mq, a.q, 3, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, a.k, 3, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, a.v, 3, dv, sv, bv, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map(&mw, a.wy, 2, dw, sw, bw, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    Fwd2Params p;
    p.d = d;
    p.gamma = a.gamma;
    p.h0 = a.h0;
    p.o = (__nv_bfloat16 *)a.o;
    p.final_state = a.final_state;
    p.h_chunks = (__nv_bfloat16 *)a.h_chunks16;
    p.delta = (__nv_bfloat16 *)a.delta16;
    p.nseg = a.nseg > 0 ? a.nseg : 1;
    p.mode = a.fwd_mode;
    p.seg_h0 = a.seg_h0;
    p.seg_c = a.seg_c;
    p.seg_P = a.seg_P;
    if (p.mode != kWhole && (p.nseg < 1 || (p.mode == kSegOut && !p.seg_h0) ||
                             (p.mode == kSegPass && (!p.seg_c || !p.seg_P || p.o))))
        return cudaErrorInvalidValue;
    p.status = a.status;
    cudaError_t e = cudaFuncSetAttribute(fwd2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    // the segment pass also carries the K operator columns
    dim3 grid(d.N * p.nseg, d.Hv, (d.V + (p.mode == kSegPass ? d.K : 0)) / kBV);
    fwd2_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mk, mv, mw, p);
    return cudaGetLastError();
}

}  // namespace gdn
