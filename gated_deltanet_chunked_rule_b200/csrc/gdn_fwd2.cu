// gdn_fwd2.cu -- chunked forward of the gated delta rule (bf16, K = V = 128):
// the sequential state chain on warp-level tensor-core MMAs, the output on
// tcgen05. Everything that does not depend on the state (w, u and the
// decay-masked P = M o Q K^T of every chunk) comes ready-made from the
// chunk-prep kernel (gdn_prep3.cu) through a TMA ring.
//
// One CTA per (sequence or segment, value head, 32-column slice of V). Per
// 64-token chunk (h the chunk-entry state, h = S^T, notation of gdn_internal.cuh):
//
//   chain (mma.sync, fp32 state in registers):
//     Delta = u - w h,     h <- e^{gamma_C} h + K^T (e^{gamma_C - gamma} o Delta)
//   output (tcgen05, TMEM accumulators, one chunk behind the chain):
//     DQ = Q h,  DP = P Delta,   o = scale (e^gamma o DQ + DP)
//
// Why this split (measured on B200): a tcgen05 MMA takes ~450 cycles from
// issue to a completed mbarrier, and the chain has two dependent products per
// chunk, whereas a dependent mma.sync costs ~20 cycles; the output products do
// not feed the chain, so they run on tcgen05 off the critical path. Shared
// memory bandwidth (128 B/clk/SM) is the next limit, which is why every
// state-independent product is hoisted into the prep kernel.
//
// Warp roles (416 threads):
//   warps 0-7   chain: h (128 x 32 fp32) in mma fragments, warp w holding
//               state rows 32 (w % 4) .. +31 and columns 16 (w / 4) .. +15.
//   warps 8-11  epilogue: o from the double-buffered DQ/DP accumulators;
//               warp 8 + q reads TMEM lanes 32 q .. +31 (rows 16 q .. +15).
//   warp 12     issuer: 3-deep TMA ring (q, k, w, u, P per chunk) and the
//               DQ/DP MMAs.
// Roles hand over through monotonically increasing shared-memory counters
// (release/acquire), which cannot alias the way mbarrier parities can when a
// producer runs ahead; mbarriers only where the hardware signals (TMA
// completion, tcgen05.commit). Every wait is bounded in time; a wait that
// expires records GDN_ERR_TIMEOUT and winds the CTA down.
//
// Modes: whole sequences from h0; the recompute for the backward (no output,
// stores every chunk's entry state and Delta in bf16); and the two passes of
// the sequence split (see Fwd2Mode).
#include <cstddef>

#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kThreads = 416;  // 8 chain + 4 epilogue + 1 issuer warps
constexpr int kRole = 256;     // chain threads
constexpr int kEpi = 128;      // epilogue threads
constexpr int kBV = 32;
constexpr int kStages = 3;

// ---- shared memory (bytes from a 1024-aligned base)
constexpr int kHb = 0;          // 2 x 8192   h (bf16): (n/8)*2048 + (k/8)*128 + (k%8)*16 (k = state row)
constexpr int kDb = 16384;      // 2 x 4096   Delta (bf16), same layout with k = token (B of DP)
constexpr int kDt = 24576;      // 4096       e^{gamma_C - gamma} Delta, chain only
constexpr int kStage0 = 28672;  // TMA ring
// per stage: q [64][128] bf16 and k, w likewise (two 64-column halves, 128-byte
// swizzle), u [64][32] fp32 (128-byte swizzle), P [64][64] bf16 (128-byte swizzle)
constexpr int kQ = 0, kK = 16384, kW = 32768, kU = 49152, kP = 57344, kStageBytes = 65536;
constexpr int kTxFull = 65536;                  // q, k, w, u, P
constexpr int kTxChain = 16384 + 16384 + 8192;  // k, w, u (no output)
constexpr int kSmall = kStage0 + kStages * kStageBytes;
constexpr int kSmemBytes = kSmall + 2048 + 1024;
static_assert(kStage0 % 1024 == 0 && kStageBytes % 1024 == 0 && kSmemBytes <= 232448, "shared memory layout");

// DQ, DP double-buffered in tensor memory: buffer b at columns 64 b.
constexpr uint32_t kColQ = 0, kColP = 32, kOBuf = 64, kTmemCols = 128;

// Hand-over counters (the number of chunks, or states, the producer has finished).
enum Ctr { kH, kDelta, kStage, kODone, kTmemO, kStored, kNumCtr };

struct Small {
    uint64_t full[kStages];
    uint64_t mmaO[2];
    uint32_t ctr[kNumCtr];
    int loads_issued, loads_landed, mma_issued, mma_seen;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Small) <= 2048, "small area");

__device__ __forceinline__ bool chain_sync(bool pred) { return role_sync_and<kRole>(1, pred); }
__device__ __forceinline__ bool epi_sync(bool pred) { return role_sync_and<kEpi>(2, pred); }

// kWhole: one CTA column per sequence, from h0.
// kSegPass: per segment, the chain on [c | P] with c from zero (V columns, u as
//   input) and P from the identity (K more columns, whose u tile is read out of
//   range and so is zero): the segment maps a start state h to P h + c.
// kSegOut: per segment, the chain and the output from the composed start state.
enum Fwd2Mode { kWhole = 0, kSegPass = 1, kSegOut = 2 };

struct Fwd2Params {
    Dims d;
    const float *gamma;   // [T_total, Hv]
    const float *h0;      // [N, Hv, K, V] or null
    __nv_bfloat16 *o;     // [T_total, Hv, V], or null: no output (the backward's recompute)
    float *final_state;   // [N, Hv, K, V] or null
    __nv_bfloat16 *h_chunks;  // [NC, Hv, K, V] entry state of every chunk (bf16, as the products read it) or null
    __nv_bfloat16 *delta;     // [T_total, Hv, V] Delta (bf16) or null
    // Sequence split: blockIdx.x = sequence * nseg + segment; a segment is a
    // contiguous run of ceil(chunks / nseg) chunks of its sequence.
    int nseg;
    int mode;             // Fwd2Mode
    const float *seg_h0;  // kSegOut: [N * nseg, Hv, K, V] start state of every segment
    float *seg_c;         // kSegPass: [N * nseg, Hv, K, V] end state from a zero start
    float *seg_P;         // kSegPass: [N * nseg, Hv, K, K] transition operator of the segment
    unsigned *status;
};

__global__ void __launch_bounds__(kThreads, 1)
fwd2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_u,
            const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_hs,
            const __grid_constant__ CUtensorMap tm_ds, const Fwd2Params prm) {
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
    const bool want_o = prm.o != nullptr;
    // chunk entry states and Delta go to global memory by TMA stores from kHb / kDb
    const bool states = prm.h_chunks != nullptr;
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
        mbar_init(&sm->mmaO[0], 1);
        mbar_init(&sm->mmaO[1], 1);
        for (int c = 0; c < kNumCtr; ++c) sm->ctr[c] = 0;
        sm->loads_issued = sm->loads_landed = sm->mma_issued = sm->mma_seen = 0;
        sm->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 12) {
        tmem_alloc(&sm->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;
    uint32_t *ctr = sm->ctr;

    // gamma of chunk j at in-chunk row r (rows past the end repeat the last live one)
    auto gamma_at = [&](int j, int r) {
        const int len = min(kChunk, sr.len - j * kChunk);
        return prm.gamma[(size_t)(sr.start + j * kChunk + min(r, len - 1)) * d.Hv + h];
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
        bool ok = chain_sync(true);
        if (tid == 0) publish(&ctr[kH], 1);  // h_0
        // gates of the current chunk, prefetched one chunk ahead
        float gl = 0.f, gt0 = 0.f, gt1 = 0.f;
        if (nch > 0) gl = gamma_at(0, 63), gt0 = gamma_at(0, 16 * p + g), gt1 = gamma_at(0, 16 * p + g + 8);

        for (int j = 0; j < nch && ok; ++j) {
            const int len = min(kChunk, sr.len - j * kChunk);
            const uint32_t st = sb + kStage0 + (j % kStages) * kStageBytes;
            ok = chain_sync(wait_bar(&sm->full[j % kStages], (j / kStages) & 1, abort_flag));
            if (!ok) break;
            if (tid == 0) sm->loads_landed = j + 1;
            const float gC = gl, gtok[2] = {gt0, gt1};
            if (j + 1 < nch) gl = gamma_at(j + 1, 63), gt0 = gamma_at(j + 1, 16 * p + g), gt1 = gamma_at(j + 1, 16 * p + g + 8);
            // ---- w h : tokens 16p..16p+15, columns of n-tiles cb, cb+1 (A = w tile, B = h)
            float acc[2][4] = {};
            {
                // all of this warp's w fragments up front (they do not depend on h),
                // the h fragments streamed three k-steps ahead
                const uint32_t wt = st + kW;
                const uint32_t hb = sb + kHb + (j & 1) * 8192;
                const int arow = 16 * p + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int mi = lane >> 3;
                uint32_t a[8][4], b[4][4];
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const int d0 = 16 * ks + (lane >> 4) * 8;
                    ldsm_x4(a[ks], wt + (d0 >> 6) * 8192 + arow * 128 + ((((d0 & 63) >> 3) ^ (arow & 7)) << 4));
                }
                auto load_b = [&](int ks) {
                    ldsm_x4_t(b[ks & 3], hb + (cb + (mi >> 1)) * 2048 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
                };
                load_b(0);
                load_b(1);
                load_b(2);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    if (ks + 3 < 8) load_b(ks + 3);
                    hmma(acc[0], a[ks], b[ks & 3][0], b[ks & 3][1]);
                    hmma(acc[1], a[ks], b[ks & 3][2], b[ks & 3][3]);
                }
            }
            // K^T fragments of the state update (independent of the chain): issued now so that
            // their latency overlaps the Delta step. A = K^T rows (state rows) 32p+16mt..,
            // cols (tokens) 16ks..: 8x8 blocks of the token-major, 128-byte-swizzled k tile
            // read transposed.
            uint32_t ka[4][2][4];
            {
                const uint32_t kt = st + kK;
                const int mi = lane >> 3;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        const int tt = 16 * ks + (lane & 7) + ((mi >> 1) & 1) * 8;
                        const int dd = 32 * p + 16 * mt + (mi & 1) * 8;
                        ldsm_x4_t(ka[ks][mt], kt + (dd >> 6) * 8192 + tt * 128 + ((((dd & 63) >> 3) ^ (tt & 7)) << 4));
                    }
            }
            // ---- Delta = u - w h -> Db[j%2] (read by DP) ; e^{gamma_C - gamma} Delta -> Dt
            // DP and the state store of chunk j-2 read Db[j%2]
            ok = chain_sync(j < 2 || ((!want_o || wait_ge(&ctr[kODone], j - 1, abort_flag)) &&
                                      (!states || wait_ge(&ctr[kStored], j - 1, abort_flag))));
            if (!ok) break;
            {
                const uint32_t db = sb + kDb + (j & 1) * 4096 + c4 * 4, dt = sb + kDt + c4 * 4;
                const float *ut = reinterpret_cast<const float *>(smem + kStage0 + (j % kStages) * kStageBytes + kU);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int tok = 16 * p + g + half * 8;
                    const bool live = tok < len;
                    const float sc = __expf(gC - gtok[half]);
                    const uint32_t off = (tok >> 3) * 128 + (tok & 7) * 16;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int col = 8 * (cb + nt) + 2 * c4;  // u tile: 32 fp32 per row, 16-B chunks XOR (row % 8)
                        const float2 uu = *reinterpret_cast<const float2 *>(
                            ut + tok * 32 + ((((col >> 2) ^ (tok & 7))) << 2) + (col & 3));
                        const float x0 = live ? uu.x - acc[nt][2 * half] : 0.f;
                        const float x1 = live ? uu.y - acc[nt][2 * half + 1] : 0.f;
                        st_shared_b32(db + (cb + nt) * 1024 + off, pack_bf16(x0, x1));
                        st_shared_b32(dt + (cb + nt) * 1024 + off, pack_bf16(sc * x0, sc * x1));
                        if (states && len < kChunk && live)  // ragged last chunk: no TMA store past its end
                            *reinterpret_cast<uint32_t *>(prm.delta + ((size_t)(sr.start + j * kChunk + tok) * d.Hv + h) * V +
                                                          c0 + col) = pack_bf16(x0, x1);
                    }
                }
            }
            chain_sync(true);  // every warp reads all 64 tokens of Dt below
            // ---- h <- e^{gamma_C} h + K^T Dt : rows 32p..32p+31, 16 columns, K = 64 tokens
            {
                const float eC = __expf(gC);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int q = 0; q < 4; ++q) hf[mt][nt][q] *= eC;
                const int mi = lane >> 3;
                uint32_t b[4][4];
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    ldsm_x4_t(b[ks], sb + kDt + (cb + (mi >> 1)) * 1024 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        hmma(hf[mt][0], ka[ks][mt], b[ks][0], b[ks][1]);
                        hmma(hf[mt][1], ka[ks][mt], b[ks][2], b[ks][3]);
                    }
            }
            chain_sync(true);
            if (tid == 0) publish(&ctr[kStage], j + 1);
            // ---- h_{j+1} -> Hb[(j+1)%2] once DQ of chunk j-1 (which read it) is done; then
            //      Delta_j and h_{j+1} go to the output MMAs behind one proxy fence
            // DQ and the state store of chunk j-1 read Hb[(j+1)%2]
            ok = chain_sync(j < 1 || ((!want_o || wait_ge(&ctr[kODone], j, abort_flag)) &&
                                      (!states || wait_ge(&ctr[kStored], j, abort_flag))));
            if (!ok) break;
            write_hb((j + 1) & 1);
            fence_proxy_async();
            chain_sync(true);
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
    } else if (warp < 12) {
        // ======================================================== epilogue
        if (want_o) {
            const int et = tid - kRole, q = warp & 3;  // TMEM lanes 32q.. = rows 16q..16q+15
            const uint32_t lane_base = (uint32_t)(q * 32) << 16;
            const int eg = lane >> 2, ec = lane & 3;
            const int rr[2] = {16 * q + eg, 16 * q + eg + 8};
            const float scl = d.scale;
            bool ok = true;
            for (int j = 0; j < nch && ok; ++j) {
                const int len = min(kChunk, sr.len - j * kChunk);
                const float g0 = gamma_at(j, rr[0]), g1 = gamma_at(j, rr[1]);
                ok = epi_sync(wait_bar(&sm->mmaO[j & 1], (j >> 1) & 1, abort_flag));
                if (!ok) break;
                if (et == 0) {
                    sm->mma_seen = j + 1;
                    publish(&ctr[kODone], j + 1);
                }
                tc_fence_after();
                float dq[16], dp[16];
                const uint32_t tb = tmem + lane_base + (j & 1) * kOBuf;
                tmem_ld16x256_x4(tb + kColQ, dq);
                tmem_ld16x256_x4(tb + kColP, dp);
                tc_fence_before();
                epi_sync(true);
                if (et == 0) publish(&ctr[kTmemO], j + 1);
                const float er[2] = {__expf(g0), __expf(g1)};
                const int t0 = sr.start + j * kChunk;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (rr[half] < len) {
                        __nv_bfloat16 *dst = prm.o + ((size_t)(t0 + rr[half]) * d.Hv + h) * V + c0 + 2 * ec;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int k = 4 * i + 2 * half;
                            *reinterpret_cast<uint32_t *>(dst + 8 * i) =
                                pack_bf16(scl * fmaf(er[half], dq[k], dp[k]), scl * fmaf(er[half], dq[k + 1], dp[k + 1]));
                        }
                    }
                }
            }
            if (!ok) {
                if (et == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
                *abort_flag = 1;
            }
        }
    } else {
        // ========================================================== issuer
        if (lane == 0) {
            bool ok = true;
            auto issue_loads = [&](int j) {
                const int s = j % kStages;
                uint8_t *stg = smem + kStage0 + s * kStageBytes;
                const int t0 = sr.start + j * kChunk;
                const int cg = sr.chunk0 + j;
                mbar_arrive_expect_tx(&sm->full[s], want_o ? kTxFull : kTxChain);
                atomicAdd(&sm->loads_issued, 1);
                if (want_o) {
                    tma_load_3d(stg + kQ, &tm_q, &sm->full[s], 0, hq, t0);
                    tma_load_3d(stg + kQ + 8192, &tm_q, &sm->full[s], 64, hq, t0);
                    tma_load_2d(stg + kP, &tm_p, &sm->full[s], 0, (cg * d.Hv + h) * kChunk);
                }
                tma_load_3d(stg + kK, &tm_k, &sm->full[s], 0, hq, t0);
                tma_load_3d(stg + kK + 8192, &tm_k, &sm->full[s], 64, hq, t0);
                tma_load_3d(stg + kW, &tm_w, &sm->full[s], 0, h, t0);
                tma_load_3d(stg + kW + 8192, &tm_w, &sm->full[s], 64, h, t0);
                tma_load_3d(stg + kU, &tm_u, &sm->full[s], c0, h, t0);  // out of range (zero) for operator columns
            };
            for (int c = 0; c < kStages && c < nch; ++c) issue_loads(c);
            const uint32_t id_O = idesc_bf16(64, 32, false, true);
            for (int j = 0; j < nch && ok; ++j) {
                // refill the stage of chunk j-1 with chunk j+2 once the chain and DQ/DP are done with it
                if (j >= 1 && j + 2 < nch) {
                    ok = wait_ge(&ctr[kStage], j, abort_flag) && (!want_o || wait_ge(&ctr[kODone], j, abort_flag));
                    if (!ok) break;
                    issue_loads(j + 2);
                }
                if (!want_o && !states) continue;
                // h_j and Delta_j are in kHb[j%2], kDb[j%2]
                ok = wait_ge(&ctr[kH], j + 1, abort_flag) && wait_ge(&ctr[kDelta], j + 1, abort_flag);
                if (!ok) break;
                if (states) {
                    // entry state (four 8-column boxes of 128 rows) and, for a full chunk, Delta
                    const int len = min(kChunk, sr.len - j * kChunk);
                    const uint32_t hb = sb + kHb + (j & 1) * 8192, db = sb + kDb + (j & 1) * 4096;
                    const int row = ((sr.chunk0 + j) * d.Hv + h) * K;
                    for (int nb = 0; nb < 4; ++nb) {
                        tma_store_2d(&tm_hs, hb + nb * 2048, c0 + 8 * nb, row);
                        if (len == kChunk) tma_store_3d(&tm_ds, db + nb * 1024, c0 + 8 * nb, h, sr.start + j * kChunk);
                    }
                    bulk_commit();
                    bulk_wait_read<0>();
                    publish(&ctr[kStored], j + 1);
                }
                if (!want_o) continue;
                // DQ = Q h_j, DP = P Delta_j into buffer j%2 once the epilogue has read chunk j-2's
                ok = wait_ge(&ctr[kTmemO], j >= 1 ? j - 1 : 0, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = sb + kStage0 + (j % kStages) * kStageBytes;
                const uint32_t hb = sb + kHb + (j & 1) * 8192, db = sb + kDb + (j & 1) * 4096;
                const uint32_t tb = tmem + (j & 1) * kOBuf;
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t aoff = (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_bf16(tb + kColQ, smem_desc(st + kQ + aoff, 16, 1024, kSw128),
                             smem_desc(hb + ks * 256, 128, 2048, kSwNone), id_O, ks > 0);
                }
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tb + kColP, smem_desc(st + kP + ks * 32, 16, 1024, kSw128),
                             smem_desc(db + ks * 256, 128, 1024, kSwNone), id_O, ks > 0);
                mma_commit(&sm->mmaO[j & 1]);
                sm->mma_issued = j + 1;
            }
            if (!ok) {
                set_status(prm.status, GDN_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            bulk_wait_all();  // state stores complete before the CTA's shared memory goes away
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        // let every TMA load still in flight land (bounded) before the CTA exits
        const uint64_t t0 = globaltimer();
        for (int c = sm->loads_landed; c < sm->loads_issued; ++c)
            while (!mbar_try_wait(smem_u32(&sm->full[c % kStages]), (c / kStages) & 1) && globaltimer() - t0 < kWaitNs) {
            }
        for (int c = sm->mma_seen; c < sm->mma_issued; ++c)  // and every output MMA
            while (!mbar_try_wait(smem_u32(&sm->mmaO[c & 1]), (c >> 1) & 1) && globaltimer() - t0 < kWaitNs) {
            }
    }
    __syncthreads();
    if (warp == 12) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, int rank, const cuuint64_t *dims,
              const cuuint64_t *strides, const cuuint32_t *box,
              CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, rank, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_fwd2(const FwdArgs &a) {
    const Dims &d = a.d;
    if (d.N == 0) return cudaSuccess;
    if (!a.w16 || !a.u32 || (a.o && !a.p16)) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mw, mu, mp, mhs, mds;
    const cuuint64_t T = (cuuint64_t)(d.T_total > 0 ? d.T_total : 1);
    const cuuint64_t dq[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hq, T};
    const cuuint64_t sq[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hq * d.K * 2};
    const cuuint32_t b64[3] = {64, 1, 64};
    const cuuint64_t dw[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hv, T};
    const cuuint64_t sw[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hv * d.K * 2};
    const cuuint64_t du[3] = {(cuuint64_t)d.V, (cuuint64_t)d.Hv, T};
    const cuuint64_t su[2] = {(cuuint64_t)d.V * 4, (cuuint64_t)d.Hv * d.V * 4};
    const cuuint32_t bu[3] = {kBV, 1, 64};
    const cuuint64_t dp[2] = {64, (cuuint64_t)(d.NC > 0 ? d.NC : 1) * d.Hv * 64};
    const cuuint64_t sp[1] = {128};
    const cuuint32_t bp[2] = {64, 64};
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    if (!make_map(&mq, BF, a.q, 3, dq, sq, b64) || !make_map(&mk, BF, a.k, 3, dq, sq, b64) ||
        !make_map(&mw, BF, a.w16, 3, dw, sw, b64) || !make_map(&mu, F32, a.u32, 3, du, su, bu) ||
        !make_map(&mp, BF, a.p16 ? a.p16 : a.w16, 2, dp, sp, bp))
        return cudaErrorInvalidValue;
    // state stores: entry states as [NC * Hv * K rows][V], Delta as [T][Hv][V]; 16-byte boxes
    const bool st = a.h_chunks16 != nullptr;
    if (st != (a.delta16 != nullptr)) return cudaErrorInvalidValue;
    const cuuint64_t dhs[2] = {(cuuint64_t)d.V, (cuuint64_t)(d.NC > 0 ? d.NC : 1) * d.Hv * d.K};
    const cuuint64_t shs[1] = {(cuuint64_t)d.V * 2};
    const cuuint32_t bhs[2] = {8, 128};
    const cuuint64_t dds[3] = {(cuuint64_t)d.V, (cuuint64_t)d.Hv, T};
    const cuuint64_t sds[2] = {(cuuint64_t)d.V * 2, (cuuint64_t)d.Hv * d.V * 2};
    const cuuint32_t bds[3] = {8, 1, 64};
    if (!make_map(&mhs, BF, st ? a.h_chunks16 : a.w16, 2, dhs, shs, bhs, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mds, BF, st ? a.delta16 : a.w16, 3, dds, sds, bds, CU_TENSOR_MAP_SWIZZLE_NONE))
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
    if (p.mode != kWhole && ((p.mode == kSegOut && !p.seg_h0) ||
                             (p.mode == kSegPass && (!p.seg_c || !p.seg_P || p.o || p.h_chunks || p.delta))))
        return cudaErrorInvalidValue;
    p.status = a.status;
    cudaError_t e = cudaFuncSetAttribute(fwd2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    // the segment pass also carries the K operator columns
    dim3 grid(d.N * p.nseg, d.Hv, (d.V + (p.mode == kSegPass ? d.K : 0)) / kBV);
    fwd2_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mk, mw, mu, mp, mhs, mds, p);
    return cudaGetLastError();
}

}  // namespace gdn
