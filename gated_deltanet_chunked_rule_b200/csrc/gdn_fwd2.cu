// gdn_fwd2.cu -- chunked forward of the gated delta rule (bf16, K = V = 128):
// the sequential state chain on warp-level tensor-core MMAs, the output on
// tcgen05. Everything that does not depend on the state (w, u and the
// decay-masked P = M o Q K^T of every chunk) comes ready-made from the
// chunk-prep kernel (gdn_prep3.cu) through TMA rings.
//
// One CTA per (sequence or segment, value head, 32-column slice of V). Per
// 64-token chunk (h the chunk-entry state, h = S^T, notation of gdn_internal.cuh):
//
//   chain (mma.sync, fp32 state in registers):
//     Delta = u - w h,     h <- e^{gamma_C} h + K^T (e^{gamma_C - gamma} o Delta)
//   output (tcgen05, TMEM accumulators, behind the chain):
//     DQ = Q h,  DP = P Delta,   o = scale (e^gamma o DQ + DP)
//
// Why this split (measured on B200): a tcgen05 MMA takes ~450 cycles from
// issue to a completed mbarrier, and the chain has two dependent products per
// chunk, whereas a dependent mma.sync costs ~20 cycles; the output products do
// not feed the chain, so they run on tcgen05 off the critical path. A chain
// warp's shared-memory reads are limited by its own issue rate (one
// ldmatrix.x4 per ~8.6 cycles), which is why every state-independent product
// is hoisted into the prep kernel, and why each chain warp owns whole rows:
// the w and K^T fragments are read once per chunk.
//
// Warp roles (320 threads):
//   warps 0-3   chain: h (128 x 32 fp32) in mma fragments, warp p holding
//               state rows 32p .. +31 (all 32 columns). The w and K^T
//               fragments and the u values of chunk j+1 are loaded into
//               registers while chunk j updates the state, so a chunk's
//               critical path only reads h and e^{gamma_C - gamma} Delta from
//               shared memory. Two barriers per chunk.
//   warps 4-7   epilogue: o from the double-buffered DQ/DP accumulators;
//               warp 4 + q reads TMEM lanes 32 q .. +31 (rows 16 q .. +15),
//               stages its rows of o in shared memory, and one TMA store per
//               full chunk writes them (fewer stores beside the chain warps;
//               a ragged last chunk is stored directly, row by row).
//   warp 8      output issuer: the DQ/DP MMAs and the (q, P) TMA ring.
//   warp 9      chain producer: the (k, w, u) TMA ring, refilled as soon as the
//               chain has a stage in registers, and the bulk copies of the
//               chunk states and Delta to global memory (in parallel with the
//               output products, since the chain reuses kHb / kDb once both
//               are done).
// Roles hand over through monotonically increasing shared-memory counters
// (release/acquire; one thread polls, a barrier passes it on), which cannot
// alias the way mbarrier parities can when a producer runs ahead; mbarriers
// only where the hardware signals (TMA completion, tcgen05.commit). Every
// wait is bounded in time; a wait that expires records GDN_ERR_TIMEOUT and
// winds the CTA down.
//
// Modes: whole sequences from h0; the recompute for the backward (no output,
// stores every chunk's entry state and Delta in bf16); and the two passes of
// the sequence split (see Fwd2Mode).
//
// Saved states and Delta are kept in the shared-memory tile layout, one
// contiguous block per (chunk, value head, 32-column slice), so that each is
// one bulk copy: entry state h [NC][Hv][V/32][4][128][8] (block of 8 columns
// n/8, state row k, 8 columns), Delta [NC][Hv][V/32][4][64][8] (token rows; rows
// past a ragged chunk's end are zero). These blocks are K-major operand tiles
// without swizzle for the backward's products.
#include <cstddef>

#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kThreads = 320;  // 4 chain + 4 epilogue + output issuer + chain producer
constexpr int kRole = 128;     // chain threads
constexpr int kEpi = 128;      // epilogue threads
constexpr int kBV = 32;
constexpr int kStages = 3;

// ---- shared memory (bytes from a 1024-aligned base)
constexpr int kHb = 0;          // 2 x 8192   h (bf16): (n/8)*2048 + (k/8)*128 + (k%8)*16 (k = state row)
constexpr int kDb = 16384;      // 2 x 4096   Delta (bf16), same layout with k = token (B of DP)
constexpr int kDt = 24576;      // 4096       e^{gamma_C - gamma} Delta, chain only
constexpr int kC0 = 28672;      // chain ring: k, w [64][128] bf16 (two 64-column halves,
                                // 128-byte swizzle), u [64][32] fp32 (128-byte swizzle)
constexpr int kK = 0, kW = 16384, kU = 32768, kCStageBytes = 40960;
constexpr int kO0 = kC0 + kStages * kCStageBytes;  // output ring: q [64][128] bf16, P [64][64] bf16
constexpr int kQ = 0, kP = 16384, kOStageBytes = 24576;
constexpr int kSmall = kO0 + kStages * kOStageBytes;
constexpr int kOs = kSmall + 2048;  // o of a full chunk, staged for its TMA store: [64][32] bf16
constexpr int kSmemBytes = kOs + 4096 + 1024;
static_assert(kC0 % 1024 == 0 && kO0 % 1024 == 0 && kCStageBytes % 1024 == 0 && kOStageBytes % 1024 == 0 &&
                  kSmemBytes <= 232448,
              "shared memory layout");

// DQ, DP double-buffered in tensor memory: buffer b at columns 64 b.
constexpr uint32_t kColQ = 0, kColP = 32, kOBuf = 64, kTmemCols = 128;

// Hand-over counters (the number of chunks, or states, the producer has finished).
// kChain, one release store per chunk: 1 once h_0 is in kHb and chunk 0's stage is
// in registers, then j + 2 after chunk j (Delta_j in kDb, h_{j+1} in kHb, chunk
// j+1's stage in registers). kODone chunks whose DQ/DP are complete, kTmemO chunks
// whose accumulators are read, kStored chunks whose state copies have read kHb / kDb.
enum Ctr { kChain, kODone, kTmemO, kStored, kNumCtr };

struct Small {
    uint64_t cfull[kStages], ofull[kStages];
    uint64_t mmaO[2];
    uint32_t ctr[kNumCtr];
    int cl_issued, cl_landed, ol_issued, ol_landed, mma_issued, mma_seen;
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
    __nv_bfloat16 *h_chunks;  // entry state of every chunk (bf16, as the products read it; blocked) or null
    __nv_bfloat16 *delta;     // Delta of every chunk (bf16; blocked) or null
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
            const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_o,
            const Fwd2Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
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
    // chunk entry states and Delta go to global memory by bulk copies from kHb / kDb
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
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm->cfull[s], 1);
            mbar_init(&sm->ofull[s], 1);
        }
        mbar_init(&sm->mmaO[0], 1);
        mbar_init(&sm->mmaO[1], 1);
        for (int c = 0; c < kNumCtr; ++c) sm->ctr[c] = 0;
        sm->cl_issued = sm->cl_landed = sm->ol_issued = sm->ol_landed = sm->mma_issued = sm->mma_seen = 0;
        sm->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 8) {
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

    if (warp < 4) {
        // =========================================================== chain
        const int p = warp;  // state rows 32p.., tokens 16p.. of the w h product
        const int g = lane >> 2, c4 = lane & 3, mi = lane >> 3;
        float hf[2][4][4];  // [m-tile][n-tile][frag]: rows 32p+16mt+g(+8), cols 8nt+2c4(+1)
        {
            const float *src = prm.mode == kWhole ? (prm.h0 ? prm.h0 + ((size_t)n * d.Hv + h) * K * V : nullptr)
                               : prm.mode == kSegOut ? prm.seg_h0 + (seg_idx * d.Hv + h) * K * V
                                                     : nullptr;
            const bool ident = prm.mode == kSegPass && c0 >= V;  // operator columns start as I
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int dim = 32 * p + 16 * mt + g + ((q >> 1) << 3);
                        const int col = 8 * nt + 2 * c4 + (q & 1);
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
                    for (int nt = 0; nt < 4; ++nt)
                        st_shared_b32(base + nt * 2048 + (dim >> 3) * 128 + (dim & 7) * 16,
                                      pack_bf16(hf[mt][nt][2 * half], hf[mt][nt][2 * half + 1]));
                }
        };
        // Registers of the coming chunk: w fragments (A of w h: tokens 16p.., all
        // 128 state rows), K^T fragments (A of the update: state rows 32p.., 64
        // tokens), u at this thread's (token, column) pairs.
        uint32_t wa[8][4], ka[4][2][4];
        float2 uu[2][4];
        auto load_chunk_regs = [&](int j) {
            const uint32_t st = sb + kC0 + (j % kStages) * kCStageBytes;
            const int arow = 16 * p + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int d0 = 16 * ks + (lane >> 4) * 8;
                ldsm_x4(wa[ks], st + kW + (d0 >> 6) * 8192 + arow * 128 + ((((d0 & 63) >> 3) ^ (arow & 7)) << 4));
            }
            // u tile: 32 fp32 per row, 16-byte chunks XOR (row % 8)
            const float *ut = reinterpret_cast<const float *>(smem + kC0 + (j % kStages) * kCStageBytes + kU);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int tok = 16 * p + g + half * 8;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const int col = 8 * nt + 2 * c4;
                    uu[half][nt] = *reinterpret_cast<const float2 *>(ut + tok * 32 + (((col >> 2) ^ (tok & 7)) << 2) + (col & 3));
                }
            }
        };
        auto load_chunk_ka = [&](int j) {
            // K^T rows (state rows) 32p+16mt.., cols (tokens) 16ks..: 8x8 blocks of the
            // token-major, 128-byte-swizzled k tile read transposed
            const uint32_t kt = sb + kC0 + (j % kStages) * kCStageBytes + kK;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    const int tt = 16 * ks + (lane & 7) + ((mi >> 1) & 1) * 8;
                    const int dd = 32 * p + 16 * mt + (mi & 1) * 8;
                    ldsm_x4_t(ka[ks][mt], kt + (dd >> 6) * 8192 + tt * 128 + ((((dd & 63) >> 3) ^ (tt & 7)) << 4));
                }
        };
        write_hb(0);
        fence_proxy_async();
        bool ok = true;
        if (nch > 0) {
            ok = wait_bar(&sm->cfull[0], 0, abort_flag);
            if (ok) {
                load_chunk_regs(0);
                load_chunk_ka(0);
            }
        }
        ok = chain_sync(ok);
        if (tid == 0) {
            sm->cl_landed = nch > 0 ? 1 : 0;
            publish(&ctr[kChain], 1);  // h_0; chunk 0's stage is in registers
        }
        // gates of the current chunk and of the next, prefetched ahead
        float gl = 0.f, gt0 = 0.f, gt1 = 0.f;
        if (nch > 0) gl = gamma_at(0, 63), gt0 = gamma_at(0, 16 * p + g), gt1 = gamma_at(0, 16 * p + g + 8);

        for (int j = 0; j < nch && ok; ++j) {
            const int len = min(kChunk, sr.len - j * kChunk);
            const float gC = gl, gtok[2] = {gt0, gt1};
            if (j + 1 < nch) gl = gamma_at(j + 1, 63), gt0 = gamma_at(j + 1, 16 * p + g), gt1 = gamma_at(j + 1, 16 * p + g + 8);
            // ---- w h : tokens 16p..16p+15, all 32 columns (A = w fragments, B = h from kHb)
            float acc[4][4] = {};
            {
                const uint32_t hb = sb + kHb + (j & 1) * 8192;
                uint32_t b[3][2][4];
                auto load_b = [&](int ks) {
#pragma unroll
                    for (int np = 0; np < 2; ++np)
                        ldsm_x4_t(b[ks % 3][np], hb + (2 * np + (mi >> 1)) * 2048 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
                };
                load_b(0);
                load_b(1);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    if (ks + 2 < 8) load_b(ks + 2);
#pragma unroll
                    for (int np = 0; np < 2; ++np) {
                        hmma(acc[2 * np], wa[ks], b[ks % 3][np][0], b[ks % 3][np][1]);
                        hmma(acc[2 * np + 1], wa[ks], b[ks % 3][np][2], b[ks % 3][np][3]);
                    }
                }
            }
            // ---- Delta = u - w h -> Db[j%2] (read by DP and the state store) ; e^{gamma_C - gamma} Delta -> Dt
            {
                const uint32_t db = sb + kDb + (j & 1) * 4096 + c4 * 4, dt = sb + kDt + c4 * 4;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int tok = 16 * p + g + half * 8;
                    const bool live = tok < len;
                    const float sc = __expf(gC - gtok[half]);
                    const uint32_t off = (tok >> 3) * 128 + (tok & 7) * 16;
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) {
                        const float x0 = live ? uu[half][nt].x - acc[nt][2 * half] : 0.f;
                        const float x1 = live ? uu[half][nt].y - acc[nt][2 * half + 1] : 0.f;
                        st_shared_b32(db + nt * 1024 + off, pack_bf16(x0, x1));
                        st_shared_b32(dt + nt * 1024 + off, pack_bf16(sc * x0, sc * x1));
                    }
                }
            }
            // every warp reads all 64 tokens of Dt below; the stage of chunk j+1 has landed;
            // kHb[(j+1)%2] (written below) and kDb[(j+1)%2] (written in chunk j+1) are free once
            // the outputs and state stores of chunk j-1 are done
            ok = chain_sync((j + 1 >= nch || wait_bar(&sm->cfull[(j + 1) % kStages], ((j + 1) / kStages) & 1, abort_flag)) &&
                            (tid != 0 || ((!want_o || wait_ge(&ctr[kODone], j, abort_flag)) &&
                                          (!states || wait_ge(&ctr[kStored], j, abort_flag)))));
            if (!ok) break;
            // ---- h <- e^{gamma_C} h + K^T Dt : rows 32p..32p+31, 32 columns, K = 64 tokens
            {
                uint32_t bt[4][2][4];
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int np = 0; np < 2; ++np)
                        ldsm_x4_t(bt[ks][np], sb + kDt + (2 * np + (mi >> 1)) * 1024 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
                if (j + 1 < nch) load_chunk_regs(j + 1);  // w, u of the next chunk (w fragments are dead)
                const float eC = __expf(gC);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int q = 0; q < 4; ++q) hf[mt][nt][q] *= eC;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int np = 0; np < 2; ++np) {
                            hmma(hf[mt][2 * np], ka[ks][mt], bt[ks][np][0], bt[ks][np][1]);
                            hmma(hf[mt][2 * np + 1], ka[ks][mt], bt[ks][np][2], bt[ks][np][3]);
                        }
                if (j + 1 < nch) load_chunk_ka(j + 1);  // after the products that read these registers
            }
            // ---- h_{j+1} -> Hb[(j+1)%2]; Delta_j and h_{j+1} go to the output MMAs behind one proxy fence
            write_hb((j + 1) & 1);
            fence_proxy_async();
            chain_sync(true);
            if (tid == 0) {
                sm->cl_landed = j + 2 < nch ? j + 2 : nch;
                publish(&ctr[kChain], j + 2);
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
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const int dim = 32 * p + 16 * mt + g + half * 8;
                            *reinterpret_cast<float2 *>(dst + (size_t)dim * ld + 8 * nt + 2 * c4) =
                                make_float2(hf[mt][nt][2 * half], hf[mt][nt][2 * half + 1]);
                        }
            }
        }
    } else if (warp < 8) {
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
                if (et == 0) bulk_wait_read<0>();  // the previous chunk's o has left the staging tile
                epi_sync(true);
                if (et == 0) publish(&ctr[kTmemO], j + 1);
                const float er[2] = {__expf(g0), __expf(g1)};
                const int t0 = sr.start + j * kChunk;
                const bool full = len == kChunk;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    __nv_bfloat16 *dst = prm.o + ((size_t)(t0 + rr[half]) * d.Hv + h) * V + c0 + 2 * ec;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int k = 4 * i + 2 * half;
                        const uint32_t x =
                            pack_bf16(scl * fmaf(er[half], dq[k], dp[k]), scl * fmaf(er[half], dq[k + 1], dp[k + 1]));
                        if (full)  // a ragged chunk's tile would spill into the next sequence
                            st_shared_b32(sb + kOs + rr[half] * 64 + (8 * i + 2 * ec) * 2, x);
                        else if (rr[half] < len)
                            *reinterpret_cast<uint32_t *>(dst + 8 * i) = x;
                    }
                }
                if (full) {
                    fence_proxy_async();
                    epi_sync(true);
                    if (et == 0) {
                        tma_store_3d(&tm_o, sb + kOs, c0, h, t0);
                        bulk_commit();
                    }
                }
            }
            if (et == 0) bulk_wait_all();  // the o stores read shared memory until they complete
            if (!ok) {
                if (et == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
                *abort_flag = 1;
            }
        }
    } else if (warp == 8) {
        // =================================================== output issuer
        if (lane == 0 && want_o) {
            bool ok = true;
            auto issue_out_loads = [&](int j) {
                const int s = j % kStages;
                uint8_t *stg = smem + kO0 + s * kOStageBytes;
                const int t0 = sr.start + j * kChunk;
                const int cg = sr.chunk0 + j;
                mbar_arrive_expect_tx(&sm->ofull[s], kOStageBytes);
                ++sm->ol_issued;
                tma_load_3d(stg + kQ, &tm_q, &sm->ofull[s], 0, hq, t0);
                tma_load_3d(stg + kQ + 8192, &tm_q, &sm->ofull[s], 64, hq, t0);
                tma_load_2d(stg + kP, &tm_p, &sm->ofull[s], 0, (cg * d.Hv + h) * kChunk);
            };
            if (want_o)
                for (int c = 0; c < kStages && c < nch; ++c) issue_out_loads(c);
            const uint32_t id_O = idesc_bf16(64, 32, false, true);
            for (int j = 0; j < nch && ok; ++j) {
                // h_j and Delta_j are in kHb[j%2], kDb[j%2]
                ok = wait_ge(&ctr[kChain], j + 2, abort_flag);
                if (!ok) break;
                const uint32_t hb = sb + kHb + (j & 1) * 8192, db = sb + kDb + (j & 1) * 4096;
                {
                    // DQ = Q h_j, DP = P Delta_j into buffer j%2 once q, P have landed and the
                    // epilogue has read chunk j-2's accumulators
                    ok = wait_bar(&sm->ofull[j % kStages], (j / kStages) & 1, abort_flag) &&
                         wait_ge(&ctr[kTmemO], j >= 1 ? j - 1 : 0, abort_flag);
                    if (!ok) break;
                    sm->ol_landed = j + 1;
                    tc_fence_after();
                    const uint32_t st = sb + kO0 + (j % kStages) * kOStageBytes;
                    const uint32_t tb = tmem + (j & 1) * kOBuf;
                    const uint64_t qd = smem_desc(st + kQ, 16, 1024, kSw128), hd = smem_desc(hb, 128, 2048, kSwNone);
                    const uint64_t pd = smem_desc(st + kP, 16, 1024, kSw128), dd = smem_desc(db, 128, 1024, kSwNone);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16(tb + kColQ, qd + (uint64_t)((((ks >> 2) * 8192 + (ks & 3) * 32)) >> 4),
                                 hd + (uint64_t)(ks * 256 >> 4), id_O, ks > 0);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(tb + kColP, pd + (uint64_t)(ks * 32 >> 4), dd + (uint64_t)(ks * 256 >> 4), id_O, ks > 0);
                    mma_commit(&sm->mmaO[j & 1]);
                    sm->mma_issued = j + 1;
                }
                // the (q, P) stage of chunk j-1 is free once its products are complete: chunk j+2
                if (want_o && j >= 1 && j + 2 < nch) {
                    ok = wait_ge(&ctr[kODone], j, abort_flag);
                    if (!ok) break;
                    issue_out_loads(j + 2);
                }
            }
            if (!ok) {
                set_status(prm.status, GDN_ERR_TIMEOUT);
                *abort_flag = 1;
            }
        }
        __syncwarp();
    } else {
        // =================================================== chain producer
        if (lane == 0) {
            bool ok = true;
            auto issue_chain_loads = [&](int c) {
                const int s = c % kStages;
                uint8_t *stg = smem + kC0 + s * kCStageBytes;
                const int t0 = sr.start + c * kChunk;
                mbar_arrive_expect_tx(&sm->cfull[s], kCStageBytes);
                ++sm->cl_issued;
                tma_load_3d(stg + kK, &tm_k, &sm->cfull[s], 0, hq, t0);
                tma_load_3d(stg + kK + 8192, &tm_k, &sm->cfull[s], 64, hq, t0);
                tma_load_3d(stg + kW, &tm_w, &sm->cfull[s], 0, h, t0);
                tma_load_3d(stg + kW + 8192, &tm_w, &sm->cfull[s], 64, h, t0);
                tma_load_3d(stg + kU, &tm_u, &sm->cfull[s], c0, h, t0);  // out of range (zero) for operator columns
            };
            for (int c = 0; c < kStages && c < nch; ++c) issue_chain_loads(c);
            // chunk 3 into stage 0 once the chain has chunk 0 in registers (kChain >= 1)
            if (kStages < nch) {
                ok = wait_ge(&ctr[kChain], 1, abort_flag);
                if (ok) issue_chain_loads(kStages);
            }
            for (int j = 0; j < nch && ok; ++j) {
                // chunk j done (kChain >= j+2): its entry state and Delta out of kHb[j%2], kDb[j%2];
                // chunk j+1's stage is in registers, so stage (j+1)%3 takes chunk j+4
                ok = wait_ge(&ctr[kChain], j + 2, abort_flag);
                if (!ok) break;
                if (j + 1 + kStages < nch) issue_chain_loads(j + 1 + kStages);
                if (states) {
                    // one block each per (chunk, head, column slice)
                    const size_t blk = ((size_t)(sr.chunk0 + j) * d.Hv + h) * (V / kBV) + blockIdx.z;
                    bulk_store(prm.h_chunks + blk * (K * kBV), sb + kHb + (j & 1) * 8192, K * kBV * 2);
                    bulk_store(prm.delta + blk * (kChunk * kBV), sb + kDb + (j & 1) * 4096, kChunk * kBV * 2);
                    bulk_commit();
                    bulk_wait_read<0>();
                    publish(&ctr[kStored], j + 1);
                }
            }
            if (!ok) {
                set_status(prm.status, GDN_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            bulk_wait_all();  // state copies complete before the CTA's shared memory goes away
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        // let every TMA load and output MMA still in flight finish (bounded) before the CTA exits
        const uint64_t t0 = globaltimer();
        for (int c = sm->cl_landed; c < sm->cl_issued; ++c)
            while (!mbar_try_wait(smem_u32(&sm->cfull[c % kStages]), (c / kStages) & 1) && globaltimer() - t0 < kWaitNs) {
            }
        for (int c = sm->ol_landed; c < sm->ol_issued; ++c)
            while (!mbar_try_wait(smem_u32(&sm->ofull[c % kStages]), (c / kStages) & 1) && globaltimer() - t0 < kWaitNs) {
            }
        for (int c = sm->mma_seen; c < sm->mma_issued; ++c)
            while (!mbar_try_wait(smem_u32(&sm->mmaO[c & 1]), (c >> 1) & 1) && globaltimer() - t0 < kWaitNs) {
            }
    }
    __syncthreads();
    if (warp == 8) {
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
    CUtensorMap mq, mk, mw, mu, mp, mo;
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
    // o [T, Hv, V] bf16 in 32-column, 64-row boxes (stores of full chunks)
    const cuuint64_t dov[3] = {(cuuint64_t)d.V, (cuuint64_t)d.Hv, T};
    const cuuint64_t sov[2] = {(cuuint64_t)d.V * 2, (cuuint64_t)d.Hv * d.V * 2};
    const cuuint32_t bov[3] = {kBV, 1, 64};
    if (!make_map(&mo, BF, a.o ? a.o : a.w16, 3, dov, sov, bov, CU_TENSOR_MAP_SWIZZLE_NONE)) return cudaErrorInvalidValue;
    // chunk entry states and Delta: both or neither
    if ((a.h_chunks16 != nullptr) != (a.delta16 != nullptr)) return cudaErrorInvalidValue;
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
    fwd2_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mk, mw, mu, mp, mo, p);
    return cudaGetLastError();
}

}  // namespace gdn
