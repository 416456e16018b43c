// gdn_fwd3.cu -- chunked forward of the gated delta rule (bf16, K = V = 128):
// the sequential state chain on warp-level MMAs with the state held
// transposed in registers, the output on tcgen05. w, u and the decay-masked
// P = M o Q K^T of every chunk come ready-made from the chunk-prep kernel
// (gdn_prep3.cu) through TMA rings.
//
// One CTA per (sequence or segment, value head, 32-column slice of V). Per
// 64-token chunk (h the chunk-entry state, h = S^T, notation of gdn_internal.cuh):
//
//   chain (mma.sync, fp32 state in registers):
//     Delta = u - w h,     h <- e^{gamma_C} h + K^T (e^{gamma_C - gamma} o Delta)
//   output (tcgen05, TMEM accumulators, behind the chain):
//     DQ = Q h,  DP = P Delta,   o = scale (e^gamma o DQ + DP)
//
// The chain works on the transposed state h^T (rows: value columns v, columns:
// key dimensions d), so that both chained products have the state or Delta as
// their A operand:
//     D1 = h^T w^T - u^T = -Delta^T        (16 v x 16 tokens per warp, contraction over d)
//     h^T <- e^{gamma_C} h^T + (Delta~)^T K  (16 v x 32 d per warp, contraction over tokens)
// An m16n8 accumulator fragment, packed to bf16 pairs, is exactly the A
// fragment of the next m16n8k16 product along its column index, so the state
// and Delta~ never pass through shared memory on their way into the next
// product of the same warp. Four chain warps, one per scheduler, each hold all
// 32 value columns of the slice (two m16 tiles, so that every w and K fragment
// read from shared memory feeds two MMAs): warp x holds the fp32 state for
// d in [32x, 32x+32) and computes Delta for the tokens [16x, 16x+16). Per
// chunk they exchange, through shared memory and two 128-thread barriers, only
// bf16 data: the state quarters (the chunk's entry state, which the output
// products read anyway) and the Delta~ quarters (1 KB per warp). Each warp
// issues 64 MMAs per chunk, into one accumulator set per product: with ten
// warps, three share a scheduler's register file, which caps a thread at 168
// registers, and a second set (to split the dependent MMAs) made the compiler
// spill inside the chain, costing 15 % of the kernel. Shared memory is read
// with ld.shared / ldmatrix on 32-bit shared addresses throughout (generic
// loads would take the long path).
//
// Warp roles (320 threads):
//   warps 0-3    chain (above).
//   warps 4-7    epilogue: o from the double-buffered DQ/DP accumulators;
//                warp 4 + q reads TMEM lanes 32 q .. +31 (rows 16 q .. +15),
//                stages its rows of o, and one TMA store per full chunk writes
//                them (a ragged last chunk is stored row by row).
//   warp 8       output issuer: the DQ/DP MMAs and the (q, P) TMA ring.
//   warp 9       producer: the (k, w, u) TMA ring with each chunk's gates,
//                L2 prefetches a few chunks ahead, and the bulk copies of the
//                chunk states and Delta to global memory.
// Hardware completions (TMA, tcgen05.commit) and the chain's per-chunk
// hand-over use mbarriers, each waited on once per use and in order; the
// "buffer is free again" conditions use monotonically increasing counters
// (release/acquire), which cannot alias the way an mbarrier parity can when
// a waiter skips uses. Every wait is bounded in time; a wait that expires
// records GDN_ERR_TIMEOUT and winds the CTA down, draining the TMA loads and
// MMAs it has in flight.
//
// Modes: whole sequences from h0; the recompute for the backward (no output,
// stores every chunk's entry state and Delta in bf16); and the two passes of
// the sequence split (see Fwd3Mode). Saved states and Delta keep the blocked
// tile layout of the output operands, one contiguous block per (chunk, value
// head, 32-column slice): entry state [NC][Hv][V/32][4][128][8] (block of 8
// columns, state row d, 8 columns), Delta [NC][Hv][V/32][4][64][8] (token
// rows; rows past a ragged chunk's end are zero).
#include <cstddef>

#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kChainWarps = 4;
constexpr int kEpiWarp0 = 4;     // warps 4..7
constexpr int kIssuerWarp = 8;
constexpr int kProdWarp = 9;
constexpr int kThreads = 10 * 32;
static_assert(kThreads == (kProdWarp + 1) * 32, "the producer is the last warp");
constexpr int kBV = 32;
constexpr int kCS = 3;  // chain ring stages
constexpr int kOS = 2;  // output ring stages
constexpr int kHB = 3;  // entry-state / Delta buffers (chain -> output products, state copies)
constexpr int kPrefetch = 4;  // chunks beyond the ring that the producer prefetches into L2

// ---- shared memory (bytes from a 1024-aligned base)
constexpr int kC0 = 0;  // chain ring: k, w [64][128] bf16 (two 64-column halves, 128-byte swizzle),
                        // u [64][32] fp32 (128-byte swizzle)
constexpr int kK = 0, kW = 16384, kU = 32768, kCStageBytes = 40960;
constexpr int kO0 = kC0 + kCS * kCStageBytes;  // output ring: q [64][128] bf16, P [64][64] bf16
constexpr int kQ = 0, kP = 16384, kOStageBytes = 24576;
constexpr int kHb = kO0 + kOS * kOStageBytes;  // kHB x 8192: h^T (bf16): (v/8)*2048 + d*16 + (v%8)*2
constexpr int kDb = kHb + kHB * 8192;          // kHB x 4096: Delta (bf16): (v/8)*1024 + t*16 + (v%8)*2
constexpr int kXb = kDb + kHB * 4096;          // 4096: Delta~ A fragments, [group][quarter][lane] x 16 bytes
constexpr int kOs = kXb + 4096;                // 4096: o of a full chunk, staged for its TMA store
                                               // ([64][32] bf16, 64-byte swizzle)
constexpr int kGam = kOs + 4096;               // kCS x 64 fp32: gamma of each staged chunk
constexpr int kSmall = kGam + 1024;
constexpr int kSmemBytes = kSmall + 2048 + 1024;
static_assert(kC0 % 1024 == 0 && kO0 % 1024 == 0 && kHb % 1024 == 0 && kCStageBytes % 1024 == 0 &&
                  kOStageBytes % 1024 == 0 && kCS * 64 * 4 <= 1024 && kSmemBytes <= 232448,
              "shared memory layout");

// DQ, DP double-buffered in tensor memory: buffer b at columns 64 b.
constexpr uint32_t kColQ = 0, kColP = 32, kOBuf = 64, kTmemCols = 128;

// Counters: kODone chunks whose output MMAs are known complete (epilogue),
// kTRead chunks whose accumulators the epilogue has read, kStored chunks whose
// state copies have finished reading shared memory (producer).
enum Ctr { kODone, kTRead, kStored, kNumCtr };

struct Small {
    uint64_t cfull[kCS], cempty[kCS], ofull[kOS], hready[kHB], mmaO[2];
    uint32_t ctr[kNumCtr];
    int c_issued[kCS], o_issued[kOS], mma_issued[2];
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Small) <= 2048, "small area");

__device__ __forceinline__ bool epi_sync(bool pred) { return role_sync_and<128>(3, pred); }

// kWhole: one CTA column per sequence, from h0.
// kSegPass: per segment, the chain on [c | P] with c from zero (V columns, u as
//   input) and P from the identity (K more columns, whose u tile is read out of
//   range and so is zero): the segment maps a start state h to P h + c.
// kSegOut: per segment, the chain and the output from the composed start state.
enum Fwd3Mode { kWhole = 0, kSegPass = 1, kSegOut = 2 };

struct Fwd3Params {
    Dims d;
    const float *gamma;   // [T_total, Hv]
    const float *h0;      // [N, Hv, K, V] or null
    __nv_bfloat16 *o;     // [T_total, Hv, V], or null: no output (the backward's recompute)
    float *final_state;   // [N, Hv, K, V] or null
    __nv_bfloat16 *h_chunks;  // entry state of every chunk (bf16, blocked) or null
    __nv_bfloat16 *delta;     // Delta of every chunk (bf16, blocked) or null
    // Sequence split: each sequence runs as nseg segments, contiguous runs of
    // ceil(chunks / nseg) chunks (CTA slot = sequence rank * nseg + segment).
    int nseg;
    int mode;             // Fwd3Mode
    const float *seg_h0;  // kSegOut: [N * nseg, Hv, K, V] start state of every segment
    float *seg_c;         // kSegPass: [N * nseg, Hv, K, V] end state from a zero start
    float *seg_P;         // kSegPass: [N * nseg, Hv, K, K] transition operator of the segment
    unsigned *status;
};

// Byte offset of (row, col) in a [rows][128] bf16 tile stored as two 64-column
// halves of 128-byte rows with 128-byte swizzle (what the TMA loads produce).
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
    return (uint32_t)((col >> 6) * 8192 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(kThreads, 1)
fwd3_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_u,
            const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_o,
            const __grid_constant__ Fwd3Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    Small *sm = reinterpret_cast<Small *>(smem + kSmall);
    volatile int *abort_flag = &sm->abort_flag;
    const uint32_t sb = smem_u32(smem);
    float *gam = reinterpret_cast<float *>(smem + kGam);

    const Dims &d = prm.d;
    const int nseg = prm.nseg;
    // 1-D grid, sequence-major in longest-first order: the CTAs of the longest
    // sequences (all their heads and column slices) are dispatched first
    const int nsl = (d.V + (prm.mode == kSegPass ? d.K : 0)) / kBV;
    const int slot = blockIdx.x / (d.Hv * nsl), rem = blockIdx.x % (d.Hv * nsl);
    const int n = seq_by_length(d, slot / nseg), sseg = slot % nseg, h = rem / nsl, zs = rem % nsl;
    const int c0 = zs * kBV;
    const int hq = h / (d.Hv / d.Hq);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int K = 128, V = 128;
    const bool want_o = prm.o != nullptr;
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
        for (int s = 0; s < kCS; ++s) {
            mbar_init(&sm->cfull[s], 1);
            mbar_init(&sm->cempty[s], kChainWarps);
            sm->c_issued[s] = 0;
        }
        for (int s = 0; s < kOS; ++s) {
            mbar_init(&sm->ofull[s], 1);
            sm->o_issued[s] = 0;
        }
        for (int b = 0; b < kHB; ++b) mbar_init(&sm->hready[b], kChainWarps);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->mmaO[b], 1);
            sm->mma_issued[b] = 0;
        }
        for (int c = 0; c < kNumCtr; ++c) sm->ctr[c] = 0;
        sm->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kIssuerWarp) {
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

    if (warp < kChainWarps) {
        // =========================================================== chain
        const int x = warp;  // d quarter of the state, token quarter of Delta
        const int g = lane >> 2, cq = lane & 3, li = lane & 7, mi = lane >> 3;
        const uint32_t gam_sb = sb + kGam;
        // hs[mt][nt][e]: h^T[v = 16mt + g + 8(e>>1)][d = 32x + 8nt + 2cq + (e&1)]
        float hs[2][4][4];
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
                    for (int e = 0; e < 4; ++e) {
                        const int v = 16 * mt + g + 8 * (e >> 1), dd = 32 * x + 8 * nt + 2 * cq + (e & 1);
                        hs[mt][nt][e] = src ? src[(size_t)dd * V + c0 + v] : (ident && dd == c0 - V + v ? 1.f : 0.f);
                    }
        }
        bool ok = true;
        for (int j = 0; j < nch; ++j) {
            const int s = j % kCS, hb = j % kHB;
            const int len = min(kChunk, sr.len - j * kChunk);
            const uint32_t st = sb + kC0 + s * kCStageBytes;
            const uint32_t hbuf = sb + kHb + hb * 8192, dbuf = sb + kDb + hb * 4096;
            bool good = wait_bar(&sm->cfull[s], (j / kCS) & 1, abort_flag);
            if (lane == 0 && j >= kHB)  // buffer hb was last read by chunk j - kHB's products / copies
                good = good && (!want_o || wait_ge(&ctr[kODone], j - kHB + 1, abort_flag)) &&
                       (!states || wait_ge(&ctr[kStored], j - kHB + 1, abort_flag));
            good = __all_sync(0xffffffffu, good);
            // own quarter of h_j as bf16 A fragments: ao[mt][kk] for k-step 2x + kk
            uint32_t ao[2][2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    ao[mt][kk][0] = pack_bf16(hs[mt][2 * kk][0], hs[mt][2 * kk][1]);
                    ao[mt][kk][1] = pack_bf16(hs[mt][2 * kk][2], hs[mt][2 * kk][3]);
                    ao[mt][kk][2] = pack_bf16(hs[mt][2 * kk + 1][0], hs[mt][2 * kk + 1][1]);
                    ao[mt][kk][3] = pack_bf16(hs[mt][2 * kk + 1][2], hs[mt][2 * kk + 1][3]);
                }
            // D1 accumulators [m-tile][token n-tile]
            float acc[2][2][4] = {};
            float gC = 0.f, sc[2][2] = {};
            uint32_t bw[8][4];  // w fragments (B of D1): bw[2 o + kk] is k-step 2((x + o) & 3) + kk
            if (good) {
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        stsm_x4_t(hbuf + (2 * mt + (mi & 1)) * 2048 + (32 * x + 16 * kk + 8 * (mi >> 1) + li) * 16,
                                  ao[mt][kk]);
#pragma unroll
                for (int o = 0; o < 4; ++o)
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        ldsm_x4(bw[2 * o + kk],
                                st + kW + sw_off(16 * x + 8 * (mi >> 1) + li, 16 * (2 * ((x + o) & 3) + kk) + 8 * (mi & 1)));
                const uint32_t gm = gam_sb + s * kChunk * 4;
                gC = ld_shared_f32(gm + (kChunk - 1) * 4);
                // acc = -u at this thread's (v, token) pairs; u tile: 32 fp32 per row, 16-byte chunks XOR (row % 8)
                const uint32_t ut = st + kU;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) sc[nt][e] = __expf(gC - ld_shared_f32(gm + (16 * x + 8 * nt + 2 * cq + e) * 4));
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int t = 16 * x + 8 * nt + 2 * cq + (e & 1), v = 16 * mt + g + 8 * (e >> 1);
                            acc[mt][nt][e] = -ld_shared_f32(ut + (t * 32 + (((v >> 2) ^ (t & 7)) << 2) + (v & 3)) * 4);
                        }
                }
                if (len < kChunk) {
                    // a ragged chunk: zero the key rows past its end (their Delta~ is zero, but a
                    // non-finite value of the next packed sequence would still turn 0 * x into NaN
                    // in the state update); the barrier below orders this before every D2 load
                    for (int i = tid; i < (kChunk - len) * 16; i += kChainWarps * 32) {
                        const int r = len + (i >> 4), c = i & 15;
                        st_shared_v4(st + kK + (c >> 3) * 8192 + r * 128 + (c & 7) * 16, 0u, 0u, 0u, 0u);
                    }
                }
                // D1 over this warp's own quarter of d (registers): k-steps 2x, 2x+1
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    hmma(acc[mt][0], ao[mt][0], bw[0][0], bw[0][1]);
                    hmma(acc[mt][1], ao[mt][0], bw[0][2], bw[0][3]);
                    hmma(acc[mt][0], ao[mt][1], bw[1][0], bw[1][1]);
                    hmma(acc[mt][1], ao[mt][1], bw[1][2], bw[1][3]);
                }
            }
            ok = role_sync_and<128>(1, good);  // every quarter of h_j is in hbuf
            if (!ok) break;
            // D1 over the other three quarters, A fragments of h_j from hbuf
#pragma unroll
            for (int o = 1; o < 4; ++o) {
                uint32_t ah[2][2][4];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        ldsm_x4_t(ah[mt][kk], hbuf + (2 * mt + (mi & 1)) * 2048 +
                                                  (16 * (2 * ((x + o) & 3) + kk) + 8 * (mi >> 1) + li) * 16);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        float(&A)[2][2][4] = acc;
                        hmma(A[mt][0], ah[mt][kk], bw[2 * o + kk][0], bw[2 * o + kk][1]);
                        hmma(A[mt][1], ah[mt][kk], bw[2 * o + kk][2], bw[2 * o + kk][3]);
                    }
            }
            // Delta = -acc on live tokens (a select, so nothing past the end leaks in);
            // Delta~ = e^{gamma_C - gamma} Delta as the A fragment of D2 for this token quarter
            uint32_t da[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                float dl[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dl[nt][e] = 16 * x + 8 * nt + 2 * cq + (e & 1) < len ? -acc[mt][nt][e] : 0.f;
                uint32_t du[4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    da[mt][2 * nt] = pack_bf16(dl[nt][0] * sc[nt][0], dl[nt][1] * sc[nt][1]);
                    da[mt][2 * nt + 1] = pack_bf16(dl[nt][2] * sc[nt][0], dl[nt][3] * sc[nt][1]);
                    du[2 * nt] = pack_bf16(dl[nt][0], dl[nt][1]);
                    du[2 * nt + 1] = pack_bf16(dl[nt][2], dl[nt][3]);
                }
                // A fragment order: (v 0-7, t 0-7), (v 8-15, t 0-7), (v 0-7, t 8-15), (v 8-15, t 8-15)
                st_shared_v4(sb + kXb + (mt * 4 + x) * 512 + lane * 16, da[mt][0], da[mt][1], da[mt][2], da[mt][3]);
                stsm_x4_t(dbuf + (2 * mt + (mi & 1)) * 1024 + (16 * x + 8 * (mi >> 1) + li) * 16, du);
            }
            // K fragments (B of D2): bk[o] is token quarter (x + o) & 3, this warp's d quarter
            uint32_t bk[4][2][4];
#pragma unroll
            for (int o = 0; o < 4; ++o)
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    const int tq = (x + o) & 3;
                    ldsm_x4_t(bk[o][np], st + kK + sw_off(16 * tq + 8 * (mi & 1) + li, 32 * x + 16 * np + 8 * (mi >> 1)));
                }
            const float eC = __expf(gC);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) hs[mt][nt][e] *= eC;
            // D2 for the own token quarter: h^T[:, own d quarter] += Delta~^T K
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    hmma(hs[mt][2 * np], da[mt], bk[0][np][0], bk[0][np][1]);
                    hmma(hs[mt][2 * np + 1], da[mt], bk[0][np][2], bk[0][np][3]);
                }
            named_sync<128>(1);  // every token quarter of Delta~ is in kXb
            // (eight independent accumulator tiles per token quarter cover the MMA latency)
#pragma unroll
            for (int o = 1; o < 4; ++o) {
                uint32_t pa[2][4];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    const uint4 p = ld_shared_v4(sb + kXb + (mt * 4 + ((x + o) & 3)) * 512 + lane * 16);
                    pa[mt][0] = p.x, pa[mt][1] = p.y, pa[mt][2] = p.z, pa[mt][3] = p.w;
                }
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int np = 0; np < 2; ++np) {
                        hmma(hs[mt][2 * np], pa[mt], bk[o][np][0], bk[o][np][1]);
                        hmma(hs[mt][2 * np + 1], pa[mt], bk[o][np][2], bk[o][np][3]);
                    }
            }
            // h_j and Delta_j (shared memory, generic writes) go to the output MMAs and
            // the state copies (async proxy); the stage is free for the producer
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm->hready[hb]);
                mbar_arrive(&sm->cempty[s]);
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
                        for (int e = 0; e < 4; ++e) {
                            const int v = 16 * mt + g + 8 * (e >> 1), dd = 32 * x + 8 * nt + 2 * cq + (e & 1);
                            dst[(size_t)dd * ld + v] = hs[mt][nt][e];
                        }
            }
        }
    } else if (warp < kEpiWarp0 + 4) {
        // ======================================================== epilogue
        if (want_o) {
            const int et = tid - kEpiWarp0 * 32, q = warp & 3;  // TMEM lanes 32q.. = rows 16q..16q+15
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
                if (et == 0) publish(&ctr[kODone], j + 1);
                tc_fence_after();
                float dq[16], dp[16];
                const uint32_t tb = tmem + lane_base + (j & 1) * kOBuf;
                tmem_ld16x256_x4(tb + kColQ, dq);
                tmem_ld16x256_x4(tb + kColP, dp);
                tc_fence_before();
                if (et == 0) bulk_wait_read<0>();  // the previous chunk's o has left the staging tile
                epi_sync(true);
                if (et == 0) publish(&ctr[kTRead], j + 1);
                const float er[2] = {__expf(g0), __expf(g1)};
                const int t0 = sr.start + j * kChunk;
                const bool full = len == kChunk;
                // o in the m16n8 accumulator layout the 16x256b loads deliver: ov[i][half] is the
                // 8 x 8 block (rows 16q + 8 half .., columns 8i ..), this lane holding row eg,
                // columns 2ec, 2ec + 1
                uint32_t ov[4][2];
#pragma unroll
                for (int half = 0; half < 2; ++half)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int k = 4 * i + 2 * half;
                        ov[i][half] = pack_bf16(scl * fmaf(er[half], dq[k], dp[k]), scl * fmaf(er[half], dq[k + 1], dp[k + 1]));
                    }
                if (full) {
                    // staging tile [64][32] bf16 with the 64-byte swizzle of its TMA store (16-byte
                    // chunk c of row r at chunk c ^ ((r / 2) % 4)): two conflict-free stmatrix.x4
                    const int li = lane & 7, mi = lane >> 3;
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        const int i = 2 * a + (mi >> 1), r = 16 * q + 8 * (mi & 1) + li;
                        const uint32_t regs[4] = {ov[2 * a][0], ov[2 * a][1], ov[2 * a + 1][0], ov[2 * a + 1][1]};
                        stsm_x4(sb + kOs + r * 64 + ((i ^ ((r >> 1) & 3)) << 4), regs);
                    }
                } else {
                    // a ragged chunk's tile would spill into the next sequence: row by row
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        __nv_bfloat16 *dst = prm.o + ((size_t)(t0 + rr[half]) * d.Hv + h) * V + c0 + 2 * ec;
                        if (rr[half] < len)
#pragma unroll
                            for (int i = 0; i < 4; ++i) *reinterpret_cast<uint32_t *>(dst + 8 * i) = ov[i][half];
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
    } else if (warp == kIssuerWarp) {
        // =================================================== output issuer
        if (lane == 0 && want_o) {
            bool ok = true;
            auto issue_out_loads = [&](int j) {
                const int s = j % kOS;
                uint8_t *stg = smem + kO0 + s * kOStageBytes;
                const int t0 = sr.start + j * kChunk;
                const int cg = sr.chunk0 + j;
                mbar_arrive_expect_tx(&sm->ofull[s], kOStageBytes);
                ++sm->o_issued[s];
                tma_load_3d(stg + kQ, &tm_q, &sm->ofull[s], 0, hq, t0);
                tma_load_3d(stg + kQ + 8192, &tm_q, &sm->ofull[s], 64, hq, t0);
                tma_load_2d(stg + kP, &tm_p, &sm->ofull[s], 0, (cg * d.Hv + h) * kChunk);
            };
            for (int c = 0; c < kOS && c < nch; ++c) issue_out_loads(c);
            const uint32_t id_O = idesc_bf16(64, 32, false, true);
            for (int j = 0; j < nch && ok; ++j) {
                // h_j and Delta_j are in the chain's buffer j % kHB; q, P in stage j % kOS;
                // the epilogue has read chunk j-2's accumulators out of TMEM buffer j % 2
                ok = wait_bar(&sm->hready[j % kHB], (j / kHB) & 1, abort_flag) &&
                     wait_bar(&sm->ofull[j % kOS], (j / kOS) & 1, abort_flag) &&
                     (j < 2 || wait_ge(&ctr[kTRead], j - 1, abort_flag));
                if (!ok) break;
                tc_fence_after();
                const uint32_t hbuf = sb + kHb + (j % kHB) * 8192, dbuf = sb + kDb + (j % kHB) * 4096;
                const uint32_t stq = sb + kO0 + (j % kOS) * kOStageBytes;
                const uint32_t tb = tmem + (j & 1) * kOBuf;
                const uint64_t qd = smem_desc(stq + kQ, 16, 1024, kSw128), hd = smem_desc(hbuf, 128, 2048, kSwNone);
                const uint64_t pd = smem_desc(stq + kP, 16, 1024, kSw128), dd = smem_desc(dbuf, 128, 1024, kSwNone);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tb + kColQ, qd + (uint64_t)((((ks >> 2) * 8192 + (ks & 3) * 32)) >> 4),
                             hd + (uint64_t)(ks * 256 >> 4), id_O, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tb + kColP, pd + (uint64_t)(ks * 32 >> 4), dd + (uint64_t)(ks * 256 >> 4), id_O, ks > 0);
                mma_commit(&sm->mmaO[j & 1]);
                ++sm->mma_issued[j & 1];
                // chunk j-1's products are complete once its commit lands: its (q, P) stage
                // takes chunk j-1+kOS
                if (j >= 1 && j - 1 + kOS < nch) {
                    ok = wait_bar(&sm->mmaO[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag);
                    if (!ok) break;
                    issue_out_loads(j - 1 + kOS);
                }
            }
            if (!ok) {
                set_status(prm.status, GDN_ERR_TIMEOUT);
                *abort_flag = 1;
            }
        }
        __syncwarp();
    } else {
        // ========================================================= producer
        bool ok = true;
        // the stage's gates come in by cp.async from every lane, tracked by the stage's mbarrier
        // (each lane's arrival raises its pending count until the copies land), then k, w, u by TMA
        auto stage_chunk = [&](int c) {
            const int s = c % kCS;
            const int t0 = sr.start + c * kChunk, len = min(kChunk, sr.len - c * kChunk);
            const uint32_t gdst = smem_u32(gam + s * kChunk);
            cp_async4(gdst + 4 * lane, prm.gamma + (size_t)(t0 + min(lane, len - 1)) * d.Hv + h);
            cp_async4(gdst + 4 * (lane + 32), prm.gamma + (size_t)(t0 + min(lane + 32, len - 1)) * d.Hv + h);
            cp_async_mbar_arrive(&sm->cfull[s]);
            __syncwarp();
            if (lane == 0) {
                uint8_t *stg = smem + kC0 + s * kCStageBytes;
                mbar_arrive_expect_tx(&sm->cfull[s], kCStageBytes);
                ++sm->c_issued[s];
                tma_load_3d(stg + kK, &tm_k, &sm->cfull[s], 0, hq, t0);
                tma_load_3d(stg + kK + 8192, &tm_k, &sm->cfull[s], 64, hq, t0);
                tma_load_3d(stg + kW, &tm_w, &sm->cfull[s], 0, h, t0);
                tma_load_3d(stg + kW + 8192, &tm_w, &sm->cfull[s], 64, h, t0);
                tma_load_3d(stg + kU, &tm_u, &sm->cfull[s], c0, h, t0);  // out of range (zero) for operator columns
            }
            __syncwarp();
        };
        auto prefetch_l2 = [&](int c) {
            if (lane == 0 && c < nch) {
                const int t0 = sr.start + c * kChunk;
                tma_prefetch_3d(&tm_k, 0, hq, t0);
                tma_prefetch_3d(&tm_k, 64, hq, t0);
                tma_prefetch_3d(&tm_w, 0, h, t0);
                tma_prefetch_3d(&tm_w, 64, h, t0);
                if (c0 < V) tma_prefetch_3d(&tm_u, c0, h, t0);
                if (want_o) {
                    tma_prefetch_3d(&tm_q, 0, hq, t0);
                    tma_prefetch_3d(&tm_q, 64, hq, t0);
                    tma_prefetch_2d(&tm_p, 0, ((sr.chunk0 + c) * d.Hv + h) * kChunk);
                }
            }
        };
        for (int c = 0; c < kCS && c < nch; ++c) stage_chunk(c);
        for (int c = kCS; c < kCS + kPrefetch; ++c) prefetch_l2(c);
        for (int j = 0; j < nch && ok; ++j) {
            // chunk j done by the chain: its stage takes chunk j + kCS
            if (j + kCS < nch) {
                ok = wait_bar(&sm->cempty[j % kCS], (j / kCS) & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                stage_chunk(j + kCS);
                prefetch_l2(j + kCS + kPrefetch);
            }
            if (states) {
                // chunk j's entry state and Delta out of buffer j % kHB, one bulk copy each
                ok = wait_bar(&sm->hready[j % kHB], (j / kHB) & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                if (lane == 0) {
                    const size_t blk = ((size_t)(sr.chunk0 + j) * d.Hv + h) * (V / kBV) + zs;
                    bulk_store(prm.h_chunks + blk * (K * kBV), sb + kHb + (j % kHB) * 8192, K * kBV * 2);
                    bulk_store(prm.delta + blk * (kChunk * kBV), sb + kDb + (j % kHB) * 4096, kChunk * kBV * 2);
                    bulk_commit();
                    bulk_wait_read<0>();
                    publish(&ctr[kStored], j + 1);
                }
                __syncwarp();
            }
        }
        if (!ok) {
            if (lane == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        if (lane == 0) bulk_wait_all();  // state copies complete before the CTA's shared memory goes away
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        // let every TMA load and output MMA still in flight finish (bounded) before the CTA exits:
        // each barrier has at most one use outstanding, the last one issued
        const uint64_t t0 = globaltimer();
        for (int s = 0; s < kCS; ++s)
            if (sm->c_issued[s] > 0)
                while (!mbar_try_wait(smem_u32(&sm->cfull[s]), (sm->c_issued[s] - 1) & 1) && globaltimer() - t0 < kWaitNs) {
                }
        for (int s = 0; s < kOS; ++s)
            if (sm->o_issued[s] > 0)
                while (!mbar_try_wait(smem_u32(&sm->ofull[s]), (sm->o_issued[s] - 1) & 1) && globaltimer() - t0 < kWaitNs) {
                }
        for (int b = 0; b < 2; ++b)
            if (sm->mma_issued[b] > 0)
                while (!mbar_try_wait(smem_u32(&sm->mmaO[b]), (sm->mma_issued[b] - 1) & 1) && globaltimer() - t0 < kWaitNs) {
                }
    }
    __syncthreads();
    if (warp == kIssuerWarp) {
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

cudaError_t launch_fwd3(const FwdArgs &a) {
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
    if (!make_map(&mo, BF, a.o ? a.o : a.w16, 3, dov, sov, bov, CU_TENSOR_MAP_SWIZZLE_64B)) return cudaErrorInvalidValue;
    // chunk entry states and Delta: both or neither
    if ((a.h_chunks16 != nullptr) != (a.delta16 != nullptr)) return cudaErrorInvalidValue;
    Fwd3Params p;
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
    cudaError_t e = cudaFuncSetAttribute(fwd3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    // the segment pass also carries the K operator columns
    const long long nctas = (long long)d.N * p.nseg * d.Hv * ((d.V + (p.mode == kSegPass ? d.K : 0)) / kBV);
    if (nctas >= (1ll << 31)) return cudaErrorInvalidValue;
    dim3 grid((unsigned)nctas);
    fwd3_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mk, mw, mu, mp, mo, p);
    return cudaGetLastError();
}

}  // namespace gdn
