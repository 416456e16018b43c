// gdn_bwd_dh.cu -- reverse state-gradient scan of the chunked backward (bf16,
// K = V = 128): the sequential part of the backward.
//
// Walking the chunks of a sequence backwards with dh' = the gradient w.r.t.
// the chunk's exit state (dht for the last chunk, zero if absent):
//
//   dDelta = scale (M o Q K^T)^T dO + diag(e^{gamma_C - gamma}) K dh'      (C x V)
//   dh     = e^{gamma_C} dh' + scale Q^T diag(e^gamma) dO - w^T dDelta     (K x V)
//
// (the adjoint of Delta = u - w h, o = scale (diag(e^gamma) Q h + (M o Q K^T) Delta),
// h' = e^{gamma_C} h + K^T diag(e^{gamma_C - gamma}) Delta). Every chunk's dh'
// and dDelta (bf16) are stored for the per-chunk gradient kernel in the blocked
// tile layout, one contiguous block per (chunk, value head, 32-column slice):
// dh' [NC][Hv][V/32][4][128][8], dDelta [NC][Hv][V/32][4][64][8]; dh0 (fp32) is
// the gradient at the sequence start.
//
// Organised like the forward chain kernel (gdn_fwd3.cu), whose chain this one
// mirrors: one CTA per (sequence, value head, 32-column slice of V), and the
// scan runs on the transposed gradient dh'^T (rows: value columns v, columns:
// key dimensions d), held in fp32 registers by four chain warps (warp x: the
// state for d in [32x, 32x+32), dDelta for the tokens [16x, 16x+16)):
//
//   D1 = dh'^T K^T                       (v x tokens, contraction over d)
//   dDelta^T = e^{gamma_C - gamma} o D1 + scale Y^T,      Y^T = dO^T P
//   dh^T = e^{gamma_C} dh'^T + X^T - dDelta^T w,           X^T = dO'^T Q,  dO' = scale e^gamma o dO
//
// D1 and the update are warp-level MMAs whose A operands (the state, dDelta)
// come from the accumulators of the previous product; the quarters the warps
// exchange pass through shared memory in bf16. Y^T and X^T do not depend on
// the chain: they run on tcgen05 one or two chunks ahead, with M = 128 rows
// that repeat the slice's 32 value columns four times (the dO tile read with a
// zero stride between its 32-column atoms), so that every chain warp finds all
// 32 value rows in its own TMEM lane quarter, in the mma.sync accumulator
// layout of the 16x256b load, and adds them to its fragments directly.
//
// Warp roles (256 threads):
//   warps 0-3  chain (above).
//   warps 4-5  dO' = scale e^gamma o dO into shared memory, then one of their
//              threads issues the X^T MMAs.
//   warp 6     issuer: the (q, P, dO) TMA ring and the Y^T MMAs.
//   warp 7     producer: the (k, w) TMA ring with each chunk's gates, and the
//              bulk copies of dh' and dDelta to global memory. (L2 prefetches
//              a few chunks ahead, as the forward chain issues them, measured
//              a few percent slower here.)
// Y^T and X^T go into double-buffered tensor memory, each chunk's pair
// completing one mbarrier (an arrival from each issuing thread): a single
// thread spends tens of cycles per tcgen05.mma, so the two products are
// issued side by side. Two dO' warps measured faster than one or four (eight
// warps in all: no scheduler holds more than two, so the register cap is 255).
// Hand-over by mbarriers (hardware completions, the chain's per-chunk
// hand-over) and release/acquire counters ("buffer free" conditions); every
// wait is bounded, and a wait that expires records GDN_ERR_TIMEOUT and winds
// the CTA down after draining its TMA loads and MMAs in flight.
//
// Sequence split (long sequences, few heads): a chunk maps its exit-state
// gradient dh' to dh = A dh' + b with A = e^{gamma_C} I - w^T diag(e^{gamma_C -
// gamma}) K, the transpose of the forward chunk's transition operator, so a
// segment of chunks maps the gradient at its end to Q dh_end + r. The segment
// pass runs the scan on [r | Q]: r from zero with the real dO, Q from the identity
// on K more columns whose dO tile is read out of range (zero), so Y = X = 0
// there. A composition walks the segments backwards from dht (gdn_split.cu), and
// the output pass reruns every segment from its composed dh_end.
//
// Rows past the end of a ragged chunk hold the next packed sequence: dDelta is
// zero there (a select), dO' too, and the w, q and dO rows they would meet in a
// product are zeroed in shared memory first, so that a non-finite value of the
// next sequence cannot turn 0 * x into NaN in this one.
#include <cstddef>

#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kChainWarps = 4;
constexpr int kAuxWarps = 2;  // dO' makers: warps kAuxWarp0 ..
constexpr int kAuxWarp0 = 4;
constexpr int kAuxThreads = kAuxWarps * 32;
constexpr int kIssuerWarp = kAuxWarp0 + kAuxWarps;
constexpr int kProdWarp = kIssuerWarp + 1;
constexpr int kThreads = (kProdWarp + 1) * 32;
static_assert(kThreads == (kProdWarp + 1) * 32, "the producer is the last warp");
constexpr int kBV = 32;
constexpr int kCS = 3;        // chain ring stages (k, w)
constexpr int kOS = 3;        // Y / X ring stages (q, P, dO)
constexpr int kHB = 2;        // dh' / dDelta buffers (chain -> copies)

// ---- shared memory (bytes from a 1024-aligned base)
constexpr int kC0 = 0;  // chain ring: k, w [64][128] bf16 (two 64-column halves, 128-byte swizzle)
constexpr int kK = 0, kW = 16384, kCStageBytes = 32768;
constexpr int kO0 = kC0 + kCS * kCStageBytes;  // Y / X ring: q [64][128], P [64][64] (128-byte
                                               // swizzle), dO [64][32] bf16 (64-byte swizzle)
constexpr int kQ = 0, kP = 16384, kDO = 24576, kOStageBytes = 28672;
constexpr int kHb = kO0 + kOS * kOStageBytes;  // kHB x 8192: dh'^T (bf16): (v/8)*2048 + d*16 + (v%8)*2
constexpr int kDb = kHb + kHB * 8192;          // kHB x 4096: dDelta (bf16): (v/8)*1024 + t*16 + (v%8)*2
constexpr int kXb = kDb + kHB * 4096;          // 4096: -dDelta^T A fragments, [group][quarter][lane] x 16 bytes
constexpr int kDO2 = kXb + 4096;               // 2 x 4096: dO' in the layout of the dO tile
constexpr int kGam = kDO2 + 2 * 4096;          // kCS x 64 fp32: gamma of each staged chunk
constexpr int kSmall = kGam + 1024;
constexpr int kSmemBytes = kSmall + 2048 + 1024;
static_assert(kO0 % 1024 == 0 && kHb % 1024 == 0 && kDO2 % 1024 == 0 && kOStageBytes % 1024 == 0 &&
                  kCS * 64 * 4 <= 1024 && kSmemBytes <= 232448,
              "shared memory layout");

// Y^T (M = 128, N = 64 tokens) and X^T (M = 128, N = 128 key dims), double-buffered.
constexpr uint32_t kColY = 0, kColX = 64, kYXBuf = 192, kTmemCols = 512;

// Counters: kTRead iterations whose Y^T, X^T the chain has read out of tensor
// memory; kStored iterations whose dh' / dDelta copies have finished reading
// shared memory; kMasked iterations whose (q, dO) stage the dO' warps have
// finished with (for a ragged chunk: its rows past the end zeroed).
enum Ctr { kTRead, kStored, kMasked, kNumCtr };

struct Small {
    uint64_t cfull[kCS], cempty[kCS], ofull[kOS], hready[kHB], mmaB[2];
    uint32_t ctr[kNumCtr];
    int c_issued[kCS], o_issued[kOS], y_issued[2], x_issued[2];
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Small) <= 2048, "small area");

struct BwdDhParams {
    Dims d;
    const float *gamma;          // [T_total, Hv]
    const float *dht;            // [N, Hv, K, V] or null
    __nv_bfloat16 *dh_chunks;    // gradient w.r.t. each chunk's exit state, blocked: per (chunk, head)
                                 // V/32 slices of [4][128][8] (the tile layout of kHb)
    __nv_bfloat16 *ddelta;       // dDelta, blocked: per (chunk, head) V/32 slices of [4][64][8]
    float *dh0;                  // [N, Hv, K, V] or null
    float scale;
    // Sequence split: each sequence runs as nseg segments, contiguous runs of
    // ceil(chunks / nseg) chunks (CTA slot = sequence rank * nseg + segment).
    int nseg;
    int mode;                    // BwdDhMode
    const float *seg_dh;         // kBSegOut: [N * nseg, Hv, K, V] gradient at every segment's end
    float *seg_r;                // kBSegPass: [N * nseg, Hv, K, V] gradient at the start from a zero end
    float *seg_Q;                // kBSegPass: [N * nseg, Hv, K, K] the segment's operator
    unsigned *status;
};

enum BwdDhMode { kBWhole = 0, kBSegPass = 1, kBSegOut = 2 };

// Waits for the six 16x256b.x2 TMEM loads of a chain step (see tmem_wait_ld).
__device__ __forceinline__ void tmem_wait_ld6(uint32_t (&a)[8], uint32_t (&b)[8], uint32_t (&c)[8], uint32_t (&e)[8],
                                              uint32_t (&f)[8], uint32_t (&g)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]),
                   "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7]),
                   "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3]), "+r"(c[4]), "+r"(c[5]), "+r"(c[6]), "+r"(c[7]),
                   "+r"(e[0]), "+r"(e[1]), "+r"(e[2]), "+r"(e[3]), "+r"(e[4]), "+r"(e[5]), "+r"(e[6]), "+r"(e[7]),
                   "+r"(f[0]), "+r"(f[1]), "+r"(f[2]), "+r"(f[3]), "+r"(f[4]), "+r"(f[5]), "+r"(f[6]), "+r"(f[7]),
                   "+r"(g[0]), "+r"(g[1]), "+r"(g[2]), "+r"(g[3]), "+r"(g[4]), "+r"(g[5]), "+r"(g[6]), "+r"(g[7])
                 :
                 : "memory");
}

// dO' of a ragged chunk (kept out of line, off the full chunks' path): rows past
// the end get dO' = 0, and the dO rows there (read by Y^T) and the q rows (read
// by X^T) are zeroed in the stage; kAuxThreads threads, thread at.
__device__ __noinline__ void make_dop_ragged(uint32_t src, uint32_t dst, uint32_t qt, uint32_t gm, float scl, int len,
                                             int at) {
    for (int i = 0; i < 256 / kAuxThreads; ++i) {
        const int p = at + kAuxThreads * i, t = p >> 2;  // 16-byte piece p of row t
        uint32_t o4[4] = {0u, 0u, 0u, 0u};
        if (t < len) {
            const float f = scl * __expf(ld_shared_f32(gm + t * 4));
            const uint4 raw = ld_shared_v4(src + p * 16);
            const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
            for (int e = 0; e < 4; ++e) {
                const float2 v2 = unpack_bf16(w4[e]);
                o4[e] = pack_bf16(f * v2.x, f * v2.y);
            }
        } else {
            st_shared_v4(src + p * 16, 0u, 0u, 0u, 0u);
        }
        st_shared_v4(dst + p * 16, o4[0], o4[1], o4[2], o4[3]);
    }
    for (int i = at; i < (kChunk - len) * 16; i += kAuxThreads) {
        const int r = len + (i >> 4), c = i & 15;
        st_shared_v4(qt + (c >> 3) * 8192 + r * 128 + (c & 7) * 16, 0u, 0u, 0u, 0u);
    }
}

// Byte offset of (row, col) in a [rows][128] bf16 tile stored as two 64-column
// halves of 128-byte rows with 128-byte swizzle (what the TMA loads produce).
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
    return (uint32_t)((col >> 6) * 8192 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(kThreads, 1)
bwd_dh_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_p,
              const __grid_constant__ CUtensorMap tm_do, const BwdDhParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    Small *sm = reinterpret_cast<Small *>(smem + kSmall);
    volatile int *abort_flag = &sm->abort_flag;
    const uint32_t sb = smem_u32(smem);
    float *gam = reinterpret_cast<float *>(smem + kGam);

    const Dims &d = prm.d;
    const int nseg = prm.nseg;
    // 1-D grid, sequence-major in longest-first order (the longest scans start first)
    const int nsl = (d.V + (prm.mode == kBSegPass ? d.K : 0)) / kBV;
    const int slot = blockIdx.x / (d.Hv * nsl), rem = blockIdx.x % (d.Hv * nsl);
    const int n = seq_by_length(d, slot / nseg), sseg = slot % nseg, h = rem / nsl, zs = rem % nsl;
    const int c0 = zs * kBV;
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
    const bool outputs = prm.mode != kBSegPass;  // dh' and dDelta of every chunk

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
            mbar_init(&sm->mmaB[b], 2);  // the Y^T and the X^T issuer
            sm->y_issued[b] = sm->x_issued[b] = 0;
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

    // iteration it handles chunk nch - 1 - it of the sequence
    auto chunk_of = [&](int it) { return nch - 1 - it; };
    auto chunk_len = [&](int it) { return min(kChunk, sr.len - chunk_of(it) * kChunk); };

    if (warp < kChainWarps) {
        // =========================================================== chain
        const int x = warp;  // d quarter of the state, token quarter of dDelta
        const int g = lane >> 2, cq = lane & 3, li = lane & 7, mi = lane >> 3;
        const uint32_t gam_sb = sb + kGam;
        const float scl = prm.scale;
        // hs[mt][nt][e]: dh'^T[v = 16mt + g + 8(e>>1)][d = 32x + 8nt + 2cq + (e&1)]
        float hs[2][4][4];
        {
            const float *src = prm.mode == kBWhole ? (prm.dht ? prm.dht + ((size_t)n * d.Hv + h) * K * V : nullptr)
                               : prm.mode == kBSegOut ? prm.seg_dh + (seg_idx * d.Hv + h) * K * V
                                                      : nullptr;
            const bool ident = prm.mode == kBSegPass && c0 >= V;  // operator columns start as I
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
        for (int it = 0; it < nch; ++it) {
            const int s = it % kCS, hb = it % kHB;
            const int len = chunk_len(it);
            const uint32_t st = sb + kC0 + s * kCStageBytes;
            const uint32_t hbuf = sb + kHb + hb * 8192, dbuf = sb + kDb + hb * 4096;
            bool good = wait_bar(&sm->cfull[s], (it / kCS) & 1, abort_flag);
            if (lane == 0 && outputs && it >= kHB)  // buffer hb was last copied out for iteration it - kHB
                good = good && wait_ge(&ctr[kStored], it - kHB + 1, abort_flag);
            good = __all_sync(0xffffffffu, good);
            // own quarter of dh' as bf16 A fragments: ao[mt][kk] for k-step 2x + kk
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
            // D1 accumulators [m-tile][token n-tile], two independent sets (even / odd k-steps)
            float acc[2][2][4] = {}, acc2[2][2][4] = {};
            float gC = 0.f, sc[2][2] = {};
            uint32_t bk[8][4];  // K fragments (B of D1): bk[2 o + kk] is k-step 2((x + o) & 3) + kk
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
                        ldsm_x4(bk[2 * o + kk],
                                st + kK + sw_off(16 * x + 8 * (mi >> 1) + li, 16 * (2 * ((x + o) & 3) + kk) + 8 * (mi & 1)));
                const uint32_t gm = gam_sb + s * kChunk * 4;
                gC = ld_shared_f32(gm + (kChunk - 1) * 4);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) sc[nt][e] = __expf(gC - ld_shared_f32(gm + (16 * x + 8 * nt + 2 * cq + e) * 4));
                if (len < kChunk) {
                    // a ragged chunk: zero the w rows past its end (their dDelta is zero, but a
                    // non-finite value of the next packed sequence would still turn 0 * x into NaN
                    // in the update); the barrier below orders this before every update load
                    for (int i = tid; i < (kChunk - len) * 16; i += kChainWarps * 32) {
                        const int r = len + (i >> 4), c = i & 15;
                        st_shared_v4(st + kW + (c >> 3) * 8192 + r * 128 + (c & 7) * 16, 0u, 0u, 0u, 0u);
                    }
                }
                // D1 over this warp's own quarter of d (registers): k-steps 2x, 2x+1
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    hmma(acc[mt][0], ao[mt][0], bk[0][0], bk[0][1]);
                    hmma(acc[mt][1], ao[mt][0], bk[0][2], bk[0][3]);
                    hmma(acc2[mt][0], ao[mt][1], bk[1][0], bk[1][1]);
                    hmma(acc2[mt][1], ao[mt][1], bk[1][2], bk[1][3]);
                }
            }
            ok = role_sync_and<128>(1, good);  // every quarter of dh' is in hbuf
            if (!ok) break;
            // Y^T and X^T of this chunk (issued a chunk or more ahead): this warp's token quarter
            // of Y^T and d quarter of X^T for all 32 value rows (lanes 32x + 16mt + .., the
            // M = 128 rows repeating the slice), loaded now and waited for after D1
            bool yx = true;
            if (lane == 0) yx = wait_bar(&sm->mmaB[it & 1], (it >> 1) & 1, abort_flag);
            __syncwarp();
            tc_fence_after();
            uint32_t yr[2][8], xr[2][2][8];
            {
                const uint32_t tb = tmem + (it & 1) * kYXBuf;
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    const uint32_t lb = (uint32_t)(32 * x + 16 * mt) << 16;
                    tmem_ld16x256_x2_nowait(tb + lb + kColY + 16 * x, yr[mt]);
                    tmem_ld16x256_x2_nowait(tb + lb + kColX + 32 * x, xr[mt][0]);
                    tmem_ld16x256_x2_nowait(tb + lb + kColX + 32 * x + 16, xr[mt][1]);
                }
            }
            // D1 over the other three quarters, A fragments of dh' from hbuf
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
                        float(&A)[2][2][4] = kk ? acc2 : acc;
                        hmma(A[mt][0], ah[mt][kk], bk[2 * o + kk][0], bk[2 * o + kk][1]);
                        hmma(A[mt][1], ah[mt][kk], bk[2 * o + kk][2], bk[2 * o + kk][3]);
                    }
            }
            tmem_wait_ld6(yr[0], yr[1], xr[0][0], xr[0][1], xr[1][0], xr[1][1]);
            tc_fence_before();
            // dDelta = e^{gamma_C - gamma} D1 + scale Y on live tokens (a select, so nothing past
            // the end leaks in); -dDelta^T as the A fragment of the update for this token quarter
            uint32_t da[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                float dl[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dl[nt][e] = 16 * x + 8 * nt + 2 * cq + (e & 1) < len
                                        ? fmaf(sc[nt][e & 1], acc[mt][nt][e] + acc2[mt][nt][e],
                                               scl * __uint_as_float(yr[mt][4 * nt + e]))
                                        : 0.f;
                uint32_t du[4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    da[mt][2 * nt] = pack_bf16(-dl[nt][0], -dl[nt][1]);
                    da[mt][2 * nt + 1] = pack_bf16(-dl[nt][2], -dl[nt][3]);
                    du[2 * nt] = pack_bf16(dl[nt][0], dl[nt][1]);
                    du[2 * nt + 1] = pack_bf16(dl[nt][2], dl[nt][3]);
                }
                // A fragment order: (v 0-7, t 0-7), (v 8-15, t 0-7), (v 0-7, t 8-15), (v 8-15, t 8-15)
                st_shared_v4(sb + kXb + (mt * 4 + x) * 512 + lane * 16, da[mt][0], da[mt][1], da[mt][2], da[mt][3]);
                if (outputs) stsm_x4_t(dbuf + (2 * mt + (mi & 1)) * 1024 + (16 * x + 8 * (mi >> 1) + li) * 16, du);
            }
            // w fragments (B of the update): bw[o] is token quarter (x + o) & 3, this warp's d quarter
            uint32_t bw[4][2][4];
#pragma unroll
            for (int o = 0; o < 4; ++o)
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    const int tq = (x + o) & 3;
                    ldsm_x4_t(bw[o][np], st + kW + sw_off(16 * tq + 8 * (mi & 1) + li, 32 * x + 16 * np + 8 * (mi >> 1)));
                }
            const float eC = __expf(gC);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        hs[mt][nt][e] = fmaf(eC, hs[mt][nt][e], __uint_as_float(xr[mt][nt >> 1][4 * (nt & 1) + e]));
            // update for the own token quarter: dh^T[:, own d quarter] += (-dDelta)^T w
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    hmma(hs[mt][2 * np], da[mt], bw[0][np][0], bw[0][np][1]);
                    hmma(hs[mt][2 * np + 1], da[mt], bw[0][np][2], bw[0][np][3]);
                }
            // every token quarter of -dDelta^T is in kXb, and every warp has read Y^T, X^T
            ok = role_sync_and<128>(1, __all_sync(0xffffffffu, yx));
            if (!ok) break;
            if (tid == 0) publish(&ctr[kTRead], it + 1);
            {
                float h2[2][4][4] = {};  // second accumulator set (latency)
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
                            float(&H)[2][4][4] = (o & 1) ? h2 : hs;
                            hmma(H[mt][2 * np], pa[mt], bw[o][np][0], bw[o][np][1]);
                            hmma(H[mt][2 * np + 1], pa[mt], bw[o][np][2], bw[o][np][3]);
                        }
                }
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) hs[mt][nt][e] += h2[mt][nt][e];
            }
            // dh' and dDelta of this chunk (generic writes) go to the bulk copies (async
            // proxy); the stage is free for the producer, and kXb for the next chunk
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
                if (outputs) mbar_arrive(&sm->hready[hb]);
                mbar_arrive(&sm->cempty[s]);
            }
        }
        if (!ok) {
            if (tid == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        } else {
            // end state: dh0 (from the CTA holding the sequence's first chunk), or the
            // segment's r / Q columns
            float *dst = nullptr;
            int ld = V;
            if (prm.mode == kBSegPass) {
                if (c0 < V) dst = prm.seg_r + (seg_idx * d.Hv + h) * K * V + c0;
                else dst = prm.seg_Q + (seg_idx * d.Hv + h) * K * K + (c0 - V), ld = K;
            } else if (prm.dh0 && sseg == 0) {
                dst = prm.dh0 + ((size_t)n * d.Hv + h) * K * V + c0;
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
    } else if (warp < kAuxWarp0 + kAuxWarps) {
        // ======================================================= dO' makers
        // dO' = scale e^gamma o dO of iteration it, in the layout of the dO tile (a row of 32
        // values is 64 contiguous bytes whatever the swizzle), once the tile has landed and
        // X^T of iteration it - 2 (the buffer's last reader) has been read by the chain; then
        // thread 0 of the role issues X^T
        const int at = tid - kAuxWarp0 * 32;
        const float scl = prm.scale;
        bool ok = true;
        for (int it = 0; it < nch && ok; ++it) {
            const int s = it % kOS, len = chunk_len(it);
            // the dO tile, and the chunk's gates in the chain ring (staged before the chain
            // reaches the chunk; the stage cannot be refilled before this chunk's X^T is read)
            bool good = wait_bar(&sm->ofull[s], (it / kOS) & 1, abort_flag) &&
                        wait_bar(&sm->cfull[it % kCS], (it / kCS) & 1, abort_flag);
            if (good && at == 0 && it >= 2) good = wait_ge(&ctr[kTRead], it - 1, abort_flag);
            ok = role_sync_and<kAuxThreads>(2, good);
            if (!ok) break;
            const uint32_t src = sb + kO0 + s * kOStageBytes + kDO, dst = sb + kDO2 + (it & 1) * 4096;
            const uint32_t gm = sb + kGam + (it % kCS) * kChunk * 4;
            if (len == kChunk) {
#pragma unroll
                for (int i = 0; i < 256 / kAuxThreads; ++i) {
                    const int p = at + kAuxThreads * i, t = p >> 2;  // 16-byte piece p of row t
                    const float f = scl * __expf(ld_shared_f32(gm + t * 4));
                    const uint4 raw = ld_shared_v4(src + p * 16);
                    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
                    uint32_t o4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 v2 = unpack_bf16(w4[e]);
                        o4[e] = pack_bf16(f * v2.x, f * v2.y);
                    }
                    st_shared_v4(dst + p * 16, o4[0], o4[1], o4[2], o4[3]);
                }
            } else {
                make_dop_ragged(src, dst, sb + kO0 + s * kOStageBytes + kQ, gm, scl, len, at);
            }
            fence_proxy_async();
            named_sync<kAuxThreads>(2);  // all of dO' is written (and a ragged chunk's rows zeroed)
            if (at == 0) publish(&ctr[kMasked], it + 1);
            if (at == 0) {
                // X^T = dO'^T Q: A = dO' read transposed (MN-major), its one 32-column atom repeated
                // over the M = 128 rows (zero stride between atoms); B = the q tile (MN-major, two
                // 64-column halves)
                tc_fence_after();
                const uint32_t tb = tmem + (it & 1) * kYXBuf, stq = sb + kO0 + s * kOStageBytes;
                const uint32_t id_X = idesc_bf16(128, 128, true, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tb + kColX, smem_desc(dst + ks * 1024, 0, 512, kSw64),
                             smem_desc(stq + kQ + ks * 2048, 8192, 1024, kSw128), id_X, ks > 0);
                mma_commit(&sm->mmaB[it & 1]);
                ++sm->x_issued[it & 1];
            }
        }
        if (!ok) {
            if (at == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        }
    } else if (warp == kIssuerWarp) {
        // ========================================================== issuer
        if (lane == 0) {
            bool ok = true;
            auto issue_out_loads = [&](int it) {
                const int s = it % kOS, ci = chunk_of(it);
                uint8_t *stg = smem + kO0 + s * kOStageBytes;
                const int t0 = sr.start + ci * kChunk, cg = sr.chunk0 + ci;
                mbar_arrive_expect_tx(&sm->ofull[s], kOStageBytes);
                ++sm->o_issued[s];
                tma_load_3d(stg + kQ, &tm_q, &sm->ofull[s], 0, hq, t0);
                tma_load_3d(stg + kQ + 8192, &tm_q, &sm->ofull[s], 64, hq, t0);
                tma_load_2d(stg + kP, &tm_p, &sm->ofull[s], 0, (cg * d.Hv + h) * kChunk);
                tma_load_3d(stg + kDO, &tm_do, &sm->ofull[s], c0, h, t0);  // out of range (zero) for operator columns
            };
            for (int c = 0; c < kOS && c < nch; ++c) issue_out_loads(c);
            const uint32_t id_Y = idesc_bf16(128, 64, true, true);
            for (int it = 0; it < nch && ok; ++it) {
                // the tiles of iteration it landed, and the chain has read the TMEM buffer's
                // previous contents (iteration it - 2)
                const int s = it % kOS;
                ok = wait_bar(&sm->ofull[s], (it / kOS) & 1, abort_flag) &&
                     (it < 2 || wait_ge(&ctr[kTRead], it - 1, abort_flag)) &&
                     (chunk_len(it) == kChunk || wait_ge(&ctr[kMasked], it + 1, abort_flag));  // dO rows zeroed
                if (!ok) break;
                tc_fence_after();
                const uint32_t stq = sb + kO0 + s * kOStageBytes;
                const uint32_t tb = tmem + (it & 1) * kYXBuf;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    // Y^T = dO^T P: A = the dO tile read transposed (MN-major), its one 32-column atom
                    // repeated over the M = 128 rows (zero stride between atoms); B = P (MN-major)
                    mma_bf16(tb + kColY, smem_desc(stq + kDO + ks * 1024, 0, 512, kSw64),
                             smem_desc(stq + kP + ks * 2048, 8192, 1024, kSw128), id_Y, ks > 0);
                mma_commit(&sm->mmaB[it & 1]);
                ++sm->y_issued[it & 1];
                // iteration it - 1's products are complete once the chain has read them: its
                // (q, P, dO) stage takes iteration it - 1 + kOS
                if (it >= 1 && it - 1 + kOS < nch) {
                    ok = wait_ge(&ctr[kTRead], it, abort_flag);
                    if (!ok) break;
                    issue_out_loads(it - 1 + kOS);
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
        // (each lane's arrival raises its pending count until the copies land), then k, w by TMA
        auto stage_chunk = [&](int it) {
            const int s = it % kCS, ci = chunk_of(it);
            const int t0 = sr.start + ci * kChunk, len = chunk_len(it);
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
            }
            __syncwarp();
        };
        for (int c = 0; c < kCS && c < nch; ++c) stage_chunk(c);
        for (int it = 0; it < nch && ok; ++it) {
            // iteration it done by the chain: its stage takes iteration it + kCS
            if (it + kCS < nch) {
                ok = wait_bar(&sm->cempty[it % kCS], (it / kCS) & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                stage_chunk(it + kCS);
            }
            if (outputs) {
                // dh' and dDelta of iteration it out of buffer it % kHB, one bulk copy each
                ok = wait_bar(&sm->hready[it % kHB], (it / kHB) & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                if (lane == 0) {
                    const size_t blk = ((size_t)(sr.chunk0 + chunk_of(it)) * d.Hv + h) * (V / kBV) + zs;
                    bulk_store(prm.dh_chunks + blk * (K * kBV), sb + kHb + (it % kHB) * 8192, K * kBV * 2);
                    bulk_store(prm.ddelta + blk * (kChunk * kBV), sb + kDb + (it % kHB) * 4096, kChunk * kBV * 2);
                    bulk_commit();
                    bulk_wait_read<0>();
                    publish(&ctr[kStored], it + 1);
                }
                __syncwarp();
            }
        }
        if (!ok) {
            if (lane == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        if (lane == 0) bulk_wait_all();  // the copies complete before the CTA's shared memory goes away
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        // let every TMA load and MMA still in flight finish (bounded) before the CTA exits:
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
        // (a use whose other product was never issued cannot complete: that wait runs out)
        for (int b = 0; b < 2; ++b) {
            const int uses = max(sm->y_issued[b], sm->x_issued[b]);
            if (uses > 0)
                while (!mbar_try_wait(smem_u32(&sm->mmaB[b]), (uses - 1) & 1) && globaltimer() - t0 < kWaitNs) {
                }
        }
    }
    __syncthreads();
    if (warp == kIssuerWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool tc_bwd_supported(const Dims &d, int dtype) {
    return dtype == GDN_DTYPE_BF16 && d.K == 128 && d.V == 128;
}

cudaError_t launch_bwd_dh_tc(const BwdArgs &a, const void *w16, const void *p16, void *dh_chunks16, void *ddelta16,
                             const BwdSplit &split) {
    const Dims &d = a.d;
    if (d.N == 0) return cudaSuccess;
    CUtensorMap mq, mk, mw, mp, mdo;
    const cuuint64_t T = (cuuint64_t)(d.T_total > 0 ? d.T_total : 1);
    const cuuint64_t dq[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hq, T};
    const cuuint64_t sq[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hq * d.K * 2};
    const cuuint32_t b64[3] = {64, 1, 64};
    const cuuint64_t dw[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hv, T};
    const cuuint64_t sw[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hv * d.K * 2};
    const cuuint64_t dv[3] = {(cuuint64_t)d.V, (cuuint64_t)d.Hv, T};
    const cuuint64_t sv[2] = {(cuuint64_t)d.V * 2, (cuuint64_t)d.Hv * d.V * 2};
    const cuuint32_t bv[3] = {kBV, 1, 64};
    const cuuint64_t dp[2] = {64, (cuuint64_t)(d.NC > 0 ? d.NC : 1) * d.Hv * 64};
    const cuuint64_t sp[1] = {128};
    const cuuint32_t bp[2] = {64, 64};
    if (!make_bf16_map(&mq, a.q, 3, dq, sq, b64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map(&mk, a.k, 3, dq, sq, b64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map(&mw, w16, 3, dw, sw, b64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map(&mp, p16, 2, dp, sp, bp, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map(&mdo, a.d_o, 3, dv, sv, bv, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    BwdDhParams p;
    p.d = d;
    p.gamma = a.gamma;
    p.dht = a.dht;
    p.dh_chunks = (__nv_bfloat16 *)dh_chunks16;
    p.ddelta = (__nv_bfloat16 *)ddelta16;
    p.dh0 = a.dh0;
    p.scale = d.scale;
    p.nseg = split.nseg > 0 ? split.nseg : 1;
    p.mode = split.mode;
    p.seg_dh = split.seg_dh;
    p.seg_r = split.seg_r;
    p.seg_Q = split.seg_Q;
    if ((p.mode == kBSegPass && (!p.seg_r || !p.seg_Q)) || (p.mode == kBSegOut && !p.seg_dh) || p.mode < 0 ||
        p.mode > kBSegOut)
        return cudaErrorInvalidValue;
    p.status = a.status;
    cudaError_t e = cudaFuncSetAttribute(bwd_dh_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    // the segment pass also carries the K operator columns
    const long long nctas = (long long)d.N * p.nseg * d.Hv * ((d.V + (p.mode == kBSegPass ? d.K : 0)) / kBV);
    if (nctas >= (1ll << 31)) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)nctas);
    bwd_dh_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mk, mw, mp, mdo, p);
    return cudaGetLastError();
}

}  // namespace gdn
