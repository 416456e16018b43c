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
// Organised like the forward chain kernel (gdn_fwd3.cu): one CTA per
// (sequence, value head, 32-column slice of V), w and P = M o Q K^T of every
// chunk from the chunk-prep kernel through a TMA ring, 416 threads:
//   warps 0-7   chain: dh' (128 x 32 fp32) in mma.sync fragments; per chunk
//               A = K dh', dDelta = e^{gamma_C - gamma} A + scale Y, then
//               dh = e^{gamma_C} dh' + X - w^T dDelta, with Y and X read
//               straight from tensor memory (the 16x256b load layout is the
//               mma.sync accumulator layout, and chain warp p sits on TMEM
//               sub-partition p);
//   warps 8-11  aux: dO' = scale e^gamma o dO into shared memory, one chunk
//               ahead of the chain, and the copies of dh' and dDelta from
//               shared memory to global memory, off the chain's path;
//   warp 12     issuer: TMA ring (q, k, w, P, dO per chunk) and, on tcgen05,
//               Y = P^T dO and X = Q^T dO' into double-buffered TMEM.
// Y and X do not depend on the chain, so they are ready one or two chunks
// ahead of it. Hand-over by release/acquire counters and mbarriers; every wait
// is bounded.
//
// Sequence split (long sequences, few heads): a chunk maps its exit-state
// gradient dh' to dh = A dh' + b with A = e^{gamma_C} I - w^T diag(e^{gamma_C -
// gamma}) K, the transpose of the forward chunk's transition operator, so a
// segment of chunks maps the gradient at its end to Q dh_end + r. The segment
// pass runs the scan on [r | Q]: r from zero with the real dO, Q from the identity
// on K more columns whose dO tile is read out of range (zero), so Y = X = 0
// there. A composition walks the segments backwards from dht (gdn_split.cu), and
// the output pass reruns every segment from its composed dh_end.
#include <cstddef>

#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kThreads = 416;
constexpr int kRole = 256;  // chain threads
constexpr int kAux = 128;
constexpr int kBV = 32;
constexpr int kStages = 3;

// ---- shared memory (bytes from a 1024-aligned base)
constexpr int kHb = 0;          // 8192       dh' (bf16): (n/8)*2048 + (k/8)*128 + (k%8)*16
constexpr int kDb = 8192;       // 4096       -dDelta (bf16): (n/8)*1024 + (t/8)*128 + (t%8)*16
constexpr int kDO2 = 12288;     // 2 x 4096   dO' (bf16), layout of kDb (B of X)
constexpr int kStage0 = 20480;  // TMA ring
// per stage: q, k, w [64][128] bf16 (two 64-column halves, 128-byte swizzle),
// P [64][64] bf16 (128-byte swizzle), dO [64][32] bf16 (64-byte swizzle)
constexpr int kQ = 0, kK = 16384, kW = 32768, kP = 49152, kDO = 57344, kStageBytes = 61440;
constexpr int kTxBytes = 3 * 16384 + 8192 + 4096;
constexpr int kSmall = kStage0 + kStages * kStageBytes;
constexpr int kSmemBytes = kSmall + 2048 + 1024;
static_assert(kStage0 % 1024 == 0 && kStageBytes % 1024 == 0 && kSmemBytes <= 232448, "shared memory layout");

// Tensor memory: two buffers of 64 columns, Y (M = 64) | X (M = 128).
constexpr uint32_t kColY = 0, kColX = 32, kYBuf = 64, kTmemCols = 128;

// kHbFull / kDbFull: the chain has put dh' / -dDelta of an iteration in kHb / kDb;
// kHbRead / kDbRead: the aux warps have copied them to global memory.
enum Ctr { kPReady, kStage, kHbFull, kDbFull, kHbRead, kDbRead, kNumCtr };

struct Small {
    uint64_t full[kStages];
    uint64_t mmaB[2];
    uint32_t ctr[kNumCtr];
    int loads_issued, loads_landed, mma_issued, mma_seen;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Small) <= 2048, "small area");

__device__ __forceinline__ bool chain_sync(bool pred) { return role_sync_and<kRole>(1, pred); }
__device__ __forceinline__ bool aux_sync(bool pred) { return role_sync_and<kAux>(2, pred); }

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

__global__ void __launch_bounds__(kThreads, 1)
bwd_dh_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_p,
              const __grid_constant__ CUtensorMap tm_do, const BwdDhParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    Small *sm = reinterpret_cast<Small *>(smem + kSmall);
    volatile int *abort_flag = &sm->abort_flag;
    const uint32_t sb = smem_u32(smem);

    const Dims &d = prm.d;
    const int nseg = prm.nseg;
    // 1-D grid, sequence-major in longest-first order (the longest scans start first)
    const int nsl = (d.V + (prm.mode == kBSegPass ? d.K : 0)) / kBV;
    const int slot = blockIdx.x / (d.Hv * nsl), rem = blockIdx.x % (d.Hv * nsl);
    const int n = seq_by_length(d, slot / nseg), sseg = slot % nseg, h = rem / nsl, zs = rem % nsl;
    const int c0 = zs * kBV;
    const int hq = h / (d.Hv / d.Hq);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
    constexpr int K = 128, V = 128;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&sm->full[s], 1);
        mbar_init(&sm->mmaB[0], 1);
        mbar_init(&sm->mmaB[1], 1);
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

    // iteration it handles chunk nch - 1 - it of the sequence
    auto chunk_of = [&](int it) { return nch - 1 - it; };
    auto gamma_at = [&](int it, int r) {
        const int ci = chunk_of(it), len = min(kChunk, sr.len - ci * kChunk);
        return prm.gamma[(size_t)(sr.start + ci * kChunk + min(r, len - 1)) * d.Hv + h];
    };

    if (warp < 8) {
        // =========================================================== chain
        const int p = warp & 3, cb = (warp >> 2) * 2;  // state rows 32p.., n-tiles cb, cb+1
        const int g = lane >> 2, c4 = lane & 3;
        const uint32_t lane_base = (uint32_t)(p * 32) << 16;
        const float scl = prm.scale;
        float hf[2][2][4];  // [m-tile][n-tile][frag]: rows 32p+16mt+g(+8), cols 8(cb+nt)+2c4(+1)
        {
            const float *src = prm.mode == kBWhole ? (prm.dht ? prm.dht + ((size_t)n * d.Hv + h) * K * V : nullptr)
                               : prm.mode == kBSegOut ? prm.seg_dh + (seg_idx * d.Hv + h) * K * V
                                                      : nullptr;
            const bool ident = prm.mode == kBSegPass && c0 >= V;  // operator columns start as I
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
        auto write_hb = [&]() {
            const uint32_t base = sb + kHb + c4 * 4;
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
        write_hb();
        bool ok = true;
        float gl = 0.f, gt0 = 0.f, gt1 = 0.f;
        if (nch > 0) gl = gamma_at(0, 63), gt0 = gamma_at(0, 16 * p + g), gt1 = gamma_at(0, 16 * p + g + 8);
        for (int it = 0; it < nch && ok; ++it) {
            const int ci = chunk_of(it);
            const int len = min(kChunk, sr.len - ci * kChunk);
            const uint32_t st = sb + kStage0 + (it % kStages) * kStageBytes;
            // stage landed (and every warp's dh' is in kHb: the barrier orders them)
            ok = chain_sync(wait_bar(&sm->full[it % kStages], (it / kStages) & 1, abort_flag));
            if (!ok) break;
            if (tid == 0) {
                sm->loads_landed = it + 1;
                publish(&ctr[kHbFull], it + 1);  // kHb holds dh' of this chunk (written before the barrier)
            }
            const float gC = gl, gtok[2] = {gt0, gt1};
            if (it + 1 < nch) gl = gamma_at(it + 1, 63), gt0 = gamma_at(it + 1, 16 * p + g), gt1 = gamma_at(it + 1, 16 * p + g + 8);
            // ---- Y and X of this chunk from tensor memory (issued now, waited after A)
            // Y, X of this chunk computed; the aux has copied the previous -dDelta out of kDb
            ok = chain_sync(wait_bar(&sm->mmaB[it & 1], (it >> 1) & 1, abort_flag) &&
                            (tid != 0 || it < 1 || wait_ge(&ctr[kDbRead], it, abort_flag)));
            if (!ok) break;
            if (tid == 0) sm->mma_seen = it + 1;
            tc_fence_after();
            uint32_t yr[8], xr0[8], xr1[8];
            {
                const uint32_t tb = tmem + (it & 1) * kYBuf + 8 * cb;
                tmem_ld16x256_x2_nowait(tb + lane_base + kColY, yr);                       // tokens 16p + (g, g+8)
                tmem_ld16x256_x2_nowait(tb + lane_base + kColX, xr0);                      // state rows 32p + (g, g+8)
                tmem_ld16x256_x2_nowait(tb + lane_base + ((uint32_t)16 << 16) + kColX, xr1);  // rows 32p + 16 + ..
            }
            // ---- A = K dh' : tokens 16p..16p+15, columns of n-tiles cb, cb+1
            float acc[2][4] = {};
            {
                const uint32_t kt = st + kK;
                const int arow = 16 * p + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int mi = lane >> 3;
                uint32_t a[2][4], b[2][4];
                auto load = [&](int ks, int buf) {
                    const int d0 = 16 * ks + (lane >> 4) * 8;
                    ldsm_x4(a[buf], kt + (d0 >> 6) * 8192 + arow * 128 + ((((d0 & 63) >> 3) ^ (arow & 7)) << 4));
                    ldsm_x4_t(b[buf], sb + kHb + (cb + (mi >> 1)) * 2048 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
                };
                load(0, 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    if (ks + 1 < 8) load(ks + 1, (ks + 1) & 1);
                    hmma(acc[0], a[ks & 1], b[ks & 1][0], b[ks & 1][1]);
                    hmma(acc[1], a[ks & 1], b[ks & 1][2], b[ks & 1][3]);
                }
            }
            tmem_wait_ld3(yr, xr0, xr1);
            tc_fence_before();
            // ---- dDelta = e^{gamma_C - gamma} A + scale Y; -dDelta -> kDb
            {
                const uint32_t db = sb + kDb + c4 * 4;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int tok = 16 * p + g + half * 8;
                    const bool live = tok < len;
                    const float sc = __expf(gC - gtok[half]);
                    const uint32_t off = (tok >> 3) * 128 + (tok & 7) * 16;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const float y0 = __uint_as_float(yr[4 * nt + 2 * half]), y1 = __uint_as_float(yr[4 * nt + 2 * half + 1]);
                        const float x0 = live ? fmaf(sc, acc[nt][2 * half], scl * y0) : 0.f;
                        const float x1 = live ? fmaf(sc, acc[nt][2 * half + 1], scl * y1) : 0.f;
                        st_shared_b32(db + (cb + nt) * 1024 + off, pack_bf16(-x0, -x1));
                    }
                }
            }
            chain_sync(true);  // every warp reads all 64 tokens of dDelta below
            if (tid == 0) publish(&ctr[kDbFull], it + 1);
            // ---- dh = e^{gamma_C} dh' + X + w^T (-dDelta) : rows 32p..+31, 16 columns, K = 64 tokens
            {
                const float eC = __expf(gC);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    const uint32_t(&xr)[8] = mt ? xr1 : xr0;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int q = 0; q < 4; ++q) hf[mt][nt][q] = fmaf(eC, hf[mt][nt][q], __uint_as_float(xr[4 * nt + q]));
                }
                const uint32_t wt = st + kW;
                const int mi = lane >> 3;
                uint32_t b[2][4], a[2][2][4];
                auto load = [&](int ks, int buf) {
                    ldsm_x4_t(b[buf], sb + kDb + (cb + (mi >> 1)) * 1024 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        // A = w^T rows (state rows) 32p+16mt.., cols (tokens) 16ks..: the
                        // token-major, 128-byte-swizzled w tile read transposed
                        const int tt = 16 * ks + (lane & 7) + ((mi >> 1) & 1) * 8;
                        const int dd = 32 * p + 16 * mt + (mi & 1) * 8;
                        ldsm_x4_t(a[buf][mt], wt + (dd >> 6) * 8192 + tt * 128 + ((((dd & 63) >> 3) ^ (tt & 7)) << 4));
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
            // all reads of kHb, kDb, the stage and this TMEM buffer are done; dh' of this
            // chunk has been copied out of kHb
            ok = chain_sync(tid != 0 || wait_ge(&ctr[kHbRead], it + 1, abort_flag));
            if (!ok) break;
            if (tid == 0) publish(&ctr[kStage], it + 1);
            write_hb();
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
        // ============================================================= aux
        const int atid = tid - kRole;
        const float scl = prm.scale;
        bool ok = true;
        // thread: 16-byte chunks e = atid and atid + 128 of the 64 x 32 dO tile
        const int ta = atid >> 2, tb2 = (atid + kAux) >> 2, cc = atid & 3;
        float ga = 0.f, gb = 0.f;
        if (nch > 0) ga = gamma_at(0, ta), gb = gamma_at(0, tb2);
        // dO' of iteration it into dO'[it % 2] once its stage has landed and X of
        // iteration it - 2 (the buffer's last reader) is done
        auto make_do = [&](int it) -> bool {
            const int ci = chunk_of(it);
            const int len = min(kChunk, sr.len - ci * kChunk);
            if (!aux_sync(wait_bar(&sm->full[it % kStages], (it / kStages) & 1, abort_flag) &&
                          (atid != 0 || it < 2 || wait_ge(&ctr[kStage], it - 1, abort_flag))))
                return false;
            const float fa = ta < len ? scl * __expf(ga) : 0.f, fb = tb2 < len ? scl * __expf(gb) : 0.f;
            if (it + 1 < nch) ga = gamma_at(it + 1, ta), gb = gamma_at(it + 1, tb2);
            const uint32_t stg = sb + kStage0 + (it % kStages) * kStageBytes + kDO;
            const uint32_t ob = sb + kDO2 + (it & 1) * 4096;
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
                const int t = e2 ? tb2 : ta;
                const float f = e2 ? fb : fa;
                // dO tile: 64-byte rows, 16-byte chunks XOR ((row / 2) % 4)
                const uint4 raw = ld_shared_v4(stg + t * 64 + ((cc ^ ((t >> 1) & 3)) << 4));
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = unpack_bf16(w[e]);
                    o[e] = pack_bf16(f * x.x, f * x.y);
                }
                st_shared_v4(ob + cc * 1024 + (t >> 3) * 128 + (t & 7) * 16, o[0], o[1], o[2], o[3]);
            }
            fence_proxy_async();
            aux_sync(true);
            if (atid == 0) publish(&ctr[kPReady], it + 1);
            return true;
        };
        if (nch > 0) ok = make_do(0);
        for (int it = 0; it < nch && ok; ++it) {
            const int ci = chunk_of(it);
            if (it + 1 < nch) {
                ok = make_do(it + 1);  // one iteration ahead of the chain
                if (!ok) break;
            }
            // dh' of this iteration: kHb -> dh_chunks, one contiguous block per (chunk, head,
            // column slice) in the tile layout
            ok = aux_sync(atid != 0 || wait_ge(&ctr[kHbFull], it + 1, abort_flag));
            if (!ok) break;
            {
                __nv_bfloat16 *hc = prm.dh_chunks + (((size_t)(sr.chunk0 + ci) * d.Hv + h) * (V / kBV) + zs) * (K * kBV);
#pragma unroll
                for (int i = 0; i < 4 && outputs; ++i) {
                    const int e = atid + kAux * i;  // 16-byte piece e = (n/8) * 128 + k
                    *reinterpret_cast<uint4 *>(hc + 8 * e) = ld_shared_v4(sb + kHb + e * 16);
                }
            }
            aux_sync(true);
            if (atid == 0) publish(&ctr[kHbRead], it + 1);
            // dDelta of this iteration: kDb holds -dDelta -> ddelta, one contiguous block per
            // (chunk, head, column slice) in the tile layout (rows past a ragged chunk's end
            // are zero), sign restored
            ok = aux_sync(atid != 0 || wait_ge(&ctr[kDbFull], it + 1, abort_flag));
            if (!ok) break;
            {
                __nv_bfloat16 *dc = prm.ddelta + (((size_t)(sr.chunk0 + ci) * d.Hv + h) * (V / kBV) + zs) * (kChunk * kBV);
#pragma unroll
                for (int i = 0; i < 2 && outputs; ++i) {
                    const int e = atid + kAux * i;  // 16-byte piece e = (n/8) * 64 + t
                    uint4 v4 = ld_shared_v4(sb + kDb + e * 16);
                    v4.x ^= 0x80008000u, v4.y ^= 0x80008000u, v4.z ^= 0x80008000u, v4.w ^= 0x80008000u;
                    *reinterpret_cast<uint4 *>(dc + 8 * e) = v4;
                }
            }
            aux_sync(true);
            if (atid == 0) publish(&ctr[kDbRead], it + 1);
        }
        if (!ok) {
            if (atid == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        }
    } else {
        // ========================================================== issuer
        if (lane == 0) {
            bool ok = true;
            auto issue_loads = [&](int it) {
                const int s = it % kStages;
                uint8_t *stg = smem + kStage0 + s * kStageBytes;
                const int ci = chunk_of(it);
                const int t0 = sr.start + ci * kChunk;
                const int cg = sr.chunk0 + ci;
                mbar_arrive_expect_tx(&sm->full[s], kTxBytes);
                atomicAdd(&sm->loads_issued, 1);
                tma_load_3d(stg + kQ, &tm_q, &sm->full[s], 0, hq, t0);
                tma_load_3d(stg + kQ + 8192, &tm_q, &sm->full[s], 64, hq, t0);
                tma_load_3d(stg + kK, &tm_k, &sm->full[s], 0, hq, t0);
                tma_load_3d(stg + kK + 8192, &tm_k, &sm->full[s], 64, hq, t0);
                tma_load_3d(stg + kW, &tm_w, &sm->full[s], 0, h, t0);
                tma_load_3d(stg + kW + 8192, &tm_w, &sm->full[s], 64, h, t0);
                tma_load_2d(stg + kP, &tm_p, &sm->full[s], 0, (cg * d.Hv + h) * kChunk);
                tma_load_3d(stg + kDO, &tm_do, &sm->full[s], c0, h, t0);
            };
            for (int c = 0; c < kStages && c < nch; ++c) issue_loads(c);
            const uint32_t id_Y = idesc_bf16(64, 32, true, true);
            const uint32_t id_X = idesc_bf16(128, 32, true, true);
            for (int it = 0; it < nch && ok; ++it) {
                // Y, X of iteration it into buffer it % 2 once dO' is written and the chain
                // has read that buffer's previous contents (iteration it - 2). They depend on
                // loaded tiles only, so they are issued before the refill below, which waits
                // for the chain to finish iteration it - 1.
                ok = wait_ge(&ctr[kPReady], it + 1, abort_flag) && wait_ge(&ctr[kStage], it >= 1 ? it - 1 : 0, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = sb + kStage0 + (it % kStages) * kStageBytes;
                const uint32_t tb = tmem + (it & 1) * kYBuf, ob = sb + kDO2 + (it & 1) * 4096;
                for (int ks = 0; ks < 4; ++ks) {
                    // Y = P^T dO: A = P read transposed (MN-major), B = the dO tile; 16 rows of P per step
                    mma_bf16(tb + kColY, smem_desc(st + kP + ks * 2048, 8192, 1024, kSw128),
                             smem_desc(st + kDO + ks * 1024, 4096, 512, kSw64), id_Y, ks > 0);
                    // X = Q^T dO': A = the q tile read transposed (MN-major, two 64-row halves)
                    mma_bf16(tb + kColX, smem_desc(st + kQ + ks * 2048, 8192, 1024, kSw128),
                             smem_desc(ob + ks * 256, 128, 1024, kSwNone), id_X, ks > 0);
                }
                mma_commit(&sm->mmaB[it & 1]);
                sm->mma_issued = it + 1;
                // refill the stage of iteration it - 1 with iteration it + 2 once the chain is
                // done with it (which also means its Y, X and dO' are consumed)
                if (it >= 1 && it + 2 < nch) {
                    ok = wait_ge(&ctr[kStage], it, abort_flag);
                    if (!ok) break;
                    issue_loads(it + 2);
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
        // let every TMA load and every MMA still in flight finish (bounded) before the CTA exits
        const uint64_t t0 = globaltimer();
        for (int c = sm->loads_landed; c < sm->loads_issued; ++c)
            while (!mbar_try_wait(smem_u32(&sm->full[c % kStages]), (c / kStages) & 1) && globaltimer() - t0 < kWaitNs) {
            }
        for (int c = sm->mma_seen; c < sm->mma_issued; ++c)
            while (!mbar_try_wait(smem_u32(&sm->mmaB[c & 1]), (c >> 1) & 1) && globaltimer() - t0 < kWaitNs) {
            }
    }
    __syncthreads();
    if (warp == 12) {
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
