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
// (bf16, [NC, Hv, K, V]) and dDelta (bf16, [T, Hv, V]) are stored for the
// per-chunk gradient kernel; dh0 (fp32) is the gradient at the sequence start.
//
// Same organisation as the forward kernel (gdn_fwd2.cu): one CTA per
// (sequence, value head, 32-column slice of V) with 576 threads,
//   warps 0-7   chain: dh' (128 x 32 fp32) in mma.sync fragments; per chunk
//               A = K dh' then dh = e^{gamma_C} dh' + X + (-w)^T dDelta;
//   warps 8-15  aux: P = scale (M o S) and dO' = scale e^gamma o dO into shared
//               memory for issuer B; -w, Y, X from tensor memory into shared
//               memory for the chain;
//   warp 16     issuer A: TMA prologue, S = Q K^T and W = Aw K (tcgen05);
//   warp 17     issuer B: Y = P^T dO and X = Q^T dO' (tcgen05), TMA refills.
// None of the tcgen05 products depends on the chain, so they run ahead of it,
// bounded by the double-buffered tensor memory and the 3-deep TMA ring.
// Hand-over is by release/acquire counters and, where the hardware signals
// completion, mbarriers with a single consumer; every wait is bounded.
#include <cstddef>

#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kThreads = 576;
constexpr int kRole = 256;
constexpr int kBV = 32;
constexpr int kStages = 3;

// ---- shared memory (bytes from a 1024-aligned base)
constexpr int kHb = 0;          // 8192       dh' (bf16): (n/8)*2048 + (k/8)*128 + (k%8)*16, chain only
constexpr int kDb = 8192;       // 4096       dDelta (bf16): (n/8)*1024 + (t/8)*128 + (t%8)*16, chain only
constexpr int kDO2 = 12288;     // 2 x 4096   dO' (bf16), layout of kDb (B of X)
constexpr int kP = 20480;       // 2 x 8192   P [r][s], 128-byte swizzle (A of Y, read transposed)
constexpr int kWs = 36864;      // 16384      -w (bf16) in the k tile's layout (two 64-column halves)
constexpr int kY = 53248;       // 9216       Y (fp32) [t][36]
constexpr int kX = 62464;       // 18432      X (fp32) [k][36]
constexpr int kStage0 = 81920;  // TMA ring
constexpr int kQ = 0, kK = 16384, kAw = 32768, kDO = 40960, kStageBytes = 45056;
constexpr int kTxBytes = 16384 + 16384 + 8192 + 4096;
constexpr int kSmall = kStage0 + kStages * kStageBytes;
constexpr int kSmemBytes = kSmall + 2560 + 1024;
static_assert(kX + 18432 <= kStage0 && kP % 1024 == 0 && kStage0 % 1024 == 0 && kStageBytes % 1024 == 0 &&
                  kSmemBytes <= 232448,
              "shared memory layout");

// Tensor memory: two buffers of 256 columns, S | W | Y | X.
constexpr uint32_t kColS = 0, kColW = 64, kColY = 192, kColX = 224, kABuf = 256, kTmemCols = 512;

struct __align__(16) Gates {
    float gam[64], egam[64];
};

// Counters (number of iterations finished by the producer).
enum Ctr { kTmemA, kPReady, kReady, kWFree, kStage, kNumCtr };

struct Small {
    uint64_t full[kStages];
    uint64_t mmaA[2], mmaB[2];
    uint32_t ctr[kNumCtr];
    int loads_issued, loads_landed;
    uint32_t tmem_base;
    int abort_flag;
    Gates gates[3];
};
static_assert(sizeof(Small) <= 2560, "small area");
static_assert(kSmall % 16 == 0 && offsetof(Small, gates) % 16 == 0, "small area alignment");

__device__ __forceinline__ bool rsync(int id, bool pred) { return role_sync_and<kRole>(id, pred); }

struct BwdDhParams {
    Dims d;
    const float *gamma;          // [T_total, Hv]
    const float *dht;            // [N, Hv, K, V] or null
    __nv_bfloat16 *dh_chunks;    // [NC, Hv, K, V]: gradient w.r.t. each chunk's exit state
    __nv_bfloat16 *ddelta;       // [T_total, Hv, V]
    float *dh0;                  // [N, Hv, K, V] or null
    float scale;
    unsigned *status;
};

__global__ void __launch_bounds__(kThreads, 1)
bwd_dh_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_wy,
              const BwdDhParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    Small *sm = reinterpret_cast<Small *>(smem + kSmall);
    volatile int *abort_flag = &sm->abort_flag;
    const uint32_t sb = smem_u32(smem);

    const Dims &d = prm.d;
    const int n = blockIdx.x, h = blockIdx.y, c0 = blockIdx.z * kBV;
    const int hq = h / (d.Hv / d.Hq);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const SeqRange sr = seq_range(d, n);
    const int nch = (sr.len + kChunk - 1) / kChunk;
    constexpr int K = 128, V = 128;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&sm->full[s], 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->mmaA[b], 1);
            mbar_init(&sm->mmaB[b], 1);
        }
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

    // iteration it handles chunk nch - 1 - it of the sequence
    auto chunk_of = [&](int it) { return nch - 1 - it; };
    auto issue_loads = [&](int it) {
        const int s = it % kStages;
        uint8_t *st = smem + kStage0 + s * kStageBytes;
        const int ci = chunk_of(it);
        const int t0 = sr.start + ci * kChunk;
        const int cg = sr.chunk0 + ci;
        mbar_arrive_expect_tx(&sm->full[s], kTxBytes);
        atomicAdd(&sm->loads_issued, 1);
        tma_load_3d(st + kQ, &tm_q, &sm->full[s], 0, hq, t0);
        tma_load_3d(st + kQ + 8192, &tm_q, &sm->full[s], 64, hq, t0);
        tma_load_3d(st + kK, &tm_k, &sm->full[s], 0, hq, t0);
        tma_load_3d(st + kK + 8192, &tm_k, &sm->full[s], 64, hq, t0);
        tma_load_2d(st + kAw, &tm_wy, &sm->full[s], 0, ((cg * d.Hv + h) * 2 + 1) * kChunk);
        tma_load_3d(st + kDO, &tm_do, &sm->full[s], c0, h, t0);
    };

    if (warp < 8) {
        // =========================================================== chain
        const int p = warp & 3, cb = (warp >> 2) * 2;  // state rows 32p.., n-tiles cb, cb+1
        const int g = lane >> 2, c4 = lane & 3;
        float hf[2][2][4];  // [m-tile][n-tile][frag]: rows 32p+16mt+g(+8), cols 8(cb+nt)+2c4(+1)
        {
            const float *src = prm.dht ? prm.dht + ((size_t)n * d.Hv + h) * K * V : nullptr;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int dim = 32 * p + 16 * mt + g + ((q >> 1) << 3);
                        const int col = 8 * (cb + nt) + 2 * c4 + (q & 1);
                        hf[mt][nt][q] = src ? src[(size_t)dim * V + c0 + col] : 0.f;
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
        for (int it = 0; it < nch && ok; ++it) {
            const int ci = chunk_of(it);
            const int len = min(kChunk, sr.len - ci * kChunk);
            const int t0 = sr.start + ci * kChunk;
            {  // dh' of this chunk, rounded as the products read it
                __nv_bfloat16 *hc = prm.dh_chunks + ((size_t)(sr.chunk0 + ci) * d.Hv + h) * K * V + c0;
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
            // -w, Y, X of this chunk are in shared memory (and dh' in kHb from every warp)
            ok = rsync(1, wait_ge(&ctr[kReady], it + 1, abort_flag));
            if (!ok) break;
            const Gates &G = sm->gates[it % 3];
            const float gl = G.gam[63];
            const float gtok[2] = {G.gam[16 * p + g], G.gam[16 * p + g + 8]};
            // ---- A = K dh' : tokens 16p..16p+15, columns of n-tiles cb, cb+1
            float acc[2][4] = {};
            {
                const uint32_t kt = sb + kStage0 + (it % kStages) * kStageBytes + kK;
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
            // ---- dDelta = e^{gamma_C - gamma} A + Y  -> ddelta (global) and kDb
            {
                const float *Y = reinterpret_cast<const float *>(smem + kY);
                const uint32_t db = sb + kDb + c4 * 4;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int tok = 16 * p + g + half * 8;
                    const bool live = tok < len;
                    const float sc = __expf(gl - gtok[half]);
                    const uint32_t off = (tok >> 3) * 128 + (tok & 7) * 16;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int col = 8 * (cb + nt) + 2 * c4;
                        const float2 y = *reinterpret_cast<const float2 *>(Y + tok * 36 + col);
                        const float x0 = live ? fmaf(sc, acc[nt][2 * half], y.x) : 0.f;
                        const float x1 = live ? fmaf(sc, acc[nt][2 * half + 1], y.y) : 0.f;
                        const uint32_t pk = pack_bf16(x0, x1);
                        st_shared_b32(db + (cb + nt) * 1024 + off, pk);
                        if (live)
                            *reinterpret_cast<uint32_t *>(prm.ddelta + ((size_t)(t0 + tok) * d.Hv + h) * V + c0 + col) = pk;
                    }
                }
            }
            rsync(1, true);  // every warp reads all 64 tokens of dDelta below
            // ---- dh = e^{gamma_C} dh' + X + (-w)^T dDelta : rows 32p..+31, 16 columns, K = 64 tokens
            {
                const float eC = __expf(gl);
                const float *X = reinterpret_cast<const float *>(smem + kX);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int dim = 32 * p + 16 * mt + g + half * 8;
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
                            const float2 x = *reinterpret_cast<const float2 *>(X + dim * 36 + 8 * (cb + nt) + 2 * c4);
                            hf[mt][nt][2 * half] = fmaf(eC, hf[mt][nt][2 * half], x.x);
                            hf[mt][nt][2 * half + 1] = fmaf(eC, hf[mt][nt][2 * half + 1], x.y);
                        }
                    }
                const int mi = lane >> 3;
                uint32_t b[2][4], a[2][2][4];
                auto load = [&](int ks, int buf) {
                    ldsm_x4_t(b[buf], sb + kDb + (cb + (mi >> 1)) * 1024 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        // A = (-w)^T rows (state rows) 32p+16mt.., cols (tokens) 16ks..
                        const int tt = 16 * ks + (lane & 7) + ((mi >> 1) & 1) * 8;
                        const int dd = 32 * p + 16 * mt + (mi & 1) * 8;
                        ldsm_x4_t(a[buf][mt], sb + kWs + (dd >> 6) * 8192 + tt * 128 + ((((dd & 63) >> 3) ^ (tt & 7)) << 4));
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
            rsync(1, true);  // all reads of kHb, kDb, kWs, kX, kY and the k tile are done
            if (tid == 0) {
                publish(&ctr[kWFree], it + 1);
                publish(&ctr[kStage], it + 1);
            }
            write_hb();
        }
        if (!ok) {
            if (tid == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        } else if (prm.dh0) {
            float *dst = prm.dh0 + ((size_t)n * d.Hv + h) * K * V + c0;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int dim = 32 * p + 16 * mt + g + half * 8;
                        *reinterpret_cast<float2 *>(dst + (size_t)dim * V + 8 * (cb + nt) + 2 * c4) =
                            make_float2(hf[mt][nt][2 * half], hf[mt][nt][2 * half + 1]);
                    }
        }
    } else if (warp < 16) {
        // ============================================================= aux
        const int atid = tid - kRole, aw = warp - 8;
        const int ap = aw & 3, ah = aw >> 2;
        const uint32_t lane_base = (uint32_t)(ap * 32) << 16;
        const int ag = lane >> 2, ac = lane & 3;
        const int ar0 = ap * 16 + ag, ar1 = ar0 + 8;
        const float scl = prm.scale;
        bool ok = true;
        float pg = 0.f;
        auto fetch_gate = [&](int it) {
            if (atid < kChunk && it < nch) {
                const int ci = chunk_of(it);
                const int t0 = sr.start + ci * kChunk, len = min(kChunk, sr.len - ci * kChunk);
                pg = prm.gamma[(size_t)(t0 + min(atid, len - 1)) * d.Hv + h];
            }
        };
        auto store_gate = [&](int it) {
            if (atid < kChunk) {
                sm->gates[it % 3].gam[atid] = pg;
                sm->gates[it % 3].egam[atid] = __expf(pg);
            }
        };
        // P and dO' of iteration it into buffer it & 1 (its previous readers, Y and X of
        // iteration it - 2, have completed: this role saw mmaB of it - 2)
        auto make_p = [&](int it) -> bool {
            const int len = min(kChunk, sr.len - chunk_of(it) * kChunk);
            if (!rsync(2, wait_bar(&sm->mmaA[it & 1], (it >> 1) & 1, abort_flag) &&
                              wait_bar(&sm->full[it % kStages], (it / kStages) & 1, abort_flag)))
                return false;
            tc_fence_after();
            if (atid == 0) sm->loads_landed = it + 1;
            store_gate(it);
            fetch_gate(it + 1);
            rsync(2, true);  // gates of this chunk visible to the role
            const Gates &G = sm->gates[it % 3];
            {
                float v[16];
                tmem_ld16x256_x4(tmem + lane_base + (it & 1) * kABuf + kColS + 32 * ah, v);
                const float gr0 = G.gam[ar0], gr1 = G.gam[ar1];
                const bool l0 = ar0 < len, l1 = ar1 < len;
                const uint32_t pb = sb + kP + (it & 1) * 8192;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int s0 = 32 * ah + 8 * i + 2 * ac;
                    const float2 gs = *reinterpret_cast<const float2 *>(&G.gam[s0]);
                    const float x00 = (l0 && s0 <= ar0) ? scl * __expf(gr0 - gs.x) * v[4 * i] : 0.f;
                    const float x01 = (l0 && s0 + 1 <= ar0) ? scl * __expf(gr0 - gs.y) * v[4 * i + 1] : 0.f;
                    const float x10 = (l1 && s0 <= ar1) ? scl * __expf(gr1 - gs.x) * v[4 * i + 2] : 0.f;
                    const float x11 = (l1 && s0 + 1 <= ar1) ? scl * __expf(gr1 - gs.y) * v[4 * i + 3] : 0.f;
                    const int ch = 4 * ah + i;
                    st_shared_b32(pb + (ar0 >> 3) * 1024 + (ar0 & 7) * 128 + ((ch ^ (ar0 & 7)) << 4) + 4 * ac,
                                  pack_bf16(x00, x01));
                    st_shared_b32(pb + (ar1 >> 3) * 1024 + (ar1 & 7) * 128 + ((ch ^ (ar1 & 7)) << 4) + 4 * ac,
                                  pack_bf16(x10, x11));
                }
            }
            {  // dO' = scale e^gamma dO (zero past the sequence end): one 16-byte chunk per thread
                const int t = atid >> 2, c = atid & 3;
                const uint32_t src = sb + kStage0 + (it % kStages) * kStageBytes + kDO + t * 64 +
                                     ((c ^ ((t >> 1) & 3)) << 4);
                const uint4 raw = ld_shared_v4(src);
                const float f = t < len ? scl * G.egam[t] : 0.f;
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = unpack_bf16(w[e]);
                    o[e] = pack_bf16(f * x.x, f * x.y);
                }
                st_shared_v4(sb + kDO2 + (it & 1) * 4096 + c * 1024 + (t >> 3) * 128 + (t & 7) * 16, o[0], o[1], o[2],
                             o[3]);
            }
            fence_proxy_async();
            tc_fence_before();
            rsync(2, true);
            if (atid == 0) publish(&ctr[kPReady], it + 1);
            return true;
        };
        if (nch > 0) {
            fetch_gate(0);
            ok = make_p(0);
        }
        for (int it = 0; it < nch && ok; ++it) {
            const int len = min(kChunk, sr.len - chunk_of(it) * kChunk);
            const uint32_t abuf = (it & 1) * kABuf;
            // ---- -w, Y, X -> shared memory once the chain is done with the previous chunk's
            ok = rsync(2, wait_ge(&ctr[kWFree], it, abort_flag) &&
                              wait_bar(&sm->mmaB[it & 1], (it >> 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            {
                float v[32];
                tmem_ld16x256_x8(tmem + lane_base + abuf + kColW + ah * 64, v);  // columns 64 ah .. +63 of w
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int r = half ? ar1 : ar0;
                    const bool live = r < len;
                    const uint32_t rowb = sb + kWs + ah * 8192 + r * 128 + 4 * ac;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        st_shared_b32(rowb + ((i ^ (r & 7)) << 4),
                                      live ? pack_bf16(-v[4 * i + 2 * half], -v[4 * i + 2 * half + 1]) : 0u);
                }
                float y[8];
                tmem_ld16x256_x2(tmem + lane_base + abuf + kColY + 16 * ah, y);  // columns 16 ah .. +15 of Y
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int r = half ? ar1 : ar0;
                    const bool live = r < len;
#pragma unroll
                    for (int i = 0; i < 2; ++i)
                        st_shared_v2f(sb + kY + (r * 36 + 16 * ah + 8 * i + 2 * ac) * 4, live ? y[4 * i + 2 * half] : 0.f,
                                      live ? y[4 * i + 2 * half + 1] : 0.f);
                }
                float x[16];
                tmem_ld32x16(tmem + lane_base + abuf + kColX + 16 * ah, x);  // state row 32 ap + lane
                const uint32_t xb = sb + kX + ((ap * 32 + lane) * 36 + 16 * ah) * 4;
#pragma unroll
                for (int i = 0; i < 4; ++i) st_shared_v4f(xb + 16 * i, x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
            }
            tc_fence_before();
            rsync(2, true);
            if (atid == 0) {
                publish(&ctr[kReady], it + 1);
                publish(&ctr[kTmemA], it + 1);
            }
            if (it + 1 < nch) ok = make_p(it + 1);
        }
        if (!ok) {
            if (atid == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        }
    } else if (warp == 16) {
        // ================================================== MMA issuer A
        if (lane == 0) {
            bool ok = true;
            for (int c = 0; c < kStages && c < nch; ++c) issue_loads(c);
            const uint32_t id_S = idesc_bf16(64, 64, false, false);
            const uint32_t id_W = idesc_bf16(64, 128, false, true);
            for (int it = 0; it < nch && ok; ++it) {
                const uint32_t st = sb + kStage0 + (it % kStages) * kStageBytes;
                ok = wait_bar(&sm->full[it % kStages], (it / kStages) & 1, abort_flag) &&
                     wait_ge(&ctr[kTmemA], it >= 1 ? it - 1 : 0, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t tb = tmem + (it & 1) * kABuf;
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tb + kColW, smem_desc(st + kAw + ks * 32, 16, 1024, kSw128),
                             smem_desc(st + kK + ks * 2048, 8192, 1024, kSw128), id_W, ks > 0);
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_bf16(tb + kColS, smem_desc(st + kQ + off, 16, 1024, kSw128),
                             smem_desc(st + kK + off, 16, 1024, kSw128), id_S, ks > 0);
                }
                mma_commit(&sm->mmaA[it & 1]);
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
            const uint32_t id_Y = idesc_bf16(64, 32, true, true);
            const uint32_t id_X = idesc_bf16(128, 32, true, true);
            for (int it = 0; it < nch && ok; ++it) {
                const uint32_t st = sb + kStage0 + (it % kStages) * kStageBytes;
                ok = wait_ge(&ctr[kPReady], it + 1, abort_flag) &&
                     wait_ge(&ctr[kTmemA], it >= 1 ? it - 1 : 0, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t tb = tmem + (it & 1) * kABuf;
                const uint32_t pb = sb + kP + (it & 1) * 8192, ob = sb + kDO2 + (it & 1) * 4096;
                for (int ks = 0; ks < 4; ++ks) {
                    // Y = P^T dO: A = P read transposed (MN-major), B = the dO tile; K = 16 rows of P per step
                    mma_bf16(tb + kColY, smem_desc(pb + ks * 2048, 8192, 1024, kSw128),
                             smem_desc(st + kDO + ks * 1024, 4096, 512, kSw64), id_Y, ks > 0);
                    // X = Q^T dO': A = the q tile read transposed (MN-major, two 64-row halves)
                    mma_bf16(tb + kColX, smem_desc(st + kQ + ks * 2048, 8192, 1024, kSw128),
                             smem_desc(ob + ks * 256, 128, 1024, kSwNone), id_X, ks > 0);
                }
                mma_commit(&sm->mmaB[it & 1]);
                // refill the stage of iteration it - 1 with iteration it + 2 once the chain is done
                // with its k tile and the aux role has seen this stage's products of it - 1 complete
                if (it >= 1 && it + 2 < nch) {
                    ok = wait_ge(&ctr[kStage], it, abort_flag) && wait_ge(&ctr[kTmemA], it, abort_flag);
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
        // let every TMA load still in flight land (bounded) before the CTA exits
        const uint64_t t0 = globaltimer();
        for (int c = sm->loads_landed; c < sm->loads_issued; ++c)
            while (!mbar_try_wait(smem_u32(&sm->full[c % kStages]), (c / kStages) & 1) &&
                   globaltimer() - t0 < kWaitNs) {
            }
    }
    __syncthreads();
    if (warp == 16) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool tc_bwd_supported(const Dims &d, int dtype) {
    return dtype == GDN_DTYPE_BF16 && d.K == 128 && d.V == 128;
}

cudaError_t launch_bwd_dh_tc(const BwdArgs &a, const void *wy, void *dh_chunks16, void *ddelta16) {
    const Dims &d = a.d;
    if (d.N == 0) return cudaSuccess;
    CUtensorMap mq, mk, mdo, mw;
    const cuuint64_t dq[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hq, (cuuint64_t)(d.T_total > 0 ? d.T_total : 1)};
    const cuuint64_t sq[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hq * d.K * 2};
    const cuuint32_t bq[3] = {64, 1, 64};
    const cuuint64_t dv[3] = {(cuuint64_t)d.V, (cuuint64_t)d.Hv, (cuuint64_t)(d.T_total > 0 ? d.T_total : 1)};
    const cuuint64_t sv[2] = {(cuuint64_t)d.V * 2, (cuuint64_t)d.Hv * d.V * 2};
    const cuuint32_t bv[3] = {kBV, 1, 64};
    const cuuint64_t dw[2] = {64, (cuuint64_t)(d.NC > 0 ? d.NC : 1) * d.Hv * 2 * 64};
    const cuuint64_t sw[1] = {128};
    const cuuint32_t bw[2] = {64, 64};
    if (!make_bf16_map(&mq, a.q, 3, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map(&mk, a.k, 3, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map(&mdo, a.d_o, 3, dv, sv, bv, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_bf16_map(&mw, wy, 2, dw, sw, bw, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    BwdDhParams p;
    p.d = d;
    p.gamma = a.gamma;
    p.dht = a.dht;
    p.dh_chunks = (__nv_bfloat16 *)dh_chunks16;
    p.ddelta = (__nv_bfloat16 *)ddelta16;
    p.dh0 = a.dh0;
    p.scale = d.scale;
    p.status = a.status;
    cudaError_t e = cudaFuncSetAttribute(bwd_dh_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    bwd_dh_kernel<<<dim3(d.N, d.Hv, d.V / kBV), kThreads, kSmemBytes, a.stream>>>(mq, mk, mdo, mw, p);
    return cudaGetLastError();
}

}  // namespace gdn
