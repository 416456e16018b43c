// gdn_prep3.cu -- chunk prep for the bf16, K = V = 128 tensor-core path: every
// per-chunk quantity that does not depend on the state, so that the state
// chains downstream only run their two state-dependent products.
//
// Persistent CTAs (8 warps, two per SM) walk the (64-token chunk, qk head) items;
// an item serves the value heads of the qk head's group. From k, q (per qk head)
// and v, g, beta (per value head):
//
//   G     = K K^T,   S = Q K^T                                  (once per qk head)
//   gamma = in-chunk cumulative sum of g
//   A_rs  = beta_r e^{gamma_r - gamma_s} G_rs  (s < r),   Ainv = (I + A)^-1
//   w     = Ainv diag(beta e^gamma) K         -> bf16 [T, Hv, K]
//   u     = Ainv diag(beta) V                 -> fp32 [T, Hv, V]
//   P     = M o S,  M_rs = e^{gamma_r - gamma_s} on s <= r     -> bf16 [NC, Hv, 64, 64]
//   Ainv  (bf16 [NC, Hv, 64, 64], for the backward; optional)
//
// (the WY form of the chunk: Delta = u - w h, o = scale (diag(e^gamma) Q h + P Delta).)
// The q and k tiles are double-buffered: the next item's load is issued as soon
// as this item's S and G are formed, so that a whole item's work hides its
// latency (a load issued at the start of its own item stalled the CTA for about
// 4 us). P and w of a full chunk are written by TMA stores from swizzled staging
// tiles (row by row for a ragged one, whose tile would spill into the next
// sequence); u goes out straight from the accumulator registers, four lanes per
// 32-byte sector. The four bulk products (S, G, u, w) run on tcgen05 from
// TMA-loaded, 128-byte-swizzled tiles. The unit lower-triangular inverse is
// taken block-wise in fp32, in one work matrix that holds the inverse on and below
// the diagonal and A transposed above it: 16 x 16 diagonal blocks by forward
// substitution, then two doubling steps on tf32 MMAs (16 -> 32 -> 64), each
// X_BA = -X_BB A_BA X_AA for the two halves A, B of a block, so that the critical
// path holds four dependent products and two CTA barriers. Rows past the end of a
// sequence have beta = 0, and a ragged chunk's rows past its end are zeroed in the
// q, k and v tiles before any product, so that whatever the TMA reads there (the
// next sequence, or zeros) never reaches an output.
#include <algorithm>
#include <cstddef>

#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kThreads = 256;
constexpr int C = 64, K = 128, V = 128;
constexpr int kLd = 68;  // row pitch (floats) of the fp32 work matrices

// ---- shared memory (bytes from a 1024-aligned base)
// q and k tiles are double-buffered by item, so that the next item's tiles load while
// this one is worked on; the item's q slot takes its value heads' v tiles once S is done.
constexpr int kQ0 = 0;          // 2 x q tile (then v tiles): [64][128] bf16, 128-byte swizzle, two halves
constexpr int kK0 = 32768;      // 2 x k tile, same layout
constexpr int kAu = 65536;      // Ainv diag(beta): [64][64] bf16, 128-byte swizzle (K-major A operand)
constexpr int kAw = 73728;      // Ainv diag(beta e^gamma)
constexpr int kAX = 81920;      // float [64][kLd]: X = Ainv on and below the diagonal, A^T above it
constexpr int kT = kAX + 64 * kLd * 4;     // float [3][16][17]: one 16 x 16 block product per warp
constexpr int kVec = kT + 3 * 16 * 17 * 4;
constexpr int kBar = kVec + 1024;
constexpr int kPs = 104448;     // P staging for its TMA store: [64][64] bf16, 128-byte swizzle
constexpr int kSmemBytes = kPs + 8192 + 1024;
static_assert(kBar + 64 <= kPs && kPs % 1024 == 0, "shared memory layout");
// w of a full chunk leaves through TMA stores from a 128-byte-swizzled staging tile
// (two [64][64] halves) over Au, Aw, free once the u, w products are complete; u
// (fp32) is stored straight from the accumulator registers.
constexpr int kWs = kAu;
static_assert(kSmemBytes <= 113 * 1024, "two CTAs per SM");

// tensor memory: S | G (64 columns each), later u | w (128 columns each)
constexpr uint32_t kColS = 0, kColG = 64, kColU = 0, kColW = 128, kTmemCols = 256;

__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Bounded wait on an mbarrier phase by every thread of the CTA. The result is
// the same in every thread (a barrier ANDs it), so that the CTA's control flow,
// and with it every later __syncthreads, stays uniform even when a wait expires.
__device__ __forceinline__ bool cta_wait(uint64_t *bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const uint64_t t0 = globaltimer();
    bool ok = true;
    while (!mbar_try_wait(a, parity))
        if (globaltimer() - t0 > kWaitNs) {
            ok = false;
            break;
        }
    return __syncthreads_and(ok ? 1 : 0) != 0;
}

// Zeroes rows [len, 64) of a [64][128] bf16 tile stored as two 64-column halves of
// 128-byte rows (the swizzle permutes 16-byte chunks within a row, so whole rows
// are zeroed regardless of it).
__device__ __forceinline__ void zero_rows(uint32_t tile, int len, int tid) {
    for (int i = tid; i < (C - len) * 16; i += kThreads) {
        const int r = len + (i >> 4), c = i & 15;
        st_shared_v4(tile + (c >> 3) * 8192 + r * 128 + (c & 7) * 16, 0u, 0u, 0u, 0u);
    }
}

struct Prep3Params {
    Dims d;
    const float *g, *beta;
    float *gamma_out;
    __nv_bfloat16 *ainv_out;  // nullable
    __nv_bfloat16 *w_out;
    float *u_out;
    __nv_bfloat16 *p_out;
    unsigned *status;
};

__global__ void __launch_bounds__(kThreads, 2)
prep3_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_wo,
             const __grid_constant__ CUtensorMap tm_po,
             const Prep3Params prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    const uint32_t sb = smem_u32(smem);
    const Dims &d = prm.d;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wm = warp & 3, wn = warp >> 2, g8 = lane >> 2, c4 = lane & 3;
    const int r0 = 16 * wm + g8, r1 = r0 + 8;
    const int G = d.Hv / d.Hq;

    // one fp32 work matrix: X (the inverse) on and below the diagonal, A transposed above it
    float(*AX)[kLd] = reinterpret_cast<float(*)[kLd]>(smem + kAX);
    float(*T)[16][17] = reinterpret_cast<float(*)[16][17]>(smem + kT);
    float *gam = reinterpret_cast<float *>(smem + kVec);
    float *egam = gam + 64, *bet = gam + 128, *scan = gam + 192;
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + kBar);
    uint64_t *mma_bar = tma_bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_bar + 2);
    uint64_t *qk_bar = tma_bar + 3;  // [2]: the q, k tiles of each buffer

    if (tid == 0) {
        mbar_init(tma_bar, 1);
        mbar_init(mma_bar, 1);
        mbar_init(&qk_bar[0], 1);
        mbar_init(&qk_bar[1], 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = (uint32_t)(wm * 32) << 16;  // TMEM lanes of this warp's rows (M = 64 layout)
    uint32_t tma_phase = 0, mma_phase = 0;  // phases consumed so far
    bool tma_pending = false;  // (every thread) a v tile load issued and not yet consumed
    bool mma_pending = false;  // (thread 0) products issued and not yet consumed
    bool ok = true;
    const int n_items = d.NC * d.Hq;
    // Persistent: items (chunk, qk head) in steps of the grid; the tiles of the item after
    // this CTA's next one are prefetched into L2 while it works on the current one. Copies
    // and prefetches are issued by warps that idle during the inverse (a copy's setup holds
    // its thread for hundreds of cycles, and with it the CTA at the next barrier).
    auto prefetch_item = [&](int item) {  // by one thread
        if (item >= n_items) return;
        const int cg2 = item / d.Hq, hq2 = item % d.Hq;
        const int n2 = chunk_owner(d, cg2);
        if (n2 < 0) return;
        const SeqRange s2 = seq_range(d, n2);
        const int t2 = s2.start + (cg2 - s2.chunk0) * C;
        tma_prefetch_3d(&tm_q, 0, hq2, t2);
        tma_prefetch_3d(&tm_q, 64, hq2, t2);
        tma_prefetch_3d(&tm_k, 0, hq2, t2);
        tma_prefetch_3d(&tm_k, 64, hq2, t2);
        for (int gi = 0; gi < G; ++gi) {
            tma_prefetch_3d(&tm_v, 0, hq2 * G + gi, t2);
            tma_prefetch_3d(&tm_v, 64, hq2 * G + gi, t2);
        }
    };
    // q, k tiles of the CTA's k-th item go to buffer k % 2 (a consistent sequence table
    // has an owner for every chunk, an inconsistent one for none, so items are either
    // all valid or all skipped and the buffer alternation holds)
    int qk_issued = 0;  // (every thread) q, k loads issued
    auto issue_qk = [&](int item, int issuer) {  // by every thread; thread `issuer` copies
        if (item >= n_items) return;
        const int cg2 = item / d.Hq, hq2 = item % d.Hq;
        const int n2 = chunk_owner(d, cg2);
        if (n2 < 0) return;
        const SeqRange s2 = seq_range(d, n2);
        const int t2 = s2.start + (cg2 - s2.chunk0) * C;
        const int b = qk_issued & 1;
        if (tid == issuer) {
            mbar_arrive_expect_tx(&qk_bar[b], 4 * 8192);
            tma_load_3d(smem + kQ0 + b * 16384, &tm_q, &qk_bar[b], 0, hq2, t2);
            tma_load_3d(smem + kQ0 + b * 16384 + 8192, &tm_q, &qk_bar[b], 64, hq2, t2);
            tma_load_3d(smem + kK0 + b * 16384, &tm_k, &qk_bar[b], 0, hq2, t2);
            tma_load_3d(smem + kK0 + b * 16384 + 8192, &tm_k, &qk_bar[b], 64, hq2, t2);
        }
        ++qk_issued;
    };
    issue_qk(blockIdx.x, 0);
    int it_k = 0;  // this CTA's item count
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++it_k) {
    const int cg = item / d.Hq, hq = item % d.Hq;
    const int n = chunk_owner(d, cg);
    if (n < 0) continue;  // the whole CTA
    const SeqRange sr = seq_range(d, n);
    const int ci = cg - sr.chunk0;
    const int t0 = sr.start + ci * C, len = min(C, sr.len - ci * C);
    const int buf = it_k & 1;
    const uint32_t qv = sb + kQ0 + buf * 16384, kt = sb + kK0 + buf * 16384;  // q (then v), k tiles

    // ---- q, k tiles (loaded during the previous item); S = Q K^T and G = K K^T on tcgen05
    float g_next = 0.f, b_next = 0.f;  // g, beta of the next value head, prefetched
    if (tid < C && tid < len) {
        g_next = prm.g[(size_t)(t0 + tid) * d.Hv + hq * G];
        b_next = prm.beta[(size_t)(t0 + tid) * d.Hv + hq * G];
    }
    ok = cta_wait(&qk_bar[buf], (it_k >> 1) & 1);
    if (len < C) {
        // a ragged chunk: rows past its end hold the next packed sequence (or zeros); zero them so that
        // a non-finite value there cannot reach this sequence through a product with a zero weight
        zero_rows(qv, len, tid);
        zero_rows(kt, len, tid);
        fence_proxy_async();
        __syncthreads();
    }
    if (ok && tid == 0) {
        tc_fence_after();
        const uint32_t id_S = idesc_bf16(64, 64, false, false);
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
            mma_bf16(tmem + kColS, smem_desc(qv + off, 16, 1024, kSw128), smem_desc(kt + off, 16, 1024, kSw128), id_S,
                     ks > 0);
            mma_bf16(tmem + kColG, smem_desc(kt + off, 16, 1024, kSw128), smem_desc(kt + off, 16, 1024, kSw128), id_S,
                     ks > 0);
        }
        mma_commit(mma_bar);
        mma_pending = true;
    }
    ok = ok && cta_wait(mma_bar, mma_phase & 1);
    if (ok) ++mma_phase, mma_pending = false;
    tc_fence_after();
    // S, G: rows r0, r1, columns 32 wn + 8 j + 2 c4 (+1) -- the warp MMA fragment layout
    float sacc[4][4], gacc[4][4];
    {
        float v[16];
        tmem_ld16x256_x4(tmem + lane_base + kColS + 32 * wn, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) sacc[i >> 2][i & 3] = v[i];
        tmem_ld16x256_x4(tmem + lane_base + kColG + 32 * wn, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) gacc[i >> 2][i & 3] = v[i];
    }
    tc_fence_before();
    __syncthreads();  // q tile and S, G columns free
    // v tiles go into the q slot. The first value head's is issued by the last warp, which
    // idles during the inverse: issued by thread 0 here, it held the whole CTA at the next
    // barrier and cost 4 % of the kernel.
    auto load_v = [&](int h) {  // by one thread
        mbar_arrive_expect_tx(tma_bar, 2 * 8192);
        tma_load_3d(smem + (qv - sb), &tm_v, tma_bar, 0, h, t0);
        tma_load_3d(smem + (qv - sb) + 8192, &tm_v, tma_bar, 64, h, t0);
    };

    for (int gi = 0; gi < G && ok; ++gi) {
        const int h = hq * G + gi;
        // ---- gamma: two warps scan 32 rows each, then combine
        if (tid < C) {
            float x = g_next;
            const float bt = b_next;
            if (gi + 1 < G && tid < len) {
                g_next = prm.g[(size_t)(t0 + tid) * d.Hv + h + 1];
                b_next = prm.beta[(size_t)(t0 + tid) * d.Hv + h + 1];
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            scan[tid] = x;
            bet[tid] = bt;
        }
        __syncthreads();
        if (tid < C) {
            const float x = tid >= 32 ? scan[tid] + scan[31] : scan[tid];
            const float gl = tid < len ? x : (len > 32 ? scan[len - 1] + scan[31] : scan[len - 1]);
            gam[tid] = gl;  // rows past the end repeat the last live value
            egam[tid] = __expf(gl);
            if (tid < len) prm.gamma_out[(size_t)(t0 + tid) * d.Hv + h] = gl;
        }
        if (tid == 0) bulk_wait_read<0>();  // the previous head's P, u, w stores have read their staging
        __syncthreads();
        // ---- A (strictly lower), X = 0, and P = M o S -> global
        {
            const float gr[2] = {gam[r0], gam[r1]}, br[2] = {bet[r0], bet[r1]};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int s = 32 * wn + 8 * j + 2 * c4;
                const float gs0 = gam[s], gs1 = gam[s + 1];
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = hi ? r1 : r0;
                    const float e0 = s <= r ? __expf(gr[hi] - gs0) : 0.f;
                    const float e1 = s + 1 <= r ? __expf(gr[hi] - gs1) : 0.f;
                    // A_rs (s < r) goes transposed above the diagonal; X fills the rest later
                    if (s < r) AX[s][r] = br[hi] * e0 * gacc[j][2 * hi];
                    if (s + 1 < r) AX[s + 1][r] = br[hi] * e1 * gacc[j][2 * hi + 1];
                    const bool live = r < len;
                    st_shared_b32(sb + kPs + r * 128 + (((s >> 3) ^ (r & 7)) << 4) + (s & 7) * 2,
                                  pack_bf16(live ? e0 * sacc[j][2 * hi] : 0.f, live ? e1 * sacc[j][2 * hi + 1] : 0.f));
                }
            }
        }
        fence_proxy_async();  // P -> its TMA store
        __syncthreads();
        if (tid == 0) {
            tma_store_2d(&tm_po, sb + kPs, 0, (cg * d.Hv + h) * C);
            bulk_commit();
        }
        // ---- the inverse X = (I + A)^-1, unit lower triangular, in two steps of doubling:
        //  (1) warps 0, 1: the diagonal 16 x 16 blocks of their 32 x 32 block by forward
        //      substitution (lane -> block lane / 16, column lane % 16), then that block's
        //      off-diagonal 16 x 16 block X_10 = -X_11 (A_10 X_00) on tf32 MMAs;
        //  (2) warps 0..3, one 8-column strip each: X_BA = -X_BB (A_BA X_AA) on the 32 x 32
        //      blocks (A = rows and columns 0..31, B = 32..63).
        //  Warps 4..7 take no part; during the item's first value head, three of them issue
        //  the copies of the next tiles meanwhile.
        if (gi == 0 && ok) {
            if (tid == kThreads - 32) load_v(hq * G);
            tma_pending = true;
            // the other q, k buffer was last read by the previous item's products, all
            // complete: the next item's tiles go there now
            issue_qk(item + gridDim.x, kThreads - 64);
            if (tid == kThreads - 96) prefetch_item(item + 2 * gridDim.x);
        }
        if (warp < 2) {
            {
                const int o = 32 * warp + 16 * (lane >> 4), cc = lane & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) x[r] = r == cc ? 1.f : 0.f;
                // right-looking: once x_j is final, rows r > j take -A_rj x_j; row j of A^T
                // (A_rj for r > j) lies contiguous at AX[o + j][o + r]
#pragma unroll
                for (int j = 0; j < 15; ++j) {
#pragma unroll
                    for (int q = (j + 1) >> 2; q < 4; ++q) {
                        const float4 a = *reinterpret_cast<const float4 *>(&AX[o + j][o + 4 * q]);
                        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (4 * q + e > j) x[4 * q + e] = fmaf(-av[e], x[j], x[4 * q + e]);
                    }
                }
                // only on and below the diagonal: above it lies A
#pragma unroll
                for (int r = 0; r < 16; ++r)
                    if (r >= cc) AX[o + r][o + cc] = x[r];
            }
            __syncwarp();
            // X_10 = -X_11 (A_10 X_00) for this warp's 32 x 32 block: rows i0 .., columns j0 ..
            const int j0 = 32 * warp, i0 = j0 + 16;
            float t[2][4] = {};
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int ac = j0 + kk * 8 + c4;
                // A_{i0 + row, ac} (below the diagonal) is stored transposed
                const uint32_t a[4] = {tf32(AX[ac][i0 + g8]), tf32(AX[ac][i0 + g8 + 8]), tf32(AX[ac + 4][i0 + g8]),
                                       tf32(AX[ac + 4][i0 + g8 + 8])};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int bc = j0 + nt * 8 + g8;
                    // X_00: zero above the diagonal (A lies there)
                    const float x0 = bc > ac ? 0.f : AX[ac][bc];
                    const float x1 = bc > ac + 4 ? 0.f : AX[ac + 4][bc];
                    mma_tf32(t[nt], a, tf32(x0), tf32(x1));
                }
            }
            float(*Tw)[17] = T[warp];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int col = nt * 8 + 2 * c4;
                Tw[g8][col] = t[nt][0];
                Tw[g8][col + 1] = t[nt][1];
                Tw[g8 + 8][col] = t[nt][2];
                Tw[g8 + 8][col + 1] = t[nt][3];
            }
            __syncwarp();
            float x[2][4] = {};
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int ac = i0 + kk * 8 + c4;
                const int ra = i0 + g8, rb = ra + 8;
                const uint32_t a[4] = {tf32(ac > ra ? 0.f : AX[ra][ac]), tf32(ac > rb ? 0.f : AX[rb][ac]),
                                       tf32(ac + 4 > ra ? 0.f : AX[ra][ac + 4]), tf32(ac + 4 > rb ? 0.f : AX[rb][ac + 4])};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int bc = nt * 8 + g8;
                    mma_tf32(x[nt], a, tf32(Tw[kk * 8 + c4][bc]), tf32(Tw[kk * 8 + c4 + 4][bc]));
                }
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int col = j0 + nt * 8 + 2 * c4;
                AX[i0 + g8][col] = -x[nt][0];
                AX[i0 + g8][col + 1] = -x[nt][1];
                AX[i0 + g8 + 8][col] = -x[nt][2];
                AX[i0 + g8 + 8][col + 1] = -x[nt][3];
            }
        }
        if (warp < 4) {
            named_sync<128>(1);  // warps 0..3 only: the others go on to the next CTA barrier
            // columns 8 ct .. 8 ct + 7 of X_BA; T = A_BA X_AA is staged where X_BA goes
            // (rows 32.., columns 0..31 of the work matrix, free until now), then overwritten
            const int ct = warp, cb = 8 * ct;
            float t[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                if (ks < ct) continue;  // X_AA is zero above the diagonal
                const int ac = 8 * ks + c4;
                const float x0 = cb + g8 > ac ? 0.f : AX[ac][cb + g8];
                const float x1 = cb + g8 > ac + 4 ? 0.f : AX[ac + 4][cb + g8];
#pragma unroll
                for (int rt = 0; rt < 2; ++rt) {
                    const int rr = 32 + 16 * rt + g8;
                    const uint32_t a[4] = {tf32(AX[ac][rr]), tf32(AX[ac][rr + 8]), tf32(AX[ac + 4][rr]),
                                           tf32(AX[ac + 4][rr + 8])};
                    mma_tf32(t[rt], a, tf32(x0), tf32(x1));
                }
            }
#pragma unroll
            for (int rt = 0; rt < 2; ++rt) {
                const int rr = 32 + 16 * rt + g8;
                AX[rr][cb + 2 * c4] = t[rt][0];
                AX[rr][cb + 2 * c4 + 1] = t[rt][1];
                AX[rr + 8][cb + 2 * c4] = t[rt][2];
                AX[rr + 8][cb + 2 * c4 + 1] = t[rt][3];
            }
            __syncwarp();
            // every row of this strip of T is read before any of it is overwritten
            uint32_t tb[4][2];
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                tb[ks][0] = tf32(AX[32 + 8 * ks + c4][cb + g8]);
                tb[ks][1] = tf32(AX[32 + 8 * ks + c4 + 4][cb + g8]);
            }
            __syncwarp();
            float x[2][4] = {};
#pragma unroll
            for (int rt = 0; rt < 2; ++rt) {
                const int ra = 16 * rt + g8, rb = ra + 8;  // rows of X_BB (offset 32)
#pragma unroll
                for (int ks = 0; ks < 2 + 2 * rt; ++ks) {
                    const int ac = 8 * ks + c4;  // columns of X_BB (offset 32): zero above the diagonal
                    const uint32_t a[4] = {tf32(ac > ra ? 0.f : AX[32 + ra][32 + ac]),
                                           tf32(ac > rb ? 0.f : AX[32 + rb][32 + ac]),
                                           tf32(ac + 4 > ra ? 0.f : AX[32 + ra][32 + ac + 4]),
                                           tf32(ac + 4 > rb ? 0.f : AX[32 + rb][32 + ac + 4])};
                    mma_tf32(x[rt], a, tb[ks][0], tb[ks][1]);
                }
            }
#pragma unroll
            for (int rt = 0; rt < 2; ++rt) {
                const int rr = 32 + 16 * rt + g8;
                AX[rr][cb + 2 * c4] = -x[rt][0];
                AX[rr][cb + 2 * c4 + 1] = -x[rt][1];
                AX[rr + 8][cb + 2 * c4] = -x[rt][2];
                AX[rr + 8][cb + 2 * c4 + 1] = -x[rt][3];
            }
        }
        __syncthreads();
        // ---- Ainv diag(beta), Ainv diag(beta e^gamma) -> 128-byte-swizzled bf16 tiles
        //      (the K-major A operands of the u and w products); Ainv -> global (optional)
        for (int e = tid; e < C * C / 2; e += kThreads) {
            const int r = e >> 5, s = (e & 31) * 2;
            const float x0 = s <= r ? AX[r][s] : 0.f, x1 = s + 1 <= r ? AX[r][s + 1] : 0.f;
            const float u0 = x0 * bet[s], u1 = x1 * bet[s + 1];
            const uint32_t off = (r >> 3) * 1024 + (r & 7) * 128 + ((((s >> 3) ^ (r & 7))) << 4) + (s & 7) * 2;
            st_shared_b32(sb + kAu + off, pack_bf16(u0, u1));
            st_shared_b32(sb + kAw + off, pack_bf16(u0 * egam[s], u1 * egam[s + 1]));
            if (prm.ainv_out)
                *reinterpret_cast<uint32_t *>(prm.ainv_out + ((size_t)cg * d.Hv + h) * C * C + r * C + s) =
                    pack_bf16(x0, x1);
        }
        fence_proxy_async();
        __syncthreads();
        // ---- u = Au V, w = Aw K on tcgen05 once this head's v tile has landed
        ok = cta_wait(tma_bar, tma_phase & 1);
        if (ok) ++tma_phase, tma_pending = false;
        if (len < C) {
            zero_rows(qv, len, tid);  // the v tile's rows past the end, as for q and k
            fence_proxy_async();
            __syncthreads();
        }
        if (ok && tid == 0) {
            tc_fence_after();
            const uint32_t id_W = idesc_bf16(64, 128, false, true);
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(tmem + kColU, smem_desc(sb + kAu + ks * 32, 16, 1024, kSw128),
                         smem_desc(qv + ks * 2048, 8192, 1024, kSw128), id_W, ks > 0);
                mma_bf16(tmem + kColW, smem_desc(sb + kAw + ks * 32, 16, 1024, kSw128),
                         smem_desc(kt + ks * 2048, 8192, 1024, kSw128), id_W, ks > 0);
            }
            mma_commit(mma_bar);
            mma_pending = true;
        }
        ok = ok && cta_wait(mma_bar, mma_phase & 1);
        if (ok) ++mma_phase, mma_pending = false;
        tc_fence_after();
        if (ok && gi + 1 < G) {  // the v tile is free again
            if (tid == 0) load_v(h + 1);
            tma_pending = true;
        }
        const bool full = len == C;
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // columns 64 wn + 32 part .. +31, 16 values at a time
            float v[16];
            const int cb = 64 * wn + 32 * part;
            tmem_ld16x256_x4(tmem + lane_base + kColU + cb, v);  // u
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int col = cb + 8 * i + 2 * c4;
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = hi ? r1 : r0;
                    // u straight to global memory (four lanes write one full 32-byte sector)
                    if (r < len)
                        *reinterpret_cast<float2 *>(prm.u_out + ((size_t)(t0 + r) * d.Hv + h) * V + col) =
                            make_float2(v[4 * i + 2 * hi], v[4 * i + 2 * hi + 1]);
                }
            }
            tmem_ld16x256_x4(tmem + lane_base + kColW + cb, v);  // w
            // wx[i][hi]: the 8 x 8 block (rows 16 wm + 8 hi .., columns cb + 8 i ..) in the m16n8
            // accumulator layout (this lane: row g8, columns 2 c4, 2 c4 + 1)
            uint32_t wx[4][2];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) wx[i][hi] = pack_bf16(v[4 * i + 2 * hi], v[4 * i + 2 * hi + 1]);
            if (full) {
                // two stmatrix.x4 into the 128-byte-swizzled staging tile (conflict-free: the 8 rows
                // of a block land in 8 distinct 16-byte chunks)
                const int li = lane & 7, mi = lane >> 3;
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    const int col = cb + 8 * (2 * a + (mi >> 1)), r = 16 * wm + 8 * (mi & 1) + li;
                    const uint32_t regs[4] = {wx[2 * a][0], wx[2 * a][1], wx[2 * a + 1][0], wx[2 * a + 1][1]};
                    stsm_x4(sb + kWs + (col >> 6) * 8192 + r * 128 + ((((col & 63) >> 3) ^ (r & 7)) << 4), regs);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi) {
                        const int r = hi ? r1 : r0;
                        if (r < len)
                            *reinterpret_cast<uint32_t *>(prm.w_out + ((size_t)(t0 + r) * d.Hv + h) * K + cb + 8 * i + 2 * c4) =
                                wx[i][hi];
                    }
            }
        }
        fence_proxy_async();  // w -> its TMA stores
        tc_fence_before();
        __syncthreads();  // u, w columns free for the next value head (Au, Aw once the stores have read them)
        if (full && tid == 0) {
            tma_store_3d(&tm_wo, sb + kWs, 0, h, t0);
            tma_store_3d(&tm_wo, sb + kWs + 8192, 64, h, t0);
            bulk_commit();
        }
    }
    __syncthreads();  // every thread is done with this item's shared memory before the next one's loads
    }  // item loop
    if (!ok) {
        if (tid == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
        // a TMA load or MMA that has not completed may still be in flight: wait (bounded) for it
        if (tid == 0) {
            const uint64_t t1 = globaltimer();
            while (tma_pending && !mbar_try_wait(smem_u32(tma_bar), tma_phase & 1) && globaltimer() - t1 < kWaitNs) {
            }
            // the last q, k load issued (each buffer has at most one outstanding)
            if (qk_issued > 0) {
                const int b = (qk_issued - 1) & 1;
                while (!mbar_try_wait(smem_u32(&qk_bar[b]), ((qk_issued - 1) >> 1) & 1) && globaltimer() - t1 < kWaitNs) {
                }
            }
            while (mma_pending && !mbar_try_wait(smem_u32(mma_bar), mma_phase & 1) && globaltimer() - t1 < kWaitNs) {
            }
        }
    }
    if (tid == 0) bulk_wait_all();  // the stores read shared memory until they complete
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool prep3_supported(const FwdArgs &a) { return a.dtype == GDN_DTYPE_BF16 && a.d.K == 128 && a.d.V == 128; }

cudaError_t launch_prep3(const FwdArgs &a) {
    const Dims &d = a.d;
    if (d.NC == 0) return cudaSuccess;
    if (!a.w16 || !a.u32 || !a.p16 || !a.gamma) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mwo, mpo;
    const cuuint64_t T = (cuuint64_t)(d.T_total > 0 ? d.T_total : 1);
    const cuuint64_t dq[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hq, T};
    const cuuint64_t sq[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hq * d.K * 2};
    const cuuint64_t dv[3] = {(cuuint64_t)d.V, (cuuint64_t)d.Hv, T};
    const cuuint64_t sv[2] = {(cuuint64_t)d.V * 2, (cuuint64_t)d.Hv * d.V * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    // stores: w bf16 [T, Hv, K], P bf16 [NC * Hv * 64 rows][64] (u is stored from registers)
    const cuuint64_t dw[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hv, T};
    const cuuint64_t sw[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hv * d.K * 2};
    const cuuint64_t dp[2] = {64, (cuuint64_t)d.NC * d.Hv * 64};
    const cuuint64_t sp[1] = {128};
    const cuuint32_t bp[2] = {64, 64};
    auto enc = tensor_map_encoder();
    if (!enc || !make_bf16_map(&mq, a.q, 3, dq, sq, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map(&mk, a.k, 3, dq, sq, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map(&mv, a.v, 3, dv, sv, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map(&mwo, a.w16, 3, dw, sw, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_bf16_map(&mpo, a.p16, 2, dp, sp, bp, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    Prep3Params p;
    p.d = d;
    p.g = a.g;
    p.beta = a.beta;
    p.gamma_out = a.gamma;
    p.ainv_out = (__nv_bfloat16 *)a.ainv;
    p.w_out = (__nv_bfloat16 *)a.w16;
    p.u_out = a.u32;
    p.p_out = (__nv_bfloat16 *)a.p16;
    p.status = a.status;
    cudaError_t e = cudaFuncSetAttribute(prep3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) sms = v;
    }
    const long long items = (long long)d.NC * d.Hq;
    if (items >= (1ll << 31)) return cudaErrorInvalidValue;
    const int grid = (int)std::min<long long>(items, 2ll * sms);  // persistent, two CTAs per SM
    prep3_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mk, mv, mwo, mpo, p);
    return cudaGetLastError();
}

}  // namespace gdn
