// gdn_bwd_grad.cu -- per-chunk gradients of the chunked backward (bf16,
// K = V = 128). Fully parallel: one CTA per (chunk, value head).
//
// Per chunk (rows r, s; h the entry state, Delta, from the forward; dh' and
// dDelta from the reverse scan; Kb = diag(beta e^gamma) K, E_rs = e^{gamma_r - gamma_s},
// M = E on s <= r, A_rs = beta_r E_rs k_r.k_s on s < r):
//
//   dU   = Ainv^T dDelta                 dv = diag(beta) dU
//   P1   = dO Delta^T                    T1 = scale M o P1
//   dAkk = -dU Delta^T  (s < r)          dG = dAkk o beta_r E
//   dq   = scale diag(e^gamma) dO h^T + T1 K
//   dk   = T1^T Q + dG K + dG^T K - diag(beta e^gamma) dU h^T + diag(e^{gamma_C - gamma}) Delta dh'^T
//   dbeta_r  = dU_r.v_r + e^{gamma_r} dKb_r.k_r + sum_s dAkk_rs E_rs k_r.k_s,   dKb = -dU h^T
//   dgamma_r = rowsum_r(Z) - colsum_r(Z) + rowsum_r(Zr) - colsum_r(Zr)
//              + scale e^{gamma_r} q_r.(dO h^T)_r + beta_r e^{gamma_r} dKb_r.k_r - Z3_r
//   dgamma_C += e^{gamma_C} <dh', h> + sum_s Z3_s
//   with Z = scale M o P1 o QK^T, Zr = dAkk o A, Z3_s = e^{gamma_C - gamma_s} k_s.(Delta dh'^T)_s,
//   and dg = the in-chunk reverse cumulative sum of dgamma.
//
// All twelve products run on tcgen05 from 128-byte-swizzled shared-memory
// tiles (TMA-loaded inputs; dU, T1, dG written by the CTA), in three rounds:
//   1. S = QK^T, G = KK^T, P1 = dO Delta^T, dU = Ainv^T dDelta
//   2. dAkk, T1 K, T1^T Q, dO h^T
//   3. dU h^T, Delta dh'^T, and dG K + dG^T K accumulated onto T1^T Q
// The 8 warps read the accumulators back with the 16x256b TMEM load, whose
// register layout is the warp-MMA fragment layout (warp w: rows 16 (w % 4)..+15,
// column half w / 4), and do the elementwise terms and the row and column sums
// in a fixed order. A warp-level version of this kernel was bound by the
// load/store unit re-reading the MMA operands; here the tensor core reads them.
//
// Rows past the end of the chunk are read as whatever follows in memory (the
// next sequence, or zeros past the tensor): every term they enter is
// multiplied by an exactly-zero decay mask, Ainv or beta entry, or lands in a
// row that is not written.
//
// dq and dk go to per-value-head fp32 partials (summed over the GQA group by
// bwd_final); dv, dg, dbeta are written directly.
#include <cstddef>

#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kThreads = 256;
constexpr int kWN = 2;  // column groups: warp w owns column half w / 4
constexpr int C = 64, K = 128, V = 128;

// ---- shared memory (bytes from a 1024-aligned base); [64][128] tiles are two
//      64-column halves of [64 rows][128 B], 128-byte swizzle
constexpr int kQ = 0, kKt = 16384, kdO = 32768, kD = 49152, kdD = 65536, kVt = 81920;
constexpr int kA = 98304;     // Ainv [64 s][64 r]
constexpr int kT1 = 106496;   // T1 [64 r][64 s]
constexpr int kdG = 114688;   // dG [64 r][64 s]
constexpr int kdU = 122880;   // dU [64 r][128 v]
constexpr int kH = 139264;    // h [128 k][128 v]: two halves of [128 rows][128 B]
constexpr int kdH = 172032;   // dh'
constexpr int kVec = 204800;
constexpr int kBar = kVec + 4096;
constexpr int kSmemBytes = kBar + 64 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory layout");

// tensor memory: round 1  S 0, G 64, P1 128, dU 192;
//                round 2  dAkk 0, TK 64, T1^T Q 192, dQ1 320;
//                round 3  dKb 0, dK2 320, (T1^T Q + dG K + dG^T K) 192
constexpr uint32_t kTmemCols = 512;

struct Vecs {
    float gam[64], egam[64], bet[64];
    float rowdg[kWN][64], rowdb[kWN][64];  // per column-half partial row sums
    float coldg[4][64];                    // per row-quarter partial column sums
    float scal[kThreads / 32];             // per-warp partial of the chunk-level dgamma_C term
};
static_assert(sizeof(Vecs) <= 4096, "vector area");

// Byte offset of element (r, c) in a 128-byte-swizzled tile of 64-column halves
// (half_bytes = rows * 128).
__device__ __forceinline__ uint32_t sw_off(int r, int c, int half_bytes) {
    return (c >> 6) * half_bytes + (r >> 3) * 1024 + (r & 7) * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2;
}

__device__ __forceinline__ float2 ld_pair_sw(uint32_t base, int r, int c) {
    uint32_t u;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(u) : "r"(base + sw_off(r, c, 8192)));
    return unpack_bf16(u);
}

__device__ __forceinline__ bool cta_wait(uint64_t *bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(a, parity))
        if (globaltimer() - t0 > kWaitNs) return false;
    return true;
}

// K-major operand over a tile of 64-column halves: 16 columns per k-step.
__device__ __forceinline__ uint64_t kdesc(uint32_t base, int ks, int half_bytes) {
    return smem_desc(base + (ks >> 2) * half_bytes + (ks & 3) * 32, 16, 1024, kSw128);
}
// MN-major operand (K runs down the rows): 16 rows per k-step; halves 8192 bytes apart.
__device__ __forceinline__ uint64_t mdesc(uint32_t base, int ks) {
    return smem_desc(base + ks * 2048, 8192, 1024, kSw128);
}

struct GradParams {
    Dims d;
    const float *gamma, *beta;
    float *dq_part, *dk_part;        // [T, Hv, K]
    __nv_bfloat16 *dv;               // [T, Hv, V]
    float *dg, *dbeta;               // [T, Hv]
    unsigned *status;
};

struct GradMaps {
    CUtensorMap q, k, v, d_o, delta, ddelta, h, dh, ainv;
};

__global__ void __launch_bounds__(kThreads, 1) bwd_grad_kernel(const __grid_constant__ GradMaps tm,
                                                               const GradParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    Vecs &vec = *reinterpret_cast<Vecs *>(smem + kVec);
    const Dims &d = prm.d;
    const int cg = blockIdx.x, h = blockIdx.y;
    const int hq = h / (d.Hv / d.Hq);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wm = warp & 3, wn = warp >> 2;
    const int g = lane >> 2, c4 = lane & 3;
    const int r0 = 16 * wm + g, r1 = r0 + 8;  // rows this thread holds in every accumulator
    const int n = chunk_owner(d, cg);
    if (n < 0) return;  // whole CTA, before any allocation
    const SeqRange sr = seq_range(d, n);
    const int ci = cg - sr.chunk0;
    const int t0 = sr.start + ci * C, len = min(C, sr.len - ci * C);
    const float scale = d.scale;
    uint64_t *bar_in = reinterpret_cast<uint64_t *>(smem + kBar);  // chunk tiles
    uint64_t *bar_st = bar_in + 1;                                  // h, dh'
    uint64_t *bar_mma = bar_in + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_in + 3);

    if (tid == 0) {
        mbar_init(bar_in, 1);
        mbar_init(bar_st, 1);
        mbar_init(bar_mma, 1);
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
    const uint32_t lane_base = (uint32_t)(wm * 32) << 16;
    bool pending_in = false, pending_st = false, pending_mma = false;  // thread 0: issued, not yet consumed
    uint32_t mma_phase = 0;

    // ---- loads by TMA: the chunk tiles, then the two states (they land while round 1 runs)
    if (tid == 0) {
        const int crow = (cg * d.Hv + h) * C, krow = (cg * d.Hv + h) * K;
        mbar_arrive_expect_tx(bar_in, 6 * 16384 + 8192);
        tma_load_3d(smem + kQ, &tm.q, bar_in, 0, hq, t0);
        tma_load_3d(smem + kQ + 8192, &tm.q, bar_in, 64, hq, t0);
        tma_load_3d(smem + kKt, &tm.k, bar_in, 0, hq, t0);
        tma_load_3d(smem + kKt + 8192, &tm.k, bar_in, 64, hq, t0);
        tma_load_3d(smem + kdO, &tm.d_o, bar_in, 0, h, t0);
        tma_load_3d(smem + kdO + 8192, &tm.d_o, bar_in, 64, h, t0);
        tma_load_3d(smem + kD, &tm.delta, bar_in, 0, h, t0);
        tma_load_3d(smem + kD + 8192, &tm.delta, bar_in, 64, h, t0);
        tma_load_3d(smem + kdD, &tm.ddelta, bar_in, 0, h, t0);
        tma_load_3d(smem + kdD + 8192, &tm.ddelta, bar_in, 64, h, t0);
        tma_load_3d(smem + kVt, &tm.v, bar_in, 0, h, t0);
        tma_load_3d(smem + kVt + 8192, &tm.v, bar_in, 64, h, t0);
        tma_load_2d(smem + kA, &tm.ainv, bar_in, 0, crow);
        mbar_arrive_expect_tx(bar_st, 4 * 16384);
        tma_load_2d(smem + kH, &tm.h, bar_st, 0, krow);
        tma_load_2d(smem + kH + 16384, &tm.h, bar_st, 64, krow);
        tma_load_2d(smem + kdH, &tm.dh, bar_st, 0, krow);
        tma_load_2d(smem + kdH + 16384, &tm.dh, bar_st, 64, krow);
        pending_in = pending_st = true;
    }
    if (tid < C) {
        const int r = tid, rr = min(r, len - 1);
        const float gm = prm.gamma[(size_t)(t0 + rr) * d.Hv + h];
        vec.gam[r] = gm;
        vec.egam[r] = __expf(gm);
        vec.bet[r] = r < len ? prm.beta[(size_t)(t0 + r) * d.Hv + h] : 0.f;
    }
    bool ok = cta_wait(bar_in, 0);
    if (ok) pending_in = false;

    // ---- round 1: S, G, P1 (64 x 64) and dU (64 x 128)
    if (ok && tid == 0) {
        tc_fence_after();
        const uint32_t idCC = idesc_bf16(64, 64, false, false), idU = idesc_bf16(64, 128, true, true);
        for (int ks = 0; ks < 8; ++ks) {
            mma_bf16(tmem + 0, kdesc(sb + kQ, ks, 8192), kdesc(sb + kKt, ks, 8192), idCC, ks > 0);
            mma_bf16(tmem + 64, kdesc(sb + kKt, ks, 8192), kdesc(sb + kKt, ks, 8192), idCC, ks > 0);
            mma_bf16(tmem + 128, kdesc(sb + kdO, ks, 8192), kdesc(sb + kD, ks, 8192), idCC, ks > 0);
        }
        for (int ks = 0; ks < 4; ++ks) mma_bf16(tmem + 192, mdesc(sb + kA, ks), mdesc(sb + kdD, ks), idU, ks > 0);
        mma_commit(bar_mma);
        pending_mma = true;
    }
    __syncthreads();  // the gate vectors
    const float gC = vec.gam[63];  // gamma at the chunk's last token (padded rows repeat it)
    const float gr[2] = {vec.gam[r0], vec.gam[r1]};
    const float er[2] = {vec.egam[r0], vec.egam[r1]};
    const float br[2] = {vec.bet[r0], vec.bet[r1]};
    const bool lr[2] = {r0 < len, r1 < len};
    float rdg[2] = {0.f, 0.f}, rdb[2] = {0.f, 0.f}, cdg[8] = {}, sdg = 0.f;
    const int cc0 = 32 * wn, ck0 = 64 * wn;  // this warp's first column (C x C, C x K)
    ok = ok && cta_wait(bar_mma, mma_phase & 1);
    if (ok) ++mma_phase, pending_mma = false;
    tc_fence_after();

    float sacc[4][4], gacc[4][4];  // S -> strictly lower E, G: kept for round 2
    if (ok) {
        float v[16], pacc[4][4];
        tmem_ld16x256_x4(tmem + lane_base + 0 + cc0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) sacc[i >> 2][i & 3] = v[i];
        tmem_ld16x256_x4(tmem + lane_base + 64 + cc0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) gacc[i >> 2][i & 3] = v[i];
        tmem_ld16x256_x4(tmem + lane_base + 128 + cc0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) pacc[i >> 2][i & 3] = v[i];
        // T1 = scale M o P1, Z = T1 o S (row and column sums)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int hi = q >> 1, s = cc0 + 8 * j + 2 * c4 + (q & 1), r = hi ? r1 : r0;
                const bool on = lr[hi] && s <= r;  // s < len follows
                const float E = on ? __expf(gr[hi] - vec.gam[s]) : 0.f;
                const float t1 = scale * E * pacc[j][q];
                const float z = t1 * sacc[j][q];
                rdg[hi] += z;
                cdg[2 * j + (q & 1)] -= z;
                pacc[j][q] = t1;
                sacc[j][q] = s < r ? E : 0.f;  // strictly lower part of E for the A terms
            }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int s = cc0 + 8 * j + 2 * c4;
            st_shared_b32(sb + kT1 + sw_off(r0, s, 8192), pack_bf16(pacc[j][0], pacc[j][1]));
            st_shared_b32(sb + kT1 + sw_off(r1, s, 8192), pack_bf16(pacc[j][2], pacc[j][3]));
        }
        // dU: dv = beta dU, dbeta += dU.v, dU -> shared memory (bf16)
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int cb = ck0 + 32 * part;
            tmem_ld16x256_x4(tmem + lane_base + 192 + cb, v);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int col = cb + 8 * i + 2 * c4;
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = hi ? r1 : r0;
                    const float u0 = v[4 * i + 2 * hi], u1 = v[4 * i + 2 * hi + 1];
                    const float2 vv = ld_pair_sw(sb + kVt, r, col);
                    rdb[hi] += u0 * vv.x + u1 * vv.y;
                    if (lr[hi])
                        *reinterpret_cast<uint32_t *>(prm.dv + ((size_t)(t0 + r) * d.Hv + h) * V + col) =
                            pack_bf16(br[hi] * u0, br[hi] * u1);
                    st_shared_b32(sb + kdU + sw_off(r, col, 8192), pack_bf16(u0, u1));
                }
            }
        }
    }
    fence_proxy_async();  // T1, dU -> the tensor core
    tc_fence_before();
    __syncthreads();
    ok = ok && cta_wait(bar_st, 0);
    if (ok) pending_st = false;

    // ---- round 2: dAkk (64 x 64), T1 K, T1^T Q, dO h^T (64 x 128)
    if (ok && tid == 0) {
        tc_fence_after();
        const uint32_t idCC = idesc_bf16(64, 64, false, false);
        const uint32_t idKM = idesc_bf16(64, 128, false, true), idMM = idesc_bf16(64, 128, true, true);
        const uint32_t idKK = idesc_bf16(64, 128, false, false);
        for (int ks = 0; ks < 8; ++ks) {
            mma_bf16(tmem + 0, kdesc(sb + kdU, ks, 8192), kdesc(sb + kD, ks, 8192), idCC, ks > 0);
            mma_bf16(tmem + 320, kdesc(sb + kdO, ks, 8192), kdesc(sb + kH, ks, 16384), idKK, ks > 0);
        }
        for (int ks = 0; ks < 4; ++ks) {
            mma_bf16(tmem + 64, kdesc(sb + kT1, ks, 8192), mdesc(sb + kKt, ks), idKM, ks > 0);
            mma_bf16(tmem + 192, mdesc(sb + kT1, ks), mdesc(sb + kQ, ks), idMM, ks > 0);
        }
        mma_commit(bar_mma);
        pending_mma = true;
    }
    ok = ok && cta_wait(bar_mma, mma_phase & 1);
    if (ok) ++mma_phase, pending_mma = false;
    tc_fence_after();
    if (ok) {
        // dAkk = -dU Delta^T (s < r): dbeta, Zr, dG -> shared memory
        float v[16];
        tmem_ld16x256_x4(tmem + lane_base + 0 + cc0, v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float dgv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int hi = q >> 1;
                const float E = sacc[j][q];  // zero unless s < r < len
                const float dA = -v[4 * j + q];
                const float eg = E * gacc[j][q];
                rdb[hi] += dA * eg;
                const float zr = br[hi] * dA * eg;
                rdg[hi] += zr;
                cdg[2 * j + (q & 1)] -= zr;
                dgv[q] = dA * br[hi] * E;
            }
            const int s = cc0 + 8 * j + 2 * c4;
            st_shared_b32(sb + kdG + sw_off(r0, s, 8192), pack_bf16(dgv[0], dgv[1]));
            st_shared_b32(sb + kdG + sw_off(r1, s, 8192), pack_bf16(dgv[2], dgv[3]));
        }
        // dq = scale diag(e^gamma) dO h^T + T1 K ; dgamma += scale e^gamma q.(dO h^T)
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int cb = ck0 + 32 * part;
            float a[16], b[16];
            tmem_ld16x256_x4(tmem + lane_base + 320 + cb, a);
            tmem_ld16x256_x4(tmem + lane_base + 64 + cb, b);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int col = cb + 8 * i + 2 * c4;
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = hi ? r1 : r0;
                    const float2 qq = ld_pair_sw(sb + kQ, r, col);
                    const float f = scale * er[hi];
                    const float x0 = a[4 * i + 2 * hi], x1 = a[4 * i + 2 * hi + 1];
                    rdg[hi] += f * (x0 * qq.x + x1 * qq.y);
                    if (lr[hi])
                        *reinterpret_cast<float2 *>(prm.dq_part + ((size_t)(t0 + r) * d.Hv + h) * K + col) =
                            make_float2(fmaf(f, x0, b[4 * i + 2 * hi]), fmaf(f, x1, b[4 * i + 2 * hi + 1]));
                }
            }
        }
    }
    fence_proxy_async();  // dG -> the tensor core
    tc_fence_before();
    __syncthreads();

    // ---- round 3: dU h^T, Delta dh'^T; dG K + dG^T K onto T1^T Q
    if (ok && tid == 0) {
        tc_fence_after();
        const uint32_t idKK = idesc_bf16(64, 128, false, false);
        const uint32_t idKM = idesc_bf16(64, 128, false, true), idMM = idesc_bf16(64, 128, true, true);
        for (int ks = 0; ks < 8; ++ks) {
            mma_bf16(tmem + 0, kdesc(sb + kdU, ks, 8192), kdesc(sb + kH, ks, 16384), idKK, ks > 0);
            mma_bf16(tmem + 320, kdesc(sb + kD, ks, 8192), kdesc(sb + kdH, ks, 16384), idKK, ks > 0);
        }
        for (int ks = 0; ks < 4; ++ks) {
            mma_bf16(tmem + 192, kdesc(sb + kdG, ks, 8192), mdesc(sb + kKt, ks), idKM, true);
            mma_bf16(tmem + 192, mdesc(sb + kdG, ks), mdesc(sb + kKt, ks), idMM, true);
        }
        mma_commit(bar_mma);
        pending_mma = true;
    }
    ok = ok && cta_wait(bar_mma, mma_phase & 1);
    if (ok) ++mma_phase, pending_mma = false;
    tc_fence_after();
    if (ok) {
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int cb = ck0 + 32 * part;
            float kb[16], k2[16], ks3[16];
            tmem_ld16x256_x4(tmem + lane_base + 0 + cb, kb);     // dU h^T = -dKb
            tmem_ld16x256_x4(tmem + lane_base + 320 + cb, k2);   // Delta dh'^T
            tmem_ld16x256_x4(tmem + lane_base + 192 + cb, ks3);  // T1^T Q + dG K + dG^T K
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = hi ? r1 : r0;
                const float fk = br[hi] * er[hi];                     // dk += beta e^gamma dKb
                const float f2 = lr[hi] ? __expf(gC - gr[hi]) : 0.f;  // dk += e^{gamma_C - gamma} (Delta dh'^T)
                float dotb = 0.f, z3 = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int col = cb + 8 * i + 2 * c4;
                    const float2 kk = ld_pair_sw(sb + kKt, r, col);
                    const float b0 = -kb[4 * i + 2 * hi], b1 = -kb[4 * i + 2 * hi + 1];
                    const float e0 = k2[4 * i + 2 * hi], e1 = k2[4 * i + 2 * hi + 1];
                    dotb += b0 * kk.x + b1 * kk.y;
                    z3 += e0 * kk.x + e1 * kk.y;
                    if (lr[hi])
                        *reinterpret_cast<float2 *>(prm.dk_part + ((size_t)(t0 + r) * d.Hv + h) * K + col) =
                            make_float2(ks3[4 * i + 2 * hi] + fk * b0 + f2 * e0, ks3[4 * i + 2 * hi + 1] + fk * b1 + f2 * e1);
                }
                rdb[hi] += er[hi] * dotb;
                rdg[hi] += br[hi] * er[hi] * dotb;
                z3 *= f2;
                rdg[hi] -= z3;
                sdg += z3;
            }
        }
    }

    // ---- e^{gamma_C} <dh', h>: this thread's share of the 128 x 128 dot (same layout in both tiles)
    if (ok) {
        float s = 0.f;
        for (int e = tid; e < K * V / 8; e += kThreads) {
            const uint4 a = ld_shared_v4(sb + kH + e * 16), b = ld_shared_v4(sb + kdH + e * 16);
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 x = unpack_bf16(aw[i]), y = unpack_bf16(bw[i]);
                s += x.x * y.x + x.y * y.y;
            }
        }
        sdg += __expf(gC) * s;
    }

    // ---- fixed-order reductions: quad (row sums), column groups, then across warps
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
        rdg[hi] += __shfl_xor_sync(0xffffffffu, rdg[hi], 1);
        rdg[hi] += __shfl_xor_sync(0xffffffffu, rdg[hi], 2);
        rdb[hi] += __shfl_xor_sync(0xffffffffu, rdb[hi], 1);
        rdb[hi] += __shfl_xor_sync(0xffffffffu, rdb[hi], 2);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        cdg[i] += __shfl_xor_sync(0xffffffffu, cdg[i], 4);
        cdg[i] += __shfl_xor_sync(0xffffffffu, cdg[i], 8);
        cdg[i] += __shfl_xor_sync(0xffffffffu, cdg[i], 16);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sdg += __shfl_xor_sync(0xffffffffu, sdg, o);
    if (c4 == 0) {
        vec.rowdg[wn][r0] = rdg[0];
        vec.rowdg[wn][r1] = rdg[1];
        vec.rowdb[wn][r0] = rdb[0];
        vec.rowdb[wn][r1] = rdb[1];
    }
    if (g == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            vec.coldg[wm][cc0 + 8 * j + 2 * c4] = cdg[2 * j];
            vec.coldg[wm][cc0 + 8 * j + 2 * c4 + 1] = cdg[2 * j + 1];
        }
    }
    if (lane == 0) vec.scal[warp] = sdg;
    __syncthreads();
    if (ok && warp == 0) {
        // dgamma_r for r = lane, lane + 32; then the reverse cumulative sum over the chunk
        float dgr[2], dbr[2];
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int r = lane + 32 * hi;
            float a = 0.f, b = 0.f;
#pragma unroll
            for (int w = 0; w < kWN; ++w) a += vec.rowdg[w][r], b += vec.rowdb[w][r];
            a += ((vec.coldg[0][r] + vec.coldg[1][r]) + vec.coldg[2][r]) + vec.coldg[3][r];
            dgr[hi] = r < len ? a : 0.f;
            dbr[hi] = b;
        }
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) tot += vec.scal[w];
        // the chunk-level term belongs to the last live token
#pragma unroll
        for (int hi = 0; hi < 2; ++hi)
            if (lane + 32 * hi == len - 1) dgr[hi] += tot;
        // reverse inclusive scan over 64 values held as (lane, lane + 32)
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float x = __shfl_down_sync(0xffffffffu, dgr[1], o);
            if (lane + o < 32) dgr[1] += x;
        }
        const float hi_tot = __shfl_sync(0xffffffffu, dgr[1], 0);  // sum of the upper half
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float x = __shfl_down_sync(0xffffffffu, dgr[0], o);
            if (lane + o < 32) dgr[0] += x;
        }
        dgr[0] += hi_tot;
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int r = lane + 32 * hi;
            if (r < len) {
                prm.dg[(size_t)(t0 + r) * d.Hv + h] = dgr[hi];
                prm.dbeta[(size_t)(t0 + r) * d.Hv + h] = dbr[hi];
            }
        }
    }
    if (!ok && tid == 0) {
        set_status(prm.status, GDN_ERR_TIMEOUT);
        // a load or a round of MMAs still in flight: let it finish (bounded)
        const uint64_t t1 = globaltimer();
        while (pending_in && !mbar_try_wait(smem_u32(bar_in), 0) && globaltimer() - t1 < kWaitNs) {
        }
        while (pending_st && !mbar_try_wait(smem_u32(bar_st), 0) && globaltimer() - t1 < kWaitNs) {
        }
        while (pending_mma && !mbar_try_wait(smem_u32(bar_mma), mma_phase & 1) && globaltimer() - t1 < kWaitNs) {
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_bwd_grad_tc(const BwdArgs &a, const void *h_chunks16, const void *dh_chunks16,
                               const void *delta16, const void *ddelta16, float *dq_part, float *dk_part) {
    const Dims &d = a.d;
    if (d.NC == 0) return cudaSuccess;
    GradMaps m;
    const cuuint64_t T = (cuuint64_t)(d.T_total > 0 ? d.T_total : 1);
    const cuuint64_t dqk[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hq, T};
    const cuuint64_t sqk[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hq * d.K * 2};
    const cuuint64_t dvv[3] = {(cuuint64_t)d.V, (cuuint64_t)d.Hv, T};
    const cuuint64_t svv[2] = {(cuuint64_t)d.V * 2, (cuuint64_t)d.Hv * d.V * 2};
    const cuuint32_t b3[3] = {64, 1, 64};
    const cuuint64_t dst[2] = {(cuuint64_t)d.V, (cuuint64_t)d.NC * d.Hv * d.K};
    const cuuint64_t sst[1] = {(cuuint64_t)d.V * 2};
    const cuuint32_t bst[2] = {64, 128};
    const cuuint64_t dai[2] = {64, (cuuint64_t)d.NC * d.Hv * 64};
    const cuuint64_t sai[1] = {128};
    const cuuint32_t bai[2] = {64, 64};
    const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_bf16_map(&m.q, a.q, 3, dqk, sqk, b3, SW) || !make_bf16_map(&m.k, a.k, 3, dqk, sqk, b3, SW) ||
        !make_bf16_map(&m.v, a.v, 3, dvv, svv, b3, SW) || !make_bf16_map(&m.d_o, a.d_o, 3, dvv, svv, b3, SW) ||
        !make_bf16_map(&m.delta, delta16, 3, dvv, svv, b3, SW) ||
        !make_bf16_map(&m.ddelta, ddelta16, 3, dvv, svv, b3, SW) ||
        !make_bf16_map(&m.h, h_chunks16, 2, dst, sst, bst, SW) || !make_bf16_map(&m.dh, dh_chunks16, 2, dst, sst, bst, SW) ||
        !make_bf16_map(&m.ainv, a.ainv, 2, dai, sai, bai, SW))
        return cudaErrorInvalidValue;
    GradParams p;
    p.d = d;
    p.gamma = a.gamma;
    p.beta = a.beta;
    p.dq_part = dq_part;
    p.dk_part = dk_part;
    p.dv = (__nv_bfloat16 *)a.dv;
    p.dg = a.dg;
    p.dbeta = a.dbeta;
    p.status = a.status;
    cudaError_t e = cudaFuncSetAttribute(bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    bwd_grad_kernel<<<dim3(d.NC, d.Hv), kThreads, kSmemBytes, a.stream>>>(m, p);
    return cudaGetLastError();
}

}  // namespace gdn
