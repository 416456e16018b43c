// gdn_bwd_grad.cu -- per-chunk gradients of the chunked backward (bf16,
// K = V = 128). No dependence between chunks: a persistent grid (one CTA per
// SM) walks the (chunk, qk head) items.
//
// Per chunk and value head (rows r, s; h the entry state, Delta, from the
// forward; dh' and dDelta from the reverse scan; Kb = diag(beta e^gamma) K,
// E_rs = e^{gamma_r - gamma_s}, M = E on s <= r, A_rs = beta_r E_rs k_r.k_s on s < r):
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
// dq and dk of a qk head are the sums of these over its group of value heads.
//
// An item is one chunk of one qk head; its G = Hv / Hq value heads run one
// after another ("steps") in the CTA, so dq and dk are summed over the group
// on chip and written once, in bf16: dk stays in tensor memory (the next
// head's T1^T Q product accumulates onto it), dq is parked in spare columns.
// All twelve products of a step run on tcgen05 from 128-byte-swizzled
// shared-memory tiles, in three product batches:
//   1. S = QK^T, G = KK^T, P1 = dO Delta^T, dU = Ainv^T dDelta
//   2. dAkk, T1 K, T1^T Q (onto dk), dO h^T
//   3. dU h^T, Delta dh'^T, and dG K + dG^T K onto dk
// The 16 warps read the accumulators back with the 16x256b TMEM load, whose
// register layout is the warp-MMA fragment layout (warp w: rows 16 (w % 4)..+15,
// column quarter w / 4), and do the elementwise terms and the row and column sums
// in a fixed order. Four warps per scheduler hide the latency of these epilogues.
//
// Delta, dDelta, h and dh' arrive in the blocked layout the chain kernels keep
// them in (per 32-column slice: 8-column blocks of 16-byte rows), each one
// contiguous bulk copy per step; h, dh' and Delta are read as K-major operands
// without swizzle, dDelta as an MN-major one.
// Each input tile of the next step is loaded by TMA as soon as the current
// step is done with its buffer (Ainv and dDelta after product batch 1, dO after
// product batch 2, h and dh' after product batch 3; Delta has two buffers), so that only a new
// item's k tile waits on memory. dv, dq and dk of a full chunk are written by
// TMA stores from shared memory: dv in place of v, dq in place of q, dk in
// the T1 | dG tiles; a ragged chunk is written row by row.
//
// Rows past the end of a ragged chunk hold the next packed sequence (or zeros
// past the tensor): the q, k, v and dO tiles are zeroed there before any
// product reads them, and the gates are clamped (gamma) or zero (beta), so a
// non-finite value of the next sequence cannot reach this one; the chain
// kernels store Delta and dDelta as zero there.
#include <cstddef>

#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kThreads = 512;
constexpr int kWN = 4;              // column groups: warp w owns column quarter w / 4
constexpr int kJJ = 64 / kWN / 8;   // 8-column tiles of a C x C accumulator per warp
constexpr int kParts = 128 / kWN / 32;  // 32-column loads of a C x K accumulator per warp
constexpr int C = 64, K = 128, V = 128;
constexpr int kStoreTid = 32;  // issues the TMA stores and the loads of the buffers they read
// The products of a batch are issued by two threads (thread 0 and kStoreTid), each
// committing to the batch's mbarrier (two arrivals): a single issuing thread spends
// about 70 cycles per tcgen05.mma.

// ---- shared memory (bytes from a 1024-aligned base); [64][128] tiles are two
//      64-column halves of [64 rows][128 B], 128-byte swizzle
constexpr int kQ = 0, kKt = 16384;  // per item; dq goes out through the q tile
constexpr int kdO = 32768;
constexpr int kD = 49152;           // Delta, two buffers (step parity): (v/8)*1024 + t*16
constexpr int kdD = 81920;          // dDelta, blocked: (v/8)*1024 + t*16
constexpr int kVt = 98304;          // v; dv goes out through it
constexpr int kA = 114688;          // Ainv [64 s][64 r]
constexpr int kT1 = 122880;         // T1 [64 r][64 s]   } dk goes out through these two:
constexpr int kdG = 131072;         // dG [64 r][64 s]   } one [64][128] tile
constexpr int kdU = 139264;         // dU [64 r][128 v]
constexpr int kH = 155648;          // h [128 k][128 v]: (v/8)*2048 + k*16
constexpr int kdH = 188416;         // dh', same layout
constexpr int kVec = 221184;
constexpr int kBar = kVec + 4096;
constexpr int kSmemBytes = kBar + 128 + 1024;
static_assert(kdG == kT1 + 8192 && kSmemBytes <= 232448, "shared memory layout");

// tensor memory columns: product batch 1  S, G, P1, dU;
// product batch 2  dAkk, T1 K, dk (T1^T Q), dO h^T;
// product batch 3  dU h^T, Delta dh'^T, dk (+ dG K + dG^T K). dk lives at kCDK for the whole
// item; dq is parked at kCPark between the heads of an item (column quarter w / 4 at
// lanes 16 ((w / 4) % 2).. of the warp's sub-partition, columns 32 ((w / 4) / 2)..).
constexpr uint32_t kCS = 0, kCG = 64, kCP1 = 128, kCU = 320;
constexpr uint32_t kCAkk = 0, kCTK = 64, kCDK = 192, kCQ1 = 320;
constexpr uint32_t kCKb = 0, kCK2 = 320, kCPark = 448;
constexpr uint32_t kTmemCols = 512;

// mbarriers: one per load group, and one for the batches of MMAs
enum Bar { kBarQ, kBarK, kBarD0, kBarD1, kBarDO, kBarA, kBarV, kBarSt, kBarMma, kNumBar };

struct Vecs {
    float gam[64], egam[64], bet[64];
    float rowdg[kWN][64], rowdb[kWN][64];  // per column-group partial row sums
    float coldg[4][64];                    // per row-quarter partial column sums
    float scal[kThreads / 32];             // per-warp partial of the chunk-level dgamma_C term
};
static_assert(sizeof(Vecs) <= 4096, "vector area");

// Byte offset of element (r, c) in a 128-byte-swizzled tile of 64-column halves
// (half_bytes = rows * 128).
__device__ __forceinline__ uint32_t sw_off(int r, int c, int half_bytes) {
    return (c >> 6) * half_bytes + (r >> 3) * 1024 + (r & 7) * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2;
}

// Zeroes rows [len, 64) of a [64][128] bf16 tile of two 64-column halves of 128-byte
// rows (the swizzle permutes 16-byte chunks within a row, so whole rows are zeroed
// regardless of it). Out of line: only ragged chunks call it.
__device__ __noinline__ void zero_rows(uint32_t tile, int len, int tid) {
    for (int i = tid; i < (C - len) * 16; i += kThreads) {
        const int r = len + (i >> 4), c = i & 15;
        st_shared_v4(tile + (c >> 3) * 8192 + r * 128 + (c & 7) * 16, 0u, 0u, 0u, 0u);
    }
}

// Stores 8 fp32 per thread in the 16x256b.x2 layout (what tmem_ld16x256_x2 reads) and
// waits until the store has completed.
__device__ __forceinline__ void tmem_st16x256_x2(uint32_t taddr, const float (&v)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x2.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n\t"
        "tcgen05.wait::st.sync.aligned;"
        :
        : "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
        : "memory");
}

// This warp's kJJ 8-column tiles of a C x C accumulator (16 rows): v[4 jj + q].
static_assert(kJJ == 2, "16 columns of a C x C accumulator per warp");
__device__ __forceinline__ void ld_cc(uint32_t taddr, float (&v)[4 * kJJ]) { tmem_ld16x256_x2(taddr, v); }

__device__ __forceinline__ float2 ld_pair_sw(uint32_t base, int r, int c) {
    uint32_t u;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(u) : "r"(base + sw_off(r, c, 8192)));
    return unpack_bf16(u);
}

// Operand descriptors are built once per tile; a k-step only moves the start
// address (descriptor bits 0..13, in 16-byte units), by a constant once the
// issue loops are unrolled.
// K-major operand over a tile of 64-column halves: 16 columns per k-step.
__device__ __forceinline__ uint64_t kbase(uint32_t base) { return smem_desc(base, 16, 1024, kSw128); }
__device__ __forceinline__ constexpr uint64_t kstep(int ks, int half_bytes) {
    return (uint64_t)(((ks >> 2) * half_bytes + (ks & 3) * 32) >> 4);
}
// MN-major operand (K runs down the rows): 16 rows per k-step; halves 8192 bytes apart.
__device__ __forceinline__ uint64_t mbase(uint32_t base) { return smem_desc(base, 8192, 1024, kSw128); }
__device__ __forceinline__ constexpr uint64_t mstep(int ks) { return (uint64_t)(ks * 2048 >> 4); }
// K-major operand without swizzle, the blocked layout: core matrices of 8 rows x
// 16 bytes, 128 bytes apart down the rows, kblk bytes apart along K (Delta 1024,
// h and dh' 2048); a k-step of 16 is two core matrices along K.
__device__ __forceinline__ uint64_t bbase(uint32_t base, uint32_t kblk) { return smem_desc(base, kblk, 128, kSwNone); }
__device__ __forceinline__ constexpr uint64_t bstep(int ks, int kblk) { return (uint64_t)(ks * 2 * kblk >> 4); }

struct GradParams {
    Dims d;
    const __nv_bfloat16 *delta, *ddelta, *h, *dh;  // blocked: per (chunk, head) 4 slices of [4][64][8] / [4][128][8]
    const float *gamma, *beta;
    __nv_bfloat16 *dq, *dk;  // [T, Hq, K]
    __nv_bfloat16 *dv;       // [T, Hv, V]
    float *dg, *dbeta;       // [T, Hv]
    int n_items;             // NC * Hq
    unsigned *status;
};

struct GradMaps {
    CUtensorMap q, k, v, d_o, ainv;  // loads
    CUtensorMap dq, dk, dv;                 // stores
};

// One step: value head g of the group of qk head hq, on chunk cg.
struct Step {
    int item, cg, hq, g, t0, len;
    bool valid;
};

__device__ Step item_step(const Dims &d, int item, int stride, int n_items) {
    Step s;
    s.valid = false;
    for (; item < n_items; item += stride) {
        const int cg = item / d.Hq;
        const int n = chunk_owner(d, cg);
        if (n < 0) continue;
        const SeqRange sr = seq_range(d, n);
        const int ci = cg - sr.chunk0;
        s.item = item;
        s.cg = cg;
        s.hq = item % d.Hq;
        s.g = 0;
        s.t0 = sr.start + ci * C;
        s.len = min(C, sr.len - ci * C);
        s.valid = true;
        break;
    }
    return s;
}

__device__ __forceinline__ bool cta_wait(uint64_t *bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(a, parity))
        if (globaltimer() - t0 > kWaitNs) return false;
    return true;
}

__global__ void __launch_bounds__(kThreads, 1) bwd_grad_kernel(const __grid_constant__ GradMaps tm,
                                                               const GradParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    const uint32_t sb = smem_u32(smem);
    Vecs &vec = *reinterpret_cast<Vecs *>(smem + kVec);
    const Dims &d = prm.d;
    const int G = d.Hv / d.Hq;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wm = warp & 3, wn = warp >> 2;
    const int g = lane >> 2, c4 = lane & 3;
    const int r0 = 16 * wm + g, r1 = r0 + 8;  // rows this thread holds in every accumulator
    const float scale = d.scale;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBar);

    if (tid == 0) {
        for (int i = 0; i < kNumBar; ++i) mbar_init(&bars[i], i == kBarMma ? 2 : 1);
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
    const uint32_t park = tmem + ((uint32_t)(wm * 32 + (wn & 1) * 16) << 16) + kCPark + 32 * (wn >> 1);
    uint32_t phase = 0;  // bit b: parity of the next completion of barrier b (same in every thread)
    uint32_t pend = 0;   // issuing threads: barriers with a completion not yet waited for

    auto wait_bar = [&](int b) -> bool {
        const bool r = cta_wait(&bars[b], (phase >> b) & 1);
        if (r) {
            phase ^= 1u << b;
            pend &= ~(1u << b);
        }
        return r;
    };
    auto expect = [&](int b, uint32_t bytes) {
        mbar_arrive_expect_tx(&bars[b], bytes);
        pend |= 1u << b;
    };
    auto load_q = [&](const Step &s) {
        expect(kBarQ, 16384);
        tma_load_3d(smem + kQ, &tm.q, &bars[kBarQ], 0, s.hq, s.t0);
        tma_load_3d(smem + kQ + 8192, &tm.q, &bars[kBarQ], 64, s.hq, s.t0);
    };
    auto load_k = [&](const Step &s) {
        expect(kBarK, 16384);
        tma_load_3d(smem + kKt, &tm.k, &bars[kBarK], 0, s.hq, s.t0);
        tma_load_3d(smem + kKt + 8192, &tm.k, &bars[kBarK], 64, s.hq, s.t0);
    };
    auto head = [&](const Step &s) { return s.hq * G + s.g; };
    auto load_delta = [&](const Step &s, int buf) {
        const int b = kBarD0 + buf;
        expect(b, 16384);
        bulk_load(smem + kD + buf * 16384, prm.delta + ((size_t)s.cg * d.Hv + head(s)) * (C * V), 16384, &bars[b]);
    };
    auto load_do = [&](const Step &s) {
        expect(kBarDO, 16384);
        tma_load_3d(smem + kdO, &tm.d_o, &bars[kBarDO], 0, head(s), s.t0);
        tma_load_3d(smem + kdO + 8192, &tm.d_o, &bars[kBarDO], 64, head(s), s.t0);
    };
    auto load_a = [&](const Step &s) {  // dDelta and Ainv
        expect(kBarA, 16384 + 8192);
        bulk_load(smem + kdD, prm.ddelta + ((size_t)s.cg * d.Hv + head(s)) * (C * V), 16384, &bars[kBarA]);
        tma_load_2d(smem + kA, &tm.ainv, &bars[kBarA], 0, (s.cg * d.Hv + head(s)) * C);
    };
    auto load_v = [&](const Step &s) {
        expect(kBarV, 16384);
        tma_load_3d(smem + kVt, &tm.v, &bars[kBarV], 0, head(s), s.t0);
        tma_load_3d(smem + kVt + 8192, &tm.v, &bars[kBarV], 64, head(s), s.t0);
    };
    auto load_st = [&](const Step &s) {  // h and dh'
        const size_t off = ((size_t)s.cg * d.Hv + head(s)) * (K * V);
        expect(kBarSt, 2 * 32768);
        bulk_load(smem + kH, prm.h + off, 32768, &bars[kBarSt]);
        bulk_load(smem + kdH, prm.dh + off, 32768, &bars[kBarSt]);
    };
    auto commit_mma = [&]() {
        mma_commit(&bars[kBarMma]);
        pend |= 1u << kBarMma;
    };

    Step cur = item_step(d, blockIdx.x, gridDim.x, prm.n_items);
    if (cur.valid) {
        if (tid == 0) {
            load_delta(cur, 0);
            load_do(cur);
            load_a(cur);
            load_st(cur);
        } else if (tid == kStoreTid) {
            load_q(cur);
            load_k(cur);
            load_v(cur);
        }
    }
    float pg = 0.f, pb = 0.f;  // threads < C: gamma and beta of row tid of the coming step
    auto fetch_gate = [&](const Step &s) {
        if (tid < C) {
            const int rr = min(tid, s.len - 1);
            pg = prm.gamma[(size_t)(s.t0 + rr) * d.Hv + head(s)];
            pb = tid < s.len ? prm.beta[(size_t)(s.t0 + tid) * d.Hv + head(s)] : 0.f;
        }
    };
    if (cur.valid) fetch_gate(cur);
    bool ok = true;
    for (int j = 0; cur.valid; ++j) {
        Step nxt = cur;
        if (cur.g + 1 < G) ++nxt.g;
        else nxt = item_step(d, cur.item + gridDim.x, gridDim.x, prm.n_items);
        const int h = head(cur), t0 = cur.t0, len = cur.len, db = j & 1;
        const bool first = cur.g == 0, last = cur.g == G - 1, full = len == C;
        const uint32_t sD = sb + kD + db * 16384;

        // Delta of the next step into the other buffer (its last reader, product batch 3 of the
        // previous step, has completed)
        if (tid == 0 && nxt.valid) load_delta(nxt, db ^ 1);
        if (tid < C) {
            vec.gam[tid] = pg;  // padded rows repeat the last live gamma
            vec.egam[tid] = __expf(pg);
            vec.bet[tid] = pb;
        }
        ok = ok && (!first || (wait_bar(kBarQ) && wait_bar(kBarK))) && wait_bar(kBarD0 + db) &&
             wait_bar(kBarDO) && wait_bar(kBarA);
        if (len < C) {
            // a ragged chunk: the rows past its end hold the next packed sequence; zero them in
            // the q, k (the item's first step) and dO tiles before any product reads them
            if (first) {
                zero_rows(sb + kQ, len, tid);
                zero_rows(sb + kKt, len, tid);
            }
            zero_rows(sb + kdO, len, tid);
            fence_proxy_async();
            __syncthreads();
        }

        // ---- product batch 1: S, G, P1 (64 x 64) and dU (64 x 128)
        if (ok && tid == 0) {
            tc_fence_after();
            const uint32_t idCC = idesc_bf16(64, 64, false, false);
            const uint64_t q = kbase(sb + kQ), k = kbase(sb + kKt);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                mma_bf16(tmem + kCS, q + kstep(ks, 8192), k + kstep(ks, 8192), idCC, ks > 0);
                mma_bf16(tmem + kCG, k + kstep(ks, 8192), k + kstep(ks, 8192), idCC, ks > 0);
            }
            commit_mma();
        } else if (ok && tid == kStoreTid) {
            tc_fence_after();
            const uint32_t idCC = idesc_bf16(64, 64, false, false), idU = idesc_bf16(64, 128, true, true);
            const uint64_t o = kbase(sb + kdO), dl = bbase(sD, 1024), ai = mbase(sb + kA);
            // dDelta as the MN-major B of dU = Ainv^T dDelta, without swizzle: core matrices of
            // 8 tokens x 8 columns, 128 bytes apart along K (tokens), 1024 along N
            const uint64_t dd = smem_desc(sb + kdD, 128, 1024, kSwNone);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) mma_bf16(tmem + kCP1, o + kstep(ks, 8192), dl + bstep(ks, 1024), idCC, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) mma_bf16(tmem + kCU, ai + mstep(ks), dd + (uint64_t)(ks * 256 >> 4), idU, ks > 0);
            commit_mma();
        }
        if (tid == kStoreTid) bulk_wait_read<0>();  // the previous dk store has read T1 | dG
        ok = __syncthreads_and(ok);                 // the gate vectors
        if (!ok) break;
        if (nxt.valid) fetch_gate(nxt);
        const float gC = vec.gam[63];  // gamma at the chunk's last token (padded rows repeat it)
        const float gr[2] = {vec.gam[r0], vec.gam[r1]};
        const float er[2] = {vec.egam[r0], vec.egam[r1]};
        const float br[2] = {vec.bet[r0], vec.bet[r1]};
        const bool lr[2] = {r0 < len, r1 < len};
        float rdg[2] = {0.f, 0.f}, rdb[2] = {0.f, 0.f}, cdg[2 * kJJ] = {}, sdg = 0.f;
        const int cc0 = (64 / kWN) * wn, ck0 = (128 / kWN) * wn;  // this warp's first column (C x C, C x K)
        ok = wait_bar(kBarMma);
        tc_fence_after();
        if (ok && tid == 0 && nxt.valid) load_a(nxt);  // Ainv and dDelta are consumed
        ok = ok && wait_bar(kBarV);
        if (len < C) {
            zero_rows(sb + kVt, len, tid);  // as for q, k and dO
            __syncthreads();
        }

        float sacc[kJJ][4], gacc[kJJ][4];  // S -> strictly lower E, G: kept for product batch 2
        if (ok) {
            float v[16], pacc[kJJ][4];
            {
                float c[4 * kJJ];
                ld_cc(tmem + lane_base + kCS + cc0, c);
#pragma unroll
                for (int i = 0; i < 4 * kJJ; ++i) sacc[i >> 2][i & 3] = c[i];
                ld_cc(tmem + lane_base + kCG + cc0, c);
#pragma unroll
                for (int i = 0; i < 4 * kJJ; ++i) gacc[i >> 2][i & 3] = c[i];
                ld_cc(tmem + lane_base + kCP1 + cc0, c);
#pragma unroll
                for (int i = 0; i < 4 * kJJ; ++i) pacc[i >> 2][i & 3] = c[i];
            }
            // T1 = scale M o P1, Z = T1 o S (row and column sums)
#pragma unroll
            for (int jj = 0; jj < kJJ; ++jj)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int hi = q >> 1, s = cc0 + 8 * jj + 2 * c4 + (q & 1), r = hi ? r1 : r0;
                    const bool on = lr[hi] && s <= r;  // s < len follows
                    const float E = on ? __expf(gr[hi] - vec.gam[s]) : 0.f;
                    const float t1 = scale * E * pacc[jj][q];
                    const float z = t1 * sacc[jj][q];
                    rdg[hi] += z;
                    cdg[2 * jj + (q & 1)] -= z;
                    pacc[jj][q] = t1;
                    sacc[jj][q] = s < r ? E : 0.f;  // strictly lower part of E for the A terms
                }
#pragma unroll
            for (int jj = 0; jj < kJJ; ++jj) {
                const int s = cc0 + 8 * jj + 2 * c4;
                st_shared_b32(sb + kT1 + sw_off(r0, s, 8192), pack_bf16(pacc[jj][0], pacc[jj][1]));
                st_shared_b32(sb + kT1 + sw_off(r1, s, 8192), pack_bf16(pacc[jj][2], pacc[jj][3]));
            }
            // dU: dv = beta dU (in place of v for a full chunk), dbeta += dU.v, dU -> shared memory
#pragma unroll
            for (int part = 0; part < kParts; ++part) {
                const int cb = ck0 + 32 * part;
                tmem_ld16x256_x4(tmem + lane_base + kCU + cb, v);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int col = cb + 8 * i + 2 * c4;
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi) {
                        const int r = hi ? r1 : r0;
                        const float u0 = v[4 * i + 2 * hi], u1 = v[4 * i + 2 * hi + 1];
                        const float2 vv = ld_pair_sw(sb + kVt, r, col);
                        rdb[hi] += u0 * vv.x + u1 * vv.y;
                        const uint32_t dvp = pack_bf16(br[hi] * u0, br[hi] * u1);
                        if (full)
                            st_shared_b32(sb + kVt + sw_off(r, col, 8192), dvp);
                        else if (lr[hi])
                            *reinterpret_cast<uint32_t *>(prm.dv + ((size_t)(t0 + r) * d.Hv + h) * V + col) = dvp;
                        st_shared_b32(sb + kdU + sw_off(r, col, 8192), pack_bf16(u0, u1));
                    }
                }
            }
        }
        fence_proxy_async();  // T1, dU -> the tensor core; dv -> the TMA store
        tc_fence_before();
        ok = __syncthreads_and(ok);
        if (!ok) break;
        if (tid == kStoreTid && full) {
            tma_store_3d(&tm.dv, sb + kVt, 0, h, t0);
            tma_store_3d(&tm.dv, sb + kVt + 8192, 64, h, t0);
            bulk_commit();
        }
        ok = wait_bar(kBarSt);

        // ---- product batch 2: dAkk (64 x 64), T1 K, T1^T Q onto dk, dO h^T (64 x 128)
        if (ok && tid == 0) {
            tc_fence_after();
            const uint32_t idCC = idesc_bf16(64, 64, false, false), idKM = idesc_bf16(64, 128, false, true);
            const uint64_t du = kbase(sb + kdU), dl = bbase(sD, 1024), t1 = kbase(sb + kT1), km = mbase(sb + kKt);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) mma_bf16(tmem + kCAkk, du + kstep(ks, 8192), dl + bstep(ks, 1024), idCC, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) mma_bf16(tmem + kCTK, t1 + kstep(ks, 8192), km + mstep(ks), idKM, ks > 0);
            commit_mma();
        } else if (ok && tid == kStoreTid) {
            tc_fence_after();
            const uint32_t idMM = idesc_bf16(64, 128, true, true), idKK = idesc_bf16(64, 128, false, false);
            const uint64_t o = kbase(sb + kdO), hh = bbase(sb + kH, 2048), t1m = mbase(sb + kT1), qm = mbase(sb + kQ);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) mma_bf16(tmem + kCQ1, o + kstep(ks, 8192), hh + bstep(ks, 2048), idKK, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) mma_bf16(tmem + kCDK, t1m + mstep(ks), qm + mstep(ks), idMM, ks > 0 || !first);
            commit_mma();
            if (nxt.valid) {
                bulk_wait_read<0>();  // dv has left the v tile
                load_v(nxt);
            }
        }
        ok = ok && wait_bar(kBarMma);
        tc_fence_after();
        if (ok && tid == 0 && nxt.valid) load_do(nxt);  // dO is consumed
        if (ok) {
            // dAkk = -dU Delta^T (s < r): dbeta, Zr, dG -> shared memory
            float v[4 * kJJ];
            ld_cc(tmem + lane_base + kCAkk + cc0, v);
#pragma unroll
            for (int jj = 0; jj < kJJ; ++jj) {
                float dgv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int hi = q >> 1;
                    const float E = sacc[jj][q];  // zero unless s < r < len
                    const float dA = -v[4 * jj + q];
                    const float eg = E * gacc[jj][q];
                    rdb[hi] += dA * eg;
                    const float zr = br[hi] * dA * eg;
                    rdg[hi] += zr;
                    cdg[2 * jj + (q & 1)] -= zr;
                    dgv[q] = dA * br[hi] * E;
                }
                const int s = cc0 + 8 * jj + 2 * c4;
                st_shared_b32(sb + kdG + sw_off(r0, s, 8192), pack_bf16(dgv[0], dgv[1]));
                st_shared_b32(sb + kdG + sw_off(r1, s, 8192), pack_bf16(dgv[2], dgv[3]));
            }
            // dq = scale diag(e^gamma) dO h^T + T1 K (+ the group's earlier heads);
            // dgamma += scale e^gamma q.(dO h^T)
            // (16 columns at a time: three 16-value blocks live at once would spill at the
            // 128-register cap of sixteen warps)
#pragma unroll
            for (int part = 0; part < 2 * kParts; ++part) {
                const int cb = ck0 + 16 * part;
                float a[8], b[8], x[8];
                tmem_ld16x256_x2(tmem + lane_base + kCQ1 + cb, a);
                tmem_ld16x256_x2(tmem + lane_base + kCTK + cb, b);
                if (!first) tmem_ld16x256_x2(park + 16 * part, x);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int col = cb + 8 * i + 2 * c4;
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi) {
                        const int r = hi ? r1 : r0, e = 4 * i + 2 * hi;
                        const float2 qq = ld_pair_sw(sb + kQ, r, col);
                        const float f = scale * er[hi];
                        rdg[hi] += f * (a[e] * qq.x + a[e + 1] * qq.y);
                        const float y0 = fmaf(f, a[e], b[e]), y1 = fmaf(f, a[e + 1], b[e + 1]);
                        x[e] = first ? y0 : x[e] + y0;
                        x[e + 1] = first ? y1 : x[e + 1] + y1;
                        if (last) {
                            const uint32_t dqp = pack_bf16(x[e], x[e + 1]);
                            if (full)
                                st_shared_b32(sb + kQ + sw_off(r, col, 8192), dqp);
                            else if (lr[hi])
                                *reinterpret_cast<uint32_t *>(prm.dq + ((size_t)(t0 + r) * d.Hq + cur.hq) * K + col) = dqp;
                        }
                    }
                }
                if (!last) tmem_st16x256_x2(park + 16 * part, x);
            }
        }
        fence_proxy_async();  // dG -> the tensor core; dq -> the TMA store
        tc_fence_before();
        ok = __syncthreads_and(ok);
        if (!ok) break;

        // ---- product batch 3: dU h^T, Delta dh'^T; dG K + dG^T K onto dk
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idKK = idesc_bf16(64, 128, false, false);
            const uint64_t du = kbase(sb + kdU), hh = bbase(sb + kH, 2048), dl = bbase(sD, 1024), dh = bbase(sb + kdH, 2048);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                mma_bf16(tmem + kCKb, du + kstep(ks, 8192), hh + bstep(ks, 2048), idKK, ks > 0);
                mma_bf16(tmem + kCK2, dl + bstep(ks, 1024), dh + bstep(ks, 2048), idKK, ks > 0);
            }
            commit_mma();
        } else if (tid == kStoreTid) {
            tc_fence_after();
            const uint32_t idKM = idesc_bf16(64, 128, false, true), idMM = idesc_bf16(64, 128, true, true);
            const uint64_t dg = kbase(sb + kdG), dgm = mbase(sb + kdG), km = mbase(sb + kKt);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(tmem + kCDK, dg + kstep(ks, 8192), km + mstep(ks), idKM, true);
                mma_bf16(tmem + kCDK, dgm + mstep(ks), km + mstep(ks), idMM, true);
            }
            commit_mma();
        }
        if (tid == kStoreTid && last) {
            if (full) {
                tma_store_3d(&tm.dq, sb + kQ, 0, cur.hq, t0);
                tma_store_3d(&tm.dq, sb + kQ + 8192, 64, cur.hq, t0);
                bulk_commit();
            }
            if (nxt.valid) {
                bulk_wait_read<0>();  // dq has left the q tile
                load_q(nxt);
            }
        }
        // e^{gamma_C} <dh', h> while the products run: this thread's share of the
        // 128 x 128 dot (same layout in both tiles)
        {
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
        ok = wait_bar(kBarMma);
        tc_fence_after();
        ok = __syncthreads_and(ok);  // h and dh' are consumed
        if (!ok) break;
        if (tid == 0 && nxt.valid) load_st(nxt);
        float dotb[2] = {0.f, 0.f}, z3[2] = {0.f, 0.f};  // per row, summed over both column halves
#pragma unroll
        for (int part = 0; part < 2 * kParts; ++part) {  // 16 columns at a time, as above
            const int cb = ck0 + 16 * part;
            float kb[8], k2[8], x[8];
            tmem_ld16x256_x2(tmem + lane_base + kCKb + cb, kb);  // dU h^T = -dKb
            tmem_ld16x256_x2(tmem + lane_base + kCK2 + cb, k2);  // Delta dh'^T
            tmem_ld16x256_x2(tmem + lane_base + kCDK + cb, x);   // dk so far + T1^T Q + dG K + dG^T K
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = hi ? r1 : r0;
                const float fk = br[hi] * er[hi];                     // dk += beta e^gamma dKb
                const float f2 = lr[hi] ? __expf(gC - gr[hi]) : 0.f;  // dk += e^{gamma_C - gamma} (Delta dh'^T)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int col = cb + 8 * i + 2 * c4, e = 4 * i + 2 * hi;
                    const float2 kk = ld_pair_sw(sb + kKt, r, col);
                    const float b0 = -kb[e], b1 = -kb[e + 1];
                    const float e0 = k2[e], e1 = k2[e + 1];
                    dotb[hi] += b0 * kk.x + b1 * kk.y;
                    z3[hi] += e0 * kk.x + e1 * kk.y;
                    x[e] += fk * b0 + f2 * e0;
                    x[e + 1] += fk * b1 + f2 * e1;
                    if (last) {
                        const uint32_t dkp = pack_bf16(x[e], x[e + 1]);
                        if (full)
                            st_shared_b32(sb + kT1 + sw_off(r, col, 8192), dkp);
                        else if (lr[hi])
                            *reinterpret_cast<uint32_t *>(prm.dk + ((size_t)(t0 + r) * d.Hq + cur.hq) * K + col) = dkp;
                    }
                }
            }
            if (!last) tmem_st16x256_x2(tmem + lane_base + kCDK + cb, x);
        }
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const float f2 = lr[hi] ? __expf(gC - gr[hi]) : 0.f;
            rdb[hi] += er[hi] * dotb[hi];
            rdg[hi] += br[hi] * er[hi] * dotb[hi];
            const float z = z3[hi] * f2;
            rdg[hi] -= z;
            sdg += z;
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
        for (int i = 0; i < 2 * kJJ; ++i) {
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
            for (int jj = 0; jj < kJJ; ++jj) {
                vec.coldg[wm][cc0 + 8 * jj + 2 * c4] = cdg[2 * jj];
                vec.coldg[wm][cc0 + 8 * jj + 2 * c4 + 1] = cdg[2 * jj + 1];
            }
        }
        if (lane == 0) vec.scal[warp] = sdg;
        fence_proxy_async();  // dk -> the TMA store
        tc_fence_before();
        __syncthreads();  // also: the k tile is consumed
        if (tid == kStoreTid && last) {
            if (full) {
                tma_store_3d(&tm.dk, sb + kT1, 0, cur.hq, t0);
                tma_store_3d(&tm.dk, sb + kdG, 64, cur.hq, t0);
                bulk_commit();
            }
            if (nxt.valid) load_k(nxt);
        }
        if (warp == 0) {
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
        cur = nxt;
    }
    if (!ok && (tid == 0 || tid == kStoreTid)) {
        if (tid == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
        // loads and products this thread issued that are still in flight: let them finish (bounded)
        const uint64_t t1 = globaltimer();
        for (int b = 0; b < kNumBar; ++b)
            if (pend & (1u << b))
                while (!mbar_try_wait(smem_u32(&bars[b]), (phase >> b) & 1) && globaltimer() - t1 < kWaitNs) {
                }
    }
    if (tid == kStoreTid) bulk_wait_all();  // stores read shared memory until they complete
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_bwd_grad_tc(const BwdArgs &a, const void *h_chunks16, const void *dh_chunks16,
                               const void *delta16, const void *ddelta16) {
    const Dims &d = a.d;
    if (d.NC == 0) return cudaSuccess;
    GradMaps m;
    const cuuint64_t T = (cuuint64_t)(d.T_total > 0 ? d.T_total : 1);
    const cuuint64_t dqk[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hq, T};
    const cuuint64_t sqk[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hq * d.K * 2};
    const cuuint64_t dvv[3] = {(cuuint64_t)d.V, (cuuint64_t)d.Hv, T};
    const cuuint64_t svv[2] = {(cuuint64_t)d.V * 2, (cuuint64_t)d.Hv * d.V * 2};
    const cuuint32_t b3[3] = {64, 1, 64};
    const cuuint64_t dai[2] = {64, (cuuint64_t)d.NC * d.Hv * 64};
    const cuuint64_t sai[1] = {128};
    const cuuint32_t bai[2] = {64, 64};
    const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_bf16_map(&m.q, a.q, 3, dqk, sqk, b3, SW) || !make_bf16_map(&m.k, a.k, 3, dqk, sqk, b3, SW) ||
        !make_bf16_map(&m.v, a.v, 3, dvv, svv, b3, SW) || !make_bf16_map(&m.d_o, a.d_o, 3, dvv, svv, b3, SW) ||

        !make_bf16_map(&m.ainv, a.ainv, 2, dai, sai, bai, SW) ||
        !make_bf16_map(&m.dq, a.dq, 3, dqk, sqk, b3, SW) || !make_bf16_map(&m.dk, a.dk, 3, dqk, sqk, b3, SW) ||
        !make_bf16_map(&m.dv, a.dv, 3, dvv, svv, b3, SW))
        return cudaErrorInvalidValue;
    GradParams p;
    p.d = d;
    p.delta = (const __nv_bfloat16 *)delta16;
    p.ddelta = (const __nv_bfloat16 *)ddelta16;
    p.h = (const __nv_bfloat16 *)h_chunks16;
    p.dh = (const __nv_bfloat16 *)dh_chunks16;
    p.gamma = a.gamma;
    p.beta = a.beta;
    p.dq = (__nv_bfloat16 *)a.dq;
    p.dk = (__nv_bfloat16 *)a.dk;
    p.dv = (__nv_bfloat16 *)a.dv;
    p.dg = a.dg;
    p.dbeta = a.dbeta;
    p.n_items = d.NC * d.Hq;
    p.status = a.status;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes)) != cudaSuccess)
        return e;
    const int grid = p.n_items < sms ? p.n_items : sms;  // persistent: one CTA per SM
    bwd_grad_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(m, p);
    return cudaGetLastError();
}

}  // namespace gdn
