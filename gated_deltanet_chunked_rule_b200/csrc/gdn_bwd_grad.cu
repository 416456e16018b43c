// gdn_bwd_grad.cu -- per-chunk gradients of the chunked backward (bf16,
// K = V = 128), on warp-level tensor-core MMAs. Fully parallel: one CTA per
// (chunk, value head).
//
// Per chunk (rows r, s; h the entry state, Delta, from the recompute; dh' and
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
// dq and dk go to per-value-head fp32 partials (summed over the GQA group by
// bwd_final); dv, dg, dbeta are written directly. All row and column sums are
// taken in a fixed order (the result does not depend on scheduling).
#include "gdn_internal.cuh"
#include "gdn_warp.cuh"

namespace gdn {
namespace {

using namespace warp;

// 8 warps: warp w owns rows 16 (w % 4) .. +15 of every product and column
// group w / 4 (32 columns of the 64 x 64 products, 64 of the 64 x 128 ones).
// (More warps re-read the same operand fragments; the kernel is bound by
// shared-memory load bandwidth, measured slower with 16.)
constexpr int kThreads = 256;
constexpr int kWN = 2;                       // column groups
constexpr int NT_CC = 64 / (8 * kWN);        // n-tiles per warp, 64 x 64 products
constexpr int NT_CK = 128 / (8 * kWN);       // n-tiles per warp, 64 x 128 products
constexpr int C = 64, K = 128, V = 128;

// ---- shared memory (bytes)
constexpr int kSQ = 0, kSK = 16384, kSV = 32768 /* later dU */, kSdO = 49152, kSD = 65536, kSdD = 81920;
constexpr int kSh = 98304, kSdh = 131072, kSA = 163840, kST1 = 172032, kSdG = 180224, kSvec = 188416;
constexpr int kSmemBytes = kSvec + 4096;

struct Vecs {
    float gam[64], egam[64], bet[64];
    float rowdg[kWN][64], rowdb[kWN][64];  // per column-group partial row sums
    float coldg[4][64];                    // per row-quarter partial column sums
    float scal[kThreads / 32];             // per-warp partial of the chunk-level dgamma_C term
};
static_assert(sizeof(Vecs) <= 4096, "vector area");

struct GradParams {
    Dims d;
    const __nv_bfloat16 *q, *k, *v, *d_o;
    const float *gamma, *beta;
    const __nv_bfloat16 *ainv;       // [NC, Hv, 64, 64]
    const __nv_bfloat16 *h_chunks;   // [NC, Hv, K, V] entry states
    const __nv_bfloat16 *dh_chunks;  // [NC, Hv, K, V] exit-state gradients
    const __nv_bfloat16 *delta;      // [T, Hv, V]
    const __nv_bfloat16 *ddelta;     // [T, Hv, V]
    float *dq_part, *dk_part;        // [T, Hv, K]
    __nv_bfloat16 *dv;               // [T, Hv, V]
    float *dg, *dbeta;               // [T, Hv]
};

__global__ void __launch_bounds__(kThreads, 1) bwd_grad_kernel(const GradParams prm) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sb = smem_u32(smem);
    Vecs &vec = *reinterpret_cast<Vecs *>(smem + kSvec);
    const Dims &d = prm.d;
    const int cg = blockIdx.x, h = blockIdx.y;
    const int hq = h / (d.Hv / d.Hq);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wm = warp & 3, wn = warp >> 2;
    const int g = lane >> 2, c4 = lane & 3;
    const int r0 = 16 * wm + g, r1 = r0 + 8;  // rows this thread holds in every accumulator
    const int n = chunk_owner(d, cg);
    if (n < 0) return;  // whole CTA
    const SeqRange sr = seq_range(d, n);
    const int ci = cg - sr.chunk0;
    const int t0 = sr.start + ci * C, len = min(C, sr.len - ci * C);
    const float scale = d.scale;

    const Tile tQ{sb + kSQ, 256}, tK{sb + kSK, 256}, tV{sb + kSV, 256}, tdO{sb + kSdO, 256};
    const Tile tD{sb + kSD, 256}, tdD{sb + kSdD, 256}, th{sb + kSh, 256}, tdh{sb + kSdh, 256};
    const Tile tA{sb + kSA, 128}, tT1{sb + kST1, 128}, tdG{sb + kSdG, 128};

    // ---- loads (cp.async; rows past the chunk's end are zero). Two groups: the
    //      chunk tiles for phases A-C, then the two states, which land while A-C run.
    const size_t hbase = ((size_t)cg * d.Hv + h) * K * V;
    load_tile<kThreads>(tQ, prm.q + ((size_t)t0 * d.Hq + hq) * K, (size_t)d.Hq * K, C, K, len, tid);
    load_tile<kThreads>(tK, prm.k + ((size_t)t0 * d.Hq + hq) * K, (size_t)d.Hq * K, C, K, len, tid);
    load_tile<kThreads>(tdO, prm.d_o + ((size_t)t0 * d.Hv + h) * V, (size_t)d.Hv * V, C, V, len, tid);
    load_tile<kThreads>(tD, prm.delta + ((size_t)t0 * d.Hv + h) * V, (size_t)d.Hv * V, C, V, len, tid);
    load_tile<kThreads>(tdD, prm.ddelta + ((size_t)t0 * d.Hv + h) * V, (size_t)d.Hv * V, C, V, len, tid);
    load_tile<kThreads>(tA, prm.ainv + ((size_t)cg * d.Hv + h) * C * C, C, C, C, C, tid);
    load_tile<kThreads>(tV, prm.v + ((size_t)t0 * d.Hv + h) * V, (size_t)d.Hv * V, C, V, len, tid);
    cp_async_commit();
    load_tile<kThreads>(th, prm.h_chunks + hbase, V, K, V, K, tid);
    load_tile<kThreads>(tdh, prm.dh_chunks + hbase, V, K, V, K, tid);
    cp_async_commit();
    if (tid < C) {
        const int r = tid, rr = min(r, len - 1);
        const float gm = prm.gamma[(size_t)(t0 + rr) * d.Hv + h];
        vec.gam[r] = gm;
        vec.egam[r] = __expf(gm);
        vec.bet[r] = r < len ? prm.beta[(size_t)(t0 + r) * d.Hv + h] : 0.f;
    }
    cp_async_wait_older();
    __syncthreads();

    const float gC = vec.gam[63];  // gamma at the chunk's last token (padded rows repeat it)
    const float gr[2] = {vec.gam[r0], vec.gam[r1]};
    const float er[2] = {vec.egam[r0], vec.egam[r1]};
    const float br[2] = {vec.bet[r0], vec.bet[r1]};
    const bool lr[2] = {r0 < len, r1 < len};
    float rdg[2] = {0.f, 0.f}, rdb[2] = {0.f, 0.f}, cdg[2 * NT_CC] = {}, sdg = 0.f;
    const int cc0 = 8 * NT_CC * wn, ck0 = 8 * NT_CK * wn;  // this warp's first column (C x C, C x K)

    // ---- phase A: S = Q K^T, G = K K^T, P1 = dO Delta^T
    float sacc[NT_CC][4] = {}, gacc[NT_CC][4] = {};
    {
        float pacc[NT_CC][4] = {};
        wgemm<NT_CC, false, false>(sacc, tQ, tK, 16 * wm, cc0, K, lane);
        wgemm<NT_CC, false, false>(gacc, tK, tK, 16 * wm, cc0, K, lane);
        wgemm<NT_CC, false, false>(pacc, tdO, tD, 16 * wm, cc0, V, lane);
#pragma unroll
        for (int j = 0; j < NT_CC; ++j)
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
        // T1 -> shared memory (bf16)
#pragma unroll
        for (int j = 0; j < NT_CC; ++j) {
            const int s = cc0 + 8 * j + 2 * c4;
            st_shared_b32(toff(tT1, r0, s), pack_bf16(pacc[j][0], pacc[j][1]));
            st_shared_b32(toff(tT1, r1, s), pack_bf16(pacc[j][2], pacc[j][3]));
        }
    }

    // ---- phase B: dU = Ainv^T dDelta; dv, dbeta (dU.v); dU -> (V's space)
    {
        float uacc[NT_CK][4] = {};
        wgemm<NT_CK, true, true>(uacc, tA, tdD, 16 * wm, ck0, C, lane);
#pragma unroll
        for (int j = 0; j < NT_CK; ++j) {
            const int col = ck0 + 8 * j + 2 * c4;
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = hi ? r1 : r0;
                const float2 vv = ld_pair(tV, r, col);
                rdb[hi] += uacc[j][2 * hi] * vv.x + uacc[j][2 * hi + 1] * vv.y;
                if (lr[hi])
                    *reinterpret_cast<uint32_t *>(prm.dv + ((size_t)(t0 + r) * d.Hv + h) * V + col) =
                        pack_bf16(br[hi] * uacc[j][2 * hi], br[hi] * uacc[j][2 * hi + 1]);
            }
        }
        __syncthreads();  // every warp is done reading v
#pragma unroll
        for (int j = 0; j < NT_CK; ++j) {
            const int col = ck0 + 8 * j + 2 * c4;
            st_shared_b32(toff(tV, r0, col), pack_bf16(uacc[j][0], uacc[j][1]));
            st_shared_b32(toff(tV, r1, col), pack_bf16(uacc[j][2], uacc[j][3]));
        }
    }
    __syncthreads();  // dU and T1 visible to all warps
    const Tile &tU = tV;

    // ---- phase C: dAkk = -dU Delta^T (s < r); dbeta, Zr, dG
    {
        float aacc[NT_CC][4] = {};
        wgemm<NT_CC, false, false>(aacc, tU, tD, 16 * wm, cc0, V, lane);
#pragma unroll
        for (int j = 0; j < NT_CC; ++j) {
            float dgv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int hi = q >> 1;
                const float E = sacc[j][q];  // zero unless s < r < len
                const float dA = -aacc[j][q];
                const float eg = E * gacc[j][q];
                rdb[hi] += dA * eg;
                const float zr = br[hi] * dA * eg;
                rdg[hi] += zr;
                cdg[2 * j + (q & 1)] -= zr;
                dgv[q] = dA * br[hi] * E;
            }
            const int s = cc0 + 8 * j + 2 * c4;
            st_shared_b32(toff(tdG, r0, s), pack_bf16(dgv[0], dgv[1]));
            st_shared_b32(toff(tdG, r1, s), pack_bf16(dgv[2], dgv[3]));
        }
    }
    cp_async_wait_all();  // the two states
    __syncthreads();      // dG and the states visible

    // ---- phase D: dq = scale diag(e^gamma) dO h^T + T1 K
    {
        float acc[NT_CK][4] = {};
        wgemm<NT_CK, false, false>(acc, tdO, th, 16 * wm, ck0, V, lane);
#pragma unroll
        for (int j = 0; j < NT_CK; ++j) {
            const int col = ck0 + 8 * j + 2 * c4;
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const float2 qq = ld_pair(tQ, hi ? r1 : r0, col);
                const float f = scale * er[hi];
                rdg[hi] += f * (acc[j][2 * hi] * qq.x + acc[j][2 * hi + 1] * qq.y);
                acc[j][2 * hi] *= f;
                acc[j][2 * hi + 1] *= f;
            }
        }
        wgemm<NT_CK, false, true>(acc, tT1, tK, 16 * wm, ck0, C, lane);
#pragma unroll
        for (int j = 0; j < NT_CK; ++j) {
            const int col = ck0 + 8 * j + 2 * c4;
#pragma unroll
            for (int hi = 0; hi < 2; ++hi)
                if (lr[hi])
                    *reinterpret_cast<float2 *>(prm.dq_part + ((size_t)(t0 + (hi ? r1 : r0)) * d.Hv + h) * K + col) =
                        make_float2(acc[j][2 * hi], acc[j][2 * hi + 1]);
        }
    }

    // ---- phase E: dk
    {
        float kacc[NT_CK][4], tacc[NT_CK][4] = {};
        // -dU h^T = dKb: dk += beta e^gamma dKb; dbeta += e^gamma dKb.k; dgamma += beta e^gamma dKb.k
        wgemm<NT_CK, false, false>(tacc, tU, th, 16 * wm, ck0, V, lane);
#pragma unroll
        for (int j = 0; j < NT_CK; ++j) {
            const int col = ck0 + 8 * j + 2 * c4;
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const float2 kk = ld_pair(tK, hi ? r1 : r0, col);
                const float x0 = -tacc[j][2 * hi], x1 = -tacc[j][2 * hi + 1];
                const float dot = x0 * kk.x + x1 * kk.y;
                rdb[hi] += er[hi] * dot;
                rdg[hi] += br[hi] * er[hi] * dot;
                const float f = br[hi] * er[hi];
                kacc[j][2 * hi] = f * x0;
                kacc[j][2 * hi + 1] = f * x1;
                tacc[j][2 * hi] = tacc[j][2 * hi + 1] = 0.f;
            }
        }
        // Delta dh'^T: dk += e^{gamma_C - gamma} (.); Z3
        wgemm<NT_CK, false, false>(tacc, tD, tdh, 16 * wm, ck0, V, lane);
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int r = hi ? r1 : r0;
            const float f = lr[hi] ? __expf(gC - gr[hi]) : 0.f;
            float z3 = 0.f;
#pragma unroll
            for (int j = 0; j < NT_CK; ++j) {
                const int col = ck0 + 8 * j + 2 * c4;
                const float2 kk = ld_pair(tK, r, col);
                z3 += tacc[j][2 * hi] * kk.x + tacc[j][2 * hi + 1] * kk.y;
                kacc[j][2 * hi] += f * tacc[j][2 * hi];
                kacc[j][2 * hi + 1] += f * tacc[j][2 * hi + 1];
            }
            z3 *= f;
            rdg[hi] -= z3;
            sdg += z3;
        }
        wgemm<NT_CK, true, true>(kacc, tT1, tQ, 16 * wm, ck0, C, lane);   // T1^T Q
        wgemm<NT_CK, false, true>(kacc, tdG, tK, 16 * wm, ck0, C, lane);  // dG K
        wgemm<NT_CK, true, true>(kacc, tdG, tK, 16 * wm, ck0, C, lane);   // dG^T K
#pragma unroll
        for (int j = 0; j < NT_CK; ++j) {
            const int col = ck0 + 8 * j + 2 * c4;
#pragma unroll
            for (int hi = 0; hi < 2; ++hi)
                if (lr[hi])
                    *reinterpret_cast<float2 *>(prm.dk_part + ((size_t)(t0 + (hi ? r1 : r0)) * d.Hv + h) * K + col) =
                        make_float2(kacc[j][2 * hi], kacc[j][2 * hi + 1]);
        }
    }

    // ---- e^{gamma_C} <dh', h>: this thread's share of the 128 x 128 dot (same layout in both tiles)
    {
        float s = 0.f;
        for (int e = tid; e < K * V / 8; e += kThreads) {
            const uint4 a = ld_shared_v4(sb + kSh + e * 16), b = ld_shared_v4(sb + kSdh + e * 16);
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
    for (int i = 0; i < 2 * NT_CC; ++i) {
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
        for (int j = 0; j < NT_CC; ++j) {
            vec.coldg[wm][cc0 + 8 * j + 2 * c4] = cdg[2 * j];
            vec.coldg[wm][cc0 + 8 * j + 2 * c4 + 1] = cdg[2 * j + 1];
        }
    }
    if (lane == 0) vec.scal[warp] = sdg;
    __syncthreads();
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
        float hi_tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float x = __shfl_down_sync(0xffffffffu, dgr[1], o);
            if (lane + o < 32) dgr[1] += x;
        }
        hi_tot = __shfl_sync(0xffffffffu, dgr[1], 0);  // sum of the upper half
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
}

}  // namespace

cudaError_t launch_bwd_grad_tc(const BwdArgs &a, const void *h_chunks16, const void *dh_chunks16,
                               const void *delta16, const void *ddelta16, float *dq_part, float *dk_part) {
    const Dims &d = a.d;
    if (d.NC == 0) return cudaSuccess;
    GradParams p;
    p.d = d;
    p.q = (const __nv_bfloat16 *)a.q;
    p.k = (const __nv_bfloat16 *)a.k;
    p.v = (const __nv_bfloat16 *)a.v;
    p.d_o = (const __nv_bfloat16 *)a.d_o;
    p.gamma = a.gamma;
    p.beta = a.beta;
    p.ainv = (const __nv_bfloat16 *)a.ainv;
    p.h_chunks = (const __nv_bfloat16 *)h_chunks16;
    p.dh_chunks = (const __nv_bfloat16 *)dh_chunks16;
    p.delta = (const __nv_bfloat16 *)delta16;
    p.ddelta = (const __nv_bfloat16 *)ddelta16;
    p.dq_part = dq_part;
    p.dk_part = dk_part;
    p.dv = (__nv_bfloat16 *)a.dv;
    p.dg = a.dg;
    p.dbeta = a.dbeta;
    cudaError_t e = cudaFuncSetAttribute(bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    bwd_grad_kernel<<<dim3(d.NC, d.Hv), kThreads, kSmemBytes, a.stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
