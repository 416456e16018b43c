// gdn_tc_fwd.cu -- tensor-core (tcgen05 / TMEM / TMA) chunked forward, bf16 inputs.
//
// One CTA per (sequence, value head, 32-column slice of V) walks the 64-token
// chunks of its sequence in order. The fp32 state slice h[:, slice] (128 x 32)
// lives in registers, one row per thread; every contraction of a chunk runs on
// the tensor cores from shared memory into tensor memory (fp32 accumulate):
//
//   phase A (does not need h):   S = Q K^T,   W = (Ainv diag(beta e^gamma)) K,
//                                DW = (Ainv diag(beta)) V            (= u)
//   phase B (needs h):           DW += (-w) h  (-> Delta),   DQ = Q h
//   phase C (needs Delta):       D2 = K^T diag(e^{gamma_C - gamma}) Delta,  DP = P Delta
//   then   h <- e^{gamma_C} h + D2,   o = scale (e^gamma o DQ + DP)
//
// with P = M o (Q K^T) the causal decay-masked score (CUDA cores: exp and
// mask). Ainv = (I + A)^-1 comes from the chunk-prep kernel (bf16). The
// q, k, v and Ainv tiles of each chunk arrive by TMA into a 3-deep ring.
// Padded rows of a ragged last chunk need no masking: their beta is 0, so
// their Ainv row is e_r and their columns of diag(beta) Ainv vanish, which
// makes their rows of u, w and Delta exactly zero.
//
// Tensor-memory lane layout: an M=64 accumulator puts row r in lane
// (r % 16) + 32 * (r / 16), so thread l < 16 of warp w owns row 16 w + l of
// every M=64 result (S, W, DW, DQ, DP); an M=128 result puts row j in lane j.
#include <cudaTypedefs.h>

#include "gdn_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kThreads = 128;
constexpr int kBV = 32;
constexpr int kStages = 3;

// Shared-memory carve-up (bytes, relative to a 1024-aligned base).
constexpr int kHb = 0;                      // h in bf16, MN-major no swizzle, 128 x 32
constexpr int kDb = kHb + 8192;             // Delta, MN-major no swizzle, 64 x 32
constexpr int kDt = kDb + 4096;             // e^{gamma_C - gamma} Delta
constexpr int kAw = kDt + 4096;             // Ainv diag(beta e^gamma), 64x64 K-major SW128
constexpr int kWn = kAw + 8192;             // -w, 64x128 K-major SW128
constexpr int kP = kWn + 16384;             // P, 64x64 K-major SW128
constexpr int kStage0 = kP + 8192;          // TMA ring
constexpr int kQ = 0, kK = 16384, kAi = 32768, kVt = 40960;  // inside a stage
constexpr int kStageBytes = 45056;
constexpr int kTxBytes = 16384 + 16384 + 8192 + 4096;
constexpr int kSmall = kStage0 + kStages * kStageBytes;
constexpr int kSmemBytes = kSmall + 1024 + 1024;  // + small arrays + alignment slack
static_assert(sizeof(int) * 0 + kSmemBytes <= 232448, "shared memory budget");

// Tensor-memory columns.
constexpr uint32_t kColS = 0, kColW = 64, kColDW = 192, kColDQ = 224, kColDP = 256, kColD2 = 288;
constexpr uint32_t kTmemCols = 512;

struct Small {
    uint64_t full[kStages];
    uint64_t bar[3];
    uint32_t tmem_base;
    int abort_flag;
    float gam[64];
    float bet[64];
    float egam[64];
};

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait measured in wall-clock time (2 s).
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait(a, parity)) return true;
        if ((i & 1023u) == 0) {
            const uint64_t t = globaltimer();
            if (i == 0) t0 = t;
            else if (t - t0 > 2000000000ull) return false;
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

struct TcParams {
    Dims d;
    const float *gamma;       // [T_total, Hv]
    const float *beta;        // [T_total, Hv]
    const float *h0;          // [N, Hv, K, V] or null
    __nv_bfloat16 *o;         // [T_total, Hv, V]
    float *final_state;       // [N, Hv, K, V] or null
    unsigned *status;
};

__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
              const TcParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    Small *sm = reinterpret_cast<Small *>(smem + kSmall);
    const uint32_t sbase = smem_u32(smem);

    const Dims &d = prm.d;
    const int n = blockIdx.x, h = blockIdx.y, c0 = blockIdx.z * kBV;
    const int hq = h / (d.Hv / d.Hq);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const SeqRange sr = seq_range(d, n);
    const int nchunks = (sr.len + kChunk - 1) / kChunk;
    constexpr int K = 128, V = 128;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&sm->full[s], 1);
        for (int b = 0; b < 3; ++b) mbar_init(&sm->bar[b], 1);
        sm->abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_a);
    }
    if (warp == 0) {
        tmem_alloc(&sm->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

    auto issue_loads = [&](int ci) {
        const int s = ci % kStages;
        uint8_t *st = smem + kStage0 + s * kStageBytes;
        const int t0 = sr.start + ci * kChunk;
        const int cg = sr.chunk0 + ci;
        mbar_arrive_expect_tx(&sm->full[s], kTxBytes);
        tma_load_3d(st + kQ, &tm_q, &sm->full[s], 0, hq, t0);
        tma_load_3d(st + kQ + 8192, &tm_q, &sm->full[s], 64, hq, t0);
        tma_load_3d(st + kK, &tm_k, &sm->full[s], 0, hq, t0);
        tma_load_3d(st + kK + 8192, &tm_k, &sm->full[s], 64, hq, t0);
        tma_load_2d(st + kAi, &tm_a, &sm->full[s], 0, (cg * d.Hv + h) * kChunk);
        tma_load_3d(st + kVt, &tm_v, &sm->full[s], c0, h, t0);
    };
    int issued = 0;
    if (tid == 0)
        for (; issued < kStages && issued < nchunks; ++issued) issue_loads(issued);

    // State slice: thread owns row j = tid of h[:, c0:c0+32].
    float hreg[kBV];
    {
        const float *src = prm.h0 ? prm.h0 + (((size_t)n * d.Hv + h) * K + tid) * V + c0 : nullptr;
#pragma unroll
        for (int c = 0; c < kBV; ++c) hreg[c] = src ? src[c] : 0.f;
    }
    auto write_hb = [&]() {
        const uint32_t base = sbase + kHb + (tid >> 3) * 128 + (tid & 7) * 16;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
            st_shared_v4(base + cc * 2048, pack_bf16(hreg[8 * cc], hreg[8 * cc + 1]),
                         pack_bf16(hreg[8 * cc + 2], hreg[8 * cc + 3]),
                         pack_bf16(hreg[8 * cc + 4], hreg[8 * cc + 5]),
                         pack_bf16(hreg[8 * cc + 6], hreg[8 * cc + 7]));
    };
    write_hb();
    fence_proxy_async();

    const uint32_t id_S = idesc_bf16(64, 64, false, false);
    const uint32_t id_W = idesc_bf16(64, 128, false, true);
    const uint32_t id_U = idesc_bf16(64, 32, false, true);
    const uint32_t id_D2 = idesc_bf16(128, 32, true, true);
    const int r16 = warp * 16 + lane;  // row of M=64 results owned by lanes < 16
    bool ok = true;

    int ci = 0;
    for (; ci < nchunks; ++ci) {
        const int s = ci % kStages;
        const uint32_t st = sbase + kStage0 + s * kStageBytes;
        const int t0 = sr.start + ci * kChunk;
        const int len = min(kChunk, sr.len - ci * kChunk);
        const uint32_t par = ci & 1;

        // ---- gates of this chunk
        if (tid < kChunk) {
            const int r = tid;
            const float gm = prm.gamma[(size_t)(t0 + min(r, len - 1)) * d.Hv + h];
            sm->gam[r] = gm;
            sm->egam[r] = __expf(gm);
            sm->bet[r] = r < len ? prm.beta[(size_t)(t0 + r) * d.Hv + h] : 0.f;
        }
        ok = wait_bar(&sm->full[s], (ci / kStages) & 1);
        if (__syncthreads_or(!ok)) break;

        // ---- Ainv -> diag(beta)-scaled (in place) and diag(beta e^gamma)-scaled copy
        for (int e = tid; e < 64 * 8; e += kThreads) {
            const int r = e >> 3, p = e & 7;
            const int sblk = (p ^ (r & 7)) * 8;  // first logical column of this 16-byte chunk
            const uint32_t off = (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + p * 16);
            uint4 raw = *reinterpret_cast<const uint4 *>(smem + kStage0 + s * kStageBytes + kAi + off);
            const __nv_bfloat16 *x = reinterpret_cast<const __nv_bfloat16 *>(&raw);
            float a[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) a[q] = __bfloat162float(x[q]);
            uint32_t u[4], w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int s0 = sblk + 2 * q;
                const float b0 = sm->bet[s0], b1 = sm->bet[s0 + 1];
                u[q] = pack_bf16(a[2 * q] * b0, a[2 * q + 1] * b1);
                w[q] = pack_bf16(a[2 * q] * b0 * sm->egam[s0], a[2 * q + 1] * b1 * sm->egam[s0 + 1]);
            }
            st_shared_v4(st + kAi + off, u[0], u[1], u[2], u[3]);
            st_shared_v4(sbase + kAw + off, w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async();
        __syncthreads();

        // ---- phase A: S = Q K^T, W = Aw K, DW = Au V
        if (tid == 0) {
            tc_fence_after();
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                mma_bf16(tmem + kColS, smem_desc(st + kQ + off, 16, 1024, kSw128),
                         smem_desc(st + kK + off, 16, 1024, kSw128), id_S, ks > 0);
            }
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(tmem + kColW, smem_desc(sbase + kAw + ks * 32, 16, 1024, kSw128),
                         smem_desc(st + kK + ks * 2048, 8192, 1024, kSw128), id_W, ks > 0);
                mma_bf16(tmem + kColDW, smem_desc(st + kAi + ks * 32, 16, 1024, kSw128),
                         smem_desc(st + kVt + ks * 1024, 4096, 512, kSw64), id_U, ks > 0);
            }
            mma_commit(&sm->bar[0]);
        }
        ok = wait_bar(&sm->bar[0], par);
        if (__syncthreads_or(!ok)) break;
        tc_fence_after();

        // ---- P = causal decay mask o S ; -w -> bf16 tiles
        {
            const int r = r16;
            const float gr = sm->gam[r & 63];
            float v[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld32(tmem + lane_base + kColS + half * 32, v);
                if (lane < 16) {
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        uint32_t pk[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int s0 = half * 32 + cc * 8 + 2 * q;
                            const float p0 = s0 <= r ? __expf(gr - sm->gam[s0]) * v[cc * 8 + 2 * q] : 0.f;
                            const float p1 = s0 + 1 <= r ? __expf(gr - sm->gam[s0 + 1]) * v[cc * 8 + 2 * q + 1] : 0.f;
                            pk[q] = pack_bf16(p0, p1);
                        }
                        st_shared_v4(sbase + kP + sw128_offset(r, half * 32 + cc * 8, 64), pk[0], pk[1],
                                     pk[2], pk[3]);
                    }
                }
            }
#pragma unroll
            for (int quarter = 0; quarter < 4; ++quarter) {
                tmem_ld32(tmem + lane_base + kColW + quarter * 32, v);
                if (lane < 16) {
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        st_shared_v4(sbase + kWn + sw128_offset(r, quarter * 32 + cc * 8, 64),
                                     pack_bf16(-v[cc * 8], -v[cc * 8 + 1]),
                                     pack_bf16(-v[cc * 8 + 2], -v[cc * 8 + 3]),
                                     pack_bf16(-v[cc * 8 + 4], -v[cc * 8 + 5]),
                                     pack_bf16(-v[cc * 8 + 6], -v[cc * 8 + 7]));
                }
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- phase B: DW += (-w) h ; DQ = Q h
        if (tid == 0) {
            tc_fence_after();
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t aoff = (ks >> 2) * 8192 + (ks & 3) * 32;
                const uint64_t bd = smem_desc(sbase + kHb + ks * 256, 128, 2048, kSwNone);
                mma_bf16(tmem + kColDW, smem_desc(sbase + kWn + aoff, 16, 1024, kSw128), bd, id_U, true);
                mma_bf16(tmem + kColDQ, smem_desc(st + kQ + aoff, 16, 1024, kSw128), bd, id_U, ks > 0);
            }
            mma_commit(&sm->bar[1]);
        }
        ok = wait_bar(&sm->bar[1], par);
        if (__syncthreads_or(!ok)) break;
        tc_fence_after();

        // ---- Delta and e^{gamma_C - gamma} Delta -> bf16 tiles
        const float gl = sm->gam[63];
        {
            float v[32];
            tmem_ld32(tmem + lane_base + kColDW, v);
            if (lane < 16) {
                const int r = r16;
                const float sc = __expf(gl - sm->gam[r]);
                const bool live = r < len;
                const uint32_t base = (uint32_t)((r >> 3) * 128 + (r & 7) * 16);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float x[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) x[q] = live ? v[cc * 8 + q] : 0.f;
                    st_shared_v4(sbase + kDb + base + cc * 1024, pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]),
                                 pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
                    st_shared_v4(sbase + kDt + base + cc * 1024, pack_bf16(sc * x[0], sc * x[1]),
                                 pack_bf16(sc * x[2], sc * x[3]), pack_bf16(sc * x[4], sc * x[5]),
                                 pack_bf16(sc * x[6], sc * x[7]));
                }
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- phase C: D2 = K^T Dt ; DP = P Db
        if (tid == 0) {
            tc_fence_after();
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t bt = smem_desc(sbase + kDt + ks * 256, 128, 1024, kSwNone);
                const uint64_t bb = smem_desc(sbase + kDb + ks * 256, 128, 1024, kSwNone);
                mma_bf16(tmem + kColD2, smem_desc(st + kK + ks * 2048, 8192, 1024, kSw128), bt, id_D2, ks > 0);
                mma_bf16(tmem + kColDP, smem_desc(sbase + kP + ks * 32, 16, 1024, kSw128), bb, id_U, ks > 0);
            }
            mma_commit(&sm->bar[2]);
        }
        ok = wait_bar(&sm->bar[2], par);
        if (__syncthreads_or(!ok)) break;
        tc_fence_after();

        // ---- h <- e^{gamma_C} h + D2 ; o = scale (e^gamma DQ + DP)
        {
            float v[32];
            tmem_ld32(tmem + lane_base + kColD2, v);
            const float eC = __expf(gl);
#pragma unroll
            for (int c = 0; c < kBV; ++c) hreg[c] = fmaf(eC, hreg[c], v[c]);
            write_hb();
            float dq[32];
            tmem_ld32(tmem + lane_base + kColDQ, dq);
            tmem_ld32(tmem + lane_base + kColDP, v);
            if (lane < 16 && r16 < len) {
                const int r = r16;
                const float er = sm->egam[r], scl = d.scale;
                uint4 *dst = reinterpret_cast<uint4 *>(prm.o + ((size_t)(t0 + r) * d.Hv + h) * V + c0);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 pk;
                    pk.x = pack_bf16(scl * fmaf(er, dq[cc * 8 + 0], v[cc * 8 + 0]), scl * fmaf(er, dq[cc * 8 + 1], v[cc * 8 + 1]));
                    pk.y = pack_bf16(scl * fmaf(er, dq[cc * 8 + 2], v[cc * 8 + 2]), scl * fmaf(er, dq[cc * 8 + 3], v[cc * 8 + 3]));
                    pk.z = pack_bf16(scl * fmaf(er, dq[cc * 8 + 4], v[cc * 8 + 4]), scl * fmaf(er, dq[cc * 8 + 5], v[cc * 8 + 5]));
                    pk.w = pack_bf16(scl * fmaf(er, dq[cc * 8 + 6], v[cc * 8 + 6]), scl * fmaf(er, dq[cc * 8 + 7], v[cc * 8 + 7]));
                    dst[cc] = pk;
                }
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        // the stage of chunk ci is free again: refill it with chunk ci + kStages
        if (tid == 0 && issued < nchunks) {
            issue_loads(issued);
            ++issued;
        }
    }

    if (ci < nchunks) {
        // A wait expired: record it, let every load already issued land (bounded),
        // then release tensor memory and return without writing the final state.
        if (tid == 0) {
            set_status(prm.status, GDN_ERR_TIMEOUT);
            for (int c = ci; c < issued; ++c) wait_bar(&sm->full[c % kStages], (c / kStages) & 1);
        }
        __syncthreads();
    } else if (prm.final_state) {
        float4 *dst = reinterpret_cast<float4 *>(prm.final_state + (((size_t)n * d.Hv + h) * K + tid) * V + c0);
#pragma unroll
        for (int c = 0; c < kBV / 4; ++c)
            dst[c] = make_float4(hreg[4 * c], hreg[4 * c + 1], hreg[4 * c + 2], hreg[4 * c + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool make_map(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
              const cuuint32_t *box, CUtensorMapSwizzle sw) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_fwd_supported(const FwdArgs &a) {
    return a.dtype == GDN_DTYPE_BF16 && a.d.K == 128 && a.d.V == 128 &&
           (long long)a.d.NC * a.d.Hv * kChunk < (1ll << 31) && a.h_chunks == nullptr &&
           a.delta == nullptr;
}

cudaError_t launch_fwd_tc(const FwdArgs &a) {
    const Dims &d = a.d;
    if (d.N == 0) return cudaSuccess;
    CUtensorMap mq, mk, mv, ma;
    // q, k: [T_total, Hq, K] bf16, box 64 (K) x 1 (head) x 64 (tokens)
    const cuuint64_t dq[3] = {(cuuint64_t)d.K, (cuuint64_t)d.Hq, (cuuint64_t)(d.T_total > 0 ? d.T_total : 1)};
    const cuuint64_t sq[2] = {(cuuint64_t)d.K * 2, (cuuint64_t)d.Hq * d.K * 2};
    const cuuint32_t bq[3] = {64, 1, 64};
    const cuuint64_t dv[3] = {(cuuint64_t)d.V, (cuuint64_t)d.Hv, (cuuint64_t)(d.T_total > 0 ? d.T_total : 1)};
    const cuuint64_t sv[2] = {(cuuint64_t)d.V * 2, (cuuint64_t)d.Hv * d.V * 2};
    const cuuint32_t bv[3] = {kBV, 1, 64};
    const cuuint64_t da[2] = {64, (cuuint64_t)(d.NC > 0 ? d.NC : 1) * d.Hv * 64};
    const cuuint64_t sa[1] = {128};
    const cuuint32_t ba[2] = {64, 64};
    if (!make_map(&mq, a.q, 3, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, a.k, 3, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, a.v, 3, dv, sv, bv, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map(&ma, a.ainv, 2, da, sa, ba, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    TcParams p;
    p.d = d;
    p.gamma = a.gamma;
    p.beta = a.beta;
    p.h0 = a.h0;
    p.o = (__nv_bfloat16 *)a.o;
    p.final_state = a.final_state;
    p.status = a.status;
    cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(d.N, d.Hv, d.V / kBV);
    fwd_tc_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mk, mv, ma, p);
    return cudaGetLastError();
}

}  // namespace gdn
