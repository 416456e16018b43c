// gdn_fwd2.cu -- warp-specialised chunked forward (bf16, K = V = 128): the
// state chain on warp-level tensor-core MMAs, everything else on tcgen05.
//
// One CTA per (sequence, value head, 32-column slice of V). Per 64-token chunk
// (notation of gdn_internal.cuh):
//
//   off the chain (tcgen05, TMEM accumulators, issued by two MMA warps):
//     S = Q K^T,  W = (Ainv diag(beta e^gamma)) K,  U = (Ainv diag(beta)) V,
//     DQ = Q h,   DP = P Delta    ->   o = scale (e^gamma o DQ + DP)
//   on the chain (mma.sync m16n8k16, fp32 state in registers):
//     Delta = U + (-w) h,    h <- e^{gamma_C} h + K^T (e^{gamma_C - gamma} o Delta)
//
// The chain is a strict sequence over chunks. On sm_100a a tcgen05 MMA pays
// roughly 450 cycles from issue to a completed mbarrier, twice per chunk on the
// chain, whereas a dependent mma.sync costs about 20 cycles, so the chain's two
// products (64x32x128 and 128x32x64 per chunk) run register-resident on
// mma.sync. The bulk products that do not depend on h, and the output
// products, stay on tcgen05 where their latency overlaps the chain.
//
// Warp roles (320 threads):
//   warps 0-3  chain: h (128 x 32 fp32) in mma fragments; Delta; state update.
//   warps 4-7  aux:   scales Ainv, turns S/W/U from TMEM into P (masked,
//                     decayed), -w and u in shared memory for the next chunk,
//                     and writes o of the previous chunk from DQ/DP.
//   warp 8     MMA issuer A: TMA prologue, S/W/U MMAs.
//   warp 9     MMA issuer B: DQ/DP MMAs, TMA refills of the 3-deep ring.
// Roles hand work over through monotonically increasing shared-memory counters
// (release/acquire), which cannot alias the way mbarrier phase parities can
// when a producer runs two phases ahead of a consumer. mbarriers are used only
// where the hardware requires them: TMA completion (full[], one consumer) and
// tcgen05.commit (mmaA for the aux warps, mmaO for issuer B, each with a single
// consumer that its producer cannot lap). Every wait is bounded in time; a
// wait that expires records GDN_ERR_TIMEOUT and winds the CTA down.
#include <cudaTypedefs.h>

#include <cstddef>

#include "gdn_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kThreads = 320;
constexpr int kBV = 32;
constexpr int kStages = 3;

// ---- shared memory (bytes from a 1024-aligned base)
constexpr int kHb = 0;          // 3 x 8192   h (bf16), MN-major, no swizzle: (n/8)*2048 + (k/8)*128 + (k%8)*16
constexpr int kDb = 24576;      // 3 x 4096   Delta (bf16), same layout with K = 64 tokens
constexpr int kDt = 36864;      // 4096       e^{gamma_C - gamma} Delta, chain only
constexpr int kAw = 40960;      // 8192       Ainv diag(beta e^gamma), K-major SW128
constexpr int kP = 49152;       // 2 x 8192   P, K-major SW128
constexpr int kWn = 65536;      // 16384      -w (bf16), row-major 256 B rows, 16-B chunks XOR (row % 8)
constexpr int kU = 81920;       // 9216       u (fp32), row stride 36 floats
constexpr int kStage0 = 91136;  // TMA ring
constexpr int kQ = 0, kK = 16384, kAi = 32768, kVt = 40960, kStageBytes = 45056;
constexpr int kTxBytes = 16384 + 16384 + 8192 + 4096;
constexpr int kSmall = kStage0 + kStages * kStageBytes;
constexpr int kSmemBytes = kSmall + 2560 + 1024;
static_assert(kStage0 % 1024 == 0 && kSmemBytes <= 232448, "shared memory layout");

// S, W, U double-buffered (buffer b at +224 b), DQ and DP single.
constexpr uint32_t kColS = 0, kColW = 64, kColU = 192, kABuf = 224, kColQ = 448, kColP = 480, kTmemCols = 512;

struct __align__(16) Gates {  // read with 16-byte vector loads
    float gam[64], bet[64], egam[64];
};

// Hand-over counters: each holds the number of chunks (or states) its producer
// has finished; consumers wait until it reaches the count they need.
enum Ctr { kScaled, kTmemA, kReady, kPReady, kWnFree, kDelta, kH, kStage, kODone, kTmemO, kNumCtr };

struct Small {
    uint64_t full[kStages];
    uint64_t mmaA[2], mmaO;
    uint32_t ctr[kNumCtr];
    int loads_issued, loads_landed;  // TMA chunk loads issued / observed complete
    uint32_t tmem_base;
    int abort_flag;
    Gates gates[3];
};
static_assert(sizeof(Small) <= 2560, "small area");
static_assert(offsetof(Small, gates) % 16 == 0 && sizeof(Gates) % 16 == 0, "gate vectors are read as float4");
static_assert(kSmall % 16 == 0, "small area alignment");

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait (2 s of wall-clock time); false if it expired or the CTA is aborting.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    const uint32_t a = smem_u32(bar);
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait(a, parity)) return true;
        if ((i & 1023u) == 0) {
            if (*abort_flag) return false;
            const uint64_t t = globaltimer();
            if (i == 0) t0 = t;
            else if (t - t0 > 2000000000ull) return false;
        }
    }
}

__device__ __forceinline__ void publish(uint32_t *ctr, uint32_t v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(ctr)), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *ctr) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(ctr)) : "memory");
    return v;
}

// Waits (bounded, 2 s) until *ctr >= need; false if it expired or the CTA is aborting.
__device__ __forceinline__ bool wait_ge(const uint32_t *ctr, uint32_t need, volatile int *abort_flag) {
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        if (ld_acquire(ctr) >= need) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            const uint64_t t = globaltimer();
            if (i == 0) t0 = t;
            else if (t - t0 > 2000000000ull) return false;
        }
    }
}

// Named barrier over one 128-thread role that also ANDs a predicate across it.
__device__ __forceinline__ bool role_sync_and(int id, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, %2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Per-access shared-memory stores and fragment loads carry no "memory" clobber
// so the compiler may overlap them; ordering across roles comes from the
// barrier, fence and release/acquire statements, which do clobber memory.
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d));
}
__device__ __forceinline__ void st_shared_b32(uint32_t addr, uint32_t a) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a));
}
__device__ __forceinline__ void st_shared_v2f(uint32_t addr, float a, float b) {
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void hmma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct Fwd2Params {
    Dims d;
    const float *gamma;   // [T_total, Hv]
    const float *beta;    // [T_total, Hv]
    const float *h0;      // [N, Hv, K, V] or null
    __nv_bfloat16 *o;     // [T_total, Hv, V]
    float *final_state;   // [N, Hv, K, V] or null
    unsigned *status;
};

__global__ void __launch_bounds__(kThreads, 1)
fwd2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
            const Fwd2Params prm) {
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
        mbar_init(&sm->mmaA[0], 1);
        mbar_init(&sm->mmaA[1], 1);
        mbar_init(&sm->mmaO, 1);
        for (int c = 0; c < kNumCtr; ++c) sm->ctr[c] = 0;
        sm->loads_issued = sm->loads_landed = 0;
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

    auto issue_loads = [&](int ci) {
        const int s = ci % kStages;
        uint8_t *st = smem + kStage0 + s * kStageBytes;
        const int t0 = sr.start + ci * kChunk;
        const int cg = sr.chunk0 + ci;
        mbar_arrive_expect_tx(&sm->full[s], kTxBytes);
        atomicAdd(&sm->loads_issued, 1);
        tma_load_3d(st + kQ, &tm_q, &sm->full[s], 0, hq, t0);
        tma_load_3d(st + kQ + 8192, &tm_q, &sm->full[s], 64, hq, t0);
        tma_load_3d(st + kK, &tm_k, &sm->full[s], 0, hq, t0);
        tma_load_3d(st + kK + 8192, &tm_k, &sm->full[s], 64, hq, t0);
        tma_load_2d(st + kAi, &tm_a, &sm->full[s], 0, (cg * d.Hv + h) * kChunk);
        tma_load_3d(st + kVt, &tm_v, &sm->full[s], c0, h, t0);
    };

    uint32_t *ctr = sm->ctr;
    if (warp < 4) {
        // =========================================================== chain
        const int cw = warp, g = lane >> 2, c4 = lane & 3;
        float hf[2][4][4];  // [m-tile][n-tile][frag]: dims 32cw+16mt+g(+8), cols 8nt+2c4(+1)
        {
            const float *src = prm.h0 ? prm.h0 + ((size_t)n * d.Hv + h) * K * V : nullptr;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int dim = 32 * cw + 16 * mt + g + ((q >> 1) << 3);
                        const int col = 8 * nt + 2 * c4 + (q & 1);
                        hf[mt][nt][q] = src ? src[(size_t)dim * V + c0 + col] : 0.f;
                    }
        }
        auto write_hb = [&](int buf) {
            const uint32_t base = sb + kHb + buf * 8192 + c4 * 4;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int dim = 32 * cw + 16 * mt + g + half * 8;
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
                        st_shared_b32(base + nt * 2048 + (dim >> 3) * 128 + (dim & 7) * 16,
                                      pack_bf16(hf[mt][nt][2 * half], hf[mt][nt][2 * half + 1]));
                }
        };
        write_hb(0);
        fence_proxy_async();
        bool ok = role_sync_and(1, true);
        if (tid == 0) publish(&ctr[kH], 1);  // h_0

        for (int j = 0; j < nch && ok; ++j) {
            const int len = min(kChunk, sr.len - j * kChunk);
            ok = role_sync_and(1, wait_ge(&ctr[kReady], j + 1, abort_flag));
            if (!ok) break;
            // gate scalars of chunk j (the slot is refilled once this chunk's -w is consumed)
            const Gates &G = sm->gates[j % 3];
            const float gl = G.gam[63];
            const float gtok[2] = {G.gam[16 * cw + g], G.gam[16 * cw + g + 8]};
            // ---- Delta = u + (-w) h : rows 16cw..16cw+15 (tokens), 32 columns
            float acc[4][4];
            {
                const float *U = reinterpret_cast<const float *>(smem + kU);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const int r0 = 16 * cw + g, col = 8 * nt + 2 * c4;
                    const float2 a = *reinterpret_cast<const float2 *>(U + r0 * 36 + col);
                    const float2 b = *reinterpret_cast<const float2 *>(U + (r0 + 8) * 36 + col);
                    acc[nt][0] = a.x; acc[nt][1] = a.y; acc[nt][2] = b.x; acc[nt][3] = b.y;
                }
                const uint32_t hb = sb + kHb + (j % 3) * 8192;
                const int arow = 16 * cw + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int mi = lane >> 3;  // (kg, nb): (2ks,2np) (2ks+1,2np) (2ks,2np+1) (2ks+1,2np+1)
                uint32_t a[2][4], b[2][2][4];
                auto load = [&](int ks, int buf) {
                    const int ch = 2 * ks + (lane >> 4);
                    ldsm_x4(a[buf], sb + kWn + arow * 256 + ((ch ^ (arow & 7)) << 4));
#pragma unroll
                    for (int np = 0; np < 2; ++np)
                        ldsm_x4_t(b[buf][np], hb + (2 * np + (mi >> 1)) * 2048 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
                };
                load(0, 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    if (ks + 1 < 8) load(ks + 1, (ks + 1) & 1);
#pragma unroll
                    for (int np = 0; np < 2; ++np) {
                        hmma(acc[2 * np], a[ks & 1], b[ks & 1][np][0], b[ks & 1][np][1]);
                        hmma(acc[2 * np + 1], a[ks & 1], b[ks & 1][np][2], b[ks & 1][np][3]);
                    }
                }
            }
            role_sync_and(1, true);
            if (tid == 0) publish(&ctr[kWnFree], j + 1);
            // ---- Delta -> Db[j%3] (read by the output MMA) ; e^{gamma_C - gamma} Delta -> Dt
            ok = role_sync_and(1, j < 3 || wait_ge(&ctr[kODone], j - 2, abort_flag));  // DP of j-3 read Db[j%3]
            if (!ok) break;
            {
                const uint32_t db = sb + kDb + (j % 3) * 4096 + c4 * 4, dt = sb + kDt + c4 * 4;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int tok = 16 * cw + g + half * 8;
                    const bool live = tok < len;
                    const float sc = __expf(gl - gtok[half]);
                    const uint32_t off = (tok >> 3) * 128 + (tok & 7) * 16;
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) {
                        const float x0 = live ? acc[nt][2 * half] : 0.f, x1 = live ? acc[nt][2 * half + 1] : 0.f;
                        st_shared_b32(db + nt * 1024 + off, pack_bf16(x0, x1));
                        st_shared_b32(dt + nt * 1024 + off, pack_bf16(sc * x0, sc * x1));
                    }
                }
            }
            fence_proxy_async();
            role_sync_and(1, true);
            if (tid == 0) publish(&ctr[kDelta], j + 1);
            // ---- h <- e^{gamma_C} h + K^T Dt : dims 32cw..32cw+31, 32 columns, K = 64 tokens
            {
                const float eC = __expf(gl);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int q = 0; q < 4; ++q) hf[mt][nt][q] *= eC;
                const uint32_t kt = sb + kStage0 + (j % kStages) * kStageBytes + kK;
                const int mi = lane >> 3;
                uint32_t b[2][2][4], a[2][2][4];
                auto load = [&](int ks, int buf) {
#pragma unroll
                    for (int np = 0; np < 2; ++np)
                        ldsm_x4_t(b[buf][np], sb + kDt + (2 * np + (mi >> 1)) * 1024 + (2 * ks + (mi & 1)) * 128 + (lane & 7) * 16);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        // A = K^T rows (dims) m0.., cols (tokens) 16ks..: 8x8 blocks of the
                        // token-major, 128-byte-swizzled k tile read transposed
                        const int tt = 16 * ks + (lane & 7) + ((mi >> 1) & 1) * 8;
                        const int dd = 32 * cw + 16 * mt + (mi & 1) * 8;
                        ldsm_x4_t(a[buf][mt], kt + (dd >> 6) * 8192 + tt * 128 + ((((dd & 63) >> 3) ^ (tt & 7)) << 4));
                    }
                };
                load(0, 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    if (ks + 1 < 4) load(ks + 1, (ks + 1) & 1);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int np = 0; np < 2; ++np) {
                            hmma(hf[mt][2 * np], a[ks & 1][mt], b[ks & 1][np][0], b[ks & 1][np][1]);
                            hmma(hf[mt][2 * np + 1], a[ks & 1][mt], b[ks & 1][np][2], b[ks & 1][np][3]);
                        }
                }
            }
            fence_proxy_async();  // generic reads of the k tile before the next TMA into it
            role_sync_and(1, true);
            if (tid == 0) publish(&ctr[kStage], j + 1);
            // ---- h_{j+1} -> Hb[(j+1)%3] once DQ of chunk j-2 (which read that buffer) is done
            ok = role_sync_and(1, j < 2 || wait_ge(&ctr[kODone], j - 1, abort_flag));
            if (!ok) break;
            write_hb((j + 1) % 3);
            fence_proxy_async();
            role_sync_and(1, true);
            if (tid == 0) publish(&ctr[kH], j + 2);
        }
        if (!ok) {
            if (tid == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        } else if (prm.final_state) {
            float *dst = prm.final_state + ((size_t)n * d.Hv + h) * K * V + c0;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int dim = 32 * cw + 16 * mt + g + half * 8;
                        *reinterpret_cast<float2 *>(dst + (size_t)dim * V + 8 * nt + 2 * c4) =
                            make_float2(hf[mt][nt][2 * half], hf[mt][nt][2 * half + 1]);
                    }
        }
    } else if (warp < 8) {
        // ============================================================= aux
        const int atid = tid - 128, aw = warp - 4;
        const uint32_t lane_base = (uint32_t)(aw * 32) << 16;
        const int ag = lane >> 2, ac = lane & 3;
        const int ar0 = aw * 16 + ag, ar1 = ar0 + 8;  // rows of M=64 results this thread holds
        bool ok = true;
        auto output = [&](int jo) -> bool {  // o of chunk jo from DQ, DP
            if (!wait_ge(&ctr[kODone], jo + 1, abort_flag)) return false;
            tc_fence_after();
            const Gates &G = sm->gates[jo % 3];
            const int len = min(kChunk, sr.len - jo * kChunk);
            const int t0 = sr.start + jo * kChunk;
            float dq[16], dp[16];
            tmem_ld16x256_x4(tmem + lane_base + kColQ, dq);
            tmem_ld16x256_x4(tmem + lane_base + kColP, dp);
            tc_fence_before();
            const float scl = d.scale;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = half ? ar1 : ar0;
                if (r < len) {
                    const float er = G.egam[r];
                    __nv_bfloat16 *dst = prm.o + ((size_t)(t0 + r) * d.Hv + h) * V + c0 + 2 * ac;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int k = 4 * i + 2 * half;
                        *reinterpret_cast<uint32_t *>(dst + 8 * i) =
                            pack_bf16(scl * fmaf(er, dq[k], dp[k]), scl * fmaf(er, dq[k + 1], dp[k + 1]));
                    }
                }
            }
            return true;
        };
        // gates of chunk jj -> registers (threads < 64), then into their slot
        float pg = 0.f, pb = 0.f;
        auto fetch_gates = [&](int jj) {
            if (atid < kChunk && jj < nch) {
                const int t0 = sr.start + jj * kChunk, len = min(kChunk, sr.len - jj * kChunk);
                pg = prm.gamma[(size_t)(t0 + min(atid, len - 1)) * d.Hv + h];
                pb = atid < len ? prm.beta[(size_t)(t0 + atid) * d.Hv + h] : 0.f;
            }
        };
        // scale Ainv of chunk jj: diag(beta) in place (A of U), diag(beta e^gamma) copy (A of W)
        auto scale = [&](int jj) -> bool {
            const int s = jj % kStages;
            const uint32_t st = sb + kStage0 + s * kStageBytes;
            Gates &G = sm->gates[jj % 3];
            if (atid < kChunk) {
                G.gam[atid] = pg;
                G.egam[atid] = __expf(pg);
                G.bet[atid] = pb;
            }
            if (!role_sync_and(2, wait_bar(&sm->full[s], (jj / kStages) & 1, abort_flag))) return false;
            if (atid == 0) sm->loads_landed = jj + 1;
#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int e = atid + it * 128;
                const int r = e >> 3, p = e & 7;
                const int sblk = (p ^ (r & 7)) * 8;
                const uint32_t off = (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + p * 16);
                const uint4 raw = *reinterpret_cast<const uint4 *>(smem + kStage0 + s * kStageBytes + kAi + off);
                const float4 b0 = *reinterpret_cast<const float4 *>(&G.bet[sblk]);
                const float4 b1 = *reinterpret_cast<const float4 *>(&G.bet[sblk + 4]);
                const float4 e0 = *reinterpret_cast<const float4 *>(&G.egam[sblk]);
                const float4 e1 = *reinterpret_cast<const float4 *>(&G.egam[sblk + 4]);
                const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                const float ee[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
                const __nv_bfloat16 *x = reinterpret_cast<const __nv_bfloat16 *>(&raw);
                uint32_t u[4], w[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float a0 = __bfloat162float(x[2 * q]) * bb[2 * q];
                    const float a1 = __bfloat162float(x[2 * q + 1]) * bb[2 * q + 1];
                    u[q] = pack_bf16(a0, a1);
                    w[q] = pack_bf16(a0 * ee[2 * q], a1 * ee[2 * q + 1]);
                }
                st_shared_v4(st + kAi + off, u[0], u[1], u[2], u[3]);
                st_shared_v4(sb + kAw + off, w[0], w[1], w[2], w[3]);
            }
            fence_proxy_async();
            role_sync_and(2, true);
            if (atid == 0) publish(&ctr[kScaled], jj + 1);
            return true;
        };
        if (nch > 0) {
            fetch_gates(0);
            ok = scale(0);
            fetch_gates(1);
        }
        for (int j = 0; j < nch && ok; ++j) {
            const int len = min(kChunk, sr.len - j * kChunk);
            const uint32_t abuf = (j & 1) * kABuf;
            const Gates &G = sm->gates[j % 3];
            // ---- S, W, U of chunk j have landed; Aw is free again -> scale chunk j + 1
            ok = role_sync_and(2, wait_bar(&sm->mmaA[j & 1], (j >> 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            if (j + 1 < nch) {
                ok = scale(j + 1);
                if (!ok) break;
                fetch_gates(j + 2);
            }
            // ---- W, U -> -w (for the chain's ldmatrix) and u, once the chain is done with chunk j-1's
            ok = role_sync_and(2, wait_ge(&ctr[kWnFree], j, abort_flag));
            if (!ok) break;
            {
                float v[32];
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {  // columns 64 hc .. 64 hc + 63 of -w
                    tmem_ld16x256_x8(tmem + lane_base + abuf + kColW + hc * 64, v);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int r = half ? ar1 : ar0;
                        const uint32_t rowb = sb + kWn + r * 256 + 4 * ac;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int ch = 8 * hc + i;
                            st_shared_b32(rowb + ((ch ^ (r & 7)) << 4),
                                          pack_bf16(-v[4 * i + 2 * half], -v[4 * i + 2 * half + 1]));
                        }
                    }
                }
                float u[16];
                tmem_ld16x256_x4(tmem + lane_base + abuf + kColU, u);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int r = half ? ar1 : ar0;
                    const bool live = r < len;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        st_shared_v2f(sb + kU + (r * 36 + 8 * i + 2 * ac) * 4, live ? u[4 * i + 2 * half] : 0.f,
                                      live ? u[4 * i + 2 * half + 1] : 0.f);
                }
            }
            role_sync_and(2, true);
            if (atid == 0) publish(&ctr[kReady], j + 1);
            // ---- S -> P (causal decay mask, SW128 for tcgen05) once DP of chunk j-2 is done with P[j%2]
            ok = role_sync_and(2, j < 2 || wait_ge(&ctr[kODone], j - 1, abort_flag));
            if (!ok) break;
            {
                float v[32];
                tmem_ld16x256_x8(tmem + lane_base + abuf + kColS, v);
                float gs[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float2 t = *reinterpret_cast<const float2 *>(&G.gam[8 * i + 2 * ac]);
                    gs[2 * i] = t.x;
                    gs[2 * i + 1] = t.y;
                }
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int r = half ? ar1 : ar0;
                    const float gr = G.gam[r];
                    const uint32_t pb = sb + kP + (j & 1) * 8192 + (r >> 3) * 1024 + (r & 7) * 128 + 4 * ac;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int s0 = 8 * i + 2 * ac;
                        const float p0 = s0 <= r ? __expf(gr - gs[2 * i]) * v[4 * i + 2 * half] : 0.f;
                        const float p1 = s0 + 1 <= r ? __expf(gr - gs[2 * i + 1]) * v[4 * i + 2 * half + 1] : 0.f;
                        st_shared_b32(pb + ((i ^ (r & 7)) << 4), pack_bf16(p0, p1));
                    }
                }
            }
            fence_proxy_async();
            tc_fence_before();
            role_sync_and(2, true);
            if (atid == 0) {
                publish(&ctr[kPReady], j + 1);
                publish(&ctr[kTmemA], j + 1);
            }
            // ---- output of the previous chunk
            if (j >= 1) {
                ok = role_sync_and(2, output(j - 1));
                if (!ok) break;
                if (atid == 0) publish(&ctr[kTmemO], j);
            }
        }
        if (ok && nch > 0) {
            ok = role_sync_and(2, output(nch - 1));
            if (ok && atid == 0) publish(&ctr[kTmemO], nch);
        }
        if (!ok) {
            if (atid == 0) set_status(prm.status, GDN_ERR_TIMEOUT);
            *abort_flag = 1;
        }
    } else if (warp == 8) {
        // ================================================== MMA issuer A
        if (lane == 0) {
            bool ok = true;
            for (int c = 0; c < kStages && c < nch; ++c) issue_loads(c);
            const uint32_t id_S = idesc_bf16(64, 64, false, false);
            const uint32_t id_W = idesc_bf16(64, 128, false, true);
            const uint32_t id_U = idesc_bf16(64, 32, false, true);
            for (int j = 0; j < nch && ok; ++j) {
                const uint32_t st = sb + kStage0 + (j % kStages) * kStageBytes;
                // buffer j%2 was last read (by the aux warps) for chunk j-2
                ok = wait_ge(&ctr[kScaled], j + 1, abort_flag) && wait_ge(&ctr[kTmemA], j >= 1 ? j - 1 : 0, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t tb = tmem + (j & 1) * kABuf;
                for (int ks = 0; ks < 4; ++ks) {
                    mma_bf16(tb + kColW, smem_desc(sb + kAw + ks * 32, 16, 1024, kSw128),
                             smem_desc(st + kK + ks * 2048, 8192, 1024, kSw128), id_W, ks > 0);
                    mma_bf16(tb + kColU, smem_desc(st + kAi + ks * 32, 16, 1024, kSw128),
                             smem_desc(st + kVt + ks * 1024, 4096, 512, kSw64), id_U, ks > 0);
                }
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_bf16(tb + kColS, smem_desc(st + kQ + off, 16, 1024, kSw128),
                             smem_desc(st + kK + off, 16, 1024, kSw128), id_S, ks > 0);
                }
                mma_commit(&sm->mmaA[j & 1]);
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
            const uint32_t id_O = idesc_bf16(64, 32, false, true);
            int issued = min(kStages, nch);
            for (int j = 0; j < nch && ok; ++j) {
                const uint32_t st = sb + kStage0 + (j % kStages) * kStageBytes;
                ok = wait_ge(&ctr[kH], j + 1, abort_flag) && wait_ge(&ctr[kDelta], j + 1, abort_flag) &&
                     wait_ge(&ctr[kPReady], j + 1, abort_flag) && wait_ge(&ctr[kTmemO], j, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t hb = sb + kHb + (j % 3) * 8192, db = sb + kDb + (j % 3) * 4096;
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t aoff = (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_bf16(tmem + kColQ, smem_desc(st + kQ + aoff, 16, 1024, kSw128),
                             smem_desc(hb + ks * 256, 128, 2048, kSwNone), id_O, ks > 0);
                }
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + kColP, smem_desc(sb + kP + (j & 1) * 8192 + ks * 32, 16, 1024, kSw128),
                             smem_desc(db + ks * 256, 128, 1024, kSwNone), id_O, ks > 0);
                mma_commit(&sm->mmaO);
                ok = wait_bar(&sm->mmaO, j & 1, abort_flag);
                if (!ok) break;
                tc_fence_before();
                publish(&ctr[kODone], j + 1);
                // refill the stage of chunk j with chunk j + 3 once the chain is done with its k tile
                if (issued < nch) {
                    ok = wait_ge(&ctr[kStage], j + 1, abort_flag);
                    if (!ok) break;
                    issue_loads(issued);
                    ++issued;
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
                   globaltimer() - t0 < 2000000000ull) {
            }
    }
    __syncthreads();
    if (warp == 8) {
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

cudaError_t launch_fwd2(const FwdArgs &a) {
    const Dims &d = a.d;
    if (d.N == 0) return cudaSuccess;
    CUtensorMap mq, mk, mv, ma;
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
    Fwd2Params p;
    p.d = d;
    p.gamma = a.gamma;
    p.beta = a.beta;
    p.h0 = a.h0;
    p.o = (__nv_bfloat16 *)a.o;
    p.final_state = a.final_state;
    p.status = a.status;
    cudaError_t e = cudaFuncSetAttribute(fwd2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(d.N, d.Hv, d.V / kBV);
    fwd2_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mk, mv, ma, p);
    return cudaGetLastError();
}

}  // namespace gdn
