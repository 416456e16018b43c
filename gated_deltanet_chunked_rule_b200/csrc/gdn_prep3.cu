// gdn_prep3.cu -- chunk prep for the bf16, K = V = 128 tensor-core path: every
// per-chunk quantity that does not depend on the state, so that the state
// chains downstream only run their two state-dependent products.
//
// One CTA (8 warps) per (64-token chunk, qk head) serves the value heads of the
// qk head's group. From k, q (per qk head) and v, g, beta (per value head):
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
// Products on warp-level bf16 MMAs from swizzled shared-memory tiles; the unit
// lower-triangular inverse block-wise on 16 x 16 blocks: diagonal blocks by
// forward substitution, off-diagonal blocks one block diagonal at a time on
// tf32 MMAs. Rows past the end of a sequence have k = q = v = 0 and beta = 0,
// so their rows of A vanish and the inverse is the identity there.
#include "gdn_internal.cuh"
#include "gdn_warp.cuh"

namespace gdn {
namespace {

using namespace warp;

constexpr int kThreads = 256;
constexpr int C = 64, K = 128, V = 128;

// ---- shared memory (bytes)
constexpr int kSK = 0;          // k tile [64][128] bf16
constexpr int kSQV = 16384;     // q tile, then the current value head's v tile
constexpr int kSA = 32768;      // float [64][65]
constexpr int kSX = kSA + 16640;
constexpr int kST = kSX + 16640;
constexpr int kSAw = kST + 16640;  // bf16 [64][64] Ainv diag(beta e^gamma)
constexpr int kSAu = kSAw + 8192;  // bf16 [64][64] Ainv diag(beta)
constexpr int kSvec = kSAu + 8192;
constexpr int kSmemBytes = kSvec + 1024;
static_assert(kSAw % 16 == 0 && kSmemBytes <= 113 * 1024, "two CTAs per SM");

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

struct Prep3Params {
    Dims d;
    const __nv_bfloat16 *q, *k, *v;
    const float *g, *beta;
    float *gamma_out;
    __nv_bfloat16 *ainv_out;  // nullable
    __nv_bfloat16 *w_out;
    float *u_out;
    __nv_bfloat16 *p_out;
};

__global__ void __launch_bounds__(kThreads, 2) prep3_kernel(const Prep3Params prm) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sb = smem_u32(smem);
    const Dims &d = prm.d;
    const int cg = blockIdx.x, hq = blockIdx.y;
    const int n = chunk_owner(d, cg);
    if (n < 0) return;
    const SeqRange sr = seq_range(d, n);
    const int ci = cg - sr.chunk0;
    const int t0 = sr.start + ci * C, len = min(C, sr.len - ci * C);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wm = warp & 3, wn = warp >> 2, g8 = lane >> 2, c4 = lane & 3;
    const int r0 = 16 * wm + g8, r1 = r0 + 8;
    const int G = d.Hv / d.Hq;

    float(*A)[65] = reinterpret_cast<float(*)[65]>(smem + kSA);
    float(*X)[65] = reinterpret_cast<float(*)[65]>(smem + kSX);
    float(*T)[65] = reinterpret_cast<float(*)[65]>(smem + kST);
    float *gam = reinterpret_cast<float *>(smem + kSvec);
    float *egam = gam + 64, *bet = gam + 128, *scan = gam + 192;
    const Tile tK{sb + kSK, 256}, tQV{sb + kSQV, 256}, tAw{sb + kSAw, 128}, tAu{sb + kSAu, 128};

    // ---- k, q tiles; g, beta of the first value head (prefetched one head ahead)
    load_tile<kThreads>(tK, prm.k + ((size_t)t0 * d.Hq + hq) * K, (size_t)d.Hq * K, C, K, len, tid);
    load_tile<kThreads>(tQV, prm.q + ((size_t)t0 * d.Hq + hq) * K, (size_t)d.Hq * K, C, K, len, tid);
    cp_async_commit();
    float g_next = 0.f, b_next = 0.f;
    if (tid < C && tid < len) {
        g_next = prm.g[(size_t)(t0 + tid) * d.Hv + hq * G];
        b_next = prm.beta[(size_t)(t0 + tid) * d.Hv + hq * G];
    }
    cp_async_wait_all();
    __syncthreads();

    // ---- S = Q K^T, G = K K^T: 16 x 32 per warp, kept in registers for every value head
    float sacc[4][4] = {}, gacc[4][4] = {};
    wgemm<4, false, false>(sacc, tQV, tK, 16 * wm, 32 * wn, K, lane);
    wgemm<4, false, false>(gacc, tK, tK, 16 * wm, 32 * wn, K, lane);
    __syncthreads();  // q tile no longer read: its space takes v

    for (int gi = 0; gi < G; ++gi) {
        const int h = hq * G + gi;
        load_tile<kThreads>(tQV, prm.v + ((size_t)t0 * d.Hv + h) * V, (size_t)d.Hv * V, C, V, len, tid);
        cp_async_commit();
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
        __syncthreads();
        // ---- A (strictly lower), X = 0, and P = M o S -> global
        {
            const float gr[2] = {gam[r0], gam[r1]}, br[2] = {bet[r0], bet[r1]};
            __nv_bfloat16 *pout = prm.p_out + ((size_t)cg * d.Hv + h) * C * C;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int s = 32 * wn + 8 * j + 2 * c4;
                const float gs0 = gam[s], gs1 = gam[s + 1];
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = hi ? r1 : r0;
                    const float e0 = s <= r ? __expf(gr[hi] - gs0) : 0.f;
                    const float e1 = s + 1 <= r ? __expf(gr[hi] - gs1) : 0.f;
                    A[r][s] = s < r ? br[hi] * e0 * gacc[j][2 * hi] : 0.f;
                    A[r][s + 1] = s + 1 < r ? br[hi] * e1 * gacc[j][2 * hi + 1] : 0.f;
                    X[r][s] = 0.f;
                    X[r][s + 1] = 0.f;
                    const bool live = r < len;
                    *reinterpret_cast<uint32_t *>(pout + r * C + s) =
                        pack_bf16(live ? e0 * sacc[j][2 * hi] : 0.f, live ? e1 * sacc[j][2 * hi + 1] : 0.f);
                }
            }
        }
        __syncthreads();
        // ---- diagonal 16 x 16 blocks: thread t -> block t / 16, column t % 16
        if (tid < 64) {
            const int b = tid >> 4, cc = tid & 15, o = b * 16;
            float xcol[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
                for (int j = 0; j < r; ++j) acc = fmaf(-A[o + r][o + j], xcol[j], acc);
                xcol[r] = r < cc ? 0.f : acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) X[o + r][o + cc] = xcol[r];
        }
        __syncthreads();
        // ---- off-diagonal blocks, one block diagonal at a time:
        //      X_ij = -X_ii sum_{m=j}^{i-1} A_im X_mj  (16 x 16 x 16 products on tf32 MMAs)
        for (int lvl = 1; lvl < 4; ++lvl) {
            if (warp < 4 - lvl) {
                const int i = lvl + warp, j = warp;
                float t[2][4] = {};
                for (int m = j; m < i; ++m) {
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const int ac = m * 16 + kk * 8 + c4;
                        const uint32_t a[4] = {tf32(A[i * 16 + g8][ac]), tf32(A[i * 16 + g8 + 8][ac]),
                                               tf32(A[i * 16 + g8][ac + 4]), tf32(A[i * 16 + g8 + 8][ac + 4])};
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
                            const int bc = j * 16 + nt * 8 + g8;
                            mma_tf32(t[nt], a, tf32(X[m * 16 + kk * 8 + c4][bc]), tf32(X[m * 16 + kk * 8 + c4 + 4][bc]));
                        }
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int col = j * 16 + nt * 8 + 2 * c4;
                    T[i * 16 + g8][col] = t[nt][0];
                    T[i * 16 + g8][col + 1] = t[nt][1];
                    T[i * 16 + g8 + 8][col] = t[nt][2];
                    T[i * 16 + g8 + 8][col + 1] = t[nt][3];
                }
                __syncwarp();
                float x[2][4] = {};
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int ac = i * 16 + kk * 8 + c4;
                    const uint32_t a[4] = {tf32(X[i * 16 + g8][ac]), tf32(X[i * 16 + g8 + 8][ac]),
                                           tf32(X[i * 16 + g8][ac + 4]), tf32(X[i * 16 + g8 + 8][ac + 4])};
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int bc = j * 16 + nt * 8 + g8;
                        mma_tf32(x[nt], a, tf32(T[i * 16 + kk * 8 + c4][bc]), tf32(T[i * 16 + kk * 8 + c4 + 4][bc]));
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int col = j * 16 + nt * 8 + 2 * c4;
                    X[i * 16 + g8][col] = -x[nt][0];
                    X[i * 16 + g8][col + 1] = -x[nt][1];
                    X[i * 16 + g8 + 8][col] = -x[nt][2];
                    X[i * 16 + g8 + 8][col + 1] = -x[nt][3];
                }
            }
            __syncthreads();
        }
        // ---- Ainv diag(beta), Ainv diag(beta e^gamma) -> bf16 tiles; Ainv -> global (optional)
        for (int e = tid; e < C * C / 2; e += kThreads) {
            const int r = e >> 5, s = (e & 31) * 2;
            const float x0 = X[r][s], x1 = X[r][s + 1];
            const float u0 = x0 * bet[s], u1 = x1 * bet[s + 1];
            st_shared_b32(toff(tAu, r, s), pack_bf16(u0, u1));
            st_shared_b32(toff(tAw, r, s), pack_bf16(u0 * egam[s], u1 * egam[s + 1]));
            if (prm.ainv_out)
                *reinterpret_cast<uint32_t *>(prm.ainv_out + ((size_t)cg * d.Hv + h) * C * C + r * C + s) =
                    pack_bf16(x0, x1);
        }
        cp_async_wait_all();  // this head's v tile
        __syncthreads();
        // ---- u = Au V (fp32), w = Aw K (bf16): 16 x 64 per warp
        {
            float acc[8][4] = {};
            wgemm<8, false, true>(acc, tAu, tQV, 16 * wm, 64 * wn, C, lane);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int col = 64 * wn + 8 * j + 2 * c4;
                if (r0 < len)
                    *reinterpret_cast<float2 *>(prm.u_out + ((size_t)(t0 + r0) * d.Hv + h) * V + col) =
                        make_float2(acc[j][0], acc[j][1]);
                if (r1 < len)
                    *reinterpret_cast<float2 *>(prm.u_out + ((size_t)(t0 + r1) * d.Hv + h) * V + col) =
                        make_float2(acc[j][2], acc[j][3]);
            }
        }
        {
            float acc[8][4] = {};
            wgemm<8, false, true>(acc, tAw, tK, 16 * wm, 64 * wn, C, lane);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int col = 64 * wn + 8 * j + 2 * c4;
                if (r0 < len)
                    *reinterpret_cast<uint32_t *>(prm.w_out + ((size_t)(t0 + r0) * d.Hv + h) * K + col) =
                        pack_bf16(acc[j][0], acc[j][1]);
                if (r1 < len)
                    *reinterpret_cast<uint32_t *>(prm.w_out + ((size_t)(t0 + r1) * d.Hv + h) * K + col) =
                        pack_bf16(acc[j][2], acc[j][3]);
            }
        }
        __syncthreads();  // v tile, Au, Aw, A, X free for the next value head
    }
}

}  // namespace

bool prep3_supported(const FwdArgs &a) { return a.dtype == GDN_DTYPE_BF16 && a.d.K == 128 && a.d.V == 128; }

cudaError_t launch_prep3(const FwdArgs &a) {
    if (a.d.NC == 0) return cudaSuccess;
    if (!a.w16 || !a.u32 || !a.p16 || !a.gamma) return cudaErrorInvalidValue;
    Prep3Params p;
    p.d = a.d;
    p.q = (const __nv_bfloat16 *)a.q;
    p.k = (const __nv_bfloat16 *)a.k;
    p.v = (const __nv_bfloat16 *)a.v;
    p.g = a.g;
    p.beta = a.beta;
    p.gamma_out = a.gamma;
    p.ainv_out = (__nv_bfloat16 *)a.ainv;
    p.w_out = (__nv_bfloat16 *)a.w16;
    p.u_out = a.u32;
    p.p_out = (__nv_bfloat16 *)a.p16;
    cudaError_t e = cudaFuncSetAttribute(prep3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    prep3_kernel<<<dim3(a.d.NC, a.d.Hq), kThreads, kSmemBytes, a.stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
