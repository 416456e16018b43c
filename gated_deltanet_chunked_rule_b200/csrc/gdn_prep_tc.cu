// gdn_prep_tc.cu -- chunk prep for bf16 problems with K = 128.
//
// One CTA per (64-token chunk, qk head) serves every value head of the qk
// head's group, so the Gram matrix K K^T of the chunk is formed once:
//
//   G     = K K^T                        (64 x 64, bf16 tensor cores, fp32 accumulate)
//   gamma = in-chunk cumulative sum of g (per value head)
//   A_rs  = beta_r exp(gamma_r - gamma_s) G_rs   for s < r
//   Ainv  = (I + A)^-1                   (fp32, then stored as bf16)
//   and, for the tensor-core forward, Ainv diag(beta) and Ainv diag(beta e^gamma)
//
// The unit lower-triangular inverse is taken block-wise on 16 x 16 blocks:
// the four diagonal blocks by forward substitution (one thread per column),
// then the off-diagonal blocks one block-diagonal at a time,
//   X_ij = -X_ii (sum_{j <= m < i} A_im X_mj),
// one warp per block, the 16 x 16 x 16 products on tf32 mma.sync. Padded rows
// of a ragged chunk have beta = 0 and k = 0, so their rows of A vanish and the
// inverse is the identity there.
//
// The Gram uses warp-level mma.sync (m16n8k16): the product is 64 x 64 x 128
// per CTA, far below the size where the tcgen05 issue and round-trip costs
// pay off, and the fragments stay in registers until they are written out.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 128;
constexpr int kKP = 136;  // padded bf16 row length of the k tile (272 B: conflict-free ldmatrix)

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_1688(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct PrepSmem {
    __nv_bfloat16 k[64 * kKP];  // 17408 B
    float G[64][65];            // Gram
    float A[64][65];            // beta/decay-scaled strictly lower part
    float X[64][65];            // inverse
    float T[64][65];            // block products
    float gam[64];
    float bet[64];
};

__global__ void __launch_bounds__(kThreads) prep_tc_kernel(Dims d, const __nv_bfloat16 *__restrict__ k,
                                                           const float *__restrict__ g,
                                                           const float *__restrict__ beta,
                                                           float *__restrict__ gamma_out,
                                                           __nv_bfloat16 *__restrict__ ainv_out,
                                                           __nv_bfloat16 *__restrict__ wy_out) {
    extern __shared__ uint8_t smem_raw[];
    PrepSmem &S = *reinterpret_cast<PrepSmem *>(smem_raw);
    const int c = blockIdx.x, hq = blockIdx.y;
    const int n = chunk_owner(d, c);
    if (n < 0) return;
    const SeqRange sr = seq_range(d, n);
    const int ci = c - sr.chunk0;
    const int t0 = sr.start + ci * kChunk;
    const int len = min(kChunk, sr.len - ci * kChunk);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = d.Hv / d.Hq;
    constexpr int K = 128;

    // ---- k tile -> smem (zero rows past the end of the sequence)
    for (int e = tid; e < 64 * 16; e += kThreads) {
        const int r = e >> 4, q = e & 15;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (r < len) val = *reinterpret_cast<const uint4 *>(k + ((size_t)(t0 + r) * d.Hq + hq) * K + q * 8);
        *reinterpret_cast<uint4 *>(&S.k[r * kKP + q * 8]) = val;
    }
    __syncthreads();

    // ---- G = K K^T: warp w owns rows 16w..16w+15, all 64 columns (8 n-tiles of 8)
    {
        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        const uint32_t kbase = (uint32_t)__cvta_generic_to_shared(S.k);
        const int r0 = warp * 16;
#pragma unroll
        for (int ks = 0; ks < K / 16; ++ks) {
            const int k0 = ks * 16;
            uint32_t a[4];
            {
                const int row = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int col = k0 + (lane >> 4) * 8;
                ldmatrix_x4(a, kbase + (row * kKP + col) * 2);
            }
#pragma unroll
            for (int np = 0; np < 4; ++np) {  // pairs of n-tiles
                uint32_t b[4];
                const int row = np * 16 + (lane & 7) + (lane >> 4) * 8;
                const int col = k0 + ((lane >> 3) & 1) * 8;
                ldmatrix_x4(b, kbase + (row * kKP + col) * 2);
                mma_16816(acc[2 * np], a, b[0], b[1]);
                mma_16816(acc[2 * np + 1], a, b[2], b[3]);
            }
        }
        const int gr = lane >> 2, gc = (lane & 3) * 2;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            S.G[r0 + gr][nt * 8 + gc] = acc[nt][0];
            S.G[r0 + gr][nt * 8 + gc + 1] = acc[nt][1];
            S.G[r0 + gr + 8][nt * 8 + gc] = acc[nt][2];
            S.G[r0 + gr + 8][nt * 8 + gc + 1] = acc[nt][3];
        }
    }
    __syncthreads();

    for (int gi = 0; gi < G; ++gi) {
        const int h = hq * G + gi;
        // ---- gamma = in-chunk cumsum (two warps scan 32 rows each, then combine)
        if (tid < 64) {
            const int r = tid;
            float x = r < len ? g[(size_t)(t0 + r) * d.Hv + h] : 0.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            S.gam[r] = x;
            S.bet[r] = r < len ? beta[(size_t)(t0 + r) * d.Hv + h] : 0.f;
        }
        __syncthreads();
        if (tid >= 32 && tid < 64) S.gam[tid] += S.gam[31];
        __syncthreads();
        if (tid < len) gamma_out[(size_t)(t0 + tid) * d.Hv + h] = S.gam[tid];
        // ---- A (strictly lower), X = 0
        for (int e = tid; e < 64 * 64; e += kThreads) {
            const int r = e >> 6, s = e & 63;
            S.A[r][s] = s < r ? S.bet[r] * __expf(S.gam[r] - S.gam[s]) * S.G[r][s] : 0.f;
            S.X[r][s] = 0.f;
        }
        __syncthreads();
        // ---- diagonal 16x16 blocks: thread t -> block t/16, column t%16 (64 threads)
        if (tid < 64) {
            const int b = tid >> 4, cc = tid & 15, o = b * 16;
            float xcol[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
                for (int j = 0; j < r; ++j) acc = fmaf(-S.A[o + r][o + j], xcol[j], acc);
                xcol[r] = r < cc ? 0.f : acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) S.X[o + r][o + cc] = xcol[r];
        }
        __syncthreads();
        // ---- off-diagonal block levels: X_ij = -X_ii sum_{m=j}^{i-1} A_im X_mj.
        // One warp per block of the level; 16x16x16 products on tf32 mma.sync
        // (their rounding stays below the bf16 rounding of the stored inverse).
        for (int lvl = 1; lvl < 4; ++lvl) {
            if (warp < 4 - lvl) {
                const int i = lvl + warp, j = warp;
                const int gr = lane >> 2, gc = lane & 3;
                float t[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                for (int m = j; m < i; ++m) {
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const int ac = m * 16 + kk * 8 + gc;
                        const uint32_t a[4] = {tf32(S.A[i * 16 + gr][ac]), tf32(S.A[i * 16 + gr + 8][ac]),
                                               tf32(S.A[i * 16 + gr][ac + 4]), tf32(S.A[i * 16 + gr + 8][ac + 4])};
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
                            const int bc = j * 16 + nt * 8 + gr;
                            mma_1688(t[nt], a, tf32(S.X[m * 16 + kk * 8 + gc][bc]),
                                     tf32(S.X[m * 16 + kk * 8 + gc + 4][bc]));
                        }
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int col = j * 16 + nt * 8 + 2 * gc;
                    S.T[i * 16 + gr][col] = t[nt][0];
                    S.T[i * 16 + gr][col + 1] = t[nt][1];
                    S.T[i * 16 + gr + 8][col] = t[nt][2];
                    S.T[i * 16 + gr + 8][col + 1] = t[nt][3];
                }
                __syncwarp();
                float x[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int ac = i * 16 + kk * 8 + gc;
                    const uint32_t a[4] = {tf32(S.X[i * 16 + gr][ac]), tf32(S.X[i * 16 + gr + 8][ac]),
                                           tf32(S.X[i * 16 + gr][ac + 4]), tf32(S.X[i * 16 + gr + 8][ac + 4])};
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int bc = j * 16 + nt * 8 + gr;
                        mma_1688(x[nt], a, tf32(S.T[i * 16 + kk * 8 + gc][bc]),
                                 tf32(S.T[i * 16 + kk * 8 + gc + 4][bc]));
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int col = j * 16 + nt * 8 + 2 * gc;
                    S.X[i * 16 + gr][col] = -x[nt][0];
                    S.X[i * 16 + gr][col + 1] = -x[nt][1];
                    S.X[i * 16 + gr + 8][col] = -x[nt][2];
                    S.X[i * 16 + gr + 8][col + 1] = -x[nt][3];
                }
            }
            __syncthreads();
        }
        // ---- Ainv -> bf16 (16-byte stores); optionally the two scaled inverses
        //      Ainv diag(beta) and Ainv diag(beta e^gamma) that the forward multiplies
        //      with V and K (so it needs no elementwise pass of its own)
        if (ainv_out) {
            __nv_bfloat16 *out = ainv_out + ((size_t)c * d.Hv + h) * kChunk * kChunk;
            for (int e = tid; e < 64 * 8; e += kThreads) {
                const int r = e >> 3, q = e & 7;
                __align__(16) __nv_bfloat162 v[4];
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) v[pp] = __floats2bfloat162_rn(S.X[r][q * 8 + 2 * pp], S.X[r][q * 8 + 2 * pp + 1]);
                *reinterpret_cast<uint4 *>(out + r * 64 + q * 8) = *reinterpret_cast<uint4 *>(v);
            }
        }
        if (wy_out) {
            __nv_bfloat16 *ou = wy_out + ((size_t)c * d.Hv + h) * 2 * kChunk * kChunk;
            __nv_bfloat16 *ow = ou + kChunk * kChunk;
            for (int e = tid; e < 64 * 8; e += kThreads) {
                const int r = e >> 3, q = e & 7;
                __align__(16) __nv_bfloat162 vu[4], vw[4];
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    const int s0 = q * 8 + 2 * pp;
                    const float a0 = S.X[r][s0] * S.bet[s0], a1 = S.X[r][s0 + 1] * S.bet[s0 + 1];
                    vu[pp] = __floats2bfloat162_rn(a0, a1);
                    vw[pp] = __floats2bfloat162_rn(a0 * __expf(S.gam[s0]), a1 * __expf(S.gam[s0 + 1]));
                }
                *reinterpret_cast<uint4 *>(ou + r * 64 + q * 8) = *reinterpret_cast<uint4 *>(vu);
                *reinterpret_cast<uint4 *>(ow + r * 64 + q * 8) = *reinterpret_cast<uint4 *>(vw);
            }
        }
        __syncthreads();
    }
}

}  // namespace

bool prep_tc_supported(const FwdArgs &a) { return a.dtype == GDN_DTYPE_BF16 && a.d.K == 128; }

cudaError_t launch_prep_tc(const FwdArgs &a) {
    if (a.d.NC == 0) return cudaSuccess;
    const size_t smem = sizeof(PrepSmem);
    cudaError_t e = cudaFuncSetAttribute(prep_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.d.NC, a.d.Hq);
    prep_tc_kernel<<<grid, kThreads, smem, a.stream>>>(a.d, (const __nv_bfloat16 *)a.k, a.g, a.beta, a.gamma,
                                                       (__nv_bfloat16 *)a.ainv, (__nv_bfloat16 *)a.wy);
    return cudaGetLastError();
}

}  // namespace gdn
