// gdn_simt.cu -- CUDA-core (fp32 FMA) kernels of the chunked gated delta rule.
//
// This is the full-precision instantiation of the chunk algorithm: every
// contraction runs in fp32 on CUDA cores. It serves fp32 problems (where the
// bf16 tensor-core operands of the fast path would cost more accuracy than
// fp32 inputs allow) and any dtype when GDN_IMPL=simt is set.
//
// Kernels:
//   prep_simt   one CTA per (chunk, value head): in-chunk cumsum of g, the
//               beta-scaled decay-masked Gram A, and Ainv = (I + A)^-1 by
//               column-parallel forward substitution.
//   fwd_simt    one CTA per (sequence, value head, 32-column slice of V):
//               walks the chunks of its sequence in order, carrying the fp32
//               state slice h[:, slice] in shared memory, and writes o and the
//               final state (and, for the backward, each chunk's entry state
//               and Delta).
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kBV = 32;  // state columns per CTA in fwd_simt

template <typename TA> __device__ __forceinline__ void store_a(TA *p, float x) { *p = from_f32<TA>(x); }

// ---------------------------------------------------------------- prep
template <typename Tin, typename TA, int K>
__global__ void __launch_bounds__(kThreads) prep_simt(Dims d, const Tin *__restrict__ k,
                                                      const float *__restrict__ g,
                                                      const float *__restrict__ beta,
                                                      float *__restrict__ gamma_out,
                                                      TA *__restrict__ ainv_out,
                                                      __nv_bfloat16 *__restrict__ wy_out) {
    extern __shared__ float smem[];
    float *ks = smem;                        // [64][K+1]
    float *A = ks + kChunk * (K + 1);        // [64][65]
    float *X = A + kChunk * 65;              // [64][65]
    float *gam = X + kChunk * 65;            // [64]
    float *bet = gam + kChunk;               // [64]

    const int c = blockIdx.x, h = blockIdx.y;
    const int n = chunk_owner(d, c);
    if (n < 0) return;
    const SeqRange sr = seq_range(d, n);
    const int i = c - sr.chunk0;
    const int t0 = sr.start + i * kChunk;
    const int len = min(kChunk, sr.len - i * kChunk);
    const int hq = h / (d.Hv / d.Hq);
    const int tid = threadIdx.x;

    for (int e = tid; e < kChunk * K; e += kThreads) {
        const int r = e / K, j = e % K;
        ks[r * (K + 1) + j] = r < len ? to_f32(k[((size_t)(t0 + r) * d.Hq + hq) * K + j]) : 0.f;
    }
    if (tid < kChunk) {
        gam[tid] = tid < len ? g[(size_t)(t0 + tid) * d.Hv + h] : 0.f;
        bet[tid] = tid < len ? beta[(size_t)(t0 + tid) * d.Hv + h] : 0.f;
    }
    __syncthreads();
    if (tid == 0) {
        float s = 0.f;
        for (int r = 0; r < kChunk; ++r) { s += gam[r]; gam[r] = s; }
    }
    __syncthreads();
    if (tid < len) gamma_out[(size_t)(t0 + tid) * d.Hv + h] = gam[tid];
    for (int e = tid; e < kChunk * kChunk; e += kThreads) {
        const int r = e / kChunk, s = e % kChunk;
        float a = 0.f;
        if (s < r) {
            float dot = 0.f;
#pragma unroll 8
            for (int j = 0; j < K; ++j) dot = fmaf(ks[r * (K + 1) + j], ks[s * (K + 1) + j], dot);
            a = bet[r] * expf(gam[r] - gam[s]) * dot;
        }
        A[r * 65 + s] = a;
    }
    __syncthreads();
    // Column col of X = (I + A)^-1: X[col][col] = 1, X[r][col] = -sum_{col<=j<r} A[r][j] X[j][col].
    if (tid < kChunk) {
        const int col = tid;
        for (int r = 0; r < kChunk; ++r) {
            float x;
            if (r < col) x = 0.f;
            else if (r == col) x = 1.f;
            else {
                float acc = 0.f;
                for (int j = col; j < r; ++j) acc = fmaf(A[r * 65 + j], X[j * 65 + col], acc);
                x = -acc;
            }
            X[r * 65 + col] = x;
        }
    }
    __syncthreads();
    TA *out = ainv_out + ((size_t)c * d.Hv + h) * kChunk * kChunk;
    for (int e = tid; e < kChunk * kChunk; e += kThreads)
        store_a(out + e, X[(e / kChunk) * 65 + (e % kChunk)]);
    if (wy_out) {  // Ainv diag(beta), Ainv diag(beta e^gamma) for the tensor-core kernels
        __nv_bfloat16 *ou = wy_out + ((size_t)c * d.Hv + h) * 2 * kChunk * kChunk, *ow = ou + kChunk * kChunk;
        for (int e = tid; e < kChunk * kChunk; e += kThreads) {
            const int r = e / kChunk, s = e % kChunk;
            const float a = X[r * 65 + s] * bet[s];
            ou[e] = __float2bfloat16_rn(a);
            ow[e] = __float2bfloat16_rn(a * expf(gam[s]));
        }
    }
}

// ---------------------------------------------------------------- forward
template <int K>
constexpr size_t fwd_smem_floats() {
    return (size_t)K * kBV                 // hs
           + 3 * (size_t)kChunk * (K + 1)  // qs, ks, ws
           + 2 * (size_t)kChunk * 65       // Ai, P
           + 2 * (size_t)kChunk * (kBV + 1)  // vs, us
           + 3 * kChunk;                   // gam, bet, egam
}

template <typename Tin, typename TA, int K, int V>
__global__ void __launch_bounds__(kThreads) fwd_simt(
    Dims d, const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
    const float *__restrict__ gamma, const float *__restrict__ beta, const TA *__restrict__ ainv,
    const float *__restrict__ h0, Tin *__restrict__ o, float *__restrict__ final_state,
    float *__restrict__ h_chunks, float *__restrict__ delta_out) {
    extern __shared__ float smem[];
    float *hs = smem;                          // [K][kBV]
    float *qs = hs + K * kBV;                  // [64][K+1]
    float *ks = qs + kChunk * (K + 1);         // [64][K+1]
    float *ws = ks + kChunk * (K + 1);         // [64][K+1]
    float *Ai = ws + kChunk * (K + 1);         // [64][65]
    float *P = Ai + kChunk * 65;               // [64][65]
    float *vs = P + kChunk * 65;               // [64][kBV+1]
    float *us = vs + kChunk * (kBV + 1);       // [64][kBV+1]  u, then Delta
    float *gam = us + kChunk * (kBV + 1);      // [64]
    float *bet = gam + kChunk;                 // [64]
    float *egam = bet + kChunk;                // [64] exp(gamma)

    const int n = blockIdx.x, h = blockIdx.y, c0 = blockIdx.z * kBV;
    const int hq = h / (d.Hv / d.Hq);
    const int tid = threadIdx.x;
    const SeqRange sr = seq_range(d, n);
    const int nchunks = (sr.len + kChunk - 1) / kChunk;

    for (int e = tid; e < K * kBV; e += kThreads) {
        const int j = e / kBV, cc = e % kBV;
        hs[e] = h0 ? h0[(((size_t)n * d.Hv + h) * K + j) * V + c0 + cc] : 0.f;
    }
    for (int ci = 0; ci < nchunks; ++ci) {
        const int cg = sr.chunk0 + ci;
        const int t0 = sr.start + ci * kChunk;
        const int len = min(kChunk, sr.len - ci * kChunk);
        __syncthreads();
        if (h_chunks) {
            float *hc = h_chunks + ((size_t)cg * d.Hv + h) * K * V;
            for (int e = tid; e < K * kBV; e += kThreads)
                hc[(size_t)(e / kBV) * V + c0 + (e % kBV)] = hs[e];
        }
        for (int e = tid; e < kChunk * K; e += kThreads) {
            const int r = e / K, j = e % K;
            const size_t off = ((size_t)(t0 + r) * d.Hq + hq) * K + j;
            qs[r * (K + 1) + j] = r < len ? to_f32(q[off]) : 0.f;
            ks[r * (K + 1) + j] = r < len ? to_f32(k[off]) : 0.f;
        }
        for (int e = tid; e < kChunk * kBV; e += kThreads) {
            const int r = e / kBV, cc = e % kBV;
            vs[r * (kBV + 1) + cc] =
                r < len ? to_f32(v[((size_t)(t0 + r) * d.Hv + h) * V + c0 + cc]) : 0.f;
        }
        const TA *Ag = ainv + ((size_t)cg * d.Hv + h) * kChunk * kChunk;
        for (int e = tid; e < kChunk * kChunk; e += kThreads)
            Ai[(e / kChunk) * 65 + (e % kChunk)] = to_f32(Ag[e]);
        if (tid < kChunk) {
            gam[tid] = gamma[(size_t)(t0 + min(tid, len - 1)) * d.Hv + h];
            bet[tid] = tid < len ? beta[(size_t)(t0 + tid) * d.Hv + h] : 0.f;
        }
        __syncthreads();
        if (tid < kChunk) egam[tid] = expf(gam[tid]);
        __syncthreads();
        // w = Ainv diag(beta e^gamma) K ; u = Ainv diag(beta) V ; P = M o (Q K^T)
        for (int e = tid; e < kChunk * K; e += kThreads) {
            const int r = e / K, j = e % K;
            float acc = 0.f;
            for (int s = 0; s <= r; ++s) acc = fmaf(Ai[r * 65 + s] * bet[s] * egam[s], ks[s * (K + 1) + j], acc);
            ws[r * (K + 1) + j] = acc;
        }
        for (int e = tid; e < kChunk * kBV; e += kThreads) {
            const int r = e / kBV, cc = e % kBV;
            float acc = 0.f;
            for (int s = 0; s <= r; ++s) acc = fmaf(Ai[r * 65 + s] * bet[s], vs[s * (kBV + 1) + cc], acc);
            us[r * (kBV + 1) + cc] = acc;
        }
        for (int e = tid; e < kChunk * kChunk; e += kThreads) {
            const int r = e / kChunk, s = e % kChunk;
            float acc = 0.f;
            if (s <= r) {
#pragma unroll 8
                for (int j = 0; j < K; ++j) acc = fmaf(qs[r * (K + 1) + j], ks[s * (K + 1) + j], acc);
                acc *= expf(gam[r] - gam[s]);
            }
            P[r * 65 + s] = acc;
        }
        __syncthreads();
        // Delta = u - w h (in place over u); qh = Q h kept in registers for o.
        constexpr int kPer = kChunk * kBV / kThreads;  // 8
        float qh[kPer];
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int e = tid + m * kThreads;
            const int r = e / kBV, cc = e % kBV;
            float acc_w = 0.f, acc_q = 0.f;
#pragma unroll 8
            for (int j = 0; j < K; ++j) {
                const float hv = hs[j * kBV + cc];
                acc_w = fmaf(ws[r * (K + 1) + j], hv, acc_w);
                acc_q = fmaf(qs[r * (K + 1) + j], hv, acc_q);
            }
            us[r * (kBV + 1) + cc] -= acc_w;
            qh[m] = acc_q;
        }
        __syncthreads();
        if (delta_out) {
            for (int e = tid; e < kChunk * kBV; e += kThreads) {
                const int r = e / kBV, cc = e % kBV;
                if (r < len) delta_out[((size_t)(t0 + r) * d.Hv + h) * V + c0 + cc] = us[r * (kBV + 1) + cc];
            }
        }
        // o = scale (e^gamma Q h + P Delta)
        if (o) {
#pragma unroll
            for (int m = 0; m < kPer; ++m) {
                const int e = tid + m * kThreads;
                const int r = e / kBV, cc = e % kBV;
                float acc = egam[r] * qh[m];
                for (int s = 0; s <= r; ++s) acc = fmaf(P[r * 65 + s], us[s * (kBV + 1) + cc], acc);
                if (r < len) o[((size_t)(t0 + r) * d.Hv + h) * V + c0 + cc] = from_f32<Tin>(d.scale * acc);
            }
        }
        // h' = e^{gamma_C} h + Ktil^T Delta
        const float gl = gam[kChunk - 1];
        const float eC = expf(gl);
        for (int e = tid; e < K * kBV; e += kThreads) {
            const int j = e / kBV, cc = e % kBV;
            float acc = 0.f;
            for (int s = 0; s < len; ++s)
                acc = fmaf(expf(gl - gam[s]) * ks[s * (K + 1) + j], us[s * (kBV + 1) + cc], acc);
            hs[e] = fmaf(eC, hs[e], acc);
        }
    }
    __syncthreads();
    if (final_state) {
        for (int e = tid; e < K * kBV; e += kThreads) {
            const int j = e / kBV, cc = e % kBV;
            final_state[(((size_t)n * d.Hv + h) * K + j) * V + c0 + cc] = hs[e];
        }
    }
}

template <typename Tin, typename TA, int K>
cudaError_t prep_dispatch(const FwdArgs &a) {
    const size_t smem = sizeof(float) * ((size_t)kChunk * (K + 1) + 2 * kChunk * 65 + 2 * kChunk);
    auto kern = prep_simt<Tin, TA, K>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.d.NC, a.d.Hv);
    kern<<<grid, kThreads, smem, a.stream>>>(a.d, (const Tin *)a.k, a.g, a.beta, a.gamma, (TA *)a.ainv,
                                             (__nv_bfloat16 *)a.wy);
    return cudaGetLastError();
}

template <typename Tin, typename TA, int K, int V>
cudaError_t fwd_dispatch(const FwdArgs &a) {
    const size_t smem = sizeof(float) * fwd_smem_floats<K>();
    auto kern = fwd_simt<Tin, TA, K, V>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.d.N, a.d.Hv, V / kBV);
    kern<<<grid, kThreads, smem, a.stream>>>(a.d, (const Tin *)a.q, (const Tin *)a.k, (const Tin *)a.v,
                                             a.gamma, a.beta, (const TA *)a.ainv, a.h0, (Tin *)a.o,
                                             a.final_state, a.h_chunks, a.delta);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prep_simt(const FwdArgs &a) {
    if (a.d.NC == 0) return cudaSuccess;
    if (a.dtype == GDN_DTYPE_F32)
        return a.d.K == 64 ? prep_dispatch<float, float, 64>(a) : prep_dispatch<float, float, 128>(a);
    return a.d.K == 64 ? prep_dispatch<__nv_bfloat16, __nv_bfloat16, 64>(a)
                       : prep_dispatch<__nv_bfloat16, __nv_bfloat16, 128>(a);
}

cudaError_t launch_fwd_simt(const FwdArgs &a) {
    if (a.d.N == 0) return cudaSuccess;
    const int kv = (a.d.K == 64 ? 0 : 2) + (a.d.V == 64 ? 0 : 1);
    if (a.dtype == GDN_DTYPE_F32) {
        switch (kv) {
            case 0: return fwd_dispatch<float, float, 64, 64>(a);
            case 1: return fwd_dispatch<float, float, 64, 128>(a);
            case 2: return fwd_dispatch<float, float, 128, 64>(a);
            default: return fwd_dispatch<float, float, 128, 128>(a);
        }
    }
    switch (kv) {
        case 0: return fwd_dispatch<__nv_bfloat16, __nv_bfloat16, 64, 64>(a);
        case 1: return fwd_dispatch<__nv_bfloat16, __nv_bfloat16, 64, 128>(a);
        case 2: return fwd_dispatch<__nv_bfloat16, __nv_bfloat16, 128, 64>(a);
        default: return fwd_dispatch<__nv_bfloat16, __nv_bfloat16, 128, 128>(a);
    }
}

}  // namespace gdn
