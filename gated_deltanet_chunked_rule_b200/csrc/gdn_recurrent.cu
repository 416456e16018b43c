// gdn_recurrent.cu -- token-by-token (decode) step of the gated delta rule:
// the same recurrence as the chunked path, for a few tokens per sequence, with
// the state read once and written once per call.
//
// Per sequence n, value head h (qk head hq = h / (Hv/Hq)) and token t, with the
// state as h = S^T [K, V]:
//
//   a = h^T k,   b = h^T q,   e = e^{g}
//   d = beta (v - e a)                       (the delta-rule correction of v)
//   h <- e h + k d^T                         (= e^g (I - beta k k^T) h + beta k v^T)
//   o = scale h^T q = scale (e b + d (k.q))
//
// One CTA per (sequence, value head, 32-column slice of V); warp w holds state
// rows 32w .. 32w+31 and lane l column l of the slice, so every state row moves
// as one 128-byte transaction and the state stays in registers across the
// call's tokens. The column sums a, b and the scalar k.q reduce over the warps
// through shared memory in a fixed order. Memory-bound: each call moves the
// state slice (K x 32 fp32) in and out once.
#include <cstddef>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kBV = 32;

template <typename Tin>
__device__ __forceinline__ float ld_in(const Tin *p) {
    return to_f32(*p);
}

template <typename Tin, int K>
__global__ void __launch_bounds__(K)
recurrent_kernel(Dims d, const int *__restrict__ cu, const Tin *__restrict__ q, const Tin *__restrict__ k,
                 const Tin *__restrict__ v, const float *__restrict__ g, const float *__restrict__ beta,
                 const float *__restrict__ h0, Tin *__restrict__ o, float *__restrict__ final_state,
                 unsigned *status) {
    constexpr int kWarps = K / 32;
    __shared__ float ks[K], qs[K];
    __shared__ float red[2][kWarps][kBV], kq[kWarps];
    const int n = blockIdx.x, h = blockIdx.y, c0 = blockIdx.z * kBV;
    const int hq = h / (d.Hv / d.Hq);
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int V = d.V;

    // tokens of sequence n in the flattened [B*T] axis
    int t_begin, t_len;
    if (cu) {
        const int a = cu[n], b = cu[n + 1];
        if (a < 0 || b < a || b > d.T_total) {  // inconsistent device copy: no work, no out-of-range access
            if (tid == 0) set_status(status, GDN_ERR_DEVICE_ARG);
            return;
        }
        t_begin = a, t_len = b - a;
    } else {
        t_begin = n * d.T, t_len = d.T;
    }

    // state slice: rows 32w + i (i < 32), column c0 + lane
    float hr[32];
    {
        const float *src = h0 ? h0 + ((size_t)n * d.Hv + h) * K * V + c0 + lane : nullptr;
#pragma unroll
        for (int i = 0; i < 32; ++i) hr[i] = src ? src[(size_t)(32 * w + i) * V] : 0.f;
    }
    const float scale = d.scale;
    for (int t = 0; t < t_len; ++t) {
        const size_t tok = (size_t)(t_begin + t);
        ks[tid] = ld_in(k + (tok * d.Hq + hq) * K + tid);
        qs[tid] = ld_in(q + (tok * d.Hq + hq) * K + tid);
        const float gt = g[tok * d.Hv + h], bt = beta[tok * d.Hv + h];
        const float vc = ld_in(v + (tok * d.Hv + h) * V + c0 + lane);
        __syncthreads();
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            a = fmaf(ks[32 * w + i], hr[i], a);
            b = fmaf(qs[32 * w + i], hr[i], b);
        }
        float p = ks[tid] * qs[tid];  // this warp's part of k.q
#pragma unroll
        for (int s = 16; s > 0; s >>= 1) p += __shfl_xor_sync(0xffffffffu, p, s);
        red[0][w][lane] = a;
        red[1][w][lane] = b;
        if (lane == 0) kq[w] = p;
        __syncthreads();
        a = 0.f, b = 0.f;
        float kqs = 0.f;
#pragma unroll
        for (int j = 0; j < kWarps; ++j) a += red[0][j][lane], b += red[1][j][lane], kqs += kq[j];
        const float e = __expf(gt);
        const float dc = bt * (vc - e * a);
#pragma unroll
        for (int i = 0; i < 32; ++i) hr[i] = fmaf(e, hr[i], ks[32 * w + i] * dc);
        if (w == 0) o[(tok * d.Hv + h) * V + c0 + lane] = from_f32<Tin>(scale * fmaf(e, b, dc * kqs));
        __syncthreads();  // ks, qs, red reused by the next token
    }
    if (final_state) {
        float *dst = final_state + ((size_t)n * d.Hv + h) * K * V + c0 + lane;
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[(size_t)(32 * w + i) * V] = hr[i];
    }
}

template <typename Tin>
cudaError_t dispatch(const RecurrentArgs &a) {
    const Dims &d = a.d;
    const dim3 grid(d.N, d.Hv, d.V / kBV);
    if (d.K == 128)
        recurrent_kernel<Tin, 128><<<grid, 128, 0, a.stream>>>(d, a.cu, (const Tin *)a.q, (const Tin *)a.k,
                                                                (const Tin *)a.v, a.g, a.beta, a.h0, (Tin *)a.o,
                                                                a.final_state, a.status);
    else
        recurrent_kernel<Tin, 64><<<grid, 64, 0, a.stream>>>(d, a.cu, (const Tin *)a.q, (const Tin *)a.k,
                                                              (const Tin *)a.v, a.g, a.beta, a.h0, (Tin *)a.o,
                                                              a.final_state, a.status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_recurrent(const RecurrentArgs &a) {
    if (a.d.N == 0) return cudaSuccess;
    if ((a.d.K != 64 && a.d.K != 128) || a.d.V % kBV) return cudaErrorInvalidValue;
    return a.dtype == GDN_DTYPE_BF16 ? dispatch<__nv_bfloat16>(a) : dispatch<float>(a);
}

}  // namespace gdn
