// gdn_split.cu -- composition step of the intra-GPU sequence split.
//
// A segment of chunks maps its start state h to P h + c, where c is the
// segment's end state from a zero start and P the product of its chunks'
// transition operators e^{gamma_C} I - K^T diag(e^{gamma_C - gamma}) w (each
// chunk's h' = e^{gamma_C} h + K^T diag(e^{gamma_C - gamma}) (u - w h)). The
// segment pass of the forward kernel produces (c, P) for all segments at once;
// this kernel walks each sequence's segments in order,
//
//   h_start(0) = h0,   h_start(s + 1) = P_s h_start(s) + c_s,
//
// exactly (fp32, no truncation), and the output pass then restarts every
// segment from its h_start. The backward split composes the same way in the
// other direction: a segment maps the gradient at its end to Q dh + r (Q the
// transposed product), and the walk starts at the last segment from dht. This is the "gate-driven intra-card context
// parallelism" of the FlashQLA resource digest (section 三, first key feature):
// the decay gates make P shrink geometrically, but nothing here relies on it.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256, kBV = 32;

// One CTA per (sequence, value head, 32-column slice of V).
template <int K, int V>
__global__ void __launch_bounds__(kThreads) split_compose(Dims d, int nseg, bool reverse, const float *__restrict__ h0,
                                                          const float *__restrict__ seg_c,
                                                          const float *__restrict__ seg_P,
                                                          float *__restrict__ seg_h0) {
    extern __shared__ float smem[];
    float *Ps = smem;                // [K][K + 1]
    float *hs = Ps + K * (K + 1);    // [K][kBV + 1]
    const int n = blockIdx.x, h = blockIdx.y, c0 = blockIdx.z * kBV;
    const int tid = threadIdx.x;
    constexpr int kRows = kThreads / 2, kCols = kBV / 2;  // thread: row tid / 2, 16 columns
    static_assert(K == kRows, "one thread pair per state row");
    const int row = tid >> 1, cb = (tid & 1) * kCols;

    auto seg_off = [&](int s) { return (((size_t)n * nseg + s) * d.Hv + h) * K * V; };
    auto sidx = [&](int i) { return reverse ? nseg - 1 - i : i; };  // the i-th segment walked
    {
        const float *src = h0 ? h0 + ((size_t)n * d.Hv + h) * K * V : nullptr;
        float *dst = seg_h0 + seg_off(sidx(0));
        for (int e = tid; e < K * kBV; e += kThreads) {
            const int r = e / kBV, c = e % kBV;
            const float x = src ? src[(size_t)r * V + c0 + c] : 0.f;
            hs[r * (kBV + 1) + c] = x;
            dst[(size_t)r * V + c0 + c] = x;
        }
    }
    for (int i = 0; i + 1 < nseg; ++i) {
        const int s = sidx(i);
        const float *P = seg_P + (((size_t)n * nseg + s) * d.Hv + h) * K * K;
        for (int e = tid; e < K * K; e += kThreads) Ps[(e / K) * (K + 1) + e % K] = P[e];
        __syncthreads();
        float acc[kCols];
        const float *c = seg_c + seg_off(s) + (size_t)row * V + c0 + cb;
#pragma unroll
        for (int j = 0; j < kCols; ++j) acc[j] = c[j];
#pragma unroll 4
        for (int k = 0; k < K; ++k) {
            const float a = Ps[row * (K + 1) + k];
#pragma unroll
            for (int j = 0; j < kCols; ++j) acc[j] = fmaf(a, hs[k * (kBV + 1) + cb + j], acc[j]);
        }
        __syncthreads();  // every thread is done reading hs and Ps
        float *dst = seg_h0 + seg_off(sidx(i + 1)) + (size_t)row * V + c0 + cb;
#pragma unroll
        for (int j = 0; j < kCols; ++j) {
            hs[row * (kBV + 1) + cb + j] = acc[j];
            dst[j] = acc[j];
        }
    }
}

}  // namespace

cudaError_t launch_split_compose(const FwdArgs &a) {
    const Dims &d = a.d;
    if (d.N == 0 || a.nseg < 1) return cudaSuccess;
    if (d.K != 128 || d.V != 128 || !a.seg_c || !a.seg_P || !a.seg_h0) return cudaErrorInvalidValue;
    const size_t smem = sizeof(float) * (128 * 129 + 128 * (kBV + 1));
    auto kern = split_compose<128, 128>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(d.N, d.Hv, d.V / kBV), kThreads, smem, a.stream>>>(d, a.nseg, false, a.h0, a.seg_c, a.seg_P,
                                                                    (float *)a.seg_h0);
    return cudaGetLastError();
}

cudaError_t launch_split_compose_bwd(const Dims &d, int nseg, const float *dht, const float *seg_r,
                                     const float *seg_Q, float *seg_dh, cudaStream_t stream) {
    if (d.N == 0 || nseg < 1) return cudaSuccess;
    if (d.K != 128 || d.V != 128 || !seg_r || !seg_Q || !seg_dh) return cudaErrorInvalidValue;
    const size_t smem = sizeof(float) * (128 * 129 + 128 * (kBV + 1));
    auto kern = split_compose<128, 128>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(d.N, d.Hv, d.V / kBV), kThreads, smem, stream>>>(d, nseg, true, dht, seg_r, seg_Q, seg_dh);
    return cudaGetLastError();
}

}  // namespace gdn
