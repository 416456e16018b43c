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
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace warp;

constexpr int kThreads = 256;
constexpr int kBV = 8;            // state columns per CTA
constexpr int kPLd = 132;         // row pitch (floats) of an operator in shared memory: 16-byte rows
                                  // that spread the 16-byte reads of 32 rows over all banks
constexpr int kPBytes = 128 * kPLd * 4;
constexpr size_t kSmemBytes = 2 * (size_t)kPBytes + 128 * kBV * 4 + 64;

// One CTA per (sequence, value head, 8-column slice of V). Thread t owns state row
// t % 128 and four of the slice's columns ((t / 128) * 4 ..). Each segment's 64 KB
// operator comes into shared memory by bulk copies (one per row, into 16-byte-padded
// rows) while the previous segment's product runs; at the start of its step every
// thread moves its row of it into registers, so the product reads only the state
// slice from shared memory, one 16-byte vector per row that the whole warp shares.
__global__ void __launch_bounds__(kThreads, 1) split_compose(Dims d, int nseg, bool reverse, const float *__restrict__ h0,
                                                             const float *__restrict__ seg_c,
                                                             const float *__restrict__ seg_P,
                                                             float *__restrict__ seg_h0, unsigned *status) {
    constexpr int K = 128, V = 128;
    extern __shared__ __align__(16) uint8_t smem[];
    float *Ps = reinterpret_cast<float *>(smem);                   // 2 x [K][kPLd]
    float *hs = reinterpret_cast<float *>(smem + 2 * kPBytes);     // [K][kBV]
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + 2 * kPBytes + K * kBV * 4);  // [2]
    const int n = blockIdx.x, h = blockIdx.y, c0 = blockIdx.z * kBV;
    const int tid = threadIdx.x, row = tid & (K - 1), cb = (tid >> 7) * 4;

    auto seg_off = [&](int s) { return (((size_t)n * nseg + s) * d.Hv + h) * K * V; };
    auto sidx = [&](int i) { return reverse ? nseg - 1 - i : i; };  // the i-th segment walked
    // operator of the i-th segment walked into buffer b: thread r < K copies row r
    auto fetch = [&](int i, int b) {
        const float *P = seg_P + (((size_t)n * nseg + sidx(i)) * d.Hv + h) * K * K;
        if (tid == 0) mbar_arrive_expect_tx(&bar[b], K * K * 4);
        __syncwarp();
        if (tid < K) bulk_load(smem + b * kPBytes + tid * kPLd * 4, P + (size_t)tid * K, K * 4, &bar[b]);
    };
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_barrier_init();
    }
    {
        const float *src = h0 ? h0 + ((size_t)n * d.Hv + h) * K * V : nullptr;
        float *dst = seg_h0 + seg_off(sidx(0));
        for (int e = tid; e < K * kBV; e += kThreads) {
            const int r = e / kBV, c = e % kBV;
            const float x = src ? src[(size_t)r * V + c0 + c] : 0.f;
            hs[r * kBV + c] = x;
            dst[(size_t)r * V + c0 + c] = x;
        }
    }
    __syncthreads();  // barriers initialised, state slice in place
    if (nseg > 1) fetch(0, 0);
    float4 cn = make_float4(0.f, 0.f, 0.f, 0.f);  // c of the coming step
    if (nseg > 1) cn = *reinterpret_cast<const float4 *>(seg_c + seg_off(sidx(0)) + (size_t)row * V + c0 + cb);
    bool ok = true;
    int issued = nseg > 1 ? 1 : 0;
    for (int i = 0; i + 1 < nseg; ++i) {
        const int b = i & 1;
        // this step's operator has landed (bounded wait; the result is made uniform)
        bool got = true;
        {
            const uint32_t a = smem_u32(&bar[b]);
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(a, (i >> 1) & 1))
                if (globaltimer() - t0 > kWaitNs) {
                    got = false;
                    break;
                }
        }
        ok = __syncthreads_and(got) != 0;
        if (!ok) break;
        float pr[K];
        {
            const float4 *src = reinterpret_cast<const float4 *>(Ps + b * (kPBytes / 4) + row * kPLd);
#pragma unroll
            for (int j = 0; j < K / 4; ++j) {
                const float4 v = src[j];
                pr[4 * j] = v.x, pr[4 * j + 1] = v.y, pr[4 * j + 2] = v.z, pr[4 * j + 3] = v.w;
            }
        }
        __syncthreads();  // every thread holds its row: the other buffer (read a step ago) can refill
        if (i + 2 < nseg) {
            fetch(i + 1, b ^ 1);
            ++issued;
        }
        float4 acc = cn;
        if (i + 2 < nseg) cn = *reinterpret_cast<const float4 *>(seg_c + seg_off(sidx(i + 1)) + (size_t)row * V + c0 + cb);
        const float4 *hk = reinterpret_cast<const float4 *>(hs + cb);
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const float4 x = hk[k * (kBV / 4)];
            acc.x = fmaf(pr[k], x.x, acc.x);
            acc.y = fmaf(pr[k], x.y, acc.y);
            acc.z = fmaf(pr[k], x.z, acc.z);
            acc.w = fmaf(pr[k], x.w, acc.w);
        }
        __syncthreads();  // every thread is done reading the state slice
        *reinterpret_cast<float4 *>(hs + row * kBV + cb) = acc;
        *reinterpret_cast<float4 *>(seg_h0 + seg_off(sidx(i + 1)) + (size_t)row * V + c0 + cb) = acc;
    }
    if (!ok) {
        if (tid == 0) set_status(status, GDN_ERR_TIMEOUT);
        // let the copies still in flight land (bounded) before the CTA's shared memory goes away
        if (tid == 0) {
            const uint64_t t0 = globaltimer();
            for (int u = 0; u < issued; ++u)
                while (!mbar_try_wait(smem_u32(&bar[u & 1]), (u >> 1) & 1) && globaltimer() - t0 < kWaitNs) {
                }
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_split_compose(const FwdArgs &a) {
    const Dims &d = a.d;
    if (d.N == 0 || a.nseg < 1) return cudaSuccess;
    if (d.K != 128 || d.V != 128 || !a.seg_c || !a.seg_P || !a.seg_h0) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(split_compose, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    split_compose<<<dim3(d.N, d.Hv, d.V / kBV), kThreads, kSmemBytes, a.stream>>>(d, a.nseg, false, a.h0, a.seg_c,
                                                                                 a.seg_P, (float *)a.seg_h0, a.status);
    return cudaGetLastError();
}

cudaError_t launch_split_compose_bwd(const Dims &d, int nseg, const float *dht, const float *seg_r,
                                     const float *seg_Q, float *seg_dh, unsigned *status, cudaStream_t stream) {
    if (d.N == 0 || nseg < 1) return cudaSuccess;
    if (d.K != 128 || d.V != 128 || !seg_r || !seg_Q || !seg_dh) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(split_compose, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    split_compose<<<dim3(d.N, d.Hv, d.V / kBV), kThreads, kSmemBytes, stream>>>(d, nseg, true, dht, seg_r, seg_Q,
                                                                               seg_dh, status);
    return cudaGetLastError();
}

}  // namespace gdn
