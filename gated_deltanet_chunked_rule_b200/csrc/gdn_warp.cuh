// gdn_warp.cuh -- helpers shared by the warp-specialised kernels: bounded
// waits, release/acquire hand-over counters between warp roles, named
// barriers over one role, warp-level bf16 tensor-core MMAs (mma.sync) with
// their ldmatrix fragment loads, and host-side TMA tensor-map encoding.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace gdn {
namespace warp {

using sm100::smem_u32;

// One wall-clock budget for every wait inside a CTA (2 s of globaltimer).
constexpr uint64_t kWaitNs = 2000000000ull;

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded mbarrier wait; false if it expired (limit_ns of globaltimer, checked
// every 1024 polls) or the CTA is aborting.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         uint64_t limit_ns = kWaitNs) {
    const uint32_t a = smem_u32(bar);
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        if (sm100::mbar_try_wait(a, parity)) return true;
        if ((i & 1023u) == 0) {
            if (*abort_flag) return false;
            const uint64_t t = globaltimer();
            if (i == 0) t0 = t;
            else if (t - t0 > limit_ns) return false;
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

// Bounded wait until *ctr >= need; false if it expired or the CTA is aborting.
// Within a warp role one thread polls, and a named barrier passes the result on
// (role_sync_and): every poll is a shared-memory load.
__device__ __forceinline__ bool wait_ge(const uint32_t *ctr, uint32_t need, volatile int *abort_flag,
                                        uint64_t limit_ns = kWaitNs) {
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        if (ld_acquire(ctr) >= need) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            const uint64_t t = globaltimer();
            if (i == 0) t0 = t;
            else if (t - t0 > limit_ns) return false;
        }
    }
}

// Named barrier over kCount threads (one warp role) that also ANDs a predicate across them.
template <int kCount>
__device__ __forceinline__ bool role_sync_and(int id, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "n"(kCount)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&u);
    return __bfloat1622float2(v);
}

// Per-access shared-memory stores and fragment loads carry no "memory"
// clobber so the compiler may overlap them; ordering across warps comes from
// barriers, fences and release/acquire statements, which do clobber memory.
__device__ __forceinline__ void st_shared_b32(uint32_t addr, uint32_t a) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a));
}
__device__ __forceinline__ void st_shared_v2f(uint32_t addr, float a, float b) {
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b));
}
__device__ __forceinline__ void st_shared_v4f(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d));
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d));
}
__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
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

// Stores four 8x8 bf16 matrices, each transposed: lane i of matrix q's lane
// group (lanes 8q .. 8q+7) gives the address of memory row i, which receives
// column i of the fragment matrix held in register r[q] (the m16n8 accumulator
// layout: lane l holds row l/4, columns 2(l%4) and 2(l%4)+1).
__device__ __forceinline__ void stsm_x4_t(uint32_t addr, const uint32_t (&r)[4]) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]));
}

// The same without the transpose: memory row i of matrix q receives row i of
// the fragment matrix in r[q].
__device__ __forceinline__ void stsm_x4(uint32_t addr, const uint32_t (&r)[4]) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3]));
}

// Named barrier over kCount threads.
template <int kCount>
__device__ __forceinline__ void named_sync(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kCount) : "memory");
}

// D (16 x 8, fp32) += A (16 x 16, bf16, row) * B (16 x 8, bf16, col).
__device__ __forceinline__ void hmma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16 tiles, row-major with 16-byte chunks XOR-permuted by (row % 8) so that
// ldmatrix over 8 consecutive rows touches 8 distinct bank groups.
struct Tile {
    uint32_t base;
    int pitch;  // bytes per row
};
__device__ __forceinline__ uint32_t toff(const Tile &t, int row, int col) {
    return t.base + row * t.pitch + ((((col >> 3) ^ (row & 7))) << 4) + (col & 7) * 2;
}

// C (16 x 8 NT) += A (16 x kdim) B (kdim x 8 NT) on one warp.
// A_T: A stored [k][m] (read transposed); B_KN: B stored [k][n] (else [n][k]).
template <int NT, bool A_T, bool B_KN>
__device__ __forceinline__ void wgemm(float (&c)[NT][4], const Tile &A, const Tile &B, int m0, int n0, int kdim,
                                      int lane) {
    const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll 2
    for (int k0 = 0; k0 < kdim; k0 += 16) {
        uint32_t a[4];
        if (!A_T) ldsm_x4(a, toff(A, m0 + r8 + (mi & 1) * 8, k0 + (mi >> 1) * 8));
        else ldsm_x4_t(a, toff(A, k0 + (mi >> 1) * 8 + r8, m0 + (mi & 1) * 8));
#pragma unroll
        for (int j = 0; j < NT; j += 2) {
            uint32_t b[4];
            if (!B_KN) ldsm_x4(b, toff(B, n0 + j * 8 + (mi >> 1) * 8 + r8, k0 + (mi & 1) * 8));
            else ldsm_x4_t(b, toff(B, k0 + (mi & 1) * 8 + r8, n0 + j * 8 + (mi >> 1) * 8));
            hmma(c[j], a, b[0], b[1]);
            hmma(c[j + 1], a, b[2], b[3]);
        }
    }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
// 4-byte asynchronous copy global -> shared (completion tracked by cp.async groups or,
// with cp_async_mbar_arrive, by an mbarrier).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// The mbarrier's current phase also waits for every cp.async this thread issued
// before: its pending count is raised now and lowered when those copies land.
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_older() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// rows [0, rows) of a bf16 matrix with `cols` columns, global row stride `ld` elements;
// rows >= valid are zero-filled.
template <int kThreads>
__device__ __forceinline__ void load_tile(const Tile &t, const __nv_bfloat16 *src, size_t ld, int rows, int cols,
                                          int valid, int tid) {
    const int cpr = cols / 8;
    for (int e = tid; e < rows * cpr; e += kThreads) {
        const int r = e / cpr, ch = e % cpr;
        const bool ok = r < valid;
        cp_async16(toff(t, r, ch * 8), src + (ok ? (size_t)r * ld + ch * 8 : 0), ok);
    }
}

__device__ __forceinline__ float2 ld_pair(const Tile &t, int row, int col) {
    uint32_t u;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(u) : "r"(toff(t, row, col)));
    return unpack_bf16(u);
}

// ------------------------------------------------------------------ host side
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// bf16 tiled tensor map (rank 2 or 3), zero fill out of bounds.
inline bool make_bf16_map(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                          const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle sw) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace warp
}  // namespace gdn
