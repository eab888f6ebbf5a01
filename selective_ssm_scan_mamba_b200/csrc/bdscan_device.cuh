// Device helpers for the bdscan kernels (sm_100a).
//
// Every arithmetic step on the scan path is written with explicit
// round-to-nearest intrinsics (__fmul_rn, __fmaf_rn, __ffma2_rn, ...), which
// the compiler may not contract or reorder. The forward recurrence therefore
// produces the same bits in every kernel variant that runs it, which is what
// makes a committed cache equal, bit for bit, the state of a one-shot scan.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bdk {

constexpr float kLog2e = 1.4426950408889634f;

// 2^x on the special-function unit (MUFU.EX2), subnormal results flushed to 0.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 1/x on the special-function unit.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void from_f32(float v, float &o) { o = v; }
__device__ __forceinline__ void from_f32(float v, __nv_bfloat16 &o) { o = __float2bfloat16_rn(v); }

// softplus(v) = log(1 + e^v) = max(v, 0) + log1p(u),  u = e^{-|v|} in (0, 1].
// log1p(u) = u * P(u) with P a degree-9 polynomial fitted to log1p(u)/u on
// [0, 1] (relative-error weighted least squares on Chebyshev nodes); about
// 1.5 ulp over the whole range, including u -> 0 where log1p(u) ~ u.
__device__ __forceinline__ float softplus_from_u(float v, float u) {
    float p = -0.003244000254198909f;
    p = __fmaf_rn(p, u, 0.01985134929418564f);
    p = __fmaf_rn(p, u, -0.05695932358503342f);
    p = __fmaf_rn(p, u, 0.10603633522987366f);
    p = __fmaf_rn(p, u, -0.153055801987648f);
    p = __fmaf_rn(p, u, 0.19675934314727783f);
    p = __fmaf_rn(p, u, -0.24954132735729218f);
    p = __fmaf_rn(p, u, 0.3332996368408203f);
    p = __fmaf_rn(p, u, -0.4999990165233612f);
    p = __fmaf_rn(p, u, 1.0f);
    return __fadd_rn(fmaxf(v, 0.f), __fmul_rn(u, p));
}
__device__ __forceinline__ float softplus_f32(float v) {
    return softplus_from_u(v, ex2_approx(__fmul_rn(-fabsf(v), kLog2e)));
}
// softplus(v) (the same bits as softplus_f32) and its derivative
// sigmoid(v) = (v >= 0 ? 1 : u) / (1 + u), from the one exp u = e^{-|v|}
__device__ __forceinline__ float softplus_sigmoid_f32(float v, float &sig) {
    const float u = ex2_approx(__fmul_rn(-fabsf(v), kLog2e));
    sig = __fmul_rn(v >= 0.f ? 1.f : u, rcp_approx(__fadd_rn(1.f, u)));
    return softplus_from_u(v, u);
}

// silu(z) = z / (1 + e^{-z})
__device__ __forceinline__ float silu_f32(float z) {
    const float e = ex2_approx(__fmul_rn(-z, kLog2e));
    return __fmul_rn(z, rcp_approx(__fadd_rn(1.f, e)));
}

// 16-byte global -> shared asynchronous copy; valid == false zero-fills the
// destination without reading global memory.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src, bool valid) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem_src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int PENDING>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(PENDING) : "memory");
}

// Widen 8 consecutive IO values (16 bytes) to fp32.
__device__ __forceinline__ void widen16(const float *src, float *dst) {
    *reinterpret_cast<float4 *>(dst) = *reinterpret_cast<const float4 *>(src);
}
__device__ __forceinline__ void widen16(const __nv_bfloat16 *src, float *dst) {
    const uint4 q = *reinterpret_cast<const uint4 *>(src);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
    *reinterpret_cast<float4 *>(dst) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4 *>(dst + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

}  // namespace bdk

namespace bdk {

// ---- Tensor Memory (TMEM) helpers -------------------------------------------
// TMEM is the 256 KB per-SM memory of the 5th-generation tensor cores: 128 lanes
// x 512 columns of 32 bits. Warp w of a CTA may access lanes 32*(w%4) .. +31
// (its quadrant); lane i of the warp reads and writes TMEM lane 32*(w%4) + i.
// The scan kernels use it as per-lane scratch for a block's decays and inputs,
// which frees registers without touching the shared-memory pipe.

// Allocate ncols columns (power of two, >= 32) for this CTA; the whole warp
// executes it. The TMEM address is written to *slot (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(slot));
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 8 consecutive 32-bit columns of this lane's row
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "r"(taddr)
                 : "memory");
}
// 16 consecutive 32-bit columns of this lane's row
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
        "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]), "=f"(v[8]),
          "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
        : "r"(taddr)
        : "memory");
}
// width-generic forms (8 or 16 columns)
__device__ __forceinline__ void tmem_st(uint32_t taddr, const float (&v)[8]) { tmem_st8(taddr, v); }
__device__ __forceinline__ void tmem_st(uint32_t taddr, const float (&v)[16]) { tmem_st16(taddr, v); }
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[8]) { tmem_ld8(taddr, v); }
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[16]) { tmem_ld16(taddr, v); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// Wait for this thread's outstanding TMEM loads. The loaded registers pass
// through the instruction so that no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_wait_ld(float (&u)[8], float (&v)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(u[0]), "+f"(u[1]), "+f"(u[2]), "+f"(u[3]), "+f"(u[4]), "+f"(u[5]), "+f"(u[6]), "+f"(u[7]),
                   "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]), "+f"(v[7])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld(float (&u)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(u[0]), "+f"(u[1]), "+f"(u[2]), "+f"(u[3]), "+f"(u[4]), "+f"(u[5]), "+f"(u[6]), "+f"(u[7])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld(float (&u)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(u[0]), "+f"(u[1]), "+f"(u[2]), "+f"(u[3]), "+f"(u[4]), "+f"(u[5]), "+f"(u[6]), "+f"(u[7]),
                   "+f"(u[8]), "+f"(u[9]), "+f"(u[10]), "+f"(u[11]), "+f"(u[12]), "+f"(u[13]), "+f"(u[14]), "+f"(u[15])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld(float (&u)[16], float (&v)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(u[0]), "+f"(u[1]), "+f"(u[2]), "+f"(u[3]), "+f"(u[4]), "+f"(u[5]), "+f"(u[6]), "+f"(u[7]),
                   "+f"(u[8]), "+f"(u[9]), "+f"(u[10]), "+f"(u[11]), "+f"(u[12]), "+f"(u[13]), "+f"(u[14]), "+f"(u[15]),
                   "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]), "+f"(v[7]),
                   "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15])
                 :
                 : "memory");
}

}  // namespace bdk
