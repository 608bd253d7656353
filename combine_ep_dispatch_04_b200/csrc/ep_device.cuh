// ep_device.cuh -- device helpers shared by the dispatch / combine kernels:
// bf16 unpacking, the native sm_100a format conversions (cvt ... satfinite to
// e4m3 / e2m1), the e8m0 exponent of an MX block, and streaming memory access.
//
// Arithmetic contract (matches the quantisation rules of the header): every
// scale is one IEEE division (__fdiv_rn), every scaled value one rounded
// multiply (__fmul_rn, never contracted into an FMA), conversions round to
// nearest even.  The library is built without fast-math, so subnormals are kept.
#pragma once

#include <cfloat>
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace ep {

constexpr uint32_t kFull = 0xFFFFFFFFu;

// topk_idx as stored by the caller: int64 ("Low-Latency Mode API", topk_idx)
// or int32 ("DeepEP topk_idx_t Custom Dtype Requirements": the index type
// built with 32 bits).  One uniform branch per load.
struct TopkIdx {
    const void *p;
    int i32;
    __device__ __forceinline__ int64_t operator[](int64_t i) const {
        return i32 ? (int64_t)static_cast<const int32_t *>(p)[i] : static_cast<const int64_t *>(p)[i];
    }
};

// Threads of a block whose token groups have TPT threads: one token per block
// from TPT = 128 up, 128 threads otherwise.  Small blocks spread the tokens of
// a grid that fits in one wave evenly over the SMs (a block of two 128-thread
// tokens leaves some SMs with one token more than the rest).
__host__ __device__ constexpr int block_threads(int tpt) { return tpt < 128 ? 128 : tpt; }
constexpr uint32_t kDevBadIndex = 0x1u;
constexpr uint32_t kDevCapacity = 0x2u;

// ---- bf16 ------------------------------------------------------------------
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// |x| of the two bf16 halves compared as integers: for finite values the
// magnitude order of bf16 bit patterns (sign cleared) is the numeric order.
__device__ __forceinline__ uint32_t bf2_absmax(uint32_t acc, uint32_t w) {
    return __vmaxu2(acc, w & 0x7FFF7FFFu);
}
// Block maxima leave NaN elements out (as fmaxf does).  Magnitudes compare as
// unsigned integers and a NaN's is above infinity's (0x7F80), so a running
// maximum above 0x7F80 says a NaN was seen; the maximum is then taken again
// over the pairs with their NaN halves zeroed.
__device__ __forceinline__ bool bf2_any_nan(uint32_t m) {
    return (m & 0xFFFFu) > 0x7F80u || (m >> 16) > 0x7F80u;
}
__device__ __forceinline__ uint32_t bf2_drop_nan(uint32_t w) {
    const uint32_t m = w & 0x7FFF7FFFu;
    const uint32_t t = (m + 0x007F007Fu) & 0x80008000u;  // bit 15 of each NaN half
    return m & ~((t >> 15) * 0xFFFFu);
}
__device__ __forceinline__ float bf2_fold(uint32_t m) {  // max of the two halves as fp32
    uint32_t lo = m & 0xFFFFu, hi = m >> 16;
    return __uint_as_float((lo > hi ? lo : hi) << 16);
}

// Two fp32 -> bf16x2 (round to nearest even); `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---- native format conversions (sm_100a) ----------------------------------
// cvt ... e4m3x2 / e2m1x2 put their first source operand in the upper part of
// the result, so `lo` is passed second to land at the lower address / nibble.
// (p0, p1) <- (fl(p0 * s), fl(p1 * s)) on the packed fp32 pipe (sm_100): each
// lane one IEEE multiply rounded to nearest even, exactly __fmul_rn.
__device__ __forceinline__ void mul2(float &p0, float &p1, float s) {
    asm("{\n\t.reg .b64 p, s;\n\tmov.b64 p, {%0, %1};\n\tmov.b64 s, {%2, %2};\n\t"
        "mul.rn.f32x2 p, p, s;\n\tmov.b64 {%0, %1}, p;\n\t}"
        : "+f"(p0), "+f"(p1)
        : "f"(s));
}

__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// ---- exact int8 decoding without a conversion instruction ----------------------
// int8 byte j of wx = w ^ 0x80808080: the fp32 2^23 + 128 + b, less 2^23 + 128 (both exact).
__device__ __forceinline__ float i8_exact(uint32_t wx, int j) {
    return __uint_as_float(__byte_perm(wx, 0x4B000000u, 0x7440 | j)) - 8388736.0f;
}

// ---- scales ------------------------------------------------------------------
// ceil(log2 v) for a positive finite fp32 v, exactly, from its bits.
__device__ __forceinline__ int ceil_log2_pos(float v) {
    uint32_t b = __float_as_uint(v);
    int ex = (int)(b >> 23);
    uint32_t m = b & 0x7FFFFFu;
    if (ex != 0) return ex - 127 + (m != 0u);
    return (32 - __clz((int)(m - 1u))) - 149;  // subnormal: v = m * 2^-149
}

// e8m0 exponent X of an MX block: the smallest power of two with
// amax / qmax <= 2^X, i.e. ceil(log2(amax / qmax)) with one IEEE division,
// clamped to [-127, 127]; amax == 0 gives 0, and so does a NaN amax (a block
// whose every element is NaN: the maximum of no element).
__device__ __forceinline__ int mx_exponent(float amax, float qmax) {
    if (amax == 0.0f || amax != amax) return 0;
    float v = __fdiv_rn(amax, qmax);
    if (v == 0.0f) return -127;
    int X = ceil_log2_pos(v);
    return X < -127 ? -127 : (X > 127 ? 127 : X);
}

// The same exponent without the division, for qmax = 448 (= 7 * 2^6) and
// qmax = 6 (= 3 * 2^1).  For a normal amax = m * 2^e whose quotient is normal,
// fl(amax / (q * 2^s)) = fl(amax / q) * 2^-s, and fl(m / q) is a power of two
// only for m = 1.75 (q = 7) or m = 1.5 (q = 3) exactly -- the neighbouring
// mantissas are more than half an ulp away -- so
//   X = e - 8 + [m > 1.75]   (qmax 448),   X = e - 2 + [m > 1.5]   (qmax 6).
// Zero, subnormal and tiny values (quotient below the normal range) and
// non-finite values take the division.  Checked against the division-based
// definition on every fp32 input (ep_cvt_sweep formats 2 and 3).
template <int QMAX>
__device__ __forceinline__ int mx_exponent_fast(float amax) {
    static_assert(QMAX == 448 || QMAX == 6, "exponent shortcut is derived for 448 and 6");
    const uint32_t b = __float_as_uint(amax);
    const int ex = (int)(b >> 23);  // amax >= 0: no sign bit
    const uint32_t mant = b & 0x7FFFFFu;
    if (QMAX == 448) {
        if (ex >= 10 && ex < 255) return ex - 127 - 8 + (mant > 0x600000u);
        return mx_exponent(amax, 448.0f);
    } else {
        if (ex >= 4 && ex < 255) return ex - 127 - 2 + (mant > 0x400000u);
        return mx_exponent(amax, 6.0f);
    }
}

// 2^-X as an fp32 for X in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float exp2_neg(int X) {
    int e = 127 - X;
    return e > 0 ? __uint_as_float((uint32_t)e << 23) : __uint_as_float(0x00400000u);
}

// ---- asynchronous copies global -> shared (per thread, completion by group) -----
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {  // L2 only
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem)), "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(smem)), "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- streaming memory access --------------------------------------------------
__device__ __forceinline__ uint4 ld_stream(const void *p) {
    return __ldcs(reinterpret_cast<const uint4 *>(p));
}
__device__ __forceinline__ uint4 ld_ro(const void *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}
__device__ __forceinline__ void st_v4(void *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }
__device__ __forceinline__ void st_v2(void *p, uint2 v) { *reinterpret_cast<uint2 *>(p) = v; }

// Programmatic dependent launch: every kernel of the library is launched so
// that it may start while the previous grid on the stream finishes.  Before
// touching global memory it waits until that grid has completed and its
// writes are visible (a no-op when there is no such grid), then lets its own
// dependents start launching.  Nothing is read before the wait, so this is
// safe whatever kernel precedes.
__device__ __forceinline__ void pdl_enter() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace ep
