// Shared device helpers for the banded Sinkhorn attention kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

// Debug builds (-DSA_DEBUG): device-side bounds checks.  A failed check
// records SA_ERR_BOUNDS in the status word (the first one wins) and the
// access it guards is skipped: the kernel never traps.  In the normal build the
// checks compile to nothing.
#ifdef SA_DEBUG
__device__ __forceinline__ bool debug_bounds(bool ok, int* status) {
    if (!ok && status) atomicCAS(status, 0, -8 /* SA_ERR_BOUNDS */);
    return ok;
}
#define SA_BOUNDS(cond, status) ::sa::debug_bounds((cond), (status))
#else
#define SA_BOUNDS(cond, status) true
#endif

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// 2^x on the MUFU unit (flush-to-zero; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// log2(x) on the MUFU unit.
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// A per-(batch*head) vector: element t of problem bh is p[bh * s + t].
struct Vec {
    const float* p;
    long long s;
    __device__ __forceinline__ float at(int bh, int t) const { return p[(long long)bh * s + t]; }
};
struct MVec {
    float* p;
    long long s;
    __device__ __forceinline__ float& at(int bh, int t) const { return p[(long long)bh * s + t]; }
};

// Element loads from storage dtype into fp32.
__device__ __forceinline__ void load_vec(const float* src, float* dst8, int n) {
    // n == 4: one 16-byte load
    float4 a = *reinterpret_cast<const float4*>(src);
    dst8[0] = a.x; dst8[1] = a.y; dst8[2] = a.z; dst8[3] = a.w;
    (void)n;
}
__device__ __forceinline__ void load_vec(const __nv_bfloat16* src, float* dst8, int n) {
    // n == 8: one 16-byte load of 8 bf16
    uint4 a = *reinterpret_cast<const uint4*>(src);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&a);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(h[e]);
        dst8[2 * e] = f.x;
        dst8[2 * e + 1] = f.y;
    }
    (void)n;
}

template <typename T> struct VecW { static constexpr int n = 16 / sizeof(T); };

__device__ __forceinline__ void store_elem(float* dst, float x) { *dst = x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* dst, float x) { *dst = __float2bfloat16_rn(x); }

__device__ __forceinline__ void store4(float* dst, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(dst) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void store4(__nv_bfloat16* dst, float a, float b, float c, float d) {
    __nv_bfloat162 x = __floats2bfloat162_rn(a, b);
    __nv_bfloat162 y = __floats2bfloat162_rn(c, d);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&x);
    u.y = *reinterpret_cast<uint32_t*>(&y);
    *reinterpret_cast<uint2*>(dst) = u;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Merge two (max, sum) pairs of a base-2 log-sum-exp: value = m + log2(s).
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) { m = m2; s = s2; return; }
    if (m2 > m) { s = s * ex2(m - m2) + s2; m = m2; }
    else { s = s + s2 * ex2(m2 - m); }
}

}  // namespace sa
