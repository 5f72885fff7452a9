// Shared device helpers of the transposable N:M mask kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace tsenor {

constexpr unsigned kFullMask = 0xffffffffu;

// Hardware base-2 exponential / logarithm / reciprocal (PTX approx forms, MUFU).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Shared-memory load of a float2 that the compiler may not move out of a
// loop (a hoisted loop-invariant load would hold its registers for the whole
// loop).
__device__ __forceinline__ float2 lds_keep(const float2* p) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];"
                 : "=f"(v.x), "=f"(v.y)
                 : "r"(static_cast<unsigned>(__cvta_generic_to_shared(p))));
    return v;
}

// Packed fp32 pairs (PTX f32x2, sm_100): two adds / multiplies / fmas per
// instruction, round to nearest even per element.
union F2U {
    float2 f;
    unsigned long long u;
};
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    F2U x{a}, y{b}, d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d.u) : "l"(x.u), "l"(y.u));
    return d.f;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    F2U x{a}, y{b}, d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d.u) : "l"(x.u), "l"(y.u));
    return d.f;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    F2U x{a}, y{b}, d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d.u) : "l"(x.u), "l"(y.u));
    return d.f;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    F2U x{a}, y{b}, z{c}, d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d.u) : "l"(x.u), "l"(y.u), "l"(z.u));
    return d.f;
}

// Element types of W.  Loads return |W| as fp32 (exact for both types).
struct F32 {
    using storage = float;
    static constexpr int kVec = 4;   // elements per 16-byte load
    __device__ __forceinline__ static void load16(const float* p, float* out) {
        float4 v = __ldg(reinterpret_cast<const float4*>(p));
        out[0] = fabsf(v.x); out[1] = fabsf(v.y); out[2] = fabsf(v.z); out[3] = fabsf(v.w);
    }
    __device__ __forceinline__ static float load1(const float* p) { return fabsf(__ldg(p)); }
    __device__ __forceinline__ static void smem16(const float* p, float* out) {     // 16 bytes of shared memory
        const float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = fabsf(v.x); out[1] = fabsf(v.y); out[2] = fabsf(v.z); out[3] = fabsf(v.w);
    }
};

struct BF16 {
    using storage = uint16_t;
    static constexpr int kVec = 8;
    __device__ __forceinline__ static float widen(uint32_t bits16) {
        return __uint_as_float((bits16 & 0x7fffu) << 16);
    }
    __device__ __forceinline__ static void load16(const uint16_t* p, float* out) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            out[2 * q] = widen(w[q] & 0xffffu);
            out[2 * q + 1] = widen(w[q] >> 16);
        }
    }
    __device__ __forceinline__ static float load1(const uint16_t* p) { return widen(__ldg(p)); }
    __device__ __forceinline__ static void smem16(const uint16_t* p, float* out) {  // 16 bytes of shared memory
        const uint4 v = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            out[2 * q] = widen(w[q] & 0xffffu);
            out[2 * q + 1] = widen(w[q] >> 16);
        }
    }
};

// Packed sort key of one block entry: plan bits (S >= 0, so the bit pattern
// orders like the value), |W| bits, and the flat index.  Larger key = earlier
// in the rounding order: S desc, then |W| desc, then flat index asc.
struct SortKey {
    unsigned long long k;   // S bits << 32 | |W| bits
    uint32_t idx;           // flat index i*M + j
};
__device__ __forceinline__ bool key_before(const SortKey& a, const SortKey& b) {
    return a.k > b.k || (a.k == b.k && a.idx < b.idx);
}

}  // namespace tsenor
