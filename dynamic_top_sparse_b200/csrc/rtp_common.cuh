// Device helpers shared by the sparse-decode kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "rtp.h"

namespace rtp {

constexpr int D = 128;          // head dim
constexpr int R = 16;           // indexer dim
constexpr int GMAX = 8;         // largest GQA group handled in one tile
constexpr int WARP = 32;

// ---------------------------------------------------------------------------
// status word (first 4 bytes of the workspace): the first error wins
// ---------------------------------------------------------------------------
__device__ __forceinline__ void set_status(uint32_t *status, int code) {
    atomicCAS(status, 0u, (uint32_t)code);
}

// ---------------------------------------------------------------------------
// element loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// 8 consecutive elements starting at element `i` of a row (16-byte aligned
// for bf16, two 16-byte loads for fp32).
template <typename T> struct Row;

template <> struct Row<__nv_bfloat16> {
    static __device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
        uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
        x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x);
        x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
        x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z);
        x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
    }
    static __device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&x)[4]) {
        uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
        x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x);
        x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    }
    static __device__ __forceinline__ __nv_bfloat16 from_float(float v) { return __float2bfloat16_rn(v); }
};

template <> struct Row<float> {
    static __device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
        float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
    static __device__ __forceinline__ void load4(const float *p, float (&x)[4]) {
        float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    }
    static __device__ __forceinline__ float from_float(float v) { return v; }
};

// ---------------------------------------------------------------------------
// order-preserving key of an fp32 logit (descending z <=> descending key);
// -0 is folded onto +0 so that equal values have equal keys.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t logit_key(float z) {
    uint32_t u = __float_as_uint(z);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// ---------------------------------------------------------------------------
// Level-1 mass histogram bins.  |z| in [2^E_LO, 2^E_HI) is binned by its
// exponent and the top MB mantissa bits (relative width 2^-MB), one set of
// bins per sign; |z| < 2^E_LO shares one central bin.  Bin order follows z.
// Each bin stores the sum of exp(z - U) over its tokens, U = the bin's upper
// edge, so no maximum is needed while scanning and every term is in (0, 1]
// (bin widths are at most 32 nats below 2^E_HI).
// ---------------------------------------------------------------------------
constexpr int MB = 4;
constexpr int E_LO = -6;
constexpr int E_HI = 10;
constexpr int NPOS = (E_HI - E_LO) << MB;     // 256 bins per sign
constexpr int NBIN = 2 * NPOS + 1;            // 513
constexpr int ZERO_BIN = NPOS;
constexpr float Z_LIMIT = 1024.0f;            // 2^E_HI
constexpr uint32_t BIN_BASE = (uint32_t)(127 + E_LO) << MB;

__device__ __forceinline__ int logit_bin(float z) {
    uint32_t a = __float_as_uint(z) & 0x7fffffffu;
    int k = (int)(a >> (23 - MB)) - (int)BIN_BASE;
    if (k < 0) return ZERO_BIN;
    return z > 0.0f ? ZERO_BIN + 1 + k : ZERO_BIN - 1 - k;
}

// Upper edge of a bin (an fp32 value; every z in the bin is <= it).
__host__ __device__ __forceinline__ float bin_upper(int bin) {
    if (bin == ZERO_BIN) {
        union { uint32_t u; float f; } c; c.u = BIN_BASE << (23 - MB); return c.f;
    }
    if (bin > ZERO_BIN) {
        uint32_t k = (uint32_t)(bin - ZERO_BIN - 1);
        union { uint32_t u; float f; } c; c.u = (k + 1 + BIN_BASE) << (23 - MB); return c.f;
    }
    uint32_t k = (uint32_t)(ZERO_BIN - 1 - bin);
    union { uint32_t u; float f; } c; c.u = (k + BIN_BASE) << (23 - MB); return -c.f;
}

// ---------------------------------------------------------------------------
// warp helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Flash-decoding partial of one head over a set of rows.
struct Partial {
    float m;        // max logit (-inf when empty)
    float l;        // sum of exp(logit - m)
};

}  // namespace rtp
