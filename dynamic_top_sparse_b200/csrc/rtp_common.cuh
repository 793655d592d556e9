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
// for bf16, two 16-byte loads for fp32).  Cache rows are read once per use:
// loads are cached in L2 only.
template <typename T> struct Row;

template <> struct Row<__nv_bfloat16> {
    static __device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
        uint4 u = __ldcg(reinterpret_cast<const uint4 *>(p));
        x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x);
        x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
        x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z);
        x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
    }
    static __device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&x)[4]) {
        uint2 u = __ldcg(reinterpret_cast<const uint2 *>(p));
        x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x);
        x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    }
    static __device__ __forceinline__ __nv_bfloat16 from_float(float v) { return __float2bfloat16_rn(v); }
};

template <> struct Row<float> {
    static __device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
        float4 a = __ldcg(reinterpret_cast<const float4 *>(p));
        float4 b = __ldcg(reinterpret_cast<const float4 *>(p) + 1);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
    static __device__ __forceinline__ void load4(const float *p, float (&x)[4]) {
        float4 a = __ldcg(reinterpret_cast<const float4 *>(p));
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
// mbarrier + bulk async copy (TMA, 1-D) helpers.  Every wait is bounded in
// time: after the limit the caller gets `false` and reports RTP_ERR_TIMEOUT.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
constexpr uint64_t WAIT_LIMIT_NS = 200000000ull;   // 0.2 s: far beyond any healthy wait
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > WAIT_LIMIT_NS) return false;
    return true;
}
// global -> shared bulk copy completing on `bar` (16-byte aligned, size a
// multiple of 16)
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel of the selection chain may be
// launched while its predecessor in the stream is still running; it calls
// pdl_wait() before its first global-memory access (read or write), which
// returns once every earlier grid of the stream has completed and its writes
// are visible (a no-op when the kernel was launched normally).
// pdl_trigger() lets the next kernel's CTAs be scheduled from then on.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

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

// List attention splits a head's kept rows into items of about LCH rows,
// at most LIST_MAX_SPLIT per head.
constexpr int LCH = 64;
constexpr int LIST_MAX_SPLIT = 256;
constexpr int LIST_SLOTS = 2 * LIST_MAX_SPLIT;   // partial record slots per head
// Flags by which the fused step's finalize hands a head's remaining rows to
// a list pass: the rows from the collect pass's count on, or every row.
constexpr uint32_t SPILL_FROM_FIRST = 2u, SPILL_ALL_ROWS = 3u;
__device__ __forceinline__ int list_items(int count) {
    if (count <= 0) return 0;
    return min(LIST_MAX_SPLIT, (count + LCH - 1) / LCH);
}

// Per-head counters of the selection (kept ids, boundary candidates) sit
// one per 128-byte line: every collect CTA reserves space on them at about
// the same moment, and counters sharing a line would queue those atomics on
// one L2 slice.
constexpr int CNT_STRIDE = 32;        // uint32 entries between consecutive heads' counters

// Flash-decoding partial record of one head over a set of rows (log2
// units): m = running max, l = sum of 2^(s - m), o[D] = unnormalised output.
constexpr int PSTRIDE = D + 4;         // partial record: m, l, (2 unused), o[D]
constexpr int POFF = 4;                // offset of o[] in a record (16-byte aligned)
static_assert(PSTRIDE % 4 == 0 && POFF % 4 == 0, "partial records must keep o[] 16-byte aligned");

// ---------------------------------------------------------------------------
// K/V row addressing.  Contiguous caches hold token t of (sequence b, KV
// head g) at row (b H_kv + g) N_max + t.  Paged caches (table != null) are
// pools [num_pages][H_kv][page][D]: token t of sequence b lives in page
// table[b max_pages + t / page] at slot t % page (page = 2^page_shift).  A
// page number outside the pool is reported (RTP_ERR_DEVICE_ARG) and the row
// reads as missing (-1).
// ---------------------------------------------------------------------------
struct KvMap {
    const int32_t *table;
    int page_shift, max_pages, num_pages;
    int H_kv;
    long long N_max;
    uint32_t *status;
};
__device__ __forceinline__ long long kv_row(const KvMap &m, int b, int g, long long t) {
    if (!m.table) return ((long long)b * m.H_kv + g) * m.N_max + t;
    const long long j = t >> m.page_shift;
    if (j >= m.max_pages) { set_status(m.status, RTP_ERR_DEVICE_ARG); return -1; }
    const int pg = __ldg(m.table + (long long)b * m.max_pages + j);
    if (pg < 0 || pg >= m.num_pages) { set_status(m.status, RTP_ERR_DEVICE_ARG); return -1; }
    return (((long long)pg * m.H_kv + g) << m.page_shift) + (t & ((1LL << m.page_shift) - 1));
}

// Flash-decoding partial of one head over a set of rows.
struct Partial {
    float m;        // max logit (-inf when empty)
    float l;        // sum of exp(logit - m)
};

}  // namespace rtp
