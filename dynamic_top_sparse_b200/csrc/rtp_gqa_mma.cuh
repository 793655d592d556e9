// Tensor-core decode attention of one KV group (all G <= 8 query heads) over
// a row-range set: the sink rows plus the sliding window of a local head
// ("Full Attention Strikes Back", gist.science technical summary, Method
// section 1), or every row (the dense comparison kernel).  bf16 caches.
//
// mma.sync m16n8k16 with the heads on M (8 used of 16, FlashAttention-2
// style so that the softmax output of Q.K^T is already the A operand of
// P.V):
//   S[h, t]  = sum_d q[h, d] k[t, d]       A = q (3-term bf16 split, ~24-bit
//                                          exact), B = K^T, 2 n-tiles of 8 rows
//   O[h, d] += sum_t p[h, t] v[t, d]       A = p (2-term split), B = V,
//                                          16 n-tiles of 8 dims
// The k dimension of each product is permuted so that every thread reads
// contiguous 16-byte pieces of K and V rows straight from HBM:
//   Q.K^T, k-step kk: thread (gid, tig) supplies dims 32 tig + 4 kk + {0..3};
//   P.V, n-tile j, column n: dim 16 n + j, so thread gid reads dims
//   [16 gid, 16 gid + 16) of its four rows (tokens 2tig, 2tig+1, 2tig+8,
//   2tig+9 of the 16-row tile) and pairs them with byte permutes.
// Partials (m, l, o) per head are merged over warps, then over CTAs by the
// last CTA to finish (same record layout as range_attn_kernel).
#pragma once

#include "rtp_attend.cuh"

namespace rtp {

constexpr int GQ_WARPS = 8;
constexpr int GQ_THREADS = GQ_WARPS * 32;
constexpr int GQ_TILE = 16;                 // rows per mma tile

// D[rows 0-7] = A.B + C for an A whose rows 8-15 are zero: only the two
// accumulators of rows gid are kept; rows 8-15 go to write-only temporaries
// (no dependency between independent products).
__device__ __forceinline__ void mma16816_top(float &d0, float &d1, uint32_t a0, uint32_t a2, uint32_t b0,
                                             uint32_t b1) {
    float j0, j1;
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%11,%12,%12};\n"
        : "=f"(d0), "=f"(d1), "=f"(j0), "=f"(j1)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d0), "f"(d1), "f"(0.0f));
    (void)j0;
    (void)j1;
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}

// x = hi + mid + lo, each a bf16 value
__device__ __forceinline__ void split3(float x, float &hi, float &mid, float &lo) {
    hi = __bfloat162float(__float2bfloat16_rn(x));
    const float r = x - hi;
    mid = __bfloat162float(__float2bfloat16_rn(r));
    lo = r - mid;
}

// PAGED: rows through the block table of a page pool (a.kv.table), else
// contiguous.
template <bool PAGED>
__global__ void __launch_bounds__(GQ_THREADS, 1) gqa_mma_attn_kernel(RangeArgs a) {
    __shared__ float s_m[GQ_WARPS][GMAX], s_l[GQ_WARPS][GMAX];
    __shared__ float s_o[GQ_WARPS][GMAX][D];
    __shared__ int s_last;
    const int b = blockIdx.y / a.n_grp;
    const int g = a.grp[blockIdx.y % a.n_grp];
    const int G = a.G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const size_t bg = (size_t)b * a.H_kv + g;
    const size_t bh0 = (size_t)b * a.H_q + (size_t)g * G;

    const int N = a.seq_lens[b];
    if (N < 1 || (long long)N > a.N_max) {
        if (blockIdx.x == 0) {
            if (tid == 0) set_status(a.status, RTP_ERR_DEVICE_ARG);
            if (a.part_out) {
                for (int i = tid; i < G * PSTRIDE; i += blockDim.x)
                    a.part_out[bh0 * PSTRIDE + i] = i % PSTRIDE == 0 ? -INFINITY : 0.0f;
            } else {
                for (int i = tid; i < G * D; i += blockDim.x) a.out[bh0 * D + i] = 0.0f;
            }
        }
        return;
    }
    int s1, w0;
    shard_range(a, b, N, s1, w0);
    const long long L = (long long)s1 + (N - w0);
    const long long seg = (L + a.n_split - 1) / a.n_split;
    const int n_active = L > 0 ? (int)((L + seg - 1) / seg) : 1;
    if ((int)blockIdx.x >= n_active) return;
    const long long lo = (long long)blockIdx.x * seg;
    const long long hi = min(L, lo + seg);

    // Q fragments: head gid (zero for gid >= G), dims 32 tig + 4 kk + {0..3}
    uint32_t qa[3][8][2];
    {
        const float *qh = a.q + (bh0 + (gid < G ? gid : 0)) * D + 32 * tig;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            float4 v = gid < G ? __ldg(reinterpret_cast<const float4 *>(qh + 4 * kk)) : make_float4(0.f, 0.f, 0.f, 0.f);
            float x[4] = {v.x * a.scale_log2, v.y * a.scale_log2, v.z * a.scale_log2, v.w * a.scale_log2};
            float h[4], m[4], l[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) split3(x[i], h[i], m[i], l[i]);
            qa[0][kk][0] = bf16x2(h[0], h[1]); qa[0][kk][1] = bf16x2(h[2], h[3]);
            qa[1][kk][0] = bf16x2(m[0], m[1]); qa[1][kk][1] = bf16x2(m[2], m[3]);
            qa[2][kk][0] = bf16x2(l[0], l[1]); qa[2][kk][1] = bf16x2(l[2], l[3]);
        }
    }
    const __nv_bfloat16 *kb = reinterpret_cast<const __nv_bfloat16 *>(a.k);
    const __nv_bfloat16 *vb = reinterpret_cast<const __nv_bfloat16 *>(a.v);
    // cache row of range position j (past the end: a valid row, masked
    // below; a page outside the pool is reported and read as row 0)
    const long long base = (long long)bg * a.N_max;
    auto row_of = [&](long long j) -> long long {
        j = j < hi ? j : hi - 1;
        const long long t = j < s1 ? j : w0 + (j - s1);
        if constexpr (PAGED) return max(0LL, kv_row(a.kv, b, g, t));
        return base + t;
    };

    float m_run = -INFINITY, l_run = 0.0f;        // head gid (shared by the 4 lanes of gid)
    float o[16][2];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = 0.0f;

    for (long long t0 = lo + (long long)warp * GQ_TILE; t0 < hi; t0 += GQ_WARPS * GQ_TILE) {
        // K: rows t0 + gid (n-tile 0) and t0 + 8 + gid (n-tile 1), dims [32 tig, 32 tig + 32)
        uint4 kr[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const uint4 *p = reinterpret_cast<const uint4 *>(kb + row_of(t0 + 8 * n + gid) * D + 32 * tig);
#pragma unroll
            for (int i = 0; i < 4; ++i) kr[n][i] = __ldg(p + i);
        }
        // V: rows t0 + {2tig, 2tig+1, 2tig+8, 2tig+9}, dims [16 gid, 16 gid + 16)
        uint4 vr[4][2];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int tr = 2 * tig + (r & 1) + 8 * (r >> 1);
            const uint4 *p = reinterpret_cast<const uint4 *>(vb + row_of(t0 + tr) * D + 16 * gid);
            vr[r][0] = __ldg(p);
            vr[r][1] = __ldg(p + 1);
        }
        // S = Q K^T (log2 units), n-tile n covers rows t0 + 8n .. t0 + 8n + 7;
        // one accumulator chain per (n-tile, term), summed low to high
        float sc[2][2];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            float acc[3][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                // dims 32 tig + 4 kk + {0,1} and {2,3}: words 2kk, 2kk+1 of the slice
                const uint4 &k4 = kr[n][kk >> 1];
                const uint32_t b0 = (kk & 1) ? k4.z : k4.x;
                const uint32_t b1 = (kk & 1) ? k4.w : k4.y;
#pragma unroll
                for (int term = 0; term < 3; ++term)
                    mma16816_top(acc[term][0], acc[term][1], qa[term][kk][0], qa[term][kk][1], b0, b1);
            }
            sc[n][0] = (acc[2][0] + acc[1][0]) + acc[0][0];
            sc[n][1] = (acc[2][1] + acc[1][1]) + acc[0][1];
        }
        // mask rows past the end of this CTA's range
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int c = 0; c < 2; ++c)
                if (t0 + 8 * n + 2 * tig + c >= hi) sc[n][c] = -INFINITY;
        // online softmax for head gid (4 lanes share it)
        float tmax = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
        const float m_new = fmaxf(m_run, tmax);
        const float alpha = m_new == -INFINITY ? 1.0f : exp2f(m_run - m_new);
        float p[2][2];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int c = 0; c < 2; ++c) p[n][c] = m_new == -INFINITY ? 0.0f : exp2f(sc[n][c] - m_new);
        l_run = l_run * alpha + (p[0][0] + p[0][1] + p[1][0] + p[1][1]);
        m_run = m_new;
#pragma unroll
        for (int j = 0; j < 16; ++j) { o[j][0] *= alpha; o[j][1] *= alpha; }
        // P as A operand: a0 = tokens (2tig, 2tig+1), a2 = tokens (2tig+8, 2tig+9)
        float ph[2][2], pl[2][2];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                ph[n][c] = __bfloat162float(__float2bfloat16_rn(p[n][c]));
                pl[n][c] = p[n][c] - ph[n][c];
            }
        const uint32_t pa0h = bf16x2(ph[0][0], ph[0][1]), pa2h = bf16x2(ph[1][0], ph[1][1]);
        const uint32_t pa0l = bf16x2(pl[0][0], pl[0][1]), pa2l = bf16x2(pl[1][0], pl[1][1]);
        // O += P V: n-tile j, column gid <-> dim 16 gid + j
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int wi = j >> 1;                       // word index within the 16-dim slice
            const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
            const uint32_t w_r0 = (&vr[0][wi >> 2].x)[wi & 3];
            const uint32_t w_r1 = (&vr[1][wi >> 2].x)[wi & 3];
            const uint32_t w_r2 = (&vr[2][wi >> 2].x)[wi & 3];
            const uint32_t w_r3 = (&vr[3][wi >> 2].x)[wi & 3];
            const uint32_t b0 = __byte_perm(w_r0, w_r1, sel);
            const uint32_t b1 = __byte_perm(w_r2, w_r3, sel);
            mma16816_top(o[j][0], o[j][1], pa0l, pa2l, b0, b1);
            mma16816_top(o[j][0], o[j][1], pa0h, pa2h, b0, b1);
        }
    }
    // warp partials: l summed over the 4 lanes of head gid; o[j][c] is dim
    // 16 (2 tig + c) + j of head gid
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    if (gid < GMAX && tig == 0) { s_m[warp][gid] = m_run; s_l[warp][gid] = l_run; }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        s_o[warp][gid][32 * tig + j] = o[j][0];
        s_o[warp][gid][32 * tig + 16 + j] = o[j][1];
    }
    __syncthreads();
    float *pp = a.part + (bg * a.slots + blockIdx.x) * GMAX * PSTRIDE;
    for (int i = tid; i < G * D; i += blockDim.x) {
        const int h = i / D, d = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < GQ_WARPS; ++w) M = fmaxf(M, s_m[w][h]);
        float ls = 0.0f, os = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < GQ_WARPS; ++w) {
                const float wg = s_m[w][h] == -INFINITY ? 0.0f : exp2f(s_m[w][h] - M);
                ls = fmaf(s_l[w][h], wg, ls);
                os = fmaf(s_o[w][h][d], wg, os);
            }
        }
        pp[h * PSTRIDE + POFF + d] = os;
        if (d == 0) { pp[h * PSTRIDE] = M; pp[h * PSTRIDE + 1] = ls; }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&a.arrive[bg], 1u) == (unsigned)(n_active - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    merge_partials(a.part + bg * a.slots * GMAX * PSTRIDE, n_active, GMAX * PSTRIDE, G, a.out + bh0 * D,
                   a.part_out ? a.part_out + bh0 * PSTRIDE : nullptr);
    if (tid == 0) a.arrive[bg] = 0;
}

}  // namespace rtp
