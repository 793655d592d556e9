// Tensor-core decode attention of one KV group (all G <= 8 query heads) over
// a row-range set: the sink rows plus the sliding window of a local head
// ("Full Attention Strikes Back", gist.science technical summary, Method
// section 1), or every row (the dense comparison kernel).  bf16 caches.
//
// mma.sync m16n8k16 with the tokens on M and the heads on N, so that all 16
// rows of every product do work (8 query heads fill N exactly):
//   S^T[t, h] = sum_d k[t, d] q[h, d]      A = K (16 rows of the tile),
//                                          B = q^T (3-term bf16 split, ~24-bit
//                                          exact), 8 k-steps of 16 dims
//   O^T[d, h] += sum_t v[t, d] p[h, t]     A = V^T (16 dims per m-tile, 8
//                                          m-tiles), B = p^T (2-term split)
// S^T leaves the first product in the accumulator layout (a thread holds
// tokens gid, gid + 8 of heads 2 tig, 2 tig + 1); packed to bf16 pairs it is
// the 8x8 fragment layout, and one movmatrix transpose per 8 tokens turns it
// into the B operand of the second product.
// The k and m indices are permuted so that every thread reads contiguous
// 16-byte pieces of K and V rows straight from HBM:
//   Q.K^T, k-step kk: thread (gid, tig) supplies dims 32 tig + 4 kk + {0..3}
//   of rows gid and gid + 8;
//   P.V, m-tile mt: rows gid, gid + 8 are dims 16 gid + 2 mt, 16 gid + 2 mt + 1,
//   so thread gid reads dims [16 gid, 16 gid + 16) of its four tokens (2tig,
//   2tig+1, 2tig+8, 2tig+9 of the 16-row tile) and pairs them with byte
//   permutes.
// Each warp keeps the next tile's K/V loads in flight while it computes the
// current one (two register sets).  Partials (m, l, o) per head are merged
// over warps, then over CTAs by the last CTA to finish (same record layout
// as range_attn_kernel).
#pragma once

#include "rtp_attend.cuh"

namespace rtp {

constexpr int GQ_WARPS = 8;
constexpr int GQ_THREADS = GQ_WARPS * 32;
constexpr int GQ_TILE = 16;                 // rows per mma tile

// D = A.B + D (m16n8k16, bf16 inputs, fp32 accumulators)
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// transpose of an 8x8 matrix of 16-bit values held one pair per lane (lane
// 4r + c holds row r, columns 2c and 2c + 1)
__device__ __forceinline__ uint32_t movm_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
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

    // q as the B operand: head gid (zero for gid >= G), dims 32 tig + 4 kk + {0..3}
    uint32_t qb[3][8][2];
    {
        const float *qh = a.q + (bh0 + (gid < G ? gid : 0)) * D + 32 * tig;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            float4 v = gid < G ? __ldg(reinterpret_cast<const float4 *>(qh + 4 * kk)) : make_float4(0.f, 0.f, 0.f, 0.f);
            float x[4] = {v.x * a.scale_log2, v.y * a.scale_log2, v.z * a.scale_log2, v.w * a.scale_log2};
            float h[4], m[4], l[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) split3(x[i], h[i], m[i], l[i]);
            qb[0][kk][0] = bf16x2(h[0], h[1]); qb[0][kk][1] = bf16x2(h[2], h[3]);
            qb[1][kk][0] = bf16x2(m[0], m[1]); qb[1][kk][1] = bf16x2(m[2], m[3]);
            qb[2][kk][0] = bf16x2(l[0], l[1]); qb[2][kk][1] = bf16x2(l[2], l[3]);
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

    // heads 2 tig + c, c = 0, 1 (shared by the 8 lanes of tig); l_run is this
    // lane's part (its tokens), summed over the lanes at the end
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};
    // m-tile mt: {O[2tig][16gid+2mt], O[2tig+1][16gid+2mt], O[2tig][16gid+2mt+1], O[2tig+1][16gid+2mt+1]}
    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.0f;

    // K: rows t0 + gid (+ 8 n), dims [32 tig, 32 tig + 32); V: rows t0 + {2tig,
    // 2tig+1, 2tig+8, 2tig+9}, dims [16 gid, 16 gid + 16)
    auto load_tile = [&](long long t0, uint4 (&kr)[2][4], uint4 (&vr)[4][2]) {
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const uint4 *p = reinterpret_cast<const uint4 *>(kb + row_of(t0 + 8 * n + gid) * D + 32 * tig);
#pragma unroll
            for (int i = 0; i < 4; ++i) kr[n][i] = __ldg(p + i);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int tr = 2 * tig + (r & 1) + 8 * (r >> 1);
            const uint4 *p = reinterpret_cast<const uint4 *>(vb + row_of(t0 + tr) * D + 16 * gid);
            vr[r][0] = __ldg(p);
            vr[r][1] = __ldg(p + 1);
        }
    };
    auto compute_tile = [&](long long t0, const uint4 (&kr)[2][4], const uint4 (&vr)[4][2]) {
        // S^T (log2 units): one accumulator chain per term, summed low to high
        float acc[3][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            // dims 32 tig + 4 kk + {0,1} and {2,3}: words 2kk, 2kk+1 of the slice
            const uint4 &k0 = kr[0][kk >> 1], &k1 = kr[1][kk >> 1];
            const uint32_t a0 = (kk & 1) ? k0.z : k0.x, a2 = (kk & 1) ? k0.w : k0.y;
            const uint32_t a1 = (kk & 1) ? k1.z : k1.x, a3 = (kk & 1) ? k1.w : k1.y;
#pragma unroll
            for (int term = 0; term < 3; ++term) mma16816(acc[term], a0, a1, a2, a3, qb[term][kk][0], qb[term][kk][1]);
        }
        // s[0], s[1]: token t0 + gid, heads 2tig, 2tig+1; s[2], s[3]: token t0 + gid + 8
        float s[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i] = (acc[2][i] + acc[1][i]) + acc[0][i];
        if (t0 + gid >= hi) s[0] = s[1] = -INFINITY;
        if (t0 + 8 + gid >= hi) s[2] = s[3] = -INFINITY;
        // online softmax per head; token t0 < hi, so every head's tile max is finite
        float alpha[2], mnew[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float tmax = fmaxf(s[c], s[2 + c]);
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
            mnew[c] = fmaxf(m_run[c], tmax);
            alpha[c] = exp2f(m_run[c] - mnew[c]);
            m_run[c] = mnew[c];
        }
        float p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = exp2f(s[i] - mnew[i & 1]);
#pragma unroll
        for (int c = 0; c < 2; ++c) l_run[c] = l_run[c] * alpha[c] + (p[c] + p[2 + c]);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            o[mt][0] *= alpha[0]; o[mt][1] *= alpha[1];
            o[mt][2] *= alpha[0]; o[mt][3] *= alpha[1];
        }
        // p^T as the B operand: the bf16 pairs (tokens gid / gid + 8, heads
        // 2tig, 2tig+1) transposed to (tokens 2tig, 2tig+1 / 2tig+8, 2tig+9, head gid)
        float ph[4], pl[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ph[i] = __bfloat162float(__float2bfloat16_rn(p[i]));
            pl[i] = p[i] - ph[i];
        }
        const uint32_t b0h = movm_trans(bf16x2(ph[0], ph[1])), b1h = movm_trans(bf16x2(ph[2], ph[3]));
        const uint32_t b0l = movm_trans(bf16x2(pl[0], pl[1])), b1l = movm_trans(bf16x2(pl[2], pl[3]));
        // O^T += V^T P^T: m-tile mt takes word mt (elements 2mt, 2mt+1) of each token's slice
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const uint32_t w_r0 = (&vr[0][mt >> 2].x)[mt & 3];
            const uint32_t w_r1 = (&vr[1][mt >> 2].x)[mt & 3];
            const uint32_t w_r2 = (&vr[2][mt >> 2].x)[mt & 3];
            const uint32_t w_r3 = (&vr[3][mt >> 2].x)[mt & 3];
            const uint32_t a0 = __byte_perm(w_r0, w_r1, 0x5410u), a1 = __byte_perm(w_r0, w_r1, 0x7632u);
            const uint32_t a2 = __byte_perm(w_r2, w_r3, 0x5410u), a3 = __byte_perm(w_r2, w_r3, 0x7632u);
            mma16816(o[mt], a0, a1, a2, a3, b0l, b1l);
            mma16816(o[mt], a0, a1, a2, a3, b0h, b1h);
        }
    };

    // two register sets: the next tile's loads go out before this tile's math
    {
        uint4 kA[2][4], vA[4][2], kB[2][4], vB[4][2];
        const long long step = (long long)GQ_WARPS * GQ_TILE;
        long long t0 = lo + (long long)warp * GQ_TILE;
        if (t0 < hi) load_tile(t0, kA, vA);
        while (t0 < hi) {
            const long long t1 = t0 + step;
            if (t1 < hi) load_tile(t1, kB, vB);
            compute_tile(t0, kA, vA);
            if (t1 >= hi) break;
            const long long t2 = t1 + step;
            if (t2 < hi) load_tile(t2, kA, vA);
            compute_tile(t1, kB, vB);
            t0 = t2;
        }
    }
    // warp partials: l summed over the 8 lanes of each tig
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        l_run[c] += __shfl_xor_sync(0xffffffffu, l_run[c], 4);
        l_run[c] += __shfl_xor_sync(0xffffffffu, l_run[c], 8);
        l_run[c] += __shfl_xor_sync(0xffffffffu, l_run[c], 16);
    }
    if (gid == 0) {
#pragma unroll
        for (int c = 0; c < 2; ++c) { s_m[warp][2 * tig + c] = m_run[c]; s_l[warp][2 * tig + c] = l_run[c]; }
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        *reinterpret_cast<float2 *>(&s_o[warp][2 * tig][16 * gid + 2 * mt]) = make_float2(o[mt][0], o[mt][2]);
        *reinterpret_cast<float2 *>(&s_o[warp][2 * tig + 1][16 * gid + 2 * mt]) = make_float2(o[mt][1], o[mt][3]);
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
