// Prefill attention of a prompt ("Full Attention Strikes Back", gist.science
// technical summary, Method section 1): every prompt token attends causally
// to the cached tokens at or before it; a local head keeps only the attention
// sinks and the sliding window, a retrieval head keeps every earlier token
// (the full KV cache).  bf16 queries and caches, fp32 accumulation and
// output.
//
// One CTA per (query block, sequence b, KV group g): BQ consecutive prompt
// tokens x all G query heads of the group, on the tensor cores
// (mma.sync m16n8k16, FlashAttention-2 layout).  Warp w owns 16 query rows
// of one head: head w / NSUB, tokens 16 (w % NSUB) .. + 15 of the block,
// NSUB = 8 / G sub-blocks (BQ = 16 NSUB), so that the G heads share every
// staged K/V tile.
//   S = Q K^T   A = Q (16 rows x 16 dims per k-step, from registers),
//               B = K^T from the staged tile (ldmatrix)
//   O += P V    A = P in bf16 as a 2-term split (the softmax weights keep
//               ~16 bits), B = V from the staged tile (ldmatrix.trans)
// K/V tiles of PF_BK keys stream through a 2-stage cp.async ring (rows
// padded to PF_PITCH bytes: the 8 rows of one ldmatrix matrix fall on
// distinct banks).  The key tiles a block visits are the sink range
// [0, n_sink) and the window range ending at the block's last token (the
// union, each tile once); a per-element mask makes the set exact.
#pragma once

#include "rtp_attend.cuh"

namespace rtp {

constexpr int PF_WARPS = 8;
constexpr int PF_THREADS = PF_WARPS * 32;
constexpr int PF_BK = 64;                        // keys per tile
constexpr int PF_PITCH = D * 2 + 16;             // bytes per staged row
constexpr int PF_TILE_BYTES = PF_BK * PF_PITCH;  // one K or V tile
constexpr int PF_SMEM = 2 * 2 * PF_TILE_BYTES;   // 2 stages x (K, V)

struct PrefillArgs {
    int B, H_q, H_kv, G;
    long long N_max;
    int T;                       // prompt tokens per sequence
    int nsub;                    // 16-row sub-blocks per head in a CTA (BQ = 16 nsub)
    int n_qblk;                  // query blocks per sequence
    const int32_t *seq_lens;     // [B] device
    const int32_t *pos0;         // [B] device: position of prompt token 0
    uint8_t hc[MAX_GROUPS];      // head class per KV head
    int window, n_sink;
    float scale_log2;
    const __nv_bfloat16 *q;      // [B, H_q, T, D]
    const __nv_bfloat16 *k;      // [B, H_kv, N_max, D]
    const __nv_bfloat16 *v;
    float *out;                  // [B, H_q, T, D]
    uint32_t *status;
    KvMap kv;                    // row addressing of k / v
};

__device__ __forceinline__ void pf_cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void pf_cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void pf_cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void pf_ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void pf_ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D = A.B + D, all 16 rows of A used
__device__ __forceinline__ void pf_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pf_pack_bf16(float lo, float hi) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}

// Key tiles of a query block whose tokens sit at positions [P0, P1]: the
// union of the sink tiles and the window tiles, as two tile ranges
// [0, s_tiles) and [w_t0, w_t1) that do not overlap.
struct TileRanges {
    int s_tiles, w_t0, w_t1;
    __device__ __forceinline__ int count() const { return s_tiles + (w_t1 - w_t0); }
    __device__ __forceinline__ int tile(int i) const { return i < s_tiles ? i : w_t0 + (i - s_tiles); }
};
__device__ __forceinline__ TileRanges prefill_tiles(int P0, int P1, bool local, int window, int n_sink) {
    TileRanges r;
    const int end = P1 / PF_BK + 1;                         // tiles up to the last visible key
    if (!local) { r.s_tiles = 0; r.w_t0 = 0; r.w_t1 = end; return r; }
    const long long wlo = max(0LL, (long long)P0 - window + 1);   // first key any token's window holds
    const int s_end = min(n_sink, P1 + 1);
    const int s_tiles = (s_end + PF_BK - 1) / PF_BK;
    const int w0 = (int)(wlo / PF_BK);
    if (w0 <= s_tiles) { r.s_tiles = 0; r.w_t0 = 0; r.w_t1 = end; return r; }
    r.s_tiles = s_tiles; r.w_t0 = w0; r.w_t1 = end;
    return r;
}

__global__ void __launch_bounds__(PF_THREADS, 1) prefill_attn_kernel(PrefillArgs a) {
    extern __shared__ __align__(128) uint8_t psm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int b = blockIdx.y / a.H_kv, g = blockIdx.y % a.H_kv;
    // the longest blocks (last tokens of a retrieval group) go first
    const int qb = a.n_qblk - 1 - (int)blockIdx.x;
    const int BQ = 16 * a.nsub;
    const int G = a.G;
    const int N = a.seq_lens[b];
    const int p0 = a.pos0[b];
    const int t_lo = qb * BQ;                                // first prompt token of the block
    const int t_hi = min(a.T, t_lo + BQ);                    // past the last
    const int hw = warp / a.nsub;                            // this warp's head within the group
    const bool has_rows = hw < G;
    const int tw0 = t_lo + 16 * (warp % a.nsub);             // this warp's first token
    if (p0 < 0 || N > a.N_max || (long long)p0 + a.T > (long long)N) {
        if (tid == 0) set_status(a.status, RTP_ERR_DEVICE_ARG);
        if (has_rows)
            for (int i = lane; i < 16 * D; i += 32) {
                const int t = tw0 + i / D;
                if (t < a.T) a.out[(((size_t)b * a.H_q + (size_t)g * G + hw) * a.T + t) * D + i % D] = 0.0f;
            }
        return;
    }
    const bool local = a.hc[g] == RTP_HEAD_LOCAL;
    const int P0 = p0 + t_lo, P1 = p0 + t_hi - 1;           // positions of the block's tokens
    const TileRanges tr = prefill_tiles(P0, P1, local, a.window, a.n_sink);
    const int n_tiles = tr.count();


    // stage tile i: 64 rows of K then of V, 16 bytes per thread per copy;
    // rows past P1 repeat row P1 (finite; masked below)
    auto stage = [&](int i, int s) {
        const int key0 = tr.tile(i) * PF_BK;
        uint8_t *ks = psm + s * 2 * PF_TILE_BYTES, *vs = ks + PF_TILE_BYTES;
#pragma unroll
        for (int c = tid; c < PF_BK * (D * 2 / 16); c += PF_THREADS) {
            const int r = c >> 4, piece = c & 15;
            const long long row = max(0LL, kv_row(a.kv, b, g, min(key0 + r, P1)));
            pf_cp_async16(ks + r * PF_PITCH + piece * 16, a.k + row * D + piece * 8);
            pf_cp_async16(vs + r * PF_PITCH + piece * 16, a.v + row * D + piece * 8);
        }
    };
    if (n_tiles > 0) stage(0, 0);
    pf_cp_async_commit();

    // Q fragments of this warp's 16 rows (tokens tw0 + gid, tw0 + gid + 8):
    // k-step kk covers dims 16 kk .. 16 kk + 15
    uint32_t qa[8][4];
    {
        const int t0 = min(tw0 + gid, a.T - 1), t1 = min(tw0 + gid + 8, a.T - 1);
        const size_t hrow = ((size_t)b * a.H_q + (size_t)g * G + (has_rows ? hw : 0)) * a.T;
        const uint32_t *q0 = reinterpret_cast<const uint32_t *>(a.q + (hrow + t0) * D);
        const uint32_t *q1 = reinterpret_cast<const uint32_t *>(a.q + (hrow + t1) * D);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qa[kk][0] = __ldg(q0 + 8 * kk + tig);
            qa[kk][1] = __ldg(q1 + 8 * kk + tig);
            qa[kk][2] = __ldg(q0 + 8 * kk + 4 + tig);
            qa[kk][3] = __ldg(q1 + 8 * kk + 4 + tig);
        }
    }
    const int qp0 = p0 + tw0 + gid, qp1 = qp0 + 8;          // positions of this thread's two rows
    const bool row0_ok = tw0 + gid < a.T, row1_ok = tw0 + gid + 8 < a.T;

    float o[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;

    // ldmatrix lane addresses: matrix m = lane / 8, row r = lane % 8
    const int lm = lane >> 3, lr = lane & 7;
    for (int i = 0; i < n_tiles; ++i) {
        if (i + 1 < n_tiles) stage(i + 1, (i + 1) & 1);
        pf_cp_async_commit();
        pf_cp_async_wait<1>();
        __syncthreads();
        const int key0 = tr.tile(i) * PF_BK;
        const uint8_t *ks = psm + (i & 1) * 2 * PF_TILE_BYTES, *vs = ks + PF_TILE_BYTES;
        if (has_rows) {
            // S = Q K^T over the tile's 64 keys: n-tile j = keys 8j .. 8j + 7
            float s[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.0f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
                for (int jp = 0; jp < 4; ++jp) {
                    // matrices: (n-tile 2jp, dims lo), (2jp, hi), (2jp+1, lo), (2jp+1, hi)
                    const int key = 8 * (2 * jp + (lm >> 1)) + lr;
                    const uint32_t addr = smem_u32(ks + key * PF_PITCH + (16 * kk + 8 * (lm & 1)) * 2);
                    uint32_t b0, b1, b2, b3;
                    pf_ldsm_x4(addr, b0, b1, b2, b3);
                    pf_mma(s[2 * jp], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
                    pf_mma(s[2 * jp + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
                }
            }
            // mask, scale to log2 units, row maxima
            float tmax0 = -INFINITY, tmax1 = -INFINITY;
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int kp = key0 + 8 * j + 2 * tig + c;
                    const bool v0 = row0_ok && kp <= qp0 && (!local || kp < a.n_sink || qp0 - kp < a.window);
                    const bool v1 = row1_ok && kp <= qp1 && (!local || kp < a.n_sink || qp1 - kp < a.window);
                    s[j][c] = v0 ? s[j][c] * a.scale_log2 : -INFINITY;
                    s[j][2 + c] = v1 ? s[j][2 + c] * a.scale_log2 : -INFINITY;
                    tmax0 = fmaxf(tmax0, s[j][c]);
                    tmax1 = fmaxf(tmax1, s[j][2 + c]);
                }
            tmax0 = fmaxf(tmax0, __shfl_xor_sync(0xffffffffu, tmax0, 1));
            tmax0 = fmaxf(tmax0, __shfl_xor_sync(0xffffffffu, tmax0, 2));
            tmax1 = fmaxf(tmax1, __shfl_xor_sync(0xffffffffu, tmax1, 1));
            tmax1 = fmaxf(tmax1, __shfl_xor_sync(0xffffffffu, tmax1, 2));
            const float mn0 = fmaxf(m0, tmax0), mn1 = fmaxf(m1, tmax1);
            const float al0 = mn0 == -INFINITY ? 1.0f : exp2f(m0 - mn0);
            const float al1 = mn1 == -INFINITY ? 1.0f : exp2f(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            float rs0 = 0.0f, rs1 = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    s[j][c] = mn0 == -INFINITY ? 0.0f : exp2f(s[j][c] - mn0);
                    s[j][2 + c] = mn1 == -INFINITY ? 0.0f : exp2f(s[j][2 + c] - mn1);
                    rs0 += s[j][c];
                    rs1 += s[j][2 + c];
                }
            l0 = l0 * al0 + rs0;
            l1 = l1 * al1 + rs1;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                o[j][0] *= al0; o[j][1] *= al0;
                o[j][2] *= al1; o[j][3] *= al1;
            }
            // O += P V: k-step kk2 = keys 16 kk2 .. 16 kk2 + 15 (n-tiles 2kk2,
            // 2kk2 + 1 of S), n-tile jd = dims 8 jd .. 8 jd + 7
#pragma unroll
            for (int kk2 = 0; kk2 < 4; ++kk2) {
                uint32_t ph[4], pl[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // a0: (row gid, n-tile 2kk2), a1: (row gid+8, 2kk2), a2: (gid, 2kk2+1), a3: (gid+8, 2kk2+1)
                    const int j = 2 * kk2 + (e >> 1);
                    const int c = 2 * (e & 1);
                    const float x0 = s[j][c], x1 = s[j][c + 1];
                    const float h0 = __bfloat162float(__float2bfloat16_rn(x0));
                    const float h1 = __bfloat162float(__float2bfloat16_rn(x1));
                    ph[e] = pf_pack_bf16(h0, h1);
                    pl[e] = pf_pack_bf16(x0 - h0, x1 - h1);
                }
#pragma unroll
                for (int jp = 0; jp < 8; ++jp) {
                    // matrices: (keys lo, dims 2jp), (keys hi, 2jp), (lo, 2jp+1), (hi, 2jp+1)
                    const int key = 16 * kk2 + 8 * (lm & 1) + lr;
                    const uint32_t addr = smem_u32(vs + key * PF_PITCH + 8 * (2 * jp + (lm >> 1)) * 2);
                    uint32_t b0, b1, b2, b3;
                    pf_ldsm_x4_t(addr, b0, b1, b2, b3);
                    pf_mma(o[2 * jp], pl[0], pl[1], pl[2], pl[3], b0, b1);
                    pf_mma(o[2 * jp], ph[0], ph[1], ph[2], ph[3], b0, b1);
                    pf_mma(o[2 * jp + 1], pl[0], pl[1], pl[2], pl[3], b2, b3);
                    pf_mma(o[2 * jp + 1], ph[0], ph[1], ph[2], ph[3], b2, b3);
                }
            }
        }
        __syncthreads();          // the stage is free for the copy issued next round
    }
    pf_cp_async_wait<0>();
    if (!has_rows) return;
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float inv0 = l0 > 0.0f ? 1.0f / l0 : 0.0f, inv1 = l1 > 0.0f ? 1.0f / l1 : 0.0f;
    const size_t hrow = ((size_t)b * a.H_q + (size_t)g * G + hw) * a.T;
#pragma unroll
    for (int jd = 0; jd < 16; ++jd) {
        const int dcol = 8 * jd + 2 * tig;
        if (row0_ok)
            *reinterpret_cast<float2 *>(a.out + (hrow + tw0 + gid) * D + dcol) =
                make_float2(o[jd][0] * inv0, o[jd][1] * inv0);
        if (row1_ok)
            *reinterpret_cast<float2 *>(a.out + (hrow + tw0 + gid + 8) * D + dcol) =
                make_float2(o[jd][2] * inv1, o[jd][3] * inv1);
    }
}

}  // namespace rtp
