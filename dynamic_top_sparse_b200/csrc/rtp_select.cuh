// Indexer scoring and the sort-free top-p threshold (sm_100a).
//
// "Full Attention Strikes Back" (gist.science technical summary), Method
// sections 2, 3 and 5: retrieval heads score every cached token in a
// 16-dim pre-RoPE subspace, turn the scores into softmax mass, and keep the
// smallest descending-score prefix whose mass reaches p; the kernels find
// that threshold with histograms instead of a sort.
//
// Stages (per sequence b and retrieval KV head g; all G <= 8 query heads of
// the group are scored from one read of each index-key row):
//   scan      q_idx = W_q_idx . q (in-kernel), logits z for every token, and
//             a level-1 mass histogram per head over the order-preserving
//             bits of z: sign, exponent and 4 mantissa bits for |z| in
//             [2^-6, 2^10) (512 bins, relative width 1/16; |z| < 2^-6 shares
//             the innermost bin of its sign).  Each bin sums exp(z - U_b),
//             U_b its upper edge, so every term is in (e^-32, 1], no maximum
//             is needed while streaming, and CTAs' bins add directly.  The
//             largest bin of every 32-token tile is recorded.  The last CTA
//             of the group resolves each head: R = U(top bin), bin masses
//             S_b exp(U_b - R), and the boundary bin b* where the mass
//             accumulated from the top first reaches p Z.
//   collect   re-derive the logits of tiles whose largest bin reaches b*;
//             tokens above b* are kept, tokens in b* become candidates
//             (64-bit key: order-preserving logit bits, then the inverted
//             token id, so the order is total and equal logits go to the
//             lower id first).
//   finalize  exact radix select by mass over the candidates: 8-bit digits
//             of the key from the first bit where candidates differ, digit
//             masses summed in fixed point (order-independent), down to the
//             unique boundary token; candidates at or above it are kept.
//
#pragma once

#include <type_traits>

#include <cooperative_groups.h>

#include "rtp_common.cuh"

namespace rtp {

constexpr int SC_THREADS = 256;
constexpr int SC_WARPS = SC_THREADS / 32;
constexpr int TILE = 32;                   // tokens per warp tile
constexpr int MAX_RET_GROUPS = 64;
constexpr float L2E = 1.4426950408889634f;     // log2(e)
constexpr double L2E_D = 1.4426950408889634;

enum ResolveMode : int32_t { MODE_NORMAL = 0, MODE_KEEP_ALL = 1, MODE_EMPTY = 2 };

// Level-1 bins over the fp32 logit bits: k = (exponent, top MB mantissa bits)
// of |z| relative to 2^E_LO, clamped to [0, 255]; bin = 256 + k for z > 0
// and 255 - k for z <= 0, so bin order follows z.
constexpr int MB = 4;
constexpr int E_LO = -6;
constexpr int NBIN = 512;
// Octaves: bins 16 s .. 16 s + 15 (one exponent of |z|, one sign) form
// super-bin s; each head's histogram holds its NBIN bin sums followed by the
// NSUP octave sums, so a resolve can read the 32 octave sums first and then
// only the bins of the octave that holds the boundary.
constexpr int NSUP = NBIN / 16;
// The octave sums are kept in NREP replicas (a CTA adds to replica
// blockIdx.x mod NREP; the resolve sums them): the scan's CTAs all add their
// octave sums at the same moment, and one copy packed into two lines per
// head queued ~1000 fp64 atomics per line.
constexpr int NREP = 4;
constexpr int HSTRIDE = NBIN + NREP * NSUP;   // doubles per head
constexpr uint32_t BIN_BASE = (uint32_t)(127 + E_LO) << MB;   // k = (bits >> 19) - BIN_BASE
constexpr float Z_LIMIT = 256.0f;   // logits beyond are reported (bins up to 16 nats wide stay resolvable)

// 2^x with the SFU (ex2.approx.ftz: relative error ~2^-22 on the range used
// here, |x| <= 47).
__device__ __forceinline__ float ex2_sfu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^y in fp64 range: 2^floor(y) exact (built from its exponent bits; 0 below
// the normal range), 2^frac(y) by the SFU (relative error ~2^-22).  For
// octave-level factors, which span far more than fp32's range.
__device__ __forceinline__ double exp2_wide(double y) {
    const double n = floor(y);
    const int e = (int)fmax(fmin(n, 1023.0), -1023.0);
    const double p2 = e < -1022 ? 0.0 : __longlong_as_double((long long)(e + 1023) << 52);
    return (double)ex2_sfu((float)(y - n)) * p2;
}

// Per-CTA bin sums are kept in fixed point: FX_ONE units per unit of mass
// (every term is in (e^-32, 1], so terms below 2^-20 of a bin's upper edge
// -- only possible for |z| >= 232 -- round to zero), as a 64-bit value split
// over two 32-bit shared counters; the thread whose add wraps the low word
// (seen in the value atomicAdd returns) carries into the high word, so the
// sums are exact and independent of the order of the adds.
constexpr float FX_ONE = 1048576.0f;   // 2^20

// Bin of z (z already folded so that -0 is +0) and exp(z - U_bin) in fixed point.
__device__ __forceinline__ int bin_and_fx(float z, uint32_t &fx) {
    const uint32_t u = __float_as_uint(z);
    const int s = (int)u >> 31;                                // 0 or -1
    int k = (int)((u << 1) >> (24 - MB)) - (int)BIN_BASE;
    k = min(max(k, 0), 255);
    const uint32_t eb = (uint32_t)(k + (int)BIN_BASE + 1 + s) << (23 - MB);
    const float U = __uint_as_float(eb | ((uint32_t)s & 0x80000000u));
    fx = __float2uint_rn(ex2_sfu((z - U) * L2E) * FX_ONE);
    return 256 + (k ^ s);
}

// Largest and smallest float of a bin (the bins partition the floats, with
// -0 counted as +0): z is in a bin above b  <=>  z > bin_hi_incl(b), and z is
// in b  <=>  bin_lo_incl(b) <= z <= bin_hi_incl(b).
__host__ __device__ __forceinline__ float bits_f(uint32_t u) {
    union { uint32_t u; float f; } c; c.u = u; return c.f;
}
__host__ __device__ __forceinline__ float bin_hi_incl(int bin) {
    if (bin >= 256) {
        const int k = bin - 256;
        if (k == 255) return bits_f(0x7f800000u);                         // +inf
        return bits_f(((uint32_t)(k + 1 + (int)BIN_BASE) << (23 - MB)) - 1u);
    }
    const int k = 255 - bin;
    if (k == 0) return bits_f(0x80000001u);                               // -denorm_min
    return bits_f(((uint32_t)(k + (int)BIN_BASE) << (23 - MB)) | 0x80000000u);
}
__host__ __device__ __forceinline__ float bin_lo_incl(int bin) {
    if (bin >= 256) {
        const int k = bin - 256;
        if (k == 0) return 0.0f;
        return bits_f((uint32_t)(k + (int)BIN_BASE) << (23 - MB));
    }
    const int k = 255 - bin;
    if (k == 255) return bits_f(0xff800000u);                             // -inf
    return bits_f((((uint32_t)(k + 1 + (int)BIN_BASE) << (23 - MB)) - 1u) | 0x80000000u);
}

// Upper edge of a bin, as used by bin_and_fx.
__host__ __device__ __forceinline__ float bin_upper(int bin) {
    union { uint32_t u; float f; } c;
    if (bin >= 256) {
        c.u = (uint32_t)(bin - 256 + (int)BIN_BASE + 1) << (23 - MB);
        return c.f;
    }
    c.u = (uint32_t)(255 - bin + (int)BIN_BASE) << (23 - MB);
    return -c.f;
}

// exp(U_b - U_octave(b)): a bin's mass relative to its octave's upper edge
// per unit of mass relative to its own (a constant of the bin; the scans
// tabulate it in shared memory while they stream).
__device__ __forceinline__ double octave_factor(int bin) {
    return exp2_wide((double)(bin_upper(bin) - bin_upper(bin | 15)) * L2E_D);
}

// A CTA's fixed-point bin sum v (< 2^52) times `unit` as a double, without
// a conversion instruction: v OR-ed into the mantissa of 2^52 is exactly
// 2^52 + v, and one fma removes the 2^52.
__device__ __forceinline__ double fixed_to_double(unsigned long long v, double unit) {
    return fma(__longlong_as_double((long long)(0x4330000000000000ull | v)), unit, -4503599627370496.0 * unit);
}

// The same for a 64-bit fixed-point sum: its two 32-bit halves, each exact,
// added with one rounding.
__device__ __forceinline__ double wide_fixed_to_double(unsigned long long v, double unit) {
    return fixed_to_double(v >> 32, 4294967296.0 * unit) + fixed_to_double(v & 0xffffffffull, unit);
}

// Wide bins.  A bin spans 1/16 of an octave of |z|, so from |z| = 32 on it is
// 2 to 8 nats wide and a value near its bottom weighs e^-8 of its upper
// edge: at 2^18 or 2^20 units per unit of mass such a term keeps only a
// few bits.  The scans add the values of these bins (k in [K_WIDE, K_TOP],
// |z| in [32, 256), both signs: NWIDE bins per head) to separate 64-bit
// counters at 2^38 units per unit of mass instead: an fp32 term times 2^38
// converts exactly, so every term keeps fp32's relative precision, and the
// sums stay below 2^64 for up to 2^25 values of one bin in one CTA.
constexpr int K_WIDE = (int)((127 + 5) << MB) - (int)BIN_BASE;      // |z| >= 32
constexpr int K_TOP = (int)((127 + 7) << MB) + 15 - (int)BIN_BASE;  // |z| < 256
constexpr int NWK = K_TOP - K_WIDE + 1;                            // wide k values per sign
constexpr int NWIDE = 2 * NWK;
constexpr float WIDE_Z = 32.0f;
constexpr float FX38_EXP2 = 38.0f;
constexpr double FX38_UNIT = 1.0 / 274877906944.0;                  // 2^-38
constexpr long long MAX_CTA_TOKENS = 1ll << 24;                     // per scan CTA
// slot of a bin among the head's wide counters, or -1
__host__ __device__ __forceinline__ int wide_slot(int bin) {
    const int k = bin >= 256 ? bin - 256 : 255 - bin;
    if (k < K_WIDE || k > K_TOP) return -1;
    return (bin >= 256 ? 0 : NWK) + (k - K_WIDE);
}

// Adds a CTA's bin sums of G heads to the histograms (gh0: the first head's;
// heads HSTRIDE apart).  bin_mass(i) = mass of entry i = head * NBIN + bin
// relative to the bin's upper edge; fac = the octave factors; rep = the
// CTA's octave replica.  One atomic per non-empty bin; the loop is
// warp-aligned (G * NBIN and blockDim are multiples of 32), so 16
// consecutive lanes hold one octave, whose sum relative to the octave's
// upper edge is formed across the half-warp (fixed order) and added to the
// octave's replica slot.
template <typename BinMass>
__device__ __forceinline__ void flush_hist(double *gh0, int G, const double *fac, int rep, const BinMass &bin_mass) {
    for (int i = threadIdx.x; i < G * NBIN; i += blockDim.x) {
        const double m = bin_mass(i);
        double *gh = gh0 + (size_t)(i / NBIN) * HSTRIDE;
        if (m != 0.0) atomicAdd(gh + i % NBIN, m);
        double x = m * fac[i % NBIN];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if ((threadIdx.x & 15) == 0 && x != 0.0) atomicAdd(gh + NBIN + rep * NSUP + (i % NBIN) / 16, x);
    }
}

struct Resolve {
    double Z;          // total mass, relative to exp(R)
    double above;      // mass of the bins above b*, same units
    double target;     // mass still needed inside b*, same units (inf: keep all of b*)
    float R;           // reference logit: upper edge of the top bin
    int32_t bstar;     // boundary bin
    int32_t mode;      // ResolveMode
    int32_t N;         // valid tokens
};
static_assert(sizeof(Resolve) == 40, "Resolve layout");

struct SelWs {
    uint32_t *status;
    uint32_t *cand_cnt;          // [B*H_q] at stride CNT_STRIDE
    uint32_t *list_cnt;          // [B*H_q] at stride CNT_STRIDE
    double *hist;                // [B*H_q][HSTRIDE]: bin sums, then octave sums
    Resolve *res;                // [B*H_q]
    uint16_t *tilebin;           // [B*H_kv][ntile][GMAX]: per tile, 1 + largest bin of each head (0: none)
    unsigned long long *cands;   // [B*H_q][N_max]
    float *qidx;                 // [B*H_q][R]
};

struct SelArgs {
    int B, H_q, H_kv, G;
    long long N_max;
    int ntile;
    int ctas;                    // scan/collect CTAs per (b, g)
    long long chunk;             // tokens per CTA, multiple of TILE
    int cl_ctas;                 // collect_mma_kernel CTAs per pair of groups (tile i -> CTA i mod cl_ctas)
    const int32_t *seq_lens;
    int n_ret;
    int ret_g[MAX_RET_GROUPS];
    float p;
    // > 0: keep the topk largest logits of each head instead of the top-p
    // set (static top-k, the fixed budget Method section 3 sets top-p
    // against): every token counts one unit where top-p counts its mass
    int topk;
    float idx_scale;
    const float *q;              // [B, H_q, D] pre-RoPE queries
    const float *Wq;             // [H_q, R, D]
    const void *kidx;            // [B, H_kv, N_max, R]
    const float *z;              // [B, H_q, N_max] (given logits)
    int32_t *lists;              // [B*H_q][N_max] kept ids
    int32_t *count_out;          // [B*H_q]
    float *mass_out;             // [B*H_q] or null
    // Fused sparse attention of a decode step (bf16 caches); q_rope null = off.
    // Every collect CTA attends the rows it kept and writes one partial per
    // head of its pair of groups; finalize attends the boundary bin's kept
    // rows and merges.  A head whose kept rows overflowed a CTA's staging is
    // attended wholly by finalize (ovf flag).
    const float *q_rope;                 // [B, H_q, D]
    const __nv_bfloat16 *k_cache;        // [B, H_kv, N_max, D], or page pools (kv)
    const __nv_bfloat16 *v_cache;
    KvMap kv;                            // row addressing of k_cache / v_cache
    float attn_scale_log2;
    float *out;                          // [B, H_q, D]
    float *part_sel;                     // [collect CTAs][2 GMAX][PSTRIDE] (pair-heads)
    uint32_t *ovf;                       // [B*H_q]
    // Hand-over of large heads: a head whose rows left to finalize exceed
    // spill_rows (> 0) is not attended by finalize's cluster; finalize
    // stores its partial in slot 0 of the head's list partials (part_list)
    // and flags the head in ovf (SPILL_FROM_FIRST / SPILL_ALL_ROWS) for a
    // list pass over all SMs.
    int spill_rows;
    float *part_list;                    // [B*H_q][LIST_SLOTS][PSTRIDE]
    uint32_t *spill_any;                 // set when any head was handed over (the scan clears it)
    // Context shard (all null: whole sequences).  The shard holds global
    // tokens [id_off[b], id_off[b] + seq_lens[b]); collect writes global ids
    // (kept lists, candidate keys); finalize takes every shard's boundary
    // candidates from ext_cands [B*H_q][ext_stride] with ext_cnt[bh] each,
    // and writes each head's threshold key to theta_out instead of lists
    // and counts (shard_own_kernel appends this shard's kept candidates).
    const int32_t *id_off;
    const unsigned long long *ext_cands;
    const int32_t *ext_cnt;
    long long ext_stride;
    unsigned long long *theta_out;
};

// Record `r` of a cluster (the same shared variable in CTA rank r); the CTA's
// own copy when the kernel runs without clusters.
__device__ __forceinline__ const float *cluster_rec(cooperative_groups::cluster_group &cl, float *rec, int r,
                                                    int K) {
    return K > 1 ? cl.map_shared_rank(rec, r) : rec;
}

// ---------------------------------------------------------------------------
// fused sparse attention helpers
// ---------------------------------------------------------------------------
// Running flash-decoding partial of one head held by one warp (log2 units);
// lane l holds dims 4l .. 4l + 3 of o.
struct WarpPart {
    float m, l, o[4];
    __device__ __forceinline__ void reset() {
        m = -INFINITY; l = 0.0f;
        o[0] = o[1] = o[2] = o[3] = 0.0f;
    }
    // fold in another partial (mx, lx, ox) of the same head
    __device__ __forceinline__ void add(float mx, float lx, const float (&ox)[4]) {
        if (mx == -INFINITY) return;
        const float mn = fmaxf(m, mx);
        const float a0 = m == -INFINITY ? 0.0f : exp2f(m - mn), a1 = exp2f(mx - mn);
        l = l * a0 + lx * a1;
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = o[i] * a0 + ox[i] * a1;
        m = mn;
    }
    // write as a record (m, l at [0], [1]; o at [POFF + 4 lane ..])
    __device__ __forceinline__ void store(float *rec) const {
        const int lane = threadIdx.x & 31;
        if (lane == 0) { rec[0] = m; rec[1] = l; }
        *reinterpret_cast<float4 *>(rec + POFF + 4 * lane) = make_float4(o[0], o[1], o[2], o[3]);
    }
    __device__ __forceinline__ void load_add(const float *rec) {
        const int lane = threadIdx.x & 31;
        const float mx = rec[0], lx = rec[1];
        const float4 v = *reinterpret_cast<const float4 *>(rec + POFF + 4 * lane);
        const float ox[4] = {v.x, v.y, v.z, v.w};
        add(mx, lx, ox);
    }
};

// The warp attends up to 8 rows of one head: lane u < 8 holds row id `id`
// (-1: none), all 16 row loads in flight before the dot products.  qx: the
// lane's 4 query dims times the softmax scale times log2(e).
// Pulls the K and V rows of one token (bf16, D = 128: two 128-byte lines
// each) toward L2, so that a later gather of the row finds it there.
__device__ __forceinline__ void prefetch_kv_l2(const __nv_bfloat16 *k_row, const __nv_bfloat16 *v_row) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(k_row));
    asm volatile("prefetch.global.L2 [%0];" ::"l"(k_row + 64));
    asm volatile("prefetch.global.L2 [%0];" ::"l"(v_row));
    asm volatile("prefetch.global.L2 [%0];" ::"l"(v_row + 64));
}

// PAGED: rows through the block table of a page pool (km.table), else the
// contiguous (b, g) slab with 32-bit token offsets.
template <bool PAGED>
__device__ __forceinline__ void attend8(const __nv_bfloat16 *kc, const __nv_bfloat16 *vc, const KvMap &km, int b,
                                        int g, int id, const float (&qx)[4], WarpPart &p) {
    const int lane = threadIdx.x & 31;
    float kx[8][4], vx[8][4];
    bool ok[8];
    long long ro = id;                                             // lanes 0-7: their token's row
    if constexpr (PAGED) {
        ro = id >= 0 ? kv_row(km, b, g, id) : -1LL;
    } else {
        const long long base = ((long long)b * km.H_kv + g) * km.N_max * D;
        kc += base;
        vc += base;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        long long r;
        if constexpr (PAGED) r = __shfl_sync(0xffffffffu, ro, u);
        else r = __shfl_sync(0xffffffffu, id, u);
        ok[u] = r >= 0;
        if (ok[u]) {
            Row<__nv_bfloat16>::load4(kc + r * D + lane * 4, kx[u]);
            Row<__nv_bfloat16>::load4(vc + r * D + lane * 4, vx[u]);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) kx[u][i] = vx[u][i] = 0.0f;
        }
    }
    float sc[8];
    float mb = -INFINITY;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        float sv = qx[0] * kx[u][0];
        sv = fmaf(qx[1], kx[u][1], sv);
        sv = fmaf(qx[2], kx[u][2], sv);
        sv = fmaf(qx[3], kx[u][3], sv);
        sv = warp_sum(sv);
        sc[u] = ok[u] ? sv : -INFINITY;
        mb = fmaxf(mb, sc[u]);
    }
    const float mn = fmaxf(p.m, mb);
    if (mn == -INFINITY) return;
    const float al = exp2f(p.m - mn);
    p.l *= al;
#pragma unroll
    for (int i = 0; i < 4; ++i) p.o[i] *= al;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const float pw = exp2f(sc[u] - mn);
        p.l += pw;
#pragma unroll
        for (int i = 0; i < 4; ++i) p.o[i] = fmaf(pw, vx[u][i], p.o[i]);
    }
    p.m = mn;
}

__device__ __forceinline__ int checked_len(int N, long long N_max, uint32_t *status) {
    if (N < 1 || (long long)N > N_max) {
        set_status(status, RTP_ERR_DEVICE_ARG);
        return 0;
    }
    return N;
}
__device__ __forceinline__ int valid_len(const int32_t *seq_lens, int b, long long N_max,
                                         uint32_t *status) {
    return checked_len(seq_lens[b], N_max, status);
}

// q_idx of the group's heads into shared memory.  Output o = h * R + j
// (head h, index dim j) is one warp's dot product of q[h] with row o of
// W_q_idx: lane l owns dims 4l .. 4l + 3, and the warp sums the lanes with
// warp_sum, so the value does not depend on which warp computes it (every
// CTA and every kernel gets bit-identical q_idx).  The nwarps warps of the
// caller (warp index `warp`) take outputs warp, warp + nwarps, ..., all of
// their loads in flight at once; PER_WARP >= ceil(G * R / nwarps).
template <int PER_WARP>
struct QProj {
    float acc[PER_WARP];
    // loads and per-lane partial dot products
    __device__ __forceinline__ void load(const float *__restrict__ q_bh0, const float *__restrict__ W_h0, int G,
                                         int warp, int nwarps) {
        const int lane = threadIdx.x & 31;
#pragma unroll
        for (int k = 0; k < PER_WARP; ++k) {
            const int o = warp + k * nwarps;
            acc[k] = 0.0f;
            if (o < G * R) {
                const float4 qv = __ldg(reinterpret_cast<const float4 *>(q_bh0 + (o / R) * D) + lane);
                const float4 wv = __ldg(reinterpret_cast<const float4 *>(W_h0 + (size_t)o * D) + lane);
                float x = qv.x * wv.x;
                x = fmaf(qv.y, wv.y, x);
                x = fmaf(qv.z, wv.z, x);
                x = fmaf(qv.w, wv.w, x);
                acc[k] = x;
            }
        }
    }
    // warp sums -> qs[o]
    __device__ __forceinline__ void store(float scale, float *qs, int G, int warp, int nwarps) {
        const int lane = threadIdx.x & 31;
#pragma unroll
        for (int k = 0; k < PER_WARP; ++k) {
            const int o = warp + k * nwarps;
            const float v = warp_sum(acc[k]);
            if (o < G * R && lane == 0) qs[o] = v * scale;
        }
    }
};

template <int PER_WARP>
__device__ __forceinline__ void project_query(const float *__restrict__ q_bh0,
                                              const float *__restrict__ W_h0, float scale,
                                              float *qs, int G, int warp, int nwarps) {
    QProj<PER_WARP> qp;
    qp.load(q_bh0, W_h0, G, warp, nwarps);
    qp.store(scale, qs, G, warp, nwarps);
}

// ---------------------------------------------------------------------------
// logit sources.  A warp tile is 32 consecutive tokens; each lane gets NV
// values (token offset tok(v), head slot slot(v)); slot s of a lane is head
// head(s).  XOR_LO is the first lane-xor offset over which lanes share slots.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat16 l = __float2bfloat16_rn(lo), h = __float2bfloat16_rn(hi);
    return (uint32_t)__bfloat16_as_ushort(l) | ((uint32_t)__bfloat16_as_ushort(h) << 16);
}

// bf16 index keys on the tensor cores.  m16n8k16: rows = 16 tokens, k = the
// 16 index dims, n = the 8 heads of the group.  The k order is permuted so
// that lane (gid, tig) reads dims 4*tig .. 4*tig+3 of a row with one 8-byte
// load: k slots (2tig, 2tig+1) <- dims (4tig, 4tig+1) and k slots
// (2tig+8, 2tig+9) <- dims (4tig+2, 4tig+3), in A and B alike.
struct SrcMma {
    static constexpr int NV = 8;        // 2 mma tiles x 2 rows x 2 heads
    static constexpr int NSLOT = 2;
    static constexpr int XOR_LO = 4;
    struct Frag { uint2 a[2][2]; };
    const __nv_bfloat16 *rows;          // [N_max][R] of (b, g)
    long long N_max;
    uint32_t bq[3][2];                  // q_idx split hi / mid / lo
    int gid, tig;

    __device__ __forceinline__ void init(const __nv_bfloat16 *r, long long nmax, const float *qs, int G) {
        rows = r; N_max = nmax;
        const int lane = threadIdx.x & 31;
        gid = lane >> 2; tig = lane & 3;
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (gid < G) {
#pragma unroll
            for (int i = 0; i < 4; ++i) x[i] = qs[gid * R + 4 * tig + i];
        }
        float hi[4], mid[4], lo[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            hi[i] = __bfloat162float(__float2bfloat16_rn(x[i]));
            const float r1 = x[i] - hi[i];
            mid[i] = __bfloat162float(__float2bfloat16_rn(r1));
            lo[i] = r1 - mid[i];
        }
        bq[0][0] = pack_bf16(hi[0], hi[1]); bq[0][1] = pack_bf16(hi[2], hi[3]);
        bq[1][0] = pack_bf16(mid[0], mid[1]); bq[1][1] = pack_bf16(mid[2], mid[3]);
        bq[2][0] = pack_bf16(lo[0], lo[1]); bq[2][1] = pack_bf16(lo[2], lo[3]);
    }
    __device__ __forceinline__ void load(int tb, Frag &f) const {
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                int t = tb + 16 * i + gid + 8 * r;
                t = t < N_max ? t : (int)N_max - 1;
                f.a[i][r] = __ldg(reinterpret_cast<const uint2 *>(rows + (size_t)t * R + 4 * tig));
            }
    }
    __device__ __forceinline__ void eval(const Frag &f, float (&z)[NV]) const {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int term = 2; term >= 0; --term)
                mma_bf16_16816(d, f.a[i][0].x, f.a[i][1].x, f.a[i][0].y, f.a[i][1].y, bq[term][0],
                               bq[term][1]);
#pragma unroll
            for (int j = 0; j < 4; ++j) z[4 * i + j] = d[j];
        }
    }
    __device__ __forceinline__ int tok(int v) const { return 16 * (v >> 2) + gid + 8 * ((v >> 1) & 1); }
    __device__ __forceinline__ int slot(int v) const { return v & 1; }
    __device__ __forceinline__ int head(int s) const { return 2 * tig + s; }
};

// fp32 index keys (or bf16 without tensor cores): one token per lane.
template <typename IT>
struct SrcSimt {
    static constexpr int NV = GMAX;
    static constexpr int NSLOT = GMAX;
    static constexpr int XOR_LO = 1;
    struct Frag { float k[R]; };
    const IT *rows;
    long long N_max;
    const float *qs;                    // shared [G][R]
    int G, lane;
    __device__ __forceinline__ void init(const IT *r, long long nmax, const float *q, int g) {
        rows = r; N_max = nmax; qs = q; G = g; lane = threadIdx.x & 31;
    }
    __device__ __forceinline__ void load(int tb, Frag &f) const {
        int t = tb + lane;
        t = t < N_max ? t : (int)N_max - 1;
        float a[8], b[8];
        Row<IT>::load8(rows + (size_t)t * R, a);
        Row<IT>::load8(rows + (size_t)t * R + 8, b);
#pragma unroll
        for (int j = 0; j < 8; ++j) { f.k[j] = a[j]; f.k[8 + j] = b[j]; }
    }
    __device__ __forceinline__ void eval(const Frag &f, float (&z)[NV]) const {
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            float acc = 0.0f;
            if (h < G) {
#pragma unroll
                for (int j = 0; j < R; ++j) acc = __fmaf_rn(qs[h * R + j], f.k[j], acc);
            }
            z[h] = acc;
        }
    }
    __device__ __forceinline__ int tok(int) const { return lane; }
    __device__ __forceinline__ int slot(int v) const { return v; }
    __device__ __forceinline__ int head(int s) const { return s; }
};

// Given logits [G][N_max] of the group's heads.
struct SrcBuffer {
    static constexpr int NV = GMAX;
    static constexpr int NSLOT = GMAX;
    static constexpr int XOR_LO = 1;
    struct Frag { float z[GMAX]; };
    const float *zb;
    long long N_max;
    int G, lane;
    __device__ __forceinline__ void init(const float *z, long long nmax, int g) {
        zb = z; N_max = nmax; G = g; lane = threadIdx.x & 31;
    }
    __device__ __forceinline__ void load(int tb, Frag &f) const {
        int t = tb + lane;
        t = t < N_max ? t : (int)N_max - 1;
#pragma unroll
        for (int h = 0; h < GMAX; ++h) f.z[h] = h < G ? __ldg(zb + h * N_max + t) : 0.0f;
    }
    __device__ __forceinline__ void eval(const Frag &f, float (&z)[NV]) const {
#pragma unroll
        for (int h = 0; h < GMAX; ++h) z[h] = f.z[h];
    }
    __device__ __forceinline__ int tok(int) const { return lane; }
    __device__ __forceinline__ int slot(int v) const { return v; }
    __device__ __forceinline__ int head(int s) const { return s; }
};

// Set up a source for group (b, g); qs holds the scaled q_idx (if used).
template <typename Src>
__device__ __forceinline__ void init_src(Src &src, const SelArgs &a, int b, int g, const float *qs) {
    const size_t bg = (size_t)b * a.H_kv + g;
    if constexpr (std::is_same<Src, SrcMma>::value) {
        src.init(reinterpret_cast<const __nv_bfloat16 *>(a.kidx) + bg * a.N_max * R, a.N_max, qs, a.G);
    } else if constexpr (std::is_same<Src, SrcBuffer>::value) {
        src.init(a.z + ((size_t)b * a.H_q + (size_t)g * a.G) * a.N_max, a.N_max, a.G);
    } else {
        using IT = typename std::remove_cv<typename std::remove_pointer<decltype(src.rows)>::type>::type;
        src.init(reinterpret_cast<const IT *>(a.kidx) + bg * a.N_max * R, a.N_max, qs, a.G);
    }
}

template <typename Src> struct NeedsQ : std::true_type {};
template <> struct NeedsQ<SrcBuffer> : std::false_type {};

// ---------------------------------------------------------------------------
// Resolve one head from its level-1 histogram `gh` (global memory, all of the
// scan's CTAs done).  One warp, two rounds of loads: first the 32 octave
// sums (lane s: octave s), which fix the total mass Z and the octave where
// the mass accumulated from the top first reaches p Z; then the 16 bins of
// that octave (lanes 0-15) and of the top octave (lanes 16-31).  R = upper
// edge of the top non-empty bin; all masses are returned relative to it.  In
// descending bin order b* is the first bin where the cumulative mass reaches
// p Z; `above` is the mass of the bins before it and `target` what b* must
// still supply (infinite: all of b*).  Every lane returns the same record.
// Octave factors are taken in fp64 (octaves can lie hundreds of nats apart);
// bin factors within the boundary octave use the same fp32 expression as
// finalize.
// ---------------------------------------------------------------------------
// With topk > 0 the histogram holds token counts (every octave factor is 1)
// and the target is min(topk, N) tokens; counts are exact in fp64.
__device__ __forceinline__ Resolve resolve_head(const double *__restrict__ gh, float p, int N, int topk) {
    const bool cnt = topk > 0;
    const int lane = threadIdx.x & 31;
    double ss = 0.0;
#pragma unroll
    for (int q = 0; q < NREP; ++q) ss += __ldcg(gh + NBIN + q * NSUP + lane);
    const unsigned ne = __ballot_sync(0xffffffffu, ss > 0.0);
    Resolve r;
    r.N = N;
    if (!ne || N == 0) {
        r.Z = 0; r.above = 0; r.target = 0; r.R = 0.f; r.bstar = -1; r.mode = MODE_EMPTY;
        return r;
    }
    const int stop = 31 - __clz(ne), slow = __ffs(ne) - 1;
    const float R0 = bin_upper(16 * stop + 15);
    // octave masses relative to R0, inclusive suffix sums from the top octave
    const double ms = ss > 0.0 ? (cnt ? ss : ss * exp2_wide((double)(bin_upper(16 * lane + 15) - R0) * L2E_D))
                               : 0.0;
    double incl = ms;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += t;
    }
    const double Z0 = __shfl_sync(0xffffffffu, incl, 0);
    const double target0 = cnt ? (double)min(topk, N) : p >= 1.0f ? 0.0 : p <= 0.0f ? 0.0 : (double)p * Z0;
    const unsigned hit = __ballot_sync(0xffffffffu, ms > 0.0 && incl >= target0);
    // boundary octave (rounding kept p Z out of reach: the lowest octave)
    const int sb = hit ? 31 - __clz(hit) : slow;
    const double above0 = __shfl_sync(0xffffffffu, incl - ms, sb);
    // second round: bins of the boundary octave and of the top octave
    const int bin = lane < 16 ? 16 * sb + lane : 16 * stop + (lane - 16);
    const double sv = __ldcg(gh + bin);
    const unsigned nt = __ballot_sync(0xffffffffu, lane >= 16 && sv > 0.0) >> 16;
    const int btop = 16 * stop + (nt ? 31 - __clz(nt) : 15);
    const float R = bin_upper(btop);
    const double sc = cnt ? 1.0 : exp2_wide((double)(R0 - R) * L2E_D);   // R0 units -> R units (>= 1)
    const double Z = Z0 * sc;
    r.Z = Z;
    r.R = R;
    if (cnt ? topk >= N : p >= 1.0f) {
        r.mode = MODE_KEEP_ALL; r.bstar = -1; r.above = 0; r.target = 0;
        return r;
    }
    const double target = cnt ? (double)topk : p <= 0.0f ? 0.0 : (double)p * Z;
    // the boundary octave's bins relative to R (lane 15 = its highest bin),
    // inclusive suffix sums on top of the octaves above
    const double mb = lane < 16 && sv > 0.0
                          ? (cnt ? sv : sv * (double)ex2_sfu((bin_upper(bin) - R) * L2E)) : 0.0;
    double incb = mb;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
        const double t = __shfl_down_sync(0xffffffffu, incb, o);
        if (lane + o < 16) incb += t;
    }
    incb += above0 * sc;
    const unsigned hb = __ballot_sync(0xffffffffu, lane < 16 && mb > 0.0 && incb >= target);
    const unsigned nb = __ballot_sync(0xffffffffu, lane < 16 && mb > 0.0);
    // b*: the highest bin whose cumulative mass reaches p Z; if rounding kept
    // it out of reach, the octave's lowest non-empty bin, kept whole
    const int L = hb ? 31 - __clz(hb) : nb ? __ffs(nb) - 1 : 0;
    r.mode = MODE_NORMAL;
    r.bstar = 16 * sb + L;
    r.above = __shfl_sync(0xffffffffu, incb - mb, L);
    r.target = hb ? target - r.above : INFINITY;
    return r;
}

// ---------------------------------------------------------------------------
// scan: level-1 histograms + tile maxima; the last CTA of a group resolves.
// grid = (ctas, B * n_ret), SCAN_THREADS threads
// ---------------------------------------------------------------------------
constexpr int SCAN_THREADS = 512;
constexpr int SCAN_WARPS = SCAN_THREADS / 32;

template <typename Src>
__global__ void __launch_bounds__(SCAN_THREADS, 2) scan_kernel(SelArgs a, SelWs w) {
    __shared__ __align__(16) float qs[GMAX * R];
    __shared__ __align__(16) uint32_t shl[2 * GMAX * NBIN];   // fixed-point bin sums: low words, then high words
    uint32_t *const shh = shl + GMAX * NBIN;
    __shared__ unsigned long long shw[GMAX * NWIDE];             // wide bins, 2^38 fixed point
    __shared__ double s_fac[NBIN];                               // octave factors
    __shared__ int s_err;
    const int b = blockIdx.y / a.n_ret;
    const int g = a.ret_g[blockIdx.y % a.n_ret];
    const int G = a.G;
    const size_t bg = (size_t)b * a.H_kv + g;
    const size_t bh0 = (size_t)b * a.H_q + (size_t)g * G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) s_err = 0;
    // this call's collect pass appends from zero
    if (blockIdx.x == 0 && threadIdx.x < G) {
        w.cand_cnt[(bh0 + threadIdx.x) * CNT_STRIDE] = 0u;
        w.list_cnt[(bh0 + threadIdx.x) * CNT_STRIDE] = 0u;
        if (a.ovf) a.ovf[bh0 + threadIdx.x] = 0u;
    }
    for (int i = threadIdx.x; i < 2 * GMAX * NBIN; i += blockDim.x) shl[i] = 0u;
    for (int i = threadIdx.x; i < GMAX * NWIDE; i += blockDim.x) shw[i] = 0ull;
    for (int i = threadIdx.x; i < NBIN; i += blockDim.x) s_fac[i] = a.topk ? 1.0 : octave_factor(i);
    // one value's mass into its head's bin counters
    auto add_value = [&](int h, float zz) -> int {
        uint32_t fx;
        const int bin = bin_and_fx(zz, fx);
        const int wsl = a.topk ? -1 : wide_slot(bin);
        if (wsl >= 0) {
            atomicAdd(&shw[h * NWIDE + wsl],
                      (unsigned long long)__float2ull_rn(ex2_sfu(fmaf(zz - bin_upper(bin), L2E, FX38_EXP2))));
            return bin;
        }
        if (a.topk) fx = (uint32_t)FX_ONE;
        uint32_t *cell = &shl[h * NBIN + bin];
        const uint32_t old = atomicAdd(cell, fx);
        if (old + fx < old) atomicAdd(cell + GMAX * NBIN, 1u);
        return bin;
    };
    if constexpr (NeedsQ<Src>::value) {
        project_query<(GMAX * R + SCAN_WARPS - 1) / SCAN_WARPS>(a.q + bh0 * D, a.Wq + (size_t)g * G * R * D,
                                                               a.idx_scale, qs, G, warp, SCAN_WARPS);
    }
    __syncthreads();
    if constexpr (NeedsQ<Src>::value) {
        if (blockIdx.x == 0)
            for (int i = threadIdx.x; i < G * R; i += blockDim.x) w.qidx[bh0 * R + i] = qs[i];
    }
    const int N = valid_len(a.seq_lens, b, a.N_max, w.status);
    Src src;
    init_src(src, a, b, g, qs);
    const int t_lo = (int)((long long)blockIdx.x * a.chunk);
    const int t_hi = (int)min((long long)N, (long long)t_lo + a.chunk);
    uint16_t *tbin = w.tilebin + bg * a.ntile * GMAX;

    int err = 0;
    typename Src::Frag cur, nxt;
    int tb = t_lo + warp * TILE;
    if (tb < t_hi) src.load(tb, cur);
    for (; tb < t_hi; tb += SCAN_WARPS * TILE) {
        const int tn = tb + SCAN_WARPS * TILE;
        if (tn < t_hi) src.load(tn, nxt);
        float z[Src::NV];
        src.eval(cur, z);
        const int nvalid = t_hi - tb;
        int tmax[Src::NSLOT];
#pragma unroll
        for (int i = 0; i < Src::NSLOT; ++i) tmax[i] = -1;
        if (nvalid >= TILE && G == GMAX) {
            // full tile, full group: no per-value validity tests
#pragma unroll
            for (int v = 0; v < Src::NV; ++v) {
                const int sl = src.slot(v);
                const float zz = z[v] + 0.0f;      // folds -0 onto +0
                err |= !(fabsf(zz) < Z_LIMIT);
                const int bin = add_value(src.head(sl), zz);
                tmax[sl] = max(tmax[sl], bin);
            }
        } else {
#pragma unroll
            for (int v = 0; v < Src::NV; ++v) {
                const int sl = src.slot(v);
                const int h = src.head(sl);
                if (h >= G || src.tok(v) >= nvalid) continue;
                const float zz = z[v] + 0.0f;
                if (!(fabsf(zz) < Z_LIMIT)) { err = 1; continue; }
                const int bin = add_value(h, zz);
                tmax[sl] = max(tmax[sl], bin);
            }
        }
#pragma unroll
        for (int i = 0; i < Src::NSLOT; ++i)
#pragma unroll
            for (int o = Src::XOR_LO; o < 32; o <<= 1) tmax[i] = max(tmax[i], __shfl_xor_sync(0xffffffffu, tmax[i], o));
        if (lane < Src::XOR_LO) {
#pragma unroll
            for (int i = 0; i < Src::NSLOT; ++i) {
                const int h = src.head(i);
                if (h < G) tbin[(size_t)(tb / TILE) * GMAX + h] = (uint16_t)(tmax[i] + 1);
            }
        }
        cur = nxt;
    }
    if (err) s_err = 1;
    __syncthreads();
    if (s_err && threadIdx.x == 0) set_status(w.status, RTP_ERR_RANGE);
    flush_hist(w.hist + bh0 * HSTRIDE, G, s_fac, blockIdx.x % NREP, [&](int i) {
        const int wsl = wide_slot(i % NBIN);
        const double m = fixed_to_double(((unsigned long long)shh[i] << 32) | shl[i], 1.0 / FX_ONE);
        return wsl < 0 ? m : m + wide_fixed_to_double(shw[(i / NBIN) * NWIDE + wsl], FX38_UNIT);
    });
}

// ---------------------------------------------------------------------------
// scan for bf16 index keys: TMA bulk-copy ring.  One producer warp streams
// the CTA's contiguous index-key range into NSTAGE shared-memory stages
// (cp.async.bulk, completion on mbarriers); TC_WARPS consumer warps take
// one 32-token tile each per stage, compute the logits on the tensor cores
// (fragments read from shared memory), and add their level-1 masses to
// 32-bit fixed-point bin counters (2^18 units per unit of mass).  Every
// SPILL_STAGES stages (<= 7680 tokens, so a counter cannot wrap) the
// counters are moved into 64-bit accumulators.  All waits are bounded.
// grid = (ctas, B * n_ret), TC_THREADS threads, TC_SMEM dynamic smem.
// ---------------------------------------------------------------------------
constexpr int TC_WARPS = 24;                             // consumer warps
constexpr int TC_THREADS = (TC_WARPS + 1) * 32;          // + one producer warp
constexpr int TPW = 2;                                   // tiles per consumer warp per stage
constexpr int ST_TOK = TC_WARPS * TPW * TILE;            // tokens per stage
constexpr int ST_BYTES = ST_TOK * R * 2;                 // bf16 index keys
constexpr int NSTAGE = 3;
constexpr int SPILL_STAGES = 10;                         // 15360 tokens
constexpr float FX18 = 262144.0f;                        // 2^18
// shared memory: the ring, the 32-bit and 64-bit bin sums, the wide bins'
// 64-bit sums, then the ring's mbarriers
constexpr int TC_OFF_H64 = NSTAGE * ST_BYTES + GMAX * NBIN * 4;
constexpr int TC_OFF_HW = TC_OFF_H64 + GMAX * NBIN * 8;
constexpr int TC_OFF_BAR = TC_OFF_HW + GMAX * NWIDE * 8;
constexpr int TC_SMEM = TC_OFF_BAR + 2 * NSTAGE * 8;
static_assert(TC_OFF_H64 % 8 == 0 && TC_OFF_HW % 8 == 0 && TC_OFF_BAR % 8 == 0, "8-byte aligned regions");
// largest single add: 2^18 e^(2^-6) < 266240 (values of the k = 0 bins may
// sit slightly above the bin's upper edge)
static_assert((long long)SPILL_STAGES * ST_TOK * 266240LL < 4294967296LL, "bin counters would wrap");

// Hot path of the scan for one value z (already folded so that -0 is +0):
// adds exp(z - U_bin) in 2^18 fixed point to the head's bin counter at
// shared address `row` (32-bit, bins of 4 bytes) and returns the raw
// (unclamped) k, whose maximum the caller checks once (k > KMAX_OK: z out
// of range or not finite).  The clamped bin index is returned in `bin`.
// CNT (static top-k): every value adds one unit, 2^18, instead of its mass.
// The fixed-point value round(v) of v in [0, 2^22) is taken with one fp32 add
// of 1.5 * 2^23 (the sum's unit in the last place is 1, so the add rounds v
// to the nearest integer, ties to even, like a conversion instruction) and
// one integer subtract of the sum's constant high bits, which keeps the
// conversion off the pipe that also serves ex2.
__device__ __forceinline__ uint32_t round_fx(float v) {
    return __float_as_uint(v + 12582912.0f) - 0x4B400000u;
}
constexpr int KMAX_OK = (int)((127 + 7) << MB) + 15 - (int)BIN_BASE;   // |z| < 256
constexpr uint32_t CNT_UNIT = 1u << 18;
template <bool CNT>
__device__ __forceinline__ int scan_value(float z, uint32_t row, int &bin) {
    const uint32_t u = __float_as_uint(z);
    const int s = (int)u >> 31;                                          // 0 or -1
    const int kr = (int)((u << 1) >> (24 - MB)) - (int)BIN_BASE;
    const int k = max(kr, 0) & 255;
    const uint32_t eb = ((uint32_t)(k + (int)BIN_BASE + 1 + s) << (23 - MB)) | (u & 0x80000000u);
    const uint32_t fx = CNT ? CNT_UNIT : round_fx(ex2_sfu(fmaf(z - __uint_as_float(eb), L2E, 18.0f)));
    bin = 256 + (k ^ s);
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(row + 4u * (uint32_t)bin), "r"(fx) : "memory");
    return kr;
}

// scan_value for a tile that holds values of |z| >= 32: the values of the
// wide bins go to their 64-bit counters at `wrow` (2^38 fixed point), the
// others as in scan_value.
__device__ __forceinline__ int scan_value_wide(float z, uint32_t row, uint32_t wrow, int &bin) {
    const uint32_t u = __float_as_uint(z);
    const int s = (int)u >> 31;                                          // 0 or -1
    const int kr = (int)((u << 1) >> (24 - MB)) - (int)BIN_BASE;
    const int k = max(kr, 0) & 255;
    const uint32_t eb = ((uint32_t)(k + (int)BIN_BASE + 1 + s) << (23 - MB)) | (u & 0x80000000u);
    const float d = z - __uint_as_float(eb);
    bin = 256 + (k ^ s);
    if (k >= K_WIDE && kr <= K_TOP) {
        const unsigned long long fx = __float2ull_rn(ex2_sfu(fmaf(d, L2E, FX38_EXP2)));
        const uint32_t slot = (uint32_t)((s ? NWK : 0) + (k - K_WIDE));
        asm volatile("red.shared.add.u64 [%0], %1;" ::"r"(wrow + 8u * slot), "l"(fx) : "memory");
    } else {
        const uint32_t fx = round_fx(ex2_sfu(fmaf(d, L2E, 18.0f)));
        asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(row + 4u * (uint32_t)bin), "r"(fx) : "memory");
    }
    return kr;
}

// The two head slots of one token at once: scan_value's bin arithmetic on
// the top 16 bits of both floats (sign, exponent and the top MB mantissa
// bits all sit there, and so does the upper edge of a bin) packed into one
// register and worked in 16-bit halves.  Per half: a = exponent and top MB
// mantissa bits of |z|; kc = a clamped to [BIN_BASE, BIN_BASE + 255]; nm =
// 0xffff where z < 0; bin = kc - BIN_BASE + 256 (z >= 0) or BIN_BASE + 255 -
// kc (z < 0), computed as (kc ^ nm) minus P_POS or P_NEG; the bin's upper
// edge has top bits (kc + 1) << 3 (z >= 0) or kc << 3 | 0x8000 (z < 0).  No
// half carries into or borrows from the other.  amax keeps the largest a of
// each slot (above A_OK: out of range or not finite), bmax the largest bin.
// Same bins and edges as scan_value for every value in range.
static_assert(MB == 4, "scan_pair's packed layout assumes 4 mantissa bits per bin");
constexpr uint32_t P_POS = (uint32_t)BIN_BASE - 256u;
constexpr uint32_t P_NEG = 65535u - ((uint32_t)BIN_BASE + 255u);
constexpr uint32_t A_OK = (uint32_t)BIN_BASE + (uint32_t)KMAX_OK;
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
template <bool CNT>
__device__ __forceinline__ void scan_pair(float z0, float z1, uint32_t row0, uint32_t row1, uint32_t &amax,
                                          uint32_t &bmax) {
    const uint32_t h = prmt(__float_as_uint(z0), __float_as_uint(z1), 0x7632u);   // [top(z1) : top(z0)]
    const uint32_t a = (h >> 3) & 0x0fff0fffu;
    amax = max_u16x2(amax, a);
    const uint32_t kc = min_u16x2(max_u16x2(a, (uint32_t)BIN_BASE * 0x10001u), ((uint32_t)BIN_BASE + 255u) * 0x10001u);
    const uint32_t nm = prmt(h, 0u, 0xbb99u);              // each half: its sign bit replicated
    // (the mask changes no bin; it keeps every address inside the head's row
    // whatever the halves hold)
    const uint32_t bin2 = ((kc ^ nm) - (P_POS * 0x10001u + (nm & ((P_NEG - P_POS) * 0x10001u)))) & 0x01ff01ffu;
    bmax = max_u16x2(bmax, bin2);
    const uint32_t hu = (kc << 3) + (nm & 0x7ff87ff8u) + 0x00080008u;
    const float U0 = __uint_as_float(hu << 16), U1 = __uint_as_float(hu & 0xffff0000u);
    const uint32_t fx0 = CNT ? CNT_UNIT : round_fx(ex2_sfu(fmaf(z0 - U0, L2E, 18.0f)));
    const uint32_t fx1 = CNT ? CNT_UNIT : round_fx(ex2_sfu(fmaf(z1 - U1, L2E, 18.0f)));
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(row0 + 4u * (bin2 & 0xffffu)), "r"(fx0) : "memory");
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(row1 + 4u * (bin2 >> 16)), "r"(fx1) : "memory");
}

// Producer of a TMA ring (lane 0 of the producer warp): streams the index
// keys of tokens [t_lo, t_hi) stage by stage into `ring` (ST_TOK tokens per
// stage).  Waits are bounded: on a timeout it records RTP_ERR_TIMEOUT and
// sets *abort.  Returns the number of stages issued; ring_drain then waits
// for the copies still in flight (none may land after the CTA exits).
template <int NS>
__device__ __forceinline__ int ring_produce(int t_lo, int t_hi, const __nv_bfloat16 *rows, uint8_t *ring,
                                            uint64_t *full, uint64_t *empty, uint32_t *status, int *abort) {
    const int n_st = t_hi > t_lo ? (t_hi - t_lo + ST_TOK - 1) / ST_TOK : 0;
    int issued = 0;
    for (int it = 0; it < n_st; ++it) {
        const int st = it % NS;
        if (it >= NS && !mbar_wait(&empty[st], (uint32_t)((it / NS - 1) & 1))) {
            set_status(status, RTP_ERR_TIMEOUT);
            *abort = 1;
            break;
        }
        if (*(volatile int *)abort) break;
        fence_proxy_async();
        const int tok0 = t_lo + it * ST_TOK;
        const uint32_t bytes = (uint32_t)min(ST_TOK, t_hi - tok0) * (uint32_t)(R * 2);
        mbar_expect_tx(&full[st], bytes);
        bulk_g2s(ring + st * ST_BYTES, rows + (size_t)tok0 * R, bytes, &full[st]);
        issued = it + 1;
    }
    return issued;
}
template <int NS>
__device__ __forceinline__ void ring_drain(uint64_t *full, int issued) {
    for (int it = max(0, issued - NS); it < issued; ++it)
        mbar_wait(&full[it % NS], (uint32_t)((it / NS) & 1));
}

template <bool CNT>
__global__ void __launch_bounds__(TC_THREADS, 1) scan_tma_kernel(SelArgs a, SelWs w) {
    extern __shared__ __align__(128) uint8_t dsm[];
    uint8_t *ring = dsm;
    uint32_t *h32 = reinterpret_cast<uint32_t *>(dsm + NSTAGE * ST_BYTES);
    unsigned long long *h64 = reinterpret_cast<unsigned long long *>(dsm + TC_OFF_H64);
    unsigned long long *hw = reinterpret_cast<unsigned long long *>(dsm + TC_OFF_HW);
    uint64_t *full = reinterpret_cast<uint64_t *>(dsm + TC_OFF_BAR);
    uint64_t *empty = full + NSTAGE;
    __shared__ __align__(16) float qs[GMAX * R];
    __shared__ double s_fac[NBIN];              // octave factors (the producer warp's idle lanes)
    __shared__ int s_err, s_abort;
    const int b = blockIdx.y / a.n_ret;
    const int g = a.ret_g[blockIdx.y % a.n_ret];
    const int G = a.G;
    const size_t bg = (size_t)b * a.H_kv + g;
    const size_t bh0 = (size_t)b * a.H_q + (size_t)g * G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        s_err = 0;
        s_abort = 0;
        for (int i = 0; i < NSTAGE; ++i) { mbar_init(&full[i], 1u); mbar_init(&empty[i], (uint32_t)TC_WARPS); }
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < GMAX * NBIN; i += blockDim.x) { h32[i] = 0u; h64[i] = 0ull; }
    for (int i = threadIdx.x; i < GMAX * NWIDE; i += blockDim.x) hw[i] = 0ull;
    pdl_wait();
    pdl_trigger();
    // the consumers' q_idx loads go out before the producer's first bulk copy
    QProj<(GMAX * R + TC_WARPS - 1) / TC_WARPS> qp;
    if (warp < TC_WARPS) qp.load(a.q + bh0 * D, a.Wq + (size_t)g * G * R * D, G, warp, TC_WARPS);
    __syncthreads();
    const int N = valid_len(a.seq_lens, b, a.N_max, w.status);
    const int t_lo = (int)((long long)blockIdx.x * a.chunk);
    const int t_hi = (int)min((long long)N, (long long)t_lo + a.chunk);
    const int n_st = t_hi > t_lo ? (t_hi - t_lo + ST_TOK - 1) / ST_TOK : 0;
    const __nv_bfloat16 *rows = reinterpret_cast<const __nv_bfloat16 *>(a.kidx) + bg * a.N_max * R;

    if (warp == TC_WARPS) {
        // lane 0 streams; once it has issued the last stage the other lanes
        // fill the octave factor table (needed only by the flush) while lane
        // 0 waits for its copies in flight
        int issued = 0;
        if (lane == 0) issued = ring_produce<NSTAGE>(t_lo, t_hi, rows, ring, full, empty, w.status, &s_abort);
        __syncwarp();
        if (lane == 0)
            ring_drain<NSTAGE>(full, issued);
        else
            for (int i = lane - 1; i < NBIN; i += 31) s_fac[i] = CNT ? 1.0 : octave_factor(i);
    } else {
        // consumers: finish q_idx of the group (the producer is already streaming)
        qp.store(a.idx_scale, qs, G, warp, TC_WARPS);
        asm volatile("bar.sync 1, %0;" ::"r"(TC_WARPS * 32) : "memory");
        // q_idx for the collect pass, and its counters from zero (these
        // stores come after the barriers of the prologue, which would wait
        // for them)
        if (blockIdx.x == 0) {
            if (blockIdx.y == 0 && threadIdx.x == 0 && a.spill_any) *a.spill_any = 0u;
            for (int i = threadIdx.x; i < G * R; i += TC_WARPS * 32) w.qidx[bh0 * R + i] = qs[i];
            if (threadIdx.x < G) {
                w.cand_cnt[(bh0 + threadIdx.x) * CNT_STRIDE] = 0u;
                w.list_cnt[(bh0 + threadIdx.x) * CNT_STRIDE] = 0u;
                if (a.ovf) a.ovf[bh0 + threadIdx.x] = 0u;
            }
        }
        SrcMma src;
        src.init(rows, a.N_max, qs, G);
        const int gid = lane >> 2, tig = lane & 3;
        const uint32_t hrow0 = smem_u32(h32 + (2 * tig) * NBIN), hrow1 = smem_u32(h32 + (2 * tig + 1) * NBIN);
        const uint32_t hwrow0 = smem_u32(hw + (2 * tig) * NWIDE), hwrow1 = smem_u32(hw + (2 * tig + 1) * NWIDE);
        const bool full_group = G == GMAX;
        int kmax = 0;
        uint32_t amax = 0u;                // packed largest exponent bits per slot (scan_pair)
        uint32_t *tbin = reinterpret_cast<uint32_t *>(w.tilebin + bg * a.ntile * GMAX);

        // One 32-token tile: logits on the tensor cores, level-1 masses into
        // the bin counters, the tile's largest bin per head into its record.
        auto scan_tile = [&](const uint8_t *tile, int tb, int nvalid) {
            SrcMma::Frag f;
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int r = 0; r < 2; ++r)
                    f.a[i][r] = *reinterpret_cast<const uint2 *>(tile + (16 * i + gid + 8 * r) * (R * 2) + 8 * tig);
            float z[SrcMma::NV];
            src.eval(f, z);
            // the lane's largest bin per head slot, both slots in one word:
            // (1 + max bin) per 16-bit half (0: no value)
            uint32_t pk;
            // a tile with a value of |z| >= 32 (or not finite) anywhere in
            // the warp takes the per-value path with the wide bins' counters
            bool wide = false;
            if constexpr (!CNT) {
                float zm = 0.0f;
#pragma unroll
                for (int v = 0; v < SrcMma::NV; ++v) zm = fmaxf(zm, fabsf(z[v]));
                wide = __any_sync(0xffffffffu, !(zm < WIDE_Z));
            }
            if (wide) {
                int tmax[2] = {-1, -1};
#pragma unroll
                for (int v = 0; v < SrcMma::NV; ++v) {
                    const int sl = v & 1;
                    if (2 * tig + sl >= G || src.tok(v) >= nvalid) continue;
                    int bin;
                    kmax = max(kmax, scan_value_wide(z[v] + 0.0f, sl ? hrow1 : hrow0, sl ? hwrow1 : hwrow0, bin));
                    tmax[sl] = max(tmax[sl], bin);
                }
                pk = (uint32_t)(tmax[0] + 1) | ((uint32_t)(tmax[1] + 1) << 16);
            } else if (nvalid >= TILE && full_group) {
                // value v is slot v & 1 of its token: pairs (v, v + 1)
                uint32_t bmax = 0u;
#pragma unroll
                for (int v = 0; v < SrcMma::NV; v += 2)
                    scan_pair<CNT>(z[v] + 0.0f, z[v + 1] + 0.0f, hrow0, hrow1, amax, bmax);
                pk = bmax + 0x00010001u;
            } else {
                int tmax[2] = {-1, -1};
#pragma unroll
                for (int v = 0; v < SrcMma::NV; ++v) {
                    const int sl = v & 1;
                    if (2 * tig + sl >= G || src.tok(v) >= nvalid) continue;
                    int bin;
                    kmax = max(kmax, scan_value<CNT>(z[v] + 0.0f, sl ? hrow1 : hrow0, bin));
                    tmax[sl] = max(tmax[sl], bin);
                }
                pk = (uint32_t)(tmax[0] + 1) | ((uint32_t)(tmax[1] + 1) << 16);
            }
            // max over the warp's lanes of the same slots
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                const uint32_t other = __shfl_xor_sync(0xffffffffu, pk, o);
                asm("max.u16x2 %0, %0, %1;" : "+r"(pk) : "r"(other));
            }
            // lane l < 4 writes heads 2l, 2l + 1 of the tile's record
            if (lane < 4) tbin[(size_t)(tb / TILE) * (GMAX / 2) + lane] = pk;
        };
        // After a timeout every consumer warp keeps iterating without
        // waiting or working, so the named barrier below stays balanced.
        bool dead = false;
        int st = 0, phase = 0, spill_in = SPILL_STAGES;
        for (int it = 0; it < n_st; ++it) {
            // one decision for the warp, so scan_tile (tensor cores, full-warp
            // shuffles) runs with all 32 lanes or none; every lane waits on
            // the barrier itself (its own acquire of the stage)
            int live = dead ? 0 : (*(volatile int *)&s_abort == 0);
            live = __shfl_sync(0xffffffffu, live, 0);
            if (live && !mbar_wait(&full[st], (uint32_t)phase)) {
                set_status(w.status, RTP_ERR_TIMEOUT);
                s_abort = 1;
                live = 0;
            }
            dead = !__all_sync(0xffffffffu, live);
            if (!dead) {
                const int tb0 = t_lo + it * ST_TOK + warp * TILE;
                const uint8_t *tiles = ring + st * ST_BYTES + warp * (TILE * R * 2);
#pragma unroll
                for (int tt = 0; tt < TPW; ++tt) {
                    const int tb = tb0 + tt * TC_WARPS * TILE;
                    if (t_hi - tb > 0) scan_tile(tiles + tt * (TC_WARPS * TILE * R * 2), tb, t_hi - tb);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
            if (++st == NSTAGE) { st = 0; phase ^= 1; }
            if (--spill_in == 0 && it + 1 < n_st) {
                spill_in = SPILL_STAGES;
                asm volatile("bar.sync 1, %0;" ::"r"(TC_WARPS * 32) : "memory");
                for (int i = threadIdx.x; i < GMAX * NBIN; i += TC_WARPS * 32) {
                    h64[i] += h32[i];
                    h32[i] = 0u;
                }
                asm volatile("bar.sync 1, %0;" ::"r"(TC_WARPS * 32) : "memory");
            }
        }
        if (kmax > KMAX_OK || max(amax & 0xffffu, amax >> 16) > A_OK) s_err = 1;
    }
    __syncthreads();
    if (s_err && threadIdx.x == 0) set_status(w.status, RTP_ERR_RANGE);
    flush_hist(w.hist + bh0 * HSTRIDE, G, s_fac, blockIdx.x % NREP,
               [&](int i) {
                   const int wsl = wide_slot(i % NBIN);
                   const double m = fixed_to_double(h64[i] + h32[i], 1.0 / FX18);
                   return wsl < 0 ? m : m + wide_fixed_to_double(hw[(i / NBIN) * NWIDE + wsl], FX38_UNIT);
               });
}

// ---------------------------------------------------------------------------
// collect: kept ids above b*, candidates in b*.  grid as scan.
// ---------------------------------------------------------------------------
constexpr int COL_THREADS = 512;
constexpr int COL_WARPS = COL_THREADS / 32;

constexpr int KCAP = 256;     // kept ids staged per head per CTA
constexpr int CCAP = 128;     // candidates staged per head per CTA

template <typename Src>
__global__ void __launch_bounds__(COL_THREADS, 2) collect_kernel(SelArgs a, SelWs w) {
    __shared__ __align__(16) float qs[GMAX * R];
    __shared__ int s_bstar[GMAX];
    __shared__ int s_mode[GMAX];
    __shared__ unsigned s_kc[GMAX], s_cc[GMAX];
    __shared__ float s_khi[GMAX], s_clo[GMAX];      // keep: z > s_khi; candidate: s_clo <= z <= s_khi
    __shared__ int32_t s_kbuf[GMAX * KCAP];
    __shared__ unsigned long long s_cbuf[GMAX * CCAP];
    const int b = blockIdx.y / a.n_ret;
    const int g = a.ret_g[blockIdx.y % a.n_ret];
    const int G = a.G;
    const size_t bh0 = (size_t)b * a.H_q + (size_t)g * G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_trigger();
    // Every CTA resolves the group's heads from the finished histograms
    // (warp h: head h); the group's first CTA records them for finalize.
    const int N = valid_len(a.seq_lens, b, a.N_max, w.status);
    if (warp < GMAX) {
        int mode = MODE_EMPTY, bs = NBIN;
        if (warp < G) {
            const Resolve r = resolve_head(w.hist + (bh0 + warp) * HSTRIDE, a.p, N, a.topk);
            if (blockIdx.x == 0 && lane == 0) w.res[bh0 + warp] = r;
            mode = r.mode;
            bs = r.bstar;
        }
        if (lane == 0) {
            s_mode[warp] = mode;
            // keep-all heads need no collect pass: finalize lists every token
            s_bstar[warp] = mode == MODE_NORMAL ? bs : NBIN;
            s_khi[warp] = mode == MODE_NORMAL ? bin_hi_incl(bs) : INFINITY;
            s_clo[warp] = mode == MODE_NORMAL ? bin_lo_incl(bs) : INFINITY;
            s_kc[warp] = 0u;
            s_cc[warp] = 0u;
        }
    }
    if constexpr (NeedsQ<Src>::value)
        for (int i = threadIdx.x; i < G * R; i += blockDim.x) qs[i] = w.qidx[bh0 * R + i];
    __syncthreads();
    Src src;
    init_src(src, a, b, g, qs);
    const int t_lo = (int)((long long)blockIdx.x * a.chunk);
    const int t_hi = (int)min((long long)N, (long long)t_lo + a.chunk);
    const uint16_t *tbin = w.tilebin + ((size_t)b * a.H_kv + g) * a.ntile * GMAX;
    int bst[GMAX];
#pragma unroll
    for (int h = 0; h < GMAX; ++h) bst[h] = s_bstar[h];

    // Warp w owns tiles w, w + COL_WARPS, ...; windows of 32 of them are
    // screened at once (lane i: the i-th tile of the window, all heads),
    // then the needed ones are processed with the next one's load in flight.
    for (int wbase = 0;; wbase += 32) {
        const int tb_l = t_lo + (warp + (wbase + lane) * COL_WARPS) * TILE;
        unsigned hm = 0u;                        // heads that need lane's tile
        if (tb_l < t_hi) {
            const int ti = tb_l / TILE;
#pragma unroll
            for (int h = 0; h < GMAX; ++h)
                if (h < G && (int)tbin[(size_t)ti * GMAX + h] - 1 >= bst[h]) hm |= 1u << h;
        }
        const unsigned any_valid = __ballot_sync(0xffffffffu, tb_l < t_hi);
        if (!any_valid) break;
        unsigned todo = __ballot_sync(0xffffffffu, hm != 0u);
        if (!todo) continue;
        int i = __ffs(todo) - 1;
        typename Src::Frag cur, nxt;
        src.load(__shfl_sync(0xffffffffu, tb_l, i), cur);
        while (true) {
            const int tb = __shfl_sync(0xffffffffu, tb_l, i);
            const unsigned hmask = __shfl_sync(0xffffffffu, hm, i);
            todo &= todo - 1u;
            const int inext = todo ? __ffs(todo) - 1 : -1;
            if (inext >= 0) src.load(__shfl_sync(0xffffffffu, tb_l, inext), nxt);
            float z[Src::NV];
            src.eval(cur, z);
#pragma unroll
            for (int v = 0; v < Src::NV; ++v) {
                const int h = src.head(src.slot(v));
                const int t = tb + src.tok(v);
                if (h < G && t < t_hi && ((hmask >> h) & 1u)) {
                    const float zz = z[v] + 0.0f;
                    if (fabsf(zz) < Z_LIMIT) {
                        const float khi = s_khi[h];
                        if (zz > khi) {
                            const unsigned p = atomicAdd(&s_kc[h], 1u);
                            if (p < (unsigned)KCAP) {
                                s_kbuf[h * KCAP + p] = t;
                            } else {
                                const unsigned q = atomicAdd(&w.list_cnt[(bh0 + h) * CNT_STRIDE], 1u);
                                a.lists[(bh0 + h) * a.N_max + q] = t;
                            }
                        } else if (zz >= s_clo[h]) {
                            const unsigned long long key =
                                ((unsigned long long)logit_key(zz) << 32) |
                                (unsigned long long)(0xffffffffu - (uint32_t)t);
                            const unsigned p = atomicAdd(&s_cc[h], 1u);
                            if (p < (unsigned)CCAP) {
                                s_cbuf[h * CCAP + p] = key;
                            } else {
                                const unsigned q = atomicAdd(&w.cand_cnt[(bh0 + h) * CNT_STRIDE], 1u);
                                w.cands[(bh0 + h) * a.N_max + q] = key;
                            }
                        }
                    }
                }
            }
            if (inext < 0) break;
            i = inext;
            cur = nxt;
        }
    }
    // flush the staged ids: one global reservation per head and kind
    __syncthreads();
    if (warp < G) {
        const size_t bh = bh0 + warp;
        const unsigned nk = min(s_kc[warp], (unsigned)KCAP);
        const unsigned ncd = min(s_cc[warp], (unsigned)CCAP);
        unsigned kb = 0u, cb = 0u;
        if (lane == 0) {
            if (nk) kb = atomicAdd(&w.list_cnt[bh * CNT_STRIDE], nk);
            if (ncd) cb = atomicAdd(&w.cand_cnt[bh * CNT_STRIDE], ncd);
        }
        kb = __shfl_sync(0xffffffffu, kb, 0);
        cb = __shfl_sync(0xffffffffu, cb, 0);
        for (unsigned j = lane; j < nk; j += 32) a.lists[bh * a.N_max + kb + j] = s_kbuf[warp * KCAP + j];
        for (unsigned j = lane; j < ncd; j += 32) w.cands[bh * a.N_max + cb + j] = s_cbuf[warp * CCAP + j];
    }
}

// ---------------------------------------------------------------------------
// collect for bf16 index keys.  The retrieval groups are taken in pairs
// (groups 2p and 2p + 1 in (b, g) order; with an odd count the last pair has
// one): the CTAs of a pair share its tiles, so a group with many needed
// tiles borrows its partner's CTAs.  Every CTA first resolves the pair's
// heads from the finished histograms (warp w: pair-head w = head w mod GMAX
// of the pair's group w / GMAX; the pair's first CTA records them for
// finalize) while loading q_idx and the tile records of its first window.
// The pair's tiles (its first group's, then its second's) are dealt to its
// CTAs round-robin; warp w of a CTA takes its tiles w, w + CL_WARPS, ...,
// screened 32 at a time by their records (a tile is needed when some head's
// largest bin in it reaches b*).  The needed ones are loaded CL_BATCH at a
// time, all loads in flight, and their logits recomputed with the scan's
// tensor-core arithmetic; one compare per value finds those at or above the
// floor of the head's boundary bin, and only these are sorted into kept ids
// (z above b*) and b*'s candidates, staged per pair-head.
// grid = (cl_ctas, pairs), CL_THREADS threads.
// ---------------------------------------------------------------------------
constexpr int CL_WARPS = 16;
constexpr int CL_THREADS = CL_WARPS * 32;
constexpr int CL_BATCH = 4;
constexpr int PAIR = 2;                    // retrieval groups per collect CTA
constexpr int HP = PAIR * GMAX;            // pair-heads: group-in-pair * GMAX + head
constexpr int CL_KCAP = 512;               // kept ids staged per pair-head per CTA
constexpr int CL_SLOTS = 32;               // attention partial slots (one round of heads)
static_assert(CL_WARPS == HP, "one resolving and one flushing warp per pair-head");
static_assert(HP * D % CL_THREADS == 0 && HP * R <= CL_THREADS, "collect prologue load split");
static_assert(CL_SLOTS >= CL_WARPS, "a round holds every warp's partial of any one head");
// dynamic shared memory: staged kept ids and candidates, the scaled q_rope of
// the pair's heads, and the attention partial slots
constexpr int CL_SMEM = HP * CL_KCAP * 4 + HP * CCAP * 8 + HP * D * 4 + CL_SLOTS * PSTRIDE * 4;

template <bool PAGED>
__global__ void __launch_bounds__(CL_THREADS, 1) collect_mma_kernel(SelArgs a, SelWs w) {
    extern __shared__ __align__(16) uint8_t csm[];
    int32_t *s_kbuf = reinterpret_cast<int32_t *>(csm);                                          // [HP][CL_KCAP]
    unsigned long long *s_cbuf = reinterpret_cast<unsigned long long *>(csm + HP * CL_KCAP * 4);  // [HP][CCAP]
    float *s_qr = reinterpret_cast<float *>(csm + HP * CL_KCAP * 4 + HP * CCAP * 8);              // [HP][D]
    float *s_slot = s_qr + HP * D;                                                        // [CL_SLOTS][PSTRIDE]
    __shared__ __align__(16) float qs[PAIR][GMAX * R];
    __shared__ int s_bstar[HP];
    __shared__ unsigned s_kc[HP], s_cc[HP];
    __shared__ float s_khi[HP], s_clo[HP];      // keep: z > s_khi; candidate: s_clo <= z <= s_khi
    __shared__ Resolve s_res[HP];               // the pair's first CTA records them at the end
    const int G = a.G;
    const int groups = a.B * a.n_ret;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = gridDim.x, cx = blockIdx.x;
    // the pair's groups: group y = b * n_ret + i is (b, ret_g[i])
    const int y0 = PAIR * blockIdx.y, y1 = y0 + 1;
    const bool has1 = y1 < groups;
    const int b0 = y0 / a.n_ret, b1 = has1 ? y1 / a.n_ret : b0;
    const int g0 = a.ret_g[y0 % a.n_ret], g1 = has1 ? a.ret_g[y1 % a.n_ret] : g0;
    const size_t bg0 = (size_t)b0 * a.H_kv + g0, bg1 = (size_t)b1 * a.H_kv + g1;
    // global position of this shard's token 0 in each group's sequence
    const int off0 = a.id_off ? a.id_off[b0] : 0, off1 = a.id_off ? a.id_off[b1] : 0;
    const size_t bh00 = (size_t)b0 * a.H_q + (size_t)g0 * G, bh01 = (size_t)b1 * a.H_q + (size_t)g1 * G;
    // pair-head ph is valid when its group exists and its head is < G
    auto ph_ok = [&](int ph) { return (ph < GMAX || has1) && ph % GMAX < G; };
    auto ph_bh = [&](int ph) { return (ph < GMAX ? bh00 : bh01) + ph % GMAX; };
    if (threadIdx.x < HP) { s_kc[threadIdx.x] = 0u; s_cc[threadIdx.x] = 0u; }
    // inputs of the call (no earlier kernel writes them) load before the wait
    const int n0 = a.seq_lens[b0], n1 = has1 ? a.seq_lens[b1] : 0;
    constexpr int QR_PER = HP * D / CL_THREADS;
    float qrv[QR_PER];
#pragma unroll
    for (int k = 0; k < QR_PER; ++k) {
        const int i = threadIdx.x + k * CL_THREADS, ph = i / D;
        qrv[k] = a.q_rope && ph_ok(ph) ? a.q_rope[ph_bh(ph) * D + i % D] : 0.0f;
    }
    pdl_wait();
    pdl_trigger();
    const int N0 = checked_len(n0, a.N_max, w.status);
    const int N1 = has1 ? checked_len(n1, a.N_max, w.status) : 0;
    const int nt0 = (N0 + TILE - 1) / TILE;
    const int ntot = nt0 + (N1 + TILE - 1) / TILE;
    const uint4 *recs0 = reinterpret_cast<const uint4 *>(w.tilebin + bg0 * a.ntile * GMAX);
    const uint4 *recs1 = reinterpret_cast<const uint4 *>(w.tilebin + bg1 * a.ntile * GMAX);
    // The pair's tile T (< ntot) is tile T of its first group, or T - nt0 of
    // its second; tile T goes to CTA T mod C.  Tile of lane `lane` in window
    // `win` of this warp:
    auto tile_of = [&](int win) { return cx + C * (warp + (win * 32 + lane) * CL_WARPS); };
    uint4 rec = make_uint4(0u, 0u, 0u, 0u);
    {
        const int T = tile_of(0);
        if (T < ntot) rec = __ldcg(T < nt0 ? recs0 + T : recs1 + (T - nt0));
    }
    // q_idx of the pair's heads (the scan wrote it): loaded now, stored to
    // shared memory after the resolve, with the scaled q_rope
    float qv = 0.0f;
    {
        const int i = threadIdx.x, ph = i / R;
        if (i < HP * R && ph_ok(ph)) qv = w.qidx[ph_bh(ph) * R + i % R];
    }
    {
        int bs = NBIN, mode = MODE_EMPTY;
        if (ph_ok(warp)) {
            const size_t bh = ph_bh(warp);
            const Resolve r = resolve_head(w.hist + bh * HSTRIDE, a.p, warp < GMAX ? N0 : N1, a.topk);
            if (cx == 0 && lane == 0) s_res[warp] = r;
            mode = r.mode;
            bs = r.bstar;
        }
        if (lane == 0) {
            // keep-all heads need no collect pass: finalize lists every token
            s_bstar[warp] = mode == MODE_NORMAL ? bs : NBIN;
            s_khi[warp] = mode == MODE_NORMAL ? bin_hi_incl(bs) : INFINITY;
            s_clo[warp] = mode == MODE_NORMAL ? bin_lo_incl(bs) : INFINITY;
        }
    }
    if (threadIdx.x < HP * R) (&qs[0][0])[threadIdx.x] = qv;
#pragma unroll
    for (int k = 0; k < QR_PER; ++k) s_qr[threadIdx.x + k * CL_THREADS] = qrv[k] * a.attn_scale_log2;
    __syncthreads();
    const size_t cta = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
    if (cx >= ntot) {
        // no tile for this CTA: empty partials for the fused attention
        if (cx == 0 && lane == 0 && ph_ok(warp)) w.res[ph_bh(warp)] = s_res[warp];
        if (a.q_rope)
            for (int i = threadIdx.x; i < HP * PSTRIDE; i += blockDim.x)
                a.part_sel[cta * HP * PSTRIDE + i] = i % PSTRIDE == 0 ? -INFINITY : 0.0f;
        return;
    }
    const __nv_bfloat16 *rows0 = reinterpret_cast<const __nv_bfloat16 *>(a.kidx) + bg0 * a.N_max * R;
    const __nv_bfloat16 *rows1 = reinterpret_cast<const __nv_bfloat16 *>(a.kidx) + bg1 * a.N_max * R;
    SrcMma src0, src1;
    src0.init(rows0, a.N_max, qs[0], G);
    src1.init(rows1, a.N_max, qs[1], G);
    const int tig = lane & 3;
    // thresholds of the lane's two head slots (heads 2 tig, 2 tig + 1) in
    // either group: kept z > khi, candidate clo <= z <= khi
    const float khi00 = s_khi[2 * tig], khi01 = s_khi[2 * tig + 1];
    const float khi10 = s_khi[GMAX + 2 * tig], khi11 = s_khi[GMAX + 2 * tig + 1];
    const float clo00 = s_clo[2 * tig], clo01 = s_clo[2 * tig + 1];
    const float clo10 = s_clo[GMAX + 2 * tig], clo11 = s_clo[GMAX + 2 * tig + 1];

    for (int win = 0; cx + C * (warp + win * 32 * CL_WARPS) < ntot; ++win) {
        const int T = tile_of(win);
        const int tg = T < nt0 ? 0 : 1;                     // the lane's tile: group in pair, tile index
        const int ti = T - (tg ? nt0 : 0);
        if (win > 0) rec = T < ntot ? __ldcg(tg ? recs1 + ti : recs0 + ti) : make_uint4(0u, 0u, 0u, 0u);
        // heads whose largest bin in the lane's tile reaches their b*
        const uint32_t rw[4] = {rec.x, rec.y, rec.z, rec.w};
        unsigned hm = 0u;
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            const int tbmax = (int)((rw[h >> 1] >> (16 * (h & 1))) & 0xffffu) - 1;
            if (tbmax >= s_bstar[tg * GMAX + h]) hm |= 1u << h;
        }
        if (T >= ntot) hm = 0u;
        unsigned todo = __ballot_sync(0xffffffffu, hm != 0u);
        while (todo) {
            // up to CL_BATCH needed tiles, all loads in flight
            int sel[CL_BATCH];
            SrcMma::Frag f[CL_BATCH];
#pragma unroll
            for (int k = 0; k < CL_BATCH; ++k) {
                sel[k] = todo ? __ffs(todo) - 1 : -1;
                if (todo) todo &= todo - 1u;
                if (sel[k] >= 0) {
                    const int gk = __shfl_sync(0xffffffffu, tg, sel[k]);
                    const int tb = __shfl_sync(0xffffffffu, ti, sel[k]) * TILE;
                    if (gk) src1.load(tb, f[k]); else src0.load(tb, f[k]);
                }
            }
#pragma unroll
            for (int k = 0; k < CL_BATCH; ++k) {
                if (sel[k] < 0) break;
                const int gk = __shfl_sync(0xffffffffu, tg, sel[k]);
                const int tb = __shfl_sync(0xffffffffu, ti, sel[k]) * TILE;
                const unsigned hmask = __shfl_sync(0xffffffffu, hm, sel[k]);
                float z[SrcMma::NV];
                if (gk) src1.eval(f[k], z); else src0.eval(f[k], z);
                // fast pass: bit v marks a value at or above the floor of its
                // head's boundary bin (heads whose tile maximum reaches b*)
                const float cl0 = (hmask >> (2 * tig)) & 1u ? (gk ? clo10 : clo00) : INFINITY;
                const float cl1 = (hmask >> (2 * tig + 1)) & 1u ? (gk ? clo11 : clo01) : INFINITY;
                unsigned mk = 0u;
#pragma unroll
                for (int v = 0; v < SrcMma::NV; ++v) mk |= (unsigned)(z[v] >= ((v & 1) ? cl1 : cl0)) << v;
                const int Ng = gk ? N1 : N0;
                if (Ng - tb < TILE) {
#pragma unroll
                    for (int v = 0; v < SrcMma::NV; ++v)
                        if (tb + src0.tok(v) >= Ng) mk &= ~(1u << v);
                }
                // rare pass: kept (above the bin) or candidate (in it), staged
                const float kh0 = gk ? khi10 : khi00, kh1 = gk ? khi11 : khi01;
                while (mk) {
                    const int v = __ffs(mk) - 1;
                    mk &= mk - 1u;
                    float zv = 0.0f;                      // z[v] without dynamic register indexing
#pragma unroll
                    for (int u = 0; u < SrcMma::NV; ++u) zv = u == v ? z[u] : zv;
                    const int h = src0.head(src0.slot(v));
                    const int ph = gk * GMAX + h;
                    const size_t bh = (gk ? bh01 : bh00) + h;
                    const int t = tb + src0.tok(v);
                    if (zv > ((v & 1) ? kh1 : kh0)) {
                        const unsigned p = atomicAdd(&s_kc[ph], 1u);
                        if (p < (unsigned)CL_KCAP) {
                            s_kbuf[ph * CL_KCAP + p] = t;
                        } else {
                            const unsigned q = atomicAdd(&w.list_cnt[bh * CNT_STRIDE], 1u);
                            a.lists[bh * a.N_max + q] = t + (gk ? off1 : off0);
                        }
                    } else {
                        const unsigned long long key =
                            ((unsigned long long)logit_key(zv + 0.0f) << 32) |
                            (unsigned long long)(0xffffffffu - (uint32_t)(t + (gk ? off1 : off0)));
                        const unsigned p = atomicAdd(&s_cc[ph], 1u);
                        if (p < (unsigned)CCAP) {
                            s_cbuf[ph * CCAP + p] = key;
                        } else {
                            const unsigned q = atomicAdd(&w.cand_cnt[bh * CNT_STRIDE], 1u);
                            w.cands[bh * a.N_max + q] = key;
                        }
                        // finalize attends the candidates it keeps: their rows
                        // start toward L2 now (there are few of them)
                        if (a.q_rope) {
                            if constexpr (PAGED) {
                                const long long row = kv_row(a.kv, gk ? b1 : b0, gk ? g1 : g0, t);
                                if (row >= 0) prefetch_kv_l2(a.k_cache + row * D, a.v_cache + row * D);
                            } else {
                                const size_t row = ((gk ? bg1 : bg0) * a.N_max + t) * D;
                                prefetch_kv_l2(a.k_cache + row, a.v_cache + row);
                            }
                        }
                    }
                }
            }
        }
    }
    // the staged ids go out with one global reservation per pair-head and
    // kind (warp w: pair-head w); the reservations are taken here and used
    // after the fused attention, which hides their round trip
    __syncthreads();
    const bool wok = ph_ok(warp);
    const size_t wbh = ph_bh(warp);
    unsigned kb = 0u, cb = 0u;
    const unsigned nk = wok ? min(s_kc[warp], (unsigned)CL_KCAP) : 0u;
    const unsigned ncd = wok ? min(s_cc[warp], (unsigned)CCAP) : 0u;
    if (lane == 0) {
        if (nk) kb = atomicAdd(&w.list_cnt[wbh * CNT_STRIDE], nk);
        if (ncd) cb = atomicAdd(&w.cand_cnt[wbh * CNT_STRIDE], ncd);
    }
    auto flush_ids = [&]() {
        // (a global store before a block barrier would make the barrier wait
        // for it, so the resolve records go out here, at the end)
        if (cx == 0 && lane == 0 && wok) w.res[wbh] = s_res[warp];
        kb = __shfl_sync(0xffffffffu, kb, 0);
        cb = __shfl_sync(0xffffffffu, cb, 0);
        const int offw = warp < GMAX ? off0 : off1;
        for (unsigned j = lane; j < nk; j += 32) a.lists[wbh * a.N_max + kb + j] = s_kbuf[warp * CL_KCAP + j] + offw;
        for (unsigned j = lane; j < ncd; j += 32) w.cands[wbh * a.N_max + cb + j] = s_cbuf[warp * CCAP + j];
    };
    if (!a.q_rope) {
        flush_ids();
        return;
    }

    // Fused attention over the rows staged here, in rounds of pair-heads
    // whose partial slots fit CL_SLOTS.  A round's rows form chunks of 8 of
    // one head (heads in order), dealt round-robin to the warps; a warp
    // keeps one running partial and files it when its head changes, in the
    // slot of the head numbered by the warp's first chunk in the head (the
    // first CL_WARPS chunks of a head belong to distinct warps, so a head
    // with c chunks fills min(c, CL_WARPS) slots, each once).  Every warp
    // derives the round layout itself (lane h: pair-head h), so no block
    // barrier -- which would wait for the reservations above -- precedes the
    // attention.  A head whose staging overflowed is left to finalize (ovf
    // flag, empty partial).
    if (lane == 0 && wok && s_kc[warp] > (unsigned)CL_KCAP) a.ovf[wbh] = 1u;

    const int nrow_l = lane < HP && ph_ok(lane) && s_kc[lane] <= (unsigned)CL_KCAP ? (int)s_kc[lane] : 0;
    for (int h_lo = 0; h_lo < HP;) {
        // lane h in [h_lo, HP): its chunks and slots, inclusive prefix sums
        const int c = lane >= h_lo ? (nrow_l + 7) / 8 : 0;
        const int sl = min(c, CL_WARPS);
        int cs = c, ss = sl;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int tc = __shfl_up_sync(0xffffffffu, cs, o), ts = __shfl_up_sync(0xffffffffu, ss, o);
            if (lane >= o) { cs += tc; ss += ts; }
        }
        // the round: heads h_lo .. h_hi - 1, as many as fit (at least one)
        const unsigned fit = __ballot_sync(0xffffffffu, lane >= h_lo && lane < HP && ss <= CL_SLOTS);
        const int h_hi = 32 - __clz(fit);
        const int nchunk = __shfl_sync(0xffffffffu, cs, h_hi - 1);
        const int c0_l = cs - c, s0_l = ss - sl;          // lane's first chunk and slot
        WarpPart part;
        part.reset();
        int cur = -1, kfirst = 0, cur_c0 = 0, cur_s0 = 0;
        float qx[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k = warp; k < nchunk; k += CL_WARPS) {
            // the chunk's head: the last non-empty head of the round starting at or before k
            const unsigned st = __ballot_sync(0xffffffffu, lane >= h_lo && lane < h_hi && c > 0 && c0_l <= k);
            const int ph = 31 - __clz(st);
            const int c0 = __shfl_sync(0xffffffffu, c0_l, ph), s0 = __shfl_sync(0xffffffffu, s0_l, ph);
            if (ph != cur) {
                if (cur >= 0) part.store(s_slot + (cur_s0 + kfirst - cur_c0) * PSTRIDE);
                part.reset();
                cur = ph;
                kfirst = k;
                cur_c0 = c0;
                cur_s0 = s0;
                const float4 q4 = *reinterpret_cast<const float4 *>(s_qr + ph * D + 4 * lane);
                qx[0] = q4.x; qx[1] = q4.y; qx[2] = q4.z; qx[3] = q4.w;
            }
            const int r = (k - c0) * 8 + lane;
            const int id = lane < 8 && r < (int)s_kc[ph] ? s_kbuf[ph * CL_KCAP + r] : -1;
            if (ph < GMAX) attend8<PAGED>(a.k_cache, a.v_cache, a.kv, b0, g0, id, qx, part);
            else attend8<PAGED>(a.k_cache, a.v_cache, a.kv, b1, g1, id, qx, part);
        }
        if (cur >= 0) part.store(s_slot + (cur_s0 + kfirst - cur_c0) * PSTRIDE);
        __syncthreads();
        // merge each head's slots into this CTA's record of the head: one
        // warp per head, lane l folding dims 4 l .. 4 l + 3 slot by slot
        for (int ph = h_lo + warp; ph < h_hi; ph += CL_WARPS) {
            const int s0 = __shfl_sync(0xffffffffu, s0_l, ph), s1 = __shfl_sync(0xffffffffu, ss, ph);
            WarpPart acc;
            acc.reset();
            for (int q = s0; q < s1; ++q) acc.load_add(s_slot + q * PSTRIDE);
            acc.store(a.part_sel + (cta * HP + ph) * PSTRIDE);
        }
        // the slots are reused only by a further round (no barrier after the
        // last: it would wait for the record stores)
        if (h_hi < HP) __syncthreads();
        h_lo = h_hi;
    }
    flush_ids();
}

// ---------------------------------------------------------------------------
// finalize: exact selection inside the boundary bin.  One CTA per head.
// grid = (B * n_ret * G)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float cand_logit(unsigned long long c) { return key_logit((uint32_t)(c >> 32)); }

constexpr int FIN_THREADS = 512;
constexpr int FIN_WARPS = FIN_THREADS / 32;
constexpr int FIN_CAP = 3072;             // candidates staged in shared memory
constexpr int FIN_CLUSTER = 4;            // CTAs per head with the fused attention
constexpr int FIN_FOLD = 3;               // collect records a warp loads at once
constexpr int FIN_SPILL = 2048;           // rows above which finalize hands a head to the list pass
// Exact selection inside the boundary bin.  One CTA per retrieval head, or
// a cluster of FIN_CLUSTER CTAs per head with the fused attention (each
// rank runs the same selection); grid = (1 or FIN_CLUSTER, B * n_ret * G).
// Candidate masses relative to the boundary bin's upper edge U* are each in
// (e^-32, 1]; they are summed in fixed point with S = (2^31 - 1) / nc
// (staged in shared memory) or 2^62 / nc units per unit of mass, so sums
// cannot wrap and do not depend on the order of the adds.  Rank 0 clears
// the head's level-1 histogram for the next call, last.
template <bool PAGED>
__global__ void __launch_bounds__(FIN_THREADS) finalize_kernel(SelArgs a, SelWs w) {
    __shared__ unsigned long long hfx[256];
    __shared__ uint32_t hfx32[256];
    __shared__ unsigned hcnt[256];
    __shared__ __align__(16) unsigned long long cbuf[FIN_CAP];
    __shared__ __align__(16) uint32_t fbuf[FIN_CAP];
    // ids of the kept candidates (staged case), compacted over the start of
    // cbuf once the keys are read
    int32_t *const s_kid = reinterpret_cast<int32_t *>(cbuf);
    __shared__ unsigned long long s_min, s_max, s_theta, s_excl, s_kept;
    __shared__ unsigned s_base2, s_wcnt[FIN_WARPS];
    __shared__ int s_digit;
    __shared__ unsigned s_dcnt;
    __shared__ __align__(16) float s_crec[FIN_CLUSTER * PSTRIDE];   // the ranks' attention partials (fused)
    const int G = a.G;
    // grid (K, heads): with the fused attention the K CTAs of a head form a
    // cluster; each runs the (cheap, identical) selection, rank 0 writes its
    // results, and the ranks split the attention and merge through DSMEM
    const int K = gridDim.x;
    const int rank = blockIdx.x;
    const int hb = blockIdx.y;
    const int b = hb / (a.n_ret * G);
    const int gi = (hb / G) % a.n_ret;
    const int h = a.ret_g[gi] * G + hb % G;
    const size_t bh = (size_t)b * a.H_q + h;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // fused attention: this head's query (scaled), an input of the call that
    // no earlier kernel writes, loads before the wait
    float qx_f[4] = {0.f, 0.f, 0.f, 0.f};
    if (a.q_rope) {
        const float4 q4 = *reinterpret_cast<const float4 *>(a.q_rope + bh * D + 4 * lane);
        qx_f[0] = q4.x * a.attn_scale_log2; qx_f[1] = q4.y * a.attn_scale_log2;
        qx_f[2] = q4.z * a.attn_scale_log2; qx_f[3] = q4.w * a.attn_scale_log2;
    }
    pdl_wait();
    pdl_trigger();
    // the head's resolve record and both counters in one round of loads
    const Resolve r = w.res[bh];
    const unsigned nc_all = a.ext_cnt ? (unsigned)a.ext_cnt[bh] : w.cand_cnt[bh * CNT_STRIDE];
    const unsigned base0 = w.list_cnt[bh * CNT_STRIDE];
    const unsigned ovf = a.q_rope ? a.ovf[bh] : 0u;
    const unsigned long long *cg = a.ext_cands ? a.ext_cands + bh * a.ext_stride : w.cands + bh * a.N_max;
    // first candidate of each thread, loaded before the count is known (the
    // buffer holds N_max -- or ext_stride -- entries, so the read is in bounds)
    const unsigned long long c_first = tid < (a.ext_cands ? a.ext_stride : a.N_max) ? __ldcg(cg + tid) : 0ull;
    // fused attention: fold the collect CTAs' partials of this head while the
    // selection's own loads are in flight (discarded below after an overflow)
    WarpPart part;
    part.reset();
    if (a.q_rope) {
        // the records of this head's pair-head in every CTA of its pair,
        // FIN_FOLD per warp at a time with all their loads issued first (one
        // round trip, not one per record)
        const size_t y = (size_t)b * a.n_ret + gi;
        const float *recs = a.part_sel + ((y % PAIR) * GMAX + (size_t)(hb % G)) * PSTRIDE +
                            (y / PAIR) * a.cl_ctas * HP * PSTRIDE;
        for (int x0 = rank * FIN_WARPS + warp; x0 < a.cl_ctas; x0 += FIN_FOLD * K * FIN_WARPS) {
            float mx[FIN_FOLD], lx[FIN_FOLD];
            float4 ox[FIN_FOLD];
#pragma unroll
            for (int j = 0; j < FIN_FOLD; ++j) {
                const int x = x0 + j * K * FIN_WARPS;
                mx[j] = -INFINITY; lx[j] = 0.0f; ox[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (x < a.cl_ctas) {
                    const float *rc = recs + (size_t)x * HP * PSTRIDE;
                    mx[j] = rc[0];
                    lx[j] = rc[1];
                    ox[j] = *reinterpret_cast<const float4 *>(rc + POFF + 4 * lane);
                }
            }
#pragma unroll
            for (int j = 0; j < FIN_FOLD; ++j) {
                const float o4[4] = {ox[j].x, ox[j].y, ox[j].z, ox[j].w};
                part.add(mx[j], lx[j], o4);
            }
        }
    }
    unsigned long long fin_theta = ~0ull;            // kept boundary candidates: key >= fin_theta
    bool fin_staged = false;                         // the kept candidates' ids are compacted in s_kid
    const unsigned nc = r.mode == MODE_NORMAL ? nc_all : 0u;
    int32_t *lst = a.lists + bh * a.N_max;
    int count = 0;
    float mass = 0.0f;

    if (r.mode == MODE_KEEP_ALL) {
        count = r.N;
        mass = 1.0f;
    } else if (r.mode != MODE_NORMAL || nc == 0u) {
        count = r.mode == MODE_EMPTY ? 0 : (int)base0;
        mass = r.mode == MODE_EMPTY ? 0.0f : (float)(r.above / r.Z);
    } else {
        const float Ub = bin_upper(r.bstar);
        // Staged candidates: 32-bit fixed point, S = floor((2^31 - 1) / nc)
        // units per unit of mass (sums cannot wrap; with nc <= FIN_CAP each
        // mass keeps >= 19 bits).  Otherwise 64-bit, S = 2^62 / nc.
        // (a wide boundary bin -- |z| >= 32, terms down to e^-8 of its edge --
        // always takes the 64-bit path: 32-bit units would leave such terms
        // too few bits)
        const bool staged = nc <= (unsigned)FIN_CAP && wide_slot(r.bstar) < 0;
        fin_staged = staged;
        const double S = staged ? (double)(0x7fffffffu / nc) : ldexp(1.0, 62) / (double)nc;
        // static top-k: every candidate weighs one unit and the target is a
        // whole number of units (exact integers)
        const unsigned long long unit = (unsigned long long)S;
        auto fx_of = [&](unsigned long long v) -> unsigned long long {
            if (a.topk > 0) return unit;
            const float m = ex2_sfu((cand_logit(v) - Ub) * L2E);
            return (unsigned long long)((double)m * S);
        };
        if (tid == 0) { s_min = ~0ull; s_max = 0ull; s_kept = 0ull; s_base2 = 0u; }
        __syncthreads();
        {
            unsigned long long lo = ~0ull, hi = 0ull;
            for (unsigned c = tid; c < nc; c += blockDim.x) {
                const unsigned long long v = c == (unsigned)tid ? c_first : __ldcg(cg + c);
                if (staged) { cbuf[c] = v; fbuf[c] = (uint32_t)fx_of(v); }
                lo = v < lo ? v : lo;
                hi = v > hi ? v : hi;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const unsigned long long l2 = __shfl_xor_sync(0xffffffffu, lo, o);
                const unsigned long long h2 = __shfl_xor_sync(0xffffffffu, hi, o);
                lo = l2 < lo ? l2 : lo;
                hi = h2 > hi ? h2 : hi;
            }
            if (lane == 0) {
                atomicMin(&s_min, lo);
                atomicMax(&s_max, hi);
            }
        }
        __syncthreads();
        const double tS = r.target / (double)ex2_sfu((Ub - r.R) * L2E) * S;
        unsigned long long T = a.topk > 0 ? (r.target < (double)nc ? (unsigned long long)r.target * unit : ~0ull)
                               : !(tS < 9.0e18) ? ~0ull : (unsigned long long)llrint(tS);
        const unsigned long long diff = s_min ^ s_max;
        unsigned long long theta = s_min;          // one candidate (or all equal): keep all
        if (diff != 0ull) {
            int shift = 63 - __clzll((long long)diff);
            shift = shift >= 7 ? shift - 7 : 0;
            unsigned long long pmask = shift + 8 >= 64 ? 0ull : ~((1ull << (shift + 8)) - 1ull);
            unsigned long long prefix = s_min & pmask;
            for (int level = 0; level < 16; ++level) {
                for (int i = tid; i < 256; i += blockDim.x) { hfx[i] = 0ull; hfx32[i] = 0u; hcnt[i] = 0u; }
                __syncthreads();
                if (staged) {
                    for (unsigned c = tid; c < nc; c += blockDim.x) {
                        const unsigned long long v = cbuf[c];
                        if ((v & pmask) != prefix) continue;
                        const int dg = (int)((v >> shift) & 255ull);
                        atomicAdd(&hfx32[dg], fbuf[c]);
                        atomicAdd(&hcnt[dg], 1u);
                    }
                    __syncthreads();
                    for (int i = tid; i < 256; i += blockDim.x) hfx[i] = hfx32[i];
                } else {
                    for (unsigned c = tid; c < nc; c += blockDim.x) {
                        const unsigned long long v = cg[c];
                        if ((v & pmask) != prefix) continue;
                        const int dg = (int)((v >> shift) & 255ull);
                        atomicAdd(&hfx[dg], fx_of(v));
                        atomicAdd(&hcnt[dg], 1u);
                    }
                }
                __syncthreads();
                if (warp == 0) {
                    // lane covers digits 255 - 8 lane - i (descending)
                    unsigned long long seg = 0ull;
                    unsigned segc = 0u;
#pragma unroll
                    for (int i = 0; i < 8; ++i) { seg += hfx[255 - 8 * lane - i]; segc += hcnt[255 - 8 * lane - i]; }
                    unsigned long long incl = seg;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += v;
                    }
                    const unsigned long long excl = incl - seg;
                    const unsigned hit = __ballot_sync(0xffffffffu, segc > 0u && incl >= T);
                    const unsigned ne = __ballot_sync(0xffffffffu, segc > 0u);
                    const int L = hit ? __ffs(hit) - 1 : 31 - __clz(ne);
                    if (lane == L) {
                        unsigned long long cum = excl, before = excl;
                        int dsel = -1;
                        for (int i = 0; i < 8; ++i) {
                            const int dg = 255 - 8 * lane - i;
                            if (hcnt[dg] == 0u) continue;
                            dsel = dg;
                            before = cum;
                            if (hit && cum + hfx[dg] >= T) break;
                            cum += hfx[dg];
                        }
                        s_digit = dsel;
                        s_dcnt = hcnt[dsel];
                        s_excl = before;
                    }
                }
                __syncthreads();
                const int dsel = s_digit;
                T = T >= s_excl ? T - s_excl : 0ull;
                prefix |= (unsigned long long)dsel << shift;
                pmask |= 255ull << shift;
                if (s_dcnt == 1u) {
                    for (unsigned c = tid; c < nc; c += blockDim.x) {
                        const unsigned long long v = staged ? cbuf[c] : cg[c];
                        if ((v & pmask) == prefix) s_theta = v;
                    }
                    __syncthreads();
                    theta = s_theta;
                    break;
                }
                if (shift == 0) { theta = prefix; break; }    // every bit fixed
                shift = shift >= 8 ? shift - 8 : 0;
                __syncthreads();
            }
        }
        // kept = candidates at or above theta: their count and mass, and
        // (staged) their ids, compacted in candidate order -- the same order
        // in every rank of the cluster, which split the list by position --
        // for the attention and for the list append rank 0 makes at the end
        unsigned long long kept = 0ull;
        const unsigned lt = (1u << lane) - 1u;
        unsigned kbase = 0u;                         // kept candidates before this chunk
        for (unsigned c0 = 0; c0 < nc; c0 += blockDim.x) {
            const unsigned c = c0 + tid;
            unsigned long long v = 0ull;
            bool k = false;
            if (c < nc) {
                v = staged ? cbuf[c] : cg[c];
                k = v >= theta;
            }
            const unsigned bal = __ballot_sync(0xffffffffu, k);
            if (k) kept += staged ? fbuf[c] : fx_of(v);
            if (lane == 0) s_wcnt[warp] = (unsigned)__popc(bal);
            // every key of the chunk is read (id i lands on key i / 2, below
            // c0 + blockDim.x / 2) and the warps' counts are in
            __syncthreads();
            unsigned before = 0u, total = 0u;
#pragma unroll
            for (int w2 = 0; w2 < FIN_WARPS; ++w2) {
                const unsigned n = s_wcnt[w2];
                before += w2 < warp ? n : 0u;
                total += n;
            }
            if (staged && k)
                s_kid[kbase + before + __popc(bal & lt)] = (int32_t)(0xffffffffu - (uint32_t)(v & 0xffffffffull));
            kbase += total;
            __syncthreads();                          // the counts are read before the next chunk
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) kept += __shfl_xor_sync(0xffffffffu, kept, o);
        if (lane == 0) atomicAdd(&s_kept, kept);
        __syncthreads();
        count = (int)(base0 + kbase);
        fin_theta = theta;
        const double kept_mass = a.topk > 0 ? (double)(s_kept / unit)
                                            : (double)s_kept / S * (double)ex2_sfu((Ub - r.R) * L2E);
        mass = (float)((r.above + kept_mass) / r.Z);
    }
    // Rank 0's global writes go out last (a global store before a block or
    // cluster barrier makes that barrier wait for it): count and mass, the
    // kept ids (every token for keep-all; the kept boundary candidates after
    // the collect pass's ids), and the cleared histogram for the next call.
    bool spill = false;
    auto finish = [&]() {
        if (rank != 0) return;
        if (a.theta_out) {
            // context shard: the threshold key (every key at or above it is
            // kept; 0 keeps all, ~0 none of the candidates) and the mass
            if (tid == 0) {
                a.theta_out[bh] = r.mode == MODE_KEEP_ALL ? 0ull
                                  : (r.mode == MODE_NORMAL && nc > 0u) ? fin_theta : ~0ull;
                if (a.mass_out) a.mass_out[bh] = mass;
            }
            for (int i = tid; i < HSTRIDE; i += blockDim.x) w.hist[bh * HSTRIDE + i] = 0.0;
            return;
        }
        if (tid == 0) {
            a.count_out[bh] = count;
            if (a.mass_out) a.mass_out[bh] = mass;
            if (spill) {
                a.ovf[bh] = (ovf || r.mode == MODE_KEEP_ALL) ? SPILL_ALL_ROWS : SPILL_FROM_FIRST;
                atomicExch(a.spill_any, 1u);
            }
        }
        if (r.mode == MODE_KEEP_ALL) {
            for (int t = tid; t < r.N; t += blockDim.x) lst[t] = t;
        } else if (r.mode == MODE_NORMAL && nc > 0u) {
            if (fin_staged) {
                for (int i = tid; i < count - (int)base0; i += blockDim.x) lst[base0 + i] = s_kid[i];
            } else {
                for (unsigned c = tid; c < nc; c += blockDim.x) {
                    const unsigned long long v = cg[c];
                    if (v >= fin_theta)
                        lst[base0 + atomicAdd(&s_base2, 1u)] =
                            (int32_t)(0xffffffffu - (uint32_t)(v & 0xffffffffull));
                }
            }
        }
        for (int i = tid; i < HSTRIDE; i += blockDim.x) w.hist[bh * HSTRIDE + i] = 0.0;
    };
    if (!a.q_rope) {
        finish();
        return;
    }

    // Fused attention: the kept rows the collect pass did not attend (the
    // boundary bin's kept candidates, plus, after a staging overflow, the
    // collect pass's rows) are split over the cluster's ranks and warps;
    // each rank merges its warps and the collect records it folded into one
    // partial, stores it into rank 0's shared memory, and rank 0 merges.
    namespace cgr = cooperative_groups;
    cgr::cluster_group cluster = cgr::this_cluster();
    if (count <= 0) {
        // nothing kept (invalid input): zeros and a status
        if (rank == 0) {
            for (int d = tid; d < D; d += blockDim.x) a.out[bh * D + d] = 0.0f;
            if (tid == 0) set_status(w.status, RTP_ERR_DEVICE_ARG);
        }
        finish();
        return;
    }
    if (ovf) part.reset();                           // a collect CTA could not attend all its kept rows
    {
        // rows this cluster would attend: hand them over to the list pass
        // when there are many (the same decision in every rank)
        const long long att = (r.mode == MODE_KEEP_ALL ? (long long)count : (long long)count - base0) +
                              (ovf ? (long long)base0 : 0LL);
        spill = a.spill_rows > 0 && att > (long long)a.spill_rows;
    }
    if (!spill) {
        const int g = h / G;
        const int worker = rank * FIN_WARPS + warp, workers = K * FIN_WARPS;
        if (ovf) {
            // the collect pass's rows, from its list
            for (int rb = worker * 8; rb < (int)base0; rb += workers * 8) {
                const int id = lane < 8 && rb + lane < (int)base0 ? __ldcg(lst + rb + lane) : -1;
                attend8<PAGED>(a.k_cache, a.v_cache, a.kv, b, g, id, qx_f, part);
            }
        }
        if (r.mode == MODE_KEEP_ALL) {
            for (int rb = worker * 8; rb < count; rb += workers * 8) {
                const int id = lane < 8 && rb + lane < count ? rb + lane : -1;
                attend8<PAGED>(a.k_cache, a.v_cache, a.kv, b, g, id, qx_f, part);
            }
        } else if (r.mode == MODE_NORMAL) {
            // boundary-bin candidates at or above theta: the compacted ids
            // (staged), else eight candidate slots at a time
            if (fin_staged) {
                const int nk = count - (int)base0;
                for (int rb = worker * 8; rb < nk; rb += workers * 8)
                    attend8<PAGED>(a.k_cache, a.v_cache, a.kv, b, g, lane < 8 && rb + lane < nk ? s_kid[rb + lane] : -1, qx_f, part);
            } else {
                for (int cb = worker * 8; cb < (int)nc; cb += workers * 8) {
                    int id = -1;
                    if (lane < 8 && cb + lane < (int)nc) {
                        const unsigned long long v = __ldcg(cg + cb + lane);
                        if (v >= fin_theta) id = (int)(0xffffffffu - (uint32_t)(v & 0xffffffffull));
                    }
                    attend8<PAGED>(a.k_cache, a.v_cache, a.kv, b, g, id, qx_f, part);
                }
            }
        }
    }
    // the warps' partials go into the mass buffer (no longer needed; the
    // candidates stay for the list append at the end)
    float *slots = reinterpret_cast<float *>(fbuf);
    static_assert(FIN_WARPS * PSTRIDE <= FIN_CAP, "partial slots fit the mass buffer");
    __syncthreads();                                 // every thread is done with the masses
    part.store(slots + warp * PSTRIDE);
    __syncthreads();
    // this rank's partial goes into slot `rank` of rank 0's s_crec
    float *dst = K > 1 ? cluster.map_shared_rank(s_crec, 0) + rank * PSTRIDE : s_crec;
    for (int d = tid; d < D; d += blockDim.x) {
        float M = -INFINITY;
#pragma unroll
        for (int w2 = 0; w2 < FIN_WARPS; ++w2) M = fmaxf(M, slots[w2 * PSTRIDE]);
        float L = 0.0f, O = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w2 = 0; w2 < FIN_WARPS; ++w2) {
                const float *sl = slots + w2 * PSTRIDE;
                const float wg = sl[0] == -INFINITY ? 0.0f : exp2f(sl[0] - M);
                L = fmaf(sl[1], wg, L);
                O = fmaf(sl[POFF + d], wg, O);
            }
        }
        dst[POFF + d] = O;
        if (d == 0) { dst[0] = M; dst[1] = L; }
    }
    if (K > 1) cluster.sync(); else __syncthreads();
    if (rank == 0) {
        for (int d = tid; d < D; d += blockDim.x) {
            float M = -INFINITY;
            for (int r2 = 0; r2 < K; ++r2) M = fmaxf(M, s_crec[r2 * PSTRIDE]);
            float L = 0.0f, O = 0.0f;
            if (M != -INFINITY) {
                for (int r2 = 0; r2 < K; ++r2) {
                    const float *rc = s_crec + r2 * PSTRIDE;
                    const float wg = rc[0] == -INFINITY ? 0.0f : exp2f(rc[0] - M);
                    L = fmaf(rc[1], wg, L);
                    O = fmaf(rc[POFF + d], wg, O);
                }
            }
            if (spill) {
                // the list pass adds the remaining rows and merges
                float *pl = a.part_list + bh * (size_t)LIST_SLOTS * PSTRIDE;
                pl[POFF + d] = O;
                if (d == 0) { pl[0] = M; pl[1] = L; }
            } else {
                a.out[bh * D + d] = O * (L > 0.0f ? 1.0f / L : 0.0f);
            }
        }
    }
    finish();
}

// ---------------------------------------------------------------------------
// Context shard: this shard's kept list of each retrieval head -- the ids
// the collect pass kept (global, already in the list) plus the shard's own
// boundary candidates at or above the head's threshold key (their global
// ids), or every token of the shard for a keep-all head.  grid = (B * n_ret
// * G), OWN_THREADS threads.
// ---------------------------------------------------------------------------
constexpr int OWN_THREADS = 256;
__global__ void __launch_bounds__(OWN_THREADS) shard_own_kernel(SelArgs a, SelWs w) {
    __shared__ unsigned s_n;
    const int hb = blockIdx.x;
    const int G = a.G;
    const int b = hb / (a.n_ret * G);
    const int gi = (hb / G) % a.n_ret;
    const int h = a.ret_g[gi] * G + hb % G;
    const size_t bh = (size_t)b * a.H_q + h;
    const int N = a.seq_lens[b];
    const int off = a.id_off[b];
    int32_t *lst = a.lists + bh * a.N_max;
    if (N < 1 || (long long)N > a.N_max) {
        if (threadIdx.x == 0) a.count_out[bh] = 0;
        return;
    }
    const Resolve r = w.res[bh];
    if (r.mode == MODE_KEEP_ALL) {
        for (int t = threadIdx.x; t < N; t += blockDim.x) lst[t] = off + t;
        if (threadIdx.x == 0) a.count_out[bh] = N;
        return;
    }
    const unsigned base0 = r.mode == MODE_NORMAL ? w.list_cnt[bh * CNT_STRIDE] : 0u;
    const unsigned nc = r.mode == MODE_NORMAL ? w.cand_cnt[bh * CNT_STRIDE] : 0u;
    const unsigned long long theta = a.theta_out[bh];
    if (threadIdx.x == 0) s_n = 0u;
    __syncthreads();
    const unsigned long long *cg = w.cands + bh * a.N_max;
    for (unsigned c = threadIdx.x; c < nc; c += blockDim.x) {
        const unsigned long long v = cg[c];
        if (v >= theta) lst[base0 + atomicAdd(&s_n, 1u)] = (int32_t)(0xffffffffu - (uint32_t)(v & 0xffffffffull));
    }
    __syncthreads();
    if (threadIdx.x == 0) a.count_out[bh] = (int)(base0 + s_n);
}

// ---------------------------------------------------------------------------
// rtp_index_scores: write z for every retrieval head (same logit sources)
// ---------------------------------------------------------------------------
template <typename Src>
__global__ void __launch_bounds__(SC_THREADS) scores_kernel(SelArgs a, SelWs w, float *z_out) {
    __shared__ __align__(16) float qs[GMAX * R];
    const int b = blockIdx.y / a.n_ret;
    const int g = a.ret_g[blockIdx.y % a.n_ret];
    const int G = a.G;
    const size_t bh0 = (size_t)b * a.H_q + (size_t)g * G;
    project_query<(GMAX * R + SC_WARPS - 1) / SC_WARPS>(a.q + bh0 * D, a.Wq + (size_t)g * G * R * D, a.idx_scale,
                                                         qs, G, threadIdx.x >> 5, SC_WARPS);
    __syncthreads();
    const int N = valid_len(a.seq_lens, b, a.N_max, w.status);
    Src src;
    init_src(src, a, b, g, qs);
    const int warp = threadIdx.x >> 5;
    const int t_lo = (int)((long long)blockIdx.x * a.chunk);
    const int t_hi = (int)min((long long)N, (long long)t_lo + a.chunk);
    float *zb = z_out + bh0 * a.N_max;
    for (int tb = t_lo + warp * TILE; tb < t_hi; tb += SC_WARPS * TILE) {
        typename Src::Frag f;
        src.load(tb, f);
        float z[Src::NV];
        src.eval(f, z);
#pragma unroll
        for (int v = 0; v < Src::NV; ++v) {
            const int h = src.head(src.slot(v));
            const int t = tb + src.tok(v);
            if (h < G && t < t_hi) zb[h * a.N_max + t] = z[v];
        }
    }
}

}  // namespace rtp
