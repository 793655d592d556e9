// Indexer scoring and the sort-free top-p threshold (sm_100a).
//
// "Full Attention Strikes Back" (gist.science technical summary), Method
// sections 2, 3 and 5: retrieval heads score every cached token in a
// 16-dim pre-RoPE subspace, turn the scores into softmax mass, and keep the
// smallest descending-score prefix whose mass reaches p; the kernels find
// that threshold with histograms instead of a sort.
//
// Stages (per sequence b and retrieval KV head g, all G query heads of the
// group at once so each index-key row is read once per pass):
//   hist     stream the logits (from the index keys, or from a logit
//            buffer), accumulate a per-head level-1 mass histogram over the
//            order-preserving bits of z (rtp_common.cuh), record the
//            largest bin of every 32-token tile; the last CTA of the group
//            resolves the boundary bin b* of each head.
//   collect  re-derive the logits of tiles whose largest bin reaches b*,
//            append tokens above b* to the head's kept list and tokens in
//            b* to its candidate list (64-bit composite key: logit key,
//            then inverted token id, so the order is total).
//   finalize exact radix select by mass over the candidates (8-bit digits
//            of the composite key, most significant first) to the unique
//            boundary token, then append the candidates at or above it.
#pragma once

#include <type_traits>

#include "rtp_common.cuh"

namespace rtp {

constexpr int SEL_THREADS = 256;
constexpr int SEL_CHUNK = 4096;            // tokens per CTA in hist/collect
constexpr int TILE = 32;                   // tokens per warp tile
constexpr int MAX_RET_GROUPS = 64;

enum ResolveMode : int32_t { MODE_NORMAL = 0, MODE_KEEP_ALL = 1, MODE_EMPTY = 2 };

struct Resolve {
    double Z;          // sum of masses, relative to exp(R)
    double above;      // mass of bins above b*, same units
    double target;     // mass still needed inside b*, same units
    float R;           // reference logit: upper edge of the top bin
    int32_t bstar;     // boundary bin
    int32_t mode;      // ResolveMode
    int32_t N;         // valid tokens
    int32_t pad[2];
};
static_assert(sizeof(Resolve) == 48, "Resolve layout");

// Pointers into the workspace used by the selection stages.
struct SelWs {
    uint32_t *status;
    uint32_t *arrive;      // [B*H_kv] hist arrivals
    uint32_t *list_cnt;    // [B*H_q]
    uint32_t *cand_cnt;    // [B*H_q]
    double *hist;          // [B*H_q*NBIN]
    Resolve *res;          // [B*H_q]
    uint16_t *tilebin;     // [B*H_q*ntile]: 1 + largest bin of the tile (0: empty)
    unsigned long long *cands;  // [B*H_q*N_max]
    float *qidx;           // [B*H_q*R] scaled query projections
};

struct SelArgs {
    int B, H_q, H_kv, G;
    long long N_max;
    int ntile;             // ceil(N_max / TILE)
    const int32_t *seq_lens;
    int n_ret;             // retrieval KV heads
    int ret_g[MAX_RET_GROUPS];
    float p;
    const void *kidx;      // [B, H_kv, N_max, R] (FromIndex)
    const float *z;        // [B, H_q, N_max] (FromBuffer)
    int32_t *lists;        // [B*H_q*N_max] kept ids
    int32_t *count_out;    // [B*H_q]
    float *mass_out;       // [B*H_q] or null
};

__device__ __forceinline__ int valid_len(const int32_t *seq_lens, int b, long long N_max,
                                         uint32_t *status) {
    int N = seq_lens[b];
    if (N < 1 || (long long)N > N_max) {
        set_status(status, RTP_ERR_DEVICE_ARG);
        return 0;
    }
    return N;
}

// ---------------------------------------------------------------------------
// q_idx[b, h, :] = scale * W_q_idx[h] . q[b, h]   (one CTA per (b, h))
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(512) qidx_kernel(const float *__restrict__ q,
                                                   const float *__restrict__ W,
                                                   float *__restrict__ qidx, int H_q,
                                                   int G, unsigned long long ret_mask,
                                                   float scale) {
    const int bh = blockIdx.x;
    const int h = bh % H_q;
    if (!((ret_mask >> (h / G)) & 1ull)) return;
    const int j = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float4 qv = __ldg(reinterpret_cast<const float4 *>(q + (size_t)bh * D) + lane);
    const float4 wv = __ldg(reinterpret_cast<const float4 *>(W + ((size_t)h * R + j) * D) + lane);
    float acc = qv.x * wv.x;
    acc = fmaf(qv.y, wv.y, acc);
    acc = fmaf(qv.z, wv.z, acc);
    acc = fmaf(qv.w, wv.w, acc);
    acc = warp_sum(acc);
    if (lane == 0) qidx[(size_t)bh * R + j] = acc * scale;
}

// ---------------------------------------------------------------------------
// logit sources.  Both passes derive z through the same code, so the
// histogram pass and the collect pass see bit-identical logits.
// ---------------------------------------------------------------------------
template <typename IT>
struct FromIndex {
    const IT *rows;   // kidx of (b, g): [N_max, R]
    const float *qs;  // shared [G][R]
    int G;
    __device__ __forceinline__ void logits(long long t, float (&z)[GMAX]) const {
        float k[R];
        float lo[8], hi[8];
        Row<IT>::load8(rows + t * R, lo);
        Row<IT>::load8(rows + t * R + 8, hi);
#pragma unroll
        for (int j = 0; j < 8; ++j) { k[j] = lo[j]; k[8 + j] = hi[j]; }
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            if (h < G) {
                const float4 *qh = reinterpret_cast<const float4 *>(qs + h * R);
                float acc = 0.0f;
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4) {
                    float4 w = qh[j4];
                    acc = __fmaf_rn(w.x, k[4 * j4 + 0], acc);
                    acc = __fmaf_rn(w.y, k[4 * j4 + 1], acc);
                    acc = __fmaf_rn(w.z, k[4 * j4 + 2], acc);
                    acc = __fmaf_rn(w.w, k[4 * j4 + 3], acc);
                }
                z[h] = acc;
            }
        }
    }
};

struct FromBuffer {
    const float *zb;  // z of head (b, g*G): [G][N_max]
    long long N_max;
    int G;
    __device__ __forceinline__ void logits(long long t, float (&z)[GMAX]) const {
#pragma unroll
        for (int h = 0; h < GMAX; ++h)
            if (h < G) z[h] = __ldg(zb + h * N_max + t);
    }
};

// ---------------------------------------------------------------------------
// rtp_index_scores: write z for every retrieval head
// ---------------------------------------------------------------------------
template <typename IT>
__global__ void __launch_bounds__(SEL_THREADS) scores_kernel(SelArgs a, SelWs w, float *z_out) {
    __shared__ __align__(16) float qs[GMAX * R];
    const int b = blockIdx.y / a.n_ret;
    const int g = a.ret_g[blockIdx.y % a.n_ret];
    const int G = a.G;
    for (int i = threadIdx.x; i < G * R; i += blockDim.x)
        qs[i] = w.qidx[((size_t)b * a.H_q + g * G) * R + i];
    __syncthreads();
    const int N = valid_len(a.seq_lens, b, a.N_max, w.status);
    const FromIndex<IT> src{reinterpret_cast<const IT *>(a.kidx) + ((size_t)b * a.H_kv + g) * a.N_max * R, qs, G};
    float *zb = z_out + ((size_t)b * a.H_q + g * G) * a.N_max;
    const long long t0 = (long long)blockIdx.x * SEL_CHUNK;
    for (long long t = t0 + threadIdx.x; t < t0 + SEL_CHUNK && t < N; t += blockDim.x) {
        float z[GMAX];
        src.logits(t, z);
#pragma unroll
        for (int h = 0; h < GMAX; ++h)
            if (h < G) zb[h * a.N_max + t] = z[h];
    }
}

// ---------------------------------------------------------------------------
// resolve: one warp per head, after the group's histogram is complete.
// Bin masses M_b = S_b * exp(U_b - R) (fp64), R = U(top bin).  The boundary
// bin is the first one, walking down from the top, whose inclusive
// cumulative mass reaches p * Z.
// ---------------------------------------------------------------------------
__device__ void resolve_head(double *gh, Resolve *out, float p, int N) {
    const int lane = threadIdx.x & 31;
    int top = -1;
    for (int bin = lane; bin < NBIN; bin += 32)
        if (gh[bin] > 0.0) top = bin;
    top = __reduce_max_sync(0xffffffffu, top);
    Resolve r;
    r.N = N;
    r.pad[0] = r.pad[1] = 0;
    if (top < 0 || N == 0) {
        r.Z = 0; r.above = 0; r.target = 0; r.R = 0.f; r.bstar = -1; r.mode = MODE_EMPTY;
        if (lane == 0) *out = r;
        __syncwarp();
        for (int bin = lane; bin < NBIN; bin += 32) gh[bin] = 0.0;
        return;
    }
    const float R = bin_upper(top);
    constexpr int SEG = (NBIN + 31) / 32;
    // lane l covers bins top - l*SEG - i, i = 0..SEG-1 (descending)
    double seg = 0.0;
    for (int i = 0; i < SEG; ++i) {
        int bin = top - lane * SEG - i;
        if (bin < 0) break;
        double s = gh[bin];
        if (s > 0.0) seg += s * exp((double)bin_upper(bin) - (double)R);
    }
    double incl = seg;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const double Z = __shfl_sync(0xffffffffu, incl, 31);
    const double excl = incl - seg;
    r.Z = Z;
    r.R = R;
    if (p >= 1.0f) {
        r.mode = MODE_KEEP_ALL; r.bstar = -1; r.above = 0; r.target = 0;
    } else {
        const double target = p <= 0.0f ? 0.0 : (double)p * Z;
        unsigned hit = __ballot_sync(0xffffffffu, seg > 0.0 && excl + seg >= target);
        int L;
        double cum;
        int bstar = -1;
        double above = 0.0, tin = 0.0;
        if (hit) {
            L = __ffs(hit) - 1;
            cum = __shfl_sync(0xffffffffu, excl, L);
            if (lane == L) {
                for (int i = 0; i < SEG; ++i) {
                    int bin = top - lane * SEG - i;
                    if (bin < 0) break;
                    double s = gh[bin];
                    if (s <= 0.0) continue;
                    double m = s * exp((double)bin_upper(bin) - (double)R);
                    // if rounding never crosses, the last nonempty bin is kept whole
                    bstar = bin;
                    above = cum;
                    if (cum + m >= target) { tin = target - cum; break; }
                    cum += m;
                    tin = INFINITY;
                }
            }
            bstar = __shfl_sync(0xffffffffu, bstar, L);
            above = __shfl_sync(0xffffffffu, above, L);
            tin = __shfl_sync(0xffffffffu, tin, L);
        } else {
            // rounding kept p * Z out of reach: keep everything down to the
            // lowest nonempty bin
            int low = NBIN;
            for (int bin = lane; bin < NBIN; bin += 32)
                if (gh[bin] > 0.0) low = min(low, bin);
            low = __reduce_min_sync(0xffffffffu, low);
            bstar = low;
            double m = gh[low] * exp((double)bin_upper(low) - (double)R);
            above = Z - m;
            tin = INFINITY;
        }
        r.mode = MODE_NORMAL;
        r.bstar = bstar;
        r.above = above;
        r.target = tin;
    }
    if (lane == 0) *out = r;
    __syncwarp();
    for (int bin = lane; bin < NBIN; bin += 32) gh[bin] = 0.0;
}

// ---------------------------------------------------------------------------
// hist: level-1 histogram + tile maxima; last CTA per (b, g) resolves.
// grid = (ceil(N_max / SEL_CHUNK), B * n_ret)
// ---------------------------------------------------------------------------
template <typename Src, typename IT>
__global__ void __launch_bounds__(SEL_THREADS) hist_kernel(SelArgs a, SelWs w) {
    __shared__ __align__(16) float qs[GMAX * R];
    __shared__ float sh[GMAX][NBIN];
    __shared__ int s_last;
    __shared__ int s_err;
    const int b = blockIdx.y / a.n_ret;
    const int g = a.ret_g[blockIdx.y % a.n_ret];
    const int G = a.G;
    const size_t bh0 = (size_t)b * a.H_q + g * G;
    for (int i = threadIdx.x; i < GMAX * NBIN; i += blockDim.x) (&sh[0][0])[i] = 0.0f;
    if (threadIdx.x == 0) s_err = 0;
    if constexpr (!std::is_same<Src, FromBuffer>::value)
        for (int i = threadIdx.x; i < G * R; i += blockDim.x) qs[i] = w.qidx[bh0 * R + i];
    __syncthreads();
    const int N = valid_len(a.seq_lens, b, a.N_max, w.status);
    Src src;
    if constexpr (std::is_same<Src, FromBuffer>::value) {
        src = FromBuffer{a.z + bh0 * a.N_max, a.N_max, G};
    } else {
        src = Src{reinterpret_cast<const IT *>(a.kidx) + ((size_t)b * a.H_kv + g) * a.N_max * R, qs, G};
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long c0 = (long long)blockIdx.x * SEL_CHUNK;
    int err = 0;
    for (long long tb = c0 + warp * TILE; tb < c0 + SEL_CHUNK && tb < N; tb += (SEL_THREADS / 32) * TILE) {
        const long long t = tb + lane;
        const bool valid = t < N;
        float z[GMAX];
        if (valid) src.logits(t, z);
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            if (h >= G) break;
            int bin = -1;
            if (valid) {
                float zz = z[h];
                if (!(fabsf(zz) < Z_LIMIT)) {
                    err = 1;
                } else {
                    bin = logit_bin(zz);
                    atomicAdd(&sh[h][bin], __expf(zz - bin_upper(bin)));
                }
            }
            int mx = __reduce_max_sync(0xffffffffu, bin);
            if (lane == h) w.tilebin[(bh0 + h) * a.ntile + (tb / TILE)] = (uint16_t)(mx + 1);
        }
    }
    if (err) s_err = 1;
    __syncthreads();
    if (s_err && threadIdx.x == 0) set_status(w.status, RTP_ERR_RANGE);
    for (int i = threadIdx.x; i < G * NBIN; i += blockDim.x) {
        float v = (&sh[0][0])[i];
        if (v != 0.0f) atomicAdd(&w.hist[bh0 * NBIN + i], (double)v);
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned old = atomicAdd(&w.arrive[(size_t)b * a.H_kv + g], 1u);
        s_last = (old == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (warp < G) {
        const size_t bh = bh0 + warp;
        resolve_head(w.hist + bh * NBIN, w.res + bh, a.p, N);
        if (lane == 0) { w.list_cnt[bh] = 0; w.cand_cnt[bh] = 0; }
    }
    if (threadIdx.x == 0) w.arrive[(size_t)b * a.H_kv + g] = 0;
}

// ---------------------------------------------------------------------------
// collect: kept ids and boundary-bin candidates.  grid as hist_kernel.
// ---------------------------------------------------------------------------
template <typename Src, typename IT>
__global__ void __launch_bounds__(SEL_THREADS) collect_kernel(SelArgs a, SelWs w) {
    __shared__ __align__(16) float qs[GMAX * R];
    __shared__ int s_bstar[GMAX];
    __shared__ int s_mode[GMAX];
    const int b = blockIdx.y / a.n_ret;
    const int g = a.ret_g[blockIdx.y % a.n_ret];
    const int G = a.G;
    const size_t bh0 = (size_t)b * a.H_q + g * G;
    if (threadIdx.x < G) {
        const Resolve &r = w.res[bh0 + threadIdx.x];
        s_bstar[threadIdx.x] = r.bstar;
        s_mode[threadIdx.x] = r.mode;
    }
    if constexpr (!std::is_same<Src, FromBuffer>::value)
        for (int i = threadIdx.x; i < G * R; i += blockDim.x) qs[i] = w.qidx[bh0 * R + i];
    __syncthreads();
    const int N = w.res[bh0].N;
    Src src;
    if constexpr (std::is_same<Src, FromBuffer>::value) {
        src = FromBuffer{a.z + bh0 * a.N_max, a.N_max, G};
    } else {
        src = Src{reinterpret_cast<const IT *>(a.kidx) + ((size_t)b * a.H_kv + g) * a.N_max * R, qs, G};
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    const long long c0 = (long long)blockIdx.x * SEL_CHUNK;
    for (long long tb = c0 + warp * TILE; tb < c0 + SEL_CHUNK && tb < N; tb += (SEL_THREADS / 32) * TILE) {
        // skip tiles whose largest bin is below every head's boundary bin
        bool need = false;
        for (int h = 0; h < G; ++h) {
            int mode = s_mode[h];
            if (mode == MODE_KEEP_ALL) { need = true; break; }
            if (mode == MODE_NORMAL &&
                (int)w.tilebin[(bh0 + h) * a.ntile + tb / TILE] - 1 >= s_bstar[h]) { need = true; break; }
        }
        if (!need) continue;
        const long long t = tb + lane;
        const bool valid = t < N;
        float z[GMAX];
        if (valid) src.logits(t, z);
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            if (h >= G) break;
            const int mode = s_mode[h];
            if (mode == MODE_EMPTY) continue;
            bool keep = false, cand = false;
            uint32_t key = 0;
            if (valid) {
                if (mode == MODE_KEEP_ALL) {
                    keep = true;
                } else if (fabsf(z[h]) < Z_LIMIT) {
                    const int bin = logit_bin(z[h]);
                    keep = bin > s_bstar[h];
                    cand = bin == s_bstar[h];
                    key = logit_key(z[h]);
                }
            }
            const size_t bh = bh0 + h;
            unsigned bk = __ballot_sync(0xffffffffu, keep);
            if (bk) {
                unsigned base = 0;
                if (lane == 0) base = atomicAdd(&w.list_cnt[bh], (unsigned)__popc(bk));
                base = __shfl_sync(0xffffffffu, base, 0);
                if (keep) a.lists[bh * a.N_max + base + __popc(bk & lt_mask)] = (int32_t)t;
            }
            unsigned bc = __ballot_sync(0xffffffffu, cand);
            if (bc) {
                unsigned base = 0;
                if (lane == 0) base = atomicAdd(&w.cand_cnt[bh], (unsigned)__popc(bc));
                base = __shfl_sync(0xffffffffu, base, 0);
                if (cand)
                    w.cands[bh * a.N_max + base + __popc(bc & lt_mask)] =
                        ((unsigned long long)key << 32) | (unsigned long long)(0xffffffffu - (uint32_t)t);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// finalize: exact selection inside the boundary bin.  One CTA per head.
// grid = (B * n_ret * G)
// ---------------------------------------------------------------------------
__device__ __forceinline__ double cand_mass(unsigned long long c, float R) {
    return exp((double)key_logit((uint32_t)(c >> 32)) - (double)R);
}

__global__ void __launch_bounds__(SEL_THREADS) finalize_kernel(SelArgs a, SelWs w) {
    __shared__ double smass[256];
    __shared__ unsigned scnt[256];
    __shared__ int s_digit;
    __shared__ unsigned s_dcnt;
    __shared__ double s_excl;
    __shared__ unsigned long long s_theta;
    __shared__ double s_red[SEL_THREADS / 32];
    const int G = a.G;
    const int hb = blockIdx.x;                  // (b, ret group, head in group)
    const int b = hb / (a.n_ret * G);
    const int gi = (hb / G) % a.n_ret;
    const int h = a.ret_g[gi] * G + hb % G;
    const size_t bh = (size_t)b * a.H_q + h;
    const Resolve r = w.res[bh];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (r.mode != MODE_NORMAL) {
        if (tid == 0) {
            a.count_out[bh] = r.mode == MODE_KEEP_ALL ? (int32_t)w.list_cnt[bh] : 0;
            if (a.mass_out) a.mass_out[bh] = r.mode == MODE_KEEP_ALL ? 1.0f : 0.0f;
        }
        return;
    }
    const unsigned nc = w.cand_cnt[bh];
    const unsigned long long *cs = w.cands + bh * a.N_max;
    double t = r.target;
    unsigned long long prefix = 0;
    unsigned long long theta = 0;
    bool found = false;
    for (int level = 0; level < 8 && !found; ++level) {
        const int shift = 56 - 8 * level;
        for (int i = tid; i < 256; i += blockDim.x) { smass[i] = 0.0; scnt[i] = 0; }
        __syncthreads();
        for (unsigned c = tid; c < nc; c += blockDim.x) {
            unsigned long long v = cs[c];
            if (level > 0 && (v >> (shift + 8)) != prefix) continue;
            int dg = (int)((v >> shift) & 255ull);
            atomicAdd(&smass[dg], cand_mass(v, r.R));
            atomicAdd(&scnt[dg], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            // lane covers digits 255 - 8*lane - i, i = 0..7 (descending)
            double seg = 0.0;
            for (int i = 0; i < 8; ++i) seg += smass[255 - 8 * lane - i];
            unsigned segc = 0;
            for (int i = 0; i < 8; ++i) segc += scnt[255 - 8 * lane - i];
            double incl = seg;
            for (int o = 1; o < 32; o <<= 1) {
                double v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const double excl = incl - seg;
            unsigned hit = __ballot_sync(0xffffffffu, segc > 0 && excl + seg >= t);
            int L;
            if (hit) {
                L = __ffs(hit) - 1;
            } else {
                unsigned ne = __ballot_sync(0xffffffffu, segc > 0);
                L = 31 - __clz(ne);   // lowest nonempty segment: keep everything above
            }
            if (lane == L) {
                double cum = excl;
                int dsel = -1;
                for (int i = 0; i < 8; ++i) {
                    int dg = 255 - 8 * lane - i;
                    if (scnt[dg] == 0) continue;
                    dsel = dg;
                    if (hit && cum + smass[dg] >= t) break;
                    if (!hit) { /* keep scanning to the last nonempty digit */ }
                    cum += smass[dg];
                }
                if (!hit) {
                    // every candidate under this prefix is kept: cum counts all but dsel
                    cum = excl;
                    for (int i = 0; i < 8; ++i) {
                        int dg = 255 - 8 * lane - i;
                        if (dg == dsel) break;
                        cum += smass[dg];
                    }
                }
                s_digit = dsel;
                s_dcnt = scnt[dsel];
                s_excl = cum;
            }
        }
        __syncthreads();
        const int dsel = s_digit;
        t -= s_excl;
        prefix = (prefix << 8) | (unsigned long long)dsel;
        if (s_dcnt == 1u || level == 7) {
            if (level == 7) {
                theta = prefix;
            } else {
                if (tid == 0) s_theta = 0;
                __syncthreads();
                for (unsigned c = tid; c < nc; c += blockDim.x) {
                    unsigned long long v = cs[c];
                    if ((v >> shift) == prefix) s_theta = v;
                }
                __syncthreads();
                theta = s_theta;
            }
            found = true;
        }
        __syncthreads();
    }
    // append candidates at or above theta
    double kept = 0.0;
    for (unsigned c = tid; c < nc; c += blockDim.x) {
        unsigned long long v = cs[c];
        if (v >= theta) {
            unsigned pos = atomicAdd(&w.list_cnt[bh], 1u);
            a.lists[bh * a.N_max + pos] = (int32_t)(0xffffffffu - (uint32_t)(v & 0xffffffffull));
            kept += cand_mass(v, r.R);
        }
    }
    kept = warp_sum_d(kept);
    if (lane == 0) s_red[warp] = kept;
    __syncthreads();
    if (tid == 0) {
        double tot = 0.0;
        for (int i = 0; i < SEL_THREADS / 32; ++i) tot += s_red[i];
        a.count_out[bh] = (int32_t)w.list_cnt[bh];
        if (a.mass_out) a.mass_out[bh] = (float)((r.above + tot) / r.Z);
    }
}

}  // namespace rtp
