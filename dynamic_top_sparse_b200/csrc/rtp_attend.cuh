// Decode attention kernels (sm_100a): exact softmax attention of one new
// query per head over a set of cached rows, fp32 accumulation.
//
//   range_attn_kernel  all G query heads of a KV head over a row range
//                      set: the sink rows plus the sliding window of a
//                      local head ("Full Attention Strikes Back",
//                      gist.science technical summary, Method section 1),
//                      or every row (dense comparison kernel).  Each K/V row
//                      is read once for the whole GQA group.
//   list_attn_kernel   one retrieval head over its kept rows (same summary,
//                      Method section 5: sparse decode gathers only the
//                      selected K/V rows).  Persistent CTAs walk a work list
//                      of (head, row slice) items built on the device from
//                      the kept-set sizes.
// Both split the rows over CTAs and merge the flash-decoding partials
// (running max m, sum l, unnormalised o, in log2 units) in the last CTA to
// finish, found with an arrival counter.
#pragma once

#include <type_traits>

#include "rtp_common.cuh"

namespace rtp {

constexpr int ATT_THREADS = 256;
constexpr int RCH = 256;               // rows per range sub-chunk (one per thread)
constexpr int MAX_GROUPS = 64;
constexpr int MAX_RET_Q = 512;
constexpr int MAX_LIST_HEADS = 4096;

// Merge n flash-decoding partial records (stride `rec` floats between
// records; record h of a group at + h * PSTRIDE) for heads [0, nh) into
// out[h * D + d].  Every thread owns 4 dims of one head and merges in one
// pass with a running max, keeping 16 records' loads in flight.
// raw != null: the merged records (m, l, unnormalised o) go to raw + h
// PSTRIDE instead of the normalised outputs (a shard's partial of a
// context-sharded step).
__device__ __forceinline__ void merge_partials(const float *__restrict__ pb, int n, int rec, int nh,
                                               float *__restrict__ out, float *__restrict__ raw = nullptr) {
    constexpr int U = 16;
    for (int i = threadIdx.x; i < nh * (D / 4); i += blockDim.x) {
        const int h = i / (D / 4), d4 = i % (D / 4);
        const float *base = pb + h * PSTRIDE;
        float M = -INFINITY, l = 0.0f;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp = 0; sp < n; sp += U) {
            float mm[U], ll[U];
            float4 oo[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (sp + u < n) {
                    const float *r = base + (size_t)(sp + u) * rec;
                    mm[u] = __ldcg(r);
                    ll[u] = __ldcg(r + 1);
                    oo[u] = __ldcg(reinterpret_cast<const float4 *>(r + POFF) + d4);
                } else {
                    mm[u] = -INFINITY; ll[u] = 0.0f; oo[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            float Mb = M;
#pragma unroll
            for (int u = 0; u < U; ++u) Mb = fmaxf(Mb, mm[u]);
            if (Mb == -INFINITY) continue;
            const float sc = M == -INFINITY ? 0.0f : exp2f(M - Mb);
            l *= sc;
            o.x *= sc; o.y *= sc; o.z *= sc; o.w *= sc;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const float wg = mm[u] == -INFINITY ? 0.0f : exp2f(mm[u] - Mb);
                l = fmaf(ll[u], wg, l);
                o.x = fmaf(oo[u].x, wg, o.x); o.y = fmaf(oo[u].y, wg, o.y);
                o.z = fmaf(oo[u].z, wg, o.z); o.w = fmaf(oo[u].w, wg, o.w);
            }
            M = Mb;
        }
        if (raw) {
            float *rr = raw + (size_t)h * PSTRIDE;
            reinterpret_cast<float4 *>(rr + POFF)[d4] = o;
            if (d4 == 0) { rr[0] = M; rr[1] = l; }
            continue;
        }
        const float inv = l > 0.0f ? 1.0f / l : 0.0f;
        reinterpret_cast<float4 *>(out + h * D)[d4] = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    }
}

struct RangeArgs {
    int B, H_q, H_kv, G;
    long long N_max;
    const int32_t *seq_lens;
    int n_grp;
    int grp[MAX_GROUPS];
    int dense;
    int window, n_sink;
    int n_split;
    int slots;          // partial slots reserved per KV group (>= n_split)
    float scale_log2;
    const float *q;
    const void *k;
    const void *v;
    float *out;
    float *part;        // [B*H_kv][slots][GMAX][PSTRIDE]
    uint32_t *arrive;   // [B*H_kv]
    uint32_t *status;
    KvMap kv;           // row addressing of k / v
    // context shard (null: the whole sequence): this shard holds global
    // tokens [id_off[b], id_off[b] + seq_lens[b]) of a sequence of
    // glob_len[b] tokens; sinks and window are taken in global positions and
    // the merged partials go to part_out [B*H_q][PSTRIDE] unnormalised
    const int32_t *glob_len;
    const int32_t *id_off;
    float *part_out;
};

// The row set of a range launch in the shard's own positions 0..N-1: rows
// [0, s1) and [w0, N).  Dense: every row.  Sinks and window: the first
// n_sink and the last `window` positions of the (global) sequence, as seen
// from the shard's offset.
__device__ __forceinline__ void shard_range(const RangeArgs &a, int b, int N, int &s1, int &w0) {
    if (a.dense) { s1 = N; w0 = N; return; }
    if (!a.glob_len) {
        s1 = min(a.n_sink, N);
        w0 = max(s1, N - a.window);
        return;
    }
    const long long off = a.id_off[b], Ng = a.glob_len[b];
    const long long sg = min((long long)a.n_sink, Ng), wg = max(sg, Ng - a.window);   // global [0, sg), [wg, Ng)
    s1 = (int)max(0LL, min((long long)N, sg - off));
    w0 = (int)max((long long)s1, min((long long)N, wg - off));
}

template <typename KT>
__global__ void __launch_bounds__(ATT_THREADS) range_attn_kernel(RangeArgs a) {
    __shared__ __align__(16) float qs[GMAX][D];
    __shared__ float S[GMAX][RCH];
    __shared__ float s_m[GMAX], s_l[GMAX], s_alpha[GMAX];
    __shared__ float O[GMAX][D];
    __shared__ int s_last;
    const int b = blockIdx.y / a.n_grp;
    const int g = a.grp[blockIdx.y % a.n_grp];
    const int G = a.G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t bg = (size_t)b * a.H_kv + g;
    const size_t bh0 = (size_t)b * a.H_q + (size_t)g * G;

    int N = a.seq_lens[b];
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

    for (int i = tid; i < G * D; i += blockDim.x)
        (&qs[0][0])[i] = a.q[bh0 * D + i] * a.scale_log2;
    for (int i = tid; i < GMAX * D; i += blockDim.x) (&O[0][0])[i] = 0.0f;
    if (tid < GMAX) { s_m[tid] = -INFINITY; s_l[tid] = 0.0f; }
    __syncthreads();

    const KT *kc = reinterpret_cast<const KT *>(a.k);
    const KT *vc = reinterpret_cast<const KT *>(a.v);
    float acc[GMAX][4];
#pragma unroll
    for (int h = 0; h < GMAX; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][i] = 0.0f;

    for (long long c = lo; c < hi; c += RCH) {
        // phase 1: one row per thread, logits for every head of the group
        {
            const long long j = c + tid;
            float s[GMAX];
#pragma unroll
            for (int h = 0; h < GMAX; ++h) s[h] = 0.0f;
            const long long kr_row = j < hi ? kv_row(a.kv, b, g, j < s1 ? j : w0 + (j - s1)) : -1LL;
            if (kr_row >= 0) {
                const KT *kr = kc + kr_row * D;
#pragma unroll 4
                for (int piece = 0; piece < D / 8; ++piece) {
                    float kx[8];
                    Row<KT>::load8(kr + piece * 8, kx);
#pragma unroll
                    for (int h = 0; h < GMAX; ++h) {
                        if (h < G) {
                            const float4 q0 = *reinterpret_cast<const float4 *>(&qs[h][piece * 8]);
                            const float4 q1 = *reinterpret_cast<const float4 *>(&qs[h][piece * 8 + 4]);
                            float t = s[h];
                            t = fmaf(q0.x, kx[0], t); t = fmaf(q0.y, kx[1], t);
                            t = fmaf(q0.z, kx[2], t); t = fmaf(q0.w, kx[3], t);
                            t = fmaf(q1.x, kx[4], t); t = fmaf(q1.y, kx[5], t);
                            t = fmaf(q1.z, kx[6], t); t = fmaf(q1.w, kx[7], t);
                            s[h] = t;
                        }
                    }
                }
            } else {
#pragma unroll
                for (int h = 0; h < GMAX; ++h) s[h] = -INFINITY;
            }
#pragma unroll
            for (int h = 0; h < GMAX; ++h)
                if (h < G) S[h][tid] = s[h];
        }
        __syncthreads();
        // phase 2: per-head running max and weights (warp h <-> head h)
        if (warp < G) {
            float mc = -INFINITY;
            for (int i = lane; i < RCH; i += 32) mc = fmaxf(mc, S[warp][i]);
            mc = warp_max(mc);
            const float mold = s_m[warp];
            const float mnew = fmaxf(mold, mc);
            float lc = 0.0f;
            if (mnew != -INFINITY) {
                for (int i = lane; i < RCH; i += 32) {
                    float e = exp2f(S[warp][i] - mnew);
                    S[warp][i] = e;
                    lc += e;
                }
            }
            lc = warp_sum(lc);
            if (lane == 0) {
                const float al = (mnew == -INFINITY) ? 1.0f : exp2f(mold - mnew);
                s_alpha[warp] = al;
                s_l[warp] = s_l[warp] * al + lc;
                s_m[warp] = mnew;
            }
        }
        __syncthreads();
        // phase 3: P.V, warp w owns rows w*32 .. w*32+31 of the sub-chunk
        {
#pragma unroll
            for (int h = 0; h < GMAX; ++h) {
                const float al = h < G ? s_alpha[h] : 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[h][i] *= al;
            }
            const long long rbase = c + warp * 32;
            const int nr = (int)max(0LL, min(32LL, hi - rbase));
#pragma unroll 8
            for (int i = 0; i < nr; ++i) {
                const long long j = rbase + i;
                const long long row = kv_row(a.kv, b, g, j < s1 ? j : w0 + (j - s1));
                float vx[4] = {0.f, 0.f, 0.f, 0.f};
                if (row >= 0) Row<KT>::load4(vc + row * D + lane * 4, vx);
#pragma unroll
                for (int h = 0; h < GMAX; ++h) {
                    if (h < G) {
                        const float pw = S[h][warp * 32 + i];
                        acc[h][0] = fmaf(pw, vx[0], acc[h][0]);
                        acc[h][1] = fmaf(pw, vx[1], acc[h][1]);
                        acc[h][2] = fmaf(pw, vx[2], acc[h][2]);
                        acc[h][3] = fmaf(pw, vx[3], acc[h][3]);
                    }
                }
            }
        }
        __syncthreads();
    }
    // reduce the warps' accumulators and publish this CTA's partial
#pragma unroll
    for (int h = 0; h < GMAX; ++h)
        if (h < G)
#pragma unroll
            for (int i = 0; i < 4; ++i) atomicAdd(&O[h][lane * 4 + i], acc[h][i]);
    __syncthreads();
    float *pp = a.part + (bg * a.slots + blockIdx.x) * GMAX * PSTRIDE;
    for (int i = tid; i < G * PSTRIDE; i += blockDim.x) {
        const int h = i / PSTRIDE, e = i % PSTRIDE;
        pp[i] = e == 0 ? s_m[h] : (e == 1 ? s_l[h] : (e < POFF ? 0.0f : O[h][e - POFF]));
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

// ---------------------------------------------------------------------------
// list attention
// ---------------------------------------------------------------------------
// The rows of a head may be attended in one pass (phase LIST_ALL) or in two
// (the prefix of the list that the collect pass wrote -- rows clearly above
// the boundary bin -- while the boundary is still being resolved, then the
// rest): LIST_FIRST writes partials only; LIST_REST adds the remaining rows
// and merges everything.  Partials live in per-head slots: the first pass
// uses slots [0, it_first), the second [it_first, it_first + it_rest).
// LIST_SPILL finishes the heads that the fused step's finalize handed over
// (their kept rows were too many for its cluster to attend quickly): flag
// spill[bh] = 2 (the rows from first[bh] on) or 3 (every row), finalize's
// partial in slot 0; heads without a flag are left alone.
enum ListPhase : int32_t { LIST_ALL = 0, LIST_FIRST = 1, LIST_REST = 2, LIST_SPILL = 3 };

struct ListArgs {
    int B, H_q, H_kv, G;
    long long N_max;
    const int32_t *seq_lens;
    int n_rq;                    // retrieval query heads per sequence
    int ret_h[MAX_RET_Q];
    float scale_log2;
    const float *q;
    const void *k;
    const void *v;
    const int32_t *lists;        // [B*H_q*N_max]
    const int32_t *counts;       // [B*H_q] kept rows per head (read by LIST_ALL and LIST_REST)
    // [B*H_q] at stride CNT_STRIDE: rows of the collect pass (LIST_FIRST,
    // LIST_REST), or null
    const int32_t *first;
    const uint32_t *spill;       // [B*H_q] hand-over flags (LIST_SPILL)
    const uint32_t *spill_any;   // nonzero when some head was handed over (LIST_SPILL)
    // context shard (null: whole sequences): list ids are global positions,
    // this shard's rows are id - id_off[b]; per-head merged partials go to
    // part_out [B*H_q][PSTRIDE] unnormalised (empty record for no rows)
    const int32_t *id_off;
    float *part_out;
    int phase;
    float *out;
    float *part;                 // [B*H_q][LIST_SLOTS][PSTRIDE]
    uint32_t *arrive;            // [B*H_q]
    uint32_t *status;
    KvMap kv;                    // row addressing of k / v
};

// Dynamic shared memory of list_attn_kernel: per head the item prefix, the
// rows of this pass, the first row and the first partial slot; per sequence
// its length.
__host__ __device__ constexpr size_t list_smem_bytes(int nh, int B) {
    return (size_t)(4 * nh + 1 + B) * sizeof(int);
}

// One item = a slice of one head's rows for this pass.  Warp w takes rows
// r0 + 8w .. r0 + 8w + 7, then every 64th: the 8 row ids come in one load and
// all 8 rows' K and V loads are issued before the first dot product.
constexpr int MAX_LIST_B = 1024;        // sequences per call
static_assert(65535 / MAX_GROUPS < MAX_LIST_B, "the argument checks must bound B below MAX_LIST_B");
template <typename KT>
__global__ void __launch_bounds__(ATT_THREADS, 2) list_attn_kernel(ListArgs a) {
    extern __shared__ int lsm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nh = a.B * a.n_rq;
    int *pre = lsm;                  // [nh + 1] item prefix
    int *s_rows = pre + nh + 1;      // [nh] rows of this pass (0 when invalid)
    int *s_row0 = s_rows + nh;       // [nh] first row of this pass in the head's list
    int *s_slot0 = s_row0 + nh;      // [nh] first partial slot of this pass
    int *s_len = s_slot0 + nh;       // [B] sequence lengths
    __shared__ int s_scan[ATT_THREADS / 32];
    __shared__ float wm[ATT_THREADS / 32], wl[ATT_THREADS / 32];
    __shared__ float wo[ATT_THREADS / 32][D];
    __shared__ int s_last;
    pdl_wait();
    pdl_trigger();
    // the hand-over pass has nothing to do unless finalize flagged a head
    if (a.phase == LIST_SPILL && __ldcg(a.spill_any) == 0u) return;

    // items per head -> exclusive prefix, built by every CTA: thread t owns
    // heads [t * per, t * per + per), then a block-wide exclusive scan
    {
        const int per = (nh + ATT_THREADS - 1) / ATT_THREADS;
        int loc = 0;
#pragma unroll 4
        for (int i = 0; i < per; ++i) {
            const int hi = tid * per + i;
            int it = 0;
            if (hi < nh) {
                const int b = hi / a.n_rq, h = a.ret_h[hi % a.n_rq];
                const size_t bh = (size_t)b * a.H_q + h;
                const int N = a.seq_lens[b];
                const bool okN = N >= 1 && (long long)N <= a.N_max;
                int rows = 0, row0 = 0, slot0 = 0;
                if (a.phase == LIST_ALL) {
                    const int cnt = __ldcg(a.counts + bh);
                    if (okN && cnt >= 1 && cnt <= N) { rows = cnt; it = list_items(cnt); }
                } else if (a.phase == LIST_FIRST) {
                    const int nf = (int)__ldcg(a.first + bh * CNT_STRIDE);
                    if (okN && nf >= 1 && nf <= N) { rows = nf; it = list_items(nf); }
                } else if (a.phase == LIST_SPILL) {
                    const uint32_t fl = __ldcg(a.spill + bh);
                    const int cnt = fl >= SPILL_FROM_FIRST ? __ldcg(a.counts + bh) : 0;
                    const int nf = fl == SPILL_FROM_FIRST ? __ldcg(a.first + bh * CNT_STRIDE) : 0;
                    if (okN && fl >= SPILL_FROM_FIRST && cnt >= 1 && cnt <= N && nf >= 0 && nf <= cnt) {
                        row0 = nf;
                        rows = cnt - nf;
                        slot0 = 1;                                   // finalize's partial
                        it = max(1, list_items(rows));
                    }
                } else {
                    const int cnt = __ldcg(a.counts + bh);
                    const int nf = __ldcg(a.first + bh * CNT_STRIDE);
                    if (okN && cnt >= 1 && cnt <= N && nf >= 0 && nf <= cnt) {
                        row0 = nf;
                        rows = cnt - nf;
                        slot0 = list_items(nf);
                        it = max(1, list_items(rows));       // at least one item: it merges the head
                    }
                }
                pre[hi] = it;
                s_rows[hi] = rows;
                s_row0[hi] = row0;
                s_slot0[hi] = slot0;
                s_len[b] = N;
            }
            loc += it;
        }
        int incl = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) s_scan[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int t = lane < ATT_THREADS / 32 ? s_scan[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += v;
            }
            if (lane < ATT_THREADS / 32) s_scan[lane] = t;
        }
        __syncthreads();
        int run = (warp > 0 ? s_scan[warp - 1] : 0) + incl - loc;
        for (int i = 0; i < per; ++i) {
            const int hi = tid * per + i;
            if (hi < nh) { const int it = pre[hi]; pre[hi] = run; run += it; }
        }
        if (tid == 0) pre[nh] = s_scan[ATT_THREADS / 32 - 1];
        __syncthreads();
    }
    const int total = pre[nh];
    // heads with nothing to attend over get zeros (and a status: invalid input)
    if (blockIdx.x == 0 && a.phase != LIST_FIRST) {
        for (int hi = warp; hi < nh; hi += ATT_THREADS / 32) {
            if (pre[hi + 1] != pre[hi]) continue;
            const int b = hi / a.n_rq, h = a.ret_h[hi % a.n_rq];
            if (a.phase == LIST_SPILL && __ldcg(a.spill + (size_t)b * a.H_q + h) < SPILL_FROM_FIRST) continue;
            if (a.part_out) {
                // a shard that keeps no row of this head: an empty partial
                float *r = a.part_out + ((size_t)b * a.H_q + h) * PSTRIDE;
                *reinterpret_cast<float4 *>(r + POFF + 4 * lane) = make_float4(0.f, 0.f, 0.f, 0.f);
                if (lane == 0) { r[0] = -INFINITY; r[1] = 0.0f; }
                continue;
            }
            float *o = a.out + ((size_t)b * a.H_q + h) * D + lane * 4;
            o[0] = o[1] = o[2] = o[3] = 0.0f;
            if (lane == 0) set_status(a.status, RTP_ERR_DEVICE_ARG);
        }
    }

    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        int lo_h = 0, hi_h = nh;
        while (hi_h - lo_h > 1) {
            const int mid = (lo_h + hi_h) >> 1;
            if (pre[mid] <= item) lo_h = mid; else hi_h = mid;
        }
        const int hix = lo_h;
        const int b = hix / a.n_rq, h = a.ret_h[hix % a.n_rq];
        const int g = h / a.G;
        const size_t bh = (size_t)b * a.H_q + h;
        const int rows = s_rows[hix];
        const int N = s_len[b];
        const int nit = pre[hix + 1] - pre[hix];
        const int sub = item - pre[hix];
        const int slot = s_slot0[hix] + sub;
        const int nrec = s_slot0[hix] + nit;       // partials the merge of this head reads
        const int per_item = (rows + nit - 1) / nit;
        const int r0 = s_row0[hix] + sub * per_item;
        const int r1 = s_row0[hix] + min(rows, sub * per_item + per_item);

        const KT *kc = reinterpret_cast<const KT *>(a.k);
        const KT *vc = reinterpret_cast<const KT *>(a.v);
        const int32_t *lst = a.lists + bh * a.N_max;
        const int id0 = a.id_off ? a.id_off[b] : 0;
        if constexpr (std::is_same<KT, __nv_bfloat16>::value) {
            // bf16 rows: a half-warp per row (lane l holds dims 8 (l % 16) ..
            // + 7, one 16-byte load per row and tensor), 16 rows per warp per
            // pass with all their loads in flight; the next pass's row ids
            // are loaded while this pass computes.  Each half keeps its own
            // running (m, l, o), merged with the other half's at the end.
            const int half = lane >> 4, hl = lane & 15;
            float qx[8];
            {
                const float4 qa = *reinterpret_cast<const float4 *>(a.q + bh * D + hl * 8);
                const float4 qb = *reinterpret_cast<const float4 *>(a.q + bh * D + hl * 8 + 4);
                qx[0] = qa.x * a.scale_log2; qx[1] = qa.y * a.scale_log2; qx[2] = qa.z * a.scale_log2;
                qx[3] = qa.w * a.scale_log2; qx[4] = qb.x * a.scale_log2; qx[5] = qb.y * a.scale_log2;
                qx[6] = qb.z * a.scale_log2; qx[7] = qb.w * a.scale_log2;
            }
            float m = -INFINITY, l = 0.0f, o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = 0.0f;
            constexpr int U2 = 16;                  // rows per warp per pass
            constexpr int STEP = (ATT_THREADS / 32) * U2;
            const uint4 *kc4 = reinterpret_cast<const uint4 *>(kc);
            const uint4 *vc4 = reinterpret_cast<const uint4 *>(vc);
            int rb = r0 + warp * U2;
            int nid = -1;                           // lanes 0-15: the ids of the pass at rb
            if (lane < U2 && rb + lane < r1) nid = __ldcg(lst + rb + lane) - id0;
            for (; rb < r1; rb += STEP) {
                const int myid = nid;
                nid = -1;
                if (lane < U2 && rb + STEP + lane < r1) nid = __ldcg(lst + rb + STEP + lane) - id0;
                const long long myrow = myid >= 0 && myid < N ? kv_row(a.kv, b, g, myid) : -1LL;
                // row u of this half: pass row 2 u + half
                uint4 kw[U2 / 2], vw[U2 / 2];
                bool ok[U2 / 2];
#pragma unroll
                for (int u = 0; u < U2 / 2; ++u) {
                    const int j = 2 * u + half;
                    const long long r = __shfl_sync(0xffffffffu, myrow, j);
                    ok[u] = rb + j < r1 && r >= 0;
                    if (ok[u]) {
                        kw[u] = __ldcg(kc4 + (r * D) / 8 + hl);
                        vw[u] = __ldcg(vc4 + (r * D) / 8 + hl);
                    } else {
                        kw[u] = vw[u] = make_uint4(0u, 0u, 0u, 0u);
                    }
                    if (rb + j < r1 && !ok[u] && hl == 0) set_status(a.status, RTP_ERR_DEVICE_ARG);
                }
                float sc[U2 / 2];
                float mb = -INFINITY;
#pragma unroll
                for (int u = 0; u < U2 / 2; ++u) {
                    const uint32_t w4[4] = {kw[u].x, kw[u].y, kw[u].z, kw[u].w};
                    float s = 0.0f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        s = fmaf(qx[2 * i], bf16_lo(w4[i]), s);
                        s = fmaf(qx[2 * i + 1], bf16_hi(w4[i]), s);
                    }
#pragma unroll
                    for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                    sc[u] = ok[u] ? s : -INFINITY;
                    mb = fmaxf(mb, sc[u]);
                }
                // (a half with no row yet skips the update; no shuffle inside,
                // so the halves may differ here)
                const float mn = fmaxf(m, mb);
                if (mn != -INFINITY) {
                    const float al = exp2f(m - mn);
                    l *= al;
#pragma unroll
                    for (int i = 0; i < 8; ++i) o[i] *= al;
#pragma unroll
                    for (int u = 0; u < U2 / 2; ++u) {
                        const float pw = exp2f(sc[u] - mn);
                        l += pw;
                        const uint32_t w4[4] = {vw[u].x, vw[u].y, vw[u].z, vw[u].w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            o[2 * i] = fmaf(pw, bf16_lo(w4[i]), o[2 * i]);
                            o[2 * i + 1] = fmaf(pw, bf16_hi(w4[i]), o[2 * i + 1]);
                        }
                    }
                    m = mn;
                }
            }
            // the two halves' partials into lanes 0-15 (dims 8 hl .. 8 hl + 7)
            {
                const float m2 = __shfl_xor_sync(0xffffffffu, m, 16);
                const float l2 = __shfl_xor_sync(0xffffffffu, l, 16);
                const float M = fmaxf(m, m2);
                const float w1 = m == -INFINITY ? 0.0f : exp2f(m - M);
                const float w2 = m2 == -INFINITY ? 0.0f : exp2f(m2 - M);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float o2 = __shfl_xor_sync(0xffffffffu, o[i], 16);
                    o[i] = o[i] * w1 + o2 * w2;
                }
                l = l * w1 + l2 * w2;
                m = M;
            }
            if (lane == 0) { wm[warp] = m; wl[warp] = l; }
            if (half == 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) wo[warp][hl * 8 + i] = o[i];
            }
        } else {
        const float4 q4 = *reinterpret_cast<const float4 *>(a.q + bh * D + lane * 4);
        const float qx[4] = {q4.x * a.scale_log2, q4.y * a.scale_log2, q4.z * a.scale_log2,
                             q4.w * a.scale_log2};
        float m = -INFINITY, l = 0.0f, o[4] = {0.f, 0.f, 0.f, 0.f};
        constexpr int U = 8;       // rows per warp per pass: all their K/V loads in flight
        for (int rb = r0 + warp * U; rb < r1; rb += (ATT_THREADS / 32) * U) {
            int myid = -1;
            if (lane < U && rb + lane < r1) myid = __ldcg(lst + rb + lane) - id0;
            // lanes 0-7: the cache row of their token (-1: none or invalid)
            const long long myrow = myid >= 0 && myid < N ? kv_row(a.kv, b, g, myid) : -1LL;
            float kx[U][4], vx[U][4];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const long long r = __shfl_sync(0xffffffffu, myrow, u);
                ok[u] = rb + u < r1 && r >= 0;
                if (ok[u]) {
                    Row<KT>::load4(kc + r * D + lane * 4, kx[u]);
                    Row<KT>::load4(vc + r * D + lane * 4, vx[u]);
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) kx[u][i] = vx[u][i] = 0.0f;
                }
                if (rb + u < r1 && !ok[u] && lane == 0) set_status(a.status, RTP_ERR_DEVICE_ARG);
            }
            float sc[U];
            float mb = -INFINITY;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                float s = qx[0] * kx[u][0];
                s = fmaf(qx[1], kx[u][1], s);
                s = fmaf(qx[2], kx[u][2], s);
                s = fmaf(qx[3], kx[u][3], s);
                s = warp_sum(s);
                sc[u] = ok[u] ? s : -INFINITY;
                mb = fmaxf(mb, sc[u]);
            }
            const float mn = fmaxf(m, mb);
            if (mn == -INFINITY) continue;
            const float al = exp2f(m - mn);
            l *= al;
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] *= al;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const float pw = exp2f(sc[u] - mn);
                l += pw;
#pragma unroll
                for (int i = 0; i < 4; ++i) o[i] = fmaf(pw, vx[u][i], o[i]);
            }
            m = mn;
        }
        // merge warps
        if (lane == 0) { wm[warp] = m; wl[warp] = l; }
#pragma unroll
        for (int i = 0; i < 4; ++i) wo[warp][lane * 4 + i] = o[i];
        }
        __syncthreads();
        float *hp = a.part + bh * (size_t)LIST_SLOTS * PSTRIDE;
        float *pp = hp + (size_t)slot * PSTRIDE;
        // a head attended by this one item only: normalise and write directly
        const bool direct = a.phase != LIST_FIRST && nrec == 1 && !a.part_out;
        if (tid < D) {
            float M = -INFINITY;
            for (int w = 0; w < ATT_THREADS / 32; ++w) M = fmaxf(M, wm[w]);
            float ls = 0.0f, os = 0.0f;
            if (M != -INFINITY) {
                for (int w = 0; w < ATT_THREADS / 32; ++w) {
                    const float wg = wm[w] == -INFINITY ? 0.0f : exp2f(wm[w] - M);
                    ls = fmaf(wl[w], wg, ls);
                    os = fmaf(wo[w][tid], wg, os);
                }
            }
            if (direct) {
                a.out[bh * D + tid] = os * (ls > 0.0f ? 1.0f / ls : 0.0f);
            } else {
                pp[POFF + tid] = os;
                if (tid == 0) { pp[0] = M; pp[1] = ls; }
            }
        }
        if (direct || a.phase == LIST_FIRST) {
            __syncthreads();
            continue;
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) s_last = atomicAdd(&a.arrive[bh], 1u) == (unsigned)(nit - 1);
        __syncthreads();
        if (s_last) {
            __threadfence();
            merge_partials(hp, nrec, PSTRIDE, 1, a.out + bh * D, a.part_out ? a.part_out + bh * PSTRIDE : nullptr);
            if (tid == 0) a.arrive[bh] = 0;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Context shards: the P shards' partial records of each head (parts
// [P][n_heads][PSTRIDE], m and l in log2 units) merged into the output.
// grid = (n_heads), 32 threads.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) merge_shards_kernel(const float *parts, int P, int nh, float *out) {
    const int h = blockIdx.x;
    merge_partials(parts + (size_t)h * PSTRIDE, P, nh * PSTRIDE, 1, out + (size_t)h * D);
}

// ---------------------------------------------------------------------------
// Forced local rows for retrieval heads: each retrieval head's kept list
// S_h (the first counts[bh] entries) becomes S_h united with the sink and
// window rows L of the sequence (the local heads' set).  One CTA per
// retrieval head: a bitmap over L's rows in shared memory marks the kept
// ids that fall in L, then the unmarked rows of L are appended.
// grid = (B * n_rq), FR_THREADS threads, dynamic smem = fr_smem_bytes(L_max).
// ---------------------------------------------------------------------------
constexpr int FR_THREADS = 256;
constexpr int FR_MAX_ROWS = 48 * 1024 * 8;       // |L| covered by the bitmap (48 KB)
__host__ __device__ constexpr size_t fr_smem_bytes(long long rows) {
    return (size_t)((rows + 31) / 32) * 4;
}
struct ForceArgs {
    int B, H_q, G;
    long long N_max;
    const int32_t *seq_lens;
    int n_rq;
    int ret_h[MAX_RET_Q];
    int window, n_sink;
    int32_t *lists;              // [B*H_q*N_max]
    int32_t *counts;             // [B*H_q]
    uint32_t *status;
};
__global__ void __launch_bounds__(FR_THREADS) force_rows_kernel(ForceArgs a) {
    extern __shared__ uint32_t fbm[];
    __shared__ unsigned s_add;
    pdl_wait();
    pdl_trigger();
    const int hi = blockIdx.x;
    const int b = hi / a.n_rq, h = a.ret_h[hi % a.n_rq];
    const size_t bh = (size_t)b * a.H_q + h;
    const int N = a.seq_lens[b];
    const int cnt = __ldcg(a.counts + bh);
    if (N < 1 || (long long)N > a.N_max || cnt < 0 || cnt > N) return;     // reported by the step's kernels
    const int s1 = min(a.n_sink, N);
    const int w0 = max(s1, N - a.window);
    const int nl = s1 + (N - w0);                                          // |L|
    const int words = (nl + 31) / 32;
    for (int i = threadIdx.x; i < words; i += blockDim.x) fbm[i] = 0u;
    if (threadIdx.x == 0) s_add = 0u;
    __syncthreads();
    int32_t *lst = a.lists + bh * a.N_max;
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
        const int t = __ldcg(lst + i);
        const int li = t < s1 ? t : (t >= w0 && t < N ? s1 + (t - w0) : -1);
        if (li >= 0) atomicOr(&fbm[li >> 5], 1u << (li & 31));
    }
    __syncthreads();
    for (int li = threadIdx.x; li < nl; li += blockDim.x) {
        if (fbm[li >> 5] & (1u << (li & 31))) continue;
        const int t = li < s1 ? li : w0 + (li - s1);
        lst[cnt + atomicAdd(&s_add, 1u)] = t;
    }
    __syncthreads();
    if (threadIdx.x == 0) a.counts[bh] = cnt + (int)s_add;
}

}  // namespace rtp
