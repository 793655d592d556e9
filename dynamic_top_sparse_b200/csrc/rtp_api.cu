// C ABI of librtp.so: argument checks, workspace layout and kernel launches
// for the RTPurbo sparse decode step.  Contract: include/rtp.h.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <functional>

#include "rtp.h"
#include "rtp_common.cuh"
#include "rtp_select.cuh"
#include "rtp_attend.cuh"
#include "rtp_append.cuh"
#include "rtp_gqa_mma.cuh"
#include "rtp_prefill.cuh"

using namespace rtp;

namespace {

constexpr int RANGE_SPLIT_MAX = 256;
// context above which the fused step adds the hand-over pass after finalize
constexpr long long SPILL_MIN_CTX = 256 * 1024;
// SMs given to the local heads while the selection runs beside them
constexpr int LOCAL_SMS = 12;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace regions, in the order ops need them (each op needs a prefix).
struct Layout {
    size_t status, arrive_range, arrive_list, cand_cnt, list_cnt, hist;
    size_t ctrl_end;
    size_t res, qidx, counts;
    size_t end_scores;      // append / index_scores need up to here
    size_t part_range;
    size_t end_range;       // local / dense
    size_t part_list;
    size_t end_list;        // sparse decode
    size_t tilebin, lists, cands, part_sel, ovf, theta;
    size_t total;           // topp_select / decode_step
};

constexpr int SCAN_CTAS_MAX = 1024;

int num_sms();

Layout make_layout(const rtp_dims *d) {
    Layout L{};
    const size_t BHq = (size_t)d->B * d->H_q, BHkv = (size_t)d->B * d->H_kv;
    const size_t ntile = (size_t)((d->N_max + TILE - 1) / TILE);
    size_t o = 0;
    L.status = o; o += 256;
    L.arrive_range = o; o = align_up(o + BHkv * 4, 256);
    L.arrive_list = o; o = align_up(o + BHq * 4, 256);
    L.cand_cnt = o; o = align_up(o + BHq * CNT_STRIDE * 4, 256);
    L.list_cnt = o; o = align_up(o + BHq * CNT_STRIDE * 4, 256);
    L.hist = o; o = align_up(o + BHq * HSTRIDE * 8, 256);
    L.ctrl_end = o;
    L.res = o; o = align_up(o + BHq * sizeof(Resolve), 256);
    L.qidx = o; o = align_up(o + BHq * R * 4, 256);
    L.counts = o; o = align_up(o + BHq * 4, 256);
    L.end_scores = o;
    L.part_range = o; o = align_up(o + BHkv * RANGE_SPLIT_MAX * GMAX * PSTRIDE * 4, 256);
    L.end_range = o;
    L.part_list = o; o = align_up(o + BHq * LIST_SLOTS * PSTRIDE * 4, 256);
    L.end_list = o;
    L.tilebin = o; o = align_up(o + BHkv * ntile * GMAX * 2, 256);
    L.lists = o; o = align_up(o + BHq * (size_t)d->N_max * 4, 256);
    L.cands = o; o = align_up(o + BHq * (size_t)d->N_max * 8, 256);
    // one record per collect CTA and head slot: the bf16 selection grid has
    // max(1, SMs / groups) CTAs per (b, g), at most max(SMs, B * H_kv) in all,
    // and the collect grid twice as many
    L.part_sel = o; o = align_up(o + 2 * std::max((size_t)num_sms(), BHkv) * GMAX * PSTRIDE * 4, 256);
    L.ovf = o; o = align_up(o + BHq * 4, 256);
    L.theta = o; o = align_up(o + BHq * 8, 256);
    L.total = o;
    return L;
}

size_t op_bytes(const Layout &L, int op) {
    switch (op) {
        case RTP_OP_APPEND_INDEX_KEYS: return L.ctrl_end;
        case RTP_OP_INDEX_SCORES: return L.end_scores;
        case RTP_OP_LOCAL_DECODE:
        case RTP_OP_DENSE_DECODE: return L.end_range;
        case RTP_OP_SPARSE_DECODE: return L.end_list;
        case RTP_OP_TOPP_SELECT:
        case RTP_OP_DECODE_STEP: return L.total;
        case RTP_OP_PREFILL: return L.status + 256;
        default: return 0;
    }
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
bool aligned4(const void *p) { return ((uintptr_t)p & 3u) == 0; }

int check_dims(const rtp_dims *d) {
    if (!d) return RTP_ERR_INVALID_ARG;
    if (d->B < 1 || d->H_q < 1 || d->H_kv < 1 || d->N_max < 1 || !d->seq_lens)
        return RTP_ERR_INVALID_ARG;
    if (d->N_max > 0x7fffffffLL - 64) return RTP_ERR_INVALID_ARG;
    if (d->H_q % d->H_kv != 0) return RTP_ERR_INVALID_ARG;
    if (d->d != D || d->r != R) return RTP_ERR_UNSUPPORTED;
    if (d->H_q / d->H_kv > GMAX) return RTP_ERR_UNSUPPORTED;
    if (d->H_kv > MAX_GROUPS) return RTP_ERR_UNSUPPORTED;
    if ((d->kv_dtype != RTP_F32 && d->kv_dtype != RTP_BF16) ||
        (d->idx_dtype != RTP_F32 && d->idx_dtype != RTP_BF16))
        return RTP_ERR_UNSUPPORTED;
    if ((size_t)d->B * d->H_q > MAX_LIST_HEADS) return RTP_ERR_UNSUPPORTED;
    if (d->B > 65535 / MAX_GROUPS) return RTP_ERR_UNSUPPORTED;   // grid.y = B * groups
    return RTP_OK;
}

int check_ws(const rtp_dims *d, void *ws, size_t ws_bytes, int op) {
    if (!ws || ((uintptr_t)ws & 255u)) return RTP_ERR_WORKSPACE;
    if (ws_bytes < op_bytes(make_layout(d), op)) return RTP_ERR_WORKSPACE;
    return RTP_OK;
}

int check_head_class(const rtp_dims *d, const uint8_t *hc) {
    if (!hc) return RTP_ERR_INVALID_ARG;
    for (int g = 0; g < d->H_kv; ++g)
        if (hc[g] != RTP_HEAD_LOCAL && hc[g] != RTP_HEAD_RETRIEVAL) return RTP_ERR_INVALID_ARG;
    return RTP_OK;
}

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) return 148;
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Launch helper: records profiling events around a launch when asked.
struct Launcher {
    cudaStream_t st;
    rtp_prof *prof;
    // Launch the next kernels with programmatic stream serialization: they
    // may start while the previous kernel of the stream drains, and wait for
    // it on the device (pdl_wait).  Only for kernels that call pdl_wait
    // before touching global memory.
    bool pdl = false;
    // Launch the next kernels in thread-block clusters of this many CTAs
    // along x (0: no clusters).
    unsigned cluster_x = 0;
    // Inside stream capture an event becomes a timestamp node of the graph
    // only when recorded as external.
    cudaError_t record(void *ev, bool capturing) {
        return capturing ? cudaEventRecordWithFlags((cudaEvent_t)ev, st, cudaEventRecordExternal)
                         : cudaEventRecord((cudaEvent_t)ev, st);
    }
    template <typename K, typename... Args>
    int run(const char *name, K kernel, dim3 grid, dim3 block, Args... args) {
        return run_smem(name, kernel, grid, block, 0, args...);
    }
    template <typename K, typename... Args>
    int run_smem(const char *name, K kernel, dim3 grid, dim3 block, size_t smem, Args... args) {
        if (grid.x == 0 || grid.y == 0 || grid.z == 0) return RTP_OK;
        int slot = -1;
        bool capturing = false;
        if (prof && prof->count < prof->capacity && (!prof->filter || std::strstr(name, prof->filter))) {
            slot = prof->count++;
            prof->name[slot] = name;
            cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
            if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return RTP_ERR_CUDA;
            capturing = cs == cudaStreamCaptureStatusActive;
            if (record(prof->ev_start[slot], capturing) != cudaSuccess) return RTP_ERR_CUDA;
        }
        if (pdl || cluster_x) {
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = grid;
            cfg.blockDim = block;
            cfg.dynamicSmemBytes = smem;
            cfg.stream = st;
            cudaLaunchAttribute at[2];
            unsigned n = 0;
            if (pdl) {
                at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
                at[n].val.programmaticStreamSerializationAllowed = 1;
                ++n;
            }
            if (cluster_x) {
                at[n].id = cudaLaunchAttributeClusterDimension;
                at[n].val.clusterDim.x = cluster_x;
                at[n].val.clusterDim.y = 1;
                at[n].val.clusterDim.z = 1;
                ++n;
            }
            cfg.attrs = at;
            cfg.numAttrs = n;
            if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) return RTP_ERR_CUDA;
        } else {
            kernel<<<grid, block, smem, st>>>(args...);
        }
        if (cudaGetLastError() != cudaSuccess) return RTP_ERR_CUDA;
        if (slot >= 0 && record(prof->ev_stop[slot], capturing) != cudaSuccess) return RTP_ERR_CUDA;
        return RTP_OK;
    }
};

#define RTP_TRY(x)                      \
    do {                                \
        int _e = (x);                   \
        if (_e != RTP_OK) return _e;    \
    } while (0)

float scale_or_default(float s) { return s > 0.0f ? s : 1.0f / std::sqrt((float)D); }

// Paged K/V option: checked on the host, then turned into the kernels' row map.
int check_kv(const rtp_dims *d, const rtp_opts *opts) {
    const rtp_kv_pages *pg = opts ? opts->kv_pages : nullptr;
    if (!pg) return RTP_OK;
    if (!pg->block_table || ((uintptr_t)pg->block_table & 3u)) return RTP_ERR_INVALID_ARG;
    const int ps = pg->page_size;
    if (ps < 16 || ps > (1 << 20) || (ps & (ps - 1))) return RTP_ERR_INVALID_ARG;
    if (pg->num_pages < 1 || pg->max_pages < 1) return RTP_ERR_INVALID_ARG;
    if ((long long)pg->max_pages * ps < d->N_max) return RTP_ERR_INVALID_ARG;
    return RTP_OK;
}
KvMap make_kv(const rtp_dims *d, const rtp_opts *opts, void *status) {
    KvMap m{};
    m.H_kv = d->H_kv;
    m.N_max = d->N_max;
    m.status = static_cast<uint32_t *>(status);
    const rtp_kv_pages *pg = opts ? opts->kv_pages : nullptr;
    if (pg) {
        m.table = pg->block_table;
        int sh = 0;
        while ((1 << sh) < pg->page_size) ++sh;
        m.page_shift = sh;
        m.max_pages = pg->max_pages;
        m.num_pages = pg->num_pages;
    }
    return m;
}

// ----------------------------------------------------------------- selection
struct SelPlan {
    SelArgs a;
    SelWs w;
};

// CTAs per (b, g) for the scan: two 512-thread CTAs per SM over the whole
// GPU (one wave), each on a contiguous, tile-aligned token range.
void plan_chunks(SelArgs &a, long long N_max) {
    const long long groups = (long long)a.B * std::max(a.n_ret, 1);
    long long ctas = std::max(1LL, 2LL * num_sms() / groups);
    const long long tiles = (N_max + TILE - 1) / TILE;
    ctas = std::max(1LL, std::min({ctas, tiles, (long long)SCAN_CTAS_MAX}));
    // at most MAX_CTA_TOKENS tokens per CTA (its 64-bit wide-bin sums cannot wrap)
    ctas = std::max(ctas, (tiles * TILE + MAX_CTA_TOKENS - 1) / MAX_CTA_TOKENS);
    long long chunk = (tiles + ctas - 1) / ctas * TILE;
    ctas = (N_max + chunk - 1) / chunk;
    a.ctas = (int)ctas;
    a.chunk = chunk;
}

SelPlan make_sel(const rtp_dims *d, const uint8_t *hc, char *ws, const Layout &L) {
    SelPlan s{};
    SelArgs &a = s.a;
    a.B = d->B; a.H_q = d->H_q; a.H_kv = d->H_kv; a.G = d->H_q / d->H_kv;
    a.N_max = d->N_max;
    a.ntile = (int)((d->N_max + TILE - 1) / TILE);
    a.seq_lens = d->seq_lens;
    a.n_ret = 0;
    for (int g = 0; g < d->H_kv; ++g)
        if (hc[g] == RTP_HEAD_RETRIEVAL) a.ret_g[a.n_ret++] = g;
    plan_chunks(a, d->N_max);
    SelWs &w = s.w;
    w.status = reinterpret_cast<uint32_t *>(ws + L.status);
    w.cand_cnt = reinterpret_cast<uint32_t *>(ws + L.cand_cnt);
    w.list_cnt = reinterpret_cast<uint32_t *>(ws + L.list_cnt);
    w.hist = reinterpret_cast<double *>(ws + L.hist);
    w.res = reinterpret_cast<Resolve *>(ws + L.res);
    w.tilebin = reinterpret_cast<uint16_t *>(ws + L.tilebin);
    w.cands = reinterpret_cast<unsigned long long *>(ws + L.cands);
    w.qidx = reinterpret_cast<float *>(ws + L.qidx);
    return s;
}

// Work queued right after the collect kernel (in a decode step: the
// attention over the rows the collect pass kept, forked onto a side stream
// so that it overlaps finalize).
using AfterCollect = std::function<int()>;

// scan + collect + finalize over a logit source
template <typename Src>
int launch_select(Launcher &ln, const rtp_dims *d, const SelPlan &s, const AfterCollect &after_collect = {}) {
    const dim3 grid((unsigned)s.a.ctas, (unsigned)(d->B * s.a.n_ret));
    RTP_TRY(ln.run("hist", scan_kernel<Src>, grid, dim3(SCAN_THREADS), s.a, s.w));
    RTP_TRY(ln.run("collect", collect_kernel<Src>, grid, dim3(COL_THREADS), s.a, s.w));
    if (after_collect) RTP_TRY(after_collect());
    RTP_TRY(ln.run("finalize", finalize_kernel<false>, dim3(1u, (unsigned)(d->B * s.a.n_ret * s.a.G)),
                   dim3(FIN_THREADS), s.a, s.w));
    return RTP_OK;
}

// reserve_sms: SMs left free for work running beside the selection (the
// local heads of a decode step), so that neither waits for the other.
// which kernels of the TMA selection chain to launch (a context shard runs
// them one at a time, with exchanges in between)
enum SelPhases : int { SEL_SCAN = 1, SEL_COLLECT = 2, SEL_FINALIZE = 4, SEL_ALL = 7 };

int select_from_index(Launcher &ln, const rtp_dims *d, SelPlan s, int reserve_sms = 0,
                      const AfterCollect &after_collect = {}, int phases = SEL_ALL) {
    if (d->idx_dtype != RTP_BF16) return launch_select<SrcSimt<float>>(ln, d, s, after_collect);
    // bf16 index keys: the TMA-ring scan, one CTA per SM over all groups
    static int attr_set[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RTP_ERR_CUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(scan_tma_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, TC_SMEM) !=
                cudaSuccess ||
            cudaFuncSetAttribute(scan_tma_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, TC_SMEM) !=
                cudaSuccess ||
            cudaFuncSetAttribute(collect_mma_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, CL_SMEM) !=
                cudaSuccess ||
            cudaFuncSetAttribute(collect_mma_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, CL_SMEM) !=
                cudaSuccess)
            return RTP_ERR_CUDA;
        attr_set[dev] = 1;
    }
    const long long groups = (long long)d->B * s.a.n_ret;
    const long long tiles = (d->N_max + TILE - 1) / TILE;
    const long long sms = std::max(1LL, (long long)num_sms() - std::max(0, reserve_sms));
    long long ctas = std::max(1LL, std::min(sms / std::max(groups, 1LL), tiles));
    ctas = std::max(ctas, (tiles * TILE + MAX_CTA_TOKENS - 1) / MAX_CTA_TOKENS);
    s.a.chunk = (tiles + ctas - 1) / ctas * TILE;
    s.a.ctas = (int)((d->N_max + s.a.chunk - 1) / s.a.chunk);
    // collect: the groups in pairs, one CTA per SM, the pair's tiles dealt
    // round-robin over its CTAs
    const long long pairs = (groups + PAIR - 1) / PAIR;
    s.a.cl_ctas = (int)std::max(1LL, std::min(sms / pairs, PAIR * tiles));
    const dim3 grid((unsigned)s.a.ctas, (unsigned)groups);
    const dim3 cl_grid((unsigned)s.a.cl_ctas, (unsigned)pairs);
    // scan, collect and finalize wait on the device for their predecessor
    // (programmatic dependent launch), so each one's launch overlaps the
    // previous kernel's tail
    const bool pdl0 = ln.pdl;
    ln.pdl = phases == SEL_ALL;
    int rc = RTP_OK;
    if (phases & SEL_SCAN)
        rc = s.a.topk > 0 ? ln.run_smem("hist", scan_tma_kernel<true>, grid, dim3(TC_THREADS), TC_SMEM, s.a, s.w)
                          : ln.run_smem("hist", scan_tma_kernel<false>, grid, dim3(TC_THREADS), TC_SMEM, s.a, s.w);
    const bool paged = s.a.kv.table != nullptr;
    if (rc == RTP_OK && (phases & SEL_COLLECT))
        rc = paged ? ln.run_smem("collect", collect_mma_kernel<true>, cl_grid, dim3(CL_THREADS), CL_SMEM, s.a, s.w)
                   : ln.run_smem("collect", collect_mma_kernel<false>, cl_grid, dim3(CL_THREADS), CL_SMEM, s.a, s.w);
    if (rc == RTP_OK && after_collect) rc = after_collect();
    if (rc == RTP_OK && (phases & SEL_FINALIZE)) {
        // with the fused attention the CTAs of a head form a cluster
        const unsigned K = s.a.q_rope ? (unsigned)FIN_CLUSTER : 1u;
        ln.cluster_x = K > 1 ? K : 0u;
        const dim3 fgrid(K, (unsigned)(d->B * s.a.n_ret * s.a.G));
        rc = paged ? ln.run("finalize", finalize_kernel<true>, fgrid, dim3(FIN_THREADS), s.a, s.w)
                   : ln.run("finalize", finalize_kernel<false>, fgrid, dim3(FIN_THREADS),
                    s.a, s.w);
        ln.cluster_x = 0;
    }
    ln.pdl = pdl0;
    return rc;
}

unsigned long long ret_mask(const rtp_dims *d, const uint8_t *hc) {
    unsigned long long m = 0;
    for (int g = 0; g < d->H_kv; ++g)
        if (hc[g] == RTP_HEAD_RETRIEVAL) m |= 1ull << g;
    return m;
}

// Side stream per device and host thread, for work that overlaps the
// retrieval pipeline (local heads).  Created on first use.
struct Side {
    cudaStream_t st = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};

int side_stream(Side *&out, int slot = 0) {
    static thread_local Side sides[64][2];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || slot < 0 || slot > 1) return RTP_ERR_CUDA;
    Side &sd = sides[dev][slot];
    if (!sd.st) {
        if (cudaStreamCreateWithFlags(&sd.st, cudaStreamNonBlocking) != cudaSuccess) return RTP_ERR_CUDA;
        if (cudaEventCreateWithFlags(&sd.fork, cudaEventDisableTiming) != cudaSuccess) return RTP_ERR_CUDA;
        if (cudaEventCreateWithFlags(&sd.join, cudaEventDisableTiming) != cudaSuccess) return RTP_ERR_CUDA;
    }
    out = &sd;
    return RTP_OK;
}

// ----------------------------------------------------------------- attention
int launch_range(Launcher &ln, const rtp_dims *d, const float *q, const void *k, const void *v,
                 const uint8_t *hc, int want_class, bool dense, int window, int n_sink, float *out,
                 char *ws, const Layout &L, float attn_scale, int max_ctas = 0, const KvMap *kv = nullptr,
                 const int32_t *glob_len = nullptr, const int32_t *id_off = nullptr, float *part_out = nullptr) {
    RangeArgs a{};
    a.B = d->B; a.H_q = d->H_q; a.H_kv = d->H_kv; a.G = d->H_q / d->H_kv;
    a.N_max = d->N_max; a.seq_lens = d->seq_lens;
    a.n_grp = 0;
    for (int g = 0; g < d->H_kv; ++g)
        if (want_class < 0 || hc[g] == want_class) a.grp[a.n_grp++] = g;
    if (a.n_grp == 0) return RTP_OK;
    a.dense = dense ? 1 : 0;
    a.window = window; a.n_sink = n_sink;
    const long long Lmax = dense ? d->N_max : std::min<long long>(d->N_max, (long long)window + n_sink);
    // at least two 16-row tiles per warp; one CTA per SM
    const int rows_min = 2 * GQ_WARPS * GQ_TILE;
    const int per_sm = 1;
    const long long chunks = (Lmax + rows_min - 1) / rows_min;
    // whole waves: a CTA count just above the SM count would leave a second
    // wave of a few CTAs running alone
    long long want = std::max(1LL, (long long)per_sm * num_sms() / ((long long)d->B * a.n_grp));
    if (max_ctas > 0) want = std::max(1LL, (long long)max_ctas / ((long long)d->B * a.n_grp));
    a.n_split = (int)std::max(1LL, std::min(want, std::min(chunks, (long long)RANGE_SPLIT_MAX)));
    // Slots are indexed by (b, g) at a fixed stride, not by this launch's
    // split count: the local and the dense retrieval launches of one step run
    // at the same time on two streams with different n_split.
    a.slots = RANGE_SPLIT_MAX;
    a.scale_log2 = attn_scale * L2E;
    a.q = q; a.k = k; a.v = v; a.out = out;
    a.part = reinterpret_cast<float *>(ws + L.part_range);
    a.arrive = reinterpret_cast<uint32_t *>(ws + L.arrive_range);
    a.status = reinterpret_cast<uint32_t *>(ws + L.status);
    a.kv = kv ? *kv : make_kv(d, nullptr, a.status);
    a.glob_len = glob_len;
    a.id_off = id_off;
    a.part_out = part_out;
    const dim3 grid((unsigned)a.n_split, (unsigned)(d->B * a.n_grp));
    const char *name = dense ? "dense_attn" : "local_attn";
    if (d->kv_dtype == RTP_BF16)
        return a.kv.table ? ln.run(name, gqa_mma_attn_kernel<true>, grid, dim3(GQ_THREADS), a)
                          : ln.run(name, gqa_mma_attn_kernel<false>, grid, dim3(GQ_THREADS), a);
    return ln.run(name, range_attn_kernel<float>, grid, dim3(ATT_THREADS), a);
}

int launch_list(Launcher &ln, const rtp_dims *d, const float *q, const void *k, const void *v,
                const int32_t *lists, const int32_t *counts, const uint8_t *hc, float *out,
                char *ws, const Layout &L, float attn_scale, int phase = LIST_ALL,
                const int32_t *first = nullptr, const uint32_t *spill = nullptr, const KvMap *kv = nullptr,
                const int32_t *id_off = nullptr, float *part_out = nullptr) {
    static int attr_set[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RTP_ERR_CUDA;
    if (!attr_set[dev]) {
        const int mx = (int)list_smem_bytes(MAX_LIST_HEADS, MAX_LIST_B);
        if (cudaFuncSetAttribute(list_attn_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 mx) != cudaSuccess ||
            cudaFuncSetAttribute(list_attn_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx) !=
                cudaSuccess)
            return RTP_ERR_CUDA;
        attr_set[dev] = 1;
    }
    ListArgs a{};
    a.B = d->B; a.H_q = d->H_q; a.H_kv = d->H_kv; a.G = d->H_q / d->H_kv;
    a.N_max = d->N_max; a.seq_lens = d->seq_lens;
    a.n_rq = 0;
    for (int h = 0; h < d->H_q; ++h)
        if (hc[h / a.G] == RTP_HEAD_RETRIEVAL) a.ret_h[a.n_rq++] = h;
    if (a.n_rq == 0) return RTP_OK;
    a.scale_log2 = attn_scale * L2E;
    a.q = q; a.k = k; a.v = v; a.lists = lists; a.counts = counts; a.out = out;
    a.first = first;
    a.spill = spill;
    a.spill_any = reinterpret_cast<const uint32_t *>(ws + L.status) + 1;
    a.phase = phase;
    a.part = reinterpret_cast<float *>(ws + L.part_list);
    a.arrive = reinterpret_cast<uint32_t *>(ws + L.arrive_list);
    a.status = reinterpret_cast<uint32_t *>(ws + L.status);
    a.kv = kv ? *kv : make_kv(d, nullptr, a.status);
    a.id_off = id_off;
    a.part_out = part_out;
    const long long max_items = (long long)d->B * a.n_rq *
        std::min<long long>(LIST_MAX_SPLIT, (d->N_max + LCH - 1) / LCH);
    const unsigned grid = (unsigned)std::max(1LL, std::min<long long>(max_items, 2LL * num_sms()));
    const size_t smem = list_smem_bytes(d->B * a.n_rq, d->B);
    const char *name = phase == LIST_FIRST ? "sparse_attn_first" : phase == LIST_SPILL ? "sparse_attn_spill"
                                                                                       : "sparse_attn";
    if (d->kv_dtype == RTP_BF16)
        return ln.run_smem(name, list_attn_kernel<__nv_bfloat16>, dim3(grid), dim3(ATT_THREADS), smem, a);
    return ln.run_smem(name, list_attn_kernel<float>, dim3(grid), dim3(ATT_THREADS), smem, a);
}

int launch_force(Launcher &ln, const rtp_dims *d, int32_t *lists, int32_t *counts, const uint8_t *hc, int window,
                 int n_sink, char *ws, const Layout &L) {
    ForceArgs a{};
    a.B = d->B; a.H_q = d->H_q; a.G = d->H_q / d->H_kv;
    a.N_max = d->N_max; a.seq_lens = d->seq_lens;
    a.n_rq = 0;
    for (int h = 0; h < d->H_q; ++h)
        if (hc[h / a.G] == RTP_HEAD_RETRIEVAL) a.ret_h[a.n_rq++] = h;
    if (a.n_rq == 0) return RTP_OK;
    a.window = window; a.n_sink = n_sink;
    a.lists = lists; a.counts = counts;
    a.status = reinterpret_cast<uint32_t *>(ws + L.status);
    const size_t smem = fr_smem_bytes(std::min<long long>(d->N_max, (long long)window + n_sink));
    return ln.run_smem("force_rows", force_rows_kernel, dim3((unsigned)(d->B * a.n_rq)), dim3(FR_THREADS), smem, a);
}

}  // namespace

// Scratch of rtp_dense_decode_noalloc: one fixed array per device, so
// callers that cannot allocate still get the split-K partials, arrival
// counters and status word the dense kernel needs.  Host code must not use
// the symbol's host-side name as a device address: the device address comes
// from cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[RTP_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr size_t NOALLOC_ARRIVE_OFF = 256;                       // after the status word
constexpr size_t NOALLOC_PART_OFF = 256 + RTP_NOALLOC_MAX_GROUPS * 4;

// The address is cached per device in an atomic slot: threads that make
// their first call at the same time may both look it up, and both store the
// same value.  The cache assumes the device is not reset (cudaDeviceReset)
// after the first call; the array's address would then change.
int noalloc_scratch(char *&out) {
    static std::atomic<void *> ptrs[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RTP_ERR_CUDA;
    void *p = ptrs[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RTP_ERR_CUDA;
        ptrs[dev].store(p, std::memory_order_release);
    }
    out = static_cast<char *>(p);
    return RTP_OK;
}

// Self-test of the bounded device-side wait: one thread waits on an
// mbarrier that nothing completes (no copy is in flight on it), gives up
// after WAIT_LIMIT_NS and records RTP_ERR_TIMEOUT.
__global__ void wait_timeout_kernel(uint32_t *status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1u);
    fence_mbar_init();
    if (!mbar_wait(&bar, 0u)) set_status(status, RTP_ERR_TIMEOUT);
}

}  // namespace

// =========================================================================
// public entry points
// =========================================================================
extern "C" {

int rtp_version(void) { return 100; }

const char *rtp_error_string(int code) {
    switch (code) {
        case RTP_OK: return "ok";
        case RTP_ERR_INVALID_ARG: return "invalid argument";
        case RTP_ERR_UNSUPPORTED: return "unsupported shape or dtype (d=128, r=16, G<=8, f32/bf16)";
        case RTP_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case RTP_ERR_CUDA: return "CUDA error";
        case RTP_ERR_TIMEOUT: return "device-side wait timed out";
        case RTP_ERR_DEVICE_ARG: return "device-resident argument out of range";
        case RTP_ERR_RANGE: return "index logit not finite";
        default: return "unknown error";
    }
}

size_t rtp_workspace_size(const rtp_dims *dims, int op) {
    if (check_dims(dims) != RTP_OK) return 0;
    return op_bytes(make_layout(dims), op);
}

int rtp_workspace_init(void *ws, size_t ws_bytes, rtp_stream_t stream) {
    // The control region is a prefix whose size depends on the shapes; the
    // caller's buffer is at least that large, so zero min(ws_bytes, 64 MiB)
    // conservatively covers it for every shape this library accepts.
    if (!ws || ((uintptr_t)ws & 255u) || ws_bytes == 0) return RTP_ERR_WORKSPACE;
    const size_t n = ws_bytes < ((size_t)64 << 20) ? ws_bytes : ((size_t)64 << 20);
    if (cudaMemsetAsync(ws, 0, n, (cudaStream_t)stream) != cudaSuccess) return RTP_ERR_CUDA;
    return RTP_OK;
}

int rtp_check(void *ws, rtp_stream_t stream) {
    if (!ws) return RTP_ERR_WORKSPACE;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return RTP_ERR_CUDA;
    uint32_t st = 0;
    if (cudaMemcpy(&st, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return RTP_ERR_CUDA;
    if (st != 0) {
        if (cudaMemset(ws, 0, 4) != cudaSuccess) return RTP_ERR_CUDA;
    }
    return (int)st;
}

int rtp_append_index_keys(const rtp_dims *dims, const void *k_pre, int32_t T, const float *W_k_idx,
                          const int32_t *pos, const uint8_t *head_class, void *kidx_cache,
                          void *ws, size_t ws_bytes, rtp_stream_t stream) {
    RTP_TRY(check_dims(dims));
    if (!k_pre || !W_k_idx || !pos || !kidx_cache || T < 1) return RTP_ERR_INVALID_ARG;
    if (T > dims->N_max) return RTP_ERR_INVALID_ARG;
    if (!aligned16(k_pre) || !aligned16(W_k_idx) || !aligned16(kidx_cache)) return RTP_ERR_INVALID_ARG;
    if (head_class) RTP_TRY(check_head_class(dims, head_class));
    RTP_TRY(check_ws(dims, ws, ws_bytes, RTP_OP_APPEND_INDEX_KEYS));
    const Layout L = make_layout(dims);
    uint32_t *status = reinterpret_cast<uint32_t *>((char *)ws + L.status);
    unsigned long long mask = head_class ? ret_mask(dims, head_class)
                                         : (dims->H_kv >= 64 ? ~0ull : ((1ull << dims->H_kv) - 1));
    Launcher ln{(cudaStream_t)stream, nullptr};
    // the append waits on the device for the previous kernel of the stream,
    // so its launch overlaps that kernel's tail
    ln.pdl = true;
    // about eight CTAs per SM over all (b, g), so that a long append (a
    // prompt) keeps many keys in flight; runs of APP_TOK tokens
    const long long units = (long long)dims->B * dims->H_kv;
    const long long per_bg = std::max(1LL, 8LL * num_sms() / units);
    long long tpc = std::max<long long>(APP_TOK, (T + per_bg - 1) / per_bg);
    tpc = (tpc + APP_TOK - 1) / APP_TOK * APP_TOK;
    const dim3 grid((unsigned)((T + tpc - 1) / tpc), (unsigned)units);
    const dim3 block(APP_THREADS);
    const int tp = (int)tpc;
    const bool kb = dims->kv_dtype == RTP_BF16, ib = dims->idx_dtype == RTP_BF16;
    if (kb && ib)
        return ln.run("append", append_kernel<__nv_bfloat16, __nv_bfloat16>, grid, block,
                      (const __nv_bfloat16 *)k_pre, W_k_idx, pos, (__nv_bfloat16 *)kidx_cache,
                      dims->H_kv, (int)T, tp, (long long)dims->N_max, mask, status);
    if (kb && !ib)
        return ln.run("append", append_kernel<__nv_bfloat16, float>, grid, block,
                      (const __nv_bfloat16 *)k_pre, W_k_idx, pos, (float *)kidx_cache, dims->H_kv,
                      (int)T, tp, (long long)dims->N_max, mask, status);
    if (!kb && ib)
        return ln.run("append", append_kernel<float, __nv_bfloat16>, grid, block,
                      (const float *)k_pre, W_k_idx, pos, (__nv_bfloat16 *)kidx_cache, dims->H_kv,
                      (int)T, tp, (long long)dims->N_max, mask, status);
    return ln.run("append", append_kernel<float, float>, grid, block, (const float *)k_pre, W_k_idx,
                  pos, (float *)kidx_cache, dims->H_kv, (int)T, tp, (long long)dims->N_max, mask, status);
}

int rtp_index_scores(const rtp_dims *dims, const rtp_opts *opts, const float *q,
                     const float *W_q_idx, const void *kidx_cache, const uint8_t *head_class,
                     float *z_out, void *ws, size_t ws_bytes, rtp_stream_t stream) {
    RTP_TRY(check_dims(dims));
    if (!q || !W_q_idx || !kidx_cache || !z_out) return RTP_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(W_q_idx) || !aligned16(kidx_cache) || !aligned16(z_out))
        return RTP_ERR_INVALID_ARG;
    RTP_TRY(check_head_class(dims, head_class));
    RTP_TRY(check_ws(dims, ws, ws_bytes, RTP_OP_INDEX_SCORES));
    const Layout L = make_layout(dims);
    char *w = (char *)ws;
    SelPlan s = make_sel(dims, head_class, w, L);
    if (s.a.n_ret == 0) return RTP_OK;
    s.a.kidx = kidx_cache;
    s.a.q = q;
    s.a.Wq = W_q_idx;
    s.a.idx_scale = scale_or_default(opts ? opts->idx_scale : 0.f);
    Launcher ln{(cudaStream_t)stream, opts ? opts->prof : nullptr};
    const dim3 grid((unsigned)s.a.ctas, (unsigned)(dims->B * s.a.n_ret));
    if (dims->idx_dtype == RTP_BF16)
        return ln.run("scores", scores_kernel<SrcMma>, grid, dim3(SC_THREADS), s.a, s.w, z_out);
    return ln.run("scores", scores_kernel<SrcSimt<float>>, grid, dim3(SC_THREADS), s.a, s.w, z_out);
}

int rtp_topp_select(const rtp_dims *dims, const float *z, const uint8_t *head_class, float p,
                    int32_t *idx_out, int32_t *count_out, float *mass_out, void *ws, size_t ws_bytes,
                    rtp_stream_t stream) {
    RTP_TRY(check_dims(dims));
    if (!z || !idx_out || !count_out) return RTP_ERR_INVALID_ARG;
    if (std::isnan(p)) return RTP_ERR_INVALID_ARG;
    if (!aligned16(z)) return RTP_ERR_INVALID_ARG;
    RTP_TRY(check_head_class(dims, head_class));
    RTP_TRY(check_ws(dims, ws, ws_bytes, RTP_OP_TOPP_SELECT));
    const Layout L = make_layout(dims);
    SelPlan s = make_sel(dims, head_class, (char *)ws, L);
    if (s.a.n_ret == 0) return RTP_OK;
    s.a.z = z;
    s.a.p = p;
    s.a.lists = idx_out;
    s.a.count_out = count_out;
    s.a.mass_out = mass_out;
    Launcher ln{(cudaStream_t)stream, nullptr};
    return launch_select<SrcBuffer>(ln, dims, s);
}

int rtp_topk_select(const rtp_dims *dims, const float *z, const uint8_t *head_class, int32_t k,
                    int32_t *idx_out, int32_t *count_out, void *ws, size_t ws_bytes, rtp_stream_t stream) {
    RTP_TRY(check_dims(dims));
    if (!z || !idx_out || !count_out || k < 1) return RTP_ERR_INVALID_ARG;
    if (!aligned16(z)) return RTP_ERR_INVALID_ARG;
    RTP_TRY(check_head_class(dims, head_class));
    RTP_TRY(check_ws(dims, ws, ws_bytes, RTP_OP_TOPP_SELECT));
    const Layout L = make_layout(dims);
    SelPlan s = make_sel(dims, head_class, (char *)ws, L);
    if (s.a.n_ret == 0) return RTP_OK;
    s.a.z = z;
    s.a.p = 0.0f;           // not used with topk
    s.a.topk = k;
    s.a.lists = idx_out;
    s.a.count_out = count_out;
    s.a.mass_out = nullptr;
    Launcher ln{(cudaStream_t)stream, nullptr};
    return launch_select<SrcBuffer>(ln, dims, s);
}

int rtp_sparse_decode(const rtp_dims *dims, const rtp_opts *opts, const float *q_rope,
                      const void *k_cache, const void *v_cache, const int32_t *idx,
                      const int32_t *count, const uint8_t *head_class, float *out, void *ws,
                      size_t ws_bytes, rtp_stream_t stream) {
    RTP_TRY(check_dims(dims));
    if (!q_rope || !k_cache || !v_cache || !idx || !count || !out) return RTP_ERR_INVALID_ARG;
    if (!aligned16(q_rope) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return RTP_ERR_INVALID_ARG;
    RTP_TRY(check_head_class(dims, head_class));
    RTP_TRY(check_ws(dims, ws, ws_bytes, RTP_OP_SPARSE_DECODE));
    RTP_TRY(check_kv(dims, opts));
    const Layout L = make_layout(dims);
    const KvMap kv = make_kv(dims, opts, (char *)ws + L.status);
    Launcher ln{(cudaStream_t)stream, opts ? opts->prof : nullptr};
    return launch_list(ln, dims, q_rope, k_cache, v_cache, idx, count, head_class, out, (char *)ws, L,
                       scale_or_default(opts ? opts->attn_scale : 0.f), LIST_ALL, nullptr, nullptr, &kv);
}

int rtp_local_decode(const rtp_dims *dims, const rtp_opts *opts, const float *q_rope,
                     const void *k_cache, const void *v_cache, const uint8_t *head_class,
                     int32_t window, int32_t n_sink, float *out, void *ws, size_t ws_bytes,
                     rtp_stream_t stream) {
    RTP_TRY(check_dims(dims));
    if (!q_rope || !k_cache || !v_cache || !out) return RTP_ERR_INVALID_ARG;
    if (window < 1 || n_sink < 0) return RTP_ERR_INVALID_ARG;
    if (!aligned16(q_rope) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return RTP_ERR_INVALID_ARG;
    RTP_TRY(check_head_class(dims, head_class));
    RTP_TRY(check_ws(dims, ws, ws_bytes, RTP_OP_LOCAL_DECODE));
    RTP_TRY(check_kv(dims, opts));
    const Layout L = make_layout(dims);
    const KvMap kv = make_kv(dims, opts, (char *)ws + L.status);
    Launcher ln{(cudaStream_t)stream, opts ? opts->prof : nullptr};
    return launch_range(ln, dims, q_rope, k_cache, v_cache, head_class, RTP_HEAD_LOCAL, false, window,
                        n_sink, out, (char *)ws, L, scale_or_default(opts ? opts->attn_scale : 0.f), 0, &kv);
}

int rtp_dense_decode(const rtp_dims *dims, const rtp_opts *opts, const float *q_rope,
                     const void *k_cache, const void *v_cache, float *out, void *ws, size_t ws_bytes,
                     rtp_stream_t stream) {
    RTP_TRY(check_dims(dims));
    if (!q_rope || !k_cache || !v_cache || !out) return RTP_ERR_INVALID_ARG;
    if (!aligned16(q_rope) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return RTP_ERR_INVALID_ARG;
    RTP_TRY(check_ws(dims, ws, ws_bytes, RTP_OP_DENSE_DECODE));
    RTP_TRY(check_kv(dims, opts));
    const Layout L = make_layout(dims);
    const KvMap kv = make_kv(dims, opts, (char *)ws + L.status);
    Launcher ln{(cudaStream_t)stream, opts ? opts->prof : nullptr};
    return launch_range(ln, dims, q_rope, k_cache, v_cache, nullptr, -1, true, 1, 0, out, (char *)ws, L,
                        scale_or_default(opts ? opts->attn_scale : 0.f), 0, &kv);
}

int rtp_prefill_attention(const rtp_dims *dims, const rtp_opts *opts, const void *q, int32_t T,
                          const int32_t *pos0, const void *k_cache, const void *v_cache,
                          const uint8_t *head_class, int32_t window, int32_t n_sink, float *out, void *ws,
                          size_t ws_bytes, rtp_stream_t stream) {
    RTP_TRY(check_dims(dims));
    if (!q || !pos0 || !k_cache || !v_cache || !out) return RTP_ERR_INVALID_ARG;
    if (T < 1 || T > dims->N_max || window < 1 || n_sink < 0) return RTP_ERR_INVALID_ARG;
    if (dims->kv_dtype != RTP_BF16) return RTP_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned4(pos0))
        return RTP_ERR_INVALID_ARG;
    RTP_TRY(check_head_class(dims, head_class));
    RTP_TRY(check_ws(dims, ws, ws_bytes, RTP_OP_PREFILL));
    RTP_TRY(check_kv(dims, opts));
    static bool attr_set[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RTP_ERR_CUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM) !=
            cudaSuccess)
            return RTP_ERR_CUDA;
        attr_set[dev] = true;
    }
    // head classes go to the device through the kernel parameters
    PrefillArgs a{};
    a.B = dims->B; a.H_q = dims->H_q; a.H_kv = dims->H_kv; a.G = dims->H_q / dims->H_kv;
    a.N_max = dims->N_max; a.T = T;
    a.nsub = std::max(1, PF_WARPS / a.G);
    a.n_qblk = (T + 16 * a.nsub - 1) / (16 * a.nsub);
    a.seq_lens = dims->seq_lens; a.pos0 = pos0;
    for (int g = 0; g < dims->H_kv; ++g) a.hc[g] = head_class[g];
    a.window = window; a.n_sink = n_sink;
    a.scale_log2 = scale_or_default(opts ? opts->attn_scale : 0.f) * L2E;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.k = static_cast<const __nv_bfloat16 *>(k_cache);
    a.v = static_cast<const __nv_bfloat16 *>(v_cache);
    a.out = out;
    a.status = reinterpret_cast<uint32_t *>(static_cast<char *>(ws));
    a.kv = make_kv(dims, opts, a.status);
    if ((long long)a.n_qblk > 0x7fffffffLL) return RTP_ERR_UNSUPPORTED;
    Launcher ln{(cudaStream_t)stream, opts ? opts->prof : nullptr};
    return ln.run_smem("prefill_attn", prefill_attn_kernel, dim3((unsigned)a.n_qblk, (unsigned)(dims->B * dims->H_kv)),
                       dim3(PF_THREADS), PF_SMEM, a);
}

int rtp_dense_decode_noalloc(const rtp_dims *dims, const rtp_opts *opts, const float *q_rope,
                             const void *k_cache, const void *v_cache, float *out, int32_t *dev_status,
                             rtp_stream_t stream) {
    RTP_TRY(check_dims(dims));
    if (!q_rope || !k_cache || !v_cache || !out) return RTP_ERR_INVALID_ARG;
    if (!aligned16(q_rope) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return RTP_ERR_INVALID_ARG;
    RTP_TRY(check_kv(dims, opts));
    const long long groups = (long long)dims->B * dims->H_kv;
    if (groups > RTP_NOALLOC_MAX_GROUPS) return RTP_ERR_WORKSPACE;
    char *scr = nullptr;
    RTP_TRY(noalloc_scratch(scr));
    const cudaStream_t st = (cudaStream_t)stream;
    // status word and arrival counters must start at zero
    if (cudaMemsetAsync(scr, 0, NOALLOC_PART_OFF, st) != cudaSuccess) return RTP_ERR_CUDA;
    RangeArgs a{};
    a.B = dims->B; a.H_q = dims->H_q; a.H_kv = dims->H_kv; a.G = dims->H_q / dims->H_kv;
    a.N_max = dims->N_max; a.seq_lens = dims->seq_lens;
    a.n_grp = dims->H_kv;
    for (int g = 0; g < dims->H_kv; ++g) a.grp[g] = g;
    a.dense = 1;
    a.window = 1;
    a.n_sink = 0;
    const long long rec = (long long)GMAX * PSTRIDE * 4;            // bytes per split per group
    const long long cap = ((long long)RTP_NOALLOC_SCRATCH_BYTES - (long long)NOALLOC_PART_OFF) / (groups * rec);
    const long long chunks = (dims->N_max + 255) / 256;
    const long long want = std::max(1LL, (long long)num_sms() / groups);   // one CTA per SM, one wave
    a.n_split = (int)std::max(1LL, std::min({want, chunks, cap, (long long)RANGE_SPLIT_MAX}));
    a.slots = a.n_split;
    a.scale_log2 = scale_or_default(opts ? opts->attn_scale : 0.f) * L2E;
    a.q = q_rope; a.k = k_cache; a.v = v_cache; a.out = out;
    a.part = reinterpret_cast<float *>(scr + NOALLOC_PART_OFF);
    a.arrive = reinterpret_cast<uint32_t *>(scr + NOALLOC_ARRIVE_OFF);
    a.status = reinterpret_cast<uint32_t *>(scr);
    a.kv = make_kv(dims, opts, scr);
    Launcher ln{st, opts ? opts->prof : nullptr};
    const dim3 grid((unsigned)a.n_split, (unsigned)groups);
    if (dims->kv_dtype == RTP_BF16) {
        if (a.kv.table) {
            RTP_TRY(ln.run("dense_attn", gqa_mma_attn_kernel<true>, grid, dim3(GQ_THREADS), a));
        } else {
            RTP_TRY(ln.run("dense_attn", gqa_mma_attn_kernel<false>, grid, dim3(GQ_THREADS), a));
        }
    } else {
        RTP_TRY(ln.run("dense_attn", range_attn_kernel<float>, grid, dim3(ATT_THREADS), a));
    }
    if (dev_status && cudaMemcpyAsync(dev_status, scr, 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return RTP_ERR_CUDA;
    return RTP_OK;
}

int rtp_decode_step(const rtp_dims *dims, const rtp_opts *opts, const float *q, const float *q_rope,
                    const void *k_cache, const void *v_cache, const void *kidx_cache,
                    const float *W_q_idx, const uint8_t *head_class, float p, int32_t window,
                    int32_t n_sink, float *out, void *ws, size_t ws_bytes, rtp_stream_t stream) {
    RTP_TRY(check_dims(dims));
    if (!q || !k_cache || !v_cache || !kidx_cache || !W_q_idx || !out) return RTP_ERR_INVALID_ARG;
    if (std::isnan(p) || window < 1 || n_sink < 0) return RTP_ERR_INVALID_ARG;
    if (!q_rope) q_rope = q;
    if (!aligned16(q) || !aligned16(q_rope) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(kidx_cache) || !aligned16(W_q_idx) || !aligned16(out))
        return RTP_ERR_INVALID_ARG;
    RTP_TRY(check_head_class(dims, head_class));
    RTP_TRY(check_ws(dims, ws, ws_bytes, RTP_OP_DECODE_STEP));
    RTP_TRY(check_kv(dims, opts));
    const Layout L = make_layout(dims);
    char *w = (char *)ws;
    const KvMap kv = make_kv(dims, opts, w + L.status);
    Launcher ln{(cudaStream_t)stream, opts ? opts->prof : nullptr};
    const float asc = scale_or_default(opts ? opts->attn_scale : 0.f);
    const float isc = scale_or_default(opts ? opts->idx_scale : 0.f);

    SelPlan s = make_sel(dims, head_class, w, L);
    const bool any_local = s.a.n_ret < dims->H_kv;
    const cudaStream_t main = (cudaStream_t)stream;
    Side *side = nullptr;
    // Local heads run on a side stream forked at the start of the step and
    // joined at its end.  Beside the selection they get a few SMs of their
    // own (the selection kernels take one CTA per SM on the rest), so that
    // neither waits for the other's CTAs to drain.
    const int topk = opts ? opts->topk : 0;
    if (topk < 0) return RTP_ERR_INVALID_ARG;
    const bool force_local = opts && opts->force_local;
    if (force_local && std::min<long long>(dims->N_max, (long long)window + n_sink) > FR_MAX_ROWS)
        return RTP_ERR_UNSUPPORTED;
    const bool selecting = s.a.n_ret > 0 && (topk > 0 || p < 1.0f);
    int local_ctas = 0;
    if (any_local && s.a.n_ret > 0) {
        int max_ctas = 0;
        if (selecting) {
            // SMs for the local heads in proportion to their bytes against
            // the selection's (the index keys, read by the scan and again by
            // the collect pass); both move about the same bytes per SM and
            // microsecond.  At least LOCAL_SMS, at most half the GPU.
            const int groups = dims->B * (dims->H_kv - s.a.n_ret);
            const double kv_el = dims->kv_dtype == RTP_BF16 ? 2.0 : 4.0;
            const double ix_el = dims->idx_dtype == RTP_BF16 ? 2.0 : 4.0;
            const double rows = std::min<double>((double)dims->N_max, (double)window + (double)n_sink);
            const double lb = (double)groups * rows * 2.0 * D * kv_el;
            const double sb = 2.0 * dims->B * s.a.n_ret * (double)dims->N_max * R * ix_el;
            int want = (int)std::lround(num_sms() * lb / std::max(1.0, lb + sb));
            want = std::max(LOCAL_SMS, std::min(want, num_sms() / 2));
            local_ctas = groups * std::max(1, want / groups);
            local_ctas = std::min(local_ctas, num_sms() / 2);
            max_ctas = local_ctas;
        }
        RTP_TRY(side_stream(side));
        if (cudaEventRecord(side->fork, main) != cudaSuccess) return RTP_ERR_CUDA;
        if (cudaStreamWaitEvent(side->st, side->fork, 0) != cudaSuccess) return RTP_ERR_CUDA;
        Launcher lside{side->st, ln.prof};
        RTP_TRY(launch_range(lside, dims, q_rope, k_cache, v_cache, head_class, RTP_HEAD_LOCAL, false, window,
                             n_sink, out, w, L, asc, max_ctas, &kv));
        if (cudaEventRecord(side->join, side->st) != cudaSuccess) return RTP_ERR_CUDA;
    } else if (any_local) {
        RTP_TRY(launch_range(ln, dims, q_rope, k_cache, v_cache, head_class, RTP_HEAD_LOCAL, false, window,
                             n_sink, out, w, L, asc, 0, &kv));
    }
    int rc = RTP_OK;
    if (s.a.n_ret > 0) {
        if (!selecting) {
            // every token is kept: the retrieval heads' attention is dense
            rc = launch_range(ln, dims, q_rope, k_cache, v_cache, head_class, RTP_HEAD_RETRIEVAL, true, 1, 0,
                              out, w, L, asc, 0, &kv);
        } else {
            s.a.kidx = kidx_cache;
            s.a.q = q;
            s.a.Wq = W_q_idx;
            s.a.idx_scale = isc;
            s.a.p = p;
            s.a.topk = topk;
            s.a.lists = opts && opts->sel_idx ? opts->sel_idx : reinterpret_cast<int32_t *>(w + L.lists);
            s.a.count_out = opts && opts->sel_count ? opts->sel_count : reinterpret_cast<int32_t *>(w + L.counts);
            s.a.mass_out = opts ? opts->sel_mass : nullptr;
            const bool fused = dims->kv_dtype == RTP_BF16 && dims->idx_dtype == RTP_BF16 && !force_local;
            if (force_local) {
                // selection alone, then each retrieval head's list united
                // with the sink and window rows, then attention over the lists
                s.a.ovf = nullptr;
                rc = select_from_index(ln, dims, s, local_ctas);
                if (rc == RTP_OK) rc = launch_force(ln, dims, s.a.lists, s.a.count_out, head_class, window, n_sink, w, L);
                if (rc == RTP_OK)
                    rc = launch_list(ln, dims, q_rope, k_cache, v_cache, s.a.lists, s.a.count_out, head_class, out,
                                     w, L, asc, LIST_ALL, nullptr, nullptr, &kv);
                if (side && cudaStreamWaitEvent(main, side->join, 0) != cudaSuccess && rc == RTP_OK)
                    rc = RTP_ERR_CUDA;
                return rc;
            }
            if (fused) {
                // the sparse attention runs inside collect and finalize
                s.a.q_rope = q_rope;
                s.a.k_cache = static_cast<const __nv_bfloat16 *>(k_cache);
                s.a.v_cache = static_cast<const __nv_bfloat16 *>(v_cache);
                s.a.kv = kv;
                s.a.attn_scale_log2 = asc * L2E;
                s.a.out = out;
                s.a.part_sel = reinterpret_cast<float *>(w + L.part_sel);
                s.a.ovf = reinterpret_cast<uint32_t *>(w + L.ovf);
                // heads that keep many rows beyond what the collect pass
                // attended are finished by a list pass over every SM (a
                // 4-CTA cluster per head would take long over them).  The
                // pass costs a launch in the chain (~2 us) even when no head
                // needs it, so it is used from SPILL_MIN_CTX tokens on; below
                // that a cluster attends at most SPILL_MIN_CTX rows per head.
                const bool can_spill = dims->N_max > SPILL_MIN_CTX;
                s.a.spill_rows = can_spill ? FIN_SPILL : 0;
                s.a.part_list = reinterpret_cast<float *>(w + L.part_list);
                s.a.spill_any = reinterpret_cast<uint32_t *>(w + L.status) + 1;
                rc = select_from_index(ln, dims, s, local_ctas);
                if (rc == RTP_OK && can_spill) {
                    const bool pdl0 = ln.pdl;
                    ln.pdl = true;
                    rc = launch_list(ln, dims, q_rope, k_cache, v_cache, s.a.lists, s.a.count_out, head_class, out,
                                     w, L, asc, LIST_SPILL, reinterpret_cast<const int32_t *>(w + L.list_cnt),
                                     s.a.ovf, &kv);
                    ln.pdl = pdl0;
                }
                if (side && cudaStreamWaitEvent(main, side->join, 0) != cudaSuccess && rc == RTP_OK)
                    rc = RTP_ERR_CUDA;
                return rc;
            }
            // The rows the collect pass kept (clearly above the boundary bin)
            // are attended on a side stream while finalize resolves the
            // boundary bin; the rest and the merge follow finalize.
            Side *side2 = nullptr;
            const int32_t *first = reinterpret_cast<const int32_t *>(w + L.list_cnt);
            auto first_pass = [&]() -> int {
                RTP_TRY(side_stream(side2, 1));
                if (cudaEventRecord(side2->fork, main) != cudaSuccess) return RTP_ERR_CUDA;
                if (cudaStreamWaitEvent(side2->st, side2->fork, 0) != cudaSuccess) return RTP_ERR_CUDA;
                Launcher l2{side2->st, ln.prof};
                RTP_TRY(launch_list(l2, dims, q_rope, k_cache, v_cache, s.a.lists, s.a.count_out, head_class, out,
                                    w, L, asc, LIST_FIRST, first, nullptr, &kv));
                if (cudaEventRecord(side2->join, side2->st) != cudaSuccess) return RTP_ERR_CUDA;
                return RTP_OK;
            };
            rc = select_from_index(ln, dims, s, local_ctas, first_pass);
            if (side2 && cudaStreamWaitEvent(main, side2->join, 0) != cudaSuccess && rc == RTP_OK) rc = RTP_ERR_CUDA;
            if (rc == RTP_OK)
                rc = launch_list(ln, dims, q_rope, k_cache, v_cache, s.a.lists, s.a.count_out, head_class, out,
                                 w, L, asc, LIST_REST, first, nullptr, &kv);
        }
    }
    if (side && cudaStreamWaitEvent(main, side->join, 0) != cudaSuccess && rc == RTP_OK) rc = RTP_ERR_CUDA;
    return rc;
}

// ------------------------------------------------------------ context shards

namespace {
int check_shard(const rtp_dims *dims, const uint8_t *head_class, void *ws, size_t ws_bytes) {
    RTP_TRY(check_dims(dims));
    if (dims->kv_dtype != RTP_BF16 || dims->idx_dtype != RTP_BF16) return RTP_ERR_UNSUPPORTED;
    RTP_TRY(check_head_class(dims, head_class));
    return check_ws(dims, ws, ws_bytes, RTP_OP_DECODE_STEP);
}
}  // namespace

int rtp_shard_scan(const rtp_dims *dims, const rtp_opts *opts, const float *q, const void *kidx_cache,
                   const float *W_q_idx, const uint8_t *head_class, float p, void *ws, size_t ws_bytes,
                   rtp_stream_t stream) {
    RTP_TRY(check_shard(dims, head_class, ws, ws_bytes));
    if (!q || !kidx_cache || !W_q_idx || std::isnan(p)) return RTP_ERR_INVALID_ARG;
    if (p >= 1.0f) return RTP_OK;                    // every token kept: no threshold
    if (!aligned16(q) || !aligned16(kidx_cache) || !aligned16(W_q_idx)) return RTP_ERR_INVALID_ARG;
    const Layout L = make_layout(dims);
    SelPlan s = make_sel(dims, head_class, (char *)ws, L);
    if (s.a.n_ret == 0) return RTP_OK;
    s.a.kidx = kidx_cache;
    s.a.q = q;
    s.a.Wq = W_q_idx;
    s.a.idx_scale = scale_or_default(opts ? opts->idx_scale : 0.f);
    Launcher ln{(cudaStream_t)stream, opts ? opts->prof : nullptr};
    return select_from_index(ln, dims, s, 0, {}, SEL_SCAN);
}

int rtp_shard_hist(const rtp_dims *dims, void *ws, double **hist, int64_t *count) {
    RTP_TRY(check_dims(dims));
    if (!ws || !hist || !count) return RTP_ERR_INVALID_ARG;
    const Layout L = make_layout(dims);
    *hist = reinterpret_cast<double *>((char *)ws + L.hist);
    *count = (int64_t)dims->B * dims->H_q * HSTRIDE;
    return RTP_OK;
}

int rtp_shard_collect(const rtp_dims *dims, const rtp_opts *opts, const void *kidx_cache, const uint8_t *head_class,
                      float p, const int32_t *shard_off, void *ws, size_t ws_bytes, rtp_stream_t stream) {
    RTP_TRY(check_shard(dims, head_class, ws, ws_bytes));
    if (std::isnan(p) || !kidx_cache || !aligned16(kidx_cache) || !shard_off || !aligned4(shard_off))
        return RTP_ERR_INVALID_ARG;
    const Layout L = make_layout(dims);
    char *w = (char *)ws;
    SelPlan s = make_sel(dims, head_class, w, L);
    if (s.a.n_ret == 0 || p >= 1.0f) return RTP_OK;
    s.a.kidx = kidx_cache;
    s.a.p = p;
    s.a.id_off = shard_off;
    s.a.lists = opts && opts->sel_idx ? opts->sel_idx : reinterpret_cast<int32_t *>(w + L.lists);
    s.a.count_out = opts && opts->sel_count ? opts->sel_count : reinterpret_cast<int32_t *>(w + L.counts);
    Launcher ln{(cudaStream_t)stream, opts ? opts->prof : nullptr};
    return select_from_index(ln, dims, s, 0, {}, SEL_COLLECT);
}

int rtp_shard_cands(const rtp_dims *dims, void *ws, uint64_t **cands, uint32_t **counts, int64_t *stride,
                    int64_t *count_stride) {
    RTP_TRY(check_dims(dims));
    if (!ws || !cands || !counts || !stride || !count_stride) return RTP_ERR_INVALID_ARG;
    const Layout L = make_layout(dims);
    *cands = reinterpret_cast<uint64_t *>((char *)ws + L.cands);
    *counts = reinterpret_cast<uint32_t *>((char *)ws + L.cand_cnt);
    *stride = dims->N_max;
    *count_stride = CNT_STRIDE;
    return RTP_OK;
}

int rtp_shard_finish(const rtp_dims *dims, const rtp_opts *opts, const float *q_rope, const void *k_cache,
                     const void *v_cache, const void *kidx_cache, const uint8_t *head_class, float p, int32_t window,
                     int32_t n_sink, const int32_t *shard_off, const int32_t *glob_len, const uint64_t *all_cands,
                     const int32_t *all_counts, int64_t all_stride, float *part_out, void *ws, size_t ws_bytes,
                     rtp_stream_t stream) {
    RTP_TRY(check_shard(dims, head_class, ws, ws_bytes));
    if (std::isnan(p) || window < 1 || n_sink < 0) return RTP_ERR_INVALID_ARG;
    if (!q_rope || !k_cache || !v_cache || !kidx_cache || !shard_off || !glob_len || !part_out)
        return RTP_ERR_INVALID_ARG;
    if (!aligned16(q_rope) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(part_out) ||
        !aligned4(shard_off) || !aligned4(glob_len))
        return RTP_ERR_INVALID_ARG;
    RTP_TRY(check_kv(dims, opts));
    const Layout L = make_layout(dims);
    char *w = (char *)ws;
    const KvMap kv = make_kv(dims, opts, w + L.status);
    SelPlan s = make_sel(dims, head_class, w, L);
    const bool selecting = s.a.n_ret > 0 && p < 1.0f;
    if (selecting && (!all_cands || !all_counts || all_stride < 1 || !aligned16(all_cands) || !aligned4(all_counts)))
        return RTP_ERR_INVALID_ARG;
    Launcher ln{(cudaStream_t)stream, opts ? opts->prof : nullptr};
    const float asc = scale_or_default(opts ? opts->attn_scale : 0.f);
    // local heads: their rows of the shard (sinks and window in global positions)
    if (s.a.n_ret < dims->H_kv) {
        RTP_TRY(launch_range(ln, dims, q_rope, k_cache, v_cache, head_class, RTP_HEAD_LOCAL, false, window, n_sink,
                             nullptr, w, L, asc, 0, &kv, glob_len, shard_off, part_out));
    }
    if (s.a.n_ret == 0) return RTP_OK;
    if (!selecting)   // every token kept: the shard's rows of the retrieval heads, densely
        return launch_range(ln, dims, q_rope, k_cache, v_cache, head_class, RTP_HEAD_RETRIEVAL, true, 1, 0, nullptr,
                            w, L, asc, 0, &kv, glob_len, shard_off, part_out);
    s.a.kidx = kidx_cache;
    s.a.p = p;
    s.a.id_off = shard_off;
    s.a.ext_cands = reinterpret_cast<const unsigned long long *>(all_cands);
    s.a.ext_cnt = all_counts;
    s.a.ext_stride = all_stride;
    s.a.theta_out = reinterpret_cast<unsigned long long *>(w + L.theta);
    s.a.lists = opts && opts->sel_idx ? opts->sel_idx : reinterpret_cast<int32_t *>(w + L.lists);
    s.a.count_out = opts && opts->sel_count ? opts->sel_count : reinterpret_cast<int32_t *>(w + L.counts);
    s.a.mass_out = opts ? opts->sel_mass : nullptr;
    RTP_TRY(select_from_index(ln, dims, s, 0, {}, SEL_FINALIZE));
    RTP_TRY(ln.run("shard_own", shard_own_kernel, dim3((unsigned)(dims->B * s.a.n_ret * s.a.G)), dim3(OWN_THREADS),
                   s.a, s.w));
    return launch_list(ln, dims, q_rope, k_cache, v_cache, s.a.lists, s.a.count_out, head_class, nullptr, w, L, asc,
                       LIST_ALL, nullptr, nullptr, &kv, shard_off, part_out);
}

int rtp_merge_shards(const float *parts, int32_t P, int32_t n_heads, float *out, rtp_stream_t stream) {
    if (!parts || !out || P < 1 || n_heads < 1 || !aligned16(parts) || !aligned16(out)) return RTP_ERR_INVALID_ARG;
    merge_shards_kernel<<<(unsigned)n_heads, 32, 0, (cudaStream_t)stream>>>(parts, P, n_heads, out);
    return cudaGetLastError() == cudaSuccess ? RTP_OK : RTP_ERR_CUDA;
}

int rtp_prof_init(rtp_prof *prof, int32_t capacity) {
    if (!prof || capacity < 1) return RTP_ERR_INVALID_ARG;
    prof->capacity = 0;
    prof->count = 0;
    prof->filter = nullptr;
    prof->ev_start = (void **)std::calloc((size_t)capacity, sizeof(void *));
    prof->ev_stop = (void **)std::calloc((size_t)capacity, sizeof(void *));
    prof->name = (const char **)std::calloc((size_t)capacity, sizeof(char *));
    if (!prof->ev_start || !prof->ev_stop || !prof->name) return RTP_ERR_INVALID_ARG;
    for (int i = 0; i < capacity; ++i) {
        cudaEvent_t a, b;
        if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return RTP_ERR_CUDA;
        prof->ev_start[i] = a;
        prof->ev_stop[i] = b;
        prof->capacity = i + 1;
    }
    return RTP_OK;
}

int rtp_prof_elapsed(const rtp_prof *prof, int32_t slot, float *ms) {
    if (!prof || !ms || slot < 0 || slot >= prof->count) return RTP_ERR_INVALID_ARG;
    if (cudaEventElapsedTime(ms, (cudaEvent_t)prof->ev_start[slot], (cudaEvent_t)prof->ev_stop[slot]) !=
        cudaSuccess)
        return RTP_ERR_CUDA;
    return RTP_OK;
}

int rtp_prof_destroy(rtp_prof *prof) {
    if (!prof) return RTP_ERR_INVALID_ARG;
    for (int i = 0; i < prof->capacity; ++i) {
        if (prof->ev_start && prof->ev_start[i]) cudaEventDestroy((cudaEvent_t)prof->ev_start[i]);
        if (prof->ev_stop && prof->ev_stop[i]) cudaEventDestroy((cudaEvent_t)prof->ev_stop[i]);
    }
    std::free(prof->ev_start);
    std::free(prof->ev_stop);
    std::free((void *)prof->name);
    prof->ev_start = prof->ev_stop = nullptr;
    prof->name = nullptr;
    prof->capacity = prof->count = 0;
    return RTP_OK;
}

int rtp_selftest_wait_timeout(int32_t *dev_status, rtp_stream_t stream) {
    if (!dev_status || !aligned4(dev_status)) return RTP_ERR_INVALID_ARG;
    wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(reinterpret_cast<uint32_t *>(dev_status));
    return cudaGetLastError() == cudaSuccess ? RTP_OK : RTP_ERR_CUDA;
}

}  // extern "C"
