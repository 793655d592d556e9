/*
 * rtp.h -- C ABI of librtp.so: the per-head sparse decode step of RTPurbo
 * ("Full Attention Strikes Back: Transferring Full Attention into Sparse
 * within Hundred Training Steps", arXiv 2605.16928) on NVIDIA B200 (sm_100a).
 *
 * What the step computes, per sequence b and query head h of one layer
 * (query head h reads KV head g = h / G, G = H_q / H_kv):
 *
 *   - local KV heads (gist.science technical summary, Method section 1):
 *     exact softmax attention over the attention-sink rows [0, n_sink) and
 *     the sliding window [N - window, N), as one set;
 *   - retrieval KV heads (same summary, Method sections 2, 3 and 5; arXiv
 *     abstract): score every cached token with the 16-dim indexer,
 *     z_t = idx_scale * (W_q_idx[h] . q_h) . kidx[b, g, t], with q_h the
 *     pre-RoPE query and kidx the pre-RoPE index keys; turn the scores into
 *     softmax mass pi_t; keep the smallest set of tokens, taken by
 *     descending z (equal z: lower index first), whose mass reaches p; then
 *     run exact full-dimension softmax attention of the post-RoPE query over
 *     only the kept K/V rows (softmax renormalised over the kept set).
 *
 * The threshold is found without sorting (same summary, Method section 5:
 * sort-free histogram threshold and bandwidth-optimised sparse decode): one
 * streaming pass over the index keys builds, per head, a histogram of
 * softmax mass over the fp32 bits of z (512 bins: sign, exponent and 4
 * mantissa bits, each bin's mass kept relative to its upper edge, plus
 * per-octave sums); from it, the boundary bin -- where the mass accumulated
 * from the top first reaches p Z -- and Z itself.  Tokens above that bin
 * are kept outright; the tokens inside it are ranked by an exact radix
 * select on the order-preserving bits of z (then the token id), with
 * per-digit mass histograms, down to the boundary token.  The binned range
 * is |z| < 256: a logit outside it, or not finite, is reported as
 * RTP_ERR_RANGE.
 *
 * Conventions shared by every call
 *   - Tensor pointers are DEVICE pointers owned by the caller, dense
 *     row-major in the layouts given below, 16-byte aligned.  The library
 *     never allocates or frees device memory and keeps no pointer after a
 *     call returns.
 *   - `head_class` is a HOST array of H_kv bytes (RTP_HEAD_LOCAL or
 *     RTP_HEAD_RETRIEVAL), read during the call only: the split of heads is
 *     fixed offline per layer (Method section 1), so launch shapes are built
 *     from it on the host.
 *   - `dims->seq_lens` is a DEVICE array of B int32 valid lengths N_b
 *     (1 <= N_b <= N_max; the current token is row N_b - 1 and is already in
 *     the caches).  A length out of range is reported by rtp_check() as
 *     RTP_ERR_DEVICE_ARG and that sequence's outputs are written as zeros.
 *   - Scratch memory comes from a caller workspace `ws` of at least
 *     rtp_workspace_size(dims, op) bytes, 256-byte aligned, zeroed once by
 *     rtp_workspace_init() before first use.  Calls that share a workspace
 *     must be ordered on one stream.  The library keeps the workspace's
 *     control words consistent between calls itself.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream)
 *     and never synchronises it; calls can be captured in a CUDA graph.
 *   - Argument errors are detected on the host, before any launch, and
 *     returned; nothing is launched then.  Errors found on the device are
 *     recorded in the workspace status word and returned by rtp_check().
 *   - State kept by the library (created on first use, held until exit):
 *     per device, the SM count and whether each kernel's shared-memory
 *     attribute is set; per host thread and device, two side streams with
 *     their fork/join events, on which rtp_decode_step runs the local
 *     heads (and, for fp32 caches, the first list pass) beside the
 *     selection.  Two rtp_decode_step calls issued from one host thread on
 *     different caller streams share those side streams, so the second
 *     call's side work queues behind the first's; issue concurrent steps
 *     from different host threads.  rtp_dense_decode_noalloc's scratch array
 *     is described at that call.
 */
#ifndef RTP_H_
#define RTP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every entry point below is exported from librtp.so (built with hidden
 * default visibility). */
#if defined(__GNUC__)
#define RTP_API __attribute__((visibility("default")))
#else
#define RTP_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *rtp_stream_t;

/* Return codes. */
enum {
    RTP_OK = 0,
    RTP_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment, NaN p, ...   */
    RTP_ERR_UNSUPPORTED = 2, /* d != 128, r != 16, G > 8, dtype not f32/bf16 */
    RTP_ERR_WORKSPACE = 3,   /* ws NULL, misaligned or smaller than needed  */
    RTP_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed        */
    RTP_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out          */
    RTP_ERR_DEVICE_ARG = 6,  /* device-resident argument out of range       */
    RTP_ERR_RANGE = 7        /* an index logit was not finite               */
};

/* Element types of the caches. */
enum { RTP_F32 = 0, RTP_BF16 = 1 };

/* Head classes (per KV head). */
enum { RTP_HEAD_LOCAL = 0, RTP_HEAD_RETRIEVAL = 1 };

/* Operation ids for rtp_workspace_size(). */
enum {
    RTP_OP_APPEND_INDEX_KEYS = 0,
    RTP_OP_INDEX_SCORES = 1,
    RTP_OP_TOPP_SELECT = 2,
    RTP_OP_SPARSE_DECODE = 3,
    RTP_OP_LOCAL_DECODE = 4,
    RTP_OP_DENSE_DECODE = 5,
    RTP_OP_DECODE_STEP = 6, /* covers every other op */
    RTP_OP_PREFILL = 7
};

/* Shapes of one layer.  d must be 128 and r must be 16 on this path. */
typedef struct rtp_dims {
    int32_t B;                /* sequences                                  */
    int32_t H_q;              /* query heads                                */
    int32_t H_kv;             /* KV heads; H_q % H_kv == 0, H_q/H_kv <= 8   */
    int32_t d;                /* head dim (128)                             */
    int32_t r;                /* indexer dim (16)                           */
    int32_t kv_dtype;         /* RTP_F32 or RTP_BF16: k/v caches, k_pre     */
    int32_t idx_dtype;        /* RTP_F32 or RTP_BF16: index-key cache       */
    int32_t reserved;
    int64_t N_max;            /* cache capacity in rows (row stride)        */
    const int32_t *seq_lens;  /* device [B]: valid rows N_b per sequence    */
} rtp_dims;

/* Optional launch accounting: when rtp_opts.prof is set, every kernel a
 * call launches whose name contains `filter` (NULL: all) is bracketed by a
 * pair of CUDA events recorded on the call's stream.  Slots are used from
 * `count` upwards and `count` is advanced; recording stops at `capacity`.
 * Create the events with rtp_prof_init(), read them with rtp_prof_elapsed()
 * once the stream has reached them, release with rtp_prof_destroy(). */
typedef struct rtp_prof {
    int32_t capacity;
    int32_t count;
    void **ev_start;          /* cudaEvent_t[capacity]                     */
    void **ev_stop;           /* cudaEvent_t[capacity]                     */
    const char **name;        /* kernel name per slot (static strings)     */
    const char *filter;
} rtp_prof;

/* Paged K/V caches (a serving layout beside the method): k_cache and
 * v_cache are pools of num_pages pages, each [H_kv, page_size, d] in the
 * cache dtype (pool layout [num_pages, H_kv, page_size, d]); token t of
 * sequence b sits in page block_table[b * max_pages + t / page_size] at slot
 * t % page_size.  block_table is a DEVICE int32 array [B, max_pages];
 * page_size is a power of two in [16, 2^20]; max_pages * page_size >=
 * N_max.  A page number outside [0, num_pages) is reported by rtp_check()
 * as RTP_ERR_DEVICE_ARG (the outputs it touches are then unspecified).
 * The index-key cache stays contiguous ([B, H_kv, N_max, r]: 1/8 of the
 * K/V bytes per token at r = 16, d = 128). */
typedef struct rtp_kv_pages {
    const int32_t *block_table;
    int32_t page_size;
    int32_t max_pages;
    int32_t num_pages;
    int32_t reserved;
} rtp_kv_pages;

/* Options; pass NULL for all defaults. */
typedef struct rtp_opts {
    float idx_scale;          /* index logit scale; 0 -> 1/sqrt(d)          */
    float attn_scale;         /* attention scale;   0 -> 1/sqrt(d)          */
    /* rtp_decode_step only, optional device outputs describing the kept
     * sets (NULL: not written): */
    int32_t *sel_idx;         /* [B, H_q, N_max]: kept token ids of each
                                 retrieval head, first sel_count entries,
                                 order unspecified                          */
    int32_t *sel_count;       /* [B, H_q]: |S_h| (retrieval heads only)      */
    float *sel_mass;          /* [B, H_q]: index-softmax mass of S_h (with
                                 topk: the kept fraction of the N_b tokens) */
    rtp_prof *prof;           /* optional launch accounting                 */
    /* rtp_decode_step only: > 0 selects static top-k instead of top-p for
     * the retrieval heads (Method section 3 sets the dynamic top-p rule
     * against this fixed budget): each head keeps its topk tokens of
     * largest index logit (equal logits: lower index first), all N_b when
     * topk >= N_b; p is then not used.  0: top-p. */
    int32_t topk;
    /* rtp_decode_step only: nonzero unites each retrieval head's kept set
     * with the local heads' rows (sinks [0, n_sink) and the window of the
     * last `window` positions): S_h u L.  A serving option beside the
     * method (Method section 1 keeps sinks and window for local heads only);
     * the selection itself is unchanged.  sel_idx / sel_count then describe
     * the union, sel_mass the selected set alone.  Needs
     * min(N_max, window + n_sink) <= 393216, else RTP_ERR_UNSUPPORTED. */
    int32_t force_local;
    /* Paged K/V caches (NULL: contiguous [B, H_kv, N_max, d]); honoured by
     * rtp_decode_step, rtp_sparse_decode, rtp_local_decode,
     * rtp_dense_decode, rtp_dense_decode_noalloc and rtp_prefill_attention. */
    const rtp_kv_pages *kv_pages;
} rtp_opts;

/* Workspace bytes `op` needs for these shapes (0 on invalid dims).  The
 * size for RTP_OP_DECODE_STEP is at least the size of every other op. */
RTP_API size_t rtp_workspace_size(const rtp_dims *dims, int op);

/* Zero the workspace's control region (status word, counters, histograms)
 * on `stream`.  Call once after allocating a workspace. */
RTP_API int rtp_workspace_init(void *ws, size_t ws_bytes, rtp_stream_t stream);

/* Synchronise `stream`, then return (and clear) the first device-side error
 * recorded in `ws` since the last check, or RTP_ERR_CUDA if the stream
 * reports a CUDA error; RTP_OK otherwise. */
RTP_API int rtp_check(void *ws, rtp_stream_t stream);

/* Static description of a return code. */
RTP_API const char *rtp_error_string(int code);

/* Library version: major * 10000 + minor * 100 + patch. */
RTP_API int rtp_version(void);

/*
 * a0 -- index keys of new tokens (Method section 2: the projector acts on
 * the key before RoPE).  For every sequence b, retrieval KV head g and
 * t < T:  kidx_cache[b, g, pos[b] + t, :] = W_k_idx[g] . k_pre[b, g, t, :],
 * accumulated in fp32 and rounded to nearest-even into dims->idx_dtype.
 * Rows of local KV heads are not written (they keep no index keys).
 *   k_pre      [B, H_kv, T, d]   dims->kv_dtype (pre-RoPE keys)
 *   W_k_idx    [H_kv, r, d]      fp32
 *   pos        device [B] int32: first row to write; 0 <= pos, pos + T <=
 *              N_max, else RTP_ERR_DEVICE_ARG (that sequence is skipped)
 *   head_class host [H_kv] (NULL: every head is written)
 *   kidx_cache [B, H_kv, N_max, r] dims->idx_dtype (written)
 */
RTP_API int rtp_append_index_keys(const rtp_dims *dims, const void *k_pre, int32_t T,
                          const float *W_k_idx, const int32_t *pos,
                          const uint8_t *head_class, void *kidx_cache,
                          void *ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * a1 + a2 -- index logits (Method sections 2 and 3).  For retrieval heads:
 * z_out[b, h, t] = idx_scale * (W_q_idx[h] . q[b, h]) . kidx[b, g, t] for
 * t < N_b (fp32 accumulation).  Rows t >= N_b and local heads' rows are not
 * written.
 *   q          [B, H_q, d]       fp32 pre-RoPE queries
 *   W_q_idx    [H_q, r, d]       fp32
 *   kidx_cache [B, H_kv, N_max, r] dims->idx_dtype
 *   z_out      [B, H_q, N_max]   fp32
 */
RTP_API int rtp_index_scores(const rtp_dims *dims, const rtp_opts *opts, const float *q,
                     const float *W_q_idx, const void *kidx_cache,
                     const uint8_t *head_class, float *z_out,
                     void *ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * a3 + a4 + a5 -- dynamic top-p selection (Method section 3) from given
 * logits z [B, H_q, N_max] fp32 (rows t < N_b of retrieval heads are read).
 * Writes, for each retrieval head, the smallest set S of tokens taken by
 * descending z (equal z: lower index first) whose softmax mass reaches p:
 *   idx_out   [B, H_q, N_max] int32: S in the first count entries (any order)
 *   count_out [B, H_q] int32:   |S| (>= 1)
 *   mass_out  [B, H_q] fp32:    mass of S (optional, NULL: not written)
 * p >= 1 keeps all N_b tokens; p <= 0 keeps the top token; p NaN is
 * RTP_ERR_INVALID_ARG.  A logit that is not finite or has |z| >= 256 is
 * reported as RTP_ERR_RANGE (the call's outputs are then unspecified).
 */
RTP_API int rtp_topp_select(const rtp_dims *dims, const float *z, const uint8_t *head_class,
                    float p, int32_t *idx_out, int32_t *count_out, float *mass_out,
                    void *ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Static top-k selection from given logits (gist.science technical summary,
 * Method section 3: the fixed budget that the dynamic top-p rule is set
 * against): for each retrieval head the k tokens of largest z (equal z:
 * lower index first), or all N_b tokens when k >= N_b.
 *   z         [B, H_q, N_max] fp32 logits (local heads' rows not read)
 *   idx_out   [B, H_q, N_max] int32: the set in the first count entries,
 *             any order
 *   count_out [B, H_q] int32: min(k, N_b)
 * k < 1 is RTP_ERR_INVALID_ARG; logits out of the binned range or not
 * finite as for rtp_topp_select.  Workspace: the size rtp_topp_select needs
 * (RTP_OP_TOPP_SELECT).  The same level-1 histogram and boundary-bin radix
 * select as top-p, with every token counting one unit instead of its mass,
 * so the kept set is exact.
 */
RTP_API int rtp_topk_select(const rtp_dims *dims, const float *z, const uint8_t *head_class, int32_t k,
                            int32_t *idx_out, int32_t *count_out, void *ws, size_t ws_bytes,
                            rtp_stream_t stream);

/*
 * a6 -- sparse decode (Method section 5): exact softmax attention of each
 * retrieval head over only its listed rows,
 * out[b, h] = sum_{t in S} softmax_S(attn_scale * q_rope[b,h] . k[b,g,t]) v[b,g,t].
 *   q_rope     [B, H_q, d]       fp32 (post-RoPE queries)
 *   k_cache, v_cache [B, H_kv, N_max, d] dims->kv_dtype
 *   idx        [B, H_q, N_max] int32 row ids, first count[b, h] valid
 *   count      [B, H_q] int32, 1 <= count <= N_b
 *   out        [B, H_q, d] fp32: retrieval heads written, others untouched
 * Ids outside [0, N_b) or counts out of range: RTP_ERR_DEVICE_ARG; the
 * offending rows are skipped.
 */
RTP_API int rtp_sparse_decode(const rtp_dims *dims, const rtp_opts *opts, const float *q_rope,
                      const void *k_cache, const void *v_cache, const int32_t *idx,
                      const int32_t *count, const uint8_t *head_class, float *out,
                      void *ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * a7 -- local heads (Method section 1): exact softmax attention over the
 * sink rows [0, min(n_sink, N)) and the window rows [max(0, N - window), N)
 * as one set.  window >= 1, n_sink >= 0.  Writes out[b, h] for the query
 * heads of local KV heads only.
 */
RTP_API int rtp_local_decode(const rtp_dims *dims, const rtp_opts *opts, const float *q_rope,
                     const void *k_cache, const void *v_cache, const uint8_t *head_class,
                     int32_t window, int32_t n_sink, float *out,
                     void *ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Comparison kernel: dense decode attention of every query head over all
 * N_b rows (what the sparse step is measured against).
 */
RTP_API int rtp_dense_decode(const rtp_dims *dims, const rtp_opts *opts, const float *q_rope,
                     const void *k_cache, const void *v_cache, float *out,
                     void *ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * The fused decode step (a1-a8): local heads as rtp_local_decode, retrieval
 * heads as rtp_index_scores -> rtp_topp_select -> rtp_sparse_decode, without
 * writing the logits to memory: the index keys are streamed once to build
 * the mass histogram, re-read (skipping tiles that cannot hold a kept
 * token) to compact the kept set, and the kept K/V rows are gathered once.
 *   q          [B, H_q, d] fp32 pre-RoPE queries (indexer input)
 *   q_rope     [B, H_q, d] fp32 post-RoPE queries (attention); NULL: q
 *   k_cache, v_cache [B, H_kv, N_max, d] dims->kv_dtype
 *   kidx_cache [B, H_kv, N_max, r] dims->idx_dtype
 *   W_q_idx    [H_q, r, d] fp32
 *   p, window, n_sink as above
 *   out        [B, H_q, d] fp32 (every head written)
 * With p >= 1 retrieval heads attend densely over all N_b rows.
 */
RTP_API int rtp_decode_step(const rtp_dims *dims, const rtp_opts *opts, const float *q,
                    const float *q_rope, const void *k_cache, const void *v_cache,
                    const void *kidx_cache, const float *W_q_idx,
                    const uint8_t *head_class, float p, int32_t window, int32_t n_sink,
                    float *out, void *ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Prefill attention of a prompt (gist.science technical summary, Method
 * section 1: local heads keep a sliding window with attention sinks,
 * retrieval heads keep the full KV cache; arXiv abstract: only retrieval
 * heads keep the full cache).  The T prompt tokens of sequence b sit at
 * positions pos0[b] .. pos0[b] + T - 1 and their keys and values are
 * already in the caches (write them first; the index keys of the prompt
 * come from rtp_append_index_keys with the same T).  The token at position
 * P attends causally, exactly, over
 *   local KV heads:     the rows j <= P with j < n_sink or P - j < window
 *                       (the decode step's set for N = P + 1);
 *   retrieval KV heads: every row j <= P.
 *   q    [B, H_q, T, d] bf16, post-RoPE queries of the prompt tokens
 *   pos0 [B] int32 DEVICE array: position of prompt token 0
 *   k_cache, v_cache [B, H_kv, N_max, d] bf16 (dims->kv_dtype == RTP_BF16)
 *   out  [B, H_q, T, d] fp32
 * Needs 0 <= pos0[b] and pos0[b] + T <= seq_lens[b] <= N_max (else
 * RTP_ERR_DEVICE_ARG in the status word and zeros for that sequence);
 * window >= 1, n_sink >= 0, 1 <= T <= N_max.  Workspace:
 * rtp_workspace_size(dims, RTP_OP_PREFILL) bytes (the status word only).
 * Softmax scale opts->attn_scale (0: 1/sqrt(d)).  A kv_dtype of RTP_F32 is
 * RTP_ERR_UNSUPPORTED.
 */
RTP_API int rtp_prefill_attention(const rtp_dims *dims, const rtp_opts *opts, const void *q, int32_t T,
                                  const int32_t *pos0, const void *k_cache, const void *v_cache,
                                  const uint8_t *head_class, int32_t window, int32_t n_sink, float *out,
                                  void *ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Dense decode without a caller workspace.  (The paper has no counterpart:
 * this is a deployment variant of rtp_dense_decode.)
 *
 * For callers that cannot allocate device memory -- for example a plug-in
 * inside a host framework that owns every device allocation and hands the
 * plug-in none, or a serving path where cudaMalloc is off limits because it
 * can synchronise the device or fail under memory pressure.  The scratch
 * this call needs (status word, arrival counters, split partials) lives in
 * one fixed device array inside librtp.so, RTP_NOALLOC_SCRATCH_BYTES per
 * device; every GPU that loads the library holds it until the process
 * exits.  The call allocates nothing and frees nothing.
 *
 * Inputs and outputs are as for rtp_dense_decode; dev_status, if not NULL,
 * is a device int32 that receives this call's device-side status (0: ok,
 * else an RTP_ERR_* code such as RTP_ERR_DEVICE_ARG for a bad sequence
 * length).  Returns RTP_ERR_WORKSPACE when B * H_kv exceeds
 * RTP_NOALLOC_MAX_GROUPS (the partials would not fit), before any launch.
 *
 * The first call on a device, with that device current, looks up the
 * array's device address (cudaGetSymbolAddress) and keeps it for the
 * process; make that first call before any stream capture, and do not
 * reset the device (cudaDeviceReset) after it.  All calls share the one array and it keeps
 * the last call's contents: each call clears the part that must start at
 * zero, and calls whose executions overlap on the GPU (different streams,
 * no ordering between them) race on it -- order them on one stream.
 */
#define RTP_NOALLOC_SCRATCH_BYTES (8u << 20)
#define RTP_NOALLOC_MAX_GROUPS 1024
RTP_API int rtp_dense_decode_noalloc(const rtp_dims *dims, const rtp_opts *opts, const float *q_rope,
                                     const void *k_cache, const void *v_cache, float *out,
                                     int32_t *dev_status, rtp_stream_t stream);

/*
 * Context-sharded decode step (a multi-GPU layout beside the method: one
 * long sequence split over P GPUs, each holding a contiguous range of its
 * tokens).  The result is the step of the whole sequence -- the same kept
 * sets and output as rtp_decode_step over all tokens -- reached with three
 * exchanges that the caller makes between these calls (over NCCL or any
 * transport; every shard runs the same calls in the same order):
 *
 *   1. rtp_shard_scan      index-key scan of this shard: per-head level-1
 *                          mass histograms in the workspace;
 *      exchange 1          sum the histograms of all shards in place
 *                          (rtp_shard_hist gives their address and length,
 *                          fp64);
 *   2. rtp_shard_collect   the boundary bin of every head from the summed
 *                          histograms; this shard's tokens above it (kept) and
 *                          in it (boundary candidates, 64-bit keys: logit bits,
 *                          then the inverted GLOBAL token id);
 *      exchange 2          gather every shard's candidates of each head
 *                          (rtp_shard_cands gives this shard's, count at
 *                          stride count_stride) into all_cands [B*H_q][stride]
 *                          with all_counts [B*H_q];
 *   3. rtp_shard_finish    the exact threshold from all candidates, this
 *                          shard's kept list (global ids; opts->sel_idx /
 *                          sel_count if given) and the attention over its kept
 *                          rows and, for local heads, its rows among the
 *                          sinks and window of the global sequence: one
 *                          partial record per head in part_out [B*H_q][132]
 *                          fp32 (m and l in log2 units, then 2 unused, then
 *                          the 128 unnormalised output dims);
 *      exchange 3          gather every shard's part_out into parts
 *                          [P][B*H_q][132];
 *   4. rtp_merge_shards    merge the P records of each head into out
 *                          [B*H_q][128] (the same on every shard).
 *
 * dims describe this shard: seq_lens[b] its tokens of sequence b (>= 1),
 * N_max its capacity; shard_off[b] (device int32) the global position of
 * its token 0, glob_len[b] (device int32) the sequence's global length.
 * bf16 caches and index keys only (else RTP_ERR_UNSUPPORTED); top-p only
 * (opts->topk and force_local are not used).  p >= 1 makes the scan and
 * collect calls no-ops (the histograms are then not summed either) and the
 * finish call attend the shard's rows densely.
 * The workspace is rtp_workspace_size(dims, RTP_OP_DECODE_STEP) and must
 * stay untouched between the calls of one step.  Argument errors as for
 * rtp_decode_step.
 */
RTP_API int rtp_shard_scan(const rtp_dims *dims, const rtp_opts *opts, const float *q, const void *kidx_cache,
                           const float *W_q_idx, const uint8_t *head_class, float p, void *ws, size_t ws_bytes,
                           rtp_stream_t stream);
RTP_API int rtp_shard_hist(const rtp_dims *dims, void *ws, double **hist, int64_t *count);
RTP_API int rtp_shard_collect(const rtp_dims *dims, const rtp_opts *opts, const void *kidx_cache,
                              const uint8_t *head_class, float p, const int32_t *shard_off, void *ws,
                              size_t ws_bytes, rtp_stream_t stream);
RTP_API int rtp_shard_cands(const rtp_dims *dims, void *ws, uint64_t **cands, uint32_t **counts, int64_t *stride,
                            int64_t *count_stride);
RTP_API int rtp_shard_finish(const rtp_dims *dims, const rtp_opts *opts, const float *q_rope, const void *k_cache,
                             const void *v_cache, const void *kidx_cache, const uint8_t *head_class, float p,
                             int32_t window, int32_t n_sink, const int32_t *shard_off, const int32_t *glob_len,
                             const uint64_t *all_cands, const int32_t *all_counts, int64_t all_stride,
                             float *part_out, void *ws, size_t ws_bytes, rtp_stream_t stream);
RTP_API int rtp_merge_shards(const float *parts, int32_t P, int32_t n_heads, float *out, rtp_stream_t stream);

/* Self-test of failure detection (no counterpart in the pages).  The
 * library's device-side waits -- the index scan's waits on its own bulk
 * copies -- are bounded: after 0.2 s a waiting kernel records
 * RTP_ERR_TIMEOUT and returns, and the context stays usable.  This call
 * launches one kernel whose single waiting thread waits on a barrier that
 * nothing completes, so its wait runs out by construction (about 0.2 s of
 * device time) and it writes RTP_ERR_TIMEOUT into *dev_status (a device
 * int32, 4-byte aligned, which the caller zeroes first: the first error
 * written wins).  Returns RTP_ERR_INVALID_ARG for a null or misaligned
 * pointer, RTP_ERR_CUDA if the launch fails, else RTP_OK (asynchronous:
 * read dev_status after synchronising the stream). */
RTP_API int rtp_selftest_wait_timeout(int32_t *dev_status, rtp_stream_t stream);

/* Launch accounting helpers (see rtp_prof). */
RTP_API int rtp_prof_init(rtp_prof *prof, int32_t capacity);
RTP_API int rtp_prof_elapsed(const rtp_prof *prof, int32_t slot, float *ms);
RTP_API int rtp_prof_destroy(rtp_prof *prof);

#ifdef __cplusplus
}
#endif

#endif /* RTP_H_ */
