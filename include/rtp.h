/*
 * rtp.h -- C ABI of the head-wise sparse attention layer (RTPurbo) on NVIDIA B200 (sm_100a).
 *
 * The layer follows "Full Attention Strikes Back" (arXiv:2605.16928) as described on the
 * pages it was built from:
 *   - heads split into retrieval heads (~15%, keep the full KV cache) and local heads
 *     (~85%, sliding window plus attention sinks)      -- techwalker page, section 2;
 *   - retrieval heads score every causal key with a 16-dim pre-RoPE indexer
 *     s_j = (Wq_h^T q).(Wk_h^T k_j)                    -- techwalker page, section 3;
 *     ngjoo digest, "Core method" (pre-RoPE projections);
 *   - they keep the smallest highest-score set whose index-softmax mass is >= p, ties to
 *     the lower position                                -- zhichai page, insight 3;
 *     techwalker page, section 4 (dynamic top-p);
 *   - and run exact RoPE'd attention in the full head dim over that set
 *                                                        -- techwalker page, section 3;
 *   - local heads attend to the last W keys plus the first S keys
 *                                                        -- techwalker page, section 8
 *     (window 8192, 4 sinks).
 *
 * Conventions shared by every entry point
 *   - All device pointers are plain CUDA device addresses on the layer's device; every
 *     call is asynchronous and ordered on the stream it is given.  Of the per-call entry
 *     points only rtp_check synchronises its stream (and rtp_profile_read waits for the
 *     profiled kernels); rtp_create and rtp_destroy synchronise the device.
 *   - The caller owns q/k/v/out and the streams.  The layer owns its KV cache, index-key
 *     cache, weight copies and all scratch, and frees them in rtp_destroy.
 *   - Argument errors are detected on the host before any launch and return RTP_EINVAL
 *     (or RTP_ECAPACITY) without side effects.  Errors found by a kernel (a selection
 *     larger than max_select, a value outside the fp16 cache range, a bounded wait that
 *     ran out) are recorded in a device word and reported by the next rtp_check.
 *   - No call allocates device memory after rtp_create.
 *   - rtp_last_error returns a host string describing the most recent failure of a call
 *     on that layer; it stays valid until the next call on the layer.
 *   - A layer is not thread-safe: calls on one layer must be serialised by the caller and
 *     issued on streams whose work does not overlap on the GPU.
 */
#ifndef RTP_H_
#define RTP_H_

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RTP_OK = 0,
  RTP_EINVAL = 1,     /* bad argument (NULL pointer, unsupported size, p outside (0,1], ...) */
  RTP_ENOMEM = 2,     /* device allocation failed in rtp_create */
  RTP_ECAPACITY = 3,  /* append would exceed max_seq; nothing was written */
  RTP_EOVERFLOW = 4,  /* a selected set exceeded max_select; it was truncated */
  RTP_ECUDA = 5,      /* a CUDA runtime call or launch failed */
  RTP_ETIMEOUT = 6,   /* a bounded in-kernel wait gave up; results of that call are invalid */
  RTP_EINTERNAL = 7,  /* an internal consistency check failed */
  RTP_ERANGE = 8      /* a RoPE'd key or a value lies outside the fp16 cache range */
} rtp_status;

typedef struct rtp_layer rtp_layer; /* opaque; owned by the library */

typedef struct {
  int32_t batch;              /* B sequences, 1 <= B <= 256; each has its own length */
  int32_t n_q_heads;          /* Hq >= 1 */
  int32_t n_kv_heads;         /* Hkv >= 1, divides Hq (GQA: q head h reads KV head h / (Hq/Hkv)) */
  int32_t head_dim;           /* D; must be 128 */
  int32_t index_dim;          /* r; must be 16 */
  int64_t max_seq;            /* KV capacity per sequence (positions 0..max_seq-1) */
  const uint8_t* head_class;  /* HOST [Hq]: 1 = retrieval head, 0 = local head; copied */
  float top_p;                /* p in (0, 1]; p == 1 keeps every causal key */
  int32_t window;             /* W >= 1: a local head sees keys j with i - j < W */
  int32_t n_sink;             /* S >= 0: ... and keys j < S */
  double rope_base;           /* RoPE base (1e6 in the pages' models) */
  float sm_scale;             /* attention scale; 0 selects 1/sqrt(D) */
  const float* wq_index;      /* HOST [Hr][D][r] fp32, retrieval heads in ascending order; copied */
  const float* wk_index;      /* HOST [Hr][D][r] fp32; copied */
  int64_t max_select;         /* capacity of one selected set; 0 selects max_seq */
  int32_t max_chunk;          /* largest prefill chunk C; 0 selects 16384 */
  int32_t index_bf16;         /* 0: index keys stored in fp32; 1: in bf16, rounded to nearest
                                 even from an fp64 projection (half the decode index stream;
                                 the selection then follows the rounded keys) */
  int32_t prefill_dense;      /* 1: in prefill, retrieval heads attend to every causal key (the
                                 pages' own prefill, techwalker page Q&A; ngjoo digest,
                                 limitations); decode keeps its selection.  0: per-row selection */
  int64_t top_k;              /* 0: top-p selection; k > 0: retrieval heads keep the first
                                 min(k, n) keys of the order (s desc, j asc) instead -- the
                                 pages' fixed-budget ablation (techwalker page, section 4);
                                 sel_mass and threshold are then reported as -1 */
  int32_t n_clusters;         /* 0: no clustering.  K in [1, 1024]: the layer can cluster each
                                 retrieval head's index keys into K clusters (rtp_cluster_build)
                                 and then select by clusters in decode (RTPurboV2, aitntnews page,
                                 finding 3).  Needs index_bf16 = 1 and top_k = 0 */
} rtp_config;

/* Optional decode statistics, DEVICE arrays [B][Hr] (retrieval heads ascending).  Any
 * member may be NULL. */
typedef struct {
  int32_t* sel_count;  /* |J|, capped at max_select */
  float* sel_mass;     /* index-softmax mass of J (>= p); clustered selection: the weight
                          fraction of the clusters hit (>= p) */
  float* threshold;    /* index-softmax mass of the last member of J; clustered selection: the
                          weight fraction of the last cluster taken */
  int32_t* sel_index;  /* [B][Hr][sel_index_cap]: the first min(|J|, cap) positions of J, ascending */
  int64_t sel_index_cap;
} rtp_decode_stats;

/* Optional prefill statistics, DEVICE arrays (retrieval heads ascending).  Any member may be
 * NULL.  sel_bitmap holds, for every row i and retrieval head, bitmap_words 32-bit words: bit
 * (j % 32) of word j / 32 is set iff key j is in row i's selected set.  Words the kernel writes:
 * those covering keys 0 .. (last position of the row's 128-row tile), rounded up to 64 keys
 * and capped at bitmap_words; the caller zeroes the rest.  Keys past 32 * bitmap_words are not
 * reported (the selection itself is unaffected).
 *
 * Row-subset positions (cheap at any chunk size, where a full bitmap is not): for each of the
 * n_rows distinct chunk rows listed in `rows` (DEVICE int32, 0 <= row < C; other values are
 * ignored) and each retrieval head, row_sel receives the row's selected positions in
 * ascending order, the first min(|J_i|, row_sel_cap) of them; |J_i| itself is in sel_count,
 * which must then be non-NULL.  Entries past the count are not written. */
typedef struct {
  int32_t* sel_count;    /* [B][C][Hr] |J_i| */
  float* sel_mass;       /* [B][C][Hr] index-softmax mass of J_i (>= p) */
  uint32_t* sel_bitmap;  /* [B][C][Hr][bitmap_words] */
  int64_t bitmap_words;
  const int32_t* rows;   /* [n_rows] chunk rows whose selected positions are listed, or NULL */
  int32_t n_rows;
  int32_t* row_sel;      /* [B][n_rows][Hr][row_sel_cap] */
  int64_t row_sel_cap;
} rtp_prefill_stats;

/* Device-side view of the layer's caches (for tests and tools; read-only use). */
typedef struct {
  const void* k;    /* fp16 [B][Hkv][max_seq][D]: RoPE'd keys */
  const void* v;    /* fp16 [B][Hkv][max_seq][D] */
  const float* idx; /* fp32 [B][Hr][max_seq][r]: pre-RoPE index keys Wk_h^T k_j (NULL with bf16 keys) */
  int64_t max_seq;
  int32_t n_retrieval;
  const void* idx_bf16; /* bf16 [B][Hr][max_seq][r] when the layer stores bf16 index keys, else NULL */
} rtp_cache_view;

/* Device-side view of a layer's K-cache clustering (read-only use).  P = B * Hr problems,
 * retrieval heads ascending within a sequence. */
typedef struct {
  const double* centres;  /* fp64 [P][K][r] cluster centres in the index space */
  const int32_t* counts;  /* [P][K] keys per cluster */
  const uint16_t* assign; /* [P][assign_stride] cluster of each clustered key (positions < rtp_cluster_len) */
  int32_t n_clusters;     /* K (0: the layer cannot cluster) */
  int32_t ready;          /* 1 while the clustering is in use by decode, else 0 */
  int64_t max_seq;
  int64_t assign_stride;  /* entries per row of assign: max_seq rounded up to a multiple of 16 */
} rtp_cluster_view;

/* Create a layer on the current CUDA device: validates cfg, allocates the caches and all
 * scratch, uploads the weights.  Synchronous.  On success *out receives the layer. */
rtp_status rtp_create(const rtp_config* cfg, rtp_layer** out);

/* Release everything the layer owns.  Synchronises the device first.  NULL is a no-op. */
rtp_status rtp_destroy(rtp_layer* layer);

/* Append T >= 1 tokens to every sequence, each at its own positions len_b .. len_b+T-1: k, v
 * are DEVICE bf16 [B][T][Hkv][D], k pre-RoPE.  Writes RoPE(k) and v into the fp16 KV cache and,
 * for every retrieval head h, the pre-RoPE index key Wk_h^T k into the index cache (the pages'
 * 16-dim indexer: techwalker page section 3; ngjoo digest, pre-RoPE projections).  Advances
 * every length by T.  RTP_ECAPACITY (nothing written) if some len_b + T > max_seq. */
rtp_status rtp_append_kv(rtp_layer* layer, const void* k, const void* v, int32_t T,
                         cudaStream_t stream);

/* Ragged batches: append T >= 1 tokens to sequence b alone (k, v DEVICE bf16 [T][Hkv][D], k
 * pre-RoPE) at positions len_b .. len_b+T-1, and advance len_b by T.  RTP_EINVAL for b outside
 * [0, B); RTP_ECAPACITY (nothing written) if len_b + T > max_seq. */
rtp_status rtp_append_kv_seq(rtp_layer* layer, int32_t b, const void* k, const void* v, int32_t T,
                             cudaStream_t stream);

/* One decode step for every sequence: q is DEVICE bf16 [B][Hq][D] pre-RoPE, sequence b's row at
 * position len_b-1 (append its own key first; every len_b >= 1, else RTP_EINVAL).  Sequences of
 * a ragged batch select and attend over their own keys only.  out is DEVICE fp32 [B][Hq][D].  Retrieval heads run
 * index scoring, exact top-p selection and sparse attention; local heads run window+sink
 * attention, on an internal stream forked from `stream` (an event) after the selection and
 * joined back (an event) before the call's work ends in `stream` order.  stats may be NULL. */
rtp_status rtp_decode(rtp_layer* layer, const void* q, float* out, const rtp_decode_stats* stats,
                      cudaStream_t stream);

/* Chunked prefill: the last C appended tokens of every sequence are its chunk; q is DEVICE bf16
 * [B][C][Hq][D] pre-RoPE, row i of sequence b at position len_b-C+i (ragged batches too).  Every row runs its own top-p selection over its causal
 * prefix (retrieval heads) or its own window (local heads).  out is DEVICE fp32 [B][C][Hq][D].
 * Requires 1 <= C <= min(shortest len_b, max_chunk).  The local heads run on an internal stream forked
 * from `stream` (an event) and joined back (an event).  stats may be NULL. */
rtp_status rtp_prefill_chunk(rtp_layer* layer, const void* q, int32_t C, float* out,
                             const rtp_prefill_stats* stats, cudaStream_t stream);

/* Change p for later calls (0 < p <= 1).  Takes effect in stream order of later calls. */
rtp_status rtp_set_top_p(rtp_layer* layer, float top_p);

/* Test knob: the limit, in SM clock cycles, on each wait of the decode selection's grid-wide
 * barriers and of the clustered selection's compaction look-back (0 restores the default,
 * about one second).  A wait past its limit makes the
 * kernel record RTP_ETIMEOUT and leave; the next rtp_check reports it and resets the
 * selection's scratch, so later calls start clean.  A tiny limit makes the barrier give up
 * at once, which is how the timeout path is tested.  The tensor-core completion waits of the
 * prefill kernels keep their fixed limit.  RTP_EINVAL if cycles < 0. */
rtp_status rtp_set_wait_limit(rtp_layer* layer, int64_t cycles);

/* The longest sequence's length (host-side counters advanced by the appends): the common
 * length of a batch whose sequences have one.  -1 for a NULL layer. */
int64_t rtp_seq_len(const rtp_layer* layer);

/* Length of sequence b; -1 for a NULL layer or b outside [0, B). */
int64_t rtp_seq_len_of(const rtp_layer* layer, int32_t b);

/* Forget every token (every length back to 0); the caches are overwritten by later appends. */
rtp_status rtp_reset(rtp_layer* layer);

/* Roll every sequence longer than new_len back to new_len (e.g. to re-run a step or drop
 * rejected speculative tokens); later appends overwrite the dropped positions.  RTP_EINVAL if
 * new_len is negative or above the longest length. */
rtp_status rtp_truncate(rtp_layer* layer, int64_t new_len);

/* Roll sequence b back to new_len <= its length.  RTP_EINVAL for b outside [0, B) or new_len
 * outside [0, len_b]. */
rtp_status rtp_truncate_seq(rtp_layer* layer, int32_t b, int64_t new_len);

/* K-cache clustering (RTPurboV2, aitntnews page, finding 3: the two-level funnel).  For every
 * sequence b and retrieval head, clusters the stored bf16 index keys of positions 0 .. len_b - 1
 * into K = n_clusters clusters by Lloyd's k-means with `iters` passes (0..1000), and records
 * len_b as the sequence's clustered length.  The keys are taken on the fixed-point grid 2^-27;
 * centre k starts at key floor((2k+1) len_b / (2K)); each pass assigns every key to the centre
 * of least squared distance (fp64, ties to the lower centre) and moves every non-empty centre
 * to its keys' mean; a final assignment follows the last pass.  Every step is deterministic.
 *
 * From then on rtp_decode (for p < 1) selects by clusters: centre scores c_k = q~ . mu_k with
 * the index query q~, cluster weights n_k exp(c_k - max c), clusters taken in (c desc, k asc)
 * order while the weight before them is below p of the total; the selected set J is every
 * clustered key of a hit cluster plus every key appended after the clustering, and the
 * retrieval head attends exactly over J.  Truncating a sequence below its clustered length,
 * rtp_reset or rtp_cluster_drop ends the clustered selection (decode returns to the per-key
 * top-p).  RTP_EINVAL (nothing launched) if the layer has no n_clusters or no retrieval heads,
 * iters is out of range, or some len_b is below K or above 2^21.  An index key of magnitude
 * >= 2^15 is counted as 0 and reported as RTP_ERANGE by the next rtp_check. */
rtp_status rtp_cluster_build(rtp_layer* layer, int32_t iters, cudaStream_t stream);
rtp_status rtp_cluster_drop(rtp_layer* layer);
/* Clustered length of sequence b (0 when no clustering is in use; -1 for a NULL layer or b
 * outside [0, B)). */
int64_t rtp_cluster_len(const rtp_layer* layer, int32_t b);
rtp_status rtp_get_clusters(const rtp_layer* layer, rtp_cluster_view* view);

/* Per-kernel device timing.  While enabled, the library records a CUDA event pair on the
 * launch stream around every kernel it launches, and runs every kernel on the call's stream
 * in order (no internal fork), so each recorded time belongs to one kernel alone.  rtp_profile_read synchronises on the
 * recorded events, returns the summed device time (ms) and launch count of the named kernel
 * ("append_kv", "q_prep", "decode_select", "decode_topk", "decode_gather", "decode_swa", "swa_merge",
 * "dense_fill", "cluster_*", "prefill_*"; NULL: all kernels together), and clears that kernel's record. */
rtp_status rtp_profile_enable(rtp_layer* layer, int on);
rtp_status rtp_profile_read(rtp_layer* layer, const char* kernel, double* total_ms, int64_t* launches);

/* Synchronise `stream`, then report and clear errors recorded by kernels since the last
 * check (RTP_EOVERFLOW, RTP_ERANGE, RTP_ETIMEOUT, ...). */
rtp_status rtp_check(rtp_layer* layer, cudaStream_t stream);

/* Device pointers of the caches. */
rtp_status rtp_get_cache(const rtp_layer* layer, rtp_cache_view* view);

/* Exact attention over caller-given key lists, with no layer and no device allocation.
 * (No counterpart on the pages: this serves callers that cannot allocate device memory --
 * code running while a CUDA graph is captured, engines that own all device memory through
 * their own pool, processes whose device memory is fully committed.)
 *
 * For each problem p < P (one decode query): o_p = softmax_j(sm_scale * q_p . K_j) V_j over the
 * positions j = idx[p][0 .. min(cnt[p], max_count)).  K_j and V_j are fp16 rows of 128 values at
 * k / v + kv_block[p] * kv_stride + j * 128 (kv_block NULL: block p); q is DEVICE fp32 [P][128]
 * (already RoPE'd), idx DEVICE int32 [P][idx_stride], cnt DEVICE int32 [P], out DEVICE fp32
 * [P][128].  Rows of the layer's cache (rtp_get_cache) can be passed directly.  A problem whose
 * count is <= 0 has an empty list; its output row is written as zeros.
 *
 * Alignment: k, v and q must be 16-byte aligned and kv_stride a multiple of 8 elements (rows
 * are read as 16-byte vectors); otherwise RTP_EINVAL, nothing launched.  Every listed position
 * must lie inside its block: positions are not checked.
 *
 * Scratch: one built-in device array of about 2.1 MB (4096 work items of 128 keys); the call
 * returns RTP_EINVAL without launching when P * ceil(max_count / 128) exceeds 4096 or P > 2048.
 * The first call on each device (with that device current) looks the array's address up and
 * caches it for the life of the process (the cache assumes the device's primary context is
 * never reset): make that first call before any stream capture.  Every call on a device shares
 * the array, so calls whose kernels overlap on the GPU race; serialise them (one stream).
 * Errors are reported through rtp_last_error(NULL). */
rtp_status rtp_gather_attn_noalloc(const void* k, const void* v, const int32_t* kv_block, int64_t kv_stride,
                                   const float* q, const int32_t* idx, int64_t idx_stride,
                                   const int32_t* cnt, int32_t P, int64_t max_count, float sm_scale,
                                   float* out, cudaStream_t stream);

/* Measurement probe, not part of the method: launches `blocks` CTAs of 256 threads that each
 * evaluate 8 * iters dependent-free chains of ex2.approx (the exponential the prefill selection
 * uses once per causal (row, key) pair), writing one float per thread to out (DEVICE,
 * blocks * 256 floats).  *n_exp receives the number of exponentials launched; the caller times
 * the launch on `stream` with CUDA events to measure the exponential issue rate that bounds
 * the prefill selection.  RTP_EINVAL on a non-positive size or a NULL pointer. */
rtp_status rtp_probe_ex2(int32_t blocks, int32_t iters, float* out, int64_t* n_exp, cudaStream_t stream);

/* Host string for the last failure on this layer ("" if none).  layer may be NULL, which
 * returns the last failure of rtp_create in this thread. */
const char* rtp_last_error(const rtp_layer* layer);

#ifdef __cplusplus
}
#endif

#endif /* RTP_H_ */
