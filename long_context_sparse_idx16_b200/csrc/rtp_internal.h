// rtp_internal.h -- layer state and kernel launch entry points (host side, internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <map>
#include <string>
#include <utility>
#include <vector>

#include "rtp.h"
#include "tma.cuh"

namespace rtp {

// Work-split and scratch sizes of the fused decode index-stream + top-p select kernel.
constexpr int kSelThreads = 1024;
constexpr int kSelBins = 2048;   // level-1 score bins (width 1/64 below the row max) and radix digits
constexpr int kSelMaxSeg = 16;   // (problem, CTA) segments one CTA may hold
constexpr int kSelCand = 1024;   // crossing-bin keys resolved by an in-CTA sort
constexpr int kSelFine = 1024;   // level-1 fine bins (width 1/64 below the row max, 16 deep)
constexpr int kSelMaxGrid = 256; // CTAs of the selection grid (<= SM count)
// Share of a CTA pair's keys taken by the even SM of a TPC when every SM holds one selection
// CTA.  The two SMs of a TPC share its bandwidth unevenly: with equal key counts the index
// stream took 57 us on even and 66 us on odd SMs; with a 0.537 share, 61.5 and 54.9 us (the odd
// SM speeds up as its partner's share grows); with 0.521, 59.6 and 63.5 us.  Interpolating the
// difference to zero gives 0.527.
constexpr double kSelEvenShare = 0.527;

// Sparse-attention gather (decode): the item kernel's chunk of selected positions and its
// item cap per problem (the flat kernel needs two partials per CTA).
constexpr int kGatherChunk = 128;
constexpr int kGatherMaxItems = 64;

// Prefill selection: keys of a row's crossing range captured per refinement walk.
constexpr int kPfCapture = 2048;
// Prefill attention: key tiles (64 keys) per CTA when long rows split their keys (256K keys).
constexpr int kAttSplitTiles = 4096;

// Fixed top-k decode selection (ablation mode): keys per chunk of its radix-select kernels.
constexpr int kTopkChunk = 4096;

// Sequences of a layer, and their per-sequence positions passed to kernels by value (a
// sequence's length, or the position of its first new row).
constexpr int kMaxBatch = 256;
struct SeqPos {
  int32_t v[kMaxBatch];
};

// Window + sink decode attention: keys per CTA tile and threads.
constexpr int kSwaTile = 128;
constexpr int kSwaThreads = 128;

}  // namespace rtp

struct rtp_layer {
  // configuration
  int B = 0, Hq = 0, Hkv = 0, Hr = 0, group = 0;
  int64_t max_seq = 0, max_select = 0;
  int64_t len = 0;                 // the longest sequence's length (sizes the launches)
  std::vector<int64_t> lens;       // [B] each sequence's length (ragged batches)
  int max_chunk = 0;
  float top_p = 0.9f, sm_scale = 0.f;
  double rope_base = 1e6;
  int W = 0, S = 0;
  std::vector<int> ret_heads;        // retrieval slot -> q head
  std::vector<int> head_slot;        // q head -> retrieval slot or -1
  int device = 0, sm_count = 0;
  size_t smem_optin = 0;

  // caches
  __half* kc = nullptr;  // [B][Hkv][max_seq][D] RoPE'd keys
  __half* vc = nullptr;  // [B][Hkv][max_seq][D]
  float* idx = nullptr;  // [B][Hr][max_seq][r] fp32 index keys (fp32 storage)
  __nv_bfloat16* idx_b = nullptr;  // [B][Hr][max_seq][r] bf16 index keys (bf16 storage)
  bool index_bf16 = false;
  bool prefill_dense = false;       // retrieval heads dense in prefill (the pages' own prefill)
  int64_t top_k = 0;                // > 0: fixed-budget selection instead of top-p
  uint32_t* tk_keys = nullptr;      // [B*Hr][max_seq] order keys of the scores (top-k mode)
  uint32_t* tk_hist = nullptr;      // [B*Hr][4][256] radix histograms (top-k mode)
  uint32_t* tk_cnt = nullptr;       // [B*Hr][chunks][2] per-chunk counts (top-k mode)
  float* wq = nullptr;   // [Hr][D][r]
  float* wk = nullptr;   // [Hr][D][r]
  double* theta = nullptr;  // [D/2] RoPE frequencies base^(-2c/D)
  int16_t* d_head_slot = nullptr;  // [Hq]
  int16_t* d_ret_head = nullptr;   // [Hr]
  int16_t* d_loc_head = nullptr;   // [Hkv][kMaxGroup] local q heads of each KV head (-1 pad)
  int32_t* d_loc_cnt = nullptr;    // [Hkv]
  int16_t* d_local_list = nullptr; // [n_local] local q heads, ascending
  __half* idx_hl = nullptr;        // [B][Hr][max_seq][2 r]: index keys split as fp16 hi | lo
  // TMA tensor maps of the prefill kernels: the split index cache as [rows][4 chunks][8 values]
  // (64-key boxes per chunk), the K and V caches as [rows][128 values] (64-key x 64-value boxes,
  // 128-byte swizzle)
  CUtensorMap tm_idx, tm_k, tm_v;
  bool tm_ready = false;
  uint2* pf_cut = nullptr;
  unsigned long long* pf_capture = nullptr;  // [B][Hr][max_chunk / 128][kPfCapture][128] selection lists
  int attn_split_max = 1;          // key splits of a prefill attention row tile (max_seq / 256K)
  float* attn_part = nullptr;      // [B][Hr][max_chunk / 128][attn_split_max][128][4 + D] partials
  uint32_t* attn_ticket = nullptr; // [B][Hr][max_chunk / 128]
  // decode: the local heads' window attention runs on a second stream, forked after the
  // selection and joined back, so it overlaps the retrieval heads' gather attention
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;         // [B][Hr][max_chunk] prefill per-row cut (t_key, tiecut)
  int n_local = 0;

  // decode scratch
  float* q_rot = nullptr;    // [B*max_rows][Hq][D] fp32 RoPE'd queries
  float* q_idx = nullptr;    // [B*max_rows][Hr][r]
  int32_t* sel_idx = nullptr;  // [B*Hr][max_select]
  int32_t* sel_cnt = nullptr;  // [B*Hr]
  float* sel_mass = nullptr;   // [B*Hr]
  float* sel_thr = nullptr;    // [B*Hr]
  float* seg_max = nullptr;    // [P + G]
  uint32_t* sel_words = nullptr;  // [12][P][bins]: level-1 and radix histograms (lo, hi, count)
  uint32_t* cand_cnt = nullptr;   // [P]
  unsigned long long* cand = nullptr;  // [P][kSelCand]
  uint32_t* sel_keep = nullptr;   // [P][max_seq] keep lists of the selection (global-score mode)
  uint32_t* sel_flags = nullptr;  // [1] radix fallback flag (the epoch of the launch that set it)
  uint32_t sel_epoch = 0;         // launches of the decode selection (its flag epochs)
  uint32_t* sel_cum = nullptr;    // [P + G][1024] cumulative fine-bin counts per (problem, CTA)
  unsigned long long* sel_psum = nullptr;   // [P][8] per-problem crossing summaries and cut keys
  long long* sel_cres = nullptr;            // [P + G][2] per-(problem, CTA) compaction offsets
  uint32_t* sel_pticket = nullptr;          // [P] phase completion tickets
  uint32_t* slot_cnt = nullptr;  // [P + G][2]
  unsigned long long* bar = nullptr;  // [2] grid barrier arrival / exit counters
  float* gscores = nullptr;      // [P][max_seq] when scores do not fit in shared memory
  size_t gscores_elems = 0;
  float* gpart = nullptr;        // gather partials [items][D + 2]
  int64_t gpart_items = 0;
  uint32_t* gticket = nullptr;   // [B*Hr]
  float* spart = nullptr;        // window partials
  int64_t spart_elems = 0;
  uint32_t* sticket = nullptr;   // [B*Hkv]
  uint32_t* err = nullptr;       // device error word
  long long wait_limit = 0;      // decode grid-barrier wait limit in cycles (0: the default, ~1 s)

  // K-cache clustering of the index keys (n_clusters > 0, bf16 index keys)
  int n_clusters = 0;
  bool cl_ready = false;                 // centres and assignments valid (rtp_cluster_build)
  std::vector<int64_t> cl_len;           // [B] keys clustered per sequence
  double* cl_cent = nullptr;             // [P][K][r] fp64 centres
  int32_t* cl_count = nullptr;           // [P][K] cluster sizes
  uint16_t* cl_assign = nullptr;         // [P][cl_stride] cluster of each clustered key
  int64_t cl_stride = 0;                 // max_seq rounded up to 16 entries (32-byte rows)
  unsigned long long* cl_sum = nullptr;  // [P][K][r] integer centre sums (two's complement)
  unsigned long long* cl_acc = nullptr;  // [P][K] counts being accumulated
  uint8_t* cl_hit = nullptr;             // [P][K] clusters hit by the current decode query
  unsigned long long* cl_flags = nullptr;  // [P][max_seq / 4096] compaction chunk flags
  uint32_t* cl_ctr = nullptr;              // [P][2] compaction chunk counter, finished chunks
  uint32_t cl_epoch = 0;                   // compaction launches (flag epochs, 24 bits)

  // per-kernel event timing (rtp_profile_enable)
  bool prof_on = false;
  std::map<std::string, std::vector<std::pair<cudaEvent_t, cudaEvent_t>>> prof;
  std::vector<cudaEvent_t> prof_pool;

  std::string last_error;
};

namespace rtp {

// Scoped event pair around one kernel launch when profiling is on.
struct ProfScope {
  rtp_layer* L;
  const char* name;
  cudaStream_t st;
  cudaEvent_t e0 = nullptr;
  ProfScope(rtp_layer* L_, const char* n, cudaStream_t s);
  ~ProfScope();
};

rtp_status fail(rtp_layer* L, rtp_status st, const std::string& msg);
rtp_status cuda_fail(rtp_layer* L, cudaError_t e, const char* what);

// Kernel launchers (return cudaGetLastError() of the launch).
// per-sequence lengths plus delta (a sequence's decode row: delta -1; first prefill row: -C)
SeqPos seq_pos(const rtp_layer* L, int64_t delta);
// append T tokens to sequences b0 .. b0 + nb - 1 (k, v: [nb][T][Hkv][D]) at their own lengths
cudaError_t launch_append_kv(const rtp_layer* L, const __nv_bfloat16* k, const __nv_bfloat16* v, int T, int b0,
                             int nb, cudaStream_t st);
cudaError_t launch_q_prep(const rtp_layer* L, const __nv_bfloat16* q, int rows, const SeqPos& pos0,
                          cudaStream_t st);
// q_raw: the decode queries ([B][Hq][D] bf16): the kernel then also writes q_rot and forms its
// own index queries (no q_prep launch); NULL: it reads q_idx written by q_prep
cudaError_t launch_decode_select(rtp_layer* L, const __nv_bfloat16* q_raw, cudaStream_t st);
cudaError_t launch_decode_topk(rtp_layer* L, cudaStream_t st);
cudaError_t launch_prefill_dense_retrieval(const rtp_layer* L, int C, float* out, cudaStream_t st);
cudaError_t launch_prefill_dense_stats(const rtp_layer* L, int C, int32_t* cnt, float* mass, cudaStream_t st);
// flat: the streaming kernel for long lists (p = 1, fixed top-k, clustered selection); else the
// item kernel for the short lists of per-key top-p
cudaError_t launch_decode_gather(const rtp_layer* L, bool dense, bool flat, float* out, cudaStream_t st);
cudaError_t launch_dense_stats(const rtp_layer* L, cudaStream_t st);
cudaError_t launch_iota_rows(const rtp_layer* L, int32_t* dst, int64_t cap, cudaStream_t st);
cudaError_t launch_decode_swa(const rtp_layer* L, float* out, cudaStream_t st);
// K-cache clustering: `iters` k-means passes over every sequence's keys 0 .. len_b - 1, and the
// clustered decode selection (sel_idx, sel_cnt, sel_mass, sel_thr)
cudaError_t launch_cluster_build(rtp_layer* L, int iters, cudaStream_t st);
cudaError_t launch_cluster_select(rtp_layer* L, cudaStream_t st);
int64_t cluster_chunks(int64_t max_seq);
cudaError_t launch_prefill_local(const rtp_layer* L, int C, float* out, cudaStream_t st);
cudaError_t launch_prefill_retrieval(rtp_layer* L, int C, float* out, const rtp_prefill_stats* stats,
                                     cudaStream_t st);

// Selection kernel geometry for the current length (host-side; also sizes scratch).
struct SelectGeom {
  int grid = 0;
  int64_t per_cta = 0;  // keys of the longest CTA range
  int64_t pair = 0;     // keys per CTA pair
  int64_t even = 0;     // keys of the even member of a pair
  bool parity = false;  // pairs split unevenly (by SM number, one CTA on every SM)
  bool smem_scores = true;
  size_t smem_bytes = 0;
};
SelectGeom select_geometry(const rtp_layer* L, int64_t N);
size_t select_fixed_smem();
size_t select_var_smem(int64_t per);

}  // namespace rtp
