// rtp_layer.cu -- the C ABI: layer creation, validation, memory layout and call sequencing.
//
// Memory layout in HBM (one layer):
//   K cache  fp16 [B][Hkv][max_seq][128]  RoPE'd keys (written once by append)
//   V cache  fp16 [B][Hkv][max_seq][128]
//   IDX      fp32 [B][Hr][max_seq][16]    pre-RoPE index keys, one 64-byte row per key
// fp16 (not bf16) caches: values are O(1)..O(100); fp16's 11-bit significand keeps the
// rounding of RoPE'd keys, of the fp16 query and of the probabilities fed to the tensor
// cores near 2.4e-4 each, which the 1e-3 relative-L2 output tolerance needs.  Inputs stay
// bf16; bf16 -> fp16 is exact inside fp16's range, and append flags anything outside it.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <string>
#include <vector>

#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {

int64_t swa_part_elems(const rtp_layer* L);

static thread_local std::string g_create_error;

rtp_status fail(rtp_layer* L, rtp_status st, const std::string& msg) {
  if (L) L->last_error = msg;
  else g_create_error = msg;
  return st;
}

rtp_status cuda_fail(rtp_layer* L, cudaError_t e, const char* what) {
  std::string m = std::string(what) + ": " + cudaGetErrorString(e);
  return fail(L, RTP_ECUDA, m);
}

template <typename T>
static cudaError_t dalloc(T** p, size_t elems) {
  *p = nullptr;
  if (elems == 0) elems = 1;
  return cudaMalloc((void**)p, elems * sizeof(T));
}

// Selection scratch that kernels expect zeroed on entry (they re-zero it after use).
static cudaError_t reset_select_scratch(rtp_layer* L) {
  const size_t P = (size_t)L->B * L->Hr > 0 ? (size_t)L->B * L->Hr : 1;
  cudaError_t e = cudaMemset(L->sel_words, 0, 12 * P * kSelBins * sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(L->cand_cnt, 0, P * sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(L->bar, 0, 2 * sizeof(unsigned long long));
  if (e == cudaSuccess) e = cudaMemset(L->sel_flags, 0, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(L->sel_pticket, 0, P * sizeof(uint32_t));
  return e;
}

static cudaEvent_t prof_event(rtp_layer* L) {
  if (!L->prof_pool.empty()) {
    cudaEvent_t e = L->prof_pool.back();
    L->prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

ProfScope::ProfScope(rtp_layer* L_, const char* n, cudaStream_t s) : L(L_), name(n), st(s) {
  if (L && L->prof_on) {
    e0 = prof_event(L);
    cudaEventRecord(e0, st);
  }
}

ProfScope::~ProfScope() {
  if (e0) {
    cudaEvent_t e1 = prof_event(L);
    cudaEventRecord(e1, st);
    L->prof[name].push_back({e0, e1});
  }
}

static void prof_release(rtp_layer* L) {
  for (auto& kv : L->prof)
    for (auto& pr : kv.second) {
      cudaEventDestroy(pr.first);
      cudaEventDestroy(pr.second);
    }
  L->prof.clear();
  for (cudaEvent_t e : L->prof_pool) cudaEventDestroy(e);
  L->prof_pool.clear();
}

static void free_all(rtp_layer* L) {
  prof_release(L);
  if (L->ev_fork) cudaEventDestroy(L->ev_fork);
  if (L->ev_join) cudaEventDestroy(L->ev_join);
  if (L->side) cudaStreamDestroy(L->side);
  L->ev_fork = L->ev_join = nullptr;
  L->side = nullptr;
  void* ptrs[] = {L->kc, L->vc, L->idx, L->idx_b, L->wq, L->wk, L->theta, L->d_head_slot, L->d_ret_head,
                  L->d_loc_head, L->d_loc_cnt, L->d_local_list, L->pf_cut, L->idx_hl, L->q_rot, L->q_idx, L->sel_idx, L->sel_cnt,
                  L->sel_mass, L->sel_thr, L->seg_max, L->sel_words, L->cand_cnt, L->cand,
                  L->sel_keep, L->sel_flags, L->slot_cnt, L->bar, L->gscores, L->gpart, L->gticket, L->spart,
                  L->sticket, L->err, L->tk_keys, L->tk_hist, L->tk_cnt, L->pf_capture, L->attn_part,
                  L->attn_ticket, L->sel_cum, L->sel_psum, L->sel_pticket, L->sel_cres, L->cl_cent,
                  L->cl_count, L->cl_assign, L->cl_sum, L->cl_acc, L->cl_hit, L->cl_flags, L->cl_ctr};
  for (void* p : ptrs)
    if (p) cudaFree(p);
}

}  // namespace rtp

namespace rtp {
namespace {
// With dense retrieval prefill row i of sequence b (position P0_b + i) keeps all its
// P0_b + i + 1 causal keys.
__global__ void prefill_dense_stats_kernel(int32_t* cnt, float* mass, int C, int Hr, const SeqPos P0, int64_t n) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n) return;
  const int64_t i = (t / Hr) % C, b = t / ((int64_t)Hr * C);
  if (cnt) cnt[t] = (int32_t)(P0.v[b] + i + 1);
  if (mass) mass[t] = 1.f;
}
}  // namespace

cudaError_t launch_prefill_dense_stats(const rtp_layer* L, int C, int32_t* cnt, float* mass, cudaStream_t st) {
  const int64_t n = (int64_t)L->B * C * L->Hr;
  prefill_dense_stats_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(cnt, mass, C, L->Hr, seq_pos(L, -C), n);
  return cudaGetLastError();
}
}  // namespace rtp

using namespace rtp;

extern "C" {

rtp_status rtp_create(const rtp_config* cfg, rtp_layer** out) {
  if (!cfg || !out) return fail(nullptr, RTP_EINVAL, "rtp_create: NULL argument");
  *out = nullptr;
  const rtp_config& c = *cfg;
  if (c.batch < 1 || c.n_q_heads < 1 || c.n_kv_heads < 1 || c.n_q_heads % c.n_kv_heads != 0)
    return fail(nullptr, RTP_EINVAL, "rtp_create: need batch >= 1 and n_kv_heads dividing n_q_heads");
  if (c.batch > kMaxBatch) return fail(nullptr, RTP_EINVAL, "rtp_create: at most 256 sequences");
  if (c.head_dim != kD || c.index_dim != kR)
    return fail(nullptr, RTP_EINVAL, "rtp_create: head_dim must be 128 and index_dim 16");
  if (c.n_q_heads / c.n_kv_heads > kMaxGroup)
    return fail(nullptr, RTP_EINVAL, "rtp_create: at most 16 query heads per KV head");
  if (c.max_seq < 1 || c.max_seq > (int64_t)INT32_MAX)
    return fail(nullptr, RTP_EINVAL, "rtp_create: max_seq must be in [1, 2^31)");
  if (!c.head_class) return fail(nullptr, RTP_EINVAL, "rtp_create: head_class is NULL");
  if (!(c.top_p > 0.f && c.top_p <= 1.f)) return fail(nullptr, RTP_EINVAL, "rtp_create: top_p must be in (0, 1]");
  if (c.window < 1 || c.n_sink < 0) return fail(nullptr, RTP_EINVAL, "rtp_create: need window >= 1, n_sink >= 0");
  if (!(c.rope_base > 1.0)) return fail(nullptr, RTP_EINVAL, "rtp_create: rope_base must be > 1");
  if (c.sm_scale < 0.f) return fail(nullptr, RTP_EINVAL, "rtp_create: sm_scale must be >= 0");
  if (c.max_select < 0 || c.max_select > c.max_seq)
    return fail(nullptr, RTP_EINVAL, "rtp_create: max_select must be in [0, max_seq]");
  if (c.max_chunk < 0) return fail(nullptr, RTP_EINVAL, "rtp_create: max_chunk must be >= 0");
  if (c.index_bf16 != 0 && c.index_bf16 != 1) return fail(nullptr, RTP_EINVAL, "rtp_create: index_bf16 must be 0 or 1");
  if (c.prefill_dense != 0 && c.prefill_dense != 1)
    return fail(nullptr, RTP_EINVAL, "rtp_create: prefill_dense must be 0 or 1");
  if (c.top_k < 0) return fail(nullptr, RTP_EINVAL, "rtp_create: top_k must be >= 0");
  if (c.n_clusters < 0 || c.n_clusters > 1024)
    return fail(nullptr, RTP_EINVAL, "rtp_create: n_clusters must be in [0, 1024]");
  if (c.n_clusters > 0 && (c.index_bf16 != 1 || c.top_k != 0))
    return fail(nullptr, RTP_EINVAL, "rtp_create: n_clusters needs index_bf16 = 1 and top_k = 0");

  rtp_layer* L = new rtp_layer();
  L->B = c.batch;
  L->lens.assign((size_t)c.batch, 0);
  L->Hq = c.n_q_heads;
  L->Hkv = c.n_kv_heads;
  L->group = c.n_q_heads / c.n_kv_heads;
  L->max_seq = c.max_seq;
  L->max_select = c.max_select ? c.max_select : c.max_seq;
  L->max_chunk = c.max_chunk ? c.max_chunk : 16384;
  L->index_bf16 = c.index_bf16 == 1;
  L->prefill_dense = c.prefill_dense == 1;
  L->top_k = c.top_k;
  L->n_clusters = c.n_clusters;
  L->cl_len.assign((size_t)c.batch, 0);
  L->top_p = c.top_p;
  L->sm_scale = c.sm_scale > 0.f ? c.sm_scale : 1.0f / sqrtf((float)kD);
  L->rope_base = c.rope_base;
  L->W = c.window;
  L->S = c.n_sink;
  L->head_slot.assign(L->Hq, -1);
  std::vector<int16_t> loc_head((size_t)L->Hkv * kMaxGroup, (int16_t)-1);
  std::vector<int32_t> loc_cnt(L->Hkv, 0);
  for (int h = 0; h < L->Hq; ++h) {
    if (c.head_class[h] > 1) {
      delete L;
      return fail(nullptr, RTP_EINVAL, "rtp_create: head_class entries must be 0 or 1");
    }
    if (c.head_class[h] == 1) {
      L->head_slot[h] = (int)L->ret_heads.size();
      L->ret_heads.push_back(h);
    } else {
      const int g = h / L->group;
      loc_head[(size_t)g * kMaxGroup + loc_cnt[g]++] = (int16_t)h;
      ++L->n_local;
    }
  }
  L->Hr = (int)L->ret_heads.size();
  if (L->Hr > 0 && (!c.wq_index || !c.wk_index)) {
    delete L;
    return fail(nullptr, RTP_EINVAL, "rtp_create: retrieval heads need wq_index and wk_index");
  }
  if ((int64_t)L->B * L->Hr > 2048) {
    delete L;
    return fail(nullptr, RTP_EINVAL, "rtp_create: batch * retrieval heads must be <= 2048");
  }
  cudaError_t e = cudaGetDevice(&L->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&L->sm_count, cudaDevAttrMultiProcessorCount, L->device);
  int optin = 0;
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, L->device);
  if (e != cudaSuccess) {
    delete L;
    return cuda_fail(nullptr, e, "rtp_create: device query");
  }
  L->smem_optin = (size_t)optin;

  const int64_t B = L->B, Hkv = L->Hkv, Hr = L->Hr, Hq = L->Hq, P = B * Hr;
  const int64_t rows = B * L->max_chunk;
  const int64_t G = L->sm_count;
  // Largest per-CTA score count the shared-memory variant can hold; beyond it the
  // selection keeps scores in global scratch.
  const int64_t smem_cap = ((int64_t)L->smem_optin - (int64_t)select_fixed_smem() - 2 * 32 * 34 - 2) * 4 / 19;
  const bool need_gscores = P * L->max_seq > smem_cap * G;
  // gather partials: the item kernel's items (at most 64 per problem), or two per CTA of the
  // flat kernel
  const int64_t gchunks = (L->max_seq + kGatherChunk - 1) / kGatherChunk;
  const int64_t gitems_i = P * (gchunks < kGatherMaxItems ? gchunks : kGatherMaxItems);
  const int64_t gitems = gitems_i > 2 * G ? gitems_i : 2 * G;

#define RTP_ALLOC(ptr, n)                                         \
  do {                                                            \
    if (e == cudaSuccess) e = dalloc(&(ptr), (size_t)(n));         \
  } while (0)
  e = cudaSuccess;
  RTP_ALLOC(L->kc, B * Hkv * L->max_seq * kD);
  RTP_ALLOC(L->vc, B * Hkv * L->max_seq * kD);
  if (L->top_k > 0 && Hr > 0) {
    RTP_ALLOC(L->tk_keys, P * L->max_seq);
    RTP_ALLOC(L->tk_hist, P * 4 * 256);
    RTP_ALLOC(L->tk_cnt, P * 2 * ((L->max_seq + kTopkChunk - 1) / kTopkChunk));
  }
  if (L->index_bf16) RTP_ALLOC(L->idx_b, P * L->max_seq * kR);
  else RTP_ALLOC(L->idx, P * L->max_seq * kR);
  RTP_ALLOC(L->wq, Hr * kD * kR);
  RTP_ALLOC(L->wk, Hr * kD * kR);
  RTP_ALLOC(L->theta, kHalfD);
  RTP_ALLOC(L->d_head_slot, Hq);
  RTP_ALLOC(L->d_ret_head, Hr);
  RTP_ALLOC(L->d_loc_head, Hkv * kMaxGroup);
  RTP_ALLOC(L->d_loc_cnt, Hkv);
  RTP_ALLOC(L->d_local_list, L->n_local);
  RTP_ALLOC(L->idx_hl, (int64_t)B * Hr * L->max_seq * 2 * kR);
  RTP_ALLOC(L->pf_cut, (int64_t)B * (Hr > 0 ? Hr : 1) * L->max_chunk);
  if (Hr > 0 && !L->prefill_dense) {
    const int64_t row_tiles = (L->max_chunk + 127) / 128;
    RTP_ALLOC(L->pf_capture, (int64_t)B * Hr * row_tiles * kPfCapture * 128);
    const int64_t key_tiles = (L->max_seq + 63) / 64;
    L->attn_split_max = (int)((key_tiles + kAttSplitTiles - 1) / kAttSplitTiles);
    if (L->attn_split_max > 1) {
      RTP_ALLOC(L->attn_part, (int64_t)B * Hr * row_tiles * L->attn_split_max * 128 * (4 + kD));
      RTP_ALLOC(L->attn_ticket, (int64_t)B * Hr * row_tiles);
      if (e == cudaSuccess) e = cudaMemset(L->attn_ticket, 0, sizeof(uint32_t) * (size_t)(B * Hr * row_tiles));
    }
  }
  RTP_ALLOC(L->q_rot, rows * Hq * kD);
  RTP_ALLOC(L->q_idx, rows * Hr * kR);
  RTP_ALLOC(L->sel_idx, P * L->max_select);
  RTP_ALLOC(L->sel_cnt, P);
  RTP_ALLOC(L->sel_mass, P);
  RTP_ALLOC(L->sel_thr, P);
  RTP_ALLOC(L->seg_max, P + G);
  RTP_ALLOC(L->sel_words, 12 * P * kSelBins);
  RTP_ALLOC(L->cand_cnt, P);
  RTP_ALLOC(L->cand, P * kSelCand);
  RTP_ALLOC(L->sel_keep, P * L->max_seq);
  RTP_ALLOC(L->sel_flags, 1);
  RTP_ALLOC(L->sel_cum, (P + G) * kSelFine);
  RTP_ALLOC(L->sel_psum, 8 * P);
  RTP_ALLOC(L->sel_cres, 2 * (P + G));
  RTP_ALLOC(L->sel_pticket, P);
  RTP_ALLOC(L->slot_cnt, 2 * (P + G));
  RTP_ALLOC(L->bar, 2);
  if (L->n_clusters > 0 && Hr > 0) {
    const int64_t K = L->n_clusters;
    RTP_ALLOC(L->cl_cent, P * K * kR);
    RTP_ALLOC(L->cl_count, P * K);
    L->cl_stride = (L->max_seq + 15) / 16 * 16;
    RTP_ALLOC(L->cl_assign, P * L->cl_stride);
    RTP_ALLOC(L->cl_sum, P * K * kR);
    RTP_ALLOC(L->cl_acc, P * K);
    RTP_ALLOC(L->cl_hit, P * K);
    RTP_ALLOC(L->cl_flags, P * cluster_chunks(L->max_seq));
    RTP_ALLOC(L->cl_ctr, 2 * P);
    if (e == cudaSuccess) e = cudaMemset(L->cl_flags, 0, sizeof(unsigned long long) * (size_t)(P * cluster_chunks(L->max_seq)));
    if (e == cudaSuccess) e = cudaMemset(L->cl_ctr, 0, sizeof(uint32_t) * (size_t)(2 * P));
  }
  if (need_gscores) {
    L->gscores_elems = (size_t)(P * L->max_seq);
    RTP_ALLOC(L->gscores, L->gscores_elems);
  }
  L->gpart_items = gitems;
  RTP_ALLOC(L->gpart, gitems * (kD + 2));
  RTP_ALLOC(L->gticket, P);
  L->spart_elems = swa_part_elems(L);
  RTP_ALLOC(L->spart, L->spart_elems);
  RTP_ALLOC(L->err, 1);
#undef RTP_ALLOC
  if (e != cudaSuccess) {
    free_all(L);
    delete L;
    return fail(nullptr, RTP_ENOMEM, std::string("rtp_create: device allocation failed: ") + cudaGetErrorString(e));
  }

  // weights, maps, RoPE frequencies, zeroed counters
  std::vector<double> theta(kHalfD);
  for (int i = 0; i < kHalfD; ++i) theta[i] = pow(c.rope_base, -2.0 * (double)i / (double)kD);
  std::vector<int16_t> slot16(Hq), ret16(Hr > 0 ? Hr : 1);
  for (int h = 0; h < Hq; ++h) slot16[h] = (int16_t)L->head_slot[h];
  for (int i = 0; i < Hr; ++i) ret16[i] = (int16_t)L->ret_heads[i];
  if (Hr > 0) {
    e = cudaMemcpy(L->wq, c.wq_index, sizeof(float) * Hr * kD * kR, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(L->wk, c.wk_index, sizeof(float) * Hr * kD * kR, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(L->d_ret_head, ret16.data(), sizeof(int16_t) * Hr, cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess) e = cudaMemcpy(L->theta, theta.data(), sizeof(double) * kHalfD, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(L->d_head_slot, slot16.data(), sizeof(int16_t) * Hq, cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(L->d_loc_head, loc_head.data(), sizeof(int16_t) * Hkv * kMaxGroup, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(L->d_loc_cnt, loc_cnt.data(), sizeof(int32_t) * Hkv, cudaMemcpyHostToDevice);
  {
    std::vector<int16_t> local_list;
    for (int h = 0; h < Hq; ++h)
      if (c.head_class[h] == 0) local_list.push_back((int16_t)h);
    if (e == cudaSuccess && !local_list.empty())
      e = cudaMemcpy(L->d_local_list, local_list.data(), sizeof(int16_t) * local_list.size(), cudaMemcpyHostToDevice);
  }
  // tensor maps of the prefill kernels (the caches never move)
  {
    const uint64_t kv_rows = (uint64_t)(B * Hkv * L->max_seq);
    const uint64_t kv_dims[2] = {(uint64_t)kD, kv_rows}, kv_str[1] = {(uint64_t)kD * 2};
    const uint32_t kv_box[2] = {64u, 64u};
    bool okm = tma_encode(&L->tm_k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, L->kc, kv_dims, kv_str, kv_box,
                          CU_TENSOR_MAP_SWIZZLE_128B) &&
               tma_encode(&L->tm_v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, L->vc, kv_dims, kv_str, kv_box,
                          CU_TENSOR_MAP_SWIZZLE_128B);
    if (okm && Hr > 0) {
      const uint64_t idx_dims[3] = {8u, 4u, (uint64_t)(P * L->max_seq)}, idx_str[2] = {16u, (uint64_t)(4 * kR)};
      const uint32_t idx_box[3] = {8u, 1u, 64u};
      okm = tma_encode(&L->tm_idx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, L->idx_hl, idx_dims, idx_str, idx_box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    L->tm_ready = okm;
    if (!okm && e == cudaSuccess) e = cudaErrorInvalidValue;
  }
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&L->side, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->ev_fork, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->ev_join, cudaEventDisableTiming);
  if (e == cudaSuccess) e = reset_select_scratch(L);
  if (e == cudaSuccess) e = cudaMemset(L->gticket, 0, sizeof(uint32_t) * (P > 0 ? P : 1));
  if (e == cudaSuccess) e = cudaMemset(L->err, 0, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(L->sel_cnt, 0, sizeof(int32_t) * (P > 0 ? P : 1));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    free_all(L);
    delete L;
    return cuda_fail(nullptr, e, "rtp_create: upload");
  }
  *out = L;
  return RTP_OK;
}

rtp_status rtp_destroy(rtp_layer* L) {
  if (!L) return RTP_OK;
  cudaDeviceSynchronize();
  free_all(L);
  delete L;
  return RTP_OK;
}

namespace {
void update_len(rtp_layer* L) {
  int64_t mx = 0;
  for (int64_t n : L->lens) mx = n > mx ? n : mx;
  L->len = mx;
}
// A truncation below the clustered prefix of some sequence invalidates the clustering.
void drop_stale_clusters(rtp_layer* L) {
  for (int b = 0; b < L->B && L->cl_ready; ++b)
    if (L->lens[(size_t)b] < L->cl_len[(size_t)b]) L->cl_ready = false;
}
int64_t min_len(const rtp_layer* L) {
  int64_t mn = L->lens.empty() ? 0 : L->lens[0];
  for (int64_t n : L->lens) mn = n < mn ? n : mn;
  return mn;
}
}  // namespace

rtp_status rtp_append_kv(rtp_layer* L, const void* k, const void* v, int32_t T, cudaStream_t stream) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_append_kv: layer is NULL");
  if (!k || !v) return fail(L, RTP_EINVAL, "rtp_append_kv: k or v is NULL");
  if (T < 1) return fail(L, RTP_EINVAL, "rtp_append_kv: T must be >= 1");
  if (L->len + T > L->max_seq) return fail(L, RTP_ECAPACITY, "rtp_append_kv: max_seq exceeded");
  cudaError_t e;
  {
    ProfScope ps(L, "append_kv", stream);
    e = launch_append_kv(L, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, T, 0, L->B, stream);
  }
  if (e != cudaSuccess) return cuda_fail(L, e, "rtp_append_kv: launch");
  for (int64_t& n : L->lens) n += T;
  update_len(L);
  L->last_error.clear();
  return RTP_OK;
}

rtp_status rtp_append_kv_seq(rtp_layer* L, int32_t b, const void* k, const void* v, int32_t T,
                             cudaStream_t stream) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_append_kv_seq: layer is NULL");
  if (b < 0 || b >= L->B) return fail(L, RTP_EINVAL, "rtp_append_kv_seq: sequence index out of range");
  if (!k || !v) return fail(L, RTP_EINVAL, "rtp_append_kv_seq: k or v is NULL");
  if (T < 1) return fail(L, RTP_EINVAL, "rtp_append_kv_seq: T must be >= 1");
  if (L->lens[b] + T > L->max_seq) return fail(L, RTP_ECAPACITY, "rtp_append_kv_seq: max_seq exceeded");
  cudaError_t e;
  {
    ProfScope ps(L, "append_kv", stream);
    e = launch_append_kv(L, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, T, b, 1, stream);
  }
  if (e != cudaSuccess) return cuda_fail(L, e, "rtp_append_kv_seq: launch");
  L->lens[b] += T;
  update_len(L);
  L->last_error.clear();
  return RTP_OK;
}

rtp_status rtp_decode(rtp_layer* L, const void* q, float* out, const rtp_decode_stats* stats, cudaStream_t stream) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_decode: layer is NULL");
  if (!q || !out) return fail(L, RTP_EINVAL, "rtp_decode: q or out is NULL");
  if (min_len(L) < 1) return fail(L, RTP_EINVAL, "rtp_decode: a sequence is empty (append its token first)");
  cudaError_t e = cudaSuccess;
  // per-key top-p: the selection kernel prepares the queries itself (RoPE'd rows for the
  // attention kernels, its own index queries), so no query-prep launch precedes it
  const bool per_key = L->Hr > 0 && L->top_k == 0 && L->top_p < 1.f && !L->cl_ready;
  if (!per_key) {
    ProfScope ps(L, "q_prep", stream);
    e = launch_q_prep(L, (const __nv_bfloat16*)q, 1, seq_pos(L, -1), stream);
  }
  if (e != cudaSuccess) return cuda_fail(L, e, "rtp_decode: q_prep");
  bool forked = false;
  if (L->Hr > 0) {
    // p == 1 (without a fixed budget) keeps every causal key: the gather reads 0..len-1 directly
    const bool dense = L->top_k == 0 && L->top_p >= 1.f;
    if (!dense && L->cl_ready) {
      e = launch_cluster_select(L, stream);  // times its kernels itself ("cluster_*")
    } else {
      ProfScope ps(L, dense ? "dense_fill" : (L->top_k > 0 ? "decode_topk" : "decode_select"), stream);
      e = dense ? launch_dense_stats(L, stream)
                : (L->top_k > 0 ? launch_decode_topk(L, stream)
                                : launch_decode_select(L, (const __nv_bfloat16*)q, stream));
    }
    if (e != cudaSuccess) return cuda_fail(L, e, "rtp_decode: select");
    if (L->n_local > 0 && !L->prof_on) {  // the window attention needs only the RoPE'd queries: fork it off
      e = cudaEventRecord(L->ev_fork, stream);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(L->side, L->ev_fork, 0);
      if (e == cudaSuccess) e = launch_decode_swa(L, out, L->side);
      if (e == cudaSuccess) e = cudaEventRecord(L->ev_join, L->side);
      if (e != cudaSuccess) return cuda_fail(L, e, "rtp_decode: window attention");
      forked = true;
    }
    {
      ProfScope ps(L, "decode_gather", stream);
      e = launch_decode_gather(L, dense, dense || L->top_k > 0 || L->cl_ready, out, stream);
    }
    if (e != cudaSuccess) {
      if (forked) cudaStreamWaitEvent(stream, L->ev_join, 0);
      return cuda_fail(L, e, "rtp_decode: gather");
    }
    if (stats) {
      const size_t P = (size_t)L->B * L->Hr;
      if (stats->sel_count)
        e = cudaMemcpyAsync(stats->sel_count, L->sel_cnt, P * 4, cudaMemcpyDeviceToDevice, stream);
      if (e == cudaSuccess && stats->sel_mass)
        e = cudaMemcpyAsync(stats->sel_mass, L->sel_mass, P * 4, cudaMemcpyDeviceToDevice, stream);
      if (e == cudaSuccess && stats->threshold)
        e = cudaMemcpyAsync(stats->threshold, L->sel_thr, P * 4, cudaMemcpyDeviceToDevice, stream);
      if (e == cudaSuccess && stats->sel_index && stats->sel_index_cap > 0) {
        if (dense) {
          e = launch_iota_rows(L, stats->sel_index, stats->sel_index_cap, stream);
        } else {
          const int64_t w = stats->sel_index_cap < L->max_select ? stats->sel_index_cap : L->max_select;
          e = cudaMemcpy2DAsync(stats->sel_index, (size_t)stats->sel_index_cap * 4, L->sel_idx,
                                (size_t)L->max_select * 4, (size_t)w * 4, P, cudaMemcpyDeviceToDevice, stream);
        }
      }
      if (e != cudaSuccess) {
        if (forked) cudaStreamWaitEvent(stream, L->ev_join, 0);
        return cuda_fail(L, e, "rtp_decode: stats");
      }
    }
  }
  if (forked) {
    e = cudaStreamWaitEvent(stream, L->ev_join, 0);  // join: the output is complete in stream order
    if (e != cudaSuccess) return cuda_fail(L, e, "rtp_decode: join");
  } else if (L->n_local > 0) {
    e = launch_decode_swa(L, out, stream);  // times itself ("decode_swa", "swa_merge")
    if (e != cudaSuccess) return cuda_fail(L, e, "rtp_decode: window attention");
  }
  L->last_error.clear();
  return RTP_OK;
}

rtp_status rtp_prefill_chunk(rtp_layer* L, const void* q, int32_t C, float* out, const rtp_prefill_stats* stats,
                             cudaStream_t stream) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_prefill_chunk: layer is NULL");
  if (!q || !out) return fail(L, RTP_EINVAL, "rtp_prefill_chunk: q or out is NULL");
  if (C < 1 || C > L->max_chunk || C > min_len(L))
    return fail(L, RTP_EINVAL, "rtp_prefill_chunk: need 1 <= C <= min(shortest length, max_chunk)");
  if (stats && stats->sel_bitmap && stats->bitmap_words < 1)
    return fail(L, RTP_EINVAL, "rtp_prefill_chunk: sel_bitmap needs bitmap_words >= 1");
  if (stats && stats->rows &&
      (stats->n_rows < 1 || !stats->row_sel || stats->row_sel_cap < 1 || !stats->sel_count))
    return fail(L, RTP_EINVAL, "rtp_prefill_chunk: rows needs n_rows >= 1, row_sel, row_sel_cap >= 1 and sel_count");
  if (stats && L->prefill_dense && (stats->sel_bitmap || stats->rows))
    return fail(L, RTP_EINVAL, "rtp_prefill_chunk: with dense retrieval prefill every causal key is selected; "
                               "no bitmap or row lists are written");
  cudaError_t e;
  {
    ProfScope ps(L, "q_prep", stream);
    e = launch_q_prep(L, (const __nv_bfloat16*)q, C, seq_pos(L, -C), stream);
  }
  if (e != cudaSuccess) return cuda_fail(L, e, "rtp_prefill_chunk: q_prep");
  // with both head classes, the local heads run on the internal stream (forked after q_prep,
  // launched after the retrieval kernels) so they fill the SMs the retrieval kernels leave
  const bool fork = L->Hr > 0 && L->n_local > 0 && !L->prof_on;
  if (fork) {
    e = cudaEventRecord(L->ev_fork, stream);
    if (e != cudaSuccess) return cuda_fail(L, e, "rtp_prefill_chunk: fork");
  }
  if (L->Hr > 0 && L->prefill_dense) {
    // the pages' own prefill: retrieval heads attend to every causal key
    {
      ProfScope ps(L, "prefill_dense", stream);
      e = launch_prefill_dense_retrieval(L, C, out, stream);
    }
    if (e == cudaSuccess && stats && (stats->sel_count || stats->sel_mass))
      e = launch_prefill_dense_stats(L, C, stats->sel_count, stats->sel_mass, stream);
    if (e != cudaSuccess) return cuda_fail(L, e, "rtp_prefill_chunk: retrieval heads (dense)");
  } else if (L->Hr > 0) {
    e = launch_prefill_retrieval(L, C, out, stats, stream);  // profiled as prefill_select + prefill_attn
    if (e != cudaSuccess) return cuda_fail(L, e, "rtp_prefill_chunk: retrieval heads");
  }
  if (L->n_local > 0) {
    cudaStream_t ls = fork ? L->side : stream;
    if (fork) e = cudaStreamWaitEvent(ls, L->ev_fork, 0);
    if (e == cudaSuccess) {
      ProfScope ps(L, "prefill_local", ls);
      e = launch_prefill_local(L, C, out, ls);
    }
    if (fork && e == cudaSuccess) e = cudaEventRecord(L->ev_join, ls);
    if (fork) {
      const cudaError_t j = cudaStreamWaitEvent(stream, L->ev_join, 0);
      if (e == cudaSuccess) e = j;
    }
    if (e != cudaSuccess) return cuda_fail(L, e, "rtp_prefill_chunk: local heads");
  }
  L->last_error.clear();
  return RTP_OK;
}

rtp_status rtp_set_top_p(rtp_layer* L, float top_p) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_set_top_p: layer is NULL");
  if (!(top_p > 0.f && top_p <= 1.f)) return fail(L, RTP_EINVAL, "rtp_set_top_p: top_p must be in (0, 1]");
  L->top_p = top_p;
  return RTP_OK;
}

rtp_status rtp_set_wait_limit(rtp_layer* L, int64_t cycles) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_set_wait_limit: layer is NULL");
  if (cycles < 0) return fail(L, RTP_EINVAL, "rtp_set_wait_limit: cycles must be >= 0");
  L->wait_limit = (long long)cycles;
  return RTP_OK;
}

int64_t rtp_seq_len(const rtp_layer* L) { return L ? L->len : -1; }

int64_t rtp_seq_len_of(const rtp_layer* L, int32_t b) { return (L && b >= 0 && b < L->B) ? L->lens[b] : -1; }

rtp_status rtp_truncate(rtp_layer* L, int64_t new_len) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_truncate: layer is NULL");
  if (new_len < 0 || new_len > L->len) return fail(L, RTP_EINVAL, "rtp_truncate: need 0 <= new_len <= length");
  for (int64_t& n : L->lens) n = n < new_len ? n : new_len;
  update_len(L);
  drop_stale_clusters(L);
  return RTP_OK;
}

rtp_status rtp_truncate_seq(rtp_layer* L, int32_t b, int64_t new_len) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_truncate_seq: layer is NULL");
  if (b < 0 || b >= L->B) return fail(L, RTP_EINVAL, "rtp_truncate_seq: sequence index out of range");
  if (new_len < 0 || new_len > L->lens[b])
    return fail(L, RTP_EINVAL, "rtp_truncate_seq: need 0 <= new_len <= the sequence's length");
  L->lens[b] = new_len;
  update_len(L);
  drop_stale_clusters(L);
  return RTP_OK;
}

rtp_status rtp_cluster_build(rtp_layer* L, int32_t iters, cudaStream_t stream) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_cluster_build: layer is NULL");
  if (L->n_clusters < 1 || L->Hr < 1)
    return fail(L, RTP_EINVAL, "rtp_cluster_build: the layer has no n_clusters or no retrieval heads");
  if (iters < 0 || iters > 1000) return fail(L, RTP_EINVAL, "rtp_cluster_build: iters must be in [0, 1000]");
  for (int64_t n : L->lens) {
    if (n < L->n_clusters) return fail(L, RTP_EINVAL, "rtp_cluster_build: a sequence has fewer keys than n_clusters");
    if (n > ((int64_t)1 << 21)) return fail(L, RTP_EINVAL, "rtp_cluster_build: a sequence has more than 2^21 keys");
  }
  L->cl_ready = false;
  const cudaError_t e = launch_cluster_build(L, iters, stream);
  if (e != cudaSuccess) return cuda_fail(L, e, "rtp_cluster_build: launch");
  L->cl_len = L->lens;
  L->cl_ready = true;
  L->last_error.clear();
  return RTP_OK;
}

rtp_status rtp_cluster_drop(rtp_layer* L) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_cluster_drop: layer is NULL");
  L->cl_ready = false;
  return RTP_OK;
}

int64_t rtp_cluster_len(const rtp_layer* L, int32_t b) {
  if (!L || b < 0 || b >= L->B) return -1;
  return L->cl_ready ? L->cl_len[(size_t)b] : 0;
}

rtp_status rtp_get_clusters(const rtp_layer* L, rtp_cluster_view* view) {
  if (!L || !view) return fail(nullptr, RTP_EINVAL, "rtp_get_clusters: NULL argument");
  view->centres = L->cl_cent;
  view->counts = L->cl_count;
  view->assign = L->cl_assign;
  view->n_clusters = L->n_clusters;
  view->ready = L->cl_ready ? 1 : 0;
  view->max_seq = L->max_seq;
  view->assign_stride = L->cl_stride;
  return RTP_OK;
}

rtp_status rtp_profile_enable(rtp_layer* L, int on) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_profile_enable: layer is NULL");
  L->prof_on = on != 0;
  return RTP_OK;
}

rtp_status rtp_profile_read(rtp_layer* L, const char* kernel, double* total_ms, int64_t* launches) {
  if (!L || !total_ms || !launches) return fail(L, RTP_EINVAL, "rtp_profile_read: NULL argument");
  double ms = 0.0;
  int64_t n = 0;
  for (auto it = L->prof.begin(); it != L->prof.end();) {
    if (kernel && it->first != kernel) {
      ++it;
      continue;
    }
    for (auto& pr : it->second) {
      cudaError_t e = cudaEventSynchronize(pr.second);
      if (e != cudaSuccess) return cuda_fail(L, e, "rtp_profile_read");
      float t = 0.f;
      cudaEventElapsedTime(&t, pr.first, pr.second);
      ms += t;
      ++n;
      L->prof_pool.push_back(pr.first);
      L->prof_pool.push_back(pr.second);
    }
    it = L->prof.erase(it);
  }
  *total_ms = ms;
  *launches = n;
  return RTP_OK;
}

rtp_status rtp_reset(rtp_layer* L) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_reset: layer is NULL");
  for (int64_t& n : L->lens) n = 0;
  L->len = 0;
  L->cl_ready = false;
  return RTP_OK;
}

rtp_status rtp_check(rtp_layer* L, cudaStream_t stream) {
  if (!L) return fail(nullptr, RTP_EINVAL, "rtp_check: layer is NULL");
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(L, e, "rtp_check: stream");
  uint32_t w = 0;
  e = cudaMemcpy(&w, L->err, sizeof w, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(L, e, "rtp_check: read error word");
  if (w == 0) return RTP_OK;
  cudaMemset(L->err, 0, sizeof(uint32_t));
  if (w & kErrTimeout) {
    // a barrier gave up: its counters are inconsistent; start the next launch from zero
    reset_select_scratch(L);
    cudaMemset(L->gticket, 0, sizeof(uint32_t) * (size_t)(L->B * L->Hr > 0 ? L->B * L->Hr : 1));
    if (L->cl_ctr) cudaMemset(L->cl_ctr, 0, sizeof(uint32_t) * (size_t)(2 * L->B * L->Hr));
    if (L->attn_ticket)
      cudaMemset(L->attn_ticket, 0, sizeof(uint32_t) * (size_t)L->B * L->Hr * ((L->max_chunk + 127) / 128));
    return fail(L, RTP_ETIMEOUT, "a bounded in-kernel wait gave up");
  }
  if (w & kErrInternal) return fail(L, RTP_EINTERNAL, "an internal consistency check failed");
  if (w & kErrOverflow) return fail(L, RTP_EOVERFLOW, "a selected set exceeded max_select and was truncated");
  if (w & kErrRange) return fail(L, RTP_ERANGE, "a key or value lies outside the fp16 cache range");
  return fail(L, RTP_EINTERNAL, "unknown device error");
}

rtp_status rtp_get_cache(const rtp_layer* L, rtp_cache_view* view) {
  if (!L || !view) return fail(nullptr, RTP_EINVAL, "rtp_get_cache: NULL argument");
  view->k = L->kc;
  view->v = L->vc;
  view->idx = L->idx;
  view->idx_bf16 = L->idx_b;
  view->max_seq = L->max_seq;
  view->n_retrieval = L->Hr;
  return RTP_OK;
}

const char* rtp_last_error(const rtp_layer* L) {
  return L ? L->last_error.c_str() : g_create_error.c_str();
}

}  // extern "C"
