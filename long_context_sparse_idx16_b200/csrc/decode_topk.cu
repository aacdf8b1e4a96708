// decode_topk.cu -- fixed top-k selection in decode (the pages' fixed-budget ablation).
//
// The techwalker page (section 4 and its Q&A) sets the dynamic top-p budget against a fixed
// one: every query keeps its k highest-scoring tokens (4096 or 16384 in the ablation), whatever
// their attention mass.  With the layer's top_k > 0 each retrieval head of a decode step keeps
// the first min(k, N) keys of the order (s desc, j asc) instead of the top-p set; the sparse
// attention over the list is unchanged.
//
// An exact radix select over the scores' order keys, 8 bits per level, in plain kernels (no
// grid-wide waits):
//   score  -- index scores of 4096-key chunks (the same 16-dim dot products as the top-p
//             stream), stored as order keys, with the histogram of their top 8 bits;
//   hist   -- three more levels: each CTA recomputes the digits fixed so far from the
//             histograms (a scan of at most 4 x 256 counts), then histograms the next 8 bits
//             of the keys that match them;
//   count  -- after four levels the cut key t and the number of tied keys to take are exact;
//             each chunk counts its keys above t and equal to t;
//   write  -- each chunk's output offset from the counts of the chunks before it, then an
//             ordered compaction: the list holds the keys above t and the first tied keys
//             (lowest positions), ascending.
#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr int kTkThreads = 256;
constexpr int kTkPer = kTopkChunk / kTkThreads;  // keys per thread in a chunk (16)
constexpr int kTkLevels = 4;

struct TopkArgs {
  const float* idx;             // fp32 index keys [P][pstride], or
  const __nv_bfloat16* idx_b;   // bf16 index keys
  int64_t idx_pstride;
  const float* q_idx;           // [P][r]
  int P, Hr;
  SeqPos lens;  // each sequence's length: problem p sees keys 0 .. lens[p / Hr] - 1
  int64_t k;
  int nchunks;
  uint32_t* keys;               // [P][max_seq] order keys of the scores
  int64_t keys_pstride;
  uint32_t* hist;               // [P][4][256]
  uint32_t* cnt;                // [P][nchunks][2]: keys above the cut, keys tied at it
  int32_t* sel_idx;
  int64_t max_select;
  int32_t* sel_cnt;
  float* sel_mass;
  float* sel_thr;
  uint32_t* err;
};

// Digits fixed by the first `levels` levels of problem p, and how many keys are still needed
// among the keys that match them (counted from the highest key down).
__device__ __forceinline__ int64_t nkeys(const TopkArgs& a, int p) { return a.lens.v[p / a.Hr]; }

__device__ void topk_state(const TopkArgs& a, int p, int levels, uint32_t* prefix, uint32_t* mask, int64_t* rem) {
  int64_t need = min(a.k, nkeys(a, p));
  uint32_t pre = 0u, msk = 0u;
  for (int l = 0; l < levels; ++l) {
    const uint32_t* h = a.hist + ((int64_t)p * kTkLevels + l) * 256;
    int64_t cum = 0;
    int d = 255;
    for (; d > 0; --d) {
      const uint32_t c = __ldcg(h + d);
      if (cum + c >= need) break;
      cum += c;
    }
    need -= cum;
    const int sh = 24 - 8 * l;
    pre |= (uint32_t)d << sh;
    msk |= 0xFFu << sh;
  }
  *prefix = pre;
  *mask = msk;
  *rem = need;
}

template <bool kBf16>
__global__ void __launch_bounds__(kTkThreads) topk_score_kernel(TopkArgs a) {
  __shared__ uint32_t h[256];
  __shared__ float q[kR];
  const int p = blockIdx.y, tid = threadIdx.x;
  const int64_t j0 = (int64_t)blockIdx.x * kTopkChunk;
  h[tid] = 0u;
  if (tid < kR) q[tid] = a.q_idx[(int64_t)p * kR + tid];
  __syncthreads();
  uint32_t* keys = a.keys + (int64_t)p * a.keys_pstride;
#pragma unroll 4
  for (int u = 0; u < kTkPer; ++u) {
    const int64_t j = j0 + u * kTkThreads + tid;
    if (j >= nkeys(a, p)) break;
    float s;
    if constexpr (kBf16) {
      const uint4* row = reinterpret_cast<const uint4*>(a.idx_b + (int64_t)p * a.idx_pstride + j * kR);
      s = 0.f;
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const uint4 w = row[v];
        const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(hb[e]);
          s = fmaf(f.x, q[8 * v + 2 * e], s);
          s = fmaf(f.y, q[8 * v + 2 * e + 1], s);
        }
      }
    } else {
      const float4* row = reinterpret_cast<const float4*>(a.idx + (int64_t)p * a.idx_pstride + j * kR);
      s = 0.f;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float4 w = row[v];
        s = fmaf(w.x, q[4 * v], s);
        s = fmaf(w.y, q[4 * v + 1], s);
        s = fmaf(w.z, q[4 * v + 2], s);
        s = fmaf(w.w, q[4 * v + 3], s);
      }
    }
    const uint32_t key = order_key(s + 0.0f);  // -0 -> +0: equal scores, equal keys
    keys[j] = key;
    atomicAdd(&h[key >> 24], 1u);
  }
  __syncthreads();
  if (h[tid]) atomicAdd(a.hist + (int64_t)p * kTkLevels * 256 + tid, h[tid]);
}

__global__ void __launch_bounds__(kTkThreads) topk_hist_kernel(TopkArgs a, int level) {
  __shared__ uint32_t h[256];
  __shared__ uint32_t s_pre, s_msk;
  const int p = blockIdx.y, tid = threadIdx.x;
  const int64_t j0 = (int64_t)blockIdx.x * kTopkChunk;
  h[tid] = 0u;
  if (tid == 0) {
    uint32_t pre, msk;
    int64_t rem;
    topk_state(a, p, level, &pre, &msk, &rem);
    s_pre = pre;
    s_msk = msk;
  }
  __syncthreads();
  const uint32_t pre = s_pre, msk = s_msk;
  const int sh = 24 - 8 * level;
  const uint32_t* keys = a.keys + (int64_t)p * a.keys_pstride;
#pragma unroll 4
  for (int u = 0; u < kTkPer; ++u) {
    const int64_t j = j0 + u * kTkThreads + tid;
    if (j >= nkeys(a, p)) break;
    const uint32_t key = keys[j];
    if ((key & msk) == pre) atomicAdd(&h[(key >> sh) & 0xFFu], 1u);
  }
  __syncthreads();
  if (h[tid]) atomicAdd(a.hist + ((int64_t)p * kTkLevels + level) * 256 + tid, h[tid]);
}

__device__ __forceinline__ void block_counts(uint32_t* red, uint32_t above, uint32_t eq, uint32_t* tot_above,
                                             uint32_t* tot_eq) {
  above = warp_sum(above);
  eq = warp_sum(eq);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    red[w] = above;
    red[8 + w] = eq;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t x = 0u, y = 0u;
    for (int i = 0; i < kTkThreads / 32; ++i) {
      x += red[i];
      y += red[8 + i];
    }
    *tot_above = x;
    *tot_eq = y;
  }
}

__global__ void __launch_bounds__(kTkThreads) topk_count_kernel(TopkArgs a) {
  __shared__ uint32_t red[16];
  __shared__ uint32_t s_t;
  const int p = blockIdx.y, c = blockIdx.x, tid = threadIdx.x;
  if (tid == 0) {
    uint32_t pre, msk;
    int64_t rem;
    topk_state(a, p, kTkLevels, &pre, &msk, &rem);
    s_t = pre;
  }
  __syncthreads();
  const uint32_t t = s_t;
  const int64_t j0 = (int64_t)c * kTopkChunk;
  const uint32_t* keys = a.keys + (int64_t)p * a.keys_pstride;
  uint32_t above = 0u, eq = 0u;
  for (int u = 0; u < kTkPer; ++u) {
    const int64_t j = j0 + u * kTkThreads + tid;
    if (j >= nkeys(a, p)) break;
    const uint32_t key = keys[j];
    above += key > t ? 1u : 0u;
    eq += key == t ? 1u : 0u;
  }
  uint32_t ta, te;
  block_counts(red, above, eq, &ta, &te);
  if (tid == 0) {
    a.cnt[((int64_t)p * a.nchunks + c) * 2] = ta;
    a.cnt[((int64_t)p * a.nchunks + c) * 2 + 1] = te;
  }
}

// exclusive block scan of one count per thread (thread order); *total receives the sum
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t* red, uint32_t v, uint32_t* total) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (l >= o) incl += y;
  }
  __syncthreads();
  if (l == 31) red[w] = incl;
  __syncthreads();
  uint32_t base = 0u, tot = 0u;
  for (int i = 0; i < kTkThreads / 32; ++i) {
    if (i < w) base += red[i];
    tot += red[i];
  }
  *total = tot;
  return base + incl - v;
}

__global__ void __launch_bounds__(kTkThreads) topk_write_kernel(TopkArgs a) {
  __shared__ uint32_t red[8];
  __shared__ uint32_t s_t;
  __shared__ long long s_before, s_eqbefore, s_need;
  const int p = blockIdx.y, c = blockIdx.x, tid = threadIdx.x;
  if (tid == 0) {
    uint32_t pre, msk;
    int64_t rem;
    topk_state(a, p, kTkLevels, &pre, &msk, &rem);
    s_t = pre;
    s_need = rem;  // tied keys (== t) to take, lowest positions first
    long long before = 0, eqb = 0;
    for (int cc = 0; cc < c; ++cc) {
      const long long ga = __ldcg(a.cnt + ((int64_t)p * a.nchunks + cc) * 2);
      const long long ge = __ldcg(a.cnt + ((int64_t)p * a.nchunks + cc) * 2 + 1);
      long long take = rem - eqb;
      take = take < 0 ? 0 : (take > ge ? ge : take);
      before += ga + take;
      eqb += ge;
    }
    s_before = before;
    s_eqbefore = eqb;
    if (c == a.nchunks - 1) {
      const int64_t K = min(a.k, nkeys(a, p));
      if (K > a.max_select) atomicOr(a.err, kErrOverflow);
      a.sel_cnt[p] = (int32_t)(K < a.max_select ? K : a.max_select);
      if (a.sel_mass) a.sel_mass[p] = -1.f;  // the fixed budget does not sum masses
      if (a.sel_thr) a.sel_thr[p] = -1.f;
    }
  }
  __syncthreads();
  const uint32_t t = s_t;
  const long long need = s_need;
  // thread tid owns the kTkPer consecutive keys j0 + kTkPer * tid ..
  const int64_t j0 = (int64_t)c * kTopkChunk + (int64_t)kTkPer * tid;
  const uint32_t* keys = a.keys + (int64_t)p * a.keys_pstride;
  uint32_t kv[kTkPer];
  uint32_t above = 0u, eq = 0u;
#pragma unroll
  for (int i = 0; i < kTkPer; ++i) {
    const int64_t j = j0 + i;
    const bool in = j < nkeys(a, p);
    kv[i] = in ? keys[j] : 0u;
    above += (in && kv[i] > t) ? 1u : 0u;
    eq += (in && kv[i] == t) ? 1u : 0u;
  }
  uint32_t tot;
  const uint32_t eq_base = block_excl_scan(red, eq, &tot);
  long long tie_rank = s_eqbefore + eq_base;  // tied keys before this thread's first key
  // selected keys of this thread: those above t, and ties while their rank is below need
  uint32_t mine = above;
  {
    const long long take = need - tie_rank;
    mine += (uint32_t)(take <= 0 ? 0 : (take > eq ? eq : take));
  }
  const uint32_t out_base = block_excl_scan(red, mine, &tot);
  long long o = s_before + out_base;
  int32_t* dst = a.sel_idx + (int64_t)p * a.max_select;
#pragma unroll
  for (int i = 0; i < kTkPer; ++i) {
    const int64_t j = j0 + i;
    if (j >= nkeys(a, p)) break;
    bool sel = kv[i] > t;
    if (kv[i] == t) {
      sel = tie_rank < need;
      ++tie_rank;
    }
    if (sel) {
      if (o < a.max_select) dst[o] = (int32_t)j;
      ++o;
    }
  }
}

}  // namespace

cudaError_t launch_decode_topk(rtp_layer* L, cudaStream_t st) {
  TopkArgs a;
  a.idx = L->idx;
  a.idx_b = L->idx_b;
  a.idx_pstride = L->max_seq * kR;
  a.q_idx = L->q_idx;
  a.P = L->B * L->Hr;
  a.Hr = L->Hr;
  a.lens = seq_pos(L, 0);
  a.k = L->top_k;
  a.nchunks = (int)((L->len + kTopkChunk - 1) / kTopkChunk);
  a.keys = L->tk_keys;
  a.keys_pstride = L->max_seq;
  a.hist = L->tk_hist;
  a.cnt = L->tk_cnt;
  a.sel_idx = L->sel_idx;
  a.max_select = L->max_select;
  a.sel_cnt = L->sel_cnt;
  a.sel_mass = L->sel_mass;
  a.sel_thr = L->sel_thr;
  a.err = L->err;
  cudaError_t e = cudaMemsetAsync(L->tk_hist, 0, sizeof(uint32_t) * (size_t)a.P * kTkLevels * 256, st);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.nchunks, a.P);
  if (L->index_bf16) topk_score_kernel<true><<<grid, kTkThreads, 0, st>>>(a);
  else topk_score_kernel<false><<<grid, kTkThreads, 0, st>>>(a);
  for (int l = 1; l < kTkLevels; ++l) topk_hist_kernel<<<grid, kTkThreads, 0, st>>>(a, l);
  topk_count_kernel<<<grid, kTkThreads, 0, st>>>(a);
  topk_write_kernel<<<grid, kTkThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
