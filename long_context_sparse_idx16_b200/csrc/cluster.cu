// cluster.cu -- K-cache clustering of the retrieval heads' index keys and the clustered decode
// selection built on it (RTPurboV2, aitntnews page, finding 3: redundancy along the sequence,
// the two-level funnel of a coarse match against K cluster centres and exact attention inside
// the clusters hit).
//
// Clustering (rtp_cluster_build): Lloyd's k-means, per (sequence, retrieval head), of the stored
// bf16 index keys kt_j in the r = 16 index space.  The keys are put on the fixed-point grid
// 2^-27 (xq = rint(kt * 2^27) / 2^27, the integer numerators exact in int64), so a centre's sum
// is an exact integer sum in whatever order the atomics add it, and every step repeats bit for
// bit:
//   init    centre k starts at key floor((2k + 1) n / (2K));
//   assign  each key goes to the centre of least squared distance, the 16 fp64 terms (x - mu)^2
//           accumulated by fused multiply-adds in dimension order; ties to the lower centre;
//   update  every non-empty centre moves to (integer sum of its keys) / count / 2^27 (fp64,
//           correctly rounded divisions); an empty centre stays;
// and a final assignment after the last move gives the cluster sizes.
//
// Clustered decode: the centre scores c_k = q~ . mu_k (fp64, from the fp32 index query), the
// cluster weights n_k exp(c_k - max c), the clusters taken in (c desc, k asc) order while the
// weight before them is below p of the total; the selected set is every clustered key of a hit
// cluster plus every key cached after the clustering, in ascending position order (one
// single-pass compaction), which the sparse-attention gather then attends to exactly.
#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {
namespace {

constexpr double kClScale = 134217728.0;  // 2^27
constexpr double kClKeyLimit = 32768.0;   // |kt| < 2^15: sums of up to 2^21 keys stay in int64
constexpr int kClThreads = 256;
constexpr int kClAssignKeys = 256;        // keys per CTA of the assignment (one per thread)
constexpr int kClAccumKeys = 16384;       // keys per CTA of the centre-sum accumulation

// A stored bf16 index key component on the clustering grid; out-of-range values (and NaN) map
// to 0 and are reported by the accumulation kernel.
__device__ __forceinline__ double cl_grid(float f) {
  const double x = (double)f;
  return fabs(x) < kClKeyLimit ? rint(x * kClScale) / kClScale : 0.0;
}

__device__ __forceinline__ double cl_sqdist(const double* x, const double* mu) {
  double acc = 0.0;
#pragma unroll
  for (int c = 0; c < kR; ++c) {
    const double d = __dsub_rn(x[c], mu[c]);
    acc = __fma_rn(d, d, acc);
  }
  return acc;
}

__global__ void cl_init_kernel(const __nv_bfloat16* __restrict__ idx, double* __restrict__ cent,
                               unsigned long long* __restrict__ sum, unsigned long long* __restrict__ cnt, int K,
                               int Hr, int64_t max_seq, const SeqPos lens) {
  const int p = blockIdx.x;
  const int64_t n = lens.v[p / Hr];
  for (int i = threadIdx.x; i < K * kR; i += blockDim.x) {
    const int k = i / kR, c = i % kR;
    const int64_t j = ((int64_t)(2 * k + 1) * n) / (2 * (int64_t)K);
    cent[(int64_t)p * K * kR + i] = cl_grid(__bfloat162float(idx[((int64_t)p * max_seq + j) * kR + c]));
    sum[(int64_t)p * K * kR + i] = 0ull;
  }
  for (int k = threadIdx.x; k < K; k += blockDim.x) cnt[(int64_t)p * K + k] = 0ull;
}

// One key per thread against all K centres (staged in shared memory, read as broadcasts).
// Four centres per step give four independent fma chains; each chain keeps dimension order.
__global__ void __launch_bounds__(kClThreads) cl_assign_kernel(const __nv_bfloat16* __restrict__ idx,
                                                               const double* __restrict__ cent,
                                                               uint16_t* __restrict__ assign, int64_t a_stride,
                                                               int K, int Hr, int64_t max_seq, const SeqPos lens) {
  extern __shared__ double s_cent[];  // [K][r]
  const int p = blockIdx.y;
  const int64_t n = lens.v[p / Hr];
  const int64_t j0 = (int64_t)blockIdx.x * kClAssignKeys;
  if (j0 >= n) return;  // the whole CTA leaves before its only barrier
  const double2* cg = reinterpret_cast<const double2*>(cent + (int64_t)p * K * kR);
  for (int i = threadIdx.x; i < K * kR / 2; i += kClThreads) reinterpret_cast<double2*>(s_cent)[i] = cg[i];
  const int64_t j = j0 + threadIdx.x;
  double x[kR];
  if (j < n) {
    const uint4* src = reinterpret_cast<const uint4*>(idx + ((int64_t)p * max_seq + j) * kR);
    const uint4 u0 = src[0], u1 = src[1];
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // element 2i is the low half of word i
      x[2 * i] = cl_grid(__uint_as_float(w[i] << 16));
      x[2 * i + 1] = cl_grid(__uint_as_float(w[i] & 0xffff0000u));
    }
  }
  __syncthreads();
  if (j >= n) return;
  int best = 0;
  double bd = cl_sqdist(x, s_cent);
  int k = 1;
  for (; k + 3 < K; k += 4) {
    const double d0 = cl_sqdist(x, s_cent + (k + 0) * kR);
    const double d1 = cl_sqdist(x, s_cent + (k + 1) * kR);
    const double d2 = cl_sqdist(x, s_cent + (k + 2) * kR);
    const double d3 = cl_sqdist(x, s_cent + (k + 3) * kR);
    if (d0 < bd) { bd = d0; best = k; }
    if (d1 < bd) { bd = d1; best = k + 1; }
    if (d2 < bd) { bd = d2; best = k + 2; }
    if (d3 < bd) { bd = d3; best = k + 3; }
  }
  for (; k < K; ++k) {
    const double d = cl_sqdist(x, s_cent + k * kR);
    if (d < bd) { bd = d; best = k; }
  }
  assign[(int64_t)p * a_stride + j] = (uint16_t)best;
}

// Integer centre sums and counts of the current assignment: 16 lanes per key (one component
// each) add into a CTA-private shared-memory table, flushed to the global sums by atomics.
__global__ void __launch_bounds__(kClThreads) cl_accum_kernel(const __nv_bfloat16* __restrict__ idx,
                                                              const uint16_t* __restrict__ assign, int64_t a_stride,
                                                              unsigned long long* __restrict__ sum,
                                                              unsigned long long* __restrict__ cnt, int K, int Hr,
                                                              int64_t max_seq, const SeqPos lens,
                                                              uint32_t* __restrict__ err) {
  extern __shared__ unsigned long long s_sum[];  // [K][r], then [K] counts as uint32
  uint32_t* s_cnt = reinterpret_cast<uint32_t*>(s_sum + (size_t)K * kR);
  const int p = blockIdx.y;
  const int64_t n = lens.v[p / Hr];
  const int64_t j0 = (int64_t)blockIdx.x * kClAccumKeys;
  if (j0 >= n) return;
  for (int i = threadIdx.x; i < K * kR; i += kClThreads) s_sum[i] = 0ull;
  for (int i = threadIdx.x; i < K; i += kClThreads) s_cnt[i] = 0u;
  __syncthreads();
  const int c = threadIdx.x & (kR - 1);
  const int64_t jend = n < j0 + kClAccumKeys ? n : j0 + kClAccumKeys;
  bool bad = false;
  for (int64_t j = j0 + (threadIdx.x >> 4); j < jend; j += kClThreads / kR) {
    const int a = assign[(int64_t)p * a_stride + j];
    const double x = (double)__bfloat162float(idx[((int64_t)p * max_seq + j) * kR + c]);
    long long q = 0;
    if (fabs(x) < kClKeyLimit) q = (long long)rint(x * kClScale);
    else bad = true;
    if (q != 0) atomicAdd(&s_sum[a * kR + c], (unsigned long long)q);
    if (c == 0) atomicAdd(&s_cnt[a], 1u);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < K * kR; i += kClThreads)
    if (s_sum[i] != 0ull) atomicAdd(&sum[(int64_t)p * K * kR + i], s_sum[i]);
  for (int i = threadIdx.x; i < K; i += kClThreads)
    if (s_cnt[i] != 0u) atomicAdd(&cnt[(int64_t)p * K + i], (unsigned long long)s_cnt[i]);
  if (bad) atomicOr(err, kErrRange);
}

// Cluster sizes of the current assignment; with `move`, every non-empty centre moves to the
// mean of its keys.  Clears the accumulators for the next pass.
__global__ void cl_update_kernel(double* __restrict__ cent, unsigned long long* __restrict__ sum,
                                 unsigned long long* __restrict__ cnt, int32_t* __restrict__ counts, int K,
                                 int move) {
  const int p = blockIdx.x;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const int64_t pk = (int64_t)p * K + k;
    const unsigned long long m = cnt[pk];
    counts[pk] = (int32_t)m;
    for (int c = 0; c < kR; ++c) {
      if (move && m > 0ull)
        cent[pk * kR + c] = __ddiv_rn(__ddiv_rn(__ll2double_rn((long long)sum[pk * kR + c]), __ull2double_rn(m)),
                                      kClScale);
      sum[pk * kR + c] = 0ull;
    }
    cnt[pk] = 0ull;
  }
}

// ---------------------------------------------------------------- clustered decode selection

constexpr int kClSelThreads = 1024;  // one thread per cluster (K <= 1024)
constexpr int kClChunk = 4096;       // positions per CTA of the compaction

template <typename T, typename Op>
__device__ __forceinline__ T cl_block_reduce(T v, T* s_red, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();  // s_red may still be read by a previous reduction
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  v = s_red[0];
  for (int w = 1; w < nw; ++w) v = op(v, s_red[w]);
  return v;
}

struct DMax {
  __device__ double operator()(double a, double b) const { return a > b ? a : b; }
};
struct DSum {
  __device__ double operator()(double a, double b) const { return a + b; }
};
struct IMax {
  __device__ int operator()(int a, int b) const { return a > b ? a : b; }
};

// The coarse match of one problem's index query against its K centres: hit flags, the hit
// clusters' weight fraction (sel_mass) and the weight fraction of the last cluster taken
// (threshold).  A cluster's place in the (c desc, k asc) order and the weight before it come
// from a direct count over all K clusters, so no sort is needed.
__global__ void __launch_bounds__(kClSelThreads) cl_select_kernel(const float* __restrict__ q_idx,
                                                                  const double* __restrict__ cent,
                                                                  const int32_t* __restrict__ counts, int K,
                                                                  float top_p, uint8_t* __restrict__ hit,
                                                                  float* __restrict__ sel_mass,
                                                                  float* __restrict__ sel_thr) {
  __shared__ double s_c[kClSelThreads], s_w[kClSelThreads];
  __shared__ double s_red[32];
  __shared__ int s_ired[32];
  const int p = blockIdx.x, k = threadIdx.x;  // blockDim.x: K rounded up to a warp multiple
  const bool live = k < K && counts[(int64_t)p * K + k] > 0;
  double ck = -INFINITY;
  if (live) {
    const float* q = q_idx + (int64_t)p * kR;
    const double* mu = cent + ((int64_t)p * K + k) * kR;
    double acc = 0.0;
#pragma unroll
    for (int c = 0; c < kR; ++c) acc = __dadd_rn(acc, __dmul_rn((double)q[c], mu[c]));
    ck = acc;
  }
  const double cmax = cl_block_reduce(ck, s_red, DMax());
  const double wk = live ? (double)counts[(int64_t)p * K + k] * exp(ck - cmax) : 0.0;
  s_c[k] = ck;
  s_w[k] = wk;
  const double tot = cl_block_reduce(wk, s_red, DSum());  // its barriers publish s_c, s_w
  double before = 0.0;
  int rank = 0;
  if (live) {
    for (int o = 0; o < K; ++o) {
      const double co = s_c[o];
      if (o != k && co != -INFINITY && (co > ck || (co == ck && o < k))) {  // -inf: empty cluster
        before += s_w[o];
        ++rank;
      }
    }
  }
  const bool h = live && (top_p >= 1.f || before / tot < (double)top_p);
  if (k < K) hit[(int64_t)p * K + k] = h ? 1 : 0;
  const double mass = cl_block_reduce(h ? wk : 0.0, s_red, DSum());
  const int last = cl_block_reduce(h ? rank : -1, s_ired, IMax());
  if (k == 0) sel_mass[p] = (float)(mass / tot);
  if (h && rank == last) sel_thr[p] = (float)(wk / tot);
}

constexpr int kClPer = kClChunk / kClThreads;  // consecutive positions per thread of a chunk

// The assignments of positions jb .. jb + 15 (jb a multiple of 16; rows padded to 16 entries),
// loaded as two 16-byte vectors when any of them is clustered.
__device__ __forceinline__ void cl_load16(const uint16_t* __restrict__ asg, uint16_t* av, int64_t jb, int64_t ncl) {
  uint4 u0 = make_uint4(0, 0, 0, 0), u1 = u0;
  if (jb < ncl) {
    const uint4* src = reinterpret_cast<const uint4*>(asg + jb);
    u0 = __ldg(src);
    u1 = __ldg(src + 1);
  }
  const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    av[2 * i] = (uint16_t)(w[i] & 0xffffu);
    av[2 * i + 1] = (uint16_t)(w[i] >> 16);
  }
}

// Selected positions of problem p: clustered keys (j < ncl) of hit clusters, and every key
// cached after the clustering (ncl <= j < n).
__device__ __forceinline__ bool cl_take(uint16_t a, const uint8_t* s_hit, int64_t j, int64_t ncl, int64_t n) {
  return j < n && (j >= ncl || s_hit[a] != 0);
}

// Taken positions among this thread's kClPer consecutive ones, as a bit mask.
__device__ __forceinline__ uint32_t cl_mask(const uint16_t* __restrict__ asg, const uint8_t* s_hit, int64_t jb,
                                            int64_t ncl, int64_t n) {
  uint16_t av[kClPer];
  cl_load16(asg, av, jb, ncl);
  uint32_t msk = 0u;
#pragma unroll
  for (int i = 0; i < kClPer; ++i) msk |= cl_take(av[i], s_hit, jb + i, ncl, n) ? (1u << i) : 0u;
  return msk;
}

// Chunk flags of the single-pass compaction: launch epoch (24 bits) | status (2 bits: 1 the
// chunk's own count, 2 the inclusive count of chunks 0 .. this one) | value (38 bits).
constexpr int kFlagEpochBits = 24;
constexpr unsigned long long kFlagValueMask = (1ull << 38) - 1ull;

__device__ __forceinline__ unsigned long long cl_flag(uint32_t epoch, uint32_t status, long long v) {
  return ((unsigned long long)epoch << 40) | ((unsigned long long)status << 38) | ((unsigned long long)v & kFlagValueMask);
}
__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Single-pass ordered compaction of one problem's selected positions (chunks of kClChunk
// positions, thread t of a chunk owning positions 16 t .. 16 t + 15).  A CTA takes the next
// chunk of its problem from a counter, so every chunk it waits on belongs to a CTA that is
// already running; it publishes its own count, then sums its predecessors' flags, 32 per step,
// back to the first one that carries an inclusive count (decoupled look-back, every wait
// bounded), publishes
// its inclusive count and writes its positions.  The last chunk writes the set size; the last
// CTA to finish resets the counters for the next launch.
__global__ void __launch_bounds__(kClThreads) cl_compact_kernel(const uint16_t* __restrict__ assign,
                                                                int64_t a_stride, const uint8_t* __restrict__ hit,
                                                                int K, int Hr, int64_t max_select,
                                                                const SeqPos lens, const SeqPos ncl_b,
                                                                unsigned long long* __restrict__ flags,
                                                                uint32_t* __restrict__ ctr, uint32_t epoch,
                                                                long long wait_limit, int32_t* __restrict__ sel_idx,
                                                                int32_t* __restrict__ sel_cnt,
                                                                uint32_t* __restrict__ err) {
  __shared__ uint8_t s_hit[1024];
  __shared__ int s_wsum[kClThreads / 32];
  __shared__ int s_chunk;
  __shared__ long long s_base;
  const int p = blockIdx.y, b = p / Hr, nch = gridDim.x;
  if (threadIdx.x == 0) s_chunk = (int)atomicAdd(&ctr[2 * p], 1u);
  for (int i = threadIdx.x; i < K; i += kClThreads) s_hit[i] = hit[(int64_t)p * K + i];
  __syncthreads();
  const int chunk = s_chunk;
  const int64_t n = lens.v[b], ncl = ncl_b.v[b];
  const int64_t j0 = (int64_t)chunk * kClChunk;
  const int64_t jb = j0 + (int64_t)threadIdx.x * kClPer;
  uint32_t msk = j0 < n ? cl_mask(assign + (int64_t)p * a_stride, s_hit, jb, ncl, n) : 0u;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = __popc(msk);
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  int off = incl - c, tot = 0;
  for (int w = 0; w < kClThreads / 32; ++w) {
    off += w < warp ? s_wsum[w] : 0;
    tot += s_wsum[w];
  }
  if (warp == 0) {
    // warp 0: publish this chunk's count, then look back 32 predecessors at a time (lane l
    // reads chunk top - l) down to the nearest one that carries an inclusive count
    unsigned long long* fl = flags + (int64_t)p * nch;
    long long prefix = 0;
    if (chunk > 0) {
      if (lane == 0) st_release_u64(fl + chunk, cl_flag(epoch, 1u, tot));
      const long long t0 = clock64();
      for (int top = chunk - 1; top >= 0;) {
        const int j = top - lane;
        unsigned long long f = 0ull;
        bool ok = true, inc = true;  // before chunk 0: an inclusive count of 0
        if (j >= 0) {
          f = ld_acquire_u64(fl + j);
          const uint32_t st = (uint32_t)(f >> 38) & 3u;
          ok = (uint32_t)(f >> 40) == epoch && st != 0u;
          inc = ok && st == 2u;
        }
        const uint32_t pub = __ballot_sync(0xffffffffu, ok), incm = __ballot_sync(0xffffffffu, inc);
        const int L = incm ? __ffs(incm) - 1 : 31;  // lanes 0 .. L-1 add counts, lane L its inclusive
        const uint32_t need = L == 31 ? 0xffffffffu : ((1u << (L + 1)) - 1u);
        if ((pub & need) == need) {
          long long v = (lane <= L && j >= 0) ? (long long)(f & kFlagValueMask) : 0;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          prefix += v;
          if (incm) break;
          top -= 32;
        } else if (clock64() - t0 > wait_limit) {
          if (lane == 0) atomicOr(err, kErrTimeout);  // the set of this call is invalid; rtp_check reports it
          break;
        } else {
          __nanosleep(20);
        }
      }
    }
    if (lane == 0) {
      st_release_u64(fl + chunk, cl_flag(epoch, 2u, prefix + tot));
      s_base = prefix;
      if (chunk == nch - 1) {
        const long long total = prefix + tot;
        sel_cnt[p] = (int32_t)(total < max_select ? total : max_select);
        if (total > max_select) atomicOr(err, kErrOverflow);
      }
    }
  }
  __syncthreads();
  int64_t slot = s_base + off;
  int32_t* dst = sel_idx + (int64_t)p * max_select;
  while (msk) {
    const int i = __ffs(msk) - 1;
    msk &= msk - 1u;
    if (slot < max_select) dst[slot] = (int32_t)(jb + i);
    ++slot;
  }
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&ctr[2 * p + 1], 1u) == (uint32_t)(nch - 1)) {  // every chunk taken and done
      ctr[2 * p] = 0u;
      ctr[2 * p + 1] = 0u;
    }
  }
}

}  // namespace

cudaError_t launch_cluster_build(rtp_layer* L, int iters, cudaStream_t st) {
  const int K = L->n_clusters, P = L->B * L->Hr;
  const SeqPos lens = seq_pos(L, 0);
  const int64_t nmax = L->len;
  cudaError_t e;
  {
    ProfScope ps(L, "cluster_init", st);
    cl_init_kernel<<<P, kClThreads, 0, st>>>(L->idx_b, L->cl_cent, L->cl_sum, L->cl_acc, K, L->Hr, L->max_seq, lens);
    e = cudaGetLastError();
  }
  const size_t smem_a = (size_t)K * kR * sizeof(double);
  const size_t smem_s = (size_t)K * kR * sizeof(unsigned long long) + (size_t)K * sizeof(uint32_t);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(cl_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(cl_accum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s);
  const dim3 ga((unsigned)((nmax + kClAssignKeys - 1) / kClAssignKeys), (unsigned)P);
  const dim3 gs((unsigned)((nmax + kClAccumKeys - 1) / kClAccumKeys), (unsigned)P);
  for (int it = 0; it <= iters && e == cudaSuccess; ++it) {
    {
      ProfScope ps(L, "cluster_assign", st);
      cl_assign_kernel<<<ga, kClThreads, smem_a, st>>>(L->idx_b, L->cl_cent, L->cl_assign, L->cl_stride, K, L->Hr,
                                                       L->max_seq, lens);
      e = cudaGetLastError();
    }
    if (e != cudaSuccess) break;
    {
      ProfScope ps(L, "cluster_accum", st);
      cl_accum_kernel<<<gs, kClThreads, smem_s, st>>>(L->idx_b, L->cl_assign, L->cl_stride, L->cl_sum, L->cl_acc, K, L->Hr,
                                                      L->max_seq, lens, L->err);
      e = cudaGetLastError();
    }
    if (e != cudaSuccess) break;
    {
      ProfScope ps(L, "cluster_update", st);
      cl_update_kernel<<<P, kClThreads, 0, st>>>(L->cl_cent, L->cl_sum, L->cl_acc, L->cl_count, K, it < iters ? 1 : 0);
      e = cudaGetLastError();
    }
  }
  return e;
}

cudaError_t launch_cluster_select(rtp_layer* L, cudaStream_t st) {
  const int K = L->n_clusters, P = L->B * L->Hr;
  const SeqPos lens = seq_pos(L, 0);
  SeqPos ncl{};
  for (int b = 0; b < L->B; ++b) ncl.v[b] = (int32_t)L->cl_len[(size_t)b];
  cudaError_t e;
  {
    ProfScope ps(L, "cluster_select", st);
    cl_select_kernel<<<P, (K + 31) / 32 * 32, 0, st>>>(L->q_idx, L->cl_cent, L->cl_count, K, L->top_p, L->cl_hit,
                                                  L->sel_mass, L->sel_thr);
    e = cudaGetLastError();
  }
  const dim3 g((unsigned)((L->len + kClChunk - 1) / kClChunk), (unsigned)P);
  if (e == cudaSuccess) {
    if (++L->cl_epoch >= (1u << kFlagEpochBits)) {  // epochs wrapped: clear every flag once
      e = cudaMemsetAsync(L->cl_flags, 0, sizeof(unsigned long long) * (size_t)P * cluster_chunks(L->max_seq), st);
      L->cl_epoch = 1u;
    }
  }
  if (e == cudaSuccess) {
    ProfScope ps(L, "cluster_compact", st);
    cl_compact_kernel<<<g, kClThreads, 0, st>>>(L->cl_assign, L->cl_stride, L->cl_hit, K, L->Hr, L->max_select, lens,
                                                ncl, L->cl_flags, L->cl_ctr, L->cl_epoch,
                                                L->wait_limit > 0 ? L->wait_limit : kWaitLimitCycles, L->sel_idx,
                                                L->sel_cnt, L->err);
    e = cudaGetLastError();
  }
  return e;
}

int64_t cluster_chunks(int64_t max_seq) { return (max_seq + kClChunk - 1) / kClChunk; }

}  // namespace rtp
