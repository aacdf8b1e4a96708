// decode_select.cu -- decode-time index scoring fused with the exact top-p selection.
//
// For every problem p = (sequence b, retrieval head h) the kernel
//   1. streams the 16-dim index keys IDX[p][0..N) (fp32, or bf16 when the layer stores bf16
//      keys: half the bytes) from HBM and computes the pre-RoPE
//      scores s_j = qidx . IDX[p][j] (techwalker page, section 3: the 16-dim "radar");
//   2. finds the exact top-p set: the shortest prefix of the order (s desc, j asc) whose
//      index-softmax mass reaches p (zhichai page, insight 3; techwalker page, section 4),
//      without a full sort -- by a mass histogram, as the pages' kernel does (techwalker
//      page, section 6: buckets instead of sorting, fused with scoring), refined until the
//      cut is exact;
//   3. writes the selected positions in ascending order.
//
// B200 design
//   * One cooperative grid of <= #SM CTAs x 1024 threads.  The flat (problem, key) range is
//     split evenly; each CTA keeps its scores in shared memory (up to ~47K per CTA, ~7M per
//     launch), so the selection passes never touch HBM again.  Larger launches keep the
//     scores in a global scratch array instead.
//   * The index stream uses 16-byte non-allocating loads, eight in flight per thread: four
//     threads own one 64-byte row, so every warp load is a fully coalesced 512-byte segment.
//   * Masses are exp(s - m) in fp32, quantised to 64-bit fixed point (scale 2^sc with
//     N * 2^sc <= 2^62) and accumulated with 32-bit integer atomics (low word with carry into
//     the high word): integer sums are exact and order-independent, so the selection is
//     deterministic however the work is split.  The quantisation error on the total mass is
//     below N * 2^-(sc+1) of the largest key's mass (< 1.2e-7 at N = 2^20).
//   * Level 1: 1024 bins of width 1/64 for (m - s) < 16 (shared atomics, and the key joins its
//     warp's ordered keep list), one coarse bin for 16..32 (per-thread register sums: no atomics
//     for the bulk of the keys).  Later passes walk only the keep lists.  Keys 32 or more below
//     the max are never counted: each carries at most e^-32 of the top key's mass, their
//     quantised mass is 0 whenever N > 2^16, and for smaller N their total stays below
//     (1 - p) * Z for every fp32 p < 1 (1 - p >= 2^-24), so they can never be needed to reach
//     p and the cut never falls among them.
//   * The keys of the crossing bin (usually a handful, at most 1024 on the fast path) are
//     gathered into a list that every CTA of the problem sorts in shared memory (bitonic, warp
//     shuffles below distance 32) to locate the exact cut key t and how many keys tied at t
//     are taken (lowest positions first).  Larger crossing bins (massive exact ties) fall back
//     to three radix levels over the key bits, 11/11/10 bits.
//   * After the cut the selection is a key comparison: key > t, or key == t among the first
//     n_need tied positions.  Ordered compaction is two ballot passes per warp.
//   * Four grid barriers on the fast path (max, histogram, candidates, counts), three more on
//     the fallback.  Every barrier wait is bounded (about 1 s); on timeout the error word records
//     RTP_ETIMEOUT and the kernel returns.  Scratch histograms are zeroed by the launch that
//     last read them, so a launch starts on clean scratch without a memset.
#include <type_traits>

#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr int kBins = kSelBins;
constexpr int kThreads = kSelThreads;
constexpr int kWarps = kThreads / 32;
constexpr int kCand = kSelCand;  // crossing-bin keys resolved by sorting
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kUnroll = 8;  // 16-byte loads in flight per thread in the index stream
constexpr int kFine = 1024;  // level-1 bins of width 1/64 covering (m - s) in [0, 16); bin kFine: [16, 32)

// radix fallback inside the crossing bin: key bits [31:21], [20:10], [9:0]
__device__ __forceinline__ int level_shift(int l) { return l == 0 ? 21 : (l == 1 ? 10 : 0); }
__device__ __forceinline__ int level_bits(int l) { return l == 2 ? 10 : 11; }

struct Hist3 {  // a 2048-bin mass histogram in global memory: exact 64-bit mass as (hi, lo) words
  uint32_t* lo;
  uint32_t* hi;
  uint32_t* cnt;
};

struct SelectArgs {
  const float* idx;           // fp32 index keys, or
  const __nv_bfloat16* idx_b; // bf16 index keys (one of the two is set)
  int64_t idx_pstride;  // floats between problems (max_seq * r)
  const float* q_idx;   // [P][r]
  int P;
  int64_t N;
  int64_t L;  // keys per CTA
  int sc_bits;
  float top_p;
  int32_t* sel_idx;
  int64_t max_select;
  int32_t* sel_cnt;
  float* sel_mass;
  float* sel_thr;
  float* seg_max;     // [P + G]
  Hist3 h1;           // [P][bins]
  Hist3 hr;           // [3][P][bins] radix fallback levels
  uint32_t* cand_cnt;         // [P]
  unsigned long long* cand;   // [P][kCand] packed (key << 32) | ~j
  uint32_t* slot_cnt;         // [P + G][2]: (gt, eq) per (problem, CTA)
  unsigned long long* bar;    // [2]: grid barrier arrival counter (monotonic), exit counter
  uint32_t* keep;             // global keep lists when the scores live in global memory
  uint32_t* flags;            // [1]: some problem needs the radix fallback
  uint32_t* err;
  float* gscores;
  long long wait_limit;       // clock cycles a grid-barrier wait may take before it gives up
};

struct Seg {
  int p;
  int radix;     // 1: crossing bin too large for the candidate list (fallback path)
  int full;      // 1: a warp's keep list overflowed; later passes scan the whole chunk
  int kbase;     // this segment's keep lists start at keep[kbase]; warp w at + w * kcap
  int kcap;      // keep-list capacity per warp
  int bstar;
  uint32_t prefix;
  int64_t jlo, jhi, off;
  float m;
  uint32_t t_key;
  unsigned long long Z, T, rem, e_t, n_need, msel;
};

struct Smem {
  union {
    struct {
      uint32_t lo[kBins];
      uint32_t hi[kBins];
    } w;
    unsigned long long m[kBins];
  } h;
  uint32_t hc[kBins];
  unsigned long long sk[kCand];
  Seg seg[kSelMaxSeg];
  unsigned long long red64[kWarps];
  uint32_t red32[kWarps];
  float redf[kWarps];
  uint32_t wcnt[kSelMaxSeg][kWarps][2];  // (gt, eq) per warp chunk, then exclusive bases
  uint32_t lcnt[kSelMaxSeg][kWarps];     // keep-list length per warp chunk
  uint32_t slot[2 * kSelMaxGrid];
  int cross, cut_idx;
  unsigned long long cross_above, cut_cum;
  long long before, take;
};

// ---------------------------------------------------------------- small helpers

// Fixed-point mass of a score: round(2^sc * exp(s - m)), as (hi, lo) 32-bit words.
__device__ __forceinline__ void mass_words(float s, float m, float scale, uint32_t* hi, uint32_t* lo) {
  const float q = fast_exp2((s - m) * kLog2e) * scale;  // < 2^63; an integer once >= 2^24
  const float qh = floorf(q * 2.3283064365386963e-10f);  // q / 2^32
  *hi = (uint32_t)qh;
  *lo = __float2uint_rn(fmaf(qh, -4294967296.0f, q));
}
__device__ __forceinline__ unsigned long long mass64(float s, float m, float scale) {
  uint32_t hi, lo;
  mass_words(s, m, scale, &hi, &lo);
  return ((unsigned long long)hi << 32) | lo;
}
__device__ __forceinline__ int bin_of(float s, float m) {
  const float x = m - s;  // >= 0; NaN lands in the tail
  if (x < 16.f) return (int)(x * 64.f);
  if (x < 32.f) return kFine;
  return kBins - 1;
}

// exact 64-bit add into a (hi, lo) pair of 32-bit counters with 32-bit atomics
__device__ __forceinline__ void add_words(uint32_t* lo_w, uint32_t* hi_w, uint32_t hi, uint32_t lo) {
  const uint32_t old = atomicAdd(lo_w, lo);
  const uint32_t carry = (old + lo < old) ? 1u : 0u;
  if (hi + carry) atomicAdd(hi_w, hi + carry);
}

// Monotonic grid barrier: one atomic per CTA on a 64-bit counter that only grows, then an
// acquire spin until the counter reaches the next multiple of the grid size.  Bounded by
// `limit` clock cycles.  A CTA that gives up has still arrived, so the CTAs that do pass the
// barrier see every CTA's writes from before it; a CTA that gave up never arrives at the next
// barrier, which therefore nobody passes.
__device__ __forceinline__ bool grid_sync(unsigned long long* bar, uint32_t nblocks, uint32_t* err,
                                          long long limit) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    const unsigned long long old = atomicAdd(bar, 1ull);
    const unsigned long long target = (old / nblocks + 1) * nblocks;
    const long long t0 = clock64();
    while (true) {
      unsigned long long v;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(bar) : "memory");
      if (v >= target) break;
      if (clock64() - t0 > limit) {
        atomicOr(err, kErrTimeout);
        ok = 0;
        break;
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

__device__ float block_max(float v, Smem& S) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) S.redf[w] = v;
  __syncthreads();
  if (w == 0) {
    v = S.redf[l];
    v = warp_max(v);
    if (l == 0) S.redf[0] = v;
  }
  __syncthreads();
  return S.redf[0];
}

__device__ unsigned long long block_sum_u64(unsigned long long v, Smem& S) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) S.red64[w] = v;
  __syncthreads();
  if (w == 0) {
    v = S.red64[l];
    v = warp_sum(v);
    if (l == 0) S.red64[0] = v;
  }
  __syncthreads();
  return S.red64[0];
}

// Inclusive block scan of one u64 per thread (thread order); returns the inclusive value.
__device__ unsigned long long block_incl_scan_u64(unsigned long long v, Smem& S) {
  const int t = threadIdx.x, w = t >> 5, l = t & 31;
  unsigned long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (l >= o) incl += y;
  }
  __syncthreads();
  if (l == 31) S.red64[w] = incl;
  __syncthreads();
  if (w == 0) {
    unsigned long long x = S.red64[l];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (l >= o) x += y;
    }
    S.red64[l] = x;
  }
  __syncthreads();
  return (w > 0 ? S.red64[w - 1] : 0ull) + incl;
}

// In S.h.m order (reverse: index kBins-1 first), find the first position whose inclusive
// cumulative mass reaches target.  Result: S.cross = bin (-1 if none), S.cross_above = mass
// before it.
__device__ void find_crossing(Smem& S, bool reverse, unsigned long long target) {
  const int t = threadIdx.x;
  const int b0 = reverse ? kBins - 1 - 2 * t : 2 * t;
  const int b1 = reverse ? b0 - 1 : b0 + 1;
  const unsigned long long m0 = S.h.m[b0], m1 = S.h.m[b1];
  if (t == 0) S.cross = -1;
  const unsigned long long incl = block_incl_scan_u64(m0 + m1, S);
  const unsigned long long base = incl - (m0 + m1);
  if (base < target && base + m0 >= target) {
    S.cross = b0;
    S.cross_above = base;
  } else if (base + m0 < target && base + m0 + m1 >= target) {
    S.cross = b1;
    S.cross_above = base + m0;
  }
  __syncthreads();
}

__device__ __forceinline__ void zero_words(Smem& S) {
  for (int i = threadIdx.x; i < kBins; i += kThreads) {
    S.h.w.lo[i] = 0u;
    S.h.w.hi[i] = 0u;
    S.hc[i] = 0u;
  }
}

__device__ __forceinline__ void flush_words(Smem& S, const Hist3& g, int64_t base) {
  for (int i = threadIdx.x; i < kBins; i += kThreads) {
    const uint32_t c = S.hc[i];
    if (c) {
      add_words(g.lo + base + i, g.hi + base + i, S.h.w.hi[i], S.h.w.lo[i]);
      atomicAdd(g.cnt + base + i, c);
    }
  }
}

// Load a global histogram as 64-bit masses + counts (then synchronise).
__device__ __forceinline__ void load_hist(Smem& S, const Hist3& g, int64_t base) {
  for (int i = threadIdx.x; i < kBins; i += kThreads) {
    const uint32_t lo = __ldcg(g.lo + base + i), hi = __ldcg(g.hi + base + i);
    S.hc[i] = __ldcg(g.cnt + base + i);
    S.h.m[i] = ((unsigned long long)hi << 32) | lo;
  }
  __syncthreads();
}

__device__ __forceinline__ void zero_global_hist(const Hist3& g, int64_t n, int c, uint32_t G) {
  for (int64_t i = (int64_t)c * kThreads + threadIdx.x; i < n; i += (int64_t)G * kThreads) {
    g.lo[i] = 0u;
    g.hi[i] = 0u;
    g.cnt[i] = 0u;
  }
}

// Sort S.sk[0..n) descending (n a power of two, 32 <= n <= kCand); thread t ends with element t.
__device__ unsigned long long bitonic_desc(Smem& S, int n, unsigned long long v) {
  const int t = threadIdx.x;
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      unsigned long long pv;
      if (j >= 32) {
        __syncthreads();
        if (t < n) S.sk[t] = v;
        __syncthreads();
        pv = t < n ? S.sk[t ^ j] : 0ull;
      } else {
        pv = __shfl_xor_sync(0xffffffffu, v, j);
      }
      const bool desc = (t & k) == 0;
      const bool lower = (t & j) == 0;
      const unsigned long long hi_v = v > pv ? v : pv, lo_v = v > pv ? pv : v;
      v = (lower == desc) ? hi_v : lo_v;
    }
  }
  return v;
}

// first CTA that holds keys of problem p
__device__ __forceinline__ int cf_of(int p, const SelectArgs& a) { return (int)(((int64_t)p * a.N) / a.L); }

// ---------------------------------------------------------------- the kernel

template <bool kSmemScores, bool kBf16>
__global__ void __launch_bounds__(kThreads, 1) decode_select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  const int c = blockIdx.x;
  const uint32_t G = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t total = (int64_t)a.P * a.N;
  const int64_t r0 = (int64_t)c * a.L;
  const int64_t r1 = min(total, r0 + a.L);
  float* sc = kSmemScores ? reinterpret_cast<float*>(smem_raw + sizeof(Smem)) : a.gscores + r0;
  // Keep lists: 16-bit in shared memory after the scores, 32-bit in global memory otherwise.
  using KeepT = typename std::conditional<kSmemScores, uint16_t, uint32_t>::type;
  KeepT* keep = kSmemScores ? reinterpret_cast<KeepT*>(smem_raw + sizeof(Smem) + 4 * ((a.L + 3) / 4 * 4))
                            : reinterpret_cast<KeepT*>(a.keep + r0);
  const float scale = __uint_as_float((uint32_t)(127 + a.sc_bits) << 23);  // 2^sc
  const int64_t nh = (int64_t)a.P * kBins;

  // ---- segments of this CTA: [jlo, jhi) of problem p, stored at sc[off ...]
  int nseg = 0;
  if (r0 < r1) {
    const int p_first = (int)(r0 / a.N), p_last = (int)((r1 - 1) / a.N);
    nseg = p_last - p_first + 1;
    if (tid < nseg) {
      Seg& s = S.seg[tid];
      s.p = p_first + tid;
      s.jlo = max((int64_t)0, r0 - (int64_t)s.p * a.N);
      s.jhi = min(a.N, r1 - (int64_t)s.p * a.N);
      s.off = (int64_t)s.p * a.N + s.jlo - r0;
      s.radix = 0;
      s.full = 0;
      s.prefix = 0;
    }
  }
  __syncthreads();
  if (tid == 0) {  // per-warp keep capacity: a quarter of the warp chunk, rounded up
    int acc = 0;
    for (int si = 0; si < nseg; ++si) {
      const int rows = (int)(S.seg[si].jhi - S.seg[si].jlo);
      const int wlen = (rows + kWarps - 1) / kWarps;
      S.seg[si].kcap = (wlen + 3) / 4;
      S.seg[si].kbase = acc;
      acc += kWarps * S.seg[si].kcap;
    }
  }
  __syncthreads();

  // ---- phase A: stream index keys -> scores, segment maxima.  fp32 keys: four threads per
  // 64-byte key row, 16 bytes each; bf16 keys: two threads per 32-byte row.
  constexpr int kPer = kBf16 ? 2 : 4;      // threads per key
  constexpr int kKeysIt = kThreads / kPer;  // keys per unrolled step
  const int quad = tid / kPer, part = tid % kPer;
  for (int si = 0; si < nseg; ++si) {
    const Seg s = S.seg[si];
    const int64_t rows = s.jhi - s.jlo;
    const float4* src = kBf16 ? reinterpret_cast<const float4*>(a.idx_b + (int64_t)s.p * a.idx_pstride) + s.jlo * 2
                              : reinterpret_cast<const float4*>(a.idx + (int64_t)s.p * a.idx_pstride) + s.jlo * 4;
    float qv[kBf16 ? 8 : 4];
    {
      const float4* qp = reinterpret_cast<const float4*>(a.q_idx + (int64_t)s.p * kR) + part * (kBf16 ? 2 : 1);
#pragma unroll
      for (int i = 0; i < (kBf16 ? 2 : 1); ++i) {
        const float4 q4 = qp[i];
        qv[4 * i] = q4.x;
        qv[4 * i + 1] = q4.y;
        qv[4 * i + 2] = q4.z;
        qv[4 * i + 3] = q4.w;
      }
    }
    float mx = -INFINITY;
    // The trip count is the same for every thread (the shuffles below are full-warp);
    // rows past the end are loaded as zeros and not stored.
    for (int64_t base = 0; base < rows; base += kUnroll * kKeysIt) {
      const int64_t k0 = base + quad;
      float4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t k = k0 + u * kKeysIt;
        v[u] = k < rows ? ld_stream_f4(src + k * kPer + part) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        float d;
        if constexpr (kBf16) {  // eight bf16 components
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
          float2 f = __bfloat1622float2(h[0]);
          d = f.x * qv[0];
          d = fmaf(f.y, qv[1], d);
#pragma unroll
          for (int e = 1; e < 4; ++e) {
            f = __bfloat1622float2(h[e]);
            d = fmaf(f.x, qv[2 * e], d);
            d = fmaf(f.y, qv[2 * e + 1], d);
          }
          d += __shfl_xor_sync(0xffffffffu, d, 1);
        } else {  // four fp32 components
          d = v[u].x * qv[0];
          d = fmaf(v[u].y, qv[1], d);
          d = fmaf(v[u].z, qv[2], d);
          d = fmaf(v[u].w, qv[3], d);
          d += __shfl_xor_sync(0xffffffffu, d, 1);
          d += __shfl_xor_sync(0xffffffffu, d, 2);
        }
        d += 0.0f;  // -0 -> +0: equal scores must get equal order keys
        const int64_t k = k0 + u * kKeysIt;
        if (k < rows) {
          mx = fmaxf(mx, d);
          if (part == 0) sc[s.off + k] = d;
        }
      }
    }
    mx = block_max(mx, S);
    if (tid == 0) a.seg_max[s.p + c] = mx;
  }
  if (!grid_sync(a.bar, G, a.err, a.wait_limit)) return;

  // ---- phase B: row maxima; level-1 mass histogram; keep lists.  Warp w walks a contiguous
  // chunk of the segment.  Keys within 16 of the max join the warp's ordered keep list (their
  // fine-bin masses are added afterwards from the list, every lane busy); keys 16..32 below the
  // max add their exact mass to a per-thread register sum for the single coarse bin.
  const bool small_mass = a.sc_bits <= 54;  // then every coarse-bin mass fits 32 bits
  for (int si = 0; si < nseg; ++si) {
    const int p = S.seg[si].p;
    const int cf = cf_of(p, a), cl = (int)(((int64_t)p * a.N + a.N - 1) / a.L);
    float mv = -INFINITY;
    for (int cc = cf + tid; cc <= cl; cc += kThreads) mv = fmaxf(mv, __ldcg(a.seg_max + p + cc));
    const float m = block_max(mv, S);
    zero_words(S);
    if (tid == 0) S.seg[si].m = m;
    __syncthreads();
    const int off = (int)S.seg[si].off, rows = (int)(S.seg[si].jhi - S.seg[si].jlo);
    const int wlen = (rows + kWarps - 1) / kWarps;
    const int w_lo = min(rows, warp * wlen), w_hi = min(rows, w_lo + wlen);
    const int kcap = S.seg[si].kcap;
    KeepT* kl = keep + S.seg[si].kbase + warp * kcap;
    unsigned long long coarse = 0;
    int nkeep = 0;
    const uint32_t lt = (1u << lane) - 1u;
    for (int k0 = w_lo; k0 < w_hi; k0 += 32) {
      const int k = k0 + lane;
      const float v = k < w_hi ? sc[off + k] : -INFINITY;
      const float x = m - v;
      const bool fine = x < 16.f;
      if (!fine && x < 32.f) {
        if (small_mass) {
          coarse += __float2uint_rn(fast_exp2((v - m) * kLog2e) * scale);
        } else {
          coarse += mass64(v, m, scale);
        }
      }
      const uint32_t bf = __ballot_sync(0xffffffffu, fine);
      if (fine) {
        const int pos = nkeep + __popc(bf & lt);
        if (pos < kcap) {
          kl[pos] = (KeepT)k;
        } else {  // list full: count this key now
          uint32_t hi, lo;
          mass_words(v, m, scale, &hi, &lo);
          add_words(&S.h.w.lo[(int)(x * 64.f)], &S.h.w.hi[(int)(x * 64.f)], hi, lo);
        }
      }
      nkeep += __popc(bf);
    }
    if (lane == 0) {
      S.lcnt[si][warp] = (uint32_t)min(nkeep, kcap);
      if (nkeep > kcap) S.seg[si].full = 1;
    }
    const int nl = min(nkeep, kcap);
    __syncwarp();  // list entries written by other lanes of this warp
    for (int i = lane; i < nl; i += 32) {
      const float v = sc[off + (int)kl[i]];
      const float x = m - v;
      uint32_t hi, lo;
      mass_words(v, m, scale, &hi, &lo);
      add_words(&S.h.w.lo[(int)(x * 64.f)], &S.h.w.hi[(int)(x * 64.f)], hi, lo);
    }
    coarse = warp_sum(coarse);
    if (lane == 0 && coarse) add_words(&S.h.w.lo[kFine], &S.h.w.hi[kFine], (uint32_t)(coarse >> 32), (uint32_t)coarse);
    __syncthreads();
    for (int i = tid; i <= kFine; i += kThreads) {
      const uint32_t lo = S.h.w.lo[i], hi = S.h.w.hi[i];
      if (lo | hi) add_words(a.h1.lo + (int64_t)p * kBins + i, a.h1.hi + (int64_t)p * kBins + i, hi, lo);
    }
    __syncthreads();
  }
  if (!grid_sync(a.bar, G, a.err, a.wait_limit)) return;

  // ---- phase C: total mass, target, crossing bin; its keys become candidates.  A crossing in
  // the coarse bin, or more than kCand keys in the crossing bin, takes the radix fallback.
  for (int si = 0; si < nseg; ++si) {
    const int p = S.seg[si].p;
    for (int i = tid; i < kBins; i += kThreads) {
      uint32_t lo = 0, hi = 0;
      if (i <= kFine) {
        lo = __ldcg(a.h1.lo + (int64_t)p * kBins + i);
        hi = __ldcg(a.h1.hi + (int64_t)p * kBins + i);
      }
      S.h.m[i] = ((unsigned long long)hi << 32) | lo;
    }
    __syncthreads();
    {  // one scan gives Z (the total), then T, then the crossing bin
      const unsigned long long m0 = S.h.m[2 * tid], m1 = S.h.m[2 * tid + 1];
      if (tid == 0) S.cross = -1;
      const unsigned long long incl = block_incl_scan_u64(m0 + m1, S);
      const unsigned long long Z = S.red64[kWarps - 1];
      unsigned long long T = (unsigned long long)ceil((double)a.top_p * (double)Z);
      if (T < 1ull) T = 1ull;
      if (T > Z) T = Z;
      const unsigned long long base = incl - (m0 + m1);
      if (base < T && base + m0 >= T) {
        S.cross = 2 * tid;
        S.cross_above = base;
      } else if (base + m0 < T && base + m0 + m1 >= T) {
        S.cross = 2 * tid + 1;
        S.cross_above = base + m0;
      }
      if (tid == 0) {
        S.seg[si].Z = Z;
        S.seg[si].T = T;
      }
    }
    __syncthreads();
    if (tid == 0) {
      Seg& sg = S.seg[si];
      if (S.cross < 0) {
        atomicOr(a.err, kErrInternal);
        S.cross = 0;
        S.cross_above = 0;
      }
      sg.bstar = S.cross;
      sg.rem = sg.T - S.cross_above;
      // the coarse bin cannot be resolved from the keep lists: force the fallback
      if (S.cross == kFine) {
        atomicOr(a.flags, 1u);
        if (c == cf_of(p, a)) atomicAdd(a.cand_cnt + p, (uint32_t)kCand + 1u);
      }
    }
    __syncthreads();
    const int bstar = S.seg[si].bstar;
    if (bstar < kFine) {
      const int off = (int)S.seg[si].off, jlo = (int)S.seg[si].jlo, rows = (int)(S.seg[si].jhi - S.seg[si].jlo);
      const float m = S.seg[si].m;
      const bool full = S.seg[si].full;
      const int wlen = (rows + kWarps - 1) / kWarps;
      const int w_lo = min(rows, warp * wlen), w_hi = min(rows, w_lo + wlen);
      const KeepT* kl = keep + S.seg[si].kbase + warp * S.seg[si].kcap;
      const int n_it = full ? (w_hi - w_lo) : (int)S.lcnt[si][warp];
      for (int i = lane; i < n_it; i += 32) {
        const int k = full ? w_lo + i : (int)kl[i];
        const float v = sc[off + k];
        if (bin_of(v, m) != bstar) continue;
        const uint32_t slot = atomicAdd(a.cand_cnt + p, 1u);
        if (slot < (uint32_t)kCand)
          a.cand[(int64_t)p * kCand + slot] = ((unsigned long long)order_key(v) << 32) | (0xFFFFFFFFu - (uint32_t)(jlo + k));
        else
          atomicOr(a.flags, 1u);
      }
    }
    __syncthreads();
  }
  if (!grid_sync(a.bar, G, a.err, a.wait_limit)) return;

  // ---- phase D: exact cut.  Problems whose crossing bin fits the candidate list sort it;
  // the others (decided identically by every CTA from the global counts) refine by radix.
  if (tid == 0) S.cut_idx = (int)__ldcg(a.flags);
  __syncthreads();
  const bool fallback = S.cut_idx != 0;
  __syncthreads();
  for (int si = 0; si < nseg; ++si) {
    const int p = S.seg[si].p;
    // one round trip: the count and the candidate slots together
    const unsigned long long vraw = tid < kCand ? __ldcg(a.cand + (int64_t)p * kCand + tid) : 0ull;
    const uint32_t ncand = __ldcg(a.cand_cnt + p);
    if (tid == 0) S.seg[si].radix = ncand > (uint32_t)kCand;
    if (ncand > (uint32_t)kCand) continue;
    const int nc = (int)ncand;
    const float m = S.seg[si].m;
    const unsigned long long rem = S.seg[si].rem;
    int n = 32;
    while (n < nc) n <<= 1;
    const unsigned long long v = bitonic_desc(S, n, tid < nc ? vraw : 0ull);
    // masses in sorted order; the cut is the first key whose running mass reaches rem
    const uint32_t key = (uint32_t)(v >> 32);
    unsigned long long mq = 0ull;
    if (tid < nc) mq = mass64(key_to_float(key), m, scale);
    const unsigned long long cum = block_incl_scan_u64(mq, S);
    if (tid == 0) S.cut_idx = -1;
    __syncthreads();
    if (tid < nc && cum >= rem && cum - mq < rem) {
      S.cut_idx = tid;
      S.cut_cum = cum;
      S.seg[si].t_key = key;
      S.seg[si].e_t = mq;
    }
    __syncthreads();
    if (tid < nc) S.sk[tid] = v;  // publish the sorted keys to find the start of the tie run
    __syncthreads();
    if (tid == 0) {
      Seg& sg = S.seg[si];
      int ci = S.cut_idx;
      if (ci < 0) {  // unreachable with exact sums; keep every candidate
        atomicOr(a.err, kErrInternal);
        ci = nc - 1;
        sg.t_key = (uint32_t)(S.sk[ci] >> 32);
        sg.e_t = mass64(key_to_float(sg.t_key), sg.m, scale);
        S.cut_cum = sg.rem;
      }
      int lo = ci;
      while (lo > 0 && (uint32_t)(S.sk[lo - 1] >> 32) == sg.t_key) --lo;
      sg.n_need = (unsigned long long)(ci - lo + 1);
      sg.msel = (sg.T - sg.rem) + S.cut_cum;
    }
    __syncthreads();
  }
  __syncthreads();
  if (fallback) {
    // radix levels over the key bits of the crossing bin: build level l, sync, read it
    for (int lev = 0; lev <= 2; ++lev) {
      for (int si = 0; si < nseg; ++si) {
        if (!S.seg[si].radix) continue;
        const int p = S.seg[si].p;
        const int off = (int)S.seg[si].off, rows = (int)(S.seg[si].jhi - S.seg[si].jlo);
        const int bstar = S.seg[si].bstar;
        const float m = S.seg[si].m;
        const uint32_t prefix = S.seg[si].prefix;
        const int sh = lev > 0 ? level_shift(lev - 1) : 32;
        zero_words(S);
        __syncthreads();
        for (int k = tid; k < rows; k += kThreads) {
          const float v = sc[off + k];
          if (bin_of(v, m) != bstar) continue;
          const uint32_t key = order_key(v);
          if (sh < 32 && (key >> sh) != prefix) continue;
          const uint32_t d = (key >> level_shift(lev)) & ((1u << level_bits(lev)) - 1u);
          uint32_t hi, lo;
          mass_words(v, m, scale, &hi, &lo);
          add_words(&S.h.w.lo[d], &S.h.w.hi[d], hi, lo);
          atomicAdd(&S.hc[d], 1u);
        }
        __syncthreads();
        flush_words(S, a.hr, (int64_t)lev * nh + (int64_t)p * kBins);
        __syncthreads();
      }
      if (!grid_sync(a.bar, G, a.err, a.wait_limit)) return;
      for (int si = 0; si < nseg; ++si) {
        if (!S.seg[si].radix) continue;
        const int p = S.seg[si].p;
        load_hist(S, a.hr, (int64_t)lev * nh + (int64_t)p * kBins);
        find_crossing(S, true, S.seg[si].rem);
        if (tid == 0) {
          Seg& sg = S.seg[si];
          int d = S.cross;
          if (d < 0 || S.hc[d] == 0u) {
            atomicOr(a.err, kErrInternal);
            d = d < 0 ? 0 : d;
          }
          sg.prefix = (lev == 0) ? (uint32_t)d : ((sg.prefix << level_bits(lev)) | (uint32_t)d);
          sg.rem -= S.cross_above;
          if (lev == 2) {  // full key: every member of the group has the same mass
            const uint32_t cnt = S.hc[d] ? S.hc[d] : 1u;
            sg.t_key = sg.prefix;
            sg.e_t = S.h.m[d] / cnt;
            sg.n_need = sg.e_t ? (sg.rem + sg.e_t - 1) / sg.e_t : (unsigned long long)cnt;
            if (sg.n_need > cnt) sg.n_need = cnt;
            sg.msel = (sg.T - sg.rem) + sg.n_need * sg.e_t;
          }
        }
        __syncthreads();
      }
    }
  }
  // counts above the cut and at it, per warp (kept for the write pass) and per CTA.  The keep
  // list holds every key above a fine-bin cut; a coarse-bin cut scans the whole chunk.
  for (int si = 0; si < nseg; ++si) {
    const int off = (int)S.seg[si].off, rows = (int)(S.seg[si].jhi - S.seg[si].jlo);
    const uint32_t tk = S.seg[si].t_key;
    const bool full = S.seg[si].bstar >= kFine || S.seg[si].full;
    const int wlen = (rows + kWarps - 1) / kWarps;
    const int w_lo = min(rows, warp * wlen), w_hi = min(rows, w_lo + wlen);
    const KeepT* kl = keep + S.seg[si].kbase + warp * S.seg[si].kcap;
    const int n_it = full ? (w_hi - w_lo) : (int)S.lcnt[si][warp];
    uint32_t wg = 0, we = 0;
    for (int i0 = 0; i0 < n_it; i0 += 32) {
      const int i = i0 + lane;
      uint32_t key = 0u;
      if (i < n_it) key = order_key(sc[off + (full ? w_lo + i : (int)kl[i])]);
      wg += __popc(__ballot_sync(0xffffffffu, i < n_it && key > tk));
      we += __popc(__ballot_sync(0xffffffffu, i < n_it && key == tk));
    }
    if (lane == 0) {
      S.wcnt[si][warp][0] = wg;
      S.wcnt[si][warp][1] = we;
    }
    __syncthreads();
    if (warp == 0) {
      const uint32_t g1 = warp_sum(S.wcnt[si][lane][0]), e1 = warp_sum(S.wcnt[si][lane][1]);
      if (lane == 0) {
        a.slot_cnt[2 * (S.seg[si].p + c)] = g1;
        a.slot_cnt[2 * (S.seg[si].p + c) + 1] = e1;
      }
    }
    __syncthreads();
  }
  if (!grid_sync(a.bar, G, a.err, a.wait_limit)) return;
  // Every CTA has passed its last barrier: the last one to get here rewinds the barrier
  // counter so the next launch (whatever its grid size) starts from zero.
  if (tid == 0 && atomicAdd(a.bar + 1, 1ull) == (unsigned long long)(G - 1)) {
    a.bar[0] = 0ull;
    a.bar[1] = 0ull;
  }

  // ---- phase E: offsets across CTAs; ordered compaction; clean the scratch for the next launch
  for (int64_t i = (int64_t)c * kThreads + tid; i < nh; i += (int64_t)G * kThreads) {
    a.h1.lo[i] = 0u;
    a.h1.hi[i] = 0u;
  }
  if (fallback) zero_global_hist(a.hr, 3 * nh, c, G);
  for (int i = c * kThreads + tid; i < a.P; i += G * kThreads) a.cand_cnt[i] = 0u;
  if (c == 0 && tid == 0) a.flags[0] = 0u;

  for (int si = 0; si < nseg; ++si) {
    const Seg& s = S.seg[si];
    const int p = s.p;
    const int cf = cf_of(p, a), cl = (int)(((int64_t)p * a.N + a.N - 1) / a.L);
    for (int cc = cf + tid; cc <= c; cc += kThreads) {
      S.slot[2 * (cc - cf)] = __ldcg(a.slot_cnt + 2 * (p + cc));
      S.slot[2 * (cc - cf) + 1] = __ldcg(a.slot_cnt + 2 * (p + cc) + 1);
    }
    __syncthreads();
    if (tid == 0) {
      long long eq_before = 0, before = 0;
      for (int cc = cf; cc < c; ++cc) {
        const long long g2 = S.slot[2 * (cc - cf)];
        const long long e2 = S.slot[2 * (cc - cf) + 1];
        long long take = (long long)s.n_need - eq_before;
        take = take < 0 ? 0 : (take > e2 ? e2 : take);
        before += g2 + take;
        eq_before += e2;
      }
      const long long e_own = S.slot[2 * (c - cf) + 1];
      long long take = (long long)s.n_need - eq_before;
      take = take < 0 ? 0 : (take > e_own ? e_own : take);
      S.before = before;
      S.take = take;
      uint32_t g_acc = 0, e_acc = 0;  // exclusive warp bases
      for (int w = 0; w < kWarps; ++w) {
        const uint32_t g1 = S.wcnt[si][w][0], e1 = S.wcnt[si][w][1];
        S.wcnt[si][w][0] = g_acc;
        S.wcnt[si][w][1] = e_acc;
        g_acc += g1;
        e_acc += e1;
      }
      if (c == cl) {
        const long long K = before + g_acc + take;
        a.sel_cnt[p] = (int32_t)(K < a.max_select ? K : a.max_select);
        a.sel_mass[p] = (float)((double)s.msel / (double)s.Z);
        a.sel_thr[p] = (float)((double)s.e_t / (double)s.Z);
      }
    }
    __syncthreads();
    // write positions in ascending order: warp lists in warp order, ballots within 32-key steps
    const long long before = S.before, take = S.take;
    const int off = (int)s.off, rows = (int)(s.jhi - s.jlo), jlo = (int)s.jlo;
    const uint32_t tk = s.t_key;
    const bool full = s.bstar >= kFine || s.full;
    const int wlen = (rows + kWarps - 1) / kWarps;
    const int w_lo = min(rows, warp * wlen), w_hi = min(rows, w_lo + wlen);
    const KeepT* kl = keep + s.kbase + warp * s.kcap;
    const int n_it = full ? (w_hi - w_lo) : (int)S.lcnt[si][warp];
    long long g_run = S.wcnt[si][warp][0], e_run = S.wcnt[si][warp][1];
    const uint32_t lt = (1u << lane) - 1u;
    int32_t* dst = a.sel_idx + (int64_t)p * a.max_select;
    for (int i0 = 0; i0 < n_it; i0 += 32) {
      const int i = i0 + lane;
      int k = 0;
      uint32_t key = 0u;
      if (i < n_it) {
        k = full ? w_lo + i : (int)kl[i];
        key = order_key(sc[off + k]);
      }
      const bool isg = i < n_it && key > tk;
      const bool ise = i < n_it && key == tk;
      const uint32_t bg = __ballot_sync(0xffffffffu, isg), be = __ballot_sync(0xffffffffu, ise);
      const long long g_le = g_run + __popc(bg & lt), e_le = e_run + __popc(be & lt);
      if (isg || (ise && e_le < take)) {
        const long long pos = before + g_le + (e_le < take ? e_le : take);
        if (pos < a.max_select) dst[pos] = jlo + k;
        else atomicOr(a.err, kErrOverflow);
      }
      g_run += __popc(bg);
      e_run += __popc(be);
    }
    __syncthreads();
  }
}

}  // namespace

size_t select_fixed_smem() { return (sizeof(Smem) + 127) / 128 * 128; }

// scores (fp32) + keep lists (16-bit, a quarter of the keys plus per-warp rounding)
size_t select_var_smem(int64_t per) {
  return 4 * (size_t)((per + 3) / 4 * 4) + 2 * (size_t)(per / 4 + kWarps * (2 * kSelMaxSeg + 2));
}

SelectGeom select_geometry(const rtp_layer* L, int64_t N) {
  SelectGeom g;
  const int64_t P = (int64_t)L->B * L->Hr;
  const int64_t total = P * N;
  int G = L->sm_count;
  const int64_t want = (total + 4095) / 4096;
  if (want < G) G = (int)(want < 1 ? 1 : want);
  int64_t per = (total + G - 1) / G;
  // one CTA may hold at most kSelMaxSeg problem segments
  if (per > (int64_t)(kSelMaxSeg - 1) * N) per = (int64_t)(kSelMaxSeg - 1) * N;
  G = (int)((total + per - 1) / per);
  g.grid = G;
  g.per_cta = per;
  const size_t fixed = select_fixed_smem();
  const size_t need = fixed + select_var_smem(per);
  g.smem_scores = need <= L->smem_optin;
  g.smem_bytes = g.smem_scores ? need : fixed;
  return g;
}

cudaError_t launch_decode_select(rtp_layer* L, cudaStream_t st) {
  const int64_t N = L->len;
  const SelectGeom g = select_geometry(L, N);
  SelectArgs a;
  a.idx = L->idx;
  a.idx_b = L->idx_b;
  a.idx_pstride = L->max_seq * kR;
  a.q_idx = L->q_idx;
  a.P = L->B * L->Hr;
  a.N = N;
  a.L = g.per_cta;
  int lg = 0;
  while ((1ll << lg) < N) ++lg;
  a.sc_bits = 62 - lg;
  a.top_p = L->top_p;
  a.sel_idx = L->sel_idx;
  a.max_select = L->max_select;
  a.sel_cnt = L->sel_cnt;
  a.sel_mass = L->sel_mass;
  a.sel_thr = L->sel_thr;
  a.seg_max = L->seg_max;
  const int64_t nh = (int64_t)a.P * kBins;
  a.h1 = Hist3{L->sel_words, L->sel_words + nh, L->sel_words + 2 * nh};
  a.hr = Hist3{L->sel_words + 3 * nh, L->sel_words + 6 * nh, L->sel_words + 9 * nh};
  a.cand_cnt = L->cand_cnt;
  a.cand = L->cand;
  a.slot_cnt = L->slot_cnt;
  a.bar = L->bar;
  a.err = L->err;
  a.gscores = L->gscores;
  a.keep = L->sel_keep;
  a.flags = L->sel_flags;
  a.wait_limit = L->wait_limit > 0 ? L->wait_limit : kWaitLimitCycles;
  if (!g.smem_scores && L->gscores == nullptr) return cudaErrorInvalidValue;
  if (g.grid > L->sm_count || g.grid > kSelMaxGrid) return cudaErrorInvalidValue;
  void* args[] = {&a};
  const void* fn = L->index_bf16
                       ? (g.smem_scores ? (const void*)decode_select_kernel<true, true>
                                        : (const void*)decode_select_kernel<false, true>)
                       : (g.smem_scores ? (const void*)decode_select_kernel<true, false>
                                        : (const void*)decode_select_kernel<false, false>);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.smem_bytes);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kThreads, g.smem_bytes);
  if (e != cudaSuccess) return e;
  if (occ < 1 || g.grid > occ * L->sm_count) return cudaErrorCooperativeLaunchTooLarge;
  return cudaLaunchCooperativeKernel(fn, dim3(g.grid), dim3(kThreads), args, g.smem_bytes, st);
}

}  // namespace rtp
