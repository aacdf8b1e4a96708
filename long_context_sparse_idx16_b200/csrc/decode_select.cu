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
//   * Each (problem, CTA) segment publishes its cumulative fine-bin key counts.  One CTA per
//     problem (the one holding the middle of its keys) waits for all of them (an arrival count)
//     and finds Z, the target and the crossing bin.  After the second barrier every CTA adds its
//     crossing-bin keys (usually a handful, at most 1024 on the fast path) to the problem's
//     candidate list, and the same CTA sorts the list in shared memory (bitonic, warp shuffles
//     below distance 32) to locate the exact cut key t and how many keys tied at t are taken
//     (lowest positions first), and from the cumulative counts and the sorted list the number of
//     keys each CTA's predecessors select.  After the third barrier each CTA writes its own
//     positions.
//   * After the cut the selection is a key comparison: key > t, or key == t among the first
//     n_need tied positions.  Ordered compaction is two ballot passes per warp.
//   * The ranges of the flat (problem, key) space follow the SM number when every SM holds one
//     CTA: the even SM of each TPC takes a larger share (measured: it streams faster while both
//     stream).
//   * Three grid barriers on the fast path (max, histogram, cut).  A crossing in the coarse bin
//     or one holding more keys than the sort takes (massive exact ties) sets the launch's
//     fallback flag: then every CTA sorts the candidates of the problems that fit, and the
//     others refine by three radix levels over the key bits (11/11/10), with five barriers
//     after the second.  Every barrier wait is bounded (about 1 s); on timeout the error word
//     records RTP_ETIMEOUT and the kernel returns.  Scratch histograms and lists are reset by
//     the launch that last read them, so a launch starts on clean scratch without a memset.
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
constexpr int kPsum = 8;     // words of a problem's summary
constexpr int kUnroll = 8;  // 16-byte loads in flight per thread in the index stream
constexpr int kFine = kSelFine;  // level-1 bins of width 1/64 covering (m - s) in [0, 16); bin kFine: [16, 32)
static_assert(kFine == kThreads, "one fine bin per thread in the count scans");
static_assert(kWarps == 32, "one lane per warp in the warp-base scans");

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
  const float* q_idx;   // [P][r], read when q_raw is NULL
  // With q_raw set the kernel also does the query preparation: it writes the RoPE'd rows of
  // every head (q_rot, for the attention kernels) and forms its own segments' index queries.
  const __nv_bfloat16* q_raw;  // [B][Hq][D] pre-RoPE decode queries, or NULL
  const double* theta;         // [D/2] RoPE frequencies
  const float* wq;             // [Hr][D][r]
  const int16_t* ret_head;     // [Hr] query head of each retrieval slot
  int Hq;
  float* q_rot;                // [B][Hq][D]
  int P;
  int64_t N;
  int64_t L;   // keys of the longest CTA range (sizes the shared-memory score array)
  int64_t Lp;  // keys per CTA pair (virtual indices 2k, 2k + 1) ...
  int64_t Le;  // ... of which the even member takes the first Le
  int use_smid;  // 1: the virtual index of a CTA is its SM (one CTA on every SM)
  int Hr;        // retrieval heads: problem p belongs to sequence p / Hr
  SeqPos lens;   // each sequence's length; problems span N = the longest, keys past a
                 // sequence's length score -inf (never counted, never selected)
  int sc_bits;
  float top_p;
  int32_t* sel_idx;
  int64_t max_select;
  int32_t* sel_cnt;
  float* sel_mass;
  float* sel_thr;
  float* seg_max;     // [P + G]
  unsigned long long* h1;  // [P][bins]: level-1 masses (64-bit words)
  Hist3 hr;           // [3][P][bins] radix fallback levels
  uint32_t* cand_cnt;         // [P]
  unsigned long long* cand;   // [P][kCand] packed (key << 32) | ~j
  uint32_t* slot_cnt;         // [P + G][2]: (gt, eq) per (problem, CTA)
  unsigned long long* bar;    // [2]: grid barrier arrival counter (monotonic), exit counter
  uint32_t* keep;             // global keep lists when the scores live in global memory
  uint32_t* flags;            // [1]: == epoch when some problem of this launch needs the fallback
  uint32_t epoch;             // this launch's number (never 0)
  uint32_t* cum;              // [P + G][kFine]: cumulative fine-bin key counts per (problem, CTA)
  unsigned long long* psum;   // [P][kPsum]: Z, T, rem, (crossing-bin keys << 32) | crossing bin, cut key
  long long* cres;            // [P + G][2]: keys the CTAs before select, tied keys this CTA takes
  uint32_t* pticket;          // [P]: CTAs of the problem done with phase B (the last resets it)
  uint32_t* err;
  float* gscores;
  long long wait_limit;       // clock cycles a grid-barrier wait may take before it gives up
};

struct Seg {
  int p;
  int radix;     // 1: crossing bin too large for the candidate list (fallback path)
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
  uint32_t lres[kSelMaxSeg][kWarps];     // first key of the warp chunk its full keep list missed
  uint32_t slot[2 * kSelMaxGrid];
  int cross, cut_idx;
  unsigned long long cross_above, cut_cum;
  long long before, take;
};

// ---------------------------------------------------------------- small helpers

// The keys a pass over a warp chunk's fine keys visits: its keep list, then, when the list
// filled up, every key from the first one it missed to the end of the chunk (keys that are not
// fine fail every test those passes make).  `whole`: every key of the chunk (a cut in the coarse
// bin, whose keys are not listed).
__device__ __forceinline__ int visit_count(bool whole, int w_lo, int w_hi, int n_list, int res) {
  return whole ? (w_hi - w_lo) : n_list + (w_hi - res);
}
template <typename KeepT>
__device__ __forceinline__ int visit_key(int i, bool whole, int w_lo, const KeepT* kl, int n_list, int res) {
  return whole ? w_lo + i : (i < n_list ? (int)kl[i] : res + (i - n_list));
}

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

// Wait (bounded by `limit` clock cycles) until the counter reaches target; false, with
// RTP_ETIMEOUT recorded, if it does not.  Only counters that co-resident CTAs of this
// cooperative grid advance are waited on.
__device__ __forceinline__ bool wait_count(const uint32_t* ctr, uint32_t target, uint32_t* err, long long limit) {
  const long long t0 = clock64();
  while (true) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if (clock64() - t0 > limit) {
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
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

// CTA ranges of the flat (problem, key) index space: virtual CTA v starts at r_start(v); the
// two members of a pair split Lp keys as Le + (Lp - Le).
__device__ __forceinline__ int64_t r_start(int v, const SelectArgs& a) {
  return (int64_t)(v >> 1) * a.Lp + ((v & 1) ? a.Le : 0);
}
// the CTA whose range holds flat index x
__device__ __forceinline__ int cta_of(int64_t x, const SelectArgs& a) {
  const int64_t k = x / a.Lp;
  return (int)(2 * k + (x - k * a.Lp >= a.Le ? 1 : 0));
}
// first and last CTA that hold keys of problem p
__device__ __forceinline__ int cf_of(int p, const SelectArgs& a) { return cta_of((int64_t)p * a.N, a); }
__device__ __forceinline__ int cl_of(int p, const SelectArgs& a) { return cta_of((int64_t)p * a.N + a.N - 1, a); }

// The virtual index of this CTA.  Of the two SMs of a TPC, the odd-numbered one streams about
// 15% slower while both stream (measured), so with one CTA on every SM the ranges follow the SM
// number: even SMs take the larger share of a pair.  Otherwise the block index.
__device__ __forceinline__ int virtual_cta(const SelectArgs& a) {
  if (a.use_smid) {
    uint32_t smid, nsmid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    asm volatile("mov.u32 %0, %%nsmid;" : "=r"(nsmid));
    if (nsmid == gridDim.x) return (int)smid;  // then the SM numbers are exactly 0 .. G-1
  }
  return (int)blockIdx.x;
}

// Z, the target T and the crossing bin of problem p, found once by its designated CTA after
// every CTA of the problem has finished phase B (S.h.m holds the problem's level-1 masses, every CTA of the problem has
// published its cumulative fine-bin counts).  A crossing in the coarse bin, or one holding more
// than kCand keys, is left to the fallback path (the launch's flag).
__device__ void select_summary(const SelectArgs& a, Smem& S, int p, int cf, int cl) {
  const int tid = threadIdx.x;
  // one scan gives Z (the total), then T, then the crossing bin
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
  __syncthreads();
  if (tid == 0 && S.cross < 0) {
    atomicOr(a.err, kErrInternal);
    S.cross = 0;
    S.cross_above = 0;
  }
  __syncthreads();
  const int cross = S.cross;
  // keys in the crossing bin, over the problem's CTAs
  unsigned long long nk = 0;
  if (cross < kFine) {
    for (int cc = cf + tid; cc <= cl; cc += kThreads) {
      const uint32_t* cu = a.cum + (int64_t)(p + cc) * kFine;
      nk += __ldcg(cu + cross) - (cross > 0 ? __ldcg(cu + cross - 1) : 0u);
    }
  }
  nk = block_sum_u64(nk, S);
  if (tid == 0) {
    unsigned long long* ps = a.psum + kPsum * (int64_t)p;
    ps[0] = Z;
    ps[1] = T;
    ps[2] = T - S.cross_above;
    ps[3] = (nk << 32) | (uint32_t)cross;
    if (cross >= kFine || nk > (unsigned long long)kCand) atomicExch(a.flags, a.epoch);
    a.pticket[p] = 0u;
  }
}

// The exact cut of problem p, found once by its designated CTA after every CTA of the problem
// has added its crossing-bin keys to the problem's candidate list: the candidates sorted (key desc, then position asc), the
// cut key t and the number of tied keys taken; then, per CTA of the problem, the count of keys
// its predecessors select (their keys above the crossing bin, from the cumulative counts, plus
// their candidates above the cut and the ties taken) and how many of its own tied keys it
// takes.  Also the problem's outputs (count, mass, threshold); the list is reset for the next
// launch.
__device__ void select_cut(const SelectArgs& a, Smem& S, int p, int cf, int cl, float m, float scale) {
  const int tid = threadIdx.x;
  unsigned long long* ps = a.psum + kPsum * (int64_t)p;
  const unsigned long long Z = __ldcg(ps), T = __ldcg(ps + 1), rem = __ldcg(ps + 2);
  const int cross = (int)(uint32_t)__ldcg(ps + 3);
  const int nct = cl - cf + 1;
  const unsigned long long vraw = tid < kCand ? __ldcg(a.cand + (int64_t)p * kCand + tid) : 0ull;
  const int nc = min((int)__ldcg(a.cand_cnt + p), kCand);
  // per CTA of the problem: keys above the crossing bin
  for (int t = tid; t < nct; t += kThreads) {
    const uint32_t* cu = a.cum + (int64_t)(p + cf + t) * kFine;
    S.slot[t] = cross > 0 ? __ldcg(cu + cross - 1) : 0u;
  }
  int n = 32;
  while (n < nc) n <<= 1;
  const unsigned long long v = bitonic_desc(S, n, tid < nc ? vraw : 0ull);  // key desc, then position asc
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
  }
  if (tid < nc) S.sk[tid] = v;
  __syncthreads();
  int ci = S.cut_idx;
  if (ci < 0) {  // unreachable with exact sums; keep every candidate
    if (tid == 0) atomicOr(a.err, kErrInternal);
    ci = nc - 1;
  }
  // the cut key (an empty list, also unreachable, selects nothing from the crossing bin)
  const uint32_t tk = ci >= 0 ? (uint32_t)(S.sk[ci] >> 32) : 0xFFFFFFFFu;
  // the start of the tie run at the cut (sorted: equal keys are adjacent)
  if (tid == 0) S.cross = ci + 1;
  for (int t = tid; t < 2 * nct; t += kThreads) S.hc[t] = 0u;
  __syncthreads();
  if (tid < nc && key == tk && (tid == 0 || (uint32_t)(S.sk[tid - 1] >> 32) != tk)) S.cross = tid;
  // per CTA: crossing-bin keys above the cut, and at it
  if (tid < nc && key >= tk) {
    const uint32_t j = 0xFFFFFFFFu - (uint32_t)v;
    const int t = cta_of((int64_t)p * a.N + j, a) - cf;
    atomicAdd(&S.hc[2 * t + (key == tk ? 1 : 0)], 1u);
  }
  __syncthreads();
  if (tid == 0) {
    const long long n_need = (long long)(ci - S.cross + 1);
    long long before = 0, eq_seen = 0;
    for (int t = 0; t < nct; ++t) {
      const long long eq = S.hc[2 * t + 1];
      long long take = n_need - eq_seen;
      take = take < 0 ? 0 : (take > eq ? eq : take);
      a.cres[2 * (int64_t)(p + cf + t)] = before;
      a.cres[2 * (int64_t)(p + cf + t) + 1] = take;
      before += (long long)S.slot[t] + (long long)S.hc[2 * t] + take;
      eq_seen += eq;
    }
    const unsigned long long e_t = mass64(key_to_float(tk), m, scale);
    const unsigned long long cut_cum = S.cut_idx >= 0 ? S.cut_cum : rem;
    a.sel_cnt[p] = (int32_t)(before < a.max_select ? before : a.max_select);
    a.sel_mass[p] = (float)((double)((T - rem) + cut_cum) / (double)Z);
    a.sel_thr[p] = (float)((double)e_t / (double)Z);
    ps[4] = tk;
    a.cand_cnt[p] = 0u;
    a.pticket[p] = 0u;
  }
}

// ---------------------------------------------------------------- the kernel

template <bool kSmemScores, bool kBf16>
__global__ void __launch_bounds__(kThreads, 1) decode_select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  const int c = virtual_cta(a);
  const uint32_t G = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t total = (int64_t)a.P * a.N;
  const int64_t r0 = min(total, r_start(c, a));
  const int64_t r1 = min(total, r_start(c + 1, a));
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
      s.prefix = 0;
    }
  }
  __syncthreads();
  if (tid == 0) {  // per-warp keep capacity: 3/8 of the warp chunk, rounded up
    int acc = 0;
    for (int si = 0; si < nseg; ++si) {
      const int rows = (int)(S.seg[si].jhi - S.seg[si].jlo);
      const int wlen = (rows + kWarps - 1) / kWarps;
      S.seg[si].kcap = (3 * wlen + 7) / 8;
      S.seg[si].kbase = acc;
      acc += kWarps * S.seg[si].kcap;
    }
  }
  __syncthreads();

  // ---- query preparation (q_raw set), first part: the index queries of this CTA's segments,
  // kept in the candidate buffer (not used before the cut).  The RoPE'd rows follow the stream.
  float* s_qt = reinterpret_cast<float*>(S.sk);  // [kSelMaxSeg][r]
  if (a.q_raw) {
    // index query of segment w (warp w): lane l holds dims 4l .. 4l + 3 of q and their 16
    // weights each, then the 16 sums are reduced over the warp
    if (warp < nseg) {
      const int p = S.seg[warp].p, hr = p % a.Hr;
      const __nv_bfloat16* qr = a.q_raw + ((int64_t)(p / a.Hr) * a.Hq + a.ret_head[hr]) * kD + 4 * lane;
      const float4* w4 = reinterpret_cast<const float4*>(a.wq + ((int64_t)hr * kD + 4 * lane) * kR);
      float acc[kR];
#pragma unroll
      for (int o = 0; o < kR; ++o) acc[o] = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float x = __bfloat162float(qr[i]);
#pragma unroll
        for (int o4 = 0; o4 < kR / 4; ++o4) {
          const float4 w = w4[i * (kR / 4) + o4];
          acc[4 * o4] = fmaf(x, w.x, acc[4 * o4]);
          acc[4 * o4 + 1] = fmaf(x, w.y, acc[4 * o4 + 1]);
          acc[4 * o4 + 2] = fmaf(x, w.z, acc[4 * o4 + 2]);
          acc[4 * o4 + 3] = fmaf(x, w.w, acc[4 * o4 + 3]);
        }
      }
#pragma unroll
      for (int o = 0; o < kR; ++o) {
#pragma unroll
        for (int sh = 16; sh >= 1; sh >>= 1) acc[o] += __shfl_xor_sync(0xffffffffu, acc[o], sh);
      }
      if (lane == 0) {
#pragma unroll
        for (int o = 0; o < kR; ++o) s_qt[warp * kR + o] = acc[o];
      }
    }
    __syncthreads();
  }

  // ---- phase A: stream index keys -> scores, segment maxima.  fp32 keys: four threads per
  // 64-byte key row, 16 bytes each; bf16 keys: two threads per 32-byte row.
  constexpr int kPer = kBf16 ? 2 : 4;      // threads per key
  constexpr int kKeysIt = kThreads / kPer;  // keys per unrolled step
  const int quad = tid / kPer, part = tid % kPer;
  for (int si = 0; si < nseg; ++si) {
    const Seg s = S.seg[si];
    const int64_t rows = s.jhi - s.jlo;
    // keys of the segment inside its sequence (a shorter sequence of a ragged batch)
    const int64_t valid = max((int64_t)0, min(rows, (int64_t)a.lens.v[s.p / a.Hr] - s.jlo));
    const float4* src = kBf16 ? reinterpret_cast<const float4*>(a.idx_b + (int64_t)s.p * a.idx_pstride) + s.jlo * 2
                              : reinterpret_cast<const float4*>(a.idx + (int64_t)s.p * a.idx_pstride) + s.jlo * 4;
    float qv[kBf16 ? 8 : 4];
    {
      const float4* qp = reinterpret_cast<const float4*>(a.q_raw ? s_qt + si * kR : a.q_idx + (int64_t)s.p * kR) +
                         part * (kBf16 ? 2 : 1);
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
    // bf16 keys: four 16-byte loads in flight per thread (eight, with the bf16 unpacking, spill
    // out of the 64 registers a thread has, which cost a third of the stream's speed)
    constexpr int kU = kBf16 ? 4 : kUnroll;
    for (int64_t base = 0; base < rows; base += kU * kKeysIt) {
      const int64_t k0 = base + quad;
      float4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t k = k0 + u * kKeysIt;
        v[u] = k < valid ? ld_stream_f4(src + k * kPer + part) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
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
          if (k >= valid) d = -INFINITY;
          mx = fmaxf(mx, d);
          if (part == 0) sc[s.off + k] = d;
        }
      }
    }
    mx = block_max(mx, S);
    if (tid == 0) a.seg_max[s.p + c] = mx;
  }
  if (a.q_raw) {
    // query preparation, second part, while the slowest CTAs finish the stream: RoPE'd rows
    // b * Hq + h for the attention kernels, 128 threads per row (rows spread over all CTAs):
    // first half x cos - partner sin, second half x cos + partner sin, the angle reduced in fp64
    const int n_rows = a.P / a.Hr * a.Hq, d = tid & (kD - 1);
    for (int r = blockIdx.x * (kThreads / kD) + tid / kD; r < n_rows; r += gridDim.x * (kThreads / kD)) {
      const int b = r / a.Hq;
      const __nv_bfloat16* qr = a.q_raw + (int64_t)r * kD;
      const float x = __bfloat162float(qr[d]), xp = __bfloat162float(qr[d ^ kHalfD]);
      float cs, sn;
      rope_cos_sin((int64_t)a.lens.v[b] - 1, a.theta[d & (kHalfD - 1)], &cs, &sn);
      a.q_rot[(int64_t)r * kD + d] = d < kHalfD ? x * cs - xp * sn : x * cs + xp * sn;
    }
  }
  if (!grid_sync(a.bar, G, a.err, a.wait_limit)) return;

  // ---- phase B: row maxima; level-1 mass histogram; keep lists; the fine keys by bin.  Warp w
  // walks a contiguous chunk of the segment.  Keys within 16 of the max join the warp's ordered
  // keep list (their fine-bin masses and counts are added afterwards from the list, every lane
  // busy); keys 16..32 below the max add their exact mass to a per-thread register sum for the
  // single coarse bin.  Each segment then publishes its cumulative fine-bin counts and its fine
  // keys grouped by bin, so that after the next barrier any CTA can read the crossing bin's keys
  // of every other CTA directly.  The last CTA of a problem to finish (a ticket) reads the
  // problem's histogram and records Z, the target T, the crossing bin and its key count.
  const bool small_mass = a.sc_bits <= 54;  // then every coarse-bin mass fits 32 bits
  for (int si = 0; si < nseg; ++si) {
    const int p = S.seg[si].p;
    const int cf = cf_of(p, a), cl = cl_of(p, a);
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
    if (lane == 0) S.lres[si][warp] = (uint32_t)w_hi;
    __syncwarp();
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
        } else {  // list full: count this key now (later passes rescan from the first one)
          if (pos == kcap) S.lres[si][warp] = (uint32_t)k;
          uint32_t hi, lo;
          mass_words(v, m, scale, &hi, &lo);
          const int bi = (int)(x * 64.f);
          add_words(&S.h.w.lo[bi], &S.h.w.hi[bi], hi, lo);
          atomicAdd(&S.hc[bi], 1u);
        }
      }
      nkeep += __popc(bf);
    }
    if (lane == 0) S.lcnt[si][warp] = (uint32_t)min(nkeep, kcap);
    const int nl = min(nkeep, kcap);
    __syncwarp();  // list entries written by other lanes of this warp
    for (int i = lane; i < nl; i += 32) {
      const float v = sc[off + (int)kl[i]];
      const float x = m - v;
      uint32_t hi, lo;
      mass_words(v, m, scale, &hi, &lo);
      const int bi = (int)(x * 64.f);
      add_words(&S.h.w.lo[bi], &S.h.w.hi[bi], hi, lo);
      atomicAdd(&S.hc[bi], 1u);
    }
    coarse = warp_sum(coarse);
    if (lane == 0 && coarse) add_words(&S.h.w.lo[kFine], &S.h.w.hi[kFine], (uint32_t)(coarse >> 32), (uint32_t)coarse);
    __syncthreads();
    for (int i = tid; i <= kFine; i += kThreads) {
      const uint32_t lo = S.h.w.lo[i], hi = S.h.w.hi[i];
      if (lo | hi) atomicAdd(a.h1 + (int64_t)p * kBins + i, ((unsigned long long)hi << 32) | lo);
    }
    // cumulative fine-bin counts of this segment (one bin per thread), published
    a.cum[(int64_t)(p + c) * kFine + tid] = (uint32_t)block_incl_scan_u64(S.hc[tid], S);
    // the problem's arrival count: its designated CTA (the one holding the middle of its keys,
    // which holds no other problem whenever the problem spans three CTAs or more) waits for all
    // of them and summarises the histogram.  Waits only point to CTAs' contributions to the same
    // or lower-numbered problems, which no wait precedes, so they cannot form a cycle.
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      atomicAdd(a.pticket + p, 1u);
      S.cut_idx = c == cta_of((int64_t)p * a.N + a.N / 2, a) &&
                          wait_count(a.pticket + p, (uint32_t)(cl - cf + 1), a.err, a.wait_limit)
                      ? 1
                      : 0;
    }
    __syncthreads();
    if (S.cut_idx) {
      __threadfence();
      for (int i = tid; i < kBins; i += kThreads) {
        unsigned long long v = 0ull;
        if (i <= kFine) {
          v = __ldcg(a.h1 + (int64_t)p * kBins + i);
          a.h1[(int64_t)p * kBins + i] = 0ull;  // clean for the next launch
        }
        S.h.m[i] = v;
      }
      __syncthreads();
      select_summary(a, S, p, cf, cl);
    }
    __syncthreads();
  }
  if (!grid_sync(a.bar, G, a.err, a.wait_limit)) return;

  // Unless some problem needs the fallback (the launch's flag): each CTA adds its crossing-bin
  // keys to the problem's candidate list; the last CTA of the problem to do so finds the cut
  // for all of them; after the barrier every CTA writes its own positions.
  if (tid == 0) S.cut_idx = __ldcg(a.flags) == a.epoch ? 1 : 0;
  __syncthreads();
  if (S.cut_idx == 0) {
    __syncthreads();
    for (int si = 0; si < nseg; ++si) {
      const int p = S.seg[si].p;
      const int cf = cf_of(p, a), cl = cl_of(p, a);
      const int bstar = (int)(uint32_t)__ldcg(a.psum + kPsum * (int64_t)p + 3);
      const int off = (int)S.seg[si].off, jlo = (int)S.seg[si].jlo, rows = (int)(S.seg[si].jhi - S.seg[si].jlo);
      const float m = S.seg[si].m;
      const int wlen = (rows + kWarps - 1) / kWarps;
      const int w_lo = min(rows, warp * wlen), w_hi = min(rows, w_lo + wlen);
      const KeepT* kl = keep + S.seg[si].kbase + warp * S.seg[si].kcap;
      const int n_list = (int)S.lcnt[si][warp], res = (int)S.lres[si][warp];
      const int n_it = visit_count(false, w_lo, w_hi, n_list, res);
      for (int i = lane; i < n_it; i += 32) {
        const int k = visit_key(i, false, w_lo, kl, n_list, res);
        const float v = sc[off + k];
        if (bin_of(v, m) != bstar) continue;
        const uint32_t slot = atomicAdd(a.cand_cnt + p, 1u);
        if (slot < (uint32_t)kCand)
          a.cand[(int64_t)p * kCand + slot] = ((unsigned long long)order_key(v) << 32) | (0xFFFFFFFFu - (uint32_t)(jlo + k));
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) {  // arrive; the problem's designated CTA waits for all and finds the cut
        atomicAdd(a.pticket + p, 1u);
        S.cut_idx = c == cta_of((int64_t)p * a.N + a.N / 2, a) &&
                            wait_count(a.pticket + p, (uint32_t)(cl - cf + 1), a.err, a.wait_limit)
                        ? 1
                        : 0;
      }
      __syncthreads();
      if (S.cut_idx) {
        __threadfence();
        select_cut(a, S, p, cf, cl, m, scale);
      }
      __syncthreads();
    }
    if (!grid_sync(a.bar, G, a.err, a.wait_limit)) return;
    // every CTA has passed its last barrier: the last one to get here rewinds the barrier
    // counter so the next launch (whatever its grid size) starts from zero
    if (tid == 0 && atomicAdd(a.bar + 1, 1ull) == (unsigned long long)(G - 1)) {
      a.bar[0] = 0ull;
      a.bar[1] = 0ull;
    }
    for (int si = 0; si < nseg; ++si) {
      const Seg& s = S.seg[si];
      const int p = s.p;
      const uint32_t tk = (uint32_t)__ldcg(a.psum + kPsum * (int64_t)p + 4);
      const long long before = __ldcg(a.cres + 2 * (int64_t)(p + c)), take = __ldcg(a.cres + 2 * (int64_t)(p + c) + 1);
      // per-warp counts over the keep list (or the whole chunk), exclusive warp bases, then the
      // positions in ascending order: warp lists in warp order, ballots within 32-key steps
      const int off = (int)s.off, rows = (int)(s.jhi - s.jlo), jlo = (int)s.jlo;
      const int wlen = (rows + kWarps - 1) / kWarps;
      const int w_lo = min(rows, warp * wlen), w_hi = min(rows, w_lo + wlen);
      const KeepT* kl = keep + s.kbase + warp * s.kcap;
      const int n_list = (int)S.lcnt[si][warp], res = (int)S.lres[si][warp];
      const int n_it = visit_count(false, w_lo, w_hi, n_list, res);
      uint32_t wg = 0, we = 0;
      for (int i0 = 0; i0 < n_it; i0 += 32) {
        const int i = i0 + lane;
        uint32_t kk = 0u;
        if (i < n_it) kk = order_key(sc[off + visit_key(i, false, w_lo, kl, n_list, res)]);
        wg += __popc(__ballot_sync(0xffffffffu, i < n_it && kk > tk));
        we += __popc(__ballot_sync(0xffffffffu, i < n_it && kk == tk));
      }
      if (lane == 0) {
        S.wcnt[si][warp][0] = wg;
        S.wcnt[si][warp][1] = we;
      }
      __syncthreads();
      if (warp == 0) {  // exclusive warp bases (one warp, one lane per warp)
        uint32_t g1 = S.wcnt[si][lane][0], e1 = S.wcnt[si][lane][1];
        uint32_t gi = g1, ei = e1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t gy = __shfl_up_sync(0xffffffffu, gi, o), ey = __shfl_up_sync(0xffffffffu, ei, o);
          if (lane >= o) {
            gi += gy;
            ei += ey;
          }
        }
        S.wcnt[si][lane][0] = gi - g1;
        S.wcnt[si][lane][1] = ei - e1;
      }
      __syncthreads();
      long long g_run = S.wcnt[si][warp][0], e_run = S.wcnt[si][warp][1];
      const uint32_t lt = (1u << lane) - 1u;
      int32_t* dst = a.sel_idx + (int64_t)p * a.max_select;
      for (int i0 = 0; i0 < n_it; i0 += 32) {
        const int i = i0 + lane;
        int k = 0;
        uint32_t kk = 0u;
        if (i < n_it) {
          k = visit_key(i, false, w_lo, kl, n_list, res);
          kk = order_key(sc[off + k]);
        }
        const bool isg = i < n_it && kk > tk;
        const bool ise = i < n_it && kk == tk;
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
    return;
  }

  // ---- fallback (some problem's crossing bin is the coarse bin or holds more than kCand keys;
  // decided identically by every CTA from the launch's flag): the candidates of the problems
  // that fit are gathered by atomics, the others refine by radix levels over the key bits.
  for (int si = 0; si < nseg; ++si) {
    const int p = S.seg[si].p;
    if (tid == 0) {
      Seg& sg = S.seg[si];
      const unsigned long long* ps = a.psum + kPsum * (int64_t)p;
      sg.Z = __ldcg(ps);
      sg.T = __ldcg(ps + 1);
      sg.rem = __ldcg(ps + 2);
      const unsigned long long w3 = __ldcg(ps + 3);
      sg.bstar = (int)(uint32_t)w3;
      // the coarse bin cannot be resolved from the keep lists, nor a crossing bin with more keys
      // than the candidate list holds: those problems refine by radix
      sg.radix = sg.bstar >= kFine || (w3 >> 32) > (unsigned long long)kCand;
      if (sg.radix && c == cf_of(p, a)) atomicAdd(a.cand_cnt + p, (uint32_t)kCand + 1u);
    }
    __syncthreads();
    const int bstar = S.seg[si].bstar;
    if (!S.seg[si].radix) {
      const int off = (int)S.seg[si].off, jlo = (int)S.seg[si].jlo, rows = (int)(S.seg[si].jhi - S.seg[si].jlo);
      const float m = S.seg[si].m;
      const int wlen = (rows + kWarps - 1) / kWarps;
      const int w_lo = min(rows, warp * wlen), w_hi = min(rows, w_lo + wlen);
      const KeepT* kl = keep + S.seg[si].kbase + warp * S.seg[si].kcap;
      const int n_list = (int)S.lcnt[si][warp], res = (int)S.lres[si][warp];
      const int n_it = visit_count(false, w_lo, w_hi, n_list, res);
      for (int i = lane; i < n_it; i += 32) {
        const int k = visit_key(i, false, w_lo, kl, n_list, res);
        const float v = sc[off + k];
        if (bin_of(v, m) != bstar) continue;
        const uint32_t slot = atomicAdd(a.cand_cnt + p, 1u);
        if (slot < (uint32_t)kCand)
          a.cand[(int64_t)p * kCand + slot] = ((unsigned long long)order_key(v) << 32) | (0xFFFFFFFFu - (uint32_t)(jlo + k));
      }
    }
    __syncthreads();
  }
  if (!grid_sync(a.bar, G, a.err, a.wait_limit)) return;

  // exact cut.  Problems whose crossing bin fits the candidate list sort it; the others
  // (decided identically by every CTA from the global counts) refine by radix.
  constexpr bool fallback = true;
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
    const bool whole = S.seg[si].bstar >= kFine;
    const int wlen = (rows + kWarps - 1) / kWarps;
    const int w_lo = min(rows, warp * wlen), w_hi = min(rows, w_lo + wlen);
    const KeepT* kl = keep + S.seg[si].kbase + warp * S.seg[si].kcap;
    const int n_list = (int)S.lcnt[si][warp], res = (int)S.lres[si][warp];
    const int n_it = visit_count(whole, w_lo, w_hi, n_list, res);
    uint32_t wg = 0, we = 0;
    for (int i0 = 0; i0 < n_it; i0 += 32) {
      const int i = i0 + lane;
      uint32_t key = 0u;
      if (i < n_it) key = order_key(sc[off + visit_key(i, whole, w_lo, kl, n_list, res)]);
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
  if (fallback) zero_global_hist(a.hr, 3 * nh, c, G);
  for (int i = c * kThreads + tid; i < a.P; i += G * kThreads) a.cand_cnt[i] = 0u;

  for (int si = 0; si < nseg; ++si) {
    const Seg& s = S.seg[si];
    const int p = s.p;
    const int cf = cf_of(p, a), cl = cl_of(p, a);
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
    const bool whole = s.bstar >= kFine;
    const int wlen = (rows + kWarps - 1) / kWarps;
    const int w_lo = min(rows, warp * wlen), w_hi = min(rows, w_lo + wlen);
    const KeepT* kl = keep + s.kbase + warp * s.kcap;
    const int n_list = (int)S.lcnt[si][warp], res = (int)S.lres[si][warp];
    const int n_it = visit_count(whole, w_lo, w_hi, n_list, res);
    long long g_run = S.wcnt[si][warp][0], e_run = S.wcnt[si][warp][1];
    const uint32_t lt = (1u << lane) - 1u;
    int32_t* dst = a.sel_idx + (int64_t)p * a.max_select;
    for (int i0 = 0; i0 < n_it; i0 += 32) {
      const int i = i0 + lane;
      int k = 0;
      uint32_t key = 0u;
      if (i < n_it) {
        k = visit_key(i, whole, w_lo, kl, n_list, res);
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

// scores (fp32) + keep lists (16-bit, 3/8 of the keys plus per-warp rounding)
size_t select_var_smem(int64_t per) {
  return 4 * (size_t)((per + 3) / 4 * 4) + 2 * (size_t)(per * 3 / 8 + 1 + kWarps * (2 * kSelMaxSeg + 2));
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
  g.pair = 2 * per;
  g.even = per;
  const size_t fixed = select_fixed_smem();
  const size_t need = fixed + select_var_smem(per);
  g.smem_scores = need <= L->smem_optin;
  g.smem_bytes = g.smem_scores ? need : fixed;
  // one CTA on every SM: the even SM of each TPC takes the larger share of a pair's keys, if
  // the larger range still fits the same score storage and segment limit
  if (G == L->sm_count && G >= 2) {
    int64_t le = (int64_t)llround((double)(2 * per) * kSelEvenShare);
    if (le > (int64_t)(kSelMaxSeg - 1) * N) le = (int64_t)(kSelMaxSeg - 1) * N;
    if (le > per) {
      const size_t need_e = fixed + select_var_smem(le);
      if (!g.smem_scores || need_e <= L->smem_optin) {
        g.even = le;
        g.per_cta = le;
        if (g.smem_scores) g.smem_bytes = need_e;
        g.parity = true;
      }
    }
  }
  return g;
}

cudaError_t launch_decode_select(rtp_layer* L, const __nv_bfloat16* q_raw, cudaStream_t st) {
  const int64_t N = L->len;
  const SelectGeom g = select_geometry(L, N);
  SelectArgs a;
  a.idx = L->idx;
  a.idx_b = L->idx_b;
  a.idx_pstride = L->max_seq * kR;
  a.q_idx = L->q_idx;
  a.q_raw = q_raw;
  a.theta = L->theta;
  a.wq = L->wq;
  a.ret_head = L->d_ret_head;
  a.Hq = L->Hq;
  a.q_rot = L->q_rot;
  a.P = L->B * L->Hr;
  a.N = N;
  a.L = g.per_cta;
  a.Lp = g.pair;
  a.Le = g.even;
  a.use_smid = 0;
  a.Hr = L->Hr;
  a.lens = seq_pos(L, 0);
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
  a.h1 = reinterpret_cast<unsigned long long*>(L->sel_words);  // the first 2 * nh words
  a.hr = Hist3{L->sel_words + 3 * nh, L->sel_words + 6 * nh, L->sel_words + 9 * nh};
  a.cand_cnt = L->cand_cnt;
  a.cand = L->cand;
  a.slot_cnt = L->slot_cnt;
  a.bar = L->bar;
  a.err = L->err;
  a.gscores = L->gscores;
  a.keep = L->sel_keep;
  a.flags = L->sel_flags;
  if (++L->sel_epoch == 0u) L->sel_epoch = 1u;
  a.epoch = L->sel_epoch;
  a.cum = L->sel_cum;
  a.psum = L->sel_psum;
  a.cres = L->sel_cres;
  a.pticket = L->sel_pticket;
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
  // SM-numbered ranges need exactly one CTA on every SM; otherwise the same split by block index
  if (g.parity) a.use_smid = occ == 1 ? 1 : 0;
  return cudaLaunchCooperativeKernel(fn, dim3(g.grid), dim3(kThreads), args, g.smem_bytes, st);
}

}  // namespace rtp
