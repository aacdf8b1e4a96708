// decode_select.cu -- decode-time index scoring fused with the exact top-p selection.
//
// For every problem p = (sequence b, retrieval head h) the kernel
//   1. streams the 16-dim index keys IDX[p][0..N) from HBM and computes the pre-RoPE
//      scores s_j = qidx . IDX[p][j] (techwalker page, section 3: the 16-dim "radar");
//   2. finds the exact top-p set: the shortest prefix of the order (s desc, j asc) whose
//      index-softmax mass reaches p (zhichai page, insight 3; techwalker page, section 4),
//      without sorting -- by mass histograms, as the pages' kernel does (techwalker page,
//      section 6: 256 buckets, no sort, fused with scoring), refined until the cut is exact;
//   3. writes the selected positions in ascending order.
//
// B200 design
//   * One cooperative grid of <= #SM CTAs x 1024 threads.  The flat (problem, key) range is
//     split evenly; each CTA keeps its scores in shared memory (up to ~50K per CTA, 7.4M per
//     launch), so the histogram passes never touch HBM again.  Larger launches keep the
//     scores in a global scratch array (L2-resident at these sizes) instead.
//   * The index stream uses 16-byte non-allocating loads: four threads own one 64-byte row,
//     so every warp load is a fully coalesced 512-byte segment.
//   * Softmax masses are exp(s - m) in fp32, quantised to 64-bit fixed point (2^sc scale with
//     N * 2^sc < 2^63).  Integer sums are exact and associative, so the selection is
//     deterministic and identical however the work is split; integer atomics build the
//     histograms.  The quantisation error on the total mass is below N * 2^-(sc+1)
//     (< 1.2e-7 of the largest key's mass at N = 2^20).
//   * Level 1: 2048 bins of width 1/64 in (m - s) (last bin: everything 32 or more below
//     the max).  Levels 2-4: radix digits (11, 11, 10 bits) of the order-preserving key bits
//     of the elements in the crossing bin.  Each level stops early when its crossing group
//     holds a single key.  After the last level the cut score t is exact; ties at t are
//     taken in ascending position order.
//   * Grid barriers are bounded waits (about 1 s); on timeout the error word records
//     RTP_ETIMEOUT and the kernel returns.
#include <cooperative_groups.h>

#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr int kBins = kSelBins;
constexpr int kThreads = kSelThreads;
constexpr int kWarps = kThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;
// radix levels inside the crossing bin: key bits [31:21], [20:10], [9:0]
__device__ __forceinline__ int level_shift(int l) { return l == 0 ? 21 : (l == 1 ? 10 : 0); }
__device__ __forceinline__ int level_bits(int l) { return l == 2 ? 10 : 11; }

struct SelectArgs {
  const float* idx;
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
  float* seg_max;  // [P + G]
  unsigned long long* h1_mass;
  uint32_t* h1_cnt;
  unsigned long long* hr_mass;  // [3][P][bins]
  uint32_t* hr_cnt;
  uint32_t* slot_cnt;  // [P + G][2]
  uint32_t* bar;
  uint32_t* err;
  float* gscores;
};

struct Seg {
  int p;
  int done;      // 1 once the tie group is known
  int shift_f;   // 32: tie group = the whole crossing bin; else key >> shift_f == prefix
  int bstar;
  int64_t jlo, jhi, off;
  float m;
  uint32_t prefix;
  unsigned long long Z, T, rem, e_t, n_need;
};

struct Smem {
  unsigned long long hm[kBins];
  uint32_t hc[kBins];
  Seg seg[kSelMaxSeg];
  unsigned long long red64[kWarps];
  uint32_t red32[kWarps];
  float redf[kWarps];
  int cross;
  unsigned long long cross_above;
  long long before, take;
  uint32_t slot[2 * kThreads];  // (gt, eq) counts of the CTAs that share a problem
};

__device__ __forceinline__ unsigned long long mass_of(float s, float m, float scale) {
  return __float2ull_rn(fast_exp2((s - m) * kLog2e) * scale);
}
__device__ __forceinline__ int bin_of(float s, float m) {
  int b = (int)((m - s) * 64.f);
  return b < kBins - 1 ? b : kBins - 1;
}

__device__ float block_max(float v, Smem& S) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) S.redf[w] = v;
  __syncthreads();
  if (w == 0) {
    v = l < kWarps ? S.redf[l] : -INFINITY;
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
    v = l < kWarps ? S.red64[l] : 0ull;
    v = warp_sum(v);
    if (l == 0) S.red64[0] = v;
  }
  __syncthreads();
  return S.red64[0];
}

// In S.hm order (reverse: index kBins-1 first), find the first position whose inclusive
// cumulative mass reaches target.  Result: S.cross = bin, S.cross_above = mass before it.
__device__ void find_crossing(Smem& S, bool reverse, unsigned long long target) {
  const int t = threadIdx.x, w = t >> 5, l = t & 31;
  const int p0 = 2 * t, p1 = 2 * t + 1;
  const int b0 = reverse ? kBins - 1 - p0 : p0;
  const int b1 = reverse ? kBins - 1 - p1 : p1;
  const unsigned long long m0 = S.hm[b0], m1 = S.hm[b1];
  unsigned long long incl = m0 + m1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (l >= o) incl += y;
  }
  __syncthreads();
  if (l == 31) S.red64[w] = incl;
  if (t == 0) S.cross = -1;
  __syncthreads();
  if (w == 0) {
    unsigned long long x = S.red64[l];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (l >= o) x += y;
    }
    S.red64[l] = x;  // inclusive warp totals
  }
  __syncthreads();
  const unsigned long long base = (w > 0 ? S.red64[w - 1] : 0ull) + incl - (m0 + m1);
  if (base < target && base + m0 >= target) {
    S.cross = b0;
    S.cross_above = base;
  } else if (base + m0 < target && base + m0 + m1 >= target) {
    S.cross = b1;
    S.cross_above = base + m0;
  }
  __syncthreads();
}

__device__ __forceinline__ void zero_smem_hist(Smem& S) {
  for (int i = threadIdx.x; i < kBins; i += kThreads) {
    S.hm[i] = 0ull;
    S.hc[i] = 0u;
  }
}

__device__ __forceinline__ void flush_hist(Smem& S, unsigned long long* gm, uint32_t* gc) {
  for (int i = threadIdx.x; i < kBins; i += kThreads) {
    const uint32_t c = S.hc[i];
    if (c) {
      atomicAdd(gm + i, S.hm[i]);
      atomicAdd(gc + i, c);
    }
  }
}

__device__ __forceinline__ void load_hist(Smem& S, const unsigned long long* gm, const uint32_t* gc) {
  for (int i = threadIdx.x; i < kBins; i += kThreads) {
    S.hm[i] = __ldcg(gm + i);
    S.hc[i] = __ldcg(gc + i);
  }
  __syncthreads();
}

// Exclusive block scan of a packed (gt << 16 | eq) counter; returns the exclusive prefix,
// total in *tot.
__device__ uint32_t block_scan_u32(uint32_t v, Smem& S, uint32_t* tot) {
  const int t = threadIdx.x, w = t >> 5, l = t & 31;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (l >= o) incl += y;
  }
  __syncthreads();
  if (l == 31) S.red32[w] = incl;
  __syncthreads();
  if (w == 0) {
    uint32_t x = S.red32[l];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (l >= o) x += y;
    }
    S.red32[l] = x;
  }
  __syncthreads();
  *tot = S.red32[kWarps - 1];
  return (w > 0 ? S.red32[w - 1] : 0u) + incl - v;
}

template <bool kSmemScores>
__global__ void __launch_bounds__(kThreads, 1) decode_select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  const int c = blockIdx.x;
  const uint32_t G = gridDim.x;
  const int tid = threadIdx.x;
  const int64_t total = (int64_t)a.P * a.N;
  const int64_t r0 = (int64_t)c * a.L;
  const int64_t r1 = min(total, r0 + a.L);
  float* sc = kSmemScores ? reinterpret_cast<float*>(smem_raw + sizeof(Smem)) : a.gscores + r0;
  const float scale = __uint_as_float((uint32_t)(127 + a.sc_bits) << 23);  // 2^sc

  // ---- segments of this CTA
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
      s.done = 0;
      s.shift_f = 32;
      s.prefix = 0;
    }
  }
  __syncthreads();

  // ---- phase A: zero global histograms; stream index keys -> scores, segment maxima
  {
    const int64_t nh = (int64_t)a.P * kBins;
    for (int64_t i = (int64_t)c * kThreads + tid; i < nh; i += (int64_t)G * kThreads) {
      a.h1_mass[i] = 0ull;
      a.h1_cnt[i] = 0u;
      a.hr_mass[i] = 0ull;
      a.hr_cnt[i] = 0u;
      a.hr_mass[nh + i] = 0ull;
      a.hr_cnt[nh + i] = 0u;
      a.hr_mass[2 * nh + i] = 0ull;
      a.hr_cnt[2 * nh + i] = 0u;
    }
  }
  const int quad = tid >> 2, part = tid & 3;
  for (int si = 0; si < nseg; ++si) {
    const Seg s = S.seg[si];
    const int64_t rows = s.jhi - s.jlo;
    const float4* src = reinterpret_cast<const float4*>(a.idx + (int64_t)s.p * a.idx_pstride) + s.jlo * 4;
    const float4 qv = reinterpret_cast<const float4*>(a.q_idx + (int64_t)s.p * kR)[part];
    float mx = -INFINITY;
    // The trip count is the same for every thread (the shuffles below are full-warp);
    // rows past the end are loaded as zeros and not stored.
    for (int64_t base = 0; base < rows; base += 4 * (kThreads / 4)) {
      const int64_t k0 = base + quad;
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t k = k0 + u * (kThreads / 4);
        v[u] = k < rows ? ld_stream_f4(src + k * 4 + part) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float d = v[u].x * qv.x;
        d = fmaf(v[u].y, qv.y, d);
        d = fmaf(v[u].z, qv.z, d);
        d = fmaf(v[u].w, qv.w, d);
        d += __shfl_xor_sync(0xffffffffu, d, 1);
        d += __shfl_xor_sync(0xffffffffu, d, 2);
        d += 0.0f;  // -0 -> +0: equal scores must get equal order keys
        const int64_t k = k0 + u * (kThreads / 4);
        if (k < rows) {
          mx = fmaxf(mx, d);
          if (part == 0) sc[s.off + k] = d;
        }
      }
    }
    mx = block_max(mx, S);
    if (tid == 0) a.seg_max[s.p + c] = mx;
  }
  if (!grid_barrier(a.bar, a.bar + 1, G, a.err)) return;

  // ---- phase B: row maxima; level-1 mass histograms
  for (int si = 0; si < nseg; ++si) {
    const int p = S.seg[si].p;
    const int cf = (int)(((int64_t)p * a.N) / a.L), cl = (int)(((int64_t)p * a.N + a.N - 1) / a.L);
    float mv = -INFINITY;
    for (int cc = cf + tid; cc <= cl; cc += kThreads) mv = fmaxf(mv, __ldcg(a.seg_max + p + cc));
    const float m = block_max(mv, S);
    zero_smem_hist(S);
    if (tid == 0) S.seg[si].m = m;
    __syncthreads();
    const Seg& s = S.seg[si];
    const int64_t rows = s.jhi - s.jlo;
    for (int64_t k = tid; k < rows; k += kThreads) {
      const float v = sc[s.off + k];
      const int b = bin_of(v, m);
      atomicAdd(&S.hm[b], mass_of(v, m, scale));
      atomicAdd(&S.hc[b], 1u);
    }
    __syncthreads();
    flush_hist(S, a.h1_mass + (int64_t)p * kBins, a.h1_cnt + (int64_t)p * kBins);
    __syncthreads();
  }
  if (!grid_barrier(a.bar, a.bar + 1, G, a.err)) return;

  // ---- phase C: total mass, target, crossing bin; radix level 0 inside it
  for (int si = 0; si < nseg; ++si) {
    const int p = S.seg[si].p;
    load_hist(S, a.h1_mass + (int64_t)p * kBins, a.h1_cnt + (int64_t)p * kBins);
    unsigned long long part_sum = 0;
    for (int i = tid; i < kBins; i += kThreads) part_sum += S.hm[i];
    const unsigned long long Z = block_sum_u64(part_sum, S);
    unsigned long long T = (unsigned long long)ceil((double)a.top_p * (double)Z);
    if (T < 1ull) T = 1ull;
    if (T > Z) T = Z;
    find_crossing(S, false, T);
    if (tid == 0) {
      Seg& s = S.seg[si];
      s.Z = Z;
      s.T = T;
      s.bstar = S.cross;
      s.rem = T - S.cross_above;
      if (S.cross < 0) {
        atomicOr(a.err, kErrInternal);
        s.bstar = 0;
        s.rem = 1;
      }
      if (S.hc[s.bstar] == 1u) {  // a single key carries the cut
        s.done = 1;
        s.shift_f = 32;
        s.e_t = S.hm[s.bstar];
        s.n_need = 1;
      }
    }
    __syncthreads();
    const Seg& s = S.seg[si];
    if (s.done) continue;
    zero_smem_hist(S);
    __syncthreads();
    const int64_t rows = s.jhi - s.jlo;
    for (int64_t k = tid; k < rows; k += kThreads) {
      const float v = sc[s.off + k];
      if (bin_of(v, s.m) != s.bstar) continue;
      const uint32_t d = order_key(v) >> level_shift(0);
      atomicAdd(&S.hm[d], mass_of(v, s.m, scale));
      atomicAdd(&S.hc[d], 1u);
    }
    __syncthreads();
    flush_hist(S, a.hr_mass + (int64_t)p * kBins, a.hr_cnt + (int64_t)p * kBins);
    __syncthreads();
  }
  if (!grid_barrier(a.bar, a.bar + 1, G, a.err)) return;

  // ---- phases D, E: radix levels 1 and 2 (after reading levels 0 and 1)
  for (int lev = 1; lev <= 2; ++lev) {
    const int64_t nh = (int64_t)a.P * kBins;
    for (int si = 0; si < nseg; ++si) {
      const Seg s0 = S.seg[si];
      if (s0.done) continue;
      const int p = s0.p;
      load_hist(S, a.hr_mass + (lev - 1) * nh + (int64_t)p * kBins,
                a.hr_cnt + (lev - 1) * nh + (int64_t)p * kBins);
      find_crossing(S, true, s0.rem);
      if (tid == 0) {
        Seg& s = S.seg[si];
        const int d = S.cross < 0 ? 0 : S.cross;
        if (S.cross < 0) atomicOr(a.err, kErrInternal);
        s.prefix = (lev == 1) ? (uint32_t)d : ((s.prefix << level_bits(lev - 1)) | (uint32_t)d);
        s.rem -= S.cross_above;
        s.shift_f = level_shift(lev - 1);
        if (S.hc[d] == 1u) {
          s.done = 1;
          s.e_t = S.hm[d];
          s.n_need = 1;
        }
      }
      __syncthreads();
      const Seg& s = S.seg[si];
      if (s.done) continue;
      zero_smem_hist(S);
      __syncthreads();
      const int64_t rows = s.jhi - s.jlo;
      for (int64_t k = tid; k < rows; k += kThreads) {
        const float v = sc[s.off + k];
        if (bin_of(v, s.m) != s.bstar) continue;
        const uint32_t key = order_key(v);
        if ((key >> s.shift_f) != s.prefix) continue;
        const uint32_t d = (key >> level_shift(lev)) & ((1u << level_bits(lev)) - 1u);
        atomicAdd(&S.hm[d], mass_of(v, s.m, scale));
        atomicAdd(&S.hc[d], 1u);
      }
      __syncthreads();
      flush_hist(S, a.hr_mass + lev * nh + (int64_t)p * kBins, a.hr_cnt + lev * nh + (int64_t)p * kBins);
      __syncthreads();
    }
    if (!grid_barrier(a.bar, a.bar + 1, G, a.err)) return;
  }

  // ---- phase F: exact cut from level 2; count keys above the tie group and in it
  {
    const int64_t nh = (int64_t)a.P * kBins;
    for (int si = 0; si < nseg; ++si) {
      const Seg s0 = S.seg[si];
      const int p = s0.p;
      if (!s0.done) {
        load_hist(S, a.hr_mass + 2 * nh + (int64_t)p * kBins, a.hr_cnt + 2 * nh + (int64_t)p * kBins);
        find_crossing(S, true, s0.rem);
        if (tid == 0) {
          Seg& s = S.seg[si];
          const int d = S.cross < 0 ? 0 : S.cross;
          if (S.cross < 0 || S.hc[d] == 0u) atomicOr(a.err, kErrInternal);
          s.prefix = (s.prefix << level_bits(2)) | (uint32_t)d;
          s.rem -= S.cross_above;
          s.shift_f = 0;
          const uint32_t cnt = S.hc[d] ? S.hc[d] : 1u;
          s.e_t = S.hm[d] / cnt;  // equal keys carry equal masses
          s.n_need = s.e_t ? (s.rem + s.e_t - 1) / s.e_t : (unsigned long long)cnt;
          if (s.n_need > cnt) s.n_need = cnt;
          s.done = 1;
        }
        __syncthreads();
      }
      const Seg& s = S.seg[si];
      uint32_t gt = 0, eq = 0;
      const int64_t rows = s.jhi - s.jlo;
      for (int64_t k = tid; k < rows; k += kThreads) {
        const float v = sc[s.off + k];
        const int b = bin_of(v, s.m);
        if (b < s.bstar) {
          ++gt;
        } else if (b == s.bstar) {
          if (s.shift_f == 32) {
            ++eq;
          } else {
            const uint32_t kk = order_key(v) >> s.shift_f;
            gt += kk > s.prefix;
            eq += kk == s.prefix;
          }
        }
      }
      gt = (uint32_t)block_sum_u64(gt, S);
      eq = (uint32_t)block_sum_u64(eq, S);
      if (tid == 0) {
        a.slot_cnt[2 * (p + c)] = gt;
        a.slot_cnt[2 * (p + c) + 1] = eq;
      }
    }
  }
  if (!grid_barrier(a.bar, a.bar + 1, G, a.err)) return;

  // ---- phase G: offsets across CTAs, ordered compaction of the selected positions
  for (int si = 0; si < nseg; ++si) {
    const Seg& s = S.seg[si];
    const int p = s.p;
    const int cf = (int)(((int64_t)p * a.N) / a.L), cl = (int)(((int64_t)p * a.N + a.N - 1) / a.L);
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
    }
    __syncthreads();
    const long long before = S.before, take = S.take;
    long long gt_run = 0, eq_run = 0;
    const int64_t rows = s.jhi - s.jlo;
    for (int64_t k0 = 0; k0 < rows; k0 += kThreads) {
      const int64_t k = k0 + tid;
      uint32_t isgt = 0, iseq = 0;
      if (k < rows) {
        const float v = sc[s.off + k];
        const int b = bin_of(v, s.m);
        if (b < s.bstar) {
          isgt = 1;
        } else if (b == s.bstar) {
          if (s.shift_f == 32) {
            iseq = 1;
          } else {
            const uint32_t kk = order_key(v) >> s.shift_f;
            isgt = kk > s.prefix;
            iseq = kk == s.prefix;
          }
        }
      }
      uint32_t tot;
      const uint32_t ex = block_scan_u32((isgt << 16) | iseq, S, &tot);
      const long long gt_b = gt_run + (ex >> 16), eq_b = eq_run + (ex & 0xFFFFu);
      const bool take_me = isgt || (iseq && eq_b < take);
      if (take_me) {
        const long long pos = before + gt_b + (eq_b < take ? eq_b : take);
        if (pos < a.max_select) {
          a.sel_idx[(int64_t)p * a.max_select + pos] = (int32_t)(s.jlo + k);
        } else {
          atomicOr(a.err, kErrOverflow);
        }
      }
      gt_run += tot >> 16;
      eq_run += tot & 0xFFFFu;
    }
    if (c == cl && tid == 0) {
      const long long K = before + gt_run + take;
      a.sel_cnt[p] = (int32_t)(K < a.max_select ? K : a.max_select);
      const unsigned long long msel = (s.T - s.rem) + s.n_need * s.e_t;
      a.sel_mass[p] = (float)((double)msel / (double)s.Z);
      a.sel_thr[p] = (float)((double)s.e_t / (double)s.Z);
    }
    __syncthreads();
  }
}

}  // namespace

size_t select_fixed_smem() { return (sizeof(Smem) + 127) / 128 * 128; }

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
  const size_t need = fixed + (size_t)per * sizeof(float);
  g.smem_scores = need <= L->smem_optin;
  g.smem_bytes = g.smem_scores ? need : fixed;
  return g;
}

cudaError_t launch_decode_select(rtp_layer* L, cudaStream_t st) {
  const int64_t N = L->len;
  const SelectGeom g = select_geometry(L, N);
  SelectArgs a;
  a.idx = L->idx;
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
  a.h1_mass = L->h1_mass;
  a.h1_cnt = L->h1_cnt;
  a.hr_mass = L->hr_mass;
  a.hr_cnt = L->hr_cnt;
  a.slot_cnt = L->slot_cnt;
  a.bar = L->bar;
  a.err = L->err;
  a.gscores = L->gscores;
  if (!g.smem_scores && L->gscores == nullptr) return cudaErrorInvalidValue;
  if (g.grid > L->sm_count) return cudaErrorInvalidValue;
  void* args[] = {&a};
  const void* fn = g.smem_scores ? (const void*)decode_select_kernel<true> : (const void*)decode_select_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.smem_bytes);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kThreads, g.smem_bytes);
  if (e != cudaSuccess) return e;
  if (occ < 1 || g.grid > occ * L->sm_count) return cudaErrorCooperativeLaunchTooLarge;
  e = cudaLaunchCooperativeKernel(fn, dim3(g.grid), dim3(kThreads), args, g.smem_bytes, st);
  return e;
}

}  // namespace rtp
