// prefill_retrieval.cu -- retrieval heads in chunked prefill: per-row exact top-p, then sparse
// attention over the selected keys.
//
// Every query row i of the chunk (position pos = len - C + i) runs its own selection over its
// causal prefix j <= pos: pre-RoPE index scores s_j = qidx_i . kidx_j (techwalker page, section
// 3), the shortest prefix of the order (s desc, j asc) whose index-softmax mass reaches p
// (zhichai page, insight 3; techwalker page, section 4), then exact RoPE'd attention over that
// set.  (The pages' own prefill keeps retrieval heads dense -- techwalker page, Q&A; ngjoo
// digest, limitations -- the per-row selection here is the chunked-prefill counterpart of the
// decode selection.)
//
// Two kernels, one CTA per (64-row tile, retrieval head, sequence), 128 threads each; scores
// come from index_mma.cuh (tensor cores, identical bits in every pass):
//
//  prefill_select_kernel -- the exact cut (t_key, tiecut) of each row, in passes over the
//    row's causal keys, all arithmetic exact in 64-bit fixed point (mass of key j =
//    round(2^sc * e^(s_j - m)), sc = 62 - ceil(log2 len)):
//      A  row maxima m;
//      B  16 bins of m - s rounded to an integer (the last one holding everything from 14.5
//         down) -> Z, T = ceil(p Z), crossing bin, whose exact order-key range is found by
//         bisection;
//      R  refinement: the crossing range of order keys is split 16 ways by bit slices, with
//         the mass of each slice and the first keys of the range captured; once a row's
//         range holds <= 16 keys they are sorted (key desc, j asc) for the exact cut; a range
//         that shrinks to one key value is an exact tie group, resolved by
//      T  an ordered count of the tied positions.
//  prefill_attn_kernel -- recomputes the scores, applies each row's cut, ORs the rows' masks
//    of every 64-key tile into the tile's union, compacts the union keys of successive tiles
//    into 64-key chunks (positions + per-row bits) and runs the attention tiles (fa_tile.cuh)
//    on the gathered K/V rows of each full chunk; tiles no row selects cost only their scores.
#include "fa_tile.cuh"
#include "index_mma.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr int kRows = 64;
constexpr int kThreads = kIdxThreads;  // 128
constexpr int kBins = 16;
constexpr int kCand = 4;               // candidates captured per thread and row slot
constexpr float kLog2e = 1.4426950408889634f;

enum : int { kModeKeys = 1, kModeTie = 2, kModeDone = 3 };

struct RetArgs {
  const __half* idx;          // [B][Hr][max_seq][hi r | lo r]: the split index cache
  const __half* kc;
  const __half* vc;
  int64_t max_seq;
  int Hkv, Hq, Hr, group, C;
  int64_t P0;
  float top_p;
  int sc_bits;
  const int16_t* ret_head;    // [Hr]
  const float* q_rot;         // [B][C][Hq][D]
  const float* q_idx;         // [B][C][Hr][r]
  uint2* cut;                 // [B][Hr][C]: (t_key, tiecut)
  float scale_log2;
  float* out;                 // [B][C][Hq][D]
  int32_t* sel_count;         // [B][C][Hr] or nullptr
  float* sel_mass;            // [B][C][Hr] or nullptr
  uint32_t* bitmap;           // [B][C][Hr][bitmap_words] or nullptr
  int64_t bitmap_words;
  const int32_t* rows;        // [n_rows] chunk rows whose positions are listed, or nullptr
  int n_rows;
  int32_t* row_sel;           // [B][n_rows][Hr][row_sel_cap]
  int64_t row_sel_cap;
  uint32_t* err;
};

struct RowS {
  float m;
  int mode, cb, shift, found, tiecut;
  uint32_t klo, khi, t_key;
  unsigned long long Z, rem, above, n_need, tie_before;
};

// Per-thread exact histograms: a 64-bit mass is added as three 21-bit limbs with shared-memory
// reductions (no read-modify-write chains); limb sums stay below 2^32 because every thread
// folds its carries at least every kFoldTiles tiles (at most 16 keys per row slot per tile).
constexpr int kLimbs = 3;
constexpr int kFoldTiles = 128;

struct SmemSel {
  IdxRing st;                                     // 12 KB
  uint32_t h[kBins][2][kLimbs][kThreads];         // 48 KB
  unsigned long long cand[kCand][2][kThreads];    // 8 KB
  int nc[2][kThreads];
  RowS row[kRows];
};

__device__ __forceinline__ void red_add(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Add mass v to bin b of row slot sl of this thread (three limb reductions).
__device__ __forceinline__ void hist_add(SmemSel& S, int b, int sl, int tid, unsigned long long v) {
  const uint32_t a0 = smem_u32(&S.h[b][sl][0][tid]);
  red_add(a0, (uint32_t)v & 0x1FFFFFu);
  red_add(a0 + kThreads * 4, (uint32_t)(v >> 21) & 0x1FFFFFu);
  red_add(a0 + 2 * kThreads * 4, (uint32_t)(v >> 42));
}

__device__ __forceinline__ unsigned long long hist_get(const SmemSel& S, int b, int sl, int t) {
  return (unsigned long long)S.h[b][sl][0][t] + ((unsigned long long)S.h[b][sl][1][t] << 21) +
         ((unsigned long long)S.h[b][sl][2][t] << 42);
}

// Fold this thread's limb carries (its own entries only; same-thread order suffices).
__device__ __forceinline__ void hist_fold(SmemSel& S, int tid) {
  for (int b = 0; b < kBins; ++b)
    for (int sl = 0; sl < 2; ++sl) {
      const unsigned long long v = hist_get(S, b, sl, tid);
      S.h[b][sl][0][tid] = (uint32_t)v & 0x1FFFFFu;
      S.h[b][sl][1][tid] = (uint32_t)(v >> 21) & 0x1FFFFFu;
      S.h[b][sl][2][tid] = (uint32_t)(v >> 42);
    }
}

__device__ __forceinline__ void hist_zero(SmemSel& S, int tid) {
  for (int b = 0; b < kBins; ++b)
    for (int sl = 0; sl < 2; ++sl)
      for (int l = 0; l < kLimbs; ++l) S.h[b][sl][l][tid] = 0u;
}

// Fixed-point mass of a score s below the row max m: e^(s - m) * 2^sc truncated to an integer
// (scale = 2^sc as a float, exact).
__device__ __forceinline__ unsigned long long mass64(float s, float m, float scale) {
  return __float2ull_rz(fast_exp2((s - m) * kLog2e) * scale);
}

// level-1 bin of x = m - s >= 0: x rounded to the nearest integer (adding 2^23 does the rounding),
// with everything from 14.5 down in the last bin.  Non-increasing in s.
__device__ __forceinline__ int bin1_of(float x) {
  const uint32_t r = __float_as_uint(x + 8388608.0f) - 0x4B000000u;
  return (int)min(r, (uint32_t)(kBins - 1));
}

// Exact order-key range [lo, hi] of the finite scores s <= m whose level-1 bin is b (bisection
// on the monotone map key -> bin).
__device__ __forceinline__ void bin_key_range(float m, int b, uint32_t* lo, uint32_t* hi) {
  const uint32_t kmin = order_key(-3.4028234663852886e38f), kmax = order_key(m);
  auto bin_of_key = [&](uint32_t k) { return bin1_of(m - key_to_float(k)); };
  // first key with bin <= b
  uint32_t l = kmin, h = kmax;
  while (l < h) {
    const uint32_t mid = l + ((h - l) >> 1);
    if (bin_of_key(mid) <= b) h = mid;
    else l = mid + 1;
  }
  *lo = l;
  // last key with bin >= b: one below the first key with bin < b (kmax + 1 if none)
  if (b == 0) {
    *hi = kmax;
    return;
  }
  l = *lo;
  h = kmax;
  if (bin_of_key(h) >= b) {
    *hi = h;
    return;
  }
  while (l < h) {
    const uint32_t mid = l + ((h - l) >> 1);
    if (bin_of_key(mid) < b) h = mid;
    else l = mid + 1;
  }
  *hi = l - 1;
}

__device__ __forceinline__ int slice_shift(uint32_t klo, uint32_t khi) {
  const uint32_t d = khi - klo;  // span - 1
  const int bits = 32 - __clz(d);
  return bits > 4 ? bits - 4 : 0;
}

struct RowCtx {
  int tid, warp, gr, tq;
  int ra, rb;          // CTA rows of slot 0 / 1
  int64_t pa, pb;      // their positions (-1: inactive row)
  int64_t pos_lo;      // position of CTA row 0 (every active row is at or after it)
  int64_t nkeys;       // keys the CTA's rows can see
};

__device__ __forceinline__ RowCtx row_ctx(const RetArgs& a, int i0, int nrows) {
  RowCtx x;
  x.tid = threadIdx.x;
  x.warp = x.tid >> 5;
  x.gr = (x.tid & 31) >> 2;
  x.tq = x.tid & 3;
  x.ra = 16 * x.warp + x.gr;
  x.rb = x.ra + 8;
  x.pa = x.ra < nrows ? a.P0 + i0 + x.ra : -1;
  x.pb = x.rb < nrows ? a.P0 + i0 + x.rb : -1;
  x.pos_lo = a.P0 + i0;
  x.nkeys = a.P0 + i0 + nrows;
  return x;
}

// Pipelined walk over the index tiles of keys [0, nkeys): body(t, stage) runs once tile t is
// in ring stage `stage` (kIdxStages - 1 tiles in flight, one barrier per tile).
template <typename Body>
__device__ __forceinline__ void idx_walk(IdxRing& R, const __half* base, int64_t nkeys, Body body) {
  const int64_t ntiles = (nkeys + kIdxKeys - 1) / kIdxKeys;
#pragma unroll
  for (int s = 0; s < kIdxStages - 1; ++s) {
    if (s < ntiles) idx_issue(R, s, base, s, nkeys);
    cp_async_commit();
  }
  for (int64_t t = 0; t < ntiles; ++t) {
    cp_async_wait<kIdxStages - 2>();
    __syncthreads();  // tile t landed for every thread; stage (t - 1) % kIdxStages is free
    const int64_t tn = t + kIdxStages - 1;
    if (tn < ntiles) idx_issue(R, (int)(tn % kIdxStages), base, tn, nkeys);
    cp_async_commit();
    body(t, (int)(t % kIdxStages));
  }
  cp_async_wait<0>();
  __syncthreads();
}

// Run f(slot, j, s) over this thread's causal (row, key) pairs, tile by tile; fold() runs
// after every kFoldTiles tiles.
template <typename F, typename G>
__device__ __forceinline__ void scan(IdxRing& S, const RowCtx& x, const __half* ibase, const uint32_t qh[4],
                                     const uint32_t ql[4], F f, G fold) {
  idx_walk(S, ibase, x.nkeys, [&](int64_t t, int stage) {
    if (t > 0 && t % kFoldTiles == 0) fold();
    float c[8][4];
    idx_scores(c, qh, ql, S, stage);
    const int64_t base = t * kIdxKeys;
    // causal limits of the two rows inside this tile (-1: none, 63: all)
    const int la = (int)max((int64_t)-1, min((int64_t)(kIdxKeys - 1), x.pa - base));
    const int lb = (int)max((int64_t)-1, min((int64_t)(kIdxKeys - 1), x.pb - base));
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int p = 8 * nt + 2 * x.tq + e;
        if (p <= la) f(0, base + p, c[nt][e]);
        if (p <= lb) f(1, base + p, c[nt][2 + e]);
      }
    }
  });
}

// As scan, for passes that touch few keys: gate(slot, s) is evaluated branch-free for every
// pair, and f runs only on pairs that pass it, after one warp vote per tile.
template <typename Gate, typename F, typename G>
__device__ __forceinline__ void scan_gated(IdxRing& S, const RowCtx& x, const __half* ibase, const uint32_t qh[4],
                                           const uint32_t ql[4], Gate gate, F f, G fold) {
  idx_walk(S, ibase, x.nkeys, [&](int64_t t, int stage) {
    if (t > 0 && t % kFoldTiles == 0) fold();
    float c[8][4];
    idx_scores(c, qh, ql, S, stage);
    const int64_t base = t * kIdxKeys;
    const int la = (int)max((int64_t)-1, min((int64_t)(kIdxKeys - 1), x.pa - base));
    const int lb = (int)max((int64_t)-1, min((int64_t)(kIdxKeys - 1), x.pb - base));
    uint32_t hit = 0;  // bit 2*(2nt+e)+slot
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int p = 8 * nt + 2 * x.tq + e;
        const int k = 2 * nt + e;
        hit |= (uint32_t)(p <= la && gate(0, c[nt][e])) << (2 * k);
        hit |= (uint32_t)(p <= lb && gate(1, c[nt][2 + e])) << (2 * k + 1);
      }
    }
    if (!__any_sync(0xffffffffu, hit != 0u)) return;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int p = 8 * nt + 2 * x.tq + e;
        const int k = 2 * nt + e;
        if (hit & (1u << (2 * k))) f(0, base + p, c[nt][e]);
        if (hit & (1u << (2 * k + 1))) f(1, base + p, c[nt][2 + e]);
      }
    }
  });
}

__global__ void __launch_bounds__(kThreads) prefill_select_kernel(RetArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SmemSel& S = *reinterpret_cast<SmemSel*>(smem_raw);
  const int tile = gridDim.x - 1 - blockIdx.x, hr = blockIdx.y, b = blockIdx.z;  // longest rows first
  const int i0 = tile * kRows;
  const int nrows = min(kRows, a.C - i0);
  const RowCtx x = row_ctx(a, i0, nrows);
  const int tid = x.tid;
  const bool owner = x.tq == 0;
  const float scale = __uint_as_float((uint32_t)(127 + a.sc_bits) << 23);  // 2^sc_bits
  const __half* ibase = a.idx + ((int64_t)b * a.Hr + hr) * a.max_seq * (2 * kR);
  uint2* cut = a.cut + ((int64_t)b * a.Hr + hr) * a.C + i0;

  if (a.top_p >= 1.f) {  // p = 1 keeps every causal key (also those whose mass rounds to 0)
    if (owner) {
      if (x.pa >= 0) cut[x.ra] = make_uint2(0u, 0x7FFFFFFFu);
      if (x.pb >= 0) cut[x.rb] = make_uint2(0u, 0x7FFFFFFFu);
      if (a.sel_mass) {
        if (x.pa >= 0) a.sel_mass[((int64_t)b * a.C + i0 + x.ra) * a.Hr + hr] = 1.f;
        if (x.pb >= 0) a.sel_mass[((int64_t)b * a.C + i0 + x.rb) * a.Hr + hr] = 1.f;
      }
    }
    return;
  }

  uint32_t qh[4], ql[4];
  {
    const int64_t qs = (int64_t)a.Hr * kR;
    const float* q0 = a.q_idx + ((int64_t)b * a.C + i0) * qs + (int64_t)hr * kR;
    idx_load_q(qh, ql, x.pa >= 0 ? q0 + x.ra * qs : nullptr, x.pb >= 0 ? q0 + x.rb * qs : nullptr);
  }

  // ---- pass A: row maxima (the 4 threads of a quad share their two rows)
  float m[2] = {-INFINITY, -INFINITY};
  scan(S.st, x, ibase, qh, ql, [&](int sl, int64_t, float s) { m[sl] = fmaxf(m[sl], s); }, [] {});
#pragma unroll
  for (int sl = 0; sl < 2; ++sl) {
    m[sl] = fmaxf(m[sl], __shfl_xor_sync(0xffffffffu, m[sl], 1));
    m[sl] = fmaxf(m[sl], __shfl_xor_sync(0xffffffffu, m[sl], 2));
  }

  // ---- pass B: 16 bins of width 1 below the max -> Z, T, crossing bin
  hist_zero(S, tid);
  scan(S.st, x, ibase, qh, ql, [&](int sl, int64_t, float s) {
    hist_add(S, bin1_of(m[sl] - s), sl, tid, mass64(s, m[sl], scale));
  }, [&] { hist_fold(S, tid); });
  if (owner) {
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      const int r = sl ? x.rb : x.ra;
      RowS& R = S.row[r];
      R.m = m[sl];
      R.found = 0;
      R.tie_before = 0;
      if ((sl ? x.pb : x.pa) < 0) {
        R.mode = kModeDone;
        continue;
      }
      unsigned long long hb[kBins];
      unsigned long long Z = 0;
      for (int i = 0; i < kBins; ++i) {
        hb[i] = hist_get(S, i, sl, tid) + hist_get(S, i, sl, tid + 1) + hist_get(S, i, sl, tid + 2) +
                hist_get(S, i, sl, tid + 3);
        Z += hb[i];
      }
      unsigned long long T = (unsigned long long)ceil((double)a.top_p * (double)Z);
      if (T < 1ull) T = 1ull;
      if (T > Z) T = Z;
      unsigned long long cum = 0;
      int cb = kBins - 1;  // bins run from the highest scores down
      for (int i = 0; i < kBins; ++i) {
        if (cum + hb[i] >= T) {
          cb = i;
          break;
        }
        cum += hb[i];
      }
      R.Z = Z;
      R.cb = cb;
      R.rem = T - cum;
      R.above = cum;
      bin_key_range(m[sl], cb, &R.klo, &R.khi);
      R.shift = slice_shift(R.klo, R.khi);
      R.mode = kModeKeys;
    }
  }
  __syncthreads();

  // ---- refinement: 16-way bit slices of the crossing key range until <= 16 keys remain
  for (int level = 0; level < 10; ++level) {
    const int need = (S.row[x.ra].mode == kModeKeys) || (S.row[x.rb].mode == kModeKeys);
    if (!__syncthreads_or(need)) break;
    bool mine[2];
    int sh[2];
    uint32_t klo[2], khi[2];
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      const RowS& R = S.row[sl ? x.rb : x.ra];
      mine[sl] = R.mode == kModeKeys;
      sh[sl] = R.shift;
      klo[sl] = R.klo;
      khi[sl] = R.khi;
    }
    hist_zero(S, tid);
    int nc[2] = {0, 0};
    RowCtx xm = x;  // rows outside refinement see no keys
    if (!mine[0]) xm.pa = -1;
    if (!mine[1]) xm.pb = -1;
    const uint32_t span[2] = {khi[0] - klo[0], khi[1] - klo[1]};
    scan_gated(S.st, xm, ibase, qh, ql, [&](int sl, float s) { return order_key(s) - klo[sl] <= span[sl]; },
               [&](int sl, int64_t j, float s) {
      const uint32_t key = order_key(s);
      {
        hist_add(S, (int)((key - klo[sl]) >> sh[sl]), sl, tid, mass64(s, m[sl], scale));
        if (nc[sl] < kCand) S.cand[nc[sl]][sl][tid] = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)j);
        ++nc[sl];
      }
    }, [&] { hist_fold(S, tid); });
    S.nc[0][tid] = nc[0];
    S.nc[1][tid] = nc[1];
    __syncthreads();
    if (owner) {
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        if (!mine[sl]) continue;
        RowS& W = S.row[sl ? x.rb : x.ra];
        const int n0 = S.nc[sl][tid], n1 = S.nc[sl][tid + 1], n2 = S.nc[sl][tid + 2], n3 = S.nc[sl][tid + 3];
        if (n0 <= kCand && n1 <= kCand && n2 <= kCand && n3 <= kCand) {
          // every key of the range is a captured candidate: exact cut by sorting them
          unsigned long long c[4 * kCand];
          int n = 0;
          const int nq[4] = {n0, n1, n2, n3};
          for (int q = 0; q < 4; ++q)
            for (int i = 0; i < nq[q]; ++i) c[n++] = S.cand[i][sl][tid + q];
          for (int i = 1; i < n; ++i) {  // insertion sort, descending: key desc, then j asc
            const unsigned long long v = c[i];
            int k = i - 1;
            while (k >= 0 && c[k] < v) {
              c[k + 1] = c[k];
              --k;
            }
            c[k + 1] = v;
          }
          unsigned long long cum = 0;
          int ci = -1;
          for (int i = 0; i < n; ++i) {
            cum += mass64(key_to_float((uint32_t)(c[i] >> 32)), m[sl], scale);
            if (cum >= W.rem) {
              ci = i;
              break;
            }
          }
          if (ci < 0) {  // not reached: the range was chosen to hold at least rem
            atomicOr(a.err, kErrInternal);
            W.t_key = 0xFFFFFFFFu;
            W.tiecut = -1;
          } else {
            W.t_key = (uint32_t)(c[ci] >> 32);
            W.tiecut = (int)(0xFFFFFFFFu - (uint32_t)c[ci]);
            W.above += cum;
          }
          W.mode = kModeDone;
        } else {
          unsigned long long cum = 0;
          int cs = -1;
          for (int i = kBins - 1; i >= 0; --i) {  // highest slice first
            const unsigned long long hs = hist_get(S, i, sl, tid) + hist_get(S, i, sl, tid + 1) +
                                          hist_get(S, i, sl, tid + 2) + hist_get(S, i, sl, tid + 3);
            if (cum + hs >= W.rem) {
              cs = i;
              break;
            }
            cum += hs;
          }
          if (cs < 0) {
            atomicOr(a.err, kErrInternal);
            W.t_key = 0xFFFFFFFFu;
            W.tiecut = -1;
            W.mode = kModeDone;
          } else {
            const uint32_t nlo = W.klo + ((uint32_t)cs << W.shift);
            const uint32_t top = nlo + ((1u << W.shift) - 1u);
            const uint32_t nhi = top < W.khi && top >= nlo ? top : W.khi;
            W.rem -= cum;
            W.above += cum;
            W.klo = nlo;
            W.khi = nhi;
            W.shift = slice_shift(nlo, nhi);
            if (nlo == nhi) {  // one key value with more than 16 members: an exact tie group
              W.t_key = nlo;
              const unsigned long long e = mass64(key_to_float(nlo), m[sl], scale);
              W.n_need = e ? (W.rem + e - 1) / e : 1ull;
              W.mode = kModeTie;
            }
          }
        }
      }
    }
    __syncthreads();
  }
  if (owner) {
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      RowS& W = S.row[sl ? x.rb : x.ra];
      if (W.mode == kModeKeys) {  // not reached: ten 16-way levels split 32 bits
        atomicOr(a.err, kErrInternal);
        W.t_key = 0xFFFFFFFFu;
        W.tiecut = -1;
        W.mode = kModeDone;
      }
    }
  }

  // ---- exact ties: the cutoff is the n_need-th tied position in ascending order
  {
    const int need = S.row[x.ra].mode == kModeTie || S.row[x.rb].mode == kModeTie;
    if (__syncthreads_or(need)) {
      bool mine[2];
      uint32_t tk[2];
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        const RowS& R = S.row[sl ? x.rb : x.ra];
        mine[sl] = R.mode == kModeTie;
        tk[sl] = R.t_key;
      }
      idx_walk(S.st, ibase, x.nkeys, [&](int64_t t, int stage) {
        float c[8][4];
        idx_scores(c, qh, ql, S.st, stage);
        unsigned long long mk[2] = {0ull, 0ull};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int p = 8 * nt + 2 * x.tq + e;
            const int64_t j = t * kIdxKeys + p;
#pragma unroll
            for (int sl = 0; sl < 2; ++sl) {
              const float s = c[nt][2 * sl + e];
              if (mine[sl] && j <= (sl ? x.pb : x.pa) && order_key(s) == tk[sl])
                mk[sl] |= 1ull << p;
            }
          }
        }
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          mk[sl] |= __shfl_xor_sync(0xffffffffu, mk[sl], 1);
          mk[sl] |= __shfl_xor_sync(0xffffffffu, mk[sl], 2);
        }
        if (owner) {
#pragma unroll
          for (int sl = 0; sl < 2; ++sl) {
            if (!mine[sl]) continue;
            RowS& W = S.row[sl ? x.rb : x.ra];
            if (W.found) continue;
            const int cnt = __popcll(mk[sl]);
            if (W.tie_before + cnt >= W.n_need) {
              int want = (int)(W.n_need - W.tie_before);
              unsigned long long v = mk[sl];
              while (--want > 0) v &= v - 1;  // drop the lowest (want - 1) set bits
              W.tiecut = (int)(t * kIdxKeys + (__ffsll((long long)v) - 1));
              W.found = 1;
            }
            W.tie_before += cnt;
          }
        }
      });
      if (owner) {
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          if (!mine[sl]) continue;
          RowS& W = S.row[sl ? x.rb : x.ra];
          if (!W.found) {
            atomicOr(a.err, kErrInternal);
            W.tiecut = 0x7FFFFFFF;
          } else {
            W.above += (unsigned long long)W.n_need * mass64(key_to_float(W.t_key), m[sl], scale);
          }
          W.mode = kModeDone;
        }
      }
    }
  }

  if (owner) {
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      const int r = sl ? x.rb : x.ra;
      if ((sl ? x.pb : x.pa) < 0) continue;
      const RowS& W = S.row[r];
      cut[r] = make_uint2(W.t_key, (uint32_t)W.tiecut);
      if (a.sel_mass)
        a.sel_mass[((int64_t)b * a.C + i0 + r) * a.Hr + hr] = (float)((double)W.above / (double)W.Z);
    }
  }
}

// ------------------------------------------------------------------ sparse attention

struct SmemAttn {
  IdxRing st;                             // 12 KB
  unsigned char kv[2][2 * kFaTileBytes];  // 64 KB: gathered K and V rows of two chunks in flight
  uint32_t cm[kRows][4];                  // per-row bits of the (up to 128) filling slots
  int32_t jl[128];                        // filling slot -> key position
  uint32_t cmc[2][kRows][2];              // per-row bits of the two issued chunks
  int32_t jlc[2][64];                     // their key positions
  unsigned long long wun[2][4];           // per-warp union of a tile's row masks (two tiles)
  int32_t lslot[kRows];                   // row -> its entry in the listed rows (-1: not listed)
};

__global__ void __launch_bounds__(kThreads) prefill_attn_kernel(RetArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SmemAttn& S = *reinterpret_cast<SmemAttn*>(smem_raw);
  const int tile = gridDim.x - 1 - blockIdx.x, hr = blockIdx.y, b = blockIdx.z;  // longest rows first
  const int i0 = tile * kRows;
  const int nrows = min(kRows, a.C - i0);
  const RowCtx x = row_ctx(a, i0, nrows);
  const int tid = x.tid;
  const bool owner = x.tq == 0;
  const int h = a.ret_head[hr], g = h / a.group;
  const __half* ibase = a.idx + ((int64_t)b * a.Hr + hr) * a.max_seq * (2 * kR);
  const __half* kb = a.kc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD;
  const __half* vb = a.vc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD;
  const int64_t qs = (int64_t)a.Hq * kD;

  uint32_t qh[4], ql[4];
  {
    const int64_t is = (int64_t)a.Hr * kR;
    const float* q0 = a.q_idx + ((int64_t)b * a.C + i0) * is + (int64_t)hr * kR;
    idx_load_q(qh, ql, x.pa >= 0 ? q0 + x.ra * is : nullptr, x.pb >= 0 ? q0 + x.rb * is : nullptr);
  }
  const uint2* cut = a.cut + ((int64_t)b * a.Hr + hr) * a.C + i0;
  uint32_t tk[2];
  int64_t tc[2];
  {
    const uint2 ca = x.pa >= 0 ? cut[x.ra] : make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
    const uint2 cbv = x.pb >= 0 ? cut[x.rb] : make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
    tk[0] = ca.x;
    tc[0] = (int32_t)ca.y;
    tk[1] = cbv.x;
    tc[1] = (int32_t)cbv.y;
  }
  uint32_t* brow[2] = {nullptr, nullptr};
  if (a.bitmap && owner) {
    if (x.pa >= 0) brow[0] = a.bitmap + (((int64_t)b * a.C + i0 + x.ra) * a.Hr + hr) * a.bitmap_words;
    if (x.pb >= 0) brow[1] = a.bitmap + (((int64_t)b * a.C + i0 + x.rb) * a.Hr + hr) * a.bitmap_words;
  }

  uint32_t qa[8][4];
  fa_load_q(qa, a.q_rot + ((int64_t)b * a.C + i0) * qs + (int64_t)h * kD, qs, x.warp * 16, nrows);
  FaAcc A;
  fa_init(A);

  for (int i = tid; i < kRows * 4; i += kThreads) (&S.cm[0][0])[i] = 0u;
  for (int i = tid; i < kRows; i += kThreads) S.lslot[i] = -1;
  __syncthreads();
  for (int i = tid; i < a.n_rows; i += kThreads) {
    const int r = a.rows[i] - i0;
    if (r >= 0 && r < nrows) S.lslot[r] = i;
  }
  __syncthreads();
  int32_t* lrow[2] = {nullptr, nullptr};  // this owner's listed rows: where their positions go
  if (a.row_sel && owner) {
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      const int r = sl ? x.rb : x.ra;
      const int li = (sl ? x.pb : x.pa) >= 0 ? S.lslot[r] : -1;
      if (li >= 0) lrow[sl] = a.row_sel + (((int64_t)b * a.n_rows + li) * a.Hr + hr) * a.row_sel_cap;
    }
  }
  int fill = 0;
  int nsel[2] = {0, 0};

  // Chunks are double-buffered: issuing chunk n starts its K/V gather, and only then is chunk
  // n - 1 (gathered meanwhile) run through the attention tile.
  int pend = -1;  // buffer of the issued chunk not yet attended (-1: none)
  int nbuf = 0;   // buffer the next chunk goes to
  auto attend = [&](int buf) {
    fa_tile(A, qa, S.kv[buf], S.kv[buf] + kFaTileBytes, a.scale_log2,
            [&](int r, int tt) { return ((S.cmc[buf][r][tt >> 5] >> (tt & 31)) & 1u) != 0u; });
  };
  auto issue = [&](int n) {  // move filling slots 0 .. n-1 into a chunk buffer and gather it
    const int k = nbuf;
    for (int i = tid; i < kRows; i += kThreads) {
      S.cmc[k][i][0] = S.cm[i][0];
      S.cmc[k][i][1] = S.cm[i][1];
      S.cm[i][0] = S.cm[i][2];
      S.cm[i][1] = S.cm[i][3];
      S.cm[i][2] = S.cm[i][3] = 0u;
    }
    if (tid < 64) {
      S.jlc[k][tid] = tid < n ? S.jl[tid] : 0;
      S.jl[tid] = S.jl[64 + tid];
    }
    __syncthreads();
    fa_stage(S.kv[k], S.kv[k] + kFaTileBytes, kb, vb, n, [&](int r) { return (int64_t)S.jlc[k][r]; });
    cp_async_commit();
    if (pend >= 0) {
      cp_async_wait<1>();  // everything but this chunk's gather has landed
      __syncthreads();
      attend(pend);
      __syncthreads();
    }
    pend = k;
    nbuf ^= 1;
  };

  // The union of tile t is published in shared memory and appended to the chunk during tile
  // t + 1, after that tile's ring barrier: one barrier per tile.
  unsigned long long own_prev[2] = {0ull, 0ull};
  auto append = [&](int64_t t) {  // tile t's union keys -> chunk slots fill, fill + 1, ...
    const int pb = (int)(t & 1);
    const unsigned long long U = S.wun[pb][0] | S.wun[pb][1] | S.wun[pb][2] | S.wun[pb][3];
    if (U == 0ull) return;  // uniform: no row selects a key of this tile
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      unsigned long long v = own_prev[sl];
      const int r = sl ? x.rb : x.ra;
      while (v) {
        const int p = __ffsll((long long)v) - 1;
        v &= v - 1;
        const int slot = fill + __popcll(U & ((1ull << p) - 1ull));
        atomicOr(&S.cm[r][slot >> 5], 1u << (slot & 31));
      }
    }
    if (tid < 64 && ((U >> tid) & 1ull))
      S.jl[fill + __popcll(U & ((1ull << tid) - 1ull))] = (int32_t)(t * kIdxKeys + tid);
    fill += __popcll(U);
    if (fill >= 64) {
      __syncthreads();  // every slot of the chunk is written
      issue(64);
      fill -= 64;
    }
  };

  idx_walk(S.st, ibase, x.nkeys, [&](int64_t t, int stage) {
    if (t > 0) append(t - 1);
    float c[8][4];
    idx_scores(c, qh, ql, S.st, stage);
    const int64_t base = t * kIdxKeys;
    const int la = (int)max((int64_t)-1, min((int64_t)(kIdxKeys - 1), x.pa - base));
    const int lb = (int)max((int64_t)-1, min((int64_t)(kIdxKeys - 1), x.pb - base));
    const int ca = (int)max((int64_t)-1, min((int64_t)kIdxKeys, tc[0] - base));
    const int cbt = (int)max((int64_t)-1, min((int64_t)kIdxKeys, tc[1] - base));
    unsigned long long mk[2] = {0ull, 0ull};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int p = 8 * nt + 2 * x.tq + e;
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          const uint32_t key = order_key(c[nt][2 * sl + e]);
          const int lim = sl ? lb : la, cut_p = sl ? cbt : ca;
          const bool sel = p <= lim && (key > tk[sl] || (key == tk[sl] && p <= cut_p));
          mk[sl] |= (unsigned long long)sel << p;
        }
      }
    }
    own_prev[0] = mk[0];  // this thread's selected keys, appended during the next tile
    own_prev[1] = mk[1];
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      mk[sl] |= __shfl_xor_sync(0xffffffffu, mk[sl], 1);
      mk[sl] |= __shfl_xor_sync(0xffffffffu, mk[sl], 2);
    }
    if (owner) {
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        if (lrow[sl]) {  // a listed row: its positions, ascending (tiles come in order)
          unsigned long long v = mk[sl];
          int n = nsel[sl];
          while (v && n < a.row_sel_cap) {
            const int p = __ffsll((long long)v) - 1;
            v &= v - 1;
            lrow[sl][n++] = (int32_t)(t * kIdxKeys + p);
          }
        }
        nsel[sl] += __popcll(mk[sl]);
        if (brow[sl]) {
          const int64_t w = 2 * t;
          if (w < a.bitmap_words) brow[sl][w] = (uint32_t)mk[sl];
          if (w + 1 < a.bitmap_words) brow[sl][w + 1] = (uint32_t)(mk[sl] >> 32);
        }
      }
    }
    unsigned long long u = mk[0] | mk[1];
    u |= __shfl_xor_sync(0xffffffffu, u, 4);
    u |= __shfl_xor_sync(0xffffffffu, u, 8);
    u |= __shfl_xor_sync(0xffffffffu, u, 16);
    if ((tid & 31) == 0) S.wun[t & 1][x.warp] = u;
  });
  {
    const int64_t ntiles = (x.nkeys + kIdxKeys - 1) / kIdxKeys;  // the walk ended with a barrier
    append(ntiles - 1);
  }
  __syncthreads();
  if (fill > 0) issue(fill);
  if (pend >= 0) {
    cp_async_wait<0>();
    __syncthreads();
    attend(pend);
  }
  fa_store(A, a.out + ((int64_t)b * a.C + i0) * qs + (int64_t)h * kD, qs, x.warp * 16, nrows);
  if (a.sel_count && owner) {
    if (x.pa >= 0) a.sel_count[((int64_t)b * a.C + i0 + x.ra) * a.Hr + hr] = nsel[0];
    if (x.pb >= 0) a.sel_count[((int64_t)b * a.C + i0 + x.rb) * a.Hr + hr] = nsel[1];
  }
}

}  // namespace

cudaError_t launch_prefill_retrieval(rtp_layer* L, int C, float* out, const rtp_prefill_stats* stats,
                                     cudaStream_t st) {
  RetArgs a;
  a.idx = L->idx_hl;
  a.kc = L->kc;
  a.vc = L->vc;
  a.max_seq = L->max_seq;
  a.Hkv = L->Hkv;
  a.Hq = L->Hq;
  a.Hr = L->Hr;
  a.group = L->group;
  a.C = C;
  a.P0 = L->len - C;
  a.top_p = L->top_p;
  int lg = 0;
  while ((1ll << lg) < L->len) ++lg;
  a.sc_bits = 62 - lg;
  a.ret_head = L->d_ret_head;
  a.q_rot = L->q_rot;
  a.q_idx = L->q_idx;
  a.cut = L->pf_cut;
  a.scale_log2 = L->sm_scale * 1.4426950408889634f;
  a.out = out;
  a.sel_count = stats ? stats->sel_count : nullptr;
  a.sel_mass = stats ? stats->sel_mass : nullptr;
  a.bitmap = stats ? stats->sel_bitmap : nullptr;
  a.bitmap_words = stats ? stats->bitmap_words : 0;
  a.rows = stats ? stats->rows : nullptr;
  a.n_rows = (stats && stats->rows) ? stats->n_rows : 0;
  a.row_sel = (stats && stats->rows) ? stats->row_sel : nullptr;
  a.row_sel_cap = (stats && stats->rows) ? stats->row_sel_cap : 0;
  a.err = L->err;
  dim3 grid((C + kRows - 1) / kRows, L->Hr, L->B);
  cudaError_t e;
  {
    ProfScope ps(L, "prefill_select", st);
    e = cudaFuncSetAttribute(prefill_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(SmemSel));
    if (e != cudaSuccess) return e;
    prefill_select_kernel<<<grid, kThreads, sizeof(SmemSel), st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    ProfScope ps(L, "prefill_attn", st);
    e = cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(SmemAttn));
    if (e != cudaSuccess) return e;
    prefill_attn_kernel<<<grid, kThreads, sizeof(SmemAttn), st>>>(a);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace rtp
