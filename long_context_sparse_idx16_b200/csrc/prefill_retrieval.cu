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
// Both kernels take 128-row tiles (one CTA per (row tile, retrieval head, sequence)) and score
// 64-key tiles on the tensor cores (index_tc.cuh: three tcgen05.mma into TMEM, key tiles
// copied by TMA), so both see identical score bits:
//
//  prefill_select_kernel -- 128 threads, one query row per thread (its TMEM lane).  The exact
//    cut (t_key, tiecut) of each row, in walks over the row's causal keys, all masses exact in
//    64-bit fixed point (mass of key j = trunc(2^sc * e^(s_j - m)), sc = 62 - ceil(log2 len)),
//    each row's histograms in its own shared-memory column (no atomics):
//      A  row maxima m;
//      B  16 bins of m - s rounded to an integer (the last one holding everything from 14.5
//         down) -> Z, T = ceil(p Z), crossing bin, whose exact order-key range is found by
//         bisection;
//      R  refinement: each walk sums the mass of 16 bit slices of the crossing range of order
//         keys and captures the range's keys (in position order) into a per-row global list;
//         a row whose range holds at most 2048 keys finishes from its list (narrowing it 16
//         ways at a time, then sorting the last <= 8 keys, key desc, j asc, for the exact cut;
//         a single key value is an exact tie group, cut at its n-th position); otherwise the
//         range narrows to the crossing slice for the next walk, and a range that shrinks to
//         one key value with more members than the list holds is resolved by
//      T  an ordered count of the tied positions.
//  prefill_attn_kernel -- 256 threads, two per row (each on half of a tile's 64 columns).
//    Rows with more than 256K keys split them over several CTAs (partial softmax states merged
//    by the last CTA of the row tile).  Walks the key tiles in order: the index scores of tile
//    t + 1 (computed one tile ahead)
//    and each row's cut give the rows' selection masks; a tile no row selects is skipped,
//    otherwise its K and V rows come in by TMA, S = Q K^T runs on the tensor cores into TMEM,
//    the masked online softmax forms P in shared memory and O += P V accumulates in TMEM.
#include "index_tc.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr int kRowsR = kTcRows;  // 128 query rows per CTA (TMEM lanes)
constexpr int kKeysR = kTcKeys;  // 64 keys per tile
constexpr int kBins = 16;        // pass B: bins of width 1 below the row max
constexpr int kSlices = 16;      // refinement: slices of the crossing key range per level
constexpr int kCand = 8;         // keys sorted in registers for the final cut
constexpr int kCapG = kPfCapture; // keys of the crossing range captured per row in a refinement walk
constexpr int kLevels = 10;      // refinement levels (4 key bits each, with margin)
constexpr float kLog2e = 1.4426950408889634f;

enum : int { kModeKeys = 1, kModeTie = 2, kModeDone = 3 };

struct RetArgs {
  int64_t max_seq;
  int Hkv, Hq, Hr, group, C;
  SeqPos P0;                  // per sequence: position of chunk row 0 (its length - C)
  float top_p;
  int64_t top_k;              // > 0: fixed budget (counts instead of masses)
  int sc_bits;                // fixed-point scale of the selection masses (62 - ceil(log2 len))
  const int16_t* ret_head;    // [Hr]
  const float* q_rot;         // [B][C][Hq][D]
  const float* q_idx;         // [B][C][Hr][r]
  uint2* cut;                 // [B][Hr][C]: (t_key, tiecut)
  unsigned long long* capture; // [B][Hr][C / 128][kCapG][128]: (key << 32 | ~j) of a row's crossing range
  int attn_splits;            // CTAs per row tile of the attention, each on attn_split_tiles key tiles
  int64_t attn_split_tiles;
  float* attn_part;           // [B][Hr][C / 128][attn_splits][128][4 + D]: (m, l, count, -, o) per row
  uint32_t* attn_ticket;      // [B][Hr][C / 128]: splits of a row tile done (the last merges)
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

// Fixed-point mass of a score s below the row max m: e^(s - m) * 2^sc truncated to an integer
// (scale = 2^sc as a float, exact).
__device__ __forceinline__ unsigned long long mass64(float s, float m, float scale) {
  return __float2ull_rz(fast_exp2((s - m) * kLog2e) * scale);
}

// pass-B bin of x = m - s >= 0: x rounded to the nearest integer (adding 2^23 does the
// rounding), with everything from 14.5 down in the last bin.  Non-increasing in s.
__device__ __forceinline__ int bin1_of(float x) {
  const uint32_t r = __float_as_uint(x + 8388608.0f) - 0x4B000000u;
  return (int)min(r, (uint32_t)(kBins - 1));
}

// Exact order-key range [lo, hi] of the finite scores s <= m whose pass-B bin is b (bisection
// on the monotone map key -> bin).
__device__ __forceinline__ void bin_key_range(float m, int b, uint32_t* lo, uint32_t* hi) {
  const uint32_t kmin = order_key(-3.4028234663852886e38f), kmax = order_key(m);
  auto bin_of_key = [&](uint32_t k) { return bin1_of(m - key_to_float(k)); };
  uint32_t l = kmin, h = kmax;  // first key with bin <= b
  while (l < h) {
    const uint32_t mid = l + ((h - l) >> 1);
    if (bin_of_key(mid) <= b) h = mid;
    else l = mid + 1;
  }
  *lo = l;
  if (b == 0) {
    *hi = kmax;
    return;
  }
  l = *lo;  // last key with bin >= b: one below the first key with bin < b
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

// slices of 2^shift keys cover [klo, khi] in at most kSlices (16) pieces
__device__ __forceinline__ int slice_shift(uint32_t klo, uint32_t khi) {
  const int bits = 32 - __clz(khi - klo);
  return bits > 4 ? bits - 4 : 0;
}

// last causal column of a 64-key tile for a row at position pos (-1: none)
__device__ __forceinline__ int causal_lim(int64_t pos, int64_t t) {
  return (int)max((int64_t)-1, min((int64_t)(kKeysR - 1), pos - t * kKeysR));
}

// ------------------------------------------------------------------ exact per-row top-p

constexpr int kPsThreads = kRowsR;  // one thread per row
constexpr uint32_t kSelStages = 3;   // key tiles of the TMA ring
constexpr uint32_t kSOffQ = 0;                                       // query tile, 8 KB
constexpr uint32_t kSOffK = kSOffQ + kTcQBytes;                      // key ring, 3 x 4 KB
constexpr uint32_t kSOffH = kSOffK + kSelStages * kTcKBytes;         // [slice][row] u64, 16 KB
constexpr uint32_t kSOffBar = kSOffH + kSlices * kRowsR * 8;         // full[3], done, TMEM base
constexpr uint32_t kSelSmem = kSOffBar + 64;  // about 36 KB: five CTAs (5 x 64 TMEM columns) per SM
static_assert(kSelStages <= 3, "the barrier block holds three stage barriers");
// One 64-column TMEM score buffer per CTA: five CTAs fit an SM (TMEM 512 columns, shared
// memory 228 KB), so the 640 CTAs of a 16K-row chunk with 5 retrieval heads run in one wave;
// the scores of tile t + 1 are issued as soon as every thread has read tile t.
constexpr uint32_t kSelTmemCols = 64;

// Walks over the key tiles [0, ntiles) of one (sequence, retrieval head): thread 0 keeps
// kSelStages TMA copies in flight and issues the scores of tile t + 1 once tile t is read;
// body(t, c0, s, lim) gets this thread's row's scores of tile t in groups of 16 (columns c0 ..
// c0 + 15, s[0..15]) and the last causal column lim of the tile.  g counts tiles over all walks
// (mbarrier phases).  A wait that runs out clears ok in every thread; later walks then do
// nothing, and drain() waits (bounded) for the copies and MMAs still in flight.
struct SelWalk {
  uint32_t sbase, tmem, lane_addr;
  const CUtensorMap* map;
  int64_t row0, pos;  // pos: this thread's row position (-1: no row)
  uint32_t g;
  bool ok;
  uint32_t inflight_lo, inflight_hi;  // tiles [lo, hi) whose copies thread 0 has not waited on
  bool mma_pending;                   // scores of tile g issued and not waited on

  __device__ uint32_t full_bar(uint32_t gt) const { return sbase + kSOffBar + 8u * (gt % kSelStages); }
  __device__ uint32_t done_bar(uint32_t) const { return sbase + kSOffBar + 24u; }
  __device__ uint32_t ktile(uint32_t gt) const { return sbase + kSOffK + (gt % kSelStages) * kTcKBytes; }

  template <typename Body>
  __device__ __forceinline__ void run(int64_t ntiles, Body body) {
    const int tid = threadIdx.x;
    if (!ok || ntiles <= 0) return;
    bool okw = true;
    if (tid == 0) {
      inflight_lo = g;
      for (int64_t i = 0; i < (int64_t)kSelStages && i < ntiles; ++i)
        tc_load_keys(ktile(g + (uint32_t)i), map, row0, i, full_bar(g + (uint32_t)i));
      inflight_hi = g + (uint32_t)min((int64_t)kSelStages, ntiles);
      okw = mbar_wait(full_bar(g), (g / kSelStages) & 1u);
      inflight_lo = g + 1;
      if (okw) tc_issue_scores(tmem, sbase + kSOffQ, ktile(g), done_bar(g));
      mma_pending = okw;
    }
    for (int64_t t = 0; t < ntiles; ++t) {
      const uint32_t gt = g + (uint32_t)t;
      // the scores of tile gt: one completion of the done barrier per tile (parity gt & 1)
      if (tid != 0 || mma_pending) okw = mbar_wait(done_bar(gt), gt & 1u) && okw;
      tc_fence_after();
      __syncwarp();  // the loads are warp-collective: reconverge after thread 0's work
      // the body sees the tile in four 16-column groups, each loaded from TMEM on its own (one
      // copy of the unrolled body per walk), with the last causal column lim of the tile
      const int lim = causal_lim(pos, t);
#pragma unroll 1
      for (int q = 0; q < kTcKeys / 16; ++q) {
        float s[16];
        tmem_ld16(lane_addr + 16u * q, s);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) s[i] += 0.0f;  // -0 -> +0: equal scores, equal order keys
        body(t, 16 * q, s, lim);
      }
      tc_fence_before();
      // every thread has read tile gt: the buffer takes the scores of tile gt + 1 next
      if (!__syncthreads_and(okw ? 1 : 0)) {
        ok = false;
        if (tid == 0) mma_pending = false;
        g = gt + 1;
        return;
      }
      if (tid == 0) {
        mma_pending = false;
        if (t + kSelStages < ntiles) {  // the stage of tile gt is free: its scores are done
          tc_load_keys(ktile(gt), map, row0, t + kSelStages, full_bar(gt));
          inflight_hi = gt + kSelStages + 1;
        }
        if (t + 1 < ntiles) {
          okw = mbar_wait(full_bar(gt + 1), ((gt + 1) / kSelStages) & 1u);
          inflight_lo = gt + 2;
          if (okw) tc_issue_scores(tmem, sbase + kSOffQ, ktile(gt + 1), done_bar(gt + 1));
          mma_pending = okw;
        }
      }
    }
    g += (uint32_t)ntiles;
  }

  // after a timeout: wait (bounded) for the copies and the scores still in flight
  __device__ void drain() {
    if (threadIdx.x != 0) return;
    for (uint32_t gt = inflight_lo; gt < inflight_hi; ++gt) mbar_wait(full_bar(gt), (gt / kSelStages) & 1u);
    if (mma_pending) mbar_wait(done_bar(g), g & 1u);
  }
};

__global__ void __launch_bounds__(kPsThreads, 6) prefill_select_kernel(RetArgs a,
                                                                     const __grid_constant__ CUtensorMap tm_idx) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int tile = gridDim.x - 1 - blockIdx.x, hr = blockIdx.y, b = blockIdx.z;  // longest rows first
  const int i0 = tile * kRowsR;
  const int nrows = min(kRowsR, a.C - i0);
  const bool live = tid < nrows;
  const int64_t P0 = a.P0.v[b];
  const int64_t pos = live ? P0 + i0 + tid : -1;
  const int64_t nkeys = P0 + i0 + nrows;
  const int64_t ntiles = (nkeys + kKeysR - 1) / kKeysR;
  const float scale = __uint_as_float((uint32_t)(127 + a.sc_bits) << 23);  // 2^sc_bits
  uint2* cut = a.cut + ((int64_t)b * a.Hr + hr) * a.C + i0;
  float* mass_out = (a.sel_mass && live) ? a.sel_mass + ((int64_t)b * a.C + i0 + tid) * a.Hr + hr : nullptr;

  const bool topk = a.top_k > 0;  // fixed budget: every key weighs 1, the target is min(k, n)
  if (!topk && a.top_p >= 1.f) {  // p = 1 keeps every causal key (also those whose mass rounds to 0)
    if (live) {
      cut[tid] = make_uint2(0u, 0x7FFFFFFFu);
      if (mass_out) *mass_out = 1.f;
    }
    return;
  }
  if (sbase & 127u) {  // TMA destinations and operand tiles need aligned shared memory
    if (tid == 0) atomicOr(a.err, kErrInternal);
    return;
  }
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kSOffBar + 48);
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kSelTmemCols);
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(sbase + kSOffBar + 8u * i, 1);
    fence_mbar_init();
  }
  {
    const float* qrow = a.q_idx + (((int64_t)b * a.C + i0 + (live ? tid : 0)) * a.Hr + hr) * kR;
    tc_put_query(sm + kSOffQ, tid, live ? qrow : nullptr);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  SelWalk W;
  W.sbase = sbase;
  W.tmem = tmem;
  W.lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
  W.map = &tm_idx;
  W.row0 = ((int64_t)b * a.Hr + hr) * a.max_seq;
  W.pos = pos;
  W.g = 0;
  W.ok = true;
  W.inflight_lo = W.inflight_hi = 0;
  W.mma_pending = false;
  // the weight a key adds to the histograms: its fixed-point softmax mass, or 1 with a fixed
  // budget (then the sums are counts)
  auto weight = [&](float s, float mx) -> unsigned long long { return topk ? 1ull : mass64(s, mx, scale); };
  unsigned long long* hist = reinterpret_cast<unsigned long long*>(sm + kSOffH) + tid;  // [slice * 128]
  // this row's capture list, entry k at cap[k * 128] (the CTA's rows interleaved: coalesced)
  unsigned long long* cap = a.capture + (((int64_t)b * a.Hr + hr) * ((a.C + kRowsR - 1) / kRowsR) + tile) *
                                             (int64_t)kCapG * kRowsR + tid;

  // ---- pass A: the row max
  float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // four chains: no serial max
  W.run(ntiles, [&](int64_t t, int c0, const float* s, int lim) {
    if (lim >= c0 + 15) {
#pragma unroll
      for (int c = 0; c < 16; ++c) mq[c & 3] = fmaxf(mq[c & 3], s[c]);
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c)
        if (c0 + c <= lim) mq[c & 3] = fmaxf(mq[c & 3], s[c]);
    }
  });
  const float m = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));

  // ---- pass B: 16 bins of width 1 below the max (the last, most populated bin in a register)
  for (int i = 0; i < kBins; ++i) hist[i * kRowsR] = 0ull;
  unsigned long long far = 0ull;
  W.run(ntiles, [&](int64_t t, int c0, const float* s, int lim) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      if (c0 + c <= lim) {
        const int bi = bin1_of(m - s[c]);
        const unsigned long long ms = weight(s[c], m);
        if (bi == kBins - 1) far += ms;
        else hist[bi * kRowsR] += ms;
      }
    }
  });
  int mode = kModeDone, shift = 0, tiecut = -1;
  uint32_t klo = 0u, khi = 0u, t_key = 0xFFFFFFFFu;
  unsigned long long Z = 0ull, rem = 0ull, above = 0ull, n_need = 0ull;
  if (live) {
    unsigned long long hb[kBins];
    for (int i = 0; i < kBins - 1; ++i) {
      hb[i] = hist[i * kRowsR];
      Z += hb[i];
    }
    hb[kBins - 1] = far;
    Z += far;
    unsigned long long T = topk ? (unsigned long long)a.top_k : (unsigned long long)ceil((double)a.top_p * (double)Z);
    if (T < 1ull) T = 1ull;
    if (T > Z) T = Z;
    unsigned long long cum = 0ull;
    int cb = kBins - 1;  // bins run from the highest scores down
    for (int i = 0; i < kBins; ++i) {
      if (cum + hb[i] >= T) {
        cb = i;
        break;
      }
      cum += hb[i];
    }
    rem = T - cum;
    above = cum;
    bin_key_range(m, cb, &klo, &khi);
    shift = slice_shift(klo, khi);
    mode = kModeKeys;
  }

  // ---- refinement: each walk captures the keys of a row's crossing key range (in position
  // order) into its global list while it sums the mass of 16 bit slices of the range.  A row
  // whose range holds at most kCapG keys then finishes from its list alone (no further walk);
  // otherwise its range narrows to the crossing slice for the next walk.
  for (int level = 0; level < kLevels; ++level) {
    if (!__syncthreads_or(mode == kModeKeys)) break;
    const bool mine = mode == kModeKeys;
    if (mine)
      for (int i = 0; i < kSlices; ++i) hist[i * kRowsR] = 0ull;
    int nc = 0;
    const uint32_t span = khi - klo;
    W.run(ntiles, [&](int64_t t, int c0, const float* s, int lim) {
      if (!mine) return;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t key = order_key(s[c]);
        if (c0 + c <= lim && key - klo <= span) {
          hist[(int)((key - klo) >> shift) * kRowsR] += weight(s[c], m);
          if (nc < kCapG)
            cap[(int64_t)nc * kRowsR] = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)(t * kKeysR + c0 + c));
          ++nc;
        }
      }
    });
    if (!mine) continue;
    if (nc <= kCapG) {
      // every key of the range is in the list: narrow the range over the list until at most
      // kCand keys remain (a single key value is an exact tie group), then sort those
      int n_in = nc;
      while (n_in > kCand && klo != khi) {
        for (int i = 0; i < kSlices; ++i) hist[i * kRowsR] = 0ull;
        const uint32_t sp = khi - klo;
        for (int i = 0; i < nc; ++i) {
          const uint32_t key = (uint32_t)(cap[(int64_t)i * kRowsR] >> 32);
          if (key - klo <= sp) hist[(int)((key - klo) >> shift) * kRowsR] += weight(key_to_float(key), m);
        }
        unsigned long long cum = 0ull;
        int cs = 0;
        for (int i = kSlices - 1; i >= 0; --i) {  // highest slice first
          const unsigned long long hs = hist[i * kRowsR];
          if (cum + hs >= rem) {
            cs = i;
            break;
          }
          cum += hs;
        }
        const uint32_t nlo = klo + ((uint32_t)cs << shift);
        const uint32_t top = nlo + ((1u << shift) - 1u);
        khi = top < khi && top >= nlo ? top : khi;
        klo = nlo;
        rem -= cum;
        above += cum;
        shift = slice_shift(klo, khi);
        n_in = 0;
        for (int i = 0; i < nc; ++i) n_in += ((uint32_t)(cap[(int64_t)i * kRowsR] >> 32) - klo <= khi - klo) ? 1 : 0;
      }
      if (n_in <= kCand) {
        unsigned long long cv[kCand];
        int n = 0;
        for (int i = 0; i < nc && n < kCand; ++i) {
          const unsigned long long e = cap[(int64_t)i * kRowsR];
          if ((uint32_t)(e >> 32) - klo <= khi - klo) cv[n++] = e;
        }
        for (int i = 1; i < n; ++i) {  // insertion sort, descending: key desc, then j asc
          const unsigned long long v = cv[i];
          int k = i - 1;
          while (k >= 0 && cv[k] < v) {
            cv[k + 1] = cv[k];
            --k;
          }
          cv[k + 1] = v;
        }
        unsigned long long cum = 0ull;
        int ci = -1;
        for (int i = 0; i < n; ++i) {
          cum += weight(key_to_float((uint32_t)(cv[i] >> 32)), m);
          if (cum >= rem) {
            ci = i;
            break;
          }
        }
        if (ci < 0) {  // not reached: the range was chosen to hold at least rem
          atomicOr(a.err, kErrInternal);
          t_key = 0xFFFFFFFFu;
          tiecut = -1;
        } else {
          t_key = (uint32_t)(cv[ci] >> 32);
          tiecut = (int)(0xFFFFFFFFu - (uint32_t)cv[ci]);
          above += cum;
        }
      } else {
        // one key value with more than kCand members: the n_need-th of them in position order
        // (the list is in position order)
        t_key = klo;
        const unsigned long long e = weight(key_to_float(klo), m);
        const unsigned long long need = e ? (rem + e - 1) / e : 1ull;
        unsigned long long seen = 0ull;
        tiecut = -1;
        for (int i = 0; i < nc; ++i) {
          const unsigned long long v = cap[(int64_t)i * kRowsR];
          if ((uint32_t)(v >> 32) == klo && ++seen == need) {
            tiecut = (int)(0xFFFFFFFFu - (uint32_t)v);
            break;
          }
        }
        if (tiecut < 0) {
          atomicOr(a.err, kErrInternal);
          tiecut = 0x7FFFFFFF;
        } else {
          above += need * e;
        }
      }
      mode = kModeDone;
    } else {
      unsigned long long cum = 0ull;
      int cs = -1;
      for (int i = kSlices - 1; i >= 0; --i) {  // highest slice first
        const unsigned long long hs = hist[i * kRowsR];
        if (cum + hs >= rem) {
          cs = i;
          break;
        }
        cum += hs;
      }
      if (cs < 0) {
        atomicOr(a.err, kErrInternal);
        t_key = 0xFFFFFFFFu;
        tiecut = -1;
        mode = kModeDone;
      } else {
        const uint32_t nlo = klo + ((uint32_t)cs << shift);
        const uint32_t top = nlo + ((1u << shift) - 1u);
        const uint32_t nhi = top < khi && top >= nlo ? top : khi;
        rem -= cum;
        above += cum;
        klo = nlo;
        khi = nhi;
        shift = slice_shift(nlo, nhi);
        if (nlo == nhi) {  // one key value with more than kCapG members: an exact tie group
          t_key = nlo;
          const unsigned long long e = weight(key_to_float(nlo), m);
          n_need = e ? (rem + e - 1) / e : 1ull;
          mode = kModeTie;
        }
      }
    }
  }
  if (mode == kModeKeys) {  // not reached: the walks narrow the range 16-fold each
    atomicOr(a.err, kErrInternal);
    t_key = 0xFFFFFFFFu;
    tiecut = -1;
    mode = kModeDone;
  }

  // ---- exact ties: the cutoff is the n_need-th tied position in ascending order
  if (__syncthreads_or(mode == kModeTie)) {
    const bool mine = mode == kModeTie;
    unsigned long long before = 0ull;
    bool found = false;
    W.run(ntiles, [&](int64_t t, int c0, const float* s, int lim) {
      if (!mine || found) return;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        if (c0 + c <= lim && order_key(s[c]) == t_key && !found) {
          if (++before == n_need) {
            tiecut = (int)(t * kKeysR + c0 + c);
            found = true;
          }
        }
      }
    });
    if (mine) {
      if (!found) {
        atomicOr(a.err, kErrInternal);
        tiecut = 0x7FFFFFFF;
      } else {
        above += n_need * weight(key_to_float(t_key), m);
      }
      mode = kModeDone;
    }
  }

  if (!W.ok) {
    W.drain();
    if (tid == 0) atomicOr(a.err, kErrTimeout);
  } else if (live) {
    cut[tid] = make_uint2(t_key, (uint32_t)tiecut);
    if (mass_out) *mass_out = topk ? -1.f : (float)((double)above / (double)Z);  // no masses with a fixed budget
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_free(tmem, kSelTmemCols);
  }
}

// ------------------------------------------------------------------ sparse attention

constexpr int kAttThreads = 256;          // two threads per row
constexpr uint32_t kAttTmemCols = 256;    // index scores [0,64), S [64,128), O [128,256)
constexpr uint32_t kColIdx = 0, kColS = 64, kColO = 128;
constexpr float kRescale = 11.f;          // log2 headroom before the reference max moves (P <= 2^11)
constexpr uint32_t kIdxStages = 3;
constexpr uint32_t kAOffQ = 0;                                  // Q tile (128-byte swizzle), 32 KB
constexpr uint32_t kAOffIQ = kAOffQ + kRowsR * 256;              // index query tile, 8 KB
constexpr uint32_t kAOffIK = kAOffIQ + kTcQBytes;                // index key ring, 3 x 4 KB
constexpr uint32_t kAOffK = kAOffIK + kIdxStages * kTcKBytes;    // K tile, 16 KB
constexpr uint32_t kAOffV = kAOffK + kKeysR * 256;               // V tile, 16 KB
constexpr uint32_t kAOffP = kAOffV + kKeysR * 256;               // P tile, 16 KB
constexpr uint32_t kAOffX = kAOffP + kRowsR * 128;               // mask exchange [2][128] u32, count [128]
constexpr uint32_t kAOffXf = kAOffX + 3 * kRowsR * 4;            // per-thread float exchange [256]
constexpr uint32_t kAOffBar = kAOffXf + kAttThreads * 4;         // ifull[3], idone, kfull, vfull, sdone, odone
constexpr uint32_t kAttSmem = kAOffBar + 8 * 8 + 16;
static_assert(kAOffK % 1024 == 0 && kAOffV % 1024 == 0 && kAOffP % 1024 == 0, "swizzled tiles need 1 KB alignment");
constexpr uint32_t kKVTileBytes = kKeysR * 256;
constexpr int kPartStride = 4 + kD;  // floats per row of a split's partial: m, l, count, pad, o[D]

__device__ __forceinline__ uint32_t pack_half2_r(float x, float y) {
  __half2 h = __floats2half2_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(kAttThreads, 2) prefill_attn_kernel(RetArgs a,
                                                                       const __grid_constant__ CUtensorMap tm_idx,
                                                                       const __grid_constant__ CUtensorMap tm_k,
                                                                       const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int half = tid >> 7, r = tid & (kRowsR - 1);
  // a row tile's keys may be split over attn_splits CTAs (key tiles [tb, tb + ntl) each), whose
  // partial (m, l, o) the last to finish merges; row tiles run longest first
  const int n_split = a.attn_splits;
  const int split = (int)(blockIdx.x % n_split);
  const int n_tiles_c = (int)(gridDim.x / n_split);
  const int tile = n_tiles_c - 1 - (int)(blockIdx.x / n_split), hr = blockIdx.y, b = blockIdx.z;
  const int i0 = tile * kRowsR;
  const int nrows = min(kRowsR, a.C - i0);
  const bool live = r < nrows;
  const int64_t P0 = a.P0.v[b];
  const int64_t pos = live ? P0 + i0 + r : -1;
  const int64_t nkeys = P0 + i0 + nrows;
  const int64_t nt = (nkeys + kKeysR - 1) / kKeysR;
  const int64_t tb = (int64_t)split * a.attn_split_tiles;
  const int64_t ntl = max((int64_t)0, min(nt, tb + a.attn_split_tiles) - tb);
  const int h = a.ret_head[hr], g = h / a.group;
  const int64_t qs = (int64_t)a.Hq * kD;
  const int64_t idx_row0 = ((int64_t)b * a.Hr + hr) * a.max_seq;
  const int64_t kv_row0 = ((int64_t)b * a.Hkv + g) * a.max_seq;
  const uint32_t barI = sbase + kAOffBar, barIdone = barI + 24, barK = barI + 32, barV = barI + 40,
                 barS = barI + 48, barO = barI + 56;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kAOffBar + 64);
  uint32_t* xm = reinterpret_cast<uint32_t*>(sm + kAOffX);  // [2][128]: half 1's masks of a tile
  int32_t* xcnt = reinterpret_cast<int32_t*>(sm + kAOffX + 2 * kRowsR * 4);

  if (sbase & 1023u) {  // the swizzle is a function of address bits: tiles on 1 KB boundaries
    if (tid == 0) atomicOr(a.err, kErrInternal);
    return;
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kAttTmemCols);
  if (tid == 0) {
    for (int i = 0; i < 8; ++i) mbar_init(barI + 8u * i, 1);
    fence_mbar_init();
  }
  // query rows: RoPE'd q as fp16 into the swizzled Q tile (each half writes 8 of the row's 16
  // chunks); the index queries (hi | lo) into the index query tile (half 0)
  {
    const float* qrow = a.q_rot + ((int64_t)b * a.C + i0 + (live ? r : 0)) * qs + (int64_t)h * kD;
#pragma unroll 4
    for (int cc = 0; cc < 8; ++cc) {
      const int c = 8 * half + cc;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (live) {
        const float4 x0 = *reinterpret_cast<const float4*>(qrow + 8 * c);
        const float4 x1 = *reinterpret_cast<const float4*>(qrow + 8 * c + 4);
        v.x = pack_half2_r(x0.x, x0.y);
        v.y = pack_half2_r(x0.z, x0.w);
        v.z = pack_half2_r(x1.x, x1.y);
        v.w = pack_half2_r(x1.z, x1.w);
      }
      *reinterpret_cast<uint4*>(sm + kAOffQ + sw128_off(r, c, kRowsR)) = v;
    }
    if (half == 0) {
      const float* iq = a.q_idx + (((int64_t)b * a.C + i0 + (live ? r : 0)) * a.Hr + hr) * kR;
      tc_put_query(sm + kAOffIQ, r, live ? iq : nullptr);
    }
  }
  // this row's cut
  uint32_t tk = 0xFFFFFFFFu;
  int64_t tcut = -1;
  if (live) {
    const uint2 cv = a.cut[((int64_t)b * a.Hr + hr) * a.C + i0 + r];
    tk = cv.x;
    tcut = (int32_t)cv.y;
  }
  // outputs of the selection statistics
  uint32_t* brow = (a.bitmap && live) ? a.bitmap + (((int64_t)b * a.C + i0 + r) * a.Hr + hr) * a.bitmap_words : nullptr;
  int32_t* lrow = nullptr;  // a listed row: where half 0 writes its positions
  if (a.row_sel && live && half == 0) {
    for (int i = 0; i < a.n_rows; ++i)
      if (a.rows[i] == i0 + r) lrow = a.row_sel + (((int64_t)b * a.n_rows + i) * a.Hr + hr) * a.row_sel_cap;
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);

  // phase counters of the mbarriers (each completion is waited exactly once, in order)
  uint32_t n_idone = 0, n_k = 0, n_v = 0, n_s = 0, n_o = 0;
  bool okw = true, ok = true, any_pv = false;
  auto ikt = [&](int64_t t) { return sbase + kAOffIK + (uint32_t)(t % kIdxStages) * kTcKBytes; };
  auto load_kv = [&](uint32_t bar, uint32_t dst, const CUtensorMap* map, int64_t t) {
    mbar_expect_tx(bar, kKVTileBytes);
    const int y = (int)(kv_row0 + t * kKeysR);
    tma_load_2d(dst, map, 0, y, bar);
    tma_load_2d(dst + kKeysR * 128, map, 64, y, bar);
  };
  // The row's cut as a float: key j is selected iff s_j > tf, or s_j == tf at a position
  // j <= tcut.  Float order equals the order of the (canonical, +0 for -0) order keys.  A row
  // without a cut has tk = 0xFFFFFFFF, whose float is a NaN that no score exceeds or equals;
  // the cut of p = 1 is tk = 0, below every finite score (-inf here).
  const float tf = tk == 0u ? -INFINITY : key_to_float(tk);
  // columns 0 .. x of this thread's 32 (none for x < 0, all for x >= 31)
  auto prefix_bits = [](int64_t x) -> uint32_t {
    return x < 0 ? 0u : (x >= 31 ? 0xFFFFFFFFu : (2u << (uint32_t)x) - 1u);
  };
  // this thread's selection mask of tile t (its 32 columns) from the index scores in TMEM
  auto read_mask = [&](int64_t t) -> uint32_t {
    okw = mbar_wait(barIdone, n_idone & 1u) && okw;
    ++n_idone;
    tc_fence_after();
    __syncwarp();
    float s[32];
    tmem_ld32(lane_addr + kColIdx + 32u * half, s);
    tmem_ld_wait();
    const int64_t j0 = t * kKeysR + 32 * half;  // position of column 0
    uint32_t gt[4] = {0u, 0u, 0u, 0u}, eq[4] = {0u, 0u, 0u, 0u};  // independent chains
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      gt[i & 3] |= (s[i] > tf ? 1u : 0u) << i;
      eq[i & 3] |= (s[i] == tf ? 1u : 0u) << i;
    }
    const uint32_t g = (gt[0] | gt[1]) | (gt[2] | gt[3]), e = (eq[0] | eq[1]) | (eq[2] | eq[3]);
    return (g | (e & prefix_bits(tcut - j0))) & prefix_bits(pos - j0);
  };
  // exchange one float per row between the two halves (threads tid and tid ^ 128) through
  // shared memory; consecutive calls are separated by at least one CTA barrier
  float* xf = reinterpret_cast<float*>(sm + kAOffXf);
  auto swap_half = [&](float v) -> float {
    xf[tid] = v;
    tc_fence_before();  // also orders this thread's TMEM reads before the barrier
    __syncthreads();
    tc_fence_after();
    return xf[tid ^ kRowsR];
  };

  // ---- prologue: index key tiles tb .. tb + 2 in flight, the scores of tile tb, its masks
  // (ring stages and barrier phases count tiles from tb; coordinates are absolute)
  uint32_t mask_cur = 0u;
  bool any_cur = false;
  if (ntl > 0) {
    if (tid == 0) {
      for (int64_t i = 0; i < (int64_t)kIdxStages && i < ntl; ++i)
        tc_load_keys(ikt(i), &tm_idx, idx_row0, tb + i, barI + 8u * (uint32_t)i);
      okw = mbar_wait(barI, 0u);
      if (okw) tc_issue_scores(tmem + kColIdx, sbase + kAOffIQ, ikt(0), barIdone);
    }
    mask_cur = read_mask(tb);
    tc_fence_before();
    if (half == 1) xm[(tb & 1) * kRowsR + r] = mask_cur;
    any_cur = __syncthreads_or(mask_cur != 0u) != 0;
    ok = __syncthreads_and(okw ? 1 : 0) != 0;
    if (ok && tid == 0) {
      if (ntl > 1) {
        okw = mbar_wait(barI + 8u, 0u);
        if (okw) tc_issue_scores(tmem + kColIdx, sbase + kAOffIQ, ikt(1), barIdone);
      }
      if (ntl > 3) tc_load_keys(ikt(3), &tm_idx, idx_row0, tb + 3, barI);  // stage 0: tile tb is scored
      if (any_cur) load_kv(barK, sbase + kAOffK, &tm_k, tb);
    }
  }

  float m_ref = -INFINITY, l = 0.f;  // reference max of row r; this half's share of the sum
  int nsel = 0;
  int64_t lbase = 0;  // listed positions written so far (half 0 of a listed row)
  for (int64_t u = 0; ok && u < ntl; ++u) {
    const int64_t t = tb + u;  // the absolute key tile
    // ---- statistics of tile t: count, bitmap words, listed positions
    nsel += __popc(mask_cur);
    if (brow) {
      const int64_t w = 2 * t + half;
      if (w < a.bitmap_words) brow[w] = mask_cur;
    }
    if (lrow) {  // half 0 writes both halves' positions, ascending
      uint32_t v = mask_cur;
      while (v && lbase < a.row_sel_cap) {
        const int p = __ffs(v) - 1;
        v &= v - 1;
        lrow[lbase++] = (int32_t)(t * kKeysR + p);
      }
      v = xm[(t & 1) * kRowsR + r];
      while (v && lbase < a.row_sel_cap) {
        const int p = __ffs(v) - 1;
        v &= v - 1;
        lrow[lbase++] = (int32_t)(t * kKeysR + 32 + p);
      }
    }
    // ---- (a) the masks of tile t + 1 (scored one tile ahead); the scores of tile t + 2
    uint32_t mask_next = 0u;
    bool any_next = false;
    if (u + 1 < ntl) {
      mask_next = read_mask(t + 1);
      tc_fence_before();
      if (half == 1) xm[((t + 1) & 1) * kRowsR + r] = mask_next;
      // one barrier: does any row select a key of tile t + 1, and has any wait given up
      const int f = __syncthreads_or((mask_next != 0u ? 1 : 0) | (okw ? 0 : 2));
      any_next = (f & 1) != 0;
      if (f & 2) ok = false;
      if (tid == 0 && u + 2 < ntl && okw) {
        okw = mbar_wait(barI + 8u * (uint32_t)((u + 2) % kIdxStages), (uint32_t)(((u + 2) / kIdxStages) & 1));
        if (okw) tc_issue_scores(tmem + kColIdx, sbase + kAOffIQ, ikt(u + 2), barIdone);
        if (u + 4 < ntl)  // the stage of tile t + 1 is free: its scores are done
          tc_load_keys(ikt(u + 4), &tm_idx, idx_row0, t + 4, barI + 8u * (uint32_t)((u + 4) % kIdxStages));
      }
    }
    // ---- (b) attention over tile t
    if (any_cur) {
      if (tid == 0) {
        if (any_pv && okw) okw = mbar_wait(barO, (n_o - 1) & 1u);  // V and P are free
        if (okw) load_kv(barV, sbase + kAOffV, &tm_v, t);
        if (okw) okw = mbar_wait(barK, n_k & 1u);
        if (okw) {
          tc_fence_after();
          constexpr uint32_t kIdS = umma_idesc_f16(kKeysR, false);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t ad = umma_desc(sbase + kAOffQ + (kk >> 2) * (kRowsR * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = umma_desc(sbase + kAOffK + (kk >> 2) * (kKeysR * 128) + (kk & 3) * 32, 16, 1024);
            umma_f16(tmem + kColS, ad, bd, kIdS, kk > 0 ? 1u : 0u);
          }
          umma_commit(barS);
        }
      }
      ++n_k;
      okw = mbar_wait(barS, n_s & 1u) && okw;
      ++n_s;
      tc_fence_after();
      __syncwarp();
      float sv[32];
      tmem_ld32(lane_addr + kColS + 32u * half, sv);
      tmem_ld_wait();
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // independent chains
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        sv[i] = ((mask_cur >> i) & 1u) ? sv[i] * a.scale_log2 : -INFINITY;
        m4[i & 3] = fmaxf(m4[i & 3], sv[i]);
      }
      float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      mx = fmaxf(mx, swap_half(mx));  // the row max over both halves (also orders the S reads)
      // S of tile t is done, and so is P V of the previous tile: K, P and O are free
      if (tid == 0 && any_next && okw) load_kv(barK, sbase + kAOffK, &tm_k, t + 1);
      const bool move = mx > m_ref + kRescale;
      if (any_pv && __any_sync(0xffffffffu, move)) {
        const float cf = move ? fast_exp2(m_ref - mx) : 1.f;  // warp-collective ld / st below
        const uint32_t oAddr = lane_addr + kColO + 64u * half;
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          float ov[32];
          tmem_ld32(oAddr + c0, ov);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= cf;
          tmem_st32(oAddr + c0, ov);
        }
        tmem_st_wait();
      }
      if (move) {
        l *= fast_exp2(m_ref - mx);  // 0 while m_ref is still -inf
        m_ref = mx;
      }
      float rs4[4] = {0.f, 0.f, 0.f, 0.f};
      const float mref = m_ref == -INFINITY ? 0.f : m_ref;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pv[e] = fast_exp2(sv[8 * q + e] - mref);
          rs4[e & 3] += pv[e];
        }
        uint4 w;
        w.x = pack_half2_r(pv[0], pv[1]);
        w.y = pack_half2_r(pv[2], pv[3]);
        w.z = pack_half2_r(pv[4], pv[5]);
        w.w = pack_half2_r(pv[6], pv[7]);
        *reinterpret_cast<uint4*>(sm + kAOffP + sw128_off(r, 4 * half + q, kRowsR)) = w;
      }
      l += (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
      fence_async_smem();
      tc_fence_before();
      ok = __syncthreads_and(okw ? 1 : 0) != 0;
      if (!ok) break;
      // ---- O += P V (one thread); V is read MN-major (rows = keys)
      if (tid == 0) {
        okw = mbar_wait(barV, n_v & 1u);
        if (okw) {
          tc_fence_after();
          constexpr uint32_t kIdO = umma_idesc_f16(kD, true);
#pragma unroll
          for (int kk = 0; kk < kKeysR / 16; ++kk) {
            const uint64_t ad = umma_desc(sbase + kAOffP + kk * 32, 16, 1024);
            const uint64_t bd = umma_desc(sbase + kAOffV + kk * 2048, kKeysR * 128, 1024);
            umma_f16(tmem + kColO, ad, bd, kIdO, (any_pv || kk > 0) ? 1u : 0u);
          }
          umma_commit(barO);
        }
      }
      ++n_v;
      ++n_o;
      any_pv = true;
    } else if (tid == 0 && any_next && okw) {
      load_kv(barK, sbase + kAOffK, &tm_k, t + 1);  // K is free: every earlier S has completed
    }
    mask_cur = mask_next;
    any_cur = any_next;
    // (no barrier here: the next tile's mask barrier also carries the wait status; a wait that
    // gives up after it is seen by the attention barrier of the tile that follows, or the exit)
  }

  if (ok && any_pv && tid == 0) okw = mbar_wait(barO, (n_o - 1) & 1u) && okw;
  ok = __syncthreads_and((ok && okw) ? 1 : 0) != 0;
  if (ok) {
    tc_fence_after();
    const float lt = l + swap_half(l);
    if (half == 1) xcnt[r] = nsel;  // selected counts: half 1 hands its count to half 0
    __syncthreads();
    const int cnt_row = nsel + xcnt[r];  // (half 0)
    float ov[64];
    const uint32_t oAddr = lane_addr + kColO + 64u * half;
    tmem_ld32(oAddr, ov);
    tmem_ld32(oAddr + 32u, ov + 32);
    tmem_ld_wait();
    if (!any_pv) {
#pragma unroll
      for (int i = 0; i < 64; ++i) ov[i] = 0.f;
    }
    float* orow = a.out + ((int64_t)b * a.C + i0 + (live ? r : 0)) * qs + (int64_t)h * kD + 64 * half;
    int32_t* crow = (a.sel_count && live && half == 0) ? a.sel_count + ((int64_t)b * a.C + i0 + r) * a.Hr + hr : nullptr;
    if (n_split == 1) {
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      if (live) {
#pragma unroll
        for (int i = 0; i < 64; i += 4)
          *reinterpret_cast<float4*>(orow + i) = make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
      }
      if (crow) *crow = cnt_row;
    } else {
      // this split's partial, then the last split of the row tile merges them all (log-sum-exp
      // in base 2: the o and l of each split are relative to its reference max m)
      const int64_t tix = ((int64_t)b * a.Hr + hr) * n_tiles_c + tile;
      float* pt = a.attn_part + tix * n_split * (int64_t)kRowsR * kPartStride;
      float* mine = pt + ((int64_t)split * kRowsR + r) * kPartStride;
#pragma unroll
      for (int i = 0; i < 64; i += 4)
        *reinterpret_cast<float4*>(mine + 4 + 64 * half + i) = make_float4(ov[i], ov[i + 1], ov[i + 2], ov[i + 3]);
      if (half == 0) *reinterpret_cast<float4*>(mine) = make_float4(m_ref, lt, __int_as_float(cnt_row), 0.f);
      __threadfence();
      __syncthreads();
      if (tid == 0) xcnt[0] = atomicAdd(a.attn_ticket + tix, 1u) == (uint32_t)(n_split - 1) ? 1 : 0;
      __syncthreads();
      if (xcnt[0]) {
        __threadfence();
        float M = -INFINITY;
        for (int sp = 0; sp < n_split; ++sp) M = fmaxf(M, __ldcg(pt + ((int64_t)sp * kRowsR + r) * kPartStride));
        float Ls = 0.f, o[64];
        int cnt = 0;
#pragma unroll
        for (int i = 0; i < 64; ++i) o[i] = 0.f;
        for (int sp = 0; sp < n_split; ++sp) {
          const float* q = pt + ((int64_t)sp * kRowsR + r) * kPartStride;
          const float ms = __ldcg(q);
          cnt += __float_as_int(__ldcg(q + 2));
          if (ms == -INFINITY) continue;  // no selected key of this row in that split
          const float f = fast_exp2(ms - M);
          Ls += __ldcg(q + 1) * f;
#pragma unroll
          for (int i = 0; i < 64; ++i) o[i] += __ldcg(q + 4 + 64 * half + i) * f;
        }
        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
        if (live) {
#pragma unroll
          for (int i = 0; i < 64; i += 4)
            *reinterpret_cast<float4*>(orow + i) = make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
        }
        if (crow) *crow = cnt;
        if (tid == 0) a.attn_ticket[tix] = 0u;
      }
    }
  } else if (tid == 0) {
    atomicOr(a.err, kErrTimeout);
    // wait (bounded) for the copies and MMAs this CTA may still have in flight: the next
    // phase of every barrier that has one pending
    mbar_wait(barIdone, n_idone & 1u);
    mbar_wait(barS, n_s & 1u);
    if (any_pv) mbar_wait(barO, (n_o - 1) & 1u);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_free(tmem, kAttTmemCols);
  }
}

}  // namespace

cudaError_t launch_prefill_retrieval(rtp_layer* L, int C, float* out, const rtp_prefill_stats* stats,
                                     cudaStream_t st) {
  if (!L->tm_ready) return cudaErrorInvalidValue;
  RetArgs a;
  a.max_seq = L->max_seq;
  a.Hkv = L->Hkv;
  a.Hq = L->Hq;
  a.Hr = L->Hr;
  a.group = L->group;
  a.C = C;
  a.P0 = seq_pos(L, -C);
  a.top_p = L->top_p;
  a.top_k = L->top_k;
  int lg = 0;
  while ((1ll << lg) < L->len) ++lg;
  a.sc_bits = 62 - lg;
  a.ret_head = L->d_ret_head;
  a.q_rot = L->q_rot;
  a.q_idx = L->q_idx;
  a.cut = L->pf_cut;
  a.capture = L->pf_capture;
  // long rows split their keys over several attention CTAs (one wave holds 2 per SM), unless a
  // row's positions are to be listed in order
  {
    const int64_t nt_max = (L->len + kKeysR - 1) / kKeysR;
    int64_t n_split = (nt_max + kAttSplitTiles - 1) / kAttSplitTiles;
    if (n_split < 1 || (stats && stats->rows)) n_split = 1;
    if (n_split > L->attn_split_max) n_split = L->attn_split_max;
    a.attn_splits = (int)n_split;
    a.attn_split_tiles = (nt_max + n_split - 1) / n_split;  // every key tile in some split
  }
  a.attn_part = L->attn_part;
  a.attn_ticket = L->attn_ticket;
  a.scale_log2 = L->sm_scale * 1.4426950408889634f;
  a.out = out;
  a.sel_count = stats ? stats->sel_count : nullptr;
  a.sel_mass = stats ? stats->sel_mass : nullptr;
  a.bitmap = stats ? stats->sel_bitmap : nullptr;
  a.bitmap_words = stats ? stats->bitmap_words : 0;
  a.rows = (stats && stats->rows) ? stats->rows : nullptr;
  a.n_rows = (stats && stats->rows) ? stats->n_rows : 0;
  a.row_sel = (stats && stats->rows) ? stats->row_sel : nullptr;
  a.row_sel_cap = (stats && stats->rows) ? stats->row_sel_cap : 0;
  a.err = L->err;
  const dim3 grid((C + kRowsR - 1) / kRowsR, L->Hr, L->B);
  const dim3 agrid(grid.x * a.attn_splits, L->Hr, L->B);
  cudaError_t e;
  {
    ProfScope ps(L, "prefill_select", st);
    e = cudaFuncSetAttribute(prefill_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSelSmem);
    if (e != cudaSuccess) return e;
    prefill_select_kernel<<<grid, kPsThreads, kSelSmem, st>>>(a, L->tm_idx);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    ProfScope ps(L, "prefill_attn", st);
    e = cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttSmem);
    if (e != cudaSuccess) return e;
    prefill_attn_kernel<<<agrid, kAttThreads, kAttSmem, st>>>(a, L->tm_idx, L->tm_k, L->tm_v);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace rtp
