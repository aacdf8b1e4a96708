// prefill_retrieval.cu -- retrieval heads in chunked prefill: per-row top-p + sparse attention.
//
// Every query row i of the chunk (position pos = len - C + i) runs its own selection over its
// causal prefix j <= pos: pre-RoPE index scores s_j = qidx_i . IDX[j] (techwalker page,
// section 3), the shortest prefix of the order (s desc, j asc) whose index-softmax mass reaches
// p (zhichai page, insight 3; techwalker page, section 4), then exact RoPE'd attention over
// that set.  (The pages' own prefill keeps retrieval heads dense -- techwalker page, limits;
// ngjoo digest, limitations -- the per-row selection here is the chunked-prefill counterpart
// of the decode selection.)
//
// One CTA per (64-row tile, retrieval head, sequence), 128 threads.  Rows are independent,
// so every step stays inside the CTA:
//   * scoring: thread t owns row t % 64 and half (t / 64) of every 64-key index tile (staged in
//     shared memory, read as broadcasts); a score is a fixed-order fp32 dot product, so every
//     pass -- and the attention mask -- recomputes bit-identical scores;
//   * pass A: row maxima;  pass B: fixed-point mass histogram (64 bins of width 1/4 below the
//     max, keys 16..32 below summed apart, the rest negligible -- same argument as the decode
//     selection) -> total mass Z, target T = ceil(p Z), crossing bin;
//   * refinement passes: inside the crossing bin, 64-way splits of the order-key range (exact
//     integer arithmetic) until a row's range holds <= 32 keys, which are sorted to give the
//     exact cut key t and tie cutoff; a range that shrinks to one key value with more members
//     is an exact tie, resolved by an ordered count of the tied positions;
//   * attention pass: for each key tile the selection mask (s > t, or s == t and j <= cutoff)
//     is recomputed; tiles no row selects are skipped, the others run on tensor cores
//     (fa_tile.cuh) with the mask.
#include "fa_tile.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr int kRows = kFaRows;          // 64 query rows per CTA
constexpr int kKeys = 64;               // index keys per tile
constexpr int kThreads = kFaThreads;    // 128: two threads per row
constexpr int kHalf = kKeys / 2;        // keys per thread per tile
constexpr int kBins = 64;
constexpr int kCandPerThread = 16;
constexpr float kLog2e = 1.4426950408889634f;

enum : int { kModeHist = 0, kModeKeys = 1, kModeTie = 2, kModeDone = 3 };

struct RetArgs {
  const float* idx;           // [B][Hr][max_seq][r]
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
  float scale_log2;
  float* out;                 // [B][C][Hq][D]
  int32_t* sel_count;         // [B][C][Hr] or nullptr
  float* sel_mass;            // [B][C][Hr] or nullptr
  uint32_t* bitmap;           // [B][C][Hr][bitmap_words] or nullptr
  int64_t bitmap_words;
  uint32_t* err;
};

struct RowSel {
  float m;
  int mode;
  int bin1;           // crossing level-1 bin (kBins: the 16..32 band)
  int found;          // tie mode: cutoff located
  uint32_t klo, khi;  // current order-key range (inclusive) inside bin1
  uint32_t t_key;     // exact cut key
  int tiecut;         // positions j <= tiecut with key t_key are selected
  unsigned long long Z, rem, n_need, tie_before;
};

// Per-thread arrays are stored [item][thread] so that a warp touching item i of its own rows
// hits consecutive words.
struct SmemR {
  RowSel row[kRows];
  float ik[2][kKeys][kR];                          // index key tiles (8 KB)
  unsigned long long cand[kCandPerThread][kThreads];  // refinement candidates (16 KB)
  unsigned long long coarse[kThreads];
  int ncand[kThreads];
  uint32_t mask[kRows][2];                         // per-row 64-key masks (two halves)
  union {
    unsigned long long hist[kBins][kThreads];      // 64 KB: per-thread mass histograms
    unsigned char kv[2 * kFaTileBytes];            // 32 KB: one K and one V tile
  } u;
};

__device__ __forceinline__ unsigned long long mass64(float s, float m, float scale) {
  const float q = fast_exp2((s - m) * kLog2e) * scale;
  const float qh = floorf(q * 2.3283064365386963e-10f);
  const uint32_t hi = (uint32_t)qh, lo = __float2uint_rn(fmaf(qh, -4294967296.0f, q));
  return ((unsigned long long)hi << 32) | lo;
}

// level-1 bin of a score below the row max: 0..63 (width 1/4), kBins (16..32), kBins+1 (tail)
__device__ __forceinline__ int bin1_of(float s, float m) {
  const float x = m - s;
  if (x < 16.f) return (int)(x * 4.f);
  if (x < 32.f) return kBins;
  return kBins + 1;
}

__device__ __forceinline__ float score16(const float* qt, const float* k) {
  const float4* k4 = reinterpret_cast<const float4*>(k);
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4 v = k4[c];
    s = fmaf(qt[4 * c + 0], v.x, s);
    s = fmaf(qt[4 * c + 1], v.y, s);
    s = fmaf(qt[4 * c + 2], v.z, s);
    s = fmaf(qt[4 * c + 3], v.w, s);
  }
  return s + 0.0f;  // -0 -> +0: equal scores get equal order keys
}

// Order-key range [lo, hi] that contains every score whose level-1 bin is b (with margin;
// membership is always re-tested with bin1_of).
__device__ __forceinline__ void bin_key_range(float m, int b, uint32_t* lo, uint32_t* hi) {
  const float x_lo = b < kBins ? 0.25f * b : 16.f;
  const float x_hi = b < kBins ? 0.25f * (b + 1) : 32.f;
  const float eps = 4.f * fmaxf(fabsf(m), 32.f) * 1.1920929e-7f;
  *lo = order_key(m - x_hi - eps);
  *hi = order_key(m - x_lo + eps);
}

// Stage index-key tile t (keys t*64 .. +63, zero beyond nkeys) into buffer buf.
__device__ __forceinline__ void stage_ik(SmemR& S, int buf, const float* base, int64_t t, int64_t nkeys) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int i = 0; i < (kKeys * kR / 4) / kThreads; ++i) {  // 2 x 16 bytes per thread
    const int idx = i * kThreads + tid;
    const int r = idx >> 2, c4 = idx & 3;
    const int64_t j = t * kKeys + r;
    const bool ok = j < nkeys;
    cp_async16(&S.ik[buf][r][c4 * 4], base + (ok ? j : 0) * kR + c4 * 4, ok ? 16 : 0);
  }
  cp_async_commit();
}

// Run f(j, s) over this thread's keys j <= pos (its half of every tile), tiles double-buffered.
template <typename F>
__device__ __forceinline__ void scan_keys(SmemR& S, const float* ibase, int64_t nkeys, int64_t pos, bool active,
                                          const float* qt, F f) {
  const int hf = threadIdx.x >> 6;
  const int64_t ntiles = (nkeys + kKeys - 1) / kKeys;
  stage_ik(S, 0, ibase, 0, nkeys);
  for (int64_t t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) {
      stage_ik(S, (t + 1) & 1, ibase, t + 1, nkeys);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (active) {
      const int buf = t & 1;
#pragma unroll 4
      for (int k = 0; k < kHalf; ++k) {
        const int64_t j = t * kKeys + hf * kHalf + k;
        if (j > pos) break;
        f(j, score16(qt, S.ik[buf][hf * kHalf + k]));
      }
    }
    __syncthreads();
  }
}

// Exact top-p cut of each row of the tile: on return S.row[r] holds (t_key, tiecut) such that
// key j of row r is selected iff order_key(s_j) > t_key, or == t_key and j <= tiecut.
__device__ void select_rows(SmemR& S, const RetArgs& a, const float* ibase, const float* qt, int64_t pos,
                            int64_t nkeys, bool active, float scale) {
  const int tid = threadIdx.x, r = tid & (kRows - 1), hf = tid >> 6;

  // ---- pass A: row maxima
  float mx = -INFINITY;
  scan_keys(S, ibase, nkeys, pos, active, qt, [&](int64_t, float s) { mx = fmaxf(mx, s); });
  S.u.hist[0][tid] = __float_as_uint(mx);  // exchange of the two halves
  __syncthreads();
  if (hf == 0) {
    RowSel& R = S.row[r];
    R.m = fmaxf(mx, __uint_as_float((uint32_t)S.u.hist[0][tid + kRows]));
    R.mode = active ? kModeHist : kModeDone;
    R.found = 0;
    R.tie_before = 0;
  }
  __syncthreads();

  // ---- pass B: level-1 mass histogram -> Z, T = ceil(p Z), crossing bin
  {
    const float m = S.row[r].m;
    for (int i = 0; i < kBins; ++i) S.u.hist[i][tid] = 0ull;
    unsigned long long co = 0;
    scan_keys(S, ibase, nkeys, pos, active, qt, [&](int64_t, float s) {
      const int bb = bin1_of(s, m);
      if (bb < kBins) S.u.hist[bb][tid] += mass64(s, m, scale);
      else if (bb == kBins) co += mass64(s, m, scale);
    });
    S.coarse[tid] = co;
    __syncthreads();
    if (hf == 0 && active) {
      RowSel& R = S.row[r];
      unsigned long long Z = S.coarse[tid] + S.coarse[tid + kRows];
      for (int i = 0; i < kBins; ++i) {
        S.u.hist[i][tid] += S.u.hist[i][tid + kRows];
        Z += S.u.hist[i][tid];
      }
      unsigned long long T = (unsigned long long)ceil((double)a.top_p * (double)Z);
      if (T < 1ull) T = 1ull;
      if (T > Z) T = Z;
      unsigned long long cum = 0;
      int cb = kBins;  // bins run from the highest scores down
      for (int i = 0; i < kBins; ++i) {
        if (cum + S.u.hist[i][tid] >= T) {
          cb = i;
          break;
        }
        cum += S.u.hist[i][tid];
      }
      R.Z = Z;
      R.bin1 = cb;
      R.rem = T - cum;
      bin_key_range(R.m, cb, &R.klo, &R.khi);
      R.mode = kModeKeys;
    }
    __syncthreads();
  }

  // ---- refinement: split the key range of the crossing bin 64 ways until <= 2 x 16 keys remain
  for (int level = 0; level < 8; ++level) {
    const int need = (hf == 0 && S.row[r].mode == kModeKeys) ? 1 : 0;
    if (!__syncthreads_or(need)) break;
    const bool mine = active && S.row[r].mode == kModeKeys;
    const float m = S.row[r].m;
    const int b1 = S.row[r].bin1;
    const uint32_t klo = S.row[r].klo, khi = S.row[r].khi;
    const unsigned long long span = (unsigned long long)(khi - klo) + 1ull;
    for (int i = 0; i < kBins; ++i) S.u.hist[i][tid] = 0ull;
    int nc = 0;
    scan_keys(S, ibase, nkeys, pos, mine, qt, [&](int64_t j, float s) {
      if (bin1_of(s, m) != b1) return;
      const uint32_t key = order_key(s);
      if (key < klo || key > khi) return;
      const int sub = (int)(((unsigned long long)(key - klo) * kBins) / span);  // 0 = lowest keys
      S.u.hist[sub][tid] += mass64(s, m, scale);
      if (nc < kCandPerThread) S.cand[nc][tid] = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)j);
      ++nc;
    });
    S.ncand[tid] = nc;
    __syncthreads();
    if (hf == 0 && mine) {
      RowSel& W = S.row[r];
      const int n0 = S.ncand[tid], n1 = S.ncand[tid + kRows];
      if (n0 <= kCandPerThread && n1 <= kCandPerThread) {
        // few keys left: the exact cut from the candidates sorted by (key desc, j asc)
        unsigned long long c[2 * kCandPerThread];
        int n = 0;
        for (int i = 0; i < n0; ++i) c[n++] = S.cand[i][tid];
        for (int i = 0; i < n1; ++i) c[n++] = S.cand[i][tid + kRows];
        for (int i = 1; i < n; ++i) {
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
          cum += mass64(key_to_float((uint32_t)(c[i] >> 32)), m, scale);
          if (cum >= W.rem) {
            ci = i;
            break;
          }
        }
        if (ci < 0) {  // cannot happen: the range was chosen to hold at least rem
          atomicOr(a.err, kErrInternal);
          W.t_key = 0xFFFFFFFFu;
          W.tiecut = -1;
        } else {
          W.t_key = (uint32_t)(c[ci] >> 32);
          W.tiecut = (int)(0xFFFFFFFFu - (uint32_t)c[ci]);
        }
        W.mode = kModeDone;
      } else {
        unsigned long long cum = 0;
        int cs = -1;
        for (int i = kBins - 1; i >= 0; --i) {  // highest sub-range first
          const unsigned long long hs = S.u.hist[i][tid] + S.u.hist[i][tid + kRows];
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
          const uint32_t nlo = klo + (uint32_t)(((unsigned long long)cs * span + kBins - 1) / kBins);
          const uint32_t nhi = klo + (uint32_t)((((unsigned long long)(cs + 1)) * span + kBins - 1) / kBins) - 1u;
          W.rem -= cum;
          W.klo = nlo;
          W.khi = nhi;
          if (nlo == nhi) {  // one key value with more than 32 members: an exact tie group
            W.t_key = nlo;
            const unsigned long long e = mass64(key_to_float(nlo), m, scale);
            W.n_need = e ? (W.rem + e - 1) / e : 1ull;
            W.mode = kModeTie;
          }
        }
      }
    }
    __syncthreads();
  }
  if (hf == 0 && active && S.row[r].mode == kModeKeys) {  // not reached: six levels split 32 bits
    atomicOr(a.err, kErrInternal);
    S.row[r].t_key = 0xFFFFFFFFu;
    S.row[r].tiecut = -1;
    S.row[r].mode = kModeDone;
  }
  __syncthreads();

  // ---- exact ties: the cutoff is the position of the n_need-th tied key in ascending order
  const int need = (hf == 0 && S.row[r].mode == kModeTie) ? 1 : 0;
  if (!__syncthreads_or(need)) return;
  const bool mine = active && S.row[r].mode == kModeTie;
  const uint32_t tk = S.row[r].t_key;
  const float m = S.row[r].m;
  const int b1 = S.row[r].bin1;
  const int64_t ntiles = (nkeys + kKeys - 1) / kKeys;
  for (int64_t t = 0; t < ntiles; ++t) {
    stage_ik(S, 0, ibase, t, nkeys);
    cp_async_wait<0>();
    __syncthreads();
    uint32_t bits = 0;
    if (mine) {
      for (int k = 0; k < kHalf; ++k) {
        const int64_t j = t * kKeys + hf * kHalf + k;
        if (j > pos) break;
        const float s = score16(qt, S.ik[0][hf * kHalf + k]);
        if (bin1_of(s, m) == b1 && order_key(s) == tk) bits |= 1u << k;
      }
    }
    S.mask[r][hf] = bits;
    __syncthreads();
    if (hf == 0 && mine) {
      RowSel& W = S.row[r];
      if (!W.found) {
        const unsigned long long mk = ((unsigned long long)S.mask[r][1] << 32) | S.mask[r][0];
        const int cnt = __popcll(mk);
        if (W.tie_before + cnt >= W.n_need) {
          int want = (int)(W.n_need - W.tie_before);
          unsigned long long x = mk;
          while (--want > 0) x &= x - 1;  // drop the lowest (want - 1) set bits
          W.tiecut = (int)(t * kKeys + (__ffsll((long long)x) - 1));
          W.found = 1;
        }
        W.tie_before += cnt;
      }
    }
    __syncthreads();
  }
  if (hf == 0 && mine) {
    if (!S.row[r].found) {
      atomicOr(a.err, kErrInternal);
      S.row[r].tiecut = 0x7FFFFFFF;
    }
    S.row[r].mode = kModeDone;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads) prefill_retrieval_kernel(RetArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SmemR& S = *reinterpret_cast<SmemR*>(smem_raw);
  const int tile = blockIdx.x, hr = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, r = tid & (kRows - 1), hf = tid >> 6, warp = tid >> 5;
  const int h = a.ret_head[hr], g = h / a.group;
  const int i0 = tile * kRows;
  const int nrows = min(kRows, a.C - i0);
  const bool active = r < nrows;
  const int64_t pos = a.P0 + i0 + r;                 // this thread's row position
  const int64_t pos_max = a.P0 + i0 + nrows - 1;
  const int64_t nkeys = pos_max + 1;
  const float scale = __uint_as_float((uint32_t)(127 + a.sc_bits) << 23);
  const float* ibase = a.idx + ((int64_t)b * a.Hr + hr) * a.max_seq * kR;

  float qt[kR];
  {
    const float* qp = a.q_idx + (((int64_t)b * a.C + (active ? i0 + r : i0)) * a.Hr + hr) * kR;
#pragma unroll
    for (int c = 0; c < kR; ++c) qt[c] = qp[c];
  }

  if (a.top_p < 1.f) {
    select_rows(S, a, ibase, qt, pos, nkeys, active, scale);
  } else {  // p = 1 keeps every causal key (also those whose mass rounds to 0)
    if (hf == 0) {
      S.row[r].t_key = 0u;
      S.row[r].tiecut = 0x7FFFFFFF;
    }
    __syncthreads();
  }

  // ---- attention over the selected keys of each row
  const __half* kb = a.kc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD;
  const __half* vb = a.vc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD;
  const int64_t qs = (int64_t)a.Hq * kD;
  uint32_t qa[8][4];
  fa_load_q(qa, a.q_rot + ((int64_t)b * a.C + i0) * qs + (int64_t)h * kD, qs, warp * 16, nrows);
  FaAcc A;
  fa_init(A);
  const uint32_t tk = S.row[r].t_key;
  const int tcut = S.row[r].tiecut;
  const bool want_mass = a.sel_mass != nullptr && a.top_p < 1.f;
  const float m = want_mass ? S.row[r].m : 0.f;
  uint32_t* brow = (a.bitmap && active) ? a.bitmap + (((int64_t)b * a.C + i0 + r) * a.Hr + hr) * a.bitmap_words
                                        : nullptr;
  int nsel = 0;
  unsigned long long msum = 0;
  const int64_t ntiles = (nkeys + kKeys - 1) / kKeys;
  for (int64_t t = 0; t < ntiles; ++t) {
    stage_ik(S, 0, ibase, t, nkeys);
    cp_async_wait<0>();
    __syncthreads();
    uint32_t bits = 0;
    if (active) {
      for (int k = 0; k < kHalf; ++k) {
        const int64_t j = t * kKeys + hf * kHalf + k;
        if (j > pos) break;
        const float s = score16(qt, S.ik[0][hf * kHalf + k]);
        const uint32_t key = order_key(s);
        if (key > tk || (key == tk && j <= tcut)) {
          bits |= 1u << k;
          if (want_mass) msum += mass64(s, m, scale);
        }
      }
      const int64_t w = 2 * t + hf;
      if (brow && w < a.bitmap_words) brow[w] = bits;
    }
    S.mask[r][hf] = bits;
    nsel += __popc(bits);
    if (!__syncthreads_or(bits != 0u)) continue;  // no row selects a key of this tile
    fa_stage(S.u.kv, S.u.kv + kFaTileBytes, kb, vb, (int)min((int64_t)kKeys, nkeys - t * kKeys),
             [&](int rr) { return t * kKeys + rr; });
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    fa_tile(A, qa, S.u.kv, S.u.kv + kFaTileBytes, a.scale_log2,
            [&](int rr, int tt) { return ((S.mask[rr][tt >> 5] >> (tt & 31)) & 1u) != 0u; });
    __syncthreads();
  }
  fa_store(A, a.out + ((int64_t)b * a.C + i0) * qs + (int64_t)h * kD, qs, warp * 16, nrows);
  if (a.sel_count || a.sel_mass) {
    S.ncand[tid] = nsel;
    S.coarse[tid] = msum;
    __syncthreads();
    if (hf == 0 && active) {
      const int64_t o = ((int64_t)b * a.C + i0 + r) * a.Hr + hr;
      if (a.sel_count) a.sel_count[o] = S.ncand[tid] + S.ncand[tid + kRows];
      if (a.sel_mass)
        a.sel_mass[o] = a.top_p < 1.f ? (float)((double)(S.coarse[tid] + S.coarse[tid + kRows]) / (double)S.row[r].Z)
                                      : 1.f;
    }
  }
}

}  // namespace

cudaError_t launch_prefill_retrieval(const rtp_layer* L, int C, float* out, const rtp_prefill_stats* stats,
                                     cudaStream_t st) {
  RetArgs a;
  a.idx = L->idx;
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
  a.scale_log2 = L->sm_scale * 1.4426950408889634f;
  a.out = out;
  a.sel_count = stats ? stats->sel_count : nullptr;
  a.sel_mass = stats ? stats->sel_mass : nullptr;
  a.bitmap = stats ? stats->sel_bitmap : nullptr;
  a.bitmap_words = stats ? stats->bitmap_words : 0;
  a.err = L->err;
  const size_t smem = sizeof(SmemR);
  cudaError_t e = cudaFuncSetAttribute(prefill_retrieval_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((C + kRows - 1) / kRows, L->Hr, L->B);
  prefill_retrieval_kernel<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
