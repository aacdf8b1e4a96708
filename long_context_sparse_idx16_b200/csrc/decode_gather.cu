// decode_gather.cu -- exact attention of one decode query over its selected keys.
//
// Retrieval heads attend, in the full head dim, to the keys their top-p selection kept
// (techwalker page, section 3: "full 128-dim exact computation on the selected tokens";
// section 6: the sparse-KV kernel splits long selections across CTAs and the last CTA to
// finish merges the results).
//
// B200 design: two kernels over the same selected lists, chosen by the selection mode.
//   * Item kernel (per-key top-p, whose lists are short): work items are (problem, run of
//     consecutive 128-key chunks), enumerated on the device from the selection counts; a
//     problem has at most 64 items (runs of one chunk until it has more than 64 chunks).  A
//     half-warp owns one key row (16 lanes x 16 bytes = one 256-byte fp16 K or V row); all rows
//     of the lane's chunk share are loaded into registers before any math.  Many CTAs per SM,
//     one item each, keep short lists at their latency floor.
//   * Flat kernel (p = 1, fixed top-k budgets, clustered selection: long lists): the lists of
//     all problems form one flat list of T keys; CTA c of a persistent grid (one per SM) takes
//     keys [c T / G, (c + 1) T / G), so every SM streams the same number of rows whatever the
//     list sizes.  Rows stream through shared memory by cp.async in stages of 64 keys, four
//     buffers deep, across the boundaries between lists; a half-warp reads back exactly the
//     slices it copied, so the stream needs no CTA barrier, and the two rows a half-warp holds
//     per stage share one running-max update.
//   * Scores and the running softmax stay in fp32 registers; the query stays fp32.  Partials
//     (m, l, o[128]) of a list split between items or CTAs are merged in order by the CTA that
//     takes the last ticket (deterministic, no waiting), which also resets the ticket.
#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

// item kernel
constexpr int kIChunk = kGatherChunk;
constexpr int kIThreads = 256;
constexpr int kIWarps = kIThreads / 32;
constexpr int kIRowsPerHalf = kIChunk / (2 * kIWarps);  // rows per half-warp per chunk
// flat kernel: stages of 64 keys (K and V, 32 KB), kStages buffers deep, one CTA per SM
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kStageKeys = 64;
constexpr int kRowsPerStage = kStageKeys / (2 * kWarps);  // rows per half-warp per stage (2)
constexpr int kStages = 4;  // 128 KB: the window kernel (64 KB) still fits beside it
constexpr size_t kGatherSmem = (size_t)kStages * 2 * kStageKeys * kD * sizeof(__half);
constexpr int kMaxProblems = 2048;

struct GatherArgs {
  const __half* kc;
  const __half* vc;
  int64_t max_seq;
  int Hkv, Hq, Hr, group;
  const float* q_rot;  // [B][Hq][D]
  const int32_t* sel_idx;
  int64_t max_select;
  const int32_t* sel_cnt;
  const int16_t* ret_head;
  int P;
  int dense;
  SeqPos lens;  // each sequence's length (a dense step attends to all its keys)
  float scale_log2;
  float* part;
  uint32_t* ticket;
  uint32_t* err;
  float* out;  // [B][Hq][D]
};

__device__ __forceinline__ void unpack8(uint4 u, float* f) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 x = __half22float2(h[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}

__global__ void __launch_bounds__(kIThreads) decode_gather_items_kernel(GatherArgs a) {
  __shared__ int s_base[kMaxProblems + 1];
  __shared__ int s_span[kMaxProblems];
  __shared__ float s_m[kIWarps], s_l[kIWarps];
  __shared__ float s_o[kIWarps][kD];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, hl = lane & 15;

  // item prefix over problems: counts loaded in parallel, summed by one thread from smem
  for (int p = tid; p < a.P; p += kIThreads) {
    const int64_t K = a.dense ? (int64_t)a.lens.v[p / a.Hr] : (int64_t)a.sel_cnt[p];
    const int chunks = (int)((K + kIChunk - 1) / kIChunk);
    const int span = chunks > kGatherMaxItems ? (chunks + kGatherMaxItems - 1) / kGatherMaxItems : 1;
    s_span[p] = span;
    s_base[p + 1] = (chunks + span - 1) / span;
  }
  __syncthreads();
  if (tid == 0) {
    s_base[0] = 0;
    for (int p = 0; p < a.P; ++p) s_base[p + 1] += s_base[p];
  }
  __syncthreads();
  const int total_items = s_base[a.P];

  for (int it = blockIdx.x; it < total_items; it += gridDim.x) {
    // the problem of this item: the largest p with s_base[p] <= it (skips problems with no items)
    int p = 0;
    {
      int hi = a.P - 1;
      while (p < hi) {
        const int mid = (p + hi + 1) >> 1;
        if (s_base[mid] <= it) p = mid;
        else hi = mid - 1;
      }
    }
    const int item = it - s_base[p];
    const int n_items = s_base[p + 1] - s_base[p];
    const int b = p / a.Hr, hr = p % a.Hr;
    const int h = a.ret_head[hr], g = h / a.group;
    const int64_t Nb = a.lens.v[b];  // this sequence's keys
    const int64_t K = a.dense ? Nb : (int64_t)a.sel_cnt[p];
    const int64_t r_begin = (int64_t)item * s_span[p] * kIChunk;
    const int64_t r_end = min(K, r_begin + (int64_t)s_span[p] * kIChunk);

    const __half* kbase = a.kc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD + hl * 8;
    const __half* vbase = a.vc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD + hl * 8;
    const int32_t* ids = a.sel_idx + (int64_t)p * a.max_select;
    float q[8];
    {
      const float4* qp = reinterpret_cast<const float4*>(a.q_rot + ((int64_t)b * a.Hq + h) * kD + hl * 8);
      const float4 q0 = qp[0], q1 = qp[1];
      q[0] = q0.x; q[1] = q0.y; q[2] = q0.z; q[3] = q0.w;
      q[4] = q1.x; q[5] = q1.y; q[6] = q1.z; q[7] = q1.w;
    }
    float m = -INFINITY, l = 0.f, o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = 0.f;
    for (int64_t r_lo = r_begin; r_lo < r_end; r_lo += kIChunk) {
      const int64_t r_hi = min(r_end, r_lo + kIChunk);
      // rows of this half-warp: r_lo + (warp * 2 + half) + 16 * u
      uint4 kr[kIRowsPerHalf], vr[kIRowsPerHalf];
#pragma unroll
      for (int u = 0; u < kIRowsPerHalf; ++u) {
        const int64_t r = r_lo + (warp * 2 + half) + 2 * kIWarps * u;
        if (r < r_hi) {
          int64_t j = a.dense ? r : (int64_t)__ldg(ids + r);
          if ((uint64_t)j >= (uint64_t)Nb) {  // never expected: a stale or corrupt list
            atomicOr(a.err, kErrInternal);
            j = 0;
          }
          kr[u] = ld_nc_u4(kbase + j * kD);
          vr[u] = ld_nc_u4(vbase + j * kD);
        } else {
          kr[u] = make_uint4(0, 0, 0, 0);
          vr[u] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < kIRowsPerHalf; ++u) {
        const int64_t r = r_lo + (warp * 2 + half) + 2 * kIWarps * u;
        float kf[8];
        unpack8(kr[u], kf);
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) s = fmaf(q[i], kf[i], s);
        s += __shfl_xor_sync(0xffffffffu, s, 8);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        if (r < r_hi) {
          s *= a.scale_log2;
          const float mn = fmaxf(m, s);
          const float corr = fast_exp2(m - mn);
          const float w = fast_exp2(s - mn);
          float vf[8];
          unpack8(vr[u], vf);
          l = l * corr + w;
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = fmaf(w, vf[i], o[i] * corr);
          m = mn;
        }
      }
    }  // chunks of the item
    // merge the two half-warps
    {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, 16);
      const float l2 = __shfl_xor_sync(0xffffffffu, l, 16);
      const float mn = fmaxf(m, m2);
      const float c1 = (m == -INFINITY) ? 0.f : fast_exp2(m - mn);
      const float c2 = (m2 == -INFINITY) ? 0.f : fast_exp2(m2 - mn);
      l = l * c1 + l2 * c2;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float o2 = __shfl_xor_sync(0xffffffffu, o[i], 16);
        o[i] = o[i] * c1 + o2 * c2;
      }
      m = mn;
    }
    if (half == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) s_o[warp][hl * 8 + i] = o[i];
      if (hl == 0) {
        s_m[warp] = m;
        s_l[warp] = l;
      }
    }
    __syncthreads();
    // CTA merge: thread d < 128 owns output dim d
    float cm = -INFINITY, cl = 0.f, co = 0.f;
    if (tid < kD) {
#pragma unroll
      for (int w = 0; w < kIWarps; ++w) cm = fmaxf(cm, s_m[w]);
#pragma unroll
      for (int w = 0; w < kIWarps; ++w) {
        const float c = (s_m[w] == -INFINITY) ? 0.f : fast_exp2(s_m[w] - cm);
        cl += s_l[w] * c;
        co += s_o[w][tid] * c;
      }
    }
    float* outp = a.out + ((int64_t)b * a.Hq + h) * kD;
    if (n_items == 1) {
      if (tid < kD) outp[tid] = co / cl;
    } else {
      float* pp = a.part + (int64_t)it * (kD + 2);
      if (tid < kD) pp[2 + tid] = co;
      if (tid == 0) {
        pp[0] = cm;
        pp[1] = cl;
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) s_last = (atomicAdd(a.ticket + p, 1u) == (uint32_t)(n_items - 1));
      __syncthreads();
      if (s_last) {
        __threadfence();
        const float* base = a.part + (int64_t)s_base[p] * (kD + 2);
        // M = max over item maxima (all threads), then warp w folds items w, w+8, ... with
        // lane-owned float4 column slices; the 8 warp results are combined in smem.
        float mv = -INFINITY;
        for (int i = tid; i < n_items; i += kIThreads) mv = fmaxf(mv, __ldcg(base + (int64_t)i * (kD + 2)));
        mv = warp_max(mv);
        if (lane == 0) s_m[warp] = mv;
        __syncthreads();
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kIWarps; ++w) M = fmaxf(M, s_m[w]);
        __syncthreads();
        float lsum = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int i = warp; i < n_items; i += kIWarps) {
          const float* pi = base + (int64_t)i * (kD + 2);
          const float mi = __ldcg(pi), li = __ldcg(pi + 1);
          const float2 o01 = __ldcg(reinterpret_cast<const float2*>(pi + 2 + lane * 4));
          const float2 o23 = __ldcg(reinterpret_cast<const float2*>(pi + 4 + lane * 4));
          const float c = (mi == -INFINITY) ? 0.f : fast_exp2(mi - M);
          lsum += li * c;
          acc.x += o01.x * c;
          acc.y += o01.y * c;
          acc.z += o23.x * c;
          acc.w += o23.y * c;
        }
        s_o[warp][lane * 4 + 0] = acc.x;
        s_o[warp][lane * 4 + 1] = acc.y;
        s_o[warp][lane * 4 + 2] = acc.z;
        s_o[warp][lane * 4 + 3] = acc.w;
        if (lane == 0) s_l[warp] = lsum;
        __syncthreads();
        if (tid < kD) {
          float O = 0.f, Lt = 0.f;
#pragma unroll
          for (int w = 0; w < kIWarps; ++w) {
            O += s_o[w][tid];
            Lt += s_l[w];
          }
          outp[tid] = O / Lt;
        }
        if (tid == 0) a.ticket[p] = 0u;
      }
    }
    __syncthreads();
  }
}


// The CTA that owns global key x of the flat list of G CTA ranges [floor(c T / G), floor((c+1) T / G)).
__device__ __forceinline__ int owner_cta(long long x, long long T, int G) {
  return (int)(((x + 1) * (long long)G - 1) / T);
}

// A stage: rows [g0, g1) of the flat list, all inside problem p's list (which starts at `off`).
struct Stage {
  int p;
  long long g0, g1, off;
};

// Walks the stages of a CTA's range [lo, hi) in order: at most kStageKeys rows, never across
// the end of a problem's list.
struct StageWalk {
  int p;
  long long g;
  __device__ __forceinline__ Stage next(const long long* s_off, long long hi) {
    Stage st;
    st.p = p;
    st.g0 = g;
    st.off = s_off[p];
    if (g >= hi) {
      st.g1 = g;  // past the range: an empty stage
      return st;
    }
    const long long pend = s_off[p + 1] < hi ? s_off[p + 1] : hi;
    st.g1 = g + kStageKeys < pend ? g + kStageKeys : pend;
    g = st.g1;
    while (g < hi && s_off[p + 1] <= g) ++p;  // the next non-empty problem
    return st;
  }
};

__global__ void __launch_bounds__(kThreads, 1) decode_gather_kernel(GatherArgs a) {
  extern __shared__ __align__(16) __half s_kv[];  // [kStages][K, V][kStageKeys][kD]
  __shared__ long long s_off[kMaxProblems + 1];  // start of each problem's list in the flat list
  __shared__ int s_kvb[kMaxProblems];            // K/V row block (b * Hkv + g) of each problem
  __shared__ int s_nb[kMaxProblems];             // each problem's sequence length
  __shared__ float s_m[kWarps], s_l[kWarps];
  __shared__ float s_o[kWarps][kD];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hl = lane & 15;
  const int hw = tid >> 4;  // half-warp: copies and consumes rows hw + 32 u of every stage
  const int c = blockIdx.x;

  for (int p = tid; p < a.P; p += kThreads) {
    const int b = p / a.Hr, g = a.ret_head[p % a.Hr] / a.group;
    s_off[p + 1] = a.dense ? (long long)a.lens.v[b] : (long long)a.sel_cnt[p];
    s_kvb[p] = b * a.Hkv + g;
    s_nb[p] = a.lens.v[b];
  }
  __syncthreads();
  if (tid == 0) {
    s_off[0] = 0;
    for (int p = 0; p < a.P; ++p) s_off[p + 1] += s_off[p];
  }
  __syncthreads();
  const long long T = s_off[a.P];
  // CTAs in use: at most one per 32 keys, so every CTA below G has a non-empty range
  const int G = (int)(T / 32 < (long long)gridDim.x ? (T / 32 > 0 ? T / 32 : 1) : gridDim.x);
  if (T == 0 || c >= G) return;  // the whole CTA: no keys of its own
  const long long lo = T * c / G, hi = T * (c + 1) / G;

  // the problem of the first key: the largest p with s_off[p] <= lo (a non-empty one)
  int p0 = 0;
  {
    int ph = a.P - 1;
    while (p0 < ph) {
      const int mid = (p0 + ph + 1) >> 1;
      if (s_off[mid] <= lo) p0 = mid;
      else ph = mid - 1;
    }
  }
  // positions of this thread's rows of stage st (dense: the row numbers themselves)
  auto positions = [&](const Stage& st, int32_t* jv) {
    const int32_t* ids = a.sel_idx + (int64_t)st.p * a.max_select - st.off;
    const long long nb = s_nb[st.p];
#pragma unroll
    for (int u = 0; u < kRowsPerStage; ++u) {
      const long long gr = st.g0 + hw + 32 * u;
      long long j = 0;
      if (gr < st.g1) {
        j = a.dense ? gr - st.off : (long long)__ldg(ids + gr);
        if ((unsigned long long)j >= (unsigned long long)nb) {  // never expected: a stale or corrupt list
          atomicOr(a.err, kErrInternal);
          j = 0;
        }
      }
      jv[u] = (int32_t)j;
    }
  };
  // thread tid copies the 16-byte slice hl of its rows of a stage, K and V
  auto issue = [&](int slot, const Stage& st, const int32_t* jv) {
    if (st.g1 > st.g0) {
      __half* sk = s_kv + (size_t)slot * 2 * kStageKeys * kD + hl * 8;
      __half* sv = sk + kStageKeys * kD;
      const int64_t kvb = (int64_t)s_kvb[st.p] * a.max_seq * kD + hl * 8;
      const __half* kg = a.kc + kvb;
      const __half* vg = a.vc + kvb;
#pragma unroll
      for (int u = 0; u < kRowsPerStage; ++u) {
        const int row = hw + 32 * u;
        if (st.g0 + row < st.g1) {
          cp_async16(sk + row * kD, kg + (int64_t)jv[u] * kD, 16);
          cp_async16(sv + row * kD, vg + (int64_t)jv[u] * kD, 16);
        }
      }
    }
    cp_async_commit();
  };

  // producer: the first kStages - 1 stages, all position loads in flight at once
  StageWalk pw{p0, lo};
  Stage pst[kStages - 1];
  int32_t jp[kStages - 1][kRowsPerStage];
#pragma unroll
  for (int t = 0; t < kStages - 1; ++t) {
    pst[t] = pw.next(s_off, hi);
    positions(pst[t], jp[t]);
  }
  Stage nst = pw.next(s_off, hi);  // the next stage to issue, and its positions
  int32_t jn[kRowsPerStage];
  positions(nst, jn);
#pragma unroll
  for (int t = 0; t < kStages - 1; ++t) issue(t, pst[t], jp[t]);

  // consumer: stages in the same order; a segment is the part of one problem's list in range
  StageWalk cw{p0, lo};
  float q[8], m = -INFINITY, l = 0.f, o[8];
  for (int t = 0;; ++t) {
    const Stage st = cw.next(s_off, hi);
    if (st.g1 <= st.g0) break;  // uniform: every thread walks the same stages
    issue((t + kStages - 1) % kStages, nst, jn);
    nst = pw.next(s_off, hi);
    positions(nst, jn);
    const long long seg_lo = st.off > lo ? st.off : lo;
    const long long seg_hi = s_off[st.p + 1] < hi ? s_off[st.p + 1] : hi;
    const int b = st.p / a.Hr, h = a.ret_head[st.p % a.Hr];
    if (st.g0 == seg_lo) {  // a segment starts: its query, a fresh softmax state
      const float4* qp = reinterpret_cast<const float4*>(a.q_rot + ((int64_t)b * a.Hq + h) * kD + hl * 8);
      const float4 q0 = qp[0], q1 = qp[1];
      q[0] = q0.x; q[1] = q0.y; q[2] = q0.z; q[3] = q0.w;
      q[4] = q1.x; q[5] = q1.y; q[6] = q1.z; q[7] = q1.w;
      m = -INFINITY;
      l = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = 0.f;
    }
    // Each thread reads back exactly the slices it copied itself, so its own wait is enough,
    // and its next copy into this buffer follows its reads.
    cp_async_wait<kStages - 1>();
    {
      const __half* sk = s_kv + (size_t)(t % kStages) * 2 * kStageKeys * kD + hl * 8;
      const __half* sv = sk + kStageKeys * kD;
      // the half-warp's rows of this stage: scores first (independent chains), then one
      // running-max update for all of them
      float sc[kRowsPerStage];
#pragma unroll
      for (int u = 0; u < kRowsPerStage; ++u) {
        float kf[8];
        unpack8(*reinterpret_cast<const uint4*>(sk + (hw + 32 * u) * kD), kf);
        float x0 = q[0] * kf[0], x1 = q[1] * kf[1];
#pragma unroll
        for (int i = 2; i < 8; i += 2) {
          x0 = fmaf(q[i], kf[i], x0);
          x1 = fmaf(q[i + 1], kf[i + 1], x1);
        }
        sc[u] = x0 + x1;
      }
#pragma unroll
      for (int o2 = 8; o2 >= 1; o2 >>= 1)
#pragma unroll
        for (int u = 0; u < kRowsPerStage; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o2);
      float mn = m;
#pragma unroll
      for (int u = 0; u < kRowsPerStage; ++u) {
        sc[u] = (st.g0 + hw + 32 * u < st.g1) ? sc[u] * a.scale_log2 : -INFINITY;
        mn = fmaxf(mn, sc[u]);
      }
      if (mn != -INFINITY) {
        const float corr = fast_exp2(m - mn);
        l *= corr;
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] *= corr;
#pragma unroll
        for (int u = 0; u < kRowsPerStage; ++u) {
          if (sc[u] != -INFINITY) {
            const float w = fast_exp2(sc[u] - mn);
            float vf[8];
            unpack8(*reinterpret_cast<const uint4*>(sv + (hw + 32 * u) * kD), vf);
            l += w;
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = fmaf(w, vf[i], o[i]);
          }
        }
        m = mn;
      }
    }
    if (st.g1 < seg_hi) continue;

    // ---- the segment ends: merge the two half-warps, then the warps
    {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, 16);
      const float l2 = __shfl_xor_sync(0xffffffffu, l, 16);
      const float mx = fmaxf(m, m2);
      const float c1 = (m == -INFINITY) ? 0.f : fast_exp2(m - mx);
      const float c2 = (m2 == -INFINITY) ? 0.f : fast_exp2(m2 - mx);
      l = l * c1 + l2 * c2;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float o2 = __shfl_xor_sync(0xffffffffu, o[i], 16);
        o[i] = o[i] * c1 + o2 * c2;
      }
      m = mx;
    }
    if (lane < 16) {
#pragma unroll
      for (int i = 0; i < 8; ++i) s_o[warp][hl * 8 + i] = o[i];
      if (hl == 0) {
        s_m[warp] = m;
        s_l[warp] = l;
      }
    }
    __syncthreads();
    float cm = -INFINITY, cl = 0.f, co = 0.f;
    if (tid < kD) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) cm = fmaxf(cm, s_m[w]);
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float cw2 = (s_m[w] == -INFINITY) ? 0.f : fast_exp2(s_m[w] - cm);
        cl += s_l[w] * cw2;
        co += s_o[w][tid] * cw2;
      }
    }
    float* outp = a.out + ((int64_t)b * a.Hq + h) * kD;
    const long long p_lo = st.off, p_hi = s_off[st.p + 1];
    if (seg_lo == p_lo && seg_hi == p_hi) {  // the whole list in this CTA
      if (tid < kD) outp[tid] = co / cl;
    } else {
      // partial slots: 2c for a CTA's first segment (the only one that can start inside a
      // list), 2c + 1 for its last (the only other one that can end inside a list)
      const int slot = seg_lo > p_lo ? 2 * c : 2 * c + 1;
      float* pp = a.part + (int64_t)slot * (kD + 2);
      if (tid < kD) pp[2 + tid] = co;
      if (tid == 0) {
        pp[0] = cm;
        pp[1] = cl;
      }
      const int c_first = owner_cta(p_lo, T, G), c_last = owner_cta(p_hi - 1, T, G);
      const int n_seg = c_last - c_first + 1;
      __threadfence();
      __syncthreads();
      if (tid == 0) s_last = (atomicAdd(a.ticket + st.p, 1u) == (uint32_t)(n_seg - 1));
      __syncthreads();
      if (s_last) {
        __threadfence();
        // the partial of segment i (CTA c_first + i) and its slot
        auto part_of = [&](int i) -> const float* {
          const int cc = c_first + i;
          const long long lo_c = T * cc / G;
          return a.part + (int64_t)(lo_c > p_lo ? 2 * cc : 2 * cc + 1) * (kD + 2);
        };
        float mv = -INFINITY;
        for (int i = tid; i < n_seg; i += kThreads) mv = fmaxf(mv, __ldcg(part_of(i)));
        mv = warp_max(mv);
        if (lane == 0) s_m[warp] = mv;
        __syncthreads();
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_m[w]);
        __syncthreads();
        float lsum = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int i = warp; i < n_seg; i += kWarps) {
          const float* pi = part_of(i);
          const float mi = __ldcg(pi), li = __ldcg(pi + 1);
          const float2 o01 = __ldcg(reinterpret_cast<const float2*>(pi + 2 + lane * 4));
          const float2 o23 = __ldcg(reinterpret_cast<const float2*>(pi + 4 + lane * 4));
          const float cc = (mi == -INFINITY) ? 0.f : fast_exp2(mi - M);
          lsum += li * cc;
          acc.x += o01.x * cc;
          acc.y += o01.y * cc;
          acc.z += o23.x * cc;
          acc.w += o23.y * cc;
        }
        s_o[warp][lane * 4 + 0] = acc.x;
        s_o[warp][lane * 4 + 1] = acc.y;
        s_o[warp][lane * 4 + 2] = acc.z;
        s_o[warp][lane * 4 + 3] = acc.w;
        if (lane == 0) s_l[warp] = lsum;
        __syncthreads();
        if (tid < kD) {
          float O = 0.f, Lt = 0.f;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) {
            O += s_o[w][tid];
            Lt += s_l[w];
          }
          outp[tid] = O / Lt;
        }
        if (tid == 0) a.ticket[st.p] = 0u;
      }
    }
    __syncthreads();  // s_o, s_m, s_l are free for the next segment
  }
  cp_async_wait<0>();
}

// p == 1: every causal key is selected.
__global__ void dense_stats_kernel(int32_t* cnt, float* mass, float* thr, int P, int Hr, const SeqPos lens) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p < P) {
    cnt[p] = lens.v[p / Hr];
    mass[p] = 1.0f;
    thr[p] = 0.0f;
  }
}

// dst[r][i] = i for i < min(n_r, cap), n_r the length of row r's sequence: the selected list of
// a p == 1 step.
__global__ void iota_rows_kernel(int32_t* dst, int64_t cap, int Hr, const SeqPos lens) {
  const int64_t n = lens.v[blockIdx.y / Hr];
  const int64_t w = n < cap ? n : cap;
  int32_t* row = dst + (int64_t)blockIdx.y * cap;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < w; i += (int64_t)gridDim.x * blockDim.x)
    row[i] = (int32_t)i;
}

}  // namespace

cudaError_t launch_iota_rows(const rtp_layer* L, int32_t* dst, int64_t cap, cudaStream_t st) {
  iota_rows_kernel<<<dim3(64, L->B * L->Hr), 256, 0, st>>>(dst, cap, L->Hr, seq_pos(L, 0));
  return cudaGetLastError();
}

cudaError_t launch_dense_stats(const rtp_layer* L, cudaStream_t st) {
  const int P = L->B * L->Hr;
  dense_stats_kernel<<<(P + 127) / 128, 128, 0, st>>>(L->sel_cnt, L->sel_mass, L->sel_thr, P, L->Hr, seq_pos(L, 0));
  return cudaGetLastError();
}

cudaError_t launch_decode_gather(const rtp_layer* L, bool dense, bool flat, float* out, cudaStream_t st) {
  GatherArgs a;
  a.kc = L->kc;
  a.vc = L->vc;
  a.max_seq = L->max_seq;
  a.Hkv = L->Hkv;
  a.Hq = L->Hq;
  a.Hr = L->Hr;
  a.group = L->group;
  a.q_rot = L->q_rot;
  a.sel_idx = L->sel_idx;
  a.max_select = L->max_select;
  a.sel_cnt = L->sel_cnt;
  a.ret_head = L->d_ret_head;
  a.P = L->B * L->Hr;
  a.dense = dense ? 1 : 0;
  a.lens = seq_pos(L, 0);
  a.scale_log2 = L->sm_scale * 1.4426950408889634f;
  a.part = L->gpart;
  a.ticket = L->gticket;
  a.err = L->err;
  a.out = out;
  if (a.P > kMaxProblems) return cudaErrorInvalidValue;
  if (!flat) {
    decode_gather_items_kernel<<<4 * L->sm_count, kIThreads, 0, st>>>(a);
    return cudaGetLastError();
  }
  cudaError_t e = cudaFuncSetAttribute(decode_gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kGatherSmem);
  if (e != cudaSuccess) return e;
  decode_gather_kernel<<<L->sm_count, kThreads, kGatherSmem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
