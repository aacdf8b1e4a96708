// decode_gather.cu -- exact attention of one decode query over its selected keys.
//
// Retrieval heads attend, in the full head dim, to the keys their top-p selection kept
// (techwalker page, section 3: "full 128-dim exact computation on the selected tokens";
// section 6: the sparse-KV kernel splits long selections across CTAs and the last CTA to
// finish merges the results).
//
// B200 design
//   * Work items are (problem, chunk of kGatherChunk selected positions), enumerated on the
//     device from the selection counts, so one persistent grid covers any mix of 2..10^5
//     selected keys without a host round trip.
//   * A half-warp owns one key row: 16 lanes x 16 bytes = one 256-byte fp16 K row (and V
//     row), loaded with 16-byte vector loads, all rows of the lane's share issued before any
//     math so every lane has 256 bytes in flight.  Scores and the running softmax stay in
//     fp32 registers; the query stays fp32 (no rounding of q).
//   * Partials (m, l, o[128]) of the items of one problem are merged in item order by the
//     CTA that takes the last ticket (deterministic, no waiting), which also resets the
//     ticket for the next call.
#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr int kChunk = kGatherChunk;
constexpr int kThreads = kGatherThreads;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerHalf = kChunk / (2 * kWarps);  // rows per half-warp per item
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

__global__ void __launch_bounds__(kThreads) decode_gather_kernel(GatherArgs a) {
  __shared__ int s_base[kMaxProblems + 1];
  __shared__ float s_m[kWarps], s_l[kWarps];
  __shared__ float s_o[kWarps][kD];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, hl = lane & 15;

  // item prefix over problems: counts loaded in parallel, summed by one thread from smem
  for (int p = tid; p < a.P; p += kThreads) {
    const int64_t K = a.dense ? (int64_t)a.lens.v[p / a.Hr] : (int64_t)a.sel_cnt[p];
    s_base[p + 1] = (int)((K + kChunk - 1) / kChunk);
  }
  __syncthreads();
  if (tid == 0) {
    s_base[0] = 0;
    for (int p = 0; p < a.P; ++p) s_base[p + 1] += s_base[p];
  }
  __syncthreads();
  const int total_items = s_base[a.P];

  for (int it = blockIdx.x; it < total_items; it += gridDim.x) {
    // locate the problem of this item (P is small; linear search over the prefix)
    int p = 0;
    while (p + 1 < a.P && s_base[p + 1] <= it) ++p;
    const int chunk = it - s_base[p];
    const int n_items = s_base[p + 1] - s_base[p];
    const int b = p / a.Hr, hr = p % a.Hr;
    const int h = a.ret_head[hr], g = h / a.group;
    const int64_t Nb = a.lens.v[b];  // this sequence's keys
    const int64_t K = a.dense ? Nb : (int64_t)a.sel_cnt[p];
    const int64_t r_lo = (int64_t)chunk * kChunk;
    const int64_t r_hi = min(K, r_lo + kChunk);

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
    // rows of this half-warp: r_lo + (warp * 2 + half) + 16 * u
    uint4 kr[kRowsPerHalf], vr[kRowsPerHalf];
#pragma unroll
    for (int u = 0; u < kRowsPerHalf; ++u) {
      const int64_t r = r_lo + (warp * 2 + half) + 2 * kWarps * u;
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
    float m = -INFINITY, l = 0.f, o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = 0.f;
#pragma unroll
    for (int u = 0; u < kRowsPerHalf; ++u) {
      const int64_t r = r_lo + (warp * 2 + half) + 2 * kWarps * u;
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
      for (int w = 0; w < kWarps; ++w) cm = fmaxf(cm, s_m[w]);
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
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
        for (int i = tid; i < n_items; i += kThreads) mv = fmaxf(mv, __ldcg(base + (int64_t)i * (kD + 2)));
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
        for (int i = warp; i < n_items; i += kWarps) {
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
          for (int w = 0; w < kWarps; ++w) {
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

cudaError_t launch_decode_gather(const rtp_layer* L, bool dense, float* out, cudaStream_t st) {
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
  const int grid = 4 * L->sm_count;
  decode_gather_kernel<<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
