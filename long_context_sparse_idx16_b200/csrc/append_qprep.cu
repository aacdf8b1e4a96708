// append_qprep.cu -- K/V append with RoPE and 16-dim index keys; query preparation.
//
// Append (rtp_append_kv): for each new token at position pos and KV head g,
//   K[g][pos] = fp16(RoPE(k, pos)), V[g][pos] = fp16(v), and for every retrieval head h
//   whose KV head is g: IDX[h][pos] = Wk_h^T k (pre-RoPE; stored in fp32, or in bf16 when the
//   layer keeps bf16 index keys), also kept split as fp16 hi + lo for the tensor-core scoring
//   of prefill.
// The indexer projects pre-RoPE keys (ngjoo digest, core method: "low-dimensional pre-RoPE
// projections"; aitntnews page, finding 2: project D=128 down to r=16 so that the
// high-frequency RoPE components do not disturb long-range matching).
//
// Query prep: q_rot = RoPE(q, pos) in fp32 and q_idx = Wq_h^T q (pre-RoPE) for retrieval heads.
//
// RoPE is the rotate-half form: pair (c, c + D/2) turns by pos * base^(-2c/D).  The angle is
// formed and reduced in fp64 (pos reaches 2^20, where an fp32 angle is off by ~0.06 rad),
// then the rotation runs in fp32.
#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr float kFp16Max = 65504.f;

// Append work split: blockIdx.z == 0 writes RoPE(k) and v of up to kAppTok tokens; blockIdx.z
// == 1 + hr computes retrieval head hr's index keys of the same tokens (its 8 KB of weights
// read once for the group).  A one-token decode append is 1 + Hr small CTAs per sequence, all
// in flight at once.
constexpr int kAppThreads = 128;
constexpr int kAppTok = 8;

template <bool kBf16>
__global__ void __launch_bounds__(kAppThreads) append_kv_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, int T, int Hkv,
    int Hr, const SeqPos pos0, int b0, int64_t max_seq, const double* __restrict__ theta,
    const float* __restrict__ wk, const int16_t* __restrict__ ret_head, int group,
    __half* __restrict__ kc, __half* __restrict__ vc, float* __restrict__ idx, __nv_bfloat16* __restrict__ idx_b,
    __half* __restrict__ idx_hl, uint32_t* __restrict__ err) {
  // bl: the sequence's slot in this call's k / v; b: its index in the layer (caches, positions)
  const int t0 = blockIdx.x * kAppTok, bl = blockIdx.y, b = b0 + bl, role = blockIdx.z;
  const int nt = min(kAppTok, T - t0);
  const int tid = threadIdx.x;
  if (role == 0) {
    // ---- K (RoPE'd) and V rows into the fp16 cache
    __shared__ float cs[kHalfD], sn[kHalfD];
    bool bad = false;
    for (int u = 0; u < nt; ++u) {
      const int t = t0 + u;
      const int64_t pos = (int64_t)pos0.v[b] + t;
      __syncthreads();  // the previous token's angles are consumed
      if (tid < kHalfD) rope_cos_sin(pos, theta[tid], &cs[tid], &sn[tid]);
      __syncthreads();
      const __nv_bfloat16* kt = k + ((int64_t)bl * T + t) * Hkv * kD;
      const __nv_bfloat16* vt = v + ((int64_t)bl * T + t) * Hkv * kD;
      for (int i = tid; i < Hkv * kD; i += kAppThreads) {
        const int g = i / kD, d = i % kD;
        const float x = __bfloat162float(vt[i]);
        bad |= !(fabsf(x) <= kFp16Max);
        vc[(((int64_t)b * Hkv + g) * max_seq + pos) * kD + d] = __float2half_rn(x);
      }
      for (int i = tid; i < Hkv * kHalfD; i += kAppThreads) {
        const int g = i / kHalfD, c = i % kHalfD;
        const float x0 = __bfloat162float(kt[g * kD + c]), x1 = __bfloat162float(kt[g * kD + c + kHalfD]);
        const float y0 = x0 * cs[c] - x1 * sn[c];
        const float y1 = x1 * cs[c] + x0 * sn[c];
        bad |= !(fabsf(y0) <= kFp16Max) || !(fabsf(y1) <= kFp16Max);
        __half* dst = kc + (((int64_t)b * Hkv + g) * max_seq + pos) * kD;
        dst[c] = __float2half_rn(y0);
        dst[c + kHalfD] = __float2half_rn(y1);
      }
    }
    if (bad) atomicOr(err, kErrRange);
    return;
  }
  // ---- index keys of retrieval head hr: 16 outputs x 8 partial sums of 16 dims, a fixed
  // order (then a 3-step shuffle tree) so every append gives the same bits
  const int hr = role - 1;
  const int o = tid >> 3, part = tid & 7;
  const int g = ret_head[hr] / group;
  float w[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) w[e] = wk[((int64_t)hr * kD + part * 16 + e) * kR + o];
  for (int u = 0; u < nt; ++u) {
    const int t = t0 + u;
    const int64_t pos = (int64_t)pos0.v[b] + t;
    const __nv_bfloat16* kt = k + (((int64_t)bl * T + t) * Hkv + g) * kD + part * 16;
    float x[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) x[e] = __bfloat162float(kt[e]);
    const int64_t row = ((int64_t)b * Hr + hr) * max_seq + pos;
    float acc;
    if (kBf16) {
      // bf16 storage: the projection in fp64, then one rounding to the nearest bf16 (even on
      // ties), so the stored key is the exact projection's bf16 rounding
      double a64 = 0.0;
#pragma unroll
      for (int e = 0; e < 16; ++e) a64 = fma((double)w[e], (double)x[e], a64);
      a64 += __shfl_xor_sync(0xffffffffu, a64, 1);
      a64 += __shfl_xor_sync(0xffffffffu, a64, 2);
      a64 += __shfl_xor_sync(0xffffffffu, a64, 4);
      const __nv_bfloat16 kb = __double2bfloat16(a64);
      if (part == 0) idx_b[row * kR + o] = kb;
      acc = __bfloat162float(kb);
    } else {
      acc = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) acc = fmaf(w[e], x[e], acc);
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (part == 0) idx[row * kR + o] = acc;
    }
    if (part == 0) {  // the same key split as fp16 hi + lo, for the tensor-core scoring of prefill
      const __half hh = __float2half_rn(acc);
      idx_hl[row * (2 * kR) + o] = hh;
      idx_hl[row * (2 * kR) + kR + o] = __float2half_rn(acc - __half2float(hh));
    }
  }
}

// One CTA per (row, batch, group of kQHeads heads): RoPE'd fp32 query for each head, and the
// pre-RoPE index query Wq_h^T q for the retrieval heads among them.
constexpr int kQHeads = 4;

__global__ void __launch_bounds__(128) q_prep_kernel(
    const __nv_bfloat16* __restrict__ q, int rows, int Hq, int Hr, const SeqPos pos0,
    const double* __restrict__ theta, const float* __restrict__ wq,
    const int16_t* __restrict__ head_slot, float* __restrict__ q_rot, float* __restrict__ q_idx) {
  const int i = blockIdx.x, b = blockIdx.y, h0 = blockIdx.z * kQHeads;
  const int64_t pos = (int64_t)pos0.v[b] + i;  // row i of sequence b
  const int d = threadIdx.x;
  __shared__ float cs[kHalfD], sn[kHalfD];
  __shared__ float qs[kQHeads][kD];
  const int64_t row = (int64_t)b * rows + i;
  const __nv_bfloat16* qr = q + row * Hq * kD;
  float x[kQHeads], xp[kQHeads];
#pragma unroll
  for (int u = 0; u < kQHeads; ++u) {
    const int h = h0 + u;
    x[u] = h < Hq ? __bfloat162float(qr[h * kD + d]) : 0.f;
    xp[u] = h < Hq ? __bfloat162float(qr[h * kD + (d ^ kHalfD)]) : 0.f;
  }
  // this thread's index weights (16 dims of one output per retrieval head), read together with
  // q so the kernel waits on memory once
  const int o = d >> 3, part = d & 7;
  int hrs[kQHeads];
  float wv[kQHeads][16];
#pragma unroll
  for (int u = 0; u < kQHeads; ++u) {
    const int h = h0 + u;
    hrs[u] = h < Hq ? head_slot[h] : -1;
    const float* w = wq + (int64_t)(hrs[u] < 0 ? 0 : hrs[u]) * kD * kR + o;
#pragma unroll
    for (int e = 0; e < 16; ++e) wv[u][e] = hrs[u] < 0 ? 0.f : w[(part * 16 + e) * kR];
  }
  if (d < kHalfD) rope_cos_sin(pos, theta[d], &cs[d], &sn[d]);
#pragma unroll
  for (int u = 0; u < kQHeads; ++u) qs[u][d] = x[u];
  __syncthreads();
  const int c = d & (kHalfD - 1);
#pragma unroll
  for (int u = 0; u < kQHeads; ++u) {
    const int h = h0 + u;
    if (h >= Hq) break;
    // first half: x*cos - partner*sin; second half: x*cos + partner*sin
    const float y = d < kHalfD ? x[u] * cs[c] - xp[u] * sn[c] : x[u] * cs[c] + xp[u] * sn[c];
    q_rot[(row * Hq + h) * kD + d] = y;
  }
  // index queries: 16 outputs x 8 partial sums of 16 dims each
#pragma unroll
  for (int u = 0; u < kQHeads; ++u) {
    const int hr = hrs[u];
    if (hr < 0) continue;  // uniform over the CTA: the head (or its absence) is blockIdx-derived
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) acc = fmaf(wv[u][e], qs[u][part * 16 + e], acc);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (part == 0) q_idx[(row * Hr + hr) * kR + o] = acc;
  }
}

}  // namespace

SeqPos seq_pos(const rtp_layer* L, int64_t delta) {
  SeqPos s{};
  for (int b = 0; b < L->B; ++b) s.v[b] = (int32_t)(L->lens[b] + delta);
  return s;
}

cudaError_t launch_append_kv(const rtp_layer* L, const __nv_bfloat16* k, const __nv_bfloat16* v, int T, int b0,
                             int nb, cudaStream_t st) {
  dim3 grid((T + kAppTok - 1) / kAppTok, nb, 1 + L->Hr);
  auto fn = L->index_bf16 ? append_kv_kernel<true> : append_kv_kernel<false>;
  fn<<<grid, kAppThreads, 0, st>>>(k, v, T, L->Hkv, L->Hr, seq_pos(L, 0), b0, L->max_seq, L->theta, L->wk,
                                   L->d_ret_head, L->group, L->kc, L->vc, L->idx, L->idx_b, L->idx_hl, L->err);
  return cudaGetLastError();
}

cudaError_t launch_q_prep(const rtp_layer* L, const __nv_bfloat16* q, int rows, const SeqPos& pos0,
                          cudaStream_t st) {
  dim3 grid(rows, L->B, (L->Hq + kQHeads - 1) / kQHeads);
  q_prep_kernel<<<grid, 128, 0, st>>>(q, rows, L->Hq, L->Hr, pos0, L->theta, L->wq, L->d_head_slot,
                                      L->q_rot, L->q_idx);
  return cudaGetLastError();
}

}  // namespace rtp
