// prefill_local.cu -- local heads in chunked prefill: causal window of W keys plus the first S.
//
// Local heads attend only to nearby tokens and a few attention sinks (techwalker page, section
// 2; section 8: window 8192 with 4 sinks).  Query row i of the chunk sits at position
// pos = len - C + i and sees keys j <= pos with pos - j < W or j < S.
//
// One CTA per (64-row tile, local head, sequence).  The tile's keys -- the sinks, then the
// union of its rows' windows -- stream through a two-stage cp.async pipeline of 64-key K/V
// tiles; attention runs on tensor cores (fa_tile.cuh) with the per-element window mask.
#include "fa_tile.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

struct LocalArgs {
  const __half* kc;
  const __half* vc;
  int64_t max_seq;
  int Hkv, Hq, group, C;
  int64_t P0;  // position of chunk row 0
  int W, S;
  const int16_t* local_heads;  // [n_local]
  const float* q_rot;          // [B][C][Hq][D]
  float scale_log2;
  float* out;                  // [B][C][Hq][D]
};

__global__ void __launch_bounds__(kFaThreads) prefill_local_kernel(LocalArgs a) {
  extern __shared__ __align__(128) unsigned char sm[];
  const int tile = blockIdx.x, b = blockIdx.z;
  const int h = a.local_heads[blockIdx.y], g = h / a.group;
  const int warp = threadIdx.x >> 5;
  const int i0 = tile * kFaRows;
  const int nrows = min(kFaRows, a.C - i0);
  const int64_t pos_min = a.P0 + i0, pos_max = a.P0 + i0 + nrows - 1;
  const int64_t s_cnt = min((int64_t)a.S, pos_max + 1);
  int64_t w_lo = pos_min - a.W + 1;
  if (w_lo < s_cnt) w_lo = s_cnt;
  const int64_t n_keys = s_cnt + (pos_max - w_lo + 1);
  auto pos_of = [&](int64_t u) -> int64_t { return u < s_cnt ? u : w_lo + (u - s_cnt); };

  const __half* kb = a.kc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD;
  const __half* vb = a.vc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD;
  const int64_t qs = (int64_t)a.Hq * kD;
  const float* qbase = a.q_rot + ((int64_t)b * a.C + i0) * qs + (int64_t)h * kD;

  uint32_t qa[8][4];
  fa_load_q(qa, qbase, qs, warp * 16, nrows);
  FaAcc A;
  fa_init(A);

  const int n_tiles = (int)((n_keys + kFaKeys - 1) / kFaKeys);
  auto stage = [&](int t) {
    unsigned char* ks = sm + (t & 1) * 2 * kFaTileBytes;
    const int64_t u0 = (int64_t)t * kFaKeys;
    const int nv = (int)min((int64_t)kFaKeys, n_keys - u0);
    fa_stage(ks, ks + kFaTileBytes, kb, vb, nv, [&](int r) { return pos_of(u0 + r); });
    cp_async_commit();
  };
  stage(0);
  for (int t = 0; t < n_tiles; ++t) {
    if (t + 1 < n_tiles) {
      stage(t + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const unsigned char* ks = sm + (t & 1) * 2 * kFaTileBytes;
    const int64_t u0 = (int64_t)t * kFaKeys;
    auto vis = [&](int r, int tt) {
      const int64_t u = u0 + tt;
      if (r >= nrows || u >= n_keys) return false;
      const int64_t j = pos_of(u), pos = pos_min + r;
      return j <= pos && (j < a.S || pos - j < a.W);
    };
    // a tile whose keys every row of the CTA sees needs no mask: a full tile of one segment
    // (sinks or window), with its last key at or before the first row and, for window keys,
    // its first key inside the last row's window
    bool full = false;
    if (nrows == kFaRows && u0 + kFaKeys <= n_keys) {
      const int64_t j_lo = pos_of(u0), j_hi = pos_of(u0 + kFaKeys - 1);
      const bool one_seg = (u0 + kFaKeys <= s_cnt) || (u0 >= s_cnt);
      full = one_seg && j_hi <= pos_min && (j_hi < a.S || pos_max - j_lo < a.W);
    }
    if (full) fa_tile<false>(A, qa, ks, ks + kFaTileBytes, a.scale_log2, vis);
    else fa_tile<true>(A, qa, ks, ks + kFaTileBytes, a.scale_log2, vis);
    __syncthreads();
  }
  float* obase = a.out + ((int64_t)b * a.C + i0) * qs + (int64_t)h * kD;
  fa_store(A, obase, qs, warp * 16, nrows);
}

}  // namespace

cudaError_t launch_prefill_local(const rtp_layer* L, int C, float* out, cudaStream_t st) {
  LocalArgs a;
  a.kc = L->kc;
  a.vc = L->vc;
  a.max_seq = L->max_seq;
  a.Hkv = L->Hkv;
  a.Hq = L->Hq;
  a.group = L->group;
  a.C = C;
  a.P0 = L->len - C;
  a.W = L->W;
  a.S = L->S;
  a.local_heads = L->d_local_list;
  a.q_rot = L->q_rot;
  a.scale_log2 = L->sm_scale * 1.4426950408889634f;
  a.out = out;
  const size_t smem = 4 * (size_t)kFaTileBytes;  // two stages of K and V
  cudaError_t e = cudaFuncSetAttribute(prefill_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((C + kFaRows - 1) / kFaRows, L->n_local, L->B);
  prefill_local_kernel<<<grid, kFaThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
