// prefill_local_tc.cu -- local heads in chunked prefill on 5th-generation tensor cores (and
// the retrieval heads too, with a window covering every causal key, when the layer runs the
// pages' own dense prefill for them).
//
// Local heads attend only to nearby tokens and a few attention sinks (techwalker page, section
// 2; section 8: window 8192 with 4 sinks).  Query row i of the chunk sits at position
// pos = len - C + i and sees keys j <= pos with pos - j < W or j < S.
//
// One CTA per (128-row tile, local head, sequence), 256 threads: query row r is TMEM lane r,
// served by threads r (columns 0..31 of each step's S, output columns 0..63) and r + 128 (the
// other halves), which share the row max through shared memory.  The tile's keys -- the sinks, then the union of its rows' windows -- are
// taken in 64-key steps t, software-pipelined so the tensor cores, the copies and the softmax
// overlap:
//   * K and V rows go through two 128-byte-swizzled slots each (cp.async): K of step t + 2
//     loads once S_t is done, V of step t + 1 once P_{t-1} V_{t-1} is done;
//   * S_t = Q K_t^T (tcgen05.mma, M 128, N 64, K 16 per instruction, Q and K from shared
//     memory) lands in one of two TMEM buffers; S_{t+1} is issued before the softmax of S_t;
//   * each thread reads its row of S_t from TMEM, applies the window mask and forms
//     P = exp2(S - m) in fp16 (one P buffer) against a reference max m that only moves when
//     the row max exceeds it by more than 11 (in log2 units): then the running sum and, in the
//     warps concerned, the output accumulator in TMEM are rescaled (this bounds P by 2^11);
//   * O += P_t V_t (tcgen05.mma, M 128, N 128, V read as an MN-major operand) accumulates in
//     TMEM across all steps and is read once at the end.
// Completions are tracked with mbarriers (tcgen05.commit); every wait is bounded, and on
// timeout the error word is set and the CTA leaves after freeing its TMEM.
#include "rtp_internal.h"
#include "tc_umma.cuh"

namespace rtp {

namespace {

constexpr int kRowsT = 128;   // query rows per CTA (= TMEM lanes)
constexpr int kKeysT = 64;    // keys per step
constexpr int kThreadsT = 256;   // two threads per row, each on half the columns
constexpr uint32_t kTmemCols = 256;  // S0 [0,64), S1 [64,128), O [128,256)
constexpr float kRescale = 11.f;     // log2 headroom before the reference max moves (P <= 2^11)
constexpr uint32_t kQBytes = kRowsT * 256;   // 32 KB
constexpr uint32_t kKVBytes = kKeysT * 256;  // 16 KB per K or V tile
constexpr uint32_t kPBytes = kRowsT * 128;   // 16 KB
// layout: Q | K x 2 | V x 2 | P | mbarriers (S0, S1, O0, O1), TMEM base -- under 113 KB, so
// two CTAs share an SM
constexpr uint32_t kOffK = kQBytes;
constexpr uint32_t kOffV = kOffK + 2 * kKVBytes;
constexpr uint32_t kOffP = kOffV + 2 * kKVBytes;
constexpr uint32_t kOffBar = kOffP + kPBytes;
constexpr uint32_t kSmemT = kOffBar + 48;

__device__ __forceinline__ uint32_t pack_half2_tc(float x, float y) {
  __half2 h = __floats2half2_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&h);
}

struct LocalTcArgs {
  const __half* kc;
  const __half* vc;
  int64_t max_seq;
  int Hkv, Hq, group, C;
  SeqPos P0;  // per sequence: position of chunk row 0
  int W, S;
  const int16_t* local_heads;
  const float* q_rot;  // [B][C][Hq][D]
  float scale_log2;
  float* out;          // [B][C][Hq][D]
  uint32_t* err;
};

__global__ void __launch_bounds__(kThreadsT, 2) prefill_local_tc_kernel(LocalTcArgs a) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const uint32_t sbase = smem_u32(sm);
  const uint32_t barS0 = sbase + kOffBar, barO0 = barS0 + 16;  // barS[i] = barS0 + 8i, barO likewise
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffBar + 32);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int half = tid >> 7, r = tid & (kRowsT - 1);  // row r, S columns [32 half, 32 half + 32)
  const int tile = blockIdx.x, b = blockIdx.z;
  const int h = a.local_heads[blockIdx.y], g = h / a.group;
  const int i0 = tile * kRowsT;
  const int nrows = min(kRowsT, a.C - i0);
  const int64_t pos_min = (int64_t)a.P0.v[b] + i0, pos_max = pos_min + nrows - 1;
  const int64_t s_cnt = min((int64_t)a.S, pos_max + 1);
  int64_t w_lo = pos_min - a.W + 1;
  if (w_lo < s_cnt) w_lo = s_cnt;
  const int64_t n_keys = s_cnt + (pos_max - w_lo + 1);
  auto pos_of = [&](int64_t u) -> int64_t { return u < s_cnt ? u : w_lo + (u - s_cnt); };
  const __half* kb = a.kc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD;
  const __half* vb = a.vc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD;
  const int64_t qs = (int64_t)a.Hq * kD;
  const bool live = r < nrows;
  const int64_t pos = pos_min + r;

  // the swizzle is a function of address bits: the tiles must sit on 1024-byte boundaries
  if (sbase & 1023u) {
    if (tid == 0) atomicOr(a.err, kErrInternal);
    return;
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(barS0 + 8 * i, 1);
  }

  // query row r as fp16 into the swizzled Q tile (zero rows past the chunk); each half writes
  // eight of the row's sixteen 16-byte chunks
  {
    const float* qrow = a.q_rot + ((int64_t)b * a.C + i0 + (live ? r : 0)) * qs + (int64_t)h * kD;
#pragma unroll 4
    for (int cc = 0; cc < 8; ++cc) {
      const int c = 8 * half + cc;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (live) {
        const float4 x0 = *reinterpret_cast<const float4*>(qrow + 8 * c);
        const float4 x1 = *reinterpret_cast<const float4*>(qrow + 8 * c + 4);
        v.x = pack_half2_tc(x0.x, x0.y);
        v.y = pack_half2_tc(x0.z, x0.w);
        v.z = pack_half2_tc(x1.x, x1.y);
        v.w = pack_half2_tc(x1.z, x1.w);
      }
      *reinterpret_cast<uint4*>(sm + sw128_off(r, c, kRowsT)) = v;
    }
  }

  const int n_steps = (int)((n_keys + kKeysT - 1) / kKeysT);
  // K rows of step t into K slot t % 2, V rows into V slot t % 2; each call commits one group
  auto stage_k = [&](int t) {
    if (t < n_steps) {
      const int64_t u0 = (int64_t)t * kKeysT;
      unsigned char* dst = sm + kOffK + (t & 1) * kKVBytes;
#pragma unroll
      for (int i = 0; i < (kKeysT * 16) / kThreadsT; ++i) {
        const int idx = i * kThreadsT + tid;
        const int key = idx >> 4, c = idx & 15;
        const int64_t u = u0 + key;
        const bool ok = u < n_keys;
        cp_async16(dst + sw128_off(key, c, kKeysT), kb + (ok ? pos_of(u) : 0) * kD + c * 8, ok ? 16 : 0);
      }
    }
    cp_async_commit();
  };
  auto stage_v = [&](int t) {
    if (t < n_steps) {
      const int64_t u0 = (int64_t)t * kKeysT;
      unsigned char* dst = sm + kOffV + (t & 1) * kKVBytes;
#pragma unroll
      for (int i = 0; i < (kKeysT * 16) / kThreadsT; ++i) {
        const int idx = i * kThreadsT + tid;
        const int key = idx >> 4, c = idx & 15;
        const int64_t u = u0 + key;
        const bool ok = u < n_keys;
        cp_async16(dst + sw128_off(key, c, kKeysT), vb + (ok ? pos_of(u) : 0) * kD + c * 8, ok ? 16 : 0);
      }
    }
    cp_async_commit();
  };
  constexpr uint32_t kIdS = umma_idesc_f16(kKeysT, false);
  constexpr uint32_t kIdO = umma_idesc_f16(kD, true);
  auto issue_s = [&](uint32_t tmem, int t) {  // S_t = Q K_t^T into TMEM buffer t & 1 (one thread)
    tc_fence_after();
    const uint32_t k0 = sbase + kOffK + (t & 1) * kKVBytes;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      const uint64_t ad = umma_desc(sbase + (kk >> 2) * (kRowsT * 128) + (kk & 3) * 32, 16, 1024);
      const uint64_t bd = umma_desc(k0 + (kk >> 2) * (kKeysT * 128) + (kk & 3) * 32, 16, 1024);
      umma_f16(tmem + (uint32_t)((t & 1) * kKeysT), ad, bd, kIdS, kk > 0 ? 1u : 0u);
    }
    umma_commit(barS0 + 8 * (t & 1));
  };
  // clamp a column bound (relative to the step) into [-1, kKeysT]
  auto cl = [](int64_t v) -> int { return (int)max((int64_t)-1, min((int64_t)kKeysT, v)); };
  // group order: K(0), K(1), V(0), then per step t: K(t + 2), V(t + 1)
  stage_k(0);
  stage_k(1);
  stage_v(0);
  cp_async_wait<1>();  // K(0), K(1) landed
  fence_async_smem();
  __syncthreads();  // Q and K(0) in shared memory, mbarriers initialised, TMEM base written
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_base_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  // exchange one float per row between the two halves through TMEM: half h writes column
  // col + 32 h of its lane (a column it has already read), then reads the partner's
  auto swap_half = [&](uint32_t col, float v) -> float {
    float w[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i] = v;
    tmem_st32(tmem_base_lane + col + 32u * half, w);
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem_ld32(tmem_base_lane + col + 32u * (1 - half), w);
    tmem_ld_wait();
    return w[0];
  };

  if (tid == 0) issue_s(tmem, 0);

  float m_ref = -INFINITY, l = 0.f;  // reference max of row r; this half's share of the sum
  bool ok = true, okw = true;
  for (int t = 0; t < n_steps; ++t) {
    // ---- S_{t+1} = Q K_{t+1}^T (K_{t+1} landed one step ago; its TMEM buffer was last read by
    // the softmax of t - 1)
    if (t + 1 < n_steps) {
      if (t > 0) {
        cp_async_wait<1>();  // everything but V(t)
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
      }
      if (tid == 0) issue_s(tmem, t + 1);
    }
    // ---- this half's 32 columns of S_t, masked to the row's sinks and window
    okw = mbar_wait(barS0 + 8 * (t & 1), (uint32_t)(t >> 1) & 1u) && okw;
    tc_fence_after();
    const uint32_t sCol = (uint32_t)((t & 1) * kKeysT);
    float sv[32];
    tmem_ld32(tmem_base_lane + sCol + 32u * half, sv);
    tmem_ld_wait();
    stage_k(t + 2);  // K slot t % 2 is free: S_t has completed
    const int64_t u0 = (int64_t)t * kKeysT;
    // column c (of the step) is visible iff c <= s_hi (a sink) or w_a <= c <= w_b and
    // (c <= d_hi or c >= e_lo) (a window key j = c + base: causal, in the cache, and a sink
    // position or within W of the row)
    int s_hi = -1, w_a = kKeysT, w_b = -1, d_hi = -1, e_lo = kKeysT;
    if (live) {
      const int64_t sink_end = s_cnt - u0;
      const int64_t base = w_lo - s_cnt + u0;
      s_hi = cl(min(sink_end - 1, pos - u0));
      w_a = cl(sink_end);
      w_b = cl(min(pos - base, n_keys - 1 - u0));
      d_hi = cl((int64_t)a.S - 1 - base);
      e_lo = cl(pos - a.W + 1 - base);
    }
    // a step whose keys every row of the CTA sees (one segment, last key at or before the
    // first row, first key inside the last row's window) needs no mask
    bool full = false;
    if (nrows == kRowsT && u0 + kKeysT <= n_keys) {
      const int64_t j_lo = pos_of(u0), j_hi = pos_of(u0 + kKeysT - 1);
      const bool one_seg = (u0 + kKeysT <= s_cnt) || (u0 >= s_cnt);
      full = one_seg && j_hi <= pos_min && (j_hi < a.S || pos_max - j_lo < a.W);
    }
    float mx = -INFINITY;
    if (full) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        sv[i] *= a.scale_log2;
        mx = fmaxf(mx, sv[i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int c = 32 * half + i;
        const bool vis = c <= s_hi || (c >= w_a && c <= w_b && (c <= d_hi || c >= e_lo));
        sv[i] = vis ? sv[i] * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, sv[i]);
      }
    }
    mx = fmaxf(mx, swap_half(sCol, mx));  // the row max over both halves
    // the reference max moves only when the row max exceeds it by more than kRescale
    const bool move = mx > m_ref + kRescale;
    // P V of step t - 1 must be done before P is rewritten (and before a rescale)
    if (t >= 1) okw = mbar_wait(barO0 + 8 * ((t - 1) & 1), (uint32_t)((t - 1) >> 1) & 1u) && okw;
    tc_fence_after();
    if (t > 0 && __any_sync(0xffffffffu, move)) {
      const float cf = move ? fast_exp2(m_ref - mx) : 1.f;  // warp-collective ld / st below
      const uint32_t oAddr = tmem_base_lane + 128u + 64u * half;
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
    // ---- P_t (this half's four 16-byte chunks)
    float rs = 0.f;
    unsigned char* pbuf = sm + kOffP;
    // a row with no visible key yet has m_ref = -inf and only -inf scores: exp2(-inf - 0) = 0
    const float mref = m_ref == -INFINITY ? 0.f : m_ref;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float pv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        pv[e] = fast_exp2(sv[8 * q + e] - mref);
        rs += pv[e];
      }
      uint4 w;
      w.x = pack_half2_tc(pv[0], pv[1]);
      w.y = pack_half2_tc(pv[2], pv[3]);
      w.z = pack_half2_tc(pv[4], pv[5]);
      w.w = pack_half2_tc(pv[6], pv[7]);
      *reinterpret_cast<uint4*>(pbuf + sw128_off(r, 4 * half + q, kRowsT)) = w;
    }
    l += rs;
    cp_async_wait<1>();  // V(t) landed (K(t + 2) may still be in flight)
    fence_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(okw);
    if (!ok) break;
    // ---- O += P_t V_t (one thread); V is read MN-major (rows = keys)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t v0 = sbase + kOffV + (t & 1) * kKVBytes;
      const uint32_t p0 = sbase + kOffP;
#pragma unroll
      for (int kk = 0; kk < kKeysT / 16; ++kk) {
        const uint64_t ad = umma_desc(p0 + kk * 32, 16, 1024);
        const uint64_t bd = umma_desc(v0 + kk * 2048, kKeysT * 128, 1024);
        umma_f16(tmem + 128u, ad, bd, kIdO, (t > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(barO0 + 8 * (t & 1));
    }
    stage_v(t + 1);  // V slot (t + 1) % 2 held V(t - 1), whose P V is done
  }

  if (ok) {
    const int tl = n_steps - 1;
    okw = mbar_wait(barO0 + 8 * (tl & 1), (uint32_t)(tl >> 1) & 1u) && okw;
    ok = __syncthreads_and(okw);
  }
  if (ok) {
    tc_fence_after();
    const float lt = l + swap_half(0u, l);  // S buffer 0 is free now
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    float* orow = a.out + ((int64_t)b * a.C + i0 + (live ? r : 0)) * qs + (int64_t)h * kD + 64 * half;
    const uint32_t oAddr = tmem_base_lane + 128u + 64u * half;
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 32) {
      float ov[32];
      tmem_ld32(oAddr + c0, ov);
      tmem_ld_wait();
      if (live) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(orow + c0 + i) =
              make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
      }
    }
  } else if (tid == 0) {
    atomicOr(a.err, kErrTimeout);
  }
  cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_free(tmem, kTmemCols);
  }
}

}  // namespace

// The kernel over a list of heads with a given window and sink count: the local heads, or (the
// pages' own prefill) the retrieval heads with a window that covers every causal key.
static cudaError_t launch_prefill_heads(const rtp_layer* L, int C, float* out, cudaStream_t st,
                                        const int16_t* heads, int n_heads, int W, int S) {
  LocalTcArgs a;
  a.kc = L->kc;
  a.vc = L->vc;
  a.max_seq = L->max_seq;
  a.Hkv = L->Hkv;
  a.Hq = L->Hq;
  a.group = L->group;
  a.C = C;
  a.P0 = seq_pos(L, -C);
  a.W = W;
  a.S = S;
  a.local_heads = heads;
  a.q_rot = L->q_rot;
  a.scale_log2 = L->sm_scale * 1.4426950408889634f;
  a.out = out;
  a.err = L->err;
  cudaError_t e = cudaFuncSetAttribute(prefill_local_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemT);
  if (e != cudaSuccess) return e;
  dim3 grid((C + kRowsT - 1) / kRowsT, n_heads, L->B);
  prefill_local_tc_kernel<<<grid, kThreadsT, kSmemT, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_prefill_local(const rtp_layer* L, int C, float* out, cudaStream_t st) {
  return launch_prefill_heads(L, C, out, st, L->d_local_list, L->n_local, L->W, L->S);
}

cudaError_t launch_prefill_dense_retrieval(const rtp_layer* L, int C, float* out, cudaStream_t st) {
  const int W = L->len < (int64_t)0x7FFFFFFF ? (int)L->len : 0x7FFFFFFF;  // every causal key
  return launch_prefill_heads(L, C, out, st, L->d_ret_head, L->Hr, W, 0);
}

}  // namespace rtp
