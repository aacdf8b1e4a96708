// index_mma.cuh -- 16-dim index scores of 64 query rows x 64 keys on tensor cores.
//
// The retrieval-head indexer scores s_j = qidx . kidx_j (techwalker page, section 3; 16 dims,
// aitntnews page, finding 3) for every (row, causal key) pair of a prefill chunk.  The fp32
// operands are split into fp16 hi + lo parts (x = hi + lo to about 22 bits) and the score is
// hi.hi + hi.lo + lo.hi, three m16n8k16 MMAs with fp32 accumulation -- about fp32 accuracy.
// The same instruction sequence on the same inputs gives the same bits, so every selection
// pass and the attention mask see identical scores.
//
// Layout (4 warps, 128 threads): warp w owns rows 16w .. 16w+15; a thread (gr = lane / 4,
// tq = lane % 4) holds rows 16w+gr (slot 0) and 16w+gr+8 (slot 1) and, of every 8-key group nt,
// keys 8nt + 2tq and 8nt + 2tq + 1:  c[nt][e] is slot 0, c[nt][2+e] slot 1.
#pragma once

#include "mma_tile.cuh"
#include "rtp_device.cuh"

namespace rtp {

constexpr int kIdxKeys = 64;     // keys per tile
constexpr int kIdxThreads = 128;
constexpr int kIdxStages = 3;    // index tiles in flight

// Ring of index-key tiles in shared memory, copied straight from the split index cache
// ([key][hi 16 | lo 16] fp16, 64 bytes per key): per stage a hi and a lo tile of 64 keys x 16
// dims, 32-byte rows with swizzled 16-byte chunks (4 KB per stage).
struct IdxRing {
  __half t[kIdxStages][2][kIdxKeys * kR];
};

// byte offset of 16-byte chunk ch (0: dims 0..7, 1: dims 8..15) of key row r
__device__ __forceinline__ uint32_t idx_swz(int r, int ch) { return (uint32_t)(r * 32 + ((ch ^ ((r >> 2) & 1)) << 4)); }

// Issue the cp.async copy of index tile t (keys 64t .. 64t+63; rows >= nkeys zero-filled)
// into ring stage `stage`.  The caller commits.
__device__ __forceinline__ void idx_issue(IdxRing& R, int stage, const __half* base, int64_t t, int64_t nkeys) {
  const int tid = threadIdx.x;
  unsigned char* dst = reinterpret_cast<unsigned char*>(R.t[stage][0]);
#pragma unroll
  for (int i = 0; i < (kIdxKeys * 4) / kIdxThreads; ++i) {  // 256 chunks of 16 bytes
    const int idx = i * kIdxThreads + tid;
    const int r = idx >> 2, part = (idx >> 1) & 1, ch = idx & 1;
    const int64_t j = t * kIdxKeys + r;
    const bool ok = j < nkeys;
    cp_async16(dst + part * (kIdxKeys * kR * 2) + idx_swz(r, ch), base + (ok ? j : 0) * (2 * kR) + part * kR + ch * 8,
               ok ? 16 : 0);
  }
}

// x = hi + lo in fp16 (about 22 significant bits; the index cache stores keys split this way)
__device__ __forceinline__ void split_half(float x, __half* hi, __half* lo) {
  const __half h = __float2half_rn(x);
  *hi = h;
  *lo = __float2half_rn(x - __half2float(h));
}

// A fragments (hi, lo) of the 16-dim index queries of rows ra (slot 0) and rb (slot 1);
// q points at row ra's 16 floats, rs is the row stride in floats; invalid rows are zero.
__device__ __forceinline__ void idx_load_q(uint32_t qh[4], uint32_t ql[4], const float* qa, const float* qb) {
  const int tq = threadIdx.x & 3;
  float x[8];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int c = 2 * tq + 8 * i;
    x[4 * i + 0] = qa ? qa[c] : 0.f;
    x[4 * i + 1] = qa ? qa[c + 1] : 0.f;
    x[4 * i + 2] = qb ? qb[c] : 0.f;
    x[4 * i + 3] = qb ? qb[c + 1] : 0.f;
  }
  // register order: a0 = (row a, dims 2tq..+1), a1 = (row b, same), a2 = (row a, dims 2tq+8..),
  // a3 = (row b, dims 2tq+8..)
  const int src[4][2] = {{0, 1}, {2, 3}, {4, 5}, {6, 7}};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __half h0, l0, h1, l1;
    split_half(x[src[k][0]], &h0, &l0);
    split_half(x[src[k][1]], &h1, &l1);
    __half2 hh = __halves2half2(h0, h1), ll = __halves2half2(l0, l1);
    qh[k] = *reinterpret_cast<uint32_t*>(&hh);
    ql[k] = *reinterpret_cast<uint32_t*>(&ll);
  }
}

// Scores of the warp's 16 rows against the 64 keys of ring stage `stage`.
__device__ __forceinline__ void idx_scores(float c[8][4], const uint32_t qh[4], const uint32_t ql[4],
                                           const IdxRing& R, int stage) {
  const int lane = threadIdx.x & 31;
  const uint32_t hi = smem_u32(R.t[stage][0]), lo = smem_u32(R.t[stage][1]);
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.f;
#pragma unroll
  for (int np = 0; np < 4; ++np) {
    const int mi = lane >> 3;
    const int key = np * 16 + (mi >> 1) * 8 + (lane & 7);
    const uint32_t off = idx_swz(key, mi & 1);
    uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
    ldsm_x4(hi + off, h0, h1, h2, h3);
    ldsm_x4(lo + off, l0, l1, l2, l3);
    // small terms first
    mma16816(c[2 * np], ql, h0, h1);
    mma16816(c[2 * np], qh, l0, l1);
    mma16816(c[2 * np], qh, h0, h1);
    mma16816(c[2 * np + 1], ql, h2, h3);
    mma16816(c[2 * np + 1], qh, l2, l3);
    mma16816(c[2 * np + 1], qh, h2, h3);
  }
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) c[nt][e] += 0.0f;  // -0 -> +0: equal scores, equal order keys
  }
}

}  // namespace rtp
