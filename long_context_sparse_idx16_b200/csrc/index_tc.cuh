// index_tc.cuh -- 16-dim index scores of a 128-row prefill tile on 5th-generation tensor cores.
//
// The retrieval-head indexer scores s_j = qidx . kidx_j (techwalker page, section 3: a 16-dim
// "radar" over pre-RoPE projections; aitntnews page, finding 3: r = 16) for every (row, causal
// key) pair of a prefill chunk.  The fp32 operands are split into fp16 hi + lo (x = hi + lo to
// about 22 bits) and the score is lo.hi + hi.lo + hi.hi accumulated in fp32: three
// tcgen05.mma (kind::f16, M 128, N 64, K 16) into one TMEM accumulator of 128 lanes x 64
// columns, row r of the tile in lane r.  The selection and the attention kernels run the same
// instructions on the same operand bytes, so both see identical score bits.
//
// Operands sit in shared memory in the no-swizzle K-major layout: 16-byte chunk c of row r at
// c * (rows * 16) + r * 16, i.e. core matrices of 8 rows x 16 bytes, the rows of a chunk
// contiguous.  A row is [hi 0..7 | hi 8..15 | lo 0..7 | lo 8..15] (chunks 0-3); the hi and lo
// K-slices start 2 * rows * 16 bytes apart.  The split index cache ([key][hi 16 | lo 16] fp16)
// is copied into key tiles by TMA as four boxes of 64 keys x 8 values, one per chunk.
#pragma once

#include "tc_umma.cuh"
#include "tma.cuh"

namespace rtp {

constexpr int kTcRows = 128;                              // rows of the scoring tile (TMEM lanes)
constexpr int kTcKeys = 64;                               // keys per scoring tile (TMEM columns)
constexpr uint32_t kTcQBytes = kTcRows * 64;              // 8 KB query tile
constexpr uint32_t kTcKBytes = kTcKeys * 64;              // 4 KB key tile
constexpr uint32_t kTcIdesc = umma_idesc_f16(kTcKeys, false);

// no-swizzle K-major descriptor: LBO = byte stride between core matrices along K (one chunk of
// all rows), SBO = byte stride between 8-row groups
__device__ __forceinline__ uint64_t umma_desc_ns(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // version; layout type 0 (no swizzle) in bits 61-63
  return d;
}

__device__ __forceinline__ uint32_t ns_off(int r, int c, int rows) { return (uint32_t)(c * rows * 16 + r * 16); }

// Write row r of the query tile from 16 fp32 index-query values (nullptr: a zero row).
__device__ __forceinline__ void tc_put_query(unsigned char* qtile, int r, const float* q) {
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = q ? q[8 * k + 2 * e] : 0.f, x1 = q ? q[8 * k + 2 * e + 1] : 0.f;
      const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
      const __half l0 = __float2half_rn(x0 - __half2float(h0)), l1 = __float2half_rn(x1 - __half2float(h1));
      __half2 hh = __halves2half2(h0, h1), ll = __halves2half2(l0, l1);
      hi[e] = *reinterpret_cast<uint32_t*>(&hh);
      lo[e] = *reinterpret_cast<uint32_t*>(&ll);
    }
    *reinterpret_cast<uint4*>(qtile + ns_off(r, k, kTcRows)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(qtile + ns_off(r, 2 + k, kTcRows)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// TMA copy of key tile t of index block `blk_row0` (the tensor-map row of key 0 of this
// (sequence, retrieval head)) into a key-tile buffer; completion on mbar (one thread).
// The map views the split cache as [rows][4 chunks][8 values].
__device__ __forceinline__ void tc_load_keys(uint32_t ktile, const CUtensorMap* map, int64_t blk_row0, int64_t t,
                                             uint32_t mbar) {
  mbar_expect_tx(mbar, kTcKBytes);
  const int y = (int)(blk_row0 + t * kTcKeys);
#pragma unroll
  for (int c = 0; c < 4; ++c) tma_load_3d(ktile + c * (kTcKeys * 16), map, 0, c, y, mbar);
}

// Scores of the query tile against one key tile into TMEM columns [col, col + 64), then an
// arrive on the mbarrier when they are complete.  One thread issues; the query tile must be
// visible to the async proxy (fence.proxy.async after its writes, then a barrier).
__device__ __forceinline__ void tc_issue_scores(uint32_t tmem_col, uint32_t qtile, uint32_t ktile, uint32_t mbar) {
  tc_fence_after();
  const uint64_t qh = umma_desc_ns(qtile, kTcRows * 16, 128), ql = umma_desc_ns(qtile + 2 * kTcRows * 16, kTcRows * 16, 128);
  const uint64_t kh = umma_desc_ns(ktile, kTcKeys * 16, 128), kl = umma_desc_ns(ktile + 2 * kTcKeys * 16, kTcKeys * 16, 128);
  // small terms first: lo.hi, hi.lo, then hi.hi
  umma_f16(tmem_col, ql, kh, kTcIdesc, 0u);
  umma_f16(tmem_col, qh, kl, kTcIdesc, 1u);
  umma_f16(tmem_col, qh, kh, kTcIdesc, 1u);
  umma_commit(mbar);
}

}  // namespace rtp
