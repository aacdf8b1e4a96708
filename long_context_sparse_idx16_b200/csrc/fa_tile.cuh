// fa_tile.cuh -- one 64-query-row attention tile for the prefill kernels (4 warps x 16 rows).
//
// Online-softmax attention over a stream of 64-key tiles staged in shared memory:
// S = Q K^T and O += P V on tensor cores (mma.m16n8k16, fp16 operands, fp32 accumulation),
// the mask supplied per element by the caller.  Each warp owns 16 query rows; a thread holds
// rows gr and gr + 8 of its warp (gr = lane / 4) and, for each 8-wide column tile, the two
// columns 2 * (lane % 4) and 2 * (lane % 4) + 1.
#pragma once

#include "mma_tile.cuh"
#include "rtp_device.cuh"

namespace rtp {

constexpr int kFaRows = 64;   // query rows per CTA
constexpr int kFaKeys = 64;   // keys per tile
constexpr int kFaThreads = 128;
constexpr int kFaTileBytes = kFaKeys * kRowBytes;  // 16 KB per K or V tile

struct FaAcc {
  float o[16][4];  // 16 rows x 128 dims per warp: [dim tile][c0..c3]
  float m0, m1, l0, l1;
};

__device__ __forceinline__ void fa_init(FaAcc& A) {
#pragma unroll
  for (int i = 0; i < 16; ++i) A.o[i][0] = A.o[i][1] = A.o[i][2] = A.o[i][3] = 0.f;
  A.m0 = A.m1 = -INFINITY;
  A.l0 = A.l1 = 0.f;
}

// Q fragments (fp16) of query rows row0 .. row0+15 from fp32 rows q[row][128] (row stride qs
// floats); rows >= nrows are zero.
__device__ __forceinline__ void fa_load_q(uint32_t qa[8][4], const float* q, int64_t qs, int row0, int nrows) {
  const int lane = threadIdx.x & 31, gr = lane >> 2, tq = lane & 3;
  const float* q0 = (row0 + gr < nrows) ? q + (int64_t)(row0 + gr) * qs : nullptr;
  const float* q1 = (row0 + gr + 8 < nrows) ? q + (int64_t)(row0 + gr + 8) * qs : nullptr;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const int c0 = kk * 16 + 2 * tq, c1 = c0 + 8;
    qa[kk][0] = q0 ? pack_half2(q0[c0], q0[c0 + 1]) : 0u;
    qa[kk][1] = q1 ? pack_half2(q1[c0], q1[c0 + 1]) : 0u;
    qa[kk][2] = q0 ? pack_half2(q0[c1], q0[c1 + 1]) : 0u;
    qa[kk][3] = q1 ? pack_half2(q1[c1], q1[c1 + 1]) : 0u;
  }
}

// Stage a 64-key K and V tile (rows given by pos_of(t), t < nvalid) into swizzled smem with
// cp.async (128 threads, 8 chunks of K and 8 of V per thread); invalid rows are zero-filled.
template <typename PosFn>
__device__ __forceinline__ void fa_stage(unsigned char* ksm, unsigned char* vsm, const __half* kb, const __half* vb,
                                         int nvalid, PosFn pos_of) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int i = 0; i < (kFaKeys * 16) / kFaThreads; ++i) {
    const int idx = i * kFaThreads + tid;
    const int r = idx >> 4, ch = idx & 15;
    const bool ok = r < nvalid;
    const int64_t pos = ok ? pos_of(r) : 0;
    cp_async16(ksm + swz(r, ch), kb + pos * kD + ch * 8, ok ? 16 : 0);
    cp_async16(vsm + swz(r, ch), vb + pos * kD + ch * 8, ok ? 16 : 0);
  }
}

// One key tile: visible(r, t) says whether row r (0..63 within the CTA) may attend to tile key t
// (not consulted when kMasked is false: every row sees every key of the tile).
template <bool kMasked = true, typename VisFn>
__device__ __forceinline__ void fa_tile(FaAcc& A, const uint32_t qa[8][4], const unsigned char* ksm,
                                        const unsigned char* vsm, float scale_log2, VisFn visible) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gr = lane >> 2, tq = lane & 3;
  float s[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      const int mi = lane >> 3;
      const int key = np * 16 + (mi >> 1) * 8 + (lane & 7);
      const int ch = kk * 2 + (mi & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(smem_u32(ksm) + swz(key, ch), b0, b1, b2, b3);
      mma16816(s[2 * np], qa[kk], b0, b1);
      mma16816(s[2 * np + 1], qa[kk], b2, b3);
    }
  }
  const int r0 = warp * 16 + gr, r1 = r0 + 8;
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = nt * 8 + 2 * tq + e;
      if (kMasked) {
        s[nt][e] = visible(r0, t) ? s[nt][e] * scale_log2 : -INFINITY;
        s[nt][2 + e] = visible(r1, t) ? s[nt][2 + e] * scale_log2 : -INFINITY;
      } else {
        s[nt][e] *= scale_log2;
        s[nt][2 + e] *= scale_log2;
      }
      mx0 = fmaxf(mx0, s[nt][e]);
      mx1 = fmaxf(mx1, s[nt][2 + e]);
    }
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float mn0 = fmaxf(A.m0, mx0), mn1 = fmaxf(A.m1, mx1);
  const float c0 = mn0 == -INFINITY ? 1.f : fast_exp2(A.m0 - mn0);
  const float c1 = mn1 == -INFINITY ? 1.f : fast_exp2(A.m1 - mn1);
  A.m0 = mn0;
  A.m1 = mn1;
  uint32_t pa[4][4];
  float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const float p0 = mn0 == -INFINITY ? 0.f : fast_exp2(s[nt][0] - mn0);
    const float p1 = mn0 == -INFINITY ? 0.f : fast_exp2(s[nt][1] - mn0);
    const float p2 = mn1 == -INFINITY ? 0.f : fast_exp2(s[nt][2] - mn1);
    const float p3 = mn1 == -INFINITY ? 0.f : fast_exp2(s[nt][3] - mn1);
    rs0 += p0 + p1;
    rs1 += p2 + p3;
    const int ks = nt >> 1, hi = nt & 1;
    pa[ks][hi ? 2 : 0] = pack_half2(p0, p1);
    pa[ks][hi ? 3 : 1] = pack_half2(p2, p3);
  }
  A.l0 = A.l0 * c0 + rs0;
  A.l1 = A.l1 * c1 + rs1;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    A.o[i][0] *= c0;
    A.o[i][1] *= c0;
    A.o[i][2] *= c1;
    A.o[i][3] *= c1;
  }
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {
      const int mi = lane >> 3;
      const int key = ks * 16 + (mi & 1) * 8 + (lane & 7);
      const int ch = dp * 2 + (mi >> 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(vsm) + swz(key, ch), b0, b1, b2, b3);
      mma16816(A.o[2 * dp], pa[ks], b0, b1);
      mma16816(A.o[2 * dp + 1], pa[ks], b2, b3);
    }
  }
}

// Normalise and store rows row0+gr and row0+gr+8 of the warp: out row r at out + r * os.
__device__ __forceinline__ void fa_store(FaAcc& A, float* out, int64_t os, int row0, int nrows) {
  const int lane = threadIdx.x & 31, gr = lane >> 2, tq = lane & 3;
  float l0 = A.l0, l1 = A.l1;
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
  const int ra = row0 + gr, rb = ra + 8;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int d = i * 8 + 2 * tq;
    if (ra < nrows) *reinterpret_cast<float2*>(out + (int64_t)ra * os + d) = make_float2(A.o[i][0] * i0, A.o[i][1] * i0);
    if (rb < nrows) *reinterpret_cast<float2*>(out + (int64_t)rb * os + d) = make_float2(A.o[i][2] * i1, A.o[i][3] * i1);
  }
}

}  // namespace rtp
