// decode_swa.cu -- local heads at decode: causal window of W keys plus the first S keys.
//
// Local heads (~85% of heads) only look at nearby tokens and a few attention sinks
// (techwalker page, section 2; section 8: window 8192 with 4 sinks).  For the decode
// query at position i the key set is J = [0, S) U [max(S, i-W+1), i].
//
// B200 design
//   * GQA: all local query heads of one KV head share each K/V tile, so a tile is read from
//     HBM once per KV group.  The rows of the MMA tile are those query heads (<= 16), the
//     columns the keys: S = Q K^T and O += P V run on tensor cores with mma.m16n8k16
//     (fp16 operands, fp32 accumulation).  Decode has at most 16 query rows per KV group, far
//     below the 64/128-row tcgen05 tile, and the kernel is bound by HBM, so the warp-level MMA
//     is the right size here.
//   * Each warp streams its own 16-key slices with cp.async into XOR-swizzled shared tiles,
//     two buffers deep: the next slice's copies are in flight while the current slice's MMAs
//     run.  Fragments are read with ldmatrix, conflict-free.
//   * The window is split into chunks over the grid (enough CTAs for all SMs even at B=1);
//     per-chunk partials (m, l, o) are merged by a small second kernel.
#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr int kThreads = kSwaThreads;  // 4 warps
constexpr int kWarps = kThreads / 32;
constexpr int kTile = kSwaTile;        // keys per chunking unit (chunks are whole tiles)
constexpr int kWarpKeys = 16;          // keys per warp stage
constexpr int kStepKeys = kWarps * kWarpKeys;  // keys per CTA step (64)
constexpr int kRowBytes = kD * 2;      // one fp16 row
constexpr int kStageBytes = 2 * kWarpKeys * kRowBytes;  // one warp stage: K rows, then V rows (8 KB)

struct SwaArgs {
  const __half* kc;
  const __half* vc;
  int64_t max_seq;
  int Hkv, Hq;
  const float* q_rot;        // [B][Hq][D]
  const int16_t* loc_head;   // [Hkv][16]
  const int32_t* loc_cnt;    // [Hkv]
  SeqPos lens;               // each sequence's length N_b; its query sits at N_b - 1
  int64_t W, S;              // window and sinks: keys [0, min(S, N_b)) and [max(.., N_b - W), N_b)
  int64_t chunk_keys;        // keys per chunk (chunks of the longest key set; a shorter
                             // sequence's later chunks are empty)
  int n_chunks;
  float scale_log2;
  float* part;  // [B][Hkv][n_chunks][16][D+2]
  float* out;   // [B][Hq][D]
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_half2(float x, float y) {
  __half2 h = __floats2half2_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&h);
}
// byte offset of 16-byte chunk `ch` of row `r` in a swizzled [rows][128] fp16 tile
__device__ __forceinline__ uint32_t swz(int r, int ch) { return (uint32_t)(r * kRowBytes + ((ch ^ (r & 7)) << 4)); }

__global__ void __launch_bounds__(kThreads) decode_swa_kernel(SwaArgs a) {
  extern __shared__ __align__(128) unsigned char sm[];
  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, tq = lane & 3;  // mma groupID / thread-in-group
  const int n_rows = a.loc_cnt[g];
  if (n_rows == 0) return;
  unsigned char* wsm = sm + warp * (2 * kStageBytes);  // this warp's two stage buffers

  // Q fragments: rows = local heads of this KV group (zero beyond n_rows)
  uint32_t qa[8][4];
  {
    const int h0 = gr < n_rows ? a.loc_head[g * kMaxGroup + gr] : -1;
    const int h1 = gr + 8 < n_rows ? a.loc_head[g * kMaxGroup + gr + 8] : -1;
    const float* q0 = h0 >= 0 ? a.q_rot + ((int64_t)b * a.Hq + h0) * kD : nullptr;
    const float* q1 = h1 >= 0 ? a.q_rot + ((int64_t)b * a.Hq + h1) * kD : nullptr;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int c0 = kk * 16 + 2 * tq, c1 = c0 + 8;
      qa[kk][0] = q0 ? pack_half2(q0[c0], q0[c0 + 1]) : 0u;
      qa[kk][1] = q1 ? pack_half2(q1[c0], q1[c0 + 1]) : 0u;
      qa[kk][2] = q0 ? pack_half2(q0[c1], q0[c1 + 1]) : 0u;
      qa[kk][3] = q1 ? pack_half2(q1[c1], q1[c1 + 1]) : 0u;
    }
  }
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  const __half* kb = a.kc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD;
  const __half* vb = a.vc + ((int64_t)b * a.Hkv + g) * a.max_seq * kD;
  // this sequence's key set J = [0, s_cnt) U [w0, N_b), enumerated by u = 0 .. nJ - 1
  const int64_t Nb = a.lens.v[b];
  const int64_t s_cnt = min(a.S, Nb);
  const int64_t w0 = max(s_cnt, Nb - a.W);
  const int64_t nJ = s_cnt + (Nb - w0);
  const int64_t u_lo = (int64_t)chunk * a.chunk_keys;
  const int64_t u_hi = min(nJ, u_lo + a.chunk_keys);

  // stage `it` of this warp: keys u_lo + it * kStepKeys + warp * kWarpKeys + (0 .. 15), into
  // buffer it & 1 (keys past the chunk are zero-filled and masked below)
  auto issue = [&](int64_t t0, int buf) {
    unsigned char* ksm = wsm + buf * kStageBytes;
    unsigned char* vsm = ksm + kWarpKeys * kRowBytes;
    const int64_t wbase = t0 + warp * kWarpKeys;
#pragma unroll
    for (int i = 0; i < (kWarpKeys * 16) / 32; ++i) {
      const int idx = i * 32 + lane;
      const int r = idx >> 4, ch = idx & 15;
      const int64_t u = wbase + r;
      const bool ok = u < u_hi;
      const int64_t pos = u < s_cnt ? u : w0 + (u - s_cnt);
      const int64_t safe = ok ? pos : 0;
      cp_async16(ksm + swz(r, ch), kb + safe * kD + ch * 8, ok ? 16 : 0);
      cp_async16(vsm + swz(r, ch), vb + safe * kD + ch * 8, ok ? 16 : 0);
    }
  };
  if (u_lo < u_hi) issue(u_lo, 0);
  cp_async_commit();
  int it = 0;
  for (int64_t t0 = u_lo; t0 < u_hi; t0 += kStepKeys, ++it) {
    const int buf = it & 1;
    if (t0 + kStepKeys < u_hi) issue(t0 + kStepKeys, buf ^ 1);  // the next stage, into the other buffer
    cp_async_commit();
    cp_async_wait<1>();  // every group but the newest: this stage has landed
    __syncwarp();
    const unsigned char* ksm = wsm + buf * kStageBytes;
    const unsigned char* vsm = ksm + kWarpKeys * kRowBytes;
    const int64_t wbase = t0 + warp * kWarpKeys;

    // S = Q K^T over 16 keys: 2 n-tiles of 8 keys
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      // matrices: (ntile 0, k lo), (0, k hi), (1, k lo), (1, k hi)
      const int mi = lane >> 3;
      const int key = (mi >> 1) * 8 + (lane & 7);
      const int ch = kk * 2 + (mi & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(smem_u32(ksm) + swz(key, ch), b0, b1, b2, b3);
      mma16816(s[0], qa[kk], b0, b1);
      mma16816(s[1], qa[kk], b2, b3);
    }
    // mask keys past the chunk, scale, online softmax (rows gr and gr+8)
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int64_t u = wbase + nt * 8 + 2 * tq + e;
        const bool ok = u < u_hi;
        s[nt][e] = ok ? s[nt][e] * a.scale_log2 : -INFINITY;
        s[nt][2 + e] = ok ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, s[nt][e]);
        mx1 = fmaxf(mx1, s[nt][2 + e]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float c0 = mn0 == -INFINITY ? 1.f : fast_exp2(m0 - mn0);
    const float c1 = mn1 == -INFINITY ? 1.f : fast_exp2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    uint32_t pa[4];
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const float p0 = mn0 == -INFINITY ? 0.f : fast_exp2(s[nt][0] - mn0);
      const float p1 = mn0 == -INFINITY ? 0.f : fast_exp2(s[nt][1] - mn0);
      const float p2 = mn1 == -INFINITY ? 0.f : fast_exp2(s[nt][2] - mn1);
      const float p3 = mn1 == -INFINITY ? 0.f : fast_exp2(s[nt][3] - mn1);
      rs0 += p0 + p1;
      rs1 += p2 + p3;
      // A fragment of P (one k-step of 16 keys): (row gr, keys 2tq..) from tile 0, (+8) from tile 1
      pa[nt ? 2 : 0] = pack_half2(p0, p1);
      pa[nt ? 3 : 1] = pack_half2(p2, p3);
    }
    l0 = l0 * c0 + rs0;
    l1 = l1 * c1 + rs1;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= c0;
      o[i][1] *= c0;
      o[i][2] *= c1;
      o[i][3] *= c1;
    }
    // O += P V: one k-step of 16 keys; 8 pairs of 8-dim n-tiles
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {
      // matrices: (keys lo, dims 16dp..+7), (keys hi, same), (keys lo, dims +8..), (keys hi, +8..)
      const int mi = lane >> 3;
      const int key = (mi & 1) * 8 + (lane & 7);
      const int ch = dp * 2 + (mi >> 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(vsm) + swz(key, ch), b0, b1, b2, b3);
      mma16816(o[2 * dp], pa, b0, b1);
      mma16816(o[2 * dp + 1], pa, b2, b3);
    }
    __syncwarp();  // this buffer is refilled two stages on
  }
  cp_async_wait<0>();  // no copy may still land in the tile space the merge below reuses

  // row sums across the 4 threads of a group
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

  // merge the 4 warps through shared memory (reuses the tile space)
  __syncthreads();
  float* so = reinterpret_cast<float*>(sm);            // [warps][16][D]
  float* sml = so + kWarps * 16 * kD;                   // [warps][16][2]
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int d = i * 8 + 2 * tq;
    so[(warp * 16 + gr) * kD + d] = o[i][0];
    so[(warp * 16 + gr) * kD + d + 1] = o[i][1];
    so[(warp * 16 + gr + 8) * kD + d] = o[i][2];
    so[(warp * 16 + gr + 8) * kD + d + 1] = o[i][3];
  }
  if (tq == 0) {
    sml[(warp * 16 + gr) * 2] = m0;
    sml[(warp * 16 + gr) * 2 + 1] = l0;
    sml[(warp * 16 + gr + 8) * 2] = m1;
    sml[(warp * 16 + gr + 8) * 2 + 1] = l1;
  }
  __syncthreads();
  // thread d owns dim d; loop over rows
  for (int r = 0; r < n_rows; ++r) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sml[(w * 16 + r) * 2]);
    float Ls = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = sml[(w * 16 + r) * 2];
      const float c = mw == -INFINITY ? 0.f : fast_exp2(mw - M);
      Ls += sml[(w * 16 + r) * 2 + 1] * c;
      O += so[(w * 16 + r) * kD + tid] * c;
    }
    if (a.n_chunks == 1) {
      const int h = a.loc_head[g * kMaxGroup + r];
      a.out[((int64_t)b * a.Hq + h) * kD + tid] = O / Ls;
    } else {
      float* pp = a.part + ((((int64_t)b * a.Hkv + g) * a.n_chunks + chunk) * kMaxGroup + r) * (kD + 2);
      pp[2 + tid] = O;
      if (tid == 0) {
        pp[0] = M;
        pp[1] = Ls;
      }
    }
  }
}

// Merge the per-chunk partials of one (query row, KV head, sequence): warps fold chunks
// w, w+8, ... with lane-owned column slices; the warp results combine in shared memory.
__global__ void __launch_bounds__(256) swa_merge_kernel(const float* __restrict__ part, int n_chunks, int Hkv,
                                                        int Hq, const int16_t* __restrict__ loc_head,
                                                        const int32_t* __restrict__ loc_cnt,
                                                        float* __restrict__ out) {
  const int r = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  if (r >= loc_cnt[g]) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ float s_m[8], s_l[8], s_o[8][kD];
  const float* base = part + (((int64_t)b * Hkv + g) * n_chunks * kMaxGroup + r) * (kD + 2);
  const int64_t stride = (int64_t)kMaxGroup * (kD + 2);
  float mv = -INFINITY;
  for (int i = tid; i < n_chunks; i += 256) mv = fmaxf(mv, base[i * stride]);
  mv = warp_max(mv);
  if (lane == 0) s_m[warp] = mv;
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < 8; ++w) M = fmaxf(M, s_m[w]);
  float ls = 0.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int i = warp; i < n_chunks; i += 8) {
    const float* pi = base + i * stride;
    const float mi = pi[0];
    const float c = mi == -INFINITY ? 0.f : fast_exp2(mi - M);
    ls += pi[1] * c;
    const float2 x = *reinterpret_cast<const float2*>(pi + 2 + lane * 4);
    const float2 y = *reinterpret_cast<const float2*>(pi + 4 + lane * 4);
    acc[0] += x.x * c;
    acc[1] += x.y * c;
    acc[2] += y.x * c;
    acc[3] += y.y * c;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) s_o[warp][lane * 4 + k] = acc[k];
  if (lane == 0) s_l[warp] = ls;
  __syncthreads();
  if (tid < kD) {
    float O = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      O += s_o[w][tid];
      L += s_l[w];
    }
    const int h = loc_head[g * kMaxGroup + r];
    out[((int64_t)b * Hq + h) * kD + tid] = O / L;
  }
}

}  // namespace

// Chunking, in whole 128-key tiles: at most three CTAs per SM over the whole grid, so the grid
// runs as one wave (166 registers per thread at 128 threads and 64 KB of shared memory let
// three CTAs share an SM; a fourth would wait for a second wave).
constexpr int64_t kSwaCtasPerSm = 3;
static void swa_chunks(const rtp_layer* L, int64_t nJ, int64_t* chunk_keys, int* n_chunks) {
  const int64_t pairs = (int64_t)L->B * L->Hkv;
  int64_t want = (kSwaCtasPerSm * L->sm_count) / pairs;  // chunks per (b, g)
  if (want < 1) want = 1;
  int64_t ck = (nJ + want - 1) / want;
  ck = (ck + kTile - 1) / kTile * kTile;
  if (ck < kTile) ck = kTile;
  *chunk_keys = ck;
  *n_chunks = (int)((nJ + ck - 1) / ck);
}

// Upper bound on chunks for any length: chunk_keys >= nJ / want, so n_chunks <= want, and
// want is at most this.
static int64_t swa_max_chunks(const rtp_layer* L) {
  const int64_t pairs = (int64_t)L->B * L->Hkv;
  return (kSwaCtasPerSm * L->sm_count + pairs - 1) / pairs;
}

int64_t swa_part_elems(const rtp_layer* L) {
  return (int64_t)L->B * L->Hkv * (swa_max_chunks(L) + 1) * kMaxGroup * (kD + 2);
}

cudaError_t launch_decode_swa(const rtp_layer* L, float* out, cudaStream_t st) {
  SwaArgs a;
  a.kc = L->kc;
  a.vc = L->vc;
  a.max_seq = L->max_seq;
  a.Hkv = L->Hkv;
  a.Hq = L->Hq;
  a.q_rot = L->q_rot;
  a.loc_head = L->d_loc_head;
  a.loc_cnt = L->d_loc_cnt;
  a.lens = seq_pos(L, 0);
  a.W = L->W;
  a.S = L->S;
  // chunking of the longest sequence's key set (at most S + W keys)
  int64_t nJ_max = 0;
  for (int b = 0; b < L->B; ++b) {
    const int64_t n = L->lens[b], sc = L->S < n ? L->S : n;
    const int64_t w0 = n - L->W > sc ? n - L->W : sc;
    const int64_t nj = sc + (n - w0);
    nJ_max = nj > nJ_max ? nj : nJ_max;
  }
  swa_chunks(L, nJ_max, &a.chunk_keys, &a.n_chunks);
  if ((int64_t)L->B * L->Hkv * a.n_chunks * kMaxGroup * (kD + 2) > L->spart_elems) return cudaErrorInvalidValue;
  a.scale_log2 = L->sm_scale * 1.4426950408889634f;
  a.part = L->spart;
  a.out = out;
  const size_t tile_smem = (size_t)kWarps * 2 * kStageBytes;  // 64 KB: two stage buffers per warp
  const size_t merge_smem = (size_t)kWarps * 16 * kD * 4 + kWarps * 16 * 2 * 4;
  const size_t smem = tile_smem > merge_smem ? tile_smem : merge_smem;
  cudaError_t e = cudaFuncSetAttribute(decode_swa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  {
    ProfScope ps(const_cast<rtp_layer*>(L), "decode_swa", st);
    decode_swa_kernel<<<dim3(a.n_chunks, L->Hkv, L->B), kThreads, smem, st>>>(a);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess || a.n_chunks == 1) return e;
  ProfScope ps(const_cast<rtp_layer*>(L), "swa_merge", st);
  swa_merge_kernel<<<dim3(kMaxGroup, L->Hkv, L->B), 256, 0, st>>>(L->spart, a.n_chunks, L->Hkv, L->Hq,
                                                                L->d_loc_head, L->d_loc_cnt, out);
  return cudaGetLastError();
}

}  // namespace rtp
