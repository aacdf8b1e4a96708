// noalloc_gather.cu -- exact attention over caller-given key lists, without any allocation.
//
// Some callers cannot call cudaMalloc: code that runs while a CUDA graph is being captured
// (allocation is not capturable), engines that own all device memory through their own pool
// and forbid other allocations, and processes whose device memory is already fully committed.
// rtp_gather_attn_noalloc serves them: it needs no layer and allocates nothing.  The caller
// passes inputs and outputs; the split-K partials and merge tickets live in one file-scope
// device array of fixed size (kScratchItems work items), shared by every call on a device.
//
// The scratch array's host-side name is not a device address.  The first call on each device
// (with that device current) looks the address up with cudaGetSymbolAddress and caches it;
// make that first call before any stream capture.  Because all calls share the array, two
// calls whose kernels overlap on the GPU race on it; issue them on one stream or serialise
// them.  Each call clears the merge tickets it uses before its kernel runs.
#include <mutex>
#include <string>

#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr int kChunk = 128;                 // listed keys per work item
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerHalf = kChunk / (2 * kWarps);
constexpr int kMaxProblems = 2048;
constexpr int kScratchItems = 4096;         // work items (problem x chunk) per call
constexpr int kMaxDevices = 64;

// [kScratchItems][D + 2] partials (m, l, o[128]) followed by [kMaxProblems] merge tickets.
constexpr size_t kScratchFloats = (size_t)kScratchItems * (kD + 2) + kMaxProblems;
static __device__ __align__(256) float g_noalloc_scratch[kScratchFloats];

struct Args {
  const __half* k;
  const __half* v;
  const int32_t* kv_block;  // [P] or nullptr (block p)
  int64_t kv_stride;        // elements between KV blocks
  const float* q;           // [P][128]
  const int32_t* idx;
  int64_t idx_stride;
  const int32_t* cnt;
  int P;
  int64_t max_count;        // counts are clamped to this (the scratch is sized from it)
  float scale_log2;
  float* out;               // [P][128]
  float* part;
  uint32_t* ticket;
};

__device__ __forceinline__ void unpack8(uint4 u, float* f) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __half22float2(h[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}

__global__ void __launch_bounds__(kThreads) noalloc_gather_kernel(Args a) {
  __shared__ int s_base[kMaxProblems + 1];
  __shared__ float s_m[kWarps], s_l[kWarps];
  __shared__ float s_o[kWarps][kD];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, hl = lane & 15;

  for (int p = tid; p < a.P; p += kThreads) {
    const int64_t K = min((int64_t)max(a.cnt[p], 0), a.max_count);
    s_base[p + 1] = (int)((K + kChunk - 1) / kChunk);
  }
  __syncthreads();
  if (tid == 0) {
    s_base[0] = 0;
    for (int p = 0; p < a.P; ++p) s_base[p + 1] += s_base[p];
  }
  __syncthreads();
  const int total = min(s_base[a.P], kScratchItems);  // the host bounds it by kScratchItems

  // a problem with an empty list has no work item: its output is defined as zeros
  for (int p = blockIdx.x; p < a.P; p += gridDim.x)
    if (s_base[p + 1] == s_base[p] && tid < kD) a.out[(int64_t)p * kD + tid] = 0.f;

  for (int it = blockIdx.x; it < total; it += gridDim.x) {
    // the item's problem: the last p with s_base[p] <= it (then s_base[p + 1] > it; problems
    // with empty lists share their base with the next problem and are skipped over)
    int p = 0;
    for (int lo = 0, hi = a.P - 1; lo <= hi;) {
      const int mid = (lo + hi) >> 1;
      if (s_base[mid] <= it) {
        p = mid;
        lo = mid + 1;
      } else {
        hi = mid - 1;
      }
    }
    const int chunk = it - s_base[p];
    const int n_items = s_base[p + 1] - s_base[p];
    const int64_t K = min((int64_t)max(a.cnt[p], 0), a.max_count);
    const int64_t r_lo = (int64_t)chunk * kChunk, r_hi = min(K, r_lo + kChunk);
    const int64_t blk = a.kv_block ? a.kv_block[p] : p;
    const __half* kb = a.k + blk * a.kv_stride + hl * 8;
    const __half* vb = a.v + blk * a.kv_stride + hl * 8;
    const int32_t* ids = a.idx + (int64_t)p * a.idx_stride;
    float q[8];
    {
      const float4* qp = reinterpret_cast<const float4*>(a.q + (int64_t)p * kD + hl * 8);
      const float4 q0 = qp[0], q1 = qp[1];
      q[0] = q0.x; q[1] = q0.y; q[2] = q0.z; q[3] = q0.w;
      q[4] = q1.x; q[5] = q1.y; q[6] = q1.z; q[7] = q1.w;
    }
    uint4 kr[kRowsPerHalf], vr[kRowsPerHalf];
#pragma unroll
    for (int u = 0; u < kRowsPerHalf; ++u) {
      const int64_t r = r_lo + (warp * 2 + half) + 2 * kWarps * u;
      if (r < r_hi) {
        const int64_t j = ids[r];
        kr[u] = ld_nc_u4(kb + j * kD);
        vr[u] = ld_nc_u4(vb + j * kD);
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
    float* outp = a.out + (int64_t)p * kD;
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
        if (tid < kD) {
          float M = -INFINITY;
          for (int i = 0; i < n_items; ++i) M = fmaxf(M, __ldcg(base + (int64_t)i * (kD + 2)));
          float Ls = 0.f, O = 0.f;
          for (int i = 0; i < n_items; ++i) {
            const float mi = __ldcg(base + (int64_t)i * (kD + 2));
            const float c = (mi == -INFINITY) ? 0.f : fast_exp2(mi - M);
            Ls += __ldcg(base + (int64_t)i * (kD + 2) + 1) * c;
            O += __ldcg(base + (int64_t)i * (kD + 2) + 2 + tid) * c;
          }
          outp[tid] = O / Ls;
        }
        if (tid == 0) a.ticket[p] = 0u;
      }
    }
    __syncthreads();
  }
}

// Device address of the scratch array, looked up once per device and kept for the life of the
// process: the cache assumes the device's primary context is never torn down (no
// cudaDeviceReset between calls).
std::mutex g_addr_mu;
float* g_addr[kMaxDevices] = {};

}  // namespace

}  // namespace rtp

using namespace rtp;

extern "C" rtp_status rtp_gather_attn_noalloc(const void* k, const void* v, const int32_t* kv_block,
                                              int64_t kv_stride, const float* q, const int32_t* idx,
                                              int64_t idx_stride, const int32_t* cnt, int32_t P,
                                              int64_t max_count, float sm_scale, float* out,
                                              cudaStream_t stream) {
  if (!k || !v || !q || !idx || !cnt || !out)
    return fail(nullptr, RTP_EINVAL, "rtp_gather_attn_noalloc: NULL pointer");
  if (P < 1 || P > kMaxProblems)
    return fail(nullptr, RTP_EINVAL, "rtp_gather_attn_noalloc: need 1 <= P <= 2048");
  if (max_count < 1 || idx_stride < max_count || kv_stride < kD || !(sm_scale > 0.f))
    return fail(nullptr, RTP_EINVAL, "rtp_gather_attn_noalloc: bad max_count, strides or scale");
  // K/V rows and queries are read as 16-byte vectors
  if ((((uintptr_t)k | (uintptr_t)v | (uintptr_t)q) & 15u) != 0u || kv_stride % 8 != 0)
    return fail(nullptr, RTP_EINVAL,
                "rtp_gather_attn_noalloc: k, v and q must be 16-byte aligned and kv_stride a multiple of 8");
  const int64_t worst = (int64_t)P * ((max_count + kChunk - 1) / kChunk);
  if (worst > kScratchItems)
    return fail(nullptr, RTP_EINVAL,
                "rtp_gather_attn_noalloc: P * ceil(max_count / 128) exceeds the 4096 work items of the "
                "built-in scratch (about 2.1 MB); split the call");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "rtp_gather_attn_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(nullptr, RTP_EINVAL, "rtp_gather_attn_noalloc: device id");
  float* scratch;
  {
    std::lock_guard<std::mutex> g(g_addr_mu);
    if (!g_addr[dev]) {  // first call on this device: look up the array's device address
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(nullptr, e, "rtp_gather_attn_noalloc: cudaGetSymbolAddress");
      g_addr[dev] = static_cast<float*>(ptr);
    }
    scratch = g_addr[dev];
  }
  Args a;
  a.k = static_cast<const __half*>(k);
  a.v = static_cast<const __half*>(v);
  a.kv_block = kv_block;
  a.kv_stride = kv_stride;
  a.q = q;
  a.idx = idx;
  a.idx_stride = idx_stride;
  a.cnt = cnt;
  a.P = P;
  a.max_count = max_count;
  a.scale_log2 = sm_scale * 1.4426950408889634f;
  a.out = out;
  a.part = scratch;
  a.ticket = reinterpret_cast<uint32_t*>(scratch + (size_t)kScratchItems * (kD + 2));
  // tickets of this call start at zero (a previous call may have been cut short)
  e = cudaMemsetAsync(a.ticket, 0, sizeof(uint32_t) * (size_t)P, stream);
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "rtp_gather_attn_noalloc: clear tickets");
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  noalloc_gather_kernel<<<4 * sms, kThreads, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "rtp_gather_attn_noalloc: launch");
  return RTP_OK;
}
