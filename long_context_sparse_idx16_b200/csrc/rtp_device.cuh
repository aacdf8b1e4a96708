// rtp_device.cuh -- device helpers shared by the CUDA kernels of the sparse attention layer.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rtp {

constexpr int kD = 128;        // head dim
constexpr int kR = 16;         // index dim
constexpr int kHalfD = kD / 2; // RoPE pairs (c, c + D/2)
constexpr int kMaxGroup = 16;  // query heads per KV head handled by one MMA row tile

// Device error word bits (reported by rtp_check).
enum : uint32_t {
  kErrOverflow = 1u,  // selected set larger than max_select
  kErrRange = 2u,     // value outside the fp16 cache range
  kErrTimeout = 4u,   // a bounded wait gave up
  kErrInternal = 8u,  // consistency check failed
};

// Bounded-wait limit for grid barriers: about one second at the B200 clock.
constexpr long long kWaitLimitCycles = 2000000000LL;

// cos/sin of the RoPE angle pos * theta.  The angle is formed in fp64 (pos reaches 2^20, where
// an fp32 product is off by ~0.06 rad) and reduced to [-pi, pi] by Cody-Waite subtraction of
// k * 2pi with 2pi split into two doubles; the short reduced angle then goes to fp32 sincosf.
__device__ __forceinline__ void rope_cos_sin(int64_t pos, double theta, float* c, float* s) {
  const double kTwoPiHi = 6.283185307179586;        // 2pi rounded to double
  const double kTwoPiLo = 2.4492935982947064e-16;   // 2pi - kTwoPiHi
  const double a = (double)pos * theta;
  const double k = rint(a * (1.0 / 6.283185307179586));
  double r = fma(-k, kTwoPiHi, a);
  r = fma(-k, kTwoPiLo, r);
  sincosf((float)r, s, c);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Order-preserving map of a float's bits to uint32 (larger float -> larger key).
// Callers canonicalise -0 to +0 first so equal scores get equal keys.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

__device__ __forceinline__ float4 ld_stream_f4(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_nc_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier for a cooperative launch (all CTAs co-resident).  count/gen live in
// global memory and start at 0.  Every wait is bounded: on timeout the error word gets
// kErrTimeout and the function returns false; callers then leave the kernel.
__device__ __forceinline__ bool grid_barrier(uint32_t* count, uint32_t* gen, uint32_t nblocks,
                                             uint32_t* err) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    uint32_t my_gen = ld_acquire_u32(gen);
    __threadfence();
    uint32_t prev = atomicAdd(count, 1u);
    if (prev == nblocks - 1) {
      atomicExch(count, 0u);
      __threadfence();
      atomicAdd(gen, 1u);
    } else {
      long long t0 = clock64();
      while (ld_acquire_u32(gen) == my_gen) {
        __nanosleep(32);
        if (clock64() - t0 > kWaitLimitCycles) {
          atomicOr(err, kErrTimeout);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// cp.async 16 bytes global -> shared; src_bytes = 0 fills zeros.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes) {
  uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace rtp
