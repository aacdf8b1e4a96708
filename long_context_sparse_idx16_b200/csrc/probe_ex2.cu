// probe_ex2.cu -- issue-rate probe of the exponential (MUFU ex2) pipe.
//
// The prefill selection evaluates one exponential per causal (row, key) pair, so its roofline is
// the rate at which the SMs retire ex2.approx.  This kernel measures that rate instead of
// assuming it: every thread runs eight independent chains y <- ex2(y) * (-0.5) (the multiply
// runs on the FMA pipe and keeps y in [-0.5, -0.25]), so nothing but the ex2 issue rate bounds
// it.  The caller times the launch with CUDA events and divides the exponentials by the time.
#include "rtp_device.cuh"
#include "rtp_internal.h"

namespace rtp {

namespace {

constexpr int kProbeThreads = 256;
constexpr int kChains = 8;

__global__ void __launch_bounds__(kProbeThreads) probe_ex2_kernel(int iters, float* out) {
  float y[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) y[c] = -0.25f - 0.01f * (float)c - 1e-7f * (float)threadIdx.x;
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < kChains; ++c) y[c] = fast_exp2(y[c]) * -0.5f;
  }
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) s += y[c];
  out[(int64_t)blockIdx.x * kProbeThreads + threadIdx.x] = s;
}

}  // namespace

}  // namespace rtp

using namespace rtp;

extern "C" rtp_status rtp_probe_ex2(int32_t blocks, int32_t iters, float* out, int64_t* n_exp,
                                    cudaStream_t stream) {
  if (blocks < 1 || iters < 1 || !out || !n_exp) return fail(nullptr, RTP_EINVAL, "rtp_probe_ex2: bad argument");
  probe_ex2_kernel<<<blocks, kProbeThreads, 0, stream>>>(iters, out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "rtp_probe_ex2: launch");
  *n_exp = (int64_t)blocks * kProbeThreads * kChains * iters;
  return RTP_OK;
}
