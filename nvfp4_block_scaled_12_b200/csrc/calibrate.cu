// Per-tensor scale calibration: g = amax(|x|) / (6 * 448) on the device
// (ModelOpt's `input_scale` / `weight_scale_2`, "BFL (fp8r / nvfp4)" diffusers
// doc, `nvfp4` bullet: a calibrated fp32 activation scale and a global fp32
// weight scale).  Two launches: a grid-stride max-reduction into out[0]
// (atomicMax on the float's bit pattern, valid because every |x| >= 0), then
// one thread computes out[1] = out[0] / 2688 with a single IEEE division.
#include "internal.h"

namespace nvfp4 {
namespace {

__global__ void __launch_bounds__(256) amax_kernel(const uint4* __restrict__ x, int64_t n_vec, float* out) {
  float m = 0.0f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_vec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = ld_stream_v4(x + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))), fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))));
    m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))), fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float warp_max[8];
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) m = fmaxf(m, warp_max[w]);
    atomicMax(reinterpret_cast<unsigned int*>(out), __float_as_uint(m));
  }
}

__global__ void scale_from_amax_kernel(float* out) { out[1] = __fdiv_rn(out[0], 2688.0f); }

}  // namespace

cudaError_t launch_calibrate(const void* x, int64_t n, float* out, cudaStream_t stream, const DeviceInfo& dev) {
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float), stream);
  if (e != cudaSuccess) return e;
  const int64_t n_vec = n / 8;
  int64_t blocks = (n_vec + 255) / 256;
  const int64_t cap = static_cast<int64_t>(dev.num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  amax_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(static_cast<const uint4*>(x), n_vec, out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  scale_from_amax_kernel<<<1, 1, 0, stream>>>(out);
  return cudaGetLastError();
}

}  // namespace nvfp4
