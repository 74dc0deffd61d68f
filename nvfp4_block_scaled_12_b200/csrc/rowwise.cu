// Row-wise FP8 activation quantization ("BFL (fp8r / nvfp4)" diffusers doc,
// `fp8r` bullet: activations are quantized to E4M3 row by row at run time,
// next to E4M3 weights with one fp32 scale per row).  Per row:
//     s = fl(amax / 448)        q_i = E4M3_satfinite(fl(x_i / s))
// and a row of zeros gets s = 0 and the codes of +-0.
//
// HBM-bound: 2 bytes read and 1 byte written per element, plus 4 bytes per
// row.  One warp per row, eight rows per CTA.  Rows of 1024-4096 elements are
// held in registers (one read); longer rows take two passes, the second
// hitting L1/L2, each lane streaming 16-byte vectors, four in flight.
#include "internal.h"

namespace nvfp4 {
namespace {

constexpr int kRowsPerCta = 8;

// Eight bf16 values (one 16-byte vector) -> eight E4M3 codes, each
// E4M3_satfinite(fl(x / d)) with an IEEE division.
__device__ __forceinline__ uint2 encode8_e4m3(const uint4& v, float d) {
  const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                      bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint16_t lo, hi;
    // cvt puts its first source in the high byte: pass (odd, even)
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(__fdiv_rn(f[4 * h + 1], d)),
        "f"(__fdiv_rn(f[4 * h + 0], d)));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(__fdiv_rn(f[4 * h + 3], d)),
        "f"(__fdiv_rn(f[4 * h + 2], d)));
    w[h] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  }
  return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ float absmax8(const uint4& v) {
  return fmaxf(fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))), fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))),
               fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))), fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
}

// Rows of K = 256 * kNv elements: each lane holds kNv 16-byte vectors of its
// row in registers, so the row is read from HBM once and all its loads are in
// flight together; amax, scale and codes come from the registers.
template <int kNv>
__global__ void __launch_bounds__(kRowsPerCta * 32)
    quantize_rowwise_regs_kernel(const uint4* __restrict__ x, int64_t M, uint8_t* __restrict__ codes,
                                 float* __restrict__ scale) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + warp;
  if (row >= M) return;
  const uint4* xr = x + row * (32 * kNv);
  uint4 v[kNv];
#pragma unroll
  for (int u = 0; u < kNv; ++u) v[u] = xr[lane + 32 * u];
  float m = 0.0f;
#pragma unroll
  for (int u = 0; u < kNv; ++u) m = fmaxf(m, absmax8(v[u]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float s = __fdiv_rn(m, 448.0f);
  if (lane == 0) scale[row] = s;
  const float d = s > 0.0f ? s : 1.0f;  // a zero row divides by 1: codes of +-0
  uint2* cr = reinterpret_cast<uint2*>(codes + row * (256 * kNv));
#pragma unroll
  for (int u = 0; u < kNv; ++u) cr[lane + 32 * u] = encode8_e4m3(v[u], d);
}

__global__ void __launch_bounds__(kRowsPerCta * 32)
    quantize_rowwise_kernel(const uint4* __restrict__ x, int64_t M, int64_t K, uint8_t* __restrict__ codes,
                            float* __restrict__ scale) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + warp;
  if (row >= M) return;
  const int64_t nvec = K >> 3;  // 16-byte vectors of 8 bf16
  const uint4* xr = x + row * nvec;

  float m = 0.0f;
  int64_t i = lane;
  for (; i + 96 < nvec; i += 128) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = xr[i + 32 * u];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v[u].x)), fabsf(bf16_hi(v[u].x))),
                         fmaxf(fabsf(bf16_lo(v[u].y)), fabsf(bf16_hi(v[u].y)))));
      m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v[u].z)), fabsf(bf16_hi(v[u].z))),
                         fmaxf(fabsf(bf16_lo(v[u].w)), fabsf(bf16_hi(v[u].w)))));
    }
  }
  for (; i < nvec; i += 32) {
    const uint4 v = xr[i];
    m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))), fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))));
    m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))), fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float s = __fdiv_rn(m, 448.0f);
  if (lane == 0) scale[row] = s;
  const float d = s > 0.0f ? s : 1.0f;  // a zero row divides by 1: codes of +-0

  auto encode8 = [&](const uint4& v) -> uint2 { return encode8_e4m3(v, d); };
  uint2* cr = reinterpret_cast<uint2*>(codes + row * K);
  i = lane;
  for (; i + 96 < nvec; i += 128) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = xr[i + 32 * u];
#pragma unroll
    for (int u = 0; u < 4; ++u) cr[i + 32 * u] = encode8(v[u]);
  }
  for (; i < nvec; i += 32) cr[i] = encode8(xr[i]);
}

}  // namespace

cudaError_t launch_quantize_rowwise(const void* x, int64_t M, int64_t K, uint8_t* codes, float* scale,
                                    cudaStream_t stream) {
  const int64_t blocks = (M + kRowsPerCta - 1) / kRowsPerCta;
  const auto* xv = static_cast<const uint4*>(x);
  switch (K) {  // register-resident rows for the usual hidden sizes
    case 1024:
      quantize_rowwise_regs_kernel<4><<<static_cast<unsigned>(blocks), kRowsPerCta * 32, 0, stream>>>(xv, M, codes, scale);
      return cudaGetLastError();
    case 2048:
      quantize_rowwise_regs_kernel<8><<<static_cast<unsigned>(blocks), kRowsPerCta * 32, 0, stream>>>(xv, M, codes, scale);
      return cudaGetLastError();
    case 3072:
      quantize_rowwise_regs_kernel<12><<<static_cast<unsigned>(blocks), kRowsPerCta * 32, 0, stream>>>(xv, M, codes, scale);
      return cudaGetLastError();
    case 4096:
      quantize_rowwise_regs_kernel<16><<<static_cast<unsigned>(blocks), kRowsPerCta * 32, 0, stream>>>(xv, M, codes, scale);
      return cudaGetLastError();
    default:
      break;
  }
  quantize_rowwise_kernel<<<static_cast<unsigned>(blocks), kRowsPerCta * 32, 0, stream>>>(
      static_cast<const uint4*>(x), M, K, codes, scale);
  return cudaGetLastError();
}

}  // namespace nvfp4
