// Row-wise FP8 activation quantization ("BFL (fp8r / nvfp4)" diffusers doc,
// `fp8r` bullet: activations are quantized to E4M3 row by row at run time,
// next to E4M3 weights with one fp32 scale per row).  Per row:
//     s = fl(amax / 448)        q_i = E4M3_satfinite(fl(x_i / s))
// and a row of zeros gets s = 0 and the codes of +-0.
//
// Algorithmic traffic: 2 bytes read and 1 byte written per element, plus 4
// bytes per row; the per-element division is branch-free (div_fast) so that
// the arithmetic keeps up with it.  One warp per row, eight rows per CTA.
// Rows of 1024-4096 elements are held in registers (one read); longer rows
// take two passes, the second hitting L1/L2, each lane streaming 16-byte
// vectors, four in flight.
#include <type_traits>

#include "internal.h"

namespace nvfp4 {
namespace {

constexpr int kRowsPerCta = 8;

// Row scales whose quotients the branch-free division below gets right.
constexpr float kFastMin = 0x1p-90f;
constexpr float kFastMax = 0x1p100f;

// fl(a / d) for d in [2^-90, 2^100] and |a| <= 449 d, given y = RN(1/d):
// q1 = RN(a y) is within 1.5 ulp of a/d; one residual step (r = a - d q,
// exact with an FMA, q + r y) makes it faithful, and a second one rounds it
// correctly (Markstein's theorem, IBM J. Res. Dev. 34(1), 1990: y the
// correctly rounded reciprocal and q faithful give RN(q + r y) = RN(a/d)).
// Within that range of d every residual of a quotient >= 2^-11 is exact;
// smaller quotients (only reached by |a| that far below the row maximum) can
// miss their last bit when a residual underflows, but every value below 2^-10
// is an E4M3 zero, so the code is the same.  The sign is copied from a, since
// RN(-0 + +0) would turn -0 / d into +0.  Five FP operations and no branch,
// where the IEEE division takes a range check and a slow-path branch per
// element, which kept the kernel issue-bound at a third of HBM bandwidth.
__device__ __forceinline__ float div_fast(float a, float d, float y) {
  const float q1 = __fmul_rn(a, y);
  const float q2 = __fmaf_rn(__fmaf_rn(-q1, d, a), y, q1);
  const float q3 = __fmaf_rn(__fmaf_rn(-q2, d, a), y, q2);
  return __uint_as_float((__float_as_uint(q3) & 0x7fffffffu) | (__float_as_uint(a) & 0x80000000u));
}

// Eight bf16 values (one 16-byte vector) -> eight E4M3 codes, each
// E4M3_satfinite(fl(x / d)): the branch-free correctly rounded division when
// kFast (d in [kFastMin, kFastMax], y = RN(1/d)), else the IEEE division.
template <bool kFast>
__device__ __forceinline__ uint2 encode8_e4m3(const uint4& v, float d, float y) {
  const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                      bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
  float q[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if constexpr (kFast) q[j] = div_fast(f[j], d, y);
    else q[j] = __fdiv_rn(f[j], d);
  }
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint16_t lo, hi;
    // cvt puts its first source in the high byte: pass (odd, even)
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(q[4 * h + 1]), "f"(q[4 * h + 0]));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(q[4 * h + 3]), "f"(q[4 * h + 2]));
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
  if (d >= kFastMin && d <= kFastMax) {  // the same for the whole warp
    const float y = __frcp_rn(d);
#pragma unroll
    for (int u = 0; u < kNv; ++u) cr[lane + 32 * u] = encode8_e4m3<true>(v[u], d, y);
  } else {
#pragma unroll
    for (int u = 0; u < kNv; ++u) cr[lane + 32 * u] = encode8_e4m3<false>(v[u], d, 0.0f);
  }
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

  uint2* cr = reinterpret_cast<uint2*>(codes + row * K);
  auto encode_row = [&](auto fast, float y) {
    int64_t j = lane;
    for (; j + 96 < nvec; j += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = xr[j + 32 * u];
#pragma unroll
      for (int u = 0; u < 4; ++u) cr[j + 32 * u] = encode8_e4m3<decltype(fast)::value>(v[u], d, y);
    }
    for (; j < nvec; j += 32) cr[j] = encode8_e4m3<decltype(fast)::value>(xr[j], d, y);
  };
  if (d >= kFastMin && d <= kFastMax) encode_row(std::true_type{}, __frcp_rn(d));
  else encode_row(std::false_type{}, 0.0f);
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
