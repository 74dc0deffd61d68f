// NVFP4 -> bf16 dequantization for the W4A16 path ("BFL (fp8r / nvfp4)"
// diffusers doc, section "Kernels", last paragraph: where the fused NVFP4
// kernels do not run, the weights are dequantized to the compute dtype on
// every forward pass and the layer runs as a regular linear, its activations
// left unquantized).  Per element: v = fl(fl(e2m1(q) * e4m3(s)) * g) (the
// first product is exact in fp32), then rounded to bf16.
//
// HBM-bound: 0.5 + 1/16 bytes in, 2 bytes out per element.  A thread turns
// 4-byte code words (8 elements) into 16-byte bf16 chunks, so that a warp's
// loads and stores are contiguous.
#include <cuda_fp16.h>

#include "internal.h"

namespace nvfp4 {
namespace {

// Eight E2M1 codes (a 32-bit word, element 2j in the low nibble of byte j)
// to fp32, exactly: the hardware conversion to f16 pairs, then f16 -> f32.
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t w, float (&f)[8]) {
  uint32_t h[4];
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&h[i]));
    f[2 * i] = v.x;      // low half: the byte's low nibble
    f[2 * i + 1] = v.y;
  }
}

constexpr int kWordsPerThread = 4;

__global__ void __launch_bounds__(256) dequantize_kernel(const uint32_t* __restrict__ codes,
                                                         const uint8_t* __restrict__ sf, float g, int64_t K,
                                                         int64_t row0, uint4* __restrict__ out) {
  // grid: x = chunks of 256 * kWordsPerThread code words of a row, y = row - row0.
  // Code word w of the row holds elements 8w .. 8w+7 and becomes 16 bytes of
  // bf16; the threads of a warp take consecutive words, so its loads and
  // stores are contiguous.
  const int64_t row = row0 + blockIdx.y;
  const int64_t words = K >> 3;
  const int64_t katoms = K >> 6;
  const uint32_t* cr = codes + row * words;
  uint4* orow = out + row * words;
#pragma unroll
  for (int u = 0; u < kWordsPerThread; ++u) {
    const int64_t w_idx = (static_cast<int64_t>(blockIdx.x) * kWordsPerThread + u) * 256 + threadIdx.x;
    if (w_idx < words) {
      const uint32_t w = cr[w_idx];
      const float s = e4m3_to_f32(sf[sf_offset(row, w_idx >> 1, katoms)]);
      float f[8];
      e2m1x8_to_f32(w, f);
      uint32_t packed[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        packed[e] = pack_bf16x2(__fmul_rn(__fmul_rn(f[2 * e], s), g), __fmul_rn(__fmul_rn(f[2 * e + 1], s), g));
      orow[w_idx] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
  }
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* sf, float g, int64_t rows, int64_t K, void* out,
                              cudaStream_t stream) {
  const int64_t words = K >> 3;
  const int64_t per_block = 256 * kWordsPerThread;
  for (int64_t r0 = 0; r0 < rows; r0 += 65535) {  // gridDim.y is at most 65535
    const int64_t nr = rows - r0 < 65535 ? rows - r0 : 65535;
    const dim3 grid(static_cast<unsigned>((words + per_block - 1) / per_block), static_cast<unsigned>(nr));
    dequantize_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint32_t*>(codes), sf, g, K, r0,
                                                  static_cast<uint4*>(out));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace nvfp4
