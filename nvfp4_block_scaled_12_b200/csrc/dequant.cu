// NVFP4 -> bf16 dequantization for the W4A16 path ("BFL (fp8r / nvfp4)"
// diffusers doc, section "Kernels", last paragraph: where the fused NVFP4
// kernels do not run, the weights are dequantized to the compute dtype on
// every forward pass and the layer runs as a regular linear, its activations
// left unquantized).  Per element: v = fl(fl(e2m1(q) * e4m3(s)) * g) (the
// first product is exact in fp32), then rounded to bf16.
//
// HBM-bound: 0.5 + 1/16 bytes in, 2 bytes out per element.
#include "internal.h"

namespace nvfp4 {
namespace {

// One thread per 16 bytes of codes (32 elements, two 16-element blocks):
// a 16-byte load, the blocks' two scale bytes as one 16-bit load (they are
// adjacent bytes of the same swizzled scale word), and 64 bytes of bf16 out.
// A warp reads 512 contiguous bytes of codes and writes 2 KB of output.
__global__ void __launch_bounds__(256) dequantize_kernel(const uint4* __restrict__ codes,
                                                         const uint8_t* __restrict__ sf, float g, int64_t K,
                                                         int64_t n_chunks, bool out32, uint8_t* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n_chunks) return;
  const int64_t per_row = K >> 5;
  const int64_t row = i / per_row, c = i % per_row;
  const uint4 w4 = codes[i];
  const uint16_t sp = *reinterpret_cast<const uint16_t*>(sf + sf_offset(row, 2 * c, K >> 6));
  const uint32_t words[4] = {w4.x, w4.y, w4.z, w4.w};
  uint32_t packed[16];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float s = e4m3_to_f32(u < 2 ? (sp & 0xFFu) : (sp >> 8));
    float f[8];
    e2m1x8_to_f32(words[u], f);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      packed[4 * u + e] = pack_bf16x2(__fmul_rn(__fmul_rn(f[2 * e], s), g), __fmul_rn(__fmul_rn(f[2 * e + 1], s), g));
  }
  uint8_t* o = out + (row * K + 32 * c) * 2;
  if (out32) {  // two whole 32-byte sectors
    st_global_v8(o, *reinterpret_cast<const uint32_t(*)[8]>(packed));
    st_global_v8(o + 32, *reinterpret_cast<const uint32_t(*)[8]>(packed + 8));
  } else {
#pragma unroll
    for (int v = 0; v < 4; ++v)
      reinterpret_cast<uint4*>(o)[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
  }
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* sf, float g, int64_t rows, int64_t K, void* out,
                              cudaStream_t stream) {
  const int64_t n_chunks = rows * (K >> 5);
  const int threads = 256;
  const int64_t blocks = (n_chunks + threads - 1) / threads;
  const bool out32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
  dequantize_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      reinterpret_cast<const uint4*>(codes), sf, g, K, n_chunks, out32, static_cast<uint8_t*>(out));
  return cudaGetLastError();
}

}  // namespace nvfp4
