// Runtime activation quantization bf16 -> NVFP4 and the scale-factor swizzle
// used for weight preparation ("BFL (fp8r / nvfp4)" diffusers doc, section
// "Kernels": `nvfp4_quantize` runs on the activations at every forward).
//
// The quantize kernel is HBM-bound (2 bytes read, 0.5 + 1/16 bytes written per
// element).  Each CTA owns a 128-row x 128-column tile: the scales of such a
// tile are exactly two 512-byte atoms of the swizzled scale layout, so they
// are assembled in shared memory and written with full 16-byte stores.
// Every thread issues all eight of its 16-byte loads before doing any math to
// keep enough bytes in flight per SM.
#include "internal.h"

namespace nvfp4 {

namespace {

constexpr int kQRows = 128;
constexpr int kQCols = 128;
constexpr int kQThreads = 256;
constexpr int kQLoads = kQRows * kQCols / 8 / kQThreads;  // 16-byte loads per thread (8)

__global__ void __launch_bounds__(kQThreads) quantize_kernel(const __nv_bfloat16* __restrict__ x, int64_t M,
                                                             int64_t K, float g, uint8_t* __restrict__ codes,
                                                             uint8_t* __restrict__ sf, int64_t tiles_k,
                                                             int64_t n_tiles) {
  __shared__ __align__(16) uint8_t sf_tile[2 * 512];
  const int tid = threadIdx.x;
  const int cg = tid & 15;    // 8-column group inside the tile
  const int rsub = tid >> 4;  // first row of this thread (0..15), then +16 per load
  const float d6 = __fmul_rn(6.0f, g);
  const int64_t katoms = K >> 6;

  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t row0 = (tile / tiles_k) * kQRows;
    const int64_t col0 = (tile % tiles_k) * kQCols;
    const int64_t col = col0 + cg * 8;
    const bool col_ok = col < K;  // K % 64 == 0: 64-column halves are all-in or all-out

    uint4 v[kQLoads];
#pragma unroll
    for (int i = 0; i < kQLoads; ++i) {
      const int64_t row = row0 + rsub + 16 * i;
      v[i] = (row < M && col_ok) ? ld_stream_v4(x + row * K + col) : make_uint4(0u, 0u, 0u, 0u);
    }

#pragma unroll
    for (int i = 0; i < kQLoads; ++i) {
      const int rloc = rsub + 16 * i;
      const int64_t row = row0 + rloc;
      float f[8] = {bf16_lo(v[i].x), bf16_hi(v[i].x), bf16_lo(v[i].y), bf16_hi(v[i].y),
                    bf16_lo(v[i].z), bf16_hi(v[i].z), bf16_lo(v[i].w), bf16_hi(v[i].w)};
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));  // partner holds the other 8
      const uint32_t s = e4m3_from_f32_satfinite(__fdiv_rn(amax, d6));
      uint32_t word = 0u;
      if (s != 0u) {
        const float r = __frcp_rn(__fmul_rn(e4m3_to_f32(s), g));
        word = e2m1x8_from_f32(__fmul_rn(f[0], r), __fmul_rn(f[1], r), __fmul_rn(f[2], r),
                               __fmul_rn(f[3], r), __fmul_rn(f[4], r), __fmul_rn(f[5], r),
                               __fmul_rn(f[6], r), __fmul_rn(f[7], r));
      }
      if (row < M && col_ok) *reinterpret_cast<uint32_t*>(codes + row * (K >> 1) + (col >> 1)) = word;
      if ((cg & 1) == 0) {
        const int c = cg >> 1;  // scale column inside the tile, 0..7
        sf_tile[(c >> 2) * 512 + (rloc & 31) * 16 + (rloc >> 5) * 4 + (c & 3)] = static_cast<uint8_t>(s);
      }
    }
    __syncthreads();
    if (tid < 64) {
      const int atom = tid >> 5;
      const int64_t katom = (col0 >> 6) + atom;
      if (katom < katoms) {
        const uint4 w = *reinterpret_cast<const uint4*>(sf_tile + tid * 16);
        *reinterpret_cast<uint4*>(sf + ((row0 >> 7) * katoms + katom) * 512 + (tid & 31) * 16) = w;
      }
    }
    __syncthreads();
  }
}

// One thread per 16-byte line of an atom: gathers rows r, r+32, r+64, r+96
// x 4 scale columns of the row-major input.
__global__ void swizzle_sf_kernel(const uint8_t* __restrict__ sf_lin, int64_t rows, int64_t cols,
                                  int64_t katoms, int64_t n_lines, uint8_t* __restrict__ out) {
  const int64_t line = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (line >= n_lines) return;
  const int64_t atom = line >> 5;
  const int l = static_cast<int>(line & 31);
  const int64_t rb = atom / katoms, cb = atom % katoms;
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int64_t r = rb * 128 + q * 32 + l;
    uint32_t word = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t c = cb * 4 + j;
      if (r < rows && c < cols) word |= static_cast<uint32_t>(sf_lin[r * cols + c]) << (8 * j);
    }
    w[q] = word;
  }
  *reinterpret_cast<uint4*>(out + line * 16) = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, float g, uint8_t* codes, uint8_t* sf,
                            cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t tiles_m = (M + kQRows - 1) / kQRows;
  const int64_t tiles_k = (K + kQCols - 1) / kQCols;
  const int64_t n_tiles = tiles_m * tiles_k;
  const int64_t resident = static_cast<int64_t>(dev.num_sms) * 8;
  const int grid = static_cast<int>(n_tiles < resident ? n_tiles : resident);
  quantize_kernel<<<grid, kQThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), M, K, g, codes, sf,
                                                  tiles_k, n_tiles);
  return cudaGetLastError();
}

cudaError_t launch_swizzle_sf(const uint8_t* sf_lin, int64_t rows, int64_t k, uint8_t* out,
                              cudaStream_t stream) {
  const int64_t katoms = k >> 6;
  const int64_t n_lines = ((rows + 127) / 128) * katoms * 32;
  const int threads = 256;
  const int64_t blocks = (n_lines + threads - 1) / threads;
  swizzle_sf_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(sf_lin, rows, k >> 4, katoms,
                                                                           n_lines, out);
  return cudaGetLastError();
}

}  // namespace nvfp4
