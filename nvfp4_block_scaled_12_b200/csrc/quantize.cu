// Runtime activation quantization bf16 -> NVFP4 and the scale-factor swizzle
// used for weight preparation ("BFL (fp8r / nvfp4)" diffusers doc, section
// "Kernels": `nvfp4_quantize` runs on the activations at every forward).
//
// The quantize kernel is HBM-bound (2 bytes read, 0.5 + 1/16 bytes written per
// element).  One persistent CTA per SM streams tiles of 128 rows x 64 columns
// (16 KB of bf16, the width of one scale atom) through 12 TMA stages in
// shared memory (192 KB in flight per SM), loaded with the 128-byte swizzle so
// that 32 threads reading 32 different rows hit distinct banks.  Sixteen
// consumer warps work independently, with no block-wide barrier: four groups
// of four warps take every fourth tile, and warp q of a group owns rows
// 32q..32q+31 of it.  Each group has its own three stages: an mbarrier wait
// only tells phases apart by parity, so a stage must be consumed in order by
// one consumer (a group running ahead on a shared ring could take a stage's
// previous phase for its next one).  A thread owns one row's 64 elements (four 16-element
// blocks), so it produces exactly one 4-byte word of the swizzled scale layout
// and 32 bytes of codes.
//
// The dynamic variant measures the per-tensor scale in the same launch: every
// CTA first takes max |x| over its own tiles (plain 16-byte loads), folds it
// into a grid-wide maximum and arrives on a grid-wide counter; the producer
// then starts the TMA ring at once (the tiles do not depend on the scale)
// while the consumers wait for the counter to reach the grid size, so the
// second read of a tile usually comes from L2.  The grid is launched
// cooperatively (every CTA resident), and the wait is bounded.
#include "internal.h"

namespace nvfp4 {

namespace {

constexpr int kQRows = 128;
constexpr int kQCols = 64;
constexpr int kQGroups = 4;                         // tiles processed concurrently per CTA
constexpr int kQStagesPerGroup = 3;
constexpr int kQStages = kQGroups * kQStagesPerGroup;
constexpr int kQConsumerWarps = 4 * kQGroups;       // 4 quarter-warps per tile
constexpr int kQThreads = (kQConsumerWarps + 1) * 32;  // + one producer warp
constexpr uint32_t kQTileBytes = kQRows * kQCols * 2;  // 16 KB of bf16
constexpr uint32_t kQOffBar = kQStages * kQTileBytes;
constexpr uint32_t kQOffMax = kQOffBar + 2 * kQStages * 8 + 16;  // per-warp maxima of the amax pass
constexpr uint32_t kQSmemBytes = kQOffMax + 32 * 4 + 1024;        // + alignment slack

template <bool kDynamic, bool kMx>
__global__ void __launch_bounds__(kQThreads, 1)
    quantize_kernel(const __grid_constant__ CUtensorMap tmap_x, int64_t M, int64_t K, float g,
                    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, int64_t tiles_k, int64_t n_tiles,
                    unsigned* fault_word, DynamicScaleArgs dyn) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQOffBar);
  uint64_t* empty = full + kQStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kQStages);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);  // the four quarter-warps of the tile
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  unsigned fault = 0u;
  // This CTA's tiles are blockIdx.x + j * gridDim.x, j = 0 .. my_tiles-1.
  // The ring carries a sequence of n_seq loads, entry jj = 4i + g going to
  // consumer group g, stage g * kQStagesPerGroup + i % 3.  The static variant
  // loads each tile once (entry jj = tile j).  The dynamic one loads them
  // twice: entries 0 .. my_tiles-1 for the amax pass in order, then the
  // quantize pass in reverse order, so that its first tiles are the ones
  // read last (the likeliest to still be in L2).
  const int64_t my_tiles = n_tiles > blockIdx.x ? (n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const int64_t n_seq = kDynamic ? 2 * my_tiles : my_tiles;
  auto seq_tile = [&](int64_t jj) -> int64_t {
    const int64_t j = (!kDynamic || jj < my_tiles) ? jj : 2 * my_tiles - 1 - jj;
    return blockIdx.x + j * gridDim.x;
  };

  if (warp == kQConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmap_x);
      int64_t jj = 0;
      for (; jj < n_seq; ++jj) {
        const int64_t i = jj / kQGroups;
        const int stage = static_cast<int>(jj % kQGroups) * kQStagesPerGroup + static_cast<int>(i % kQStagesPerGroup);
        const uint32_t phase = static_cast<uint32_t>((i / kQStagesPerGroup) & 1);
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
          fault = kFaultProducerWait;
          break;
        }
        const int64_t tile = seq_tile(jj);
        mbar_arrive_expect_tx(&full[stage], kQTileBytes);
        tma_load_2d(smem + stage * kQTileBytes, &tmap_x, &full[stage], static_cast<int32_t>((tile % tiles_k) * kQCols),
                    static_cast<int32_t>((tile / tiles_k) * kQRows));
      }
      if (fault != 0u) {
        *abort_flag = 1;
        // let the copies already issued (the last kQStages entries) land
        for (int64_t k = jj - 1; k >= 0 && k >= jj - kQStages; --k) {
          const int64_t i = k / kQGroups;
          const int stage = static_cast<int>(k % kQGroups) * kQStagesPerGroup + static_cast<int>(i % kQStagesPerGroup);
          mbar_wait(&full[stage], static_cast<uint32_t>((i / kQStagesPerGroup) & 1), nullptr);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int group = warp >> 2;
    const int q = warp & 3;         // rows 32q..32q+31 of each tile
    const int rloc = q * 32 + lane; // this thread's row inside the tile
    float amax_part = 0.0f;         // dynamic: max |x| over the rows this thread saw
    bool have_scale = !kDynamic;
    float d6 = __fmul_rn(6.0f, g);
    const int64_t katoms = K >> 6;
    const int64_t mx_katoms = (K / 32 + 3) / 4;  // MXFP8 scale atoms per 128-row block

    // Dynamic variant, once per consumer warp (every one of the 16 reaches
    // it exactly once, so the named barriers below always complete): fold
    // this CTA's maximum into the grid-wide one, wait (bounded) until every
    // CTA has, and derive g.
    auto grid_scale = [&]() {
      float m = amax_part;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      volatile float* warp_max = reinterpret_cast<volatile float*>(smem + kQOffMax);
      if (lane == 0) warp_max[warp] = m;
      named_barrier_sync(1, kQConsumerWarps * 32);
      if (warp == 0 && lane == 0) {
        for (int w = 1; w < kQConsumerWarps; ++w) m = fmaxf(m, warp_max[w]);
        // |x| >= 0, so the float's bit pattern orders like the value
        atomicMax(dyn.scratch, __float_as_uint(m));
        __threadfence();
        atomicAdd(dyn.scratch + 1, 1u);
        const uint64_t t0 = global_timer_ns();
        uint32_t arrived;
        while ((arrived = ld_acquire_gpu(dyn.scratch + 1)) < gridDim.x) {
          if (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs) break;
          __nanosleep(64);
        }
        warp_max[kQConsumerWarps] = arrived >= gridDim.x ? __uint_as_float(ld_acquire_gpu(dyn.scratch)) : -1.0f;
      }
      named_barrier_sync(1, kQConsumerWarps * 32);
      const float amax = warp_max[kQConsumerWarps];
      if (amax < 0.0f) {
        fault = kFaultGridWait;
        *abort_flag = 1;
        return false;
      }
      // g = fl(amax / 2688) clamped into [2^-64, 2^64]; 0 for an all-zero tensor
      g = amax > 0.0f ? fminf(fmaxf(__fdiv_rn(amax, 2688.0f), 0x1p-64f), 0x1p64f) : 0.0f;
      d6 = __fmul_rn(6.0f, g);
      if (blockIdx.x == 0 && warp == 0 && lane == 0) {
        dyn.scale_out[0] = amax;
        dyn.scale_out[1] = g;
      }
      return true;
    };

    for (int64_t jj = group; jj < n_seq; jj += kQGroups) {
      if (!have_scale && jj >= my_tiles) {
        have_scale = true;
        if (!grid_scale()) break;
      }
      const int64_t i = jj / kQGroups;
      const int stage = group * kQStagesPerGroup + static_cast<int>(i % kQStagesPerGroup);
      const uint32_t phase = static_cast<uint32_t>((i / kQStagesPerGroup) & 1);
      const bool got = mbar_wait(&full[stage], phase, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        fault = kFaultEpilogueWait;
        break;
      }
      // row rloc: 128 bytes, 16-byte chunk c stored at chunk c ^ (rloc % 8)
      const uint8_t* row_s = smem + stage * kQTileBytes + rloc * 128;
      uint4 v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] = *reinterpret_cast<const uint4*>(row_s + ((c ^ (rloc & 7)) * 16));
      // The stage is refilled by TMA (the async proxy) once all four warps
      // have arrived: order this thread's shared-memory reads before that
      // write, or a load still in flight can return the next tile's data.
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);  // this quarter is in registers

      if (kDynamic && jj < my_tiles) {
        // amax pass (rows past M arrived zero-filled)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          amax_part = fmaxf(amax_part, fmaxf(fmaxf(fabsf(bf16_lo(v[c].x)), fabsf(bf16_hi(v[c].x))),
                                             fmaxf(fabsf(bf16_lo(v[c].y)), fabsf(bf16_hi(v[c].y)))));
          amax_part = fmaxf(amax_part, fmaxf(fmaxf(fabsf(bf16_lo(v[c].z)), fabsf(bf16_hi(v[c].z))),
                                             fmaxf(fabsf(bf16_lo(v[c].w)), fabsf(bf16_hi(v[c].w)))));
        }
        continue;
      }

      const int64_t tile = seq_tile(jj);
      const int64_t row = (tile / tiles_k) * kQRows + rloc;
      const int64_t katom = tile % tiles_k;  // 64-column group of the tile
      if constexpr (kMx) {
        // MXFP8: two 32-element blocks -> 64 E4M3 bytes and two E8M0 scale
        // bytes (scale columns 2*katom, 2*katom + 1: half of a 4-byte word)
        uint32_t sfh = 0u;
        uint32_t cw[16];
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          float f[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 u = v[4 * blk + c];
            f[8 * c + 0] = bf16_lo(u.x);
            f[8 * c + 1] = bf16_hi(u.x);
            f[8 * c + 2] = bf16_lo(u.y);
            f[8 * c + 3] = bf16_hi(u.y);
            f[8 * c + 4] = bf16_lo(u.z);
            f[8 * c + 5] = bf16_hi(u.z);
            f[8 * c + 6] = bf16_lo(u.w);
            f[8 * c + 7] = bf16_hi(u.w);
          }
          uint32_t w[8];
          sfh |= quantize_mx_block32(f, w) << (8 * blk);
#pragma unroll
          for (int i = 0; i < 8; ++i) cw[8 * blk + i] = w[i];
        }
        if (row < M) {
          uint8_t* crow = codes + row * K + katom * 64;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(crow + 16 * c) = make_uint4(cw[4 * c], cw[4 * c + 1], cw[4 * c + 2], cw[4 * c + 3]);
        }
        // rows past M: zero-filled data, amax 0, scale bytes 0 (the padding).
        // The last tile of a K that is 64 mod 128 also zeroes the two padding
        // columns of its word.
        if ((katom & 1) == 0 && katom == tiles_k - 1)
          *reinterpret_cast<uint32_t*>(sf + sf_offset(row, katom * 2, mx_katoms)) = sfh;
        else
          *reinterpret_cast<uint16_t*>(sf + sf_offset(row, katom * 2, mx_katoms)) = static_cast<uint16_t>(sfh);
        continue;
      }
      uint32_t sfw = 0u;
      uint32_t cw[8];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        float f[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 u = v[2 * b + h];
          f[8 * h + 0] = bf16_lo(u.x);
          f[8 * h + 1] = bf16_hi(u.x);
          f[8 * h + 2] = bf16_lo(u.y);
          f[8 * h + 3] = bf16_hi(u.y);
          f[8 * h + 4] = bf16_lo(u.z);
          f[8 * h + 5] = bf16_hi(u.z);
          f[8 * h + 6] = bf16_lo(u.w);
          f[8 * h + 7] = bf16_hi(u.w);
        }
        if (kDynamic && g == 0.0f) {  // all-zero tensor: zero codes and scales
          cw[2 * b] = 0u;
          cw[2 * b + 1] = 0u;
        } else {
          sfw |= quantize_block16(f, g, d6, cw[2 * b], cw[2 * b + 1]) << (8 * b);
        }
      }
      if (row < M) {
        uint8_t* crow = codes + row * (K >> 1) + katom * 32;
        *reinterpret_cast<uint4*>(crow) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        *reinterpret_cast<uint4*>(crow + 16) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
      }
      // rows past M belong to the zero padding of the scale buffer (their
      // data was zero-filled by the TMA, so sfw == 0)
      *reinterpret_cast<uint32_t*>(sf + sf_offset(row, katom * 4, katoms)) = sfw;
    }
    // a group whose entries ended inside the amax pass (or that gave up
    // there) still takes part in the CTA's scale exchange
    if (!have_scale) grid_scale();
    if (fault != 0u) *abort_flag = 1;
  }
  if (fault != 0u && lane == 0 && fault_word != nullptr) atomicOr(fault_word, fault);
  __syncthreads();
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

cudaError_t launch_quantize(const CUtensorMap& tmap_x, int64_t M, int64_t K, float g, uint8_t* codes, uint8_t* sf,
                            cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t tiles_m = (M + kQRows - 1) / kQRows;
  const int64_t tiles_k = (K + kQCols - 1) / kQCols;
  const int64_t n_tiles = tiles_m * tiles_k;
  const int grid = static_cast<int>(n_tiles < dev.num_sms ? n_tiles : dev.num_sms);
  cudaError_t err =
      cudaFuncSetAttribute(quantize_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmemBytes);
  if (err != cudaSuccess) return err;
  quantize_kernel<false, false><<<grid, kQThreads, kQSmemBytes, stream>>>(tmap_x, M, K, g, codes, sf, tiles_k, n_tiles,
                                                                   dev.fault, DynamicScaleArgs{});
  return cudaGetLastError();
}

cudaError_t launch_quantize_mxfp8(const CUtensorMap& tmap_x, int64_t M, int64_t K, uint8_t* codes, uint8_t* sf,
                                  cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t tiles_m = (M + kQRows - 1) / kQRows;
  const int64_t tiles_k = (K + kQCols - 1) / kQCols;
  const int64_t n_tiles = tiles_m * tiles_k;
  const int grid = static_cast<int>(n_tiles < dev.num_sms ? n_tiles : dev.num_sms);
  auto kernel = quantize_kernel<false, true>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmemBytes);
  if (err != cudaSuccess) return err;
  kernel<<<grid, kQThreads, kQSmemBytes, stream>>>(tmap_x, M, K, 0.0f, codes, sf, tiles_k, n_tiles, dev.fault,
                                                   DynamicScaleArgs{});
  return cudaGetLastError();
}

cudaError_t launch_quantize_dynamic(const CUtensorMap& tmap_x, const void* x, int64_t M, int64_t K, uint8_t* codes,
                                    uint8_t* sf, float* scale_out, uint32_t* scratch, cudaStream_t stream,
                                    const DeviceInfo& dev) {
  const int64_t tiles_m = (M + kQRows - 1) / kQRows;
  const int64_t tiles_k = (K + kQCols - 1) / kQCols;
  const int64_t n_tiles = tiles_m * tiles_k;
  const int grid = static_cast<int>(n_tiles < dev.num_sms ? n_tiles : dev.num_sms);
  auto kernel = quantize_kernel<true, false>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmemBytes);
  if (err != cudaSuccess) return err;
  // the grid-wide maximum and the arrival counter start at zero
  err = cudaMemsetAsync(scratch, 0, kDynamicScratchBytes, stream);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = kQSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid-wide wait can complete
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const DynamicScaleArgs dyn{static_cast<const uint8_t*>(x), scratch, scale_out};
  err = cudaLaunchKernelEx(&cfg, kernel, tmap_x, M, K, 0.0f, codes, sf, tiles_k, n_tiles, dev.fault, dyn);
  if (err != cudaSuccess) return err;
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
