// Runtime activation quantization bf16 -> NVFP4 and the scale-factor swizzle
// used for weight preparation ("BFL (fp8r / nvfp4)" diffusers doc, section
// "Kernels": `nvfp4_quantize` runs on the activations at every forward).
//
// The quantize kernel is HBM-bound (2 bytes read, 0.5 + 1/16 bytes written per
// element).  One persistent CTA per SM streams tiles of 256 rows x 64 columns
// (32 KB of bf16, the width of one scale atom) through 6 TMA stages in shared
// memory (192 KB in flight per SM), loaded with the 128-byte swizzle so that
// 32 threads reading 32 different rows hit distinct banks.  24 consumer warps
// work independently, with no block-wide barrier: three groups of eight warps
// take every third tile, and warp q of a group owns rows 32q..32q+31 of it.
// Each group has its own two stages: an mbarrier wait only tells phases apart
// by parity, so a stage must be consumed in order by one consumer (a group
// running ahead on a shared ring could take a stage's previous phase for its
// next one).  A thread owns one row's 64 elements (four 16-element blocks),
// so it produces exactly one 4-byte word of the swizzled scale layout and 32
// bytes of codes, written as one whole 32-byte sector.  The consumers' work,
// not HBM, set the pace with 16 warps; 24 keep more rows in flight.
//
// The dynamic variant measures the per-tensor scale in the same launch: every
// CTA first takes max |x| over its own tiles (plain 16-byte loads), folds it
// into a grid-wide maximum and arrives on a grid-wide counter; the producer
// then starts the TMA ring at once (the tiles do not depend on the scale)
// while the consumers wait for the counter to reach the grid size, so the
// second read of a tile usually comes from L2.  The grid is launched
// cooperatively (every CTA resident), and the wait is bounded (by default
// kWaitLimitNs; a test of the time-out path shortens it and adds arrivals that
// never come, see nvfp4_testing_set_grid_wait).
#include "internal.h"

namespace nvfp4 {

namespace {

// Tile shape and ring of one launch: 128-row tiles (four groups of four
// warps, three stages each) keep enough tiles per CTA in flight for small
// tensors; 256-row tiles (three groups of eight warps, two stages each) put
// 24 consumer warps to work on large ones.  Both hold 192 KB per SM.
template <int kRows>
struct QCfg {
  static constexpr int kTileRows = kRows;
  static constexpr int kCols = 64;
  static constexpr int kGroups = kRows == 256 ? 3 : 4;       // tiles processed concurrently per CTA
  static constexpr int kStagesPerGroup = kRows == 256 ? 2 : 3;
  static constexpr int kStages = kGroups * kStagesPerGroup;
  static constexpr int kWarpsPerTile = kRows / 32;           // one row per thread
  static constexpr int kConsumerWarps = kWarpsPerTile * kGroups;
  static constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
  static constexpr uint32_t kTileBytes = kRows * kCols * 2;
  static constexpr uint32_t kOffBar = kStages * kTileBytes;
  static constexpr uint32_t kOffMax = kOffBar + 2 * kStages * 8 + 16;  // per-warp maxima of the amax pass
  static constexpr uint32_t kOffRtab = (kOffMax + (kConsumerWarps + 1) * 4 + 15) & ~15u;  // 128 block reciprocals
  static constexpr uint32_t kSmemBytes = kOffRtab + 128 * 4 + 1024;  // + alignment slack
  static_assert(kRows == 128 || kRows == 256, "tile rows");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

template <bool kDynamic, bool kMx, int kRows>
__global__ void __launch_bounds__(QCfg<kRows>::kThreads, 1)
    quantize_kernel(const __grid_constant__ CUtensorMap tmap_x, int64_t M, int64_t K, float g,
                    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, int64_t tiles_k, int64_t n_tiles,
                    unsigned* fault_word, DynamicScaleArgs dyn) {
  using Q = QCfg<kRows>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Q::kOffBar);
  uint64_t* empty = full + Q::kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + Q::kStages);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < Q::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], Q::kWarpsPerTile);  // every consumer warp of the tile
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  unsigned fault = 0u;
  // This CTA's tiles are blockIdx.x + j * gridDim.x, j = 0 .. my_tiles-1.
  // The ring carries a sequence of n_seq loads, entry jj = 4i + g going to
  // consumer group g, stage g * Q::kStagesPerGroup + i % 3.  The static variant
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

  if (warp == Q::kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmap_x);
      int64_t jj = 0;
      for (; jj < n_seq; ++jj) {
        const int64_t i = jj / Q::kGroups;
        const int stage = static_cast<int>(jj % Q::kGroups) * Q::kStagesPerGroup + static_cast<int>(i % Q::kStagesPerGroup);
        const uint32_t phase = static_cast<uint32_t>((i / Q::kStagesPerGroup) & 1);
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
          fault = kFaultProducerWait;
          break;
        }
        const int64_t tile = seq_tile(jj);
        mbar_arrive_expect_tx(&full[stage], Q::kTileBytes);
        tma_load_2d(smem + stage * Q::kTileBytes, &tmap_x, &full[stage], static_cast<int32_t>((tile % tiles_k) * Q::kCols),
                    static_cast<int32_t>((tile / tiles_k) * Q::kTileRows));
      }
      if (fault != 0u) *abort_flag = 1;
      // Every copy this warp issued (the last Q::kStages entries at most) has
      // landed before the CTA may exit, also when the consumers gave up before
      // taking them (normally they have taken them all and these waits return
      // at once).
      for (int64_t k = jj - 1; k >= 0 && k >= jj - Q::kStages; --k) {
        const int64_t i = k / Q::kGroups;
        const int stage = static_cast<int>(k % Q::kGroups) * Q::kStagesPerGroup + static_cast<int>(i % Q::kStagesPerGroup);
        mbar_wait(&full[stage], static_cast<uint32_t>((i / Q::kStagesPerGroup) & 1), nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int group = warp / Q::kWarpsPerTile;
    const int q = warp % Q::kWarpsPerTile;  // rows 32q..32q+31 of each tile
    const int rloc = q * 32 + lane;       // this thread's row inside the tile
    const int64_t m_padded = (M + 127) & ~int64_t(127);  // rows of the scale buffer
    float amax_part = 0.0f;         // dynamic: max |x| over the rows this thread saw
    bool have_scale = !kDynamic;
    // rtab[s] = RN(1 / fl(e4m3(s) g)): the block reciprocal for every scale
    // code, filled by the consumers once g is known
    float* rtab = reinterpret_cast<float*>(smem + Q::kOffRtab);
    auto fill_rtab = [&]() {
      const int ct = warp * 32 + lane;
      if (ct < 128) rtab[ct] = (ct >= 1 && ct <= 126) ? __frcp_rn(__fmul_rn(e4m3_to_f32(ct), g)) : 0.0f;
      named_barrier_sync(1, Q::kConsumerWarps * 32);
    };
    if (!kDynamic && dyn.amax_in != nullptr) {
      // one-pass variant: the scale comes from an amax measured elsewhere
      const float amax = *dyn.amax_in;
      g = scale_from_amax(amax);
      if (blockIdx.x == 0 && warp == 0 && lane == 0) {
        dyn.scale_out[0] = amax;
        dyn.scale_out[1] = g;
      }
    }
    float d6 = __fmul_rn(6.0f, g);
    float rd6 = __frcp_rn(d6);
    if (!kDynamic && !kMx) fill_rtab();
    const int64_t katoms = K >> 6;
    // 32-byte aligned codes rows (the usual case: every row starts at a
    // multiple of 32 bytes when the buffer does) take one 32-byte store
    const bool codes32 = (reinterpret_cast<uintptr_t>(codes) & 31u) == 0;
    const int64_t mx_katoms = (K / 32 + 3) / 4;  // MXFP8 scale atoms per 128-row block

    // Dynamic variant, once per consumer warp (every one of the 16 reaches
    // it exactly once, so the named barriers below always complete): fold
    // this CTA's maximum into the grid-wide one, wait (bounded) until every
    // CTA has, and derive g.
    auto grid_scale = [&]() {
      float m = amax_part;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      volatile float* warp_max = reinterpret_cast<volatile float*>(smem + Q::kOffMax);
      if (lane == 0) warp_max[warp] = m;
      named_barrier_sync(1, Q::kConsumerWarps * 32);
      if (warp == 0 && lane == 0) {
        for (int w = 1; w < Q::kConsumerWarps; ++w) m = fmaxf(m, warp_max[w]);
        // |x| >= 0, so the float's bit pattern orders like the value
        atomicMax(dyn.scratch, __float_as_uint(m));
        __threadfence();
        atomicAdd(dyn.scratch + 1, 1u);
        const uint64_t t0 = global_timer_ns();
        uint32_t arrived;
        while ((arrived = ld_acquire_gpu(dyn.scratch + 1)) < dyn.expect) {
          if (*abort_flag || global_timer_ns() - t0 > dyn.wait_limit_ns) break;
          __nanosleep(64);
        }
        warp_max[Q::kConsumerWarps] = arrived >= dyn.expect ? __uint_as_float(ld_acquire_gpu(dyn.scratch)) : -1.0f;
      }
      named_barrier_sync(1, Q::kConsumerWarps * 32);
      const float amax = warp_max[Q::kConsumerWarps];
      if (amax < 0.0f) {
        fault = kFaultGridWait;
        *abort_flag = 1;
        return false;
      }
      g = scale_from_amax(amax);
      d6 = __fmul_rn(6.0f, g);
      rd6 = __frcp_rn(d6);
      fill_rtab();
      if (blockIdx.x == 0 && warp == 0 && lane == 0) {
        dyn.scale_out[0] = amax;
        dyn.scale_out[1] = g;
      }
      return true;
    };

    for (int64_t jj = group; jj < n_seq; jj += Q::kGroups) {
      if (!have_scale && jj >= my_tiles) {
        have_scale = true;
        if (!grid_scale()) break;
      }
      const int64_t i = jj / Q::kGroups;
      const int stage = group * Q::kStagesPerGroup + static_cast<int>(i % Q::kStagesPerGroup);
      const uint32_t phase = static_cast<uint32_t>((i / Q::kStagesPerGroup) & 1);
      const bool got = mbar_wait(&full[stage], phase, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        fault = kFaultEpilogueWait;
        break;
      }
      // row rloc: 128 bytes, 16-byte chunk c stored at chunk c ^ (rloc % 8)
      const uint8_t* row_s = smem + stage * Q::kTileBytes + rloc * 128;
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
      const int64_t row = (tile / tiles_k) * Q::kTileRows + rloc;
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
          if (codes32) {
            st_global_v8(crow, *reinterpret_cast<const uint32_t(*)[8]>(cw));
            st_global_v8(crow + 32, *reinterpret_cast<const uint32_t(*)[8]>(cw + 8));
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4*>(crow + 16 * c) = make_uint4(cw[4 * c], cw[4 * c + 1], cw[4 * c + 2], cw[4 * c + 3]);
          }
        }
        // rows past M: zero-filled data, amax 0, scale bytes 0 (the padding).
        // The last tile of a K that is 64 mod 128 also zeroes the two padding
        // columns of its word.
        if (row < m_padded) {
          if ((katom & 1) == 0 && katom == tiles_k - 1)
            *reinterpret_cast<uint32_t*>(sf + sf_offset(row, katom * 2, mx_katoms)) = sfh;
          else
            *reinterpret_cast<uint16_t*>(sf + sf_offset(row, katom * 2, mx_katoms)) = static_cast<uint16_t>(sfh);
        }
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
        if (g == 0.0f) {  // measured scale of an all-zero tensor: zero codes and scales
          cw[2 * b] = 0u;
          cw[2 * b + 1] = 0u;
        } else {
          sfw |= quantize_block16_tab(f, d6, rd6, rtab, cw[2 * b], cw[2 * b + 1]) << (8 * b);
        }
      }
      if (row < M) {
        uint8_t* crow = codes + row * (K >> 1) + katom * 32;
        if (codes32)  // one full 32-byte sector per thread
          st_global_v8(crow, cw);
        else {
          *reinterpret_cast<uint4*>(crow) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
          *reinterpret_cast<uint4*>(crow + 16) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
        }
      }
      // rows past M up to the next multiple of 128 are the zero padding of
      // the scale buffer (their data was zero-filled by the TMA, so sfw == 0)
      if (row < m_padded) *reinterpret_cast<uint32_t*>(sf + sf_offset(row, katom * 4, katoms)) = sfw;
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

int quantize_tile_rows(int64_t M, int64_t K, int num_sms) {
  // 256-row tiles once every CTA gets at least eight of them
  const int64_t tiles256 = ((M + 255) / 256) * ((K + 63) / 64);
  return tiles256 >= 8 * static_cast<int64_t>(num_sms) ? 256 : 128;
}

namespace {

template <bool kDynamic, bool kMx, int kRows>
cudaError_t launch_q(const CUtensorMap& tmap_x, const void* x, int64_t M, int64_t K, float g, uint8_t* codes,
                     uint8_t* sf, float* scale_out, uint32_t* scratch, const GridWaitSettings& wait,
                     cudaStream_t stream, const DeviceInfo& dev) {
  using Q = QCfg<kRows>;
  const int64_t tiles_m = (M + kRows - 1) / kRows;
  const int64_t tiles_k = (K + Q::kCols - 1) / Q::kCols;
  const int64_t n_tiles = tiles_m * tiles_k;
  const int grid = static_cast<int>(n_tiles < dev.num_sms ? n_tiles : dev.num_sms);
  auto kernel = quantize_kernel<kDynamic, kMx, kRows>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Q::kSmemBytes);
  if (err != cudaSuccess) return err;
  if (!kDynamic) {
    kernel<<<grid, Q::kThreads, Q::kSmemBytes, stream>>>(tmap_x, M, K, g, codes, sf, tiles_k, n_tiles, dev.fault,
                                                         DynamicScaleArgs{});
    return cudaGetLastError();
  }
  // the grid-wide maximum and the arrival counter start at zero
  err = cudaMemsetAsync(scratch, 0, kDynamicScratchBytes, stream);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(Q::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Q::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid-wide wait can complete
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const DynamicScaleArgs dyn{static_cast<const uint8_t*>(x), scratch, scale_out, wait.limit_ns,
                             static_cast<uint32_t>(grid) + wait.extra_arrivals};
  err = cudaLaunchKernelEx(&cfg, kernel, tmap_x, M, K, 0.0f, codes, sf, tiles_k, n_tiles, dev.fault, dyn);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

// The one-pass quantize with g from a device amax: the static kernel's grid.
template <int kRows>
cudaError_t launch_q_amax(const CUtensorMap& tmap_x, int64_t M, int64_t K, uint8_t* codes, uint8_t* sf,
                          const DynamicScaleArgs& dyn, cudaStream_t stream, const DeviceInfo& dev) {
  using Q = QCfg<kRows>;
  const int64_t tiles_m = (M + kRows - 1) / kRows;
  const int64_t tiles_k = (K + Q::kCols - 1) / Q::kCols;
  const int64_t n_tiles = tiles_m * tiles_k;
  const int grid = static_cast<int>(n_tiles < dev.num_sms ? n_tiles : dev.num_sms);
  auto kernel = quantize_kernel<false, false, kRows>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Q::kSmemBytes);
  if (err != cudaSuccess) return err;
  kernel<<<grid, Q::kThreads, Q::kSmemBytes, stream>>>(tmap_x, M, K, 0.0f, codes, sf, tiles_k, n_tiles, dev.fault, dyn);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const CUtensorMap& tmap_x, int tile_rows, int64_t M, int64_t K, float g, uint8_t* codes,
                            uint8_t* sf, cudaStream_t stream, const DeviceInfo& dev) {
  const GridWaitSettings none;
  return tile_rows == 256 ? launch_q<false, false, 256>(tmap_x, nullptr, M, K, g, codes, sf, nullptr, nullptr, none, stream, dev)
                          : launch_q<false, false, 128>(tmap_x, nullptr, M, K, g, codes, sf, nullptr, nullptr, none, stream, dev);
}

cudaError_t launch_quantize_mxfp8(const CUtensorMap& tmap_x, int tile_rows, int64_t M, int64_t K, uint8_t* codes,
                                  uint8_t* sf, cudaStream_t stream, const DeviceInfo& dev) {
  const GridWaitSettings none;
  return tile_rows == 256 ? launch_q<false, true, 256>(tmap_x, nullptr, M, K, 0.0f, codes, sf, nullptr, nullptr, none, stream, dev)
                          : launch_q<false, true, 128>(tmap_x, nullptr, M, K, 0.0f, codes, sf, nullptr, nullptr, none, stream, dev);
}

cudaError_t launch_quantize_from_amax(const CUtensorMap& tmap_x, int tile_rows, int64_t M, int64_t K,
                                      const float* amax_in, uint8_t* codes, uint8_t* sf, float* scale_out,
                                      cudaStream_t stream, const DeviceInfo& dev) {
  DynamicScaleArgs dyn{};
  dyn.scale_out = scale_out;
  dyn.amax_in = amax_in;
  return tile_rows == 256 ? launch_q_amax<256>(tmap_x, M, K, codes, sf, dyn, stream, dev)
                          : launch_q_amax<128>(tmap_x, M, K, codes, sf, dyn, stream, dev);
}

cudaError_t launch_quantize_dynamic(const CUtensorMap& tmap_x, int tile_rows, const void* x, int64_t M, int64_t K,
                                    uint8_t* codes, uint8_t* sf, float* scale_out, uint32_t* scratch,
                                    const GridWaitSettings& wait, cudaStream_t stream, const DeviceInfo& dev) {
  return tile_rows == 256
             ? launch_q<true, false, 256>(tmap_x, x, M, K, 0.0f, codes, sf, scale_out, scratch, wait, stream, dev)
             : launch_q<true, false, 128>(tmap_x, x, M, K, 0.0f, codes, sf, scale_out, scratch, wait, stream, dev);
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
