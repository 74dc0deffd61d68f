// Block-scaled NVFP4 x NVFP4 GEMM on the sm_100a tensor cores ("BFL (fp8r /
// nvfp4)" diffusers doc, section "Kernels": the `mm_fp4` GEMM of an NVFP4
// linear layer), with the dequant y = alpha * acc + bias folded into the
// epilogue and an optional fused epilogue that quantizes the result for the
// next layer.
//
// Design (one persistent CTA per SM, 10 warps, warp-specialised):
//   warp 0      TMA producer: 128x256 A tile, 192x256 B tile and their scale
//               atoms into a 4-stage shared-memory ring (mbarrier expect-tx).
//   warp 1      allocates TMEM; one thread issues tcgen05.mma kind::mxf4nvf4
//               (M=128, N=192, K=64, one UE4M3 scale per 16 elements) into a
//               double-buffered fp32 accumulator in TMEM.
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time, alpha*acc + bias,
//               bf16, swizzled staging in shared memory, TMA store; they
//               drain accumulator i while the MMA fills accumulator i^1.
//   warps 6-9   scale-factor movers: copy each stage's scale atoms from shared
//               memory into a double-buffered TMEM slot with tcgen05.st, one
//               warp per 32-lane TMEM quarter.  The MMA reads every scale row
//               from all four quarters, so each quarter holds a full copy.
//               Register-path stores run beside the tensor pipe; tcgen05.cp
//               copies of the same data would serialize with the MMAs.
// TMEM columns: [0,192) and [192,384) accumulators; [384,432) and [432,480)
// scale slots, each 16 columns of A scales (4 per MMA k-block) then 32 of B
// scales (8 per k-block).  Scale atom column j of lane l holds the 4 scales
// of row 32*j + l, so row i of a tile is read from column i/32; a 192-wide B
// tile that starts at row 64 of a 128-row atom block skips 2 columns.
// Every barrier wait is bounded (see mbar_wait); a role that gives up sets
// the CTA's abort flag and the device fault word, lets the copies it issued
// land, and the CTA still frees its TMEM before exiting.
#include "internal.h"

namespace nvfp4 {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 192;
constexpr int kBKBytes = 128;  // 256 fp4 elements per row per stage
constexpr int kStages = 4;
constexpr int kThreads = 320;
constexpr int kChunks = kBN / 32;

constexpr uint32_t kABytes = kBM * kBKBytes;  // 16 KB
constexpr uint32_t kBBytes = kBN * kBKBytes;  // 24 KB
constexpr uint32_t kSfaBytes = 4 * 512;       // 4 k-blocks x one 128-row atom
constexpr uint32_t kSfbBytes = 2 * 4 * 512;   // two 128-row atom blocks x 4 k-blocks

constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kABytes;
constexpr uint32_t kOffSfa = kOffB + kStages * kBBytes;
constexpr uint32_t kOffSfb = kOffSfa + kStages * kSfaBytes;
constexpr uint32_t kOffEpi = kOffSfb + kStages * kSfbBytes;  // 4 warps x 2 x 2 KB
constexpr uint32_t kOffBar = kOffEpi + 4 * 2 * 2048;
constexpr uint32_t kNumBars = 2 * kStages + 2 + 2 + 1 + 2 + 2;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol = 384;       // first scale slot
constexpr uint32_t kSfSlotCols = 48;   // 16 A-scale + 32 B-scale columns per k-tile
constexpr uint32_t kSfbOff = 16;       // B scales inside a slot
static_assert(2 * kBN <= kSfCol && kSfCol + 2 * kSfSlotCols <= kTmemCols, "TMEM layout");
static_assert(kABytes % 1024 == 0 && kBBytes % 1024 == 0, "stage bases must stay 1024-byte aligned");

__device__ __forceinline__ float gelu_tanh_f32(float v) {
  const float u = 0.7978845608028654f * (v + 0.044715f * v * v * v);
  return 0.5f * v * (1.0f + tanhf(u));
}

// Round to bf16 and back (the value the bf16 output holds).
__device__ __forceinline__ float round_bf16(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// Stage 32 rows x 32 bf16 columns (this warp's slice of one chunk) in the
// 64-byte-swizzled layout the Y tensor map expects, then TMA-store it.
__device__ __forceinline__ void store_chunk_bf16(const CUtensorMap* tmap, uint8_t* buf, const uint32_t (&w)[16],
                                                 int lane, int32_t x, int32_t y) {
  if (lane == 0) bulk_wait_read<1>();  // the store that last read this buffer is done
  __syncwarp();
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    const int phys = ch ^ ((lane >> 1) & 3);
    *reinterpret_cast<uint4*>(buf + lane * 64 + phys * 16) =
        make_uint4(w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
  }
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmap, buf, x, y);
    bulk_commit();
  }
}

template <bool kFused>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_y, const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = bars + 2 * kStages + 2;
  uint64_t* drain = bars + 2 * kStages + 4;
  uint64_t* sf_full = bars + 2 * kStages + 5;
  uint64_t* sf_empty = bars + 2 * kStages + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(drain, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sf_full[t], 4);
      mbar_init(&sf_empty[t], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_y);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  unsigned fault = 0u;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_phase[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
      for (int tile = blockIdx.x; tile < p.num_tiles && fault == 0u; tile += gridDim.x) {
        const int tm = tile % p.tiles_m;
        const int n0 = (tile / p.tiles_m) * kBN;
        const int rb0 = n0 >> 7;
        const bool has_rb1 = rb0 + 1 < p.sfb_row_blocks;
        for (int kt = 0; kt < p.num_kt; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            fault = kFaultProducerWait;
            break;
          }
          const int nkb = min(4, p.k64 - kt * 4);
          const uint32_t sf_bytes = static_cast<uint32_t>(nkb) * 512u;
          mbar_arrive_expect_tx(&full[stage], kABytes + kBBytes + sf_bytes * (has_rb1 ? 3u : 2u));
          tma_load_2d(smem + kOffA + stage * kABytes, &tmap_a, &full[stage], kt * kBKBytes, tm * kBM);
          tma_load_2d(smem + kOffB + stage * kBBytes, &tmap_b, &full[stage], kt * kBKBytes, n0);
          bulk_load(smem + kOffSfa + stage * kSfaBytes,
                    p.sfa + (static_cast<size_t>(tm) * p.k64 + kt * 4) * 512, sf_bytes, &full[stage]);
          bulk_load(smem + kOffSfb + stage * kSfbBytes,
                    p.sfb + (static_cast<size_t>(rb0) * p.k64 + kt * 4) * 512, sf_bytes, &full[stage]);
          if (has_rb1)
            bulk_load(smem + kOffSfb + stage * kSfbBytes + 4 * 512,
                      p.sfb + (static_cast<size_t>(rb0 + 1) * p.k64 + kt * 4) * 512, sf_bytes, &full[stage]);
          last_phase[stage] = static_cast<int>(phase);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (fault != 0u) {
        *abort_flag = 1;
        // let every copy already issued land before shared memory goes away
        for (int s = 0; s < kStages; ++s)
          if (last_phase[s] >= 0) mbar_wait(&full[s], static_cast<uint32_t>(last_phase[s]), nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_nvf4(kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int slot = 0;
      uint32_t slot_phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && fault == 0u; tile += gridDim.x) {
        const int n0 = (tile / p.tiles_m) * kBN;
        const uint32_t sfb_shift = (n0 & 127) ? 2u : 0u;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
          fault = kFaultMmaWait;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        for (int kt = 0; kt < p.num_kt; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag) || !mbar_wait(&sf_full[slot], slot_phase, abort_flag)) {
            fault = kFaultMmaWait;
            break;
          }
          tc_fence_after();
          const int nkb = min(4, p.k64 - kt * 4);
          const uint32_t sa = smem_u32(smem + kOffA + stage * kABytes);
          const uint32_t sb = smem_u32(smem + kOffB + stage * kBBytes);
          const uint32_t sf = tmem_base + kSfCol + static_cast<uint32_t>(slot) * kSfSlotCols;
          for (int kb = 0; kb < nkb; ++kb) {
            tc_mma_nvf4(d_tmem, sdesc_kmajor_sw128(sa + kb * 32), sdesc_kmajor_sw128(sb + kb * 32), idesc,
                        sf + kb * 4, sf + kSfbOff + kb * 8 + sfb_shift, (kt | kb) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);    // frees the smem stage once these MMAs have read it
          tc_commit(&sf_empty[slot]);  // and the scale slot
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
          slot ^= 1;
          if (slot == 0) slot_phase ^= 1u;
        }
        if (fault != 0u) break;
        tc_commit(&acc_full[acc]);  // accumulator ready for the epilogue
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (fault != 0u) *abort_flag = 1;
      // every tcgen05 op issued must complete before TMEM is released
      tc_commit(drain);
      if (!mbar_wait(drain, 0u, nullptr)) fault |= kFaultDrainWait;
    }
    __syncwarp();
  } else if (warp >= 6) {
    // ------------------------------------------------------------ scale movers
    const uint32_t q = static_cast<uint32_t>(warp & 3);  // TMEM lane quarter of this warp
    int stage = 0;
    uint32_t phase = 0;
    int slot = 0;
    uint32_t slot_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles && fault == 0u; tile += gridDim.x) {
      for (int kt = 0; kt < p.num_kt; ++kt) {
        const bool got = mbar_wait(&full[stage], phase, abort_flag) &&
                         mbar_wait(&sf_empty[slot], slot_phase ^ 1u, abort_flag);
        __syncwarp();
        if (!__all_sync(0xffffffffu, got)) {
          fault = kFaultMmaWait;
          break;
        }
        tc_fence_after();
        const int nkb = min(4, p.k64 - kt * 4);
        const uint8_t* ssfa = smem + kOffSfa + stage * kSfaBytes + lane * 16;
        const uint8_t* ssfb = smem + kOffSfb + stage * kSfbBytes + lane * 16;
        const uint32_t t = tmem_base + ((q * 32u) << 16) + kSfCol + static_cast<uint32_t>(slot) * kSfSlotCols;
        for (int kb = 0; kb < nkb; ++kb) {
          const uint4 a = *reinterpret_cast<const uint4*>(ssfa + kb * 512);
          const uint4 b0 = *reinterpret_cast<const uint4*>(ssfb + kb * 512);
          const uint4 b1 = *reinterpret_cast<const uint4*>(ssfb + 4 * 512 + kb * 512);
          tmem_st_32x32b_x4(t + kb * 4, a);
          tmem_st_32x32b_x8(t + kSfbOff + kb * 8, b0, b1);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full[slot]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
        slot ^= 1;
        if (slot == 0) slot_phase ^= 1u;
      }
    }
    if (fault != 0u) *abort_flag = 1;
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint8_t* stage_buf = smem + kOffEpi + (warp - 2) * 4096;
    int buf = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      const int tm = tile % p.tiles_m;
      const int n0 = (tile / p.tiles_m) * kBN;
      const bool got = mbar_wait(&acc_full[acc], acc_phase, abort_flag);
      __syncwarp();  // tcgen05.ld below needs the whole warp converged
      if (!__all_sync(0xffffffffu, got)) {
        fault = kFaultEpilogueWait;
        break;
      }
      tc_fence_after();
      const int row_base = tm * kBM + q * 32;
      const int row = row_base + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kBN);
      uint32_t sf_word = 0u;
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + c * 32, r);
        tmem_ld_wait(r);
        if (c == kChunks - 1) {
          // accumulator fully read: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[acc]);
        }
        const int n = n0 + c * 32;
        if (n >= p.N) continue;

        // which output, and which activation, this chunk goes to
        int act = NVFP4_ACT_NONE, dst = NVFP4_DST_BF16, out_col = n;
        if (kFused) {
          int hit = -1;
          for (int i = 0; i < p.n_ranges; ++i)
            if (n >= p.ranges[i].begin && n < p.ranges[i].end) hit = i;
          if (hit < 0) continue;
          act = p.ranges[hit].act;
          dst = p.ranges[hit].dst;
          out_col = p.ranges[hit].dst_col + (n - p.ranges[hit].begin);
        }

        float bias[32];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint4 b = make_uint4(0u, 0u, 0u, 0u);
          if (p.bias != nullptr && n + 8 * g < p.N) b = __ldg(reinterpret_cast<const uint4*>(p.bias + n + 8 * g));
          bias[8 * g + 0] = bf16_lo(b.x);
          bias[8 * g + 1] = bf16_hi(b.x);
          bias[8 * g + 2] = bf16_lo(b.y);
          bias[8 * g + 3] = bf16_hi(b.y);
          bias[8 * g + 4] = bf16_lo(b.z);
          bias[8 * g + 5] = bf16_hi(b.z);
          bias[8 * g + 6] = bf16_lo(b.w);
          bias[8 * g + 7] = bf16_hi(b.w);
        }
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = round_bf16(fmaf(p.alpha, __uint_as_float(r[j]), bias[j]));
        if (kFused && act == NVFP4_ACT_GELU_TANH) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = round_bf16(gelu_tanh_f32(v[j]));
        }

        if (!kFused || dst == NVFP4_DST_BF16) {
          if (row_base < p.M) {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
            store_chunk_bf16(&tmap_y, stage_buf + buf * 2048, w, lane, out_col, row_base);
            buf ^= 1;
          }
        } else {
          // next layer's NVFP4 input: two 16-element blocks per chunk
          const float g = p.g_next;
          const float d6 = __fmul_rn(6.0f, g);
          float blk[16];
          uint32_t c0, c1, c2, c3;
#pragma unroll
          for (int j = 0; j < 16; ++j) blk[j] = v[j];
          const uint32_t s0 = quantize_block16(blk, g, d6, c0, c1);
#pragma unroll
          for (int j = 0; j < 16; ++j) blk[j] = v[16 + j];
          const uint32_t s1 = quantize_block16(blk, g, d6, c2, c3);
          if (row < p.M)
            *reinterpret_cast<uint4*>(p.codes_next + static_cast<size_t>(row) * (p.k_next >> 1) + (out_col >> 1)) =
                make_uint4(c0, c1, c2, c3);
          const int csf = out_col >> 4;  // scale column of the first block (even)
          sf_word |= (s0 | (s1 << 8)) << (8 * (csf & 3));
          if ((csf & 3) == 2) {  // the 64-column group is complete
            const uint32_t word = row < p.M ? sf_word : 0u;  // padding rows of the scale buffer are zero
            *reinterpret_cast<uint32_t*>(p.sf_next + sf_offset(row, csf & ~3, p.k_next >> 6)) = word;
            sf_word = 0u;
          }
        }
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait<0>();
    if (fault != 0u) *abort_flag = 1;
  }

  if (fault != 0u && lane == 0 && p.fault != nullptr) atomicOr(p.fault, fault);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm(const CUtensorMap& tmap_a, const CUtensorMap& tmap_b, const CUtensorMap& tmap_y,
                        const GemmParams& p, bool fused, cudaStream_t stream, const DeviceInfo& dev) {
  auto kernel = fused ? gemm_nvf4_kernel<true> : gemm_nvf4_kernel<false>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (err != cudaSuccess) return err;
  const int grid = p.num_tiles < dev.num_sms ? p.num_tiles : dev.num_sms;
  kernel<<<grid, kThreads, kSmemBytes, stream>>>(tmap_a, tmap_b, tmap_y, p);
  return cudaGetLastError();
}

int gemm_tile_n() { return kBN; }

}  // namespace nvfp4
