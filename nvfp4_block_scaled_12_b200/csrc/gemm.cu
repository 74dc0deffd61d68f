// Block-scaled NVFP4 x NVFP4 GEMM on the sm_100a tensor cores ("BFL (fp8r /
// nvfp4)" diffusers doc, section "Kernels": the `mm_fp4` GEMM of an NVFP4
// linear layer), with the dequant y = alpha * acc + bias folded into the
// epilogue and an optional fused epilogue that quantizes the result for the
// next layer.
//
// One persistent kernel, templated on the tile shape (the same rule for the
// NVFP4, fused, MXFP8 and row-wise FP8 GEMMs; gemm_config below):
//   256 x 256 (wide)  a CTA pair (cluster of 2) owns the tile: each CTA loads
//            its 128 rows of A and 128 rows of B, and the pair leader issues
//            tcgen05.mma.cta_group::2 (M=256, N=256, K=64) into one
//            256-column accumulator.  Used with at least one tile per pair.
//   256 x 192  a CTA pair with 96 rows of B per CTA and two accumulators
//            (M > 128 with fewer wide tiles than pairs).
//   256 x 128  as 256 x 192 with 64 rows of B per CTA, when these tiles still
//            fit in one wave and the 192-wide ones would leave pairs idle.
//   128 x 192  one CTA per tile (M <= 128).
// Every pipeline step (one 128-byte k-tile: four MMAs) costs the MMA-issuing
// thread a barrier wait, a commit and its bookkeeping, during which the
// tensor pipe runs dry; the wide tile does a third more MMA work per step.
// Warps, standard layout (11 per CTA):
//   0, 10 TMA producers, alternating k-tiles: A/B tiles (128-byte rows,
//         128-byte swizzle) and the scale atoms (3-D boxes, zero-filled past
//         K and past the last row block) into a shared-memory ring.  A TMA
//         instruction holds its issuing thread long enough that one thread
//         cannot keep the SM's TMA unit busy; two issuing warps reach about
//         twice the load rate.
//   1     allocates TMEM; in the leader one thread waits for one barrier per
//         k-tile, issues the MMAs and commits once: that commit frees the
//         shared-memory stage and the TMEM scale slot of the k-tile together.
//   2-5   epilogue: tcgen05.ld 32 columns at a time, alpha*acc + bias, bf16,
//         swizzled staging in shared memory, TMA store (or the fused
//         quantize); drains accumulator i while the MMA fills i^1.
//   6-9   scale movers: copy each stage's scale atoms from shared memory into
//         a ring of TMEM slots with tcgen05.st, one warp per 32-lane TMEM
//         quarter, and arrive on the same barrier as the A/B bytes.  The MMA
//         reads every scale row from all four quarters, so each quarter holds
//         a full copy.  Register-path stores run beside the tensor pipe, where
//         tcgen05.cp copies of the same (replicated) data would serialize with
//         the MMAs.
// Wide layout (16 warps = four warpgroups with their own register budgets):
//   0, 2 producers, 1 MMA issuer, 3 idle; 4-11 epilogue, two warps per lane
//   quarter (one per 128-column half), each reading its whole 128-column
//   slice into registers before releasing the accumulator; 12-15 movers.
// TMEM columns: the accumulators first, then the scale slots: 16 columns of A
// scales each (4 per MMA k-block), then kBN/8 columns of B scales each
// (kBN/32 per k-block).  Scale column j of lane l holds the 4 scales of row
// 32*j + l, so row i of a tile is read from column i/32; the movers pick the
// kBN/32 row groups of the tile out of the 128-row atom blocks it touches (a
// 192-wide tile may start at row 64 of a block).
// Every barrier wait is bounded (see mbar_wait); a role that gives up sets
// the CTA's abort flag and the device fault word, lets the copies it issued
// land, and the CTA still reaches the final barrier and frees its TMEM.
#include <atomic>

#include "internal.h"

namespace nvfp4 {

namespace {

constexpr int kBKBytes = 128;   // per row per stage: 256 fp4 or 128 fp8 elements
constexpr uint32_t kABytes = 128 * kBKBytes;  // 16 KB: this CTA's 128 rows of A
constexpr int kProducers = 2;
constexpr uint32_t kTmemCols = 512;

// kCG: CTAs per tile; kBN: tile width; kAcc: accumulator buffers in TMEM;
// kMx: 8-bit E4M3 operands (K = 32 per MMA) instead of NVFP4; with kRow they
// carry no block scales at all (row-wise FP8: one scale per row of A and of
// B, applied in the epilogue), otherwise one E8M0 scale per 32 elements.
// kW16: W4A16, bf16 activations (K = 16 per MMA, 64 elements = 128 bytes per
// k-tile) against NVFP4 weights that the transform warps dequantize to bf16
// in shared memory (the stage holds this CTA's B codes and scale atoms as
// loaded, and the bf16 B tile the MMA reads).
template <int kCG, int kBN, int kAcc, bool kMx, bool kRow = false, bool kW16 = false>
struct Cfg {
  // Wide tiles (256 columns, one accumulator): the accumulator is drained into
  // the registers of eight epilogue warps, so the next tile's MMAs can start
  // before the epilogue's arithmetic and stores.  Other shapes keep four
  // epilogue warps that read the accumulator chunk by chunk while the MMAs
  // fill the other buffer.
  static constexpr bool kWide = kBN == 256 && kAcc == 1;
  static constexpr int kEpiWarps = kWide ? 8 : 4;
  static constexpr int kThreads = kWide ? 512 : 352;
  // 512-byte scale atoms (128 rows x 4 scale columns) per 128-row block and
  // k-tile: NVFP4's k-tile is 4 MMA k-blocks of 64 elements with one 4-scale
  // word per row each; MXFP8's is 4 k-blocks of 32 whose scales share one word.
  // (W4A16: a k-tile of 64 elements is one atom, read for B only)
  static constexpr int kAtoms = (kMx || kW16) ? 1 : 4;
  static constexpr uint32_t kSfaBytes = (kRow || kW16) ? 0 : kAtoms * 512;
  static constexpr int kBNc = kBN / kCG;  // B rows per CTA
  static constexpr uint32_t kBBytes = kBNc * kBKBytes;
  static constexpr int kChunks = kBN / 32;
  // 128-row scale blocks a B tile can touch (a 192-wide tile may start mid-block)
  static constexpr int kSfbBlocks = kBN % 128 == 0 ? kBN / 128 : kBN / 128 + 1;
  static constexpr uint32_t kSfbBytes = kRow ? 0 : kSfbBlocks * kAtoms * 512;
  static constexpr uint32_t kCodeBytes = kW16 ? kBNc * 32 : 0;  // W4A16: this CTA's B codes (64 elements a row)
  static constexpr uint32_t kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes + kCodeBytes;
  static constexpr uint32_t kEpiBytes = kEpiWarps * 2 * 2048;  // double-buffered 32 x 32 bf16 staging per warp
  static constexpr uint32_t kBiasBytes = kWide ? kEpiWarps * 256 : 0;  // each wide epilogue warp's 128 bias values
  static constexpr int kStagesFit = (224 * 1024 - kEpiBytes - kBiasBytes) / kStageBytes;
  // The producers alternate k-tiles.  An mbarrier wait tells phases apart
  // only by parity, so a waiter must never be two phases behind: a producer
  // has seen the commit of its own previous k-tile (kProducers back), hence
  // of every k-tile before it, which covers the stage's previous phase as
  // long as kStages >= kProducers.
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  // TMEM: accumulators, then the scale slots.  Slot j % kSfSlots holds the
  // scales of k-tile j; the movers refill it once the commit of k-tile
  // j - kSfSlots has arrived on that k-tile's empty barrier, which can only
  // be the phase they wait for while kSfSlots <= kStages.
  static constexpr uint32_t kSfbGroups = kBN / 32;       // 32-row groups of B scales per k-block
  static constexpr uint32_t kSfaSlotCols = kMx ? 4 : 16;
  static constexpr uint32_t kSfbSlotCols = kMx ? (kSfbGroups + 7) / 8 * 8 : 4 * kSfbGroups;
  static constexpr int kSfSlotsFit = (kTmemCols - kAcc * kBN) / (kSfaSlotCols + kSfbSlotCols);
  static constexpr int kSfSlots = kSfSlotsFit < kStages ? (kSfSlotsFit > 8 ? 8 : kSfSlotsFit) : kStages;
  static constexpr uint32_t kSfaCol = kAcc * kBN;
  static constexpr uint32_t kSfbCol = (kSfaCol + kSfaSlotCols * kSfSlots + 7) / 8 * 8;
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffB = kOffA + kStages * kABytes;
  static constexpr uint32_t kOffSfa = kOffB + kStages * kBBytes;
  static constexpr uint32_t kOffSfb = kOffSfa + kStages * kSfaBytes;
  static constexpr uint32_t kOffCode = kOffSfb + kStages * kSfbBytes;
  static constexpr uint32_t kOffEpi = kOffCode + kStages * kCodeBytes;
  static constexpr uint32_t kOffBias = kOffEpi + kEpiBytes;
  static constexpr uint32_t kOffBar = kOffBias + kBiasBytes;
  // full, empty, sfin per stage; acc_full, acc_empty per accumulator; drain
  static constexpr uint32_t kNumBars = 3 * kStages + 2 * kAcc + 1;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  // A/B bytes of the whole group (W4A16: A only; B is written by the transform warps)
  static constexpr uint32_t kFullTx = kW16 ? kCG * kABytes : kCG * (kABytes + kBBytes);
  static_assert(kBN % 32 == 0 && kChunks * 32 == kBN && kBN / kCG % 8 == 0, "tile width");
  static_assert(kBBytes % 1024 == 0, "stage bases must stay 1024-byte aligned");
  static_assert(kSfSlots >= 2 && kSfSlots <= kStages, "TMEM budget");
  static_assert(kSfaCol % kSfaSlotCols == 0 && kSfbCol % 8 == 0 && kSfbSlotCols % 8 == 0, "tcgen05.st column alignment");
  static_assert(kSfbCol + kSfSlots * kSfbSlotCols <= kTmemCols, "TMEM budget");
  static_assert(kStages >= 3 && kStages >= kProducers, "pipeline depth");
  static_assert(!kWide || kCG == 2, "wide tiles are CTA pairs");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(!kW16 || (!kMx && !kRow), "W4A16 has bf16 activations and NVFP4 weights");
  // K split: a CTA's fp32 partial tile, 128 rows of kBN + 4 floats (the pad
  // spreads the rows over the banks), in the idle stage ring
  static constexpr uint32_t kPartStride = (kBN + 4) * 4;
  static_assert(kWide || 128 * kPartStride <= kOffEpi, "the partial tile fits the stage ring");
  static_assert(kCodeBytes % 128 == 0 && kSfbBytes % 128 == 0, "TMA destinations stay 128-byte aligned");
};

// GELU, tanh form, 0.5 v (1 + tanh(u)), u = sqrt(2/pi) (v + 0.044715 v^3), in
// fp32 with the hardware tanh (tanh.approx.f32, relative error about 2^-11:
// below the bf16 rounding the result goes through next, far below the GEMM
// tolerance; accurate tanhf made the activation the slowest part of the
// fused epilogue).
__device__ __forceinline__ float gelu_tanh_f32(float v) {
  const float u = 0.7978845608028654f * (v + 0.044715f * v * v * v);
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(u));
  return 0.5f * v * (1.0f + t);
}


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

template <int kCG, int kBN, int kAcc, bool kFused, bool kMx, bool kRow, bool kW16 = false>
__global__ void __launch_bounds__(Cfg<kCG, kBN, kAcc, kMx, kRow, kW16>::kThreads, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                     const __grid_constant__ CUtensorMap tmap_y, const __grid_constant__ GemmParams p) {
  using C = Cfg<kCG, kBN, kAcc, kMx, kRow, kW16>;
  static_assert(!(kFused && kW16), "the fused quantize epilogue follows an NVFP4 GEMM");
  static_assert(!(kFused && kMx), "the fused quantize epilogue writes NVFP4 after an NVFP4 GEMM");
  static_assert(!kRow || kMx, "row-wise FP8 uses the 8-bit operand layout");
  constexpr int S = C::kStages;
  constexpr int R = C::kSfSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;            // leader: A/B of the whole group landed, scales in TMEM
  uint64_t* empty = bars + S;       // this CTA's stage and the k-tile's scale slot may be refilled
  uint64_t* sfin = bars + 2 * S;    // this CTA's scale atoms (W4A16: B codes and scale atoms) landed
  uint64_t* acc_full = bars + 3 * S;
  uint64_t* acc_empty = acc_full + kAcc;   // leader
  uint64_t* drain = acc_empty + kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // A cluster is one tile group of kCG CTAs, or, with a K split, p.k_split
  // such groups that share one output tile over disjoint k-tile ranges; a CTA
  // pair is cluster ranks 2i, 2i + 1.
  const uint32_t crank = (kCG == 2 || p.k_split > 1) ? cluster_ctarank() : 0u;
  const uint32_t rank = crank % kCG;          // CTA within its tile group
  const uint32_t lead_rank = crank - rank;    // cluster rank of the group leader
  const bool leader = rank == 0;
  const int split = static_cast<int>(crank) / kCG;  // this group's k-tile range
  const int kt_begin = static_cast<int>(static_cast<int64_t>(p.num_kt) * split / p.k_split);
  const int kt_end = static_cast<int>(static_cast<int64_t>(p.num_kt) * (split + 1) / p.k_split);
  const int my_kt = kt_end - kt_begin;
  // Warp roles.  Standard layout (11 warps): 0 and 10 TMA producers, 1 MMA,
  // 2-5 epilogue, 6-9 scale movers.  Wide layout (16 warps, four warpgroups):
  // 0 and 2 producers, 1 MMA, 3 idle, 4-11 epilogue (two per TMEM lane
  // quarter, one per 128-column half), 12-15 scale movers.
  const bool is_producer = C::kWide ? (warp == 0 || warp == 2) : (warp == 0 || warp == 10);
  const bool is_mover = C::kWide ? warp >= 12 : (warp >= 6 && warp <= 9);
  const bool is_epilogue = C::kWide ? (warp >= 4 && warp < 12) : (warp >= 2 && warp <= 5);
  const int cluster = blockIdx.x / (kCG * p.k_split);
  const int num_clusters = gridDim.x / (kCG * p.k_split);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // the producer's expect_tx and every scale mover of the group
      mbar_init(&full[s], kRow ? 1 : 1 + 4 * kCG);
      mbar_init(&empty[s], 1);
      mbar_init(&sfin[s], 1);
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], C::kEpiWarps * kCG);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    if (!kRow && !kW16) prefetch_tmap(&tmap_sfa);
    if (!kRow) prefetch_tmap(&tmap_sfb);
    prefetch_tmap(&tmap_y);
  }
  if (warp == 1) {
    tmem_alloc<kCG>(tmem_slot, kTmemCols);
    tmem_relinquish<kCG>();
  }
  tc_fence_before();
  __syncthreads();
  if (kCG == 2 || p.k_split > 1) cluster_sync();  // the peer's barriers are initialised before anyone signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  unsigned fault = 0u;

  // arrive on a barrier that lives in the group leader
  auto arrive_leader = [&](uint64_t* bar) {
    if (kCG == 2 && !leader)
      mbar_arrive_cluster(peer_smem(smem_u32(bar), lead_rank));
    else
      mbar_arrive(bar);
  };
  // commit to a barrier in every CTA of the group
  auto commit_group = [&](uint64_t* bar) {
    if (kCG == 2)
      tc_commit_pair(bar, static_cast<uint16_t>(0x3u << lead_rank));
    else
      tc_commit(bar);
  };

  auto run_producer = [&]() {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      const int pid = warp == 0 ? 0 : 1;
      // flattened (tile, k-tile) sequence of this CTA group; producer pid
      // issues the entries j with j % kProducers == pid into stage j % S
      const int my_tiles = p.num_tiles > cluster ? (p.num_tiles - cluster + num_clusters - 1) / num_clusters : 0;
      const int64_t total = static_cast<int64_t>(my_tiles) * my_kt;
      // entry j = t_i * my_kt + (kt - kt_begin) of this CTA group's t_i-th
      // tile; stage, phase, tile and k-tile advance incrementally (no 64-bit
      // division on the way to the first loads)
      int t_i = 0, kt = kt_begin + pid;
      while (kt >= kt_end) {
        kt -= my_kt;
        ++t_i;
      }
      int stage = pid, cur_t = -1, tm = 0, n0 = 0;
      uint32_t phase = 0;
      int64_t j = pid;
      for (; j < total; j += kProducers) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
          fault = kFaultProducerWait;
          break;
        }
        if (t_i != cur_t) {
          cur_t = t_i;
          const int tile = cluster + t_i * num_clusters;
          tm = tile % p.tiles_m;
          n0 = (tile / p.tiles_m) * kBN;
        }
        const int row_block = tm * kCG + static_cast<int>(rank);  // this CTA's 128-row block
        if (leader) mbar_arrive_expect_tx(&full[stage], C::kFullTx);
        if (!kRow) mbar_arrive_expect_tx(&sfin[stage], C::kSfaBytes + C::kSfbBytes + C::kCodeBytes);
        uint8_t* sa = smem + C::kOffA + stage * kABytes;
        uint8_t* sb = smem + C::kOffB + stage * C::kBBytes;
        // A's x coordinate counts elements of its map: bytes for the 4- and
        // 8-bit codes, bf16 elements (64 per 128-byte k-tile) for W4A16
        const int32_t xa = kW16 ? kt * 64 : kt * kBKBytes;
        const int brow = n0 + static_cast<int>(rank) * C::kBNc;  // this CTA's first B row
        if (kCG == 2) {
          const uint32_t fb = peer_smem(smem_u32(&full[stage]), lead_rank);
          tma_load_2d_pair(sa, &tmap_a, fb, xa, row_block * 128);
          if (!kW16) tma_load_2d_pair(sb, &tmap_b, fb, kt * kBKBytes, brow);
        } else {
          tma_load_2d(sa, &tmap_a, &full[stage], xa, row_block * 128);
          if (!kW16) tma_load_2d(sb, &tmap_b, &full[stage], kt * kBKBytes, n0);
        }
        if (kW16) {
          // this CTA's B codes (32 bytes = 64 elements a row) and the B scale
          // atoms of the k-tile, for the transform warps
          tma_load_2d(smem + C::kOffCode + stage * C::kCodeBytes, &tmap_b, &sfin[stage], kt * 32, brow);
          tma_load_3d(smem + C::kOffSfb + stage * C::kSfbBytes, &tmap_sfb, &sfin[stage], 0, kt, n0 >> 7);
        } else if (!kRow) {
          tma_load_3d(smem + C::kOffSfa + stage * C::kSfaBytes, &tmap_sfa, &sfin[stage], 0, kt * C::kAtoms, row_block);
          tma_load_3d(smem + C::kOffSfb + stage * C::kSfbBytes, &tmap_sfb, &sfin[stage], 0, kt * C::kAtoms, n0 >> 7);
        }
        kt += kProducers;
        while (kt >= kt_end) {
          kt -= my_kt;
          ++t_i;
        }
        stage += kProducers;
        if (stage >= S) {
          stage -= S;
          phase ^= 1u;
        }
      }
      if (fault != 0u) {
        *abort_flag = 1;
        // let the copies this producer issued (its last S / kProducers entries) land
        for (int64_t i = j - kProducers; i >= 0 && i >= j - S; i -= kProducers) {
          const int stage = static_cast<int>(i % S);
          const uint32_t phase = static_cast<uint32_t>((i / S) & 1);
          if (!kRow) mbar_wait(&sfin[stage], phase, nullptr);
          if (leader) mbar_wait(&full[stage], phase, nullptr);
        }
      }
    }
  };
  auto run_mma = [&]() {
    // ------------------------------------------------------------ MMA issuer (group leader)
    if (lane == 0 && leader) {
      // one MMA k-block: NVFP4 reads 4 scale columns per k-block; MXFP8 reads
      // byte kb of the k-tile's scale words (named in the descriptor and in
      // the top two bits of the scale addresses)
      auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t sfa, uint32_t sfb, int kb, uint32_t accum) {
        if constexpr (kW16) {
          constexpr uint32_t idesc = idesc_bf16(128 * kCG, kBN);
          if (kCG == 2)
            tc_mma_bf16_pair(d, ad, bd, idesc, accum);
          else
            tc_mma_bf16(d, ad, bd, idesc, accum);
        } else if constexpr (kRow) {
          constexpr uint32_t idesc = idesc_f8(128 * kCG, kBN);
          if (kCG == 2)
            tc_mma_f8_pair(d, ad, bd, idesc, accum);
          else
            tc_mma_f8(d, ad, bd, idesc, accum);
        } else if constexpr (kMx) {
          const uint32_t idesc = idesc_mxf8(128 * kCG, kBN, static_cast<uint32_t>(kb));
          const uint32_t sel = static_cast<uint32_t>(kb) << 30;
          if (kCG == 2)
            tc_mma_mxf8_pair(d, ad, bd, idesc, sfa | sel, sfb | sel, accum);
          else
            tc_mma_mxf8(d, ad, bd, idesc, sfa | sel, sfb | sel, accum);
        } else {
          constexpr uint32_t idesc = idesc_nvf4(128 * kCG, kBN);
          if (kCG == 2)
            tc_mma_nvf4_pair(d, ad, bd, idesc, sfa + kb * 4, sfb + kb * C::kSfbGroups, accum);
          else
            tc_mma_nvf4(d, ad, bd, idesc, sfa + kb * 4, sfb + kb * C::kSfbGroups, accum);
        }
      };
      int stage = 0;
      uint32_t phase = 0;
      int slot = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = cluster; tile < p.num_tiles && fault == 0u; tile += num_clusters) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
          fault = kFaultMmaWait;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        for (int kt = kt_begin; kt < kt_end; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            fault = kFaultMmaWait;
            break;
          }
          tc_fence_after();
          const int nkb = min(4, p.kblocks - kt * 4);
          const uint32_t sa = smem_u32(smem + C::kOffA + stage * kABytes);
          const uint32_t sb = smem_u32(smem + C::kOffB + stage * C::kBBytes);
          const uint32_t sfa = tmem_base + C::kSfaCol + static_cast<uint32_t>(slot) * C::kSfaSlotCols;
          const uint32_t sfb = tmem_base + C::kSfbCol + static_cast<uint32_t>(slot) * C::kSfbSlotCols;
          // One thread issues the MMAs and the tensor pipe queues few of them,
          // so the instructions between two MMAs are on the critical path: the
          // full k-tile takes a straight-line path with every operand address
          // formed up front (a descriptor's start address field counts 16-byte
          // units, so the next 32-byte k-block is +2).
          const uint64_t ad = sdesc_kmajor_sw128(sa), bd = sdesc_kmajor_sw128(sb);
          if (nkb == 4) {
            const uint32_t first = kt != kt_begin ? 1u : 0u;  // the range's first k-tile starts the sum
            mma(d_tmem, ad, bd, sfa, sfb, 0, first);
            mma(d_tmem, ad + 2, bd + 2, sfa, sfb, 1, 1u);
            mma(d_tmem, ad + 4, bd + 4, sfa, sfb, 2, 1u);
            mma(d_tmem, ad + 6, bd + 6, sfa, sfb, 3, 1u);
          } else {
            for (int kb = 0; kb < nkb; ++kb)
              mma(d_tmem, ad + 2 * kb, bd + 2 * kb, sfa, sfb, kb, (kt != kt_begin || kb != 0) ? 1u : 0u);
          }
          // frees the smem stage and the scale slot once these MMAs have read them
          commit_group(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
          if (++slot == R) slot = 0;
        }
        if (fault != 0u) break;
        commit_group(&acc_full[acc]);  // accumulators ready for both epilogues
        if (++acc == kAcc) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (fault != 0u) *abort_flag = 1;
      // every tcgen05 op issued must complete before TMEM is released
      if (kCG == 2)
        tc_commit_pair_local(drain);
      else
        tc_commit(drain);
      if (!mbar_wait(drain, 0u, nullptr)) fault |= kFaultDrainWait;
    }
    __syncwarp();
  };
  auto run_movers = [&]() {
    // ------------------------------------------------------------ scale movers
    const uint32_t q = static_cast<uint32_t>(warp & 3);  // TMEM lane quarter of this warp
    const uint32_t t_quarter = tmem_base + ((q * 32u) << 16);
    int stage = 0;
    uint32_t phase = 0;
    int lag_stage = 0;  // stage and phase of k-tile j - R, whose commit frees slot j % R
    uint32_t lag_phase = 0;
    int slot = 0;
    int64_t j = 0;
    for (int tile = cluster; tile < p.num_tiles && fault == 0u; tile += num_clusters) {
      // a 192-wide tile that starts at row 64 of a 128-row scale block
      const bool mid = ((tile / p.tiles_m) * kBN & 127) != 0;
      for (int kt = kt_begin; kt < kt_end; ++kt, ++j) {
        const bool landed = mbar_wait(&sfin[stage], phase, abort_flag);
        __syncwarp();
        if (!__all_sync(0xffffffffu, landed)) {
          fault = kFaultMmaWait;
          break;
        }
        // The scales are read into registers first; only the TMEM stores wait
        // for slot j % R to be free (the commit of k-tile j - R).
        auto slot_free = [&]() {
          bool ok = true;
          if (j >= R) {
            ok = mbar_wait(&empty[lag_stage], lag_phase, abort_flag);
            if (++lag_stage == S) {
              lag_stage = 0;
              lag_phase ^= 1u;
            }
          }
          __syncwarp();
          ok = __all_sync(0xffffffffu, ok);
          tc_fence_after();
          return ok;
        };
        // All loads first (atoms past K arrived zero-filled), then a few wide
        // stores: a shared load is not reordered across a tcgen05.st.
        const uint8_t* ssfa = smem + C::kOffSfa + stage * C::kSfaBytes + lane * 16;
        const uint8_t* ssfb = smem + C::kOffSfb + stage * C::kSfbBytes + lane * 16;
        if constexpr (kMx) {
          // one atom per 128-row block: word j of lane l's chunk = the four
          // 32-element-block scales of row 32j + l
          const uint4 a = *reinterpret_cast<const uint4*>(ssfa);
          uint32_t w[4 * C::kSfbBlocks];
#pragma unroll
          for (int blk = 0; blk < C::kSfbBlocks; ++blk) {
            const uint4 u = *reinterpret_cast<const uint4*>(ssfb + blk * 512);
            w[4 * blk + 0] = u.x;
            w[4 * blk + 1] = u.y;
            w[4 * blk + 2] = u.z;
            w[4 * blk + 3] = u.w;
          }
          uint32_t sb[C::kSfbSlotCols];
#pragma unroll
          for (int g = 0; g < static_cast<int>(C::kSfbSlotCols); ++g) {
            if (g >= static_cast<int>(C::kSfbGroups))
              sb[g] = 0u;
            else if constexpr (kBN % 128 != 0)
              sb[g] = mid ? w[g + 2] : w[g];
            else
              sb[g] = w[g];
          }
          if (!slot_free()) {
            fault = kFaultMmaWait;
            break;
          }
          tmem_st_32x32b_x4(t_quarter + C::kSfaCol + static_cast<uint32_t>(slot) * C::kSfaSlotCols, a);
#pragma unroll
          for (int c = 0; c < static_cast<int>(C::kSfbSlotCols / 8); ++c)
            tmem_st_32x32b_x8(t_quarter + C::kSfbCol + static_cast<uint32_t>(slot) * C::kSfbSlotCols + c * 8,
                              sb + 8 * c);
        } else {
          uint32_t sa[16];
          uint32_t sb[4 * C::kSfbGroups];
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint4 v = *reinterpret_cast<const uint4*>(ssfa + kb * 512);
            sa[4 * kb + 0] = v.x;
            sa[4 * kb + 1] = v.y;
            sa[4 * kb + 2] = v.z;
            sa[4 * kb + 3] = v.w;
            uint32_t w[4 * C::kSfbBlocks];
#pragma unroll
            for (int blk = 0; blk < C::kSfbBlocks; ++blk) {
              const uint4 u = *reinterpret_cast<const uint4*>(ssfb + blk * 4 * 512 + kb * 512);
              w[4 * blk + 0] = u.x;
              w[4 * blk + 1] = u.y;
              w[4 * blk + 2] = u.z;
              w[4 * blk + 3] = u.w;
            }
#pragma unroll
            for (int g = 0; g < static_cast<int>(C::kSfbGroups); ++g) {
              if constexpr (kBN % 128 != 0)
                sb[kb * C::kSfbGroups + g] = mid ? w[g + 2] : w[g];
              else
                sb[kb * C::kSfbGroups + g] = w[g];
            }
          }
          if (!slot_free()) {
            fault = kFaultMmaWait;
            break;
          }
          tmem_st_32x32b_x16(t_quarter + C::kSfaCol + static_cast<uint32_t>(slot) * C::kSfaSlotCols, sa);
#pragma unroll
          for (int c = 0; c < static_cast<int>(C::kSfbSlotCols / 8); ++c)
            tmem_st_32x32b_x8(t_quarter + C::kSfbCol + static_cast<uint32_t>(slot) * C::kSfbSlotCols + c * 8,
                              sb + 8 * c);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_leader(&full[stage]);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
        if (++slot == R) slot = 0;
      }
    }
    if (fault != 0u) *abort_flag = 1;
  };
  auto run_transform = [&]() {
    // ------------------------------------------------------------ W4A16 transform warps
    // Dequantize this CTA's B rows of each k-tile, as landed (codes 32 bytes
    // a row, the k-tile's scale atoms), into the stage's bf16 B tile in the
    // 128-byte-swizzled K-major layout the MMA descriptors describe:
    //   w = bf16_rn(fl(fl(e2m1(q) * e4m3(s)) * g))   (the first product exact)
    // Work item i of the 2 * kBNc per k-tile = half i % 2 (32 elements, two
    // 16-element blocks) of row i / 2; the four warps take every 128th item,
    // two at a time (one transform warp per scheduler: the second item's
    // independent chain hides the first one's latencies).
    if constexpr (kW16) {
      const int t = (warp & 3) * 32 + lane;
      const float g = p.w_scale;  // the weight's per-tensor scale
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = cluster; tile < p.num_tiles && fault == 0u; tile += num_clusters) {
        const int n0 = (tile / p.tiles_m) * kBN;
        const int brow = n0 + static_cast<int>(rank) * C::kBNc;
        for (int kt = kt_begin; kt < kt_end; ++kt) {
          const bool landed = mbar_wait(&sfin[stage], phase, abort_flag);
          __syncwarp();
          if (!__all_sync(0xffffffffu, landed)) {
            fault = kFaultMmaWait;
            break;
          }
          const uint8_t* cb = smem + C::kOffCode + stage * C::kCodeBytes;
          const uint8_t* sb = smem + C::kOffSfb + stage * C::kSfbBytes;
          uint8_t* bb = smem + C::kOffB + stage * C::kBBytes;
#pragma unroll 2
          for (int i = t; i < 2 * C::kBNc; i += 128) {
            const int row = i >> 1, half = i & 1;
            const int rg = brow + row;  // B row in the weight (rows past N arrived zero-filled)
            const uint4 c = *reinterpret_cast<const uint4*>(cb + row * 32 + half * 16);
            const int blk = (rg >> 7) - (n0 >> 7);
            const uint32_t sw = *reinterpret_cast<const uint32_t*>(sb + blk * 512 + (rg & 31) * 16 + ((rg & 127) >> 5) * 4);
            const uint32_t words[4] = {c.x, c.y, c.z, c.w};
            // this half's two block scales as an f16 pair (low half: the first block)
            const uint32_t s01 = e4m3x2_to_f16x2(sw >> (16 * half));
            const uint32_t sb0 = __byte_perm(s01, 0u, 0x1010), sb1 = __byte_perm(s01, 0u, 0x3232);
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // 8 elements = one 16-byte chunk of bf16
              uint32_t o[4];
              nvfp4x8_to_bf16(words[j], j < 2 ? sb0 : sb1, g, o);
              const int chunk = half * 4 + j;
              *reinterpret_cast<uint4*>(bb + row * 128 + ((chunk ^ (row & 7)) * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
          // The MMA (async proxy) reads what these generic stores wrote: the
          // proxy fence, then an arrival released at CTA scope, as the scale
          // movers do for TMEM.  The stores are performed in this CTA's own
          // shared memory before its arrival leaves the CTA, and the pair MMA
          // reads this CTA's half of B from there.  (A cluster-scope release
          // on every arrival gave bit-identical results at half the speed.)
          fence_async_smem();
          __syncwarp();
          if (lane == 0) arrive_leader(&full[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (fault != 0u) *abort_flag = 1;
    }
  };
  // One 32-column chunk of a 32-row slice, as bf16 words (w[j] = columns 2j,
  // 2j+1 of this thread's row): the fused epilogue's column ranges pick the
  // destination and activation; bf16 chunks go out through the TMA, NVFP4
  // chunks are quantized (two 16-element blocks) into the next layer's codes
  // and swizzled scales (sf_word collects the 64-column group's scale word).
  const int m_padded = (p.M + 127) & ~127;  // rows of the next layer's scale buffer
  // (pend holds the codes of a 64-column group's first chunk until its second
  // one completes the row's 32 bytes, written as one whole sector)
  const bool codes32 = (reinterpret_cast<uintptr_t>(p.codes_next) & 31u) == 0;
  // the fused epilogue's quantize: d6 = fl(6 g_next) and its reciprocal, once
  const float next_d6 = __fmul_rn(6.0f, p.g_next);
  const float next_rd6 = __frcp_rn(next_d6);
  // plain epilogue with an amax output: this thread's largest |Y| so far (two
  // bf16 lanes), folded into p.amax_out once per warp when its role ends
  const bool want_amax = !kFused && p.amax_out != nullptr;
  uint32_t amax2 = 0u;
  auto flush_amax = [&]() {
    if (!want_amax) return;
    __syncwarp();
    const uint32_t m = __reduce_max_sync(0xffffffffu, max(amax2 & 0xFFFFu, amax2 >> 16));
    if (lane == 0 && m != 0u) atomicMax(p.amax_out, m << 16);  // the bf16 bits as float bits
  };
  auto emit_chunk = [&](uint32_t (&w)[16], int n, int row_base, uint8_t* stage_buf, int& buf, uint32_t& sf_word,
                        uint32_t (&pend)[4]) {
    const int row = row_base + lane;
    int act = NVFP4_ACT_NONE, dst = NVFP4_DST_BF16, out_col = n;
    if (kFused) {
      int hit = -1;
      for (int i = 0; i < p.n_ranges; ++i)
        if (n >= p.ranges[i].begin && n < p.ranges[i].end) hit = i;
      if (hit < 0) return;
      act = p.ranges[hit].act;
      dst = p.ranges[hit].dst;
      out_col = p.ranges[hit].dst_col + (n - p.ranges[hit].begin);
    }
    if (kFused && act == NVFP4_ACT_GELU_TANH) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        w[j] = pack_bf16x2(gelu_tanh_f32(bf16_lo(w[j])), gelu_tanh_f32(bf16_hi(w[j])));
    }
    if (!kFused || dst == NVFP4_DST_BF16) {
      if (row_base < p.M) {
        store_chunk_bf16(&tmap_y, stage_buf + buf * 2048, w, lane, out_col, row_base);
        if (want_amax && row < p.M) {
#pragma unroll
          for (int j = 0; j < 16; ++j) amax2 = bf16x2_absmax(amax2, w[j]);
        }
        buf ^= 1;
      }
    } else {
      // next layer's NVFP4 input: two 16-element blocks per chunk
      const float g = p.g_next;
      float blk[16];
      uint32_t c0, c1, c2, c3;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        blk[2 * j] = bf16_lo(w[j]);
        blk[2 * j + 1] = bf16_hi(w[j]);
      }
      const uint32_t s0 = quantize_block16_rd(blk, g, next_d6, next_rd6, c0, c1);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        blk[2 * j] = bf16_lo(w[8 + j]);
        blk[2 * j + 1] = bf16_hi(w[8 + j]);
      }
      const uint32_t s1 = quantize_block16_rd(blk, g, next_d6, next_rd6, c2, c3);
      const int csf = out_col >> 4;  // scale column of the first block (even)
      uint8_t* crow = p.codes_next + static_cast<size_t>(row) * (p.k_next >> 1) + (out_col >> 1);
      if ((csf & 3) == 0) {
        pend[0] = c0;
        pend[1] = c1;
        pend[2] = c2;
        pend[3] = c3;
      } else if (row < p.M) {  // the row's 32 bytes of this 64-column group
        if (codes32) {
          const uint32_t cw[8] = {pend[0], pend[1], pend[2], pend[3], c0, c1, c2, c3};
          st_global_v8(crow - 16, cw);
        } else {
          *reinterpret_cast<uint4*>(crow - 16) = make_uint4(pend[0], pend[1], pend[2], pend[3]);
          *reinterpret_cast<uint4*>(crow) = make_uint4(c0, c1, c2, c3);
        }
      }
      sf_word |= (s0 | (s1 << 8)) << (8 * (csf & 3));
      if ((csf & 3) == 2) {  // the 64-column group is complete
        const uint32_t word = row < p.M ? sf_word : 0u;  // padding rows of the scale buffer are zero
        if (row < m_padded) *reinterpret_cast<uint32_t*>(p.sf_next + sf_offset(row, csf & ~3, p.k_next >> 6)) = word;
        sf_word = 0u;
      }
    }
  };

  auto run_epilogue_wide = [&]() {
    if constexpr (C::kWide) {
    // ------------------------------------------------------------ epilogue, wide tiles
    // Warp e (0-7) owns TMEM lane quarter e % 4 (rows 32q..32q+31 of this
    // CTA's 128) and columns 128h..128h+127 of the tile, h = e / 4.  It reads
    // its whole slice into registers, hands the accumulator back at once, and
    // only then applies alpha and bias and stores bf16 through the TMA.
    const int e = warp - 4;
    const int q = warp & 3;
    const int h = e >> 2;
    uint8_t* stage_buf = smem + C::kOffEpi + e * 4096;
    uint8_t* bias_buf = smem + C::kOffBias + e * 256;
    int buf = 0;
    uint32_t acc_phase = 0;
    const float alpha = __fmul_rn(p.alpha, p.alpha_scale != nullptr ? *p.alpha_scale : p.alpha_mul);
    for (int tile = cluster; tile < p.num_tiles; tile += num_clusters) {
      const int tm = tile % p.tiles_m;
      const int c0 = (tile / p.tiles_m) * kBN + h * 128;  // first column of this warp's slice
      // this slice's bias (4 values per lane), staged while the MMAs run
      __syncwarp();  // every lane is done with the previous tile's values
      {
        uint2 bv = make_uint2(0u, 0u);
        const int cb = c0 + lane * 4;
        if (p.bias != nullptr && cb < p.N) bv = __ldg(reinterpret_cast<const uint2*>(p.bias + cb));
        *reinterpret_cast<uint2*>(bias_buf + lane * 8) = bv;
      }
      const bool got = mbar_wait(&acc_full[0], acc_phase, abort_flag);
      __syncwarp();  // tcgen05.ld below needs the whole warp converged
      if (!__all_sync(0xffffffffu, got)) {
        fault = kFaultEpilogueWait;
        break;
      }
      tc_fence_after();
      const int row_base = (tm * kCG + static_cast<int>(rank)) * 128 + q * 32;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(h * 128);
      // two 64-column loads: with four 32-column ones the compiler spilled
      // parts of the slice to local memory (and the MLP-up GEMM ran 8% slower)
      uint32_t r[128];
      tmem_ld_32x32b_x64(t_row, r);
      tmem_ld_32x32b_x64(t_row + 64, r + 64);
      tmem_ld_wait_n<128>(r);
      // the accumulator is in registers: the next tile's MMAs may start
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(&acc_empty[0]);
      acc_phase ^= 1u;
      // y = bf16(alpha * acc + bias) (row-wise FP8: fl(s_a[row] * s_b[n]) in
      // place of alpha), packed two columns per word
      const int row = row_base + lane;
      const float sa = kRow ? (row < p.M ? __ldg(p.row_scale + row) : 0.0f) : 0.0f;
      uint32_t sf_word = 0u;
      uint32_t pend[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int n = c0 + c * 32;
        if (n >= p.N) break;
        uint32_t w[16];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint4 b = *reinterpret_cast<const uint4*>(bias_buf + c * 64 + g * 16);
          const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
          float4 cs0 = make_float4(0.0f, 0.0f, 0.0f, 0.0f), cs1 = cs0;
          if constexpr (kRow) {
            if (n + 8 * g < p.N) {
              cs0 = __ldg(reinterpret_cast<const float4*>(p.col_scale + n + 8 * g));
              cs1 = __ldg(reinterpret_cast<const float4*>(p.col_scale + n + 8 * g + 4));
            }
          }
          const float csv[8] = {cs0.x, cs0.y, cs0.z, cs0.w, cs1.x, cs1.y, cs1.z, cs1.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int j = c * 32 + g * 8 + 2 * t;
            const float a0 = kRow ? __fmul_rn(sa, csv[2 * t]) : alpha;
            const float a1 = kRow ? __fmul_rn(sa, csv[2 * t + 1]) : alpha;
            w[4 * g + t] = pack_bf16x2(fmaf(a0, __uint_as_float(r[j]), bf16_lo(bw[t])),
                                       fmaf(a1, __uint_as_float(r[j + 1]), bf16_hi(bw[t])));
          }
        }
        emit_chunk(w, n, row_base, stage_buf, buf, sf_word, pend);
      }
    }
    flush_amax();
    if (lane == 0) bulk_wait<0>();
    if (fault != 0u) *abort_flag = 1;
    }
  };
  auto run_epilogue = [&]() {
    if constexpr (!C::kWide) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint8_t* stage_buf = smem + C::kOffEpi + (warp - 2) * 4096;
    int buf = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    // alpha = fl(g_a * g_b) when the two scales are passed apart (alpha_mul,
    // or g_a measured on the device and read here); fl(alpha * 1) = alpha
    const float alpha = __fmul_rn(p.alpha, p.alpha_scale != nullptr ? *p.alpha_scale : p.alpha_mul);
    for (int tile = cluster; tile < p.num_tiles; tile += num_clusters) {
      const int tm = tile % p.tiles_m;
      const int n0 = (tile / p.tiles_m) * kBN;
      const bool got = mbar_wait(&acc_full[acc], acc_phase, abort_flag);
      __syncwarp();  // tcgen05.ld below needs the whole warp converged
      if (!__all_sync(0xffffffffu, got)) {
        fault = kFaultEpilogueWait;
        break;
      }
      tc_fence_after();
      const int row_base = (tm * kCG + static_cast<int>(rank)) * 128 + q * 32;
      const int row = row_base + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kBN);
      if constexpr (!kFused && !kMx) {
        if (p.k_split > 1) {
          // K split: this group's raw partial sums to this CTA's shared memory
          // (the stage ring is idle: one tile per cluster, all of its k-tiles
          // consumed), summed across the cluster once every role is done
          uint8_t* prow = smem + (q * 32 + lane) * C::kPartStride;
#pragma unroll 1
          for (int c = 0; c < C::kChunks; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + c * 32, r);
            tmem_ld_wait(r);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              *reinterpret_cast<uint4*>(prow + c * 128 + v * 16) = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
          }
          continue;
        }
      }
      uint32_t sf_word = 0u;
      uint32_t pend[4] = {0u, 0u, 0u, 0u};
#pragma unroll 1
      for (int c = 0; c < C::kChunks; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + c * 32, r);
        tmem_ld_wait(r);
        if (c == C::kChunks - 1) {
          // accumulator fully read: hand it back to the MMA issuer
          tc_fence_before();
          __syncwarp();
          if (lane == 0) arrive_leader(&acc_empty[acc]);
        }
        const int n = n0 + c * 32;
        if (n >= p.N) continue;
        if (kFused) {  // chunks outside every column range are not written
          bool hit = false;
          for (int i = 0; i < p.n_ranges; ++i) hit |= n >= p.ranges[i].begin && n < p.ranges[i].end;
          if (!hit) continue;
        }
        uint32_t w[16];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint4 b = make_uint4(0u, 0u, 0u, 0u);
          if (p.bias != nullptr && n + 8 * g < p.N) b = __ldg(reinterpret_cast<const uint4*>(p.bias + n + 8 * g));
          const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
          if constexpr (kRow) {
            // row-wise FP8: y = fl(s_a[row] * s_b[n]) * acc + bias
            const float sa = row < p.M ? __ldg(p.row_scale + row) : 0.0f;
            float4 cs0 = make_float4(0.0f, 0.0f, 0.0f, 0.0f), cs1 = cs0;
            if (n + 8 * g < p.N) {
              cs0 = __ldg(reinterpret_cast<const float4*>(p.col_scale + n + 8 * g));
              cs1 = __ldg(reinterpret_cast<const float4*>(p.col_scale + n + 8 * g + 4));
            }
            const float csv[8] = {cs0.x, cs0.y, cs0.z, cs0.w, cs1.x, cs1.y, cs1.z, cs1.w};
#pragma unroll
            for (int t = 0; t < 4; ++t)
              w[4 * g + t] = pack_bf16x2(fmaf(__fmul_rn(sa, csv[2 * t]), __uint_as_float(r[8 * g + 2 * t]), bf16_lo(bw[t])),
                                         fmaf(__fmul_rn(sa, csv[2 * t + 1]), __uint_as_float(r[8 * g + 2 * t + 1]),
                                              bf16_hi(bw[t])));
          } else {
#pragma unroll
            for (int t = 0; t < 4; ++t)
              w[4 * g + t] = pack_bf16x2(fmaf(alpha, __uint_as_float(r[8 * g + 2 * t]), bf16_lo(bw[t])),
                                         fmaf(alpha, __uint_as_float(r[8 * g + 2 * t + 1]), bf16_hi(bw[t])));
          }
        }
        emit_chunk(w, n, row_base, stage_buf, buf, sf_word, pend);
      }
      if (++acc == kAcc) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    flush_amax();
    if (lane == 0) bulk_wait<0>();
    if (fault != 0u) *abort_flag = 1;
    }
  };

  if constexpr (C::kWide) {
    // One role per warpgroup, each with its own register budget (512 threads
    // x 128 at launch): the two epilogue warpgroups hold a 128-column
    // accumulator slice per thread; 56 + 88 + 2 x 184 = 4 x 128.
    const int wg = warp >> 2;
    if (wg == 0) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
      if (warp == 0 || warp == 2)
        run_producer();
      else if (warp == 1)
        run_mma();
    } else if (wg == 3) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 88;" ::: "memory");
      if constexpr (kW16)
        run_transform();
      else if constexpr (!kRow)
        run_movers();  // row-wise FP8 has no block scales to move
    } else {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 184;" ::: "memory");
      run_epilogue_wide();
    }
  } else {
    if (is_producer)
      run_producer();
    else if (warp == 1)
      run_mma();
    else if (is_mover) {
      if constexpr (kW16)
        run_transform();
      else if constexpr (!kRow)
        run_movers();  // row-wise FP8 has no block scales to move
    } else if (is_epilogue)
      run_epilogue();
  }

  if constexpr (!C::kWide && !kFused && !kMx) {
    if (p.k_split > 1) {
      // ------------------------------------------------------------ K-split reduction
      // Every group's partial tile is in its CTA's shared memory once the
      // cluster barrier completes.  CTA (split s, pair rank r) then finishes
      // rows [s * 128 / k_split, (s + 1) * 128 / k_split) of the r-th 128-row
      // half: the k_split partials summed in split order (so the result is
      // deterministic), y = bf16(alpha * sum + bias), 16 bytes a thread.
      tc_fence_before();
      __syncthreads();
      cluster_sync();
      const float alpha = __fmul_rn(p.alpha, p.alpha_scale != nullptr ? *p.alpha_scale : p.alpha_mul);
      const int rows = 128 / p.k_split;
      constexpr int kGroupsN = kBN / 8;
      const int tm = cluster % p.tiles_m;  // one tile per cluster
      const int n0 = (cluster / p.tiles_m) * kBN;
      const uint32_t part = smem_u32(smem);
      for (int it = threadIdx.x; it < rows * kGroupsN; it += C::kThreads) {
        const int rr = split * rows + it / kGroupsN;
        const int cg = it % kGroupsN;
        const int m = (tm * kCG + static_cast<int>(rank)) * 128 + rr;
        const int n = n0 + cg * 8;
        if (m >= p.M || n >= p.N) continue;
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int s2 = 0; s2 < p.k_split; ++s2) {
          const uint32_t src = peer_smem(part + static_cast<uint32_t>(rr) * C::kPartStride + cg * 32,
                                         static_cast<uint32_t>(s2 * kCG) + rank);
          const float4 a = ld_shared_cluster_f4(src), b = ld_shared_cluster_f4(src + 16);
          v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
          v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
        }
        uint4 bv = make_uint4(0u, 0u, 0u, 0u);
        if (p.bias != nullptr) bv = __ldg(reinterpret_cast<const uint4*>(p.bias + n));
        const uint4 o = make_uint4(pack_bf16x2(fmaf(alpha, v[0], bf16_lo(bv.x)), fmaf(alpha, v[1], bf16_hi(bv.x))),
                                   pack_bf16x2(fmaf(alpha, v[2], bf16_lo(bv.y)), fmaf(alpha, v[3], bf16_hi(bv.y))),
                                   pack_bf16x2(fmaf(alpha, v[4], bf16_lo(bv.z)), fmaf(alpha, v[5], bf16_hi(bv.z))),
                                   pack_bf16x2(fmaf(alpha, v[6], bf16_lo(bv.w)), fmaf(alpha, v[7], bf16_hi(bv.w))));
        *reinterpret_cast<uint4*>(p.y + static_cast<size_t>(m) * p.ldy + n) = o;
        if (want_amax) amax2 = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(amax2, o.x), o.y), o.z), o.w);
      }
      flush_amax();
    }
  }
  if (fault != 0u && lane == 0 && p.fault != nullptr) atomicOr(p.fault, fault);
  tc_fence_before();
  __syncthreads();
  // the peers no longer read this CTA's shared memory (the pair MMA, the
  // K-split reduction) or signal its barriers
  if (kCG == 2 || p.k_split > 1) cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc<kCG>(tmem_base, kTmemCols);
  }
}

template <int kCG, int kBN, int kAcc, bool kFused, bool kMx, bool kRow = false, bool kW16 = false>
cudaError_t launch(const GemmTensorMaps& m, const GemmParams& p, cudaStream_t stream, const DeviceInfo& dev) {
  using C = Cfg<kCG, kBN, kAcc, kMx, kRow, kW16>;
  auto kernel = gemm_nvf4_kernel<kCG, kBN, kAcc, kFused, kMx, kRow, kW16>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kCG == 2 ? 1 : 0;
  if (p.k_split > 1) {
    // K split: one tile per cluster of kCG * k_split CTAs (at most 8, the
    // portable cluster size); the clusters are independent, so they need not
    // all be resident at once
    if (C::kWide || kFused || kMx || kCG * p.k_split > 8) return cudaErrorInvalidConfiguration;
    attr[0].val.clusterDim.x = static_cast<unsigned>(kCG * p.k_split);
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(p.num_tiles * kCG * p.k_split), 1, 1);
    err = cudaLaunchKernelEx(&cfg, kernel, m.a, m.b, m.sfa, m.sfb, m.y, p);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
  }
  // A persistent grid must be co-resident: as many CTA groups as fit at once,
  // found once per template instance and device (two host threads that race
  // on the first launch compute and store the same value).
  static std::atomic<int> groups_cache[kMaxDevices];
  int max_groups = groups_cache[dev.device].load(std::memory_order_relaxed);
  if (max_groups == 0) {
    int n = dev.num_sms / kCG;
    if (kCG == 2) {
      cfg.gridDim = dim3(static_cast<unsigned>(2 * n), 1, 1);
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) == cudaSuccess && clusters > 0 && clusters < n)
        n = clusters;
    }
    max_groups = n;
    groups_cache[dev.device].store(n, std::memory_order_relaxed);
  }
  const int groups = p.num_tiles < max_groups ? p.num_tiles : max_groups;
  cfg.gridDim = dim3(static_cast<unsigned>(groups * kCG), 1, 1);
  err = cudaLaunchKernelEx(&cfg, kernel, m.a, m.b, m.sfa, m.sfb, m.y, p);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

GemmConfig gemm_config(int64_t M, int64_t N, int num_sms) {
  if (M <= 128) return GemmConfig{1, 192, 2};
  // 256 x 256 tiles do a third more MMA work per pipeline step than 256 x 192
  // ones for the same per-k-tile synchronisation, but leave SMs idle when
  // there are fewer tiles than CTA pairs.
  const int64_t pairs = num_sms / 2;
  const int64_t wide_tiles = ((M + 255) / 256) * ((N + 255) / 256);
  if (wide_tiles >= pairs) return GemmConfig{2, 256, 1};
  // Few tiles (a few hundred tokens): narrower 256 x 128 tiles put more CTA
  // pairs to work as long as they still fit in one wave.
  const int64_t tiles192 = ((M + 255) / 256) * ((N + 191) / 192);
  const int64_t tiles128 = ((M + 255) / 256) * ((N + 127) / 128);
  if (tiles192 < pairs && tiles128 <= pairs) return GemmConfig{2, 128, 2};
  return GemmConfig{2, 192, 2};
}

GemmPlan gemm_plan(int64_t M, int64_t N, int num_kt, int num_sms) {
  const GemmConfig base = gemm_config(M, N, num_sms);
  if (base.cta_group == 2 && base.tile_n == 256) return GemmPlan{base, 1};  // a tile for every CTA pair
  // Cost of a shape, in k-tiles of one CTA group: the tiles in waves of the
  // co-resident groups; or, with few tiles, the share of the K range of a
  // power-of-two split plus kSplitCost for the split's own work (writing the
  // partial tile, two cluster barriers, the reduction through distributed
  // shared memory).  A split keeps every cluster within 4 CTAs and all of them
  // resident at once (at most 7/8 of the SMs: clusters of 4 CTAs with this
  // kernel's shared memory fit 33 at a time on 148 SMs, of 8 only 15), and at
  // least one k-tile to a range.
  constexpr int64_t kSplitCost = 6;
  auto cost = [&](const GemmConfig& c, int* ks_out) {
    const int64_t groups = num_sms / c.cta_group;
    const int64_t tiles = ((M + 128 * c.cta_group - 1) / (128 * c.cta_group)) * ((N + c.tile_n - 1) / c.tile_n);
    *ks_out = 1;
    if (tiles > groups) return static_cast<int64_t>(num_kt) * ((tiles + groups - 1) / groups);
    int64_t best_c = num_kt;
    for (int ks = 2; ks * c.cta_group <= 4 && ks <= num_kt && tiles * ks * c.cta_group * 8 <= num_sms * 7; ks *= 2) {
      const int64_t cc = (num_kt + ks - 1) / ks + kSplitCost;
      if (cc < best_c) {
        best_c = cc;
        *ks_out = ks;
      }
    }
    return best_c;
  };
  GemmPlan best{base, 1};
  int64_t best_cost = cost(base, &best.k_split);
  if (M > 128) {
    for (const GemmConfig c : {GemmConfig{2, 192, 2}, GemmConfig{2, 128, 2}}) {
      int ks = 1;
      const int64_t cc = cost(c, &ks);
      if (cc < best_cost) {
        best = GemmPlan{c, ks};
        best_cost = cc;
      }
    }
  }
  return best;
}

cudaError_t launch_gemm_w4a16(const GemmTensorMaps& m, const GemmParams& p, const GemmConfig& c, cudaStream_t stream,
                              const DeviceInfo& dev) {
  if (c.cta_group == 2 && c.tile_n == 256 && c.acc_bufs == 1)
    return launch<2, 256, 1, false, false, false, true>(m, p, stream, dev);
  if (c.cta_group == 2 && c.tile_n == 192 && c.acc_bufs == 2)
    return launch<2, 192, 2, false, false, false, true>(m, p, stream, dev);
  if (c.cta_group == 2 && c.tile_n == 128 && c.acc_bufs == 2)
    return launch<2, 128, 2, false, false, false, true>(m, p, stream, dev);
  if (c.cta_group == 1 && c.tile_n == 192 && c.acc_bufs == 2)
    return launch<1, 192, 2, false, false, false, true>(m, p, stream, dev);
  return cudaErrorInvalidConfiguration;
}

cudaError_t launch_gemm(const GemmTensorMaps& m, const GemmParams& p, const GemmConfig& c, bool fused, bool mx,
                        cudaStream_t stream, const DeviceInfo& dev, bool row) {
  if (row) {  // row-wise FP8: the default tile shapes, no fused epilogue
    if (fused || !mx) return cudaErrorInvalidConfiguration;
    if (c.cta_group == 2 && c.tile_n == 256 && c.acc_bufs == 1)
      return launch<2, 256, 1, false, true, true>(m, p, stream, dev);
    if (c.cta_group == 2 && c.tile_n == 192 && c.acc_bufs == 2)
      return launch<2, 192, 2, false, true, true>(m, p, stream, dev);
    if (c.cta_group == 2 && c.tile_n == 128 && c.acc_bufs == 2)
      return launch<2, 128, 2, false, true, true>(m, p, stream, dev);
    if (c.cta_group == 1 && c.tile_n == 192 && c.acc_bufs == 2)
      return launch<1, 192, 2, false, true, true>(m, p, stream, dev);
    return cudaErrorInvalidConfiguration;
  }
  if (mx) {  // MXFP8 operands: the default tile shapes, no fused epilogue
    if (fused) return cudaErrorInvalidConfiguration;
    if (c.cta_group == 2 && c.tile_n == 256 && c.acc_bufs == 1) return launch<2, 256, 1, false, true>(m, p, stream, dev);
    if (c.cta_group == 2 && c.tile_n == 192 && c.acc_bufs == 2) return launch<2, 192, 2, false, true>(m, p, stream, dev);
    if (c.cta_group == 2 && c.tile_n == 128 && c.acc_bufs == 2) return launch<2, 128, 2, false, true>(m, p, stream, dev);
    if (c.cta_group == 1 && c.tile_n == 192 && c.acc_bufs == 2) return launch<1, 192, 2, false, true>(m, p, stream, dev);
    return cudaErrorInvalidConfiguration;
  }
#define NVFP4_GEMM_CASE(CG, BN, ACC)                                                                          \
  if (c.cta_group == CG && c.tile_n == BN && c.acc_bufs == ACC)                                             \
    return fused ? launch<CG, BN, ACC, true, false>(m, p, stream, dev)                                      \
                 : launch<CG, BN, ACC, false, false>(m, p, stream, dev);
  NVFP4_GEMM_CASE(2, 256, 1)
  NVFP4_GEMM_CASE(2, 192, 2)
  NVFP4_GEMM_CASE(2, 128, 2)
  NVFP4_GEMM_CASE(1, 192, 2)
#undef NVFP4_GEMM_CASE
  return cudaErrorInvalidConfiguration;
}

}  // namespace nvfp4
