// Declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "device.cuh"
#include "nvfp4.h"

namespace nvfp4 {

// Devices the per-device caches of the library cover (device index < this).
constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int device = -1;
  int num_sms = 0;
  int cc_major = 0, cc_minor = 0;
  size_t max_smem_optin = 0;
  unsigned* fault = nullptr;  // device address of the fault word
};

// One column range of the fused epilogue, as the kernel sees it.
struct EpiRange {
  int32_t begin, end, act, dst, dst_col;
};

struct GemmParams {
  int32_t M, N, K;
  int32_t tiles_m, tiles_n, num_tiles;  // tiles_m counts (128 * CTA-group)-row tiles
  int32_t num_kt;  // k-tiles of 256 elements (last one may be partial)
  int32_t kblocks; // MMA k-blocks in total: K / 64 (NVFP4) or K / 32 (MXFP8)
  float alpha;
  float alpha_mul;            // the epilogue uses fl(alpha * alpha_mul) (1 when alpha is given whole)
  const float* alpha_scale;   // nullable: if set, the epilogue uses fl(alpha * alpha_scale[0]) instead
  const float* row_scale;     // row-wise FP8: [M] scales of A's rows
  const float* col_scale;     // row-wise FP8: [N] scales of B's rows (output columns)
  float w_scale;              // W4A16: the weight's per-tensor scale, applied by the transform warps
  int32_t k_split;            // tile groups per cluster that share one output tile (K split); 1 = none
  __nv_bfloat16* y;           // K split: the bf16 output [M, ldy], written by the cluster's reduction
  int32_t ldy;
  const __nv_bfloat16* bias;  // nullable
  unsigned* amax_out;         // nullable (plain epilogue): atomic max of |Y| as float bits
  unsigned* fault;
  // fused epilogue (only read by the fused kernel)
  int32_t n_ranges;
  EpiRange ranges[NVFP4_MAX_RANGES];
  float g_next;
  uint8_t* codes_next;
  uint8_t* sf_next;
  int32_t k_next;
};

// TMA descriptors of one GEMM launch.
struct GemmTensorMaps {
  CUtensorMap a, b;      // codes, [rows, K/2] uint8, 128-byte swizzle
  CUtensorMap sfa, sfb;  // swizzled scales as [row blocks][K/64 atoms][128 x u32]
  CUtensorMap y;         // bf16 destination of the plain or BF16-range epilogue
};

// Per-call state of the dynamic-scale quantize.
struct DynamicScaleArgs {
  const uint8_t* x;  // bf16 [M, K], for the amax pass
  uint32_t* scratch; // [0] bits of the grid-wide max |x|, [1] CTAs arrived; both start at zero
  float* scale_out;  // [0] amax, [1] g, written by CTA 0
  uint64_t wait_limit_ns;  // longest wait for the other CTAs' arrivals
  uint32_t expect;         // arrivals that complete the wait (the grid size, plus any test-only extra)
  const float* amax_in;    // one-pass variant: g derived on the device from this amax (no amax pass)
};

// Grid-wait settings of the dynamic quantize (normally kWaitLimitNs and no
// extra arrivals; a test of the time-out path changes them for its thread).
struct GridWaitSettings {
  uint64_t limit_ns = kWaitLimitNs;
  uint32_t extra_arrivals = 0;
};
// Bytes of scratch one dynamic-scale quantize uses (zeroed by the launch).
constexpr size_t kDynamicScratchBytes = 8;

// Rows of one quantize tile for a [M, K] input (128 or 256): the TMA box
// height of the bf16 input's tensor map, passed back to the launch.
int quantize_tile_rows(int64_t M, int64_t K, int num_sms);
// tmap_x: bf16 [M, K], box tile_rows rows x 64 columns, 128-byte swizzle.
cudaError_t launch_quantize(const CUtensorMap& tmap_x, int tile_rows, int64_t M, int64_t K, float g, uint8_t* codes,
                            uint8_t* sf, cudaStream_t stream, const DeviceInfo& dev);
// MXFP8 (E4M3 codes [M, K], E8M0 scales, one per 32 elements, swizzled).
cudaError_t launch_quantize_mxfp8(const CUtensorMap& tmap_x, int tile_rows, int64_t M, int64_t K, uint8_t* codes,
                                  uint8_t* sf, cudaStream_t stream, const DeviceInfo& dev);
// Same, with g derived on the device from amax_in[0] (as the dynamic
// variant derives it from its own amax pass); scale_out gets [amax, g].
cudaError_t launch_quantize_from_amax(const CUtensorMap& tmap_x, int tile_rows, int64_t M, int64_t K,
                                      const float* amax_in, uint8_t* codes, uint8_t* sf, float* scale_out,
                                      cudaStream_t stream, const DeviceInfo& dev);
// Same, with g measured on x in the same (cooperative) launch.
cudaError_t launch_quantize_dynamic(const CUtensorMap& tmap_x, int tile_rows, const void* x, int64_t M, int64_t K,
                                    uint8_t* codes, uint8_t* sf, float* scale_out, uint32_t* scratch,
                                    const GridWaitSettings& wait, cudaStream_t stream, const DeviceInfo& dev);
cudaError_t launch_calibrate(const void* x, int64_t n, float* out, cudaStream_t stream, const DeviceInfo& dev);
cudaError_t launch_swizzle_sf(const uint8_t* sf_lin, int64_t rows, int64_t k, uint8_t* out, cudaStream_t stream);

// Tile configuration of one GEMM launch.
struct GemmConfig {
  int cta_group;  // 1: one CTA per 128-row tile; 2: CTA pairs with 256-row tiles
  int tile_n;     // output tile width
  int acc_bufs;   // accumulator buffers in TMEM
};
GemmConfig gemm_config(int64_t M, int64_t N, int num_sms);
// Tile shape and K split of a GEMM whose epilogue is the plain one (NVFP4 and
// W4A16 with bias): when the tiles cannot fill the SMs, up to 8 CTAs (4 CTA
// pairs) of a cluster share one tile over disjoint k-tile ranges.  num_kt:
// k-tiles of the problem (256 elements for NVFP4, 64 for W4A16).
struct GemmPlan {
  GemmConfig c;
  int k_split;
};
GemmPlan gemm_plan(int64_t M, int64_t N, int num_kt, int num_sms);
// mx: MXFP8 operands (E4M3 codes [rows, K], E8M0 scales) instead of NVFP4.
// row: row-wise FP8 (8-bit operands without block scales; requires mx).
cudaError_t launch_gemm(const GemmTensorMaps& m, const GemmParams& p, const GemmConfig& c, bool fused, bool mx,
                        cudaStream_t stream, const DeviceInfo& dev, bool row = false);
// W4A16: bf16 activations [M, K] x NVFP4 weights [N, K] dequantized in shared
// memory (p.w_scale is the weight's per-tensor scale; p.alpha = 1);
// maps: a = bf16 activations (64-element boxes), b = weight codes (32-byte
// boxes of this CTA's B rows), sfb = weight scales (one atom per k-tile).
cudaError_t launch_gemm_w4a16(const GemmTensorMaps& m, const GemmParams& p, const GemmConfig& c, cudaStream_t stream,
                              const DeviceInfo& dev);
// NVFP4 [rows, K] (codes, swizzled scales, g) -> bf16 [rows, K].
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* sf, float g, int64_t rows, int64_t K, void* out,
                              cudaStream_t stream);
// Row-wise FP8 quantize: x bf16 [M, K] -> codes [M, K] E4M3, scale [M] fp32.
cudaError_t launch_quantize_rowwise(const void* x, int64_t M, int64_t K, uint8_t* codes, float* scale,
                                    cudaStream_t stream);

}  // namespace nvfp4
