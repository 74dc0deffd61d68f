// The library's C ABI (declared in include/nvfp4.h): argument validation,
// device checks, TMA descriptor construction and kernel launch.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "internal.h"

namespace nvfp4 {

namespace {

// Fault word: kernels OR a code in here when a barrier wait times out.
__device__ unsigned int g_fault_word;

thread_local std::string t_last_error;

// Grid-wait settings the calling thread's dynamic quantizes launch with
// (changed only by nvfp4_testing_set_grid_wait).
thread_local GridWaitSettings t_grid_wait;

nvfp4_status fail(nvfp4_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
nvfp4_status fail(nvfp4_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

nvfp4_status ok() {
  t_last_error.clear();
  return NVFP4_OK;
}

nvfp4_status cuda_fail(cudaError_t e, const char* what) {
  return fail(NVFP4_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

DeviceInfo g_devices[kMaxDevices];
std::mutex g_dev_mutex;

// Properties of the current device (cached); EARCH unless it is cc 10.0.
nvfp4_status current_device(const DeviceInfo** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(NVFP4_ECUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& d = g_devices[dev];
  if (d.device != dev) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    DeviceInfo n;
    n.device = dev;
    n.num_sms = prop.multiProcessorCount;
    n.cc_major = prop.major;
    n.cc_minor = prop.minor;
    n.max_smem_optin = prop.sharedMemPerBlockOptin;
    if (n.cc_major == 10 && n.cc_minor == 0) {
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, g_fault_word);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(fault word)");
      n.fault = static_cast<unsigned*>(addr);
    }
    d = n;
  }
  if (d.cc_major != 10 || d.cc_minor != 0)
    return fail(NVFP4_EARCH, "device %d has compute capability %d.%d; this library is built for 10.0 (sm_100a)",
                dev, d.cc_major, d.cc_minor);
  *out = &d;
  return NVFP4_OK;
}

// ---------------------------------------------------------------------------
// Scratch of the no-allocation dynamic quantize.  Callers that cannot hand
// the library a workspace (a host program or plugin given only its input and
// output buffers, with no device allocator to draw one from) get the grid
// state from this fixed array in the library's own device memory instead.
// One array per device: calls that overlap in time on a device race on it.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = 256;  // the most scratch one call may use
static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoAllocScratchBytes / sizeof(uint32_t)];
uint32_t* g_noalloc_ptr[kMaxDevices];  // device address of g_noalloc_scratch, looked up once per device
std::mutex g_noalloc_mutex;

// Address of the scratch on device `dev`, which must be current.  The first
// call per device looks it up (this may load the module on the device, so it
// belongs outside any stream capture).
nvfp4_status noalloc_scratch(int dev, uint32_t** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* addr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
    g_noalloc_ptr[dev] = static_cast<uint32_t*>(addr);
  }
  *out = g_noalloc_ptr[dev];
  return NVFP4_OK;
}

// ---------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major tensor of `rank` dims (innermost first) with byte strides of
// dims 1.. in `strides`.
nvfp4_status make_tmap_nd(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int rank, const uint64_t* dims,
                          const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw, const char* what) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(NVFP4_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t d[3], st[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
  const CUresult r = fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, st, bx, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NVFP4_ECUDA, "cuTensorMapEncodeTiled(%s) failed with %d", what, (int)r);
  return NVFP4_OK;
}

// 2-D row-major tensor [outer, inner] with rows `row_bytes` apart.
nvfp4_status make_tmap(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw,
                       const char* what) {
  const uint64_t dims[2] = {inner, outer};
  const uint64_t strides[1] = {row_bytes};
  const uint32_t box[2] = {box_inner, box_outer};
  return make_tmap_nd(m, dt, base, 2, dims, strides, box, sw, what);
}

// Swizzled scale buffer of a [rows, k] tensor seen as [row blocks][atoms]
// [128 x u32]; one box = box_atoms atoms (4 = one 256-wide NVFP4 k-tile) of
// box_blocks row blocks.  Out-of-range atoms and blocks read as zero.
nvfp4_status make_sf_tmap(CUtensorMap* m, const void* sf, int64_t rows, int64_t atoms, uint32_t box_atoms,
                          uint32_t box_blocks, const char* what) {
  const uint64_t dims[3] = {128, static_cast<uint64_t>(atoms), static_cast<uint64_t>((rows + 127) / 128)};
  const uint64_t strides[2] = {512, static_cast<uint64_t>(atoms) * 512};
  const uint32_t box[3] = {128, box_atoms, box_blocks};
  return make_tmap_nd(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, sf, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                      what);
}

bool finite_f(float v) { return isfinite(v) != 0; }

// Largest row count and K of any entry point: keeps every row index and TMA
// tile coordinate inside int32.
constexpr int64_t kMaxDim = INT32_MAX / 2;

// 1 <= rows <= kMaxDim; 64 <= K <= kMaxDim with K % 64 == 0.
nvfp4_status check_rows_k(const char* rname, int64_t rows, const char* kname, int64_t K) {
  if (rows < 1 || rows > kMaxDim)
    return fail(NVFP4_EINVAL, "%s=%lld must be in [1, %lld]", rname, (long long)rows, (long long)kMaxDim);
  if (K < 64 || K % 64 != 0 || K > kMaxDim)
    return fail(NVFP4_EINVAL, "%s=%lld must be a positive multiple of 64, at most %lld", kname, (long long)K,
                (long long)kMaxDim);
  return NVFP4_OK;
}

// A one-dimensional grid of `threads`-thread blocks over `items` must fit
// gridDim.x.
bool grid_fits(int64_t items, int threads) { return (items + threads - 1) / threads <= INT32_MAX; }

bool scale_ok(float g) { return finite_f(g) && g >= 0x1p-64f && g <= 0x1p64f; }

// Two per-tensor scales whose fp32 product (the epilogue's alpha) is finite.
bool product_ok(float g_a, float g_b) {
  return finite_f(g_a) && finite_f(g_b) && finite_f(static_cast<float>(static_cast<double>(g_a) * g_b));
}

// Checks shared by the two GEMM entry points; fills the operand part of p
// and the operand tensor maps.
// mx: 8-bit operands (one E4M3 byte per element), with E8M0 scales per 32
// (MXFP8) or, with row, one fp32 scale per row passed as sfa / sfb.
// y (bf16 [M, N]) non-null: the plain NVFP4 epilogue, which may split K
// across a cluster (gemm_plan) and then writes y directly from the cluster's
// reduction.
nvfp4_status gemm_common(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb, int64_t M,
                         int64_t N, int64_t K, float alpha, const void* bias, GemmParams* p, GemmTensorMaps* maps,
                         GemmConfig* cfg, const DeviceInfo** dev, bool mx = false, bool row = false,
                         bool fused = false, void* split_y = nullptr) {
  if (!a || !sfa || !b || !sfb) return fail(NVFP4_EINVAL, "null operand pointer");
  nvfp4_status st = check_rows_k("M", M, "K", K);
  if (st != NVFP4_OK) return st;
  if (N < 8 || N % 8 != 0 || N > kMaxDim)
    return fail(NVFP4_EINVAL, "N=%lld must be a positive multiple of 8, at most %lld", (long long)N,
                (long long)kMaxDim);
  if (!finite_f(alpha)) return fail(NVFP4_EINVAL, "alpha must be finite");
  if (!aligned16(a) || !aligned16(sfa) || !aligned16(b) || !aligned16(sfb) || !aligned16(bias))
    return fail(NVFP4_EALIGN, "operand pointers must be 16-byte aligned");
  st = current_device(dev);
  if (st != NVFP4_OK) return st;

  // a k-tile is 128 bytes of every operand row: 256 fp4 or 128 fp8 elements
  const int64_t row_bytes = mx ? K : K / 2;
  const int num_kt = static_cast<int>((row_bytes + 127) / 128);
  int k_split = 1;
  if (split_y != nullptr && !mx && !row && !fused) {
    const GemmPlan plan = gemm_plan(M, N, num_kt, (*dev)->num_sms);
    *cfg = plan.c;
    k_split = plan.k_split;
  } else {
    *cfg = gemm_config(M, N, (*dev)->num_sms);
  }
  const int bn = cfg->tile_n;
  const int cg = cfg->cta_group;
  *p = GemmParams{};
  p->k_split = k_split;
  p->y = static_cast<__nv_bfloat16*>(split_y);
  p->ldy = static_cast<int32_t>(N);
  p->M = static_cast<int32_t>(M);
  p->N = static_cast<int32_t>(N);
  p->K = static_cast<int32_t>(K);
  p->tiles_m = static_cast<int32_t>((M + 128 * cg - 1) / (128 * cg));
  p->tiles_n = static_cast<int32_t>((N + bn - 1) / bn);
  const int64_t tiles = static_cast<int64_t>(p->tiles_m) * p->tiles_n;
  if (tiles > INT32_MAX) return fail(NVFP4_EINVAL, "problem too large");
  p->num_tiles = static_cast<int32_t>(tiles);
  p->num_kt = static_cast<int32_t>(num_kt);
  p->kblocks = static_cast<int32_t>(mx ? K / 32 : K / 64);
  p->alpha = alpha;
  p->alpha_mul = 1.0f;
  p->bias = static_cast<const __nv_bfloat16*>(bias);
  p->fault = (*dev)->fault;

  st = make_tmap(&maps->a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a, row_bytes, M, row_bytes, 128, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B, "A");
  if (st != NVFP4_OK) return st;
  st = make_tmap(&maps->b, CU_TENSOR_MAP_DATA_TYPE_UINT8, b, row_bytes, N, row_bytes, 128, bn / cg,
                 CU_TENSOR_MAP_SWIZZLE_128B, "B");
  if (st != NVFP4_OK) return st;
  if (row) {  // no block scales: the kernel reads the row scales in its epilogue
    p->row_scale = reinterpret_cast<const float*>(sfa);
    p->col_scale = reinterpret_cast<const float*>(sfb);
    return NVFP4_OK;
  }
  // scale atoms per 128-row block, and atoms per k-tile
  const int64_t atoms = mx ? (K / 32 + 3) / 4 : K / 64;
  const uint32_t box_atoms = mx ? 1u : 4u;
  st = make_sf_tmap(&maps->sfa, sfa, M, atoms, box_atoms, 1, "A scales");
  if (st != NVFP4_OK) return st;
  // 128-row scale blocks one B tile can touch: a width that is not a
  // multiple of 128 may start in the middle of a block
  const uint32_t sfb_blocks = static_cast<uint32_t>(bn % 128 == 0 ? bn / 128 : bn / 128 + 1);
  return make_sf_tmap(&maps->sfb, sfb, N, atoms, box_atoms, sfb_blocks, "B scales");
}

// nvfp4_gemm_quant with alpha = fl(alpha * alpha_mul) formed on the device.
nvfp4_status gemm_quant_impl(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb,
                             int64_t M, int64_t N, int64_t K, float alpha, float alpha_mul, const void* bias,
                             const nvfp4_colrange* ranges, int32_t n_ranges, void* y_bf16, int64_t ldy,
                             float g_next, uint8_t* codes_next, uint8_t* sf_next, int64_t k_next, void* stream) {
  if (!ranges || n_ranges < 1 || n_ranges > NVFP4_MAX_RANGES)
    return fail(NVFP4_EINVAL, "n_ranges=%d must be in [1, %d]", n_ranges, NVFP4_MAX_RANGES);
  bool any_bf16 = false, any_fp4 = false;
  for (int i = 0; i < n_ranges; ++i) {
    const nvfp4_colrange& r = ranges[i];
    if (r.begin < 0 || r.end <= r.begin || r.end > N || r.begin % 64 || r.end % 64 || r.dst_col < 0 ||
        r.dst_col % 64)
      return fail(NVFP4_EINVAL, "range %d [%lld, %lld) -> %lld: bounds must be multiples of 64 within [0, N]", i,
                  (long long)r.begin, (long long)r.end, (long long)r.dst_col);
    if (r.act != NVFP4_ACT_NONE && r.act != NVFP4_ACT_GELU_TANH)
      return fail(NVFP4_EINVAL, "range %d: unknown activation %d", i, r.act);
    if (r.dst == NVFP4_DST_BF16) {
      any_bf16 = true;
      if (r.dst_col + (r.end - r.begin) > ldy) return fail(NVFP4_EINVAL, "range %d overruns ldy", i);
    } else if (r.dst == NVFP4_DST_NVFP4) {
      any_fp4 = true;
      if (r.dst_col + (r.end - r.begin) > k_next) return fail(NVFP4_EINVAL, "range %d overruns k_next", i);
    } else {
      return fail(NVFP4_EINVAL, "range %d: unknown destination %d", i, r.dst);
    }
    for (int j = 0; j < i; ++j)
      if (ranges[j].begin < r.end && r.begin < ranges[j].end)
        return fail(NVFP4_EINVAL, "ranges %d and %d overlap", j, i);
  }
  if (any_bf16) {
    if (!y_bf16) return fail(NVFP4_EINVAL, "a BF16 range needs y_bf16");
    if (ldy < 8 || ldy % 8 != 0) return fail(NVFP4_EINVAL, "ldy=%lld must be a positive multiple of 8", (long long)ldy);
    if (!aligned16(y_bf16)) return fail(NVFP4_EALIGN, "y_bf16 must be 16-byte aligned");
  }
  if (any_fp4) {
    if (!codes_next || !sf_next) return fail(NVFP4_EINVAL, "an NVFP4 range needs codes_next and sf_next");
    if (k_next < 64 || k_next % 64 != 0 || k_next > INT32_MAX / 2)
      return fail(NVFP4_EINVAL, "k_next=%lld must be a positive multiple of 64", (long long)k_next);
    if (!scale_ok(g_next)) return fail(NVFP4_EINVAL, "g_next must be finite and in [2^-64, 2^64]");
    if (!aligned16(codes_next) || !aligned16(sf_next))
      return fail(NVFP4_EALIGN, "codes_next and sf_next must be 16-byte aligned");
  }
  GemmParams p;
  GemmTensorMaps maps;
  GemmConfig cg;
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = gemm_common(a, sfa, b, sfb, M, N, K, alpha, bias, &p, &maps, &cg, &dev, false, false, true);
  if (st != NVFP4_OK) return st;
  if (any_bf16) {
    st = make_tmap(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y_bf16, ldy, M, ldy * 2, 32, 32,
                   CU_TENSOR_MAP_SWIZZLE_64B, "Y");
  } else {
    // never used for a store; a valid descriptor keeps the prefetch harmless
    st = make_tmap(&maps.y, CU_TENSOR_MAP_DATA_TYPE_UINT8, a, 16, 1, 16, 16, 1, CU_TENSOR_MAP_SWIZZLE_NONE,
                   "dummy");
  }
  if (st != NVFP4_OK) return st;
  p.n_ranges = n_ranges;
  for (int i = 0; i < n_ranges; ++i) {
    p.ranges[i].begin = static_cast<int32_t>(ranges[i].begin);
    p.ranges[i].end = static_cast<int32_t>(ranges[i].end);
    p.ranges[i].act = ranges[i].act;
    p.ranges[i].dst = ranges[i].dst;
    p.ranges[i].dst_col = static_cast<int32_t>(ranges[i].dst_col);
  }
  p.g_next = g_next;
  p.codes_next = codes_next;
  p.sf_next = sf_next;
  p.k_next = static_cast<int32_t>(k_next);
  p.alpha_mul = alpha_mul;
  cudaError_t e = launch_gemm(maps, p, cg, true, false, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "gemm_quant launch");
  return ok();
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

static_assert(kDynamicScratchBytes == NVFP4_DYNAMIC_WORKSPACE_BYTES, "workspace size in the header");
static_assert(kNoAllocScratchBytes == NVFP4_NOALLOC_SCRATCH_BYTES, "no-allocation scratch size in the header");

extern "C" {

size_t nvfp4_mxfp8_sf_bytes(int64_t rows, int64_t k) {
  if (rows < 1 || k < 32 || k % 32 != 0) return 0;
  const int64_t rp = (rows + 127) / 128 * 128;
  const int64_t cp = (k / 32 + 3) / 4 * 4;
  return static_cast<size_t>(rp) * static_cast<size_t>(cp);
}

nvfp4_status nvfp4_mxfp8_quantize(const void* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* sf, void* stream) {
  if (!x || !codes || !sf) return fail(NVFP4_EINVAL, "null pointer");
  if (check_rows_k("M", M, "K", K) != NVFP4_OK) return NVFP4_EINVAL;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sf))
    return fail(NVFP4_EALIGN, "pointers must be 16-byte aligned");
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  CUtensorMap tx;
  const int tile_rows = quantize_tile_rows(M, K, dev->num_sms);
  st = make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, K * 2, 64, static_cast<uint32_t>(tile_rows),
                 CU_TENSOR_MAP_SWIZZLE_128B, "x");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_quantize_mxfp8(tx, tile_rows, M, K, codes, sf, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "mxfp8 quantize launch");
  return ok();
}

nvfp4_status nvfp4_mxfp8_gemm(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb, int64_t M,
                              int64_t N, int64_t K, float alpha, const void* bias, void* y, void* stream) {
  if (!y) return fail(NVFP4_EINVAL, "null output pointer");
  if (!aligned16(y)) return fail(NVFP4_EALIGN, "y must be 16-byte aligned");
  GemmParams p;
  GemmTensorMaps maps;
  GemmConfig cg;
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = gemm_common(a, sfa, b, sfb, M, N, K, alpha, bias, &p, &maps, &cg, &dev, true);
  if (st != NVFP4_OK) return st;
  st = make_tmap(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B, "Y");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_gemm(maps, p, cg, false, true, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "mxfp8 gemm launch");
  return ok();
}

nvfp4_status nvfp4_fp8row_quantize(const void* x, int64_t M, int64_t K, uint8_t* codes, float* scale,
                                   void* stream) {
  if (!x || !codes || !scale) return fail(NVFP4_EINVAL, "null pointer");
  if (check_rows_k("M", M, "K", K) != NVFP4_OK) return NVFP4_EINVAL;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scale))
    return fail(NVFP4_EALIGN, "pointers must be 16-byte aligned");
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_quantize_rowwise(x, M, K, codes, scale, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "row-wise fp8 quantize launch");
  return ok();
}

nvfp4_status nvfp4_fp8row_gemm(const uint8_t* a, const float* a_scale, const uint8_t* b, const float* b_scale,
                               int64_t M, int64_t N, int64_t K, const void* bias, void* y, void* stream) {
  if (!y) return fail(NVFP4_EINVAL, "null output pointer");
  if (!aligned16(y)) return fail(NVFP4_EALIGN, "y must be 16-byte aligned");
  GemmParams p;
  GemmTensorMaps maps;
  GemmConfig cg;
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = gemm_common(a, reinterpret_cast<const uint8_t*>(a_scale), b,
                                reinterpret_cast<const uint8_t*>(b_scale), M, N, K, 1.0f, bias, &p, &maps, &cg, &dev,
                                true, true);
  if (st != NVFP4_OK) return st;
  st = make_tmap(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B, "Y");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_gemm(maps, p, cg, false, true, static_cast<cudaStream_t>(stream), *dev, true);
  if (e != cudaSuccess) return cuda_fail(e, "row-wise fp8 gemm launch");
  return ok();
}

nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* sf, float g, int64_t rows, int64_t K, void* out,
                              void* stream) {
  if (!codes || !sf || !out) return fail(NVFP4_EINVAL, "null pointer");
  if (check_rows_k("rows", rows, "K", K) != NVFP4_OK) return NVFP4_EINVAL;
  if (!grid_fits(rows * (K / 32), 256)) return fail(NVFP4_EINVAL, "rows*K=%lld is too large", (long long)(rows * K));
  if (!finite_f(g)) return fail(NVFP4_EINVAL, "g must be finite");
  if (!aligned16(codes) || !aligned16(sf) || !aligned16(out))
    return fail(NVFP4_EALIGN, "pointers must be 16-byte aligned");
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_dequantize(codes, sf, g, rows, K, out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return ok();
}

size_t nvfp4_sf_bytes(int64_t rows, int64_t k) {
  if (rows < 1 || k < 16 || k % 16 != 0) return 0;
  const int64_t rp = (rows + 127) / 128 * 128;
  const int64_t cp = (k / 16 + 3) / 4 * 4;
  return static_cast<size_t>(rp) * static_cast<size_t>(cp);
}

nvfp4_status nvfp4_calibrate(const void* x, int64_t n, float* out, void* stream) {
  if (!x || !out) return fail(NVFP4_EINVAL, "null pointer");
  if (n < 8 || n % 8 != 0) return fail(NVFP4_EINVAL, "n=%lld must be a positive multiple of 8", (long long)n);
  if (!aligned16(x)) return fail(NVFP4_EALIGN, "x must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(out) & 3u) != 0) return fail(NVFP4_EALIGN, "out must be 4-byte aligned");
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_calibrate(x, n, out, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "calibrate launch");
  return ok();
}

nvfp4_status nvfp4_quantize(const void* x, int64_t M, int64_t K, float g, uint8_t* codes, uint8_t* sf,
                            void* stream) {
  if (!x || !codes || !sf) return fail(NVFP4_EINVAL, "null pointer");
  if (check_rows_k("M", M, "K", K) != NVFP4_OK) return NVFP4_EINVAL;
  if (!scale_ok(g)) return fail(NVFP4_EINVAL, "g=%g must be finite and in [2^-64, 2^64]", (double)g);
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sf))
    return fail(NVFP4_EALIGN, "pointers must be 16-byte aligned");
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  CUtensorMap tx;
  const int tile_rows = quantize_tile_rows(M, K, dev->num_sms);
  st = make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, K * 2, 64, static_cast<uint32_t>(tile_rows),
                 CU_TENSOR_MAP_SWIZZLE_128B, "x");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_quantize(tx, tile_rows, M, K, g, codes, sf, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return ok();
}

nvfp4_status nvfp4_quantize_from_amax(const void* x, int64_t M, int64_t K, const float* amax, uint8_t* codes,
                                      uint8_t* sf, float* scale_out, void* stream) {
  if (!x || !amax || !codes || !sf || !scale_out) return fail(NVFP4_EINVAL, "null pointer");
  if (check_rows_k("M", M, "K", K) != NVFP4_OK) return NVFP4_EINVAL;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sf))
    return fail(NVFP4_EALIGN, "x, codes and sf must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(amax) & 3u) != 0 || (reinterpret_cast<uintptr_t>(scale_out) & 3u) != 0)
    return fail(NVFP4_EALIGN, "amax and scale_out must be 4-byte aligned");
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  CUtensorMap tx;
  const int tile_rows = quantize_tile_rows(M, K, dev->num_sms);
  st = make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, K * 2, 64, static_cast<uint32_t>(tile_rows),
                 CU_TENSOR_MAP_SWIZZLE_128B, "x");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_quantize_from_amax(tx, tile_rows, M, K, amax, codes, sf, scale_out,
                                            static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return ok();
}

nvfp4_status nvfp4_quantize_dynamic(const void* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* sf,
                                    float* scale_out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !codes || !sf || !scale_out || !workspace) return fail(NVFP4_EINVAL, "null pointer");
  if (check_rows_k("M", M, "K", K) != NVFP4_OK) return NVFP4_EINVAL;
  if (workspace_bytes < kDynamicScratchBytes)
    return fail(NVFP4_EINVAL, "workspace_bytes=%zu is below NVFP4_DYNAMIC_WORKSPACE_BYTES=%zu", workspace_bytes,
                kDynamicScratchBytes);
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sf))
    return fail(NVFP4_EALIGN, "pointers must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(scale_out) & 3u) != 0 || (reinterpret_cast<uintptr_t>(workspace) & 3u) != 0)
    return fail(NVFP4_EALIGN, "scale_out and workspace must be 4-byte aligned");
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  CUtensorMap tx;
  const int tile_rows = quantize_tile_rows(M, K, dev->num_sms);
  st = make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, K * 2, 64, static_cast<uint32_t>(tile_rows),
                 CU_TENSOR_MAP_SWIZZLE_128B, "x");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_quantize_dynamic(tx, tile_rows, x, M, K, codes, sf, scale_out, static_cast<uint32_t*>(workspace),
                                          t_grid_wait, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "dynamic quantize launch");
  return ok();
}

nvfp4_status nvfp4_quantize_dynamic_noalloc(const void* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* sf,
                                            float* scale_out, void* stream) {
  if (!x || !codes || !sf || !scale_out) return fail(NVFP4_EINVAL, "null pointer");
  if (check_rows_k("M", M, "K", K) != NVFP4_OK) return NVFP4_EINVAL;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sf))
    return fail(NVFP4_EALIGN, "pointers must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(scale_out) & 3u) != 0) return fail(NVFP4_EALIGN, "scale_out must be 4-byte aligned");
  // scratch this call needs (the grid-wide maximum and the arrival counter)
  const size_t need = kDynamicScratchBytes;
  if (need > kNoAllocScratchBytes)
    return fail(NVFP4_EINVAL, "this call needs %zu bytes of scratch; the no-allocation scratch holds %zu", need,
                kNoAllocScratchBytes);
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  uint32_t* scratch = nullptr;
  st = noalloc_scratch(dev->device, &scratch);
  if (st != NVFP4_OK) return st;
  CUtensorMap tx;
  const int tile_rows = quantize_tile_rows(M, K, dev->num_sms);
  st = make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, K * 2, 64, static_cast<uint32_t>(tile_rows),
                 CU_TENSOR_MAP_SWIZZLE_128B, "x");
  if (st != NVFP4_OK) return st;
  // the launch zeroes the scratch on the stream before the kernel
  cudaError_t e = launch_quantize_dynamic(tx, tile_rows, x, M, K, codes, sf, scale_out, scratch, t_grid_wait,
                                          static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "dynamic quantize launch");
  return ok();
}

nvfp4_status nvfp4_swizzle_sf(const uint8_t* sf_linear, int64_t rows, int64_t k, uint8_t* sf_swizzled,
                              void* stream) {
  if (!sf_linear || !sf_swizzled) return fail(NVFP4_EINVAL, "null pointer");
  if (check_rows_k("rows", rows, "k", k) != NVFP4_OK) return NVFP4_EINVAL;
  if (!grid_fits((rows + 127) / 128 * (k / 64) * 32, 256))
    return fail(NVFP4_EINVAL, "rows*k=%lld is too large", (long long)(rows * k));
  if (!aligned16(sf_swizzled)) return fail(NVFP4_EALIGN, "sf_swizzled must be 16-byte aligned");
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_swizzle_sf(sf_linear, rows, k, sf_swizzled, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "swizzle launch");
  return ok();
}

nvfp4_status nvfp4_gemm(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb, int64_t M,
                        int64_t N, int64_t K, float alpha, const void* bias, void* y, void* stream) {
  if (!y) return fail(NVFP4_EINVAL, "null output pointer");
  if (!aligned16(y)) return fail(NVFP4_EALIGN, "y must be 16-byte aligned");
  GemmParams p;
  GemmTensorMaps maps;
  GemmConfig cg;
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = gemm_common(a, sfa, b, sfb, M, N, K, alpha, bias, &p, &maps, &cg, &dev, false, false, false, y);
  if (st != NVFP4_OK) return st;
  st = make_tmap(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B, "Y");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_gemm(maps, p, cg, false, false, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return ok();
}

nvfp4_status nvfp4_gemm_scaled(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb,
                               int64_t M, int64_t N, int64_t K, float g_a, float g_b, const void* bias, void* y,
                               void* stream) {
  if (!y) return fail(NVFP4_EINVAL, "null output pointer");
  if (!aligned16(y)) return fail(NVFP4_EALIGN, "y must be 16-byte aligned");
  if (!product_ok(g_a, g_b)) return fail(NVFP4_EINVAL, "g_a and g_b must be finite with a finite product");
  GemmParams p;
  GemmTensorMaps maps;
  GemmConfig cg;
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = gemm_common(a, sfa, b, sfb, M, N, K, g_b, bias, &p, &maps, &cg, &dev, false, false, false, y);
  if (st != NVFP4_OK) return st;
  p.alpha_mul = g_a;
  st = make_tmap(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B, "Y");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_gemm(maps, p, cg, false, false, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return ok();
}

nvfp4_status nvfp4_w4a16_gemm(const void* x, const uint8_t* w_codes, const uint8_t* w_sf, int64_t M, int64_t N,
                              int64_t K, float g_w, const void* bias, void* y, void* stream) {
  if (!x || !w_codes || !w_sf || !y) return fail(NVFP4_EINVAL, "null pointer");
  nvfp4_status st = check_rows_k("M", M, "K", K);
  if (st != NVFP4_OK) return st;
  if (N < 8 || N % 8 != 0 || N > kMaxDim)
    return fail(NVFP4_EINVAL, "N=%lld must be a positive multiple of 8, at most %lld", (long long)N,
                (long long)kMaxDim);
  if (!finite_f(g_w)) return fail(NVFP4_EINVAL, "g_w must be finite");
  if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_sf) || !aligned16(bias) || !aligned16(y))
    return fail(NVFP4_EALIGN, "pointers must be 16-byte aligned");
  const DeviceInfo* dev = nullptr;
  st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  const GemmPlan plan = gemm_plan(M, N, static_cast<int>(K / 64), dev->num_sms);
  const GemmConfig cg = plan.c;
  GemmParams p{};
  p.k_split = plan.k_split;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.ldy = static_cast<int32_t>(N);
  p.M = static_cast<int32_t>(M);
  p.N = static_cast<int32_t>(N);
  p.K = static_cast<int32_t>(K);
  p.tiles_m = static_cast<int32_t>((M + 128 * cg.cta_group - 1) / (128 * cg.cta_group));
  p.tiles_n = static_cast<int32_t>((N + cg.tile_n - 1) / cg.tile_n);
  const int64_t tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
  if (tiles > INT32_MAX) return fail(NVFP4_EINVAL, "problem too large");
  p.num_tiles = static_cast<int32_t>(tiles);
  p.num_kt = static_cast<int32_t>(K / 64);    // 64 bf16 elements = 128 bytes of every A row
  p.kblocks = static_cast<int32_t>(K / 16);   // K = 16 per MMA
  p.alpha = 1.0f;
  p.alpha_mul = 1.0f;
  p.w_scale = g_w;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.fault = dev->fault;
  GemmTensorMaps maps;
  st = make_tmap(&maps.a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B,
                 "x");
  if (st != NVFP4_OK) return st;
  st = make_tmap(&maps.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K / 2, N, K / 2, 32,
                 static_cast<uint32_t>(cg.tile_n / cg.cta_group), CU_TENSOR_MAP_SWIZZLE_NONE, "weight codes");
  if (st != NVFP4_OK) return st;
  maps.sfa = maps.b;  // unused (the activations carry no block scales); a valid descriptor
  const uint32_t sfb_blocks = static_cast<uint32_t>(cg.tile_n % 128 == 0 ? cg.tile_n / 128 : cg.tile_n / 128 + 1);
  st = make_sf_tmap(&maps.sfb, w_sf, N, K / 64, 1, sfb_blocks, "weight scales");
  if (st != NVFP4_OK) return st;
  st = make_tmap(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B, "Y");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_gemm_w4a16(maps, p, cg, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "w4a16 gemm launch");
  return ok();
}

nvfp4_status nvfp4_gemm_dynamic(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb,
                                int64_t M, int64_t N, int64_t K, float g_b, const float* g_a, const void* bias,
                                void* y, void* stream) {
  if (!y || !g_a) return fail(NVFP4_EINVAL, "null output or scale pointer");
  if (!aligned16(y)) return fail(NVFP4_EALIGN, "y must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(g_a) & 3u) != 0) return fail(NVFP4_EALIGN, "g_a must be 4-byte aligned");
  GemmParams p;
  GemmTensorMaps maps;
  GemmConfig cg;
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = gemm_common(a, sfa, b, sfb, M, N, K, g_b, bias, &p, &maps, &cg, &dev, false, false, false, y);
  if (st != NVFP4_OK) return st;
  p.alpha_scale = g_a;
  st = make_tmap(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B, "Y");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_gemm(maps, p, cg, false, false, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return ok();
}


nvfp4_status nvfp4_gemm_amax(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb,
                             int64_t M, int64_t N, int64_t K, float g_a, const float* g_a_device, float g_b,
                             const void* bias, void* y, float* amax_out, void* stream) {
  if (!y || !amax_out) return fail(NVFP4_EINVAL, "null output pointer");
  if (!aligned16(y)) return fail(NVFP4_EALIGN, "y must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(amax_out) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(g_a_device) & 3u) != 0)
    return fail(NVFP4_EALIGN, "amax_out and g_a_device must be 4-byte aligned");
  if (g_a_device == nullptr && !product_ok(g_a, g_b))
    return fail(NVFP4_EINVAL, "g_a and g_b must be finite with a finite product");
  GemmParams p;
  GemmTensorMaps maps;
  GemmConfig cg;
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = gemm_common(a, sfa, b, sfb, M, N, K, g_b, bias, &p, &maps, &cg, &dev, false, false, false, y);
  if (st != NVFP4_OK) return st;
  p.alpha_mul = g_a;
  p.alpha_scale = g_a_device;
  p.amax_out = reinterpret_cast<unsigned*>(amax_out);
  st = make_tmap(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B, "Y");
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_gemm(maps, p, cg, false, false, static_cast<cudaStream_t>(stream), *dev);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return ok();
}

nvfp4_status nvfp4_gemm_quant(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb,
                              int64_t M, int64_t N, int64_t K, float alpha, const void* bias,
                              const nvfp4_colrange* ranges, int32_t n_ranges, void* y_bf16, int64_t ldy,
                              float g_next, uint8_t* codes_next, uint8_t* sf_next, int64_t k_next, void* stream) {
  return gemm_quant_impl(a, sfa, b, sfb, M, N, K, alpha, 1.0f, bias, ranges, n_ranges, y_bf16, ldy, g_next,
                         codes_next, sf_next, k_next, stream);
}

nvfp4_status nvfp4_gemm_quant_scaled(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb,
                                     int64_t M, int64_t N, int64_t K, float g_a, float g_b, const void* bias,
                                     const nvfp4_colrange* ranges, int32_t n_ranges, void* y_bf16, int64_t ldy,
                                     float g_next, uint8_t* codes_next, uint8_t* sf_next, int64_t k_next,
                                     void* stream) {
  if (!product_ok(g_a, g_b)) return fail(NVFP4_EINVAL, "g_a and g_b must be finite with a finite product");
  return gemm_quant_impl(a, sfa, b, sfb, M, N, K, g_b, g_a, bias, ranges, n_ranges, y_bf16, ldy, g_next,
                         codes_next, sf_next, k_next, stream);
}

nvfp4_status nvfp4_testing_set_grid_wait(uint64_t limit_ns, uint32_t extra_arrivals) {
  if (limit_ns > kWaitLimitNs) return fail(NVFP4_EINVAL, "limit_ns=%llu exceeds the default %llu",
                                          (unsigned long long)limit_ns, (unsigned long long)kWaitLimitNs);
  if (extra_arrivals > 1024u) return fail(NVFP4_EINVAL, "extra_arrivals=%u exceeds 1024", extra_arrivals);
  t_grid_wait.limit_ns = limit_ns == 0 ? kWaitLimitNs : limit_ns;
  t_grid_wait.extra_arrivals = extra_arrivals;
  return ok();
}

nvfp4_status nvfp4_check_fault(void) {
  const DeviceInfo* dev = nullptr;
  nvfp4_status st = current_device(&dev);
  if (st != NVFP4_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  unsigned v = 0;
  e = cudaMemcpyFromSymbol(&v, g_fault_word, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "read fault word");
  if (v != 0u) {
    const unsigned zero = 0u;
    e = cudaMemcpyToSymbol(g_fault_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clear fault word");
    return fail(NVFP4_ETIMEOUT, "a kernel gave up waiting on a barrier (fault bits 0x%x)", v);
  }
  return ok();
}

nvfp4_status nvfp4_gemm_tile_shape(int64_t M, int64_t N, int32_t num_sms, int32_t* out) {
  if (!out) return fail(NVFP4_EINVAL, "null output pointer");
  if (M < 1 || M > kMaxDim || N < 8 || N > kMaxDim || num_sms < 2)
    return fail(NVFP4_EINVAL, "M=%lld, N=%lld, num_sms=%d out of range", (long long)M, (long long)N, num_sms);
  const GemmConfig c = gemm_config(M, N, num_sms);
  out[0] = c.cta_group;
  out[1] = c.tile_n;
  out[2] = c.acc_bufs;
  return ok();
}

nvfp4_status nvfp4_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t num_sms, int32_t w4a16, int32_t* out) {
  if (!out) return fail(NVFP4_EINVAL, "null output pointer");
  if (M < 1 || M > kMaxDim || N < 8 || N > kMaxDim || K < 64 || K % 64 != 0 || K > kMaxDim || num_sms < 2)
    return fail(NVFP4_EINVAL, "M=%lld, N=%lld, K=%lld, num_sms=%d out of range", (long long)M, (long long)N,
                (long long)K, num_sms);
  const int num_kt = static_cast<int>(w4a16 ? K / 64 : (K / 2 + 127) / 128);
  const GemmPlan plan = gemm_plan(M, N, num_kt, num_sms);
  out[0] = plan.c.cta_group;
  out[1] = plan.c.tile_n;
  out[2] = plan.c.acc_bufs;
  out[3] = plan.k_split;
  return ok();
}

int32_t nvfp4_quantize_tile_rows(int64_t M, int64_t K, int32_t num_sms) {
  if (M < 1 || M > kMaxDim || K < 64 || K % 64 != 0 || K > kMaxDim || num_sms < 1) return 0;
  return quantize_tile_rows(M, K, num_sms);
}

const char* nvfp4_last_error(void) { return t_last_error.c_str(); }

}  // extern "C"
