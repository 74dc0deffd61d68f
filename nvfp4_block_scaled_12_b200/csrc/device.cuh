// Device-side building blocks for the sm_100a kernels: NVFP4 element/scale
// conversions, mbarriers with bounded waits, TMA / bulk copies, and the
// tcgen05 (5th-generation tensor core) instructions, all as inline PTX.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

// ---------------------------------------------------------------------------
// Fault word codes (OR-ed into the library's device fault word)
// ---------------------------------------------------------------------------
enum : unsigned {
  kFaultProducerWait = 1u << 0,
  kFaultMmaWait = 1u << 1,
  kFaultEpilogueWait = 1u << 2,
  kFaultDrainWait = 1u << 3,
  kFaultGridWait = 1u << 4,  // a grid-wide barrier did not complete
};

// Longest a kernel waits on one barrier before giving up (nanoseconds).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// ---------------------------------------------------------------------------
// NVFP4 element and scale conversions (every step one IEEE fp32 op, RNE)
// ---------------------------------------------------------------------------

// E4M3 encode of a non-negative value, round to nearest even, saturating at
// 448 (never NaN for finite or +inf input).  Returns the byte.
__device__ __forceinline__ uint32_t e4m3_from_f32_satfinite(float t) {
  uint16_t pair;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(0.0f), "f"(t));
  return pair & 0xFFu;
}

// Exact value of a non-negative E4M3 byte below 0x7F.
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  if (e == 0) return static_cast<float>(m) * 0x1p-9f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Eight values to a 32-bit word of E2M1 codes (v0 -> bits 0-3, v1 -> bits
// 4-7, ...), round to nearest even, saturating at +-6.  cvt's first source
// lands in the high nibble of its byte, so each pair is passed (odd, even).
__device__ __forceinline__ uint32_t e2m1x8_from_f32(float v0, float v1, float v2, float v3, float v4,
                                                    float v5, float v6, float v7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return out;
}

// E4M3_satfinite(fl(amax / d6)) without the IEEE division's range check and
// slow-path branch, given rd6 = RN(1/d6) and amax >= 0: q1 = fl(amax rd6) is
// within 1.5 ulp of the quotient; at 1024 or more the quotient is far above
// E4M3's largest value 448 and the code saturates; otherwise two FMA residual
// corrections make it the correctly rounded quotient (Markstein, IBM J. Res.
// Dev. 34(1), 1990: with rd6 the correctly rounded reciprocal and a faithful
// q, RN(q + rd6 (amax - d6 q)) = RN(amax / d6)).  For d6 = fl(6 g), g in
// [2^-64, 2^64], every residual of a quotient >= 2^-12 is exact; below that
// the code is zero either way.
__device__ __forceinline__ uint32_t block_scale_e4m3(float amax, float d6, float rd6) {
  const float q1 = __fmul_rn(amax, rd6);
  if (q1 >= 1024.0f) return 0x7Eu;  // 448
  const float q2 = __fmaf_rn(__fmaf_rn(-q1, d6, amax), rd6, q1);
  const float q3 = __fmaf_rn(__fmaf_rn(-q2, d6, amax), rd6, q2);
  return e4m3_from_f32_satfinite(q3);
}

// Quantize 16 fp32 values (exactly representable in bf16) that form one
// NVFP4 block, given the per-tensor scale g, d6 = fl(6*g) and rd6 = RN(1/d6):
//     s = E4M3_satfinite(fl(amax / d6))   (block_scale_e4m3)
//     code_i = E2M1_satfinite(fl(v_i * RN(1 / fl(e4m3(s) * g))))   (0 when s == 0)
// Writes the 8 code bytes as two 32-bit words (element 0 in the low nibble
// of byte 0 of lo_word) and returns the E4M3 scale byte.
__device__ __forceinline__ uint32_t quantize_block16_rd(const float (&v)[16], float g, float d6, float rd6,
                                                        uint32_t& lo_word, uint32_t& hi_word) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t s = block_scale_e4m3(amax, d6, rd6);
  lo_word = 0u;
  hi_word = 0u;
  if (s != 0u) {
    const float r = __frcp_rn(__fmul_rn(e4m3_to_f32(s), g));
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = __fmul_rn(v[i], r);
    lo_word = e2m1x8_from_f32(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
    hi_word = e2m1x8_from_f32(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]);
  }
  return s;
}

// quantize_block16_rd for the standalone quantizer, with the block's
// reciprocal from a table filled once per launch, rtab[s] = RN(1 / fl(e4m3(s)
// g)) for the codes s = 1 .. 126: the same fp32 operations, taken out of the
// per-block path.
__device__ __forceinline__ uint32_t quantize_block16_tab(const float (&v)[16], float d6, float rd6,
                                                         const float* rtab, uint32_t& lo_word, uint32_t& hi_word) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t s = block_scale_e4m3(amax, d6, rd6);
  lo_word = 0u;
  hi_word = 0u;
  if (s != 0u) {
    const float r = rtab[s];
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = __fmul_rn(v[i], r);
    lo_word = e2m1x8_from_f32(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
    hi_word = e2m1x8_from_f32(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]);
  }
  return s;
}

// The per-tensor scale a measured amax gives (the dynamic quantizer's rule):
// g = fl(amax / 2688) clamped into [2^-64, 2^64], 0 for amax == 0.
__device__ __forceinline__ float scale_from_amax(float amax) {
  return amax > 0.0f ? fminf(fmaxf(__fdiv_rn(amax, 2688.0f), 0x1p-64f), 0x1p64f) : 0.0f;
}

// Largest magnitude of the 2 x 16 bf16 values in a word, folded into acc (two
// 16-bit lanes): |v| as its bit pattern orders like the value; a NaN counts
// as infinity.
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t acc, uint32_t w) {
  return __vmaxu2(acc, __vminu2(w & 0x7FFF7FFFu, 0x7F807F80u));
}

// MXFP8 block (OCP microscaling): 32 fp32 values (exactly representable in
// bf16) -> 32 E4M3 bytes in 8 little-endian words and the E8M0 scale byte.
//   amax == 0: scale byte 0 (2^-127);  else s = clamp(floor(log2 amax) - 8,
//   -127, 127), scale byte s + 127;  code_i = E4M3_satfinite(fl(v_i * 2^-s)).
__device__ __forceinline__ uint32_t quantize_mx_block32(const float (&v)[32], uint32_t (&w)[8]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t bits = __float_as_uint(amax);
  int e;  // floor(log2(amax)) for amax > 0
  if (bits >= 0x00800000u)
    e = static_cast<int>(bits >> 23) - 127;
  else
    e = (31 - __clz(static_cast<int>(bits))) - 149;  // fp32 subnormal: bits * 2^-149
  int s = bits == 0u ? -127 : e - 8;
  s = s < -127 ? -127 : (s > 127 ? 127 : s);
  // 2^-s exactly: a normal float for s <= 126, the subnormal 2^-127 for s = 127
  const float inv = s <= 126 ? __uint_as_float(static_cast<uint32_t>(127 - s) << 23) : __uint_as_float(0x00400000u);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint16_t lo, hi;
    // cvt puts its first source in the high byte: pass (odd, even)
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(__fmul_rn(v[4 * i + 1], inv)),
        "f"(__fmul_rn(v[4 * i + 0], inv)));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(__fmul_rn(v[4 * i + 3], inv)),
        "f"(__fmul_rn(v[4 * i + 2], inv)));
    w[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  }
  return static_cast<uint32_t>(s + 127);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low 16 bits)
  return *reinterpret_cast<uint32_t*>(&h);
}

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

// Two E4M3 bytes (bits 0-7 and 8-15 of b) to an f16 pair, exactly (E4M3's
// whole range, subnormals included, is representable in f16); the low byte
// lands in the low half.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t b) {
  uint32_t h;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h) : "r"(b));
  return h;
}

// Eight NVFP4 weight elements (a 32-bit word of E2M1 codes, element 2j in the
// low nibble of byte j) of one 16-element block with E4M3 scale s, to eight
// bf16 values (four words, element 2j in the low half of word j):
//     w = bf16_rn( fl32( fl32(e2m1 * s) * g ) )
// s2 holds s in both halves of an f16 pair.  e2m1 * s has at most six
// significant bits and lies in [2^-10, 2688], so the f16 product is exact
// (as it is in fp32); the multiply by g is one fp32 rounding per element,
// done two at a time (mul.rn.f32x2), then one bf16 rounding.
__device__ __forceinline__ void nvfp4x8_to_bf16(uint32_t codes, uint32_t s2, float g, uint32_t (&o)[4]) {
  uint32_t h[4];
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(codes));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t t;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(t) : "r"(h[i]), "r"(s2));  // exact
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&t));
    float lo, hi;
    asm("{\n\t.reg .b64 a, gg;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 gg, {%4, %4};\n\t"
        "mul.rn.f32x2 a, a, gg;\n\t"
        "mov.b64 {%0, %1}, a;\n\t}"
        : "=f"(lo), "=f"(hi) : "f"(f.x), "f"(f.y), "f"(g));
    o[i] = pack_bf16x2(lo, hi);
  }
}

// Byte offset of logical scale (row r, scale column c) in the swizzled
// scale-factor buffer with `katoms` 4-column atoms per 128-row block.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t c, int64_t katoms) {
  return ((r >> 7) * katoms + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
}

// ---------------------------------------------------------------------------
// Global memory access
// ---------------------------------------------------------------------------
// One 32-byte store (a whole L2 sector) of 8 words; p must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Named barrier over `threads` threads of the CTA (a multiple of 32; every
// warp that takes part arrives with all its threads).
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// A 32-bit load with acquire semantics at GPU scope (reads what other CTAs
// released with fences or atomics).
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// Shared memory, mbarriers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0u;
}

// Same as mbar_try_wait, with acquire semantics at cluster scope: for
// barriers that threads of the peer CTA arrive on.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0u;
}

// Wait until the phase with the given parity has completed.  Gives up (and
// returns false) after kWaitLimitNs, or early once *abort is non-zero
// (abort may be null: then only the time limit applies).
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  auto poll = [&]() { return kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (poll()) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (poll()) return true;
    if ((i & 63u) == 0u) {
      if (abort != nullptr && *abort) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
  }
}

// ---------------------------------------------------------------------------
// Clusters (CTA pairs)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared-memory address of the same object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_smem(uint32_t local, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(local), "r"(rank));
  return out;
}

// Arrive on an mbarrier given by its shared::cluster address (possibly in
// the peer CTA).  Default (CTA-scope release) semantics: the data these
// arrivals publish lives in TMEM and is ordered by tcgen05.wait / fences,
// and a cluster-scope release costs hundreds of nanoseconds per arrive.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// 16 bytes (four floats) from shared memory at a shared::cluster address
// (possibly in another CTA of the cluster: distributed shared memory).
__device__ __forceinline__ float4 ld_shared_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
  return v;
}

// All threads of every CTA of the cluster.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA and bulk copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// 2-D tile load by one CTA of a pair whose completion is signalled on the
// mbarrier at `bar_cluster_addr` (the pair leader's barrier).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster_addr,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster_addr), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int32_t x, int32_t y,
                                            int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation MMA
// ---------------------------------------------------------------------------

// Allocate `ncols` TMEM columns (power of two >= 32); whole warp.  The base
// address is written to *dst in shared memory.
// kCG = 2: both CTAs of a pair execute it; the pair gets the same columns.
template <int kCG = 1>
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  if (kCG == 1)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols) : "memory");
  else
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols) : "memory");
}
template <int kCG = 1>
__device__ __forceinline__ void tmem_relinquish() {
  if (kCG == 1)
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  else
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
template <int kCG = 1>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  if (kCG == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive (once) on `bar` when every tcgen05 operation this thread issued
// before has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Pair-MMA form of tc_commit (arrive on this CTA's barrier): every tcgen05
// instruction of a kernel uses the same cta_group.
__device__ __forceinline__ void tc_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Pair MMA: arrive once on the barrier at the same shared-memory offset in
// every CTA of `cta_mask` when all prior tcgen05 ops of this thread are done.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// D (TMEM, fp32) (+)= A * B with NVFP4 operands: E2M1 elements from shared
// memory and one UE4M3 scale per 16 elements from TMEM.  M=128, K=64.
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Pair MMA (M = 256 across the two CTAs, each holding 128 rows of A, half of
// B and its own accumulator rows); issued by the pair leader.
__device__ __forceinline__ void tc_mma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Shared-memory matrix descriptor, K-major operand rows of 128 bytes with the
// 128-byte swizzle; groups of 8 rows are 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;          // leading byte offset (16 B; unused when swizzled)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;  // stride byte offset: 8 rows x 128 B
  d |= static_cast<uint64_t>(1) << 46;          // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;          // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor of the block-scaled MMA: E2M1 x E2M1 -> fp32,
// both operands K-major, UE4M3 scales, dense K = 64.
__host__ __device__ constexpr uint32_t idesc_nvf4(int m, int n) {
  return (1u << 7)                                  // A format: E2M1
         | (1u << 10)                               // B format: E2M1
         | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24);   // M / 16 (scale format bit 23 = 0: UE4M3)
}

// Instruction descriptor of the MXFP8 block-scaled MMA: E4M3 x E4M3 -> fp32,
// both operands K-major, UE8M0 scales, dense K = 32.  One 32-bit TMEM scale
// word holds the scales of four consecutive 32-element blocks; sf_id picks the
// byte this MMA uses, for A (bits 29-30) and B (bits 4-5).
__host__ __device__ constexpr uint32_t idesc_mxf8(int m, int n, uint32_t sf_id) {
  return (sf_id << 4)                               // B scale byte
         | (0u << 7)                                // A format: E4M3
         | (0u << 10)                               // B format: E4M3
         | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
         | (1u << 23)                               // scale format: UE8M0
         | (static_cast<uint32_t>(m >> 4) << 24)    // M / 16
         | (sf_id << 29);                           // A scale byte
}

// MXFP8 MMA (kind::mxf8f6f4, one E8M0 scale per 32 elements); the scale
// addresses carry the scale byte in their top two bits, as the descriptor does.
__device__ __forceinline__ void tc_mma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
__device__ __forceinline__ void tc_mma_mxf8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor of the plain FP8 MMA (kind::f8f6f4, no block
// scales): E4M3 x E4M3 -> fp32, both operands K-major, dense K = 32.
__host__ __device__ constexpr uint32_t idesc_f8(int m, int n) {
  return (1u << 4)                                  // D format: F32
         | (0u << 7)                                // A format: E4M3
         | (0u << 10)                               // B format: E4M3
         | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_mma_f8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of the bf16 MMA (kind::f16): BF16 x BF16 -> fp32,
// both operands K-major, dense K = 16.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
  return (1u << 4)                                  // D format: F32
         | (1u << 7)                                // A format: BF16
         | (1u << 10)                               // B format: BF16
         | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Registers -> TMEM: 32 lanes (this warp's quarter) x 4 / 8 consecutive
// 32-bit columns; thread i of the warp writes lane base+i.
__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, uint4 v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, uint4 a, uint4 b) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}
// 8 / 16 consecutive columns from a register array (column address aligned to
// the column count)
__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit TMEM columns -> 32 registers per thread
// (thread i of the warp gets lane base+i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// 32 lanes x 64 consecutive 32-bit TMEM columns -> r[0..63] (thread i of the
// warp gets lane base+i).
__device__ __forceinline__ void tmem_ld_32x32b_x64(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x64.b32 "
               "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                 "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
                 "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                 "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
                 "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
                 "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
                 "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
                 "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
               : "r"(taddr));
}

// Wait for this thread's outstanding tcgen05.ld, then pin the loaded
// registers behind the wait so no use of them is scheduled earlier.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}

// Same for a register array filled by several tcgen05.ld.
template <int N>
__device__ __forceinline__ void tmem_ld_wait_n(uint32_t (&r)[N]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

}  // namespace nvfp4
