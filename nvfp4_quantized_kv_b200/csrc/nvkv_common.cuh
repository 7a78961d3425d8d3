// nvkv_common.cuh -- shared device helpers of the NVFP4 paged-KV kernels.
//
// Storage format: "gzenz/ninfer" README, "Fork changes vs upstream" ->
// "Context and model", NVFP4 KV cache bullet (4-bit E2M1 codes, one E4M3
// scale per 16 elements).  The page layout is documented in include/nvkv.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvkv.h"

namespace nvkv {

constexpr int kPageTokens = 16;   // token slots per page
constexpr int kGroup = 16;        // elements per E4M3 scale
constexpr int kUnitTokens = 128;  // split-plan unit (8 pages)

// Byte offsets inside one kv-head block of a page (18*D bytes).
__host__ __device__ constexpr int kc_off(int) { return 0; }
__host__ __device__ constexpr int ks_off(int D) { return 8 * D; }
__host__ __device__ constexpr int vc_off(int D) { return 9 * D; }
__host__ __device__ constexpr int vs_off(int D) { return 17 * D; }
__host__ __device__ constexpr int head_bytes(int D) { return 18 * D; }

// Byte offsets inside one kv-head block of a K8V4 page (25*D + 64 bytes):
// K codes [16 slots][D] (one E4M3 byte per element), K scales [16 slots]
// (float), then V exactly as in an NVFP4 block: codes [D][8], scales
// [D/16][16].  Every region starts on a 16-byte boundary (D is 128 or 256).
__host__ __device__ constexpr int k8_ks_off(int D) { return 16 * D; }
__host__ __device__ constexpr int k8_vc_off(int D) { return 16 * D + 64; }
__host__ __device__ constexpr int k8_vs_off(int D) { return 24 * D + 64; }
__host__ __device__ constexpr int k8_head_bytes(int D) { return 25 * D + 64; }

// The two cache formats as compile-time layouts (the CUDA-core attention
// kernels are written once for both).
struct Nvfp4Layout {
  static constexpr bool kK8 = false;
  __device__ static int head(int D) { return head_bytes(D); }
  __device__ static int vc(int D) { return vc_off(D); }
  __device__ static int vs(int D) { return vs_off(D); }
};
struct K8v4Layout {
  static constexpr bool kK8 = true;
  __device__ static int head(int D) { return k8_head_bytes(D); }
  __device__ static int vc(int D) { return k8_vc_off(D); }
  __device__ static int vs(int D) { return k8_vs_off(D); }
};

// ---------------------------------------------------------------------------
// Split plan (see nvkv_decode_workspace_bytes in nvkv.h).  Units of 128
// tokens of every (b, h) pair, in (b, h, unit) order, are dealt to S ranges:
// range c owns units [c*U/S, (c+1)*U/S).
// ---------------------------------------------------------------------------
__host__ __device__ inline int64_t range_begin(int64_t c, int64_t U, int64_t S) {
  return (c * U) / S;
}
// The range holding unit u (0 <= u < U): the largest c with range_begin(c) <= u.
__host__ __device__ inline int64_t range_of_unit(int64_t u, int64_t U, int64_t S) {
  return ((u + 1) * S - 1) / U;
}
__host__ __device__ inline int units_of_len(int kv_len) {
  return kv_len > 0 ? (kv_len + kUnitTokens - 1) / kUnitTokens : 0;
}

// Finds the (b, h) pair holding global unit u of the split plan: its first
// unit pair_start and its unit count (0 when u is past the last unit).
__device__ inline void locate_pair(const int32_t *kv_lens, int B, int Hkv, int64_t u, int &b,
                                   int &h, int64_t &pair_start, int &units) {
  int64_t acc = 0;
  for (b = 0; b < B; ++b) {
    const int ub = units_of_len(kv_lens[b]);
    const int64_t span = (int64_t)ub * Hkv;
    if (u < acc + span) {
      h = (int)((u - acc) / ub);
      pair_start = acc + (int64_t)h * ub;
      units = ub;
      return;
    }
    acc += span;
  }
  h = 0;
  pair_start = acc;
  units = 0;
}

// ---------------------------------------------------------------------------
// Error reporting: never trap, OR a bit into the caller's word.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void report(int32_t *err, unsigned bit) {
  if (err) atomicOr(reinterpret_cast<unsigned *>(err), bit);
}

// ---------------------------------------------------------------------------
// Number formats.
// ---------------------------------------------------------------------------
// E4M3 byte -> fp32 (exact), through the hardware fp8 -> f16 conversion.
__device__ __forceinline__ float e4m3_to_float(uint8_t b) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
  return __half2float(__half(h));
}

// Scale byte for a group with max |x| = amax: E4M3 round-to-nearest-even of
// amax/6, saturating to 448.  amax/6 is the IEEE-rounded fp32 quotient; it
// can only equal an E4M3 rounding midpoint when the exact quotient does
// (the dividend has 8 significant bits, a midpoint times 6 at most 7), so
// the decision is that of exact arithmetic.
__device__ __forceinline__ uint8_t scale_byte_of_amax(float amax) {
  float t = __fdiv_rn(amax, 6.0f);
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3));
}

// E2M1 code of x under scale s (> 0): the magnitude index is the number of
// rounding midpoints m*s that |x| passes, with ties going to the even index
// (strict comparison where the lower neighbour is even, >= where the upper
// one is).  Every m*s is exact in fp32 (s has 4 significant bits, m at most
// 3), so the comparisons are exact.  A zero magnitude gives code 0.
__device__ __forceinline__ uint32_t e2m1_code(float x, float s) {
  float a = fabsf(x);
  uint32_t idx = (a > 0.25f * s) + (a >= 0.75f * s) + (a > 1.25f * s) + (a >= 1.75f * s) +
                 (a > 2.5f * s) + (a >= 3.5f * s) + (a > 5.0f * s);
  uint32_t sign = (__float_as_uint(x) >> 31) & 1u;
  return idx ? (idx | (sign << 3)) : 0u;
}

// Two E2M1 codes (low nibble = first element) -> f16x2, exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t out;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(out)
      : "r"(byte));
  return out;
}

// Two E4M3 bytes (low byte = first element) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t out;
  uint16_t in = static_cast<uint16_t>(two_bytes);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(in));
  return out;
}

// Two floats -> two E4M3 bytes (a in the low byte), rounded to nearest with
// ties to even and saturated at 448 by the hardware conversion.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float a, float b) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(a), "f"(b));
  return out;
}

// Two floats -> one byte of E2M1 codes (a in the low nibble), rounded to
// nearest with ties to even and saturated at 6 by the hardware conversion.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float a, float b) {
  uint32_t out;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(out)
      : "f"(a), "f"(b));
  return out;
}

// Four E2M1 code pairs (one 32-bit word, byte k = elements 2k, 2k+1) ->
// four f16x2.  The bytes are split by register unpacking, not converted.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t (&o)[4]) {
  asm("{\n\t.reg .b8 a, b, c, d;\n\tmov.b32 {a, b, c, d}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, a;\n\tcvt.rn.f16x2.e2m1x2 %1, b;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, c;\n\tcvt.rn.f16x2.e2m1x2 %3, d;\n\t}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
}

// Two E4M3 byte pairs (one 32-bit word, half k = bytes 2k, 2k+1) -> two f16x2.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t (&o)[2]) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(o[0]), "=r"(o[1])
      : "r"(w));
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
  return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t v) {
  return __half22float2(*reinterpret_cast<__half2 *>(&v));
}

// Packed fp32 pair arithmetic (one instruction for both lanes of the pair).
__device__ __forceinline__ float2 add_f32x2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
// (2^a, 2^b) as an f16 pair (a in the low half) with one exponential
// instruction for both: the arguments are rounded to f16 first, so this is
// for softmax weights that end up in f16 anyway.  2^-inf = +0.
__device__ __forceinline__ uint32_t ex2_f16x2(float a, float b) {
  uint32_t h, r;
  asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(h) : "f"(a), "f"(b));
  asm("ex2.approx.f16x2 %0, %1;" : "=r"(r) : "r"(h));
  return r;
}

// (2^a, 2^b) as an f16 pair (a in the low half): each exponential in fp32
// (ex2.approx, relative error about 2^-22), then one rounding to f16.
// 2^-inf = +0.
__device__ __forceinline__ uint32_t ex2_f32_to_f16x2(float a, float b) {
  float ea, eb;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(ea) : "f"(a));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(eb) : "f"(b));
  uint32_t h;
  asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(h) : "f"(ea), "f"(eb));
  return h;
}

// (q, q) as an f16 pair with q = 2^a / 4: the exponential in fp32
// (ex2.approx, relative error about 2^-22), one rounding to f16.  2^-inf = +0.
__device__ __forceinline__ uint32_t ex2_quarter_f16x2(float a) {
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(a));
  e *= 0.25f;
  uint32_t h;
  asm("cvt.rn.f16x2.f32 %0, %1, %1;" : "=r"(h) : "f"(e));
  return h;
}

// Warp reductions.
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace nvkv
