// append.cu -- quantise new bf16 K/V rows into the NVFP4 paged pool.
//
// "gzenz/ninfer" README, "Fork changes vs upstream" -> "Context and model":
// NVFP4 KV cache, 4-bit E2M1 codes plus one E4M3 scale per group of 16.
// Each group of 16 head_dim elements of one token and one kv-head gets
// scale = E4M3_RN(amax / 6) and codes = E2M1_RN(x / scale) (see
// nvkv_common.cuh for the exact decision rules).
//
// With rotary_dim > 0 (nvkv_append_rope), K is rotated at its position
// before it is quantised -- the YaRN context extension of the same README,
// stated there as linear RoPE scaling; the (cos, sin) table comes from
// nvkv_rope_table.  Element i < rotary_dim/2 pairs with i + rotary_dim/2;
// in float, x' = fma(x, c, -(y*s)) and y' = fma(y, c, x*s).  Positions
// without a table row are reported (NVKV_DEVERR_LENGTH) and not written.
//
// Work item = (sequence b, slot pair, kv-head h, group g).  V codes are
// stored transposed (byte (d, i) holds slots 2i and 2i+1), so the two slots
// of a pair share bytes; giving the whole pair to one thread makes every
// byte single-writer within a launch.  A slot of the pair that is not new
// in this call keeps its nibble (read-modify-write of the shared byte).
#include "nvkv_common.cuh"

namespace nvkv {

struct GroupQ {
  uint32_t codes_lo;  // elements 0..7, 4 bits each (element 0 in bits 0..3)
  uint32_t codes_hi;  // elements 8..15
  uint8_t scale;
};

// Quantise 16 bf16 values (two 16-byte loads).
__device__ __forceinline__ GroupQ quantize16(const __nv_bfloat16 *src) {
  uint4 raw0 = __ldg(reinterpret_cast<const uint4 *>(src));
  uint4 raw1 = __ldg(reinterpret_cast<const uint4 *>(src) + 1);
  uint32_t w[8] = {raw0.x, raw0.y, raw0.z, raw0.w, raw1.x, raw1.y, raw1.z, raw1.w};
  float x[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  GroupQ q;
  q.scale = scale_byte_of_amax(amax);
  q.codes_lo = q.codes_hi = 0;
  if (q.scale != 0) {
    float s = e4m3_to_float(q.scale);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      q.codes_lo |= e2m1_code(x[i], s) << (4 * i);
      q.codes_hi |= e2m1_code(x[8 + i], s) << (4 * i);
    }
  }
  return q;
}

// Quantise 16 float values (the rotated K): same decisions as quantize16.
__device__ __forceinline__ GroupQ quantize16_f32(const float (&x)[16]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  GroupQ q;
  q.scale = scale_byte_of_amax(amax);
  q.codes_lo = q.codes_hi = 0;
  if (q.scale != 0) {
    float s = e4m3_to_float(q.scale);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      q.codes_lo |= e2m1_code(x[i], s) << (4 * i);
      q.codes_hi |= e2m1_code(x[8 + i], s) << (4 * i);
    }
  }
  return q;
}

__device__ __forceinline__ void load16_f32(const __nv_bfloat16 *src, float (&x)[16]) {
  const uint4 raw0 = __ldg(reinterpret_cast<const uint4 *>(src));
  const uint4 raw1 = __ldg(reinterpret_cast<const uint4 *>(src) + 1);
  const uint32_t w[8] = {raw0.x, raw0.y, raw0.z, raw0.w, raw1.x, raw1.y, raw1.z, raw1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Group g (16 elements from 16*g) of a K row rotated by the table row of its
// position: its partner elements are the whole group g +- rotary_dim/32.
__device__ __forceinline__ GroupQ rope_quantize16(const __nv_bfloat16 *row, int g, int rotary_dim,
                                                  const float *cs_pos) {
  const int h = rotary_dim / 2;
  const bool first = 16 * g < h;  // this group holds the x of its pairs
  float own[16], other[16], rot[16];
  load16_f32(row + 16 * g, own);
  load16_f32(row + 16 * g + (first ? h : -h), other);
  const int i0 = first ? 16 * g : 16 * g - h;  // pair index of element 0 of the group
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float2 cs = *reinterpret_cast<const float2 *>(cs_pos + 2 * (i0 + e));
    const float ps = other[e] * cs.y;
    rot[e] = first ? fmaf(own[e], cs.x, -ps) : fmaf(own[e], cs.x, ps);
  }
  return quantize16_f32(rot);
}

__global__ void __launch_bounds__(256)
append_kernel(uint8_t *__restrict__ pool, int num_pages, int Hkv, int D,
              const int32_t *__restrict__ page_table, int max_pages,
              const int32_t *__restrict__ kv_lens, int max_kv_len,
              const __nv_bfloat16 *__restrict__ k_new, const __nv_bfloat16 *__restrict__ v_new,
              const int32_t *__restrict__ cu_new, int total_new, int max_new, int max_pairs,
              const float *__restrict__ rope_cs, int rotary_dim, int max_pos, int32_t *err) {
  const int b = blockIdx.y;
  const int groups = D / kGroup;
  const int per_pair = Hkv * groups;
  const int item = blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= max_pairs * per_pair) return;
  const int pair = item / per_pair;
  const int h = (item % per_pair) / groups;
  const int g = item % groups;

  const int row0 = cu_new[b];
  const int n = cu_new[b + 1] - row0;
  const int len = kv_lens[b];
  if (n <= 0) return;
  const int first = len - n;  // position of the first new row
  if (row0 < 0 || row0 + n > total_new || n > max_new || first < 0 || len > max_kv_len ||
      len > max_pages * kPageTokens) {
    if (pair == 0 && h == 0 && g == 0) report(err, NVKV_DEVERR_LENGTH);
    return;
  }
  const int p0 = (first >> 1) + pair;  // pair index: positions 2*p0, 2*p0+1
  const int pos_even = 2 * p0;
  if (pos_even >= len) return;
  const int page = page_table[(size_t)b * max_pages + pos_even / kPageTokens];
  if (page < 0 || page >= num_pages) {
    report(err, NVKV_DEVERR_PAGE_ID);
    return;
  }
  const int slot_even = pos_even % kPageTokens;
  uint8_t *blk = pool + (size_t)page * Hkv * head_bytes(D) + (size_t)h * head_bytes(D);

  GroupQ vq[2];
  bool is_new[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int pos = pos_even + k;
    is_new[k] = pos >= first && pos < len;
    if (is_new[k] && rotary_dim > 0 && pos >= max_pos) {  // no table row for this position
      if (h == 0 && g == 0) report(err, NVKV_DEVERR_LENGTH);
      is_new[k] = false;
    }
    if (!is_new[k]) continue;
    const size_t row = (size_t)(row0 + pos - first);
    const size_t src = (row * Hkv + h) * D + g * kGroup;
    const int slot = slot_even + k;
    // K: codes of the row are contiguous, element 2i in the low nibble.
    GroupQ kq = (rotary_dim > 0 && 16 * g < rotary_dim)
                    ? rope_quantize16(k_new + src - g * kGroup, g, rotary_dim,
                                      rope_cs + (size_t)pos * rotary_dim)
                    : quantize16(k_new + src);
    uint2 packed;
    packed.x = kq.codes_lo;
    packed.y = kq.codes_hi;
    *reinterpret_cast<uint2 *>(blk + kc_off(D) + slot * (D / 2) + g * 8) = packed;
    blk[ks_off(D) + slot * (D / 16) + g] = kq.scale;
    // V: codes go to the transposed region below; scales are [g][slot].
    vq[k] = quantize16(v_new + src);
    blk[vs_off(D) + g * kPageTokens + slot] = vq[k].scale;
  }
  // V code bytes (d, slot_even/2) for the 16 elements of group g.
  uint8_t *vc = blk + vc_off(D) + (size_t)(g * kGroup) * 8 + slot_even / 2;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    uint8_t *p = vc + i * 8;
    uint32_t lo, hi;
    if (is_new[0]) {
      lo = ((i < 8 ? vq[0].codes_lo : vq[0].codes_hi) >> (4 * (i & 7))) & 15u;
    } else {
      lo = *p & 15u;
    }
    if (is_new[1]) {
      hi = ((i < 8 ? vq[1].codes_lo : vq[1].codes_hi) >> (4 * (i & 7))) & 15u;
    } else {
      hi = *p >> 4;
    }
    *p = static_cast<uint8_t>(lo | (hi << 4));
  }
}

cudaError_t launch_append(const nvkv_cache &c, const nvkv_seqs &s, const void *k_new,
                          const void *v_new, const int32_t *cu_new, int total_new, int max_new,
                          const float *rope_cs, int rotary_dim, int max_pos, cudaStream_t stream) {
  const int max_pairs = max_new / 2 + 1;
  const int per_pair = c.num_kv_heads * (c.head_dim / kGroup);
  const long items = (long)max_pairs * per_pair;
  const int threads = 256;
  dim3 grid((unsigned)((items + threads - 1) / threads), (unsigned)s.batch);
  append_kernel<<<grid, threads, 0, stream>>>(
      c.pool, c.num_pages, c.num_kv_heads, c.head_dim, s.page_table, s.max_pages_per_seq,
      s.kv_lens, s.max_kv_len, static_cast<const __nv_bfloat16 *>(k_new),
      static_cast<const __nv_bfloat16 *>(v_new), cu_new, total_new, max_new, max_pairs, rope_cs,
      rotary_dim, max_pos, s.err_word);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K8V4 cache (the "knoopx/ninfer" README, "Capabilities and limits", lists
// K8V4 among its KV storage formats; the same README's note on its published
// measurements names an E4M3 "row-256" KV).  K: one float scale per row of
// one token and one kv-head, scale = amax / 448 (fp32 division), and one
// E4M3 byte per element, the E4M3 value nearest to x / scale (fp32
// division, ties to the even mantissa, saturating at 448; a magnitude that
// rounds to zero is stored as +0; an all-zero row has scale 0 and codes 0).
// V: NVFP4 groups exactly as in the NVFP4 cache.
//
// Work item = (sequence b, slot pair, kv-head h, group g) as in
// append_kernel.  The D/16 items of one (pair, h) are adjacent lanes of one
// warp (D/16 is 8 or 16 and divides the block size), so the row maximum of
// K is a shuffle reduction over those lanes.  Every lane of a warp takes
// part in the shuffles: lanes without work contribute 0 and write nothing,
// and the only early exits are uniform over the block.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3_byte(float q) {
  const uint32_t c = __nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
  return (c & 0x7fu) ? c : 0u;
}

__global__ void __launch_bounds__(256)
append_k8v4_kernel(uint8_t *__restrict__ pool, int num_pages, int Hkv, int D,
                   const int32_t *__restrict__ page_table, int max_pages,
                   const int32_t *__restrict__ kv_lens, int max_kv_len,
                   const __nv_bfloat16 *__restrict__ k_new,
                   const __nv_bfloat16 *__restrict__ v_new, const int32_t *__restrict__ cu_new,
                   int total_new, int max_new, int max_pairs, int32_t *err) {
  const int b = blockIdx.y;
  const int groups = D / kGroup;
  const int per_pair = Hkv * groups;
  const int item = blockIdx.x * blockDim.x + threadIdx.x;
  const int pair = item / per_pair;
  const int h = (item % per_pair) / groups;
  const int g = item % groups;

  // Checks of the sequence: the same for every thread of the block.
  const int row0 = cu_new[b];
  const int n = cu_new[b + 1] - row0;
  const int len = kv_lens[b];
  if (n <= 0) return;
  const int first = len - n;
  if (row0 < 0 || row0 + n > total_new || n > max_new || first < 0 || len > max_kv_len ||
      len > max_pages * kPageTokens) {
    if (item == 0) report(err, NVKV_DEVERR_LENGTH);
    return;
  }

  const int pos_even = 2 * ((first >> 1) + pair);
  bool live = item < max_pairs * per_pair && pos_even < len;
  int page = 0;
  if (live) {
    page = page_table[(size_t)b * max_pages + pos_even / kPageTokens];
    if (page < 0 || page >= num_pages) {
      report(err, NVKV_DEVERR_PAGE_ID);
      live = false;
    }
  }
  const int slot_even = pos_even % kPageTokens;
  uint8_t *blk = pool + ((size_t)page * Hkv + h) * k8_head_bytes(D);

  bool is_new[2];
  size_t src[2];
  float kx[2][16];
  float amax[2] = {0.f, 0.f};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int pos = pos_even + k;
    is_new[k] = live && pos >= first && pos < len;
    src[k] = ((size_t)(row0 + pos - first) * Hkv + h) * D + g * kGroup;
    if (is_new[k]) {
      load16_f32(k_new + src[k], kx[k]);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) kx[k][i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) amax[k] = fmaxf(amax[k], fabsf(kx[k][i]));
  }
  for (int o = 1; o < groups; o <<= 1) {  // row maximum over the row's D/16 lanes
    amax[0] = fmaxf(amax[0], __shfl_xor_sync(0xffffffffu, amax[0], o));
    amax[1] = fmaxf(amax[1], __shfl_xor_sync(0xffffffffu, amax[1], o));
  }

  GroupQ vq[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    if (!is_new[k]) continue;
    const int slot = slot_even + k;
    const float sc = __fdiv_rn(amax[k], 448.0f);
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (sc != 0.f) {
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i >> 2] |= e4m3_byte(__fdiv_rn(kx[k][i], sc)) << (8 * (i & 3));
    }
    *reinterpret_cast<uint4 *>(blk + (size_t)slot * D + g * kGroup) =
        make_uint4(w[0], w[1], w[2], w[3]);
    if (g == 0) *reinterpret_cast<float *>(blk + k8_ks_off(D) + 4 * slot) = sc;
    vq[k] = quantize16(v_new + src[k]);
    blk[k8_vs_off(D) + g * kPageTokens + slot] = vq[k].scale;
  }
  if (!live) return;
  // V code bytes (d, slot_even/2) for the 16 elements of group g.
  uint8_t *vc = blk + k8_vc_off(D) + (size_t)(g * kGroup) * 8 + slot_even / 2;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    uint8_t *p = vc + i * 8;
    const uint32_t lo = is_new[0] ? ((i < 8 ? vq[0].codes_lo : vq[0].codes_hi) >> (4 * (i & 7))) & 15u
                                  : *p & 15u;
    const uint32_t hi = is_new[1] ? ((i < 8 ? vq[1].codes_lo : vq[1].codes_hi) >> (4 * (i & 7))) & 15u
                                  : *p >> 4;
    *p = static_cast<uint8_t>(lo | (hi << 4));
  }
}

cudaError_t launch_append_k8v4(const nvkv_cache &c, const nvkv_seqs &s, const void *k_new,
                               const void *v_new, const int32_t *cu_new, int total_new,
                               int max_new, cudaStream_t stream) {
  const int max_pairs = max_new / 2 + 1;
  const int per_pair = c.num_kv_heads * (c.head_dim / kGroup);
  const long items = (long)max_pairs * per_pair;
  const int threads = 256;
  dim3 grid((unsigned)((items + threads - 1) / threads), (unsigned)s.batch);
  append_k8v4_kernel<<<grid, threads, 0, stream>>>(
      c.pool, c.num_pages, c.num_kv_heads, c.head_dim, s.page_table, s.max_pages_per_seq,
      s.kv_lens, s.max_kv_len, static_cast<const __nv_bfloat16 *>(k_new),
      static_cast<const __nv_bfloat16 *>(v_new), cu_new, total_new, max_new, max_pairs,
      s.err_word);
  return cudaGetLastError();
}

namespace {

// (cos, sin) of (pos / scale) * base^(-2i / rotary_dim), in double, rounded
// once to float; one thread per (pos, i).
__global__ void __launch_bounds__(256)
rope_table_kernel(float *__restrict__ cs, int max_pos, int rotary_dim, double base, double scale) {
  const int h = rotary_dim / 2;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)max_pos * h) return;
  const int pos = (int)(idx / h), i = (int)(idx % h);
  const double a = ((double)pos / scale) * pow(base, -2.0 * i / rotary_dim);
  cs[2 * idx] = (float)cos(a);
  cs[2 * idx + 1] = (float)sin(a);
}

}  // namespace

cudaError_t launch_rope_table(float *cs, int max_pos, int rotary_dim, double base, double scale,
                              cudaStream_t stream) {
  const int64_t n = (int64_t)max_pos * (rotary_dim / 2);
  rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(cs, max_pos, rotary_dim,
                                                                      base, scale);
  return cudaGetLastError();
}

}  // namespace nvkv
