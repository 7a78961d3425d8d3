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
