// combine.cu -- merge the split-K partial results of nvkv_decode_attn.
//
// Each split s of a (sequence, kv-head) pair left, per query row, the
// normalised partial output o_s and lse2_s = base-2 log-sum-exp of its
// scaled scores (-inf when the row saw no key in that split).  The exact
// softmax over the union of the splits is
//     L = max_s lse2_s,  w_s = 2^(lse2_s - L),  out = sum_s w_s o_s / sum_s w_s,
// rounded once to bf16.  One warp per query row; each lane owns D/32
// channels.
#include "nvkv_common.cuh"

namespace nvkv {

__global__ void __launch_bounds__(256)
combine_kernel(const int32_t *__restrict__ kv_lens, int B, int Hkv, int T, int Hq, int D, int S,
               const float *__restrict__ ws_o, const float *__restrict__ ws_lse,
               __nv_bfloat16 *__restrict__ out) {
  const int G = Hq / Hkv;
  const int R = T * G;
  const long wid = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (long)B * Hkv * R) return;
  const int bh = (int)(wid / R), r = (int)(wid % R);
  const int b = bh / Hkv, h = bh % Hkv;
  const int t = r / G, g = r % G;
  const int dpl = D / 32;
  __nv_bfloat16 *dst = out + ((size_t)(b * T + t) * Hq + h * G + g) * D + lane * dpl;

  int64_t U = 0, pair_start = 0;
  int units = 0;
  for (int bb = 0; bb < B; ++bb) {
    const int ub = units_of_len(kv_lens[bb]);
    if (bb == b) {
      pair_start = U + (int64_t)h * ub;
      units = ub;
    }
    U += (int64_t)ub * Hkv;
  }
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (units > 0) {
    const int64_t c0 = range_of_unit(pair_start, U, S);
    const int64_t c1 = range_of_unit(pair_start + units - 1, U, S);
    // A range that owns no unit (possible only when U < S) wrote nothing.
    const bool all_own_units = U >= S;
    // The lse of up to 32 ranges at a time, one per lane; their max.
    float L = -INFINITY;
    for (int64_t cb = c0; cb <= c1; cb += 32) {
      const int64_t c = cb + lane;
      if (c <= c1 && (all_own_units || range_begin(c, U, S) != range_begin(c + 1, U, S)))
        L = fmaxf(L, ws_lse[(size_t)(c + bh) * R + r]);
    }
    L = warp_max(L);
    if (L > -INFINITY) {
      for (int64_t cb = c0; cb <= c1; cb += 32) {
        const int64_t c = cb + lane;
        float w = 0.f;  // weight of range c; 0 for ranges without keys of this row
        if (c <= c1 && (all_own_units || range_begin(c, U, S) != range_begin(c + 1, U, S))) {
          const float lse = ws_lse[(size_t)(c + bh) * R + r];
          if (lse > -INFINITY) w = exp2f(lse - L);
        }
        const int n = c1 - cb + 1 < 32 ? (int)(c1 - cb + 1) : 32;
        for (int k = 0; k < n; ++k) {
          const float wk = __shfl_sync(0xffffffffu, w, k);
          if (wk == 0.f) continue;  // warp-uniform
          wsum += wk;
          const float *o = ws_o + ((size_t)(cb + k + bh) * R + r) * (size_t)D + lane * dpl;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (i < dpl) acc[i] = fmaf(wk, o[i], acc[i]);
        }
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i < dpl) dst[i] = __float2bfloat16_rn(acc[i] * inv);
}

cudaError_t launch_combine(const nvkv_seqs &s, const void *ws_o, const void *ws_lse, int T,
                           int Hq, int Hkv, int D, int S, void *out, cudaStream_t stream) {
  const int R = T * (Hq / Hkv);
  const long warps = (long)s.batch * Hkv * R;
  const int threads = 256;
  const long blocks = (warps * 32 + threads - 1) / threads;
  combine_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
      s.kv_lens, s.batch, Hkv, T, Hq, D, S, static_cast<const float *>(ws_o),
      static_cast<const float *>(ws_lse), static_cast<__nv_bfloat16 *>(out));
  return cudaGetLastError();
}

}  // namespace nvkv
