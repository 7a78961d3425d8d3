// decode_simt.cu -- split-K GQA decode / MTP-verify attention over the NVFP4
// paged pool on CUDA cores (reference kernel of the library).
//
// Serves the decode half of the path the "knoopx/ninfer" README describes in
// "Capabilities and limits" (batched decode, MTP verify with one to five
// drafts) over the NVFP4 KV cache of the "gzenz/ninfer" README, "Context and
// model".  For query row (t, g) of kv-head h of sequence b, at position
// pos = kv_len - T + t, it computes over the keys j <= pos of its split
//     s_j = sm_scale * q . Khat_j,   m = max s,   l = sum 2^(s_j log2e - m'),
//     o = sum p_j Vhat_j / l
// and stores o and lse2 = m' + log2(l) (base-2 log-sum-exp of the scaled
// scores) per split; nvkv_combine merges the splits.
//
// One CTA per split-plan range; one warp per query row.  Per page of 16
// tokens a warp reads the K codes of the page (two lanes per token, half of
// head_dim each), forms the 16 scores, updates the online softmax, then
// each lane accumulates D/32 output channels from the transposed V codes.
//
// The same kernels serve the K8V4 cache (the "knoopx/ninfer" README lists it
// among its KV storage formats): K rows of one E4M3 byte per element with
// one float scale per row, V as in the NVFP4 cache.  Only the K score and
// the block offsets differ; the softmax and the value sums are shared.
#include "nvkv_common.cuh"

namespace nvkv {

constexpr int kSimtWarps = 8;

// Partial score of K row `slot` of a page block: the dot product of the
// half `half` of head_dim with the same half of the query row qr.
//
// NVFP4 block: 4-bit codes, one E4M3 scale per 16 elements.
__device__ __forceinline__ float k_half_score(Nvfp4Layout, const uint8_t *blk, int D, int slot,
                                              int half, const float *qr) {
  const uint8_t *kc = blk + kc_off(D) + slot * (D / 2) + half * (D / 4);
  const uint8_t *ks = blk + ks_off(D) + slot * (D / 16) + half * (D / 32);
  const float *qh = qr + half * (D / 2);
  float s = 0.f;
  for (int c16 = 0; c16 < D / 64; ++c16) {  // 16 bytes = 32 elements = 2 groups
    uint4 w4 = *reinterpret_cast<const uint4 *>(kc + 16 * c16);
    uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int gg = 0; gg < 2; ++gg) {
      float part = 0.f;
#pragma unroll
      for (int bi = 0; bi < 8; ++bi) {
        const int byte_idx = gg * 8 + bi;
        uint32_t byte = (w[byte_idx >> 2] >> (8 * (byte_idx & 3))) & 0xffu;
        float2 v = f16x2_to_float2(e2m1x2_to_f16x2(byte));
        const int d = 32 * c16 + 2 * byte_idx;
        part = fmaf(v.x, qh[d], part);
        part = fmaf(v.y, qh[d + 1], part);
      }
      s = fmaf(part, e4m3_to_float(ks[2 * c16 + gg]), s);
    }
  }
  return s;
}

// K8V4 block: one E4M3 byte per element, one float scale per row.
__device__ __forceinline__ float k_half_score(K8v4Layout, const uint8_t *blk, int D, int slot,
                                              int half, const float *qr) {
  const uint8_t *kc = blk + slot * D + half * (D / 2);
  const float row_scale = *reinterpret_cast<const float *>(blk + k8_ks_off(D) + 4 * slot);
  const float *qh = qr + half * (D / 2);
  float part = 0.f;
  for (int c16 = 0; c16 < D / 32; ++c16) {  // 16 bytes = 16 elements
    uint4 w4 = *reinterpret_cast<const uint4 *>(kc + 16 * c16);
    uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      uint32_t h2[2];
      e4m3x4_to_f16x2x2(w[wi], h2);  // h2[k] = elements 2k, 2k+1 of the word
      const float2 a = f16x2_to_float2(h2[0]), b = f16x2_to_float2(h2[1]);
      const int d = 16 * c16 + 4 * wi;
      part = fmaf(a.x, qh[d], part);
      part = fmaf(a.y, qh[d + 1], part);
      part = fmaf(b.x, qh[d + 2], part);
      part = fmaf(b.y, qh[d + 3], part);
    }
  }
  return part * row_scale;
}

// Online softmax of one query row (qr: fp32, pre-scaled to base-2 scores)
// over keys [jb, je) of one sequence / kv-head, jb a multiple of 16, in a
// pool of layout L.  The calling warp returns the running max m, the sum l
// of 2^(s - m) and, per lane, the unnormalised value sums of channels
// [lane*D/32, (lane+1)*D/32).
template <class L>
__device__ __forceinline__ void attend_rows_simt(const uint8_t *__restrict__ pool, int num_pages,
                                                 int Hkv, int D, int h,
                                                 const int32_t *__restrict__ pt, int jb, int je,
                                                 const float *qr, float &m, float &l, float acc[8],
                                                 int32_t *err) {
  const int lane = threadIdx.x & 31;
  const int dpl = D / 32;
  m = -INFINITY;
  l = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int p0 = jb; p0 < je; p0 += kPageTokens) {
    const int page = pt[p0 / kPageTokens];
    if (page < 0 || page >= num_pages) {
      if (lane == 0) report(err, NVKV_DEVERR_PAGE_ID);
      continue;
    }
    const uint8_t *blk = pool + (size_t)page * Hkv * L::head(D) + (size_t)h * L::head(D);
    // ---- scores: lane -> (slot, half of head_dim) ----
    const int slot = lane & 15, half = lane >> 4;
    const bool valid = (p0 + slot) < je;
    float s = k_half_score(L{}, blk, D, slot, half, qr);
    s += __shfl_xor_sync(0xffffffffu, s, 16);
    const float s_eff = valid ? s : -INFINITY;
    const float m_new = fmaxf(m, warp_max(s_eff));
    const float alpha = exp2f(m - m_new);  // m = -inf on the first page -> 0
    const float p = valid ? exp2f(s - m_new) : 0.f;
    l = l * alpha + warp_sum(lane < 16 ? p : 0.f);
    m = m_new;
    // ---- values: lane -> channels [lane*dpl, lane*dpl + dpl) ----
    const int d0 = lane * dpl;
    const int g = d0 / kGroup;
    uint4 sc4 = *reinterpret_cast<const uint4 *>(blk + L::vs(D) + g * kPageTokens);
    uint32_t sc[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
    float wgt[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p, j);
      const uint8_t sb = (sc[j >> 2] >> (8 * (j & 3))) & 0xffu;
      wgt[j] = (p0 + j < je) ? pj * e4m3_to_float(sb) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= dpl) break;
      const uint2 cw = *reinterpret_cast<const uint2 *>(blk + L::vc(D) + (size_t)(d0 + i) * 8);
      uint32_t cws[2] = {cw.x, cw.y};
      float a = acc[i] * alpha;
#pragma unroll
      for (int bi = 0; bi < 8; ++bi) {
        uint32_t byte = (cws[bi >> 2] >> (8 * (bi & 3))) & 0xffu;
        float2 v = f16x2_to_float2(e2m1x2_to_f16x2(byte));
        a = fmaf(wgt[2 * bi], v.x, a);
        a = fmaf(wgt[2 * bi + 1], v.y, a);
      }
      acc[i] = a;
    }
  }
}

template <class L>
__global__ void __launch_bounds__(kSimtWarps * 32)
decode_simt_kernel(const uint8_t *__restrict__ pool, int num_pages, int Hkv, int D,
                   const int32_t *__restrict__ page_table, int max_pages,
                   const int32_t *__restrict__ kv_lens, int B, int max_kv_len,
                   const __nv_bfloat16 *__restrict__ q, int T, int Hq, float qscale,
                   int S, float *__restrict__ ws_o, float *__restrict__ ws_lse, int32_t *err) {
  extern __shared__ float qs[];  // [R][D] query rows of the current pair, pre-scaled
  const int G = Hq / Hkv;
  const int R = T * G;
  const int c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int64_t U = 0;
  for (int b = 0; b < B; ++b) U += (int64_t)units_of_len(kv_lens[b]) * Hkv;
  if (U == 0) return;
  const int64_t u0 = range_begin(c, U, S), u1 = range_begin(c + 1, U, S);
  int64_t u = u0;
  while (u < u1) {
    int b, h, units;
    int64_t pair_start;
    locate_pair(kv_lens, B, Hkv, u, b, h, pair_start, units);
    const int64_t seg_end = min(u1, pair_start + units);
    const int kv_len = kv_lens[b];
    const int tok_begin = (int)(u - pair_start) * kUnitTokens;
    const int tok_end = min((int)(seg_end - pair_start) * kUnitTokens, kv_len);
    const size_t slot = (size_t)c + (size_t)b * Hkv + h;
    const bool bad_len = kv_len > max_kv_len || kv_len > max_pages * kPageTokens;
    if (bad_len && threadIdx.x == 0) report(err, NVKV_DEVERR_LENGTH);

    __syncthreads();  // previous segment's rows are done with qs
    for (int i = threadIdx.x; i < R * D; i += blockDim.x) {
      const int r = i / D, d = i % D;
      const int t = r / G, g = r % G;
      const size_t qi = ((size_t)(b * T + t) * Hq + h * G + g) * D + d;
      qs[i] = __bfloat162float(q[qi]) * qscale;
    }
    __syncthreads();

    const int32_t *pt = page_table + (size_t)b * max_pages;
    const int dpl = D / 32;  // output channels per lane
    for (int r = warp; r < R; r += kSimtWarps) {
      const int t = r / G;
      const int n_vis = kv_len - T + t + 1;  // keys 0 .. n_vis-1 are visible
      const int jb = tok_begin, je = bad_len ? jb : min(tok_end, n_vis);
      float m, l, acc[8];
      attend_rows_simt<L>(pool, num_pages, Hkv, D, h, pt, jb, je, qs + (size_t)r * D, m, l, acc,
                          err);
      // ---- partial result of this split for row r ----
      float *o = ws_o + (slot * R + r) * (size_t)D;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      for (int i = 0; i < dpl; ++i) o[lane * dpl + i] = acc[i] * inv;
      if (lane == 0) ws_lse[slot * R + r] = l > 0.f ? m + log2f(l) : -INFINITY;
    }
    u = seg_end;
  }
}

// k8: the pool is in the K8V4 layout (else NVFP4).
cudaError_t launch_decode_simt(const nvkv_cache &c, const nvkv_seqs &s, const void *q, int T,
                               int Hq, float sm_scale, int S, float *ws_o, float *ws_lse,
                               cudaStream_t stream, bool k8) {
  const int R = T * (Hq / c.num_kv_heads);
  const size_t smem = (size_t)R * c.head_dim * sizeof(float);
  auto kernel = k8 ? decode_simt_kernel<K8v4Layout> : decode_simt_kernel<Nvfp4Layout>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const float qscale = sm_scale * 1.4426950408889634f;  // scores in base 2
  kernel<<<S, kSimtWarps * 32, smem, stream>>>(
      c.pool, c.num_pages, c.num_kv_heads, c.head_dim, s.page_table, s.max_pages_per_seq,
      s.kv_lens, s.batch, s.max_kv_len, static_cast<const __nv_bfloat16 *>(q), T, Hq, qscale, S,
      ws_o, ws_lse, s.err_word);
  return cudaGetLastError();
}

// Chunked prefill on CUDA cores: one warp per (chunk row, query head), over
// the row's whole visible prefix (keys 0 .. its position).  Used for chunks
// the tensor-core prefill kernel does not take.
template <class L>
__global__ void __launch_bounds__(kSimtWarps * 32)
prefill_simt_kernel(const uint8_t *__restrict__ pool, int num_pages, int Hkv, int D,
                    const int32_t *__restrict__ page_table, int max_pages,
                    const int32_t *__restrict__ kv_lens, int B, int max_kv_len,
                    const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ cu_q,
                    int total_q, int Hq, float qscale, __nv_bfloat16 *__restrict__ out,
                    int32_t *err) {
  extern __shared__ float qs[];  // [kSimtWarps][D]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long w = (long)blockIdx.x * kSimtWarps + warp;
  if (w >= (long)total_q * Hq) return;
  const int row = (int)(w / Hq), hq = (int)(w % Hq);
  const int G = Hq / Hkv, h = hq / G;
  int b = 0;
  while (b + 1 < B && cu_q[b + 1] <= row) ++b;
  const int n_b = cu_q[b + 1] - cu_q[b];
  const int kv_len = kv_lens[b];
  const int pos = kv_len - n_b + (row - cu_q[b]);
  float *qr = qs + warp * D;
  for (int d = lane; d < D; d += 32) qr[d] = __bfloat162float(q[((size_t)row * Hq + hq) * D + d]) * qscale;
  __syncwarp();
  int je = pos + 1;
  if (row - cu_q[b] >= n_b || pos < 0 || kv_len > max_kv_len ||
      kv_len > max_pages * kPageTokens) {
    if (lane == 0) report(err, NVKV_DEVERR_LENGTH);
    je = 0;
  }
  float m, l, acc[8];
  attend_rows_simt<L>(pool, num_pages, Hkv, D, h, page_table + (size_t)b * max_pages, 0, je, qr,
                      m, l, acc, err);
  const int dpl = D / 32;
  const float inv = l > 0.f ? 1.f / l : 0.f;
  __nv_bfloat16 *dst = out + ((size_t)row * Hq + hq) * D + lane * dpl;
  for (int i = 0; i < dpl; ++i) dst[i] = __float2bfloat16_rn(acc[i] * inv);
}

cudaError_t launch_prefill_simt(const nvkv_cache &c, const nvkv_seqs &s, const void *q,
                                const int32_t *cu_q, int total_q, int Hq, float sm_scale,
                                void *out, cudaStream_t stream, bool k8) {
  const long warps = (long)total_q * Hq;
  const long blocks = (warps + kSimtWarps - 1) / kSimtWarps;
  const size_t smem = (size_t)kSimtWarps * c.head_dim * sizeof(float);
  const float qscale = sm_scale * 1.4426950408889634f;
  auto kernel = k8 ? prefill_simt_kernel<K8v4Layout> : prefill_simt_kernel<Nvfp4Layout>;
  kernel<<<(unsigned)blocks, kSimtWarps * 32, smem, stream>>>(
      c.pool, c.num_pages, c.num_kv_heads, c.head_dim, s.page_table, s.max_pages_per_seq,
      s.kv_lens, s.batch, s.max_kv_len, static_cast<const __nv_bfloat16 *>(q), cu_q, total_q, Hq,
      qscale, static_cast<__nv_bfloat16 *>(out), s.err_word);
  return cudaGetLastError();
}

}  // namespace nvkv
