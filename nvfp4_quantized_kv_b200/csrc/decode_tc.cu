// decode_tc.cu -- split-K GQA decode / MTP-verify attention over the NVFP4
// paged pool on the 5th-generation tensor cores (tcgen05), head_dim 256.
//
// What it computes is the decode half of the path in the "knoopx/ninfer"
// README, "Capabilities and limits" (batched decode, MTP verify with one to
// five drafts), over the NVFP4 KV cache of the "gzenz/ninfer" README,
// "Fork changes vs upstream" -> "Context and model": for every query row
// (t, g) of kv-head h of sequence b, at position kv_len - T + t, the
// softmax-weighted sum of the dequantised V rows over the visible keys of
// one split, as a partial result (o, base-2 log-sum-exp) that nvkv_combine
// merges.  Same contract and workspace layout as the CUDA-core kernel.
//
// Design (one CTA per split-plan range, persistent over its units):
//  * A unit is 128 tokens = 8 pages of one (sequence, kv-head).  The TMA
//    producer warp copies each page's 4608-byte kv-head block (36 rows of
//    128 B) into a 4-stage shared-memory ring with one 2-D tiled load per page
//    (128-byte swizzle, so the dequantising reads below are bank-conflict
//    free).  No multicast.
//  * Swap-AB: the dequantised K tile (128 tokens x 256 d, f16) and V^T tile
//    (2 x 128 d x 128 tokens) are the A operands, written straight from
//    registers into Tensor Memory; the G*T query rows (Q, then P) are the
//    small N side of the MMA, in shared memory.  S^T and O^T accumulate in
//    Tensor Memory in fp32.  Dequantisation is exact in f16
//    (E2M1 x E4M3 has at most 6 significant bits).
//  * 8 worker warps dequantise (K: one token per thread; V: one head_dim row
//    per thread), run the online softmax on S^T (one token per thread,
//    column maxima across the 128 lanes through shared memory) and write
//    P^T; one thread issues the MMAs.  The running max is only raised when
//    a tile max exceeds it by more than 2^8, so O^T is rarely rescaled.
//  * Every wait is bounded; a timeout sets NVKV_DEVERR_TIMEOUT, turns all
//    later waits into no-ops and lets the kernel drain and free its Tensor
//    Memory.
#include "nvkv_common.cuh"
#include "sm100.cuh"

namespace nvkv {
namespace {

using namespace sm100;

constexpr int kD = 256;
constexpr int kRowsPerHead = 36;      // 18*D bytes / 128
constexpr int kHeadBytes = 18 * kD;   // 4608
constexpr int kPagePitch = 5120;      // staged page pitch (1024-aligned)
constexpr int kUnitPages = 8;
constexpr int kStageBytes = kUnitPages * kPagePitch;
constexpr int kWorkerWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr long long kWaitBudget = 2000000000LL;  // clock cycles (~1 s)
constexpr float kLazyRescale = 8.0f;             // log2 units

constexpr uint32_t kColK = 0;    // 128 columns: K tile (token lanes, d pairs)
constexpr uint32_t kColV = 128;  // 2 x 64 columns: V^T halves (d lanes, token pairs)
constexpr uint32_t kColS = 256;  // N columns: S^T; then O^T halves of N columns each

template <int N>
struct Cfg {
  static constexpr int NH = N / 2;               // S^T columns per worker warp
  static constexpr int NST = N <= 64 ? 4 : 3;    // pipeline stages
  static constexpr uint32_t kColO = kColS + N;
  static constexpr int kQBytes = N * kD * 2;     // Q tile, K-major, no swizzle
  static constexpr int kPBytes = N * 128 * 2;    // P^T tile, MN-major, no swizzle
  static constexpr int kRedFloats = kWorkerWarps * 40;
  static constexpr int kOffQ = NST * kStageBytes;
  static constexpr int kOffP = kOffQ + kQBytes;
  static constexpr int kOffRed = kOffP + kPBytes;
  static constexpr int kOffM = kOffRed + kRedFloats * 4;
  static constexpr int kOffAlpha = kOffM + 80 * 4;
  static constexpr int kOffL = kOffAlpha + 80 * 4;
  static constexpr int kOffFlags = kOffL + 80 * 4;     // int[4]: rescale[2], abort, pad
  static constexpr int kOffPages = kOffFlags + 16;     // int[NST][8]: staged page ids
  static constexpr int kOffBars = kOffPages + NST * kUnitPages * 4;  // 8-byte aligned
  static constexpr int kNumBars = 2 * NST + 6;
  static constexpr int kOffTmem = kOffBars + kNumBars * 8;
  static constexpr int kSmemBytes = kOffTmem + 16 + 1024;  // + alignment slack
};

struct Shared {
  uint8_t *stages, *qtile, *ptile;
  float *red, *m_s, *alpha_s, *l_s;
  volatile int *flags;
  int32_t *pages;  // [NST][8], -1 = not loaded
  uint64_t *full, *empty, *kready, *sready, *pready, *vready, *pvdone, *final_bar;
  uint32_t *tmem_slot;
};

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *flags,
                                         int32_t *err) {
  if (flags[2]) return false;  // aborted: do not wait any more
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (flags[2]) return false;
    if (clock64() - t0 > kWaitBudget) {
      flags[2] = 1;
      report(err, NVKV_DEVERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Segment of the CTA's range: units [u, seg_end) of pair (b, h).
struct Seg {
  int b, h, kv_len;
  int64_t pair_start, seg_end;
  bool bad;
};

__device__ __forceinline__ Seg segment_at(int64_t u, int64_t u1, const int32_t *kv_lens, int B,
                                          int Hkv, int max_kv_len, int max_pages) {
  Seg s;
  int units;
  locate_pair(kv_lens, B, Hkv, u, s.b, s.h, s.pair_start, units);
  s.seg_end = min(u1, s.pair_start + units);
  s.kv_len = kv_lens[s.b];
  s.bad = s.kv_len > max_kv_len || s.kv_len > max_pages * kPageTokens;
  if (s.bad) s.kv_len = 0;  // nothing of a bad sequence is read
  return s;
}

__device__ __forceinline__ int page_of(const int32_t *pt_row, int tok, int kv_len, int num_pages) {
  if (tok >= kv_len) return -1;
  const int p = pt_row[tok / kPageTokens];
  return (p >= 0 && p < num_pages) ? p : -1;
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmap, int num_pages, int Hkv,
                 const int32_t *__restrict__ page_table, int max_pages,
                 const int32_t *__restrict__ kv_lens, int B, int max_kv_len,
                 const __nv_bfloat16 *__restrict__ q, int T, int Hq, float qscale, int S,
                 float *__restrict__ ws_o, float *__restrict__ ws_lse, int32_t *err) {
  using C = Cfg<N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Shared sh;
  sh.stages = smem;
  sh.qtile = smem + C::kOffQ;
  sh.ptile = smem + C::kOffP;
  sh.red = reinterpret_cast<float *>(smem + C::kOffRed);
  sh.m_s = reinterpret_cast<float *>(smem + C::kOffM);
  sh.alpha_s = reinterpret_cast<float *>(smem + C::kOffAlpha);
  sh.l_s = reinterpret_cast<float *>(smem + C::kOffL);
  sh.flags = reinterpret_cast<volatile int *>(smem + C::kOffFlags);
  sh.pages = reinterpret_cast<int32_t *>(smem + C::kOffPages);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBars);
  sh.full = bars;
  sh.empty = bars + C::NST;
  sh.kready = bars + 2 * C::NST;
  sh.sready = sh.kready + 1;
  sh.pready = sh.kready + 2;
  sh.vready = sh.kready + 3;
  sh.pvdone = sh.kready + 4;
  sh.final_bar = sh.kready + 5;
  sh.tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = Hq / Hkv;
  const int R = T * G;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], kWorkerWarps);
    }
    mbar_init(sh.kready, kWorkerWarps);
    mbar_init(sh.sready, 1);
    mbar_init(sh.pready, kWorkerWarps);
    mbar_init(sh.vready, kWorkerWarps);
    mbar_init(sh.pvdone, 1);
    mbar_init(sh.final_bar, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 4) sh.flags[threadIdx.x] = 0;
  if (threadIdx.x < 80) sh.m_s[threadIdx.x] = -INFINITY;
  if (warp == kMmaWarp) {
    tmem_alloc(sh.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sh.tmem_slot;

  int64_t U = 0;
  for (int b = 0; b < B; ++b) U += (int64_t)units_of_len(kv_lens[b]) * Hkv;
  const int c = blockIdx.x;
  const int64_t u0 = U > 0 ? range_begin(c, U, S) : 0;
  const int64_t u1 = U > 0 ? range_begin(c + 1, U, S) : 0;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      prefetch_tmap(&tmap);
      uint32_t uc = 0;
      for (int64_t u = u0; u < u1;) {
        const Seg sg = segment_at(u, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
        const int32_t *pt = page_table + (size_t)sg.b * max_pages;
        for (; u < sg.seg_end; ++u, ++uc) {
          const int stage = uc % C::NST;
          if (uc >= (uint32_t)C::NST)
            wait_bar(&sh.empty[stage], ((uc / C::NST) + 1) & 1, sh.flags, err);
          const int tok0 = (int)(u - sg.pair_start) * kUnitTokens;
          int pages[kUnitPages];
          uint32_t bytes = 0;
#pragma unroll
          for (int p = 0; p < kUnitPages; ++p) {
            pages[p] = page_of(pt, tok0 + p * kPageTokens, sg.kv_len, num_pages);
            if (tok0 + p * kPageTokens < sg.kv_len && pages[p] < 0) report(err, NVKV_DEVERR_PAGE_ID);
            if (pages[p] >= 0) bytes += kHeadBytes;
            sh.pages[stage * kUnitPages + p] = pages[p];
          }
          // The arrive releases the page ids to the workers that wait on it.
          mbar_arrive_expect_tx(&sh.full[stage], bytes);
#pragma unroll
          for (int p = 0; p < kUnitPages; ++p)
            if (pages[p] >= 0)
              tma_load_2d(sh.stages + stage * kStageBytes + p * kPagePitch, &tmap, 0,
                          (pages[p] * Hkv + sg.h) * kRowsPerHead, &sh.full[stage]);
        }
      }
      // Drain: every issued copy must land before the CTA may exit.
      const uint32_t first = uc > (uint32_t)C::NST ? uc - C::NST : 0;
      for (uint32_t k = first; k < uc; ++k)
        mbar_wait(&sh.full[k % C::NST], (k / C::NST) & 1, kWaitBudget);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_f16_f32(128, N, false, false);
      const uint32_t idesc_pv = idesc_f16_f32(128, N, false, true);
      const uint32_t qb = smem_u32(sh.qtile), pb = smem_u32(sh.ptile);
      uint32_t uc = 0;
      bool issued = false;
      for (int64_t u = u0; u < u1;) {
        const Seg sg = segment_at(u, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
        const int64_t seg_start = u;
        for (; u < sg.seg_end; ++u, ++uc) {
          const bool first = (u == seg_start);
          if (wait_bar(sh.kready, uc & 1, sh.flags, err)) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
              const uint64_t bd = smem_desc(qb + ks * 2 * (N * 16), N * 16, 128);
              mma_f16_ts(tmem + kColS, tmem + kColK + ks * 8, bd, idesc_qk, ks > 0);
            }
            issued = true;
          }
          mma_commit(sh.sready);
          const bool ok_p = wait_bar(sh.pready, uc & 1, sh.flags, err);
          const bool ok_v = wait_bar(sh.vready, uc & 1, sh.flags, err);
          if (ok_p && ok_v) {
            tc_fence_after();
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
              for (int ks = 0; ks < 8; ++ks) {
                const uint64_t bd = smem_desc(pb + ks * 256, 128, 2048);
                mma_f16_ts(tmem + C::kColO + hf * N, tmem + kColV + hf * 64 + ks * 8, bd,
                           idesc_pv, (!first) || ks > 0);
              }
            issued = true;
          }
          mma_commit(sh.pvdone);
        }
      }
      if (issued) {
        mma_commit(sh.final_bar);
        mbar_wait(sh.final_bar, 0, kWaitBudget);
      }
    }
  } else {
    // -------------------------------------------------------------- workers
    const int lq = warp & 3, hf = warp >> 2;
    const uint32_t lane_base = (uint32_t)(32 * lq) << 16;
    const uint32_t tl = tmem + lane_base;  // this warp's lane quarter
    const int tid = threadIdx.x;           // 0..255
    constexpr int NH = C::NH;
    float l_part[NH];
    uint32_t uc = 0;
    for (int64_t u = u0; u < u1;) {
      const Seg sg = segment_at(u, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
      if (sg.bad && tid == 0) report(err, NVKV_DEVERR_LENGTH);
      const int32_t *pt = page_table + (size_t)sg.b * max_pages;
      const int64_t seg_start = u;
      const size_t slot = (size_t)c + (size_t)sg.b * Hkv + sg.h;

      // Q tile of this pair: rows n < R are (t, g) = (n / G, n % G), pre-scaled
      // to base-2 scores, f16, K-major core-matrix layout; rows >= R are zero.
      for (int ci = tid; ci < N * (kD / 8); ci += kWorkerWarps * 32) {
        const int n = ci / (kD / 8), k8 = ci % (kD / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < R) {
          const int t = n / G, g = n % G;
          const uint4 raw = *reinterpret_cast<const uint4 *>(
              q + ((size_t)(sg.b * T + t) * Hq + sg.h * G + g) * kD + k8 * 8);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = __uint_as_float(w[i] << 16) * qscale;
            const float hi = __uint_as_float(w[i] & 0xffff0000u) * qscale;
            __half2 hh = __floats2half2_rn(lo, hi);
            o[i] = *reinterpret_cast<uint32_t *>(&hh);
          }
          v = make_uint4(o[0], o[1], o[2], o[3]);
        }
        *reinterpret_cast<uint4 *>(sh.qtile + k8 * (N * 16) + (n >> 3) * 128 + (n & 7) * 16) = v;
      }
      fence_proxy_async_smem();
#pragma unroll
      for (int i = 0; i < NH; ++i) l_part[i] = 0.f;
      // Keys visible to this thread's score columns n = hf*NH + i: row n is
      // query t = n / G at position kv_len - T + t; padding rows see none.
      int n_vis[NH];
#pragma unroll
      for (int i = 0; i < NH; ++i) {
        const int n = hf * NH + i;
        n_vis[i] = n < R ? sg.kv_len - T + n / G + 1 : 0;
      }

      for (; u < sg.seg_end; ++u, ++uc) {
        const bool first = (u == seg_start);
        const int stage = uc % C::NST;
        const uint8_t *stg = sh.stages + stage * kStageBytes;
        const int tok0 = (int)(u - sg.pair_start) * kUnitTokens;
        wait_bar(&sh.full[stage], (uc / C::NST) & 1, sh.flags, err);
        const int4 pa = *reinterpret_cast<const int4 *>(sh.pages + stage * kUnitPages);
        const int4 pb = *reinterpret_cast<const int4 *>(sh.pages + stage * kUnitPages + 4);
        const int pg_id[kUnitPages] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
        const bool full_unit = tok0 + kUnitTokens <= sg.kv_len &&
                               min(min(min(pa.x, pa.y), min(pa.z, pa.w)),
                                   min(min(pb.x, pb.y), min(pb.z, pb.w))) >= 0;

        // ---- K tile: thread = token jl, d in [128*hf, 128*hf + 128) ----
        {
          const int jl = 32 * lq + lane;
          const int p = jl >> 4, slot = jl & 15;
          const bool ok = full_unit ||
                          (sh.pages[stage * kUnitPages + p] >= 0 && tok0 + jl < sg.kv_len);
          const uint8_t *pg = stg + p * kPagePitch;
          // Scale bytes of groups 8*hf .. 8*hf+7 of this token.
          uint2 sc = make_uint2(0u, 0u);
          if (ok)
            sc = *reinterpret_cast<const uint2 *>(pg + (16 + (slot >> 3)) * 128 +
                                                  (((slot & 7) ^ (slot >> 3)) << 4) + hf * 8);
#pragma unroll
          for (int ci = 0; ci < 4; ++ci) {
            const int cch = 4 * hf + ci;  // 16-byte chunk = 32 d = groups 2cch, 2cch+1
            uint32_t words[16];
            if (ok) {
              const uint4 w4 = *reinterpret_cast<const uint4 *>(pg + slot * 128 +
                                                                ((cch ^ (slot & 7)) << 4));
              const uint32_t sword = ci < 2 ? sc.x : sc.y;
              const uint32_t sb0 = (sword >> (16 * (ci & 1))) & 0xffu;
              const uint32_t sb1 = (sword >> (16 * (ci & 1) + 8)) & 0xffu;
              const uint32_t s0 = e4m3x2_to_f16x2(sb0 | (sb0 << 8));
              const uint32_t s1 = e4m3x2_to_f16x2(sb1 | (sb1 << 8));
              const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
              for (int wi = 0; wi < 4; ++wi) {
                uint32_t t4[4];
                e2m1x8_to_f16x2x4(w[wi], t4);
#pragma unroll
                for (int k = 0; k < 4; ++k) words[4 * wi + k] = hmul2_u32(t4[k], wi < 2 ? s0 : s1);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) words[i] = 0u;
            }
            tmem_st16(tl + kColK + hf * 64 + ci * 16, words);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(sh.kready);
        }

        // PV of the previous unit must be done before O^T, P^T and the V^T
        // tile are touched.
        if (uc > 0) {
          wait_bar(sh.pvdone, (uc - 1) & 1, sh.flags, err);
          tc_fence_after();
        }

        // ---- V^T tile: thread = head_dim row d, 128 tokens (overlaps QK) ----
        {
          const int d = 128 * hf + 32 * lq + lane;
          const int g = d >> 4;
          const int vrow = 18 + (d >> 4);
          const int vchunk = ((d & 15) >> 1) ^ (vrow & 7);
          const int srow = 34 + (g >> 3);
          const int schunk = (g & 7) ^ (srow & 7);
#pragma unroll
          for (int p = 0; p < kUnitPages; ++p) {
            const int ptok = tok0 + p * kPageTokens;
            uint32_t o8[8];
            if (pg_id[p] >= 0) {
              const uint8_t *pg = stg + p * kPagePitch;
              const uint2 cw = *reinterpret_cast<const uint2 *>(pg + vrow * 128 + vchunk * 16 +
                                                                (d & 1) * 8);
              const uint4 s4 = *reinterpret_cast<const uint4 *>(pg + srow * 128 + schunk * 16);
              uint32_t c0[4], c1[4], sp[8];
              e2m1x8_to_f16x2x4(cw.x, c0);
              e2m1x8_to_f16x2x4(cw.y, c1);
              {
                uint32_t t2[2];
                e4m3x4_to_f16x2x2(s4.x, t2); sp[0] = t2[0]; sp[1] = t2[1];
                e4m3x4_to_f16x2x2(s4.y, t2); sp[2] = t2[0]; sp[3] = t2[1];
                e4m3x4_to_f16x2x2(s4.z, t2); sp[4] = t2[0]; sp[5] = t2[1];
                e4m3x4_to_f16x2x2(s4.w, t2); sp[6] = t2[0]; sp[7] = t2[1];
              }
#pragma unroll
              for (int i = 0; i < 8; ++i) o8[i] = hmul2_u32(i < 4 ? c0[i] : c1[i - 4], sp[i]);
              if (!full_unit && ptok + kPageTokens > sg.kv_len) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const int t0 = ptok + 2 * i;
                  if (t0 >= sg.kv_len) o8[i] = 0u;
                  else if (t0 + 1 >= sg.kv_len) o8[i] &= 0xffffu;
                }
              }
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) o8[i] = 0u;
            }
            tmem_st8(tl + kColV + hf * 64 + 8 * p, o8);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(sh.vready);
            mbar_arrive(&sh.empty[stage]);  // every read of the stage is done
          }
        }

        // ---- softmax on S^T: thread = token jl, columns hf*NH .. +NH ----
        wait_bar(sh.sready, uc & 1, sh.flags, err);
        tc_fence_after();
        float sv[NH];
        {
          const int pos = tok0 + 32 * lq + lane;
#pragma unroll
          for (int i8 = 0; i8 < NH / 8; ++i8) {
            uint32_t r[8];
            tmem_ld8(tl + kColS + hf * NH + i8 * 8, r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              sv[i8 * 8 + j] = pos < n_vis[i8 * 8 + j] ? __uint_as_float(r[j]) : -INFINITY;
          }
#pragma unroll
          for (int i = 0; i < NH; ++i) {
            const float mx = warp_max(sv[i]);
            if (lane == 0) sh.red[warp * 40 + i] = mx;
          }
        }
        named_barrier(1, kWorkerWarps * 32);
        if (tid < N) {
          const int n = tid, hn = n / NH, i = n % NH;
          float tmax = -INFINITY;
#pragma unroll
          for (int w = 0; w < 4; ++w) tmax = fmaxf(tmax, sh.red[(w + 4 * hn) * 40 + i]);
          const float m_old = sh.m_s[n];
          float alpha = 1.f;
          if (tmax > -INFINITY && (m_old == -INFINITY || tmax > m_old + kLazyRescale)) {
            alpha = exp2f(m_old - tmax);  // 0 when m_old = -inf
            sh.m_s[n] = tmax;
            sh.alpha_s[n] = alpha;
            sh.flags[uc & 1] = 1;
          } else {
            sh.alpha_s[n] = 1.f;
          }
        }
        if (tid == 0) sh.flags[(uc + 1) & 1] = 0;
        named_barrier(1, kWorkerWarps * 32);
        const bool rescale = sh.flags[uc & 1] != 0;
        float pv[NH];
#pragma unroll
        for (int i = 0; i < NH; ++i) {
          const int n = hf * NH + i;
          const float mu = sh.m_s[n];
          if (rescale) l_part[i] *= sh.alpha_s[n];
          pv[i] = sv[i] > -INFINITY ? exp2f(sv[i] - mu) : 0.f;
          l_part[i] += pv[i];
        }
        if (rescale && !first) {
          // O^T rows d = 128*hf + 32*lq + lane: column n *= alpha_n.
#pragma unroll
          for (int j8 = 0; j8 < N / 8; ++j8) {
            uint32_t r[8];
            const uint32_t addr = tl + C::kColO + hf * N + j8 * 8;
            tmem_ld8(addr, r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              r[j] = __float_as_uint(__uint_as_float(r[j]) * sh.alpha_s[j8 * 8 + j]);
            tmem_st8(addr, r);
          }
          tmem_wait_st();
        }
        {
          // P^T (MN-major): element (n, k) at (n/8)*2048 + (k/8)*128 + (k%8)*16 + (n%8)*2.
          const int k = 32 * lq + lane;
#pragma unroll
          for (int j = 0; j < NH / 8; ++j) {
            uint32_t h2[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __half2 hh = __floats2half2_rn(pv[8 * j + 2 * e], pv[8 * j + 2 * e + 1]);
              h2[e] = *reinterpret_cast<uint32_t *>(&hh);
            }
            const int n8 = (hf * NH) / 8 + j;
            *reinterpret_cast<uint4 *>(sh.ptile + n8 * 2048 + (k >> 3) * 128 + (k & 7) * 16) =
                make_uint4(h2[0], h2[1], h2[2], h2[3]);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(sh.pready);
        }
      }

      // ---- end of segment: l totals, then O^T / l -> workspace ----
      if (uc > 0) {
        wait_bar(sh.pvdone, (uc - 1) & 1, sh.flags, err);
        tc_fence_after();
      }
#pragma unroll
      for (int i = 0; i < NH; ++i) {
        const float ls = warp_sum(l_part[i]);
        if (lane == 0) sh.red[warp * 40 + i] = ls;
      }
      named_barrier(1, kWorkerWarps * 32);
      if (tid < N) {
        const int n = tid, hn = n / NH, i = n % NH;
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) l += sh.red[(w + 4 * hn) * 40 + i];
        sh.l_s[n] = l;
        if (n < R) ws_lse[slot * R + n] = l > 0.f ? sh.m_s[n] + log2f(l) : -INFINITY;
      }
      named_barrier(1, kWorkerWarps * 32);
      {
        const int d = 128 * hf + 32 * lq + lane;
#pragma unroll
        for (int j8 = 0; j8 < N / 8; ++j8) {
          uint32_t r[8];
          tmem_ld8(tl + C::kColO + hf * N + j8 * 8, r);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int n = j8 * 8 + j;
            if (n < R) {
              const float l = sh.l_s[n];
              ws_o[(slot * R + n) * kD + d] = l > 0.f ? __uint_as_float(r[j]) / l : 0.f;
            }
          }
        }
      }
      tc_fence_before();
      named_barrier(1, kWorkerWarps * 32);
      if (tid < N) sh.m_s[tid] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

template <int N>
cudaError_t launch_n(const CUtensorMap &map, const nvkv_cache &c, const nvkv_seqs &s,
                     const void *q, int T, int Hq, float qscale, int S, float *ws_o,
                     float *ws_lse, cudaStream_t stream) {
  const int smem = Cfg<N>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<N>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  decode_tc_kernel<N><<<S, kThreads, smem, stream>>>(
      map, c.num_pages, c.num_kv_heads, s.page_table, s.max_pages_per_seq, s.kv_lens, s.batch,
      s.max_kv_len, static_cast<const __nv_bfloat16 *>(q), T, Hq, qscale, S, ws_o, ws_lse,
      s.err_word);
  return cudaGetLastError();
}

}  // namespace

// True when the tensor-core decode kernel takes this shape.
bool decode_tc_supported(const nvkv_cache &c, int T, int Hq) {
  const int R = T * (Hq / c.num_kv_heads);
  return c.head_dim == kD && R >= 1 && R <= 80 && encode_fn() != nullptr;
}

cudaError_t launch_decode_tc(const nvkv_cache &c, const nvkv_seqs &s, const void *q, int T,
                             int Hq, float sm_scale, int S, float *ws_o, float *ws_lse,
                             cudaStream_t stream) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  // The pool as a 2-D byte tensor of 128-byte rows; one box = one page's
  // kv-head block (36 rows).
  CUtensorMap map;
  const cuuint64_t rows = (cuuint64_t)c.num_pages * c.num_kv_heads * kRowsPerHead;
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {128, kRowsPerHead};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, c.pool, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const int R = T * (Hq / c.num_kv_heads);
  const float qscale = sm_scale * 1.4426950408889634f;
  if (R <= 16) return launch_n<16>(map, c, s, q, T, Hq, qscale, S, ws_o, ws_lse, stream);
  if (R <= 32) return launch_n<32>(map, c, s, q, T, Hq, qscale, S, ws_o, ws_lse, stream);
  if (R <= 48) return launch_n<48>(map, c, s, q, T, Hq, qscale, S, ws_o, ws_lse, stream);
  if (R <= 64) return launch_n<64>(map, c, s, q, T, Hq, qscale, S, ws_o, ws_lse, stream);
  return launch_n<80>(map, c, s, q, T, Hq, qscale, S, ws_o, ws_lse, stream);
}

}  // namespace nvkv
