// prefill_tc.cu -- chunked-prefill attention over the NVFP4 paged pool on the
// 5th-generation tensor cores (tcgen05), head_dim 256.
//
// Computes the chunked prefill of the "knoopx/ninfer" README, "Capabilities
// and limits": the n_b newest positions of a sequence (their K/V rows already
// quantise-appended) attend causally to the whole NVFP4 cache of the
// "gzenz/ninfer" README, "Fork changes vs upstream" -> "Context and model".
// Query row (i, g) of kv-head h is chunk token i, query head h*G + g, at
// position kv_len - n_b + i; it sees keys 0 .. that position.
//
// Here the path is a dense contraction, so it runs in the usual orientation:
// one CTA owns 128 query rows (tokens x GQA heads) of one kv-head and streams
// the keys in 64-token tiles.
//  * A TMA producer warp copies each tile's 4 page blocks into a 4-stage
//    ring (as in the decode kernel: 36-row boxes, 128-byte swizzle).
//  * 8 dequantising warps write the K tile (64 tokens x 256 d) and the V^T
//    tile (256 d x 64 tokens) as f16 into shared memory in the canonical
//    no-swizzle K-major layouts the MMA reads; both are double-buffered.
//    E2M1 x E4M3 is exact in f16.
//  * Q (128 rows x 256 d, f16, pre-scaled to base-2 scores) sits in Tensor
//    Memory as the A operand of S = Q K^T (M=128, N=64); S is double-buffered
//    in Tensor Memory and P (f16) overwrites its own S slot, as the A operand
//    of O += P V (M=128, N=256); O lives in Tensor Memory (256 columns).
//  * 4 softmax warps own one query row per thread: row max, exp2, the
//    running max (raised lazily, only when it grows by more than 2^8, then O
//    is rescaled), the denominator of the f16 weights, and the final O / l.
//  * One thread issues the MMAs, event-driven; every wait is bounded.
#include "nvkv_common.cuh"
#include "sm100.cuh"

namespace nvkv {

bool make_pool_tmap(const nvkv_cache &c, CUtensorMap *map);

namespace {

using namespace sm100;

constexpr int kD = 256;
constexpr int kRowsPerHead = 36;
constexpr int kHeadBytes = 18 * kD;
constexpr int kPagePitch = 5120;
constexpr int kTileTokens = 64;
constexpr int kTilePages = 4;
constexpr int kStages = 4;
constexpr int kStageBytes = kTilePages * kPagePitch;   // 20 KB
constexpr int kKTileBytes = kTileTokens * kD * 2;      // 32 KB
constexpr int kVTileBytes = kD * kTileTokens * 2;      // 32 KB
constexpr int kDeqWarps = 8;                           // warps 0..7
constexpr int kSmxWarp0 = 8;                           // warps 8..11
constexpr int kSmxWarps = 4;
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kThreads = 14 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr long long kWaitBudget = 2000000000LL;
// After a poll that found nothing ready the MMA thread sleeps this long,
// leaving issue slots to the dequantising and softmax warps it waits for
// (measured: +3-4 % over spinning; 1 us is too long).
constexpr unsigned kPollSleepNs = 300;
constexpr float kLazyRescale = 8.0f;

// Tensor Memory columns.
constexpr uint32_t kColQ = 0;     // 128: Q (row lanes, d pairs)
constexpr uint32_t kColS = 128;   // 2 x 64: S slots (P overwrites the first 32 columns)
constexpr uint32_t kColO = 256;   // 256: O (row lanes, fp32 d)

// Shared memory.
constexpr int kOffK = kStages * kStageBytes;
constexpr int kOffV = kOffK + 2 * kKTileBytes;
constexpr int kVscBytes = kTilePages * 16 * 8 * 4;            // V scales of a tile as f16 pairs
constexpr int kOffVsc = kOffV + 2 * kVTileBytes;              // 2 tables (tile parity)
constexpr int kOffPages = kOffVsc + 2 * kVscBytes;            // int[stages][4]
constexpr int kOffFlags = kOffPages + kStages * kTilePages * 4;
constexpr int kOffBars = kOffFlags + 16;
constexpr int kNumBars = 2 * kStages + 2 * 5 + 2;  // full, empty; kready, vready, sready, pready, pvdone; qready, final
constexpr int kOffTmem = kOffBars + kNumBars * 8;
constexpr int kSmemBytes = kOffTmem + 16 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kOffK % 1024 == 0 && kOffPages % 16 == 0 && kOffBars % 8 == 0, "alignment");

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *flags,
                                         int32_t *err) {
  return guarded_wait(bar, parity, flags + 2, err, kWaitBudget);  // flags[2]: abort
}

__device__ __forceinline__ uint32_t dup_scale(uint32_t byte) {
  return e4m3x2_to_f16x2(byte | (byte << 8));
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap, int num_pages, int Hkv,
                  const int32_t *__restrict__ page_table, int max_pages,
                  const int32_t *__restrict__ kv_lens, int max_kv_len,
                  const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ cu_q,
                  int total_q, int Hq, float qscale, __nv_bfloat16 *__restrict__ out,
                  int num_splits, float *__restrict__ ws_o, float *__restrict__ ws_lse,
                  int32_t *err) {
  // blockIdx.x = m-tile * num_splits + split: split s of an m-tile takes the
  // s-th of num_splits equal runs of its key tiles and, when num_splits > 1,
  // leaves O / l and log2(l) + m of its rows in the workspace for the merge.
  const int mt = blockIdx.x / num_splits, split = blockIdx.x % num_splits;
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv;
  const int q0 = cu_q[b];
  const int n_b = cu_q[b + 1] - q0;
  const int rows = n_b * G;
  if (128 * mt >= rows) return;  // uniform: this tile has no query row
  int kv_len = kv_lens[b];
  const bool bad = n_b < 0 || q0 < 0 || q0 + n_b > total_q || kv_len < n_b ||
                   kv_len > max_kv_len || kv_len > max_pages * kPageTokens;
  const int i_first = (128 * mt) / G;
  const int i_last = min(n_b - 1, (128 * mt + 127) / G);
  const int pos_last = kv_len - n_b + i_last;     // keys 0 .. pos_last are needed
  const int ntiles_all = bad ? 0 : pos_last / kTileTokens + 1;
  // This CTA's key tiles j0 .. j0 + ntiles - 1; every ring and barrier below
  // counts from its first tile.
  const int j0 = (int)((int64_t)split * ntiles_all / num_splits);
  const int ntiles = (int)((int64_t)(split + 1) * ntiles_all / num_splits) - j0;
  // Output rows exist only when the chunk lies inside the total_q rows.
  const bool rows_ok = n_b >= 0 && q0 >= 0 && q0 + n_b <= total_q;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *stages = smem;
  uint8_t *ktiles = smem + kOffK;
  uint8_t *vtiles = smem + kOffV;
  uint32_t *vsc = reinterpret_cast<uint32_t *>(smem + kOffVsc);  // [2][page][group][8]
  int32_t *spages = reinterpret_cast<int32_t *>(smem + kOffPages);
  volatile int *flags = reinterpret_cast<volatile int *>(smem + kOffFlags);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars);
  uint64_t *full = bars, *empty = bars + kStages;
  uint64_t *kready = bars + 2 * kStages, *vready = kready + 2, *sready = kready + 4,
           *pready = kready + 6, *pvdone = kready + 8, *qready = kready + 10,
           *final_bar = kready + 11;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffTmem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (bad && threadIdx.x == 0) report(err, NVKV_DEVERR_LENGTH);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kDeqWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kready[i], kDeqWarps);
      mbar_init(&vready[i], kDeqWarps);
      mbar_init(&sready[i], 1);
      mbar_init(&pready[i], kSmxWarps);
      mbar_init(&pvdone[i], 1);
    }
    mbar_init(qready, kSmxWarps);
    mbar_init(final_bar, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 4) flags[threadIdx.x] = 0;
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int32_t *pt = page_table + (size_t)b * max_pages;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA
    prefetch_tmap(&tmap);
    const int p = lane & 3;
    auto page_for = [&](int j) -> int {
      const int tok = j * kTileTokens + p * kPageTokens;
      if (tok > pos_last) return -1;  // keys past the last query are never needed
      const int pg = pt[tok / kPageTokens];
      if (pg < 0 || pg >= num_pages) {
        if (lane < kTilePages) report(err, NVKV_DEVERR_PAGE_ID);
        return -1;
      }
      return pg;
    };
    int cur = ntiles > 0 ? page_for(j0) : -1;
    for (int j = 0; j < ntiles; ++j) {
      const int stage = j % kStages;
      const int nxt = j + 1 < ntiles ? page_for(j0 + j + 1) : -1;
      if (j >= kStages) {
        if (lane == 0) wait_bar(&empty[stage], ((j / kStages) + 1) & 1, flags, err);
        __syncwarp();
      }
      const bool mine = lane < kTilePages && cur >= 0;
      if (lane < kTilePages) spages[stage * kTilePages + lane] = cur;
      const uint32_t bytes = __popc(__ballot_sync(0xffffffffu, mine)) * kHeadBytes;
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&full[stage], bytes);
      __syncwarp();
      if (mine)
        tma_load_2d(stages + stage * kStageBytes + lane * kPagePitch, &tmap, 0,
                    (cur * Hkv + h) * kRowsPerHead, &full[stage]);
      cur = nxt;
    }
    if (lane == 0) {
      const int first = ntiles > kStages ? ntiles - kStages : 0;
      for (int k = first; k < ntiles; ++k)
        mbar_wait(&full[k % kStages], (k / kStages) & 1, kWaitBudget);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0 && ntiles > 0) {
      const uint32_t idesc_qk = idesc_f16_f32(128, kTileTokens, false, false);
      const uint32_t idesc_pv = idesc_f16_f32(128, kD, false, false);
      const uint32_t kb = smem_u32(ktiles), vb = smem_u32(vtiles);
      wait_bar(qready, 0, flags, err);
      tc_fence_after();
      int qk = 0, pv = 0;
      bool issued = false;
      long long t_last = clock64();
      while (pv < ntiles && !flags[2]) {
        bool progress = false;
        if (pv < qk && mbar_test(&pready[pv & 1], (pv >> 1) & 1) &&
            mbar_test(&vready[pv & 1], (pv >> 1) & 1)) {
          tc_fence_after();
          const uint32_t pcol = tmem + kColS + (pv & 1) * 64;  // P: first 32 columns of the slot
          const uint32_t vt = vb + (pv & 1) * kVTileBytes;
#pragma unroll
          for (int ks = 0; ks < kTileTokens / 16; ++ks) {
            const uint64_t bd = smem_desc(vt + ks * 2 * 4096, 4096, 128);
            mma_f16_ts(tmem + kColO, pcol + ks * 8, bd, idesc_pv, (pv > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&pvdone[pv & 1]);
          ++pv;
          progress = issued = true;
        } else if (qk < ntiles &&
                   (qk < 2 || mbar_test(&pvdone[qk & 1], ((qk >> 1) + 1) & 1)) &&
                   mbar_test(&kready[qk & 1], (qk >> 1) & 1)) {
          tc_fence_after();
          const uint32_t kt = kb + (qk & 1) * kKTileBytes;
          const uint32_t scol = tmem + kColS + (qk & 1) * 64;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t bd = smem_desc(kt + ks * 2 * 1024, 1024, 128);
            mma_f16_ts(scol, tmem + kColQ + ks * 8, bd, idesc_qk, ks > 0 ? 1u : 0u);
          }
          mma_commit(&sready[qk & 1]);
          ++qk;
          progress = issued = true;
        }
        if (progress) {
          t_last = clock64();
        } else {
          if (clock64() - t_last > kWaitBudget) {
            flags[2] = 1;
            report(err, NVKV_DEVERR_TIMEOUT);
          }
          // Nothing was ready: back off briefly so the polling thread does
          // not take issue slots from the warps it is waiting for.
          if (kPollSleepNs > 0) __nanosleep(kPollSleepNs);
        }
      }
      if (issued) {
        mma_commit(final_bar);
        mbar_wait(final_bar, 0, kWaitBudget);
      }
    }
  } else if (warp < kDeqWarps) {
    // ---------------------------------------------------------- dequantise
    const int t = threadIdx.x;  // 0..255
    for (int j = 0; j < ntiles; ++j) {
      const int stage = j % kStages, slot = j & 1;
      const uint8_t *stg = stages + stage * kStageBytes;
      wait_bar(&full[stage], (j / kStages) & 1, flags, err);
      const int4 pg4 = *reinterpret_cast<const int4 *>(spages + stage * kTilePages);
      const int pgs[4] = {pg4.x, pg4.y, pg4.z, pg4.w};
      const int tok0 = (j0 + j) * kTileTokens;
      {
        // This tile's V scales, converted once: thread t takes 4 consecutive
        // tokens of one (page, group); the 16 V^T rows of a group share them.
        // (Absent pages convert stale bytes that are never used.)
        const int p = t >> 6, g = (t >> 2) & 15, q4 = t & 3;
        const int srow = 34 + (g >> 3);
        const uint32_t raw = *reinterpret_cast<const uint32_t *>(
            stg + p * kPagePitch + srow * 128 + (((g & 7) ^ (srow & 7)) << 4) + 4 * q4);
        uint32_t t2[2];
        e4m3x4_to_f16x2x2(raw, t2);
        *reinterpret_cast<uint2 *>(vsc + ((slot * kTilePages + p) * 16 + g) * 8 + 2 * q4) =
            make_uint2(t2[0], t2[1]);
      }
      // K tile slot: its previous tile's QK must be done.
      if (j >= 2) {
        wait_bar(&sready[slot], ((j >> 1) + 1) & 1, flags, err);
        tc_fence_after();
      }
      {
        // thread = token n (32 consecutive per warp), two 32-d chunks
        const int n = t & 63, cp = t >> 6;
        const int p = n >> 4, s = n & 15;
        const bool ok = pgs[p] >= 0 && tok0 + n <= pos_last;
        const uint8_t *pg = stg + p * kPagePitch;
        uint32_t sc = 0;  // scale bytes of groups 4cp .. 4cp+3
        if (ok)
          sc = *reinterpret_cast<const uint32_t *>(pg + (16 + (s >> 3)) * 128 +
                                                   (((s & 7) ^ (s >> 3)) << 4) + 4 * cp);
        uint8_t *kt = ktiles + slot * kKTileBytes + (n >> 3) * 128 + (n & 7) * 16;
#pragma unroll
        for (int ci = 0; ci < 2; ++ci) {
          const int c = 2 * cp + ci;  // 32-d chunk: groups 2c, 2c+1
          uint32_t words[16];
          if (ok) {
            const uint4 w4 =
                *reinterpret_cast<const uint4 *>(pg + s * 128 + ((c ^ (s & 7)) << 4));
            const uint32_t s0 = dup_scale((sc >> (16 * ci)) & 0xffu);
            const uint32_t s1 = dup_scale((sc >> (16 * ci + 8)) & 0xffu);
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
          // K-major core matrices: element (n, k) at (k/8)*1024 + (n/8)*128 + (n%8)*16.
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4 *>(kt + (4 * c + i) * 1024) =
                make_uint4(words[4 * i], words[4 * i + 1], words[4 * i + 2], words[4 * i + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&kready[slot]);
      // The scale table of this tile is complete once every dequantising
      // thread is here; all of them finished reading the table of tile j-2
      // before arriving here for tile j-1.
      named_barrier(1, kDeqWarps * 32);
      // V^T tile slot: its previous tile's PV must be done.
      if (j >= 2) {
        wait_bar(&pvdone[slot], ((j >> 1) + 1) & 1, flags, err);
        tc_fence_after();
      }
      {
        const int d = t;  // head_dim row
        const int g = d >> 4;
        const int vrow = 18 + (d >> 4);
        const int vchunk = ((d & 15) >> 1) ^ (vrow & 7);
        uint8_t *vt = vtiles + slot * kVTileBytes + (d >> 3) * 128 + (d & 7) * 16;
#pragma unroll
        for (int p = 0; p < kTilePages; ++p) {
          const int ptok = tok0 + p * kPageTokens;
          uint32_t o8[8];
          if (pgs[p] >= 0) {
            const uint8_t *pg = stg + p * kPagePitch;
            const uint2 cw =
                *reinterpret_cast<const uint2 *>(pg + vrow * 128 + vchunk * 16 + (d & 1) * 8);
            const uint4 *tb =
                reinterpret_cast<const uint4 *>(vsc + ((slot * kTilePages + p) * 16 + g) * 8);
            const uint4 sa = tb[0], sb = tb[1];
            const uint32_t sp[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
            uint32_t c0[4], c1[4];
            e2m1x8_to_f16x2x4(cw.x, c0);
            e2m1x8_to_f16x2x4(cw.y, c1);
#pragma unroll
            for (int i = 0; i < 8; ++i) o8[i] = hmul2_u32(i < 4 ? c0[i] : c1[i - 4], sp[i]);
            if (ptok + kPageTokens - 1 > pos_last) {  // zero the tokens past the last query
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int t0 = ptok + 2 * i;
                if (t0 > pos_last) o8[i] = 0u;
                else if (t0 + 1 > pos_last) o8[i] &= 0xffffu;
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) o8[i] = 0u;
          }
          // K-major (tokens) core matrices: element (d, t) at (t/8)*4096 + (d/8)*128 + (d%8)*16.
          *reinterpret_cast<uint4 *>(vt + (2 * p) * 4096) = make_uint4(o8[0], o8[1], o8[2], o8[3]);
          *reinterpret_cast<uint4 *>(vt + (2 * p + 1) * 4096) =
              make_uint4(o8[4], o8[5], o8[6], o8[7]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&vready[slot]);
        mbar_arrive(&empty[stage]);
      }
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int lq = warp & 3;
    const int r = 32 * lq + lane;             // query row of the tile
    const uint32_t tl = tmem + ((uint32_t)(32 * lq) << 16);
    const int gr = 128 * mt + r;
    const bool valid = gr < rows && !bad;
    const int i = gr / G, g = gr % G;
    const int pos = kv_len - n_b + i;        // keys 0 .. pos are visible
    // Q row -> Tensor Memory (A operand), f16, pre-scaled to base-2 scores.
    {
      const __nv_bfloat16 *qr = q + ((size_t)(q0 + i) * Hq + h * G + g) * kD;
#pragma unroll
      for (int c32 = 0; c32 < 4; ++c32) {
        uint32_t w[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 raw = make_uint4(0, 0, 0, 0);
          if (valid) raw = *reinterpret_cast<const uint4 *>(qr + c32 * 64 + v * 8);
          const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __half2 hh = __floats2half2_rn(__uint_as_float(rw[e] << 16) * qscale,
                                           __uint_as_float(rw[e] & 0xffff0000u) * qscale);
            w[4 * v + e] = *reinterpret_cast<uint32_t *>(&hh);
          }
        }
        tmem_st16(tl + kColQ + c32 * 32, w);
        tmem_st16(tl + kColQ + c32 * 32 + 16, w + 16);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qready);
    }
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < ntiles; ++j) {
      const int slot = j & 1;
      wait_bar(&sready[slot], (j >> 1) & 1, flags, err);
      __syncwarp();  // the Tensor Memory loads below are warp-collective
      tc_fence_after();
      const uint32_t scol = tl + kColS + slot * 64;
      float x[64];
      {
        uint32_t r0[16], r1[16], r2[16], r3[16];
        tmem_ld16(scol, r0);
        tmem_ld16(scol + 16, r1);
        tmem_ld16(scol + 32, r2);
        tmem_ld16(scol + 48, r3);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          x[e] = __uint_as_float(r0[e]);
          x[16 + e] = __uint_as_float(r1[e]);
          x[32 + e] = __uint_as_float(r2[e]);
          x[48 + e] = __uint_as_float(r3[e]);
        }
      }
      const int key0 = (j0 + j) * kTileTokens;
      float tmax = -INFINITY;
      if (valid && key0 + kTileTokens - 1 <= pos) {
#pragma unroll
        for (int e = 0; e < 64; ++e) tmax = fmaxf(tmax, x[e]);
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          if (!valid || key0 + e > pos) x[e] = -INFINITY;
          tmax = fmaxf(tmax, x[e]);
        }
      }
      // Each row decides on its own whether its running max moves, but the
      // Tensor Memory loads and stores of O are warp-collective: if any row of
      // the warp moves, the whole warp rescales, rows that stay with alpha 1.
      const bool raise = tmax > -INFINITY && (m == -INFINITY || tmax > m + kLazyRescale);
      const float alpha = raise ? exp2f(m - tmax) : 1.f;  // 0 when m = -inf
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
        // O, accumulated up to tile j-1, scales once that tile's PV is done.
        wait_bar(&pvdone[(j - 1) & 1], ((j - 1) >> 1) & 1, flags, err);
        __syncwarp();
        tc_fence_after();
#pragma unroll 1
        for (int c16 = 0; c16 < kD / 16; ++c16) {
          uint32_t rr[16];
          tmem_ld16(tl + kColO + c16 * 16, rr);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
          tmem_st16(tl + kColO + c16 * 16, rr);
        }
        tmem_wait_st();
      }
      if (raise) {
        l *= alpha;
        m = tmax;
      }
      // Weights in f16, two per exponential instruction; masked keys are
      // -inf and give 0 (a row with no visible key yet keeps m = -inf: it
      // subtracts 0 instead).  The denominator sums the same f16 weights.
      const float ms = m == -INFINITY ? 0.f : m;
      uint32_t pw[32];
      float2 lv = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 dd = add_f32x2(make_float2(x[2 * e], x[2 * e + 1]), make_float2(-ms, -ms));
        pw[e] = ex2_f16x2(dd.x, dd.y);
        lv = add_f32x2(lv, f16x2_to_float2(pw[e]));
      }
      l += lv.x + lv.y;
      // P overwrites the first 32 columns of its own S slot (already read).
      tmem_st16(scol, pw);
      tmem_st16(scol + 16, pw + 16);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pready[slot]);
    }
    // Epilogue: O / l -> bf16 out.
    if (ntiles > 0) {
      wait_bar(&pvdone[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, flags, err);
      __syncwarp();
      tc_fence_after();
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const size_t orow_idx = (size_t)(q0 + i) * Hq + h * G + g;
    const bool write = gr < rows && rows_ok;
    // Split partial: O / l (fp32) and lse = m + log2(l), -inf without a
    // visible key, in the split's plane of total_q * Hq rows.
    const size_t plane = (size_t)split * total_q * Hq;
    if (ws_o && write) ws_lse[plane + orow_idx] = l > 0.f ? m + log2f(l) : -INFINITY;
#pragma unroll 1
    for (int c16 = 0; c16 < kD / 16; ++c16) {
      uint32_t rr[16];
      if (ntiles > 0) {
        tmem_ld16(tl + kColO + c16 * 16, rr);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) rr[e] = 0u;
      }
      if (!write) continue;
      if (ws_o) {
        float4 *dst = reinterpret_cast<float4 *>(ws_o + (plane + orow_idx) * kD + c16 * 16);
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4)
          dst[e4] = make_float4(__uint_as_float(rr[4 * e4]) * inv, __uint_as_float(rr[4 * e4 + 1]) * inv,
                                __uint_as_float(rr[4 * e4 + 2]) * inv,
                                __uint_as_float(rr[4 * e4 + 3]) * inv);
      } else {
        uint32_t ow[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(rr[2 * e]) * inv,
                                                    __uint_as_float(rr[2 * e + 1]) * inv);
          ow[e] = *reinterpret_cast<uint32_t *>(&b2);
        }
        __nv_bfloat16 *orow = out + orow_idx * kD;
        *reinterpret_cast<uint4 *>(orow + c16 * 16) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        *reinterpret_cast<uint4 *>(orow + c16 * 16 + 8) = make_uint4(ow[4], ow[5], ow[6], ow[7]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// Merge of the key splits: row (token q0 + i, head hq) of sequence b is
// sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M) with M the largest lse (the
// log-sum-exp combination of partial softmax results; zero when no split saw
// a key).  One warp per row, 8 head_dim elements per lane.
constexpr int kMaxSplits = 8;
constexpr int kMergeWarps = 8;

__global__ void __launch_bounds__(kMergeWarps * 32)
prefill_merge_kernel(const float *__restrict__ ws_o, const float *__restrict__ ws_lse,
                     int num_splits, const int32_t *__restrict__ cu_q, int total_q, int Hq,
                     int G, int row_cap, __nv_bfloat16 *__restrict__ out) {
  const int b = blockIdx.y;
  const int q0 = cu_q[b], n_b = cu_q[b + 1] - q0;
  if (n_b <= 0 || q0 < 0 || q0 + n_b > total_q) return;  // no output rows (as in the attention)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t idx = (int64_t)blockIdx.x * kMergeWarps + warp;  // token idx / Hq, head idx % Hq
  if (idx >= (int64_t)n_b * Hq) return;
  // only the rows the attention grid covers (tile rows i*G + g < row_cap)
  if ((idx / Hq) * G + (idx % Hq) % G >= row_cap) return;
  const size_t row = (size_t)q0 * Hq + idx;
  const size_t plane = (size_t)total_q * Hq;
  float lse[kMaxSplits], mx = -INFINITY;
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) {
    lse[s] = s < num_splits ? ws_lse[s * plane + row] : -INFINITY;
    mx = fmaxf(mx, lse[s]);
  }
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, wsum = 0.f;
  if (mx > -INFINITY) {
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) {
      if (s < num_splits && lse[s] > -INFINITY) {
        const float w = exp2f(lse[s] - mx);
        const float4 *src = reinterpret_cast<const float4 *>(ws_o + (s * plane + row) * kD + 8 * lane);
        const float4 a = src[0], c = src[1];
        acc[0] += w * a.x; acc[1] += w * a.y; acc[2] += w * a.z; acc[3] += w * a.w;
        acc[4] += w * c.x; acc[5] += w * c.y; acc[6] += w * c.z; acc[7] += w * c.w;
        wsum += w;
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint32_t ow[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
    ow[e] = *reinterpret_cast<uint32_t *>(&b2);
  }
  *reinterpret_cast<uint4 *>(out + row * kD + 8 * lane) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
}

}  // namespace

bool prefill_tc_supported(const nvkv_cache &c) { return c.head_dim == kD; }

int prefill_max_splits() { return kMaxSplits; }

// Key splits for a grid of `items` (m-tile, kv-head, sequence) CTAs on `sms`
// SMs (one CTA per SM): the count in 1 .. kMaxSplits whose CTAs fill their
// last wave best, a larger count taken only when it raises the fill by more
// than 1 % (each split writes and merges a partial result of its rows).  The
// 384 CTAs of a 2048-token chunk at 24/4 heads fill 2.59 of 3 waves; 5
// splits fill 12.97 of 13.
int prefill_auto_splits(int64_t items, int sms) {
  if (items <= 0 || sms <= 0) return 1;
  auto fill = [&](int k) {
    const int64_t n = items * k;
    return (double)n / (double)(((n + sms - 1) / sms) * sms);
  };
  int best = 1;
  for (int k = 2; k <= kMaxSplits; ++k)
    if (fill(k) > fill(best) + 0.01) best = k;
  return best;
}

int prefill_tc_items(const nvkv_cache &c, const nvkv_seqs &s, int max_q, int Hq) {
  const int G = Hq / c.num_kv_heads;
  return (int)(((int64_t)max_q * G + 127) / 128) * c.num_kv_heads * s.batch;
}

cudaError_t launch_prefill_tc(const nvkv_cache &c, const nvkv_seqs &s, const void *q,
                              const int32_t *cu_q, int total_q, int max_q, int Hq,
                              float sm_scale, void *out, int num_splits, float *ws_o,
                              float *ws_lse, cudaStream_t stream) {
  CUtensorMap map;
  if (!make_pool_tmap(c, &map)) return cudaErrorNotSupported;
  if (num_splits < 1 || num_splits > kMaxSplits || (num_splits > 1 && (!ws_o || !ws_lse)))
    return cudaErrorInvalidValue;
  const int G = Hq / c.num_kv_heads;
  const int mtiles = (max_q * G + 127) / 128;
  cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(mtiles * num_splits), (unsigned)c.num_kv_heads, (unsigned)s.batch);
  prefill_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(
      map, c.num_pages, c.num_kv_heads, s.page_table, s.max_pages_per_seq, s.kv_lens,
      s.max_kv_len, static_cast<const __nv_bfloat16 *>(q), cu_q, total_q, Hq,
      sm_scale * 1.4426950408889634f, static_cast<__nv_bfloat16 *>(out), num_splits,
      num_splits > 1 ? ws_o : nullptr, ws_lse, s.err_word);
  if ((e = cudaGetLastError()) != cudaSuccess || num_splits == 1) return e;
  const dim3 mgrid((unsigned)(((int64_t)max_q * Hq + kMergeWarps - 1) / kMergeWarps),
                   (unsigned)s.batch);
  prefill_merge_kernel<<<mgrid, kMergeWarps * 32, 0, stream>>>(
      ws_o, ws_lse, num_splits, cu_q, total_q, Hq, G, 128 * mtiles,
      static_cast<__nv_bfloat16 *>(out));
  return cudaGetLastError();
}

}  // namespace nvkv
