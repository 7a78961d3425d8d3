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
//    128 B) into a 4-stage shared-memory ring with one 2-D tiled load per
//    page (128-byte swizzle: the dequantising reads are bank-conflict free).
//    No multicast.  (3 stages at N = 48, where the two Q tiles need room.)
//  * Swap-AB: the dequantised K tile (128 tokens x 256 d, f16) and V^T tile
//    (2 x 128 d x 128 tokens) are the A operands, written straight from
//    registers into Tensor Memory; the G*T query rows (Q, then P) are the
//    small N side of the MMA, in shared memory; q enters as two f16 terms
//    (hi, and the fp32 remainder lo), both multiplied by the same K tile
//    into the same S^T.  S^T and O^T accumulate in Tensor Memory in fp32;
//    the weights p = 2^(x - m) come from an fp32 exp2 rounded to f16, and
//    each softmax thread keeps per-row partial sums of the same f16 P the
//    value sums use, reduced once per segment.
//    Dequantisation is exact in f16 (E2M1 x E4M3 has at most 6 significant
//    bits).
//  * 16 dequantising warps (4 per SM sub-partition): each converts a quarter
//    of the K tile (one token per thread, 32 d per QK phase) and of the V^T
//    tile (one d row per thread, 64 tokens).  4 dedicated softmax warps run
//    the softmax on S^T (one token per thread): the running max of a row is only
//    raised when a score exceeds it by more than 2^8, which one warp vote per
//    row detects; the full cross-lane max (and the rescale of O^T and of the
//    denominator) runs only then -- on the first unit of a segment and rarely
//    after.  One thread issues the MMAs.
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
constexpr int kWorkerWarps = 16;      // dequantising warps 0..15
constexpr int kSoftmaxWarps = 4;      // softmax warps 16..19
constexpr int kSoftmaxWarp0 = 16;
constexpr int kProducerWarp = 20;
constexpr int kMmaWarp = 21;
constexpr int kThreads = 22 * 32;
constexpr int kSegThreads = (kWorkerWarps + kSoftmaxWarps) * 32;  // segment-end barrier
constexpr uint32_t kTmemCols = 512;
constexpr long long kWaitBudget = 2000000000LL;  // clock cycles (~1 s)
constexpr float kLazyRescale = 8.0f;             // log2 units

// Tensor Memory columns.  The K tile is dequantised in two head_dim halves
// (64 columns each, one QK phase per half); the V^T tile, S^T and the P^T tile
// are double-buffered by unit parity, so the QK of unit u+1 and the
// dequantisation of unit u+1 overlap the softmax and PV of unit u.  When
// N <= 32 the two K halves also get their own columns, so the first half of
// unit u+1 only waits for the first QK phase of unit u.
constexpr uint32_t kColK = 0;      // K half of phase A (and B when N > 32)

template <int N>
struct Cfg {
  // Stage ring depth: 3 at N = 48, where the two f16 Q tiles take the room.
  static constexpr int kStages = N > 32 ? 3 : 4;
  static constexpr bool kSplitK = N <= 32;
  static constexpr uint32_t kColKB = kSplitK ? 64 : 0;       // K half of phase B
  static constexpr uint32_t kColV = kSplitK ? 128 : 64;      // 2 slots x 128: V^T
  static constexpr uint32_t kColS = kColV + 256;             // 2 slots x N: S^T
  static constexpr uint32_t kColO = kColS + 2 * N;           // O^T half hf at kColO + hf*N
  static_assert(N % 16 == 0 && N >= 16 && N <= 48 && kColO + 2 * N <= kTmemCols, "N");
  static constexpr int kMaskWords = (N + 31) / 32;
  static constexpr int kQBytes = N * kD * 2;        // Q tile, K-major, no swizzle
  static constexpr int kPBytes = N * 128 * 2;       // one P^T tile, MN-major, no swizzle
  static constexpr int kOffQ = kStages * kStageBytes;
  static constexpr int kOffQlo = kOffQ + kQBytes;               // low f16 term of the Q tile
  static constexpr int kOffP = kOffQlo + kQBytes;               // 2 P^T tiles
  static constexpr int kOffRed = kOffP + 2 * kPBytes;           // float [4][N]
  static constexpr int kOffMask = kOffRed + kSoftmaxWarps * N * 4;  // u32 [2][4][4]
  static constexpr int kOffM = kOffMask + 2 * kSoftmaxWarps * 4 * 4;
  static constexpr int kOffAlpha = kOffM + N * 4;
  static constexpr int kOffNvis = kOffAlpha + N * 4;
  static constexpr int kOffFlags = kOffNvis + N * 4;            // int[4]: abort at [2]
  static constexpr int kOffPages = kOffFlags + 16;              // int[stages][8]
  static constexpr int kOffBars = kOffPages + kStages * kUnitPages * 4;
  static constexpr int kNumBars = 2 * kStages + 12;
  static constexpr int kOffTmem = kOffBars + kNumBars * 8;
  static constexpr int kSmemBytes = kOffTmem + 16 + 1024;      // + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert(kOffQ % 1024 == 0 && kOffP % 16 == 0 && kPBytes % 16 == 0 &&
                kOffPages % 16 == 0 && kOffBars % 8 == 0, "alignment");
};

struct Shared {
  uint8_t *stages, *qtile, *qtile_lo, *ptile;
  float *red, *m_s, *alpha_s;
  int32_t *nvis_s, *pages;
  uint32_t *masks;
  volatile int *flags;
  // sready, pready, vready and pvdone exist once per S^T / P^T / V^T slot:
  // slot s completes once per unit with (unit & 1) == s, so no wait is ever
  // more than one phase behind (a parity wait cannot tell phases two apart).
  uint64_t *full, *empty, *kready_a, *kdone_a, *kready_b, *sready, *pready, *vready, *pvdone,
      *final_bar;
  uint32_t *tmem_slot;
};

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *flags,
                                         int32_t *err) {
  return guarded_wait(bar, parity, flags + 2, err, kWaitBudget);  // flags[2]: abort
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

__device__ __forceinline__ uint32_t dup_scale(uint32_t byte) {
  return e4m3x2_to_f16x2(byte | (byte << 8));
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmap, int num_pages, int Hkv,
                 const int32_t *__restrict__ page_table, int max_pages,
                 const int32_t *__restrict__ kv_lens, int B, int max_kv_len,
                 const __nv_bfloat16 *__restrict__ q, int T, int t0, int T_all, int Hq,
                 float qscale, int S,
                 float *__restrict__ ws_o, float *__restrict__ ws_lse, int32_t *err) {
  using C = Cfg<N>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Shared sh;
  sh.stages = smem;
  sh.qtile = smem + C::kOffQ;
  sh.qtile_lo = smem + C::kOffQlo;
  sh.ptile = smem + C::kOffP;
  sh.red = reinterpret_cast<float *>(smem + C::kOffRed);
  sh.masks = reinterpret_cast<uint32_t *>(smem + C::kOffMask);
  sh.m_s = reinterpret_cast<float *>(smem + C::kOffM);
  sh.alpha_s = reinterpret_cast<float *>(smem + C::kOffAlpha);
  sh.nvis_s = reinterpret_cast<int32_t *>(smem + C::kOffNvis);
  sh.flags = reinterpret_cast<volatile int *>(smem + C::kOffFlags);
  sh.pages = reinterpret_cast<int32_t *>(smem + C::kOffPages);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBars);
  sh.full = bars;
  sh.empty = bars + kStages;
  sh.kready_a = bars + 2 * kStages;
  sh.kdone_a = sh.kready_a + 1;
  sh.kready_b = sh.kready_a + 2;
  sh.sready = sh.kready_a + 3;  // [2]
  sh.pready = sh.kready_a + 5;  // [2]
  sh.vready = sh.kready_a + 7;  // [2]
  sh.pvdone = sh.kready_a + 9;  // [2]
  sh.final_bar = sh.kready_a + 11;
  sh.tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = Hq / Hkv;
  // This launch takes queries t0 .. t0+T-1 of the step's T_all (rows
  // n < R = T*G of the chunk are rows t0*G + n of the step's R_all).
  const int R = T * G;
  const int R_all = T_all * G;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], kWorkerWarps);
    }
    mbar_init(sh.kready_a, kWorkerWarps);
    mbar_init(sh.kdone_a, 1);
    mbar_init(sh.kready_b, kWorkerWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.sready[i], 1);
      mbar_init(&sh.pready[i], kSoftmaxWarps);
    }
    mbar_init(&sh.vready[0], kWorkerWarps);
    mbar_init(&sh.vready[1], kWorkerWarps);
    mbar_init(&sh.pvdone[0], 1);
    mbar_init(&sh.pvdone[1], 1);
    mbar_init(sh.final_bar, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 4) sh.flags[threadIdx.x] = 0;
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
    // The whole warp produces: lane p < 8 owns page p of a unit.  The page
    // ids of unit u+1 are loaded while unit u's copies are issued, so the
    // page-table latency is off the critical path.
    prefetch_tmap(&tmap);
    const int p = lane & 7;
    int64_t u = u0;
    Seg sg = segment_at(u, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
    auto page_for = [&](const Seg &g, int64_t uu) -> int {
      const int tok = (int)(uu - g.pair_start) * kUnitTokens + p * kPageTokens;
      const int32_t *pt = page_table + (size_t)g.b * max_pages;
      const int pg = page_of(pt, tok, g.kv_len, num_pages);
      if (lane < kUnitPages && tok < g.kv_len && pg < 0) report(err, NVKV_DEVERR_PAGE_ID);
      return pg;
    };
    int cur = u < u1 ? page_for(sg, u) : -1;
    uint32_t uc = 0;
    for (; u < u1; ++u, ++uc) {
      const int stage = uc % kStages;
      // Next unit's page id (possibly in the next segment).
      int nxt = -1;
      Seg nsg = sg;
      if (u + 1 < u1) {
        if (u + 1 >= sg.seg_end) nsg = segment_at(u + 1, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
        nxt = page_for(nsg, u + 1);
      }
      if (uc >= (uint32_t)kStages) {
        if (lane == 0) wait_bar(&sh.empty[stage], ((uc / kStages) + 1) & 1, sh.flags, err);
        __syncwarp();
      }
      const bool mine = lane < kUnitPages && cur >= 0;
      if (lane < kUnitPages) sh.pages[stage * kUnitPages + lane] = cur;
      const uint32_t bytes = __popc(__ballot_sync(0xffffffffu, mine)) * kHeadBytes;
      __syncwarp();
      // The arrive releases the page ids to the workers that wait on it.
      if (lane == 0) mbar_arrive_expect_tx(&sh.full[stage], bytes);
      __syncwarp();
      if (mine)
        tma_load_2d(sh.stages + stage * kStageBytes + lane * kPagePitch, &tmap, 0,
                    (cur * Hkv + sg.h) * kRowsPerHead, &sh.full[stage]);
      cur = nxt;
      sg = nsg;
    }
    // Drain: every issued copy must land before the CTA may exit.
    if (lane == 0) {
      const uint32_t first = uc > (uint32_t)kStages ? uc - kStages : 0;
      for (uint32_t k = first; k < uc; ++k)
        mbar_wait(&sh.full[k % kStages], (k / kStages) & 1, kWaitBudget);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA
    // Event driven: the issuing thread polls the ready barriers without
    // blocking and issues whichever step is ready, the oldest PV first (it
    // frees a V^T and a P^T slot).  Unit qk's QK needs its S^T slot, last read
    // by the softmax of unit qk-2, so it waits until that unit's PV (issued
    // after the softmax's arrival) has been issued.  Segment boundaries need
    // no special case: the workers load a new pair's queries only after its
    // previous pair's last PV completed.
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_f16_f32(128, N, false, false);
      const uint32_t idesc_pv = idesc_f16_f32(128, N, false, true);
      const uint32_t qb = smem_u32(sh.qtile), pb = smem_u32(sh.ptile);
      const uint32_t qlb = smem_u32(sh.qtile_lo);
      const uint32_t n_units = (uint32_t)(u1 - u0);
      uint32_t qk = 0, pv = 0;
      int qk_phase = 0;
      uint32_t first_bits = 0;  // bit (unit & 31): unit starts its segment
      int64_t u = u0;
      Seg sg = segment_at(u, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
      int64_t seg_start = u;
      bool issued = false;
      long long t_last = clock64();
      while (pv < n_units && !sh.flags[2]) {
        bool progress = false;
        if (pv < qk && mbar_test(&sh.vready[pv & 1], (pv >> 1) & 1) &&
            mbar_test(&sh.pready[pv & 1], (pv >> 1) & 1)) {
          tc_fence_after();
          const bool first = (first_bits >> (pv & 31)) & 1u;
          const uint32_t pslot = pb + (pv & 1) * C::kPBytes;
          const uint32_t vslot = tmem + C::kColV + (pv & 1) * 128;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t bd = smem_desc(pslot + ks * 256, 128, 2048);
            const uint32_t acc = (!first) || ks > 0;
            mma_f16_ts(tmem + C::kColO, vslot + ks * 8, bd, idesc_pv, acc);
            mma_f16_ts(tmem + C::kColO + N, vslot + 64 + ks * 8, bd, idesc_pv, acc);
          }
          mma_commit(&sh.pvdone[pv & 1]);
          ++pv;
          progress = issued = true;
        } else if (qk_phase == 0 && qk < n_units && qk < pv + 2 &&
                   mbar_test(sh.kready_a, qk & 1)) {
          tc_fence_after();
          if (u >= sg.seg_end) {
            sg = segment_at(u, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
            seg_start = u;
          }
          if (u == seg_start) first_bits |= 1u << (qk & 31);
          else first_bits &= ~(1u << (qk & 31));
          const uint32_t sslot = tmem + C::kColS + (qk & 1) * N;
          // the high f16 terms of q, then the low ones, into the same S^T
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t bd = smem_desc(qb + ks * 2 * (N * 16), N * 16, 128);
            mma_f16_ts(sslot, tmem + kColK + ks * 8, bd, idesc_qk, ks > 0);
          }
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t bd = smem_desc(qlb + ks * 2 * (N * 16), N * 16, 128);
            mma_f16_ts(sslot, tmem + kColK + ks * 8, bd, idesc_qk, 1u);
          }
          mma_commit(sh.kdone_a);
          qk_phase = 1;
          progress = issued = true;
        } else if (qk_phase == 1 && mbar_test(sh.kready_b, qk & 1)) {
          tc_fence_after();
          const uint32_t sslot = tmem + C::kColS + (qk & 1) * N;
#pragma unroll
          for (int ks = 8; ks < 16; ++ks) {
            const uint64_t bd = smem_desc(qb + ks * 2 * (N * 16), N * 16, 128);
            mma_f16_ts(sslot, tmem + C::kColKB + (ks - 8) * 8, bd, idesc_qk, 1u);
          }
#pragma unroll
          for (int ks = 8; ks < 16; ++ks) {
            const uint64_t bd = smem_desc(qlb + ks * 2 * (N * 16), N * 16, 128);
            mma_f16_ts(sslot, tmem + C::kColKB + (ks - 8) * 8, bd, idesc_qk, 1u);
          }
          mma_commit(&sh.sready[qk & 1]);
          qk_phase = 0;
          ++qk;
          ++u;
          progress = true;
        }
        if (progress) {
          t_last = clock64();
        } else if (clock64() - t_last > kWaitBudget) {
          sh.flags[2] = 1;
          report(err, NVKV_DEVERR_TIMEOUT);
        }
      }
      if (issued) {
        mma_commit(sh.final_bar);
        mbar_wait(sh.final_bar, 0, kWaitBudget);
      }
    }
  } else {
    // -------------------------------------------------------------- workers
    const bool smx = warp >= kSoftmaxWarp0;                    // softmax warps 16..19
    const int lq = warp & 3, sub = smx ? 0 : warp >> 2;
    const uint32_t tl = tmem + ((uint32_t)(32 * lq) << 16);  // this warp's lane quarter
    const int tid = smx ? threadIdx.x - kSoftmaxWarp0 * 32 : threadIdx.x;  // 0..127 / 0..511
    // Per-token partial softmax denominators (softmax threads): the sums of
    // the same f16 weights the PV MMAs use.
    float l_part[N];
#pragma unroll
    for (int i = 0; i < N; ++i) l_part[i] = 0.f;

    uint32_t uc = 0;
    for (int64_t u = u0; u < u1;) {
      const Seg sg = segment_at(u, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
      if (sg.bad && tid == 0) report(err, NVKV_DEVERR_LENGTH);
      const int64_t seg_start = u;
      const size_t slot = (size_t)c + (size_t)sg.b * Hkv + sg.h;

      // Q tiles of this pair: rows n < R are (t, g) = (n / G, n % G), pre-scaled
      // to base-2 scores (fp32) and written as two f16 terms, hi = f16(x) and
      // lo = f16(x - hi) (the difference is exact in fp32), which carry
      // about 22 significant bits between them; K-major core-matrix layout;
      // rows >= R are zero.  The score MMAs run over both tiles into the
      // same S^T.  (The previous segment's QK MMAs completed: every worker
      // waited for its last PV, which follows them.)
      for (int ci = smx ? N * (kD / 8) : tid; ci < N * (kD / 8); ci += kWorkerWarps * 32) {
        const int n = ci / (kD / 8), k8 = ci % (kD / 8);
        uint4 v = make_uint4(0, 0, 0, 0), vl = make_uint4(0, 0, 0, 0);
        if (n < R) {
          const int t = n / G, g = n % G;
          const uint4 raw = *reinterpret_cast<const uint4 *>(
              q + ((size_t)(sg.b * T_all + t0 + t) * Hq + sg.h * G + g) * kD + k8 * 8);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t o[4], ol[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // element 2i in the low half, 2i+1 in the high half
            const float x0 = __uint_as_float(w[i] << 16) * qscale;
            const float x1 = __uint_as_float(w[i] & 0xffff0000u) * qscale;
            const __half2 hh = __floats2half2_rn(x0, x1);
            const float2 hf = __half22float2(hh);
            const __half2 ll = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
            o[i] = *reinterpret_cast<const uint32_t *>(&hh);
            ol[i] = *reinterpret_cast<const uint32_t *>(&ll);
          }
          v = make_uint4(o[0], o[1], o[2], o[3]);
          vl = make_uint4(ol[0], ol[1], ol[2], ol[3]);
        }
        const int qoff = k8 * (N * 16) + (n >> 3) * 128 + (n & 7) * 16;
        *reinterpret_cast<uint4 *>(sh.qtile + qoff) = v;
        *reinterpret_cast<uint4 *>(sh.qtile_lo + qoff) = vl;
      }
      fence_proxy_async_smem();
      if (smx) {
        if (tid < N) {
          // Keys visible to score row n (query t0 + n / G of the step, at
          // position kv_len - T_all + t0 + n / G).
          sh.nvis_s[tid] = tid < R ? sg.kv_len - T_all + t0 + tid / G + 1 : 0;
          sh.m_s[tid] = -INFINITY;
        }
#pragma unroll
        for (int i = 0; i < N; ++i) l_part[i] = 0.f;
        named_barrier(1, kSoftmaxWarps * 32);
      }

      for (; u < sg.seg_end; ++u, ++uc) {
        const bool first = (u == seg_start);
        const int stage = uc % kStages;
        const uint8_t *stg = sh.stages + stage * kStageBytes;
        const int tok0 = (int)(u - sg.pair_start) * kUnitTokens;
        if (!smx) {
          wait_bar(&sh.full[stage], (uc / kStages) & 1, sh.flags, err);
          const int4 pa = *reinterpret_cast<const int4 *>(sh.pages + stage * kUnitPages);
          const int4 pb4 = *reinterpret_cast<const int4 *>(sh.pages + stage * kUnitPages + 4);
          const bool full_unit = tok0 + kUnitTokens <= sg.kv_len &&
                                 min(min(min(pa.x, pa.y), min(pa.z, pa.w)),
                                     min(min(pb4.x, pb4.y), min(pb4.z, pb4.w))) >= 0;

          // K tile half (phase 0: d 0..127, phase 1: d 128..255): thread = token
          // jl, one 16-byte chunk (32 d, two scale groups) per warp.
          const int jl = 32 * lq + lane;
          const int kp = jl >> 4, kslot = jl & 15;
          const bool kok = full_unit ||
                           (sh.pages[stage * kUnitPages + kp] >= 0 && tok0 + jl < sg.kv_len);
          const uint8_t *kpg = stg + kp * kPagePitch;
          // Scale bytes of the chunk's two groups: 2*sub, 2*sub+1 (phase 0) and
          // 8 + 2*sub, 8 + 2*sub + 1 (phase 1); 2-byte loads at 2-byte offsets.
          uint32_t ksc = 0, ksc1 = 0;
          if (kok) {
            const uint8_t *sp = kpg + (16 + (kslot >> 3)) * 128 + (((kslot & 7) ^ (kslot >> 3)) << 4);
            ksc = *reinterpret_cast<const uint16_t *>(sp + 2 * sub);
            ksc1 = *reinterpret_cast<const uint16_t *>(sp + 8 + 2 * sub);
          }
          auto k_half = [&](int phase) {
            const int cch = 4 * phase + sub;  // chunk = 32 d = groups 2cch, 2cch+1
            const uint32_t scw = phase ? ksc1 : ksc;
            uint32_t words[16];
            if (kok) {
              const uint4 w4 = *reinterpret_cast<const uint4 *>(kpg + kslot * 128 +
                                                                ((cch ^ (kslot & 7)) << 4));
              const uint32_t s0 = dup_scale(scw & 0xffu);
              const uint32_t s1 = dup_scale((scw >> 8) & 0xffu);
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
            tmem_st16(tl + (phase ? C::kColKB : kColK) + 16 * sub, words);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
          };

          // A K half may only be rewritten once the QK phase reading it has
          // completed: phase A of unit uc-1 (split halves) or phase B of uc-1.
          if (uc > 0) {
            if (C::kSplitK)
              wait_bar(sh.kdone_a, (uc - 1) & 1, sh.flags, err);
            else
              wait_bar(&sh.sready[(uc - 1) & 1], ((uc - 1) >> 1) & 1, sh.flags, err);
            tc_fence_after();
          }
          k_half(0);
          if (lane == 0) mbar_arrive(sh.kready_a);

          // ---- V^T tile into slot uc&1: thread = head_dim row d, 4 pages ----
          // The slot was last read by the PV of unit uc-2.
          if (uc > 1) {
            wait_bar(&sh.pvdone[uc & 1], ((uc >> 1) + 1) & 1, sh.flags, err);  // PV of uc-2
            tc_fence_after();
          }
          {
            const int hv = sub & 1;
            const int d = 128 * hv + 32 * lq + lane;
            const int g = d >> 4;
            const int vrow = 18 + (d >> 4);
            const int vchunk = ((d & 15) >> 1) ^ (vrow & 7);
            const int srow = 34 + (g >> 3);
            const int schunk = (g & 7) ^ (srow & 7);
            const uint32_t vcol = C::kColV + (uc & 1) * 128 + 64 * hv;
  #pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
              const int p = 4 * (sub >> 1) + pp;
              const int ptok = tok0 + p * kPageTokens;
              uint32_t o8[8];
              if (full_unit || sh.pages[stage * kUnitPages + p] >= 0) {
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
              tmem_st8(tl + vcol + 8 * p, o8);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.vready[uc & 1]);
          }

          // Second K half, once phase A's MMAs are done with the first.
          if (C::kSplitK) {
            if (uc > 0) wait_bar(&sh.sready[(uc - 1) & 1], ((uc - 1) >> 1) & 1, sh.flags, err);
          } else {
            wait_bar(sh.kdone_a, uc & 1, sh.flags, err);
          }
          tc_fence_after();
          k_half(1);
          if (lane == 0) {
            mbar_arrive(sh.kready_b);
            mbar_arrive(&sh.empty[stage]);  // every read of the stage is done
          }
        }
        if (smx) {
          // ---- softmax on S^T slot uc&1: thread = token tok0 + 32*lq + lane ----
          wait_bar(&sh.sready[uc & 1], (uc >> 1) & 1, sh.flags, err);
          tc_fence_after();
          const int pos = tok0 + 32 * lq + lane;
          const bool vis_all = tok0 + kUnitTokens <= sg.kv_len - T_all + t0 + 1;
          const uint32_t sslot = tl + C::kColS + (uc & 1) * N;
          uint32_t *my_mask = sh.masks + ((uc & 1) * kSoftmaxWarps + lq) * 4;
          // Scores of one 16-row chunk, masked: invisible keys and padding
          // rows (n >= R) become -inf.  Branch-free over the 16 rows.
          auto load_chunk = [&](int c16, float (&x)[16]) {
            uint32_t r[16];
            tmem_ld16(sslot + 16 * c16, r);
            tmem_wait_ld();
            int nv[16];
            if (vis_all) {
#pragma unroll
              for (int j = 0; j < 16; ++j) nv[j] = 16 * c16 + j < R ? 0x7fffffff : 0;
            } else {
#pragma unroll
              for (int j4 = 0; j4 < 4; ++j4) {
                const int4 v = *reinterpret_cast<const int4 *>(sh.nvis_s + 16 * c16 + 4 * j4);
                nv[4 * j4] = v.x; nv[4 * j4 + 1] = v.y; nv[4 * j4 + 2] = v.z; nv[4 * j4 + 3] = v.w;
              }
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) x[j] = pos < nv[j] ? __uint_as_float(r[j]) : -INFINITY;
          };
          auto load_m = [&](int c16, float (&m)[16]) {
#pragma unroll
            for (int j4 = 0; j4 < 4; ++j4) {
              const float4 v = *reinterpret_cast<const float4 *>(sh.m_s + 16 * c16 + 4 * j4);
              m[4 * j4] = v.x; m[4 * j4 + 1] = v.y; m[4 * j4 + 2] = v.z; m[4 * j4 + 3] = v.w;
            }
          };
          // One pass: weights against the current running max, kept in
          // registers while the 4 softmax warps agree whether any score rose
          // more than 2^8 above its row's running max (then the max is raised,
          // the accumulators are rescaled and the weights recomputed).
          uint32_t h2[N / 2];
          bool up = false;
#pragma unroll
          for (int c16 = 0; c16 < N / 16; ++c16) {
            if (16 * c16 < R) {
              float x[16], m[16];
              load_chunk(c16, x);
              load_m(c16, m);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float2 dd = add_f32x2(make_float2(x[2 * e], x[2 * e + 1]),
                                            make_float2(-m[2 * e], -m[2 * e + 1]));
                up |= (dd.x > kLazyRescale) | (dd.y > kLazyRescale);
                h2[8 * c16 + e] = ex2_f32_to_f16x2(dd.x, dd.y);  // 2^-inf = 0
              }
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) h2[8 * c16 + e] = 0u;
            }
          }
          const uint32_t wup = __ballot_sync(0xffffffffu, up);
          if (lane == 0) my_mask[0] = wup;
          named_barrier(1, kSoftmaxWarps * 32);
          uint32_t any = 0;
#pragma unroll
          for (int w = 0; w < kSoftmaxWarps; ++w) any |= sh.masks[((uc & 1) * kSoftmaxWarps + w) * 4];
          if (any) {
            // Slow path (the first unit of a segment and rare max raises):
            // exact row maxima, new running max, rescale factor of everything
            // accumulated against the old max, weights recomputed.
#pragma unroll
            for (int c16 = 0; c16 < N / 16; ++c16) {
              if (16 * c16 < R) {
                float x[16];
                load_chunk(c16, x);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  const float wm = warp_max(x[j]);
                  if (lane == 0) sh.red[lq * N + 16 * c16 + j] = wm;
                }
              }
            }
            named_barrier(1, kSoftmaxWarps * 32);
            if (tid < N) {
              const int n = tid;
              float alpha = 1.f;
              if (n < R) {
                float tmax = -INFINITY;
#pragma unroll
                for (int w = 0; w < kSoftmaxWarps; ++w) tmax = fmaxf(tmax, sh.red[w * N + n]);
                const float m_old = sh.m_s[n];
                if (tmax > -INFINITY && (m_old == -INFINITY || tmax > m_old + kLazyRescale)) {
                  alpha = exp2f(m_old - tmax);  // 0 when the old max was -inf
                  sh.m_s[n] = tmax;
                }
              }
              sh.alpha_s[n] = alpha;
            }
            named_barrier(1, kSoftmaxWarps * 32);
#pragma unroll
            for (int n = 0; n < N; ++n) l_part[n] *= sh.alpha_s[n];
            if (!first) {
              // O^T rows d = 32*lq + lane and d + 128, accumulated up to the
              // previous unit, scale by alpha once that unit's PV has finished.
              wait_bar(&sh.pvdone[(uc - 1) & 1], ((uc - 1) >> 1) & 1, sh.flags, err);
              tc_fence_after();
#pragma unroll
              for (int reg = 0; reg < 2; ++reg) {
                const uint32_t base = C::kColO + reg * N;
#pragma unroll
                for (int j8 = 0; j8 < N / 8; ++j8) {
                  uint32_t r[8];
                  tmem_ld8(tl + base + j8 * 8, r);
                  tmem_wait_ld();
#pragma unroll
                  for (int j = 0; j < 8; ++j)
                    r[j] = __float_as_uint(__uint_as_float(r[j]) * sh.alpha_s[j8 * 8 + j]);
                  tmem_st8(tl + base + j8 * 8, r);
                }
              }
              tmem_wait_st();
            }
#pragma unroll
            for (int c16 = 0; c16 < N / 16; ++c16) {
              if (16 * c16 < R) {
                float x[16], m[16];
                load_chunk(c16, x);
                load_m(c16, m);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const float2 dd = add_f32x2(make_float2(x[2 * e], x[2 * e + 1]),
                                              make_float2(-m[2 * e], -m[2 * e + 1]));
                  h2[8 * c16 + e] = ex2_f32_to_f16x2(dd.x, dd.y);
                }
              }
            }
          }
          // P^T into slot uc&1 (MN-major): element (n, k) at
          // (n/8)*2048 + (k/8)*128 + (k%8)*16 + (n%8)*2; masked rows are 0.
          // The slot was last read by the PV of unit uc-2.
          if (uc > 1) {
            wait_bar(&sh.pvdone[uc & 1], ((uc >> 1) + 1) & 1, sh.flags, err);
            tc_fence_after();
          }
          const int k = 32 * lq + lane;
          uint8_t *ptile = sh.ptile + (uc & 1) * C::kPBytes;
#pragma unroll
          for (int c16 = 0; c16 < N / 16; ++c16) {
            uint8_t *dst = ptile + (2 * c16) * 2048 + (k >> 3) * 128 + (k & 7) * 16;
            *reinterpret_cast<uint4 *>(dst) =
                make_uint4(h2[8 * c16], h2[8 * c16 + 1], h2[8 * c16 + 2], h2[8 * c16 + 3]);
            *reinterpret_cast<uint4 *>(dst + 2048) =
                make_uint4(h2[8 * c16 + 4], h2[8 * c16 + 5], h2[8 * c16 + 6], h2[8 * c16 + 7]);
            // the denominator sums the same f16 weights the PV uses
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 lp = add_f32x2(
                  make_float2(l_part[16 * c16 + 2 * e], l_part[16 * c16 + 2 * e + 1]),
                  f16x2_to_float2(h2[8 * c16 + e]));
              l_part[16 * c16 + 2 * e] = lp.x;
              l_part[16 * c16 + 2 * e + 1] = lp.y;
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.pready[uc & 1]);
        }
      }

      // ---- end of segment: O^T / l -> workspace, lse ----
      if (uc > 0) {
        wait_bar(&sh.pvdone[(uc - 1) & 1], ((uc - 1) >> 1) & 1, sh.flags, err);  // last PV
        tc_fence_after();
      }
      {
        // Denominators from the softmax threads' partial sums -> sh.alpha_s.
        if (smx) {
#pragma unroll
          for (int n = 0; n < N; ++n) {
            const float ls = warp_sum(l_part[n]);
            if (lane == 0) sh.red[lq * N + n] = ls;
          }
        }
        named_barrier(2, kSegThreads);
        if (smx && tid < N) {
          float l = 0.f;
#pragma unroll
          for (int w = 0; w < kSoftmaxWarps; ++w) l += sh.red[w * N + tid];
          sh.alpha_s[tid] = l;
        }
        named_barrier(2, kSegThreads);
      }
      if (!smx) {
        const int hv = sub & 1, cb = (sub >> 1) * (N / 2);  // O half, first column
        const int d = 128 * hv + 32 * lq + lane;
#pragma unroll
        for (int j8 = 0; j8 < N / 16; ++j8) {
          uint32_t o[8];
          tmem_ld8(tl + C::kColO + hv * N + cb + j8 * 8, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int n = cb + j8 * 8 + j;
            if (n < R) {
              const float lv = sh.alpha_s[n];
              ws_o[(slot * R_all + t0 * G + n) * kD + d] = lv > 0.f ? __uint_as_float(o[j]) / lv : 0.f;
              if (d == 0)
                ws_lse[slot * R_all + t0 * G + n] = lv > 0.f ? sh.m_s[n] + log2f(lv) : -INFINITY;
            }
          }
        }
      }
      tc_fence_before();
      named_barrier(2, kSegThreads);
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
                     const void *q, int T, int t0, int T_all, int Hq, float qscale, int S,
                     float *ws_o, float *ws_lse, cudaStream_t stream) {
  const int smem = Cfg<N>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<N>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  decode_tc_kernel<N><<<S, kThreads, smem, stream>>>(
      map, c.num_pages, c.num_kv_heads, s.page_table, s.max_pages_per_seq, s.kv_lens, s.batch,
      s.max_kv_len, static_cast<const __nv_bfloat16 *>(q), T, t0, T_all, Hq, qscale, S, ws_o,
      ws_lse, s.err_word);
  return cudaGetLastError();
}

}  // namespace

// True when the tensor-core decode kernel takes this shape: head_dim 256
// and a GQA group of at most 48 query heads.  More than 48 query rows per
// (sequence, kv-head) run as several launches over chunks of queries.
bool decode_tc_supported(const nvkv_cache &c, int T, int Hq) {
  const int G = Hq / c.num_kv_heads;
  return c.head_dim == kD && T >= 1 && G >= 1 && G <= 48 && encode_fn() != nullptr;
}

// The pool as a 2-D byte tensor of 128-byte rows; one 36-row box is one
// page's kv-head block (head_dim 256).  Shared with the prefill kernel.
bool make_pool_tmap(const nvkv_cache &c, CUtensorMap *map) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t rows = (cuuint64_t)c.num_pages * c.num_kv_heads * kRowsPerHead;
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {128, kRowsPerHead};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, c.pool, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_decode_tc(const nvkv_cache &c, const nvkv_seqs &s, const void *q, int T,
                             int Hq, float sm_scale, int S, float *ws_o, float *ws_lse,
                             cudaStream_t stream) {
  CUtensorMap map;
  if (!make_pool_tmap(c, &map)) return cudaErrorNotSupported;
  const int G = Hq / c.num_kv_heads;
  const float qscale = sm_scale * 1.4426950408889634f;
  // Queries in chunks of at most 48 rows: each launch reads the whole KV
  // of the step and writes its rows of the shared workspace layout (the
  // same split plan, so nvkv_combine merges them as one launch's).
  const int Tc = 48 / G;
  for (int t0 = 0; t0 < T; t0 += Tc) {
    const int Tn = T - t0 < Tc ? T - t0 : Tc;
    const int R = Tn * G;
    cudaError_t e;
    if (R <= 16)
      e = launch_n<16>(map, c, s, q, Tn, t0, T, Hq, qscale, S, ws_o, ws_lse, stream);
    else if (R <= 32)
      e = launch_n<32>(map, c, s, q, Tn, t0, T, Hq, qscale, S, ws_o, ws_lse, stream);
    else
      e = launch_n<48>(map, c, s, q, Tn, t0, T, Hq, qscale, S, ws_o, ws_lse, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace nvkv
