// decode_qk4.cu -- split-K GQA decode attention over the NVFP4 paged pool,
// head_dim 256, up to 6 query rows per (sequence, kv-head): the scores on
// the NVFP4 block-scaled tensor-core MMA, straight from the cached codes.
//
// What it computes is the decode half of the path in the "knoopx/ninfer"
// README, "Capabilities and limits" (batched decode, MTP verify), over the
// NVFP4 KV cache of the "gzenz/ninfer" README, "Fork changes vs upstream" ->
// "Context and model": for every query row (t, g) of kv-head h of sequence
// b, at position kv_len - T + t, the softmax-weighted sum of the dequantised
// V rows over the visible keys of one split, as a partial result (o,
// base-2 log-sum-exp) that nvkv_combine merges.  Same contract, split plan
// and workspace layout as the other decode kernels.
//
// The cache format is the tensor core's own NVFP4 operand format: E2M1 codes
// packed two per byte (low nibble first) with one unsigned E4M3 scale per 16
// consecutive elements along the contraction.  K's groups run along
// head_dim, which is the contraction of the scores, so the K codes the TMA
// copies into shared memory are the A operand of tcgen05.mma
// kind::mxf4nvf4 as they are, and the K scale bytes are its scale factors:
// no K dequantisation at all, and 64 head_dim elements per instruction.
// The query side must be NVFP4 too.  Each query row x = q * sm_scale * log2(e)
// (fp32) is written as a sum of L = 8 NVFP4 terms, x = sum_l 2^-k_l * c_l,
// each term quantising the residual the previous terms left (scale = E4M3 of
// group amax / 6, codes = E2M1 nearest, after a power-of-two prescale 2^k_l
// that puts the row maximum in [256, 512)); every term shrinks the residual
// by at least 5.6x (at most one E2M1 half-gap, scale/1, per element), so
// the dropped remainder is below 0.177^8 = 1e-6 of each group's maximum.
// The terms are the N side of the MMA (row r, term l -> column r*L + l), and
// the softmax recombines each row's L columns with their 2^-k_l factors in
// fp32.  The products of E2M1 codes and E4M3 scales are exact; the MMA
// accumulates them in fp32.
//
// V's groups run along head_dim, not along the tokens the value sum
// contracts, so the value sum is an f16 MMA (swap-AB: V^T is the M = 128
// side, the query rows the N = 16 side).  V^T goes into Tensor Memory as
// exact f16 values: E2M1 * E4M3 has at most 6 significant bits and lies in
// [2^-10, 2688], so v * 2^-14 is an f16 number (subnormal at the bottom)
// and needs no rounding.  A 32-bit word of 8 codes becomes four f16 pairs
// with integer operations: the bit pattern (mag << 9) | (sign << 15) is
// exactly E2M1(code) * 2^-14 (the E2M1 subnormal 0.5 included), built with a
// shift, two masks and a multiply-add -- no conversion instructions, which
// run at a fraction of the rate -- and one f16 multiply by the pair's scales
// applies the scales.  A warp covers 32 head_dim rows, i.e. two scale
// groups, so it converts the 2 x 128 scale bytes of a unit once (4
// conversions a lane) into a table in shared memory that its lanes read.
// The pair of a word holds tokens (t, t+4), so P uses the same permutation
// of the tokens along K.  P = f16(2^(score - running max)) from an fp32
// exp2, at most 2^8 with the lazy maximum, and the epilogue applies
// 2^14 / denominator, the denominator summing the same f16 weights.
//
// Per 128-token unit the tensor pipe runs 4 NVFP4 MMAs (scores) and 16 f16
// MMAs (values), against 16 + 16 f16 MMAs when K is dequantised.
//
// Roles (one persistent CTA per split-plan range, 512 threads):
//  * warp 12 (TMA): per page two tiled loads, no multicast: the 16 rows of K
//    codes (128-byte swizzle, into the unit's contiguous K tile) and the 18
//    rows of V codes and V scales (no swizzle); 5-stage ring.  Warp 15 loads
//    the 2 rows of K scale bytes of each page into a separate 8-slot ring,
//    so the scale factors written one unit ahead hold no stage of the big
//    ring and the big ring keeps 5 units of loads in flight.
//  * warps 0..7 write the scaled V^T into Tensor Memory (one head_dim row
//    a lane).
//  * warps 8..11 (softmax, one token a lane): copy the K scale bytes of the
//    next unit into the Tensor Memory scale-factor layout (every lane
//    quarter holds the same 32 rows), recombine the terms, mask,
//    running max raised lazily (only when a score exceeds it by more than
//    2^8, detected by a vote), fp32 exp2, P to a 4-slot ring in shared
//    memory, the denominator from the same f16 weights; at a segment start
//    they build the query terms.
//  * warp 13 issues the score MMAs, warp 14 the value MMAs (one thread each).
//  * Every wait is bounded; a timeout sets NVKV_DEVERR_TIMEOUT, turns later
//    waits into no-ops and lets the kernel drain and free its Tensor Memory.
#include <cfloat>

#include "nvkv_common.cuh"
#include "sm100.cuh"

namespace nvkv {
namespace {

using namespace sm100;

constexpr int kD = 256;
constexpr int kRowsPerHead = 36;         // 18*D bytes / 128
constexpr int kUnitPages = 8;
constexpr int kKRows = 16;               // K-code rows of a page block (one per token)
constexpr int kKsRows = 2;               // K scales: 16 tokens x 16 groups
constexpr int kVRows = 18;               // V codes (16), V scales (2)
constexpr int kKPageBytes = kKRows * 128;         // 2048
constexpr int kVPageBytes = kVRows * 128;         // 2304
constexpr int kKsPageBytes = kKsRows * 128;       // 256
constexpr int kVc = 0, kVs = 2048;       // V codes, V scales inside a page's V block
constexpr int kKsSlotBytes = kUnitPages * kKsPageBytes;    // 2048
// K8V4 page block of one kv-head (head_dim 256): K codes [16][256] (4096 B),
// K row scales [16] fp32 (64 B), then the V codes and scales as above.
constexpr int kK8HeadBytes = 25 * kD + 64;   // 6464
constexpr int kK8KsOff = 16 * kD;            // 4096
constexpr int kK8VOff = kK8KsOff + 64;       // 4160

constexpr int kRowsCap = 6;              // query rows per pair (T * G) this kernel takes
constexpr int kTerms = 8;                // NVFP4 terms per query row
constexpr int kNSMax = kRowsCap * kTerms;   // 48: largest N of the score MMA
constexpr int kNP = 16;                  // N of the value MMA: the query rows, padded
constexpr int kPSlots = 4;               // P ring depth
constexpr int kPSlotBytes = 2 * 2048;    // rows 0..7, rows 8..15 (zero) x 128 tokens
constexpr int kVscWarpBytes = kUnitPages * 2 * 8 * 4;   // 512
constexpr int kVSlots = 3;               // V^T ring depth (Tensor Memory)

constexpr int kDeqWarps = 8;             // warps 0..7
constexpr int kSmxWarp0 = 8;             // warps 8..11
constexpr int kSmxWarps = 4;
constexpr int kProducerWarp = 12;        // K codes and V
constexpr int kMmaWarp = 13;             // issues the score MMAs
constexpr int kPvWarp = 14;              // issues the value MMAs
constexpr int kKsProducerWarp = 15;      // K scales
constexpr int kThreads = 16 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr long long kWaitBudget = 2000000000LL;  // clock cycles (~1 s)
constexpr float kLazyRescale = 8.0f;             // log2 units

// Tensor Memory columns (all 512).
constexpr uint32_t kColV = 0;      // kVSlots x 128: V^T (d-half h at +64h), f16 token pairs
constexpr uint32_t kColS = 384;    // kNSMax: S^T, fp32, one token per lane
constexpr uint32_t kColO = 432;    // 2 halves x kNP: O^T, fp32, column = query row
constexpr uint32_t kColSFA = 464;  // 2 slots x 16: K scale factors, column 4*ks + m1
constexpr uint32_t kColSFB = 496;  // 4 x 4: query-term scale factors, column 4*ks + n1 (n1 < 2)
static_assert(kColV + kVSlots * 128 <= kColS && kColS + kNSMax <= kColO &&
                  kColO + 2 * kNP <= kColSFA &&
                  kColSFB + 16 <= kTmemCols && kColSFA % 4 == 0 && kColSFB % 4 == 0,
              "tensor memory");

// Shared memory (offsets from a 1024-byte aligned base), per cache format.
// NVFP4: a stage holds the unit's K code tile [128 tokens][128 B] and the 8
// pages' V blocks; the K scale bytes go to their own ring.  K8V4: the K code
// tile is two head_dim halves [2][128 tokens][128 B], then the V blocks, then
// the 8 pages' K row scales ([8][128 B] slots, 16 fp32 used); no scale ring.
template <bool K8>
struct Fmt {
  static constexpr int kKTileBytes = K8 ? 2 * kUnitPages * kKPageBytes : kUnitPages * kKPageBytes;
  static constexpr int kVOff = kKTileBytes;                       // V blocks [page][2304]
  static constexpr int kKsOff = kVOff + kUnitPages * kVPageBytes;  // K8: row scales [page][128 B]
  static constexpr int kStageBytes = K8 ? 52224 : kKsOff;          // 1024-aligned
  static constexpr int kStages = K8 ? 3 : 5;
  static constexpr int kKsSlots = K8 ? 0 : 8;                      // K scale ring (NVFP4)
  static constexpr int kQBytes = (K8 ? 2 : 1) * kNSMax * 128;      // query terms, swizzled
  static constexpr int kOffKs = kStages * kStageBytes;
  static constexpr int kOffQ = kOffKs + kKsSlots * kKsSlotBytes;
  static constexpr int kOffP = kOffQ + kQBytes;                    // P tiles [slot], MN-major f16
  static constexpr int kOffVsc = kOffP + kPSlots * kPSlotBytes;    // V scale pairs [warp][page][group][8]
  static constexpr int kOffSfb = kOffVsc + kDeqWarps * kVscWarpBytes;  // [kNSMax][16] term scales
  static constexpr int kOffFac = kOffSfb + kNSMax * 16;            // float: 2^-k of each row
  static constexpr int kOffRed = kOffFac + kNSMax * 4;             // float [quarter][kNP]
  static constexpr int kOffM = kOffRed + 4 * kNP * 4;              // float [kNP]
  static constexpr int kOffAlpha = kOffM + kNP * 4;
  static constexpr int kOffNvis = kOffAlpha + kNP * 4;
  static constexpr int kOffFlags = kOffNvis + kNP * 4;             // int[4]: abort at [2]
  static constexpr int kOffPages = kOffFlags + 16;                 // int[stages][8]
  static constexpr int kOffKsv = kOffPages + kStages * kUnitPages * 4;  // u32 [ks slot]: pages present
  static constexpr int kOffBars = kOffKsv + ((kKsSlots > 0 ? kKsSlots : 1) * 4 + 7) / 8 * 8;
  static constexpr int kNumBars = 2 * kStages + 2 * kKsSlots + 4 + 4 * kVSlots + 2 * kPSlots + 5;
  static constexpr int kOffTmem = kOffBars + kNumBars * 8;
  static constexpr int kSmemBytes = kOffTmem + 16 + 1024;          // + alignment slack
  // (TMA destinations are 128-byte aligned: each page's 64 bytes of K row
  // scales get a 128-byte slot)
  static_assert(kKsOff + (K8 ? kUnitPages * 128 : 0) <= kStageBytes && kStageBytes % 1024 == 0 &&
                    kKsOff % 128 == 0,
                "stage");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert(kOffQ % 1024 == 0 && kOffP % 128 == 0 && kOffKs % 128 == 0 &&
                    kOffVsc % 16 == 0 && kOffSfb % 16 == 0 && kOffPages % 16 == 0 &&
                    kOffBars % 8 == 0,
                "alignment");
};

struct Shared {
  uint8_t *stages, *ks, *qtile, *ptile, *sfb;
  uint32_t *vsc;
  float *fac, *red, *m_s, *alpha_s;
  int32_t *nvis_s, *pages;
  uint32_t *ksv;  // [ks slot]: bit p set when page p of the unit is present (NVFP4)
  volatile int *flags;
  // A barrier of a ring slot completes once per unit that uses the slot.  A
  // parity wait for unit u on it is only valid once the unit before u on
  // the same slot has been seen complete (else the parity aliases); every
  // wait below states or follows from that.
  uint64_t *full, *empty;        // [kStages]
  uint64_t *ks_full, *ks_empty;  // [kKsSlots]
  uint64_t *sfa_ready;           // [2]: scale factors of K written
  uint64_t *sready, *sfree;      // S^T written; S^T read by the softmax
  uint64_t *vready, *pvdone;     // [kVSlots][half]: V^T written; value MMAs done
  uint64_t *pready, *pfree;      // [kPSlots]: P written; P read by the value MMAs
  uint64_t *qready, *final_bar, *final_pv;
  uint64_t *qfree;     // every score MMA of the segment completed (query tiles free)
  uint64_t *segstart;  // the softmax has taken the segment's row factors
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

// 2^k as a float for -126 <= k <= 127 (exact).
__device__ __forceinline__ float pow2f(int k) { return __int_as_float((k + 127) << 23); }
// x * 2^k for -252 <= k <= 254 as two exact power-of-two multiplies (the
// result is exact unless it leaves the float range).
__device__ __forceinline__ float scale_pow2(float x, int k) {
  const int k1 = k / 2;
  return x * pow2f(k1) * pow2f(k - k1);
}

// Four f16 pairs from a word of 8 E2M1 codes (code i in bits 4i..4i+3):
// pair t holds codes t (low half) and t+4 (high half), each as the f16 bit
// pattern (mag << 9) | (sign << 15) = E2M1(code) * 2^-14, exactly.  The
// shift puts code t at bits 9..12 and code t+4 at bits 25..28; the masks keep
// the magnitudes and the sign bits, and the multiply-add moves the sign bits
// 12 and 28 up to 15 and 31.
template <int t>
__device__ __forceinline__ uint32_t code_pair(uint32_t w) {
  const uint32_t a = t < 3 ? (w << (9 - 4 * t)) : (w >> 3);
  return (a & 0x10001000u) * 8u + (a & 0x0E000E00u);
}

// f16 pair product, round to nearest, subnormals kept (the V^T values at the
// bottom of the range are f16 subnormals, and exact).
__device__ __forceinline__ uint32_t mul_f16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// K8 selects the cache format: false = NVFP4 K (tmap_k: 16-row SW128 boxes of
// K codes; tmap_ks: 2-row boxes of K scales; tmap_v: 18-row boxes of V codes
// and scales, all over 128-byte rows of the pool), true = K8V4 (tmap_k: 3-D
// [block][token][256 B], 128-byte SW128 boxes of 16 tokens, one per head_dim
// half; tmap_ks: [block][64 B] row scales; tmap_v: [block][18][128 B]).
template <int RM, bool K8>
__global__ void __launch_bounds__(kThreads, 1)
decode_qk4_kernel(const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_ks,
                  const __grid_constant__ CUtensorMap tmap_v, int num_pages, int Hkv,
                  const int32_t *__restrict__ page_table, int max_pages,
                  const int32_t *__restrict__ kv_lens, int B, int max_kv_len,
                  const __nv_bfloat16 *__restrict__ q, int T, int Hq, float qscale, int S,
                  float *__restrict__ ws_o, float *__restrict__ ws_lse, int32_t *err) {
  // RM: query rows per pair rounded up to an even count (padding rows are
  // zero); the score MMA has N = RM * kTerms columns.
  static_assert(RM % 2 == 0 && RM >= 2 && RM <= kRowsCap, "rows");
  constexpr int NS = RM * kTerms;
  using F = Fmt<K8>;
  constexpr int kStages = F::kStages, kStageBytes = F::kStageBytes, kKTileBytes = F::kKTileBytes,
                kKsSlots = F::kKsSlots;
  constexpr int kOffKs = F::kOffKs, kOffQ = F::kOffQ, kOffP = F::kOffP, kOffVsc = F::kOffVsc,
                kOffSfb = F::kOffSfb, kOffFac = F::kOffFac, kOffRed = F::kOffRed,
                kOffM = F::kOffM, kOffAlpha = F::kOffAlpha,
                kOffNvis = F::kOffNvis, kOffFlags = F::kOffFlags, kOffPages = F::kOffPages,
                kOffKsv = F::kOffKsv,
                kOffBars = F::kOffBars, kOffTmem = F::kOffTmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Shared sh;
  sh.stages = smem;
  sh.ks = smem + kOffKs;
  sh.qtile = smem + kOffQ;
  sh.ptile = smem + kOffP;
  sh.vsc = reinterpret_cast<uint32_t *>(smem + kOffVsc);
  sh.sfb = smem + kOffSfb;
  sh.fac = reinterpret_cast<float *>(smem + kOffFac);
  sh.red = reinterpret_cast<float *>(smem + kOffRed);
  sh.m_s = reinterpret_cast<float *>(smem + kOffM);
  sh.alpha_s = reinterpret_cast<float *>(smem + kOffAlpha);
  sh.nvis_s = reinterpret_cast<int32_t *>(smem + kOffNvis);
  sh.flags = reinterpret_cast<volatile int *>(smem + kOffFlags);
  sh.pages = reinterpret_cast<int32_t *>(smem + kOffPages);
  sh.ksv = reinterpret_cast<uint32_t *>(smem + kOffKsv);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars);
  sh.full = bars;
  sh.empty = bars + kStages;
  sh.ks_full = bars + 2 * kStages;
  sh.ks_empty = sh.ks_full + kKsSlots;
  sh.sfa_ready = sh.ks_empty + kKsSlots;
  sh.sready = sh.sfa_ready + 2;
  sh.sfree = sh.sfa_ready + 3;
  sh.vready = sh.sfa_ready + 4;
  sh.pvdone = sh.vready + 2 * kVSlots;
  sh.pready = sh.pvdone + 2 * kVSlots;
  sh.pfree = sh.pready + kPSlots;
  sh.qready = sh.pfree + kPSlots;
  sh.final_bar = sh.qready + 1;
  sh.final_pv = sh.qready + 2;
  sh.qfree = sh.qready + 3;
  sh.segstart = sh.qready + 4;
  sh.tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffTmem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = Hq / Hkv;
  const int R = T * G;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.full[i], 1);
      // the score MMAs' commit, the V^T writers (and, for K8V4, the softmax
      // warps, which read their tokens' K row scales from the stage)
      mbar_init(&sh.empty[i], 1 + kDeqWarps + (K8 ? kSmxWarps : 0));
    }
    for (int i = 0; i < kKsSlots; ++i) {
      mbar_init(&sh.ks_full[i], 1);
      mbar_init(&sh.ks_empty[i], kSmxWarps);  // the scale-factor writers
    }
    for (int i = 0; i < 2; ++i) mbar_init(&sh.sfa_ready[i], kSmxWarps);
    mbar_init(sh.sready, 1);
    mbar_init(sh.sfree, kSmxWarps);
    for (int i = 0; i < 2 * kVSlots; ++i) {
      mbar_init(&sh.vready[i], kDeqWarps / 2);
      mbar_init(&sh.pvdone[i], 1);
    }
    for (int i = 0; i < kPSlots; ++i) {
      mbar_init(&sh.pready[i], kSmxWarps);
      mbar_init(&sh.pfree[i], 1);
    }
    mbar_init(sh.qready, 4);  // the V^T writers of lane quarters 0..3
    mbar_init(sh.qfree, 1);
    mbar_init(sh.segstart, kSmxWarps);
    mbar_init(sh.final_bar, 1);
    mbar_init(sh.final_pv, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 4) sh.flags[threadIdx.x] = 0;
  // The P tiles start as zeros: rows R..15 are never written.
  for (int i = threadIdx.x; i < kPSlots * kPSlotBytes / 16; i += kThreads)
    reinterpret_cast<uint4 *>(sh.ptile)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (warp == kMmaWarp) {
    tmem_alloc(sh.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sh.tmem_slot;

  int64_t U = 0;
  for (int b = 0; b < B; ++b) U += (int64_t)units_of_len(kv_lens[b]) * Hkv;
  const int c = blockIdx.x;
  const int64_t u0 = U > 0 ? range_begin(c, U, S) : 0;
  const int64_t u1 = U > 0 ? range_begin(c + 1, U, S) : 0;
  const uint32_t n_units = (uint32_t)(u1 - u0);

  if (K8 && warp == kKsProducerWarp) {
    // K8V4 has no K scale ring: this warp has nothing to do.
  } else if (warp == kProducerWarp || warp == kKsProducerWarp) {
    // ------------------------------------------------------------------ TMA
    // Lane p < 8 owns page p of a unit; the page ids of unit u+1 are loaded
    // while unit u's copies are issued.  One warp fills the stage ring (K
    // codes into the unit's contiguous K tile, V codes and scales, and for
    // K8V4 the K row scales), the other (NVFP4) the deeper ring of K scale
    // bytes, which the scale-factor writers read one unit ahead of the rest.
    const bool big = warp == kProducerWarp;
    const int ring = big ? kStages : kKsSlots;
    uint64_t *fullb = big ? sh.full : sh.ks_full;
    uint64_t *emptyb = big ? sh.empty : sh.ks_empty;
    if (big) {
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
    } else {
      prefetch_tmap(&tmap_ks);
    }
    const int p = lane & 7;
    int64_t u = u0;
    Seg sg = segment_at(u, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
    auto page_for = [&](const Seg &g, int64_t uu) -> int {
      const int tok = (int)(uu - g.pair_start) * kUnitTokens + p * kPageTokens;
      const int32_t *pt = page_table + (size_t)g.b * max_pages;
      const int pg = page_of(pt, tok, g.kv_len, num_pages);
      if (big && lane < kUnitPages && tok < g.kv_len && pg < 0) report(err, NVKV_DEVERR_PAGE_ID);
      return pg;
    };
    int cur = u < u1 ? page_for(sg, u) : -1;
    uint32_t uc = 0;
    for (; u < u1; ++u, ++uc) {
      const int slot = uc % ring;
      int nxt = -1;
      Seg nsg = sg;
      if (u + 1 < u1) {
        if (u + 1 >= sg.seg_end) nsg = segment_at(u + 1, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
        nxt = page_for(nsg, u + 1);
      }
      if (uc >= (uint32_t)ring) {
        if (lane == 0) wait_bar(&emptyb[slot], ((uc / ring) + 1) & 1, sh.flags, err);
        __syncwarp();
      }
      const bool mine = lane < kUnitPages && cur >= 0;
      if (big && lane < kUnitPages) sh.pages[slot * kUnitPages + lane] = cur;
      const uint32_t present = __ballot_sync(0xffffffffu, mine);
      // the K-scale ring carries the unit's present pages to the softmax
      if (!big && lane == 0) sh.ksv[slot] = present;
      const uint32_t bytes = __popc(present) *
                             (!big ? kKsPageBytes : K8 ? kK8HeadBytes : kKPageBytes + kVPageBytes);
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&fullb[slot], bytes);
      __syncwarp();
      if (mine && K8) {
        // K halves [token][128 B] (x = 0 / 128 of the 256-byte rows), the V
        // block and the 16 K row scales of this page's kv-head block
        const int blk = cur * Hkv + sg.h;
        uint8_t *st = sh.stages + slot * kStageBytes;
        tma_load_3d(st + lane * kKPageBytes, &tmap_k, 0, 0, blk, &fullb[slot]);
        tma_load_3d(st + kUnitPages * kKPageBytes + lane * kKPageBytes, &tmap_k, 128, 0, blk,
                    &fullb[slot]);
        tma_load_3d(st + F::kVOff + lane * kVPageBytes, &tmap_v, 0, 0, blk, &fullb[slot]);
        tma_load_2d(st + F::kKsOff + lane * 128, &tmap_ks, 0, blk, &fullb[slot]);
      } else if (mine) {
        const int y = (cur * Hkv + sg.h) * kRowsPerHead;
        if (big) {
          uint8_t *st = sh.stages + slot * kStageBytes;
          tma_load_2d(st + lane * kKPageBytes, &tmap_k, 0, y, &fullb[slot]);
          tma_load_2d(st + kKTileBytes + lane * kVPageBytes, &tmap_v, 0, y + kKRows + kKsRows,
                      &fullb[slot]);
        } else {
          tma_load_2d(sh.ks + slot * kKsSlotBytes + lane * kKsPageBytes, &tmap_ks, 0, y + kKRows,
                      &fullb[slot]);
        }
      }
      cur = nxt;
      sg = nsg;
    }
    // Drain: every issued copy must land before the CTA may exit.
    if (lane == 0) {
      const uint32_t first = uc > (uint32_t)ring ? uc - ring : 0;
      for (uint32_t k = first; k < uc; ++k)
        mbar_wait(&fullb[k % ring], (k / ring) & 1, kWaitBudget);
    }
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    // ------------------------------------------------------------------ MMA
    // Two issuing threads: issuing a batch of tcgen05.mma blocks the thread
    // until the batch has nearly executed, so a single thread would leave
    // the tensor pipe idle while it waits for the next step's inputs.  One
    // thread issues the scores of each unit as soon as its tiles, scale
    // factors, query terms and S^T slot are ready; the other issues the
    // value MMAs of each unit once its V^T and P are ready.  Each commits
    // its own MMAs; the tensor pipe runs both streams.
    if (lane == 0) {
      int64_t seg_end = segment_at(u0, u1, kv_lens, B, Hkv, max_kv_len, max_pages).seg_end;
      bool issued = false;
      if (warp == kMmaWarp) {
        // NVFP4: E2M1 x E2M1 block-scaled; K8V4: E4M3 x E4M3 (kind::f8f6f4,
        // format 0 = E4M3), the same descriptor layout as the f16 kind.
        const uint32_t idesc_qk = K8 ? idesc_f16_f32(128, NS, false, false) : idesc_nvf4(128, NS);
        const uint32_t qb = smem_u32(sh.qtile);
        const uint32_t kt0 = smem_u32(sh.stages);
        uint32_t seg_idx = 0;
        for (uint32_t qk = 0; qk < n_units && !sh.flags[2]; ++qk) {
          const int64_t uu = u0 + qk;
          const bool opens = qk == 0 || uu >= seg_end;
          if (uu >= seg_end) {
            seg_end = segment_at(uu, u1, kv_lens, B, Hkv, max_kv_len, max_pages).seg_end;
            ++seg_idx;
          }
          if (opens) wait_bar(sh.qready, seg_idx & 1, sh.flags, err);
          const int stage = qk % kStages;
          wait_bar(&sh.full[stage], (qk / kStages) & 1, sh.flags, err);
          if (!K8) wait_bar(&sh.sfa_ready[qk & 1], (qk >> 1) & 1, sh.flags, err);
          // S^T was read by the softmax of unit qk-1
          if (qk > 0) wait_bar(sh.sfree, (qk - 1) & 1, sh.flags, err);
          tc_fence_after();
          const uint32_t sslot = tmem + kColS;
          const uint32_t sfa = tmem + kColSFA + (qk & 1) * 16;
          const uint32_t kt = kt0 + stage * kStageBytes;
          if constexpr (K8) {
            // two head_dim halves of 128 bytes, 4 K steps of 32 elements each
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_f8_ss(sslot, smem_desc_sw128(kt + hf * kUnitPages * kKPageBytes + 32 * ks),
                          smem_desc_sw128(qb + hf * kNSMax * 128 + 32 * ks), idesc_qk,
                          (hf | ks) > 0);
          } else {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_nvf4_ss(sslot, smem_desc_sw128(kt + 32 * ks), smem_desc_sw128(qb + 32 * ks),
                          idesc_qk, ks > 0, sfa + 4 * ks, tmem + kColSFB + 4 * ks);
          }
          mma_commit(sh.sready);
          mma_commit(&sh.empty[stage]);  // the K tile has been read
          // the last score MMA of a segment that another follows: the V^T
          // writers may build the next pair's query terms
          if (uu + 1 >= seg_end && uu + 1 < u1) mma_commit(sh.qfree);
          issued = true;
        }
        if (issued) {
          mma_commit(sh.final_bar);
          mbar_wait(sh.final_bar, 0, kWaitBudget);
        }
      } else {
        const uint32_t idesc_pv = idesc_f16_f32(128, kNP, false, true);
        const uint32_t pb = smem_u32(sh.ptile);
        for (uint32_t pv = 0; pv < n_units && !sh.flags[2]; ++pv) {
          const int64_t uu = u0 + pv;
          const bool first = pv == 0 || uu >= seg_end;  // O^T starts from zero
          if (uu >= seg_end)
            seg_end = segment_at(uu, u1, kv_lens, B, Hkv, max_kv_len, max_pages).seg_end;
          const int ps = pv % kPSlots;
          wait_bar(&sh.pready[ps], (pv / kPSlots) & 1, sh.flags, err);
          const uint32_t pslot = pb + ps * kPSlotBytes;
          const int vs = pv % kVSlots;
          const uint32_t vslot = tmem + kColV + vs * 128;
          // One head_dim half at a time: each half's V^T rows are released
          // as soon as its MMAs complete.
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            wait_bar(&sh.vready[vs * 2 + hf], (pv / kVSlots) & 1, sh.flags, err);
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              mma_f16_ts(tmem + kColO + hf * kNP, vslot + 64 * hf + ks * 8,
                         smem_desc(pslot + ks * 256, 128, 2048), idesc_pv, (!first) || ks > 0);
            mma_commit(&sh.pvdone[vs * 2 + hf]);
          }
          mma_commit(&sh.pfree[ps]);
          issued = true;
        }
        if (issued) {
          mma_commit(sh.final_pv);
          mbar_wait(sh.final_pv, 0, kWaitBudget);
        }
      }
    }
  } else {
    // -------------------------------------------------------------- workers
    const bool smx = warp >= kSmxWarp0;
    const int lq = warp & 3;                     // lane quarter of Tensor Memory
    const int hv = smx ? 0 : ((warp >> 2) & 1);  // V^T half of a V^T-writing warp
    const uint32_t tl = tmem + ((uint32_t)(32 * lq) << 16);
    const int stid = threadIdx.x - kSmxWarp0 * 32;  // softmax thread 0..127
    float l_part[RM], facr[RM], mr[RM];
#pragma unroll
    for (int i = 0; i < RM; ++i) l_part[i] = facr[i] = 0.f, mr[i] = -FLT_MAX;

    // K scale factors of unit un (from the K-scale ring) into slot un&1,
    // which the score MMAs of unit un-2 read before: the softmax warps write
    // them at the start of unit un-1, after their wait for the scores of
    // unit un-2.  Every lane quarter holds the same rows.
    // Column 4*ks + m1, lane l: the 4 scale bytes of token 32*m1 + l for
    // head_dim elements 64*ks .. 64*ks+63.
    // Returns the unit's present-page mask, which travels with its K scales.
    auto write_sfa = [&](uint32_t un) -> uint32_t {
      constexpr int kRing = kKsSlots > 0 ? kKsSlots : 1;  // (NVFP4 only)
      const int ksl = un % kRing;
      const uint8_t *kb = sh.ks + ksl * kKsSlotBytes;
      wait_bar(&sh.ks_full[ksl], (un / kRing) & 1, sh.flags, err);
      tc_fence_after();
      const uint32_t present = sh.ksv[ksl];
      uint32_t w[16];
#pragma unroll
      for (int m1 = 0; m1 < 4; ++m1) {
        const uint4 v = *reinterpret_cast<const uint4 *>(kb + (32 * m1 + lane) * 16);
        w[0 * 4 + m1] = v.x;
        w[1 * 4 + m1] = v.y;
        w[2 * 4 + m1] = v.z;
        w[3 * 4 + m1] = v.w;
      }
      tmem_st16(tl + kColSFA + (un & 1) * 16, w);
      __syncwarp();  // every lane's loads are done (the store consumed them)
      if (lane == 0) mbar_arrive(&sh.ks_empty[ksl]);
      return present;
    };
    // Publishes the scale factors of unit un once the warp's stores are
    // complete (the caller waits for them, together with its own loads).
    auto finish_sfa = [&](uint32_t un) {
      if (lane == 0) mbar_arrive(&sh.sfa_ready[un & 1]);
    };
    // Present pages of the softmax's current and next unit (NVFP4: from the
    // K-scale ring; a token of an absent page is skipped like an invisible
    // one).
    uint32_t pm_cur = 0xffu, pm_next = 0xffu;
    if (!K8 && smx && n_units > 0) {
      pm_cur = write_sfa(0);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      finish_sfa(0);
    }

    // Query terms of pair pg, one row per V^T-writing warp (rows are
    // independent chains of conversions), then their scale factors into
    // Tensor Memory and the release of the pair's score MMAs.  The V^T
    // writers build them for the next pair as soon as the current segment's
    // last score MMA has completed, so the next segment's first scores are
    // computed while the softmax finishes this one.
    auto prep_q = [&](const Seg &pg) {
      // Row r of x = q * sm_scale * log2(e): one power-of-two prescale 2^k
      // puts the row maximum in [256, 512); then term l quantises the
      // residual y (group scale = E4M3 of its 16-element maximum / 6,
      // codes = nearest E2M1) and leaves y - term, exactly.  Each term
      // shrinks every group's residual at least 5.6x, so the scales of the
      // 8 terms stay inside the E4M3 range (448 down to 2^-9) until the
      // remainder is below about 2^-15 of the row maximum.  The MMA's
      // columns r*8 .. r*8+7 summed and times 2^-k give the row's scores.
      // (Any rounding of the scales and codes would do: only the residual
      // bookkeeping has to be exact.)
      for (int r = warp; r < RM; r += kDeqWarps) {
        float y[8];
        if (r < R) {
          const int t = r / G, g = r % G;
          const uint4 raw = *reinterpret_cast<const uint4 *>(
              q + ((size_t)(pg.b * T + t) * Hq + pg.h * G + g) * kD + 8 * lane);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            y[2 * i] = __uint_as_float(w[i] << 16) * qscale;
            y[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u) * qscale;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) y[i] = 0.f;
        }
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(y[i]));
        a = warp_max(a);
        // A row whose largest element is below the smallest normal float
        // (2^-126) is taken as zero: its scores would be below 2^-110.
        const int eb = (int)((__float_as_uint(a) >> 23) & 0xffu);  // biased exponent
        // a in [2^(eb-127), 2^(eb-126)): a * 2^k in [256, 512) (NVFP4), in
        // [128, 256) (K8V4, under the E4M3 maximum 448)
        const int k = (K8 ? 134 : 135) - eb;
        if (eb > 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) y[i] = scale_pow2(y[i], k);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) y[i] = 0.f;
        }
        if constexpr (K8) {
          // Term l: E4M3 codes of y * 2^(4l), its value subtracted exactly.
          // E4M3 rounding leaves at most 2^-4 of an element (or 2^-10 of
          // the term's unit in the subnormal range), so y * 2^(4(l+1))
          // stays below 256 and no term saturates; the MMA's column 8r + l
          // carries weight 2^-4l, recombined in the softmax.
#pragma unroll 1
          for (int l = 0; l < kTerms; ++l) {
            const int n = r * kTerms + l;
            const float up = pow2f(4 * l), down = pow2f(-4 * l);
            uint32_t pr[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              pr[i] = f32x2_to_e4m3x2(y[2 * i] * up, y[2 * i + 1] * up);
              const float2 v = f16x2_to_float2(e4m3x2_to_f16x2(pr[i]));
              y[2 * i] -= v.x * down;  // exact
              y[2 * i + 1] -= v.y * down;
            }
            // bytes 8*lane .. 8*lane+7 of the row: head_dim half lane/16,
            // 128-byte swizzle
            const int c16 = (lane & 15) >> 1;
            *reinterpret_cast<uint2 *>(sh.qtile + (lane >> 4) * (kNSMax * 128) + n * 128 +
                                       ((c16 ^ (n & 7)) << 4) + (lane & 1) * 8) =
                make_uint2(pr[0] | (pr[1] << 16), pr[2] | (pr[3] << 16));
          }
        } else {
#pragma unroll 1
        for (int l = 0; l < kTerms; ++l) {
          const int n = r * kTerms + l;
          float ga = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) ga = fmaxf(ga, fabsf(y[i]));
          ga = fmaxf(ga, __shfl_xor_sync(0xffffffffu, ga, 1));  // 16-element group
          const uint32_t sb = (uint32_t)__nv_cvt_float_to_fp8(ga * (1.0f / 6.0f), __NV_SATFINITE,
                                                              __NV_E4M3);
          const float sv = e4m3_to_float((uint8_t)sb);
          const float rs = sv > 0.f ? 1.0f / sv : 0.f;
          uint32_t codes = 0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // codes of y/s (the hardware's rounding; any choice is exact
            // bookkeeping below), then the chosen values, exact in f16
            const uint32_t pair = f32x2_to_e2m1x2(y[2 * i] * rs, y[2 * i + 1] * rs);
            codes |= pair << (8 * i);
            const float2 v = f16x2_to_float2(e2m1x2_to_f16x2(pair));
            y[2 * i] -= v.x * sv;  // the products are exact
            y[2 * i + 1] -= v.y * sv;
          }
          // Row n of the term tile: bytes 4*lane..4*lane+3, 128-byte swizzle.
          *reinterpret_cast<uint32_t *>(sh.qtile + n * 128 + (((lane >> 2) ^ (n & 7)) << 4) +
                                        (lane & 3) * 4) = codes;
          if ((lane & 1) == 0) sh.sfb[n * 16 + (lane >> 1)] = (uint8_t)sb;
        }
        }
        if (lane == 0) sh.fac[r] = eb > 0 ? scale_pow2(1.f, -k) : 0.f;
      }
      fence_proxy_async_smem();
      named_barrier(2, kDeqWarps * 32);
      if (warp < 4) {
        // Scale factors of the terms (each lane quarter holds all rows):
        // column 4*ks + n1, lane l -> row 32*n1 + l (every K step's block
        // starts on a multiple of 4 columns).  K8V4 has none.
        if constexpr (!K8) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = 0u;
#pragma unroll
          for (int n1 = 0; n1 < 2; ++n1) {
            const uint4 v = *reinterpret_cast<const uint4 *>(sh.sfb + (32 * n1 + lane) * 16);
            w[0 * 4 + n1] = v.x;
            w[1 * 4 + n1] = v.y;
            w[2 * 4 + n1] = v.z;
            w[3 * 4 + n1] = v.w;
          }
          tmem_st16(tl + kColSFB, w);
          tmem_wait_st();
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sh.qready);
      }
    };

    uint32_t uc = 0;
    uint32_t seg_idx = 0;
    for (int64_t u = u0; u < u1; ++seg_idx) {
      const Seg sg = segment_at(u, u1, kv_lens, B, Hkv, max_kv_len, max_pages);
      if (sg.bad && threadIdx.x == 0) report(err, NVKV_DEVERR_LENGTH);
      const int64_t seg_start = u;
      const size_t slot = (size_t)c + (size_t)sg.b * Hkv + sg.h;

      if (!smx) {
        if (seg_idx > 0) {
          // The V^T writers come here straight from the previous segment's
          // units: its query terms are replaced once the softmax has taken
          // its row factors (so the shared factors and the query-term
          // barrier run one segment ahead at most) and its score MMAs have
          // all completed.
          wait_bar(sh.segstart, (seg_idx - 1) & 1, sh.flags, err);
          wait_bar(sh.qfree, (seg_idx - 1) & 1, sh.flags, err);
          tc_fence_after();
        }
        prep_q(sg);
      } else {
        // softmax state of the pair; its query terms' row factors (the V^T
        // writers published them with the terms)
        if (stid < kNP) {
          sh.nvis_s[stid] = stid < R ? sg.kv_len - T + stid / G + 1 : 0;
          sh.m_s[stid] = -FLT_MAX;
        }
#pragma unroll
        for (int i = 0; i < RM; ++i) l_part[i] = 0.f, mr[i] = -FLT_MAX;
        wait_bar(sh.qready, seg_idx & 1, sh.flags, err);
#pragma unroll
        for (int i = 0; i < RM; ++i) facr[i] = sh.fac[i];
        __syncwarp();
        if (lane == 0) mbar_arrive(sh.segstart);
        named_barrier(1, kSmxWarps * 32);  // the row state is written
      }

      for (; u < sg.seg_end; ++u, ++uc) {
        const bool first = (u == seg_start);
        const int stage = uc % kStages;
        const uint8_t *vb = sh.stages + stage * kStageBytes + kKTileBytes;
        const int tok0 = (int)(u - sg.pair_start) * kUnitTokens;
        if (!smx) {
          wait_bar(&sh.full[stage], (uc / kStages) & 1, sh.flags, err);
          // ---- scale pairs of this warp's two groups (head_dim rows
          // d0 .. d0+31, d0 = 128*hv + 32*lq), in the token pairs of the
          // V^T words: lane (gsel, page pp, half h8) converts the pairs
          // (8*h8 + t, 8*h8 + t + 4), t < 4.  Tokens without data (past
          // kv_len, or an absent page) get scale 0: their bytes may hold
          // anything, NaN patterns included. ----
          uint32_t *vsc = sh.vsc + (warp * kVscWarpBytes) / 4;
          {
            const int gsel = lane >> 4, pp = (lane & 15) >> 1, h8 = lane & 1;
            const int g = 8 * hv + 2 * lq + gsel;
            const uint2 sw = *reinterpret_cast<const uint2 *>(vb + pp * kVPageBytes + kVs +
                                                              g * 16 + 8 * h8);
            int nval = sg.kv_len - (tok0 + 16 * pp + 8 * h8);
            if (sh.pages[stage * kUnitPages + pp] < 0) nval = 0;
            uint32_t w0 = sw.x, w1 = sw.y;
            if (nval < 8) {
              w0 = nval >= 4 ? w0 : nval <= 0 ? 0u : w0 & ((1u << (8 * nval)) - 1u);
              w1 = nval <= 4 ? 0u : w1 & ((1u << (8 * (nval - 4))) - 1u);
            }
            const uint4 t4 = make_uint4(e4m3x2_to_f16x2(__byte_perm(w0, w1, 0x40)),
                                        e4m3x2_to_f16x2(__byte_perm(w0, w1, 0x51)),
                                        e4m3x2_to_f16x2(__byte_perm(w0, w1, 0x62)),
                                        e4m3x2_to_f16x2(__byte_perm(w0, w1, 0x73)));
            __syncwarp();  // the previous unit's table has been read
            *reinterpret_cast<uint4 *>(vsc + pp * 16 + gsel * 8 + 4 * h8) = t4;
            __syncwarp();
          }
          // ---- V^T into slot uc%3, this warp's half (read by the value
          // MMAs of that half of unit uc-3): head_dim row
          // d = 128*hv + 32*lq + lane, all 8 pages. ----
          const int vs = uc % kVSlots;
          if (uc >= (uint32_t)kVSlots) {
            wait_bar(&sh.pvdone[vs * 2 + hv], ((uc / kVSlots) + 1) & 1, sh.flags, err);
            tc_fence_after();
          }
          {
            const int d = 128 * hv + 32 * lq + lane;
            const uint32_t vcol = kColV + vs * 128 + 64 * hv;
            const uint32_t *vg = vsc + (lane >> 4) * 8;
#pragma unroll
            for (int p = 0; p < kUnitPages; ++p) {
              const uint2 cw =
                  *reinterpret_cast<const uint2 *>(vb + p * kVPageBytes + kVc + d * 8);
              const uint4 s0 = *reinterpret_cast<const uint4 *>(vg + p * 16);
              const uint4 s1 = *reinterpret_cast<const uint4 *>(vg + p * 16 + 4);
              const uint32_t o8[8] = {
                  mul_f16x2(code_pair<0>(cw.x), s0.x), mul_f16x2(code_pair<1>(cw.x), s0.y),
                  mul_f16x2(code_pair<2>(cw.x), s0.z), mul_f16x2(code_pair<3>(cw.x), s0.w),
                  mul_f16x2(code_pair<0>(cw.y), s1.x), mul_f16x2(code_pair<1>(cw.y), s1.y),
                  mul_f16x2(code_pair<2>(cw.y), s1.z), mul_f16x2(code_pair<3>(cw.y), s1.w)};
              tmem_st8(tl + vcol + 8 * p, o8);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&sh.vready[vs * 2 + hv]);
              mbar_arrive(&sh.empty[stage]);  // this warp's reads of the stage are done
            }
          }
        } else {
          // ---- softmax on S^T: thread = token tok0 + 32*lq + lane.
          // First the K scale factors of the next unit, while the scores of
          // this one are computed.
          const bool sfa_next = !K8 && uc + 1 < n_units;
          if (sfa_next) pm_next = write_sfa(uc + 1);
          const int pos = tok0 + 32 * lq + lane;
          wait_bar(sh.sready, uc & 1, sh.flags, err);
          tc_fence_after();
          // Scores: the sum of each row's 8 term columns (packed fp32 adds)
          // times the row's 2^-k; invisible keys and padding rows -inf.
          float x[RM];
          {
            uint32_t rr[NS];
            const uint32_t scol = tl + kColS;
#pragma unroll
            for (int i = 0; i < NS / 16; ++i)
              tmem_ld16(scol + 16 * i, *reinterpret_cast<uint32_t(*)[16]>(rr + 16 * i));
            tmem_wait_ld();
            if (sfa_next) tmem_wait_st();  // the next unit's scale factors
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sh.sfree);  // S^T read
            if (sfa_next) finish_sfa(uc + 1);
            // K8V4: this token's K row scale, from the stage (then this
            // warp's reads of the stage are done)
            float ksc = 1.f;
            bool present;  // the token's page was loaded
            if constexpr (K8) {
              wait_bar(&sh.full[stage], (uc / kStages) & 1, sh.flags, err);
              const int j = 32 * lq + lane;
              ksc = *reinterpret_cast<const float *>(sh.stages + stage * kStageBytes + F::kKsOff +
                                                     (j >> 4) * 128 + (j & 15) * 4);
              present = sh.pages[stage * kUnitPages + (j >> 4)] >= 0;
              __syncwarp();
              if (lane == 0) mbar_arrive(&sh.empty[stage]);
            } else {
              present = (pm_cur >> ((32 * lq + lane) >> 4)) & 1u;
            }
            const bool vis_all = tok0 + kUnitTokens <= sg.kv_len - T + 1 && present;
#pragma unroll
            for (int j = 0; j < RM; ++j) {
              const uint32_t *c8 = rr + j * kTerms;
              float sc;
              if constexpr (K8) {
                // sum_l 2^-4l * column l, by Horner
                float acc = __uint_as_float(c8[kTerms - 1]);
#pragma unroll
                for (int l = kTerms - 2; l >= 0; --l) acc = fmaf(acc, 0.0625f, __uint_as_float(c8[l]));
                sc = acc * facr[j] * ksc;
              } else {
                const float2 a0 = add_f32x2(
                    make_float2(__uint_as_float(c8[0]), __uint_as_float(c8[1])),
                    make_float2(__uint_as_float(c8[2]), __uint_as_float(c8[3])));
                const float2 a1 = add_f32x2(
                    make_float2(__uint_as_float(c8[4]), __uint_as_float(c8[5])),
                    make_float2(__uint_as_float(c8[6]), __uint_as_float(c8[7])));
                const float2 a2 = add_f32x2(a0, a1);
                sc = (a2.x + a2.y) * facr[j];
              }
              const int nv = vis_all ? (j < R ? 0x7fffffff : 0) : sh.nvis_s[j];
              x[j] = pos < nv && present ? sc : -INFINITY;
            }
          }
          // Weights: p = 2^(score - running max) in fp32 (2^-inf = 0), as
          // f16 pairs of rows (2i, 2i+1).  The running max starts at -FLT_MAX
          // (no key seen yet), so a visible key always forces the slow path.
          uint32_t pw[RM / 2];
          bool up = false;
          auto weights = [&]() {
#pragma unroll
            for (int j = 0; j < RM; j += 2) {
              const float d0 = x[j] - mr[j], d1 = x[j + 1] - mr[j + 1];
              up |= (d0 > kLazyRescale) | (d1 > kLazyRescale);
              pw[j / 2] = ex2_f32_to_f16x2(d0, d1);
            }
          };
          weights();
          // one barrier of the 4 softmax warps that also ORs the votes
          const bool any = named_barrier_or(1, kSmxWarps * 32, up);
          if (any) {
            // Slow path (the first unit of a segment and rare max raises):
            // exact row maxima, new running max, rescale of everything
            // accumulated against the old max, weights recomputed.
#pragma unroll
            for (int j = 0; j < RM; ++j) {
              const float wm = warp_max(x[j]);
              if (lane == 0) sh.red[lq * kNP + j] = wm;
            }
            named_barrier(1, kSmxWarps * 32);
            if (stid < RM) {
              float alpha = 1.f;
              if (stid < R) {
                float tmax = -INFINITY;
#pragma unroll
                for (int w = 0; w < 4; ++w) tmax = fmaxf(tmax, sh.red[w * kNP + stid]);
                const float m_old = sh.m_s[stid];
                if (tmax > m_old + kLazyRescale) {
                  alpha = exp2f(m_old - tmax);  // 0 when nothing was seen before
                  sh.m_s[stid] = tmax;
                }
              }
              sh.alpha_s[stid] = alpha;
            }
            named_barrier(1, kSmxWarps * 32);
            float al[RM];
#pragma unroll
            for (int j = 0; j < RM; ++j) {
              al[j] = sh.alpha_s[j];
              l_part[j] *= al[j];
              mr[j] = sh.m_s[j];
            }
            if (!first) {
              // O^T rows d = 32*lq + lane and d + 128, accumulated up to the
              // previous unit, scale by alpha once its value MMAs finished
              // (P slot release of unit uc-1: committed after both halves;
              // the wait of unit uc-5 on that slot is behind, so the parity
              // cannot alias).
              wait_bar(&sh.pfree[(uc - 1) % kPSlots], ((uc - 1) / kPSlots) & 1, sh.flags, err);
              tc_fence_after();
#pragma unroll
              for (int half = 0; half < 2; ++half) {
                uint32_t r8[8];
                const uint32_t col = tl + kColO + half * kNP;
                tmem_ld8(col, r8);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < RM; ++j) r8[j] = __float_as_uint(__uint_as_float(r8[j]) * al[j]);
                tmem_st8(col, r8);
              }
              tmem_wait_st();
            }
            weights();
          }
          // P into ring slot uc%4 (read by the value MMAs of unit uc-4
          // before): rows 0..7 of token slot i of page pg at K position
          // k = 16*pg + 8*(i/8) + 2*(i%4) + (i/4)%2, the order of the V^T
          // token pairs; the MN-major B operand puts element (n, k) at
          // (n/8)*2048 + (k/8)*128 + (k%8)*16 + (n%8)*2.
          const int ps = uc % kPSlots;
          if (uc >= (uint32_t)kPSlots) {
            wait_bar(&sh.pfree[ps], ((uc / kPSlots) + 1) & 1, sh.flags, err);
            tc_fence_after();
          }
          {
            const int j = 32 * lq + lane, pg = j >> 4, i = j & 15;
            const int kk = 16 * pg + 8 * (i >> 3) + 2 * (i & 3) + ((i >> 2) & 1);
            uint32_t w4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int k2 = 0; k2 < RM / 2; ++k2) w4[k2] = pw[k2];
            *reinterpret_cast<uint4 *>(sh.ptile + ps * kPSlotBytes + (kk >> 3) * 128 +
                                       (kk & 7) * 16) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
          // the denominator sums the same f16 weights the value MMAs use
#pragma unroll
          for (int k2 = 0; k2 < RM / 2; ++k2) {
            const float2 f = f16x2_to_float2(pw[k2]);
            l_part[2 * k2] += f.x;
            l_part[2 * k2 + 1] += f.y;
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.pready[ps]);
          pm_cur = pm_next;
        }
      }


      if (smx) {
        // ---- end of segment: O^T / l -> workspace, lse (thread: head_dim
        // rows d = 32*lq + lane and d + 128) ----
        // the last unit's value MMAs, both halves (every softmax warp has
        // seen the value MMAs of unit uc-5 complete)
        wait_bar(&sh.pfree[(uc - 1) % kPSlots], ((uc - 1) / kPSlots) & 1, sh.flags, err);
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < RM; ++j) {
          const float ls = warp_sum(l_part[j]);
          if (lane == 0) sh.red[lq * kNP + j] = ls;
        }
        named_barrier(1, kSmxWarps * 32);
        float lv[RM];
#pragma unroll
        for (int n = 0; n < RM; ++n) {
          lv[n] = 0.f;
#pragma unroll
          for (int w = 0; w < 4; ++w) lv[n] += sh.red[w * kNP + n];
        }
        // The sums carry the 2^-14 of V^T: o = O * 2^14 / l, lse = m + log2(l).
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o8[8];
          tmem_ld8(tl + kColO + half * kNP, o8);
          tmem_wait_ld();
          const int d = 128 * half + 32 * lq + lane;
#pragma unroll
          for (int n = 0; n < RM; ++n) {
            if (n < R) {
              const float v = __uint_as_float(o8[n]);
              ws_o[(slot * R + n) * kD + d] = lv[n] > 0.f ? v * 16384.f / lv[n] : 0.f;
            }
          }
        }
        if (stid < R) {
          float l = 0.f;
#pragma unroll
          for (int n = 0; n < RM; ++n) l = n == stid ? lv[n] : l;
          ws_lse[slot * R + stid] = l > 0.f ? sh.m_s[stid] + log2f(l) : -INFINITY;
        }
        tc_fence_before();
        named_barrier(1, kSmxWarps * 32);  // the sums and maxima have been read
      }
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
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// The pool as a 2-D byte tensor of 128-byte rows; a box of `rows` rows
// starting at row (page * Hkv + h) * 36 + r0 is part of one page's kv-head
// block (head_dim 256).
bool make_map(const nvkv_cache &c, int rows, CUtensorMapSwizzle swz, CUtensorMap *map) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t total = (cuuint64_t)c.num_pages * c.num_kv_heads * kRowsPerHead;
  const cuuint64_t dims[2] = {128, total};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {128, (cuuint32_t)rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, c.pool, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K8V4 pool maps (head_dim 256): the pool as [block][...] with a block stride
// of 6464 bytes (block = page * Hkv + h).  K: [block][16 tokens][256 B],
// boxes of 128 B x 16 tokens, 128-byte swizzle (one box per head_dim half);
// K row scales: [block][64 B] from byte 4096; V codes and scales:
// [block][18][128 B] from byte 4160.
bool make_k8_maps(const nvkv_cache &c, CUtensorMap *mk, CUtensorMap *mks, CUtensorMap *mv) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t nblk = (cuuint64_t)c.num_pages * c.num_kv_heads;
  const cuuint32_t e1[3] = {1, 1, 1};
  uint8_t *pool = static_cast<uint8_t *>(c.pool);
  const cuuint64_t kd[3] = {256, 16, nblk}, ks[2] = {256, kK8HeadBytes};
  const cuuint32_t kb[3] = {128, 16, 1};
  const cuuint64_t sd[2] = {64, nblk}, ss[1] = {kK8HeadBytes};
  const cuuint32_t sb[2] = {64, 1};
  const cuuint64_t vd[3] = {128, kVRows, nblk}, vs[2] = {128, kK8HeadBytes};
  const cuuint32_t vb[3] = {128, kVRows, 1};
  return enc(mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, pool, kd, ks, kb, e1,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
             CUDA_SUCCESS &&
         enc(mks, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, pool + kK8KsOff, sd, ss, sb, e1,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
             CUDA_SUCCESS &&
         enc(mv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, pool + kK8VOff, vd, vs, vb, e1,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
             CUDA_SUCCESS;
}

template <bool K8>
cudaError_t launch_fmt(const nvkv_cache &c, const nvkv_seqs &s, const void *q, int T, int Hq,
                       float sm_scale, int S, float *ws_o, float *ws_lse, cudaStream_t stream) {
  CUtensorMap map_k, map_ks, map_v;
  const bool ok = K8 ? make_k8_maps(c, &map_k, &map_ks, &map_v)
                     : make_map(c, kKRows, CU_TENSOR_MAP_SWIZZLE_128B, &map_k) &&
                           make_map(c, kKsRows, CU_TENSOR_MAP_SWIZZLE_NONE, &map_ks) &&
                           make_map(c, kVRows, CU_TENSOR_MAP_SWIZZLE_NONE, &map_v);
  if (!ok) return cudaErrorNotSupported;
  const float qscale = sm_scale * 1.4426950408889634f;
  const int R = T * (Hq / c.num_kv_heads);
  auto kernel = R <= 2 ? decode_qk4_kernel<2, K8> : R <= 4 ? decode_qk4_kernel<4, K8>
                                                             : decode_qk4_kernel<6, K8>;
  const int smem = Fmt<K8>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kernel<<<S, kThreads, smem, stream>>>(
      map_k, map_ks, map_v, c.num_pages, c.num_kv_heads, s.page_table, s.max_pages_per_seq,
      s.kv_lens, s.batch, s.max_kv_len, static_cast<const __nv_bfloat16 *>(q), T, Hq, qscale, S,
      ws_o, ws_lse, s.err_word);
  return cudaGetLastError();
}

}  // namespace

// True when this kernel takes the shape: head_dim 256 and at most 6 query
// rows (T * Hq/Hkv) per (sequence, kv-head).  The same holds for both cache
// formats.
bool decode_qk4_supported(const nvkv_cache &c, int T, int Hq) {
  const int R = T * (Hq / c.num_kv_heads);
  return c.head_dim == kD && R >= 1 && R <= kRowsCap && encode_fn() != nullptr;
}

cudaError_t launch_decode_qk4(const nvkv_cache &c, const nvkv_seqs &s, const void *q, int T,
                              int Hq, float sm_scale, int S, float *ws_o, float *ws_lse,
                              cudaStream_t stream) {
  return launch_fmt<false>(c, s, q, T, Hq, sm_scale, S, ws_o, ws_lse, stream);
}

// The same kernel over a K8V4 cache (E4M3 K rows with an fp32 row scale,
// NVFP4 V): the scores on kind::f8f6f4 from the cached E4M3 bytes.
cudaError_t launch_decode_qk4_k8v4(const nvkv_cache &c, const nvkv_seqs &s, const void *q, int T,
                                   int Hq, float sm_scale, int S, float *ws_o, float *ws_lse,
                                   cudaStream_t stream) {
  return launch_fmt<true>(c, s, q, T, Hq, sm_scale, S, ws_o, ws_lse, stream);
}

}  // namespace nvkv
