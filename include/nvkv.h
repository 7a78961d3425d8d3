/*
 * nvkv.h -- C ABI of libnvkv: attention over an NVFP4-quantised paged KV
 * cache on NVIDIA B200 (sm_100a).
 *
 * The storage format is the one stated in the "gzenz/ninfer" README, section
 * "Fork changes vs upstream", subsection "Context and model", NVFP4 KV cache
 * bullet: every KV element is a 4-bit E2M1 code and each group of 16
 * elements (here: 16 consecutive head_dim elements of one token and one
 * kv-head) shares one E4M3 scale.  The serving features the calls follow are
 * those listed in the "knoopx/ninfer" README, section "Capabilities and
 * limits": a single KV pool, sized at startup, serving every active request,
 * batched decode replayed from CUDA Graphs, MTP speculative verify with one
 * to five draft tokens (T = drafts + 1 causal queries per sequence), and
 * chunked prefill; one GPU.
 *
 * Conventions for every call
 *  - Every pointer named "device" is GPU memory owned by the caller; the
 *    library never allocates, frees, synchronises or reads device memory
 *    from the host.  Each call only enqueues kernels on `stream` (NULL = the
 *    legacy default stream) and returns, so every call can be captured in a
 *    CUDA Graph.
 *  - Host-checkable argument errors return NVKV_ERR_INVALID_ARG or
 *    NVKV_ERR_UNSUPPORTED before anything is launched; a failed launch
 *    returns NVKV_ERR_CUDA.
 *  - Device-resident metadata (page ids, lengths) is checked by the kernels:
 *    an out-of-range page id or length is skipped (nothing is read or
 *    written through it) and, when `err_word` is non-NULL, the matching
 *    NVKV_DEVERR_* bit is OR-ed into *err_word.  Kernels never trap.
 *  - bf16 tensors are row-major and contiguous, 16-byte aligned.
 *
 * Pool layout (this library's own; the pages do not fix one).  A page holds
 * 16 consecutive token slots of one sequence for every kv-head.  Page p starts
 * at pool + p * nvkv_page_bytes(Hkv, D); inside it, kv-head h owns the
 * 18*D-byte block at offset h*18*D:
 *   [0,     8D)  K codes  [16 slots][D/2]: byte i of a slot holds element 2i
 *                in its low nibble and element 2i+1 in its high nibble
 *   [8D,    9D)  K scales [16 slots][D/16]: byte g scales elements 16g..16g+15
 *   [9D,   17D)  V codes  [D][8]: byte (d, i) holds slot 2i in its low nibble
 *                and slot 2i+1 in its high nibble (V is stored transposed so a
 *                head_dim row of 16 tokens is 8 contiguous bytes)
 *   [17D,  18D)  V scales [D/16][16 slots]
 * A code is sign<<3 | magnitude index, magnitudes {0,.5,1,1.5,2,3,4,6};
 * value = E2M1(code) * E4M3(scale).  Quantisation of a group: scale = E4M3
 * nearest to amax/6 (ties to even, saturating at 448); code = E2M1 nearest
 * to x/scale (ties to even, saturating at 6); a scale of 0 gives all codes 0;
 * a magnitude that rounds to 0 is stored as code 0.
 */
#ifndef NVKV_H
#define NVKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st *nvkv_stream_t;

typedef enum nvkv_status {
    NVKV_OK = 0,
    NVKV_ERR_INVALID_ARG = 1,  /* null pointer, negative size, inconsistent shape */
    NVKV_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels implement */
    NVKV_ERR_WORKSPACE = 3,    /* workspace missing, too small or misaligned */
    NVKV_ERR_CUDA = 4          /* a kernel launch failed (cudaGetLastError) */
} nvkv_status;

/* Bits OR-ed into *err_word by the kernels. */
#define NVKV_DEVERR_PAGE_ID 1u   /* a page-table entry outside [0, num_pages) */
#define NVKV_DEVERR_LENGTH 2u    /* kv_len outside [rows or queries, max_kv_len] or
                                    beyond max_pages_per_seq * 16 */
#define NVKV_DEVERR_TIMEOUT 4u   /* a bounded wait inside a kernel gave up */

/* The paged pool. */
typedef struct nvkv_cache {
    uint8_t *pool;          /* device, num_pages * nvkv_page_bytes() bytes, 16-B aligned */
    int32_t num_pages;
    int32_t num_kv_heads;   /* Hkv >= 1 */
    int32_t head_dim;       /* D: 128 or 256 */
} nvkv_cache;

/* The batch of sequences a call works on. */
typedef struct nvkv_seqs {
    const int32_t *page_table;  /* device [batch][max_pages_per_seq]; entry i of
                                   row b is the page holding positions 16i..16i+15 */
    int32_t max_pages_per_seq;  /* row stride of page_table */
    const int32_t *kv_lens;     /* device [batch]: tokens in the cache of each
                                   sequence, INCLUDING the rows of this step */
    int32_t batch;              /* B >= 1 */
    int32_t max_kv_len;         /* host upper bound of kv_lens (sizes grids) */
    int32_t *err_word;          /* device int32 or NULL (see NVKV_DEVERR_*) */
} nvkv_seqs;

/* Bytes of one page: 18 * num_kv_heads * head_dim (4.5 bits per element).
 * Returns 0 for non-positive arguments. */
size_t nvkv_page_bytes(int32_t num_kv_heads, int32_t head_dim);

/* Quantise new K and V rows into the pool (the NVFP4 KV cache bullet above).
 *   k_new, v_new: device bf16 [total_new][Hkv][D].
 *   cu_new:       device int32 [batch+1], cu_new[0] = 0, non-decreasing;
 *                 rows cu_new[b] .. cu_new[b+1]-1 belong to sequence b and are
 *                 written to positions kv_lens[b]-n_b .. kv_lens[b]-1,
 *                 n_b = cu_new[b+1]-cu_new[b].
 *   total_new:    cu_new[batch] (host copy); max_new >= every n_b (host bound);
 *                 NVKV_ERR_UNSUPPORTED when (max_new/2 + 1) * Hkv * D/16
 *                 exceeds 2^31 - 1 (the kernels' 32-bit work-item index).
 * Writes exactly the code nibbles and scale bytes of those positions; every
 * other pool byte, including the other nibble of a shared V code byte, is
 * left as it was.  Sequences must not share pages written by the same call. */
nvkv_status nvkv_append(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *k_new,
                        const void *v_new, const int32_t *cu_new, int32_t total_new,
                        int32_t max_new, nvkv_stream_t stream);

/* Split-K ("flash-decoding") plan used by nvkv_decode_attn / nvkv_combine.
 *
 * The KV of every (sequence, kv-head) pair is cut into 128-token units; the
 * units of all pairs, ordered by (b, h, unit), are dealt to num_splits
 * contiguous, equal-sized (+-1 unit) ranges.  Range c writes one partial
 * result per pair it touches, into workspace slot c + b*Hkv + h, so a
 * workspace holds num_splits + batch*Hkv - 1 slots.  num_splits = 0 picks
 * the default for this GPU (a multiple of its SM count).
 *
 * nvkv_decode_workspace_bytes: bytes of workspace for T queries per
 * sequence (rows = T * Hq/Hkv per pair); 0 on invalid arguments. */
int32_t nvkv_default_num_splits(void);
size_t nvkv_decode_workspace_bytes(int32_t batch, int32_t T, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t head_dim, int32_t num_splits);

/* Host-side copy of the split plan, for inspection and tests: given host
 * kv_lens[batch], writes for every pair bh = b*Hkv + h the first and last
 * split touching it (first_split[bh] > last_split[bh] when the pair has no
 * KV).  Launches nothing. */
nvkv_status nvkv_split_plan(const int32_t *kv_lens_host, int32_t batch, int32_t num_kv_heads,
                            int32_t num_splits, int32_t *first_split, int32_t *last_split);

/* Decode / MTP-verify attention, first half: partial results per split.
 *   q: device bf16 [batch*T][Hq][D]; row b*T + t is query t of sequence b,
 *      at position kv_lens[b] - T + t, which sees keys 0 .. that position
 *      (causal).  Query head hq reads kv-head hq / (Hq/Hkv).
 *   T: 1 .. 16 queries per sequence; Hq a multiple of Hkv with T*Hq/Hkv <= 128.
 *   sm_scale: scores are sm_scale * q.k (typically 1/sqrt(D)).
 *   workspace: device, >= nvkv_decode_workspace_bytes(...), 16-B aligned.
 * nvkv_combine must follow with the same T, heads and num_splits.
 *
 * Arithmetic (which kernel runs: nvkv_decode_kernel_name).  Every kernel
 * uses the cached values exactly (E2M1 x E4M3 is exact in f16 and fp32),
 * base-2 scores x = q.k * sm_scale * log2(e), an fp32 running maximum, an
 * fp32 denominator that sums the same weights the value sum uses, fp32
 * accumulation of the value sums, and an fp32 partial result per split:
 *   decode_qk4 (D = 256, T*Hq/Hkv <= 6): the scores on the NVFP4
 *     block-scaled tensor-core MMA straight from the cached K codes and
 *     scales; q * sm_scale * log2(e) (fp32) enters as 8 stacked NVFP4
 *     terms after a power-of-two prescale of each row, leaving a remainder
 *     below about 1e-6 of each 16-element group's maximum, for any finite
 *     q; the products are exact and accumulate in fp32.  Weights
 *     p = 2^(x - m) from an fp32 exp2, rounded to f16 (relative error
 *     <= 2^-11; below 2^-14 f16 subnormals, absolute error <= 2^-25); the
 *     value sum is an f16 x f16 MMA with fp32 accumulation.
 *   decode_tc (D = 256, the other shapes with Hq/Hkv <= 48; more than 48
 *     query rows per (sequence, kv-head) run as one launch per chunk of
 *     queries, each reading the KV once): q * sm_scale * log2(e) (fp32) as
 *     two f16 terms hi + lo (about 22 significant bits; |q * sm_scale| must
 *     stay below about 45000, the f16 range, and elements below 2^-14 keep
 *     an absolute precision of 2^-25), K dequantised to f16, scores on the
 *     f16 MMA over both terms with fp32 accumulation; weights and value
 *     sum as for decode_qk4.
 *   decode_simt (head_dim 128, and NVKV_DECODE_KERNEL=simt): scores,
 *     weights and value sums in fp32 on CUDA cores. */
nvkv_status nvkv_decode_attn(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                             int32_t T, int32_t num_q_heads, float sm_scale, int32_t num_splits,
                             void *workspace, size_t workspace_bytes, nvkv_stream_t stream);

/* Name of the decode kernel nvkv_decode_attn launches for this cache and
 * step shape: "decode_qk4", "decode_tc" or "decode_simt" ("none" on invalid
 * arguments).  A static string; launches nothing.  The environment variable
 * NVKV_DECODE_KERNEL ("simt", or "tc" to skip decode_qk4) is read on every
 * call, as nvkv_decode_attn does. */
const char *nvkv_decode_kernel_name(const nvkv_cache *cache, int32_t T, int32_t num_q_heads);

/* Decode / MTP-verify attention, second half: merges the per-split partial
 * results (log-sum-exp weighting) into out, device bf16 [batch*T][Hq][D].
 * A query row that sees no key (kv_len < T - t) gets zeros. */
nvkv_status nvkv_combine(const nvkv_seqs *seqs, const void *workspace, int32_t T,
                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                         int32_t num_splits, void *out, nvkv_stream_t stream);

/* Decode / MTP-verify attention without a caller workspace: the same
 * computation as nvkv_decode_attn followed by nvkv_combine (same arguments,
 * same q / out layouts), with the split-K partial results kept in a
 * library-owned device array of nvkv_decode_static_scratch_bytes() bytes
 * (8 MiB) instead of caller memory.  The pages describe no such call; it is
 * here for callers that cannot call cudaMalloc or any other allocator where
 * they run attention: runtimes whose device memory belongs to a pool they
 * may not draw from, plugins inside an application that owns all device
 * memory, and real-time paths that must not take allocator locks or face an
 * allocation failure.  It allocates and frees nothing.
 *  - Every GPU that loads the library holds the 8 MiB array until the process
 *    exits.
 *  - out must be non-NULL and 16-byte aligned (NVKV_ERR_INVALID_ARG, checked
 *    before anything is launched).  Shapes whose
 *    nvkv_decode_workspace_bytes() exceeds the array return
 *    NVKV_ERR_WORKSPACE without launching.
 *  - The first call on each device (with that device current) looks up the
 *    array's device address (cudaGetSymbolAddress) and caches it for that
 *    device's CUDA context; a new context (after a device reset) gets a new
 *    lookup on its first call.  Make that first call before any stream
 *    capture.  NVKV_ERR_CUDA if the lookup fails.
 *  - All calls on a device share the one array, and it keeps the last call's
 *    contents (nothing needs to start at zero: every slot the merge reads is
 *    written by the same call first).  Calls whose kernels overlap on the GPU
 *    (different streams without ordering) race on it: order them on one
 *    stream or with events. */
size_t nvkv_decode_static_scratch_bytes(void);
nvkv_status nvkv_decode_attn_static(const nvkv_cache *cache, const nvkv_seqs *seqs,
                                    const void *q, int32_t T, int32_t num_q_heads,
                                    float sm_scale, int32_t num_splits, void *out,
                                    nvkv_stream_t stream);

/* Chunked-prefill attention ("knoopx/ninfer" README, "Capabilities and
 * limits": chunked prefill): causal attention of a chunk of new queries
 * against the whole cache of their sequence, whose K/V rows (including the
 * chunk's own) have already been appended.
 *   q:    device bf16 [total_q][Hq][D]; cu_q device int32 [batch+1]; rows
 *         cu_q[b] .. cu_q[b+1]-1 are the n_b newest positions of sequence b
 *         (kv_lens[b]-n_b .. kv_lens[b]-1).
 *   total_q = cu_q[batch] (host), max_q >= every n_b (host bound).
 *   out:  device bf16 [total_q][Hq][D].
 * Device-side: a page id outside the pool sets NVKV_DEVERR_PAGE_ID (its keys
 * read as absent); a kv_len beyond max_kv_len or the page table, or (on the
 * tensor-core kernel) a chunk reaching past total_q, sets
 * NVKV_DEVERR_LENGTH.  No row at or past total_q is ever written. */
nvkv_status nvkv_prefill_attn(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                              const int32_t *cu_q, int32_t total_q, int32_t max_q,
                              int32_t num_q_heads, float sm_scale, void *out,
                              nvkv_stream_t stream);

/* The same chunked prefill with each query tile's keys split into
 * num_splits equal runs of 64-key tiles, one CTA each, so that the grid of
 * tile CTAs fills the GPU's last wave (one CTA of the head_dim-256
 * tensor-core kernel per SM).  Every split leaves, per query row, its
 * softmax-normalised partial output O_s and lse_s = log2 of its sum of
 * weights (in the base-2 score scale), and a merge kernel writes
 * out = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M), M = max_s lse_s:
 * the log-sum-exp combination of partial softmax results, the same merge
 * the decode splits use (the result equals one pass up to fp32 rounding;
 * a row no split sees a key of is 0).
 *   num_splits: 0 = automatic -- the count in 1..8 whose CTAs fill their
 *               last wave best on this device, a larger count only where it
 *               raises that fill by more than 1 % (nvkv_prefill_num_splits
 *               tells which); 1..8 = that count; others
 *               NVKV_ERR_INVALID_ARG.
 *   workspace:  device, 16-byte aligned, caller-owned, at least
 *               nvkv_prefill_workspace_bytes(total_q, Hq, D, num_splits)
 *               bytes when the resolved count is above 1 (else unused, may
 *               be NULL); NVKV_ERR_WORKSPACE otherwise.  Layout: fp32
 *               [S][total_q][Hq][D] partial outputs, then (at a 256-byte
 *               boundary) fp32 [S][total_q][Hq] lse.  Its contents need no
 *               initialisation.
 * Shapes the tensor-core kernel does not take (head_dim 128), and
 * NVKV_DECODE_KERNEL=simt, run the CUDA-core kernel of nvkv_prefill_attn
 * and ignore the workspace.
 * nvkv_prefill_workspace_bytes: bytes for num_splits (0: for the largest
 * count the automatic choice takes, 8); 0 when no workspace is needed
 * (num_splits 1) and on invalid arguments.
 * nvkv_prefill_num_splits: the count num_splits = 0 resolves to for batch
 * sequences of at most max_q new queries (1 where the CUDA-core kernel
 * runs); 0 on invalid arguments. */
size_t nvkv_prefill_workspace_bytes(int32_t total_q, int32_t num_q_heads, int32_t head_dim,
                                    int32_t num_splits);
int32_t nvkv_prefill_num_splits(const nvkv_cache *cache, int32_t batch, int32_t max_q,
                                int32_t num_q_heads);
nvkv_status nvkv_prefill_attn_split(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                                    const int32_t *cu_q, int32_t total_q, int32_t max_q,
                                    int32_t num_q_heads, float sm_scale, int32_t num_splits,
                                    void *workspace, size_t workspace_bytes, void *out,
                                    nvkv_stream_t stream);

/* Rotary position embedding of K fused with the quantise-append: the YaRN
 * context extension of the "gzenz/ninfer" README, "Fork changes vs
 * upstream" -> "Context and model", stated there as linear RoPE scaling
 * (--rope-scaling-factor).  The pages fix no base, rotary width or pairing;
 * this library's reading: the first rotary_dim elements of each K head
 * rotate, element i paired with element i + rotary_dim/2, by the angle
 * (pos / scale) * base^(-2i / rotary_dim); V and the other elements are
 * stored unrotated (queries are rotated by the caller with the same table).
 *
 * nvkv_rope_table fills cs (device float [max_pos][rotary_dim/2][2], 8-byte
 * aligned) with (cos, sin) of those angles, computed in double and rounded
 * once to float.  rotary_dim > 0 and a multiple of 32; base, scale > 0.
 *
 * nvkv_append_rope is nvkv_append with each K row rotated at its position
 * by row pos of rope_cs (max_pos rows) before quantisation, in float:
 * x' = fma(x, c, -(y*s)), y' = fma(y, c, x*s) (products rounded to float).
 * 0 < rotary_dim <= head_dim, rotary_dim % 32 == 0.  A new row whose
 * position has no table row (pos >= max_pos) is not written (neither K nor
 * V) and sets NVKV_DEVERR_LENGTH. */
nvkv_status nvkv_rope_table(float *cs, int32_t max_pos, int32_t rotary_dim, double base,
                            double scale, nvkv_stream_t stream);
nvkv_status nvkv_append_rope(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *k_new,
                             const void *v_new, const int32_t *cu_new, int32_t total_new,
                             int32_t max_new, const float *rope_cs, int32_t max_pos,
                             int32_t rotary_dim, nvkv_stream_t stream);

/* Host KV spill and restore ("gzenz/ninfer" README, "Context cache and
 * eviction": when device KV runs out, evicted continuations move to a pinned
 * host arena and move back when their cache is reused; placement in the
 * arena is scatter-gather, so fragmentation never blocks a spill).
 *   arena: num_slots page-sized slots, nvkv_page_bytes(Hkv, D) bytes each
 *          (slot s at arena + s * page_bytes), 16-byte aligned, in pinned
 *          host memory (cudaHostAlloc / cudaHostRegister, e.g. a torch
 *          pin_memory tensor) or in device memory.  Pageable host memory is
 *          refused with NVKV_ERR_INVALID_ARG before anything is launched.
 *   nvkv_pages_spill:   pool page page_ids[i] -> arena slot slot_ids[i]
 *   nvkv_pages_restore: arena slot slot_ids[i] -> pool page page_ids[i]
 *          for i < n; a page moves whole (every kv-head), bit-exact.
 *   page_ids, slot_ids: int32 [n], device or pinned host memory, read by
 *          the kernel; a pair with an out-of-range id is skipped and sets
 *          NVKV_DEVERR_PAGE_ID in *err_word (device int, optional).  Pairs
 *          must not share a destination.
 * One kernel per call on `stream` (pinned host memory is read and written
 * through its device-visible address, no staging copy); n = 0 is a no-op. */
nvkv_status nvkv_pages_spill(const nvkv_cache *cache, const int32_t *page_ids,
                             const int32_t *slot_ids, int32_t n, void *arena, int64_t num_slots,
                             int32_t *err_word, nvkv_stream_t stream);
nvkv_status nvkv_pages_restore(const nvkv_cache *cache, const int32_t *page_ids,
                               const int32_t *slot_ids, int32_t n, const void *arena,
                               int64_t num_slots, int32_t *err_word, nvkv_stream_t stream);

/* K8V4 cache: 8-bit K, NVFP4 V.  The "knoopx/ninfer" README, "Capabilities
 * and limits", lists K8V4 among its KV storage formats and its note on the
 * published measurements names an E4M3 "row-256" KV; the pages fix no
 * layout.  This library's reading: K rows in E4M3 with one fp32 scale per
 * row of one token and one kv-head, V exactly as in the NVFP4 cache.
 *   K scale = amax / 448 in fp32 (round to nearest even); K code = the E4M3
 *   value nearest to x / scale computed in fp32 (ties to the even mantissa,
 *   saturating at 448); an all-zero row has scale 0 and codes 0; a
 *   magnitude that rounds to 0 is stored as 0x00.  Value = E4M3(code) * scale.
 * Page layout: page p starts at pool + p * nvkv_k8v4_page_bytes(Hkv, D);
 * kv-head h owns the (25*D + 64)-byte block at offset h * (25*D + 64):
 *   [0,        16D)     K codes  [16 slots][D], one E4M3 byte per element
 *   [16D,      16D+64)  K scales [16 slots], fp32 little-endian
 *   [16D+64,   24D+64)  V codes  [D][8], as the NVFP4 V codes
 *   [24D+64,   25D+64)  V scales [D/16][16 slots], as the NVFP4 V scales
 * A K8V4 cache is an nvkv_cache whose pool holds num_pages *
 * nvkv_k8v4_page_bytes() bytes; it is used only with the *_k8v4 calls
 * (the other calls read and write the NVFP4 layout).  Each call below has
 * the arguments, layouts, checks and error behaviour of its NVFP4
 * counterpart:
 *   nvkv_append_k8v4       ~ nvkv_append
 *   nvkv_decode_attn_k8v4  ~ nvkv_decode_attn (same workspace size and
 *                            split plan; merge with nvkv_combine)
 *   nvkv_prefill_attn_k8v4 ~ nvkv_prefill_attn
 *   nvkv_pages_spill_k8v4, nvkv_pages_restore_k8v4 ~ nvkv_pages_spill,
 *                            nvkv_pages_restore, with arena slots of
 *                            nvkv_k8v4_page_bytes() bytes
 * nvkv_decode_attn_k8v4 runs the decode_qk4 pipeline over this layout for
 * head_dim 256 and T*Hq/Hkv <= 6: the scores on the E4M3 tensor-core MMA
 * (kind::f8f6f4) straight from the cached K bytes, q * sm_scale * log2(e)
 * entering as 8 stacked E4M3 terms after a power-of-two prescale of each
 * row (term l weighted 2^-4l; remainder below 2^-28 of the row maximum),
 * times each token's fp32 row scale in fp32; weights and value sum as for
 * the NVFP4 cache.  Other decode shapes and the prefill run on CUDA cores
 * (one warp per query row).  nvkv_decode_kernel_name_k8v4 names the kernel
 * ("decode_qk4_k8v4" or "decode_simt"; "none" on invalid arguments).
 * nvkv_k8v4_page_bytes returns 0 for non-positive arguments. */
size_t nvkv_k8v4_page_bytes(int32_t num_kv_heads, int32_t head_dim);
nvkv_status nvkv_append_k8v4(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *k_new,
                             const void *v_new, const int32_t *cu_new, int32_t total_new,
                             int32_t max_new, nvkv_stream_t stream);
nvkv_status nvkv_decode_attn_k8v4(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                                  int32_t T, int32_t num_q_heads, float sm_scale,
                                  int32_t num_splits, void *workspace, size_t workspace_bytes,
                                  nvkv_stream_t stream);
const char *nvkv_decode_kernel_name_k8v4(const nvkv_cache *cache, int32_t T,
                                         int32_t num_q_heads);
nvkv_status nvkv_prefill_attn_k8v4(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                                   const int32_t *cu_q, int32_t total_q, int32_t max_q,
                                   int32_t num_q_heads, float sm_scale, void *out,
                                   nvkv_stream_t stream);
nvkv_status nvkv_pages_spill_k8v4(const nvkv_cache *cache, const int32_t *page_ids,
                                  const int32_t *slot_ids, int32_t n, void *arena,
                                  int64_t num_slots, int32_t *err_word, nvkv_stream_t stream);
nvkv_status nvkv_pages_restore_k8v4(const nvkv_cache *cache, const int32_t *page_ids,
                                    const int32_t *slot_ids, int32_t n, const void *arena,
                                    int64_t num_slots, int32_t *err_word, nvkv_stream_t stream);

/* Static description of a status code. */
const char *nvkv_status_string(nvkv_status status);

#ifdef __cplusplus
}
#endif

#endif /* NVKV_H */
