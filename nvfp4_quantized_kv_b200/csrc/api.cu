// api.cu -- the extern "C" boundary of libnvkv (declared in include/nvkv.h):
// host-side argument checks, workspace carving and kernel dispatch.  Nothing
// here allocates, synchronises or reads device memory.
#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "nvkv_common.cuh"

namespace nvkv {
cudaError_t launch_append(const nvkv_cache &, const nvkv_seqs &, const void *, const void *,
                          const int32_t *, int, int, const float *, int, int, cudaStream_t);
cudaError_t launch_rope_table(float *, int, int, double, double, cudaStream_t);
cudaError_t launch_append_k8v4(const nvkv_cache &, const nvkv_seqs &, const void *, const void *,
                               const int32_t *, int, int, cudaStream_t);
cudaError_t launch_decode_simt(const nvkv_cache &, const nvkv_seqs &, const void *, int, int,
                               float, int, float *, float *, cudaStream_t, bool);
bool decode_tc_supported(const nvkv_cache &, int, int);
bool decode_qk4_supported(const nvkv_cache &, int, int);
cudaError_t launch_decode_qk4(const nvkv_cache &, const nvkv_seqs &, const void *, int, int, float,
                              int, float *, float *, cudaStream_t);
cudaError_t launch_decode_qk4_k8v4(const nvkv_cache &, const nvkv_seqs &, const void *, int, int,
                                   float, int, float *, float *, cudaStream_t);
cudaError_t launch_decode_tc(const nvkv_cache &, const nvkv_seqs &, const void *, int, int, float,
                             int, float *, float *, cudaStream_t);
bool prefill_tc_supported(const nvkv_cache &);
cudaError_t launch_prefill_tc(const nvkv_cache &, const nvkv_seqs &, const void *, const int32_t *,
                              int, int, int, float, void *, int, float *, float *, cudaStream_t);
int prefill_max_splits();
int prefill_auto_splits(int64_t, int);
int prefill_tc_items(const nvkv_cache &, const nvkv_seqs &, int, int);
cudaError_t launch_combine(const nvkv_seqs &, const void *, const void *, int, int, int, int, int,
                           void *, cudaStream_t);
cudaError_t launch_prefill_simt(const nvkv_cache &, const nvkv_seqs &, const void *,
                                const int32_t *, int, int, float, void *, cudaStream_t, bool);
cudaError_t launch_page_copy(const uint8_t *, int64_t, uint8_t *, int64_t, const int32_t *,
                             const int32_t *, int, int64_t, int32_t *, cudaStream_t);
}  // namespace nvkv

using namespace nvkv;

namespace {

constexpr int kMaxT = 16;
constexpr int kMaxRows = 128;  // T * Hq / Hkv per (sequence, kv-head)

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

nvkv_status check_cache(const nvkv_cache *c) {
  if (!c || !c->pool || !aligned16(c->pool)) return NVKV_ERR_INVALID_ARG;
  if (c->num_pages <= 0 || c->num_kv_heads <= 0) return NVKV_ERR_INVALID_ARG;
  if (c->head_dim != 128 && c->head_dim != 256) return NVKV_ERR_UNSUPPORTED;
  return NVKV_OK;
}

nvkv_status check_seqs(const nvkv_seqs *s) {
  if (!s || !s->page_table || !s->kv_lens) return NVKV_ERR_INVALID_ARG;
  if (s->batch <= 0 || s->max_pages_per_seq <= 0 || s->max_kv_len < 0) return NVKV_ERR_INVALID_ARG;
  if ((int64_t)s->max_kv_len > (int64_t)s->max_pages_per_seq * kPageTokens)
    return NVKV_ERR_INVALID_ARG;
  return NVKV_OK;
}

nvkv_status check_heads(int Hq, int Hkv, int D, int T) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return NVKV_ERR_INVALID_ARG;
  if (D != 128 && D != 256) return NVKV_ERR_UNSUPPORTED;
  if (T <= 0) return NVKV_ERR_INVALID_ARG;
  if (T > kMaxT || (int64_t)T * (Hq / Hkv) > kMaxRows) return NVKV_ERR_UNSUPPORTED;
  return NVKV_OK;
}

int resolve_splits(int num_splits) {
  return num_splits > 0 ? num_splits : nvkv_default_num_splits();
}

struct WorkspaceLayout {
  size_t o_bytes, lse_off, total;
};

WorkspaceLayout layout(int batch, int T, int Hq, int Hkv, int D, int S) {
  const size_t R = (size_t)T * (Hq / Hkv);
  const size_t slots = (size_t)S + (size_t)batch * Hkv - 1;
  WorkspaceLayout w;
  w.o_bytes = align256(slots * R * D * sizeof(float));
  w.lse_off = w.o_bytes;
  w.total = w.o_bytes + align256(slots * R * sizeof(float));
  return w;
}

nvkv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVKV_OK : NVKV_ERR_CUDA; }

// The address through which a kernel reaches p: device (or managed) memory
// as it is, pinned host memory through its mapped device address; nullptr
// for anything a kernel cannot touch (pageable host memory, unknown).
const void *device_view(const void *p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // clear the (non-sticky) error of the failed query
    return nullptr;
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return p;
  if (a.type == cudaMemoryTypeHost) return a.devicePointer;
  return nullptr;
}

// pb: bytes of one page of the cache's format.
nvkv_status pages_move(const nvkv_cache *cache, const int32_t *page_ids, const int32_t *slot_ids,
                       int32_t n, const void *arena, int64_t num_slots, int32_t *err_word,
                       nvkv_stream_t stream, bool spill, bool k8) {
  const nvkv_status st = check_cache(cache);
  if (st != NVKV_OK) return st;
  if (n < 0 || num_slots <= 0 || !page_ids || !slot_ids || !arena || !aligned16(arena))
    return NVKV_ERR_INVALID_ARG;
  if (n == 0) return NVKV_OK;
  const void *pid = device_view(page_ids), *sid = device_view(slot_ids), *ar = device_view(arena);
  if (!pid || !sid || !ar || !aligned16(ar)) return NVKV_ERR_INVALID_ARG;
  const int64_t pb = (int64_t)(k8 ? nvkv_k8v4_page_bytes(cache->num_kv_heads, cache->head_dim)
                                  : nvkv_page_bytes(cache->num_kv_heads, cache->head_dim));
  uint8_t *pool = cache->pool;
  uint8_t *arena_b = const_cast<uint8_t *>(static_cast<const uint8_t *>(ar));
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int32_t *p32 = static_cast<const int32_t *>(pid), *s32 = static_cast<const int32_t *>(sid);
  return cuda_status(spill ? launch_page_copy(pool, cache->num_pages, arena_b, num_slots, p32, s32,
                                              n, pb, err_word, s)
                           : launch_page_copy(arena_b, num_slots, pool, cache->num_pages, s32,
                                              p32, n, pb, err_word, s));
}


// The append kernels index their work items (slot pair, kv-head, group of
// 16) with 32-bit integers: max_new/2 + 1 pairs times Hkv * D/16 items
// must fit.
bool append_fits(const nvkv_cache &c, int32_t max_new) {
  return ((int64_t)max_new / 2 + 1) * c.num_kv_heads * (c.head_dim / kGroup) <= INT32_MAX;
}

// Checks shared by the decode entry points of both cache formats; on
// success `a` holds the resolved split count and the workspace regions.
struct DecodeArgs {
  int S = 0;
  float *ws_o = nullptr, *ws_lse = nullptr;
};

nvkv_status check_decode(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q, int32_t T,
                         int32_t num_q_heads, float sm_scale, int32_t num_splits, void *workspace,
                         size_t workspace_bytes, DecodeArgs &a) {
  nvkv_status st = check_cache(cache);
  if (st != NVKV_OK) return st;
  if ((st = check_seqs(seqs)) != NVKV_OK) return st;
  if ((st = check_heads(num_q_heads, cache->num_kv_heads, cache->head_dim, T)) != NVKV_OK) return st;
  if (!q || !aligned16(q) || !std::isfinite(sm_scale) || num_splits < 0) return NVKV_ERR_INVALID_ARG;
  a.S = resolve_splits(num_splits);
  const WorkspaceLayout w = layout(seqs->batch, T, num_q_heads, cache->num_kv_heads,
                                   cache->head_dim, a.S);
  if (!workspace || !aligned16(workspace) || workspace_bytes < w.total) return NVKV_ERR_WORKSPACE;
  a.ws_o = static_cast<float *>(workspace);
  a.ws_lse = reinterpret_cast<float *>(static_cast<char *>(workspace) + w.lse_off);
  return NVKV_OK;
}

// Checks shared by the prefill entry points (NVKV_OK with total_q == 0
// means there is nothing to launch).
nvkv_status check_prefill(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                          const int32_t *cu_q, int32_t total_q, int32_t max_q,
                          int32_t num_q_heads, float sm_scale, const void *out) {
  nvkv_status st = check_cache(cache);
  if (st != NVKV_OK) return st;
  if ((st = check_seqs(seqs)) != NVKV_OK) return st;
  if (num_q_heads <= 0 || num_q_heads % cache->num_kv_heads != 0) return NVKV_ERR_INVALID_ARG;
  if (total_q < 0 || max_q < 0 || !std::isfinite(sm_scale)) return NVKV_ERR_INVALID_ARG;
  if (total_q == 0) return NVKV_OK;
  if (!q || !cu_q || !out || !aligned16(q) || !aligned16(out)) return NVKV_ERR_INVALID_ARG;
  return NVKV_OK;
}

// Workspace of the key-split prefill: S planes of total_q * Hq rows, the
// rows' O / l (fp32, head_dim each) and then their lse (fp32).
struct PrefillLayout {
  size_t lse_off, total;
};
PrefillLayout prefill_layout(int64_t total_q, int Hq, int D, int S) {
  const size_t rows = (size_t)total_q * Hq * S;
  const size_t lse_off = align256(rows * D * sizeof(float));
  return {lse_off, lse_off + align256(rows * sizeof(float))};
}

// NVKV_DECODE_KERNEL=simt forces the CUDA-core decode and prefill kernels;
// NVKV_DECODE_KERNEL=tc forces the decode kernel that dequantises K for
// the f16 tensor-core scores (where it takes the shape).  The tests use
// them to cross-check the kernel families on the same shapes.
bool force_kernel(const char *name) {
  const char *v = std::getenv("NVKV_DECODE_KERNEL");
  return v && std::strcmp(v, name) == 0;
}
bool force_simt() { return force_kernel("simt"); }

}  // namespace

extern "C" {

size_t nvkv_page_bytes(int32_t num_kv_heads, int32_t head_dim) {
  if (num_kv_heads <= 0 || head_dim <= 0) return 0;
  return (size_t)18 * num_kv_heads * head_dim;
}

int32_t nvkv_default_num_splits(void) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();  // the failed query leaves a (non-sticky) error; clear it
    sms = 148;           // B200
  }
  return sms;
}

size_t nvkv_decode_workspace_bytes(int32_t batch, int32_t T, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t head_dim, int32_t num_splits) {
  if (batch <= 0 || num_splits < 0) return 0;
  if (check_heads(num_q_heads, num_kv_heads, head_dim, T) != NVKV_OK) return 0;
  return layout(batch, T, num_q_heads, num_kv_heads, head_dim, resolve_splits(num_splits)).total;
}

nvkv_status nvkv_split_plan(const int32_t *kv_lens_host, int32_t batch, int32_t num_kv_heads,
                            int32_t num_splits, int32_t *first_split, int32_t *last_split) {
  if (!kv_lens_host || !first_split || !last_split || batch <= 0 || num_kv_heads <= 0 ||
      num_splits < 0)
    return NVKV_ERR_INVALID_ARG;
  const int64_t S = resolve_splits(num_splits);
  int64_t U = 0;
  for (int b = 0; b < batch; ++b) {
    if (kv_lens_host[b] < 0) return NVKV_ERR_INVALID_ARG;
    U += (int64_t)units_of_len(kv_lens_host[b]) * num_kv_heads;
  }
  int64_t start = 0;
  for (int b = 0; b < batch; ++b) {
    const int ub = units_of_len(kv_lens_host[b]);
    for (int h = 0; h < num_kv_heads; ++h) {
      const int bh = b * num_kv_heads + h;
      if (ub == 0) {
        first_split[bh] = 0;
        last_split[bh] = -1;
      } else {
        first_split[bh] = (int32_t)range_of_unit(start, U, S);
        last_split[bh] = (int32_t)range_of_unit(start + ub - 1, U, S);
      }
      start += ub;
    }
  }
  return NVKV_OK;
}

nvkv_status nvkv_append(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *k_new,
                        const void *v_new, const int32_t *cu_new, int32_t total_new,
                        int32_t max_new, nvkv_stream_t stream) {
  nvkv_status st = check_cache(cache);
  if (st != NVKV_OK) return st;
  if ((st = check_seqs(seqs)) != NVKV_OK) return st;
  if (total_new < 0 || max_new < 0) return NVKV_ERR_INVALID_ARG;
  if (total_new == 0 || max_new == 0) return NVKV_OK;
  if (!k_new || !v_new || !cu_new || !aligned16(k_new) || !aligned16(v_new))
    return NVKV_ERR_INVALID_ARG;
  if (!append_fits(*cache, max_new)) return NVKV_ERR_UNSUPPORTED;
  return cuda_status(launch_append(*cache, *seqs, k_new, v_new, cu_new, total_new, max_new,
                                   nullptr, 0, 0, reinterpret_cast<cudaStream_t>(stream)));
}

nvkv_status nvkv_rope_table(float *cs, int32_t max_pos, int32_t rotary_dim, double base,
                            double scale, nvkv_stream_t stream) {
  if (!cs || (reinterpret_cast<uintptr_t>(cs) & 7u) || max_pos <= 0 || rotary_dim <= 0 ||
      rotary_dim % 32 != 0 || !(base > 0.0) || !(scale > 0.0) || !std::isfinite(base) ||
      !std::isfinite(scale))
    return NVKV_ERR_INVALID_ARG;
  return cuda_status(launch_rope_table(cs, max_pos, rotary_dim, base, scale,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

nvkv_status nvkv_append_rope(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *k_new,
                             const void *v_new, const int32_t *cu_new, int32_t total_new,
                             int32_t max_new, const float *rope_cs, int32_t max_pos,
                             int32_t rotary_dim, nvkv_stream_t stream) {
  nvkv_status st = check_cache(cache);
  if (st != NVKV_OK) return st;
  if ((st = check_seqs(seqs)) != NVKV_OK) return st;
  if (total_new < 0 || max_new < 0) return NVKV_ERR_INVALID_ARG;
  if (!rope_cs || (reinterpret_cast<uintptr_t>(rope_cs) & 7u) || max_pos <= 0 ||
      rotary_dim <= 0 || rotary_dim % 32 != 0 || rotary_dim > cache->head_dim)
    return NVKV_ERR_INVALID_ARG;
  if (total_new == 0 || max_new == 0) return NVKV_OK;
  if (!k_new || !v_new || !cu_new || !aligned16(k_new) || !aligned16(v_new))
    return NVKV_ERR_INVALID_ARG;
  if (!append_fits(*cache, max_new)) return NVKV_ERR_UNSUPPORTED;
  return cuda_status(launch_append(*cache, *seqs, k_new, v_new, cu_new, total_new, max_new,
                                   rope_cs, rotary_dim, max_pos,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

const char *nvkv_decode_kernel_name(const nvkv_cache *cache, int32_t T, int32_t num_q_heads) {
  if (!cache || cache->num_kv_heads <= 0 || T <= 0 || num_q_heads <= 0 ||
      num_q_heads % cache->num_kv_heads != 0)
    return "none";
  if (!force_simt() && !force_kernel("tc") && decode_qk4_supported(*cache, T, num_q_heads))
    return "decode_qk4";
  if (!force_simt() && decode_tc_supported(*cache, T, num_q_heads)) return "decode_tc";
  return "decode_simt";
}

nvkv_status nvkv_decode_attn(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                             int32_t T, int32_t num_q_heads, float sm_scale, int32_t num_splits,
                             void *workspace, size_t workspace_bytes, nvkv_stream_t stream) {
  DecodeArgs a;
  const nvkv_status st = check_decode(cache, seqs, q, T, num_q_heads, sm_scale, num_splits,
                                      workspace, workspace_bytes, a);
  if (st != NVKV_OK) return st;
  cudaStream_t st_ = reinterpret_cast<cudaStream_t>(stream);
  if (!force_simt() && !force_kernel("tc") && decode_qk4_supported(*cache, T, num_q_heads))
    return cuda_status(
        launch_decode_qk4(*cache, *seqs, q, T, num_q_heads, sm_scale, a.S, a.ws_o, a.ws_lse, st_));
  if (!force_simt() && decode_tc_supported(*cache, T, num_q_heads))
    return cuda_status(
        launch_decode_tc(*cache, *seqs, q, T, num_q_heads, sm_scale, a.S, a.ws_o, a.ws_lse, st_));
  return cuda_status(launch_decode_simt(*cache, *seqs, q, T, num_q_heads, sm_scale, a.S, a.ws_o,
                                        a.ws_lse, st_, false));
}

nvkv_status nvkv_combine(const nvkv_seqs *seqs, const void *workspace, int32_t T,
                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                         int32_t num_splits, void *out, nvkv_stream_t stream) {
  nvkv_status st = check_seqs(seqs);
  if (st != NVKV_OK) return st;
  if ((st = check_heads(num_q_heads, num_kv_heads, head_dim, T)) != NVKV_OK) return st;
  if (!out || !aligned16(out) || num_splits < 0) return NVKV_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace)) return NVKV_ERR_WORKSPACE;
  const int S = resolve_splits(num_splits);
  const WorkspaceLayout w = layout(seqs->batch, T, num_q_heads, num_kv_heads, head_dim, S);
  const void *ws_lse = static_cast<const char *>(workspace) + w.lse_off;
  return cuda_status(launch_combine(*seqs, workspace, ws_lse, T, num_q_heads, num_kv_heads,
                                    head_dim, S, out, reinterpret_cast<cudaStream_t>(stream)));
}

nvkv_status nvkv_prefill_attn(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                              const int32_t *cu_q, int32_t total_q, int32_t max_q,
                              int32_t num_q_heads, float sm_scale, void *out,
                              nvkv_stream_t stream) {
  const nvkv_status st =
      check_prefill(cache, seqs, q, cu_q, total_q, max_q, num_q_heads, sm_scale, out);
  if (st != NVKV_OK || total_q == 0) return st;
  cudaStream_t st_ = reinterpret_cast<cudaStream_t>(stream);
  if (!force_simt() && prefill_tc_supported(*cache))
    return cuda_status(launch_prefill_tc(*cache, *seqs, q, cu_q, total_q, max_q, num_q_heads,
                                         sm_scale, out, 1, nullptr, nullptr, st_));
  return cuda_status(launch_prefill_simt(*cache, *seqs, q, cu_q, total_q, num_q_heads, sm_scale,
                                         out, st_, false));
}

size_t nvkv_prefill_workspace_bytes(int32_t total_q, int32_t num_q_heads, int32_t head_dim,
                                    int32_t num_splits) {
  if (total_q < 0 || num_q_heads <= 0 || head_dim <= 0 || num_splits < 0 ||
      num_splits > prefill_max_splits())
    return 0;
  const int S = num_splits == 0 ? prefill_max_splits() : num_splits;
  return S > 1 ? prefill_layout(total_q, num_q_heads, head_dim, S).total : 0;
}

int32_t nvkv_prefill_num_splits(const nvkv_cache *cache, int32_t batch, int32_t max_q,
                                int32_t num_q_heads) {
  if (check_cache(cache) != NVKV_OK || batch <= 0 || max_q < 0 || num_q_heads <= 0 ||
      num_q_heads % cache->num_kv_heads != 0)
    return 0;
  if (force_simt() || !prefill_tc_supported(*cache)) return 1;
  nvkv_seqs s{};
  s.batch = batch;
  return prefill_auto_splits(prefill_tc_items(*cache, s, max_q, num_q_heads),
                             nvkv_default_num_splits());
}

nvkv_status nvkv_prefill_attn_split(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                                    const int32_t *cu_q, int32_t total_q, int32_t max_q,
                                    int32_t num_q_heads, float sm_scale, int32_t num_splits,
                                    void *workspace, size_t workspace_bytes, void *out,
                                    nvkv_stream_t stream) {
  const nvkv_status st =
      check_prefill(cache, seqs, q, cu_q, total_q, max_q, num_q_heads, sm_scale, out);
  if (st != NVKV_OK) return st;
  if (num_splits < 0 || num_splits > prefill_max_splits()) return NVKV_ERR_INVALID_ARG;
  if (total_q == 0) return NVKV_OK;
  cudaStream_t st_ = reinterpret_cast<cudaStream_t>(stream);
  if (force_simt() || !prefill_tc_supported(*cache))
    return cuda_status(launch_prefill_simt(*cache, *seqs, q, cu_q, total_q, num_q_heads, sm_scale,
                                           out, st_, false));
  const int S = num_splits > 0 ? num_splits
                               : prefill_auto_splits(
                                     prefill_tc_items(*cache, *seqs, max_q, num_q_heads),
                                     nvkv_default_num_splits());
  float *ws_o = nullptr, *ws_lse = nullptr;
  if (S > 1) {
    const PrefillLayout w = prefill_layout(total_q, num_q_heads, cache->head_dim, S);
    if (!workspace || !aligned16(workspace) || workspace_bytes < w.total)
      return NVKV_ERR_WORKSPACE;
    ws_o = static_cast<float *>(workspace);
    ws_lse = reinterpret_cast<float *>(static_cast<char *>(workspace) + w.lse_off);
  }
  return cuda_status(launch_prefill_tc(*cache, *seqs, q, cu_q, total_q, max_q, num_q_heads,
                                       sm_scale, out, S, ws_o, ws_lse, st_));
}

size_t nvkv_k8v4_page_bytes(int32_t num_kv_heads, int32_t head_dim) {
  if (num_kv_heads <= 0 || head_dim <= 0) return 0;
  return (size_t)num_kv_heads * (25 * (size_t)head_dim + 64);
}

nvkv_status nvkv_append_k8v4(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *k_new,
                             const void *v_new, const int32_t *cu_new, int32_t total_new,
                             int32_t max_new, nvkv_stream_t stream) {
  nvkv_status st = check_cache(cache);
  if (st != NVKV_OK) return st;
  if ((st = check_seqs(seqs)) != NVKV_OK) return st;
  if (total_new < 0 || max_new < 0) return NVKV_ERR_INVALID_ARG;
  if (total_new == 0 || max_new == 0) return NVKV_OK;
  if (!k_new || !v_new || !cu_new || !aligned16(k_new) || !aligned16(v_new))
    return NVKV_ERR_INVALID_ARG;
  if (!append_fits(*cache, max_new)) return NVKV_ERR_UNSUPPORTED;
  return cuda_status(launch_append_k8v4(*cache, *seqs, k_new, v_new, cu_new, total_new, max_new,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

nvkv_status nvkv_decode_attn_k8v4(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                                  int32_t T, int32_t num_q_heads, float sm_scale,
                                  int32_t num_splits, void *workspace, size_t workspace_bytes,
                                  nvkv_stream_t stream) {
  DecodeArgs a;
  const nvkv_status st = check_decode(cache, seqs, q, T, num_q_heads, sm_scale, num_splits,
                                      workspace, workspace_bytes, a);
  if (st != NVKV_OK) return st;
  cudaStream_t st_ = reinterpret_cast<cudaStream_t>(stream);
  if (!force_simt() && decode_qk4_supported(*cache, T, num_q_heads))
    return cuda_status(launch_decode_qk4_k8v4(*cache, *seqs, q, T, num_q_heads, sm_scale, a.S,
                                              a.ws_o, a.ws_lse, st_));
  return cuda_status(launch_decode_simt(*cache, *seqs, q, T, num_q_heads, sm_scale, a.S, a.ws_o,
                                        a.ws_lse, st_, true));
}

const char *nvkv_decode_kernel_name_k8v4(const nvkv_cache *cache, int32_t T,
                                         int32_t num_q_heads) {
  if (!cache || cache->num_kv_heads <= 0 || T <= 0 || num_q_heads <= 0 ||
      num_q_heads % cache->num_kv_heads != 0)
    return "none";
  if (!force_simt() && decode_qk4_supported(*cache, T, num_q_heads)) return "decode_qk4_k8v4";
  return "decode_simt";
}

nvkv_status nvkv_prefill_attn_k8v4(const nvkv_cache *cache, const nvkv_seqs *seqs, const void *q,
                                   const int32_t *cu_q, int32_t total_q, int32_t max_q,
                                   int32_t num_q_heads, float sm_scale, void *out,
                                   nvkv_stream_t stream) {
  const nvkv_status st =
      check_prefill(cache, seqs, q, cu_q, total_q, max_q, num_q_heads, sm_scale, out);
  if (st != NVKV_OK || total_q == 0) return st;
  return cuda_status(launch_prefill_simt(*cache, *seqs, q, cu_q, total_q, num_q_heads, sm_scale,
                                         out, reinterpret_cast<cudaStream_t>(stream), true));
}

nvkv_status nvkv_pages_spill(const nvkv_cache *cache, const int32_t *page_ids,
                             const int32_t *slot_ids, int32_t n, void *arena, int64_t num_slots,
                             int32_t *err_word, nvkv_stream_t stream) {
  return pages_move(cache, page_ids, slot_ids, n, arena, num_slots, err_word, stream, true, false);
}

nvkv_status nvkv_pages_restore(const nvkv_cache *cache, const int32_t *page_ids,
                               const int32_t *slot_ids, int32_t n, const void *arena,
                               int64_t num_slots, int32_t *err_word, nvkv_stream_t stream) {
  return pages_move(cache, page_ids, slot_ids, n, arena, num_slots, err_word, stream, false,
                    false);
}

nvkv_status nvkv_pages_spill_k8v4(const nvkv_cache *cache, const int32_t *page_ids,
                                  const int32_t *slot_ids, int32_t n, void *arena,
                                  int64_t num_slots, int32_t *err_word, nvkv_stream_t stream) {
  return pages_move(cache, page_ids, slot_ids, n, arena, num_slots, err_word, stream, true, true);
}

nvkv_status nvkv_pages_restore_k8v4(const nvkv_cache *cache, const int32_t *page_ids,
                                    const int32_t *slot_ids, int32_t n, const void *arena,
                                    int64_t num_slots, int32_t *err_word, nvkv_stream_t stream) {
  return pages_move(cache, page_ids, slot_ids, n, arena, num_slots, err_word, stream, false, true);
}

const char *nvkv_status_string(nvkv_status status) {
  switch (status) {
    case NVKV_OK: return "ok";
    case NVKV_ERR_INVALID_ARG: return "invalid argument";
    case NVKV_ERR_UNSUPPORTED: return "unsupported shape";
    case NVKV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case NVKV_ERR_CUDA: return "CUDA launch error";
  }
  return "unknown status";
}

}  // extern "C"
