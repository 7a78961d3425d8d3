// decode_static.cu -- nvkv_decode_attn_static: decode / MTP-verify attention
// (split-K partials + combine) whose split-K scratch lives in a fixed,
// library-owned device array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot call cudaMalloc (or any allocator) at
// the point where they run attention -- runtimes whose device memory belongs
// to another pool or allocator they may not draw from, plugins hosted by an
// application that owns all device memory, and real-time paths that must not
// take allocator locks or risk an allocation failure.  They pass only inputs
// and outputs.
//
// The scratch is one file-scope __device__ array of kStaticScratchBytes.
// Host code cannot use the array's name as a device address (it names a
// host-side stand-in), so the address is looked up with cudaGetSymbolAddress
// with the device current: once per device and CUDA context, on the first
// call made in that context, and cached.  The cache is keyed by the
// context's unique id, so a context torn down and recreated (a device reset)
// gets a fresh lookup instead of a stale address.
#include <cuda.h>

#include <mutex>

#include "nvkv_common.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct ScratchSlot {
  void *addr = nullptr;
  unsigned long long ctx_id = 0;
  bool keyed = false;  // ctx_id is valid
};

std::mutex g_mutex;
ScratchSlot g_slot[kMaxDevices];

template <class Fn>
Fn driver_fn(const char *name) {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return reinterpret_cast<Fn>(p);
}

// Unique id of the current CUDA context (false when there is none yet or the
// driver cannot tell).
bool current_ctx_id(unsigned long long *id) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current device's context, or
// NULL when the lookup fails.
void *scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  std::lock_guard<std::mutex> lock(g_mutex);
  ScratchSlot &s = g_slot[dev];
  if (s.addr && s.keyed && have_id && s.ctx_id == id) return s.addr;
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
    cudaGetLastError();  // leave no error behind for the caller's next call
    s = ScratchSlot();
    return nullptr;
  }
  // The lookup made the device's context current if it was not yet.
  s.addr = p;
  s.keyed = current_ctx_id(&s.ctx_id);
  return p;
}

}  // namespace

extern "C" {

size_t nvkv_decode_static_scratch_bytes(void) { return kStaticScratchBytes; }

nvkv_status nvkv_decode_attn_static(const nvkv_cache *cache, const nvkv_seqs *seqs,
                                    const void *q, int32_t T, int32_t num_q_heads,
                                    float sm_scale, int32_t num_splits, void *out,
                                    nvkv_stream_t stream) {
  if (!cache || !seqs) return NVKV_ERR_INVALID_ARG;
  // out is only written by the merge, after the partials kernel: reject a bad
  // one before anything is launched.
  if (!out || (reinterpret_cast<uintptr_t>(out) & 15u)) return NVKV_ERR_INVALID_ARG;
  const size_t need = nvkv_decode_workspace_bytes(seqs->batch, T, num_q_heads,
                                                  cache->num_kv_heads, cache->head_dim,
                                                  num_splits);
  if (need == 0) {
    // Same argument checks as nvkv_decode_attn, without touching the scratch.
    return nvkv_decode_attn(cache, seqs, q, T, num_q_heads, sm_scale, num_splits, nullptr, 0,
                            stream);
  }
  if (need > kStaticScratchBytes) return NVKV_ERR_WORKSPACE;
  void *scratch = scratch_on_current_device();
  if (!scratch) return NVKV_ERR_CUDA;
  nvkv_status st = nvkv_decode_attn(cache, seqs, q, T, num_q_heads, sm_scale, num_splits,
                                    scratch, kStaticScratchBytes, stream);
  if (st != NVKV_OK) return st;
  return nvkv_combine(seqs, scratch, T, num_q_heads, cache->num_kv_heads, cache->head_dim,
                      num_splits, out, stream);
}

}  // extern "C"
