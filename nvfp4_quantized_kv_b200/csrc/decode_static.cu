// decode_static.cu -- nvkv_decode_attn_static: decode / MTP-verify attention
// (split-K partials + combine) whose split-K scratch lives in a fixed,
// library-owned device array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory at the point
// where they run attention -- code inside a CUDA Graph capture region (an
// allocation there may synchronise and break the capture), runtimes whose
// device memory is owned by another pool or allocator, and real-time paths
// that must not take allocator locks.  They pass only inputs and outputs.
//
// The scratch is one file-scope __device__ array of kStaticScratchBytes.
// Host code cannot use the array's name as a device address, so the address
// is looked up with cudaGetSymbolAddress once per device, on the first call
// made with that device current, and cached.
#include <mutex>

#include "nvkv_common.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, or NULL.
void *scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
      cudaGetLastError();  // leave no error behind for the caller's next call
      return nullptr;
    }
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" {

size_t nvkv_decode_static_scratch_bytes(void) { return kStaticScratchBytes; }

nvkv_status nvkv_decode_attn_static(const nvkv_cache *cache, const nvkv_seqs *seqs,
                                    const void *q, int32_t T, int32_t num_q_heads,
                                    float sm_scale, int32_t num_splits, void *out,
                                    nvkv_stream_t stream) {
  if (!cache || !seqs) return NVKV_ERR_INVALID_ARG;
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
