// pages.cu -- host KV spill / restore of whole NVFP4 pages.
//
// "gzenz/ninfer" README, "Context cache and eviction": once the device pool
// runs out, the engine copies the KV of the continuations it evicts into an
// arena of pinned host memory and copies it back to the device when that
// cache is used again; the arena is filled scatter-gather, so fragmentation
// of the arena cannot make a spill fail.
// Here the arena is an array of page-sized slots and a spill or restore is
// a list of (pool page, arena slot) pairs: one kernel moves every listed
// page block in 16-byte words, reading and writing pinned host memory
// directly through its device-visible address (no staging copy, one launch
// however fragmented the lists are).
#include "nvkv_common.cuh"

namespace nvkv {
namespace {

constexpr int kCopyThreads = 256;

// Block i moves pair i: 16-byte words, strided over the block.
__global__ void __launch_bounds__(kCopyThreads)
page_copy_kernel(const uint8_t *__restrict__ src_base, int64_t src_count,
                 uint8_t *__restrict__ dst_base, int64_t dst_count,
                 const int32_t *__restrict__ src_ids, const int32_t *__restrict__ dst_ids, int n,
                 int64_t page_bytes, int32_t *err) {
  const int i = blockIdx.x;
  if (i >= n) return;
  const int64_t s = src_ids[i], d = dst_ids[i];
  if (s < 0 || s >= src_count || d < 0 || d >= dst_count) {
    if (threadIdx.x == 0) report(err, NVKV_DEVERR_PAGE_ID);
    return;
  }
  const uint4 *src = reinterpret_cast<const uint4 *>(src_base + s * page_bytes);
  uint4 *dst = reinterpret_cast<uint4 *>(dst_base + d * page_bytes);
  const int64_t words = page_bytes / 16;
  for (int64_t w = threadIdx.x; w < words; w += kCopyThreads) dst[w] = src[w];
}

}  // namespace

cudaError_t launch_page_copy(const uint8_t *src, int64_t src_count, uint8_t *dst,
                             int64_t dst_count, const int32_t *src_ids, const int32_t *dst_ids,
                             int n, int64_t page_bytes, int32_t *err, cudaStream_t stream) {
  page_copy_kernel<<<(unsigned)n, kCopyThreads, 0, stream>>>(src, src_count, dst, dst_count,
                                                             src_ids, dst_ids, n, page_bytes, err);
  return cudaGetLastError();
}

}  // namespace nvkv
