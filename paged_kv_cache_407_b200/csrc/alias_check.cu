// Check build (PKV_CHECK defined): the uniqueness guarantees of the cache
// write and the block copy, verified on the host.  Source of the rules:
// lshu.cn/news/11644, "方案：页式内存管理" (every token owns one position of
// one block, so no two tokens of a step share a slot) and "内存共享" (a
// shared block is copied before it is written: each copy makes one new
// private block from a block that is only read).  The regular build leaves
// both unchecked (the kernels would race; the result is unspecified).
#include <algorithm>
#include <new>
#include <vector>

#include "alias_check.h"

extern "C" int32_t pkv_check_build(void) {
#ifdef PKV_CHECK
  return 1;
#else
  return 0;
#endif
}

#ifdef PKV_CHECK
namespace pkv {
namespace {

// Copies n int64 values from the device to the host.  The stream must not be
// capturing: the copy is followed by a synchronisation.
pkv_status fetch(std::vector<int64_t> &h, const int64_t *d, size_t n, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return PKV_ERR_CUDA;
  h.resize(n);
  if (cudaMemcpyAsync(h.data(), d, n * sizeof(int64_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return PKV_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

bool has_repeat(std::vector<int64_t> &v) {
  std::sort(v.begin(), v.end());
  return std::adjacent_find(v.begin(), v.end()) != v.end();
}

}  // namespace

pkv_status check_unique_slots(const int64_t *slot_mapping, int32_t num_tokens, cudaStream_t stream) try {
  if (num_tokens <= 0) return PKV_OK;
  std::vector<int64_t> h;
  pkv_status st = fetch(h, slot_mapping, static_cast<size_t>(num_tokens), stream);
  if (st != PKV_OK) return st;
  std::vector<int64_t> used;
  used.reserve(h.size());
  for (const int64_t p : h)
    if (p >= 0) used.push_back(p);  // negative slots are padding: they write nothing
  return has_repeat(used) ? PKV_ERR_ALIAS : PKV_OK;
} catch (const std::bad_alloc &) {
  return PKV_ERR_TOO_LARGE;  // no host memory for the copy: nothing was queued
}

pkv_status check_copy_pairs(const int64_t *block_pairs, int32_t num_pairs, int64_t num_blocks,
                            cudaStream_t stream) try {
  if (num_pairs <= 0) return PKV_OK;
  std::vector<int64_t> h;
  pkv_status st = fetch(h, block_pairs, 2 * static_cast<size_t>(num_pairs), stream);
  if (st != PKV_OK) return st;
  std::vector<int64_t> srcs, dsts;
  for (int32_t i = 0; i < num_pairs; ++i) {
    const int64_t src = h[2 * i], dst = h[2 * i + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) continue;  // skipped by the kernel
    srcs.push_back(src);
    dsts.push_back(dst);
  }
  if (has_repeat(dsts)) return PKV_ERR_ALIAS;
  std::sort(srcs.begin(), srcs.end());
  for (const int64_t d : dsts)
    if (std::binary_search(srcs.begin(), srcs.end(), d)) return PKV_ERR_ALIAS;
  return PKV_OK;
} catch (const std::bad_alloc &) {
  return PKV_ERR_TOO_LARGE;
}

}  // namespace pkv
#endif  // PKV_CHECK
