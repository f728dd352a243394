// copy_blocks: copy-on-write of shared physical blocks.
//
// lshu.cn/news/11644 (vLLM architecture analysis), "内存共享": requests whose
// prompts share a prefix map it to the same physical blocks, read-only; when a
// request diverges inside a shared block, that block is copied first.  Each
// (src, dst) pair makes block dst of both pools a bit copy of block src.
#include "pkv_device.cuh"
#include "alias_check.h"
#include "pkv_host.h"

namespace pkv {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

// grid.x = pair, grid.y = pool (0: K, 1: V), grid.z = slice of the block.
__global__ void __launch_bounds__(kCopyThreads)
    copy_blocks_kernel(uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                       const int64_t *__restrict__ block_pairs, int64_t block_vecs,
                       int64_t num_blocks, int32_t *d_status) {
  pdl_trigger();
  pdl_wait();
  const int64_t src = block_pairs[2 * static_cast<int64_t>(blockIdx.x)];
  const int64_t dst = block_pairs[2 * static_cast<int64_t>(blockIdx.x) + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
      raise_flag(d_status, PKV_DEV_BAD_BLOCK);
    return;
  }
  uint4 *pool = blockIdx.y == 0 ? k_cache : v_cache;
  const uint4 *from = pool + src * block_vecs;
  uint4 *to = pool + dst * block_vecs;
  const int64_t step = static_cast<int64_t>(gridDim.z) * kCopyThreads;
  int64_t i = static_cast<int64_t>(blockIdx.z) * kCopyThreads + threadIdx.x;
  for (; i + (kCopyUnroll - 1) * step < block_vecs; i += kCopyUnroll * step) {
    uint4 v[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) v[u] = from[i + u * step];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) to[i + u * step] = v[u];
  }
  for (; i < block_vecs; i += step) to[i] = from[i];
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_copy_blocks(void *k_cache, void *v_cache, pkv_cache_desc cache,
                                      const int64_t *block_pairs, int32_t num_pairs,
                                      int32_t *d_status, pkv_stream_t stream) {
  using namespace pkv;
  pkv_status st = check_cache_desc(cache);
  if (st != PKV_OK) return st;
  if (num_pairs < 0) return PKV_ERR_BAD_SHAPE;
  if (num_pairs == 0) return PKV_OK;
  if (!k_cache || !v_cache || !block_pairs) return PKV_ERR_NULL_POINTER;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(block_pairs, 8))
    return PKV_ERR_MISALIGNED;
  if (num_pairs > 2147483647 / 2) return PKV_ERR_TOO_LARGE;
  if ((st = check_device()) != PKV_OK) return st;
#ifdef PKV_CHECK
  if ((st = check_copy_pairs(block_pairs, num_pairs, cache.num_blocks, reinterpret_cast<cudaStream_t>(stream))) !=
      PKV_OK)
    return st;
#endif
  const int64_t block_vecs = static_cast<int64_t>(cache.num_kv_heads) * cache.block_size *
                             cache.head_dim * elem_bytes(cache.dtype) / 16;
  const int64_t per_cta = static_cast<int64_t>(kCopyThreads) * kCopyUnroll;
  const unsigned slices = static_cast<unsigned>(std::min<int64_t>((block_vecs + per_cta - 1) / per_cta, 64));
  dim3 grid(static_cast<unsigned>(num_pairs), 2u, slices);
  const cudaError_t err =
      launch_pdl(copy_blocks_kernel, grid, dim3(kCopyThreads), 0, reinterpret_cast<cudaStream_t>(stream),
                 static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), block_pairs, block_vecs,
                 static_cast<int64_t>(cache.num_blocks), d_status);
  return err == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
