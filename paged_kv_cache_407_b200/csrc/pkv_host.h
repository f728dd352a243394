// Host-side helpers shared by the libpkv entry points.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "pkv.h"

namespace pkv {

inline bool aligned(const void *p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline bool valid_dtype(pkv_dtype t) { return t == PKV_F16 || t == PKV_BF16 || t == PKV_FP8_E4M3; }

inline bool is_16bit(pkv_dtype t) { return t == PKV_F16 || t == PKV_BF16; }

inline int elem_bytes(pkv_dtype t) { return t == PKV_FP8_E4M3 ? 1 : 2; }

// Checks shared by every call that takes a cache descriptor.
pkv_status check_cache_desc(const pkv_cache_desc &c);

constexpr int kMaxDevices = 128;

// PKV_ERR_DEVICE unless the current device is compute capability 10.0 (asked
// once per device ordinal, then remembered).
pkv_status check_device();

// cudaFuncSetAttribute(func, MaxDynamicSharedMemorySize, bytes) once per
// device (devices 0..63 remembered in the bits of *done; others set on every
// call).  `done` belongs to one kernel and starts at 0.
pkv_status set_smem_limit_once(const void *func, int bytes, std::atomic<uint64_t> *done);

// Encode a rank-4 tiled tensor map over one fp16/bf16 cache pool viewed as
// [N][Hkv][B][D] (fastest last), box = 64 elements x B rows, 128-byte swizzle.
pkv_status encode_cache_map(CUtensorMap *map, const void *pool, const pkv_cache_desc &c);

// 8-bit pools (D = 128), 128-byte swizzle, one box per (block, kv head) tile
// addressed by the row block * Hkv + head.  K [N][Hkv][B][D] bytes through a
// rank-5 view that puts the rows of each score column tile together (the
// token order is given with the encoder); V [N][Hkv][D][B] bytes as rows of
// 128 bytes.

pkv_status encode_fp8_k_map(CUtensorMap *map, const void *pool, const pkv_cache_desc &c);
pkv_status encode_fp8_v_map(CUtensorMap *map, const void *pool, const pkv_cache_desc &c);

// Rank-3 tiled map over the queries [T][Hq][D] (16-bit), box 64 x G heads x
// (128 / G) tokens, 128-byte swizzle: one box is 64 columns of a 128-row tile
// whose row t * G + h is query head g * G + h of token t.
pkv_status encode_query_map(CUtensorMap *map, const void *query, int num_tokens, int num_q_heads,
                            int head_dim, int group);

inline pkv_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

#ifdef __CUDACC__
// Launch with programmatic stream serialisation: the kernel may be launched
// while the previous kernel in the stream finishes; it must call pdl_wait()
// (pkv_device.cuh) before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// launch_pdl for a kernel that needs `smem` bytes of dynamic shared memory,
// raising its limit first (once per device, remembered in *done).  Should the
// launch fail - as it does when the device was reset and the raised limit
// went with it - the limit is raised again and the launch retried once.
template <typename... KArgs, typename... Args>
pkv_status launch_with_smem(void (*kern)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t stream,
                            std::atomic<uint64_t> *done, Args &&...args) {
  pkv_status st = set_smem_limit_once(reinterpret_cast<const void *>(kern), smem, done);
  if (st != PKV_OK) return st;
  if (launch_pdl(kern, grid, block, smem, stream, args...) == cudaSuccess) return PKV_OK;
  (void)cudaGetLastError();
  done->store(0, std::memory_order_release);
  if ((st = set_smem_limit_once(reinterpret_cast<const void *>(kern), smem, done)) != PKV_OK) return st;
  return launch_pdl(kern, grid, block, smem, stream, args...) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
#endif

}  // namespace pkv
