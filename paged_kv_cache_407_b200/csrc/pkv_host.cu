// Host helpers: status strings, descriptor and device checks, tensor maps.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "pkv_host.h"

namespace pkv {

pkv_status check_cache_desc(const pkv_cache_desc &c) {
  if (!valid_dtype(c.dtype)) return PKV_ERR_BAD_DTYPE;
  if (c.num_blocks < 1 || c.num_kv_heads < 1) return PKV_ERR_BAD_SHAPE;
  if (c.block_size != 8 && c.block_size != 16 && c.block_size != 32 && c.block_size != 64)
    return PKV_ERR_BAD_SHAPE;
  if (c.head_dim != 64 && c.head_dim != 128) return PKV_ERR_BAD_SHAPE;
  // Slots are int64 but block coordinates and per-pool element offsets are
  // formed in 64-bit; tensor-map dimensions must stay below 2^32.
  const long long rows = static_cast<long long>(c.num_blocks) * c.num_kv_heads;
  if (rows >= (1ll << 31)) return PKV_ERR_TOO_LARGE;
  return PKV_OK;
}

namespace {
// Result of the compute-capability check per device ordinal (0 = not yet
// asked, 1 = sm_100, 2 = another part); the answer cannot change while the
// process runs.
std::atomic<int8_t> g_device_kind[kMaxDevices];
}  // namespace

pkv_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PKV_ERR_DEVICE;
  int8_t kind = g_device_kind[dev].load(std::memory_order_relaxed);
  if (kind == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return PKV_ERR_CUDA;
    kind = (major == 10 && minor == 0) ? 1 : 2;
    g_device_kind[dev].store(kind, std::memory_order_relaxed);
  }
  return kind == 1 ? PKV_OK : PKV_ERR_DEVICE;
}

pkv_status set_smem_limit_once(const void *func, int bytes, std::atomic<uint64_t> *done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit != 0 && (done->load(std::memory_order_acquire) & bit) != 0) return PKV_OK;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return PKV_ERR_CUDA;
  if (bit != 0) done->fetch_or(bit, std::memory_order_release);
  return PKV_OK;
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}
}  // namespace

namespace {
// Rank-4 tiled map; dims fastest first, element size esz bytes, box inner x
// rows (the other two box extents 1).
pkv_status encode_map(CUtensorMap *map, const void *pool, CUtensorMapDataType type, cuuint64_t esz,
                      const cuuint64_t (&dims)[4], cuuint32_t box_inner, cuuint32_t box_rows,
                      CUtensorMapSwizzle swizzle) {
  auto fn = encoder();
  if (fn == nullptr) return PKV_ERR_CUDA;
  cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t strides[3] = {d[0] * esz, d[0] * d[1] * esz, d[0] * d[1] * d[2] * esz};
  cuuint32_t box[4] = {box_inner, box_rows, 1u, 1u};
  cuuint32_t estride[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, type, 4, const_cast<void *>(pool), d, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}
}  // namespace

pkv_status encode_cache_map(CUtensorMap *map, const void *pool, const pkv_cache_desc &c) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(c.head_dim), static_cast<cuuint64_t>(c.block_size),
                              static_cast<cuuint64_t>(c.num_kv_heads),
                              static_cast<cuuint64_t>(c.num_blocks)};
  return encode_map(map, pool, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, dims, 64u,
                    static_cast<cuuint32_t>(c.block_size), CU_TENSOR_MAP_SWIZZLE_128B);
}

namespace {
// Byte map of `rank` dims (fastest first) with explicit byte strides of dims
// 1.. and a full box, 128-byte swizzle.
pkv_status encode_bytes(CUtensorMap *map, const void *pool, cuuint32_t rank, const cuuint64_t *dims,
                        const cuuint64_t *strides, const cuuint32_t *box) {
  auto fn = encoder();
  if (fn == nullptr) return PKV_ERR_CUDA;
  const cuuint32_t estride[5] = {1u, 1u, 1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void *>(pool),
                  const_cast<cuuint64_t *>(dims), const_cast<cuuint64_t *>(strides),
                  const_cast<cuuint32_t *>(box), estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}
}  // namespace

pkv_status encode_query_map(CUtensorMap *map, const void *query, int num_tokens, int num_q_heads,
                            int head_dim, int group) {
  auto fn = encoder();
  if (fn == nullptr) return PKV_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                        static_cast<cuuint64_t>(num_tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                           static_cast<cuuint64_t>(head_dim) * num_q_heads * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(128 / group)};
  cuuint32_t estride[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void *>(query), dims, strides, box,
                  estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}

// The K tile of (block, kv head) is B rows of D codes.  Token t = b + 2 a + 4 c
// (b, a in {0, 1}) is addressed through dims (d, b, c, a, block*Hkv + head),
// so the box lands in shared memory with token t on row b + 2 c + (B/2) a:
// the eight tokens {0,1,4,5,8,9,12,13} + 2a + 16 j of one score column tile
// sit on eight consecutive rows.
pkv_status encode_fp8_k_map(CUtensorMap *map, const void *pool, const pkv_cache_desc &c) {
  const cuuint64_t D = static_cast<cuuint64_t>(c.head_dim);
  const cuuint64_t B = static_cast<cuuint64_t>(c.block_size);
  const cuuint64_t rows = static_cast<cuuint64_t>(c.num_blocks) * c.num_kv_heads;
  const cuuint64_t dims[5] = {D, 2, B / 4, 2, rows};
  const cuuint64_t strides[4] = {D, 4 * D, 2 * D, B * D};
  const cuuint32_t box[5] = {static_cast<cuuint32_t>(D), 2u, static_cast<cuuint32_t>(B / 4), 2u, 1u};
  return encode_bytes(map, pool, 5, dims, strides, box);
}

// The V tile of (block, kv head) is D rows of B codes, D*B contiguous bytes;
// it is moved as (D*B)/128 rows of 128 bytes.
pkv_status encode_fp8_v_map(CUtensorMap *map, const void *pool, const pkv_cache_desc &c) {
  const cuuint64_t tile = static_cast<cuuint64_t>(c.head_dim) * c.block_size;
  const cuuint64_t rows = static_cast<cuuint64_t>(c.num_blocks) * c.num_kv_heads;
  const cuuint64_t dims[3] = {128, tile / 128, rows};
  const cuuint64_t strides[2] = {128, tile};
  const cuuint32_t box[3] = {128u, static_cast<cuuint32_t>(tile / 128), 1u};
  return encode_bytes(map, pool, 3, dims, strides, box);
}

}  // namespace pkv

extern "C" const char *pkv_status_string(pkv_status s) {
  switch (s) {
    case PKV_OK: return "ok";
    case PKV_ERR_NULL_POINTER: return "a required pointer is NULL";
    case PKV_ERR_BAD_DTYPE: return "dtype not accepted here (fp16/bf16 pools, or PKV_FP8_E4M3 pools for the _fp8 calls)";
    case PKV_ERR_BAD_SHAPE: return "unsupported shape (head_dim 64/128, block_size 8/16/32/64, head counts)";
    case PKV_ERR_MISALIGNED: return "pointer or stride breaks the required alignment";
    case PKV_ERR_WORKSPACE: return "workspace missing or smaller than pkv_paged_attention_workspace_size";
    case PKV_ERR_BAD_PARTITION: return "partition_size must be a positive multiple of block_size";
    case PKV_ERR_TOO_LARGE: return "a size exceeds what the kernels can index";
    case PKV_ERR_CUDA: return "a CUDA runtime or driver call failed";
    case PKV_ERR_DEVICE: return "current device is not compute capability 10.0 (B200, sm_100a)";
    case PKV_ERR_NO_BLOCKS: return "the free block pool cannot supply the blocks asked for";
    case PKV_ERR_BAD_SEQUENCE: return "unknown, repeated or already present sequence id";
    case PKV_ERR_ALIAS: return "a slot repeats in one cache write, or a copy destination repeats or is also a source";
  }
  return "unknown pkv_status";
}

extern "C" int32_t pkv_version(void) { return 100; }
