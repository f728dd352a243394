// reshape_and_cache: scatter this step's new K/V tokens into their cache slots.
//
// lshu.cn/news/11644 (vLLM architecture analysis), "方案：页式内存管理": a token
// that a request appends goes into a position of a block of its Block Table;
// zzmblog.top "vLLM使用指南", "Transformer推理与KV缓存": the decode step appends
// the current token's K, V before computing attention.  The slot (block id *
// block_size + position) is chosen by the host; for fp16/bf16 pools the kernel
// is a bit copy, for 8-bit pools it quantises (same page, "性能关键路径与瓶颈":
// an FP8/INT8 KV cache halves the bytes decode reads).
#include <cuda_fp8.h>

#include "pkv_device.cuh"
#include "alias_check.h"
#include "pkv_host.h"

namespace pkv {
namespace {

// One thread per 16-byte chunk of one (token, kv head) row, for K and V.
__global__ void __launch_bounds__(256)
    reshape_and_cache_vec_kernel(const uint4 *__restrict__ key, const uint4 *__restrict__ value,
                                 int64_t key_stride_vec, int64_t value_stride_vec,
                                 uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                                 const int64_t *__restrict__ slot_mapping, int num_tokens,
                                 int num_kv_heads, int head_vecs, int block_size,
                                 int64_t num_slots, int32_t *d_status) {
  pdl_trigger();
  pdl_wait();
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * head_vecs;
  const int64_t total = per_token * num_tokens;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t r = i - t * per_token;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;  // padding token
    if (slot >= num_slots) {
      if (r == 0) raise_flag(d_status, PKV_DEV_BAD_SLOT);
      continue;
    }
    const int64_t h = r / head_vecs;
    const int64_t c = r - h * head_vecs;
    const int64_t blk = slot / block_size;
    const int64_t pos = slot - blk * block_size;
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + pos) * head_vecs + c;
    const uint4 kv = key[t * key_stride_vec + r];
    const uint4 vv = value[t * value_stride_vec + r];
    k_cache[dst] = kv;
    v_cache[dst] = vv;
  }
}

// Element-wise fallback for inputs whose rows are not 16-byte aligned.
__global__ void __launch_bounds__(256)
    reshape_and_cache_elem_kernel(const uint16_t *__restrict__ key,
                                  const uint16_t *__restrict__ value, int64_t key_stride,
                                  int64_t value_stride, uint16_t *__restrict__ k_cache,
                                  uint16_t *__restrict__ v_cache,
                                  const int64_t *__restrict__ slot_mapping, int num_tokens,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int64_t num_slots, int32_t *d_status) {
  pdl_trigger();
  pdl_wait();
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * head_dim;
  const int64_t total = per_token * num_tokens;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t r = i - t * per_token;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (r == 0) raise_flag(d_status, PKV_DEV_BAD_SLOT);
      continue;
    }
    const int64_t h = r / head_dim;
    const int64_t e = r - h * head_dim;
    const int64_t blk = slot / block_size;
    const int64_t pos = slot - blk * block_size;
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + pos) * head_dim + e;
    k_cache[dst] = key[t * key_stride + r];
    v_cache[dst] = value[t * value_stride + r];
  }
}

// Quantising write into 8-bit pools: one thread per 4 dimensions of one
// (token, kv head), so a warp covers a 128-wide head.  Each value x is stored
// as e4m3(x / scale) (IEEE fp32 division, round to nearest even, saturated to
// +-448).  K codes go to the token's row (one 32-bit store per thread, a
// coalesced 128-byte row per warp), V codes to the token's column of the
// transposed V tile (single bytes, B apart).  VEC: 8-byte input loads.
template <typename T, bool VEC>
__global__ void __launch_bounds__(256)
    reshape_and_cache_fp8_kernel(const T *__restrict__ key, const T *__restrict__ value,
                                 int64_t key_stride, int64_t value_stride,
                                 uint8_t *__restrict__ k_cache, uint8_t *__restrict__ v_cache,
                                 const int64_t *__restrict__ slot_mapping, int num_tokens,
                                 int num_kv_heads, int head_dim, int block_size, int64_t num_slots,
                                 float k_scale, float v_scale, int32_t *d_status) {
  pdl_trigger();
  pdl_wait();
  const int quads = head_dim / 4;
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * quads;
  const int64_t total = per_token * num_tokens;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t r = i - t * per_token;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (r == 0) raise_flag(d_status, PKV_DEV_BAD_SLOT);
      continue;
    }
    const int64_t h = r / quads;
    const int64_t d0 = (r - h * quads) * 4;
    const int64_t blk = slot / block_size;
    const int64_t pos = slot - blk * block_size;
    const T *kp = key + t * key_stride + h * head_dim + d0;
    const T *vp = value + t * value_stride + h * head_dim + d0;
    T kx[4], vx[4];
    if constexpr (VEC) {
      *reinterpret_cast<uint2 *>(kx) = *reinterpret_cast<const uint2 *>(kp);
      *reinterpret_cast<uint2 *>(vx) = *reinterpret_cast<const uint2 *>(vp);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        kx[j] = kp[j];
        vx[j] = vp[j];
      }
    }
    const uint32_t k01 = __nv_cvt_float2_to_fp8x2(
        make_float2(static_cast<float>(kx[0]) / k_scale, static_cast<float>(kx[1]) / k_scale),
        __NV_SATFINITE, __NV_E4M3);
    const uint32_t k23 = __nv_cvt_float2_to_fp8x2(
        make_float2(static_cast<float>(kx[2]) / k_scale, static_cast<float>(kx[3]) / k_scale),
        __NV_SATFINITE, __NV_E4M3);
    const uint32_t v01 = __nv_cvt_float2_to_fp8x2(
        make_float2(static_cast<float>(vx[0]) / v_scale, static_cast<float>(vx[1]) / v_scale),
        __NV_SATFINITE, __NV_E4M3);
    const uint32_t v23 = __nv_cvt_float2_to_fp8x2(
        make_float2(static_cast<float>(vx[2]) / v_scale, static_cast<float>(vx[3]) / v_scale),
        __NV_SATFINITE, __NV_E4M3);
    const int64_t base = blk * num_kv_heads + h;
    *reinterpret_cast<uint32_t *>(k_cache + (base * block_size + pos) * head_dim + d0) =
        (k01 & 0xffffu) | (k23 << 16);
    uint8_t *vrow = v_cache + (base * head_dim + d0) * block_size + pos;
    vrow[0] = static_cast<uint8_t>(v01);
    vrow[block_size] = static_cast<uint8_t>(v01 >> 8);
    vrow[2 * block_size] = static_cast<uint8_t>(v23);
    vrow[3 * block_size] = static_cast<uint8_t>(v23 >> 8);
  }
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_reshape_and_cache_fp8(const void *key, const void *value,
                                                int64_t key_token_stride,
                                                int64_t value_token_stride, pkv_dtype input_dtype,
                                                void *k_cache, void *v_cache, pkv_cache_desc cache,
                                                const int64_t *slot_mapping, int32_t num_tokens,
                                                float k_scale, float v_scale, int32_t *d_status,
                                                pkv_stream_t stream) {
  using namespace pkv;
  pkv_status st = check_cache_desc(cache);
  if (st != PKV_OK) return st;
  if (cache.dtype != PKV_FP8_E4M3 || !is_16bit(input_dtype)) return PKV_ERR_BAD_DTYPE;
  if (cache.head_dim != 128 || cache.block_size < 16) return PKV_ERR_BAD_SHAPE;
  if (!(k_scale > 0.f) || !(k_scale < INFINITY) || !(v_scale > 0.f) || !(v_scale < INFINITY))
    return PKV_ERR_BAD_SHAPE;
  if (num_tokens < 0) return PKV_ERR_BAD_SHAPE;
  if (num_tokens == 0) return PKV_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_NULL_POINTER;
  const int64_t row = static_cast<int64_t>(cache.num_kv_heads) * cache.head_dim;
  if (key_token_stride == 0) key_token_stride = row;
  if (value_token_stride == 0) value_token_stride = row;
  if (key_token_stride < row || value_token_stride < row) return PKV_ERR_BAD_SHAPE;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(slot_mapping, 8) ||
      !aligned(key, 2) || !aligned(value, 2))
    return PKV_ERR_MISALIGNED;
  if ((st = check_device()) != PKV_OK) return st;
#ifdef PKV_CHECK
  if ((st = check_unique_slots(slot_mapping, num_tokens, reinterpret_cast<cudaStream_t>(stream))) != PKV_OK)
    return st;
#endif
  const int64_t num_slots = static_cast<int64_t>(cache.num_blocks) * cache.block_size;
  const int threads = 256;
  const int64_t items = static_cast<int64_t>(num_tokens) * cache.num_kv_heads * (cache.head_dim / 4);
  const int blocks = static_cast<int>(std::min<int64_t>((items + threads - 1) / threads, 148 * 16));
  const bool vec = aligned(key, 8) && aligned(value, 8) && key_token_stride % 4 == 0 &&
                   value_token_stride % 4 == 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err;
#define PKV_FP8_WRITE(T, V)                                                                   \
  err = launch_pdl(reshape_and_cache_fp8_kernel<T, V>, dim3(blocks), dim3(threads), 0, s,     \
                   static_cast<const T *>(key), static_cast<const T *>(value),                \
                   key_token_stride, value_token_stride, static_cast<uint8_t *>(k_cache),     \
                   static_cast<uint8_t *>(v_cache), slot_mapping, num_tokens,                 \
                   cache.num_kv_heads, cache.head_dim, cache.block_size, num_slots, k_scale,  \
                   v_scale, d_status)
  if (input_dtype == PKV_BF16) {
    if (vec)
      PKV_FP8_WRITE(__nv_bfloat16, true);
    else
      PKV_FP8_WRITE(__nv_bfloat16, false);
  } else {
    if (vec)
      PKV_FP8_WRITE(__half, true);
    else
      PKV_FP8_WRITE(__half, false);
  }
#undef PKV_FP8_WRITE
  return err == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

extern "C" pkv_status pkv_reshape_and_cache(const void *key, const void *value,
                                            int64_t key_token_stride, int64_t value_token_stride,
                                            void *k_cache, void *v_cache, pkv_cache_desc cache,
                                            const int64_t *slot_mapping, int32_t num_tokens,
                                            int32_t *d_status, pkv_stream_t stream) {
  using namespace pkv;
  pkv_status st = check_cache_desc(cache);
  if (st != PKV_OK) return st;
  if (!is_16bit(cache.dtype)) return PKV_ERR_BAD_DTYPE;
  if (num_tokens < 0) return PKV_ERR_BAD_SHAPE;
  if (num_tokens == 0) return PKV_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_NULL_POINTER;
  const int64_t row = static_cast<int64_t>(cache.num_kv_heads) * cache.head_dim;
  if (key_token_stride == 0) key_token_stride = row;
  if (value_token_stride == 0) value_token_stride = row;
  if (key_token_stride < row || value_token_stride < row) return PKV_ERR_BAD_SHAPE;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(slot_mapping, 8) ||
      !aligned(key, 2) || !aligned(value, 2))
    return PKV_ERR_MISALIGNED;
  if ((st = check_device()) != PKV_OK) return st;
#ifdef PKV_CHECK
  if ((st = check_unique_slots(slot_mapping, num_tokens, reinterpret_cast<cudaStream_t>(stream))) != PKV_OK)
    return st;
#endif

  const int64_t num_slots = static_cast<int64_t>(cache.num_blocks) * cache.block_size;
  const bool vec = aligned(key, 16) && aligned(value, 16) && key_token_stride % 8 == 0 &&
                   value_token_stride % 8 == 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int threads = 256;
  cudaError_t err;
  if (vec) {
    const int head_vecs = cache.head_dim / 8;
    const int64_t items = static_cast<int64_t>(num_tokens) * cache.num_kv_heads * head_vecs;
    const int blocks = static_cast<int>(std::min<int64_t>((items + threads - 1) / threads, 148 * 16));
    err = launch_pdl(reshape_and_cache_vec_kernel, dim3(blocks), dim3(threads), 0, s,
                     static_cast<const uint4 *>(key), static_cast<const uint4 *>(value),
                     key_token_stride / 8, value_token_stride / 8, static_cast<uint4 *>(k_cache),
                     static_cast<uint4 *>(v_cache), slot_mapping, num_tokens, cache.num_kv_heads,
                     head_vecs, cache.block_size, num_slots, d_status);
  } else {
    const int64_t items = static_cast<int64_t>(num_tokens) * row;
    const int blocks = static_cast<int>(std::min<int64_t>((items + threads - 1) / threads, 148 * 16));
    err = launch_pdl(reshape_and_cache_elem_kernel, dim3(blocks), dim3(threads), 0, s,
                     static_cast<const uint16_t *>(key), static_cast<const uint16_t *>(value),
                     key_token_stride, value_token_stride, static_cast<uint16_t *>(k_cache),
                     static_cast<uint16_t *>(v_cache), slot_mapping, num_tokens, cache.num_kv_heads,
                     cache.head_dim, cache.block_size, num_slots, d_status);
  }
  return err == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
