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

// Quantising write into 8-bit pools: one thread per 16 dimensions of one
// (token, kv head).  Each value x is stored as e4m3(x / scale) (IEEE fp32
// division, round to nearest even, saturated to +-448).  K codes go to the
// token's row, V codes to the token's column of the transposed V tile.
template <typename T>
__global__ void __launch_bounds__(256)
    reshape_and_cache_fp8_kernel(const T *__restrict__ key, const T *__restrict__ value,
                                 int64_t key_stride, int64_t value_stride,
                                 uint8_t *__restrict__ k_cache, uint8_t *__restrict__ v_cache,
                                 const int64_t *__restrict__ slot_mapping, int num_tokens,
                                 int num_kv_heads, int head_dim, int block_size, int64_t num_slots,
                                 float k_scale, float v_scale, int32_t *d_status) {
  const int chunks = head_dim / 16;
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * chunks;
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
    const int64_t h = r / chunks;
    const int64_t d0 = (r - h * chunks) * 16;
    const int64_t blk = slot / block_size;
    const int64_t pos = slot - blk * block_size;
    const T *kp = key + t * key_stride + h * head_dim + d0;
    const T *vp = value + t * value_stride + h * head_dim + d0;
    uint32_t kw[4];
    uint8_t vq[16];
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
      float2 a = make_float2(static_cast<float>(kp[j]) / k_scale, static_cast<float>(kp[j + 1]) / k_scale);
      float2 b = make_float2(static_cast<float>(kp[j + 2]) / k_scale, static_cast<float>(kp[j + 3]) / k_scale);
      const uint32_t lo = __nv_cvt_float2_to_fp8x2(a, __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float2_to_fp8x2(b, __NV_SATFINITE, __NV_E4M3);
      kw[j / 4] = lo | (hi << 16);
      a = make_float2(static_cast<float>(vp[j]) / v_scale, static_cast<float>(vp[j + 1]) / v_scale);
      b = make_float2(static_cast<float>(vp[j + 2]) / v_scale, static_cast<float>(vp[j + 3]) / v_scale);
      const uint32_t vlo = __nv_cvt_float2_to_fp8x2(a, __NV_SATFINITE, __NV_E4M3);
      const uint32_t vhi = __nv_cvt_float2_to_fp8x2(b, __NV_SATFINITE, __NV_E4M3);
      vq[j] = vlo & 0xff;
      vq[j + 1] = vlo >> 8;
      vq[j + 2] = vhi & 0xff;
      vq[j + 3] = vhi >> 8;
    }
    const int64_t base = (blk * num_kv_heads + h);
    *reinterpret_cast<uint4 *>(k_cache + (base * block_size + pos) * head_dim + d0) =
        make_uint4(kw[0], kw[1], kw[2], kw[3]);
    uint8_t *vrow = v_cache + (base * head_dim + d0) * block_size + pos;
#pragma unroll
    for (int j = 0; j < 16; ++j) vrow[j * block_size] = vq[j];
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
  const int64_t num_slots = static_cast<int64_t>(cache.num_blocks) * cache.block_size;
  const int threads = 256;
  const int64_t items = static_cast<int64_t>(num_tokens) * cache.num_kv_heads * (cache.head_dim / 16);
  const int blocks = static_cast<int>(std::min<int64_t>((items + threads - 1) / threads, 148 * 16));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (input_dtype == PKV_BF16)
    reshape_and_cache_fp8_kernel<__nv_bfloat16><<<blocks, threads, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(key), static_cast<const __nv_bfloat16 *>(value),
        key_token_stride, value_token_stride, static_cast<uint8_t *>(k_cache),
        static_cast<uint8_t *>(v_cache), slot_mapping, num_tokens, cache.num_kv_heads,
        cache.head_dim, cache.block_size, num_slots, k_scale, v_scale, d_status);
  else
    reshape_and_cache_fp8_kernel<__half><<<blocks, threads, 0, s>>>(
        static_cast<const __half *>(key), static_cast<const __half *>(value), key_token_stride,
        value_token_stride, static_cast<uint8_t *>(k_cache), static_cast<uint8_t *>(v_cache),
        slot_mapping, num_tokens, cache.num_kv_heads, cache.head_dim, cache.block_size,
        num_slots, k_scale, v_scale, d_status);
  return launch_status();
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

  const int64_t num_slots = static_cast<int64_t>(cache.num_blocks) * cache.block_size;
  const bool vec = aligned(key, 16) && aligned(value, 16) && key_token_stride % 8 == 0 &&
                   value_token_stride % 8 == 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int threads = 256;
  if (vec) {
    const int head_vecs = cache.head_dim / 8;
    const int64_t items = static_cast<int64_t>(num_tokens) * cache.num_kv_heads * head_vecs;
    const int blocks = static_cast<int>(std::min<int64_t>((items + threads - 1) / threads, 148 * 16));
    reshape_and_cache_vec_kernel<<<blocks, threads, 0, s>>>(
        static_cast<const uint4 *>(key), static_cast<const uint4 *>(value), key_token_stride / 8,
        value_token_stride / 8, static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache),
        slot_mapping, num_tokens, cache.num_kv_heads, head_vecs, cache.block_size, num_slots,
        d_status);
  } else {
    const int64_t items = static_cast<int64_t>(num_tokens) * row;
    const int blocks = static_cast<int>(std::min<int64_t>((items + threads - 1) / threads, 148 * 16));
    reshape_and_cache_elem_kernel<<<blocks, threads, 0, s>>>(
        static_cast<const uint16_t *>(key), static_cast<const uint16_t *>(value), key_token_stride,
        value_token_stride, static_cast<uint16_t *>(k_cache), static_cast<uint16_t *>(v_cache),
        slot_mapping, num_tokens, cache.num_kv_heads, cache.head_dim, cache.block_size, num_slots,
        d_status);
  }
  return launch_status();
}
