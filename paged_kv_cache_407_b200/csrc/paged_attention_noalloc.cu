// pkv_paged_attention_decode_noalloc: decode attention for callers that must
// not allocate device memory.
//
// The regular entry point asks the caller for a split-K workspace.  Some callers
// cannot provide one: a serving engine that reserved all free device memory for
// its block pool up front (so any later cudaMalloc fails), a plain C host with no
// device allocator of its own, or a latency-critical loop where cudaMalloc's
// implicit device-wide synchronisation is unacceptable.  For them the scratch
// lives in a fixed buffer compiled into this library, PKV_NOALLOC_SCRATCH_BYTES
// per device; the caller still passes every input and output.
#include "pkv_host.h"

// The scratch itself.  Every GPU that loads this library holds it until the
// process exits.  Host code must not pass `g_noalloc_scratch` to a kernel: in
// host code that name is only a host-side stand-in; the device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

namespace pkv {
namespace {

constexpr size_t kScratchBytes = PKV_NOALLOC_SCRATCH_BYTES;

// Device address of the buffer on the current device.  It is looked up on
// every call rather than cached: the lookup is cheap next to a launch, and a
// cached address would go stale if the device's context were destroyed and
// created again (cudaDeviceReset), which loads the buffer anew.  The first
// lookup on a device also loads the library's device code there.
pkv_status scratch_address(void **addr) {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return PKV_ERR_CUDA;
  *addr = p;
  return PKV_OK;
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_paged_attention_decode_noalloc(
    void *out, const void *query, const void *k_cache, const void *v_cache, pkv_cache_desc cache,
    const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens,
    int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len, float scale,
    int32_t partition_size, int32_t *d_status, pkv_stream_t stream) {
  using namespace pkv;
  // Sizes whose split-K partials do not fit the buffer are refused up front.
  const size_t need = pkv_paged_attention_workspace_size(num_seqs, num_q_heads, cache.num_kv_heads,
                                                         cache.head_dim, cache.block_size,
                                                         max_context_len, partition_size);
  if (need > kScratchBytes) return PKV_ERR_TOO_LARGE;
  pkv_status st = check_device();
  if (st != PKV_OK) return st;
  void *scratch = nullptr;
  if ((st = scratch_address(&scratch)) != PKV_OK) return st;
  // The regular entry point clears what must start at zero (its split arrival
  // counters, with an async memset on the stream) and writes every partial
  // before reading it.  Two calls whose kernels overlap on the GPU (e.g. on two
  // streams) share the buffer and race.
  return pkv_paged_attention_decode(out, query, k_cache, v_cache, cache, block_tables,
                                    max_blocks_per_seq, context_lens, num_seqs, num_q_heads,
                                    max_context_len, scale, partition_size, scratch, kScratchBytes,
                                    d_status, stream);
}
