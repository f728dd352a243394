// Host block manager of a paged KV cache: free pool, reference counts, one
// Block Table per request, the append rule and copy-on-write.
//
// lshu.cn/news/11644 (vLLM architecture analysis): "整体架构" (blocks handed
// out on demand from one global pool and returned when a request finishes),
// "方案：页式内存管理" (Block Table per request; a new token goes into the last
// block while it has room, else a block is taken from the free pool) and
// "收益分析" (shared prefix blocks, copy-on-write on divergence).  The rules the
// pages leave open are fixed in pkv_block_manager.h.
#include "pkv_block_manager.h"

#include <algorithm>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

namespace {

struct Sequence {
  std::vector<int32_t> table;
  int32_t len = 0;
};

// First-in first-out queue of block ids over a fixed ring.
class FreePool {
 public:
  explicit FreePool(int32_t n) : ring_(static_cast<size_t>(n)), head_(0), size_(n) {
    for (int32_t i = 0; i < n; ++i) ring_[static_cast<size_t>(i)] = i;
  }
  int32_t size() const { return size_; }
  int32_t pop() {
    const int32_t b = ring_[static_cast<size_t>(head_)];
    head_ = next(head_);
    --size_;
    return b;
  }
  void push(int32_t b) {
    int64_t tail = static_cast<int64_t>(head_) + size_;
    if (tail >= static_cast<int64_t>(ring_.size())) tail -= static_cast<int64_t>(ring_.size());
    ring_[static_cast<size_t>(tail)] = b;
    ++size_;
  }
  int32_t at(int32_t i) const {
    int64_t k = static_cast<int64_t>(head_) + i;
    if (k >= static_cast<int64_t>(ring_.size())) k -= static_cast<int64_t>(ring_.size());
    return ring_[static_cast<size_t>(k)];
  }

 private:
  int32_t next(int32_t i) const { return i + 1 == static_cast<int32_t>(ring_.size()) ? 0 : i + 1; }
  std::vector<int32_t> ring_;
  int32_t head_;
  int32_t size_;
};

}  // namespace

struct pkv_block_manager {
  pkv_block_manager(int32_t n, int32_t b, int32_t m)
      : num_blocks(n), block_size(b), max_blocks(m), pool(n), ref(static_cast<size_t>(n), 0),
        copied(static_cast<size_t>(n), 0) {}

  const int32_t num_blocks;
  const int32_t block_size;
  const int32_t max_blocks;
  FreePool pool;
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Sequence> seqs;
  std::vector<int32_t> copied;   // scratch: copies of a block counted in one step
  std::vector<Sequence *> batch;  // scratch: the step's sequences
  mutable std::mutex mu;

  int32_t take() {
    const int32_t b = pool.pop();
    ref[static_cast<size_t>(b)] = 1;
    return b;
  }
  void release(int32_t b) {
    if (--ref[static_cast<size_t>(b)] == 0) pool.push(b);
  }

  // Resolve ids into `batch`; false for an unknown or repeated id.
  bool resolve(const int64_t *ids, int32_t n) {
    batch.clear();
    for (int32_t i = 0; i < n; ++i) {
      auto it = seqs.find(ids[i]);
      if (it == seqs.end()) return false;
      batch.push_back(&it->second);
    }
    std::vector<Sequence *> sorted(batch);
    std::sort(sorted.begin(), sorted.end());
    return std::adjacent_find(sorted.begin(), sorted.end()) == sorted.end();
  }

  // Blocks an append over `batch` takes; the scratch counts are left at zero.
  int64_t needed() {
    int64_t n = 0;
    for (Sequence *q : batch) {
      if (q->len % block_size == 0) {
        ++n;
        continue;
      }
      const size_t last = static_cast<size_t>(q->table.back());
      if (ref[last] - copied[last] > 1) {
        ++copied[last];
        ++n;
      }
    }
    for (Sequence *q : batch)
      if (!q->table.empty()) copied[static_cast<size_t>(q->table.back())] = 0;
    return n;
  }
};

// No C++ exception leaves the C ABI: the calls that allocate host memory
// return PKV_ERR_TOO_LARGE when it runs out, and they allocate before they
// change anything, so the manager is then unchanged.
extern "C" {

pkv_status pkv_bm_create(int32_t num_blocks, int32_t block_size, int32_t max_blocks_per_seq,
                         pkv_block_manager **out) try {
  if (out == nullptr) return PKV_ERR_NULL_POINTER;
  *out = nullptr;
  if (num_blocks < 1 || block_size < 1 || max_blocks_per_seq < 1) return PKV_ERR_BAD_SHAPE;
  *out = new pkv_block_manager(num_blocks, block_size, max_blocks_per_seq);
  return PKV_OK;
} catch (const std::bad_alloc &) {
  return PKV_ERR_TOO_LARGE;
}

void pkv_bm_destroy(pkv_block_manager *bm) { delete bm; }

int32_t pkv_bm_num_free_blocks(const pkv_block_manager *bm) {
  if (bm == nullptr) return -1;
  std::lock_guard<std::mutex> g(bm->mu);
  return bm->pool.size();
}

int32_t pkv_bm_num_sequences(const pkv_block_manager *bm) {
  if (bm == nullptr) return -1;
  std::lock_guard<std::mutex> g(bm->mu);
  return static_cast<int32_t>(bm->seqs.size());
}

int32_t pkv_bm_ref_count(const pkv_block_manager *bm, int32_t block) {
  if (bm == nullptr || block < 0 || block >= bm->num_blocks) return -1;
  std::lock_guard<std::mutex> g(bm->mu);
  return bm->ref[static_cast<size_t>(block)];
}

int32_t pkv_bm_context_len(const pkv_block_manager *bm, int64_t seq_id) {
  if (bm == nullptr) return -1;
  std::lock_guard<std::mutex> g(bm->mu);
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? -1 : it->second.len;
}

pkv_status pkv_bm_add_sequence(pkv_block_manager *bm, int64_t seq_id, int32_t num_tokens,
                               int64_t *slot_mapping) try {
  if (bm == nullptr) return PKV_ERR_NULL_POINTER;
  if (num_tokens < 0) return PKV_ERR_BAD_SHAPE;
  std::lock_guard<std::mutex> g(bm->mu);
  if (bm->seqs.count(seq_id)) return PKV_ERR_BAD_SEQUENCE;
  const int64_t B = bm->block_size;
  const int64_t nb = (num_tokens + B - 1) / B;
  if (nb > bm->max_blocks) return PKV_ERR_TOO_LARGE;
  if (nb > bm->pool.size()) return PKV_ERR_NO_BLOCKS;
  Sequence q;
  q.table.reserve(static_cast<size_t>(nb));
  Sequence &dst = bm->seqs.emplace(seq_id, Sequence{}).first->second;  // the last allocation
  for (int64_t j = 0; j < nb; ++j) q.table.push_back(bm->take());
  q.len = num_tokens;
  if (slot_mapping != nullptr)
    for (int64_t t = 0; t < num_tokens; ++t)
      slot_mapping[t] = static_cast<int64_t>(q.table[static_cast<size_t>(t / B)]) * B + t % B;
  dst = std::move(q);
  return PKV_OK;
} catch (const std::bad_alloc &) {
  return PKV_ERR_TOO_LARGE;
}

pkv_status pkv_bm_fork(pkv_block_manager *bm, int64_t parent_id, int64_t child_id) try {
  if (bm == nullptr) return PKV_ERR_NULL_POINTER;
  std::lock_guard<std::mutex> g(bm->mu);
  auto it = bm->seqs.find(parent_id);
  if (it == bm->seqs.end() || bm->seqs.count(child_id)) return PKV_ERR_BAD_SEQUENCE;
  Sequence child = it->second;
  const Sequence &added = bm->seqs.emplace(child_id, std::move(child)).first->second;
  for (int32_t b : added.table) ++bm->ref[static_cast<size_t>(b)];
  return PKV_OK;
} catch (const std::bad_alloc &) {
  return PKV_ERR_TOO_LARGE;
}

pkv_status pkv_bm_free_sequence(pkv_block_manager *bm, int64_t seq_id) {
  if (bm == nullptr) return PKV_ERR_NULL_POINTER;
  std::lock_guard<std::mutex> g(bm->mu);
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PKV_ERR_BAD_SEQUENCE;
  for (int32_t b : it->second.table) bm->release(b);
  bm->seqs.erase(it);
  return PKV_OK;
}

int32_t pkv_bm_blocks_needed(const pkv_block_manager *cbm, const int64_t *seq_ids, int32_t n) try {
  if (cbm == nullptr || n < 0 || (n > 0 && seq_ids == nullptr)) return -1;
  auto *bm = const_cast<pkv_block_manager *>(cbm);  // only the scratch vectors change
  std::lock_guard<std::mutex> g(bm->mu);
  if (!bm->resolve(seq_ids, n)) return -1;
  return static_cast<int32_t>(bm->needed());
} catch (const std::bad_alloc &) {
  return -1;
}

pkv_status pkv_bm_append(pkv_block_manager *bm, const int64_t *seq_ids, int32_t n,
                         int64_t *slot_mapping, int64_t *copy_pairs, int32_t copy_capacity,
                         int32_t *num_copies) try {
  if (bm == nullptr) return PKV_ERR_NULL_POINTER;
  if (n < 0 || copy_capacity < n) return PKV_ERR_BAD_SHAPE;
  if (n > 0 && (seq_ids == nullptr || slot_mapping == nullptr || copy_pairs == nullptr))
    return PKV_ERR_NULL_POINTER;
  if (num_copies == nullptr) return PKV_ERR_NULL_POINTER;
  std::lock_guard<std::mutex> g(bm->mu);
  *num_copies = 0;
  if (!bm->resolve(seq_ids, n)) return PKV_ERR_BAD_SEQUENCE;
  const int32_t B = bm->block_size;
  for (Sequence *q : bm->batch)
    if (q->len % B == 0 && static_cast<int64_t>(q->table.size()) + 1 > bm->max_blocks)
      return PKV_ERR_TOO_LARGE;
  if (bm->needed() > bm->pool.size()) return PKV_ERR_NO_BLOCKS;
  for (Sequence *q : bm->batch)  // the step's only allocations, before anything changes
    if (q->len % B == 0) q->table.reserve(q->table.size() + 1);
  int32_t copies = 0;
  for (int32_t i = 0; i < n; ++i) {
    Sequence *q = bm->batch[static_cast<size_t>(i)];
    if (q->len % B == 0) {
      q->table.push_back(bm->take());
    } else if (bm->ref[static_cast<size_t>(q->table.back())] > 1) {
      const int32_t old = q->table.back();
      const int32_t fresh = bm->take();
      --bm->ref[static_cast<size_t>(old)];  // still held by another table
      q->table.back() = fresh;
      copy_pairs[2 * copies] = old;
      copy_pairs[2 * copies + 1] = fresh;
      ++copies;
    }
    slot_mapping[i] = static_cast<int64_t>(q->table.back()) * B + q->len % B;
    ++q->len;
  }
  *num_copies = copies;
  return PKV_OK;
} catch (const std::bad_alloc &) {
  return PKV_ERR_TOO_LARGE;
}

pkv_status pkv_bm_block_tables(const pkv_block_manager *cbm, const int64_t *seq_ids, int32_t n,
                               int32_t *block_tables, int32_t row_stride, int32_t *context_lens) {
  if (cbm == nullptr) return PKV_ERR_NULL_POINTER;
  if (n < 0 || row_stride < cbm->max_blocks) return PKV_ERR_BAD_SHAPE;
  if (n > 0 && (seq_ids == nullptr || block_tables == nullptr || context_lens == nullptr))
    return PKV_ERR_NULL_POINTER;
  std::lock_guard<std::mutex> g(cbm->mu);
  for (int32_t i = 0; i < n; ++i)
    if (!cbm->seqs.count(seq_ids[i])) return PKV_ERR_BAD_SEQUENCE;
  for (int32_t i = 0; i < n; ++i) {
    const Sequence &q = cbm->seqs.find(seq_ids[i])->second;
    int32_t *row = block_tables + static_cast<int64_t>(i) * row_stride;
    const size_t used = q.table.size();
    std::copy(q.table.begin(), q.table.end(), row);
    std::fill(row + used, row + row_stride, -1);
    context_lens[i] = q.len;
  }
  return PKV_OK;
}

pkv_status pkv_bm_free_list(const pkv_block_manager *bm, int32_t *out, int32_t capacity,
                            int32_t *count) {
  if (bm == nullptr || count == nullptr) return PKV_ERR_NULL_POINTER;
  if (capacity < 0) return PKV_ERR_BAD_SHAPE;
  std::lock_guard<std::mutex> g(bm->mu);
  *count = bm->pool.size();
  const int32_t k = std::min(capacity, bm->pool.size());
  if (k > 0 && out == nullptr) return PKV_ERR_NULL_POINTER;
  for (int32_t i = 0; i < k; ++i) out[i] = bm->pool.at(i);
  return PKV_OK;
}

}  // extern "C"
