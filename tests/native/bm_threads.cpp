// Several host threads drive one block manager of libpkv at once (each its
// own requests: add, fork, one-token steps, free; some steps refused for want
// of blocks), then the pool is checked: every request has the length its
// thread gave it, each block's reference count is the number of Block Tables
// holding it, and the free blocks and the held ones partition the pool.
// Exit status 0 when consistent, 1 when not, 2 on a setup error.
// Usage: bm_threads [threads] [steps per thread]
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <iterator>
#include <map>
#include <mutex>
#include <random>
#include <thread>
#include <vector>

#include "pkv_block_manager.h"

int main(int argc, char **argv) {
  const int threads = argc > 1 ? std::atoi(argv[1]) : 8;
  const int steps = argc > 2 ? std::atoi(argv[2]) : 4000;
  const int32_t N = 1 << 14, B = 16, M = 128;
  pkv_block_manager *bm = nullptr;
  if (pkv_bm_create(N, B, M, &bm) != PKV_OK) return 2;

  std::mutex guard;
  std::map<int64_t, int32_t> expected;
  int unexpected = 0;
  auto worker = [&](int t) {
    std::mt19937_64 rng(1000 + t);
    std::map<int64_t, int32_t> live;
    std::vector<int64_t> slots(M * B), pairs(2 * M * B), ids;
    int bad = 0;
    for (int it = 0; it < steps; ++it) {
      const int64_t sid = static_cast<int64_t>(t) * 100000000 + it;
      const int r = static_cast<int>(rng() % 100);
      if (r < 30 || live.size() < 4) {
        const int32_t n = 1 + static_cast<int32_t>(rng() % 200);
        const pkv_status s = pkv_bm_add_sequence(bm, sid, n, slots.data());
        if (s == PKV_OK) live[sid] = n;
        else if (s != PKV_ERR_NO_BLOCKS) ++bad;
      } else if (r < 40) {
        auto p = std::next(live.begin(), static_cast<long>(rng() % live.size()));
        if (pkv_bm_fork(bm, p->first, sid) == PKV_OK) live[sid] = p->second;
        else ++bad;
      } else if (r < 85) {
        ids.clear();
        for (const auto &kv : live)
          if (kv.second < M * B && ids.size() < 64) ids.push_back(kv.first);
        int32_t k = 0;
        const pkv_status s = pkv_bm_append(bm, ids.data(), static_cast<int32_t>(ids.size()), slots.data(),
                                           pairs.data(), static_cast<int32_t>(ids.size()), &k);
        if (s == PKV_OK) {
          for (const int64_t id : ids) ++live[id];
        } else if (s != PKV_ERR_NO_BLOCKS) {
          ++bad;
        }
      } else {
        auto v = std::next(live.begin(), static_cast<long>(rng() % live.size()));
        if (pkv_bm_free_sequence(bm, v->first) != PKV_OK) ++bad;
        live.erase(v);
      }
    }
    std::lock_guard<std::mutex> g(guard);
    expected.insert(live.begin(), live.end());
    unexpected += bad;
  };
  std::vector<std::thread> pool;
  for (int t = 0; t < threads; ++t) pool.emplace_back(worker, t);
  for (auto &th : pool) th.join();

  int errors = unexpected;
  if (pkv_bm_num_sequences(bm) != static_cast<int32_t>(expected.size())) ++errors;
  std::vector<int64_t> held(N, 0);
  std::vector<int32_t> row(M), len(1);
  for (const auto &kv : expected) {
    if (pkv_bm_block_tables(bm, &kv.first, 1, row.data(), M, len.data()) != PKV_OK || len[0] != kv.second) {
      ++errors;
      continue;
    }
    for (int32_t j = 0; j < (len[0] + B - 1) / B; ++j) {
      if (row[j] < 0 || row[j] >= N) ++errors;
      else ++held[row[j]];
    }
  }
  for (int32_t b = 0; b < N; ++b)
    if (pkv_bm_ref_count(bm, b) != held[b]) ++errors;
  std::vector<int32_t> free_ids(N);
  int32_t nfree = 0;
  if (pkv_bm_free_list(bm, free_ids.data(), N, &nfree) != PKV_OK || nfree != pkv_bm_num_free_blocks(bm)) ++errors;
  free_ids.resize(std::min(nfree, N));
  std::vector<char> seen(N, 0);
  for (const int32_t b : free_ids) {
    if (b < 0 || b >= N || seen[b] || held[b]) ++errors;
    else seen[b] = 1;
  }
  const long used = std::count_if(held.begin(), held.end(), [](int64_t h) { return h > 0; });
  if (used + nfree != N) ++errors;
  std::printf("requests %zu, free blocks %d, inconsistencies %d\n", expected.size(), nfree, errors);
  pkv_bm_destroy(bm);
  return errors == 0 ? 0 : 1;
}
