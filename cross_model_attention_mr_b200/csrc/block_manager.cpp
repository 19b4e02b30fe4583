// Prefix-hash block manager for compressed maps: MapFlow section 5.3 ("Block Manager": prefix
// hashes map to the stored attention blocks of every sender layer, which are then streamed to the
// receiver) and section 1 (prefix-hash indexing).
//
// A sequence's compressed map row (head h, query block I) depends only on tokens 0 .. (I+1)B - 1,
// because the map is causal.  So the maps stored for one sequence serve, for their first k query
// blocks, every later request whose first k blocks of tokens are the same.  The manager keys each
// whole-block prefix by a chained hash of its tokens, remembers which stored sequences contain
// it, and answers "how many leading query blocks of this request can reuse stored maps, and
// which".  Host code only: the maps' device arrays stay owned by the caller, who frees an entry's
// arrays once the manager reports it evicted.
#include <stdint.h>

#include <algorithm>
#include <list>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "../../include/mr.h"

namespace {

// 64-bit mixing of one value into a running hash (the finaliser of the SplitMix64 generator,
// Steele, Lea and Flood, "Fast splittable pseudorandom number generators", 2014).
uint64_t mix(uint64_t h, uint64_t v) {
  uint64_t z = h ^ (v + 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2));
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  return z ^ (z >> 31);
}

struct Entry {
  std::vector<int32_t> tokens;       // whole blocks only
  std::vector<mr_bsr> maps;          // one per layer
  std::vector<uint64_t> hashes;      // prefix hash of blocks 0 .. k, k = 0 .. n_blocks - 1
  int64_t bytes = 0;
  int64_t refs = 0;
  std::list<int64_t>::iterator lru;  // position in the manager's recency list
};

}  // namespace

struct mr_block_manager {
  int block = 0;
  int64_t budget = 0;
  int64_t bytes = 0;
  int64_t next_id = 0;
  std::unordered_map<int64_t, Entry> entries;
  // prefix hash -> ids of the entries that contain that prefix (most recent last)
  std::unordered_map<uint64_t, std::vector<int64_t>> prefixes;
  std::list<int64_t> lru;            // front = most recently used
  std::vector<int64_t> evicted;      // ids whose arrays the caller may free
  int64_t lookups = 0, hits = 0, hit_blocks = 0;
  std::mutex mu;

  void touch(Entry& e, int64_t id) {
    lru.erase(e.lru);
    lru.push_front(id);
    e.lru = lru.begin();
  }

  void drop(int64_t id) {
    Entry& e = entries.at(id);
    for (uint64_t h : e.hashes) {
      auto it = prefixes.find(h);
      if (it == prefixes.end()) continue;
      auto& v = it->second;
      v.erase(std::remove(v.begin(), v.end(), id), v.end());
      if (v.empty()) prefixes.erase(it);
    }
    lru.erase(e.lru);
    bytes -= e.bytes;
    entries.erase(id);
    evicted.push_back(id);
  }

  // least recently used entries without references go until the budget holds
  void enforce_budget() {
    if (budget <= 0) return;
    std::vector<int64_t> victims;
    int64_t b = bytes;
    for (auto it = lru.rbegin(); it != lru.rend() && b > budget; ++it) {
      const Entry& e = entries.at(*it);
      if (e.refs > 0) continue;
      victims.push_back(*it);
      b -= e.bytes;
    }
    for (int64_t id : victims) drop(id);
  }
};

extern "C" {

mr_block_manager* mr_bm_create(int block, int64_t budget_bytes) {
  if (block < 1 || budget_bytes < 0) return nullptr;
  mr_block_manager* bm = new (std::nothrow) mr_block_manager();
  if (!bm) return nullptr;
  bm->block = block;
  bm->budget = budget_bytes;
  return bm;
}

void mr_bm_destroy(mr_block_manager* bm) { delete bm; }

int64_t mr_bm_insert(mr_block_manager* bm, const int32_t* tokens, int n_tokens, const mr_bsr* maps,
                     int n_layers, int64_t map_bytes) {
  if (!bm || !tokens || !maps || n_layers < 1 || map_bytes < 0) return -(int64_t)MR_ERR_INVALID_ARG;
  const int nb = n_tokens / bm->block;
  if (nb < 1) return -(int64_t)MR_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (maps[l].block != bm->block || maps[l].L < nb * bm->block) return -(int64_t)MR_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(bm->mu);
  const int64_t id = bm->next_id++;
  Entry e;
  e.tokens.assign(tokens, tokens + (size_t)nb * bm->block);
  e.maps.assign(maps, maps + n_layers);
  e.bytes = map_bytes;
  e.refs = 1;  // the caller holds the entry until it releases it
  uint64_t h = mix(0x6d61707265757365ull, (uint64_t)bm->block);
  for (int k = 0; k < nb; ++k) {
    for (int t = 0; t < bm->block; ++t) h = mix(h, (uint32_t)tokens[(size_t)k * bm->block + t]);
    e.hashes.push_back(h);
    bm->prefixes[h].push_back(id);
  }
  bm->lru.push_front(id);
  e.lru = bm->lru.begin();
  bm->bytes += map_bytes;
  bm->entries.emplace(id, std::move(e));
  bm->enforce_budget();
  return id;
}

int mr_bm_lookup(mr_block_manager* bm, const int32_t* tokens, int n_tokens, int64_t* entry) {
  if (!bm || !entry || (!tokens && n_tokens > 0) || n_tokens < 0) return -(int)MR_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(bm->mu);
  ++bm->lookups;
  *entry = -1;
  const int nb = n_tokens / bm->block;
  uint64_t h = mix(0x6d61707265757365ull, (uint64_t)bm->block);
  int best_k = 0;
  int64_t best = -1;
  for (int k = 0; k < nb; ++k) {
    for (int t = 0; t < bm->block; ++t) h = mix(h, (uint32_t)tokens[(size_t)k * bm->block + t]);
    auto it = bm->prefixes.find(h);
    if (it == bm->prefixes.end()) break;
    // the most recent entry that truly holds these tokens (a hash collision is not a hit)
    int64_t found = -1;
    for (auto r = it->second.rbegin(); r != it->second.rend(); ++r) {
      const Entry& e = bm->entries.at(*r);
      if (std::equal(tokens + (size_t)k * bm->block, tokens + (size_t)(k + 1) * bm->block,
                     e.tokens.begin() + (size_t)k * bm->block) &&
          (k == 0 || *r == best ||
           std::equal(tokens, tokens + (size_t)k * bm->block, e.tokens.begin()))) {
        found = *r;
        break;
      }
    }
    if (found < 0) break;
    best = found;
    best_k = k + 1;
  }
  if (best >= 0) {
    Entry& e = bm->entries.at(best);
    ++e.refs;
    bm->touch(e, best);
    ++bm->hits;
    bm->hit_blocks += best_k;
    *entry = best;
  }
  return best_k;
}

mr_status mr_bm_map(mr_block_manager* bm, int64_t entry, int layer, mr_bsr* out) {
  if (!bm || !out) return MR_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(bm->mu);
  auto it = bm->entries.find(entry);
  if (it == bm->entries.end() || layer < 0 || layer >= (int)it->second.maps.size()) return MR_ERR_INVALID_ARG;
  *out = it->second.maps[(size_t)layer];
  return MR_OK;
}

mr_status mr_bm_release(mr_block_manager* bm, int64_t entry) {
  if (!bm) return MR_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(bm->mu);
  auto it = bm->entries.find(entry);
  if (it == bm->entries.end() || it->second.refs < 1) return MR_ERR_INVALID_ARG;
  --it->second.refs;
  bm->enforce_budget();
  return MR_OK;
}

int mr_bm_evicted(mr_block_manager* bm, int64_t* ids, int max_ids) {
  if (!bm || (!ids && max_ids > 0) || max_ids < 0) return -(int)MR_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(bm->mu);
  const int n = std::min<int>(max_ids, (int)bm->evicted.size());
  std::copy(bm->evicted.begin(), bm->evicted.begin() + n, ids);
  bm->evicted.erase(bm->evicted.begin(), bm->evicted.begin() + n);
  return n;
}

mr_status mr_bm_stats(mr_block_manager* bm, int64_t* out) {
  if (!bm || !out) return MR_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(bm->mu);
  out[0] = (int64_t)bm->entries.size();
  out[1] = bm->bytes;
  out[2] = bm->lookups;
  out[3] = bm->hits;
  out[4] = bm->hit_blocks;
  return MR_OK;
}

}  // extern "C"
