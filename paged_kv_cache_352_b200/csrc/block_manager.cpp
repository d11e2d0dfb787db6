// Host block manager of the paged KV cache.
//
// A pool of equal blocks allocated once; per-sequence block tables mapping
// logical to physical blocks; blocks taken on demand as tokens arrive; refcounts
// so forked sequences share blocks, with a copy only when a sharer writes
// ("PagedAttention: The vLLM Paper", "Implementation Essentials" and "The OS
// paging analogy"; "PagedAttention and Continuous Batching", "Pages, from
// operating systems").
//
// Preemption by swapping: a sequence's blocks can move to a host pool and back
// ("PagedAttention: The vLLM Paper", "Implementation Essentials" and "The OS
// paging analogy", swapping). The host pool is a stack like the device pool;
// swap-out emits (device, host) copy pairs in logical order and releases device
// blocks last first, swap-in emits (host, device) pairs and releases host blocks
// last first. A swapped sequence cannot grow, fork or appear in block tables.
//
// Prefix caching across requests: the KV of shared prompt prefixes is kept and
// reused by later requests ("PagedAttention: The vLLM Paper", "Impact and
// Follow-Ups", item 1). A full prompt block is identified exactly by
// (physical block of the previous logical block or -1, its token ids); a
// sequence added with its token ids shares every leading block found. Cached
// blocks whose refcount falls to 0 stay reusable on a queue, least recently
// released first; blocks come from the free list first, then by evicting the
// queue's head together with any cached descendants.
//
// Every mutating call first works out how many free blocks it needs and fails
// before touching any state when the pool cannot cover it.
#include <algorithm>
#include <stdint.h>

#include <new>

#include "block_manager.h"
#include "pa_internal.h"

using pa::fail;

namespace {

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Physical blocks of the leading full blocks of a prompt found in the cache.
std::vector<int32_t> cached_prefix_blocks(const pa_bm* bm, const int32_t* token_ids,
                                          int num_tokens) {
  const int bs = bm->block_size;
  std::vector<int32_t> hits;
  std::vector<int32_t> key(bs + 1);
  int32_t parent = -1;
  for (int i = 0; i < num_tokens / bs; ++i) {
    key[0] = parent;
    for (int t = 0; t < bs; ++t) key[1 + t] = token_ids[i * bs + t];
    auto c = bm->cache.find(key);
    if (c == bm->cache.end()) break;
    hits.push_back(c->second);
    parent = c->second;
  }
  return hits;
}

int swapped_error(int64_t seq_id) {
  return fail(PA_ERR_SEQ_SWAPPED, "sequence %lld is swapped out", (long long)seq_id);
}

}  // namespace

extern "C" {

int pa_bm_create(int num_blocks, int block_size, const int32_t* initial_free_order,
                 pa_bm** out) {
  pa::clear_error();
  if (!out) return fail(PA_ERR_INVALID_ARG, "out must not be NULL");
  *out = nullptr;
  if (num_blocks <= 0 || block_size <= 0)
    return fail(PA_ERR_INVALID_ARG, "num_blocks and block_size must be positive");
  pa_bm* bm = new (std::nothrow) pa_bm;
  if (!bm) return fail(PA_ERR_INVALID_ARG, "out of host memory");
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->ref.assign(num_blocks, 0);
  bm->free_stack.resize(num_blocks);
  if (initial_free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t b = initial_free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        return fail(PA_ERR_INVALID_ARG, "initial_free_order is not a permutation of the pool");
      }
      seen[b] = 1;
      bm->free_stack[num_blocks - 1 - i] = b;
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) bm->free_stack[num_blocks - 1 - i] = i;
  }
  *out = bm;
  return PA_OK;
}

void pa_bm_destroy(pa_bm* bm) { delete bm; }

int pa_bm_add_seq(pa_bm* bm, int64_t seq_id, int num_tokens, int64_t* slots_out) {
  pa::clear_error();
  if (!bm) return fail(PA_ERR_INVALID_ARG, "null manager");
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens must be >= 0");
  if (num_tokens > 0 && !slots_out) return fail(PA_ERR_INVALID_ARG, "slots_out is NULL");
  if (bm->seqs.count(seq_id))
    return fail(PA_ERR_SEQ_EXISTS, "sequence %lld exists", (long long)seq_id);
  const int64_t need = ceil_div(num_tokens, bm->block_size);
  if (need > (int64_t)bm->num_free())
    return fail(PA_ERR_NO_FREE_BLOCKS, "need %lld blocks, %zu free", (long long)need,
                bm->num_free());
  pa_bm::Seq s;
  s.table.reserve(need);
  for (int64_t i = 0; i < need; ++i) s.table.push_back(bm->pop());
  s.len = num_tokens;
  for (int64_t p = 0; p < num_tokens; ++p) slots_out[p] = bm->slot(s, p);
  bm->seqs.emplace(seq_id, std::move(s));
  return PA_OK;
}

int pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child) {
  pa::clear_error();
  if (!bm) return fail(PA_ERR_INVALID_ARG, "null manager");
  auto it = bm->seqs.find(parent);
  if (it == bm->seqs.end())
    return fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)parent);
  if (it->second.swapped) return swapped_error(parent);
  if (bm->seqs.count(child))
    return fail(PA_ERR_SEQ_EXISTS, "sequence %lld exists", (long long)child);
  pa_bm::Seq s = it->second;
  for (int32_t b : s.table) ++bm->ref[b];
  bm->seqs.emplace(child, std::move(s));
  return PA_OK;
}

int pa_bm_append_slots(pa_bm* bm, int64_t seq_id, int n, int64_t* slots_out,
                       int64_t* cow_pairs_out, int* n_cow) {
  pa::clear_error();
  if (!bm) return fail(PA_ERR_INVALID_ARG, "null manager");
  if (n < 0) return fail(PA_ERR_INVALID_ARG, "n must be >= 0");
  if ((n > 0 && !slots_out) || !cow_pairs_out || !n_cow)
    return fail(PA_ERR_INVALID_ARG, "null output pointer");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
  pa_bm::Seq& s = it->second;
  if (s.swapped) return swapped_error(seq_id);
  const int bs = bm->block_size;
  const int64_t new_blocks = ceil_div(s.len + n, bs) - (int64_t)s.table.size();
  const bool cow = n > 0 && s.len % bs != 0 && bm->ref[s.table.back()] > 1;
  if (new_blocks + (cow ? 1 : 0) > (int64_t)bm->num_free())
    return fail(PA_ERR_NO_FREE_BLOCKS, "need %lld blocks, %zu free",
                (long long)(new_blocks + (cow ? 1 : 0)), bm->num_free());
  *n_cow = 0;
  if (cow) {
    const int32_t old = s.table.back();
    const int32_t fresh = bm->pop();
    --bm->ref[old];
    s.table.back() = fresh;
    cow_pairs_out[0] = old;
    cow_pairs_out[1] = fresh;
    *n_cow = 1;
  }
  for (int64_t p = s.len; p < s.len + n; ++p) {
    if (p % bs == 0) s.table.push_back(bm->pop());
    slots_out[p - s.len] = bm->slot(s, p);
  }
  s.len += n;
  return PA_OK;
}

int pa_bm_free_seq(pa_bm* bm, int64_t seq_id) {
  pa::clear_error();
  if (!bm) return fail(PA_ERR_INVALID_ARG, "null manager");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
  const std::vector<int32_t>& h = it->second.host;
  for (auto b = h.rbegin(); b != h.rend(); ++b) bm->host_free.push_back(*b);
  if (it->second.swapped) --bm->num_swapped;
  const std::vector<int32_t>& t = it->second.table;
  for (auto b = t.rbegin(); b != t.rend(); ++b) bm->release(*b);
  bm->seqs.erase(it);
  return PA_OK;
}

int pa_bm_block_tables(const pa_bm* bm, const int64_t* seq_ids, int n, int32_t* out,
                       int max_blocks) {
  pa::clear_error();
  if (!bm) return fail(PA_ERR_INVALID_ARG, "null manager");
  if (n < 0 || max_blocks < 0) return fail(PA_ERR_INVALID_ARG, "negative size");
  if (n == 0) return PA_OK;
  if (!seq_ids || !out) return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  for (int i = 0; i < n; ++i) {  // validate everything before writing anything
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end())
      return fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_ids[i]);
    if (it->second.swapped) return swapped_error(seq_ids[i]);
    if ((int64_t)it->second.table.size() > max_blocks)
      return fail(PA_ERR_INVALID_ARG, "sequence %lld holds %zu blocks > max_blocks %d",
                  (long long)seq_ids[i], it->second.table.size(), max_blocks);
  }
  for (int i = 0; i < n; ++i) {
    const std::vector<int32_t>& t = bm->seqs.find(seq_ids[i])->second.table;
    int32_t* row = out + (size_t)i * max_blocks;
    size_t k = 0;
    for (; k < t.size(); ++k) row[k] = t[k];
    for (; k < (size_t)max_blocks; ++k) row[k] = -1;
  }
  return PA_OK;
}

int pa_bm_prefix_groups(const pa_bm* bm, const int64_t* seq_ids, int n, int group_size,
                        int32_t* group_members, int32_t* group_prefix_blocks, int32_t* seq_group,
                        int32_t* seq_member, int* num_groups, int* max_prefix_blocks) {
  pa::clear_error();
  if (!bm) return fail(PA_ERR_INVALID_ARG, "null manager");
  if (n < 0 || group_size < 1) return fail(PA_ERR_INVALID_ARG, "bad n or group_size");
  if (!num_groups || !max_prefix_blocks) return fail(PA_ERR_INVALID_ARG, "null output pointer");
  if (n > 0 && (!seq_ids || !group_members || !group_prefix_blocks || !seq_group || !seq_member))
    return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  std::vector<const pa_bm::Seq*> seqs(n);
  for (int i = 0; i < n; ++i) {  // validate everything before writing anything
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end())
      return fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_ids[i]);
    if (it->second.swapped) return swapped_error(seq_ids[i]);
    seqs[i] = &it->second;
  }
  auto full = [&](int i) { return (int)(seqs[i]->len / bm->block_size); };
  std::vector<int32_t> first_keys;
  std::unordered_map<int32_t, std::vector<int>> buckets;
  for (int i = 0; i < n; ++i) {
    seq_group[i] = -1;
    seq_member[i] = -1;
    if (full(i) < 1) continue;
    const int32_t key = seqs[i]->table[0];
    auto& b = buckets[key];
    if (b.empty()) first_keys.push_back(key);
    b.push_back(i);
  }
  int ng = 0, maxp = 0;
  for (int32_t key : first_keys) {
    const std::vector<int>& b = buckets[key];
    for (size_t c = 0; c < b.size(); c += group_size) {
      const size_t m = std::min(b.size() - c, (size_t)group_size);
      if (m < 2) continue;
      const std::vector<int32_t>& lead = seqs[b[c]]->table;
      int P = full(b[c]);
      for (size_t j = 1; j < m; ++j) {
        const std::vector<int32_t>& t = seqs[b[c + j]]->table;
        P = std::min(P, full(b[c + j]));
        int k = 0;
        while (k < P && t[k] == lead[k]) ++k;
        P = k;
      }
      if (P < 1) continue;
      int32_t* row = group_members + (size_t)ng * group_size;
      for (int j = 0; j < group_size; ++j) row[j] = -1;
      for (size_t j = 0; j < m; ++j) {
        row[j] = b[c + j];
        seq_group[b[c + j]] = ng;
        seq_member[b[c + j]] = (int32_t)j;
      }
      group_prefix_blocks[ng] = P;
      maxp = std::max(maxp, P);
      ++ng;
    }
  }
  *num_groups = ng;
  *max_prefix_blocks = maxp;
  return PA_OK;
}

int pa_bm_num_free(const pa_bm* bm) { return bm ? (int)bm->num_free() : -1; }

int pa_bm_add_seq_cached(pa_bm* bm, int64_t seq_id, const int32_t* token_ids, int num_tokens,
                         int64_t* slots_out, int* num_cached_tokens) {
  pa::clear_error();
  if (!bm || !num_cached_tokens) return fail(PA_ERR_INVALID_ARG, "null argument");
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens must be >= 0");
  if (num_tokens > 0 && (!slots_out || !token_ids))
    return fail(PA_ERR_INVALID_ARG, "null token_ids or slots_out");
  if (bm->seqs.count(seq_id))
    return fail(PA_ERR_SEQ_EXISTS, "sequence %lld exists", (long long)seq_id);
  const int bs = bm->block_size;
  const int full = num_tokens / bs;
  std::vector<int32_t> hits = cached_prefix_blocks(bm, token_ids, num_tokens);
  std::vector<int32_t> key(bs + 1);
  int32_t parent = hits.empty() ? -1 : hits.back();
  const int64_t need = ceil_div(num_tokens, bs) - (int64_t)hits.size();
  int64_t revived = 0;
  for (int32_t b : hits) revived += bm->ref[b] == 0;
  if (need > (int64_t)bm->num_free() - revived)
    return fail(PA_ERR_NO_FREE_BLOCKS, "need %lld blocks, %lld free", (long long)need,
                (long long)(bm->num_free() - revived));
  for (int32_t b : hits) {
    if (bm->ref[b] == 0) {
      auto pos = bm->evictable_pos.find(b);
      bm->evictable.erase(pos->second);
      bm->evictable_pos.erase(pos);
    }
    ++bm->ref[b];
  }
  pa_bm::Seq s;
  s.table = hits;
  const int64_t nblk = ceil_div(num_tokens, bs);
  for (int64_t i = (int64_t)hits.size(); i < nblk; ++i) {
    const int32_t b = bm->pop();
    s.table.push_back(b);
    if (i < full) {
      key[0] = parent;
      for (int t = 0; t < bs; ++t) key[1 + t] = token_ids[i * bs + t];
      bm->cache[key] = b;
      bm->key_of[b] = key;
      if (parent >= 0) bm->children[parent].insert(b);
      parent = b;
    }
  }
  s.len = num_tokens;
  for (int64_t p = 0; p < num_tokens; ++p) slots_out[p] = bm->slot(s, p);
  bm->seqs.emplace(seq_id, std::move(s));
  *num_cached_tokens = (int)hits.size() * bs;
  return PA_OK;
}

int pa_bm_cached_prefix(const pa_bm* bm, const int32_t* token_ids, int num_tokens,
                        int* hit_blocks, int* revived_blocks) {
  pa::clear_error();
  if (!bm || !hit_blocks || !revived_blocks) return fail(PA_ERR_INVALID_ARG, "null argument");
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens must be >= 0");
  if (num_tokens > 0 && !token_ids) return fail(PA_ERR_INVALID_ARG, "null token_ids");
  const std::vector<int32_t> hits = cached_prefix_blocks(bm, token_ids, num_tokens);
  int revived = 0;
  for (int32_t b : hits) revived += bm->ref[b] == 0;
  *hit_blocks = (int)hits.size();
  *revived_blocks = revived;
  return PA_OK;
}

int pa_bm_num_cached(const pa_bm* bm) { return bm ? (int)bm->key_of.size() : -1; }

int pa_bm_evictable_list(const pa_bm* bm, int32_t* out, int capacity) {
  if (!bm || (!out && capacity > 0) || capacity < 0) return -1;
  int i = 0;
  for (auto it = bm->evictable.begin(); it != bm->evictable.end() && i < capacity; ++it)
    out[i++] = *it;
  return i;
}

int pa_bm_refcount(const pa_bm* bm, int32_t block) {
  if (!bm || block < 0 || block >= bm->num_blocks) {
    fail(PA_ERR_INVALID_ARG, "block id out of range");
    return -1;
  }
  return bm->ref[block];
}

int pa_bm_seq_len(const pa_bm* bm, int64_t seq_id) {
  if (!bm) return -1;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) {
    fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
    return -1;
  }
  return (int)it->second.len;
}

int pa_bm_num_seqs(const pa_bm* bm) { return bm ? (int)bm->seqs.size() : -1; }

int pa_bm_set_host_pool(pa_bm* bm, int num_host_blocks) {
  pa::clear_error();
  if (!bm) return fail(PA_ERR_INVALID_ARG, "null manager");
  if (num_host_blocks < 0) return fail(PA_ERR_INVALID_ARG, "num_host_blocks must be >= 0");
  if (bm->num_swapped > 0) return fail(PA_ERR_INVALID_ARG, "host blocks are in use");
  bm->num_host_blocks = num_host_blocks;
  bm->host_free.resize(num_host_blocks);
  for (int i = 0; i < num_host_blocks; ++i) bm->host_free[num_host_blocks - 1 - i] = i;
  return PA_OK;
}

int pa_bm_swap_out(pa_bm* bm, int64_t seq_id, int64_t* pairs_out, int capacity, int* n_pairs) {
  pa::clear_error();
  if (!bm || !n_pairs) return fail(PA_ERR_INVALID_ARG, "null argument");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
  pa_bm::Seq& s = it->second;
  if (s.swapped) return swapped_error(seq_id);
  const int n = (int)s.table.size();
  if (n > capacity || (n > 0 && !pairs_out))
    return fail(PA_ERR_INVALID_ARG, "pairs_out holds %d pairs, %d needed", capacity, n);
  if (n > (int)bm->host_free.size())
    return fail(PA_ERR_NO_FREE_BLOCKS, "need %d host blocks, %zu free", n, bm->host_free.size());
  s.host.resize(n);
  for (int i = 0; i < n; ++i) {
    s.host[i] = bm->host_free.back();
    bm->host_free.pop_back();
    pairs_out[2 * i] = s.table[i];
    pairs_out[2 * i + 1] = s.host[i];
  }
  for (int i = n - 1; i >= 0; --i) bm->release(s.table[i]);
  s.table.clear();
  s.swapped = true;
  ++bm->num_swapped;
  *n_pairs = n;
  return PA_OK;
}

int pa_bm_swap_in(pa_bm* bm, int64_t seq_id, int64_t* pairs_out, int capacity, int* n_pairs) {
  pa::clear_error();
  if (!bm || !n_pairs) return fail(PA_ERR_INVALID_ARG, "null argument");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
  pa_bm::Seq& s = it->second;
  if (!s.swapped)
    return fail(PA_ERR_SEQ_SWAPPED, "sequence %lld is not swapped out", (long long)seq_id);
  const int n = (int)s.host.size();
  if (n > capacity || (n > 0 && !pairs_out))
    return fail(PA_ERR_INVALID_ARG, "pairs_out holds %d pairs, %d needed", capacity, n);
  if (n > (int)bm->num_free())
    return fail(PA_ERR_NO_FREE_BLOCKS, "need %d blocks, %zu free", n, bm->num_free());
  s.table.resize(n);
  for (int i = 0; i < n; ++i) {
    s.table[i] = bm->pop();
    pairs_out[2 * i] = s.host[i];
    pairs_out[2 * i + 1] = s.table[i];
  }
  for (int i = n - 1; i >= 0; --i) bm->host_free.push_back(s.host[i]);
  s.host.clear();
  s.swapped = false;
  --bm->num_swapped;
  *n_pairs = n;
  return PA_OK;
}

int pa_bm_is_swapped(const pa_bm* bm, int64_t seq_id) {
  if (!bm) return -1;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) {
    fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
    return -1;
  }
  return it->second.swapped ? 1 : 0;
}

int pa_bm_num_free_host(const pa_bm* bm) { return bm ? (int)bm->host_free.size() : -1; }

int pa_bm_host_free_list(const pa_bm* bm, int32_t* out, int capacity) {
  if (!bm || (!out && capacity > 0) || capacity < 0) return -1;
  const int n = (int)bm->host_free.size();
  const int m = n < capacity ? n : capacity;
  for (int i = 0; i < m; ++i) out[i] = bm->host_free[n - 1 - i];
  return m;
}

int pa_bm_free_list(const pa_bm* bm, int32_t* out, int capacity) {
  if (!bm || (!out && capacity > 0) || capacity < 0) return -1;
  const int n = (int)bm->free_stack.size();
  const int m = n < capacity ? n : capacity;
  for (int i = 0; i < m; ++i) out[i] = bm->free_stack[n - 1 - i];
  return m;
}

}  // extern "C"
