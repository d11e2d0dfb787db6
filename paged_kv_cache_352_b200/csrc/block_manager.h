// The host block manager's state, shared by the block manager's C interface
// and the continuous-batching scheduler that drives it (both host-only).
#pragma once

#include <stdint.h>

#include <iterator>
#include <list>
#include <map>
#include <set>
#include <unordered_map>
#include <vector>

struct pa_bm {
  struct Seq {
    std::vector<int32_t> table;  // device blocks (empty while swapped out)
    std::vector<int32_t> host;   // host blocks while swapped out
    int64_t len = 0;
    bool swapped = false;
  };
  int num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_stack;  // back() is handed out next
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Seq> seqs;
  std::vector<int32_t> host_free;  // back() is handed out next
  int num_host_blocks = 0;
  int num_swapped = 0;

  // prefix cache: key = {parent block or -1, token ids of the block}
  std::map<std::vector<int32_t>, int32_t> cache;
  std::unordered_map<int32_t, std::vector<int32_t>> key_of;
  std::unordered_map<int32_t, std::set<int32_t>> children;
  std::list<int32_t> evictable;  // cached blocks with refcount 0, oldest first
  std::unordered_map<int32_t, std::list<int32_t>::iterator> evictable_pos;

  size_t num_free() const { return free_stack.size() + evictable.size(); }

  void evict(int32_t b) {
    auto ch = children.find(b);
    if (ch != children.end()) {
      const std::set<int32_t> kids = ch->second;  // ascending block ids
      children.erase(ch);
      for (int32_t c : kids) evict(c);
    }
    auto k = key_of.find(b);
    const int32_t parent = k->second[0];
    cache.erase(k->second);
    key_of.erase(k);
    if (parent >= 0) {
      auto pc = children.find(parent);
      if (pc != children.end()) pc->second.erase(b);
    }
    auto pos = evictable_pos.find(b);
    evictable.erase(pos->second);
    evictable_pos.erase(pos);
    free_stack.push_back(b);
  }

  // A block for new tokens: the free list first, else the oldest released cached block.
  int32_t pop() {
    if (free_stack.empty()) evict(evictable.front());
    const int32_t b = free_stack.back();
    free_stack.pop_back();
    ref[b] = 1;
    return b;
  }

  void release(int32_t b) {
    if (--ref[b] != 0) return;
    if (key_of.count(b)) {
      evictable.push_back(b);
      evictable_pos[b] = std::prev(evictable.end());
    } else {
      free_stack.push_back(b);
    }
  }
  int64_t slot(const Seq& s, int64_t pos) const {
    return (int64_t)s.table[pos / block_size] * block_size + pos % block_size;
  }
};
