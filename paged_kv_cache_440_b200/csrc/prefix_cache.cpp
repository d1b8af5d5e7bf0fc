// Prefix cache: a radix tree over token sequences whose nodes hold the KV
// blocks already computed for those tokens, so that a request whose prompt
// starts with a cached prefix reuses the blocks instead of recomputing them
// [bjdmk.com.cn/news/6246348, §4.1 (prefix caching), §4.2 (radix tree,
// longest-prefix match, LRU eviction from the leaves); KV Cache 原理与
// PagedAttention, §五].
//
// Each edge carries a run of whole blocks: its token label (a multiple of
// block_size tokens) and one block id per block_size tokens, with a last-use
// tick per block. Children are keyed by the tokens of their first block. A
// lookup walks whole blocks as far as they match and may end with a block that
// matches only in part (the caller copies that block before writing to it).
// The cache holds one pool reference per cached block; every block a lookup
// returns carries one more reference, owned by the caller. Eviction drops the
// least recently used leaf block that only the cache holds, repeatedly.
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <vector>

#include "internal.h"

using namespace pagedkv;

namespace {

struct Node {
  std::vector<int32_t> tokens;   // edge label: blocks.size() * bs tokens
  std::vector<int32_t> blocks;   // one pool block per bs tokens of the label
  std::vector<uint64_t> tick;    // last use of each block
  std::map<std::vector<int32_t>, std::unique_ptr<Node>> kids;  // by first block's tokens
  Node *parent = nullptr;
};

}  // namespace

struct kv_prefix_cache {
  kv_pool *pool = nullptr;
  int bs = 0;
  std::mutex mu;
  Node root;
  uint64_t clock = 0;
  int64_t nodes = 0;
  int64_t cached = 0;
  int64_t lookups = 0, hits = 0, hit_tokens = 0;
};

namespace {

std::vector<int32_t> block_key(const int32_t *t, int bs) { return std::vector<int32_t>(t, t + bs); }

int ref_of(kv_pool *p, int32_t id) {
  int32_t r = 0;
  if (kv_block_refcount(p, id, &r) != KV_OK) return -1;
  return r;
}

// Split `n` after its first `e` blocks: the head keeps them, a new child gets
// the rest (with n's children).
Node *split(kv_prefix_cache *pc, Node *n, size_t e) {
  const int bs = pc->bs;
  auto tail = std::make_unique<Node>();
  tail->tokens.assign(n->tokens.begin() + e * bs, n->tokens.end());
  tail->blocks.assign(n->blocks.begin() + e, n->blocks.end());
  tail->tick.assign(n->tick.begin() + e, n->tick.end());
  tail->kids = std::move(n->kids);
  for (auto &kv : tail->kids) kv.second->parent = tail.get();
  tail->parent = n;
  n->tokens.resize(e * bs);
  n->blocks.resize(e);
  n->tick.resize(e);
  n->kids.clear();
  std::vector<int32_t> key = block_key(tail->tokens.data(), bs);
  n->kids.emplace(std::move(key), std::move(tail));
  pc->nodes++;
  return n;
}

void collect_blocks(const Node *n, std::vector<int32_t> *out) {
  out->insert(out->end(), n->blocks.begin(), n->blocks.end());
  for (const auto &kv : n->kids) collect_blocks(kv.second.get(), out);
}

// Least recently used leaf block held by the cache alone: (node, tick, id).
void best_leaf(kv_prefix_cache *pc, Node *n, Node **best, uint64_t *bt, int32_t *bid) {
  if (n->kids.empty()) {
    if (n != &pc->root && !n->blocks.empty()) {
      const int32_t id = n->blocks.back();
      const uint64_t t = n->tick.back();
      if (ref_of(pc->pool, id) == 1 &&
          (*best == nullptr || t < *bt || (t == *bt && id < *bid))) {
        *best = n;
        *bt = t;
        *bid = id;
      }
    }
    return;
  }
  for (auto &kv : n->kids) best_leaf(pc, kv.second.get(), best, bt, bid);
}

}  // namespace

extern "C" {

kv_status kv_prefix_cache_create(kv_pool *pool, kv_prefix_cache **out) {
  if (!pool || !out) return fail(KV_ERR_INVALID, "null argument");
  auto *pc = new kv_prefix_cache();
  pc->pool = pool;
  pc->bs = pool->d.block_size;
  *out = pc;
  return ok();
}

kv_status kv_prefix_clear(kv_prefix_cache *pc) {
  if (!pc) return fail(KV_ERR_INVALID, "null cache");
  std::lock_guard<std::mutex> g(pc->mu);
  std::vector<int32_t> ids;
  for (const auto &kv : pc->root.kids) collect_blocks(kv.second.get(), &ids);
  if (!ids.empty()) {
    kv_status s = kv_free_blocks(pc->pool, static_cast<int32_t>(ids.size()), ids.data());
    if (s != KV_OK) return s;
  }
  pc->root.kids.clear();
  pc->nodes = 0;
  pc->cached = 0;
  return ok();
}

kv_status kv_prefix_cache_destroy(kv_prefix_cache *pc) {
  if (!pc) return ok();
  kv_status s = kv_prefix_clear(pc);
  delete pc;
  return s;
}

kv_status kv_prefix_match(kv_prefix_cache *pc, const int32_t *tokens, int32_t n,
                          int32_t max_blocks, int32_t *block_ids, int32_t *num_blocks,
                          int32_t *matched_tokens) {
  if (!pc || !num_blocks || !matched_tokens) return fail(KV_ERR_INVALID, "null argument");
  if (n < 0 || (n > 0 && !tokens)) return fail(KV_ERR_INVALID, "bad token array");
  const int bs = pc->bs;
  if (max_blocks < (n + bs - 1) / bs || (max_blocks > 0 && !block_ids))
    return fail(KV_ERR_INVALID, "block_ids must hold ceil(n / block_size) = %d ids",
                (n + bs - 1) / bs);
  std::lock_guard<std::mutex> g(pc->mu);
  const uint64_t now = ++pc->clock;
  std::vector<int32_t> ids;
  Node *node = &pc->root;
  int32_t pos = 0;
  // whole blocks
  Node *edge = nullptr;  // edge we stopped inside, if any
  size_t e = 0;
  while (pos + bs <= n) {
    auto it = node->kids.find(block_key(tokens + pos, bs));
    if (it == node->kids.end()) break;
    Node *c = it->second.get();
    e = 0;
    while (e < c->blocks.size() && pos + bs <= n &&
           std::memcmp(c->tokens.data() + e * bs, tokens + pos, bs * sizeof(int32_t)) == 0) {
      ids.push_back(c->blocks[e]);
      c->tick[e] = now;
      pos += bs;
      ++e;
    }
    if (e < c->blocks.size()) {
      edge = c;
      break;
    }
    node = c;
  }
  int32_t matched = pos;
  // part of one more block: the next block of the edge we stopped in, or the
  // first block of one of the node's children
  if (pos < n) {
    int best_j = 0;
    int32_t best_id = -1;
    Node *best_n = nullptr;
    size_t best_e = 0;
    auto consider = [&](Node *c, size_t ce) {
      const int32_t *lab = c->tokens.data() + ce * bs;
      int j = 0;
      while (j < bs && pos + j < n && lab[j] == tokens[pos + j]) ++j;
      const int32_t id = c->blocks[ce];
      if (j >= 1 && (j > best_j || (j == best_j && id < best_id))) {
        best_j = j;
        best_id = id;
        best_n = c;
        best_e = ce;
      }
    };
    if (edge) {
      consider(edge, e);
    } else {
      for (auto &kv : node->kids) consider(kv.second.get(), 0);
    }
    if (best_n) {
      ids.push_back(best_id);
      best_n->tick[best_e] = now;
      matched += best_j;
    }
  }
  if (!ids.empty()) {
    kv_status s = kv_share_blocks(pc->pool, static_cast<int32_t>(ids.size()), ids.data());
    if (s != KV_OK) return s;
    std::memcpy(block_ids, ids.data(), ids.size() * sizeof(int32_t));
  }
  *num_blocks = static_cast<int32_t>(ids.size());
  *matched_tokens = matched;
  pc->lookups++;
  pc->hits += matched > 0;
  pc->hit_tokens += matched;
  return ok();
}

kv_status kv_prefix_insert(kv_prefix_cache *pc, const int32_t *tokens, int32_t n,
                           const int32_t *block_ids, int32_t num_blocks,
                           int32_t *newly_cached) {
  if (!pc) return fail(KV_ERR_INVALID, "null cache");
  if (n < 0 || (n > 0 && !tokens)) return fail(KV_ERR_INVALID, "bad token array");
  const int bs = pc->bs;
  const int32_t nfull = n / bs;
  if (num_blocks < nfull || (nfull > 0 && !block_ids))
    return fail(KV_ERR_INVALID, "need one block id per full block (%d)", nfull);
  for (int32_t i = 0; i < nfull; ++i)
    if (ref_of(pc->pool, block_ids[i]) < 1)
      return fail(KV_ERR_INVALID, "block %d is not allocated", block_ids[i]);
  std::lock_guard<std::mutex> g(pc->mu);
  const uint64_t now = ++pc->clock;
  int32_t added = 0;
  Node *node = &pc->root;
  int32_t i = 0;  // next block of the prompt
  while (i < nfull) {
    const int32_t *t = tokens + static_cast<int64_t>(i) * bs;
    auto it = node->kids.find(block_key(t, bs));
    if (it == node->kids.end()) {
      // new branch with the remaining full blocks
      auto c = std::make_unique<Node>();
      c->tokens.assign(t, tokens + static_cast<int64_t>(nfull) * bs);
      c->blocks.assign(block_ids + i, block_ids + nfull);
      c->tick.assign(nfull - i, now);
      c->parent = node;
      kv_status s = kv_share_blocks(pc->pool, nfull - i, block_ids + i);
      if (s != KV_OK) return s;
      added += nfull - i;
      pc->cached += nfull - i;
      pc->nodes++;
      node->kids.emplace(block_key(t, bs), std::move(c));
      break;
    }
    Node *c = it->second.get();
    size_t e = 0;
    while (e < c->blocks.size() && i < nfull &&
           std::memcmp(c->tokens.data() + e * bs, tokens + static_cast<int64_t>(i) * bs,
                       bs * sizeof(int32_t)) == 0) {
      c->tick[e] = now;
      ++e;
      ++i;
    }
    if (e < c->blocks.size() && i < nfull) split(pc, c, e);  // diverges inside the edge
    node = c;
  }
  if (newly_cached) *newly_cached = added;
  return ok();
}

kv_status kv_prefix_evict(kv_prefix_cache *pc, int32_t want, int32_t *freed_ids,
                          int32_t *num_freed) {
  if (!pc || !num_freed) return fail(KV_ERR_INVALID, "null argument");
  if (want < 0 || (want > 0 && !freed_ids)) return fail(KV_ERR_INVALID, "bad output array");
  std::lock_guard<std::mutex> g(pc->mu);
  int32_t k = 0;
  while (k < want) {
    Node *best = nullptr;
    uint64_t bt = 0;
    int32_t bid = -1;
    best_leaf(pc, &pc->root, &best, &bt, &bid);
    if (!best) break;
    kv_status s = kv_free_blocks(pc->pool, 1, &bid);
    if (s != KV_OK) return s;
    freed_ids[k++] = bid;
    pc->cached--;
    best->blocks.pop_back();
    best->tick.pop_back();
    best->tokens.resize(best->blocks.size() * pc->bs);
    if (best->blocks.empty()) {  // the edge is gone: unlink the node
      Node *par = best->parent;
      for (auto it = par->kids.begin(); it != par->kids.end(); ++it) {
        if (it->second.get() == best) {
          par->kids.erase(it);
          break;
        }
      }
      pc->nodes--;
    }
  }
  *num_freed = k;
  return ok();
}

kv_status kv_prefix_stats(kv_prefix_cache *pc, kv_prefix_cache_stats *out) {
  if (!pc || !out) return fail(KV_ERR_INVALID, "null argument");
  std::lock_guard<std::mutex> g(pc->mu);
  out->nodes = pc->nodes;
  out->cached_blocks = pc->cached;
  out->lookups = pc->lookups;
  out->hits = pc->hits;
  out->hit_tokens = pc->hit_tokens;
  return ok();
}

}  // extern "C"
