// Host-side block manager; see block_manager.h for the policies.
#include "block_manager.h"

#include <algorithm>
#include <cstring>

namespace pa {

void MirrorDeltas::reset(int64_t space) {
  where_.assign(static_cast<size_t>(space), -1);
  idx_.clear();
  val_.clear();
}

void MirrorDeltas::set(int64_t index, int32_t value) {
  int32_t& w = where_[static_cast<size_t>(index)];
  if (w >= 0) {
    val_[w] = value;
    return;
  }
  w = static_cast<int32_t>(idx_.size());
  idx_.push_back(static_cast<int32_t>(index));
  val_.push_back(value);
}

void MirrorDeltas::consume(size_t n) {
  n = std::min(n, idx_.size());
  for (size_t k = 0; k < n; ++k) where_[idx_[k]] = -1;
  idx_.erase(idx_.begin(), idx_.begin() + n);
  val_.erase(val_.begin(), val_.begin() + n);
  for (size_t k = 0; k < idx_.size(); ++k) where_[idx_[k]] = static_cast<int32_t>(k);
}

void NodeIndex::grow() {
  std::vector<Slot> old;
  old.swap(slots_);
  slots_.assign(old.empty() ? 64 : 2 * old.size(), Slot{0, -1});
  mask_ = slots_.size() - 1;
  size_ = 0;
  for (const Slot& s : old)
    if (s.node >= 0) insert(s.key, s.node);
}

void NodeIndex::insert(uint64_t key, int32_t node) {
  if (2 * (size_ + 1) > slots_.size()) grow();
  size_t i = key & mask_;
  while (slots_[i].node >= 0) i = (i + 1) & mask_;
  slots_[i] = Slot{key, node};
  ++size_;
}

void NodeIndex::erase(uint64_t key, int32_t node) {
  if (slots_.empty()) return;
  size_t i = key & mask_;
  while (slots_[i].node >= 0 && !(slots_[i].key == key && slots_[i].node == node)) i = (i + 1) & mask_;
  if (slots_[i].node < 0) return;
  // Backward shift: move later entries of the run into the hole whenever
  // their home slot does not lie cyclically in (hole, entry].
  for (size_t j = (i + 1) & mask_; slots_[j].node >= 0; j = (j + 1) & mask_) {
    const size_t home = slots_[j].key & mask_;
    const bool stays = (i <= j) ? (i < home && home <= j) : (i < home || home <= j);
    if (!stays) {
      slots_[i] = slots_[j];
      i = j;
    }
  }
  slots_[i].node = -1;
  --size_;
}

BlockManager::BlockManager(int32_t num_blocks, int32_t block_size, int32_t max_seqs,
                           int32_t max_blocks_per_seq, const int32_t* free_order)
    : num_blocks_(num_blocks), block_size_(block_size), max_seqs_(max_seqs),
      mbps_(max_blocks_per_seq), ring_(num_blocks), ref_(num_blocks, 0), seqs_(max_seqs),
      block_node_(num_blocks, -1), lru_prev_(num_blocks, -2), lru_next_(num_blocks, -2) {
  for (int32_t b = 0; b < num_blocks; ++b) ring_[b] = free_order ? free_order[b] : b;
  free_count_ = num_blocks;
  deltas_.reset(static_cast<int64_t>(max_seqs) * max_blocks_per_seq + max_seqs);
}

int32_t BlockManager::pop_free() {
  int32_t b = ring_[head_];
  head_ = (head_ + 1 == num_blocks_) ? 0 : head_ + 1;
  --free_count_;
  return b;
}

void BlockManager::push_free(int32_t b) {
  int64_t tail = static_cast<int64_t>(head_) + free_count_;
  if (tail >= num_blocks_) tail -= num_blocks_;
  ring_[tail] = b;
  ++free_count_;
}

int32_t BlockManager::take_block() {
  if (free_count_ > 0) return pop_free();
  const int32_t b = lru_head_;
  lru_remove(b);
  unregister(b);
  return b;
}

void BlockManager::lru_push_back(int32_t b) {
  lru_prev_[b] = lru_tail_;
  lru_next_[b] = -1;
  if (lru_tail_ >= 0) lru_next_[lru_tail_] = b; else lru_head_ = b;
  lru_tail_ = b;
  ++lru_count_;
}

void BlockManager::lru_remove(int32_t b) {
  const int32_t p = lru_prev_[b], n = lru_next_[b];
  if (p >= 0) lru_next_[p] = n; else lru_head_ = n;
  if (n >= 0) lru_prev_[n] = p; else lru_tail_ = p;
  lru_prev_[b] = lru_next_[b] = -2;
  --lru_count_;
}

uint64_t BlockManager::node_key(int32_t parent, const int32_t* toks) const {
  // FNV-1a over 32-bit words (the parent id, then the tokens), then the
  // MurmurHash3 64-bit finaliser to spread the bits over the buckets.
  uint64_t h = 0xcbf29ce484222325ull;
  h = (h ^ static_cast<uint32_t>(parent)) * 0x100000001b3ull;
  for (int32_t i = 0; i < block_size_; ++i) h = (h ^ static_cast<uint32_t>(toks[i])) * 0x100000001b3ull;
  h ^= h >> 33;
  h *= 0xff51afd7ed558ccdull;
  h ^= h >> 33;
  h *= 0xc4ceb9fe1a85ec53ull;
  h ^= h >> 33;
  return h;
}

int32_t BlockManager::find_child(int32_t parent, const int32_t* toks) const {
  return index_.find(node_key(parent, toks), [&](int32_t c) {
    return nodes_[c].parent == parent &&
           std::memcmp(&node_tokens_[static_cast<size_t>(c) * block_size_], toks,
                       sizeof(int32_t) * block_size_) == 0;
  });
}

int32_t BlockManager::add_child(int32_t parent, const int32_t* toks) {
  int32_t c;
  if (!spare_nodes_.empty()) {
    c = spare_nodes_.back();
    spare_nodes_.pop_back();
  } else {
    c = static_cast<int32_t>(nodes_.size());
    nodes_.push_back({});
    node_tokens_.resize(nodes_.size() * static_cast<size_t>(block_size_));
  }
  const uint64_t key = node_key(parent, toks);
  nodes_[c] = {parent, -1, 0, key};
  std::memcpy(&node_tokens_[static_cast<size_t>(c) * block_size_], toks,
              sizeof(int32_t) * block_size_);
  index_.insert(key, c);
  if (parent >= 0) ++nodes_[parent].children;
  return c;
}

// Drop nodes that hold no block and lead to none, walking towards the root.
// A node is only dropped once no child names it as parent, so a reused node
// id never matches a stale key.
void BlockManager::prune(int32_t node) {
  while (node >= 0 && nodes_[node].block < 0 && nodes_[node].children == 0) {
    index_.erase(nodes_[node].key, node);
    const int32_t parent = nodes_[node].parent;
    spare_nodes_.push_back(node);
    if (parent >= 0) --nodes_[parent].children;
    node = parent;
  }
}

void BlockManager::unregister(int32_t block) {
  const int32_t node = block_node_[block];
  block_node_[block] = -1;
  nodes_[node].block = -1;
  prune(node);
}

void BlockManager::record_entry(int32_t seq, int32_t j, int32_t block) {
  deltas_.set(static_cast<int64_t>(seq) * mbps_ + j, block);
  ++version_;
}

void BlockManager::record_len(int32_t seq, int32_t len) {
  deltas_.set(static_cast<int64_t>(max_seqs_) * mbps_ + seq, len);
  ++version_;
}

Status BlockManager::reserve(int32_t seq, int32_t new_len, std::vector<CowPair>* cows) {
  if (seq < 0 || seq >= max_seqs_ || new_len < 0) return kInvalidArg;
  Seq& s = seqs_[seq];
  const int32_t cur = s.active ? s.len : 0;
  if (new_len < cur) return kInvalidArg;
  const int64_t want_blocks = (static_cast<int64_t>(new_len) + block_size_ - 1) / block_size_;
  if (want_blocks > mbps_) return kInvalidArg;
  const int32_t have = static_cast<int32_t>(s.active ? s.table.size() : 0);
  // A write will land in the tail block: copy it first if others share it.
  const bool cow = new_len > cur && (cur % block_size_) != 0 && ref_[s.table.back()] > 1;
  const int64_t grow = want_blocks - have;
  const int64_t need = (cow ? 1 : 0) + grow;
  if (need > static_cast<int64_t>(free_count_) + lru_count_) return kNoBlocks;
  if (fail_after_ >= 0 && need > fail_after_) return kNoBlocks;

  if (!s.active) {
    s.active = true;
    s.len = 0;
    s.table.clear();
    s.table.reserve(static_cast<size_t>(std::min<int64_t>(mbps_, want_blocks + 64)));
  }
  if (cow) {
    const int32_t src = s.table.back();
    const int32_t dst = take_block();
    --ref_[src];
    ref_[dst] = 1;
    s.table.back() = dst;
    record_entry(seq, have - 1, dst);
    cows->push_back({src, dst});
  }
  for (int64_t k = 0; k < grow; ++k) {
    const int32_t b = take_block();
    ref_[b] = 1;
    s.table.push_back(b);
    record_entry(seq, static_cast<int32_t>(s.table.size()) - 1, b);
  }
  if (fail_after_ >= 0) fail_after_ -= need;
  if (s.len != new_len || cur == 0) record_len(seq, new_len);
  s.len = new_len;
  return kOk;
}

Status BlockManager::fork(int32_t parent, int32_t child) {
  if (parent < 0 || parent >= max_seqs_ || child < 0 || child >= max_seqs_) return kInvalidArg;
  if (!seqs_[parent].active) return kNoSeq;
  if (seqs_[child].active) return kSeqExists;
  Seq& c = seqs_[child];
  const Seq& p = seqs_[parent];
  c.active = true;
  c.len = p.len;
  c.table = p.table;
  for (size_t j = 0; j < c.table.size(); ++j) {
    ++ref_[c.table[j]];
    record_entry(child, static_cast<int32_t>(j), c.table[j]);
  }
  record_len(child, c.len);
  return kOk;
}

Status BlockManager::release(int32_t seq) {
  if (seq < 0 || seq >= max_seqs_) return kInvalidArg;
  Seq& s = seqs_[seq];
  if (!s.active) return kNoSeq;
  for (int32_t b : s.table) {
    if (--ref_[b] == 0 && block_node_[b] < 0) push_free(b);
  }
  for (auto it = s.table.rbegin(); it != s.table.rend(); ++it) {
    if (ref_[*it] == 0 && block_node_[*it] >= 0) lru_push_back(*it);
  }
  s.active = false;
  s.len = 0;
  s.table.clear();
  record_len(seq, 0);
  return kOk;
}

Status BlockManager::slot(int32_t seq, int32_t pos, int64_t* slot_out) const {
  if (seq < 0 || seq >= max_seqs_) return kInvalidArg;
  const Seq& s = seqs_[seq];
  if (!s.active) return kNoSeq;
  if (pos < 0 || pos >= s.len) return kInvalidArg;
  const int32_t b = s.table[pos / block_size_];
  if (ref_[b] > 1 || block_node_[b] >= 0) return kSharedBlock;
  *slot_out = static_cast<int64_t>(b) * block_size_ + pos % block_size_;
  return kOk;
}

Status BlockManager::register_prefix(int32_t seq, int32_t n, const int32_t* tokens) {
  if (seq < 0 || seq >= max_seqs_ || n < 0 || (n > 0 && tokens == nullptr)) return kInvalidArg;
  Seq& s = seqs_[seq];
  if (!s.active) return kNoSeq;
  if (n > s.len) return kInvalidArg;
  const int32_t m = n / block_size_;
  const size_t row = sizeof(int32_t) * block_size_;
  // Validate: a block registered already must hold this very prefix.  Its node
  // is known, so that is a parent and token comparison (nodes are unique per
  // (parent, tokens)); only unregistered blocks need the index.
  int32_t node = -1;  // node of the prefix before block i (-1: the empty prefix)
  bool path = true;   // that node exists
  for (int32_t i = 0; i < m; ++i) {
    const int32_t* toks = tokens + static_cast<int64_t>(i) * block_size_;
    const int32_t bn = block_node_[s.table[i]];
    if (bn >= 0) {
      if (!path || nodes_[bn].parent != node ||
          std::memcmp(&node_tokens_[static_cast<size_t>(bn) * block_size_], toks, row) != 0)
        return kInvalidArg;
      node = bn;
    } else {
      node = path ? find_child(node, toks) : -1;
      path = node >= 0;
    }
  }
  node = -1;
  for (int32_t i = 0; i < m; ++i) {
    const int32_t b = s.table[i];
    if (block_node_[b] >= 0) {  // validated above: the node of this prefix
      node = block_node_[b];
      continue;
    }
    const int32_t* toks = tokens + static_cast<int64_t>(i) * block_size_;
    int32_t c = find_child(node, toks);
    if (c < 0) c = add_child(node, toks);
    if (nodes_[c].block < 0) {
      nodes_[c].block = b;
      block_node_[b] = c;
    }
    node = c;
  }
  return kOk;
}

int32_t BlockManager::match_prefix(int32_t n, const int32_t* tokens,
                                   std::vector<int32_t>* blocks) const {
  if (blocks) blocks->clear();
  int32_t node = -1, m = 0;
  for (; (static_cast<int64_t>(m) + 1) * block_size_ <= n; ++m) {
    const int32_t c = find_child(node, tokens + static_cast<int64_t>(m) * block_size_);
    if (c < 0 || nodes_[c].block < 0) break;
    if (blocks) blocks->push_back(nodes_[c].block);
    node = c;
  }
  return m;
}

Status BlockManager::reserve_prefix(int32_t seq, int32_t n, const int32_t* tokens,
                                    int32_t* n_cached) {
  if (seq < 0 || seq >= max_seqs_ || n < 0 || (n > 0 && tokens == nullptr)) return kInvalidArg;
  const int64_t want_blocks = (static_cast<int64_t>(n) + block_size_ - 1) / block_size_;
  if (want_blocks > mbps_) return kInvalidArg;
  Seq& s = seqs_[seq];
  if (s.active) return kSeqExists;
  std::vector<int32_t> hit;
  const int32_t m = match_prefix(n, tokens, &hit);
  int64_t idle = 0;
  for (int32_t b : hit) idle += ref_[b] == 0 ? 1 : 0;
  const int64_t need = want_blocks - m;
  if (need > static_cast<int64_t>(free_count_) + lru_count_ - idle) return kNoBlocks;
  if (fail_after_ >= 0 && need > fail_after_) return kNoBlocks;

  s.active = true;
  s.table.clear();
  s.table.reserve(static_cast<size_t>(std::min<int64_t>(mbps_, want_blocks + 64)));
  for (int32_t b : hit) {
    if (ref_[b] == 0) lru_remove(b);
    ++ref_[b];
    s.table.push_back(b);
    record_entry(seq, static_cast<int32_t>(s.table.size()) - 1, b);
  }
  for (int64_t k = 0; k < need; ++k) {
    const int32_t b = take_block();
    ref_[b] = 1;
    s.table.push_back(b);
    record_entry(seq, static_cast<int32_t>(s.table.size()) - 1, b);
  }
  if (fail_after_ >= 0) fail_after_ -= need;
  s.len = n;
  record_len(seq, n);
  *n_cached = m * block_size_;
  return kOk;
}

void BlockManager::cached_list(std::vector<int32_t>* out) const {
  out->clear();
  out->reserve(lru_count_);
  for (int32_t b = lru_head_; b >= 0; b = lru_next_[b]) out->push_back(b);
}

void BlockManager::free_list(std::vector<int32_t>* out) const {
  out->resize(free_count_);
  int32_t at = head_;
  for (int32_t k = 0; k < free_count_; ++k) {
    (*out)[k] = ring_[at];
    at = (at + 1 == num_blocks_) ? 0 : at + 1;
  }
}

}  // namespace pa
