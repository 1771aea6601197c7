// Host-side block manager; see block_manager.h for the policies.
#include "block_manager.h"

#include <algorithm>
#include <cstring>
#include <utility>

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


// ------------------------------------------------------------ state image
// int32 words:
//   magic, num_blocks, block_size, max_seqs, max_blocks_per_seq,
//   free count, the free blocks from the head,
//   ref[num_blocks], block_node[num_blocks],
//   per sequence: active, len, table size, table entries,
//   node count N, per node: parent, block, children, key low, key high;
//   then N * block_size tokens,
//   spare-node count, the spare nodes (last one reused first),
//   cached count, the idle cached blocks least recently used first.
constexpr int32_t kStateMagic = 0x50414231;

void BlockManager::save_state(std::vector<int32_t>* out) const {
  std::vector<int32_t>& o = *out;
  o.clear();
  o.insert(o.end(), {kStateMagic, num_blocks_, block_size_, max_seqs_, mbps_});
  std::vector<int32_t> fl;
  free_list(&fl);
  o.push_back(free_count_);
  o.insert(o.end(), fl.begin(), fl.end());
  o.insert(o.end(), ref_.begin(), ref_.end());
  o.insert(o.end(), block_node_.begin(), block_node_.end());
  for (const Seq& q : seqs_) {
    o.push_back(q.active ? 1 : 0);
    o.push_back(q.len);
    o.push_back(static_cast<int32_t>(q.table.size()));
    o.insert(o.end(), q.table.begin(), q.table.end());
  }
  o.push_back(static_cast<int32_t>(nodes_.size()));
  for (const Node& nd : nodes_) {
    o.insert(o.end(), {nd.parent, nd.block, nd.children, static_cast<int32_t>(nd.key & 0xffffffffu),
                       static_cast<int32_t>(nd.key >> 32)});
  }
  o.insert(o.end(), node_tokens_.begin(), node_tokens_.end());
  o.push_back(static_cast<int32_t>(spare_nodes_.size()));
  o.insert(o.end(), spare_nodes_.begin(), spare_nodes_.end());
  std::vector<int32_t> cached;
  cached_list(&cached);
  o.push_back(static_cast<int32_t>(cached.size()));
  o.insert(o.end(), cached.begin(), cached.end());
}

Status BlockManager::load_state(const int32_t* w, size_t n) {
  size_t at = 0;
  auto take = [&](int32_t* v) {
    if (at >= n) return false;
    *v = w[at++];
    return true;
  };
  auto in = [](int32_t v, int32_t lo, int32_t hi) { return v >= lo && v < hi; };
  int32_t head[5];
  for (int32_t& h : head)
    if (!take(&h)) return kInvalidArg;
  if (head[0] != kStateMagic || head[1] != num_blocks_ || head[2] != block_size_ || head[3] != max_seqs_ ||
      head[4] != mbps_)
    return kInvalidArg;
  const int32_t NB = num_blocks_;
  int32_t fc = 0;
  if (!take(&fc) || !in(fc, 0, NB + 1)) return kInvalidArg;
  std::vector<int32_t> fl(fc), ref(NB), bnode(NB);
  std::vector<char> seen(NB, 0);
  for (int32_t& b : fl)
    if (!take(&b) || !in(b, 0, NB) || seen[b]++) return kInvalidArg;
  for (int32_t& r : ref)
    if (!take(&r) || r < 0) return kInvalidArg;
  for (int32_t& x : bnode)
    if (!take(&x)) return kInvalidArg;
  std::vector<Seq> seqs(max_seqs_);
  std::vector<int32_t> counted(NB, 0);
  for (Seq& q : seqs) {
    int32_t act = 0, len = 0, nt = 0;
    if (!take(&act) || !take(&len) || !take(&nt) || !in(act, 0, 2) || !in(nt, 0, mbps_ + 1)) return kInvalidArg;
    if (len < 0 || static_cast<int64_t>(len) > static_cast<int64_t>(mbps_) * block_size_) return kInvalidArg;
    if (nt != (act ? (len + block_size_ - 1) / block_size_ : 0)) return kInvalidArg;
    q.active = act != 0;
    q.len = act ? len : 0;
    q.table.resize(nt);
    for (int32_t& b : q.table) {
      if (!take(&b) || !in(b, 0, NB)) return kInvalidArg;
      ++counted[b];
    }
  }
  int32_t nn = 0;
  if (!take(&nn) || nn < 0 || static_cast<size_t>(nn) * (5 + block_size_) > n) return kInvalidArg;
  std::vector<Node> nodes(nn);
  for (Node& nd : nodes) {
    int32_t lo = 0, hi = 0;
    if (!take(&nd.parent) || !take(&nd.block) || !take(&nd.children) || !take(&lo) || !take(&hi))
      return kInvalidArg;
    if (!in(nd.parent, -1, nn) || !in(nd.block, -1, NB) || nd.children < 0) return kInvalidArg;
    nd.key = static_cast<uint64_t>(static_cast<uint32_t>(lo)) | (static_cast<uint64_t>(static_cast<uint32_t>(hi)) << 32);
  }
  std::vector<int32_t> toks(static_cast<size_t>(nn) * block_size_);
  for (int32_t& t : toks)
    if (!take(&t)) return kInvalidArg;
  int32_t ns = 0;
  if (!take(&ns) || !in(ns, 0, nn + 1)) return kInvalidArg;
  std::vector<int32_t> spare(ns);
  std::vector<char> dead(nn, 0);
  for (int32_t& x : spare)
    if (!take(&x) || !in(x, 0, nn) || dead[x]++) return kInvalidArg;
  int32_t nc = 0;
  if (!take(&nc) || !in(nc, 0, NB + 1)) return kInvalidArg;
  std::vector<int32_t> lru(nc);
  std::vector<char> cached(NB, 0);
  for (int32_t& b : lru)
    if (!take(&b) || !in(b, 0, NB) || cached[b]++) return kInvalidArg;
  if (at != n) return kInvalidArg;
  // consistency: every block free, referenced (its count = the tables it is
  // in), or idle, registered and cached; live nodes and blocks name each other
  for (int32_t b = 0; b < NB; ++b) {
    if (ref[b] != counted[b]) return kInvalidArg;
    if (!in(bnode[b], -1, nn) || (bnode[b] >= 0 && (dead[bnode[b]] || nodes[bnode[b]].block != b)))
      return kInvalidArg;
    const int kinds = (seen[b] ? 1 : 0) + (ref[b] > 0 ? 1 : 0) + (cached[b] ? 1 : 0);
    if (kinds != 1 || (cached[b] && bnode[b] < 0) || (seen[b] && bnode[b] >= 0)) return kInvalidArg;
  }
  // the trie: a live node's parent is live, its child count is the live
  // nodes naming it, it holds a block or leads to one, and its key is the
  // hash of (parent, tokens)
  std::vector<int32_t> kids(nn, 0);
  for (int32_t c = 0; c < nn; ++c) {
    if (dead[c]) continue;
    const Node& nd = nodes[c];
    if (nd.block >= 0 && bnode[nd.block] != c) return kInvalidArg;
    if (nd.parent >= 0) {
      if (dead[nd.parent]) return kInvalidArg;
      ++kids[nd.parent];
    }
    if (nd.key != node_key(nd.parent, &toks[static_cast<size_t>(c) * block_size_])) return kInvalidArg;
  }
  for (int32_t c = 0; c < nn; ++c)
    if (!dead[c] && (nodes[c].children != kids[c] || (nodes[c].block < 0 && kids[c] == 0)))
      return kInvalidArg;
  // every parent chain reaches the root (no cycle), and no two live nodes
  // hold the same (parent, tokens)
  std::vector<char> state(nn, 0);  // 0 unvisited, 1 on the current chain, 2 reaches the root
  std::vector<int32_t> chain;
  for (int32_t c = 0; c < nn; ++c) {
    if (dead[c] || state[c] == 2) continue;
    chain.clear();
    int32_t v = c;
    while (v >= 0 && state[v] == 0) {
      state[v] = 1;
      chain.push_back(v);
      v = nodes[v].parent;
    }
    if (v >= 0 && state[v] == 1) return kInvalidArg;
    for (int32_t u : chain) state[u] = 2;
  }
  NodeIndex idx;
  for (int32_t c = 0; c < nn; ++c) {
    if (dead[c]) continue;
    const int32_t* tc = &toks[static_cast<size_t>(c) * block_size_];
    const int32_t twin = idx.find(nodes[c].key, [&](int32_t o) {
      return nodes[o].parent == nodes[c].parent &&
             std::memcmp(&toks[static_cast<size_t>(o) * block_size_], tc, sizeof(int32_t) * block_size_) == 0;
    });
    if (twin >= 0) return kInvalidArg;
    idx.insert(nodes[c].key, c);
  }

  // apply
  std::fill(ring_.begin(), ring_.end(), 0);
  std::copy(fl.begin(), fl.end(), ring_.begin());
  head_ = 0;
  free_count_ = fc;
  ref_.swap(ref);
  block_node_.swap(bnode);
  seqs_.swap(seqs);
  nodes_.swap(nodes);
  node_tokens_.swap(toks);
  spare_nodes_.swap(spare);
  index_ = std::move(idx);
  std::fill(lru_prev_.begin(), lru_prev_.end(), -2);
  std::fill(lru_next_.begin(), lru_next_.end(), -2);
  lru_head_ = lru_tail_ = -1;
  lru_count_ = 0;
  for (int32_t b : lru) lru_push_back(b);
  fail_after_ = -1;
  deltas_.reset(static_cast<int64_t>(max_seqs_) * mbps_ + max_seqs_);
  for (int32_t q = 0; q < max_seqs_; ++q) {
    const Seq& sq = seqs_[q];
    for (size_t j = 0; j < sq.table.size(); ++j)
      deltas_.set(static_cast<int64_t>(q) * mbps_ + static_cast<int64_t>(j), sq.table[j]);
    deltas_.set(static_cast<int64_t>(max_seqs_) * mbps_ + q, sq.len);
  }
  ++version_;
  return kOk;
}

}  // namespace pa
