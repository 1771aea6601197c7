// Host-side block manager of the paged KV pool.
//
// Keeps the free list, the reference count of every physical block and one
// block table per sequence.  Blocks are handed out only when a sequence
// crosses a block boundary, return to the free list once nothing references
// them, and a shared, partly filled tail block is copied before a sequence
// grows into it ("KV cache", paging paragraph; "Managing the KV Cache",
// Block Tables and Sharing and Answer Key item 2; kv-cache-pagedattention-
// serving, The bonus: sharing via copy-on-write).
//
// Policies where the pages leave a choice: the free list is FIFO (allocate
// from the head, release to the tail in logical-block order); a reservation
// that needs a copy-on-write block and new blocks takes the copy-on-write
// block first; the need is checked before any change.
//
// Block-granular prefix cache (kv-cache-pagedattention-serving, Beyond
// paging: radix trees and continuous batching; "Managing the KV Cache",
// Block Tables and Sharing): a full block whose KV is written may be
// registered under the token prefix it ends (every token from the sequence
// start to its last slot).  A new prompt reuses, from its first block on,
// each block whose whole prefix is registered, and stops at the first miss.
// The index is a trie with one node per distinct whole-block prefix, found by
// (parent node, the block's own tokens) and compared exactly, so no hash
// collision can hand out a wrong block.  Registered blocks that nothing
// references stay on a least-recently-used list with their contents and are
// evicted only when a block is needed and the free list is empty.  Where the
// pages are silent: a registered block is immutable (a write into it is
// refused like a write into a shared block); the first registration of a
// prefix wins; a release adds its registered blocks to the recently-used end
// in reverse logical order, so a longer prefix is evicted before the shorter
// one it extends.
//
// Every change that the device must see (a block-table entry, a sequence
// length) is recorded in a MirrorDeltas list, which the API layer ships to
// the device copy of the tables with the next kernel launch.
#pragma once

#include <cstdint>
#include <vector>

namespace pa {

enum Status : int32_t {
  kOk = 0,
  kInvalidArg = -1,
  kNoBlocks = -2,
  kNoSeq = -3,
  kSeqExists = -4,
  kSharedBlock = -5,
  kCuda = -6,
  kDeviceCheck = -7,
};

// Pending updates of the device mirror, keyed by flat int32 index into
// [tables: max_seqs * max_blocks_per_seq][lens: max_seqs].  A second write to
// an index overwrites the pending value, so each index appears at most once.
class MirrorDeltas {
 public:
  void reset(int64_t space);
  void set(int64_t index, int32_t value);
  size_t size() const { return idx_.size(); }
  const std::vector<int32_t>& indices() const { return idx_; }
  const std::vector<int32_t>& values() const { return val_; }
  // Forget the first `n` deltas (they were shipped).
  void consume(size_t n);

 private:
  std::vector<int32_t> where_;  // index -> position in idx_/val_, or -1
  std::vector<int32_t> idx_, val_;
};

struct CowPair {
  int32_t src, dst;
};

// Open-addressing hash table from a 64-bit key to the nodes stored under it
// (linear probing, load <= 1/2, backward-shift deletion), so inserting and
// removing a node allocates nothing once the table has grown.
class NodeIndex {
 public:
  void insert(uint64_t key, int32_t node);
  void erase(uint64_t key, int32_t node);
  // First node stored under `key` for which `same(node)` holds, or -1.
  template <class F>
  int32_t find(uint64_t key, F&& same) const {
    if (slots_.empty()) return -1;
    for (size_t i = key & mask_;; i = (i + 1) & mask_) {
      const Slot& s = slots_[i];
      if (s.node < 0) return -1;
      if (s.key == key && same(s.node)) return s.node;
    }
  }

 private:
  struct Slot {
    uint64_t key;
    int32_t node;  // -1: empty
  };
  void grow();
  std::vector<Slot> slots_;
  size_t mask_ = 0, size_ = 0;
};

class BlockManager {
 public:
  BlockManager(int32_t num_blocks, int32_t block_size, int32_t max_seqs,
               int32_t max_blocks_per_seq, const int32_t* free_order);

  // Grow (or create) `seq` to `new_len` tokens.  Appends any copy-on-write
  // pair to `cows`.  On failure nothing changes.
  Status reserve(int32_t seq, int32_t new_len, std::vector<CowPair>* cows);
  Status fork(int32_t parent, int32_t child);
  Status release(int32_t seq);
  // Flat slot id (block * block_size + offset) of token `pos` of `seq`.
  Status slot(int32_t seq, int32_t pos, int64_t* slot_out) const;

  // Prefix cache.  `tokens` holds the first `n` tokens of the sequence.
  // register_prefix: registers the full blocks of `seq` covering tokens[0, n),
  // n <= length; fails (nothing registered) if one of them is already
  // registered under another prefix.
  Status register_prefix(int32_t seq, int32_t n, const int32_t* tokens);
  // Leading full blocks of tokens[0, n) whose prefix is registered; their
  // block ids go to `blocks` if given.
  int32_t match_prefix(int32_t n, const int32_t* tokens, std::vector<int32_t>* blocks) const;
  // Create `seq` for the prompt tokens[0, n), reusing its cached leading
  // blocks; *n_cached = the prompt tokens whose KV those blocks hold.
  Status reserve_prefix(int32_t seq, int32_t n, const int32_t* tokens, int32_t* n_cached);
  int32_t cached_count() const { return lru_count_; }
  // Registered blocks with no reference, least recently used first.
  void cached_list(std::vector<int32_t>* out) const;
  bool registered(int32_t block) const { return block_node_[block] >= 0; }

  bool active(int32_t seq) const { return seq >= 0 && seq < max_seqs_ && seqs_[seq].active; }
  int32_t len(int32_t seq) const { return seqs_[seq].len; }
  const std::vector<int32_t>& table(int32_t seq) const { return seqs_[seq].table; }
  int32_t refcount(int32_t block) const { return ref_[block]; }
  int32_t free_count() const { return free_count_; }
  void free_list(std::vector<int32_t>* out) const;

  // The whole host state as int32 words (layout in block_manager.cpp), and
  // its restore into a manager of the same geometry.  load_state validates
  // the image completely first (ranges, and that every block is exactly one
  // of free, referenced by the tables it sits in, or idle and cached) and
  // changes nothing when it fails.  After a load the manager behaves exactly
  // as the saved one did from the save on, and every table entry and length
  // is queued for the device mirror.
  void save_state(std::vector<int32_t>* out) const;
  Status load_state(const int32_t* words, size_t n);

  void set_fail_after(int64_t n) { fail_after_ = n; }
  MirrorDeltas& deltas() { return deltas_; }

  // Incremented by every change of a block table or a length: equal versions
  // mean identical tables (a decode plan built from them is still valid).
  uint64_t version() const { return version_; }
  int32_t num_blocks() const { return num_blocks_; }
  int32_t block_size() const { return block_size_; }
  int32_t max_seqs() const { return max_seqs_; }
  int32_t max_blocks_per_seq() const { return mbps_; }

 private:
  uint64_t version_ = 0;
  struct Seq {
    bool active = false;
    int32_t len = 0;
    std::vector<int32_t> table;
  };
  // One distinct whole-block token prefix: its last block's tokens live at
  // node_tokens_[id * block_size].
  struct Node {
    int32_t parent;    // node of the prefix one block shorter, -1 at depth 1
    int32_t block;     // registered block holding this prefix's last block, or -1
    int32_t children;  // nodes whose parent is this one
    uint64_t key;      // hash of (parent, tokens), the index key
  };
  int32_t pop_free();
  void push_free(int32_t b);
  int32_t take_block();  // free head, else evict the least recently used cached block
  uint64_t node_key(int32_t parent, const int32_t* toks) const;
  int32_t find_child(int32_t parent, const int32_t* toks) const;
  int32_t add_child(int32_t parent, const int32_t* toks);
  void prune(int32_t node);
  void unregister(int32_t block);
  void lru_push_back(int32_t b);
  void lru_remove(int32_t b);
  void record_entry(int32_t seq, int32_t j, int32_t block);
  void record_len(int32_t seq, int32_t len);

  int32_t num_blocks_, block_size_, max_seqs_, mbps_;
  std::vector<int32_t> ring_;  // free list as a ring buffer of capacity num_blocks
  int32_t head_ = 0, free_count_ = 0;
  std::vector<int32_t> ref_;
  std::vector<Seq> seqs_;
  int64_t fail_after_ = -1;  // remaining allocations before injected failure
  MirrorDeltas deltas_;

  std::vector<Node> nodes_;
  std::vector<int32_t> node_tokens_, spare_nodes_;
  NodeIndex index_;                                   // key -> node
  std::vector<int32_t> block_node_;                   // block -> node, or -1
  std::vector<int32_t> lru_prev_, lru_next_;          // -2: not on the list
  int32_t lru_head_ = -1, lru_tail_ = -1, lru_count_ = 0;
};

}  // namespace pa
