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

  bool active(int32_t seq) const { return seq >= 0 && seq < max_seqs_ && seqs_[seq].active; }
  int32_t len(int32_t seq) const { return seqs_[seq].len; }
  const std::vector<int32_t>& table(int32_t seq) const { return seqs_[seq].table; }
  int32_t refcount(int32_t block) const { return ref_[block]; }
  int32_t free_count() const { return free_count_; }
  void free_list(std::vector<int32_t>* out) const;

  void set_fail_after(int64_t n) { fail_after_ = n; }
  MirrorDeltas& deltas() { return deltas_; }

  int32_t num_blocks() const { return num_blocks_; }
  int32_t block_size() const { return block_size_; }
  int32_t max_seqs() const { return max_seqs_; }
  int32_t max_blocks_per_seq() const { return mbps_; }

 private:
  struct Seq {
    bool active = false;
    int32_t len = 0;
    std::vector<int32_t> table;
  };
  int32_t pop_free();
  void push_free(int32_t b);
  void record_entry(int32_t seq, int32_t j, int32_t block);
  void record_len(int32_t seq, int32_t len);

  int32_t num_blocks_, block_size_, max_seqs_, mbps_;
  std::vector<int32_t> ring_;  // free list as a ring buffer of capacity num_blocks
  int32_t head_ = 0, free_count_ = 0;
  std::vector<int32_t> ref_;
  std::vector<Seq> seqs_;
  int64_t fail_after_ = -1;  // remaining allocations before injected failure
  MirrorDeltas deltas_;
};

}  // namespace pa
