// Host-side block manager; see block_manager.h for the policies.
#include "block_manager.h"

#include <algorithm>

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

BlockManager::BlockManager(int32_t num_blocks, int32_t block_size, int32_t max_seqs,
                           int32_t max_blocks_per_seq, const int32_t* free_order)
    : num_blocks_(num_blocks), block_size_(block_size), max_seqs_(max_seqs),
      mbps_(max_blocks_per_seq), ring_(num_blocks), ref_(num_blocks, 0), seqs_(max_seqs) {
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

void BlockManager::record_entry(int32_t seq, int32_t j, int32_t block) {
  deltas_.set(static_cast<int64_t>(seq) * mbps_ + j, block);
}

void BlockManager::record_len(int32_t seq, int32_t len) {
  deltas_.set(static_cast<int64_t>(max_seqs_) * mbps_ + seq, len);
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
  if (need > free_count_) return kNoBlocks;
  if (fail_after_ >= 0 && need > fail_after_) return kNoBlocks;

  if (!s.active) {
    s.active = true;
    s.len = 0;
    s.table.clear();
    s.table.reserve(static_cast<size_t>(std::min<int64_t>(mbps_, want_blocks + 64)));
  }
  if (cow) {
    const int32_t src = s.table.back();
    const int32_t dst = pop_free();
    --ref_[src];
    ref_[dst] = 1;
    s.table.back() = dst;
    record_entry(seq, have - 1, dst);
    cows->push_back({src, dst});
  }
  for (int64_t k = 0; k < grow; ++k) {
    const int32_t b = pop_free();
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
    if (--ref_[b] == 0) push_free(b);
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
  if (ref_[b] > 1) return kSharedBlock;
  *slot_out = static_cast<int64_t>(b) * block_size_ + pos % block_size_;
  return kOk;
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
