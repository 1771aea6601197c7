// Random-operation fuzz of the host block manager, built with the address and
// undefined-behaviour sanitizers by tests/test_host_sanitized.py.  After every
// operation it checks the pool invariants from the block manager's own
// accessors: each block is free, cached or referenced, and exactly one of
// these; reference counts equal the table entries that name a block; cached
// blocks are registered and unreferenced; a match never exceeds the prompt's
// whole blocks and its blocks equal those the new sequence receives.  Before
// that, the prefix index's open-addressing table runs against a std::multimap
// with keys crowded onto three home slots.  Every 250 operations the state
// image is saved and loaded into a fresh manager, which must show the same
// state, and corrupted copies of the image (random words, truncations) must
// either load into a consistent state or be refused with nothing changed.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <random>
#include <vector>

#include "block_manager.h"

namespace {

int fails = 0;
// Records a failed check; the loops stop at the first one.
#define CHECK(c)                                                            \
  do {                                                                      \
    if (!(c) && fails++ == 0)                                               \
      std::fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
  } while (0)

void check(const pa::BlockManager& bm) {
  const int nb = bm.num_blocks();
  std::vector<int> refs(nb, 0), seen(nb, 0);
  for (int s = 0; s < bm.max_seqs(); ++s) {
    if (!bm.active(s)) continue;
    const auto& t = bm.table(s);
    CHECK(static_cast<int64_t>(t.size()) ==
          (static_cast<int64_t>(bm.len(s)) + bm.block_size() - 1) / bm.block_size());
    for (int b : t) {
      CHECK(b >= 0 && b < nb);
      ++refs[b];
    }
  }
  std::vector<int32_t> fl, cl;
  bm.free_list(&fl);
  bm.cached_list(&cl);
  CHECK(static_cast<int>(cl.size()) == bm.cached_count());
  for (int b : fl) {
    CHECK(b >= 0 && b < nb && !bm.registered(b));
    ++seen[b];
  }
  for (int b : cl) {
    CHECK(b >= 0 && b < nb && bm.registered(b));
    ++seen[b];
  }
  for (int b = 0; b < nb; ++b) {
    CHECK(refs[b] == bm.refcount(b));
    CHECK(seen[b] == (refs[b] == 0 ? 1 : 0));
  }
}

bool same_state(const pa::BlockManager& a, const pa::BlockManager& b) {
  if (a.num_blocks() != b.num_blocks() || a.max_seqs() != b.max_seqs()) return false;
  for (int s = 0; s < a.max_seqs(); ++s) {
    if (a.active(s) != b.active(s)) return false;
    if (a.active(s) && (a.len(s) != b.len(s) || a.table(s) != b.table(s))) return false;
  }
  for (int k = 0; k < a.num_blocks(); ++k)
    if (a.refcount(k) != b.refcount(k) || a.registered(k) != b.registered(k)) return false;
  std::vector<int32_t> fa, fb, ca, cb;
  a.free_list(&fa);
  b.free_list(&fb);
  a.cached_list(&ca);
  b.cached_list(&cb);
  return fa == fb && ca == cb;
}

// The state image: restored into a fresh manager it gives the same state;
// corrupted, it loads into a consistent state or changes nothing.
void fuzz_state(const pa::BlockManager& bm, const std::vector<int32_t>& order, std::mt19937& g) {
  std::vector<int32_t> img;
  bm.save_state(&img);
  pa::BlockManager r(bm.num_blocks(), bm.block_size(), bm.max_seqs(), bm.max_blocks_per_seq(), order.data());
  CHECK(r.load_state(img.data(), img.size()) == pa::kOk);
  CHECK(same_state(r, bm));
  check(r);
  for (int t = 0; t < 40 && fails == 0; ++t) {
    std::vector<int32_t> bad = img;
    const int flips = 1 + static_cast<int>(g() % 3);
    for (int f = 0; f < flips; ++f) {
      const size_t at = g() % bad.size();
      switch (g() % 4) {
        case 0: bad[at] = static_cast<int32_t>(g()); break;
        case 1: bad[at] += 1; break;
        case 2: bad[at] = -1; break;
        default: bad.resize(at); break;
      }
      if (bad.empty()) break;
    }
    pa::BlockManager before = r;
    if (r.load_state(bad.data(), bad.size()) == pa::kOk) {
      check(r);
    } else {
      CHECK(same_state(r, before));
    }
  }
}

// The prefix index against a std::multimap, with keys forced onto few home
// slots (shared low bits) so that probe runs are long, wrap around the table
// end and are cut by backward-shift deletions.
void fuzz_node_index(int seed) {
  std::mt19937_64 g(seed);
  pa::NodeIndex ix;
  std::multimap<uint64_t, int32_t> ref;
  int32_t next = 0;
  for (int it = 0; it < 4000 && fails == 0; ++it) {
    const uint64_t key = ((g() % 40) << 20) | (g() % 3) * 61 | 0x3f;  // low bits: 3 homes
    if (g() % 3 != 0 || ref.empty()) {
      ix.insert(key, next);
      ref.emplace(key, next);
      ++next;
    } else {
      auto it_ref = ref.begin();
      std::advance(it_ref, static_cast<long>(g() % ref.size()));
      ix.erase(it_ref->first, it_ref->second);
      ref.erase(it_ref);
    }
    // every stored (key, node) is found; a node not stored is not
    const uint64_t probe = ((g() % 40) << 20) | (g() % 3) * 61 | 0x3f;
    auto range = ref.equal_range(probe);
    for (auto r = range.first; r != range.second; ++r) {
      const int32_t want = r->second;
      CHECK(ix.find(probe, [&](int32_t n) { return n == want; }) == want);
    }
    CHECK(ix.find(probe, [&](int32_t n) { return n == next; }) == -1);
  }
}

}  // namespace

int main(int argc, char** argv) {
  const int seeds = argc > 1 ? std::atoi(argv[1]) : 20;
  for (int seed = 0; seed < 4 && fails == 0; ++seed) fuzz_node_index(seed);
  for (int seed = 0; seed < seeds && fails == 0; ++seed) {
    std::mt19937 g(seed);
    const int B = (seed % 2) ? 32 : 16, nb = 24 + seed * 7, max_seqs = 12, mbps = 24;
    std::vector<int32_t> order(nb);
    for (int i = 0; i < nb; ++i) order[i] = i;
    std::shuffle(order.begin(), order.end(), g);
    pa::BlockManager bm(nb, B, max_seqs, mbps, order.data());
    const int vocab = 1 + seed % 4;
    std::vector<std::vector<int32_t>> hist(max_seqs), done;
    std::vector<pa::CowPair> cows;
    for (int it = 0; it < 3000 && fails == 0; ++it) {
      const int s = static_cast<int>(g() % max_seqs);
      const int op = static_cast<int>(g() % 100);
      if (op < 25 && !bm.active(s)) {  // new prompt, maybe a continuation
        std::vector<int32_t> toks = (!done.empty() && g() % 2) ? done[g() % done.size()]
                                                               : std::vector<int32_t>();
        const int extra = static_cast<int>(g() % (3 * B));
        for (int k = 0; k < extra; ++k) toks.push_back(static_cast<int32_t>(g() % vocab));
        if (static_cast<int>(toks.size()) > mbps * B) toks.resize(mbps * B);
        std::vector<int32_t> hit;
        const int m = bm.match_prefix(static_cast<int32_t>(toks.size()), toks.data(), &hit);
        CHECK(m * B <= static_cast<int>(toks.size()));
        int32_t cached = -1;
        if (bm.reserve_prefix(s, static_cast<int32_t>(toks.size()), toks.data(), &cached) == pa::kOk) {
          CHECK(cached == m * B);
          for (int j = 0; j < m; ++j) CHECK(bm.table(s)[j] == hit[j]);
          hist[s] = toks;
          CHECK(bm.register_prefix(s, static_cast<int32_t>(toks.size()), toks.data()) == pa::kOk);
        }
      } else if (op < 35 && bm.active(s)) {  // fork
        const int c = static_cast<int>(g() % max_seqs);
        if (!bm.active(c) && bm.fork(s, c) == pa::kOk) hist[c] = hist[s];
      } else if (op < 75 && bm.active(s)) {  // grow
        const int grow = 1 + static_cast<int>(g() % (2 * B));
        const int n = bm.len(s) + grow;
        cows.clear();
        if (n <= mbps * B && bm.reserve(s, n, &cows) == pa::kOk) {
          for (int k = 0; k < grow; ++k) hist[s].push_back(static_cast<int32_t>(g() % vocab));
          if (g() % 3 == 0)
            CHECK(bm.register_prefix(s, static_cast<int32_t>(hist[s].size()), hist[s].data()) == pa::kOk);
        }
      } else if (op < 90 && bm.active(s)) {  // finish
        CHECK(bm.release(s) == pa::kOk);
        done.push_back(hist[s]);
        if (done.size() > 16) done.erase(done.begin());
      } else if (bm.active(s) && bm.len(s) > 0) {  // a write must avoid shared and cached blocks
        int64_t slot = 0;
        const int pos = static_cast<int>(g() % bm.len(s));
        const int b = bm.table(s)[pos / B];
        const pa::Status st = bm.slot(s, pos, &slot);
        CHECK((st == pa::kSharedBlock) == (bm.refcount(b) > 1 || bm.registered(b)));
      }
      check(bm);
      if (it % 250 == 249) fuzz_state(bm, order, g);
    }
  }
  if (fails) return 1;
  std::printf("ok\n");
  return 0;
}
