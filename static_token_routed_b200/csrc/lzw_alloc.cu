// LZW-based embedding allocation (host code; kimjy99 review, 1. Embedding
// Allocation; papernotes note, LZW 分配). It decides d_t, the number of rows
// of W_K / W_V each token ID owns, once, before training or serving.
//
//   1. Scan a token corpus and grow a set of codewords (token tuples) with a
//      frequency each: at every position, the longest suffix of the text
//      ending there that is already a codeword, extended one token further
//      back, is a suffix not seen before. It becomes a codeword with
//      frequency 1; the suffix it extends gains 1.
//   2. Walk the codewords from most to least frequent (equal frequencies in
//      creation order); each gives the token it ends with one row.
//   3. Repeat the walk until the rows add up to v; every token holds at
//      least one row (given up front) and at most k.
//
// The codewords form a suffix-closed set, kept as a trie read backwards
// from a codeword's last token: node = codeword, edge = the token one
// position further back. The scan at position i walks the trie from the
// root along x_i, x_{i-1}, ... and hangs the new codeword under the deepest
// node reached. Children are found in one open-addressing hash table keyed
// by (parent node, token).
#include <algorithm>
#include <cstdint>
#include <new>
#include <string>
#include <vector>

#include "l3_internal.cuh"

namespace l3 {
namespace {

struct ChildTable {
  std::vector<uint64_t> keys;  // (parent + 1) << 32 | token; 0 = empty
  std::vector<int32_t> vals;
  uint64_t mask = 0;

  explicit ChildTable(size_t max_entries) {
    size_t cap = 16;
    while (cap < 2 * max_entries + 16) cap <<= 1;
    keys.assign(cap, 0);
    vals.assign(cap, -1);
    mask = cap - 1;
  }
  static uint64_t key(int32_t parent, int32_t token) {
    return ((uint64_t)(uint32_t)(parent + 1) << 32) | (uint32_t)token;
  }
  static uint64_t hash(uint64_t k) {  // splitmix64 finaliser
    k ^= k >> 30;
    k *= 0xbf58476d1ce4e5b9ull;
    k ^= k >> 27;
    k *= 0x94d049bb133111ebull;
    return k ^ (k >> 31);
  }
  int32_t find(int32_t parent, int32_t token) const {
    const uint64_t k = key(parent, token);
    for (uint64_t h = hash(k) & mask;; h = (h + 1) & mask) {
      if (keys[h] == k) return vals[h];
      if (keys[h] == 0) return -1;
    }
  }
  void insert(int32_t parent, int32_t token, int32_t child) {
    const uint64_t k = key(parent, token);
    uint64_t h = hash(k) & mask;
    while (keys[h] != 0) h = (h + 1) & mask;
    keys[h] = k;
    vals[h] = child;
  }
};

}  // namespace
}  // namespace l3

using namespace l3;

extern "C" l3_status l3_lzw_allocate(const int32_t *corpus, int64_t n, int64_t vocab, int64_t v,
                                     int64_t k, int32_t *d_out, int64_t *n_codewords) {
  set_error("");
  if ((n > 0 && !corpus) || !d_out || n < 0 || vocab < 1 || k < 1 || n > INT32_MAX - 2) {
    set_error("l3_lzw_allocate: NULL pointer or size out of range");
    return L3_ERR_INVALID_ARG;
  }
  if (v < vocab || v > vocab * k) {
    set_error("l3_lzw_allocate: need vocab <= v <= vocab * k");
    return L3_ERR_INVALID_ARG;
  }
  for (int64_t i = 0; i < n; ++i)
    if (corpus[i] < 0 || corpus[i] >= vocab) {
      set_error("l3_lzw_allocate: a corpus token is outside [0, vocab)");
      return L3_ERR_INVALID_ARG;
    }
  try {
    // nodes: 0 is the empty suffix; node j > 0 is the (j)-th codeword made
    std::vector<int64_t> count(1, 0);
    std::vector<int32_t> last(1, -1);  // token a codeword ends with
    count.reserve((size_t)n + 1);
    last.reserve((size_t)n + 1);
    ChildTable child((size_t)n);
    for (int64_t i = 0; i < n; ++i) {
      int32_t node = 0;
      int64_t depth = 0;
      while (depth <= i) {
        const int32_t c = child.find(node, corpus[i - depth]);
        if (c < 0) break;
        node = c;
        ++depth;
      }
      if (depth == i + 1) {  // the whole text up to i is a codeword
        ++count[node];
        continue;
      }
      const int32_t fresh = (int32_t)count.size();
      count.push_back(1);
      last.push_back(corpus[i]);
      child.insert(node, corpus[i - depth], fresh);
      if (node != 0) ++count[node];
    }
    const int32_t n_words = (int32_t)count.size() - 1;
    if (n_codewords) *n_codewords = n_words;

    // walk order: most frequent first, equal frequencies in creation order
    std::vector<int32_t> walk(n_words);
    for (int32_t j = 0; j < n_words; ++j) walk[j] = j + 1;
    std::stable_sort(walk.begin(), walk.end(),
                     [&](int32_t a, int32_t b) { return count[a] > count[b]; });

    for (int64_t t = 0; t < vocab; ++t) d_out[t] = 1;
    int64_t total = vocab;
    while (total < v) {
      bool gave = false;
      for (int32_t j : walk) {
        int32_t &dt = d_out[last[j]];
        if (dt < k) {
          ++dt;
          gave = true;
          if (++total == v) break;
        }
      }
      if (!gave) {
        set_error("l3_lzw_allocate: every token that ends a codeword is at k; v is out of reach");
        return L3_ERR_INVALID_ARG;
      }
    }
  } catch (const std::bad_alloc &) {
    set_error("l3_lzw_allocate: out of host memory");
    return L3_ERR_OOM;
  }
  return L3_OK;
}
