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

// Step 1 (host): the codewords and their frequencies. count[j], last[j] for
// codeword j = 1..W (index 0 is the empty suffix). Throws std::bad_alloc.
void lzw_scan(const int32_t *corpus, int64_t n, std::vector<int64_t> &count,
              std::vector<int32_t> &last) {
  // nodes: 0 is the empty suffix; node j > 0 is the (j)-th codeword made
  count.assign(1, 0);
  last.assign(1, -1);  // token a codeword ends with
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
}

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
    std::vector<int64_t> count;
    std::vector<int32_t> last;
    lzw_scan(corpus, n, count, last);
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

// ---------------------------------------------------------------------------
// Steps 2-3 on the GPU
//
// The walk of step 2 visits the codewords in a fixed order (frequency
// descending, creation order among equals), and each visit gives the
// codeword's last token one row unless it holds k. So after P complete walks
// token t holds min(k, 1 + P cnt_t), cnt_t being how many codewords end with
// t, and the rows handed out so far are T(P) = sum_t min(k, 1 + P cnt_t),
// non-decreasing in P. The walks stop inside walk P* + 1, where P* is the
// largest P with T(P) <= v: in that walk the r-th codeword (in walk order)
// ending with t gives a row iff min(k, 1 + P* cnt_t) + r < k, and giving stops
// after v - T(P*) rows. This is the sequential walk's result, reached with
// one sort by frequency, one sort by token (the rank r), a binary search over
// P and one prefix sum.
// ---------------------------------------------------------------------------
namespace l3 {
namespace {

constexpr int LZW_THREADS = 1024;

// rows of token t after P complete walks: min(k, 1 + P c), without overflow
__device__ __forceinline__ int64_t rows_after(int64_t P, int64_t c, int64_t k) {
  if (c == 0 || P == 0) return 1;
  return P > (k - 1) / c ? k : 1 + P * c;
}

__global__ void k_lzw_keys(const int32_t *__restrict__ count, int64_t W, int32_t max_count,
                           int32_t *__restrict__ keys) {
  const int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (j < W) keys[j] = max_count - count[j];  // ascending key = descending frequency
}

__global__ void k_lzw_tokens(const int32_t *__restrict__ order, const int32_t *__restrict__ last,
                             int64_t W, int32_t *__restrict__ tok, int32_t *__restrict__ cnt) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= W) return;
  const int32_t t = last[order[i]];
  tok[i] = t;
  atomicAdd(&cnt[t], 1);
}

// one CTA: T(P) over all tokens for a P
__device__ int64_t lzw_total(const int32_t *cnt, int64_t vocab, int64_t k, int64_t P,
                             int64_t *red) {
  int64_t s = 0;
  for (int64_t t = threadIdx.x; t < vocab; t += LZW_THREADS) s += rows_after(P, cnt[t], k);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();
  if (lane == 0) red[warp] = s;
  __syncthreads();
  int64_t total = 0;
  for (int w = 0; w < LZW_THREADS / 32; ++w) total += red[w];
  return total;
}

// P* and the rows left for the partial walk; state[0] = P*, state[1] = rows
// left, state[2] = 1 if v is out of reach
__global__ void __launch_bounds__(LZW_THREADS) k_lzw_passes(const int32_t *__restrict__ cnt,
                                                            int64_t vocab, int64_t v, int64_t k,
                                                            int64_t *state) {
  __shared__ int64_t red[LZW_THREADS / 32];
  // every walk after the (k-1)-th gives nothing: T(k) is the most reachable
  const int64_t t_sat = lzw_total(cnt, vocab, k, k, red);
  if (t_sat < v) {
    if (threadIdx.x == 0) {
      state[0] = 0;
      state[1] = 0;
      state[2] = 1;
    }
    return;
  }
  int64_t lo = 0, hi = k;  // T(lo) <= v (T(0) = vocab <= v); find the largest such P
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) / 2;
    if (lzw_total(cnt, vocab, k, mid, red) <= v)
      lo = mid;
    else
      hi = mid - 1;
  }
  const int64_t t_lo = lzw_total(cnt, vocab, k, lo, red);
  if (threadIdx.x == 0) {
    state[0] = lo;
    state[1] = v - t_lo;
    state[2] = 0;
  }
}

__global__ void k_lzw_base(const int32_t *__restrict__ cnt, int64_t vocab, int64_t k,
                           const int64_t *state, int32_t *__restrict__ d) {
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t < vocab) d[t] = (int32_t)rows_after(state[0], cnt[t], k);
}

// flag[i] = 1 when walk position i gives a row in the partial walk (before
// the budget cut): its rank r among the codewords ending with the same token
// is below k - d_t
__global__ void k_lzw_flags(const int32_t *__restrict__ stok, const int32_t *__restrict__ spos,
                            const int32_t *__restrict__ start, const int32_t *__restrict__ d,
                            int64_t W, int64_t k, const int64_t *state,
                            int32_t *__restrict__ flag) {
  const int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (s >= W) return;
  const int32_t t = stok[s];
  const int64_t r = s - start[t];
  flag[spos[s]] = (state[1] > 0 && (int64_t)d[t] + r < k) ? 1 : 0;
}

// after the exclusive scan of the flags: give the first `rows left` of them
__global__ void k_lzw_take(const int32_t *__restrict__ pre, const int32_t *__restrict__ tok,
                           int64_t W, const int64_t *state, int32_t *__restrict__ d) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= W) return;
  if (pre[i + 1] - pre[i] == 1 && (int64_t)pre[i] < state[1]) atomicAdd(&d[tok[i]], 1);
}

int bits_for(int64_t max_value) {
  int b = 1;
  while (b < 31 && ((int64_t)1 << b) <= max_value) ++b;
  return b;
}

unsigned grid_for(int64_t n) { return (unsigned)std::max<int64_t>(1, (n + 255) / 256); }

}  // namespace
}  // namespace l3

extern "C" l3_status l3_lzw_allocate_device(const int32_t *corpus, int64_t n, int64_t vocab,
                                            int64_t v, int64_t k, int32_t *d_out,
                                            int64_t *n_codewords, void *stream) {
  set_error("");
  if ((n > 0 && !corpus) || !d_out || n < 0 || vocab < 1 || k < 1 || n > INT32_MAX - 2 ||
      vocab > INT32_MAX - 1 || k > INT32_MAX) {
    set_error("l3_lzw_allocate_device: NULL pointer or size out of range");
    return L3_ERR_INVALID_ARG;
  }
  if (v < vocab || v > vocab * k) {
    set_error("l3_lzw_allocate_device: need vocab <= v <= vocab * k");
    return L3_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(d_out) & 3u) {
    set_error("l3_lzw_allocate_device: d_out must be 4-byte aligned");
    return L3_ERR_INVALID_ARG;
  }
  for (int64_t i = 0; i < n; ++i)
    if (corpus[i] < 0 || corpus[i] >= vocab) {
      set_error("l3_lzw_allocate_device: a corpus token is outside [0, vocab)");
      return L3_ERR_INVALID_ARG;
    }
  std::vector<int32_t> count32, last;
  int32_t max_count = 0;
  try {
    std::vector<int64_t> count;
    lzw_scan(corpus, n, count, last);
    count32.resize(count.size() - 1);
    for (size_t j = 1; j < count.size(); ++j) {
      count32[j - 1] = (int32_t)count[j];  // a frequency never exceeds n < 2^31
      max_count = std::max(max_count, count32[j - 1]);
    }
    last.erase(last.begin());
  } catch (const std::bad_alloc &) {
    set_error("l3_lzw_allocate_device: out of host memory");
    return L3_ERR_OOM;
  }
  const int64_t W = (int64_t)count32.size();
  if (n_codewords) *n_codewords = W;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // device scratch: count, last, keys, order, tok, sorted tokens, their walk
  // positions, flags / prefix (W + 1), cnt and start (vocab + 1 each), sort
  // scratch, state
  const size_t w4 = ((size_t)W * 4 + 255) / 256 * 256, w41 = ((size_t)(W + 1) * 4 + 255) / 256 * 256;
  const size_t v41 = ((size_t)(vocab + 1) * 4 + 255) / 256 * 256;
  const size_t sort4 = (radix_sort_scratch_ints(W) * 4 + 255) / 256 * 256;
  const size_t bytes = 7 * w4 + w41 + 2 * v41 + sort4 + 256;
  char *base = nullptr;
  cudaError_t e = cudaMalloc(&base, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(LZW scratch)");
  char *c = base;
  auto take = [&](size_t b) {
    char *r = c;
    c += b;
    return reinterpret_cast<int32_t *>(r);
  };
  int32_t *d_count = take(w4), *d_last = take(w4), *keys = take(w4), *skeys = take(w4),
          *order = take(w4), *tok = take(w4), *spos = take(w4), *flag = take(w41),
          *cnt = take(v41), *start = take(v41), *sort_scratch = take(sort4);
  int64_t *state = reinterpret_cast<int64_t *>(take(256));
  int64_t host_state[3] = {0, 0, 0};
  l3_status st = L3_OK;
  auto run = [&]() -> l3_status {
    if (W > 0) {
      L3_CUDA_TRY(cudaMemcpyAsync(d_count, count32.data(), W * 4, cudaMemcpyHostToDevice, s));
      L3_CUDA_TRY(cudaMemcpyAsync(d_last, last.data(), W * 4, cudaMemcpyHostToDevice, s));
    }
    L3_CUDA_TRY(cudaMemsetAsync(cnt, 0, (vocab + 1) * 4, s));
    if (W > 0) {
      LaunchTimer t("lzw_walk_order", s);
      // walk order: stable sort by (max_count - frequency), i.e. frequency
      // descending, creation order among equals
      k_lzw_keys<<<grid_for(W), 256, 0, s>>>(d_count, W, max_count, keys);
      l3_status r = radix_sort_pairs(keys, nullptr, W, bits_for(max_count), skeys, order,
                                     sort_scratch, s);
      if (r != L3_OK) return r;
      k_lzw_tokens<<<grid_for(W), 256, 0, s>>>(order, d_last, W, tok, cnt);
    }
    {
      LaunchTimer t("lzw_full_walks", s);
      k_lzw_passes<<<1, LZW_THREADS, 0, s>>>(cnt, vocab, v, k, state);
      k_lzw_base<<<grid_for(vocab), 256, 0, s>>>(cnt, vocab, k, state, d_out);
    }
    if (W > 0) {
      LaunchTimer t("lzw_partial_walk", s);
      // rank of each walk position among the codewords ending with its token
      l3_status r = radix_sort_pairs(tok, nullptr, W, bits_for(vocab - 1), skeys, spos,
                                     sort_scratch, s);
      if (r != L3_OK) return r;
      L3_CUDA_TRY(cudaMemcpyAsync(start, cnt, vocab * 4, cudaMemcpyDeviceToDevice, s));
      if ((r = exclusive_scan(start, vocab, nullptr, s)) != L3_OK) return r;
      k_lzw_flags<<<grid_for(W), 256, 0, s>>>(skeys, spos, start, d_out, W, k, state, flag);
      if ((r = exclusive_scan(flag, W, nullptr, s)) != L3_OK) return r;
      k_lzw_take<<<grid_for(W), 256, 0, s>>>(flag, tok, W, state, d_out);
    }
    L3_CUDA_TRY(cudaGetLastError());
    L3_CUDA_TRY(cudaMemcpyAsync(host_state, state, sizeof host_state, cudaMemcpyDeviceToHost, s));
    L3_CUDA_TRY(cudaStreamSynchronize(s));
    return L3_OK;
  };
  st = run();
  if (st != L3_OK) {
    // the scratch may still be in use by work already enqueued
    cudaStreamSynchronize(s);
  }
  cudaFree(base);
  if (st == L3_OK && host_state[2]) {
    set_error("l3_lzw_allocate_device: every token that ends a codeword is at k; v is out of reach");
    return L3_ERR_INVALID_ARG;
  }
  return st;
}
