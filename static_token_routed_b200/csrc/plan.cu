// Batch plan: validate, stable LSD radix sort by token ID, group build and
// work lists.
//
// "L³: Large Lookup Layers" — sciencestack page, Fig. 3 caption: since the
// layer mixes channels only, sorting the batch by token ID turns its
// attention mask block-diagonal, and the sort is cheap to invert; kimjy99
// review §2 states the same (sort B by T). The sort here is stable, so equal
// IDs keep their original order and the plan is unique.
//
// Kernels (all on the caller's stream, no host round trip until the end):
//   validate offsets -> per pass { digit histogram per tile, one-CTA scan of
//   the (digit, tile) counts, stable scatter } -> group heads + inverse
//   permutation -> scan -> group fill -> scan of d_t -> work-item counts ->
//   scans -> work-item fill.
#include <algorithm>
#include <initializer_list>
#include <mutex>

#include "l3_internal.cuh"

namespace l3 {
namespace {

constexpr int RADIX_BITS = 9;  // 18-bit IDs (vocab <= 262144) in two passes
constexpr int RADIX = 1 << RADIX_BITS;
constexpr int SORT_THREADS = 256;
constexpr int SORT_WARPS = SORT_THREADS / 32;
constexpr int SORT_ITEMS = 8;                            // per thread
constexpr int SORT_TILE = SORT_THREADS * SORT_ITEMS;     // elements per CTA
constexpr int WARP_SPAN = SORT_TILE / SORT_WARPS;        // contiguous elements per warp
constexpr int SCAN_THREADS = 1024;
constexpr int SCAN_ITEMS = 16;
constexpr int SCAN_CHUNK = SCAN_THREADS * SCAN_ITEMS;
constexpr int MAX_DT_BUCKETS = 1025;  // d_t <= k <= 1024
constexpr int N_CLASSES = 4;          // tail items with 1, 2, 3-4 and 5-8 tokens
constexpr int SMALL_PLAN_MAX_TOKENS = 4096;  // batches planned by one CTA

__host__ __device__ __forceinline__ int token_class(int nt) {
  return nt <= 1 ? 0 : nt == 2 ? 1 : nt <= 4 ? 2 : 3;
}

// d_t bucket, largest d_t first: d_t = k_cap -> 0 ... d_t = 1 -> k_cap - 1.
// Clamped so that rows from invalid offsets (reported by the plan, never
// run) still index inside the bucket arrays.
__host__ __device__ __forceinline__ int bucket_of(int rows, int k_cap) {
  return k_cap - max(0, min(rows, k_cap));
}

// slots of the device info block read back at the end of l3_plan
enum {
  INFO_ERR = 0,
  INFO_G,
  INFO_TILES,
  INFO_TAILS,
  INFO_ROWS,
  INFO_ROWS_MULTI,
  INFO_DENSE_GROUPS,
  INFO_MAX_TOKENS,
  INFO_CLS,              // 5 slots: first tail item of each token-count class, then the total
  INFO_SPLIT = INFO_CLS + 5,  // 4 slots: first item of each class with d_t <= TAIL_SMALL_ROWS
  INFO_DENSE_SMALL = INFO_SPLIT + 4,  // dense tiles of groups with d_t <= DENSE_SMALL_ROWS
  INFO_SKINNY_BIG,    // dense tiles of at most SKINNY_TOKENS tokens, d_t > DENSE_SMALL_ROWS
  INFO_SKINNY_SMALL,  // the same, d_t <= DENSE_SMALL_ROWS
  INFO_SLOTS
};
static_assert(INFO_SLOTS <= 64, "the plan zeroes 64 info words");

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__global__ void k_validate_offsets(const int32_t *__restrict__ offsets, int64_t vocab, int64_t v,
                                   int64_t k, int32_t *info) {
  int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= vocab) return;
  int64_t d = (int64_t)offsets[t + 1] - offsets[t];
  bool bad = d < 1 || d > k;
  if (t == 0 && offsets[0] != 0) bad = true;
  if (t == vocab - 1 && offsets[vocab] != v) bad = true;
  if (bad) atomicOr(&info[INFO_ERR], DEV_ERR_BAD_OFFSETS);
}

// Digit histogram of one tile; counts land digit-major: hist[d * n_tiles + tile].
// With vocab > 0 (the first pass) keys outside [0, vocab) are flagged, and
// with `offsets` the CTAs also check the offsets array as k_validate_offsets
// does (grid-stride), which saves that launch.
__global__ void __launch_bounds__(SORT_THREADS)
    k_radix_hist(const int32_t *__restrict__ keys, int64_t n, int shift, int32_t *__restrict__ hist,
                 int n_tiles, int64_t vocab, int32_t *info, const int32_t *__restrict__ offsets,
                 int64_t v, int64_t k_cap) {
  __shared__ int32_t cnt[RADIX];
  for (int i = threadIdx.x; i < RADIX; i += SORT_THREADS) cnt[i] = 0;
  if (offsets) {
    bool bad_off = false;
    for (int64_t t = blockIdx.x * (int64_t)SORT_THREADS + threadIdx.x; t < vocab;
         t += (int64_t)gridDim.x * SORT_THREADS) {
      const int64_t d = (int64_t)offsets[t + 1] - offsets[t];
      bad_off |= d < 1 || d > k_cap;
      if (t == 0 && offsets[0] != 0) bad_off = true;
      if (t == vocab - 1 && offsets[vocab] != v) bad_off = true;
    }
    if (bad_off) atomicOr(&info[INFO_ERR], DEV_ERR_BAD_OFFSETS);
  }
  __syncthreads();
  int64_t base = (int64_t)blockIdx.x * SORT_TILE;
  bool bad = false;
#pragma unroll
  for (int j = 0; j < SORT_ITEMS; ++j) {
    int64_t i = base + threadIdx.x + (int64_t)j * SORT_THREADS;
    if (i < n) {
      int32_t key = keys[i];
      if (vocab > 0 && (key < 0 || key >= vocab)) bad = true;
      atomicAdd(&cnt[((uint32_t)key >> shift) & (RADIX - 1)], 1);
    }
  }
  if (bad) atomicOr(&info[INFO_ERR], DEV_ERR_TOKEN_RANGE);
  __syncthreads();
  for (int d = threadIdx.x; d < RADIX; d += SORT_THREADS) hist[(int64_t)d * n_tiles + blockIdx.x] = cnt[d];
}

// Stable scatter of one tile. offs[d * n_tiles + tile] is the first output
// position of digit d for this tile (exclusive scan of the histogram in
// digit-major order), or, with `raw`, the histogram itself: the CTA then adds
// up digit d's counts in the earlier tiles and in all tiles (few tiles:
// FUSED_SCAN_TILES at most) and scans the digit totals itself, which saves a
// scan launch per pass. Each warp owns a contiguous span of the tile and
// walks it in order, ranking equal digits with __match_any_sync, so the output
// keeps input order among equal digits.
constexpr int FUSED_SCAN_TILES = 64;
static_assert(RADIX % SORT_THREADS == 0, "whole digits per thread");

__global__ void __launch_bounds__(SORT_THREADS)
    k_radix_scatter(const int32_t *__restrict__ keys_in, const int32_t *__restrict__ vals_in,
                    int32_t *__restrict__ keys_out, int32_t *__restrict__ vals_out, int64_t n,
                    int shift, const int32_t *__restrict__ offs, int n_tiles, int raw,
                    int32_t *__restrict__ inv_out) {
  __shared__ int32_t whist[SORT_WARPS][RADIX];
  __shared__ int32_t dbase[RADIX];
  __shared__ int32_t wtot[SORT_WARPS];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int i = threadIdx.x; i < SORT_WARPS * RADIX; i += SORT_THREADS) (&whist[0][0])[i] = 0;
  __syncthreads();

  int64_t base = (int64_t)blockIdx.x * SORT_TILE + (int64_t)warp * WARP_SPAN;
  int32_t key[SORT_ITEMS], rank[SORT_ITEMS];
  int digit[SORT_ITEMS];
  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int it = 0; it < SORT_ITEMS; ++it) {
    int64_t i = base + it * 32 + lane;
    bool valid = i < n;
    key[it] = valid ? keys_in[i] : 0;
    int d = valid ? (int)(((uint32_t)key[it] >> shift) & (RADIX - 1)) : RADIX;
    digit[it] = d;
    uint32_t peers = __match_any_sync(0xffffffffu, d);
    int prior = valid ? whist[warp][d] : 0;
    rank[it] = prior + __popc(peers & lt);
    __syncwarp();
    if (valid && lane == __ffs(peers) - 1) whist[warp][d] = prior + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  {
    // DPT consecutive digits per thread
    constexpr int DPT = RADIX / SORT_THREADS;
    int32_t pre[DPT], tot[DPT];
#pragma unroll
    for (int j = 0; j < DPT; ++j) {
      const int d = threadIdx.x * DPT + j;
      int32_t run = 0;
#pragma unroll
      for (int w = 0; w < SORT_WARPS; ++w) {
        int32_t c = whist[w][d];
        whist[w][d] = run;
        run += c;
      }
      pre[j] = tot[j] = 0;
      if (!raw) {
        dbase[d] = offs[(int64_t)d * n_tiles + blockIdx.x];
      } else {
        // digit d in earlier tiles, in all tiles
        const int32_t *row = offs + (int64_t)d * n_tiles;
        for (int t0 = 0; t0 < n_tiles; t0 += 16) {
          int32_t c[16];  // sixteen loads in flight
#pragma unroll
          for (int u = 0; u < 16; ++u) c[u] = t0 + u < n_tiles ? row[t0 + u] : 0;
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            tot[j] += c[u];
            pre[j] += t0 + u < (int)blockIdx.x ? c[u] : 0;
          }
        }
      }
    }
    if (raw) {
      // exclusive scan of the digit totals across the CTA (digits in order)
      int32_t mine = 0;
#pragma unroll
      for (int j = 0; j < DPT; ++j) mine += tot[j];
      int32_t incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (lane == 31) wtot[warp] = incl;
      __syncthreads();
      int32_t before = incl - mine;
      for (int w = 0; w < warp; ++w) before += wtot[w];
#pragma unroll
      for (int j = 0; j < DPT; ++j) {
        dbase[threadIdx.x * DPT + j] = before + pre[j];
        before += tot[j];
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < SORT_ITEMS; ++it) {
    int64_t i = base + it * 32 + lane;
    if (i < n) {
      int d = digit[it];
      int32_t pos = dbase[d] + whist[warp][d] + rank[it];
      const int32_t val = vals_in ? vals_in[i] : (int32_t)i;
      keys_out[pos] = key[it];
      vals_out[pos] = val;
      if (inv_out) inv_out[val] = pos;  // the last pass: the inverse permutation
    }
  }
}

// Exclusive scans, one array per CTA: out[i] = sum in[0..i-1] for i <= n (out
// has n + 1 entries; in == out is allowed: every value is read before the
// chunk's first store); the total also goes to *total if given.
struct ScanJob {
  const int32_t *in;
  int32_t *out;
  int64_t n;
  int32_t *total;
  const int32_t *n_dev;  // if set, only the first min(n, *n_dev) values are scanned
};
struct ScanJobs {
  ScanJob job[4];
};

__global__ void __launch_bounds__(SCAN_THREADS) k_scan_multi(ScanJobs jobs) {
  __shared__ int32_t warp_sums[SCAN_THREADS / 32];
  __shared__ int32_t chunk_total;
  // select the job without indexing the parameter array dynamically
  ScanJob J = jobs.job[0];
  if (blockIdx.x == 1) J = jobs.job[1];
  if (blockIdx.x == 2) J = jobs.job[2];
  if (blockIdx.x == 3) J = jobs.job[3];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (J.n_dev) J.n = min(J.n, (int64_t)*J.n_dev);
  // Each warp owns a contiguous segment of SCAN_ITEMS * 32 values of the chunk
  // and walks it in rounds of 32 consecutive values (coalesced loads and
  // stores); a round's inclusive warp scan plus the carry of earlier rounds
  // gives the prefix inside the segment, and segment totals are scanned
  // across warps through shared memory.
  int32_t carry = 0;
  for (int64_t base = 0; base < J.n; base += SCAN_CHUNK) {
    const int64_t seg = base + (int64_t)warp * (SCAN_ITEMS * 32);
    int32_t v[SCAN_ITEMS], incl[SCAN_ITEMS];
#pragma unroll
    for (int r = 0; r < SCAN_ITEMS; ++r) {
      const int64_t i = seg + r * 32 + lane;
      v[r] = i < J.n ? J.in[i] : 0;
    }
    int32_t run = 0;  // sum of earlier rounds in this warp's segment
#pragma unroll
    for (int r = 0; r < SCAN_ITEMS; ++r) {
      int32_t x = v[r];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
      }
      incl[r] = x + run;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) warp_sums[warp] = run;
    __syncthreads();
    if (warp == 0) {
      const int32_t w = warp_sums[lane];
      int32_t wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += t;
      }
      warp_sums[lane] = wi - w;  // exclusive prefix of segment totals
      if (lane == 31) chunk_total = wi;
    }
    __syncthreads();
    const int32_t off = carry + warp_sums[warp];
#pragma unroll
    for (int r = 0; r < SCAN_ITEMS; ++r) {
      const int64_t i = seg + r * 32 + lane;
      if (i < J.n) J.out[i] = off + incl[r] - v[r];
    }
    carry += chunk_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    J.out[J.n] = carry;
    if (J.total) *J.total = carry;
  }
}

// launch up to four independent scans as one grid
l3_status scan_multi(std::initializer_list<ScanJob> js, cudaStream_t s) {
  ScanJobs jobs{};
  int k = 0;
  for (const ScanJob &j : js) jobs.job[k++] = j;
  LaunchTimer t("plan_scan", s);
  k_scan_multi<<<k, SCAN_THREADS, 0, s>>>(jobs);
  return L3_OK;
}

// The groups of a sorted batch in one CTA: head flags (a new ID starts at
// sorted position i), their exclusive scan (the group of each head) and the
// group arrays, in the coalesced warp-segment layout of k_scan_multi.
__global__ void __launch_bounds__(SCAN_THREADS)
    k_group_scan(const int32_t *__restrict__ sorted, int64_t n,
                 const int32_t *__restrict__ offsets, int64_t vocab, int32_t *__restrict__ group_ids,
                 int32_t *__restrict__ group_tok_start, int32_t *__restrict__ group_row_start,
                 int32_t *__restrict__ group_rows, int32_t *info) {
  __shared__ int32_t warp_sums[SCAN_THREADS / 32];
  __shared__ int32_t chunk_total;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int32_t carry = 0;
  for (int64_t base = 0; base < n; base += SCAN_CHUNK) {
    const int64_t seg = base + (int64_t)warp * (SCAN_ITEMS * 32);
    int32_t id[SCAN_ITEMS], v[SCAN_ITEMS], incl[SCAN_ITEMS];
#pragma unroll
    for (int r = 0; r < SCAN_ITEMS; ++r) {
      const int64_t i = seg + r * 32 + lane;
      id[r] = i < n ? sorted[i] : 0;
      v[r] = i < n && (i == 0 || id[r] != sorted[i - 1]) ? 1 : 0;
    }
    int32_t run = 0;  // heads in earlier rounds of this warp's segment
#pragma unroll
    for (int r = 0; r < SCAN_ITEMS; ++r) {
      int32_t x = v[r];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
      }
      incl[r] = x + run;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) warp_sums[warp] = run;
    __syncthreads();
    if (warp == 0) {
      const int32_t w = warp_sums[lane];
      int32_t wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += t;
      }
      warp_sums[lane] = wi - w;
      if (lane == 31) chunk_total = wi;
    }
    __syncthreads();
    const int32_t off = carry + warp_sums[warp];
#pragma unroll
    for (int r = 0; r < SCAN_ITEMS; ++r) {
      if (v[r]) {
        const int64_t i = seg + r * 32 + lane;
        const int32_t g = off + incl[r] - 1;
        group_ids[g] = id[r];
        group_tok_start[g] = (int32_t)i;
        const bool ok = id[r] >= 0 && id[r] < vocab;
        const int32_t r0 = ok ? offsets[id[r]] : 0;
        group_row_start[g] = r0;
        group_rows[g] = ok ? offsets[id[r] + 1] - r0 : 0;
      }
    }
    carry += chunk_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    group_tok_start[carry] = (int32_t)n;
    info[INFO_G] = carry;
  }
}

__global__ void k_item_counts(const int32_t *__restrict__ group_tok_start,
                              const int32_t *__restrict__ group_rows, int64_t cap,
                              int dense_min_tokens, int dense_min_rows, int dense_max_rows,
                              int32_t *__restrict__ tiles, int32_t *__restrict__ tails,
                              int32_t *__restrict__ dcount, int32_t *__restrict__ tcount,
                              int k_cap, int32_t *info) {
  int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (g >= cap) return;
  int32_t G = info[INFO_G];
  int32_t nt = 0, nl = 0;
  if (g < G) {
    int32_t c = group_tok_start[g + 1] - group_tok_start[g];
    int32_t rows = group_rows[g];
    bool dense = dense_min_tokens > 0 && c >= dense_min_tokens && rows >= dense_min_rows &&
                 rows <= dense_max_rows;
    if (dense) {
      nt = (c + DENSE_TILE_M - 1) / DENSE_TILE_M;
      atomicAdd(&info[INFO_DENSE_GROUPS], 1);
      if (rows <= DENSE_SMALL_ROWS) atomicAdd(&info[INFO_DENSE_SMALL], nt);
      // the group's last tile holds c - (nt - 1) 128 tokens
      if (c - (nt - 1) * DENSE_TILE_M <= SKINNY_TOKENS)
        atomicAdd(&info[rows <= DENSE_SMALL_ROWS ? INFO_SKINNY_SMALL : INFO_SKINNY_BIG], 1);
      // dense tiles are listed largest d_t first (bucket k_cap - d_t): the
      // longest CTAs start first, and the d_t > DENSE_SMALL_ROWS tiles come
      // before the others
      atomicAdd(&tcount[bucket_of(rows, k_cap)], nt);
    } else {
      nl = (c + TAIL_TOKENS - 1) / TAIL_TOKENS;
    }
    if (rows > 1) atomicAdd(&info[INFO_ROWS_MULTI], rows);
    atomicMax(&info[INFO_MAX_TOKENS], c);
    // tail items are listed by token-count class, then largest d_t first:
    // bucket class * (k_cap + 1) + (k_cap - d_t), so an ascending scan gives
    // the order
    if (nl > 0) {
      const int db = bucket_of(rows, k_cap);
      const int full = c / TAIL_TOKENS, rest = c % TAIL_TOKENS;
      if (full > 0) atomicAdd(&dcount[token_class(TAIL_TOKENS) * (k_cap + 1) + db], full);
      if (rest > 0) atomicAdd(&dcount[token_class(rest) * (k_cap + 1) + db], 1);
    }
  }
  tiles[g] = nt;
  tails[g] = nl;
}

__global__ void k_item_fill(const int32_t *__restrict__ group_tok_start,
                            const int32_t *__restrict__ group_row_start,
                            const int32_t *__restrict__ group_rows,
                            const int32_t *__restrict__ perm,
                            const int32_t *__restrict__ tiles, int32_t *__restrict__ tcursor,
                            const int32_t *__restrict__ tails, int32_t *__restrict__ dcursor,
                            int k_cap, int64_t cap, DenseTile *__restrict__ dense,
                            TailItem *__restrict__ tail, int32_t *info) {
  int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (g >= cap || g >= info[INFO_G]) return;
  const int32_t start = group_tok_start[g];
  const int32_t c = group_tok_start[g + 1] - start;
  const int32_t rows = group_rows[g];
  // a group's dense tiles sit side by side (they share K_t, V_t through L2);
  // any order of the groups inside a d_t bucket gives the same results
  if (tiles[g] > 0) {
    const int32_t pos = atomicAdd(&tcursor[bucket_of(rows, k_cap)], tiles[g]);
    for (int32_t j = 0; j < tiles[g]; ++j)
      dense[pos + j] = DenseTile{(int32_t)g, start + j * DENSE_TILE_M};
  }
  for (int32_t j = 0; j < tails[g]; ++j) {
    TailItem it;
    it.r0 = group_row_start[g];
    it.d = (int16_t)rows;
    it.nt = (int16_t)min(TAIL_TOKENS, c - j * TAIL_TOKENS);
#pragma unroll
    for (int t = 0; t < TAIL_TOKENS; ++t)
      it.tok[t] = t < it.nt ? perm[start + j * TAIL_TOKENS + t] : 0;
    it.pad[0] = it.pad[1] = 0;
    // position within its bucket: any order inside a bucket gives the same results
    const int bucket = token_class(it.nt) * (k_cap + 1) + bucket_of(rows, k_cap);
    const int32_t pos = atomicAdd(&dcursor[bucket], 1);
    tail[pos] = it;
  }
}

// first tail item of each class (read before the fill kernel moves the cursors)
__global__ void k_class_starts(const int32_t *__restrict__ scanned, int k_cap, int32_t *info) {
  const int c = threadIdx.x;
  if (c <= N_CLASSES) info[INFO_CLS + c] = scanned[c * (k_cap + 1)];
  // buckets run from d_t = k_cap down to 1 inside a class
  const int small = min(TAIL_SMALL_ROWS, k_cap);
  if (c < N_CLASSES) info[INFO_SPLIT + c] = scanned[c * (k_cap + 1) + (k_cap - small)];
}

// ---------------------------------------------------------------------------
// Whole plan in one CTA for small batches (N <= SMALL_PLAN_MAX_TOKENS): the
// same outputs as the multi-kernel path, built in shared memory by 1024
// threads, so a decode-sized batch costs one launch instead of a dozen.
//   1. keys (id << 32 | original index) are bitonic-sorted: unique keys, so
//      the order is the stable sort by ID;
//   2. group heads, their exclusive scan (group positions), the group arrays;
//   3. the exclusive scan of d_t over groups (segment row offsets);
//   4. dense tiles and tail items counted per bucket, bucket starts scanned,
//      items written at their bucket's cursor (any order inside a bucket).
// Info slots are all written here (the offsets check, launched after this
// kernel, ORs its error bit into the same word).
// ---------------------------------------------------------------------------
constexpr int SMALL_THREADS = 1024;

// in-place exclusive scan of data[0..n) by the whole CTA; returns the total
// (every thread gets it). `tmp` holds SMALL_THREADS / 32 + 1 ints.
__device__ int block_exclusive_scan(int32_t *data, int n, int32_t *tmp) {
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int per = (n + SMALL_THREADS - 1) / SMALL_THREADS;
  const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
  int32_t local = 0;
  for (int i = b0; i < b1; ++i) local += data[i];
  int32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int32_t w = lane < SMALL_THREADS / 32 ? tmp[lane] : 0;
    int32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < SMALL_THREADS / 32) tmp[lane] = wi - w;
    if (lane == 31) tmp[SMALL_THREADS / 32] = wi;
  }
  __syncthreads();
  int32_t run = tmp[warp] + incl - local;
  for (int i = b0; i < b1; ++i) {
    const int32_t v = data[i];
    data[i] = run;
    run += v;
  }
  const int32_t total = tmp[SMALL_THREADS / 32];
  __syncthreads();
  return total;
}

struct SmallPlanArgs {
  const int32_t *ids;
  const int32_t *offsets;
  int64_t vocab;
  int n;            // tokens, <= SMALL_PLAN_MAX_TOKENS
  int np;           // n rounded up to a power of two (>= 2)
  int k_cap;        // buckets per class: d_t in [1, k_cap]
  int dense_min_tokens, dense_min_rows, dense_max_rows;
  bool staged;
  int32_t *perm, *inv_perm, *sorted_ids;
  int32_t *group_ids, *group_tok_start, *group_row_start, *group_row_src, *group_rows, *seg_rows;
  DenseTile *dense;
  TailItem *tail;
  int32_t *info;
};

__global__ void __launch_bounds__(SMALL_THREADS, 1) k_plan_small(SmallPlanArgs A) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x;
  const int n = A.n, np = A.np, k_cap = A.k_cap;
  const int n_buckets = N_CLASSES * (k_cap + 1);
  uint64_t *key = reinterpret_cast<uint64_t *>(smem);                  // [np]
  int32_t *gpos = reinterpret_cast<int32_t *>(key + np);               // [n + 1]
  int32_t *gstart = gpos + (n + 1);                                    // [n + 1]
  int32_t *grows = gstart + (n + 1);                                   // [n + 1]
  int32_t *dcount = grows + (n + 1);                                   // [n_buckets + 1]
  int32_t *tcount = dcount + (n_buckets + 1);                          // [k_cap + 2]
  int32_t *tmp = tcount + (k_cap + 2);                                 // [33]
  __shared__ int32_t s_err, s_rows_multi, s_max_tokens, s_dense_groups, s_dense_small;
  __shared__ int32_t s_skinny[2];  // big, small

  if (tid == 0) {
    s_err = 0;
    s_rows_multi = 0;
    s_max_tokens = 0;
    s_dense_groups = 0;
    s_dense_small = 0;
    s_skinny[0] = s_skinny[1] = 0;
  }
  for (int i = tid; i < n_buckets + 1; i += SMALL_THREADS) dcount[i] = 0;
  for (int i = tid; i < k_cap + 2; i += SMALL_THREADS) tcount[i] = 0;
  bool bad = false;
  for (int i = tid; i < np; i += SMALL_THREADS) {
    uint64_t k = ~0ull;  // padding sorts last
    if (i < n) {
      const int32_t id = A.ids[i];
      if (id < 0 || id >= A.vocab) bad = true;
      k = ((uint64_t)(uint32_t)id << 32) | (uint32_t)i;
    }
    key[i] = k;
  }
  if (bad) atomicOr(&s_err, DEV_ERR_TOKEN_RANGE);
  __syncthreads();

  // 1. bitonic sort, ascending
  for (int size = 2; size <= np; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = tid; t < np / 2; t += SMALL_THREADS) {
        const int lo = 2 * t - (t & (stride - 1));  // index whose partner is lo + stride
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t a = key[lo], b = key[hi];
        if ((a > b) == up) {
          key[lo] = b;
          key[hi] = a;
        }
      }
      __syncthreads();
    }
  }

  // 2. sorted IDs, permutation, group heads
  for (int i = tid; i < n; i += SMALL_THREADS) {
    const int32_t id = (int32_t)(key[i] >> 32), src = (int32_t)(uint32_t)key[i];
    A.sorted_ids[i] = id;
    A.perm[i] = src;
    A.inv_perm[src] = i;
    gpos[i] = (i == 0 || (int32_t)(key[i - 1] >> 32) != id) ? 1 : 0;
  }
  __syncthreads();
  const int G = block_exclusive_scan(gpos, n, tmp);
  for (int i = tid; i < n; i += SMALL_THREADS) {
    const int32_t id = (int32_t)(key[i] >> 32);
    if (i == 0 || (int32_t)(key[i - 1] >> 32) != id) {
      const int g = gpos[i];
      const bool ok = id >= 0 && id < A.vocab;
      const int32_t r0 = ok ? A.offsets[id] : 0;
      const int32_t rows = ok ? A.offsets[id + 1] - r0 : 0;
      A.group_ids[g] = id;
      A.group_tok_start[g] = i;
      A.group_row_src[g] = r0;
      A.group_rows[g] = rows;
      gstart[g] = i;
      grows[g] = rows;
    }
  }
  if (tid == 0) {
    A.group_tok_start[G] = n;
    gstart[G] = n;
  }
  __syncthreads();

  // 3. bucket counts of dense tiles and tail items (grows is still d_t here)
  for (int g = tid; g < G; g += SMALL_THREADS) {
    const int c = gstart[g + 1] - gstart[g];
    const int rows = grows[g];
    const bool dense = A.dense_min_tokens > 0 && c >= A.dense_min_tokens &&
                       rows >= A.dense_min_rows && rows <= A.dense_max_rows;
    if (rows > 1) atomicAdd(&s_rows_multi, rows);
    atomicMax(&s_max_tokens, c);
    const int db = bucket_of(rows, k_cap);
    if (dense) {
      const int nt = (c + DENSE_TILE_M - 1) / DENSE_TILE_M;
      atomicAdd(&s_dense_groups, 1);
      if (rows <= DENSE_SMALL_ROWS) atomicAdd(&s_dense_small, nt);
      if (c - (nt - 1) * DENSE_TILE_M <= SKINNY_TOKENS)
        atomicAdd(&s_skinny[rows <= DENSE_SMALL_ROWS ? 1 : 0], 1);
      atomicAdd(&tcount[db], nt);
    } else {
      const int full = c / TAIL_TOKENS, rest = c % TAIL_TOKENS;
      if (full > 0) atomicAdd(&dcount[token_class(TAIL_TOKENS) * (k_cap + 1) + db], full);
      if (rest > 0) atomicAdd(&dcount[token_class(rest) * (k_cap + 1) + db], 1);
    }
  }
  __syncthreads();
  // segment row offsets: exclusive prefix of d_t over groups
  const int rows_total = block_exclusive_scan(grows, G, tmp);
  for (int g = tid; g < G; g += SMALL_THREADS) A.seg_rows[g] = grows[g];
  if (tid == 0) A.seg_rows[G] = rows_total;
  const int n_tiles = block_exclusive_scan(tcount, k_cap + 1, tmp);
  const int n_tails = block_exclusive_scan(dcount, n_buckets, tmp);
  if (tid == 0) {
    int32_t *info = A.info;
    info[INFO_ERR] = s_err;
    info[INFO_G] = G;
    info[INFO_TILES] = n_tiles;
    info[INFO_TAILS] = n_tails;
    info[INFO_ROWS] = rows_total;
    info[INFO_ROWS_MULTI] = s_rows_multi;
    info[INFO_DENSE_GROUPS] = s_dense_groups;
    info[INFO_MAX_TOKENS] = s_max_tokens;
    const int small = min(TAIL_SMALL_ROWS, k_cap);
    for (int c = 0; c <= N_CLASSES; ++c)
      info[INFO_CLS + c] = c < N_CLASSES ? dcount[c * (k_cap + 1)] : n_tails;
    for (int c = 0; c < N_CLASSES; ++c) info[INFO_SPLIT + c] = dcount[c * (k_cap + 1) + (k_cap - small)];
    info[INFO_DENSE_SMALL] = s_dense_small;
    info[INFO_SKINNY_BIG] = s_skinny[0];
    info[INFO_SKINNY_SMALL] = s_skinny[1];
  }
  __syncthreads();

  // 4. the work items at their buckets' cursors
  for (int g = tid; g < G; g += SMALL_THREADS) {
    const int start = gstart[g];
    const int c = gstart[g + 1] - start;
    const int32_t id = (int32_t)(key[start] >> 32);
    const bool ok = id >= 0 && id < A.vocab;
    const int32_t rows = ok ? A.offsets[id + 1] - A.offsets[id] : 0;
    // a staged plan addresses the group's rows where the staging copy puts them
    const int32_t r0 = A.staged ? grows[g] : (ok ? A.offsets[id] : 0);
    A.group_row_start[g] = r0;
    const bool dense = A.dense_min_tokens > 0 && c >= A.dense_min_tokens &&
                       rows >= A.dense_min_rows && rows <= A.dense_max_rows;
    const int db = bucket_of(rows, k_cap);
    if (dense) {
      const int nt = (c + DENSE_TILE_M - 1) / DENSE_TILE_M;
      const int pos = atomicAdd(&tcount[db], nt);
      for (int j = 0; j < nt; ++j) A.dense[pos + j] = DenseTile{g, start + j * DENSE_TILE_M};
    } else {
      const int n_items = (c + TAIL_TOKENS - 1) / TAIL_TOKENS;
      for (int j = 0; j < n_items; ++j) {
        TailItem it;
        it.r0 = r0;
        it.d = (int16_t)rows;
        it.nt = (int16_t)min(TAIL_TOKENS, c - j * TAIL_TOKENS);
#pragma unroll
        for (int t = 0; t < TAIL_TOKENS; ++t)
          it.tok[t] = t < it.nt ? (int32_t)(uint32_t)key[start + j * TAIL_TOKENS + t] : 0;
        it.pad[0] = it.pad[1] = 0;
        const int pos = atomicAdd(&dcount[token_class(it.nt) * (k_cap + 1) + db], 1);
        A.tail[pos] = it;
      }
    }
  }
}

inline int blocks_for(int64_t n, int threads) { return (int)std::max<int64_t>(1, (n + threads - 1) / threads); }

}  // namespace

// Staging copy: CTA g copies group g's rows of W_V (and of W_K when d_t > 1;
// a single row's logit is never needed) from the full tables to rows
// seg_rows[g].. of the staged tables, 16 bytes per thread per load, four
// loads in flight per thread (the source may sit across PCIe).
__global__ void k_stage_rows(const int32_t *__restrict__ group_row_src,
                             const int32_t *__restrict__ seg_rows,
                             const int32_t *__restrict__ group_rows,
                             const uint4 *__restrict__ W_K, const uint4 *__restrict__ W_V,
                             uint4 *__restrict__ K_st, uint4 *__restrict__ V_st, int k_vecs,
                             int v_vecs) {
  const int64_t g = blockIdx.x;  // one CTA per group of the plan
  const int64_t src = group_row_src[g], dst = seg_rows[g];
  const int32_t d = group_rows[g];
  for (int pass = 0; pass < 2; ++pass) {
    const int vecs = pass == 0 ? v_vecs : k_vecs;
    if (pass == 1 && d == 1) break;
    const uint4 *from = (pass == 0 ? W_V : W_K) + src * vecs;
    uint4 *to = (pass == 0 ? V_st : K_st) + dst * vecs;
    const int64_t total = (int64_t)d * vecs;
    for (int64_t i = threadIdx.x; i < total; i += 4 * (int64_t)blockDim.x) {
      uint4 r[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t j = i + u * (int64_t)blockDim.x;
        if (j < total) r[u] = from[j];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t j = i + u * (int64_t)blockDim.x;
        if (j < total) to[j] = r[u];
      }
    }
  }
}

// Scratch needed while building the plan, beyond the plan's own arrays.
size_t plan_scratch_bytes(int64_t n) {
  int64_t tiles = std::max<int64_t>(1, (n + SORT_TILE - 1) / SORT_TILE);
  size_t ints = 0;
  ints += 2 * (size_t)n;                 // ping-pong keys / vals
  ints += (size_t)RADIX * tiles + 1;     // histogram / offsets
  ints += 2 * ((size_t)n + 1);           // dense tiles and tail items per group
  ints += 64;                            // info block
  ints += 2 * (N_CLASSES * MAX_DT_BUCKETS + 1);  // tail items per bucket, and their cursors
  ints += 2 * (MAX_DT_BUCKETS + 1);      // dense tiles per d_t bucket, and their cursors
  return ints * sizeof(int32_t) + 256;
}

namespace {
std::mutex g_small_attr_mu;
bool g_small_attr[64] = {};

size_t small_plan_smem(int np, int n, int k_cap) {
  return (size_t)np * 8 + 3 * (size_t)(n + 1) * 4 + (size_t)(N_CLASSES * (k_cap + 1) + 1) * 4 +
         (size_t)(k_cap + 2) * 4 + 33 * 4 + 16;
}
}  // namespace

l3_status finish_plan(l3_plan_s *p, const int32_t *info, int64_t n, cudaStream_t s);

l3_status build_plan(l3_plan_s *p, const int32_t *ids, const int32_t *offsets, cudaStream_t s,
                     void *scratch, size_t scratch_bytes) {
  const int64_t n = p->n_tokens;
  const int64_t vocab = p->dims.vocab;
  const int64_t cap = n + 1;
  int32_t *sp = reinterpret_cast<int32_t *>(scratch);
  int32_t *keys_tmp = sp;
  sp += n;
  int32_t *vals_tmp = sp;
  sp += n;
  int64_t n_tiles = std::max<int64_t>(1, (n + SORT_TILE - 1) / SORT_TILE);
  int32_t *hist = sp;
  sp += RADIX * n_tiles + 1;
  int32_t *tiles = sp;
  sp += cap;
  int32_t *tails = sp;
  sp += cap;
  int32_t *info = sp;
  sp += 64;
  int32_t *dcount = sp;
  sp += N_CLASSES * MAX_DT_BUCKETS + 1;
  int32_t *dcursor = sp;
  sp += N_CLASSES * MAX_DT_BUCKETS + 1;
  int32_t *tcount = sp;
  sp += MAX_DT_BUCKETS + 1;
  int32_t *tcursor = sp;
  sp += MAX_DT_BUCKETS + 1;
  const int k_cap = (int)std::min<int64_t>(p->dims.k, MAX_DT_BUCKETS - 1);
  if ((size_t)((char *)sp - (char *)scratch) > scratch_bytes) {
    set_error("internal: plan scratch too small");
    return L3_ERR_INVALID_ARG;
  }

  // groups with enough tokens and rows go to the tensor-core attention kernel
  int dense_min_tokens = 0, dense_min_rows = 0, dense_max_rows = 0;
  if (dense_attention_supported(p->dims)) {
    dense_min_tokens = DENSE_MIN_TOKENS;
    dense_min_rows = DENSE_MIN_ROWS;
    dense_max_rows = dense_attention_max_rows();
  }
  if (n > 0 && n <= SMALL_PLAN_MAX_TOKENS) {
    // one CTA builds the whole plan; the offsets check runs after it and ORs
    // its error bit into the info word the plan kernel wrote
    SmallPlanArgs A;
    A.ids = ids;
    A.offsets = offsets;
    A.vocab = vocab;
    A.n = (int)n;
    A.np = 2;
    while (A.np < n) A.np <<= 1;
    A.k_cap = k_cap;
    A.dense_min_tokens = dense_min_tokens;
    A.dense_min_rows = dense_min_rows;
    A.dense_max_rows = dense_max_rows;
    A.staged = p->staged;
    A.perm = p->perm;
    A.inv_perm = p->inv_perm;
    A.sorted_ids = p->sorted_ids;
    A.group_ids = p->group_ids;
    A.group_tok_start = p->group_tok_start;
    A.group_row_start = p->group_row_start;
    A.group_row_src = p->group_row_src;
    A.group_rows = p->group_rows;
    A.seg_rows = p->seg_rows;
    A.dense = p->dense_tiles;
    A.tail = p->tail_items;
    A.info = info;
    const size_t smem = small_plan_smem(A.np, (int)n, k_cap);
    {
      std::lock_guard<std::mutex> lk(g_small_attr_mu);
      int dev = p->device & 63;
      if (!g_small_attr[dev]) {
        L3_CUDA_TRY(cudaFuncSetAttribute(k_plan_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)small_plan_smem(SMALL_PLAN_MAX_TOKENS,
                                                              SMALL_PLAN_MAX_TOKENS,
                                                              MAX_DT_BUCKETS - 1)));
        g_small_attr[dev] = true;
      }
    }
    {
      LaunchTimer t("plan_small", s);
      k_plan_small<<<1, SMALL_THREADS, smem, s>>>(A);
    }
    {
      LaunchTimer t("plan_validate", s);
      k_validate_offsets<<<blocks_for(vocab, 256), 256, 0, s>>>(offsets, vocab, p->dims.v,
                                                                p->dims.k, info);
    }
    return finish_plan(p, info, n, s);
  }

  L3_CUDA_TRY(cudaMemsetAsync(info, 0, 64 * sizeof(int32_t), s));
  if (n == 0) {
    // (with tokens the first histogram pass checks the offsets)
    LaunchTimer t("plan_validate", s);
    k_validate_offsets<<<blocks_for(vocab, 256), 256, 0, s>>>(offsets, vocab, p->dims.v, p->dims.k,
                                                              info);
  }
  if (n > 0) {
    // number of radix digits that cover IDs 0..vocab-1
    int bits = 1;
    while (bits < 31 && ((int64_t)1 << bits) < vocab) ++bits;
    int passes = (bits + RADIX_BITS - 1) / RADIX_BITS;
    // ping-pong so that the last pass lands in the plan's arrays
    int32_t *kbuf[2], *vbuf[2];
    if (passes % 2 == 1) {
      kbuf[0] = keys_tmp; vbuf[0] = vals_tmp;      // (unused as input of pass 0)
      kbuf[1] = p->sorted_ids; vbuf[1] = p->perm;
    } else {
      kbuf[0] = p->sorted_ids; vbuf[0] = p->perm;
      kbuf[1] = keys_tmp; vbuf[1] = vals_tmp;
    }
    const int32_t *kin = ids;
    const int32_t *vin = nullptr;
    for (int pass = 0; pass < passes; ++pass) {
      int shift = pass * RADIX_BITS;
      int32_t *kout = kbuf[(pass + 1) % 2];
      int32_t *vout = vbuf[(pass + 1) % 2];
      {
        LaunchTimer t("plan_radix_hist", s);
        k_radix_hist<<<(int)n_tiles, SORT_THREADS, 0, s>>>(
            kin, n, shift, hist, (int)n_tiles, pass == 0 ? vocab : 0, info,
            pass == 0 ? offsets : nullptr, p->dims.v, p->dims.k);
      }
      const int raw = n_tiles <= FUSED_SCAN_TILES;
      if (!raw) scan_multi({{hist, hist, RADIX * n_tiles, nullptr}}, s);
      {
        LaunchTimer t("plan_radix_scatter", s);
        k_radix_scatter<<<(int)n_tiles, SORT_THREADS, 0, s>>>(
            kin, vin, kout, vout, n, shift, hist, (int)n_tiles, raw,
            pass == passes - 1 ? p->inv_perm : nullptr);
      }
      kin = kout;
      vin = vout;
    }
    {
      LaunchTimer t("plan_group_scan", s);
      k_group_scan<<<1, SCAN_THREADS, 0, s>>>(p->sorted_ids, n, offsets, vocab, p->group_ids,
                                              p->group_tok_start, p->group_row_start,
                                              p->group_rows, info);
    }
    const int n_buckets = N_CLASSES * (k_cap + 1);
    L3_CUDA_TRY(cudaMemsetAsync(dcount, 0, n_buckets * sizeof(int32_t), s));
    L3_CUDA_TRY(cudaMemsetAsync(tcount, 0, (k_cap + 1) * sizeof(int32_t), s));
    {
      LaunchTimer t("plan_item_counts", s);
      k_item_counts<<<blocks_for(cap, 256), 256, 0, s>>>(p->group_tok_start, p->group_rows, n,
                                                         dense_min_tokens, dense_min_rows,
                                                         dense_max_rows, tiles, tails, dcount,
                                                         tcount, k_cap, info);
    }
    // three independent scans in one launch: d_t over groups (segment row
    // offsets), dense tiles over d_t buckets, tail items over (class, d_t) buckets
    scan_multi({{p->group_rows, p->seg_rows, n, &info[INFO_ROWS], &info[INFO_G]},
                {tcount, tcursor, k_cap + 1, &info[INFO_TILES]},
                {dcount, dcursor, n_buckets, &info[INFO_TAILS]}},
               s);
    k_class_starts<<<1, 32, 0, s>>>(dcursor, k_cap, info);
    // keep each group's row in the full table; a staged plan addresses the
    // group's rows where the staging copy puts them, at seg_rows[g]
    L3_CUDA_TRY(cudaMemcpyAsync(p->group_row_src, p->group_row_start, cap * sizeof(int32_t),
                                cudaMemcpyDeviceToDevice, s));
    if (p->staged)
      L3_CUDA_TRY(cudaMemcpyAsync(p->group_row_start, p->seg_rows, cap * sizeof(int32_t),
                                  cudaMemcpyDeviceToDevice, s));
    {
      LaunchTimer t("plan_item_fill", s);
      k_item_fill<<<blocks_for(n, 256), 256, 0, s>>>(p->group_tok_start, p->group_row_start,
                                                     p->group_rows, p->perm, tiles, tcursor,
                                                     tails, dcursor, k_cap, n, p->dense_tiles,
                                                     p->tail_items, info);
    }
  } else {
    L3_CUDA_TRY(cudaMemsetAsync(p->group_tok_start, 0, sizeof(int32_t), s));
    L3_CUDA_TRY(cudaMemsetAsync(p->seg_rows, 0, sizeof(int32_t), s));
  }
  return finish_plan(p, info, n, s);
}

// read the info block back (the path's one host round trip) and fill the
// plan's host-side counts
l3_status finish_plan(l3_plan_s *p, const int32_t *info, int64_t n, cudaStream_t s) {
  L3_CUDA_TRY(cudaGetLastError());

  int32_t host_info[INFO_SLOTS];
  L3_CUDA_TRY(cudaMemcpyAsync(host_info, info, sizeof host_info, cudaMemcpyDeviceToHost, s));
  L3_CUDA_TRY(cudaStreamSynchronize(s));
  if (host_info[INFO_ERR] & DEV_ERR_BAD_OFFSETS) {
    set_error("offsets invalid: need offsets[0] = 0, offsets[vocab] = v and 1 <= d_t <= k");
    return L3_ERR_BAD_OFFSETS;
  }
  if (host_info[INFO_ERR] & DEV_ERR_TOKEN_RANGE) {
    set_error("a token id is outside [0, vocab)");
    return L3_ERR_TOKEN_RANGE;
  }
  p->n_groups = host_info[INFO_G];
  p->n_dense_tiles = host_info[INFO_TILES];
  p->n_dense_small = host_info[INFO_DENSE_SMALL];
  p->n_skinny_big = host_info[INFO_SKINNY_BIG];
  p->n_skinny_small = host_info[INFO_SKINNY_SMALL];
  p->n_tail_items = host_info[INFO_TAILS];
  p->unique_rows = host_info[INFO_ROWS];
  p->unique_rows_multi = host_info[INFO_ROWS_MULTI];
  p->n_dense_groups = host_info[INFO_DENSE_GROUPS];
  p->max_group_tokens = host_info[INFO_MAX_TOKENS];
  for (int c = 0; c <= N_CLASSES; ++c)
    p->tail_class_start[c] = n > 0 ? host_info[INFO_CLS + c] : 0;
  for (int c = 0; c < N_CLASSES; ++c)
    p->tail_class_split[c] = n > 0 ? host_info[INFO_SPLIT + c] : 0;
  return L3_OK;
}

l3_status launch_stage_rows(const l3_plan_s *p, const void *W_K, const void *W_V, void *K_staged,
                            void *V_staged, cudaStream_t s) {
  if (p->n_groups == 0) return L3_OK;
  const size_t el = p->dims.dtype == L3_BF16 ? 2 : 4;
  const int k_vecs = (int)(p->dims.d_in * el / 16), v_vecs = (int)(p->dims.d_emb * el / 16);
  LaunchTimer t("stage_rows", s);
  k_stage_rows<<<(unsigned)p->n_groups, 256, 0, s>>>(
      p->group_row_src, p->seg_rows, p->group_rows, reinterpret_cast<const uint4 *>(W_K),
      reinterpret_cast<const uint4 *>(W_V), reinterpret_cast<uint4 *>(K_staged),
      reinterpret_cast<uint4 *>(V_staged), k_vecs, v_vecs);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

// Stable LSD radix sort of int32 keys in [0, 2^bits) (pairs: vals_in, or the
// input index when NULL), for other parts of the library. Scratch: see
// radix_sort_scratch_ints. The result lands in keys_out / vals_out; neither
// may alias the inputs.
size_t radix_sort_scratch_ints(int64_t n) {
  const int64_t tiles = std::max<int64_t>(1, (n + SORT_TILE - 1) / SORT_TILE);
  return 2 * (size_t)n + (size_t)RADIX * tiles + 1;
}

l3_status radix_sort_pairs(const int32_t *keys_in, const int32_t *vals_in, int64_t n, int bits,
                           int32_t *keys_out, int32_t *vals_out, int32_t *scratch,
                           cudaStream_t s) {
  if (n == 0) return L3_OK;
  const int64_t n_tiles = std::max<int64_t>(1, (n + SORT_TILE - 1) / SORT_TILE);
  int32_t *keys_tmp = scratch, *vals_tmp = scratch + n, *hist = scratch + 2 * n;
  const int passes = std::max(1, (bits + RADIX_BITS - 1) / RADIX_BITS);
  int32_t *kbuf[2], *vbuf[2];
  if (passes % 2 == 1) {
    kbuf[0] = keys_tmp; vbuf[0] = vals_tmp;
    kbuf[1] = keys_out; vbuf[1] = vals_out;
  } else {
    kbuf[0] = keys_out; vbuf[0] = vals_out;
    kbuf[1] = keys_tmp; vbuf[1] = vals_tmp;
  }
  const int32_t *kin = keys_in, *vin = vals_in;
  for (int pass = 0; pass < passes; ++pass) {
    const int shift = pass * RADIX_BITS;
    int32_t *kout = kbuf[(pass + 1) % 2], *vout = vbuf[(pass + 1) % 2];
    k_radix_hist<<<(int)n_tiles, SORT_THREADS, 0, s>>>(kin, n, shift, hist, (int)n_tiles, 0,
                                                      nullptr, nullptr, 0, 0);
    ScanJobs jobs{};
    jobs.job[0] = ScanJob{hist, hist, RADIX * n_tiles, nullptr};
    k_scan_multi<<<1, SCAN_THREADS, 0, s>>>(jobs);
    k_radix_scatter<<<(int)n_tiles, SORT_THREADS, 0, s>>>(kin, vin, kout, vout, n, shift, hist,
                                                         (int)n_tiles, 0, nullptr);
    kin = kout;
    vin = vout;
  }
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

// in-place exclusive scan of data[0..n) (data has n + 1 entries; data[n]
// receives the total, and *total too when given), one CTA
l3_status exclusive_scan(int32_t *data, int64_t n, int32_t *total, cudaStream_t s) {
  ScanJobs jobs{};
  jobs.job[0] = ScanJob{data, data, n, total};
  k_scan_multi<<<1, SCAN_THREADS, 0, s>>>(jobs);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

}  // namespace l3

// ---------------------------------------------------------------------------
// Allocation-free stable sort by token ID
//
// Some callers cannot allocate device memory at the point where they sort a
// batch: a serving engine or framework allocator that has reserved nearly
// all of HBM up front (a cudaMalloc would fail or fight it), or a latency-
// critical loop that cannot afford the device-wide synchronisation that
// cudaMalloc / cudaFree may imply. l3_sort_tokens_noalloc gives them the
// plan's stable sort with its temporaries in the fixed array below instead of
// in memory it allocates. The array lives in every GPU that loads this
// library, until the process exits.
// ---------------------------------------------------------------------------
namespace l3 {
namespace {

constexpr int64_t NOALLOC_MAX_TOKENS = 65536;
constexpr int64_t NOALLOC_TILES = (NOALLOC_MAX_TOKENS + SORT_TILE - 1) / SORT_TILE;
// ping-pong keys and values, then the (digit, tile) histogram plus its total
constexpr int64_t NOALLOC_SCRATCH_INTS = 2 * NOALLOC_MAX_TOKENS + RADIX * NOALLOC_TILES + 64;

static __device__ __align__(256) int32_t g_sort_scratch[NOALLOC_SCRATCH_INTS];

__global__ void k_inverse_perm(const int32_t *__restrict__ perm, int64_t n,
                               int32_t *__restrict__ inv_perm) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i < n) inv_perm[perm[i]] = (int32_t)i;
}

std::mutex g_scratch_mu;
int32_t *g_scratch_ptr[64] = {};  // device address of g_sort_scratch, per device

}  // namespace
}  // namespace l3

extern "C" l3_status l3_sort_tokens_noalloc(const int32_t *token_ids, int64_t n_tokens,
                                            int64_t vocab, int32_t *perm, int32_t *inv_perm,
                                            int32_t *sorted_ids, void *stream) {
  using namespace l3;
  set_error("");
  if (n_tokens < 0 || n_tokens > NOALLOC_MAX_TOKENS) {
    set_error("l3_sort_tokens_noalloc: n_tokens must be in [0, 65536] (fixed scratch size)");
    return L3_ERR_INVALID_ARG;
  }
  if (vocab < 1 || vocab > INT32_MAX - 1) {
    set_error("l3_sort_tokens_noalloc: vocab must be in [1, 2^31 - 2]");
    return L3_ERR_INVALID_ARG;
  }
  if (n_tokens == 0) return L3_OK;
  if (!token_ids || !perm || !inv_perm || !sorted_ids) {
    set_error("l3_sort_tokens_noalloc: a pointer is NULL");
    return L3_ERR_INVALID_ARG;
  }
  {
    // the scatter of one pass reads token_ids (or the previous pass's keys)
    // while other CTAs write the outputs, so no two of the four buffers may
    // share a byte
    const uintptr_t bytes = (uintptr_t)n_tokens * sizeof(int32_t);
    const uintptr_t lo[4] = {reinterpret_cast<uintptr_t>(token_ids),
                             reinterpret_cast<uintptr_t>(perm),
                             reinterpret_cast<uintptr_t>(inv_perm),
                             reinterpret_cast<uintptr_t>(sorted_ids)};
    for (int i = 0; i < 4; ++i)
      for (int j = i + 1; j < 4; ++j)
        if (lo[i] < lo[j] + bytes && lo[j] < lo[i] + bytes) {
          set_error("l3_sort_tokens_noalloc: token_ids, perm, inv_perm and sorted_ids must not "
                    "overlap");
          return L3_ERR_INVALID_ARG;
        }
  }
  int dev = -1;
  L3_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) {
    set_error("l3_sort_tokens_noalloc: device ordinal out of range");
    return L3_ERR_INVALID_ARG;
  }
  int32_t *scratch = nullptr;
  {
    // once per device, with that device current: the host-side name of the
    // array is not a device address, so ask the runtime for the real one
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
      void *ptr = nullptr;
      L3_CUDA_TRY(cudaGetSymbolAddress(&ptr, g_sort_scratch));
      g_scratch_ptr[dev] = reinterpret_cast<int32_t *>(ptr);
    }
    scratch = g_scratch_ptr[dev];
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = n_tokens;
  const int64_t n_tiles = (n + SORT_TILE - 1) / SORT_TILE;
  int32_t *keys_tmp = scratch;
  int32_t *vals_tmp = scratch + NOALLOC_MAX_TOKENS;
  int32_t *hist = scratch + 2 * NOALLOC_MAX_TOKENS;  // RADIX * n_tiles + 1 entries

  int bits = 1;
  while (bits < 31 && ((int64_t)1 << bits) < vocab) ++bits;
  const int passes = (bits + RADIX_BITS - 1) / RADIX_BITS;
  int32_t *kbuf[2], *vbuf[2];
  if (passes % 2 == 1) {
    kbuf[0] = keys_tmp; vbuf[0] = vals_tmp;
    kbuf[1] = sorted_ids; vbuf[1] = perm;
  } else {
    kbuf[0] = sorted_ids; vbuf[0] = perm;
    kbuf[1] = keys_tmp; vbuf[1] = vals_tmp;
  }
  // Every scratch word that is read is written earlier in the same call (the
  // histogram kernel writes each (digit, tile) count, the scan and the
  // scatter write all they later read), so nothing needs clearing between
  // calls.
  const int32_t *kin = token_ids;
  const int32_t *vin = nullptr;
  for (int pass = 0; pass < passes; ++pass) {
    int shift = pass * RADIX_BITS;
    int32_t *kout = kbuf[(pass + 1) % 2];
    int32_t *vout = vbuf[(pass + 1) % 2];
    k_radix_hist<<<(int)n_tiles, SORT_THREADS, 0, s>>>(kin, n, shift, hist, (int)n_tiles, 0,
                                                      nullptr, nullptr, 0, 0);
    {
      ScanJobs jobs{};
      jobs.job[0] = ScanJob{hist, hist, RADIX * n_tiles, nullptr};
      k_scan_multi<<<1, SCAN_THREADS, 0, s>>>(jobs);
    }
    k_radix_scatter<<<(int)n_tiles, SORT_THREADS, 0, s>>>(kin, vin, kout, vout, n, shift, hist,
                                                         (int)n_tiles, 0, nullptr);
    kin = kout;
    vin = vout;
  }
  k_inverse_perm<<<(int)((n + 255) / 256), 256, 0, s>>>(perm, n, inv_perm);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}
