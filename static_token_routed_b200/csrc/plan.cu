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

constexpr int RADIX_BITS = 8;
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

__host__ __device__ __forceinline__ int token_class(int nt) {
  return nt <= 1 ? 0 : nt == 2 ? 1 : nt <= 4 ? 2 : 3;
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
  INFO_SLOTS
};

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
__global__ void __launch_bounds__(SORT_THREADS)
    k_radix_hist(const int32_t *__restrict__ keys, int64_t n, int shift, int32_t *__restrict__ hist,
                 int n_tiles, int64_t vocab, int32_t *info) {
  __shared__ int32_t cnt[RADIX];
  for (int i = threadIdx.x; i < RADIX; i += SORT_THREADS) cnt[i] = 0;
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
// digit-major order). Each warp owns a contiguous span of the tile and walks
// it in order, ranking equal digits with __match_any_sync, so the output keeps
// input order among equal digits.
__global__ void __launch_bounds__(SORT_THREADS)
    k_radix_scatter(const int32_t *__restrict__ keys_in, const int32_t *__restrict__ vals_in,
                    int32_t *__restrict__ keys_out, int32_t *__restrict__ vals_out, int64_t n,
                    int shift, const int32_t *__restrict__ offs, int n_tiles) {
  __shared__ int32_t whist[SORT_WARPS][RADIX];
  __shared__ int32_t dbase[RADIX];
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
  for (int d = threadIdx.x; d < RADIX; d += SORT_THREADS) {
    int32_t run = 0;
#pragma unroll
    for (int w = 0; w < SORT_WARPS; ++w) {
      int32_t c = whist[w][d];
      whist[w][d] = run;
      run += c;
    }
    dbase[d] = offs[(int64_t)d * n_tiles + blockIdx.x];
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < SORT_ITEMS; ++it) {
    int64_t i = base + it * 32 + lane;
    if (i < n) {
      int d = digit[it];
      int32_t pos = dbase[d] + whist[warp][d] + rank[it];
      keys_out[pos] = key[it];
      vals_out[pos] = vals_in ? vals_in[i] : (int32_t)i;
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

// head[i] = 1 where a new ID starts in sorted order; inv_perm[perm[i]] = i.
__global__ void k_group_heads(const int32_t *__restrict__ sorted, const int32_t *__restrict__ perm,
                              int64_t n, int32_t *__restrict__ head, int32_t *__restrict__ inv_perm) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n) return;
  head[i] = (i == 0 || sorted[i] != sorted[i - 1]) ? 1 : 0;
  inv_perm[perm[i]] = (int32_t)i;
}

__global__ void k_group_fill(const int32_t *__restrict__ sorted, const int32_t *__restrict__ head,
                             const int32_t *__restrict__ gpos, int64_t n,
                             const int32_t *__restrict__ offsets, int64_t vocab,
                             int32_t *__restrict__ group_ids, int32_t *__restrict__ group_tok_start,
                             int32_t *__restrict__ group_row_start, int32_t *__restrict__ group_rows,
                             const int32_t *info) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i == 0) group_tok_start[info[INFO_G]] = (int32_t)n;
  if (i >= n || !head[i]) return;
  int32_t g = gpos[i];
  int32_t id = sorted[i];
  group_ids[g] = id;
  group_tok_start[g] = (int32_t)i;
  bool ok = id >= 0 && id < vocab;
  int32_t r0 = ok ? offsets[id] : 0;
  group_row_start[g] = r0;
  group_rows[g] = ok ? offsets[id + 1] - r0 : 0;
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
      // dense tiles are listed largest d_t first (bucket k_cap - d_t): the
      // longest CTAs start first, and the d_t > DENSE_SMALL_ROWS tiles come
      // before the others
      atomicAdd(&tcount[k_cap - min(rows, k_cap)], nt);
    } else {
      nl = (c + TAIL_TOKENS - 1) / TAIL_TOKENS;
    }
    if (rows > 1) atomicAdd(&info[INFO_ROWS_MULTI], rows);
    atomicMax(&info[INFO_MAX_TOKENS], c);
    // tail items are listed by token-count class, then largest d_t first:
    // bucket class * (k_cap + 1) + (k_cap - d_t), so an ascending scan gives
    // the order
    if (nl > 0) {
      const int db = k_cap - min(rows, k_cap);
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
    const int32_t pos = atomicAdd(&tcursor[k_cap - min(rows, k_cap)], tiles[g]);
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
    const int bucket = token_class(it.nt) * (k_cap + 1) + (k_cap - min(rows, k_cap));
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
  ints += 2 * ((size_t)n + 1);           // head flags, group positions
  ints += 2 * ((size_t)n + 1);           // dense tiles and tail items per group
  ints += 64;                            // info block
  ints += 2 * (N_CLASSES * MAX_DT_BUCKETS + 1);  // tail items per bucket, and their cursors
  ints += 2 * (MAX_DT_BUCKETS + 1);      // dense tiles per d_t bucket, and their cursors
  return ints * sizeof(int32_t) + 256;
}

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
  int32_t *head = sp;
  sp += cap;
  int32_t *gpos = sp;
  sp += cap;
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

  L3_CUDA_TRY(cudaMemsetAsync(info, 0, 64 * sizeof(int32_t), s));
  {
    LaunchTimer t("plan_validate", s);
    k_validate_offsets<<<blocks_for(vocab, 256), 256, 0, s>>>(offsets, vocab, p->dims.v, p->dims.k,
                                                              info);
  }
  if (n > 0) {
    // number of 8-bit digits that cover IDs 0..vocab-1
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
        k_radix_hist<<<(int)n_tiles, SORT_THREADS, 0, s>>>(kin, n, shift, hist, (int)n_tiles,
                                                          pass == 0 ? vocab : 0, info);
      }
      scan_multi({{hist, hist, RADIX * n_tiles, nullptr}}, s);
      {
        LaunchTimer t("plan_radix_scatter", s);
        k_radix_scatter<<<(int)n_tiles, SORT_THREADS, 0, s>>>(kin, vin, kout, vout, n, shift, hist,
                                                             (int)n_tiles);
      }
      kin = kout;
      vin = vout;
    }
    {
      LaunchTimer t("plan_group_heads", s);
      k_group_heads<<<blocks_for(n, 256), 256, 0, s>>>(p->sorted_ids, p->perm, n, head,
                                                       p->inv_perm);
    }
    scan_multi({{head, gpos, n, &info[INFO_G]}}, s);
    L3_CUDA_TRY(cudaMemsetAsync(p->group_rows, 0, cap * sizeof(int32_t), s));
    {
      LaunchTimer t("plan_group_fill", s);
      k_group_fill<<<blocks_for(n, 256), 256, 0, s>>>(p->sorted_ids, head, gpos, n, offsets, vocab,
                                                      p->group_ids, p->group_tok_start,
                                                      p->group_row_start, p->group_rows, info);
    }
    // groups with enough tokens and rows go to the tensor-core attention kernel
    int dense_min_tokens = 0, dense_min_rows = 0, dense_max_rows = 0;
    if (dense_attention_supported(p->dims)) {
      dense_min_tokens = DENSE_MIN_TOKENS;
      dense_min_rows = DENSE_MIN_ROWS;
      dense_max_rows = dense_attention_max_rows();
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
    scan_multi({{p->group_rows, p->seg_rows, n, &info[INFO_ROWS]},
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
                                                      nullptr);
    {
      ScanJobs jobs{};
      jobs.job[0] = ScanJob{hist, hist, RADIX * n_tiles, nullptr};
      k_scan_multi<<<1, SCAN_THREADS, 0, s>>>(jobs);
    }
    k_radix_scatter<<<(int)n_tiles, SORT_THREADS, 0, s>>>(kin, vin, kout, vout, n, shift, hist,
                                                         (int)n_tiles);
    kin = kout;
    vin = vout;
  }
  k_inverse_perm<<<(int)((n + 255) / 256), 256, 0, s>>>(perm, n, inv_perm);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}
