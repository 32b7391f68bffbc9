// C ABI of the L³ forward library: argument checks, the plan object and its
// device memory, launch order of the forward kernels, errors and profiling.
//
// The forward pass (kimjy99 review, Method, eq. L³) runs as:
//   attention  a[n] = V_t^T softmax(K_t x_n)   (gather-attention kernels)
//   up + LN    h = LayerNorm(W_up a)           (GEMM with LayerNorm epilogue)
//   mix        y = W_mix[:, :d_up] h + W_mix[:, d_up:] x   (two accumulated K-ranges)
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "l3_internal.cuh"

namespace l3 {

size_t attn_tail_smem_bytes(const l3_dims_t &d);

namespace {
thread_local std::string g_error;

// ---- profiling registry ----
struct Record {
  const char *name;
  cudaStream_t stream;
  cudaEvent_t start, end;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
bool g_prof_plan = false;  // also time the plan's kernels
std::vector<Record> g_records;
std::vector<cudaEvent_t> g_free_events;

cudaEvent_t take_event() {
  if (!g_free_events.empty()) {
    cudaEvent_t e = g_free_events.back();
    g_free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}


// Per-device helper streams and events that let the attention kernels run
// side by side: the tensor-core dense kernel on the caller's stream, the
// CUDA-core tail classes spread over the helper streams. They write disjoint
// rows of a, and the tails' small CTAs fit next to a dense CTA on an SM.
constexpr int N_AUX = 3;
struct Aux {
  std::mutex mu;
  cudaStream_t stream[N_AUX] = {};
  cudaEvent_t fork = nullptr, join[N_AUX] = {};
};
Aux g_aux[64];

l3_status aux_for(int device, Aux **out) {
  Aux &a = g_aux[device & 63];
  std::lock_guard<std::mutex> lk(a.mu);
  if (!a.stream[0]) {
    // highest priority: the block scheduler hands freed SM slots to the tail
    // attention's short CTAs before the next dense CTA, so the two overlap
    // instead of the tails waiting behind the dense launch (1.84 -> 1.69 ms per
    // paper_shaped batch)
    int lowest = 0, highest = 0;
    L3_CUDA_TRY(cudaDeviceGetStreamPriorityRange(&lowest, &highest));
    for (int i = 0; i < N_AUX; ++i) {
      L3_CUDA_TRY(cudaStreamCreateWithPriority(&a.stream[i], cudaStreamNonBlocking, highest));
      L3_CUDA_TRY(cudaEventCreateWithFlags(&a.join[i], cudaEventDisableTiming));
    }
    L3_CUDA_TRY(cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming));
  }
  *out = &a;
  return L3_OK;
}

}  // namespace

// Plan memory cache. A destroyed plan's block goes back to a per-process list
// with an event recorded on the stream that last used it; a new plan takes a
// cached block on its device that is large enough and whose event has
// completed, so a plan per batch costs no allocator call after warm-up, and a
// plan built on one stream while an earlier forward still runs on another
// never waits for it or grows the pool. The backward pass takes its scratch
// from the same cache.
namespace {
struct CachedBlock {
  void *ptr;
  size_t bytes;
  int device;
  cudaEvent_t ready;
};
std::mutex g_cache_mu;
std::vector<CachedBlock> g_cache;
constexpr size_t CACHE_MAX_BLOCKS = 4;
}  // namespace

// returns a cached block of at least `bytes` on `device` (and its size), or nullptr
void *cache_take(int device, size_t bytes, size_t *got) {
  std::lock_guard<std::mutex> lk(g_cache_mu);
  int best = -1;
  for (int i = 0; i < (int)g_cache.size(); ++i) {
    const CachedBlock &c = g_cache[i];
    if (c.device != device || c.bytes < bytes) continue;
    if (cudaEventQuery(c.ready) != cudaSuccess) continue;  // still in use on the GPU
    if (best < 0 || c.bytes < g_cache[best].bytes) best = i;
  }
  if (best < 0) return nullptr;
  void *p = g_cache[best].ptr;
  *got = g_cache[best].bytes;
  cudaEventDestroy(g_cache[best].ready);
  g_cache.erase(g_cache.begin() + best);
  return p;
}

void cache_give(void *ptr, size_t bytes, int device, cudaStream_t s) {
  cudaEvent_t ev = nullptr;
  if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventRecord(ev, s) != cudaSuccess) {
    if (ev) cudaEventDestroy(ev);
    cudaStreamSynchronize(s);
    cudaFree(ptr);
    return;
  }
  std::lock_guard<std::mutex> lk(g_cache_mu);
  g_cache.push_back(CachedBlock{ptr, bytes, device, ev});
  while (g_cache.size() > CACHE_MAX_BLOCKS) {
    // drop the oldest block once its last user has finished
    CachedBlock old = g_cache.front();
    g_cache.erase(g_cache.begin());
    cudaEventSynchronize(old.ready);
    cudaEventDestroy(old.ready);
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != old.device) cudaSetDevice(old.device);
    cudaFree(old.ptr);
    if (cur != old.device) cudaSetDevice(cur);
  }
}

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

l3_status check_dims(const l3_dims_t *d) {
  if (!d) {
    set_error("dims is NULL");
    return L3_ERR_INVALID_ARG;
  }
  if (d->vocab < 1 || d->v < d->vocab || d->k < 1 || d->d_in < 1 || d->d_emb < 1 ||
      d->d_up < 1 || d->d_out < 1) {
    set_error("dims: need vocab >= 1, v >= vocab, k >= 1 and positive layer widths");
    return L3_ERR_INVALID_ARG;
  }
  if (d->vocab > INT32_MAX - 1 || d->v > INT32_MAX) {
    set_error("dims: vocab and v must fit int32");
    return L3_ERR_UNSUPPORTED;
  }
  if (d->dtype != L3_BF16 && d->dtype != L3_FP32) {
    set_error("dims.dtype must be L3_BF16 or L3_FP32");
    return L3_ERR_INVALID_ARG;
  }
  const int64_t mult = d->dtype == L3_BF16 ? 16 : 4;
  if (d->d_in % mult || d->d_emb % mult || d->d_up % mult || d->d_out % mult) {
    set_error(d->dtype == L3_BF16 ? "dims: bf16 widths must be multiples of 16"
                                  : "dims: fp32 widths must be multiples of 4");
    return L3_ERR_UNSUPPORTED;
  }
  if (d->k > 1024 || d->d_in > 8192 || d->d_emb > 512 || d->d_up > 4096 || d->d_out > 65536) {
    set_error("dims: supported k <= 1024, d_in <= 8192, d_emb <= 512, d_up <= 4096");
    return L3_ERR_UNSUPPORTED;
  }
  if (!(d->ln_eps >= 0.0f)) {
    set_error("dims.ln_eps must be >= 0");
    return L3_ERR_INVALID_ARG;
  }
  return L3_OK;
}

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

void set_error(const std::string &msg) { g_error = msg; }

l3_status cuda_fail(cudaError_t e, const char *what) {
  g_error = std::string("CUDA error in ") + what + ": " + cudaGetErrorString(e);
  return e == cudaErrorMemoryAllocation ? L3_ERR_OOM : L3_ERR_CUDA;
}

LaunchTimer::LaunchTimer(const char *n, cudaStream_t s) : name(n), stream(s), slot(-1) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on || (!g_prof_plan && std::strncmp(n, "plan", 4) == 0)) return;
  Record r{name, s, take_event(), take_event()};
  cudaEventRecord(r.start, s);
  slot = (int)g_records.size();
  g_records.push_back(r);
}

LaunchTimer::~LaunchTimer() {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (slot < (int)g_records.size()) cudaEventRecord(g_records[slot].end, stream);
}

}  // namespace l3

using namespace l3;

extern "C" {

const char *l3_last_error(void) { return g_error.c_str(); }

static l3_status plan_impl(const int32_t *token_ids, int64_t n_tokens, const int32_t *offsets,
                           const l3_dims_t *dims, void *stream, l3_plan_t *out, bool staged);

l3_status l3_plan(const int32_t *token_ids, int64_t n_tokens, const int32_t *offsets,
                  const l3_dims_t *dims, void *stream, l3_plan_t *out) {
  return plan_impl(token_ids, n_tokens, offsets, dims, stream, out, false);
}

l3_status l3_plan_staged(const int32_t *token_ids, int64_t n_tokens, const int32_t *offsets,
                         const l3_dims_t *dims, void *stream, l3_plan_t *out) {
  return plan_impl(token_ids, n_tokens, offsets, dims, stream, out, true);
}

l3_status l3_stage_rows(l3_plan_t p, const void *W_K, const void *W_V, void *W_K_staged,
                        void *W_V_staged, void *stream) {
  g_error.clear();
  if (!p || !p->staged) {
    set_error(p ? "l3_stage_rows needs a plan from l3_plan_staged" : "plan is NULL");
    return L3_ERR_INVALID_ARG;
  }
  if (p->n_groups == 0) return L3_OK;
  for (const void *q : {W_K, W_V, (const void *)W_K_staged, (const void *)W_V_staged}) {
    if (!q) {
      set_error("a table pointer is NULL");
      return L3_ERR_INVALID_ARG;
    }
    if (reinterpret_cast<uintptr_t>(q) & 15u) {
      set_error("table pointers must be 16-byte aligned");
      return L3_ERR_INVALID_ARG;
    }
  }
  int dev = -1;
  L3_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != p->device) {
    set_error("l3_stage_rows called on a different device than l3_plan_staged");
    return L3_ERR_INVALID_ARG;
  }
  return launch_stage_rows(p, W_K, W_V, W_K_staged, W_V_staged,
                           reinterpret_cast<cudaStream_t>(stream));
}

static l3_status plan_impl(const int32_t *token_ids, int64_t n_tokens, const int32_t *offsets,
                           const l3_dims_t *dims, void *stream, l3_plan_t *out, bool staged) {
  g_error.clear();
  if (!out) {
    set_error("out is NULL");
    return L3_ERR_INVALID_ARG;
  }
  *out = nullptr;
  l3_status st = check_dims(dims);
  if (st != L3_OK) return st;
  if (n_tokens < 0 || n_tokens > (int64_t)INT32_MAX / 2) {
    set_error("n_tokens out of range");
    return L3_ERR_INVALID_ARG;
  }
  if (!offsets || (n_tokens > 0 && !token_ids)) {
    set_error("token_ids / offsets is NULL");
    return L3_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(token_ids) & 3u) || (reinterpret_cast<uintptr_t>(offsets) & 3u)) {
    set_error("token_ids / offsets must be 4-byte aligned");
    return L3_ERR_INVALID_ARG;
  }
  if (attn_tail_smem_bytes(*dims) > 220 * 1024) {
    set_error("dims: d_in and k too large for the attention kernel's shared memory");
    return L3_ERR_UNSUPPORTED;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto *p = new l3_plan_s();
  p->staged = staged;
  p->dims = *dims;
  p->n_tokens = n_tokens;
  p->stream = s;
  L3_CUDA_TRY(cudaGetDevice(&p->device));

  const int64_t n = n_tokens, cap = n + 1;
  const size_t el = dims->dtype == L3_BF16 ? 2 : 4;
  p->tc_gemm = tc_gemm_supported(*dims);
  size_t sizes[] = {
      align256(n * 4),                                            // perm
      align256(n * 4),                                            // inv_perm
      align256(n * 4),                                            // sorted_ids
      align256(cap * 4),                                          // group_ids
      align256(cap * 4),                                          // group_tok_start
      align256(cap * 4),                                          // group_row_start
      align256(cap * 4),                                          // group_row_src
      align256(cap * 4),                                          // group_rows
      align256(cap * 4),                                          // seg_rows
      align256((n / DENSE_TILE_M + cap) * sizeof(DenseTile)),     // dense tiles
      align256((n / TAIL_TOKENS + cap) * sizeof(TailItem)),       // tail items
      align256(64),                                               // device flags
      align256(n * dims->d_emb * el),                             // a
      align256(n * dims->d_up * el),                              // h
      align256(p->tc_gemm ? 0 : n * dims->d_up * 4),              // z (CUDA-core GEMM path)
      align256(plan_scratch_bytes(n)),                            // plan-build scratch
      align256(p->tc_gemm ? dims->d_up * dims->d_emb * 2 : 0),    // fp16 W_up
      align256(p->tc_gemm ? dims->d_out * dims->d_up * 2 : 0),    // fp16 W_mix[:, :d_up] diag(gamma)
      align256(p->tc_gemm ? n * ((dims->d_up + 255) / 256) * 8 : 0),  // (mean, M2) of z per 256 columns
      align256(p->tc_gemm ? 2 * ((dims->d_out + 3) / 4 * 4) * 4 : 0),  // W' 1, W_mix[:, :d_up] beta
  };
  size_t total = 0;
  for (size_t b : sizes) total += b;
  size_t got = 0;
  p->block = cache_take(p->device, total, &got);
  cudaError_t e = cudaSuccess;
  if (p->block) {
    p->block_bytes = got;  // a cached block keeps its size for its next owner
  } else {
    e = cudaMalloc(&p->block, total);
    if (e != cudaSuccess) {
      delete p;
      return cuda_fail(e, "cudaMalloc(plan)");
    }
    p->block_bytes = total;
  }
  char *c = reinterpret_cast<char *>(p->block);
  size_t i = 0;
  auto next = [&](size_t k) {
    char *r = c;
    c += sizes[k];
    return r;
  };
  p->perm = reinterpret_cast<int32_t *>(next(i++));
  p->inv_perm = reinterpret_cast<int32_t *>(next(i++));
  p->sorted_ids = reinterpret_cast<int32_t *>(next(i++));
  p->group_ids = reinterpret_cast<int32_t *>(next(i++));
  p->group_tok_start = reinterpret_cast<int32_t *>(next(i++));
  p->group_row_start = reinterpret_cast<int32_t *>(next(i++));
  p->group_row_src = reinterpret_cast<int32_t *>(next(i++));
  p->group_rows = reinterpret_cast<int32_t *>(next(i++));
  p->seg_rows = reinterpret_cast<int32_t *>(next(i++));
  p->dense_tiles = reinterpret_cast<DenseTile *>(next(i++));
  p->tail_items = reinterpret_cast<TailItem *>(next(i++));
  p->dev_flags = reinterpret_cast<int32_t *>(next(i++));
  p->a_buf = next(i++);
  p->h_buf = next(i++);
  p->z_buf = reinterpret_cast<float *>(next(i++));
  const size_t scratch_idx = i;
  void *scratch = next(i++);
  p->w_up16 = next(i++);
  p->w_mixh16 = next(i++);
  p->ln_stats = reinterpret_cast<float2 *>(next(i++));
  p->mix_ccol = reinterpret_cast<float *>(next(i++));

  st = L3_OK;
  e = cudaMemsetAsync(p->dev_flags, 0, 64, s);
  if (e != cudaSuccess) st = cuda_fail(e, "cudaMemsetAsync(flags)");
  if (st == L3_OK) st = build_plan(p, token_ids, offsets, s, scratch, sizes[scratch_idx]);
  if (st != L3_OK) {
    std::string msg = g_error;
    cache_give(p->block, p->block_bytes, p->device, s);
    delete p;
    g_error = msg;
    return st;
  }
  *out = p;
  return L3_OK;
}

l3_status l3_plan_info(l3_plan_t p, l3_plan_info_t *info) {
  g_error.clear();
  if (!p || !info) {
    set_error("plan / info is NULL");
    return L3_ERR_INVALID_ARG;
  }
  info->n_tokens = p->n_tokens;
  info->n_groups = p->n_groups;
  info->n_dense_groups = p->n_dense_groups;
  info->n_dense_tiles = p->n_dense_tiles;
  info->n_tail_items = p->n_tail_items;
  info->unique_rows = p->unique_rows;
  info->unique_rows_multi = p->unique_rows_multi;
  return L3_OK;
}

l3_status l3_plan_export(l3_plan_t p, int32_t *perm, int32_t *inv_perm, int32_t *sorted_ids,
                         int32_t *group_ids, int32_t *group_tok_start, int32_t *seg_rows,
                         int64_t *G_out, void *stream) {
  g_error.clear();
  if (!p) {
    set_error("plan is NULL");
    return L3_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t n = (size_t)p->n_tokens, G = (size_t)p->n_groups;
  auto cp = [&](int32_t *dst, const int32_t *src, size_t count) -> l3_status {
    if (!dst || count == 0) return L3_OK;
    L3_CUDA_TRY(cudaMemcpyAsync(dst, src, count * 4, cudaMemcpyDeviceToDevice, s));
    return L3_OK;
  };
  l3_status st;
  if ((st = cp(perm, p->perm, n)) != L3_OK) return st;
  if ((st = cp(inv_perm, p->inv_perm, n)) != L3_OK) return st;
  if ((st = cp(sorted_ids, p->sorted_ids, n)) != L3_OK) return st;
  if ((st = cp(group_ids, p->group_ids, G)) != L3_OK) return st;
  if ((st = cp(group_tok_start, p->group_tok_start, G + 1)) != L3_OK) return st;
  if ((st = cp(seg_rows, p->seg_rows, G + 1)) != L3_OK) return st;
  if (G_out) *G_out = (int64_t)G;
  p->stream = s;
  return L3_OK;
}

// Dense attention on the caller's stream: the d_t > 256 tiles of more than
// SKINNY_TOKENS tokens (one CTA per SM, the longest), then every tile of at
// most SKINNY_TOKENS tokens (transposed products, one CTA per SM beside the
// tail kernels), then the other d_t <= 256 tiles. The skinny kernel takes its
// tiles only where there are at least four per SM: with fewer, its launch
// adds a ramp down of its own to the two others' (small_bf16, 271 such
// tiles: 0.266 -> 0.278 ms per batch; dense_stress, 16: 0.837 -> 0.960 ms),
// and the two configurations take all of their tiles.
static l3_status launch_dense_all(const l3_plan_s *p, const void *x, const void *W_K,
                                  const void *W_V, cudaStream_t s) {
  const bool skinny = skinny_attention_supported(p->dims) &&
                      p->n_skinny_big + p->n_skinny_small >= 4 * (int64_t)sm_count(p->device);
  l3_status st = launch_attn_dense(p, x, W_K, W_V, false, skinny, s);
  if (st == L3_OK && skinny) st = launch_attn_skinny(p, x, W_K, W_V, s);
  if (st == L3_OK) st = launch_attn_dense(p, x, W_K, W_V, true, skinny, s);
  return st;
}

l3_status l3_forward(const void *x, l3_plan_t p, const void *W_K, const void *W_V,
                     const void *W_up, const void *ln_gamma, const void *ln_beta,
                     const void *W_mix, void *y, void *stream) {
  g_error.clear();
  if (!p) {
    set_error("plan is NULL");
    return L3_ERR_INVALID_ARG;
  }
  if (p->n_tokens == 0) return L3_OK;
  const void *ptrs[] = {x, W_K, W_V, W_up, ln_gamma, ln_beta, W_mix, y};
  for (const void *q : ptrs) {
    if (!q) {
      set_error("a tensor pointer is NULL");
      return L3_ERR_INVALID_ARG;
    }
    if (!aligned16(q)) {
      set_error("tensor pointers must be 16-byte aligned");
      return L3_ERR_INVALID_ARG;
    }
  }
  int dev = -1;
  L3_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != p->device) {
    set_error("l3_forward called on a different device than l3_plan");
    return L3_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  p->stream = s;
  l3_status st = L3_OK;
  const bool has_big = p->n_dense_tiles > p->n_dense_small;
  const bool has_tail = p->n_tail_items > 0;
  if (has_tail && tail_cls_supported(p->dims)) {
    // fork: dense attention (its launches in turn, see launch_dense_all) on
    // the caller's stream; the fp16 weight copies first on the last helper
    // stream, then the tail classes over the high-priority helper streams,
    // whose short CTAs fill the SM slots the dense CTAs leave; join before
    // W_up. The launches write disjoint rows of a.
    Aux *aux = nullptr;
    if ((st = aux_for(p->device, &aux)) != L3_OK) return st;
    std::lock_guard<std::mutex> lk(aux->mu);
    L3_CUDA_TRY(cudaEventRecord(aux->fork, s));
    for (int i = 0; i < N_AUX; ++i) L3_CUDA_TRY(cudaStreamWaitEvent(aux->stream[i], aux->fork, 0));
    if (st == L3_OK) st = launch_dense_all(p, x, W_K, W_V, s);
    // the weight copies run beside the attention rather than after the tail
    // stream's last launch (paper_shaped: up_z started ~20 us later there)
    if (st == L3_OK && p->tc_gemm)
      st = launch_weights_f16(p, W_up, W_mix, ln_gamma, ln_beta, aux->stream[N_AUX - 1]);
    // next to the big dense configuration (one CTA per SM, streaming K_t)
    // the tails stay on one helper stream: spread over three they take SMs
    // and bandwidth from it (paper_shaped: 1.64 -> 1.72 ms per batch, and
    // 1.43 -> 1.49 beside the skinny kernel); with no such launch they spread
    // over all three (small_bf16: 0.41 -> 0.34 ms)
    if (st == L3_OK) st = launch_attn_tail_cls(p, x, W_K, W_V, aux->stream, has_big ? 1 : N_AUX);
    for (int i = 0; i < N_AUX; ++i) {
      L3_CUDA_TRY(cudaEventRecord(aux->join[i], aux->stream[i]));
      L3_CUDA_TRY(cudaStreamWaitEvent(s, aux->join[i], 0));
    }
  } else if (has_tail) {
    st = launch_attn_tail(p, x, W_K, W_V, s);
    if (st == L3_OK) st = launch_dense_all(p, x, W_K, W_V, s);
    if (st == L3_OK && p->tc_gemm) st = launch_weights_f16(p, W_up, W_mix, ln_gamma, ln_beta, s);
  } else {
    if (st == L3_OK) st = launch_dense_all(p, x, W_K, W_V, s);
    if (st == L3_OK && p->tc_gemm) st = launch_weights_f16(p, W_up, W_mix, ln_gamma, ln_beta, s);
  }
  if (p->tc_gemm) {
    if (st == L3_OK) st = launch_up_z_tc(p, s);
    if (st == L3_OK) st = launch_mix_tc(p, x, W_mix, y, s);
  } else {
    if (st == L3_OK) st = launch_up_ln_simt(p, W_up, ln_gamma, ln_beta, s);
    if (st == L3_OK) st = launch_mix_simt(p, x, W_mix, y, s);
  }
  return st;
}

l3_status l3_forward_status(l3_plan_t p) {
  g_error.clear();
  if (!p) {
    set_error("plan is NULL");
    return L3_ERR_INVALID_ARG;
  }
  int32_t flags[2] = {0, 0};
  L3_CUDA_TRY(cudaMemcpyAsync(flags, p->dev_flags, sizeof flags, cudaMemcpyDeviceToHost, p->stream));
  L3_CUDA_TRY(cudaStreamSynchronize(p->stream));
  if (flags[1] & DEV_ERR_TIMEOUT) {
    set_error("a bounded device-side wait in l3_forward gave up; outputs are incomplete");
    return L3_ERR_TIMEOUT;
  }
  if (flags[1] & DEV_ERR_F16_RANGE) {
    set_error("W_up, W_mix[:, :d_up] diag(ln_gamma) or z = W_up a holds a value outside "
              "fp16's finite range (|v| > 65504), which the bf16 layer's fp16 intermediate "
              "GEMMs cannot represent");
    return L3_ERR_UNSUPPORTED;
  }
  return L3_OK;
}

void l3_plan_destroy(l3_plan_t p) {
  if (!p) return;
  if (p->block) cache_give(p->block, p->block_bytes, p->device, p->stream);
  delete p;
}

void l3_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto &r : g_records) {
    g_free_events.push_back(r.start);
    g_free_events.push_back(r.end);
  }
  g_records.clear();
  g_prof_on = enable != 0;
  g_prof_plan = enable == 1;
}

int l3_profile_read(l3_kernel_time_t *out, int max_entries) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  std::vector<l3_kernel_time_t> acc;
  std::unordered_map<std::string, size_t> index;
  for (auto &r : g_records) {
    if (cudaEventSynchronize(r.end) != cudaSuccess) return -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.start, r.end) != cudaSuccess) return -1;
    auto it = index.find(r.name);
    if (it == index.end()) {
      l3_kernel_time_t k{};
      snprintf(k.name, sizeof k.name, "%s", r.name);
      index[r.name] = acc.size();
      acc.push_back(k);
      it = index.find(r.name);
    }
    acc[it->second].launches += 1;
    acc[it->second].total_ms += ms;
  }
  int n = (int)acc.size();
  for (int i = 0; i < n && i < max_entries; ++i) out[i] = acc[i];
  return n;
}

}  // extern "C"
