// Internal declarations of the L³ library: the plan object, launch helpers
// and the kernels' host-side entry points.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "../../include/l3.h"

namespace l3 {

// ---------------------------------------------------------------------------
// error plumbing
// ---------------------------------------------------------------------------
void set_error(const std::string &msg);
l3_status cuda_fail(cudaError_t e, const char *what);

#define L3_CUDA_TRY(expr)                                   \
  do {                                                      \
    cudaError_t _e = (expr);                                \
    if (_e != cudaSuccess) return ::l3::cuda_fail(_e, #expr); \
  } while (0)

// Device-side error bits, OR-ed into a flag word by kernels.
enum : int32_t {
  DEV_ERR_TOKEN_RANGE = 1,
  DEV_ERR_BAD_OFFSETS = 2,
  DEV_ERR_TIMEOUT = 4,
  DEV_ERR_F16_RANGE = 8,  // an fp16 operand (W_up, W', z) outside fp16's finite range
};

// ---------------------------------------------------------------------------
// profiling: optional CUDA-event bracketing of every launch
// ---------------------------------------------------------------------------
struct LaunchTimer {
  const char *name;
  cudaStream_t stream;
  int slot;
  LaunchTimer(const char *name, cudaStream_t s);
  ~LaunchTimer();
};

// ---------------------------------------------------------------------------
// work items built by the plan
// ---------------------------------------------------------------------------
// One 128-token tile of a group on the tensor-core attention path.
struct DenseTile {
  int32_t group;
  int32_t tok0;  // first sorted position of the tile
};
// One item of the CUDA-core attention path: up to TAIL_TOKENS tokens of one
// group, with everything a kernel needs to run it (no further lookups).
struct alignas(16) TailItem {
  int32_t r0;         // first row of K_t / V_t
  int16_t d;          // d_t
  int16_t nt;         // tokens in the item (1..TAIL_TOKENS)
  int32_t tok[8];     // original indices of the tokens
  int32_t pad[2];
};

constexpr int TAIL_TOKENS = 8;     // tokens per tail work item (size of TailItem::tok)
constexpr int DENSE_TILE_M = 128;  // tokens per dense tile
// a group runs on the tensor-core attention kernel when it has at least this
// many tokens and rows (and d_t fits the kernel); otherwise on CUDA cores
constexpr int DENSE_MIN_TOKENS = 5;
constexpr int DENSE_MIN_ROWS = 32;
// dense groups with at most this many rows run in a configuration that fits
// two CTAs per SM (256 TMEM columns, O computed in 256-column passes)
constexpr int DENSE_SMALL_ROWS = 256;
// dense tiles with at most this many tokens (a group's last tile, or its only
// one) run on the transposed-product kernel, tokens as the MMAs' N
constexpr int SKINNY_TOKENS = 32;
// tail items with at most this many rows are "small" (latency-bound)
constexpr int TAIL_SMALL_ROWS = 16;

}  // namespace l3

// The plan object behind the opaque l3_plan_t.
struct l3_plan_s {
  int device = 0;
  cudaStream_t stream = nullptr;  // last stream the plan's buffers were used on
  l3_dims_t dims{};
  int64_t n_tokens = 0;
  int64_t n_groups = 0;
  int64_t n_dense_groups = 0;
  int64_t n_dense_tiles = 0;
  int64_t n_dense_small = 0;  // the last n_dense_small tiles have d_t <= DENSE_SMALL_ROWS
  // tiles of at most SKINNY_TOKENS tokens among the first n_dense_tiles -
  // n_dense_small tiles and among the last n_dense_small
  int64_t n_skinny_big = 0, n_skinny_small = 0;
  int64_t n_tail_items = 0;
  int64_t unique_rows = 0;
  int64_t unique_rows_multi = 0;
  int64_t max_group_tokens = 0;
  int64_t tail_class_start[5] = {};  // tail items of token class c are [start[c], start[c+1])
  int64_t tail_class_split[4] = {};  // ... of which [split[c], start[c+1]) have d_t <= TAIL_SMALL_ROWS

  void *block = nullptr;  // the one device allocation backing everything below
  size_t block_bytes = 0;

  int32_t *perm = nullptr;             // [N] sorted position -> original index
  int32_t *inv_perm = nullptr;         // [N]
  int32_t *sorted_ids = nullptr;       // [N]
  int32_t *group_ids = nullptr;        // [N+1]
  int32_t *group_tok_start = nullptr;  // [N+1]
  int32_t *group_row_start = nullptr;  // [N+1] first row of group g in the table the forward reads
  int32_t *group_row_src = nullptr;    // [N+1] offsets[group_ids[g]]: first row in the full table
  bool staged = false;  // the forward reads a staged table (rows of group g at seg_rows[g])
  int32_t *group_rows = nullptr;       // [N+1] d_t of group g
  int32_t *seg_rows = nullptr;         // [N+1]
  l3::DenseTile *dense_tiles = nullptr;
  l3::TailItem *tail_items = nullptr;
  int32_t *dev_flags = nullptr;        // [0] plan errors, [1] forward errors, [4..9] dense tile counters
  void *a_buf = nullptr;               // [N x d_emb] dtype, original token order
  void *h_buf = nullptr;               // [N x d_up] h (CUDA-core path) or z = a W_up^T (fp16,
                                       // tensor-core path: the LayerNorm is applied inside W_mix)
  float *z_buf = nullptr;              // [N x d_up] fp32 (CUDA-core GEMM path only)
  void *w_up16 = nullptr;              // [d_up x d_emb] fp16 copy of W_up (tensor-core path)
  void *w_mixh16 = nullptr;            // [d_out x d_up] fp16 W_mix[:, :d_up] diag(gamma)
  float2 *ln_stats = nullptr;          // [ceil(d_up / 256) x N] (mean, M2) of z per 256 columns
  float *mix_ccol = nullptr;           // W' 1 [d_out], then W_mix[:, :d_up] beta at a 16-byte
                                       // aligned offset
  bool tc_gemm = false;                // tensor-core GEMMs in use
};

namespace l3 {

// device block cache (api.cu): cache_take returns a cached block of at
// least `bytes` on `device` whose last user has finished (its size in *got),
// or nullptr; cache_give returns a block once the work enqueued on `s` so far
// is done with it
void *cache_take(int device, size_t bytes, size_t *got);
void cache_give(void *ptr, size_t bytes, int device, cudaStream_t s);

// plan kernels (plan.cu)
// copy each group's rows of the full tables into staged tables (rows of
// group g at seg_rows[g]); the full tables may be in mapped host memory
l3_status launch_stage_rows(const l3_plan_s *p, const void *W_K, const void *W_V, void *K_staged,
                            void *V_staged, cudaStream_t s);
l3_status build_plan(l3_plan_s *p, const int32_t *token_ids, const int32_t *offsets,
                     cudaStream_t s, void *scratch, size_t scratch_bytes);
size_t plan_scratch_bytes(int64_t n_tokens);
// stable LSD radix sort of int32 keys in [0, 2^bits) with int32 values (the
// input index when vals_in is NULL); scratch of radix_sort_scratch_ints(n)
// ints; outputs must not alias inputs
size_t radix_sort_scratch_ints(int64_t n);
l3_status radix_sort_pairs(const int32_t *keys_in, const int32_t *vals_in, int64_t n, int bits,
                           int32_t *keys_out, int32_t *vals_out, int32_t *scratch,
                           cudaStream_t s);
// in-place exclusive scan of data[0..n) by one CTA; data[n] (and *total when
// given) receives the sum
l3_status exclusive_scan(int32_t *data, int64_t n, int32_t *total, cudaStream_t s);

// attention, CUDA-core path (attn_tail.cu)
l3_status launch_attn_tail(const l3_plan_s *p, const void *x, const void *W_K, const void *W_V,
                           cudaStream_t s);

// attention, CUDA-core path specialised by token count (attn_tail_cls.cu)
bool tail_cls_supported(const l3_dims_t &d);
// the class launches spread over n_streams streams (largest first, each to
// the least loaded stream)
l3_status launch_attn_tail_cls(const l3_plan_s *p, const void *x, const void *W_K,
                               const void *W_V, const cudaStream_t *streams, int n_streams);

// attention, tensor-core path (attn_dense.cu)
int sm_count(int device);  // SMs of the device (cached per device)
bool dense_attention_supported(const l3_dims_t &d);
int dense_attention_max_rows();
// one of the two launch configurations: tiles with d_t > DENSE_SMALL_ROWS
// (small = false) or the others; skip_skinny leaves the tiles of at most
// SKINNY_TOKENS tokens to launch_attn_skinny
l3_status launch_attn_dense(const l3_plan_s *p, const void *x, const void *W_K, const void *W_V,
                            bool small, bool skip_skinny, cudaStream_t s);
// backward of the dense tiles: p and g_s into the fp32 planes (bwd_scores_tc.cu)
bool bwd_scores_tc_supported(const l3_dims_t &d);
l3_status launch_bwd_scores_tc(const l3_plan_s *p, const void *x, const void *W_K,
                               const void *W_V, const float *g_a, float *slots, int slot_rows,
                               cudaStream_t s);
// dx += K_t^T g_s of the dense tiles' tokens from the g_s plane (bwd_scores_tc.cu)
bool bwd_dx_tc_supported(const l3_dims_t &d);
l3_status launch_bwd_dx_tc(const l3_plan_s *p, const void *W_K, const float *slots, int slot_rows,
                           float *dx, cudaStream_t s);
// attention for dense tiles of at most SKINNY_TOKENS tokens (attn_skinny.cu)
bool skinny_attention_supported(const l3_dims_t &d);
l3_status launch_attn_skinny(const l3_plan_s *p, const void *x, const void *W_K, const void *W_V,
                             cudaStream_t s);

// GEMMs + LayerNorm, tensor-core path (gemm_tc.cu)
bool tc_gemm_supported(const l3_dims_t &d);
l3_status launch_weights_f16(const l3_plan_s *p, const void *W_up, const void *W_mix,
                             const void *gamma, const void *beta, cudaStream_t s);
l3_status launch_up_z_tc(const l3_plan_s *p, cudaStream_t s);
l3_status launch_mix_tc(const l3_plan_s *p, const void *x, const void *W_mix, void *y,
                        cudaStream_t s);
// C[M x N] (fp32, row stride ldc) = A[M x K] B[N x K]^T (+ A1 B1^T when A1
// and B1 are given, same shapes and strides) on the pair kernel: operands
// row-major 16-bit, all fp16 (f16) or all bf16, row strides lda / ldb
// elements (multiples of 8), all pointers 16-byte aligned, N and ldc
// multiples of 4, K >= 1; anything else returns L3_ERR_UNSUPPORTED. A wait
// that gives up sets *err.
l3_status launch_gemm_nt_tc(const void *A, const void *B, const void *A1, const void *B1, bool f16,
                            int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, float *C,
                            int64_t ldc, int *err, int device, cudaStream_t s);

// GEMMs + LayerNorm, CUDA-core path (gemm_simt.cu)
l3_status launch_up_ln_simt(const l3_plan_s *p, const void *W_up, const void *gamma,
                            const void *beta, cudaStream_t s);
l3_status launch_mix_simt(const l3_plan_s *p, const void *x, const void *W_mix, void *y,
                          cudaStream_t s);

}  // namespace l3
