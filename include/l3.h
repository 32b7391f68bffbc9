/*
 * l3.h — C ABI of the B200 (sm_100a) L³ forward-pass library (libl3.so).
 *
 * The layer is the Large Lookup Layer of "L³: Large Lookup Layers" (Tseng &
 * De Sa). For a token with hidden state x [d_in] and token ID t:
 *
 *     y = W_mix [ LayerNorm(W_up (V_t^T softmax(K_t x))) ; x ]      (kimjy99
 *     review, Method, eq. L³; papernotes.org note, 整体框架)
 *
 * where K_t = W_K[offsets[t] .. offsets[t+1]-1] and V_t likewise of W_V: the
 * per-token key/value sets are contiguous row slices of two concatenated
 * tables (kimjy99 review, §2 Efficient Training and Inference). Routing
 * depends on t alone (papernotes, 关键设计: static token routing).
 *
 * A batch is handled in two calls. l3_plan sorts the batch by token ID so
 * that tokens sharing an ID form one group, the block-diagonal form of the
 * sciencestack page's Fig. 3 caption. l3_forward then runs the layer over
 * those groups and writes y back in the caller's token order (the inverse
 * sort of the same caption).
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major, caller-owned DEVICE pointers on the
 *     current CUDA device, 16-byte aligned. The library never frees them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). All device work is enqueued on it.
 *   - Errors are returned as l3_status; l3_last_error() gives a message for
 *     the calling thread. Nothing aborts the process and no exception
 *     crosses the ABI. Invalid arguments are rejected before any launch.
 *   - bf16 is IEEE bfloat16 (round to nearest even when the library rounds);
 *     accumulation is fp32 on the GPU.
 */
#ifndef L3_H
#define L3_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  L3_OK = 0,
  L3_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misaligned pointer */
  L3_ERR_TOKEN_RANGE = 2,  /* a token ID outside [0, vocab) */
  L3_ERR_BAD_OFFSETS = 3,  /* offsets[0] != 0, offsets[vocab] != v, or some d_t outside [1, k] */
  L3_ERR_UNSUPPORTED = 4,  /* dims this build does not handle (see l3_dims_t) */
  L3_ERR_CUDA = 5,         /* a CUDA runtime call failed; the message names it */
  L3_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up (kernel returned early) */
  L3_ERR_OOM = 7           /* device allocation failed */
} l3_status;

typedef enum { L3_BF16 = 0, L3_FP32 = 1 } l3_dtype;

/*
 * Layer dimensions (kimjy99 review, Method: W_mix in R^{d_out x (d_in+d_up)},
 * K_t in R^{d_t x d_in}, V_t in R^{d_t x d_emb}; v = sum_t d_t with
 * 1 <= d_t <= k, papernotes LZW 分配 / kimjy99 Embedding Allocation).
 * W_up is read as d_up x d_emb: the shape printed on the review cannot map
 * d_emb to d_up, and this is the only shape that makes the equation typecheck.
 *
 * Supported: vocab >= 1, v >= vocab, 1 <= k <= 1024; for L3_BF16 every one
 * of d_in, d_emb, d_up, d_out a multiple of 16, d_in <= 8192, d_emb <= 512,
 * d_up <= 4096; for L3_FP32 multiples of 4 with the same bounds.
 * ln_eps is the LayerNorm epsilon (added to the biased variance).
 */
typedef struct {
  int64_t vocab;   /* |tau|, number of token IDs */
  int64_t v;       /* rows of W_K and W_V */
  int64_t k;       /* cap on d_t */
  int64_t d_in;
  int64_t d_emb;
  int64_t d_up;
  int64_t d_out;
  int32_t dtype;   /* l3_dtype of x, W_K, W_V, W_up, ln_gamma, ln_beta, W_mix, y */
  float ln_eps;
} l3_dims_t;

/* Opaque plan: the sorted batch plus the library-owned device buffers that
 * l3_forward uses. Owned by the library until l3_plan_destroy. */
typedef struct l3_plan_s *l3_plan_t;

/* Host-side summary of a plan. */
typedef struct {
  int64_t n_tokens;       /* N */
  int64_t n_groups;       /* G, distinct IDs in the batch */
  int64_t n_dense_groups; /* groups run on the tensor-core attention path */
  int64_t n_dense_tiles;  /* 128-token tiles of those groups */
  int64_t n_tail_items;   /* work items of the CUDA-core attention path */
  int64_t unique_rows;    /* sum of d_t over the groups: rows of W_K/W_V touched */
  int64_t unique_rows_multi; /* the same over groups with d_t > 1 (whose K_t is read) */
} l3_plan_info_t;

/*
 * l3_plan — sort a batch by token ID and build the group structure
 * (sciencestack page, Fig. 3 caption: sorting makes the attention mask
 * block-diagonal; kimjy99 review §2: sort B by T).
 *
 *   token_ids  device int32 [n_tokens], each in [0, dims->vocab)
 *   n_tokens   N >= 0 (N = 0 gives an empty plan; l3_forward then does nothing)
 *   offsets    device int32 [vocab + 1]: K_t = W_K rows offsets[t] .. offsets[t+1]-1;
 *              offsets[0] = 0, offsets[vocab] = v, 1 <= d_t <= k
 *   dims       host pointer, copied
 *   stream     cudaStream_t
 *   out        host pointer; receives a new plan on L3_OK, NULL otherwise
 *
 * The sort is stable: tokens with equal IDs keep their order, and groups
 * come in ascending ID order. token_ids and offsets are read during this
 * call only. The call synchronizes `stream` once, to read the group counts
 * and the validation flag; it is the only host-device round trip of the
 * path. Errors: L3_ERR_INVALID_ARG, L3_ERR_UNSUPPORTED, L3_ERR_TOKEN_RANGE,
 * L3_ERR_BAD_OFFSETS, L3_ERR_OOM, L3_ERR_CUDA.
 */
l3_status l3_plan(const int32_t *token_ids, int64_t n_tokens, const int32_t *offsets,
                  const l3_dims_t *dims, void *stream, l3_plan_t *out);

/*
 * l3_plan_staged — l3_plan for tables kept outside device memory (CPU
 * offload: the papernotes note, 关键设计 / CPU offload, and the sciencestack
 * page's inference section: the rows a token needs follow from its ID alone,
 * so they can be fetched before the layer runs).
 *
 * Same arguments, sort, synchronization and errors as l3_plan. The plan
 * addresses K_t / V_t in STAGED tables holding only this batch's rows:
 * group g's d_t rows at rows seg_rows[g] .. seg_rows[g+1]-1 (see
 * l3_plan_export), info.unique_rows rows in all. Fill them with
 * l3_stage_rows, then pass the staged tables to l3_forward as W_K / W_V.
 */
l3_status l3_plan_staged(const int32_t *token_ids, int64_t n_tokens, const int32_t *offsets,
                         const l3_dims_t *dims, void *stream, l3_plan_t *out);

/*
 * l3_stage_rows — copy the rows of a staged plan's batch from the full
 * tables into staged tables.
 *
 *   plan        from l3_plan_staged
 *   W_K, W_V    full tables [v x d_in], [v x d_emb] (dims->dtype): device
 *               memory, or page-locked host memory mapped into the device's
 *               address space (cudaHostAlloc / cudaHostRegister with
 *               mapping; the kernel reads it across PCIe)
 *   W_K_staged  device [info.unique_rows x d_in], caller-allocated
 *   W_V_staged  device [info.unique_rows x d_emb], caller-allocated
 * Rows of W_K are copied only for groups with d_t > 1 (a single row's
 * logit is never used); those staged rows are left as they were. All
 * pointers 16-byte aligned. Enqueued on `stream`; does not synchronize.
 * Errors: L3_ERR_INVALID_ARG (not a staged plan, NULL or misaligned
 * pointer, wrong device), L3_ERR_CUDA.
 */
l3_status l3_stage_rows(l3_plan_t plan, const void *W_K, const void *W_V, void *W_K_staged,
                        void *W_V_staged, void *stream);

/* Host summary of a plan (no device work). */
l3_status l3_plan_info(l3_plan_t plan, l3_plan_info_t *info);

/*
 * l3_plan_export — copy the plan's sort into caller-owned device buffers
 * (for tests that compare it bit for bit with a CPU sort). Any pointer may
 * be NULL to skip that array.
 *   perm[i]            original index of the token at sorted position i      [N]
 *   inv_perm[n]        sorted position of original token n                    [N]
 *   sorted_ids[i]      token ID at sorted position i                          [N]
 *   group_ids[g]       ID of group g, ascending                               [G]
 *   group_tok_start[g] first sorted position of group g; [G] = N             [G+1]
 *   seg_rows[g]        sum of d_t over groups before g; [G] = unique rows     [G+1]
 *   G_out              host int64, number of groups
 * Enqueued on `stream`; does not synchronize.
 */
l3_status l3_plan_export(l3_plan_t plan, int32_t *perm, int32_t *inv_perm, int32_t *sorted_ids,
                         int32_t *group_ids, int32_t *group_tok_start, int32_t *seg_rows,
                         int64_t *G_out, void *stream);

/*
 * l3_forward — y = L³(x, t) for every token of the plan's batch (kimjy99
 * review, Method, eq. L³).
 *
 *   x         [N x d_in]              hidden states, caller's token order
 *   W_K       [v x d_in]              concatenated key tables
 *   W_V       [v x d_emb]             concatenated value tables
 *   W_up      [d_up x d_emb]          up projection
 *   ln_gamma  [d_up], ln_beta [d_up]  LayerNorm affine parameters
 *   W_mix     [d_out x (d_up + d_in)] columns 0..d_up-1 multiply the LayerNorm
 *                                     output, columns d_up.. multiply x
 *   y         [N x d_out]             output, caller's token order
 * All in dims->dtype. Softmax has no 1/sqrt(d) scale (none appears in the
 * equation). For a bf16 layer the intermediates a = V_t^T p and z = W_up a
 * are stored once each as fp16 (fp16's 10-bit mantissa keeps the error that
 * LayerNorm amplifies small), and the LayerNorm is applied inside the W_mix
 * product, W_mix[:, :d_up] LayerNorm(z) = r (W' z - mu W' 1) + W_mix[:, :d_up]
 * beta with W' = W_mix[:, :d_up] diag(gamma) in fp16 and each row's mean mu
 * and 1 / std r from z's fp32 values; for an fp32 layer a and h =
 * LayerNorm(z) are stored as fp32. y is rounded once to dtype. The call only
 * enqueues work on `stream` and never synchronizes; a device-side wait that
 * gives up, and (bf16 layers) a W_up, W' or z value outside fp16's finite
 * range, are reported by l3_forward_status. Errors: L3_ERR_INVALID_ARG,
 * L3_ERR_CUDA.
 */
l3_status l3_forward(const void *x, l3_plan_t plan, const void *W_K, const void *W_V,
                     const void *W_up, const void *ln_gamma, const void *ln_beta,
                     const void *W_mix, void *y, void *stream);

/*
 * l3_backward — gradients of the layer (kimjy99 review, Method, eq. L³, by
 * the chain rule) for dL/dy. bf16 layers run the dense GEMMs and the dense
 * tiles' attention GEMMs on the tensor cores (bf16 operands, fp32 accumulate;
 * fp32 intermediates such as g_z, g_a, g_s and p enter as the sum of two bf16
 * parts) and the rest on CUDA cores in fp32; fp32 layers run all of it on
 * CUDA cores in fp32.
 *
 * Call after l3_forward on the same plan and the same inputs: it reuses the
 * a = V_t^T softmax(K_t x) that forward stored in the plan, and h =
 * LayerNorm(W_up a) as forward stored it (fp32 layers) or rebuilt from the z =
 * W_up a and row statistics forward stored (bf16 layers); it also recomputes
 * W_up a.
 *   x .. W_mix   as for l3_forward (dims->dtype)
 *   dy           [N x d_out] dims->dtype, caller's token order
 *   dx           fp32 [N x d_in], out
 *   dW_K, dW_V   fp32 [v x d_in], [v x d_emb], in/out: the batch's
 *                gradient is ADDED to the rows of every ID in the batch
 *                (zero them first for a fresh gradient); other rows untouched
 *   dW_up        fp32 [d_up x d_emb], out
 *   dgamma, dbeta fp32 [d_up], out
 *   dW_mix       fp32 [d_out x (d_up + d_in)], out
 * dW_K / dW_V take atomic adds (the order of a group's partial sums may
 * differ between calls); every other output is deterministic. Scratch (about
 * 3 N d_up + N d_emb floats, plus bf16 transposes of g_y, [h ; x], g_z and a
 * on the tensor-core path) comes from the library's device block cache
 * (cudaMalloc on a miss) and goes back to it, ordered after the work on
 * `stream`. Enqueued on `stream`; does not synchronize. Errors: L3_ERR_INVALID_ARG (NULL pointer,
 * a staged plan, x / W_K / W_V / dx / dW_K / dW_V not 16-byte aligned, a
 * different device than the plan's), L3_ERR_UNSUPPORTED (k > 1024, or d_in /
 * d_emb / d_up too wide for its shared-memory layout), L3_ERR_OOM,
 * L3_ERR_CUDA. The plan's last stream becomes `stream`: l3_plan_destroy and
 * l3_forward_status order themselves after this call's work.
 */
l3_status l3_backward(const void *x, l3_plan_t plan, const void *W_K, const void *W_V,
                      const void *W_up, const void *ln_gamma, const void *ln_beta,
                      const void *W_mix, const void *dy, float *dx, float *dW_K, float *dW_V,
                      float *dW_up, float *dgamma, float *dbeta, float *dW_mix, void *stream);

/*
 * l3_sort_tokens_noalloc — the stable sort step of l3_plan, for callers that
 * cannot allocate device memory. The pages have no counterpart: this entry
 * point exists for integration, not for the method.
 *
 * Who needs it: a process whose device memory is already reserved by
 * another allocator (a serving engine or framework caching allocator that
 * takes nearly all of HBM at start-up, so a cudaMalloc would fail or compete
 * with it), or a latency-critical loop that cannot accept the device-wide
 * synchronisation cudaMalloc / cudaFree can imply. This call allocates
 * nothing: no cudaMalloc, cudaFree or allocating library routine.
 *
 *   token_ids   device int32 [n_tokens], each in [0, vocab) (not checked:
 *               an out-of-range ID gives an unspecified order, never an
 *               out-of-bounds access)
 *   n_tokens    0 <= N <= L3_SORT_NOALLOC_MAX_TOKENS (65536); larger N is
 *               rejected with L3_ERR_INVALID_ARG
 *   vocab       number of token IDs, >= 1
 *   perm        device int32 [N], out: original index at sorted position i
 *   inv_perm    device int32 [N], out: sorted position of original token n
 *   sorted_ids  device int32 [N], out: token ID at sorted position i
 * The outputs equal l3_plan's perm / inv_perm / sorted_ids for the same IDs.
 * The four buffers must not overlap one another (an overlap is rejected with
 * L3_ERR_INVALID_ARG: the sort reads its input while other blocks write).
 *
 * Scratch: a file-scope device array of 590,080 bytes (2 x 65536 keys and
 * values plus the digit histogram) that every GPU which loads libl3.so holds
 * until the process exits. The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current; make that
 * first call before any stream capture on the device. Every call shares the
 * one array and overwrites it (each call writes every scratch word before it
 * reads it, so stale contents do not matter): calls that overlap on the GPU,
 * on different streams or from different host threads, race. Serialize them.
 * Enqueued on `stream`; does not synchronize. Errors: L3_ERR_INVALID_ARG,
 * L3_ERR_CUDA.
 */
#define L3_SORT_NOALLOC_MAX_TOKENS 65536
l3_status l3_sort_tokens_noalloc(const int32_t *token_ids, int64_t n_tokens, int64_t vocab,
                                 int32_t *perm, int32_t *inv_perm, int32_t *sorted_ids,
                                 void *stream);

/*
 * l3_lzw_allocate — how many rows of W_K / W_V each token ID gets: the
 * LZW-based allocation (kimjy99 review, 1. Embedding Allocation; papernotes
 * note, LZW 分配). Host code, no device work; run once, its output turned
 * into `offsets` (prefix sums) for l3_plan.
 *
 *   corpus       host int32 [n], token IDs in [0, vocab)
 *   n            corpus length >= 0 (< 2^31 - 2)
 *   vocab        number of token IDs >= 1
 *   v            row budget, vocab <= v <= vocab * k
 *   k            cap on rows per token >= 1
 *   d_out        host int32 [vocab], out: d_t, 1 <= d_t <= k, sum = v
 *   n_codewords  host int64, out: codewords the scan made (may be NULL)
 *
 * The scan makes one codeword per corpus position: the longest suffix of
 * the text ending there that is already a codeword, extended one token
 * further back, with frequency 1, and the suffix it extends gains 1 (a
 * suffix never reaches before position 0). Codewords are then walked from
 * most to least frequent, equal frequencies in creation order; each gives
 * its last token one row unless that token holds k. Every token starts
 * with one row; walks repeat until the rows sum to v. Time grows with the
 * corpus length times the length of the matched suffixes (short on natural
 * or Zipf-like text, up to quadratic on a text that repeats itself).
 * Errors: L3_ERR_INVALID_ARG (NULL pointer, a token out of range, v outside
 * [vocab, vocab * k], or v out of reach because every token that ends a
 * codeword already holds k), L3_ERR_OOM (host memory).
 */
l3_status l3_lzw_allocate(const int32_t *corpus, int64_t n, int64_t vocab, int64_t v, int64_t k,
                          int32_t *d_out, int64_t *n_codewords);

/*
 * l3_lzw_allocate_device — the same allocation as l3_lzw_allocate, with its
 * walk over the codewords (kimjy99 review, 1. Embedding Allocation: walk
 * the codewords by decreasing frequency, one row to each one's last token,
 * repeat until the budget) on the GPU. The corpus scan that builds the
 * codewords stays on the host: each position extends a suffix found among
 * the codewords made before it, a sequential dependence.
 *
 *   corpus, n, vocab, v, k, n_codewords   as for l3_lzw_allocate; in
 *                addition vocab < 2^31 - 1 and k < 2^31
 *   d_out        DEVICE int32 [vocab], out: d_t (4-byte aligned)
 *   stream       cudaStream_t the device work is enqueued on
 *
 * The result equals l3_lzw_allocate's bit for bit. On the device: a stable
 * radix sort of the codewords by frequency (the walk order), the number P of
 * complete walks found by binary search over P on T(P) = sum_t min(k, 1 + P
 * c_t) (c_t: codewords ending with t), then the last, partial walk from each
 * position's rank among the codewords ending with its token and one prefix
 * sum. Device scratch (about 9 ints per codeword plus 2 per token) is
 * cudaMalloc'ed and freed by the call; the call synchronizes `stream` once
 * at the end. Errors as l3_lzw_allocate, plus L3_ERR_CUDA.
 */
l3_status l3_lzw_allocate_device(const int32_t *corpus, int64_t n, int64_t vocab, int64_t v,
                                 int64_t k, int32_t *d_out, int64_t *n_codewords, void *stream);

/*
 * l3_check_bounded_wait — exercise the give-up path that every kernel's
 * waits share, on the device. The pages have no counterpart: this entry
 * point exists for failure detection, not for the method.
 *
 * Launches one small kernel that waits on an mbarrier nothing completes,
 * with the kernels' own bounded wait (2 s by %globaltimer). The wait gives
 * up, raises its CTA's abort flag, reports the timeout in device memory and
 * returns; the launch ends normally and the context stays usable.
 * Synchronizes `stream` and takes about 2 s.
 * Returns L3_ERR_TIMEOUT when the give-up was reported (the expected
 * result), L3_ERR_CUDA otherwise.
 */
l3_status l3_check_bounded_wait(void *stream);

/* Synchronizes the plan's last stream and returns L3_ERR_TIMEOUT if a
 * bounded wait inside an l3_forward kernel gave up since the plan was made
 * (the outputs of that call are then incomplete), L3_ERR_UNSUPPORTED if a bf16
 * layer's fp16 operand (W_up, W_mix[:, :d_up] diag(ln_gamma), z = W_up a) fell
 * outside fp16's finite range, L3_ERR_CUDA on a CUDA error, L3_OK otherwise. */
l3_status l3_forward_status(l3_plan_t plan);

/* Releases the plan. Its device memory returns to a small per-process cache
 * (at most four blocks, reused by later plans once the work last enqueued on
 * the plan's stream has finished; older blocks are freed). NULL is a no-op. */
void l3_plan_destroy(l3_plan_t plan);

/* Message for the last error on the calling thread ("" if none). */
const char *l3_last_error(void);

/*
 * Per-kernel timing for profiling: while enabled, every kernel the library
 * launches (enable = 1), or every kernel but the plan's (enable = 2), is
 * bracketed by CUDA events recorded on the stream it is launched on;
 * enable = 0 turns timing off. l3_profile_read synchronizes those streams and
 * returns, per kernel name, the number of launches and the summed device time
 * since the last l3_profile_enable. At most `max_entries` entries are written;
 * the return value is the number of distinct kernels (or -1 on error).
 */
typedef struct {
  char name[48];
  int64_t launches;
  double total_ms;
} l3_kernel_time_t;

void l3_profile_enable(int enable);
int l3_profile_read(l3_kernel_time_t *out, int max_entries);

#ifdef __cplusplus
}
#endif

#endif /* L3_H */
