// Gather-attention on tensor cores for groups with many tokens.
//
// After the batch sort, the tokens that share an ID t form a contiguous group
// whose attention mask is one dense block (sciencestack page, Fig. 3 caption;
// kimjy99 review §2): every token of the group attends to the same d_t rows
// K_t, V_t. For such a group the per-token products become matrix products,
//     S = X_g K_t^T   (tokens x d_t),   P = exp(S - rowmax),   O = P V_t,
//     a = O / rowsum(P)
// which is the layer's V_t^T softmax(K_t x) for every token of the group at
// once (kimjy99 review, Method, eq. L³).
//
// One CTA takes one 128-token tile of one group:
//   - warps 2-3 gather the tile's x rows (through the sort permutation) into
//     128-byte-swizzled shared memory with cp.async, 64 columns at a time and
//     up to a ring's depth of slices ahead;
//   - warp 0 streams the matching 64-column slices of K_t with TMA (128 bytes
//     of each row per request: half as many, twice as long DRAM reads as
//     32-column slices, which streamed K_t markedly slower), as many slices in
//     flight as the shared-memory ring holds for this d_t;
//   - warp 1 issues tcgen05.mma (M = 128 tokens, N = d_t up to 2 x 256) so that
//     S accumulates in TMEM over d_in;
//   - warps 4-11 (two per TMEM lane quarter, so two threads per token row,
//     each with half of the row's columns) take an exact row max and the
//     exponentials, and write P as bf16 into shared memory;
//   - warp 0 then streams V_t in 16-row slices with TMA and warp 1
//     accumulates O = P V_t (bf16 x bf16, the slices as they land) in the
//     TMEM columns S no longer needs, after zeroing the rows of the last
//     slice that lie past d_t;
//   - warps 4-11 scale O by 1 / rowsum and store a[perm[i]] (fp16), i.e. already
//     in the caller's token order.
// K_t and V_t are read from HBM by the group's first tile; its other tiles run
// at the same time and find them in L2.
// Groups with d_t <= 256 run in a second launch with half the shared memory
// and TMEM per CTA (two CTAs per SM), O then computed in 256-column passes.
// P and V_t meet in bf16 (tcgen05 kind::f16 takes one type for both
// operands): V_t needs no conversion, and P's largest entry, exp(0) = 1, is
// exact, so P's rounding weighs only on the smaller weights.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "l3_internal.cuh"
#include "sm100.cuh"

namespace l3 {

l3_status make_map_2d16(CUtensorMap *m, const void *base, bool bf16, uint64_t rows, uint64_t cols,
                        uint64_t ld, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes);

namespace {

using namespace sm100;

constexpr int TM = 128;                 // tokens per tile
constexpr int CK = 64;                  // d_in columns per S-phase slice (128-byte rows)
constexpr int MAX_D = 512;              // d_t handled here (TMEM columns)
constexpr int MAX_EMB = 512;
constexpr int X_BYTES = TM * CK * 2;    // 16 KB
constexpr int MAX_STAGES = 8;

// Two launch configurations. The big one holds S for d_t up to 512 (all 512
// TMEM columns, 192 KB of shared memory: one CTA per SM). The small one takes
// groups with d_t <= 256 in half of both, so two CTAs share an SM and twice as
// many K_t / x bytes are in flight; with d_emb > 256 it computes O in
// 256-column passes through the same TMEM columns.
template <bool SMALL>
struct DenseCfg {
  static constexpr int REGION = SMALL ? 96 * 1024 : 192 * 1024;  // S ring, later P + V slices
  static constexpr int TMEM_COLS = SMALL ? 256 : 512;
  static constexpr int MIN_BLOCKS = SMALL ? 2 : 1;
};
static_assert(DenseCfg<true>::TMEM_COLS == DENSE_SMALL_ROWS, "plan and kernel disagree on small d_t");
constexpr int V_ROWS = 16;              // d_t rows per V slice (one MMA k-step)
constexpr int V_BLOCK = V_ROWS * 128;   // one 64-column block of a V slice
constexpr int DENSE_THREADS = 384;  // 0 TMA, 1 MMA, 2-3 x gather, 4-11 softmax / epilogue
constexpr int SOFTMAX_THREADS = 256;

struct DenseBars {
  uint64_t xfull[MAX_STAGES], kfull[MAX_STAGES], sempty[MAX_STAGES];
  uint64_t sfull, pready, ofull;
  uint64_t vfull[MAX_STAGES], vempty[MAX_STAGES];
  uint64_t odrained;  // the epilogue has read this O pass out of TMEM
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  float red_max[2][128];  // per row: max of each half of the columns
  float red_sum[2][128];
};

struct DenseParams {
  const __nv_bfloat16 *x;
  __half *a;
  const int32_t *perm;
  const int32_t *group_tok_start;
  const int32_t *group_row_start;
  const int32_t *group_rows;
  const DenseTile *tiles;
  int d_in, d_emb;
  int *err;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void cp_async16_zfill(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}
// wait until at most `lag` committed groups of this thread are still in flight
__device__ __forceinline__ void cp_async_wait_group_lag(int lag) {
  switch (lag) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
    case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
    case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
    case 6: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 7;" ::: "memory"); break;
  }
}

// barrier of the 256 softmax / epilogue threads that ANDs a flag across them
__device__ __forceinline__ bool softmax_sync_and(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "n"(SOFTMAX_THREADS)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void spin_bounded(uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity) && globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
  }
}

template <bool SMALL>
__global__ void __launch_bounds__(DENSE_THREADS, DenseCfg<SMALL>::MIN_BLOCKS)
    k_attn_dense(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mK16,
                 const __grid_constant__ CUtensorMap mV, DenseParams P) {
  using Cfg = DenseCfg<SMALL>;
  constexpr int REGION = Cfg::REGION;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  DenseBars *b = reinterpret_cast<DenseBars *>(smem + REGION);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const DenseTile tile = P.tiles[blockIdx.x];
  const int g = tile.group;
  const int tok0 = tile.tok0;
  const int n_valid = min(TM, P.group_tok_start[g + 1] - tok0);
  const int r0 = P.group_row_start[g];
  const int d = P.group_rows[g];
  const int d16 = (d + 15) & ~15;       // N of the S product, K extent of the PV product
  const int d32 = (d + 31) & ~31;       // softmax works in 32-column TMEM loads
  const int d64 = (d + 63) & ~63;
  const int n_kc = P.d_in / CK;
  const int n_vc = d16 / V_ROWS;
  // K_t rows per slice: whole 64-row TMA boxes, then 16-row boxes up to d16
  // (the rows the MMA reads), so no slice fetches more than 15 rows past d_t
  const int k_full = d16 / 64, k_rest = (d16 % 64) / 16;
  const uint32_t k_slice_bytes = (uint32_t)(k_full * 64 + k_rest * 16) * CK * 2;
  // O = P V_t in passes of at most TMEM_COLS columns of d_emb
  const int o_max = min(P.d_emb, Cfg::TMEM_COLS);
  const int n_op = (P.d_emb + o_max - 1) / o_max;
  const int n_vs = n_op * n_vc;         // V slices over all passes
  // pipeline depth follows from d_t: the S ring holds as many slices as fit,
  // and so do the V buffers after P
  const int s_stage = X_BYTES + d64 * CK * 2;
  const int n_s = min(MAX_STAGES, REGION / s_stage);
  const int p_bytes = (d64 / 64) * (TM * 128);
  const int v_bytes = V_ROWS * o_max * 2;
  const int n_v = min(MAX_STAGES, (REGION - p_bytes) / v_bytes);
  uint8_t *pbuf = smem;                 // P slices (PV phase)
  uint8_t *vbuf = smem + p_bytes;       // V slices (PV phase)

  if (threadIdx.x == 0) {
    for (int s = 0; s < MAX_STAGES; ++s) {
      mbar_init(&b->xfull[s], 2);
      mbar_init(&b->kfull[s], 1);
      mbar_init(&b->sempty[s], 1);
    }
    mbar_init(&b->sfull, 1);
    mbar_init(&b->pready, 8);
    mbar_init(&b->ofull, 1);
    for (int i = 0; i < MAX_STAGES; ++i) {
      mbar_init(&b->vfull[i], 1);
      mbar_init(&b->vempty[i], 1);
    }
    mbar_init(&b->odrained, 8);
    mbar_init(&b->drain, 1);
    b->abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mK);
    prefetch_tensormap(&mK16);
    prefetch_tensormap(&mV);
  }
  if (warp == 1) {
    tmem_alloc(&b->tmem_base, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = b->tmem_base;
  const Abort ab{&b->abort_flag, P.err};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      bool ok = true;
      bool armed[MAX_STAGES];
      uint32_t armed_par[MAX_STAGES];
      for (int i = 0; i < MAX_STAGES; ++i) armed[i] = false;
      for (int kc = 0; kc < n_kc; ++kc) {
        const int s = kc % n_s;
        const uint32_t ph = (kc / n_s) & 1;
        if (!mbar_wait(&b->sempty[s], ph ^ 1, ab)) {
          ok = false;
          break;
        }
        uint8_t *kdst = smem + s * s_stage + X_BYTES;
        mbar_arrive_expect_tx(&b->kfull[s], k_slice_bytes);
        armed[s] = true;
        armed_par[s] = ph;
        for (int bx = 0; bx < k_full; ++bx)
          tma_load_2d(kdst + bx * 64 * CK * 2, &mK, &b->kfull[s], kc * CK, r0 + bx * 64);
        for (int bx = 0; bx < k_rest; ++bx)
          tma_load_2d(kdst + (k_full * 64 + bx * 16) * CK * 2, &mK16, &b->kfull[s], kc * CK,
                      r0 + k_full * 64 + bx * 16);
      }
      // V slices go where the S ring was: wait until every S-phase MMA is done
      if (ok) ok = mbar_wait(&b->sfull, 0, ab);
      bool varmed[MAX_STAGES];
      uint32_t varmed_par[MAX_STAGES];
      for (int i = 0; i < MAX_STAGES; ++i) varmed[i] = false;
      for (int gv = 0; ok && gv < n_vs; ++gv) {
        const int h = gv / n_vc, vc = gv % n_vc;
        const int v_boxes = min(o_max, P.d_emb - h * o_max) / 64;
        const int i = gv % n_v;
        const uint32_t ph = (gv / n_v) & 1;
        if (!mbar_wait(&b->vempty[i], ph ^ 1, ab)) {
          ok = false;
          break;
        }
        uint8_t *vdst = vbuf + i * v_bytes;
        mbar_arrive_expect_tx(&b->vfull[i], v_boxes * V_BLOCK);
        varmed[i] = true;
        varmed_par[i] = ph;
        for (int bx = 0; bx < v_boxes; ++bx)
          tma_load_2d(vdst + bx * V_BLOCK, &mV, &b->vfull[i], h * o_max + bx * 64,
                      r0 + vc * V_ROWS);
      }
      if (!ok) {
        for (int s = 0; s < MAX_STAGES; ++s)
          if (armed[s]) spin_bounded(&b->kfull[s], armed_par[s]);
        for (int i = 0; i < MAX_STAGES; ++i)
          if (varmed[i]) spin_bounded(&b->vfull[i], varmed_par[i]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // lane 0 issues; the whole warp waits for the V slices and zeroes the
    // padding rows of the last slice of each pass
    bool ok = true;
    if (lane == 0) {
      const int n_half = d16 > 256 ? 2 : 1;
      const uint32_t id_s0 = idesc_f16(1, 0, TM, d16 > 256 ? 256 : d16);
      const uint32_t id_s1 = idesc_f16(1, 0, TM, d16 > 256 ? d16 - 256 : 16);
      for (int kc = 0; ok && kc < n_kc; ++kc) {
        const int s = kc % n_s;
        const uint32_t ph = (kc / n_s) & 1;
        if (!mbar_wait(&b->xfull[s], ph, ab) || !mbar_wait(&b->kfull[s], ph, ab)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t xa = smem_u32(smem + s * s_stage);
        const uint32_t ka = xa + X_BYTES;
#pragma unroll
        for (int k = 0; k < CK / 16; ++k) {
          const uint64_t adesc = sdesc_sw128(xa + k * 32, 16, 1024);
          umma_f16(tmem, adesc, sdesc_sw128(ka + k * 32, 16, 1024), id_s0, (kc | k) != 0);
          if (n_half == 2)
            umma_f16(tmem + 256, adesc, sdesc_sw128(ka + 256 * CK * 2 + k * 32, 16, 1024), id_s1,
                     (kc | k) != 0);
        }
        umma_commit(&b->sempty[s]);
      }
      if (ok) umma_commit(&b->sfull);
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    // P V_t into the TMEM columns S used, once the softmax warps have read S
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&b->pready, 0, ab));
    const uint32_t pa = smem_u32(pbuf);
    for (int h = 0; ok && h < n_op; ++h) {
      // a later pass reuses the TMEM columns once the epilogue has read them
      if (h > 0 && !__all_sync(0xffffffffu, mbar_wait(&b->odrained, (h - 1) & 1, ab))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int o_w = min(o_max, P.d_emb - h * o_max);
      const int o_half = o_w > 256 ? 2 : 1;
      const uint32_t id_o0 = idesc_f16(1, 1, TM, o_w > 256 ? 256 : o_w);
      const uint32_t id_o1 = idesc_f16(1, 1, TM, o_w > 256 ? o_w - 256 : 16);
      for (int vc = 0; vc < n_vc; ++vc) {
        const int gv = h * n_vc + vc;
        const int i = gv % n_v;
        const uint32_t ph = (gv / n_v) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&b->vfull[i], ph, ab))) {
          ok = false;
          break;
        }
        const int live = d - vc * V_ROWS;  // rows of this slice that belong to the group
        if (live < V_ROWS) {
          // rows at or past d_t belong to the next token IDs: zero them, so that
          // nothing in another ID's rows (an Inf, a NaN) reaches this group's
          // P V_t through a zero of P (static routing: a token's output
          // depends on its own rows only)
          const int blocks = o_w / 64, per_block = (V_ROWS - live) * 8;
          uint4 *vb = reinterpret_cast<uint4 *>(vbuf + i * v_bytes);
          for (int e = lane; e < blocks * per_block; e += 32) {
            const int bk = e / per_block, w = e - bk * per_block;
            vb[bk * (V_BLOCK / 16) + live * 8 + w] = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t va = smem_u32(vbuf + i * v_bytes);
          const int kk = vc * V_ROWS;  // column of P / row of V_t
          const uint64_t adesc =
              sdesc_sw128(pa + (kk / 64) * (TM * 128) + (kk % 64) * 2, 16, 1024);
          umma_f16(tmem, adesc, sdesc_sw128(va, V_BLOCK, 1024), id_o0, vc != 0);
          if (o_half == 2)
            umma_f16(tmem + 256, adesc, sdesc_sw128(va + 4 * V_BLOCK, V_BLOCK, 1024), id_o1,
                     vc != 0);
          umma_commit(&b->vempty[i]);
        }
        __syncwarp();
      }
      if (ok && lane == 0) umma_commit(&b->ofull);
    }
    if (!ok && lane == 0) {
      umma_commit(&b->drain);
      spin_bounded(&b->drain, 0);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ x-row gather
    // cp.async copies (16 bytes each, zero-filled past the group's tokens),
    // up to n_s - 1 slices ahead; a slice is handed to the MMA warp once this
    // thread's copies for it have landed and been made visible to the async proxy.
    const int t = (warp - 2) * 32 + lane;  // 0..63, rows t and t + 64
    const __nv_bfloat16 *src_row[2];
    uint32_t src_bytes[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = t + u * 64;
      const bool valid = r < n_valid;
      src_row[u] = P.x + (valid ? (int64_t)P.perm[tok0 + r] * P.d_in : 0);
      src_bytes[u] = valid ? 16u : 0u;
    }
    const int lag = n_s - 1;
    bool ok = true;
    int issued = 0, done = 0;
    for (int kc = 0; kc < n_kc; ++kc) {
      const int s = kc % n_s;
      const uint32_t ph = (kc / n_s) & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&b->sempty[s], ph ^ 1, ab));
      if (!ok) break;
      uint8_t *xdst = smem + s * s_stage;
      // 128-byte rows; the 128-byte swizzle XORs the 16-byte chunk index with
      // bits 0-2 of the row
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int r = t + u * 64;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          cp_async16_zfill(xdst + r * 128 + ((j ^ (r & 7)) << 4), src_row[u] + kc * CK + j * 8,
                           src_bytes[u]);
      }
      cp_async_commit();
      ++issued;
      if (issued - done > lag) {
        cp_async_wait_group_lag(lag);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b->xfull[done % n_s]);
        ++done;
      }
    }
    // the last slices, and on a give-up every copy still in flight
    cp_async_wait_all();
    fence_proxy_async_smem();
    __syncwarp();
    for (; ok && done < issued; ++done)
      if (lane == 0) mbar_arrive(&b->xfull[done % n_s]);
  } else {
    // ------------------------------------------------------------ softmax, V convert, epilogue
    // warps 4-11: two warps per TMEM lane quarter, each taking every other
    // 32-column slice of the row; row max and row sum combine through shared
    // memory at barriers of these 256 threads
    const int sw = warp - 4;  // 0..7
    const int q = warp & 3;
    const int half = sw / 4;
    const int r = q * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    float inv_sum = 0.f;
    bool ok = __all_sync(0xffffffffu, mbar_wait(&b->sfull, 0, ab));
    ok = softmax_sync_and(ok);
    if (ok) {
      tc_fence_after();
      float m = -INFINITY;
      for (int c = half * 32; c < d32; c += 64) {
        uint32_t v[32];
        tmem_ld32(trow + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c + j < d) m = fmaxf(m, __uint_as_float(v[j]));
      }
      b->red_max[half][r] = m;
    }
    ok = softmax_sync_and(ok);
    if (ok) {
      const float m = fmaxf(b->red_max[0][r], b->red_max[1][r]);
      float sum = 0.f;
      for (int c = half * 32; c < d32; c += 64) {
        uint32_t v[32];
        tmem_ld32(trow + c, v);
        tmem_wait_ld();
        // 32 columns -> four 16-byte chunks of the 128-byte swizzled P row
        uint8_t *prow = pbuf + (c / 64) * (TM * 128) + r * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 o;
          __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = c + j * 8 + 2 * e;
            const float p0 = col < d ? __expf(__uint_as_float(v[j * 8 + 2 * e]) - m) : 0.f;
            const float p1 = col + 1 < d ? __expf(__uint_as_float(v[j * 8 + 2 * e + 1]) - m) : 0.f;
            const __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
            // the sum uses the rounded values the MMA will see
            const float2 hf = __bfloat1622float2(hp);
            sum += hf.x + hf.y;
            o2[e] = hp;
          }
          const int chunk = ((c % 64) / 8) + j;  // 16-byte chunk index within the row
          *reinterpret_cast<uint4 *>(prow + ((chunk ^ (r & 7)) << 4)) = o;
        }
      }
      b->red_sum[half][r] = sum;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0 && ok) mbar_arrive(&b->pready);
    ok = softmax_sync_and(ok);
    if (ok) inv_sum = 1.0f / (b->red_sum[0][r] + b->red_sum[1][r]);

    __half *arow = P.a + (r < n_valid ? (int64_t)P.perm[tok0 + r] * P.d_emb : 0);
    for (int h = 0; ok && h < n_op; ++h) {
      const int o_w = min(o_max, P.d_emb - h * o_max);
      // epilogue: a = O / rowsum, fp16, to the token's original position
      ok = __all_sync(0xffffffffu, mbar_wait(&b->ofull, h & 1, ab));
      if (!ok) break;
      tc_fence_after();
      for (int c = half * 32; c < o_w; c += 64) {
        uint32_t v[32];
        tmem_ld32(trow + c, v);
        tmem_wait_ld();
        if (r < n_valid) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 o;
            __half2 *o2 = reinterpret_cast<__half2 *>(&o);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              o2[e] = __floats2half2_rn(__uint_as_float(v[j * 8 + 2 * e]) * inv_sum,
                                        __uint_as_float(v[j * 8 + 2 * e + 1]) * inv_sum);
            *reinterpret_cast<uint4 *>(arow + h * o_max + c + j * 8) = o;
          }
        }
      }
      if (h + 1 < n_op) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b->odrained);
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

template <bool SMALL>
constexpr size_t dense_smem() {
  return 1024 + DenseCfg<SMALL>::REGION + sizeof(DenseBars);
}

template <bool SMALL>
l3_status launch_cfg(const CUtensorMap &mK, const CUtensorMap &mK16, const CUtensorMap &mV,
                     const DenseParams &P,
                     int64_t n_tiles, int device, const char *name, cudaStream_t s) {
  if (n_tiles == 0) return L3_OK;
  static bool attr[64] = {};
  if (!attr[device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_attn_dense<SMALL>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)dense_smem<SMALL>()));
    attr[device & 63] = true;
  }
  LaunchTimer t(name, s);
  k_attn_dense<SMALL><<<(unsigned)n_tiles, DENSE_THREADS, dense_smem<SMALL>(), s>>>(mK, mK16, mV, P);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

}  // namespace

bool dense_attention_supported(const l3_dims_t &d) {
  return d.dtype == L3_BF16 && d.d_in % CK == 0 && d.d_emb % 64 == 0 && d.d_emb <= MAX_EMB;
}
int dense_attention_max_rows() { return MAX_D; }

l3_status launch_attn_dense(const l3_plan_s *p, const void *x, const void *W_K, const void *W_V,
                            bool small, cudaStream_t s) {
  // the plan lists the tiles of groups with d_t > DENSE_SMALL_ROWS first
  const int64_t n_big = p->n_dense_tiles - p->n_dense_small;
  if ((small ? p->n_dense_small : n_big) == 0) return L3_OK;
  const l3_dims_t &d = p->dims;
  CUtensorMap mK, mK16, mV;
  l3_status st;
  // rows of the tables the kernel reads: all v, or the batch's rows when staged
  // (TMA fills rows past the end with zeros, so padding never reads past it)
  const uint64_t rows = p->staged ? (uint64_t)p->unique_rows : (uint64_t)d.v;
  if ((st = make_map_2d16(&mK, W_K, true, rows, d.d_in, d.d_in, CK, 64, 128)) != L3_OK) return st;
  if ((st = make_map_2d16(&mK16, W_K, true, rows, d.d_in, d.d_in, CK, 16, 128)) != L3_OK)
    return st;
  if ((st = make_map_2d16(&mV, W_V, true, rows, d.d_emb, d.d_emb, 64, V_ROWS, 128)) != L3_OK)
    return st;
  DenseParams P;
  P.x = reinterpret_cast<const __nv_bfloat16 *>(x);
  P.a = reinterpret_cast<__half *>(p->a_buf);
  P.perm = p->perm;
  P.group_tok_start = p->group_tok_start;
  P.group_row_start = p->group_row_start;
  P.group_rows = p->group_rows;
  P.tiles = p->dense_tiles;
  P.d_in = (int)d.d_in;
  P.d_emb = (int)d.d_emb;
  P.err = p->dev_flags + 1;
  if (!small) return launch_cfg<false>(mK, mK16, mV, P, n_big, p->device, "attn_dense", s);
  P.tiles = p->dense_tiles + n_big;
  return launch_cfg<true>(mK, mK16, mV, P, p->n_dense_small, p->device, "attn_dense_small", s);
}

}  // namespace l3
