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
// The kernel is persistent: each CTA claims 128-token tiles of one group from a
// counter until none are left, and for each tile
//   - warps 2-3 gather the tile's x rows (through the sort permutation) into
//     128-byte-swizzled shared memory with cp.async, 64 columns at a time, in a
//     ring of their own; each warp instruction copies whole 128-byte row
//     segments of four rows;
//   - warp 0 streams the matching 64-column slices of K_t with TMA (128 bytes
//     of each row per request), one slice per half of S (at most 256 rows, one
//     MMA's N), as many in flight as the rest of the shared memory holds;
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
// The next tile's x and K_t slices start loading as soon as this tile's P V_t
// MMAs are done, during its epilogue, and its S MMAs as soon as the epilogue
// has read O out of TMEM.
// K_t and V_t are read from HBM by the group's first tile; its other tiles run
// at the same time and find them in L2.
// Groups with d_t <= 256 run in a second launch with half the shared memory
// and TMEM per CTA (two CTAs per SM), O then computed in 256-column passes.
// P and V_t meet in bf16 (tcgen05 kind::f16 takes one type for both
// operands): V_t needs no conversion, and P's largest entry, exp(0) = 1, is
// exact, so P's rounding weighs only on the smaller weights.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "l3_internal.cuh"
#include "attn_common.cuh"
#include "sm100.cuh"

namespace l3 {

l3_status make_map_2d16(CUtensorMap *m, const void *base, bool bf16, uint64_t rows, uint64_t cols,
                        uint64_t ld, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes);

namespace {

using namespace sm100;
using namespace attn;

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
  static constexpr int REGION = SMALL ? 96 * 1024 : 192 * 1024;  // S-phase rings, later P + V slices
  static constexpr int N_X = SMALL ? 2 : 4;  // x slices in flight (ring at the top of the region)
  static constexpr int TMEM_COLS = SMALL ? 256 : 512;
  static constexpr int MIN_BLOCKS = SMALL ? 2 : 1;
};
static_assert(DenseCfg<true>::TMEM_COLS == DENSE_SMALL_ROWS, "plan and kernel disagree on small d_t");
constexpr int V_ROWS = 16;              // d_t rows per V slice (one MMA k-step)
constexpr int V_BLOCK = V_ROWS * 128;   // one 64-column block of a V slice
constexpr int DENSE_THREADS = 384;  // 0 TMA, 1 MMA, 2-3 x gather, 4-11 softmax / epilogue
constexpr int SOFTMAX_THREADS = 256;

struct DenseBars {
  uint64_t xfull[4], xempty[4];                // x slices (fixed depth N_X)
  uint64_t kfull[MAX_STAGES], kempty[MAX_STAGES];  // K_t slices (depth from d_t)
  uint64_t vfull[MAX_STAGES], vempty[MAX_STAGES];
  uint64_t sfull;     // every S-phase MMA of the tile has completed
  uint64_t pready;    // the softmax warps have written P
  uint64_t ofull;     // an O pass has completed
  uint64_t odrained;  // the epilogue has read an O pass that a later pass of the tile overwrites
  uint64_t pvdone;    // every P V_t MMA of the tile has completed: P and the V slices are free
  uint64_t tdrained;  // the epilogue has read the tile's last O pass: TMEM is free for the next S
  uint64_t tfull[2], tempty[2];  // tile handoff from the TMA warp to the other warps
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int tile_slot[2];
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
  int n_tiles;
  int *counter;    // [0] next tile to claim, [1] CTAs finished; the last CTA zeroes both
  int skip_skinny;  // leave tiles of at most SKINNY_TOKENS tokens to attn_skinny.cu
  int d_in, d_emb;
  int *err;
};


// barrier of the 256 softmax / epilogue threads that ANDs a flag across them
__device__ __forceinline__ bool softmax_sync_and(bool ok) {
  return sync_and<1, SOFTMAX_THREADS>(ok);
}


// Per-tile geometry, the same in every warp: the S ring and the P / V layout
// follow from d_t.
struct TileGeo {
  int tok0, n_valid, r0, d, d16, d32, d64, n_vc, n_half, k_stage, n_k, p_bytes, n_v;
  int h_rows0, h_rows1;  // K_t rows of each half of S (columns 0-255, 256-511)
};

template <int REGION, int N_X>
__device__ __forceinline__ TileGeo tile_geo(const DenseParams &P, int ti, int v_bytes) {
  TileGeo t;
  const DenseTile tile = P.tiles[ti];
  const int g = tile.group;
  t.tok0 = tile.tok0;
  t.n_valid = min(TM, P.group_tok_start[g + 1] - t.tok0);
  t.r0 = P.group_row_start[g];
  t.d = P.group_rows[g];
  t.d16 = (t.d + 15) & ~15;  // N of the S product, K extent of the PV product
  t.d32 = (t.d + 31) & ~31;  // softmax works in 32-column TMEM loads
  t.d64 = (t.d + 63) & ~63;
  t.n_vc = t.d16 / V_ROWS;
  // A K_t slice is one 64-column slice of the rows of one half of S (at most
  // 256 rows, one MMA's N), so the ring turns over in steps of at most 32 KB
  t.n_half = t.d16 > 256 ? 2 : 1;
  t.h_rows0 = min(t.d16, 256);
  t.h_rows1 = t.d16 - 256;
  // pipeline depth follows from d_t: below the x ring, the K_t ring holds as
  // many slices as fit, and so do the V slices after P
  t.k_stage = (t.n_half == 2 ? 256 : t.d64) * CK * 2;
  t.n_k = min(MAX_STAGES, (REGION - N_X * X_BYTES) / t.k_stage);
  t.p_bytes = (t.d64 / 64) * (TM * 128);
  t.n_v = min(MAX_STAGES, (REGION - t.p_bytes) / v_bytes);
  return t;
}

// The next tile index from the TMA warp (-1: none left). Every warp of a
// consumer role calls this once per tile, in order.
__device__ __forceinline__ int next_tile(DenseBars *b, int u, const Abort &ab, bool &ok,
                                         int lane) {
  const int j = u & 1;
  ok = __all_sync(0xffffffffu, mbar_wait(&b->tfull[j], (u >> 1) & 1, ab));
  const int ti = *reinterpret_cast<volatile int *>(&b->tile_slot[j]);
  __syncwarp();
  if (lane == 0) mbar_arrive(&b->tempty[j]);
  return ok ? ti : -1;
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
  const int n_kc = P.d_in / CK;
  // O = P V_t in passes of at most TMEM_COLS columns of d_emb
  const int o_max = min(P.d_emb, Cfg::TMEM_COLS);
  const int n_op = (P.d_emb + o_max - 1) / o_max;
  const int v_bytes = V_ROWS * o_max * 2;
  uint8_t *pbuf = smem;  // P slices (PV phase); V slices follow at p_bytes

  if (threadIdx.x == 0) {
    for (int s = 0; s < 4; ++s) {
      mbar_init(&b->xfull[s], 2);
      mbar_init(&b->xempty[s], 1);
    }
    for (int s = 0; s < MAX_STAGES; ++s) {
      mbar_init(&b->kfull[s], 1);
      mbar_init(&b->kempty[s], 1);
      mbar_init(&b->vfull[s], 1);
      mbar_init(&b->vempty[s], 1);
    }
    mbar_init(&b->sfull, 1);
    mbar_init(&b->pready, 8);
    mbar_init(&b->ofull, 1);
    mbar_init(&b->odrained, 8);
    mbar_init(&b->pvdone, 1);
    mbar_init(&b->tdrained, 8);
    for (int j = 0; j < 2; ++j) {
      mbar_init(&b->tfull[j], 1);
      mbar_init(&b->tempty[j], 11);  // warps 1-11
    }
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

  // Persistent: each CTA claims tiles from a counter until none are left. A
  // tile's S ring overlays the previous tile's P and V slices and its S the
  // previous tile's O, so the TMA and gather warps start the next tile's
  // slices as soon as the previous tile's P V_t MMAs are done (during its
  // epilogue), and the MMA warp once the epilogue has read O. Every ring slot
  // keeps a per-slot phase bit across tiles (the ring depth changes with d_t).
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      bool ok = true;
      uint32_t ku = 0, vu = 0;  // per slot: parity of its uses so far
      bool armed[MAX_STAGES], varmed[MAX_STAGES];
      uint32_t armed_par[MAX_STAGES], varmed_par[MAX_STAGES];
      for (int i = 0; i < MAX_STAGES; ++i) armed[i] = varmed[i] = false;
      for (int u = 0; ok; ++u) {
        int ti;
        do {
          ti = atomicAdd(P.counter, 1);
        } while (P.skip_skinny && ti < P.n_tiles &&
                 P.group_tok_start[P.tiles[ti].group + 1] - P.tiles[ti].tok0 <= SKINNY_TOKENS);
        if (ti >= P.n_tiles) ti = -1;
        const int j = u & 1;
        if (!mbar_wait(&b->tempty[j], ((u >> 1) & 1) ^ 1, ab)) {
          ok = false;
          break;
        }
        b->tile_slot[j] = ti;
        mbar_arrive(&b->tfull[j]);
        if (ti < 0) break;
        const TileGeo t = tile_geo<REGION, Cfg::N_X>(P, ti, v_bytes);
        if (u > 0 && !mbar_wait(&b->pvdone, (u - 1) & 1, ab)) {
          ok = false;
          break;
        }
        for (int kh = 0; kh < n_kc * t.n_half; ++kh) {
          const int kc = kh / t.n_half, hf = kh - kc * t.n_half;
          const int s = kh % t.n_k;
          const uint32_t ph = (ku >> s) & 1;
          if (!mbar_wait(&b->kempty[s], ph ^ 1, ab)) {
            ok = false;
            break;
          }
          ku ^= 1u << s;
          uint8_t *kdst = smem + s * t.k_stage;
          // whole 64-row TMA boxes, then 16-row boxes up to d16 (the rows the
          // MMA reads), so no slice fetches more than 15 rows past d_t
          const int rows = hf ? t.h_rows1 : t.h_rows0, k_full = rows / 64, k_rest = (rows % 64) / 16;
          const int row0 = t.r0 + hf * 256;
          mbar_arrive_expect_tx(&b->kfull[s], (uint32_t)rows * CK * 2);
          armed[s] = true;
          armed_par[s] = ph;
          for (int bx = 0; bx < k_full; ++bx)
            tma_load_2d(kdst + bx * 64 * CK * 2, &mK, &b->kfull[s], kc * CK, row0 + bx * 64);
          for (int bx = 0; bx < k_rest; ++bx)
            tma_load_2d(kdst + (k_full * 64 + bx * 16) * CK * 2, &mK16, &b->kfull[s], kc * CK,
                        row0 + k_full * 64 + bx * 16);
        }
        // V slices go where the S ring was: wait until every S-phase MMA is done
        if (ok) ok = mbar_wait(&b->sfull, u & 1, ab);
        for (int gv = 0; ok && gv < n_op * t.n_vc; ++gv) {
          const int h = gv / t.n_vc, vc = gv % t.n_vc;
          const int v_boxes = min(o_max, P.d_emb - h * o_max) / 64;
          const int i = gv % t.n_v;
          const uint32_t ph = (vu >> i) & 1;
          if (!mbar_wait(&b->vempty[i], ph ^ 1, ab)) {
            ok = false;
            break;
          }
          vu ^= 1u << i;
          uint8_t *vdst = smem + t.p_bytes + i * v_bytes;
          mbar_arrive_expect_tx(&b->vfull[i], v_boxes * V_BLOCK);
          varmed[i] = true;
          varmed_par[i] = ph;
          for (int bx = 0; bx < v_boxes; ++bx)
            tma_load_2d(vdst + bx * V_BLOCK, &mV, &b->vfull[i], h * o_max + bx * 64,
                        t.r0 + vc * V_ROWS);
        }
      }
      if (!ok) {
        for (int s = 0; s < MAX_STAGES; ++s)
          if (armed[s]) spin_bounded(&b->kfull[s], armed_par[s]);
        for (int i = 0; i < MAX_STAGES; ++i)
          if (varmed[i]) spin_bounded(&b->vfull[i], varmed_par[i]);
      }
      // the last CTA to finish returns the counter to zero for the next launch
      // (every CTA has made its last claim by then)
      if (atomicAdd(P.counter + 1, 1) == (int)gridDim.x - 1) {
        P.counter[0] = 0;
        P.counter[1] = 0;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // lane 0 issues; the whole warp waits for the V slices and zeroes the
    // padding rows of the last slice of each pass
    bool ok = true;
    uint32_t mu = 0, mv = 0;  // per slot: parity of its uses so far (lane 0 / all lanes)
    int gx = 0;               // x slices consumed so far (lane 0)
    for (int u = 0; ok; ++u) {
      const int ti = next_tile(b, u, ab, ok, lane);
      if (!ok || ti < 0) break;
      const TileGeo t = tile_geo<REGION, Cfg::N_X>(P, ti, v_bytes);
      // S goes into the TMEM columns of the previous tile's O
      ok = __all_sync(0xffffffffu, mbar_wait(&b->tdrained, (u & 1) ^ 1, ab));
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t id_s0 = idesc_f16(1, 0, TM, t.h_rows0);
        const uint32_t id_s1 = idesc_f16(1, 0, TM, t.n_half == 2 ? t.h_rows1 : 16);
        int kh = 0;
        for (int kc = 0; ok && kc < n_kc; ++kc) {
          const int xs = gx % Cfg::N_X;
          if (!mbar_wait(&b->xfull[xs], (gx / Cfg::N_X) & 1, ab)) {
            ok = false;
            break;
          }
          ++gx;
          const uint32_t xa = smem_u32(smem + REGION - (Cfg::N_X - xs) * X_BYTES);
          for (int hf = 0; hf < t.n_half; ++hf, ++kh) {
            const int s = kh % t.n_k;
            if (!mbar_wait(&b->kfull[s], (mu >> s) & 1, ab)) {
              ok = false;
              break;
            }
            mu ^= 1u << s;
            tc_fence_after();
            const uint32_t ka = smem_u32(smem + s * t.k_stage);
#pragma unroll
            for (int k = 0; k < CK / 16; ++k)
              umma_f16(tmem + hf * 256, sdesc_sw128(xa + k * 32, 16, 1024),
                       sdesc_sw128(ka + k * 32, 16, 1024), hf ? id_s1 : id_s0, (kc | k) != 0);
            umma_commit(&b->kempty[s]);
          }
          if (ok) umma_commit(&b->xempty[xs]);
        }
        if (ok) umma_commit(&b->sfull);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // P V_t into the TMEM columns S used, once the softmax warps have read S
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&b->pready, u & 1, ab));
      const uint32_t pa = smem_u32(pbuf);
      for (int h = 0; ok && h < n_op; ++h) {
        // a later pass reuses the TMEM columns once the epilogue has read them
        if (h > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(&b->odrained, (u * (n_op - 1) + h - 1) & 1, ab))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int o_w = min(o_max, P.d_emb - h * o_max);
        const int o_half = o_w > 256 ? 2 : 1;
        const uint32_t id_o0 = idesc_f16(1, 1, TM, o_w > 256 ? 256 : o_w);
        const uint32_t id_o1 = idesc_f16(1, 1, TM, o_w > 256 ? o_w - 256 : 16);
        for (int vc = 0; vc < t.n_vc; ++vc) {
          const int gv = h * t.n_vc + vc;
          const int i = gv % t.n_v;
          const uint32_t ph = (mv >> i) & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(&b->vfull[i], ph, ab))) {
            ok = false;
            break;
          }
          mv ^= 1u << i;
          uint8_t *vslot = smem + t.p_bytes + i * v_bytes;
          const int live = t.d - vc * V_ROWS;  // rows of this slice that belong to the group
          if (live < V_ROWS) {
            // rows at or past d_t belong to the next token IDs: zero them, so that
            // nothing in another ID's rows (an Inf, a NaN) reaches this group's
            // P V_t through a zero of P (static routing: a token's output
            // depends on its own rows only)
            const int blocks = o_w / 64, per_block = (V_ROWS - live) * 8;
            uint4 *vb = reinterpret_cast<uint4 *>(vslot);
            for (int e = lane; e < blocks * per_block; e += 32) {
              const int bk = e / per_block, w = e - bk * per_block;
              vb[bk * (V_BLOCK / 16) + live * 8 + w] = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t va = smem_u32(vslot);
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
      if (ok && lane == 0) umma_commit(&b->pvdone);
    }
    if (!ok && lane == 0) {
      umma_commit(&b->drain);
      spin_bounded(&b->drain, 0);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ x-row gather
    // cp.async copies (16 bytes each, zero-filled past the group's tokens)
    // into a ring of N_X slices; a slice is handed to the MMA warp once this
    // thread's copies for it have landed and been made visible to the async
    // proxy, as soon as LAG later slices have been issued. With LAG = N_X - 2
    // handing over slice n needs only slice n - 2 to have been consumed, so
    // the handover does not wait for the MMAs of slice n - 1. Thread tw copies 16-byte chunk tw % 8 of rows tw / 8 + 8 i
    // (i = 0..15), so every warp instruction reads four whole 128-byte row
    // segments instead of one 16-byte piece of 32 rows.
    const int tw = (warp - 2) * 32 + lane;  // 0..63
    const int chunk = tw & 7, rb = tw >> 3;
    bool ok = true;
    int gx = 0;  // x slices gathered so far
    for (int u = 0; ok; ++u) {
      const int ti = next_tile(b, u, ab, ok, lane);
      if (!ok || ti < 0) break;
      const TileGeo t = tile_geo<REGION, Cfg::N_X>(P, ti, v_bytes);
      int src_row[16];  // original token of each of this thread's rows, -1 past the group
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = rb + 8 * i;
        src_row[i] = r < t.n_valid ? P.perm[t.tok0 + r] : -1;
      }
      if (u > 0 && !__all_sync(0xffffffffu, mbar_wait(&b->pvdone, (u - 1) & 1, ab))) {
        ok = false;
        break;
      }
      constexpr int lag = Cfg::N_X >= 3 ? Cfg::N_X - 2 : Cfg::N_X - 1;
      int issued = 0, done = 0;
      for (int kc = 0; kc < n_kc; ++kc) {
        const int xs = (gx + kc) % Cfg::N_X;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&b->xempty[xs], (((gx + kc) / Cfg::N_X) & 1) ^ 1, ab));
        if (!ok) break;
        uint8_t *xdst = smem + REGION - (Cfg::N_X - xs) * X_BYTES;
        const int col = kc * CK + chunk * 8;
        // 128-byte rows; the 128-byte swizzle XORs the 16-byte chunk index with
        // bits 0-2 of the row (here rb, since 8 i does not change them)
        uint8_t *dcol = xdst + ((chunk ^ rb) << 4);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = rb + 8 * i;
          const bool valid = src_row[i] >= 0;
          cp_async16_zfill(dcol + r * 128,
                           P.x + (valid ? (int64_t)src_row[i] * P.d_in + col : 0),
                           valid ? 16u : 0u);
        }
        cp_async_commit();
        ++issued;
        if (issued - done > lag) {
          cp_async_wait<lag>();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&b->xfull[(gx + done) % Cfg::N_X]);
          ++done;
        }
      }
      // the last slices, and on a give-up every copy still in flight
      cp_async_wait<0>();
      fence_proxy_async_smem();
      __syncwarp();
      for (; ok && done < issued; ++done)
        if (lane == 0) mbar_arrive(&b->xfull[(gx + done) % Cfg::N_X]);
      gx += n_kc;
    }
  } else {
    // ------------------------------------------------------------ softmax, epilogue
    // warps 4-11: two warps per TMEM lane quarter, each taking every other
    // 32-column slice of the row; row max and row sum combine through shared
    // memory at barriers of these 256 threads, which all of them pass the same
    // number of times
    const int sw = warp - 4;  // 0..7
    const int q = warp & 3;
    const int half = sw / 4;
    const int r = q * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    bool ok = true;
    for (int u = 0; ok; ++u) {
      const int ti = next_tile(b, u, ab, ok, lane);
      ok = softmax_sync_and(ok);
      if (!ok || ti < 0) break;
      const TileGeo t = tile_geo<REGION, Cfg::N_X>(P, ti, v_bytes);
      float inv_sum = 0.f;
      ok = __all_sync(0xffffffffu, mbar_wait(&b->sfull, u & 1, ab));
      ok = softmax_sync_and(ok);
      if (ok) {
        tc_fence_after();
        float m = -INFINITY;
        for (int c = half * 32; c < t.d32; c += 64) {
          uint32_t v[32];
          tmem_ld32(trow + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c + j < t.d) m = fmaxf(m, __uint_as_float(v[j]));
        }
        b->red_max[half][r] = m;
      }
      ok = softmax_sync_and(ok);
      if (ok) {
        const float m = fmaxf(b->red_max[0][r], b->red_max[1][r]);
        float sum = 0.f;
        for (int c = half * 32; c < t.d32; c += 64) {
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
              const float p0 = col < t.d ? __expf(__uint_as_float(v[j * 8 + 2 * e]) - m) : 0.f;
              const float p1 =
                  col + 1 < t.d ? __expf(__uint_as_float(v[j * 8 + 2 * e + 1]) - m) : 0.f;
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

      __half *arow = P.a + (r < t.n_valid ? (int64_t)P.perm[t.tok0 + r] * P.d_emb : 0);
      for (int h = 0; ok && h < n_op; ++h) {
        const int o_w = min(o_max, P.d_emb - h * o_max);
        // epilogue: a = O / rowsum, fp16, to the token's original position
        ok = __all_sync(0xffffffffu, mbar_wait(&b->ofull, (u * n_op + h) & 1, ab));
        if (!ok) break;
        tc_fence_after();
        for (int c = half * 32; c < o_w; c += 64) {
          uint32_t v[32];
          tmem_ld32(trow + c, v);
          tmem_wait_ld();
          if (r < t.n_valid) {
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
      // the tile's TMEM columns are free for the next tile's S
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&b->tdrained);
      ok = softmax_sync_and(ok);
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
                     DenseParams P, int64_t n_tiles, int64_t n_own, int device, const char *name,
                     cudaStream_t s) {
  if (n_tiles == 0) return L3_OK;
  static bool attr[64] = {};
  if (!attr[device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_attn_dense<SMALL>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)dense_smem<SMALL>()));
    attr[device & 63] = true;
  }
  // persistent: as many CTAs as fit at once, each claiming tiles until none are left
  // (n_own of the n_tiles are this launch's: the others are skinny tiles)
  const int64_t grid = std::min<int64_t>(n_own, (int64_t)sm_count(device) * DenseCfg<SMALL>::MIN_BLOCKS);
  P.n_tiles = (int)n_tiles;
  LaunchTimer t(name, s);
  k_attn_dense<SMALL><<<(unsigned)grid, DENSE_THREADS, dense_smem<SMALL>(), s>>>(mK, mK16, mV, P);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

}  // namespace

int sm_count(int device) {
  static int n[64] = {};
  if (n[device & 63] == 0) cudaDeviceGetAttribute(&n[device & 63], cudaDevAttrMultiProcessorCount, device);
  return n[device & 63];
}

bool dense_attention_supported(const l3_dims_t &d) {
  return d.dtype == L3_BF16 && d.d_in % CK == 0 && d.d_emb % 64 == 0 && d.d_emb <= MAX_EMB;
}
int dense_attention_max_rows() { return MAX_D; }

l3_status launch_attn_dense(const l3_plan_s *p, const void *x, const void *W_K, const void *W_V,
                            bool small, bool skip_skinny, cudaStream_t s) {
  // the plan lists the tiles of groups with d_t > DENSE_SMALL_ROWS first
  const int64_t n_big = p->n_dense_tiles - p->n_dense_small;
  const int64_t n_own = small ? p->n_dense_small - (skip_skinny ? p->n_skinny_small : 0)
                              : n_big - (skip_skinny ? p->n_skinny_big : 0);
  if (n_own == 0) return L3_OK;
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
  P.counter = p->dev_flags + 4;
  P.skip_skinny = skip_skinny ? 1 : 0;
  if (!small) return launch_cfg<false>(mK, mK16, mV, P, n_big, n_own, p->device, "attn_dense", s);
  P.tiles = p->dense_tiles + n_big;
  P.counter = p->dev_flags + 6;
  return launch_cfg<true>(mK, mK16, mV, P, p->n_dense_small, n_own, p->device, "attn_dense_small",
                          s);
}

}  // namespace l3
