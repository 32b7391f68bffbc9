// Gather-attention on tensor cores for dense tiles of few tokens.
//
// A group's tokens share K_t and V_t, so per group (kimjy99 review, Method,
// eq. L³; sciencestack page, Fig. 3 caption: one dense mask block per ID)
//     S = X_g K_t^T,   P = exp(S - rowmax),   a = (P V_t) / rowsum(P).
// For a tile of at most SKINNY_TOKENS tokens (a group of 5-32 tokens, or the
// last tile of a larger group) the 128-token form of attn_dense.cu spends its
// MMAs on empty rows and its TMEM on a 128 x d_t score block. Here the same
// products run transposed, the tile's 32 token slots as the MMAs' N:
//     S^T = K_t X^T     (M = 128 rows of K_t per block, N = 32, K = d_in)
//     O^T = V_t^T P^T   (M = 128 columns of d_emb per block, N = 32, K = d_t)
// so the tensor work follows the tokens, S^T takes at most 4 x 32 TMEM
// columns and O^T another 128. A CTA takes half of an SM's shared memory and
// registers: the launch puts one on each SM and the tail kernels, which run
// beside it on a helper stream, take the other half (two skinny CTAs per SM
// left the tails no room: 1.46 -> 1.48 ms per paper-shaped batch; one, 1.43).
//
// Persistent CTAs claim tiles from the plan's dense tile list (its tiles of
// more than SKINNY_TOKENS tokens are left to attn_dense.cu). Per tile:
//   - warps 2-3 gather the tile's x rows (32 slots, zero past the group's
//     tokens) 64 columns at a time with cp.async into a ring of their own,
//     128-byte swizzled rows: the B operand of S^T, K-major;
//   - warp 0 streams, per 64-column slice of d_in, the K_t rows of each
//     128-row block by TMA (A operand, K-major); then V_t in 16-row slices;
//   - warp 1 issues tcgen05.mma: S^T block b into TMEM columns 32 b, then
//     O^T block e (columns 128 e .. 128 e + 127 of d_emb) into 128 + 32 e,
//     V_t as an MN-major A operand and P as a K-major B operand [token][row];
//   - warps 4-11 (two per TMEM lane quarter) take each token's exact max and
//     exponentials over the rows (a lane holds one row, 32 tokens: the warp
//     reduces its 32 x 32 block with a butterfly in which every step halves
//     the values a lane keeps), write P as bf16 and each token's sum of the
//     rounded values the MMA sees, then scale O^T by 1 / sum and store a
//     (fp16) at the tokens' original positions through a per-warp transpose.
// Rows at or past d_t take no part: their logits are masked, their P is 0 and
// the MMA warp zeroes them in the last V_t slice, so nothing in a neighbour
// ID's rows reaches this group (static routing).
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

constexpr int TN = SKINNY_TOKENS;          // token slots per tile: N of both products
constexpr int MB = 128;                    // rows of an M block (one MMA's M)
constexpr int CK = 64;                     // d_in columns per slice (128-byte rows)
constexpr int K_STAGE = MB * CK * 2;       // 16 KB: one block of one slice
constexpr int X_SLOT = TN * CK * 2;        // 4 KB
constexpr int N_X = 3;                     // x slices in flight
constexpr int X_LAG = N_X - 2;             // a slice is handed over once X_LAG later ones are issued
constexpr int REGION = 80 * 1024;          // K_t ring, later P and the V_t slices
constexpr int N_K = REGION / K_STAGE;      // 5
constexpr int MAX_STAGES = 8;
constexpr int MAX_D = 512;
constexpr int MAX_EMB = 512;
constexpr int V_ROWS = 16;                 // d_t rows per V_t slice (one MMA k-step)
constexpr int V_BLOCK = V_ROWS * 128;      // one 64-column box of a V_t slice
constexpr int P_BLOCK = TN * 128;          // 64 rows of P^T for the 32 tokens: 4 KB
constexpr int S_COLS = 4 * TN;             // TMEM columns of S^T
constexpr int TMEM_COLS = 256;             // S^T at 0, O^T at S_COLS
constexpr int THREADS = 384;               // 0 TMA, 1 MMA, 2-3 x gather, 4-11 softmax / epilogue
constexpr int SM_THREADS = 256;
constexpr int WBUF = TN * TN * 2;          // per-warp transpose buffer of the epilogue
static_assert(MAX_D <= 4 * MB && MAX_EMB <= 4 * MB, "four M blocks at most");
static_assert(MAX_D / 64 * P_BLOCK + 16 * MAX_EMB * 2 <= REGION, "P and one V slice fit");

struct SkBars {
  uint64_t xfull[N_X], xempty[N_X];
  uint64_t kfull[MAX_STAGES], kempty[MAX_STAGES];
  uint64_t vfull[MAX_STAGES], vempty[MAX_STAGES];
  uint64_t sfull;     // every S^T MMA of the tile has completed
  uint64_t sread;     // the softmax warps have read S^T (its columns are free)
  uint64_t pready;    // the softmax warps have written P
  uint64_t ofull;     // every O^T MMA of the tile has completed
  uint64_t odrained;  // the epilogue has read O^T (its columns are free)
  uint64_t pvdone;    // P and the V_t slices are free (the region takes K_t again)
  uint64_t tfull[2], tempty[2];  // tile handoff from the TMA warp
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int tile_slot[2];
  float red[8][TN];   // per softmax warp: partial max, then partial sum, of each token
};

struct SkParams {
  const __nv_bfloat16 *x;
  __half *a;
  const int32_t *perm;
  const int32_t *group_tok_start;
  const int32_t *group_row_start;
  const int32_t *group_rows;
  const DenseTile *tiles;
  int n_tiles;
  int *counter;  // [0] next tile to claim, [1] CTAs finished; the last CTA zeroes both
  int d_in, d_emb;
  int *err;
};

// a slice is handed over once X_LAG later ones have been issued
__device__ __forceinline__ void cp_async_wait_lag() { cp_async_wait<X_LAG>(); }
__device__ __forceinline__ bool sm_sync_and(bool ok) { return sync_and<1, SM_THREADS>(ok); }

struct SkGeo {
  int tok0, n_valid, r0, d, d16, d64, n_mb, n_vc, p_bytes, n_v;
};

__device__ __forceinline__ SkGeo sk_geo(const SkParams &P, int ti, int v_bytes) {
  SkGeo t;
  const DenseTile tile = P.tiles[ti];
  const int g = tile.group;
  t.tok0 = tile.tok0;
  t.n_valid = min(DENSE_TILE_M, P.group_tok_start[g + 1] - t.tok0);
  t.r0 = P.group_row_start[g];
  t.d = P.group_rows[g];
  t.d16 = (t.d + 15) & ~15;
  t.d64 = (t.d + 63) & ~63;
  t.n_mb = (t.d16 + MB - 1) / MB;
  t.n_vc = t.d16 / V_ROWS;
  t.p_bytes = (t.d64 / 64) * P_BLOCK;
  t.n_v = min(MAX_STAGES, (REGION - t.p_bytes) / v_bytes);
  return t;
}

__device__ __forceinline__ bool tile_is_skinny(const SkParams &P, int ti) {
  const DenseTile tile = P.tiles[ti];
  return P.group_tok_start[tile.group + 1] - tile.tok0 <= TN;
}

__device__ __forceinline__ int next_tile(SkBars *b, int u, const Abort &ab, bool &ok, int lane) {
  const int j = u & 1;
  ok = __all_sync(0xffffffffu, mbar_wait(&b->tfull[j], (u >> 1) & 1, ab));
  const int ti = *reinterpret_cast<volatile int *>(&b->tile_slot[j]);
  __syncwarp();
  if (lane == 0) mbar_arrive(&b->tempty[j]);
  return ok ? ti : -1;
}

__global__ void __launch_bounds__(THREADS, 2)
    k_attn_skinny(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mK16,
                  const __grid_constant__ CUtensorMap mV, SkParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *xring = smem + REGION;  // N_X slots of 4 KB
  uint8_t *wbufs = xring + N_X * X_SLOT;  // 8 x 2 KB epilogue transposes
  SkBars *b = reinterpret_cast<SkBars *>(wbufs + 8 * WBUF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_kc = P.d_in / CK;
  const int n_eb = P.d_emb / MB;  // O^T blocks
  const int v_bytes = V_ROWS * P.d_emb * 2;
  uint8_t *pbuf = smem;

  if (threadIdx.x == 0) {
    for (int s = 0; s < N_X; ++s) {
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
    mbar_init(&b->sread, 8);
    mbar_init(&b->pready, 8);
    mbar_init(&b->ofull, 1);
    mbar_init(&b->odrained, 8);
    mbar_init(&b->pvdone, 1);
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
    tmem_alloc(&b->tmem_base, TMEM_COLS);
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
      uint32_t ku = 0, vu = 0;  // per slot: parity of its uses so far
      bool armed[MAX_STAGES], varmed[MAX_STAGES];
      uint32_t armed_par[MAX_STAGES], varmed_par[MAX_STAGES];
      for (int i = 0; i < MAX_STAGES; ++i) armed[i] = varmed[i] = false;
      int kh = 0;  // K_t stages filled so far (the ring's depth is fixed)
      for (int u = 0; ok; ++u) {
        int ti;
        do {
          ti = atomicAdd(P.counter, 1);
        } while (ti < P.n_tiles && !tile_is_skinny(P, ti));
        if (ti >= P.n_tiles) ti = -1;
        const int j = u & 1;
        if (!mbar_wait(&b->tempty[j], ((u >> 1) & 1) ^ 1, ab)) {
          ok = false;
          break;
        }
        b->tile_slot[j] = ti;
        mbar_arrive(&b->tfull[j]);
        if (ti < 0) break;
        const SkGeo t = sk_geo(P, ti, v_bytes);
        // the region holds the previous tile's P and V_t slices until its
        // P V_t MMAs are done
        if (u > 0 && !mbar_wait(&b->pvdone, (u - 1) & 1, ab)) {
          ok = false;
          break;
        }
        for (int kc = 0; ok && kc < n_kc; ++kc) {
          for (int mb = 0; mb < t.n_mb; ++mb, ++kh) {
            const int s = kh % N_K;
            const uint32_t ph = (ku >> s) & 1;
            if (!mbar_wait(&b->kempty[s], ph ^ 1, ab)) {
              ok = false;
              break;
            }
            ku ^= 1u << s;
            uint8_t *kdst = smem + s * K_STAGE;
            // the block's rows up to d16: whole 64-row boxes, then 16-row ones
            const int rows = min(MB, t.d16 - mb * MB), k_full = rows / 64, k_rest = (rows % 64) / 16;
            const int row0 = t.r0 + mb * MB;
            mbar_arrive_expect_tx(&b->kfull[s], (uint32_t)rows * CK * 2);
            armed[s] = true;
            armed_par[s] = ph;
            for (int bx = 0; bx < k_full; ++bx)
              tma_load_2d(kdst + bx * 64 * CK * 2, &mK, &b->kfull[s], kc * CK, row0 + bx * 64);
            for (int bx = 0; bx < k_rest; ++bx)
              tma_load_2d(kdst + (k_full * 64 + bx * 16) * CK * 2, &mK16, &b->kfull[s], kc * CK,
                          row0 + k_full * 64 + bx * 16);
          }
        }
        // V_t slices go where the K_t ring was: every S^T MMA must be done
        if (ok) ok = mbar_wait(&b->sfull, u & 1, ab);
        for (int vc = 0; ok && vc < t.n_vc; ++vc) {
          const int i = vc % t.n_v;
          const uint32_t ph = (vu >> i) & 1;
          if (!mbar_wait(&b->vempty[i], ph ^ 1, ab)) {
            ok = false;
            break;
          }
          vu ^= 1u << i;
          uint8_t *vdst = smem + t.p_bytes + i * v_bytes;
          mbar_arrive_expect_tx(&b->vfull[i], (P.d_emb / 64) * V_BLOCK);
          varmed[i] = true;
          varmed_par[i] = ph;
          for (int bx = 0; bx < P.d_emb / 64; ++bx)
            tma_load_2d(vdst + bx * V_BLOCK, &mV, &b->vfull[i], bx * 64, t.r0 + vc * V_ROWS);
        }
      }
      if (!ok) {
        for (int s = 0; s < MAX_STAGES; ++s)
          if (armed[s]) spin_bounded(&b->kfull[s], armed_par[s]);
        for (int i = 0; i < MAX_STAGES; ++i)
          if (varmed[i]) spin_bounded(&b->vfull[i], varmed_par[i]);
      }
      // the last CTA to finish returns the counter to zero for the next launch
      if (atomicAdd(P.counter + 1, 1) == (int)gridDim.x - 1) {
        P.counter[0] = 0;
        P.counter[1] = 0;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = true;
    uint32_t mu = 0, mv = 0;  // per slot: parity of its uses so far (lane 0 / all lanes)
    int gx = 0, kh = 0;       // x slices and K_t stages consumed so far (lane 0)
    const uint32_t id_s = idesc_f16(1, 0, MB, TN);
    const uint32_t id_o = idesc_f16_amn(1, MB, TN);
    for (int u = 0; ok; ++u) {
      const int ti = next_tile(b, u, ab, ok, lane);
      if (!ok || ti < 0) break;
      const SkGeo t = sk_geo(P, ti, v_bytes);
      // S^T goes into columns the previous tile's softmax has read
      ok = __all_sync(0xffffffffu, mbar_wait(&b->sread, (u & 1) ^ 1, ab));
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        for (int kc = 0; ok && kc < n_kc; ++kc) {
          const int xs = gx % N_X;
          if (!mbar_wait(&b->xfull[xs], (gx / N_X) & 1, ab)) {
            ok = false;
            break;
          }
          ++gx;
          const uint32_t xa = smem_u32(xring + xs * X_SLOT);
          for (int mb = 0; mb < t.n_mb; ++mb, ++kh) {
            const int s = kh % N_K;
            if (!mbar_wait(&b->kfull[s], (mu >> s) & 1, ab)) {
              ok = false;
              break;
            }
            mu ^= 1u << s;
            tc_fence_after();
            const uint32_t ka = smem_u32(smem + s * K_STAGE);
#pragma unroll
            for (int k = 0; k < CK / 16; ++k)
              umma_f16(tmem + mb * TN, sdesc_sw128(ka + k * 32, 16, 1024),
                       sdesc_sw128(xa + k * 32, 16, 1024), id_s, (kc | k) != 0);
            umma_commit(&b->kempty[s]);
          }
          if (ok) umma_commit(&b->xempty[xs]);
        }
        if (ok) umma_commit(&b->sfull);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // O^T once P is written and the previous tile's O^T has been read out
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&b->pready, u & 1, ab));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&b->odrained, (u & 1) ^ 1, ab));
      tc_fence_after();
      const uint32_t pa = smem_u32(pbuf);
      for (int vc = 0; ok && vc < t.n_vc; ++vc) {
        const int i = vc % t.n_v;
        const uint32_t ph = (mv >> i) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&b->vfull[i], ph, ab))) {
          ok = false;
          break;
        }
        mv ^= 1u << i;
        uint8_t *vslot = smem + t.p_bytes + i * v_bytes;
        const int live = t.d - vc * V_ROWS;  // rows of this slice that belong to the group
        if (live < V_ROWS) {
          // rows at or past d_t belong to the next IDs: zero them, so that an
          // Inf or NaN there never meets a zero of P
          const int blocks = P.d_emb / 64, per_block = (V_ROWS - live) * 8;
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
          const int kk = vc * V_ROWS;  // row of V_t / column of P^T's K
          const uint64_t bdesc = sdesc_sw128(pa + (kk / 64) * P_BLOCK + (kk % 64) * 2, 16, 1024);
          for (int eb = 0; eb < n_eb; ++eb)
            umma_f16(tmem + S_COLS + eb * TN, sdesc_sw128(va + 2 * eb * V_BLOCK, V_BLOCK, 1024),
                     bdesc, id_o, vc != 0);
          umma_commit(&b->vempty[i]);
        }
        __syncwarp();
      }
      if (ok && lane == 0) {
        umma_commit(&b->ofull);
        umma_commit(&b->pvdone);
      }
    }
    if (!ok && lane == 0) {
      umma_commit(&b->drain);
      spin_bounded(&b->drain, 0);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ x-row gather
    // thread tw copies 16-byte chunk tw % 8 of token slots tw / 8 + 8 i
    // (i = 0..3), zero past the tile's tokens; a slice is handed to the MMA
    // warp once X_LAG later slices have been issued
    const int tw = (warp - 2) * 32 + lane;  // 0..63
    const int chunk = tw & 7, rb = tw >> 3;
    bool ok = true;
    int gx = 0;
    for (int u = 0; ok; ++u) {
      const int ti = next_tile(b, u, ab, ok, lane);
      if (!ok || ti < 0) break;
      const SkGeo t = sk_geo(P, ti, v_bytes);
      int src_row[TN / 8];
#pragma unroll
      for (int i = 0; i < TN / 8; ++i) {
        const int r = rb + 8 * i;
        src_row[i] = r < t.n_valid ? P.perm[t.tok0 + r] : -1;
      }
      int issued = 0, done = 0;
      for (int kc = 0; kc < n_kc; ++kc) {
        const int xs = (gx + kc) % N_X;
        ok = __all_sync(0xffffffffu, mbar_wait(&b->xempty[xs], (((gx + kc) / N_X) & 1) ^ 1, ab));
        if (!ok) break;
        uint8_t *dcol = xring + xs * X_SLOT + ((chunk ^ rb) << 4);
        const int col = kc * CK + chunk * 8;
#pragma unroll
        for (int i = 0; i < TN / 8; ++i) {
          const int r = rb + 8 * i;
          const bool valid = src_row[i] >= 0;
          cp_async16_zfill(dcol + r * 128, P.x + (valid ? (int64_t)src_row[i] * P.d_in + col : 0),
                           valid ? 16u : 0u);
        }
        cp_async_commit();
        ++issued;
        if (issued - done > X_LAG) {
          cp_async_wait_lag();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&b->xfull[(gx + done) % N_X]);
          ++done;
        }
      }
      cp_async_wait<0>();
      fence_proxy_async_smem();
      __syncwarp();
      for (; ok && done < issued; ++done)
        if (lane == 0) mbar_arrive(&b->xfull[(gx + done) % N_X]);
      gx += n_kc;
    }
  } else {
    // ------------------------------------------------------------ softmax, epilogue
    // warp sw = warp - 4 reads TMEM lane quarter q = warp % 4 and takes the
    // M blocks half, half + 2 (rows of S^T; columns of d_emb for O^T)
    const int sw = warp - 4, q = warp & 3, half = sw / 4;
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
    uint8_t *wbuf = wbufs + sw * WBUF;
    bool ok = true;
    for (int u = 0; ok; ++u) {
      const int ti = next_tile(b, u, ab, ok, lane);
      ok = sm_sync_and(ok);
      if (!ok || ti < 0) break;
      const SkGeo t = sk_geo(P, ti, v_bytes);
      ok = __all_sync(0xffffffffu, mbar_wait(&b->sfull, u & 1, ab));
      ok = sm_sync_and(ok);
      float tok_max = -INFINITY, inv_sum = 0.f;  // for token `lane`
      if (ok) {
        tc_fence_after();
        float m = -INFINITY;
        for (int mb = half; mb < t.n_mb; mb += 2) {
          const int j = mb * MB + q * 32 + lane;  // this lane's row of K_t
          uint32_t v[TN];
          tmem_ld32(tq + mb * TN, v);
          tmem_wait_ld();
          float f[TN];
#pragma unroll
          for (int e = 0; e < TN; ++e) f[e] = j < t.d ? __uint_as_float(v[e]) : -INFINITY;
          m = fmaxf(m, warp_transpose_reduce<false>(f, lane));
        }
        b->red[sw][lane] = m;
      }
      ok = sm_sync_and(ok);
      if (ok) {
#pragma unroll
        for (int w = 0; w < 8; ++w) tok_max = fmaxf(tok_max, b->red[w][lane]);
      }
      ok = sm_sync_and(ok);  // every warp has read red before it takes the sums
      if (ok) {
        float s = 0.f;
        for (int mb = half; mb < t.n_mb; mb += 2) {
          const int j = mb * MB + q * 32 + lane;
          uint32_t v[TN];
          tmem_ld32(tq + mb * TN, v);
          tmem_wait_ld();
          float f[TN];
          // P^T row j: 32 tokens, bf16, into P[token][j] (K-major B operand,
          // 64-row blocks of 32 x 128 bytes, 128-byte swizzle); rows from d
          // up to d16 are written as zeros, rows past d16 not at all
          uint8_t *pcol = pbuf + (j / 64) * P_BLOCK + (j % 8) * 2;
          const int cj = (j % 64) / 8;  // 16-byte chunk of the row
#pragma unroll
          for (int e = 0; e < TN; ++e) {
            const float mt = __shfl_sync(0xffffffffu, tok_max, e);
            const float p = j < t.d ? __expf(__uint_as_float(v[e]) - mt) : 0.f;
            const __nv_bfloat16 pb = __float2bfloat16_rn(p);
            f[e] = __bfloat162float(pb);  // the sum takes the values the MMA sees
            if (j < t.d16)
              *reinterpret_cast<__nv_bfloat16 *>(pcol + e * 128 + ((cj ^ (e & 7)) << 4)) = pb;
          }
          s += warp_transpose_reduce<true>(f, lane);
        }
        b->red[sw][lane] = s;
      }
      // S^T has been read and P written: the MMA warp may start the next
      // tile's S^T and this tile's O^T
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) {
        mbar_arrive(&b->sread);
        mbar_arrive(&b->pready);
      }
      ok = sm_sync_and(ok);
      if (ok) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += b->red[w][lane];
        inv_sum = 1.0f / s;
      }
      // epilogue: a = O^T / sum, per O^T block this warp's 32 columns of
      // d_emb for all 32 tokens, through the transpose buffer: each thread
      // writes its column, then each store instruction writes eight tokens'
      // 64-byte row pieces
      const int my_tok = lane < t.n_valid ? P.perm[t.tok0 + lane] : -1;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&b->ofull, u & 1, ab));
      if (ok) {
        tc_fence_after();
        for (int eb = half; eb < n_eb; eb += 2) {
          uint32_t v[TN];
          tmem_ld32(tq + S_COLS + eb * TN, v);
          tmem_wait_ld();
          // this lane's column of d_emb: e = 128 eb + 32 q + lane
#pragma unroll
          for (int e = 0; e < TN; ++e) {
            const float is = __shfl_sync(0xffffffffu, inv_sum, e);
            const __half h = __float2half_rn(__uint_as_float(v[e]) * is);
            // row e (token), column lane; 16-byte chunks XOR-swizzled by (e >> 1) & 3
            *reinterpret_cast<__half *>(wbuf + e * 64 + ((((lane >> 3) ^ ((e >> 1) & 3))) << 4) +
                                        (lane & 7) * 2) = h;
          }
          __syncwarp();
          const int col0 = eb * MB + q * 32;
#pragma unroll
          for (int k = 0; k < TN / 8; ++k) {
            const int rr = k * 8 + (lane >> 2), c4 = lane & 3;
            const uint4 o = *reinterpret_cast<const uint4 *>(wbuf + rr * 64 + ((c4 ^ ((rr >> 1) & 3)) << 4));
            const int tk = __shfl_sync(0xffffffffu, my_tok, rr);
            if (tk >= 0)
              *reinterpret_cast<uint4 *>(P.a + (int64_t)tk * P.d_emb + col0 + c4 * 8) = o;
          }
          __syncwarp();  // the buffer is read before the next block overwrites it
        }
      }
      // O^T's columns are free for the next tile's P V_t
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&b->odrained);
      ok = sm_sync_and(ok);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

constexpr size_t skinny_smem() {
  return 1024 + REGION + N_X * X_SLOT + 8 * WBUF + sizeof(SkBars);
}
// at most half of an SM's 228 KB (1 KB of it reserved per CTA)
static_assert(2 * (skinny_smem() + 1024) <= 228 * 1024, "half an SM");

}  // namespace

bool skinny_attention_supported(const l3_dims_t &d) {
  return d.dtype == L3_BF16 && d.d_in % CK == 0 && d.d_emb % MB == 0 && d.d_emb <= MAX_EMB &&
         d.k <= MAX_D;
}

l3_status launch_attn_skinny(const l3_plan_s *p, const void *x, const void *W_K, const void *W_V,
                             cudaStream_t s) {
  const int64_t n_skinny = p->n_skinny_big + p->n_skinny_small;
  if (n_skinny == 0) return L3_OK;
  const l3_dims_t &d = p->dims;
  CUtensorMap mK, mK16, mV;
  l3_status st;
  const uint64_t rows = p->staged ? (uint64_t)p->unique_rows : (uint64_t)d.v;
  if ((st = make_map_2d16(&mK, W_K, true, rows, d.d_in, d.d_in, CK, 64, 128)) != L3_OK) return st;
  if ((st = make_map_2d16(&mK16, W_K, true, rows, d.d_in, d.d_in, CK, 16, 128)) != L3_OK)
    return st;
  if ((st = make_map_2d16(&mV, W_V, true, rows, d.d_emb, d.d_emb, 64, V_ROWS, 128)) != L3_OK)
    return st;
  SkParams P;
  P.x = reinterpret_cast<const __nv_bfloat16 *>(x);
  P.a = reinterpret_cast<__half *>(p->a_buf);
  P.perm = p->perm;
  P.group_tok_start = p->group_tok_start;
  P.group_row_start = p->group_row_start;
  P.group_rows = p->group_rows;
  P.tiles = p->dense_tiles;
  P.n_tiles = (int)p->n_dense_tiles;
  P.counter = p->dev_flags + 8;
  P.d_in = (int)d.d_in;
  P.d_emb = (int)d.d_emb;
  P.err = p->dev_flags + 1;
  static bool attr[64] = {};
  if (!attr[p->device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_attn_skinny, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)skinny_smem()));
    attr[p->device & 63] = true;
  }
  // persistent, one CTA per SM (the other half of the SM for the tail kernels)
  const int64_t grid = std::min<int64_t>(n_skinny, (int64_t)sm_count(p->device));
  LaunchTimer t("attn_dense_skinny", s);
  k_attn_skinny<<<(unsigned)grid, THREADS, skinny_smem(), s>>>(mK, mK16, mV, P);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

}  // namespace l3
