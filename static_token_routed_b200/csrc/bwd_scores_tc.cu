// Attention backward of the dense tiles, first half, on tensor cores.
//
// Per token n of a group with rows K_t, V_t (kimjy99 review, Method, eq. L³,
// differentiated by the chain rule):
//     s = K_t x,  p = softmax(s),  g_p = V_t g_a,  g_s = p (g_p - p . g_p),
// with g_a = dL/da from the LayerNorm and W_up backward. For a chunk of up to
// 32 tokens of a dense tile this kernel forms, with the tokens as the MMAs' N,
//     S^T = K_t X^T      (M = 128 rows of K_t per block, K = d_in)
//     G_p^T = V_t G_a^T  (M = 128 rows of V_t per block, K = d_emb; g_a enters
//                         as the sum of two bf16 parts, hi + lo)
// in TMEM, then the exact softmax over the rows and g_s per token, and writes
// p and g_s into the tile's two fp32 planes [row][token] that the dx and
// dK / dV kernels read. One CTA per (tile, 32-token chunk), two per SM:
//   - warp 0 streams by TMA the rows of each 128-row block, 64 columns at a
//     time: K_t's d_in columns, then V_t's d_emb columns (A operands, K-major);
//   - warps 2-3 gather the chunk's x rows (cp.async), then convert the chunk's
//     g_a rows to bf16 hi / lo parts, 64 columns at a time, into a ring of
//     128-byte swizzled slots (B operands, K-major, zero past the tokens);
//   - warp 1 issues tcgen05.mma: S^T block b into TMEM columns 32 b, G_p^T
//     block b into 128 + 32 b (hi and lo parts);
//   - warps 4-11 (two per TMEM lane quarter; a lane holds one row, 32 tokens)
//     reduce each token's max, exp-sum and sum of exp(s - max) g_p over the
//     rows with warp butterflies and shared memory, then write p and g_s.
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

constexpr int TN = 32;                   // tokens per chunk: N of both products
constexpr int MB = 128;                  // rows per M block
constexpr int CK = 64;                   // columns per slice (128-byte rows)
constexpr int K_STAGE = MB * CK * 2;     // 16 KB
constexpr int N_K = 5;                   // K_t / V_t stages in flight
constexpr int B_SLOT = TN * CK * 2;      // 4 KB: one bf16 operand slice
constexpr int N_B = 3;                   // B slots (x, or g_a hi + lo)
constexpr int MAX_D = 512;
constexpr int THREADS = 384;             // 0 TMA, 1 MMA, 2-3 B operands, 4-11 softmax
constexpr int SM_THREADS = 256;
constexpr int TMEM_COLS = 256;           // S^T at 0, G_p^T at 128
constexpr int G_COL = 4 * TN;
constexpr int V16_BOX() { return 16 * 128; }  // one 16-row, 64-column bf16 TMA box: 2 KB

struct Bars {
  uint64_t bfull[N_B], bempty[N_B];
  uint64_t kfull[N_K], kempty[N_K];
  uint64_t done;  // every MMA of the chunk has completed
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  float red[3][8][TN];  // per softmax warp and token: max, exp-sum, exp-weighted g_p sum
};

struct Params {
  const __nv_bfloat16 *x;
  const float *g_a;
  const int32_t *perm;
  const int32_t *group_tok_start;
  const int32_t *group_row_start;
  const int32_t *group_rows;
  const DenseTile *tiles;
  float *slots;
  int slot_rows;
  int d_in, d_emb;
  int *err;
};

__device__ __forceinline__ void cp_async_wait_all() { cp_async_wait<0>(); }
__device__ __forceinline__ void cp_async_wait_1() { cp_async_wait<1>(); }
__device__ __forceinline__ bool sm_sync_and(bool ok) { return sync_and<1, SM_THREADS>(ok); }

__global__ void __launch_bounds__(THREADS, 2)
    k_bwd_scores_tc(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mK16,
                    const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mV16,
                    Params P) {
  const int ti = blockIdx.x / (DENSE_TILE_M / TN), chunk = blockIdx.x % (DENSE_TILE_M / TN);
  const DenseTile tile = P.tiles[ti];
  const int g = tile.group;
  const int n_tile = min(DENSE_TILE_M, P.group_tok_start[g + 1] - tile.tok0);
  const int tok0 = tile.tok0 + chunk * TN;
  const int n_valid = min(TN, n_tile - chunk * TN);
  if (n_valid <= 0) return;  // the whole CTA, before any barrier or TMEM
  const int r0 = P.group_row_start[g], d = P.group_rows[g];
  const int d16 = (d + 15) & ~15, n_mb = (d16 + MB - 1) / MB;
  const int n_kc = P.d_in / CK, n_ec = P.d_emb / CK;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *bring = smem + N_K * K_STAGE;  // N_B slots of hi + lo (2 x 4 KB)
  Bars *b = reinterpret_cast<Bars *>(bring + N_B * 2 * B_SLOT);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < N_B; ++s) {
      mbar_init(&b->bfull[s], 2);
      mbar_init(&b->bempty[s], 1);
    }
    for (int s = 0; s < N_K; ++s) {
      mbar_init(&b->kfull[s], 1);
      mbar_init(&b->kempty[s], 1);
    }
    mbar_init(&b->done, 1);
    mbar_init(&b->drain, 1);
    b->abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mK);
    prefetch_tensormap(&mK16);
    prefetch_tensormap(&mV);
    prefetch_tensormap(&mV16);
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
  // the A operand sequence: K_t slices kc = 0..n_kc-1, then V_t slices, each
  // as n_mb blocks of 128 rows; the B sequence: x slices, then g_a slices
  const int n_steps = (n_kc + n_ec) * n_mb;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      bool ok = true;
      bool armed[N_K];
      uint32_t armed_par[N_K];
      for (int i = 0; i < N_K; ++i) armed[i] = false;
      for (int kh = 0; ok && kh < n_steps; ++kh) {
        const int s = kh % N_K;
        const uint32_t ph = (kh / N_K) & 1;
        if (!mbar_wait(&b->kempty[s], ph ^ 1, ab)) {
          ok = false;
          break;
        }
        const int sl = kh / n_mb, mb = kh % n_mb;
        const bool is_v = sl >= n_kc;
        const int col = (is_v ? sl - n_kc : sl) * CK;
        const int rows = min(MB, d16 - mb * MB), k_full = rows / 64, k_rest = (rows % 64) / 16;
        const int row0 = r0 + mb * MB;
        uint8_t *dst = smem + s * K_STAGE;
        mbar_arrive_expect_tx(&b->kfull[s], (uint32_t)rows * CK * 2);
        armed[s] = true;
        armed_par[s] = ph;
        const CUtensorMap *m64 = is_v ? &mV : &mK, *m16 = is_v ? &mV16 : &mK16;
        for (int bx = 0; bx < k_full; ++bx)
          tma_load_2d(dst + bx * 64 * CK * 2, m64, &b->kfull[s], col, row0 + bx * 64);
        for (int bx = 0; bx < k_rest; ++bx)
          tma_load_2d(dst + (k_full * 64 + bx * 16) * CK * 2, m16, &b->kfull[s], col,
                      row0 + k_full * 64 + bx * 16);
      }
      if (!ok)
        for (int s = 0; s < N_K; ++s)
          if (armed[s]) spin_bounded(&b->kfull[s], armed_par[s]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      bool ok = true;
      const uint32_t id = idesc_f16(1, 0, MB, TN);
      int kh = 0;
      for (int sl = 0; ok && sl < n_kc + n_ec; ++sl) {
        const int bs = sl % N_B;
        if (!mbar_wait(&b->bfull[bs], (sl / N_B) & 1, ab)) {
          ok = false;
          break;
        }
        const bool is_v = sl >= n_kc;
        const uint32_t ba = smem_u32(bring + bs * 2 * B_SLOT);
        const int k0 = is_v ? sl - n_kc : sl;  // slice index within the range
        for (int mb = 0; mb < n_mb; ++mb, ++kh) {
          const int s = kh % N_K;
          if (!mbar_wait(&b->kfull[s], (kh / N_K) & 1, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t aa = smem_u32(smem + s * K_STAGE);
          const uint32_t dcol = tmem + (is_v ? G_COL : 0) + mb * TN;
#pragma unroll
          for (int k = 0; k < CK / 16; ++k) {
            const uint64_t ad = sdesc_sw128(aa + k * 32, 16, 1024);
            umma_f16(dcol, ad, sdesc_sw128(ba + k * 32, 16, 1024), id, (k0 | k) != 0);
            if (is_v) umma_f16(dcol, ad, sdesc_sw128(ba + B_SLOT + k * 32, 16, 1024), id, 1);
          }
          umma_commit(&b->kempty[s]);
        }
        if (ok) umma_commit(&b->bempty[bs]);
      }
      if (ok) umma_commit(&b->done);
      if (!ok) {
        umma_commit(&b->drain);
        spin_bounded(&b->drain, 0);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ B operands
    // thread tw covers 16-byte chunk tw % 8 of token slots tw / 8 + 8 i
    const int tw = (warp - 2) * 32 + lane;  // 0..63
    const int ck = tw & 7, rb = tw >> 3;
    int src[TN / 8];
#pragma unroll
    for (int i = 0; i < TN / 8; ++i) {
      const int t = rb + 8 * i;
      src[i] = t < n_valid ? P.perm[tok0 + t] : -1;
    }
    bool ok = true;
    // x slices by cp.async, each handed over once the next one is issued
    int done = 0;
    for (int sl = 0; ok && sl < n_kc; ++sl) {
      const int bs = sl % N_B;
      ok = __all_sync(0xffffffffu, mbar_wait(&b->bempty[bs], ((sl / N_B) & 1) ^ 1, ab));
      if (!ok) break;
      uint8_t *hi = bring + bs * 2 * B_SLOT;
      const int col = sl * CK + ck * 8;
#pragma unroll
      for (int i = 0; i < TN / 8; ++i) {
        const int t = rb + 8 * i;
        cp_async16_zfill(hi + t * 128 + ((ck ^ rb) << 4),
                         P.x + (src[i] >= 0 ? (int64_t)src[i] * P.d_in + col : 0),
                         src[i] >= 0 ? 16u : 0u);
      }
      cp_async_commit();
      if (sl - done >= 1) {
        cp_async_wait_1();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b->bfull[done % N_B]);
        ++done;
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    __syncwarp();
    for (; ok && done < n_kc; ++done)
      if (lane == 0) mbar_arrive(&b->bfull[done % N_B]);
    // g_a slices: all of a slice's loads in flight at once, then the bf16
    // hi / lo parts
    for (int sl = n_kc; ok && sl < n_kc + n_ec; ++sl) {
      const int col = (sl - n_kc) * CK + ck * 8;
      float4 u[TN / 8][2];
#pragma unroll
      for (int i = 0; i < TN / 8; ++i) {
        u[i][0] = u[i][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (src[i] >= 0) {
          const float4 *gp = reinterpret_cast<const float4 *>(P.g_a + (int64_t)src[i] * P.d_emb + col);
          u[i][0] = gp[0];
          u[i][1] = gp[1];
        }
      }
      const int bs = sl % N_B;
      ok = __all_sync(0xffffffffu, mbar_wait(&b->bempty[bs], ((sl / N_B) & 1) ^ 1, ab));
      if (!ok) break;
      uint8_t *hi = bring + bs * 2 * B_SLOT, *lo = hi + B_SLOT;
#pragma unroll
      for (int i = 0; i < TN / 8; ++i) {
        const int t = rb + 8 * i;
        const float f[8] = {u[i][0].x, u[i][0].y, u[i][0].z, u[i][0].w,
                            u[i][1].x, u[i][1].y, u[i][1].z, u[i][1].w};
        uint4 h, l;
        uint32_t *hw = reinterpret_cast<uint32_t *>(&h), *lw = reinterpret_cast<uint32_t *>(&l);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 hh = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
          const float2 hf = __bfloat1622float2(hh);
          const __nv_bfloat162 ll = __floats2bfloat162_rn(f[2 * e] - hf.x, f[2 * e + 1] - hf.y);
          hw[e] = *reinterpret_cast<const uint32_t *>(&hh);
          lw[e] = *reinterpret_cast<const uint32_t *>(&ll);
        }
        *reinterpret_cast<uint4 *>(hi + t * 128 + ((ck ^ rb) << 4)) = h;
        *reinterpret_cast<uint4 *>(lo + t * 128 + ((ck ^ rb) << 4)) = l;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b->bfull[bs]);
    }
  } else {
    // ------------------------------------------------------------ softmax and g_s
    const int sw = warp - 4, q = warp & 3, half = sw / 4;
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&b->done, 0, ab));
    ok = sm_sync_and(ok);
    float m_t = -INFINITY, inv_t = 0.f, dot_t = 0.f;  // for token `lane`
    if (ok) {
      tc_fence_after();
      float m = -INFINITY;
      for (int mb = half; mb < n_mb; mb += 2) {
        const int j = mb * MB + q * 32 + lane;
        uint32_t v[TN];
        tmem_ld32(tq + mb * TN, v);
        tmem_wait_ld();
        float f[TN];
#pragma unroll
        for (int e = 0; e < TN; ++e) f[e] = j < d ? __uint_as_float(v[e]) : -INFINITY;
        m = fmaxf(m, warp_transpose_reduce<false>(f, lane));
      }
      b->red[0][sw][lane] = m;
    }
    ok = sm_sync_and(ok);
    if (ok) {
#pragma unroll
      for (int w = 0; w < 8; ++w) m_t = fmaxf(m_t, b->red[0][w][lane]);
      float s = 0.f, sg = 0.f;
      for (int mb = half; mb < n_mb; mb += 2) {
        const int j = mb * MB + q * 32 + lane;
        uint32_t v[TN], gv[TN];
        tmem_ld32(tq + mb * TN, v);
        tmem_ld32(tq + G_COL + mb * TN, gv);
        tmem_wait_ld();
        float e1[TN], e2[TN];
#pragma unroll
        for (int e = 0; e < TN; ++e) {
          const float mt = __shfl_sync(0xffffffffu, m_t, e);
          const float ex = j < d ? expf(__uint_as_float(v[e]) - mt) : 0.f;
          e1[e] = ex;
          // rows past d_t hold the next IDs' rows: 0 * Inf would be NaN
          e2[e] = j < d ? ex * __uint_as_float(gv[e]) : 0.f;
        }
        s += warp_transpose_reduce<true>(e1, lane);
        sg += warp_transpose_reduce<true>(e2, lane);
      }
      b->red[1][sw][lane] = s;
      b->red[2][sw][lane] = sg;
    }
    ok = sm_sync_and(ok);
    if (ok) {
      float s = 0.f, sg = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        s += b->red[1][w][lane];
        sg += b->red[2][w][lane];
      }
      inv_t = 1.f / s;
      dot_t = sg * inv_t;  // p . g_p
      float *pl0 = P.slots + (int64_t)ti * 2 * P.slot_rows * DENSE_TILE_M;
      float *pl1 = pl0 + (int64_t)P.slot_rows * DENSE_TILE_M;
      for (int mb = half; mb < n_mb; mb += 2) {
        const int j = mb * MB + q * 32 + lane;
        uint32_t v[TN], gv[TN];
        tmem_ld32(tq + mb * TN, v);
        tmem_ld32(tq + G_COL + mb * TN, gv);
        tmem_wait_ld();
        float *o0 = pl0 + (int64_t)j * DENSE_TILE_M + chunk * TN;
        float *o1 = pl1 + (int64_t)j * DENSE_TILE_M + chunk * TN;
        // every lane takes part in the shuffles; lanes at or past d store nothing
#pragma unroll
        for (int e = 0; e < TN; e += 4) {
          float4 pp, gs;
          float *pv = &pp.x, *gw = &gs.x;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float mt = __shfl_sync(0xffffffffu, m_t, e + k);
            const float it = __shfl_sync(0xffffffffu, inv_t, e + k);
            const float dt = __shfl_sync(0xffffffffu, dot_t, e + k);
            const float p = j < d ? expf(__uint_as_float(v[e + k]) - mt) * it : 0.f;
            pv[k] = p;
            gw[k] = p * (__uint_as_float(gv[e + k]) - dt);
          }
          if (j < d) {
            *reinterpret_cast<float4 *>(o0 + e) = pp;
            *reinterpret_cast<float4 *>(o1 + e) = gs;
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

constexpr size_t scores_smem() {
  return 1024 + N_K * K_STAGE + N_B * 2 * B_SLOT + sizeof(Bars);
}
static_assert(2 * (scores_smem() + 1024) <= 228 * 1024, "two CTAs per SM");

// ---------------------------------------------------------------------------
// dx_n += K_t^T g_s,n for the tokens of a dense tile, from the g_s plane the
// kernel above wrote: per (tile, 32-token chunk, 512 columns of d_in)
//     dx^T = K_t^T G_s     (M = 128 columns of d_in per block, N = 32, K = d_t)
// with K_t in 16-row slices as an MN-major A operand (TMA, two 64-column boxes
// per block) and G_s as a K-major B operand [token][row], bf16 hi + lo parts
// converted from the fp32 plane. Each token's dx row belongs to one chunk, so
// the epilogue adds into it without atomics: through a per-warp transpose,
// 16-byte read-modify-writes of eight tokens' 128-byte row pieces.
constexpr int DX_COLS = 512;                  // columns of d_in per CTA
constexpr int DX_MB = DX_COLS / MB;           // 4 M blocks (fewer in a last, partial group)
constexpr int DX_TMEM = DX_MB * TN;           // 128 TMEM columns
constexpr int DX_STAGE = V16_BOX() * (DX_COLS / 64);
constexpr int DX_NS = 2;                      // K_t slices in flight
constexpr int DX_THREADS = 192;               // 0 TMA, 1 MMA, 2-5 G_s conversion, then epilogue
constexpr int DX_P_BLOCK = TN * 128;          // 64 rows of G_s^T for the 32 tokens: 4 KB
constexpr int DX_WBUF = TN * TN * 4;          // fp32 32 x 32 transpose per epilogue warp

struct DxBars {
  uint64_t full[DX_NS], empty[DX_NS];
  uint64_t bready;  // the epilogue warps have written G_s^T
  uint64_t done;    // every MMA has completed
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(DX_THREADS, 2)
    k_bwd_dx_tc(const __grid_constant__ CUtensorMap mK16, Params P, float *__restrict__ dx) {
  constexpr int per_tile = DENSE_TILE_M / TN;
  const int n_cg = (P.d_in + DX_COLS - 1) / DX_COLS;
  const int ti = blockIdx.x / (per_tile * n_cg);
  const int chunk = (blockIdx.x / n_cg) % per_tile, cg = blockIdx.x % n_cg;
  const DenseTile tile = P.tiles[ti];
  const int g = tile.group;
  const int n_tile = min(DENSE_TILE_M, P.group_tok_start[g + 1] - tile.tok0);
  const int tok0 = tile.tok0 + chunk * TN;
  const int n_valid = min(TN, n_tile - chunk * TN);
  if (n_valid <= 0) return;  // the whole CTA, before any barrier or TMEM
  const int r0 = P.group_row_start[g], d = P.group_rows[g];
  const int d16 = (d + 15) & ~15, n_vc = d16 / 16;
  const int col0 = cg * DX_COLS;
  const int n_mb = min(DX_MB, (P.d_in - col0) / MB);  // d_in is a multiple of 128

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *ring = smem;                                   // DX_NS slices of K_t
  uint8_t *bhi = ring + DX_NS * DX_STAGE;                 // G_s^T hi, (d64 / 64) blocks of 4 KB
  uint8_t *blo = bhi + (MAX_D / 64) * DX_P_BLOCK;         // G_s^T lo
  // the epilogue's 4 transposes reuse G_s^T hi once every MMA has completed
  uint8_t *wbufs = bhi;
  static_assert(4 * DX_WBUF <= (MAX_D / 64) * DX_P_BLOCK, "transposes fit in G_s^T hi");
  DxBars *b = reinterpret_cast<DxBars *>(blo + (MAX_D / 64) * DX_P_BLOCK);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < DX_NS; ++s) {
      mbar_init(&b->full[s], 1);
      mbar_init(&b->empty[s], 1);
    }
    mbar_init(&b->bready, 4);
    mbar_init(&b->done, 1);
    mbar_init(&b->drain, 1);
    b->abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mK16);
  }
  if (warp == 1) {
    tmem_alloc(&b->tmem_base, DX_TMEM);
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
      bool armed[DX_NS];
      uint32_t armed_par[DX_NS];
      for (int i = 0; i < DX_NS; ++i) armed[i] = false;
      for (int vc = 0; ok && vc < n_vc; ++vc) {
        const int s = vc % DX_NS;
        const uint32_t ph = (vc / DX_NS) & 1;
        if (!mbar_wait(&b->empty[s], ph ^ 1, ab)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&b->full[s], (uint32_t)(2 * n_mb * V16_BOX()));
        armed[s] = true;
        armed_par[s] = ph;
        for (int bx = 0; bx < 2 * n_mb; ++bx)
          tma_load_2d(ring + s * DX_STAGE + bx * V16_BOX(), &mK16, &b->full[s], col0 + bx * 64,
                      r0 + vc * 16);
      }
      if (!ok)
        for (int s = 0; s < DX_NS; ++s)
          if (armed[s]) spin_bounded(&b->full[s], armed_par[s]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // lane 0 issues; the whole warp waits and zeroes, in the last slice, the
    // rows at or past d_t: they belong to the next IDs, and an Inf there
    // would meet a zero of G_s
    bool ok = __all_sync(0xffffffffu, mbar_wait(&b->bready, 0, ab));
    tc_fence_after();
    const uint32_t id = idesc_f16_amn(1, MB, TN);
    const uint32_t ph = smem_u32(bhi), pl = smem_u32(blo);
    for (int vc = 0; ok && vc < n_vc; ++vc) {
      const int s = vc % DX_NS;
      if (!__all_sync(0xffffffffu, mbar_wait(&b->full[s], (vc / DX_NS) & 1, ab))) {
        ok = false;
        break;
      }
      uint8_t *slice = ring + s * DX_STAGE;
      const int live = d - vc * 16;
      if (live < 16) {
        const int per_box = (16 - live) * 8;  // 16-byte pieces past d_t in a box
        uint4 *vb = reinterpret_cast<uint4 *>(slice);
        for (int e = lane; e < 2 * n_mb * per_box; e += 32) {
          const int bx = e / per_box, w = e - bx * per_box;
          vb[bx * (V16_BOX() / 16) + live * 8 + w] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t va = smem_u32(slice);
        const int kk = vc * 16;  // row of K_t: the K index of both operands
        const uint32_t boff = (kk / 64) * DX_P_BLOCK + (kk % 64) * 2;
        for (int mb = 0; mb < n_mb; ++mb) {
          const uint64_t ad = sdesc_sw128(va + 2 * mb * V16_BOX(), V16_BOX(), 1024);
          umma_f16(tmem + mb * TN, ad, sdesc_sw128(ph + boff, 16, 1024), id, vc != 0);
          umma_f16(tmem + mb * TN, ad, sdesc_sw128(pl + boff, 16, 1024), id, 1);
        }
        umma_commit(&b->empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) {
      if (ok) {
        umma_commit(&b->done);
      } else {
        umma_commit(&b->drain);
        spin_bounded(&b->drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ G_s^T, then the epilogue
    // warps 2-5: thread et takes rows et, et + 128, ... of the plane: its 32
    // tokens' g_s, split into bf16 hi / lo, into [token][row] (128-byte
    // swizzled 64-row blocks); rows from d up to d16 as zeros
    const int et = threadIdx.x - 64;  // 0..127
    const float *plane = P.slots + ((int64_t)ti * 2 + 1) * P.slot_rows * DENSE_TILE_M + chunk * TN;
    for (int j = et; j < d16; j += 128) {
      float f[TN];
#pragma unroll
      for (int e = 0; e < TN; e += 4) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j < d) v = *reinterpret_cast<const float4 *>(plane + (int64_t)j * DENSE_TILE_M + e);
        f[e] = v.x; f[e + 1] = v.y; f[e + 2] = v.z; f[e + 3] = v.w;
      }
      const int cj = (j % 64) / 8;
      uint8_t *ch = bhi + (j / 64) * DX_P_BLOCK + (j % 8) * 2;
      uint8_t *cl = blo + (j / 64) * DX_P_BLOCK + (j % 8) * 2;
#pragma unroll
      for (int t = 0; t < TN; ++t) {
        // tokens past the chunk's count enter as zero
        const float v = t < n_valid ? f[t] : 0.f;
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
        const int off = t * 128 + ((cj ^ (t & 7)) << 4);
        *reinterpret_cast<__nv_bfloat16 *>(ch + off) = h;
        *reinterpret_cast<__nv_bfloat16 *>(cl + off) = l;
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&b->bready);
    // epilogue: warp w reads TMEM lane quarter w % 4 of both blocks: column
    // col0 + 128 mb + 32 q + lane of d_in for the 32 tokens
    const int q = warp & 3;
    uint8_t *wbuf = wbufs + (warp - 2) * DX_WBUF;
    bool ok = __all_sync(0xffffffffu, mbar_wait(&b->done, 0, ab));
    const int my_tok = lane < n_valid ? P.perm[tok0 + lane] : -1;
    if (ok) {
      tc_fence_after();
      for (int mb = 0; mb < n_mb; ++mb) {
        uint32_t v[TN];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + mb * TN, v);
        tmem_wait_ld();
        // row t (token), column lane: 16-byte chunks XOR-swizzled by t & 7
#pragma unroll
        for (int t = 0; t < TN; ++t)
          *reinterpret_cast<uint32_t *>(wbuf + t * 128 + ((((lane >> 2) ^ (t & 7))) << 4) +
                                        (lane & 3) * 4) = v[t];
        __syncwarp();
        const int cb = col0 + mb * MB + q * 32;
#pragma unroll
        for (int k = 0; k < TN / 4; ++k) {
          const int t = k * 4 + (lane >> 3), c8 = lane & 7;  // 4 tokens x 8 chunks
          const float4 add =
              *reinterpret_cast<const float4 *>(wbuf + t * 128 + ((c8 ^ (t & 7)) << 4));
          const int tk = __shfl_sync(0xffffffffu, my_tok, t);
          if (tk >= 0) {
            float4 *o = reinterpret_cast<float4 *>(dx + (int64_t)tk * P.d_in + cb + c8 * 4);
            float4 cur = *o;
            cur.x += add.x; cur.y += add.y; cur.z += add.z; cur.w += add.w;
            *o = cur;
          }
        }
        __syncwarp();
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, DX_TMEM);
  }
}

constexpr size_t dx_smem() {
  return 1024 + DX_NS * DX_STAGE + 2 * (MAX_D / 64) * DX_P_BLOCK + sizeof(DxBars);
}
static_assert(2 * (dx_smem() + 1024) <= 228 * 1024, "two CTAs per SM");

}  // namespace

bool bwd_dx_tc_supported(const l3_dims_t &d) {
  return d.dtype == L3_BF16 && d.d_in % MB == 0 && d.k <= MAX_D;
}

l3_status launch_bwd_dx_tc(const l3_plan_s *p, const void *W_K, const float *slots, int slot_rows,
                           float *dx, cudaStream_t s) {
  if (p->n_dense_tiles == 0) return L3_OK;
  const l3_dims_t &d = p->dims;
  CUtensorMap mK16;
  l3_status st;
  if ((st = make_map_2d16(&mK16, W_K, true, (uint64_t)d.v, d.d_in, d.d_in, CK, 16, 128)) != L3_OK)
    return st;
  Params P = {};
  P.perm = p->perm;
  P.group_tok_start = p->group_tok_start;
  P.group_row_start = p->group_row_start;
  P.group_rows = p->group_rows;
  P.tiles = p->dense_tiles;
  P.slots = const_cast<float *>(slots);
  P.slot_rows = slot_rows;
  P.d_in = (int)d.d_in;
  P.d_emb = (int)d.d_emb;
  P.err = p->dev_flags + 1;
  static bool attr[64] = {};
  if (!attr[p->device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_bwd_dx_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)dx_smem()));
    attr[p->device & 63] = true;
  }
  const int64_t grid = p->n_dense_tiles * (DENSE_TILE_M / TN) * ((d.d_in + DX_COLS - 1) / DX_COLS);
  LaunchTimer t("bwd_dense_dx_tc", s);
  k_bwd_dx_tc<<<(unsigned)grid, DX_THREADS, dx_smem(), s>>>(mK16, P, dx);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

bool bwd_scores_tc_supported(const l3_dims_t &d) {
  return d.dtype == L3_BF16 && d.d_in % CK == 0 && d.d_emb % CK == 0 && d.k <= MAX_D;
}

l3_status launch_bwd_scores_tc(const l3_plan_s *p, const void *x, const void *W_K,
                               const void *W_V, const float *g_a, float *slots, int slot_rows,
                               cudaStream_t s) {
  if (p->n_dense_tiles == 0) return L3_OK;
  const l3_dims_t &d = p->dims;
  CUtensorMap mK, mK16, mV, mV16;
  l3_status st;
  const uint64_t rows = (uint64_t)d.v;
  if ((st = make_map_2d16(&mK, W_K, true, rows, d.d_in, d.d_in, CK, 64, 128)) != L3_OK) return st;
  if ((st = make_map_2d16(&mK16, W_K, true, rows, d.d_in, d.d_in, CK, 16, 128)) != L3_OK)
    return st;
  if ((st = make_map_2d16(&mV, W_V, true, rows, d.d_emb, d.d_emb, CK, 64, 128)) != L3_OK)
    return st;
  if ((st = make_map_2d16(&mV16, W_V, true, rows, d.d_emb, d.d_emb, CK, 16, 128)) != L3_OK)
    return st;
  Params P;
  P.x = reinterpret_cast<const __nv_bfloat16 *>(x);
  P.g_a = g_a;
  P.perm = p->perm;
  P.group_tok_start = p->group_tok_start;
  P.group_row_start = p->group_row_start;
  P.group_rows = p->group_rows;
  P.tiles = p->dense_tiles;
  P.slots = slots;
  P.slot_rows = slot_rows;
  P.d_in = (int)d.d_in;
  P.d_emb = (int)d.d_emb;
  P.err = p->dev_flags + 1;
  static bool attr[64] = {};
  if (!attr[p->device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_bwd_scores_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)scores_smem()));
    attr[p->device & 63] = true;
  }
  LaunchTimer t("bwd_dense_scores_tc", s);
  k_bwd_scores_tc<<<(unsigned)(p->n_dense_tiles * (DENSE_TILE_M / TN)), THREADS, scores_smem(), s>>>(
      mK, mK16, mV, mV16, P);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

}  // namespace l3
