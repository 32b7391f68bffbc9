// Tensor-core (tcgen05 + TMEM + TMA) GEMMs of the bf16 layer.
//
// kimjy99 review, Method, eq. L³:
//   h = LayerNorm(W_up a)                      (W_up: d_up x d_emb)
//   y = W_mix [h ; x] = W_mix[:, :d_up] h + W_mix[:, d_up:] x
//
// k_mix_gemm_pair: persistent, warp-specialised, on CTA pairs (cta_group::2).
// A pair computes a 256 x 256 tile of y: warp 0 of each CTA streams its own
// 128x64 A tiles and 128x64 half of the pair's B tiles into a 6-stage ring
// with TMA; warp 1 of the pair's first CTA issues tcgen05.mma (M=256, N=256,
// K=16) into one of two TMEM accumulators (each CTA's TMEM holds its 128
// rows); warps 2-5 of each CTA drain the other accumulator and store y while
// the next tile's MMAs run. The two K-ranges of W_mix (the LayerNorm output h,
// then x) accumulate into the same TMEM tile, so the concat [h ; x] never
// exists.
//
// k_up_ln_gemm: W_up a with the LayerNorm fused into the epilogue. A cluster
// of ceil(d_up / 256) CTAs covers one 128-token tile's whole d_up row: each
// CTA holds a 128 x 256 fp32 slice in TMEM, computes per-row (mean, M2) of
// its slice, the cluster exchanges them through distributed shared memory
// and merges them (Chan et al.'s pairwise update), and every CTA normalises
// its slice in place and stores h.
//
// Precision: h and a are fp16 and meet fp16 copies of W_mix[:, :d_up] and
// W_up (converted in k_to_f16), since tcgen05 kind::f16 needs both operands of
// one MMA in the same type; the x range stays bf16 x bf16.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "l3_internal.cuh"
#include "sm100.cuh"

namespace l3 {
namespace {

using namespace sm100;

constexpr int BM = 128;  // tokens per tile (TMEM lanes)
constexpr int BK = 64;   // 64 16-bit elements = one 128-byte swizzle row
constexpr int BN = 256;  // output columns per tile (max N of one MMA)
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int UP_STAGES = 2;  // two CTAs per SM: one drains its epilogue while the other computes
constexpr int GEMM_THREADS = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t IDESC_F16 = idesc_f16(0, 0, BM, BN);

struct MixParams {
  int M, N;        // tokens, d_out
  int kb0, kb1;    // 64-wide k-blocks of the h range and of the x range
  int n_tiles_n, n_tiles;
  void *y;         // bf16 (the layer's y) or fp32 (the backward pass's GEMMs)
  int64_t ldy;
  uint32_t idesc0, idesc1;  // instruction descriptors of the two ranges (fp32-output form)
  int *err;
};

struct UpParams {
  int M, N;        // tokens, d_up
  int kb;          // k-blocks of d_emb
  const __nv_bfloat16 *gamma, *beta;
  float eps;
  __half *h;
  int *err;
};

// shared-memory layout after the stage ring
struct Bars {
  uint64_t full[8], empty[8], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Make sure no TMA write or MMA is still in flight before the CTA frees TMEM
// and exits after a give-up. Normal runs have already waited for all of them.
__device__ void drain_after_abort(Bars *b, int stages, const uint32_t *armed_parity,
                                  const bool *armed, bool is_producer, bool is_mma,
                                  const Abort &ab) {
  (void)ab;  // the drain ignores the abort flag and keeps only the time bound
  if (is_producer) {
    for (int s = 0; s < stages; ++s)
      if (armed[s]) {
        // wait for the last armed phase; ignore the abort flag, keep the time bound
        const uint32_t a = smem_u32(&b->full[s]);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(a, armed_parity[s]) && globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
        }
      }
  }
  if (is_mma) {
    umma_commit(&b->drain);
    const uint32_t a = smem_u32(&b->drain);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
    }
  }
}

// ---------------------------------------------------------------------------
// y = W_mix[:, :d_up] h + W_mix[:, d_up:] x on CTA pairs (tcgen05 cta_group::2)
//
// The same kernel, instantiated with F32OUT, is the backward pass's NT GEMM
// C = A B^T with fp32 output (one K-range, operand types from the params).
//
// Two CTAs on neighbouring SMs compute one 256 x 256 tile of y: each loads its
// own 128 rows of the A operand (h or x) and its own 128 of the 256 rows of
// W_mix, and the pair's first CTA issues M = 256 MMAs that read both CTAs'
// shared memory and accumulate each CTA's 128 rows in its own TMEM. Per SM
// this moves 32 KB per 64-wide k-block instead of 48 KB (B is split between
// the two SMs instead of loaded by each), and a 32 KB stage lets six stages
// fit instead of four.
// ---------------------------------------------------------------------------
constexpr int MIX2_STAGES = 6;
constexpr int B2_ROWS = 128;                    // W_mix rows per CTA of a pair
constexpr int STAGE2_BYTES = A_BYTES + B2_ROWS * BK * 2;
constexpr uint32_t IDESC2_F16 = idesc_f16(0, 0, 2 * BM, BN);
constexpr uint32_t IDESC2_BF16 = idesc_f16(1, 0, 2 * BM, BN);

__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t cluster_addr,
                                                              uint32_t bytes) {
  // default (CTA-scope release) semantics: a cluster-scope release here is a
  // full memory fence per stage, which starved the pipeline
  asm volatile("mbarrier.arrive.expect_tx.shared::cluster.b64 _, [%0], %1;" ::"r"(
                   cluster_addr),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (no multicast)
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map,
                                                 uint32_t bar_cluster_addr, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(bar_cluster_addr), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on `bar` (same offset) in both CTAs of the pair once every MMA issued
// so far by this thread has completed
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}

template <bool F32OUT>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_mix_gemm_pair(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mB0,
                    const __grid_constant__ CUtensorMap mA1, const __grid_constant__ CUtensorMap mB1,
                    MixParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *ring = smem;
  Bars *b = reinterpret_cast<Bars *>(smem + MIX2_STAGES * STAGE2_BYTES);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();  // 0 issues the MMAs
  const int pair_id = blockIdx.x / 2, n_pairs = gridDim.x / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < MIX2_STAGES; ++s) {
      mbar_init(&b->full[s], 2);   // used in CTA 0: one arrival per CTA, plus both CTAs' bytes
      mbar_init(&b->empty[s], 1);  // MMA completion, signalled in both CTAs
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&b->tfull[a], 1);
      mbar_init(&b->tempty[a], 8);  // used in CTA 0: four epilogue warps of each CTA
    }
    mbar_init(&b->drain, 1);
    b->abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mA0);
    prefetch_tensormap(&mB0);
    prefetch_tensormap(&mA1);
    prefetch_tensormap(&mB1);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&b->tmem_base)),
                 "r"(2 * BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = b->tmem_base;
  const Abort ab{&b->abort_flag, P.err};
  const int n_kb = P.kb0 + P.kb1;

  if (warp == 0) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed_parity[MIX2_STAGES];
      bool armed[MIX2_STAGES];
      for (int s = 0; s < MIX2_STAGES; ++s) armed[s] = false;
      bool ok = true;
      for (int tile = pair_id; ok && tile < P.n_tiles; tile += n_pairs) {
        const int m0 = (tile / P.n_tiles_n) * (2 * BM) + (int)rank * BM;
        const int n0 = (tile % P.n_tiles_n) * BN + (int)rank * B2_ROWS;
        for (int kb = 0; kb < n_kb; ++kb) {
          if (!mbar_wait(&b->empty[stage], phase ^ 1, ab)) {
            ok = false;
            break;
          }
          uint8_t *sa = ring + stage * STAGE2_BYTES;
          const uint32_t full0 = map_shared_rank(&b->full[stage], 0);
          mbar_arrive_expect_tx_cluster(full0, STAGE2_BYTES);
          armed[stage] = true;
          armed_parity[stage] = phase;
          if (kb < P.kb0) {
            tma_load_2d_pair(sa, &mA0, full0, kb * BK, m0);
            tma_load_2d_pair(sa + A_BYTES, &mB0, full0, kb * BK, n0);
          } else {
            tma_load_2d_pair(sa, &mA1, full0, (kb - P.kb0) * BK, m0);
            tma_load_2d_pair(sa + A_BYTES, &mB1, full0, (kb - P.kb0) * BK, n0);
          }
          if (++stage == MIX2_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // after a give-up CTA 0 waits for the phases it armed, which complete
      // only once both CTAs' copies have landed
      if (!ok && rank == 0) drain_after_abort(b, MIX2_STAGES, armed_parity, armed, true, false, ab);
    }
  } else if (warp == 1) {
    if (rank == 0 && elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = pair_id; ok && tile < P.n_tiles; tile += n_pairs, ++it) {
        const int acc = it & 1;
        if (!mbar_wait(&b->tempty[acc], ((it >> 1) & 1) ^ 1, ab)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = 0; kb < n_kb; ++kb) {
          if (!mbar_wait(&b->full[stage], phase, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + stage * STAGE2_BYTES);
          const uint32_t sb = sa + A_BYTES;
          const uint32_t idesc = F32OUT ? (kb < P.kb0 ? P.idesc0 : P.idesc1)
                                        : (kb < P.kb0 ? IDESC2_F16 : IDESC2_BF16);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_f16_pair(d, sdesc_sw128(sa + k * 32, 16, 1024), sdesc_sw128(sb + k * 32, 16, 1024),
                          idesc, (kb | k) != 0);
          umma_commit_pair(&b->empty[stage]);
          if (++stage == MIX2_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) umma_commit_pair(&b->tfull[acc]);
      }
      if (!ok) {
        umma_commit_pair(&b->drain);
        const uint32_t a = smem_u32(&b->drain);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
        }
      }
    }
  } else {
    // epilogue: warp (2..5) % 4 selects the TMEM lane quarter it may read;
    // each CTA drains its own 128 rows of the pair's tile
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t tempty0[2] = {map_shared_rank(&b->tempty[0], 0),
                                 map_shared_rank(&b->tempty[1], 0)};
    int it = 0;
    for (int tile = pair_id; tile < P.n_tiles; tile += n_pairs, ++it) {
      const int acc = it & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&b->tfull[acc], (it >> 1) & 1, ab));
      if (!got) break;
      tc_fence_after();
      const int m = (tile / P.n_tiles_n) * (2 * BM) + (int)rank * BM + r;
      const int n0 = (tile % P.n_tiles_n) * BN;
      __nv_bfloat16 *yrow = reinterpret_cast<__nv_bfloat16 *>(P.y) + (int64_t)m * P.ldy + n0;
      float *crow = reinterpret_cast<float *>(P.y) + (int64_t)m * P.ldy + n0;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + acc * BN + c * 32, v);
        tmem_wait_ld();
        if (F32OUT) {
          if (m < P.M) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (n0 + c * 32 + j * 4 < P.N)
                *reinterpret_cast<uint4 *>(crow + c * 32 + j * 4) =
                    make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
        } else if (m < P.M) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int col = n0 + c * 32 + j * 8;
            if (col < P.N) {
              uint4 o;
              __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                o2[e] = __floats2bfloat162_rn(__uint_as_float(v[j * 8 + 2 * e]),
                                              __uint_as_float(v[j * 8 + 2 * e + 1]));
              *reinterpret_cast<uint4 *>(yrow + c * 32 + j * 8) = o;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0[acc]);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no signal crosses between the CTAs after this
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * BN)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// h = LayerNorm(W_up a), one cluster of ceil(d_up / 256) CTAs per 128 tokens
// ---------------------------------------------------------------------------
constexpr int UP_THREADS = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue

// barrier of the 256 epilogue threads of k_up_ln_gemm that ANDs a flag across them
__device__ __forceinline__ bool epi_sync_and(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, 256, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}

// (n_a, mean_a, M2_a) <- (n_a, mean_a, M2_a) (+) (n_b, mean_b, M2_b): Chan,
// Golub and LeVeque's pairwise update of a mean and a sum of squared deviations
__device__ __forceinline__ void chan_merge(float &n_a, float &mean_a, float &m2_a, float n_b,
                                           float mean_b, float m2_b) {
  const float n = n_a + n_b;
  if (n_b == 0.f) return;
  const float delta = mean_b - mean_a;
  mean_a += delta * (n_b / n);
  m2_a += m2_b + delta * delta * (n_a * n_b / n);
  n_a = n;
}

__device__ __forceinline__ void st_shared_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int x,
                                             int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
      "r"(smem_u32(src)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_and_wait_all() {
  asm volatile("cp.async.bulk.commit_group;\n\tcp.async.bulk.wait_group 0;" ::: "memory");
}

__global__ void __launch_bounds__(UP_THREADS, 2)
    k_up_ln_gemm(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB,
                 const __grid_constant__ CUtensorMap mH, UpParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *ring = smem;
  Bars *b = reinterpret_cast<Bars *>(smem + UP_STAGES * STAGE_BYTES);
  float *g_s = reinterpret_cast<float *>(b + 1);  // gamma of this CTA's 256 columns
  float *b_s = g_s + BN;                          // beta
  float(*red)[BM] = reinterpret_cast<float(*)[BM]>(b_s + BN);  // [4][BM]: mean, M2 of two halves
  // [2][8][BM]: every slice's (mean, M2) per row, written by the cluster's CTAs
  float(*st_all)[8][BM] = reinterpret_cast<float(*)[8][BM]>(red[4]);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const uint32_t n_ranks = gridDim.x;  // one cluster spans the grid's x dimension
  const int m0 = blockIdx.y * BM;
  const int n0 = (int)rank * BN;
  const int n_valid = min(BN, P.N - n0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < UP_STAGES; ++s) {
      mbar_init(&b->full[s], 1);
      mbar_init(&b->empty[s], 1);
    }
    mbar_init(&b->tfull[0], 1);
    mbar_init(&b->drain, 1);
    b->abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mA);
    prefetch_tensormap(&mB);
  }
  if (warp == 1) {
    tmem_alloc(&b->tmem_base, BN);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < BN; i += UP_THREADS) {
    const bool v = n0 + i < P.N;
    g_s[i] = v ? __bfloat162float(P.gamma[n0 + i]) : 0.f;
    b_s[i] = v ? __bfloat162float(P.beta[n0 + i]) : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // first phase of the cluster barrier: every CTA of the cluster has started
  // before any writes into another's shared memory (waited on before that)
  cluster_arrive_relaxed();
  const uint32_t tmem = b->tmem_base;
  const Abort ab{&b->abort_flag, P.err};

  if (warp == 0) {
    if (elect_one()) {
      uint32_t armed_parity[UP_STAGES];
      bool armed[UP_STAGES];
      for (int s = 0; s < UP_STAGES; ++s) armed[s] = false;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < P.kb; ++kb) {
        if (!mbar_wait(&b->empty[stage], phase ^ 1, ab)) {
          ok = false;
          break;
        }
        uint8_t *sa = ring + stage * STAGE_BYTES;
        mbar_arrive_expect_tx(&b->full[stage], STAGE_BYTES);
        armed[stage] = true;
        armed_parity[stage] = phase;
        tma_load_2d(sa, &mA, &b->full[stage], kb * BK, m0);
        tma_load_2d(sa + A_BYTES, &mB, &b->full[stage], kb * BK, n0);
        if (++stage == UP_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) drain_after_abort(b, UP_STAGES, armed_parity, armed, true, false, ab);
    }
  } else if (warp == 1) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < P.kb; ++kb) {
        if (!mbar_wait(&b->full[stage], phase, ab)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(ring + stage * STAGE_BYTES);
        const uint32_t sb = sa + A_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          umma_f16(tmem, sdesc_sw128(sa + k * 32, 16, 1024), sdesc_sw128(sb + k * 32, 16, 1024),
                   IDESC_F16, (kb | k) != 0);
        umma_commit(&b->empty[stage]);
        if (++stage == UP_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (ok) umma_commit(&b->tfull[0]);
      else drain_after_abort(b, UP_STAGES, nullptr, nullptr, false, true, ab);
    }
  }

  // epilogue part 1: per-row (mean, M2) of this CTA's slice in one pass over
  // TMEM. Warps 2-9, two per TMEM lane quarter; each takes every other
  // 32-column chunk, takes each chunk's exact mean and M2 in registers and
  // merges chunks, then the two halves of a row merge through shared memory.
  const bool epi = warp >= 2;
  const int q = warp & 3;
  const int half = (warp - 2) / 4;
  const int r = q * 32 + lane;
  const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
  bool have = false;
  __syncwarp();
  if (epi) {
    have = __all_sync(0xffffffffu, mbar_wait(&b->tfull[0], 0, ab));
    have = epi_sync_and(have);
    tc_fence_after();
    float n_acc = 0.f, mean_acc = 0.f, m2_acc = 0.f;
    if (have) {
#pragma unroll 1
      for (int c = half; c < BN / 32; c += 2) {
        const int nv = min(32, n_valid - c * 32);
        if (nv <= 0) break;
        uint32_t v[32];
        tmem_ld32(trow + c * 32, v);
        tmem_wait_ld();
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nv) sum += __uint_as_float(v[j]);
        const float mc = sum / (float)nv;
        float qc = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nv) {
            const float dlt = __uint_as_float(v[j]) - mc;
            qc = fmaf(dlt, dlt, qc);
          }
        chan_merge(n_acc, mean_acc, m2_acc, (float)nv, mc, qc);
      }
    }
    red[2 * half][r] = mean_acc;
    red[2 * half + 1][r] = m2_acc;
    epi_sync_and(true);
    if (half == 0) {
      // this slice's statistics go to every CTA of the cluster (this one
      // included); the other half's column count follows from n_valid
      float n1 = 0.f;
      for (int c = 1; c < BN / 32; c += 2) n1 += (float)max(0, min(32, n_valid - c * 32));
      chan_merge(n_acc, mean_acc, m2_acc, n1, red[2][r], red[3][r]);
      // wait for the start-up phase (every CTA of the cluster is running)
      asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
      for (uint32_t j = 0; j < n_ranks; ++j) {
        st_shared_cluster_f32(map_shared_rank(&st_all[0][rank][r], j), mean_acc);
        st_shared_cluster_f32(map_shared_rank(&st_all[1][rank][r], j), m2_acc);
      }
    } else {
      asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    }
  } else {
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  }
  __syncwarp();
  // second phase: every CTA's statistics have landed in every CTA; nothing is
  // read from or written to another CTA's shared memory after this
  cluster_arrive_release();
  cluster_wait_acquire();

  if (epi) {
    // merge the slices in rank order
    float n_acc = 0.f, mean_acc = 0.f, m2_acc = 0.f;
#pragma unroll 1
    for (uint32_t j = 0; j < n_ranks; ++j)
      chan_merge(n_acc, mean_acc, m2_acc, (float)min(BN, P.N - (int)j * BN), st_all[0][j][r],
                 st_all[1][j][r]);
    const float mu = mean_acc;
    const float rstd = 1.0f / sqrtf(m2_acc / n_acc + P.eps);
    // normalise into the (now idle) stage ring in the 128-byte-swizzled layout
    // of 64-column TMA boxes, then one thread stores the boxes with TMA
    if (have) {
#pragma unroll 1
      for (int c = half; c < BN / 32; c += 2) {
        if (c * 32 >= n_valid) break;
        uint32_t v[32];
        tmem_ld32(trow + c * 32, v);
        tmem_wait_ld();
        uint8_t *box = ring + (c / 2) * (BM * 128);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 o;
          __half2 *o2 = reinterpret_cast<__half2 *>(&o);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k0 = c * 32 + j * 8 + 2 * e;
            const float h0 = g_s[k0] * ((__uint_as_float(v[j * 8 + 2 * e]) - mu) * rstd) + b_s[k0];
            const float h1 =
                g_s[k0 + 1] * ((__uint_as_float(v[j * 8 + 2 * e + 1]) - mu) * rstd) + b_s[k0 + 1];
            o2[e] = __floats2half2_rn(h0, h1);
          }
          const int chunk = (c % 2) * 4 + j;  // 16-byte chunk within the box's 128-byte row
          *reinterpret_cast<uint4 *>(box + r * 128 + ((chunk ^ (r & 7)) << 4)) = o;
        }
      }
    }
    fence_proxy_async_smem();
    have = epi_sync_and(have);
    if (have && warp == 2 && lane == 0) {
      for (int bx = 0; bx * 64 < n_valid; ++bx)
        tma_store_2d(&mH, ring + bx * (BM * 128), n0 + bx * 64, m0);
      bulk_commit_and_wait_all();
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

// bf16 -> fp16 copy of a row-strided matrix; flags values outside fp16's range
__global__ void k_to_f16(const __nv_bfloat16 *__restrict__ src, int64_t ld_src, int64_t rows,
                         int64_t cols, __half *__restrict__ dst, int *err) {
  const int64_t vec_per_row = cols / 8;
  const int64_t total = rows * vec_per_row;
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / vec_per_row, c = (i - r * vec_per_row) * 8;
    uint4 v = *reinterpret_cast<const uint4 *>(src + r * ld_src + c);
    const __nv_bfloat162 *in = reinterpret_cast<const __nv_bfloat162 *>(&v);
    uint4 o;
    __half2 *out = reinterpret_cast<__half2 *>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(in[e]);
      bad |= fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f;
      out[e] = __floats2half2_rn(f.x, f.y);
    }
    *reinterpret_cast<uint4 *>(dst + r * cols + c) = o;
  }
  if (bad) atomicOr(err, DEV_ERR_F16_RANGE);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
int g_num_sms[64] = {};

l3_status encoder(PFN_cuTensorMapEncodeTiled_v12000 *out) {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void *fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) {
    set_error("cuTensorMapEncodeTiled is not available from the driver");
    return L3_ERR_CUDA;
  }
  *out = g_encode;
  return L3_OK;
}

// 2-D row-major [rows x cols] tensor of 16-bit elements, row stride ld elements,
// box = 64 columns x box_rows rows, 128-byte swizzle, zero fill out of bounds.
l3_status make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint64_t rows,
                   uint64_t cols, uint64_t ld, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  l3_status st = encoder(&enc);
  if (st != L3_OK) return st;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
    return L3_ERR_CUDA;
  }
  return L3_OK;
}

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  dev &= 63;
  if (g_num_sms[dev] == 0) cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
  return g_num_sms[dev];
}

constexpr size_t MIX2_SMEM = 1024 + MIX2_STAGES * STAGE2_BYTES + sizeof(Bars);
constexpr size_t UP_SMEM =
    1024 + UP_STAGES * STAGE_BYTES + sizeof(Bars) + (2 * BN + 4 * BM + 2 * 8 * BM) * sizeof(float);
static_assert(UP_STAGES * STAGE_BYTES >= (BN / 64) * BM * 128, "h staging fits the stage ring");

}  // namespace

l3_status make_map_2d16(CUtensorMap *m, const void *base, bool bf16, uint64_t rows, uint64_t cols,
                        uint64_t ld, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  l3_status st = encoder(&enc);
  if (st != L3_OK) return st;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                   const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
    return L3_ERR_CUDA;
  }
  return L3_OK;
}

bool tc_gemm_supported(const l3_dims_t &d) {
  return d.dtype == L3_BF16 && d.d_in % BK == 0 && d.d_emb % BK == 0 && d.d_up % BK == 0 &&
         d.d_up <= 8 * BN;
}

l3_status launch_weights_f16(const l3_plan_s *p, const void *W_up, const void *W_mix,
                             cudaStream_t s) {
  const l3_dims_t &d = p->dims;
  int *err = p->dev_flags + 1;
  {
    LaunchTimer t("to_f16", s);
    k_to_f16<<<num_sms() * 4, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16 *>(W_up), d.d_emb,
                                           d.d_up, d.d_emb, reinterpret_cast<__half *>(p->w_up16),
                                           err);
    k_to_f16<<<num_sms() * 4, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16 *>(W_mix),
                                           d.d_up + d.d_in, d.d_out, d.d_up,
                                           reinterpret_cast<__half *>(p->w_mixh16), err);
  }
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

l3_status launch_up_ln_tc(const l3_plan_s *p, const void *gamma, const void *beta,
                          cudaStream_t s) {
  const l3_dims_t &d = p->dims;
  CUtensorMap mA, mB;
  l3_status st;
  if ((st = make_map(&mA, p->a_buf, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p->n_tokens, d.d_emb, d.d_emb,
                     BM)) != L3_OK)
    return st;
  if ((st = make_map(&mB, p->w_up16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, d.d_up, d.d_emb, d.d_emb,
                     BN)) != L3_OK)
    return st;
  CUtensorMap mH;  // h is written with TMA from 64-column, 128-row boxes
  if ((st = make_map(&mH, p->h_buf, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p->n_tokens, d.d_up, d.d_up,
                     BM)) != L3_OK)
    return st;
  UpParams P;
  P.M = (int)p->n_tokens;
  P.N = (int)d.d_up;
  P.kb = (int)(d.d_emb / BK);
  P.gamma = reinterpret_cast<const __nv_bfloat16 *>(gamma);
  P.beta = reinterpret_cast<const __nv_bfloat16 *>(beta);
  P.eps = d.ln_eps;
  P.h = reinterpret_cast<__half *>(p->h_buf);
  P.err = p->dev_flags + 1;
  static bool attr[64] = {};
  if (!attr[p->device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_up_ln_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)UP_SMEM));
    attr[p->device & 63] = true;
  }
  const int cn = (int)((d.d_up + BN - 1) / BN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cn, (unsigned)((p->n_tokens + BM - 1) / BM), 1);
  cfg.blockDim = dim3(UP_THREADS, 1, 1);
  cfg.dynamicSmemBytes = UP_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cn;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  LaunchTimer t("up_ln_gemm_tc", s);
  L3_CUDA_TRY(cudaLaunchKernelEx(&cfg, k_up_ln_gemm, mA, mB, mH, P));
  return L3_OK;
}

l3_status launch_mix_tc(const l3_plan_s *p, const void *x, const void *W_mix, void *y,
                        cudaStream_t s) {
  const l3_dims_t &d = p->dims;
  CUtensorMap mA0, mB0, mA1, mB1;
  l3_status st;
  const uint64_t M = p->n_tokens;
  // A: 128-row boxes of h and x (each CTA of a pair loads its own rows);
  // B: 128-row halves of the pair's 256 W_mix rows
  if ((st = make_map(&mA0, p->h_buf, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, M, d.d_up, d.d_up, BM)) !=
      L3_OK)
    return st;
  if ((st = make_map(&mB0, p->w_mixh16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, d.d_out, d.d_up, d.d_up,
                     B2_ROWS)) != L3_OK)
    return st;
  if ((st = make_map(&mA1, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, M, d.d_in, d.d_in, BM)) != L3_OK)
    return st;
  const __nv_bfloat16 *wx = reinterpret_cast<const __nv_bfloat16 *>(W_mix) + d.d_up;
  if ((st = make_map(&mB1, wx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d.d_out, d.d_in, d.d_up + d.d_in,
                     B2_ROWS)) != L3_OK)
    return st;
  MixParams P;
  P.M = (int)M;
  P.N = (int)d.d_out;
  P.kb0 = (int)(d.d_up / BK);
  P.kb1 = (int)(d.d_in / BK);
  P.n_tiles_n = (int)((d.d_out + BN - 1) / BN);
  P.n_tiles = (int)((M + 2 * BM - 1) / (2 * BM)) * P.n_tiles_n;
  P.y = y;
  P.ldy = d.d_out;
  P.idesc0 = IDESC2_F16;
  P.idesc1 = IDESC2_BF16;
  P.err = p->dev_flags + 1;
  static bool attr[64] = {};
  if (!attr[p->device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_mix_gemm_pair<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)MIX2_SMEM));
    attr[p->device & 63] = true;
  }
  // persistent: one CTA pair per two SMs, 256 x 256 tiles
  const int pairs = std::min(P.n_tiles, num_sms() / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = MIX2_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  LaunchTimer t("mix_gemm_tc", s);
  L3_CUDA_TRY(cudaLaunchKernelEx(&cfg, k_mix_gemm_pair<false>, mA0, mB0, mA1, mB1, P));
  return L3_OK;
}

l3_status launch_gemm_nt_tc(const void *A, const void *B, const void *A1, const void *B1, bool f16,
                            int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, float *C,
                            int64_t ldc, int *err, int device, cudaStream_t s) {
  if (M == 0 || N == 0) return L3_OK;
  if (!A1 != !B1) {
    set_error("launch_gemm_nt_tc: the second range needs both operands");
    return L3_ERR_INVALID_ARG;
  }
  const uintptr_t mis = reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) |
                        reinterpret_cast<uintptr_t>(A1) | reinterpret_cast<uintptr_t>(B1) |
                        reinterpret_cast<uintptr_t>(C);
  if (K < 1 || M > INT32_MAX || N > INT32_MAX || (mis & 15) || lda % 8 || ldb % 8 || ldc % 4 ||
      N % 4 || lda < K || ldb < K || ldc < N) {
    set_error("launch_gemm_nt_tc: shape, stride or alignment outside the kernel's layout");
    return L3_ERR_UNSUPPORTED;
  }
  const CUtensorMapDataType dt =
      f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap mA, mB, mA1, mB1;
  l3_status st;
  if ((st = make_map(&mA, A, dt, M, K, lda, BM)) != L3_OK) return st;
  if ((st = make_map(&mB, B, dt, N, K, ldb, B2_ROWS)) != L3_OK) return st;
  if (A1) {
    if ((st = make_map(&mA1, A1, dt, M, K, lda, BM)) != L3_OK) return st;
    if ((st = make_map(&mB1, B1, dt, N, K, ldb, B2_ROWS)) != L3_OK) return st;
  } else {
    mA1 = mA;  // never read (kb1 = 0)
    mB1 = mB;
  }
  MixParams P;
  P.M = (int)M;
  P.N = (int)N;
  P.kb0 = (int)((K + BK - 1) / BK);  // the K tail is zero-filled by TMA in both operands
  P.kb1 = A1 ? P.kb0 : 0;
  P.n_tiles_n = (int)((N + BN - 1) / BN);
  P.n_tiles = (int)((M + 2 * BM - 1) / (2 * BM)) * P.n_tiles_n;
  P.y = C;
  P.ldy = ldc;
  P.idesc0 = P.idesc1 = f16 ? IDESC2_F16 : IDESC2_BF16;
  P.err = err;
  static bool attr[64] = {};
  if (!attr[device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_mix_gemm_pair<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)MIX2_SMEM));
    attr[device & 63] = true;
  }
  const int pairs = std::min(P.n_tiles, num_sms() / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = MIX2_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  L3_CUDA_TRY(cudaLaunchKernelEx(&cfg, k_mix_gemm_pair<true>, mA, mB, mA1, mB1, P));
  return L3_OK;
}

}  // namespace l3
