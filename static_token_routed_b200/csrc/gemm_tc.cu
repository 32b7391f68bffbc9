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

struct MixParams {
  int M, N;        // rows (tokens), output columns
  int kb0, kb1;    // 64-wide k-blocks of the first range (z, or A) and of the second (x, or A1)
  int n_tiles_n, n_tiles;
  void *y;         // bf16 y (MODE_MIX_LN), fp32 C (MODE_F32) or fp16 z (MODE_UP_Z)
  int64_t ldy;
  uint32_t idesc0, idesc1;  // instruction descriptors of the two ranges (MODE_F32)
  // MODE_UP_Z writes, MODE_MIX_LN reads: (mean, M2) of each row over each
  // 256-column tile of z, [n_chunks][M] (a warp's 32 rows are adjacent)
  float2 *stats;
  int n_chunks;
  const float *ccol, *dcol;  // MODE_MIX_LN: c = W' 1 and d = W_mix[:, :d_up] beta, [N] each
  float eps;
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

// Packed pairs of fp32 lanes (sm_100a `.f32x2` arithmetic): half the issue
// slots of scalar adds and FMAs in the z epilogue's row statistics.
__device__ __forceinline__ uint64_t f2_pack(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ float f2_hsum(uint64_t a) {
  uint32_t lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(a));
  return __uint_as_float(lo) + __uint_as_float(hi);
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// mean and sum of squared deviations of 32 fp32 values, in two passes (the
// mean first, then the deviations from it), lanes paired, two partial sums
// per pass
__device__ __forceinline__ void stats32(const uint32_t (&v)[32], float &mean, float &m2) {
  uint64_t s0 = f2_pack(v[0], v[1]), s1 = f2_pack(v[2], v[3]);
#pragma unroll
  for (int e = 4; e < 32; e += 4) {
    s0 = f2_add(s0, f2_pack(v[e], v[e + 1]));
    s1 = f2_add(s1, f2_pack(v[e + 2], v[e + 3]));
  }
  mean = f2_hsum(f2_add(s0, s1)) * (1.f / 32.f);
  const uint64_t mm = f2_pack(__float_as_uint(mean), __float_as_uint(mean));
  uint64_t q0 = 0, q1 = 0;  // (+0.f, +0.f)
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const uint64_t d0 = f2_sub(f2_pack(v[e], v[e + 1]), mm);
    const uint64_t d1 = f2_sub(f2_pack(v[e + 2], v[e + 3]), mm);
    q0 = f2_fma(d0, d0, q0);
    q1 = f2_fma(d1, d1, q1);
  }
  m2 = f2_hsum(f2_add(q0, q1));
}

// Kernel forms:
//   MODE_F32:    C = A B^T (+ A1 B1^T), fp32 output (the backward pass's GEMMs)
//   MODE_UP_Z:   z = a W_up^T, fp16 output through shared memory and TMA stores,
//                plus each row's (mean, M2) over each 256-column tile of z
//   MODE_MIX_LN: y = W_mix [LayerNorm(z) ; x] with the LayerNorm folded into the
//                accumulator (see below)
//
// MODE_MIX_LN. With W' = W_mix[:, :d_up] diag(gamma), c = W' 1 and
// d = W_mix[:, :d_up] beta, for a row with mean mu and 1 / std r,
//     W_mix[:, :d_up] LayerNorm(z) = r (W' z - mu c) + d,
// so the kernel accumulates W' z over the z range, the epilogue warps rewrite
// that accumulator in TMEM as r (acc - mu c) + d, and the x range then
// accumulates W_mix[:, d_up:] x on top. To keep the tensor cores busy while a
// tile's accumulator is being rewritten, a pair runs its tiles two at a time:
//     z(t) -> acc 0, z(t+1) -> acc 1, x(t) -> acc 0, x(t+1) -> acc 1
// and the epilogue warps follow: rewrite t, rewrite t+1, store t, store t+1.
enum : int { MODE_F32 = 0, MODE_UP_Z = 1, MODE_MIX_LN = 2 };

template <int MODE>
struct MixCfg {
  static constexpr int STAGES = MODE == MODE_UP_Z ? 4 : MIX2_STAGES;
  // epilogue warps: four per TMEM lane quarter for MODE_UP_Z, whose epilogue
  // has only d_emb / 64 k-blocks of MMAs to hide behind; one per quarter otherwise
  static constexpr int EPI_WARPS = MODE == MODE_UP_Z ? 16 : 4;
  // MODE_UP_Z: 128 rows x 256 columns of fp16 z, four 64-column TMA boxes,
  // then the (count, mean, M2) of each row over the chunks of warps 2-3 of a quarter
  static constexpr int STAGING =
      MODE == MODE_UP_Z ? (BN / 64) * BM * 128 + (EPI_WARPS / 4 - 1) * 3 * BM * 4 : 0;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
};

// The j-th (tile, range, accumulator) job of a pair that owns `k_tiles`
// tiles; false past the last. Ranges: 0 = the first k-range (or both, when
// the kernel does not split them), 1 = the second.
template <int MODE>
__device__ __forceinline__ bool mix_job(int j, int k_tiles, int &k, int &rng, int &acc) {
  if (MODE != MODE_MIX_LN) {
    if (j >= k_tiles) return false;
    k = j;
    rng = 0;
    acc = j & 1;
    return true;
  }
  const int n_full = k_tiles / 2;
  if (j < 4 * n_full) {
    const int w = j & 3;
    k = 2 * (j >> 2) + (w & 1);
    rng = w >> 1;
    acc = w & 1;
    return true;
  }
  const int j2 = j - 4 * n_full;
  if ((k_tiles & 1) && j2 < 2) {
    k = 2 * n_full;
    rng = j2;
    acc = 0;
    return true;
  }
  return false;
}

// barriers of the epilogue warps (N threads): a plain one, and one that ANDs
// a flag across them so that they leave their loop together
template <int N>
__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ bool epi_sync_and(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 2, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "n"(N)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void tma_store_2d_box(const CUtensorMap *map, const void *src, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
      "r"(smem_u32(src)), "r"(x), "r"(y)
      : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(MixCfg<MODE>::THREADS, 1)
    k_mix_gemm_pair(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mB0,
                    const __grid_constant__ CUtensorMap mA1, const __grid_constant__ CUtensorMap mB1,
                    const __grid_constant__ CUtensorMap mZ, MixParams P) {
  using Cfg = MixCfg<MODE>;
  // MODE_UP_Z's constant-weight statistics merge: two 32-column chunks per warp
  static_assert(MODE != MODE_UP_Z || BN / 32 == 2 * (Cfg::EPI_WARPS / 4), "z epilogue chunk split");
  constexpr int STAGES = Cfg::STAGES;
  constexpr int EPI_T = 32 * Cfg::EPI_WARPS;  // epilogue threads
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *ring = smem;
  uint8_t *staging = smem + STAGES * STAGE2_BYTES;  // MODE_UP_Z
  Bars *b = reinterpret_cast<Bars *>(staging + Cfg::STAGING);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();  // 0 issues the MMAs
  const int pair_id = blockIdx.x / 2, n_pairs = gridDim.x / 2;
  const int k_tiles = P.n_tiles > pair_id ? (P.n_tiles - pair_id + n_pairs - 1) / n_pairs : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&b->full[s], 2);   // used in CTA 0: one arrival per CTA, plus both CTAs' bytes
      mbar_init(&b->empty[s], 1);  // MMA completion, signalled in both CTAs
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&b->tfull[a], 1);
      mbar_init(&b->tempty[a], 2 * Cfg::EPI_WARPS);  // used in CTA 0: every epilogue warp of both CTAs
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
  // k-blocks of a job's range
  auto job_kb = [&](int rng) { return MODE == MODE_MIX_LN ? (rng ? P.kb1 : P.kb0) : P.kb0 + P.kb1; };

  if (warp == 0) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed_parity[STAGES];
      bool armed[STAGES];
      for (int s = 0; s < STAGES; ++s) armed[s] = false;
      bool ok = true;
      int k, rng, acc;
      for (int j = 0; ok && mix_job<MODE>(j, k_tiles, k, rng, acc); ++j) {
        const int tile = pair_id + k * n_pairs;
        const int m0 = (tile / P.n_tiles_n) * (2 * BM) + (int)rank * BM;
        const int n0 = (tile % P.n_tiles_n) * BN + (int)rank * B2_ROWS;
        const int nkb = job_kb(rng);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&b->empty[stage], phase ^ 1, ab)) {
            ok = false;
            break;
          }
          uint8_t *sa = ring + stage * STAGE2_BYTES;
          const uint32_t full0 = map_shared_rank(&b->full[stage], 0);
          mbar_arrive_expect_tx_cluster(full0, STAGE2_BYTES);
          armed[stage] = true;
          armed_parity[stage] = phase;
          // the first range: A0 / B0 (z / W', or A / B); the second: A1 / B1
          const bool first = MODE == MODE_MIX_LN ? rng == 0 : kb < P.kb0;
          const int kk = MODE == MODE_MIX_LN ? kb : (first ? kb : kb - P.kb0);
          if (first) {
            tma_load_2d_pair(sa, &mA0, full0, kk * BK, m0);
            tma_load_2d_pair(sa + A_BYTES, &mB0, full0, kk * BK, n0);
          } else {
            tma_load_2d_pair(sa, &mA1, full0, kk * BK, m0);
            tma_load_2d_pair(sa + A_BYTES, &mB1, full0, kk * BK, n0);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // after a give-up CTA 0 waits for the phases it armed, which complete
      // only once both CTAs' copies have landed
      if (!ok && rank == 0) drain_after_abort(b, STAGES, armed_parity, armed, true, false, ab);
    }
  } else if (warp == 1) {
    if (rank == 0 && elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int n_acc[2] = {0, 0};  // jobs run so far on each accumulator
      int k, rng, acc;
      for (int j = 0; ok && mix_job<MODE>(j, k_tiles, k, rng, acc); ++j) {
        const int na = acc ? n_acc[1] : n_acc[0];
        if (acc) ++n_acc[1]; else ++n_acc[0];
        // the epilogue has finished with this accumulator's previous job
        if (!mbar_wait(&b->tempty[acc], (na & 1) ^ 1, ab)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        const int nkb = job_kb(rng);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&b->full[stage], phase, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + stage * STAGE2_BYTES);
          const uint32_t sb = sa + A_BYTES;
          const bool first = MODE == MODE_MIX_LN ? rng == 0 : kb < P.kb0;
          const uint32_t idesc = MODE == MODE_F32 ? (first ? P.idesc0 : P.idesc1)
                                 : MODE == MODE_UP_Z ? IDESC2_F16
                                                     : (first ? IDESC2_F16 : IDESC2_BF16);
          // the x range adds onto the rewritten z-range accumulator
          const bool fresh = MODE == MODE_MIX_LN ? rng == 0 && kb == 0 : kb == 0;
#pragma unroll
          for (int kq = 0; kq < BK / 16; ++kq)
            umma_f16_pair(d, sdesc_sw128(sa + kq * 32, 16, 1024),
                          sdesc_sw128(sb + kq * 32, 16, 1024), idesc, !(fresh && kq == 0));
          umma_commit_pair(&b->empty[stage]);
          if (++stage == STAGES) {
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
    // epilogue: warp % 4 selects the TMEM lane quarter it may read; each CTA
    // handles its own 128 rows of the pair's tile; with several warps per
    // quarter, warp j of a quarter takes 32-column chunks j, j + (warps per quarter), ...
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int c_first = (warp - 2) / 4, c_step = Cfg::EPI_WARPS / 4;
    const uint32_t tempty0[2] = {map_shared_rank(&b->tempty[0], 0),
                                 map_shared_rank(&b->tempty[1], 0)};
    int n_acc[2] = {0, 0};
    int k, rng, acc;
    bool stored = false;  // MODE_UP_Z: TMA stores may still be reading the staging buffer
    for (int j = 0; mix_job<MODE>(j, k_tiles, k, rng, acc); ++j) {
      const int na = acc ? n_acc[1] : n_acc[0];
      if (acc) ++n_acc[1]; else ++n_acc[0];
      bool got = __all_sync(0xffffffffu, mbar_wait(&b->tfull[acc], na & 1, ab));
      // MODE_UP_Z's warps meet at named barriers below: they leave together
      if (MODE == MODE_UP_Z) got = epi_sync_and<EPI_T>(got);
      if (!got) break;
      tc_fence_after();
      const int tile = pair_id + k * n_pairs;
      const int m = (tile / P.n_tiles_n) * (2 * BM) + (int)rank * BM + r;
      const int n0 = (tile % P.n_tiles_n) * BN;
      const uint32_t tacc = tmem + ((uint32_t)(q * 32) << 16) + acc * BN;
      if (MODE == MODE_MIX_LN && rng == 0) {
        // rewrite the z-range accumulator as r (acc - mu c) + d
        float n_acc_f = 0.f, mean = 0.f, m2 = 0.f;
        if (m < P.M)
          for (int c = 0; c < P.n_chunks; ++c) {
            const float2 st = P.stats[(int64_t)c * P.M + m];
            chan_merge(n_acc_f, mean, m2, (float)min(BN, P.kb0 * BK - c * BN), st.x, st.y);
          }
        const float rs = m < P.M ? rsqrtf(m2 / n_acc_f + P.eps) : 0.f;
        const float mr = mean * rs;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const int col = n0 + c * 32 + e;
            const float4 cc = col < P.N ? __ldg(reinterpret_cast<const float4 *>(P.ccol + col))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 dd = col < P.N ? __ldg(reinterpret_cast<const float4 *>(P.dcol + col))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            v[e] = __float_as_uint(fmaf(__uint_as_float(v[e]), rs, fmaf(-mr, cc.x, dd.x)));
            v[e + 1] = __float_as_uint(fmaf(__uint_as_float(v[e + 1]), rs, fmaf(-mr, cc.y, dd.y)));
            v[e + 2] = __float_as_uint(fmaf(__uint_as_float(v[e + 2]), rs, fmaf(-mr, cc.z, dd.z)));
            v[e + 3] = __float_as_uint(fmaf(__uint_as_float(v[e + 3]), rs, fmaf(-mr, cc.w, dd.w)));
          }
          tmem_st32(tacc + c * 32, v);
        }
        tmem_wait_st();
      } else if (MODE == MODE_UP_Z) {
        // z tile: per-row (mean, M2) in 32-column chunks merged in order, and
        // the fp16 values into the staging boxes (128-byte swizzle)
        const int nv = min(BN, P.N - n0);
        // every chunk of the tile holds 32 columns (d_up a multiple of 256
        // or an inner tile): chunk sizes and merge weights are constants
        const bool full = nv == BN;
        float n_acc_f = 0.f, mean = 0.f, m2 = 0.f;
        bool range_ok = true;
        const int mrow = (tile / P.n_tiles_n) * (2 * BM) + (int)rank * BM;
        // The staging buffer's two halves (columns 0-127: every warp's first
        // chunk; 128-255: its second) go out as separate TMA store groups, the
        // first as soon as it is written, so each half has about half a tile's
        // time to be read out before the next tile writes it again. Groups are
        // committed in the order first(t-1), second(t-1), first(t), ...
#pragma unroll 1
        for (int i = 0; i < 2; ++i) {
          const int c = c_first + i * c_step;
          uint32_t v[32];
          tmem_ld32(tacc + c * 32, v);
          tmem_wait_ld();
          if (i == 1) {
            // the tile's TMEM is read: the accumulator is free for the MMAs
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty0[acc]);
            // every warp has written the first half, and the previous tile's
            // second half has been read out (the newest group): store the
            // first half
            if (warp == 2 && lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            epi_bar_sync<EPI_T>();
            if (warp == 2 && lane == 0) {
              for (int bx = 0; bx < 2 && bx * 64 < nv; ++bx)
                tma_store_2d_box(&mZ, staging + bx * (BM * 128), n0 + bx * 64, mrow);
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
          } else if (stored) {
            // the previous tile's first half has been read out (all groups
            // but the newest)
            if (warp == 2 && lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            epi_bar_sync<EPI_T>();
          }
          const int cv = min(32, nv - c * 32);
          bool check = !full;  // test each value against fp16's range
          if (full) {
            float mc, qc;
            stats32(v, mc, qc);
            if (i == 0) {
              mean = mc;
              m2 = qc;
            } else {  // two 32-column chunk sets: weights 1/2 and 32 * 32 / 64
              const float delta = mc - mean;
              mean += delta * 0.5f;
              m2 += qc + delta * delta * 16.f;
            }
            // every value lies within sqrt(qc) of mc; the margin below 65504
            // covers the rounding of mc and qc, and NaN or Inf fail the test
            const float lim = 65000.f - fabsf(mc);
            check = !(lim > 0.f && qc <= lim * lim);
          } else if (cv > 0) {
            float sum = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e < cv) sum += __uint_as_float(v[e]);
            const float mc = sum / (float)cv;
            float qc = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e < cv) {
                const float dl = __uint_as_float(v[e]) - mc;
                qc = fmaf(dl, dl, qc);
              }
            chan_merge(n_acc_f, mean, m2, (float)cv, mc, qc);
          }
          if (check)
#pragma unroll
            for (int e = 0; e < 32; ++e) range_ok &= fabsf(__uint_as_float(v[e])) <= 65504.f;
          uint8_t *box = staging + (c / 2) * (BM * 128);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            uint4 o;
            __half2 *o2 = reinterpret_cast<__half2 *>(&o);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              o2[e] = __floats2half2_rn(__uint_as_float(v[jj * 8 + 2 * e]),
                                        __uint_as_float(v[jj * 8 + 2 * e + 1]));
            const int chunk = (c % 2) * 4 + jj;  // 16-byte chunk within the box's 128-byte row
            *reinterpret_cast<uint4 *>(box + r * 128 + ((chunk ^ (r & 7)) << 4)) = o;
          }
          // this thread's staging writes, visible to the TMA store
          fence_proxy_async_smem();
        }
        if (!range_ok) atomicOr(P.err, DEV_ERR_F16_RANGE);
        // the statistics of a row's chunk sets (one per warp of its quarter)
        // merge in a fixed order
        float *part = reinterpret_cast<float *>(staging + (BN / 64) * BM * 128);
        if (c_first > 0) {
          float *pp = part + (c_first - 1) * 3 * BM;
          pp[r] = n_acc_f;
          pp[BM + r] = mean;
          pp[2 * BM + r] = m2;
        }
        epi_bar_sync<EPI_T>();
        if (c_first == 0 && m < P.M) {
          if (full) {
            // equal 64-column sets: the k-th merge weighs 1 / (k + 2) and
            // 64 (k + 1) / (k + 2)
#pragma unroll
            for (int k = 0; k < c_step - 1; ++k) {
              const float *pp = part + k * 3 * BM;
              const float delta = pp[BM + r] - mean;
              mean += delta * (1.f / (float)(k + 2));
              m2 += pp[2 * BM + r] + delta * delta * (64.f * (float)(k + 1) / (float)(k + 2));
            }
          } else {
            for (int k = 0; k < c_step - 1; ++k) {
              const float *pp = part + k * 3 * BM;
              chan_merge(n_acc_f, mean, m2, pp[r], pp[BM + r], pp[2 * BM + r]);
            }
          }
          P.stats[(int64_t)(n0 / BN) * P.M + m] = make_float2(mean, m2);
        }
        if (warp == 2 && lane == 0) {  // the second half
          for (int bx = 2; bx * 64 < nv; ++bx)
            tma_store_2d_box(&mZ, staging + bx * (BM * 128), n0 + bx * 64, mrow);
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        stored = true;
      } else {
        __nv_bfloat16 *yrow = reinterpret_cast<__nv_bfloat16 *>(P.y) + (int64_t)m * P.ldy + n0;
        float *crow = reinterpret_cast<float *>(P.y) + (int64_t)m * P.ldy + n0;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + c * 32, v);
          tmem_wait_ld();
          if (MODE == MODE_F32) {
            if (m < P.M) {
#pragma unroll
              for (int jj = 0; jj < 8; ++jj)
                if (n0 + c * 32 + jj * 4 < P.N)
                  *reinterpret_cast<uint4 *>(crow + c * 32 + jj * 4) =
                      make_uint4(v[4 * jj], v[4 * jj + 1], v[4 * jj + 2], v[4 * jj + 3]);
            }
          } else if (m < P.M) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int col = n0 + c * 32 + jj * 8;
              if (col < P.N) {
                uint4 o;
                __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  o2[e] = __floats2bfloat162_rn(__uint_as_float(v[jj * 8 + 2 * e]),
                                                __uint_as_float(v[jj * 8 + 2 * e + 1]));
                *reinterpret_cast<uint4 *>(yrow + c * 32 + jj * 8) = o;
              }
            }
          }
        }
      }
      if (MODE != MODE_UP_Z) {  // MODE_UP_Z released the accumulator after its last TMEM read
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty0[acc]);
      }
    }
    if (MODE == MODE_UP_Z && stored && warp == 2 && lane == 0)
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
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

// W' = W_mix[:, :d_up] diag(gamma) as fp16 (one warp per output row j), with
// c[j] = sum_k W'[j][k] over the rounded values the MMAs see, and
// d[j] = sum_k W_mix[j][k] beta[k]; flags products outside fp16's range
__global__ void k_mix_ln_weights(const __nv_bfloat16 *__restrict__ W_mix, int64_t ld, int d_out,
                                 int d_up, const __nv_bfloat16 *__restrict__ gamma,
                                 const __nv_bfloat16 *__restrict__ beta, __half *__restrict__ w16,
                                 float *__restrict__ ccol, float *__restrict__ dcol, int *err) {
  const int lane = threadIdx.x % 32;
  const int j = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (j >= d_out) return;
  float c = 0.f, dv = 0.f;
  bool bad = false;
  for (int k = lane * 8; k < d_up; k += 256) {
    const uint4 w = *reinterpret_cast<const uint4 *>(W_mix + (int64_t)j * ld + k);
    const uint4 g = *reinterpret_cast<const uint4 *>(gamma + k);
    const uint4 bt = *reinterpret_cast<const uint4 *>(beta + k);
    const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&w);
    const __nv_bfloat162 *g2 = reinterpret_cast<const __nv_bfloat162 *>(&g);
    const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&bt);
    uint4 o;
    __half2 *o2 = reinterpret_cast<__half2 *>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 wf = __bfloat1622float2(w2[e]), gf = __bfloat1622float2(g2[e]),
                   bf = __bfloat1622float2(b2[e]);
      const float p0 = wf.x * gf.x, p1 = wf.y * gf.y;
      bad |= fabsf(p0) > 65504.f || fabsf(p1) > 65504.f;
      o2[e] = __floats2half2_rn(p0, p1);
      const float2 r = __half22float2(o2[e]);
      c += r.x + r.y;
      dv = fmaf(wf.x, bf.x, fmaf(wf.y, bf.y, dv));
    }
    *reinterpret_cast<uint4 *>(w16 + (int64_t)j * d_up + k) = o;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c += __shfl_xor_sync(0xffffffffu, c, o);
    dv += __shfl_xor_sync(0xffffffffu, dv, o);
  }
  if (lane == 0) {
    ccol[j] = c;
    dcol[j] = dv;
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
                             const void *gamma, const void *beta, cudaStream_t s) {
  const l3_dims_t &d = p->dims;
  int *err = p->dev_flags + 1;
  {
    LaunchTimer t("to_f16", s);
    k_to_f16<<<num_sms() * 4, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16 *>(W_up), d.d_emb,
                                           d.d_up, d.d_emb, reinterpret_cast<__half *>(p->w_up16),
                                           err);
    k_mix_ln_weights<<<(unsigned)((d.d_out + 7) / 8), 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16 *>(W_mix), d.d_up + d.d_in, (int)d.d_out,
        (int)d.d_up, reinterpret_cast<const __nv_bfloat16 *>(gamma),
        reinterpret_cast<const __nv_bfloat16 *>(beta), reinterpret_cast<__half *>(p->w_mixh16),
        p->mix_ccol, p->mix_ccol + (d.d_out + 3) / 4 * 4, err);
  }
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

template <int MODE>
l3_status launch_pair(const CUtensorMap &mA0, const CUtensorMap &mB0, const CUtensorMap &mA1,
                      const CUtensorMap &mB1, const CUtensorMap &mZ, const MixParams &P,
                      int device, cudaStream_t s) {
  constexpr size_t smem =
      1024 + MixCfg<MODE>::STAGES * STAGE2_BYTES + MixCfg<MODE>::STAGING + sizeof(Bars);
  static bool attr[64] = {};
  if (!attr[device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_mix_gemm_pair<MODE>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    attr[device & 63] = true;
  }
  // persistent: one CTA pair per two SMs, 256 x 256 tiles
  const int pairs = std::min(P.n_tiles, num_sms() / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(MixCfg<MODE>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  L3_CUDA_TRY(cudaLaunchKernelEx(&cfg, k_mix_gemm_pair<MODE>, mA0, mB0, mA1, mB1, mZ, P));
  return L3_OK;
}

l3_status launch_up_z_tc(const l3_plan_s *p, cudaStream_t s) {
  const l3_dims_t &d = p->dims;
  CUtensorMap mA, mB, mZ;
  l3_status st;
  const uint64_t M = p->n_tokens;
  if ((st = make_map(&mA, p->a_buf, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, M, d.d_emb, d.d_emb, BM)) !=
      L3_OK)
    return st;
  if ((st = make_map(&mB, p->w_up16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, d.d_up, d.d_emb, d.d_emb,
                     B2_ROWS)) != L3_OK)
    return st;
  // z is stored with TMA from 64-column, 128-row boxes
  if ((st = make_map(&mZ, p->h_buf, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, M, d.d_up, d.d_up, BM)) !=
      L3_OK)
    return st;
  MixParams P = {};
  P.M = (int)M;
  P.N = (int)d.d_up;
  P.kb0 = (int)(d.d_emb / BK);
  P.kb1 = 0;
  P.n_tiles_n = (int)((d.d_up + BN - 1) / BN);
  P.n_tiles = (int)((M + 2 * BM - 1) / (2 * BM)) * P.n_tiles_n;
  P.y = p->h_buf;
  P.ldy = d.d_up;
  P.stats = p->ln_stats;
  P.n_chunks = P.n_tiles_n;
  P.err = p->dev_flags + 1;
  LaunchTimer t("up_z_gemm_tc", s);
  return launch_pair<MODE_UP_Z>(mA, mB, mA, mB, mZ, P, p->device, s);
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
  MixParams P = {};
  P.M = (int)M;
  P.N = (int)d.d_out;
  P.kb0 = (int)(d.d_up / BK);
  P.kb1 = (int)(d.d_in / BK);
  P.n_tiles_n = (int)((d.d_out + BN - 1) / BN);
  P.n_tiles = (int)((M + 2 * BM - 1) / (2 * BM)) * P.n_tiles_n;
  P.y = y;
  P.ldy = d.d_out;
  P.stats = p->ln_stats;
  P.n_chunks = (int)((d.d_up + BN - 1) / BN);
  P.ccol = p->mix_ccol;
  P.dcol = p->mix_ccol + (d.d_out + 3) / 4 * 4;
  P.eps = d.ln_eps;
  P.err = p->dev_flags + 1;
  LaunchTimer t("mix_gemm_tc", s);
  return launch_pair<MODE_MIX_LN>(mA0, mB0, mA1, mB1, mA0, P, p->device, s);
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
  MixParams P = {};
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
  return launch_pair<MODE_F32>(mA, mB, mA1, mB1, mA, P, device, s);
}

}  // namespace l3
