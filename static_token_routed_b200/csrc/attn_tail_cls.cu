// Gather-attention on CUDA cores for short groups (the long tail).
//
// Per token n with ID t (kimjy99 review, Method, eq. L³):
//     s = K_t x_n,   p = softmax(s),   a_n = V_t^T p.
// A work item is up to 8 tokens of one group. K_t and V_t are contiguous row
// ranges of W_K and W_V (kimjy99 review §2: the tables are concatenations);
// every row is read from HBM once per item, with coalesced 16-byte loads, and
// used for all of the item's tokens.
//
// The plan sorts the items by token-count class (1, 2, 3-4, 5-8 tokens) and,
// inside a class, by d_t, largest first; one kernel per class, compiled for
// that many tokens, so a singleton does a singleton's arithmetic and the
// kernel's registers and shared memory allow several CTAs per SM. One CTA per
// item (256 threads):
//   - the item's x rows go to shared memory (bf16);
//   - logits: warp w takes rows w, w + 8, ...; each lane loads its 16-byte
//     column vectors of two rows at a time straight from HBM (many loads in
//     flight per SM across the resident CTAs) and the row's logits come out
//     of one warp-shuffle sum;
//   - an exact softmax per token (warp per token);
//   - a = V_t^T p: each thread owns one 16-byte column vector of d_emb and a
//     row phase, rows of V_t stream four at a time, row phases combine with
//     shuffles; a is stored as fp16 at the token's original position.
// d_t = 1 skips K_t: one logit gives p = 1.
// Single-token items with at most TAIL_SMALL_ROWS rows (most of the
// singletons) instead run one warp per item, eight items per CTA.
#include <cuda_fp16.h>

#include <algorithm>

#include "l3_internal.cuh"
#include "sm100.cuh"

namespace l3 {
namespace {

using namespace sm100;

constexpr int THREADS = 256;
constexpr int MAX_DIN = 2048;
constexpr int MAX_K = 512;

struct Params {
  const __nv_bfloat16 *x, *W_K, *W_V;
  __half *a;
  const TailItem *items;  // this class's items
  int d_in, d_emb;
};

__device__ __forceinline__ void cvt8(const uint4 &v, float *f) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

template <int TBC>
__global__ void __launch_bounds__(THREADS, 2) k_attn_tail_cls(Params P) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const TailItem it = P.items[blockIdx.x];
  const int nt = it.nt;
  const int d = it.d;
  const int64_t r0 = it.r0;
  const int nv_in = P.d_in / 8;       // 16-byte vectors per x / K row
  const int nvl = nv_in / 32;         // of them per lane (1..8)
  const int row_bytes = P.d_in * 2;
  uint8_t *xs = smem;                                                // [TBC][d_in] bf16
  float *logit = reinterpret_cast<float *>(smem + TBC * row_bytes);  // [TBC][MAX_K]
  __shared__ float inv_sum[TBC];

  if (d > 1) {
    for (int i = tid; i < nt * nv_in; i += THREADS) {
      const int t = i / nv_in, c = i - t * nv_in;
      reinterpret_cast<uint4 *>(xs)[i] =
          reinterpret_cast<const uint4 *>(P.x + (int64_t)it.tok[t] * P.d_in)[c];
    }
    __syncthreads();

    const uint4 *Kt = reinterpret_cast<const uint4 *>(P.W_K + r0 * P.d_in);
    for (int j = warp; j < d; j += 16) {
      const int j2 = j + 8;
      const bool two = j2 < d;
      uint4 k1[8], k2[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i < nvl) {
          k1[i] = Kt[(int64_t)j * nv_in + lane + 32 * i];
          k2[i] = two ? Kt[(int64_t)j2 * nv_in + lane + 32 * i] : make_uint4(0, 0, 0, 0);
        }
      float a1[TBC], a2[TBC];
#pragma unroll
      for (int t = 0; t < TBC; ++t) a1[t] = a2[t] = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i < nvl) {
          float kf1[8], kf2[8];
          cvt8(k1[i], kf1);
          cvt8(k2[i], kf2);
#pragma unroll
          for (int t = 0; t < TBC; ++t) {
            float xv[8];
            cvt8(*reinterpret_cast<const uint4 *>(xs + t * row_bytes + (lane + 32 * i) * 16), xv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              a1[t] = fmaf(kf1[e], xv[e], a1[t]);
              a2[t] = fmaf(kf2[e], xv[e], a2[t]);
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < TBC; ++t) {
        float v1 = a1[t], v2 = a2[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          v1 += __shfl_xor_sync(0xffffffffu, v1, o);
          v2 += __shfl_xor_sync(0xffffffffu, v2, o);
        }
        if (lane == 0 && t < nt) {
          logit[t * MAX_K + j] = v1;
          if (two) logit[t * MAX_K + j2] = v2;
        }
      }
    }
    __syncthreads();
    // exact softmax per token; logits become exp(s - max)
    if (warp < nt) {
      float *sl = logit + warp * MAX_K;
      float mx = -INFINITY;
      for (int j = lane; j < d; j += 32) mx = fmaxf(mx, sl[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sum = 0.f;
      for (int j = lane; j < d; j += 32) {
        const float e = expf(sl[j] - mx);
        sl[j] = e;
        sum += e;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) inv_sum[warp] = 1.0f / sum;
    }
  } else if (tid < TBC) {
    logit[tid * MAX_K] = 1.0f;
    inv_sum[tid] = 1.0f;
  }
  __syncthreads();

  // a = V_t^T p: lane = column vector (within the warp's vpw) + vpw * row phase
  const int nv_emb = P.d_emb / 8;
  const int vpw = nv_emb / 8;
  const int rl_n = 32 / vpw;
  const int cvv = warp * vpw + lane % vpw;
  const int rl = lane / vpw;
  const uint4 *Vt = reinterpret_cast<const uint4 *>(P.W_V + r0 * P.d_emb) + cvv;
  float acc[TBC][8];
#pragma unroll
  for (int t = 0; t < TBC; ++t)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[t][e] = 0.f;
  for (int j0 = rl; j0 < d; j0 += 4 * rl_n) {
    uint4 vv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u * rl_n;
      vv[u] = j < d ? Vt[(int64_t)j * nv_emb] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u * rl_n;
      if (j < d) {
        float vf[8];
        cvt8(vv[u], vf);
#pragma unroll
        for (int t = 0; t < TBC; ++t) {
          const float p = logit[t * MAX_K + j];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[t][e] = fmaf(p, vf[e], acc[t][e]);
        }
      }
    }
  }
  for (int o = vpw; o < 32; o <<= 1)
#pragma unroll
    for (int t = 0; t < TBC; ++t)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[t][e] += __shfl_xor_sync(0xffffffffu, acc[t][e], o);
  if (rl == 0) {
#pragma unroll
    for (int t = 0; t < TBC; ++t) {
      if (t < nt) {
        const float is = inv_sum[t];
        uint4 o;
        __half2 *o2 = reinterpret_cast<__half2 *>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o2[e] = __floats2half2_rn(acc[t][2 * e] * is, acc[t][2 * e + 1] * is);
        reinterpret_cast<uint4 *>(P.a + (int64_t)it.tok[t] * P.d_emb)[cvv] = o;
      }
    }
  }
}

// Items with few rows (d_t <= 32; the bulk of the singleton groups): one WARP
// per item, eight items per CTA, so many more items are in flight per SM than
// with a CTA per item. Lane j ends up holding logit j; the softmax is a pair of
// warp reductions; V_t rows are read by all lanes, two 16-byte vectors each.
// Requires d_t <= 32 and d_emb <= 512.
template <int TBC>
__global__ void __launch_bounds__(THREADS, 2) k_attn_tail_small(Params P, int count) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int idx = blockIdx.x * (THREADS / 32) + warp;
  if (idx >= count) return;
  const TailItem it = P.items[idx];
  const int nt = it.nt;
  const int d = it.d;
  const int64_t r0 = it.r0;
  const int nv_in = P.d_in / 8, nvl = nv_in / 32;
  float p[TBC];  // lane j: softmax weight of row j for each token
  if (d > 1) {
    uint4 xr[TBC][8];
#pragma unroll
    for (int t = 0; t < TBC; ++t)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i < nvl)
          xr[t][i] = t < nt ? reinterpret_cast<const uint4 *>(P.x + (int64_t)it.tok[t] * P.d_in)[lane + 32 * i]
                            : make_uint4(0, 0, 0, 0);
    const uint4 *Kt = reinterpret_cast<const uint4 *>(P.W_K + r0 * P.d_in);
    float s[TBC];
#pragma unroll
    for (int t = 0; t < TBC; ++t) s[t] = -INFINITY;
    for (int j = 0; j < d; ++j) {
      uint4 k1[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i < nvl) k1[i] = Kt[(int64_t)j * nv_in + lane + 32 * i];
#pragma unroll
      for (int t = 0; t < TBC; ++t) {
        float a1 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (i < nvl) {
            float kf1[8], xf[8];
            cvt8(k1[i], kf1);
            cvt8(xr[t][i], xf);
#pragma unroll
            for (int e = 0; e < 8; ++e) a1 = fmaf(kf1[e], xf[e], a1);
          }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a1 += __shfl_xor_sync(0xffffffffu, a1, o);
        if (lane == j) s[t] = a1;
      }
    }
#pragma unroll
    for (int t = 0; t < TBC; ++t) {
      float m = s[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float e = lane < d ? expf(s[t] - m) : 0.f;
      float sum = e;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      p[t] = e / sum;
    }
  } else {
#pragma unroll
    for (int t = 0; t < TBC; ++t) p[t] = lane == 0 ? 1.0f : 0.f;
  }
  // a = V_t^T p: lane owns 16-byte column vectors lane, lane + 32, ...
  const int nv_emb = P.d_emb / 8;
  const uint4 *Vt = reinterpret_cast<const uint4 *>(P.W_V + r0 * P.d_emb);
  float acc[TBC][2][8];
#pragma unroll
  for (int t = 0; t < TBC; ++t)
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[t][u][e] = 0.f;
  for (int j = 0; j < d; ++j) {
    float pj[TBC];
#pragma unroll
    for (int t = 0; t < TBC; ++t) pj[t] = __shfl_sync(0xffffffffu, p[t], j);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c = lane + 32 * u;
      if (c < nv_emb) {
        float vf[8];
        cvt8(Vt[(int64_t)j * nv_emb + c], vf);
#pragma unroll
        for (int t = 0; t < TBC; ++t)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[t][u][e] = fmaf(pj[t], vf[e], acc[t][u][e]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < TBC; ++t) {
    if (t < nt) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = lane + 32 * u;
        if (c < nv_emb) {
          uint4 o;
          __half2 *o2 = reinterpret_cast<__half2 *>(&o);
#pragma unroll
          for (int e = 0; e < 4; ++e) o2[e] = __floats2half2_rn(acc[t][u][2 * e], acc[t][u][2 * e + 1]);
          reinterpret_cast<uint4 *>(P.a + (int64_t)it.tok[t] * P.d_emb)[c] = o;
        }
      }
    }
  }
}

template <int TBC>
l3_status launch_small(const l3_plan_s *p, Params P, int64_t first, int64_t count,
                       cudaStream_t s) {
  if (count <= 0) return L3_OK;
  P.items = p->tail_items + first;
  const int per_cta = THREADS / 32;
  k_attn_tail_small<TBC><<<(unsigned)((count + per_cta - 1) / per_cta), THREADS, 0, s>>>(P, (int)count);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

template <int TBC>
l3_status launch_class(const l3_plan_s *p, Params P, int64_t first, int64_t count,
                       cudaStream_t s) {
  if (count <= 0) return L3_OK;
  P.items = p->tail_items + first;
  const size_t smem = (size_t)TBC * P.d_in * 2 + (size_t)TBC * MAX_K * sizeof(float);
  // dynamic + static shared memory may pass 48 KB; raise the limit when a
  // wider layer needs more than any earlier launch on this device
  static size_t configured[64] = {};
  if (smem > configured[p->device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_attn_tail_cls<TBC>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    configured[p->device & 63] = smem;
  }
  k_attn_tail_cls<TBC><<<(unsigned)count, THREADS, smem, s>>>(P);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

// ---------------------------------------------------------------------------
// Short groups (d_t <= TAIL_SMALL_ROWS) of 2..8 tokens: the item's rows are
// TMA-staged into shared memory once and reused by every token of the item.
// A persistent CTA per SM; warp 0 issues, several items ahead, one 1-D bulk
// copy per x row plus one for the item's K_t rows and one for its V_t rows
// (both contiguous in the concatenated tables) into a ring of slots; warps
// 1-4 and 5-8 are two groups that take alternate items: logits from shared
// memory (warp per (token, row) pair, lanes across d_in), an exact softmax
// per token, a = V_t^T p with threads across d_emb, stored at the tokens'
// original positions. The slot size follows the largest d_t of the launch's
// items (its first: the plan lists them largest first).
// ---------------------------------------------------------------------------
constexpr int STG_MAX_GROUPS = 4;  // compute groups of four warps
constexpr int STG_THREADS = 32 + STG_MAX_GROUPS * 128;  // warp 0 copies, the rest compute
constexpr int STG_MAX_SLOTS = 8;
constexpr int STG_GROUP_THREADS = 128;

struct StgHdr {
  int nt, d;
  int tok[TAIL_TOKENS];
};
struct StgShared {
  uint64_t full[STG_MAX_SLOTS], empty[STG_MAX_SLOTS];
  StgHdr hdr[STG_MAX_SLOTS];
  float lg[STG_MAX_GROUPS][TAIL_TOKENS * TAIL_SMALL_ROWS];  // per group: logits, then p
  int abort_flag;
};

__device__ __forceinline__ int stg_slot_bytes(int nt, int d, int d_in, int d_emb) {
  return nt * d_in * 2 + (d > 1 ? d * d_in * 2 : 0) + d * d_emb * 2;
}

// barrier of one compute group (128 threads), ids 1..STG_MAX_GROUPS, ANDing a
// flag across the group (every thread gets the AND)
__device__ __forceinline__ bool group_sync_and(int g, bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(1 + g), "n"(STG_GROUP_THREADS)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(STG_GROUP_THREADS) : "memory");
}

template <int TBC>
__global__ void __launch_bounds__(STG_THREADS, 1)
    k_attn_tail_staged(Params P, int count, int ring_bytes, int *err) {
  extern __shared__ __align__(128) uint8_t smem_stg[];
  StgShared *S = reinterpret_cast<StgShared *>(smem_stg);
  uint8_t *ring = smem_stg + ((sizeof(StgShared) + 127) & ~size_t(127));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // every thread sizes the ring the same way, from the largest d_t
  const int dmax = P.items[0].d;
  const int slot_bytes = (stg_slot_bytes(TBC, dmax, P.d_in, P.d_emb) + 127) & ~127;
  const int raw_slots = min(STG_MAX_SLOTS, ring_bytes / slot_bytes);  // >= 2
  // item q goes to group q % n_groups and slot q % n_slots; n_slots a multiple
  // of n_groups, so a slot always serves the same group, which then never
  // waits on a phase more than one ahead of the slot's
  const int n_groups = raw_slots >= 4 ? 4 : 2;
  const int n_slots = raw_slots / n_groups * n_groups;
  if (threadIdx.x == 0) {
    for (int i = 0; i < STG_MAX_SLOTS; ++i) {
      mbar_init(&S->full[i], 1);
      mbar_init(&S->empty[i], 1);
    }
    S->abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const Abort ab{&S->abort_flag, err};
  const int n_mine = count > (int)blockIdx.x ? (count - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    // ------------------------------------------------ producer: bulk copies
    bool ok = true;
    bool armed[STG_MAX_SLOTS];
    uint32_t armed_par[STG_MAX_SLOTS];
    for (int i = 0; i < STG_MAX_SLOTS; ++i) armed[i] = false;
    for (int q0 = 0; ok && q0 < n_mine; q0 += 32) {
      // the next 32 items' records, one per lane, handed to lane 0 by shuffles
      uint4 rec[3] = {};
      if (q0 + lane < n_mine) {
        const uint4 *src = reinterpret_cast<const uint4 *>(
            P.items + blockIdx.x + (int64_t)(q0 + lane) * gridDim.x);
        rec[0] = src[0];
        rec[1] = src[1];
        rec[2] = src[2];
      }
      const int n_here = min(32, n_mine - q0);
      for (int u = 0; u < n_here; ++u) {
        uint32_t w[12];
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          w[4 * k] = __shfl_sync(0xffffffffu, rec[k].x, u);
          w[4 * k + 1] = __shfl_sync(0xffffffffu, rec[k].y, u);
          w[4 * k + 2] = __shfl_sync(0xffffffffu, rec[k].z, u);
          w[4 * k + 3] = __shfl_sync(0xffffffffu, rec[k].w, u);
        }
        const int q = q0 + u;
        const int slot = q % n_slots;
        const uint32_t par = (uint32_t)(q / n_slots) & 1;
        if (lane == 0) {
          // TailItem: r0, (d | nt << 16), tok[8], pad[2]
          const int64_t r0 = (int32_t)w[0];
          const int d = (int)(int16_t)(w[1] & 0xffff), nt = (int)(int16_t)(w[1] >> 16);
          if (!mbar_wait(&S->empty[slot], par ^ 1, ab)) ok = false;
          if (ok) {
            StgHdr &h = S->hdr[slot];
            h.nt = nt;
            h.d = d;
            for (int t = 0; t < TAIL_TOKENS; ++t) h.tok[t] = (int)w[2 + t];
            uint8_t *xs = ring + slot * slot_bytes;
            uint8_t *ks = xs + nt * P.d_in * 2;
            uint8_t *vs = ks + (d > 1 ? d * P.d_in * 2 : 0);
            mbar_arrive_expect_tx(&S->full[slot], (uint32_t)stg_slot_bytes(nt, d, P.d_in, P.d_emb));
            armed[slot] = true;
            armed_par[slot] = par;
            for (int t = 0; t < nt; ++t)
              bulk_load_1d(xs + t * P.d_in * 2, P.x + (int64_t)(int)w[2 + t] * P.d_in,
                           (uint32_t)P.d_in * 2, &S->full[slot]);
            if (d > 1)
              bulk_load_1d(ks, P.W_K + r0 * P.d_in, (uint32_t)(d * P.d_in * 2), &S->full[slot]);
            bulk_load_1d(vs, P.W_V + r0 * P.d_emb, (uint32_t)(d * P.d_emb * 2), &S->full[slot]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
    }
    if (!ok && lane == 0) {
      // after a give-up: wait (bounded) for the copies still landing
      for (int i = 0; i < STG_MAX_SLOTS; ++i)
        if (armed[i]) {
          const uint32_t a = smem_u32(&S->full[i]);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(a, armed_par[i]) && globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
          }
        }
    }
  } else {
    // ------------------------------------------------ compute groups
    const int g = (warp - 1) / 4;
    if (g >= n_groups) return;  // no barrier below involves this group
    const int gt = threadIdx.x - 32 - g * STG_GROUP_THREADS;  // 0..127
    const int gw = gt / 32;
    float *lg = S->lg[g];
    const int nvl = P.d_in / 256;  // 16-byte vectors per lane per row (d_in % 256 == 0)
    const int nc = P.d_emb / 8;    // 16-byte vectors per V / a row
    for (int q = g; q < n_mine; q += n_groups) {
      const int slot = q % n_slots;
      const uint32_t par = (uint32_t)(q / n_slots) & 1;
      // the group leaves together (a thread that gave up alone would leave the
      // others waiting at the group's barrier)
      if (!group_sync_and(g, mbar_wait(&S->full[slot], par, ab))) break;
      const StgHdr h = S->hdr[slot];
      const int nt = h.nt, d = h.d;
      const uint8_t *xs = ring + slot * slot_bytes;
      const uint8_t *ks = xs + nt * P.d_in * 2;
      const uint8_t *vs = ks + (d > 1 ? d * P.d_in * 2 : 0);
      if (d > 1) {
        // logits: warp gw takes tokens gw, gw + 4; one x vector against all
        // d_t rows per step (d_t partial sums in registers), then one warp
        // reduction per row
        for (int t = gw; t < nt; t += 4) {
          const uint4 *xr = reinterpret_cast<const uint4 *>(xs + t * P.d_in * 2);
          float acc[TAIL_SMALL_ROWS];
#pragma unroll
          for (int j = 0; j < TAIL_SMALL_ROWS; ++j) acc[j] = 0.f;
          for (int i = 0; i < nvl; ++i) {
            float xf[8];
            cvt8(xr[lane + 32 * i], xf);
#pragma unroll
            for (int j = 0; j < TAIL_SMALL_ROWS; ++j) {
              if (j < d) {
                float kf[8];
                cvt8(reinterpret_cast<const uint4 *>(ks + j * P.d_in * 2)[lane + 32 * i], kf);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[j] = fmaf(xf[e], kf[e], acc[j]);
              }
            }
          }
#pragma unroll
          for (int j = 0; j < TAIL_SMALL_ROWS; ++j) {
            if (j < d) {
              float v = acc[j];
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
              if (lane == 0) lg[t * TAIL_SMALL_ROWS + j] = v;
            }
          }
          __syncwarp();
          // exact softmax of this token: lane j holds row j
          const float s = lane < d ? lg[t * TAIL_SMALL_ROWS + lane] : -INFINITY;
          float m = s;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          const float e = lane < d ? expf(s - m) : 0.f;
          float sum = e;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          if (lane < d) lg[t * TAIL_SMALL_ROWS + lane] = e / sum;
        }
      } else if (gt < nt) {
        lg[gt * TAIL_SMALL_ROWS] = 1.0f;  // one row: p = 1
      }
      group_sync(g);
      // a = V_t^T p: thread per (token, 16-byte column vector)
      const uint4 *vr = reinterpret_cast<const uint4 *>(vs);
      for (int wi = gt; wi < nt * nc; wi += STG_GROUP_THREADS) {
        const int t = wi / nc, c = wi - t * nc;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int j = 0; j < d; ++j) {
          const float pj = lg[t * TAIL_SMALL_ROWS + j];
          float vf[8];
          cvt8(vr[j * nc + c], vf);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fmaf(pj, vf[e], acc[e]);
        }
        uint4 o;
        __half2 *o2 = reinterpret_cast<__half2 *>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) o2[e] = __floats2half2_rn(acc[2 * e], acc[2 * e + 1]);
        reinterpret_cast<uint4 *>(P.a + (int64_t)h.tok[t] * P.d_emb)[c] = o;
      }
      // every thread of the group is done with the slot and with lg
      group_sync(g);
      if (gt == 0) mbar_arrive(&S->empty[slot]);
    }
  }
}

// the staged kernel keeps several items in flight per SM only when an item
// of the class with TAIL_SMALL_ROWS rows takes at most a quarter of the ring;
// with wider rows (d_in 2048) a CTA per item keeps more bytes in flight
bool staged_pays(const Params &P, int tbc) {
  const size_t slot = (size_t)tbc * P.d_in * 2 + (size_t)TAIL_SMALL_ROWS * (P.d_in + P.d_emb) * 2;
  return slot * 4 <= 227 * 1024 - ((sizeof(StgShared) + 127) & ~size_t(127));
}

template <int TBC>
l3_status launch_staged(const l3_plan_s *p, Params P, int64_t first, int64_t count,
                        cudaStream_t s) {
  if (count <= 0) return L3_OK;
  P.items = p->tail_items + first;
  const size_t head = (sizeof(StgShared) + 127) & ~size_t(127);
  const size_t smem = 227 * 1024;
  static bool configured[64] = {};
  if (!configured[p->device & 63]) {
    L3_CUDA_TRY(cudaFuncSetAttribute(k_attn_tail_staged<TBC>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    configured[p->device & 63] = true;
  }
  int n_sms = 148;
  cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, p->device);
  const int grid = (int)std::min<int64_t>(count, n_sms);
  k_attn_tail_staged<TBC><<<grid, STG_THREADS, smem, s>>>(P, (int)count, (int)(smem - head),
                                                         p->dev_flags + 1);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

}  // namespace

bool tail_cls_supported(const l3_dims_t &d) {
  // lanes own d_in / 256 column vectors; warps own d_emb / 64 of them
  auto pow2 = [](int64_t v) { return v > 0 && (v & (v - 1)) == 0; };
  return d.dtype == L3_BF16 && d.d_in % 256 == 0 && d.d_in <= MAX_DIN && d.d_emb % 64 == 0 &&
         d.d_emb <= 512 && pow2(d.d_emb / 64) && d.k <= MAX_K;
}

l3_status launch_attn_tail_cls(const l3_plan_s *p, const void *x, const void *W_K,
                               const void *W_V, const cudaStream_t *streams, int n_streams) {
  if (p->n_tail_items == 0) return L3_OK;
  Params P;
  P.x = reinterpret_cast<const __nv_bfloat16 *>(x);
  P.W_K = reinterpret_cast<const __nv_bfloat16 *>(W_K);
  P.W_V = reinterpret_cast<const __nv_bfloat16 *>(W_V);
  P.a = reinterpret_cast<__half *>(p->a_buf);
  P.d_in = (int)p->dims.d_in;
  P.d_emb = (int)p->dims.d_emb;
  const int64_t *off = p->tail_class_start;  // [5]
  const int64_t *spl = p->tail_class_split;  // [4]
  static const char *names[8] = {"attn_tail_t1_big", "attn_tail_t1_small", "attn_tail_t2_big",
                                 "attn_tail_t2_small", "attn_tail_t4_big", "attn_tail_t4_small",
                                 "attn_tail_t8_big", "attn_tail_t8_small"};
  // the eight (token class, d_t range) launches are independent: each goes to
  // the stream with the least work so far (items, those with more than
  // TAIL_SMALL_ROWS rows weighted 4x), largest launches first, so that one
  // launch's last long items do not leave the SMs idle before the next
  int order[8], n_l = 0;
  int64_t weight[8];
  for (int i = 0; i < 8; ++i) {
    const int c = i / 2, part = i % 2;
    const int64_t n = part == 0 ? spl[c] - off[c] : off[c + 1] - spl[c];
    weight[i] = n * (part == 0 ? 4 : 1);
    if (n > 0) order[n_l++] = i;
  }
  std::sort(order, order + n_l, [&](int a, int b) { return weight[a] > weight[b]; });
  int64_t load[8] = {};
  l3_status st = L3_OK;
  for (int li = 0; li < n_l && st == L3_OK; ++li) {
    const int c = order[li] / 2, part = order[li] % 2;
    int q = 0;
    for (int j = 1; j < n_streams; ++j)
      if (load[j] < load[q]) q = j;
    load[q] += weight[order[li]];
    const cudaStream_t s = streams[q];
    {
      const int64_t first = part == 0 ? off[c] : spl[c];
      const int64_t last = part == 0 ? spl[c] : off[c + 1];
      LaunchTimer t(names[2 * c + part], s);
      // single-token items with d_t <= TAIL_SMALL_ROWS run a warp per item
      switch (c) {
        case 0:
          st = part == 0 ? launch_class<1>(p, P, first, last - first, s)
                         : launch_small<1>(p, P, first, last - first, s);
          break;
        // short groups of several tokens: rows staged in shared memory once,
        // where at least four items fit the staging ring at a time (narrow
        // layers); otherwise a CTA per item
        case 1:
          st = part == 0 || !staged_pays(P, 2) ? launch_class<2>(p, P, first, last - first, s)
                                               : launch_staged<2>(p, P, first, last - first, s);
          break;
        case 2:
          st = part == 0 || !staged_pays(P, 4) ? launch_class<4>(p, P, first, last - first, s)
                                               : launch_staged<4>(p, P, first, last - first, s);
          break;
        default:
          st = part == 0 || !staged_pays(P, 8) ? launch_class<8>(p, P, first, last - first, s)
                                               : launch_staged<8>(p, P, first, last - first, s);
          break;
      }
    }
  }
  return st;
}

}  // namespace l3
