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

#include "l3_internal.cuh"

namespace l3 {
namespace {

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

}  // namespace

bool tail_cls_supported(const l3_dims_t &d) {
  // lanes own d_in / 256 column vectors; warps own d_emb / 64 of them
  auto pow2 = [](int64_t v) { return v > 0 && (v & (v - 1)) == 0; };
  return d.dtype == L3_BF16 && d.d_in % 256 == 0 && d.d_in <= MAX_DIN && d.d_emb % 64 == 0 &&
         d.d_emb <= 512 && pow2(d.d_emb / 64) && d.k <= MAX_K;
}

l3_status launch_attn_tail_cls(const l3_plan_s *p, const void *x, const void *W_K,
                               const void *W_V, cudaStream_t s) {
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
  l3_status st = L3_OK;
  for (int c = 0; c < 4 && st == L3_OK; ++c) {
    for (int part = 0; part < 2 && st == L3_OK; ++part) {
      const int64_t first = part == 0 ? off[c] : spl[c];
      const int64_t last = part == 0 ? spl[c] : off[c + 1];
      if (last <= first) continue;
      LaunchTimer t(names[2 * c + part], s);
      // single-token items with d_t <= TAIL_SMALL_ROWS run a warp per item
      switch (c) {
        case 0:
          st = part == 0 ? launch_class<1>(p, P, first, last - first, s)
                         : launch_small<1>(p, P, first, last - first, s);
          break;
        case 1: st = launch_class<2>(p, P, first, last - first, s); break;
        case 2: st = launch_class<4>(p, P, first, last - first, s); break;
        default: st = launch_class<8>(p, P, first, last - first, s); break;
      }
    }
  }
  return st;
}

}  // namespace l3
