// Gather-attention on CUDA cores for short groups (the long tail of
// singleton and few-token groups).
//
// For every token n of a group with ID t (kimjy99 review, Method, eq. L³;
// papernotes 整体框架: per-token attention over the token's own rows):
//     s = K_t x_n,   p = softmax(s),   a_n = V_t^T p
// K_t = W_K[r0 .. r0+d-1], V_t = W_V[r0 .. r0+d-1], r0 = offsets[t], d = d_t.
//
// One CTA takes one work item: up to TAIL_TOKENS tokens of one group. Each
// K_t / V_t row is streamed from HBM once per item with 16-byte vector loads
// and reused for all tokens of the item from registers. The softmax is
// exact (max, exp, sum over all d_t logits held in shared memory). The
// d_t = 1 case skips K_t: one logit gives p = 1. The result row is written to
// a[perm[i]], i.e. back in the caller's token order, so the inverse sort of
// the batch (sciencestack page, Fig. 3 caption) costs nothing extra.
// For bf16 layers a is stored as fp16: its 10-bit mantissa keeps the error
// that LayerNorm later amplifies well inside the output tolerance, where a
// bf16 a alone would use half of it.
#include <cuda_fp16.h>

#include "l3_internal.cuh"

namespace l3 {
namespace {

constexpr int TAIL_THREADS = 256;
constexpr int TAIL_WARPS = TAIL_THREADS / 32;
constexpr int TB = TAIL_TOKENS;

template <typename T>
struct VecOps;

template <>
struct VecOps<__nv_bfloat16> {
  static constexpr int N = 8;  // elements per 16-byte vector
  __device__ __forceinline__ static void to_f32(const uint4 &v, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ __forceinline__ static uint4 from_f32(const float *f) {
    uint4 v;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return v;
  }
};

// fp16 output of the bf16 path: a holds 8 halves per 16-byte vector
struct HalfOut {
  __device__ __forceinline__ static uint4 from_f32(const float *f) {
    uint4 v;
    __half2 *h = reinterpret_cast<__half2 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
    return v;
  }
};

template <>
struct VecOps<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void to_f32(const uint4 &v, float *f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static uint4 from_f32(const float *f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

struct TailParams {
  const uint4 *x;      // [N][d_in / VEC]
  const uint4 *W_K;    // [v][d_in / VEC]
  const uint4 *W_V;    // [v][d_emb / VEC]
  uint4 *a;            // [N][d_emb / VEC]
  const TailItem *items;
  int nv_in;   // 16-byte vectors per x / K row
  int nv_emb;  // 16-byte vectors per V / a row
  int k_cap;   // d_t bound (logit buffer length)
  int red_rows;  // row phases of the V pass: TAIL_THREADS / nv_emb
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Shared memory: [union{ x rows (TB x nv_in uint4), V-pass partial sums
// (red_rows x TB x nv_emb*VEC floats) }] [logits TB x k_cap floats] [1/sum TB].
template <typename T, typename Out>
__global__ void __launch_bounds__(TAIL_THREADS) k_attn_tail(TailParams P) {
  using V = VecOps<T>;
  constexpr int VEC = V::N;
  extern __shared__ __align__(16) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  const TailItem item = P.items[blockIdx.x];
  const int nt = item.nt;
  const int64_t r0 = item.r0;
  const int d = item.d;

  const size_t xs_bytes = (size_t)TB * P.nv_in * 16;
  const size_t red_bytes = (size_t)P.red_rows * TB * P.nv_emb * VEC * sizeof(float);
  uint4 *xs = reinterpret_cast<uint4 *>(smem);
  float *red = reinterpret_cast<float *>(smem);
  float *logit = reinterpret_cast<float *>(smem + (xs_bytes > red_bytes ? xs_bytes : red_bytes));
  float *inv_sum = logit + (size_t)TB * P.k_cap;

  __shared__ int32_t tok_index[TB];
  if (tid < TB) tok_index[tid] = tid < nt ? item.tok[tid] : 0;
  __syncthreads();

  if (d > 1) {
    // x rows of the item's tokens (gathered through perm)
    for (int i = tid; i < nt * P.nv_in; i += TAIL_THREADS) {
      int t = i / P.nv_in, c = i - t * P.nv_in;
      xs[i] = P.x[(int64_t)tok_index[t] * P.nv_in + c];
    }
    __syncthreads();

    // logits: warp w takes rows w, w + 8, ...; lane l takes vectors l, l + 32, ...
    for (int j = warp; j < d; j += TAIL_WARPS) {
      const uint4 *krow = P.W_K + (r0 + j) * P.nv_in;
      float acc[TB];
#pragma unroll
      for (int t = 0; t < TB; ++t) acc[t] = 0.f;
      for (int c0 = 0; c0 < P.nv_in; c0 += 4 * 32) {
        uint4 kv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          int c = c0 + u * 32 + lane;
          kv[u] = c < P.nv_in ? krow[c] : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          int c = c0 + u * 32 + lane;
          if (c >= P.nv_in) break;
          float kf[VEC];
          V::to_f32(kv[u], kf);
#pragma unroll
          for (int t = 0; t < TB; ++t) {
            if (t < nt) {
              float xf[VEC];
              V::to_f32(xs[t * P.nv_in + c], xf);
#pragma unroll
              for (int e = 0; e < VEC; ++e) acc[t] = fmaf(kf[e], xf[e], acc[t]);
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < TB; ++t) {
        if (t < nt) {
          float s = warp_sum(acc[t]);
          if (lane == 0) logit[t * P.k_cap + j] = s;
        }
      }
    }
    __syncthreads();

    // exact softmax per token; logits are replaced by exp(s - max)
    for (int t = warp; t < nt; t += TAIL_WARPS) {
      float *s = logit + t * P.k_cap;
      float m = -INFINITY;
      for (int j = lane; j < d; j += 32) m = fmaxf(m, s[j]);
      m = warp_max(m);
      float sum = 0.f;
      for (int j = lane; j < d; j += 32) {
        float e = expf(s[j] - m);
        s[j] = e;
        sum += e;
      }
      sum = warp_sum(sum);
      if (lane == 0) inv_sum[t] = 1.0f / sum;
    }
  } else {
    if (tid < TB) {
      logit[tid * P.k_cap] = 1.0f;
      inv_sum[tid] = 1.0f;
    }
  }
  __syncthreads();

  // a = V_t^T p: thread (rg, cv) accumulates rows rg, rg + red_rows, ... of column vector cv
  const int cv = tid % P.nv_emb;
  const int rg = tid / P.nv_emb;
  if (rg < P.red_rows) {
    float acc[TB][VEC];
#pragma unroll
    for (int t = 0; t < TB; ++t)
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[t][e] = 0.f;
    const uint4 *vcol = P.W_V + r0 * P.nv_emb + cv;
    int j = rg;
    for (; j + 3 * P.red_rows < d; j += 4 * P.red_rows) {
      uint4 vv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) vv[u] = vcol[(int64_t)(j + u * P.red_rows) * P.nv_emb];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float vf[VEC];
        V::to_f32(vv[u], vf);
#pragma unroll
        for (int t = 0; t < TB; ++t) {
          if (t < nt) {
            float p = logit[t * P.k_cap + j + u * P.red_rows];
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[t][e] = fmaf(p, vf[e], acc[t][e]);
          }
        }
      }
    }
    for (; j < d; j += P.red_rows) {
      float vf[VEC];
      V::to_f32(vcol[(int64_t)j * P.nv_emb], vf);
#pragma unroll
      for (int t = 0; t < TB; ++t) {
        if (t < nt) {
          float p = logit[t * P.k_cap + j];
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[t][e] = fmaf(p, vf[e], acc[t][e]);
        }
      }
    }
    // partial sums of this row phase; they reuse the x-row buffer, which no
    // thread reads after the softmax barrier above
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      if (t < nt) {
        float *dst = red + ((size_t)(rg * TB + t) * P.nv_emb + cv) * VEC;
#pragma unroll
        for (int e = 0; e < VEC; ++e) dst[e] = acc[t][e];
      }
    }
  }
  __syncthreads();

  // fixed-order sum over row phases, scale by 1/sum, round once, store to a[perm[i]]
  for (int i = tid; i < nt * P.nv_emb; i += TAIL_THREADS) {
    int t = i / P.nv_emb, c = i - t * P.nv_emb;
    float o[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) o[e] = 0.f;
    for (int r = 0; r < P.red_rows; ++r) {
      const float *src = red + ((size_t)(r * TB + t) * P.nv_emb + c) * VEC;
#pragma unroll
      for (int e = 0; e < VEC; ++e) o[e] += src[e];
    }
    float is = inv_sum[t];
#pragma unroll
    for (int e = 0; e < VEC; ++e) o[e] *= is;
    P.a[(int64_t)tok_index[t] * P.nv_emb + c] = Out::from_f32(o);
  }
}

template <typename T>
size_t tail_smem_bytes(const TailParams &P) {
  constexpr int VEC = VecOps<T>::N;
  size_t xs = (size_t)TB * P.nv_in * 16;
  size_t red = (size_t)P.red_rows * TB * P.nv_emb * VEC * sizeof(float);
  return (xs > red ? xs : red) + (size_t)TB * P.k_cap * sizeof(float) + TB * sizeof(float);
}

template <typename T, typename Out>
l3_status launch_typed(const l3_plan_s *p, TailParams P, cudaStream_t s) {
  size_t smem = tail_smem_bytes<T>(P);
  if (smem > 48 * 1024)
    L3_CUDA_TRY(cudaFuncSetAttribute(k_attn_tail<T, Out>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  LaunchTimer t("attn_tail", s);
  k_attn_tail<T, Out><<<(unsigned)p->n_tail_items, TAIL_THREADS, smem, s>>>(P);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

}  // namespace

l3_status launch_attn_tail(const l3_plan_s *p, const void *x, const void *W_K, const void *W_V,
                           cudaStream_t s) {
  if (p->n_tail_items == 0) return L3_OK;
  const bool bf16 = p->dims.dtype == L3_BF16;
  const int vec = bf16 ? 8 : 4;
  TailParams P;
  P.x = reinterpret_cast<const uint4 *>(x);
  P.W_K = reinterpret_cast<const uint4 *>(W_K);
  P.W_V = reinterpret_cast<const uint4 *>(W_V);
  P.a = reinterpret_cast<uint4 *>(p->a_buf);
  P.items = p->tail_items;
  P.nv_in = (int)(p->dims.d_in / vec);
  P.nv_emb = (int)(p->dims.d_emb / vec);
  P.k_cap = (int)p->dims.k;
  P.red_rows = TAIL_THREADS / P.nv_emb;
  return bf16 ? launch_typed<__nv_bfloat16, HalfOut>(p, P, s)
              : launch_typed<float, VecOps<float>>(p, P, s);
}

size_t attn_tail_smem_bytes(const l3_dims_t &d) {
  const bool bf16 = d.dtype == L3_BF16;
  const int vec = bf16 ? 8 : 4;
  TailParams P{};
  P.nv_in = (int)(d.d_in / vec);
  P.nv_emb = (int)(d.d_emb / vec);
  P.k_cap = (int)d.k;
  P.red_rows = P.nv_emb > 0 ? TAIL_THREADS / P.nv_emb : 1;
  return bf16 ? tail_smem_bytes<__nv_bfloat16>(P) : tail_smem_bytes<float>(P);
}

}  // namespace l3
