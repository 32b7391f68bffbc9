// Backward pass of the layer, after an l3_forward on the same plan: it reuses
// the a and h that forward stored.
//
// kimjy99 review, Method, eq. L³, per token with rows K_t, V_t:
//   s = K_t x, p = softmax(s), a = V_t^T p, z = W_up a,
//   h = gamma (z - mean z) / sqrt(var z + eps) + beta, y = W_mix [h ; x].
// Given g_y = dL/dy (chain rule, step by step):
//   dW_mix = g_y^T [h ; x]              g_h = g_y W_mix[:, :d_up]
//   dx     = g_y W_mix[:, d_up:]  (+ K_t^T g_s below)
//   dgamma = sum g_h hhat, dbeta = sum g_h, g_hhat = g_h gamma
//   g_z    = (g_hhat - mean g_hhat - hhat mean(g_hhat hhat)) / sqrt(var z + eps)
//   dW_up  = g_z^T a                    g_a = g_z W_up
//   g_p    = V_t g_a, g_s = p (g_p - p.g_p)
//   dV_t  += p g_a^T, dK_t += g_s x^T, dx += K_t^T g_s
// bf16 layers run the six dense GEMMs on the tcgen05 pair kernel of the
// forward (fp32 output): it reads both operands K-major, so the operands
// whose K is the token axis or whose rows are the wrong way round are first
// transposed into bf16 copies (fp16 a and h become bf16 there, since one MMA
// takes one operand type); g_z is kept as a hi / lo pair of bf16 numbers.
// fp32 layers run them as one strided tiled FFMA kernel. The LayerNorm
// backward walks rows with a thread per column; its dgamma / dbeta column
// sums are per-CTA partials reduced in a fixed order (deterministic). The
// attention part runs dense tiles (up to 128 tokens of one group) as
// register-tiled warp-level MMA kernels over per-tile scratch planes, and
// tail items (up to 8 tokens) one CTA each on CUDA cores; dW_K / dW_V rows
// take atomic adds (several units of a group share them).
#include <cuda_fp16.h>

#include <algorithm>

#include "l3_internal.cuh"

namespace l3 {
namespace {

enum { T_F32 = 0, T_BF16 = 1, T_F16 = 2 };

__device__ __forceinline__ float ldx(const void *p, int type, int64_t i) {
  if (type == T_F32) return reinterpret_cast<const float *>(p)[i];
  if (type == T_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
  return __half2float(reinterpret_cast<const __half *>(p)[i]);
}

// ---------------------------------------------------------------- GEMM
// C[m][n] (+)= sum_k A(m, k) B(n, k), A(m, k) = A[m * a_sm + k * a_sk],
// B(n, k) = B[n * b_sn + k * b_sk]; fp32 accumulate and output.
struct Operand {
  const void *p;
  int64_t s_row, s_k;  // element strides along the output dimension and along k
  int type;
};

constexpr int GB_M = 64, GB_N = 64, GB_K = 16, G_THREADS = 256;

__global__ void __launch_bounds__(G_THREADS)
    k_gemm_strided(Operand A, Operand B, int M, int N, int K, float *__restrict__ C, int64_t ldc,
                   int accumulate) {
  __shared__ float As[GB_K][GB_M + 4];
  __shared__ float Bs[GB_K][GB_N + 4];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.y * GB_M, n0 = blockIdx.x * GB_N;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += GB_K) {
#pragma unroll
    for (int i = 0; i < (GB_M * GB_K) / G_THREADS; ++i) {
      const int e = tid + i * G_THREADS;
      // consecutive threads walk the operand's unit-stride dimension
      int row = A.s_k == 1 ? e / GB_K : e % GB_M, kk = A.s_k == 1 ? e % GB_K : e / GB_M;
      int gm = m0 + row, gk = k0 + kk;
      As[kk][row] = (gm < M && gk < K) ? ldx(A.p, A.type, gm * A.s_row + gk * A.s_k) : 0.f;
      row = B.s_k == 1 ? e / GB_K : e % GB_N;
      kk = B.s_k == 1 ? e % GB_K : e / GB_N;
      const int gn = n0 + row;
      gk = k0 + kk;
      Bs[kk][row] = (gn < N && gk < K) ? ldx(B.p, B.type, gn * B.s_row + gk * B.s_k) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GB_K; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= N) continue;
      float *c = C + (int64_t)gm * ldc + gn;
      *c = accumulate ? *c + acc[i][j] : acc[i][j];
    }
  }
}

l3_status gemm(Operand A, Operand B, int M, int N, int K, float *C, int64_t ldc, bool accumulate,
               cudaStream_t s) {
  if (M == 0 || N == 0) return L3_OK;
  dim3 grid((N + GB_N - 1) / GB_N, (M + GB_M - 1) / GB_M);
  k_gemm_strided<<<grid, G_THREADS, 0, s>>>(A, B, M, N, K, C, ldc, accumulate ? 1 : 0);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

// out[c][r] = in[r][c] as bf16: in is [R x C] 16-bit (fp16 or bf16) with row
// stride ld_in, out [C x ld_out]. 64 x 64 tiles, a grid-stride loop over them;
// 16-byte loads and stores, so C, ld_in and ld_out are multiples of 8 (the
// last store of a row may run into out's padding up to ld_out).
constexpr int TT = 64;

// With `ln` set, each input row r is z of the tensor-core forward and is
// normalised on the way, out[c][r] = gamma[c] (z[r][c] - mean_r) / std_r + beta[c],
// from the forward's per-256-column (mean, M2) of each row.
struct LnApply {
  const float2 *stats;  // [n_chunks][R], nullptr: plain transpose
  int n_chunks;
  const void *gamma, *beta;
  int wtype;  // weight type of gamma / beta
  float eps;
};

template <typename Tin>
__global__ void __launch_bounds__(256)
    k_transpose_bf16(const Tin *__restrict__ in, int64_t ld_in, int64_t R, int64_t C,
                     __nv_bfloat16 *__restrict__ out, int64_t ld_out, LnApply ln) {
  __shared__ float tile[TT][TT + 1];
  __shared__ float row_mu[TT], row_rs[TT];
  const int64_t tiles_c = (C + TT - 1) / TT, n_tiles = tiles_c * ((R + TT - 1) / TT);
  const int tid = threadIdx.x;
  for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x) {
    const int64_t r0 = (t / tiles_c) * TT, c0 = (t % tiles_c) * TT;
    if (ln.stats) {
      if (tid < TT && r0 + tid < R) {
        float n = 0.f, mean = 0.f, m2 = 0.f;
        for (int k = 0; k < ln.n_chunks; ++k) {
          const float2 st = ln.stats[k * R + r0 + tid];
          const float nb = (float)min((int64_t)256, C - 256 * k);
          const float nn = n + nb, dl = st.x - mean;
          mean += dl * (nb / nn);
          m2 += st.y + dl * dl * (n * nb / nn);
          n = nn;
        }
        row_mu[tid] = mean;
        row_rs[tid] = rsqrtf(m2 / n + ln.eps);
      }
      __syncthreads();
    }
    // load: 8 threads per 64-element row, 32 rows per pass
    for (int rr = tid / 8; rr < TT; rr += 32) {
      const int cc = (tid % 8) * 8;
      const int64_t r = r0 + rr, c = c0 + cc;
      float f[8];
      if (r < R && c < C) {
        const uint4 u = *reinterpret_cast<const uint4 *>(in + r * ld_in + c);
        const Tin *e = reinterpret_cast<const Tin *>(&u);
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = static_cast<float>(e[i]);
        if (ln.stats)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            f[i] = ldx(ln.gamma, ln.wtype, c + i) * ((f[i] - row_mu[rr]) * row_rs[rr]) +
                   ldx(ln.beta, ln.wtype, c + i);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) tile[rr][cc + i] = f[i];
    }
    __syncthreads();
    // store: 8 threads per 64-element output row
    for (int cc = tid / 8; cc < TT; cc += 32) {
      const int rr = (tid % 8) * 8;
      const int64_t c = c0 + cc, r = r0 + rr;
      if (c < C && r < R) {
        uint4 u;
        __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          o[i] = __floats2bfloat162_rn(tile[rr + 2 * i][cc], tile[rr + 2 * i + 1][cc]);
        *reinterpret_cast<uint4 *>(out + c * ld_out + r) = u;
      }
    }
    __syncthreads();
  }
}

template <typename Tin>
l3_status transpose_bf16(const void *in, int64_t ld_in, int64_t R, int64_t C, void *out,
                         int64_t ld_out, int n_sms, cudaStream_t s, LnApply ln = {}) {
  if (R == 0 || C == 0) return L3_OK;
  const int64_t n_tiles = ((R + TT - 1) / TT) * ((C + TT - 1) / TT);
  const unsigned grid = (unsigned)std::min<int64_t>(n_tiles, (int64_t)n_sms * 8);
  k_transpose_bf16<Tin><<<grid, 256, 0, s>>>(reinterpret_cast<const Tin *>(in), ld_in, R, C,
                                             reinterpret_cast<__nv_bfloat16 *>(out), ld_out, ln);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

// ---------------------------------------------------------------- LayerNorm
// Sum of K values over the CTA's 256 threads, the same in every thread and
// in a fixed order (deterministic); red holds 8 x 4 floats.
template <int K>
__device__ __forceinline__ void block_sum(float (&v)[K], float (*red)[4]) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
#pragma unroll
  for (int k = 0; k < K; ++k)
    for (int o = 16; o > 0; o >>= 1) v[k] += __shfl_xor_sync(0xffffffffu, v[k], o);
  if (lane == 0)
#pragma unroll
    for (int k = 0; k < K; ++k) red[warp][k] = v[k];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < K; ++k) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[w][k];
    v[k] = t;
  }
  __syncthreads();
}

// g_z from g_h and z, rows [blockIdx.x * rows, +rows) of M, one row at a
// time over the whole CTA: thread i holds columns i, i + 256, ... (NC of
// them, d_up <= 256 NC) in registers, the row's mean, variance and the two
// means of the LayerNorm gradient are CTA sums. g_z goes to g_z16 + g_z16_lo
// (its bf16 rounding and the bf16 rounding of the rest) when they are given,
// else to g_z as fp32. The CTA's column sums of g_h hhat (dgamma) and g_h
// (dbeta) go to part[cta][2][d_up].
template <int NC>
__global__ void __launch_bounds__(256)
    k_ln_backward(const float *__restrict__ z, const float *__restrict__ g_h, const void *gamma,
                  int gtype, int d_up, float eps, int64_t M, int64_t rows,
                  float *__restrict__ g_z, __nv_bfloat16 *__restrict__ g_z16,
                  __nv_bfloat16 *__restrict__ g_z16_lo, float *__restrict__ part) {
  __shared__ float red[8][4];
  const int tid = threadIdx.x;
  float gam[NC], pg[NC], pb[NC];
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int u = tid + i * 256;
    gam[i] = u < d_up ? ldx(gamma, gtype, u) : 0.f;
    pg[i] = pb[i] = 0.f;
  }
  const int64_t r_end = min(M, (int64_t)(blockIdx.x + 1) * rows);
  for (int64_t row = (int64_t)blockIdx.x * rows; row < r_end; ++row) {
    const float *zr = z + row * d_up, *gr = g_h + row * d_up;
    float zv[NC], gv[NC];
    float sum[1] = {0.f};
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int u = tid + i * 256;
      zv[i] = u < d_up ? zr[u] : 0.f;
      gv[i] = u < d_up ? gr[u] : 0.f;
      sum[0] += zv[i];
    }
    block_sum<1>(sum, red);
    const float mu = sum[0] / d_up;
    float q[1] = {0.f};
#pragma unroll
    for (int i = 0; i < NC; ++i)
      if (tid + i * 256 < d_up) q[0] = fmaf(zv[i] - mu, zv[i] - mu, q[0]);
    block_sum<1>(q, red);
    const float rstd = 1.0f / sqrtf(q[0] / d_up + eps);
    float m[2] = {0.f, 0.f};  // sums of g_hhat and g_hhat * hhat
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const float hh = (zv[i] - mu) * rstd, gh = gv[i] * gam[i];
      zv[i] = hh;  // zv holds hhat from here on
      m[0] += gh;
      m[1] = fmaf(gh, hh, m[1]);
      pg[i] = fmaf(gv[i], hh, pg[i]);
      pb[i] += gv[i];
    }
    block_sum<2>(m, red);
    const float m1 = m[0] / d_up, m2 = m[1] / d_up;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int u = tid + i * 256;
      if (u >= d_up) continue;
      const float gz = (gv[i] * gam[i] - m1 - zv[i] * m2) * rstd;
      if (g_z16) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(gz);
        g_z16[row * d_up + u] = hi;
        g_z16_lo[row * d_up + u] = __float2bfloat16_rn(gz - __bfloat162float(hi));
      } else {
        g_z[row * d_up + u] = gz;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int u = tid + i * 256;
    if (u < d_up) {
      part[(int64_t)blockIdx.x * 2 * d_up + u] = pg[i];
      part[(int64_t)blockIdx.x * 2 * d_up + d_up + u] = pb[i];
    }
  }
}

// column sums of the per-CTA partials in a fixed order: a CTA per 32
// columns, warp w adds partials w, w + 8, ..., then warp order
__global__ void __launch_bounds__(256)
    k_sum_partials(const float *__restrict__ part, int n_parts, int d_up,
                   float *__restrict__ dgamma, float *__restrict__ dbeta) {
  __shared__ float red[2][8][32];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int u = blockIdx.x * 32 + lane;
  float g = 0.f, b = 0.f;
  if (u < d_up)
    for (int i = warp; i < n_parts; i += 8) {
      g += part[(int64_t)i * 2 * d_up + u];
      b += part[(int64_t)i * 2 * d_up + d_up + u];
    }
  red[0][warp][lane] = g;
  red[1][warp][lane] = b;
  __syncthreads();
  if (warp == 0 && u < d_up) {
    g = b = 0.f;
    for (int w = 0; w < 8; ++w) {
      g += red[0][w][lane];
      b += red[1][w][lane];
    }
    dgamma[u] = g;
    dbeta[u] = b;
  }
}

template <int NC>
void launch_ln_backward(unsigned grid, int64_t rows, cudaStream_t s, const float *z,
                        const float *g_h, const void *gamma, int gtype, int d_up, float eps,
                        int64_t M, float *g_z, __nv_bfloat16 *g_z16, __nv_bfloat16 *g_z16_lo,
                        float *part) {
  k_ln_backward<NC><<<grid, 256, 0, s>>>(z, g_h, gamma, gtype, d_up, eps, M, rows, g_z, g_z16,
                                         g_z16_lo, part);
}

// ---------------------------------------------------------------- attention
constexpr int AT = 8;        // tokens per chunk
constexpr int A_MAX_K = 1024;

// Tail items (up to TAIL_TOKENS tokens of one group): one CTA per item,
// every row it reads shared by the item's tokens; dK / dV rows take atomic
// adds (several items of a group share its rows). NT = the item class's
// token bound (1, 2, 4 or 8): the plan lists items by class.
static_assert(AT == TAIL_TOKENS, "one chunk per tail item");
template <int WT>
__device__ __forceinline__ float ldt(const void *p, int64_t i) {
  if (WT == T_F32) return reinterpret_cast<const float *>(p)[i];
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
}
// four consecutive elements i .. i + 3 (i a multiple of 4) as fp32
template <int WT>
__device__ __forceinline__ float4 ldt4(const void *p, int64_t i) {
  if (WT == T_F32) return reinterpret_cast<const float4 *>(p)[i / 4];
  const uint2 u = reinterpret_cast<const uint2 *>(p)[i / 4];
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float dot4(const float4 a, const float4 b, float acc) {
  return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, acc))));
}

template <int NT, int WT>
__global__ void __launch_bounds__(256)
    k_attn_backward_tail(const void *x, const void *W_K, const void *W_V,
                         const float *__restrict__ g_a, const TailItem *__restrict__ items,
                         int d_in, int d_emb, float *__restrict__ dx, float *__restrict__ dW_K,
                         float *__restrict__ dW_V) {
  extern __shared__ float sm[];
  float *xs = sm;                  // [NT][d_in]
  float *gas = xs + NT * d_in;     // [NT][d_emb]
  float *ps = gas + NT * d_emb;    // [NT][A_MAX_K] logits, then p
  float *gs = ps + NT * A_MAX_K;   // [NT][A_MAX_K] g_p, then g_s
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __shared__ int32_t tok[AT];  // original indices of the item's tokens
  const TailItem *item = items + blockIdx.x;
  const int64_t r0 = item->r0;
  const int d = item->d, c = item->nt;
  for (int c0 = 0; c0 < c; c0 += NT) {
    const int nt = min(NT, c - c0);
    if (threadIdx.x < NT) tok[threadIdx.x] = threadIdx.x < nt ? item->tok[c0 + threadIdx.x] : 0;
    __syncthreads();
    for (int i = threadIdx.x; i < NT * d_in; i += blockDim.x) {
      const int t = i / d_in, col = i % d_in;
      xs[i] = t < nt ? ldt<WT>(x, (int64_t)tok[t] * d_in + col) : 0.f;
    }
    for (int i = threadIdx.x; i < NT * d_emb; i += blockDim.x) {
      const int t = i / d_emb, col = i % d_emb;
      gas[i] = t < nt ? g_a[(int64_t)tok[t] * d_emb + col] : 0.f;
    }
    __syncthreads();
    // logits s = K_j . x_t and g_p = V_j . g_a_t, one warp per row, four
    // columns per lane per step
    for (int j = warp; j < d; j += 8) {
      float sv[NT], gv[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) sv[t] = gv[t] = 0.f;
      if (d > 1)
#pragma unroll 2
        for (int c4 = lane * 4; c4 < d_in; c4 += 128) {
          const float4 kv = ldt4<WT>(W_K, (r0 + j) * d_in + c4);
#pragma unroll
          for (int t = 0; t < NT; ++t)
            sv[t] = dot4(kv, *reinterpret_cast<const float4 *>(xs + t * d_in + c4), sv[t]);
        }
#pragma unroll 2
      for (int c4 = lane * 4; c4 < d_emb; c4 += 128) {
        const float4 vv = ldt4<WT>(W_V, (r0 + j) * d_emb + c4);
#pragma unroll
        for (int t = 0; t < NT; ++t)
          gv[t] = dot4(vv, *reinterpret_cast<const float4 *>(gas + t * d_emb + c4), gv[t]);
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        for (int o = 16; o > 0; o >>= 1) {
          sv[t] += __shfl_xor_sync(0xffffffffu, sv[t], o);
          gv[t] += __shfl_xor_sync(0xffffffffu, gv[t], o);
        }
        if (lane == 0) {
          ps[t * A_MAX_K + j] = sv[t];
          gs[t * A_MAX_K + j] = gv[t];
        }
      }
    }
    __syncthreads();
    // softmax and g_s = p (g_p - p . g_p), one warp per token
    if (warp < nt) {
      float *pr = ps + warp * A_MAX_K, *gr = gs + warp * A_MAX_K;
      float mx = -INFINITY;
      for (int j = lane; j < d; j += 32) mx = fmaxf(mx, pr[j]);
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sum = 0.f;
      for (int j = lane; j < d; j += 32) {
        const float e = d > 1 ? expf(pr[j] - mx) : 1.f;
        pr[j] = e;
        sum += e;
      }
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      float dot = 0.f;
      for (int j = lane; j < d; j += 32) {
        pr[j] /= sum;
        dot = fmaf(pr[j], gr[j], dot);
      }
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      for (int j = lane; j < d; j += 32) gr[j] = pr[j] * (gr[j] - dot);
    }
    __syncthreads();
    // dx_t += K_t^T g_s_t and dK_j (+)= sum_t g_s[t][j] x_t: thread per four
    // columns, one vector atomic add per row
    if (d > 1) {
      for (int c4 = threadIdx.x * 4; c4 < d_in; c4 += blockDim.x * 4) {
        float4 acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
        for (int j = 0; j < d; ++j) {
          const int64_t kidx = (r0 + j) * d_in + c4;
          const float4 kv = ldt4<WT>(W_K, kidx);
          float4 gk = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float gst = gs[t * A_MAX_K + j];
            const float4 xv = *reinterpret_cast<const float4 *>(xs + t * d_in + c4);
            acc[t].x = fmaf(gst, kv.x, acc[t].x);
            acc[t].y = fmaf(gst, kv.y, acc[t].y);
            acc[t].z = fmaf(gst, kv.z, acc[t].z);
            acc[t].w = fmaf(gst, kv.w, acc[t].w);
            gk.x = fmaf(gst, xv.x, gk.x);
            gk.y = fmaf(gst, xv.y, gk.y);
            gk.z = fmaf(gst, xv.z, gk.z);
            gk.w = fmaf(gst, xv.w, gk.w);
          }
          atomicAdd(reinterpret_cast<float4 *>(dW_K + kidx), gk);
        }
        for (int t = 0; t < nt; ++t) {
          float4 *o = reinterpret_cast<float4 *>(dx + (int64_t)tok[t] * d_in + c4);
          float4 v = *o;
          v.x += acc[t].x;
          v.y += acc[t].y;
          v.z += acc[t].z;
          v.w += acc[t].w;
          *o = v;
        }
      }
    }  // one row: p = 1, no gradient reaches K
    // dV_j (+)= sum_t p[t][j] g_a_t
    for (int c4 = threadIdx.x * 4; c4 < d_emb; c4 += blockDim.x * 4) {
#pragma unroll 2
      for (int j = 0; j < d; ++j) {
        float4 gv = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float pj = ps[t * A_MAX_K + j];
          const float4 ga = *reinterpret_cast<const float4 *>(gas + t * d_emb + c4);
          gv.x = fmaf(pj, ga.x, gv.x);
          gv.y = fmaf(pj, ga.y, gv.y);
          gv.z = fmaf(pj, ga.z, gv.z);
          gv.w = fmaf(pj, ga.w, gv.w);
        }
        atomicAdd(reinterpret_cast<float4 *>(dW_V + (r0 + j) * d_emb + c4), gv);
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- dense tiles
// A dense tile (up to 128 tokens of one group, 32..512 rows) runs the
// attention backward as four register-tiled kernels over its slot in
// scratch, two [slot_rows][DENSE_TILE_M] fp32 planes (row j, token t):
//   k_bwd_dense_scores   plane 0 = S = K_t X^T, plane 1 = G_p = V_t G_a^T
//   k_bwd_dense_softmax  plane 0 = P = softmax_j(S), plane 1 = G_s = P (G_p - sum_j P G_p)
//   k_bwd_dense_dx       dx_t += K_t^T g_s_t
//   k_attn_backward_dw   dK_t += G_s X, dV_t += P G_a
// Each thread holds a 4 x 8 (or 8 x 4) block of outputs; operands pass
// through shared memory 32 k-steps at a time.
constexpr int DB_K = 32;  // k-steps per shared-memory stage
constexpr int DB_J = 64;  // rows of a scores block

__device__ __forceinline__ float *slot_plane(float *slots, int64_t b, int slot_rows, int plane) {
  return slots + (b * 2 + plane) * (int64_t)slot_rows * DENSE_TILE_M;
}

// D += A B^T on the warp's tensor cores: A 16 x 16 bf16 (row-major
// fragment), B 8 x 16 bf16 (one token per column), D 16 x 8 fp32.
__device__ __forceinline__ void mma_bf16(float (&dacc)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(dacc[0]), "+f"(dacc[1]), "+f"(dacc[2]), "+f"(dacc[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16 pair (lo element first) from two floats, and the hi / lo split of a float
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

constexpr int DS_LD = DB_K + 8;  // bf16 row stride of the staged tiles (conflict-free fragments)

// S and G_p of 64 rows x 16 NE tokens (NE = ceil(c / 16) column groups of
// the tile; columns c..16 NE - 1 come out zero, later columns are left
// alone), on mma.sync: warp w owns rows 16 (w % 4) .. + 15 and the 8-token
// column blocks w / 4, w / 4 + 2, ... S takes K_t and x as they are (bf16);
// G_p takes V_t against g_a split into two bf16 parts (hi + lo), so it keeps
// about 16 bits of g_a.
template <int NE>
__device__ __forceinline__ void dense_scores(const void *x, const void *W_K, const void *W_V,
                                             const float *__restrict__ g_a, const int64_t *tok,
                                             int64_t r0, int d, int jb, int d_in, int d_emb,
                                             float *plane0, float *plane1,
                                             __nv_bfloat16 (*as)[DS_LD],
                                             __nv_bfloat16 (*bs)[DS_LD],
                                             __nv_bfloat16 (*bl)[DS_LD]) {
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int g = lane >> 2, tg = lane & 3;
  const int jr = (warp & 3) * 16, nb0 = warp >> 2;
  constexpr int T = 16 * NE;
  for (int plane = 0; plane < 2; ++plane) {
    const int K = plane == 0 ? d_in : d_emb;
    const __nv_bfloat16 *W = reinterpret_cast<const __nv_bfloat16 *>(plane == 0 ? W_K : W_V);
    float acc[NE][4] = {};
    for (int k0 = 0; k0 < K; k0 += DB_K) {
      __syncthreads();  // tok written / the previous stage read
      {  // 64 rows x 32 k of K_t or V_t: 16 bytes per thread
        const int row = tid / 4, seg = (tid % 4) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (jb + row < d) v = *reinterpret_cast<const uint4 *>(W + (r0 + jb + row) * K + k0 + seg);
        *reinterpret_cast<uint4 *>(&as[row][seg]) = v;
      }
      for (int i = tid; i < T * 4; i += 256) {  // T tokens x 32 k
        const int t = i / 4, seg = (i % 4) * 8;
        const int64_t tk = tok[t];
        if (plane == 0) {
          uint4 v = make_uint4(0, 0, 0, 0);
          if (tk >= 0)
            v = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(x) +
                                                 tk * d_in + k0 + seg);
          *reinterpret_cast<uint4 *>(&bs[t][seg]) = v;
        } else {
          float f[8] = {};
          if (tk >= 0) {
            const float4 u0 = *reinterpret_cast<const float4 *>(g_a + tk * d_emb + k0 + seg);
            const float4 u1 = *reinterpret_cast<const float4 *>(g_a + tk * d_emb + k0 + seg + 4);
            f[0] = u0.x; f[1] = u0.y; f[2] = u0.z; f[3] = u0.w;
            f[4] = u1.x; f[5] = u1.y; f[6] = u1.z; f[7] = u1.w;
          }
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat16 h0 = __float2bfloat16_rn(f[2 * e]);
            const __nv_bfloat16 h1 = __float2bfloat16_rn(f[2 * e + 1]);
            hi[e] = pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
            lo[e] = pack_bf16(f[2 * e] - __bfloat162float(h0), f[2 * e + 1] - __bfloat162float(h1));
          }
          *reinterpret_cast<uint4 *>(&bs[t][seg]) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4 *>(&bl[t][seg]) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < DB_K; kk += 16) {
        uint32_t a[4];
        a[0] = *reinterpret_cast<const uint32_t *>(&as[jr + g][kk + 2 * tg]);
        a[1] = *reinterpret_cast<const uint32_t *>(&as[jr + g + 8][kk + 2 * tg]);
        a[2] = *reinterpret_cast<const uint32_t *>(&as[jr + g][kk + 8 + 2 * tg]);
        a[3] = *reinterpret_cast<const uint32_t *>(&as[jr + g + 8][kk + 8 + 2 * tg]);
#pragma unroll
        for (int i = 0; i < NE; ++i) {
          const int n = (nb0 + 2 * i) * 8 + g;  // this lane's token in the block
          mma_bf16(acc[i], a, *reinterpret_cast<const uint32_t *>(&bs[n][kk + 2 * tg]),
                   *reinterpret_cast<const uint32_t *>(&bs[n][kk + 8 + 2 * tg]));
          if (plane == 1)
            mma_bf16(acc[i], a, *reinterpret_cast<const uint32_t *>(&bl[n][kk + 2 * tg]),
                     *reinterpret_cast<const uint32_t *>(&bl[n][kk + 8 + 2 * tg]));
        }
      }
    }
    float *out = plane == 0 ? plane0 : plane1;
#pragma unroll
    for (int i = 0; i < NE; ++i) {
      const int col = (nb0 + 2 * i) * 8 + 2 * tg;
      const int j0 = jb + jr + g, j1 = j0 + 8;
      if (j0 < d)
        *reinterpret_cast<float2 *>(out + (int64_t)j0 * DENSE_TILE_M + col) =
            make_float2(acc[i][0], acc[i][1]);
      if (j1 < d)
        *reinterpret_cast<float2 *>(out + (int64_t)j1 * DENSE_TILE_M + col) =
            make_float2(acc[i][2], acc[i][3]);
    }
  }
}

// CTA per (tile, 64-row block): S and G_p for 64 rows x the tile's tokens.
__global__ void __launch_bounds__(256)
    k_bwd_dense_scores(const void *x, const void *W_K, const void *W_V, int wtype,
                       const float *__restrict__ g_a, const int32_t *__restrict__ perm,
                       const int32_t *__restrict__ group_tok_start,
                       const int32_t *__restrict__ group_row_start,
                       const int32_t *__restrict__ group_rows, const DenseTile *__restrict__ tiles,
                       float *__restrict__ slots, int slot_rows, int d_in, int d_emb) {
  __shared__ __align__(16) __nv_bfloat16 as[DB_J][DS_LD];          // rows of K_t or V_t
  __shared__ __align__(16) __nv_bfloat16 bs[DENSE_TILE_M][DS_LD];  // x, or g_a's hi part
  __shared__ __align__(16) __nv_bfloat16 bl[DENSE_TILE_M][DS_LD];  // g_a's lo part
  __shared__ int64_t tok[DENSE_TILE_M];
  (void)wtype;  // dense tiles exist for bf16 layers only
  const int n_jb = slot_rows / DB_J;
  const int64_t b = blockIdx.x / n_jb;
  const int jb = (blockIdx.x % n_jb) * DB_J;
  const DenseTile tl = tiles[b];
  const int d = group_rows[tl.group];
  if (jb >= d) return;  // the whole CTA leaves
  const int64_t r0 = group_row_start[tl.group];
  const int c = min(DENSE_TILE_M, group_tok_start[tl.group + 1] - tl.tok0);
  if (threadIdx.x < DENSE_TILE_M) tok[threadIdx.x] = threadIdx.x < c ? perm[tl.tok0 + threadIdx.x] : -1;
  float *p0 = slot_plane(slots, b, slot_rows, 0), *p1 = slot_plane(slots, b, slot_rows, 1);
#define L3_SCORES(NE)                                                                           \
  dense_scores<NE>(x, W_K, W_V, g_a, tok, r0, d, jb, d_in, d_emb, p0, p1, as, bs, bl);  \
  break;
  switch ((c + 15) / 16) {
    case 1: L3_SCORES(1)
    case 2: L3_SCORES(2)
    case 3: L3_SCORES(3)
    case 4: L3_SCORES(4)
    case 5: L3_SCORES(5)
    case 6: L3_SCORES(6)
    case 7: L3_SCORES(7)
    default: L3_SCORES(8)
  }
#undef L3_SCORES
}

// CTA per tile, thread per token: P = softmax over the d rows of S, and
// G_s = P (G_p - sum_j P G_p), in place.
__global__ void __launch_bounds__(DENSE_TILE_M)
    k_bwd_dense_softmax(const int32_t *__restrict__ group_tok_start,
                        const int32_t *__restrict__ group_rows, const DenseTile *__restrict__ tiles,
                        float *__restrict__ slots, int slot_rows) {
  const int64_t b = blockIdx.x;
  const DenseTile tl = tiles[b];
  const int d = group_rows[tl.group];
  const int t = threadIdx.x;
  if (t >= group_tok_start[tl.group + 1] - tl.tok0) return;
  float *S = slot_plane(slots, b, slot_rows, 0) + t, *G = slot_plane(slots, b, slot_rows, 1) + t;
  float mx = -INFINITY;
  for (int j = 0; j < d; ++j) mx = fmaxf(mx, S[j * DENSE_TILE_M]);
  float sum = 0.f;
  for (int j = 0; j < d; ++j) sum += expf(S[j * DENSE_TILE_M] - mx);
  const float inv = 1.f / sum;
  float dot = 0.f;
  for (int j = 0; j < d; ++j) {
    const float pj = expf(S[j * DENSE_TILE_M] - mx) * inv;
    S[j * DENSE_TILE_M] = pj;
    dot = fmaf(pj, G[j * DENSE_TILE_M], dot);
  }
  for (int j = 0; j < d; ++j) G[j * DENSE_TILE_M] = S[j * DENSE_TILE_M] * (G[j * DENSE_TILE_M] - dot);
}

// A fragment (16 x 16, row-major, row stride DS_LD or wider) at row r0, k0
template <int LD>
__device__ __forceinline__ void load_a(uint32_t (&a)[4], const __nv_bfloat16 (*m)[LD], int r0,
                                       int k0, int g, int tg) {
  a[0] = *reinterpret_cast<const uint32_t *>(&m[r0 + g][k0 + 2 * tg]);
  a[1] = *reinterpret_cast<const uint32_t *>(&m[r0 + g + 8][k0 + 2 * tg]);
  a[2] = *reinterpret_cast<const uint32_t *>(&m[r0 + g][k0 + 8 + 2 * tg]);
  a[3] = *reinterpret_cast<const uint32_t *>(&m[r0 + g + 8][k0 + 8 + 2 * tg]);
}

// dx[t][col] += sum_j G_s[j][t] K_t[j][col] for the tile's tokens t < c of
// 16 NE, on mma.sync: M = tokens, N = 64 columns (warp w: columns 8w..8w+7,
// all NE 16-token blocks), K = rows j, 32 per stage. G_s enters as a hi / lo
// bf16 pair, K_t as it is.
template <int NE>
__device__ __forceinline__ void dense_dx(const __nv_bfloat16 *__restrict__ Wk,
                                         const float *__restrict__ G,
                                         const int32_t *__restrict__ perm, int tok0, int64_t r0,
                                         int d, int c, int col0, int d_in, float *__restrict__ dx,
                                         __nv_bfloat16 (*ah)[DS_LD], __nv_bfloat16 (*al)[DS_LD],
                                         __nv_bfloat16 (*bt)[DS_LD]) {
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int g = lane >> 2, tg = lane & 3;
  constexpr int T = 16 * NE;
  float acc[NE][4] = {};
  for (int j0 = 0; j0 < d; j0 += DB_K) {
    __syncthreads();  // the previous stage read
    // G_s rows j0..j0+31 x tokens 0..T-1 -> ah / al [token][j]
    for (int i = tid; i < DB_K * T / 4; i += 256) {
      const int jj = i % DB_K, t4 = (i / DB_K) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + jj < d) v = *reinterpret_cast<const float4 *>(G + (int64_t)(j0 + jj) * DENSE_TILE_M + t4);
      const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat16 h = __float2bfloat16_rn(f[e]);
        ah[t4 + e][jj] = h;
        al[t4 + e][jj] = __float2bfloat16_rn(f[e] - __bfloat162float(h));
      }
    }
    {  // K_t rows j0..j0+31, columns col0..col0+63 -> bt [column][j]
      const int jj = tid % DB_K, seg = (tid / DB_K) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (j0 + jj < d) v = *reinterpret_cast<const uint4 *>(Wk + (r0 + j0 + jj) * d_in + col0 + seg);
      const __nv_bfloat16 *e8 = reinterpret_cast<const __nv_bfloat16 *>(&v);
#pragma unroll
      for (int q = 0; q < 8; ++q) bt[seg + q][jj] = e8[q];
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < DB_K; kk += 16) {
      const uint32_t b0 = *reinterpret_cast<const uint32_t *>(&bt[warp * 8 + g][kk + 2 * tg]);
      const uint32_t b1 = *reinterpret_cast<const uint32_t *>(&bt[warp * 8 + g][kk + 8 + 2 * tg]);
#pragma unroll
      for (int i = 0; i < NE; ++i) {
        uint32_t a[4];
        load_a<DS_LD>(a, ah, 16 * i, kk, g, tg);
        mma_bf16(acc[i], a, b0, b1);
        load_a<DS_LD>(a, al, 16 * i, kk, g, tg);
        mma_bf16(acc[i], a, b0, b1);
      }
    }
  }
  const int col = col0 + warp * 8 + 2 * tg;
#pragma unroll
  for (int i = 0; i < NE; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int t = 16 * i + g + 8 * h;
      if (t >= c) continue;
      float2 *o = reinterpret_cast<float2 *>(dx + (int64_t)perm[tok0 + t] * d_in + col);
      float2 v = *o;
      v.x += acc[i][2 * h];
      v.y += acc[i][2 * h + 1];
      *o = v;
    }
  }
}

// CTA per (tile, 64-column block of d_in): dx of the tile's tokens (each
// token's dx belongs to this CTA alone).
__global__ void __launch_bounds__(256)
    k_bwd_dense_dx(const void *W_K, int wtype, const int32_t *__restrict__ perm,
                   const int32_t *__restrict__ group_tok_start,
                   const int32_t *__restrict__ group_row_start,
                   const int32_t *__restrict__ group_rows, const DenseTile *__restrict__ tiles,
                   const float *__restrict__ slots, int slot_rows, int d_in,
                   float *__restrict__ dx) {
  __shared__ __align__(16) __nv_bfloat16 ah[DENSE_TILE_M][DS_LD];  // g_s hi, [token][j]
  __shared__ __align__(16) __nv_bfloat16 al[DENSE_TILE_M][DS_LD];  // g_s lo
  __shared__ __align__(16) __nv_bfloat16 bt[64][DS_LD];            // K_t, [column][j]
  (void)wtype;  // dense tiles exist for bf16 layers only
  const int n_cb = d_in / 64;
  const int64_t b = blockIdx.x / n_cb;
  const int col0 = (blockIdx.x % n_cb) * 64;
  const DenseTile tl = tiles[b];
  const int d = group_rows[tl.group];
  const int64_t r0 = group_row_start[tl.group];
  const int c = min(DENSE_TILE_M, group_tok_start[tl.group + 1] - tl.tok0);
  const float *G = slot_plane(const_cast<float *>(slots), b, slot_rows, 1);
  const __nv_bfloat16 *Wk = reinterpret_cast<const __nv_bfloat16 *>(W_K);
#define L3_DX(NE)                                                                 \
  dense_dx<NE>(Wk, G, perm, tl.tok0, r0, d, c, col0, d_in, dx, ah, al, bt); \
  break;
  switch ((c + 15) / 16) {
    case 1: L3_DX(1)
    case 2: L3_DX(2)
    case 3: L3_DX(3)
    case 4: L3_DX(4)
    case 5: L3_DX(5)
    case 6: L3_DX(6)
    case 7: L3_DX(7)
    default: L3_DX(8)
  }
#undef L3_DX
}

// dK_t (+)= G_s X and dV_t (+)= P G_a over one dense tile's tokens, from the
// planes k_bwd_dense_softmax left, on mma.sync: CTA per (tile, 64-column
// block of d_in for dK or of d_emb for dV); M = 64 rows at a time (warp w:
// rows 16 (w % 4).., columns 32 (w / 4)..), N = 64 columns, K = the tile's
// 16 NE tokens. G_s / P enter as hi / lo bf16 pairs, x as it is, g_a as a
// pair (dV adds hi x hi, lo x hi, hi x lo). One atomic add per element: the
// tiles of one group share its rows.
constexpr int DW_C = 64, DW_LD = DENSE_TILE_M + 8;

template <int NE>
__device__ __forceinline__ void dense_dw(const __nv_bfloat16 *__restrict__ x,
                                         const float *__restrict__ g_a, const float *__restrict__ A,
                                         const int32_t *__restrict__ perm, int tok0, int64_t r0,
                                         int d, int c, bool is_k, int col0, int width, int d_in,
                                         int d_emb, float *__restrict__ out,
                                         __nv_bfloat16 (*bh)[DW_LD], __nv_bfloat16 (*bl)[DW_LD],
                                         __nv_bfloat16 (*ahi)[DW_LD],
                                         __nv_bfloat16 (*alo)[DW_LD]) {
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int g = lane >> 2, tg = lane & 3;
  constexpr int T = 16 * NE;
  // B: x or g_a of tokens 0..T-1, columns col0..col0+63 -> bh / bl [column][token]
  for (int i = tid; i < T * (DW_C / 8); i += 256) {
    const int t = i % T, seg = (i / T) * 8;
    float f[8] = {};
    if (t < c) {
      const int64_t tk = perm[tok0 + t];
      if (is_k) {
        const uint4 v = *reinterpret_cast<const uint4 *>(x + tk * d_in + col0 + seg);
        const __nv_bfloat16 *e8 = reinterpret_cast<const __nv_bfloat16 *>(&v);
#pragma unroll
        for (int q = 0; q < 8; ++q) f[q] = __bfloat162float(e8[q]);
      } else {
        const float4 u0 = *reinterpret_cast<const float4 *>(g_a + tk * d_emb + col0 + seg);
        const float4 u1 = *reinterpret_cast<const float4 *>(g_a + tk * d_emb + col0 + seg + 4);
        f[0] = u0.x; f[1] = u0.y; f[2] = u0.z; f[3] = u0.w;
        f[4] = u1.x; f[5] = u1.y; f[6] = u1.z; f[7] = u1.w;
      }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const __nv_bfloat16 h = __float2bfloat16_rn(f[q]);
      bh[seg + q][t] = h;
      bl[seg + q][t] = __float2bfloat16_rn(f[q] - __bfloat162float(h));
    }
  }
  const int mr = (warp & 3) * 16, nb = (warp >> 2) * 32;
  for (int jb = 0; jb < d; jb += 64) {
    __syncthreads();  // B written / the previous block's A read
    // A: rows jb..jb+63 of G_s or P, tokens 0..T-1 -> ahi / alo [row][token]
    for (int i = tid; i < 64 * T / 4; i += 256) {
      const int jj = i / (T / 4), t4 = (i % (T / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (jb + jj < d && t4 < c)
        v = *reinterpret_cast<const float4 *>(A + (int64_t)(jb + jj) * DENSE_TILE_M + t4);
      const float fv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float fe = t4 + e < c ? fv[e] : 0.f;
        const __nv_bfloat16 h = __float2bfloat16_rn(fe);
        ahi[jj][t4 + e] = h;
        alo[jj][t4 + e] = __float2bfloat16_rn(fe - __bfloat162float(h));
      }
    }
    __syncthreads();
    float acc[4][4] = {};
#pragma unroll
    for (int kk = 0; kk < T; kk += 16) {
      uint32_t ah4[4], al4[4];
      load_a<DW_LD>(ah4, ahi, mr, kk, g, tg);
      load_a<DW_LD>(al4, alo, mr, kk, g, tg);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int n = nb + q * 8 + g;
        const uint32_t b0 = *reinterpret_cast<const uint32_t *>(&bh[n][kk + 2 * tg]);
        const uint32_t b1 = *reinterpret_cast<const uint32_t *>(&bh[n][kk + 8 + 2 * tg]);
        mma_bf16(acc[q], ah4, b0, b1);
        mma_bf16(acc[q], al4, b0, b1);
        if (!is_k)
          mma_bf16(acc[q], ah4, *reinterpret_cast<const uint32_t *>(&bl[n][kk + 2 * tg]),
                   *reinterpret_cast<const uint32_t *>(&bl[n][kk + 8 + 2 * tg]));
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int col = col0 + nb + q * 8 + 2 * tg;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = jb + mr + g + 8 * h;
        if (j >= d) continue;
        float *o = out + (r0 + j) * width + col;  // col is even: 8-byte aligned
        atomicAdd(reinterpret_cast<float2 *>(o), make_float2(acc[q][2 * h], acc[q][2 * h + 1]));
      }
    }
  }
}

__global__ void __launch_bounds__(256)
    k_attn_backward_dw(const void *x, int wtype, const float *__restrict__ g_a,
                       const int32_t *__restrict__ perm, const int32_t *__restrict__ group_tok_start,
                       const int32_t *__restrict__ group_row_start,
                       const int32_t *__restrict__ group_rows, const DenseTile *__restrict__ tiles,
                       const float *__restrict__ slots, int slot_rows, int d_in, int d_emb,
                       float *__restrict__ dW_K, float *__restrict__ dW_V) {
  extern __shared__ __align__(16) uint8_t dw_raw[];
  auto bh = reinterpret_cast<__nv_bfloat16 (*)[DW_LD]>(dw_raw);  // [64 columns][DW_LD]
  auto bl = bh + DW_C;
  auto ahi = bl + DW_C;  // [64 rows][DW_LD]
  auto alo = ahi + 64;
  (void)wtype;  // dense tiles exist for bf16 layers only
  const int n_cbk = d_in / DW_C, n_cb = n_cbk + d_emb / DW_C;
  const int64_t b = blockIdx.x / n_cb;
  const int cb = blockIdx.x % n_cb;
  const bool is_k = cb < n_cbk;
  const int width = is_k ? d_in : d_emb, col0 = (is_k ? cb : cb - n_cbk) * DW_C;
  const DenseTile tl = tiles[b];
  const int64_t r0 = group_row_start[tl.group];
  const int d = group_rows[tl.group];
  const int c = min(DENSE_TILE_M, group_tok_start[tl.group + 1] - tl.tok0);
  const float *A = slots + (b * 2 + (is_k ? 1 : 0)) * (int64_t)slot_rows * DENSE_TILE_M;
  float *out = is_k ? dW_K : dW_V;
  const __nv_bfloat16 *xb = reinterpret_cast<const __nv_bfloat16 *>(x);
#define L3_DW(NE)                                                                               \
  dense_dw<NE>(xb, g_a, A, perm, tl.tok0, r0, d, c, is_k, col0, width, d_in, d_emb, out, bh, bl, \
               ahi, alo);                                                                        \
  break;
  switch ((c + 15) / 16) {
    case 1: L3_DW(1)
    case 2: L3_DW(2)
    case 3: L3_DW(3)
    case 4: L3_DW(4)
    case 5: L3_DW(5)
    case 6: L3_DW(6)
    case 7: L3_DW(7)
    default: L3_DW(8)
  }
#undef L3_DW
}

}  // namespace
}  // namespace l3

using namespace l3;

extern "C" l3_status l3_backward(const void *x, l3_plan_t p, const void *W_K, const void *W_V,
                                 const void *W_up, const void *ln_gamma, const void *ln_beta,
                                 const void *W_mix, const void *dy, float *dx, float *dW_K,
                                 float *dW_V, float *dW_up, float *dgamma, float *dbeta,
                                 float *dW_mix, void *stream) {
  set_error("");
  if (!p) {
    set_error("plan is NULL");
    return L3_ERR_INVALID_ARG;
  }
  const l3_dims_t &d = p->dims;
  const int64_t N = p->n_tokens;
  for (const void *q : {x, W_K, W_V, W_up, ln_gamma, ln_beta, W_mix, dy, (const void *)dx,
                        (const void *)dW_K, (const void *)dW_V, (const void *)dW_up,
                        (const void *)dgamma, (const void *)dbeta, (const void *)dW_mix})
    if (!q) {
      set_error("a tensor pointer is NULL");
      return L3_ERR_INVALID_ARG;
    }
  if (p->staged) {
    set_error("l3_backward takes a plan over the full tables (l3_plan)");
    return L3_ERR_INVALID_ARG;
  }
  const size_t attn_smem = (AT * d.d_in + AT * d.d_emb + 2 * AT * A_MAX_K) * sizeof(float);
  if (d.k > A_MAX_K || attn_smem > 220 * 1024 || d.d_up > 16 * 256) {
    set_error("l3_backward: k, d_in, d_emb or d_up beyond this kernel's shared-memory layout");
    return L3_ERR_UNSUPPORTED;
  }
  int cur_dev = -1;
  L3_CUDA_TRY(cudaGetDevice(&cur_dev));
  if (cur_dev != p->device) {
    set_error("l3_backward called on a different device than l3_plan");
    return L3_ERR_INVALID_ARG;
  }
  auto a16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  // checked before anything is enqueued: the tail kernels add into dW_K / dW_V,
  // so a rejection after them would leave a partial gradient behind
  if (!(a16(x) && a16(W_K) && a16(W_V) && a16(dx) && a16(dW_K) && a16(dW_V))) {
    set_error("l3_backward: x, W_K, W_V, dx, dW_K and dW_V must be 16-byte aligned");
    return L3_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the plan's a / h buffers and flags are read on this stream from here on:
  // l3_plan_destroy and l3_forward_status order themselves after it
  p->stream = s;
  if (N == 0) {
    L3_CUDA_TRY(cudaMemsetAsync(dW_up, 0, d.d_up * d.d_emb * sizeof(float), s));
    L3_CUDA_TRY(cudaMemsetAsync(dgamma, 0, d.d_up * sizeof(float), s));
    L3_CUDA_TRY(cudaMemsetAsync(dbeta, 0, d.d_up * sizeof(float), s));
    L3_CUDA_TRY(cudaMemsetAsync(dW_mix, 0, d.d_out * (d.d_up + d.d_in) * sizeof(float), s));
    return L3_OK;
  }
  const int wt = d.dtype == L3_BF16 ? T_BF16 : T_F32;
  const int it = d.dtype == L3_BF16 ? T_F16 : T_F32;  // a and h as the forward stored them
  int n_sms = 148;
  cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, p->device);
  // LayerNorm backward: about four CTAs per SM, each over a run of rows
  const int64_t ln_rows = (N + 4 * n_sms - 1) / (4 * n_sms);
  const int64_t n_ln = (N + ln_rows - 1) / ln_rows;
  const int64_t D = d.d_up + d.d_in;  // columns of W_mix
  // tensor cores for bf16 layers whose forward ran on them (it left the fp16
  // W_up copy in the plan) and whose operands meet the TMA alignment
  const bool tc = p->tc_gemm && a16(x) && a16(W_up) && a16(W_mix) && a16(dy) && a16(dx) &&
                  a16(dW_up) && a16(dW_mix);
  const int64_t ldn = (N + 7) / 8 * 8;  // row stride of the copies whose rows run over tokens
  // scratch: g_h, z [N x d_up] fp32, g_a [N x d_emb] fp32, LayerNorm partials,
  // g_z [N x d_up] (bf16 on the tensor-core path, else fp32) and the
  // tensor-core path's bf16 transposes
  const size_t f = sizeof(float);
  size_t bytes = 0;
  auto take = [&](size_t b) {
    const size_t o = bytes;
    bytes += (b + 255) / 256 * 256;
    return o;
  };
  const size_t o_gh = take(N * d.d_up * f), o_z = take(N * d.d_up * f),
               o_ga = take(N * d.d_emb * f), o_part = take(n_ln * 2 * d.d_up * f),
               o_gz = take(N * d.d_up * (tc ? 2 : f)), o_gzlo = take(tc ? N * d.d_up * 2 : 0);
  size_t o_wmt = 0, o_gyt = 0, o_hxt = 0, o_gzt = 0, o_at = 0, o_wut = 0;
  if (tc) {
    o_wmt = take(D * d.d_out * 2);      // W_mix^T   [D x d_out]
    o_gyt = take(d.d_out * ldn * 2);    // g_y^T     [d_out x N]
    o_hxt = take(D * ldn * 2);          // [h ; x]^T [D x N]
    o_gzt = take(d.d_up * ldn * 2);     // g_z^T     [d_up x N]
    o_at = take(d.d_emb * ldn * 2);     // a^T       [d_emb x N]
    o_wut = take(d.d_emb * d.d_up * 2); // W_up^T    [d_emb x d_up]
  }
  // p and g_s of every dense tile for k_attn_backward_dw
  const int64_t n_dt = p->n_dense_tiles;
  const int slot_rows = n_dt > 0 ? dense_attention_max_rows() : 0;
  const size_t o_slots = take(n_dt * 2 * slot_rows * DENSE_TILE_M * f);
  // from the device block cache, so a backward per batch maps no memory
  // after warm-up
  size_t got = 0;
  char *scratch = reinterpret_cast<char *>(cache_take(p->device, bytes, &got));
  cudaError_t e = cudaSuccess;
  if (!scratch) {
    e = cudaMalloc(reinterpret_cast<void **>(&scratch), bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(backward scratch)");
    got = bytes;
  }
  float *g_h = reinterpret_cast<float *>(scratch + o_gh);
  float *z = reinterpret_cast<float *>(scratch + o_z);
  float *g_a = reinterpret_cast<float *>(scratch + o_ga);
  float *part = reinterpret_cast<float *>(scratch + o_part);
  float *slots = reinterpret_cast<float *>(scratch + o_slots);
  float *g_z = tc ? nullptr : reinterpret_cast<float *>(scratch + o_gz);
  __nv_bfloat16 *g_z16 = tc ? reinterpret_cast<__nv_bfloat16 *>(scratch + o_gz) : nullptr;
  __nv_bfloat16 *g_z16_lo = tc ? reinterpret_cast<__nv_bfloat16 *>(scratch + o_gzlo) : nullptr;
  auto bf = [&](size_t o) { return reinterpret_cast<__nv_bfloat16 *>(scratch + o); };
  __nv_bfloat16 *wmt = bf(o_wmt), *gyt = bf(o_gyt), *hxt = bf(o_hxt), *gzt = bf(o_gzt),
                *at = bf(o_at), *wut = bf(o_wut);
  int *err = p->dev_flags + 1;  // a tensor-core wait that gives up reports here
  const int dev = p->device;
  using BF = __nv_bfloat16;
  const int64_t ldm = D;
  const char *wmx = reinterpret_cast<const char *>(W_mix) + d.d_up * (wt == T_F32 ? 4 : 2);
  l3_status st = L3_OK;
  if (tc) {
    LaunchTimer t("bwd_transpose", s);
    if (st == L3_OK) st = transpose_bf16<BF>(W_mix, D, d.d_out, D, wmt, d.d_out, n_sms, s);
    if (st == L3_OK) st = transpose_bf16<BF>(dy, d.d_out, N, d.d_out, gyt, ldn, n_sms, s);
    // the tensor-core forward keeps z, not h: normalise it on the way (its
    // per-256-column statistics are the forward's)
    LnApply ln{p->ln_stats, (int)((d.d_up + 255) / 256), ln_gamma, ln_beta, wt, d.ln_eps};
    if (st == L3_OK)
      st = transpose_bf16<__half>(p->h_buf, d.d_up, N, d.d_up, hxt, ldn, n_sms, s, ln);
    if (st == L3_OK)
      st = transpose_bf16<BF>(x, d.d_in, N, d.d_in, hxt + d.d_up * ldn, ldn, n_sms, s);
    if (st == L3_OK) st = transpose_bf16<BF>(W_up, d.d_emb, d.d_up, d.d_emb, wut, d.d_up, n_sms, s);
    if (st == L3_OK) st = transpose_bf16<__half>(p->a_buf, d.d_emb, N, d.d_emb, at, ldn, n_sms, s);
  }
  {
    LaunchTimer t("bwd_gemms_mix", s);
    // g_h = g_y W_mix[:, :d_up];  dx = g_y W_mix[:, d_up:];  dW_mix = g_y^T [h ; x]
    if (tc) {
      if (st == L3_OK)
        st = launch_gemm_nt_tc(dy, wmt, nullptr, nullptr, false, N, d.d_up, d.d_out, d.d_out,
                               d.d_out, g_h, d.d_up, err, dev, s);
      if (st == L3_OK)
        st = launch_gemm_nt_tc(dy, wmt + d.d_up * d.d_out, nullptr, nullptr, false, N, d.d_in,
                               d.d_out, d.d_out, d.d_out, dx, d.d_in, err, dev, s);
      if (st == L3_OK)
        st = launch_gemm_nt_tc(gyt, hxt, nullptr, nullptr, false, d.d_out, D, N, ldn, ldn, dW_mix,
                               D, err, dev, s);
    } else {
      if (st == L3_OK)
        st = gemm({dy, d.d_out, 1, wt}, {W_mix, 1, ldm, wt}, (int)N, (int)d.d_up, (int)d.d_out,
                  g_h, d.d_up, false, s);
      if (st == L3_OK)
        st = gemm({dy, d.d_out, 1, wt}, {wmx, 1, ldm, wt}, (int)N, (int)d.d_in, (int)d.d_out, dx,
                  d.d_in, false, s);
      if (st == L3_OK)
        st = gemm({dy, 1, d.d_out, wt}, {p->h_buf, 1, d.d_up, it}, (int)d.d_out, (int)d.d_up,
                  (int)N, dW_mix, ldm, false, s);
      if (st == L3_OK)
        st = gemm({dy, 1, d.d_out, wt}, {x, 1, d.d_in, wt}, (int)d.d_out, (int)d.d_in, (int)N,
                  dW_mix + d.d_up, ldm, false, s);
    }
  }
  {
    LaunchTimer t("bwd_layernorm", s);
    // z = a W_up^T again (the tensor-core path with the forward's fp16
    // operands, so z is the forward's), then the LayerNorm backward
    if (st == L3_OK)
      st = tc ? launch_gemm_nt_tc(p->a_buf, p->w_up16, nullptr, nullptr, true, N, d.d_up, d.d_emb,
                                  d.d_emb, d.d_emb, z, d.d_up, err, dev, s)
              : gemm({p->a_buf, d.d_emb, 1, it}, {W_up, d.d_emb, 1, wt}, (int)N, (int)d.d_up,
                     (int)d.d_emb, z, d.d_up, false, s);
    if (st == L3_OK) {
      auto ln = d.d_up <= 4 * 256   ? launch_ln_backward<4>
                : d.d_up <= 8 * 256 ? launch_ln_backward<8>
                                    : launch_ln_backward<16>;
      ln((unsigned)n_ln, ln_rows, s, z, g_h, ln_gamma, wt, (int)d.d_up, d.ln_eps, N, g_z, g_z16,
         g_z16_lo, part);
      k_sum_partials<<<(unsigned)((d.d_up + 31) / 32), 256, 0, s>>>(part, (int)n_ln, (int)d.d_up,
                                                                     dgamma, dbeta);
      e = cudaGetLastError();
      if (e != cudaSuccess) st = cuda_fail(e, "LayerNorm backward");
    }
  }
  {
    LaunchTimer t("bwd_gemms_up", s);
    // dW_up = g_z^T a;  g_a = g_z W_up, with g_z as the sum of its two bf16
    // parts: the attention backward's g_s = p (g_p - p . g_p) cancels, and
    // bf16 rounding of g_z alone shows in dW_K beyond the bf16 bar
    if (tc) {
      if (st == L3_OK) st = transpose_bf16<BF>(g_z16, d.d_up, N, d.d_up, gzt, ldn, n_sms, s);
      if (st == L3_OK)
        st = launch_gemm_nt_tc(gzt, at, nullptr, nullptr, false, d.d_up, d.d_emb, N, ldn, ldn,
                               dW_up, d.d_emb, err, dev, s);
      if (st == L3_OK)
        st = launch_gemm_nt_tc(g_z16, wut, g_z16_lo, wut, false, N, d.d_emb, d.d_up, d.d_up,
                               d.d_up, g_a, d.d_emb, err, dev, s);
    } else {
      if (st == L3_OK)
        st = gemm({g_z, 1, d.d_up, T_F32}, {p->a_buf, 1, d.d_emb, it}, (int)d.d_up, (int)d.d_emb,
                  (int)N, dW_up, d.d_emb, false, s);
      if (st == L3_OK)
        st = gemm({g_z, d.d_up, 1, T_F32}, {W_up, 1, d.d_emb, wt}, (int)N, (int)d.d_emb,
                  (int)d.d_up, g_a, d.d_emb, false, s);
    }
  }
  const int64_t n_tail = p->n_tail_items;
  if (st == L3_OK && n_tail > 0) {
    LaunchTimer t("bwd_attention_tail", s);
    auto launch_tail = [&](auto kernel, int nt, int cls) {
      const int64_t i0 = p->tail_class_start[cls], n = p->tail_class_start[cls + 1] - i0;
      if (n <= 0 || e != cudaSuccess) return;
      const size_t smem = (nt * d.d_in + nt * d.d_emb + 2 * nt * A_MAX_K) * f;
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return;
      kernel<<<(unsigned)n, 256, smem, s>>>(x, W_K, W_V, g_a, p->tail_items + i0, (int)d.d_in,
                                            (int)d.d_emb, dx, dW_K, dW_V);
      e = cudaGetLastError();
    };
    if (wt == T_BF16) {
      launch_tail(k_attn_backward_tail<1, T_BF16>, 1, 0);
      launch_tail(k_attn_backward_tail<2, T_BF16>, 2, 1);
      launch_tail(k_attn_backward_tail<4, T_BF16>, 4, 2);
      launch_tail(k_attn_backward_tail<8, T_BF16>, 8, 3);
    } else {
      launch_tail(k_attn_backward_tail<1, T_F32>, 1, 0);
      launch_tail(k_attn_backward_tail<2, T_F32>, 2, 1);
      launch_tail(k_attn_backward_tail<4, T_F32>, 4, 2);
      launch_tail(k_attn_backward_tail<8, T_F32>, 8, 3);
    }
    if (e != cudaSuccess) st = cuda_fail(e, "attention backward (tail items)");
  }
  if (st == L3_OK && n_dt > 0) {
    if (bwd_scores_tc_supported(d)) {
      // S, G_p on tcgen05 with the tokens as N, softmax and g_s in the same kernel
      st = launch_bwd_scores_tc(p, x, W_K, W_V, g_a, slots, slot_rows, s);
    } else {
      {
        LaunchTimer t("bwd_dense_scores", s);
        k_bwd_dense_scores<<<(unsigned)(n_dt * (slot_rows / DB_J)), 256, 0, s>>>(
            x, W_K, W_V, wt, g_a, p->perm, p->group_tok_start, p->group_row_start, p->group_rows,
            p->dense_tiles, slots, slot_rows, (int)d.d_in, (int)d.d_emb);
      }
      {
        LaunchTimer t("bwd_dense_softmax", s);
        k_bwd_dense_softmax<<<(unsigned)n_dt, DENSE_TILE_M, 0, s>>>(
            p->group_tok_start, p->group_rows, p->dense_tiles, slots, slot_rows);
      }
    }
    if (st == L3_OK && bwd_dx_tc_supported(d)) {
      st = launch_bwd_dx_tc(p, W_K, slots, slot_rows, dx, s);
    } else if (st == L3_OK) {
      LaunchTimer t("bwd_dense_dx", s);
      k_bwd_dense_dx<<<(unsigned)(n_dt * (d.d_in / 64)), 256, 0, s>>>(
          W_K, wt, p->perm, p->group_tok_start, p->group_row_start, p->group_rows, p->dense_tiles,
          slots, slot_rows, (int)d.d_in, dx);
    }
    e = cudaGetLastError();
    const size_t dw_smem = 4 * 64 * DW_LD * sizeof(__nv_bfloat16);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_attn_backward_dw, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)dw_smem);
    if (e == cudaSuccess && st == L3_OK) {
      LaunchTimer t("bwd_dense_dw", s);
      const int64_t n_cb = d.d_in / DW_C + d.d_emb / DW_C;
      k_attn_backward_dw<<<(unsigned)(n_dt * n_cb), 256, dw_smem, s>>>(
          x, wt, g_a, p->perm, p->group_tok_start, p->group_row_start, p->group_rows,
          p->dense_tiles, slots, slot_rows, (int)d.d_in, (int)d.d_emb, dW_K, dW_V);
      e = cudaGetLastError();
    }
    if (e != cudaSuccess) st = cuda_fail(e, "attention backward (dense tiles)");
  }
  cache_give(scratch, got, p->device, s);
  return st;
}
