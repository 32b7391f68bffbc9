// CUDA-core (FFMA) GEMMs and LayerNorm for the fp32 layer, where tensor
// cores would need TF32 and its 10-bit mantissa.
//
// kimjy99 review, Method, eq. L³:
//   z = W_up a;  h = LayerNorm(z) over d_up (biased variance, gamma, beta, eps);
//   y = W_mix [h ; x] = W_mix[:, :d_up] h + W_mix[:, d_up:] x
// The concat [h ; x] is never materialised: W_mix is applied as two K-ranges
// accumulated into the same registers. Here every operand is widened to fp32
// (the bf16 layer's fp16 intermediates a and h included).
#include <cuda_fp16.h>

#include "l3_internal.cuh"

namespace l3 {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, THREADS = 256;
enum { ELT_F32 = 0, ELT_BF16 = 1, ELT_F16 = 2 };

template <typename T>
__device__ __forceinline__ float ld_f32(const T *p);
template <>
__device__ __forceinline__ float ld_f32<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ float ld_any(const void *p, int type, int64_t i) {
  if (type == ELT_F32) return reinterpret_cast<const float *>(p)[i];
  if (type == ELT_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
  return __half2float(reinterpret_cast<const __half *>(p)[i]);
}

template <typename T>
__device__ __forceinline__ void st_out(T *p, float v);
template <>
__device__ __forceinline__ void st_out<float>(float *p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st_out<__nv_bfloat16>(__nv_bfloat16 *p, float v) {
  *p = __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ void st_out<__half>(__half *p, float v) { *p = __float2half_rn(v); }

struct Range {
  const void *A;  // [M x K] row-major, lda
  const void *B;  // [N x K] row-major, ldb (so C = A B^T)
  int64_t lda, ldb;
  int K;
  int a_type, b_type;  // ELT_*
};

// C[m][n] = sum over ranges r of sum_k A_r[m][k] * B_r[n][k]   (fp32 accumulate)
template <typename TOut>
__global__ void __launch_bounds__(THREADS)
    k_gemm_simt(Range r0, Range r1, int n_ranges, TOut *__restrict__ C, int64_t ldc, int M, int N) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int r = 0; r < n_ranges; ++r) {
    const Range R = r == 0 ? r0 : r1;
    for (int k0 = 0; k0 < R.K; k0 += BK) {
#pragma unroll
      for (int i = 0; i < (BM * BK) / THREADS; ++i) {
        int e = tid + i * THREADS;
        int row = e / BK, kk = e % BK;
        int gm = m0 + row, gk = k0 + kk;
        As[kk][row] = (gm < M && gk < R.K) ? ld_any(R.A, R.a_type, (int64_t)gm * R.lda + gk) : 0.f;
        int gn = n0 + row;
        Bs[kk][row] = (gn < N && gk < R.K) ? ld_any(R.B, R.b_type, (int64_t)gn * R.ldb + gk) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < BK; ++kk) {
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
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int gn = n0 + tx * 4 + j;
      if (gn < N) st_out(C + (int64_t)gm * ldc + gn, acc[i][j]);
    }
  }
}

// h = gamma * (z - mean) / sqrt(var + eps) + beta, one warp per row, two-pass
// (mean first, then the biased variance about it).
template <typename T, typename TH>
__global__ void k_layernorm(const float *__restrict__ z, int d, const T *__restrict__ gamma,
                            const T *__restrict__ beta, float eps, TH *__restrict__ h, int64_t M) {
  int64_t row = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x % 32;
  if (row >= M) return;
  const float *zr = z + row * d;
  float s = 0.f;
  for (int u = lane; u < d; u += 32) s += zr[u];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  float mu = s / d;
  float q = 0.f;
  for (int u = lane; u < d; u += 32) {
    float c = zr[u] - mu;
    q = fmaf(c, c, q);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  float rstd = 1.0f / sqrtf(q / d + eps);
  TH *hr = h + row * d;
  for (int u = lane; u < d; u += 32)
    st_out(hr + u, ld_f32(gamma + u) * ((zr[u] - mu) * rstd) + ld_f32(beta + u));
}

template <typename T, typename TH>
l3_status up_ln_typed(const l3_plan_s *p, const void *W_up, const void *gamma, const void *beta,
                      cudaStream_t s) {
  const int M = (int)p->n_tokens, N = (int)p->dims.d_up;
  const int ta = sizeof(TH) == 4 ? ELT_F32 : ELT_F16;
  const int tb = sizeof(T) == 4 ? ELT_F32 : ELT_BF16;
  Range r0{p->a_buf, W_up, p->dims.d_emb, p->dims.d_emb, (int)p->dims.d_emb, ta, tb};
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  {
    LaunchTimer t("up_gemm_simt", s);
    k_gemm_simt<float><<<grid, THREADS, 0, s>>>(r0, r0, 1, p->z_buf, N, M, N);
  }
  {
    LaunchTimer t("layernorm", s);
    k_layernorm<T, TH><<<(M + 7) / 8, 256, 0, s>>>(p->z_buf, N, reinterpret_cast<const T *>(gamma),
                                                   reinterpret_cast<const T *>(beta),
                                                   p->dims.ln_eps,
                                                   reinterpret_cast<TH *>(p->h_buf), M);
  }
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

template <typename T, typename TH>
l3_status mix_typed(const l3_plan_s *p, const void *x, const void *W_mix, void *y,
                    cudaStream_t s) {
  const int M = (int)p->n_tokens, N = (int)p->dims.d_out;
  const int64_t ldw = p->dims.d_up + p->dims.d_in;
  const int th = sizeof(TH) == 4 ? ELT_F32 : ELT_F16;
  const int tw = sizeof(T) == 4 ? ELT_F32 : ELT_BF16;
  const T *W = reinterpret_cast<const T *>(W_mix);
  Range r0{p->h_buf, W, p->dims.d_up, ldw, (int)p->dims.d_up, th, tw};
  Range r1{x, W + p->dims.d_up, p->dims.d_in, ldw, (int)p->dims.d_in, tw, tw};
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  LaunchTimer t("mix_gemm_simt", s);
  k_gemm_simt<T><<<grid, THREADS, 0, s>>>(r0, r1, 2, reinterpret_cast<T *>(y), N, M, N);
  L3_CUDA_TRY(cudaGetLastError());
  return L3_OK;
}

}  // namespace

l3_status launch_up_ln_simt(const l3_plan_s *p, const void *W_up, const void *gamma,
                            const void *beta, cudaStream_t s) {
  return p->dims.dtype == L3_BF16 ? up_ln_typed<__nv_bfloat16, __half>(p, W_up, gamma, beta, s)
                                  : up_ln_typed<float, float>(p, W_up, gamma, beta, s);
}

l3_status launch_mix_simt(const l3_plan_s *p, const void *x, const void *W_mix, void *y,
                          cudaStream_t s) {
  return p->dims.dtype == L3_BF16 ? mix_typed<__nv_bfloat16, __half>(p, x, W_mix, y, s)
                                  : mix_typed<float, float>(p, x, W_mix, y, s);
}

}  // namespace l3
