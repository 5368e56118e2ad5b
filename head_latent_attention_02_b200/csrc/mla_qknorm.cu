// mla_qknorm.cu -- the query side and the weight preparation of QK-normed MLA.
//
// What it computes (the "QK-Normed MLA" abstract: an RMSNorm over the content
// query and over each token's content keys, applied after the key up-
// projection, kept compatible with the absorbed decode).  The heads form one
// group: the query statistic is taken over the H * d_n content values of a
// query row, the key statistic over the H * d_n content keys U_K c_t of a
// token.  In the absorbed form the normalised query carries both RMSNorm
// weights, q' = (q / rms(q)) * g_q * g_k, and is absorbed as usual; the key
// side reduces to one inverse RMS per cached token, which the cache writer
// stores beside the row and the decode applies per score column.
//
// The key statistic needs mean_j (U_K c_t)_j^2 = c_t^T G c_t with the Gram
// matrix G = U_K^T U_K / (H d_n) of the stacked key weights: d_c^2 products
// per token instead of H d_n d_c.  G depends on the weights only.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "mla.h"

namespace {

template <typename T> __device__ __forceinline__ float ld_f(const T* p, size_t i);
template <> __device__ __forceinline__ float ld_f<float>(const float* p, size_t i) { return p[i]; }
template <> __device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}
template <typename T> __device__ __forceinline__ void st_f(T* p, size_t i, float x);
template <> __device__ __forceinline__ void st_f<float>(float* p, size_t i, float x) { p[i] = x; }
template <> __device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16* p, size_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

constexpr int kNormThreads = 256;

// One block per query row: the sum of squares over its n = H * d_n content
// values (fp32, block tree reduction), then q' = q * rsqrt(mean + eps) *
// g_q * g_k rounded to the storage type.
template <typename T>
__global__ void __launch_bounds__(kNormThreads) qknorm_query_kernel(int n, const T* q,
                                                                     const float* g_q,
                                                                     const float* g_k, float eps,
                                                                     T* out) {
  __shared__ float red[kNormThreads / 32];
  const size_t base = (size_t)blockIdx.x * n;
  float ss = 0.f;
  for (int i = threadIdx.x; i < n; i += kNormThreads) {
    const float x = ld_f(q, base + i);
    ss = fmaf(x, x, ss);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kNormThreads / 32; ++w) tot += red[w];
  const float inv = rsqrtf(tot / (float)n + eps);
  for (int i = threadIdx.x; i < n; i += kNormThreads)
    st_f(out, base + i, ld_f(q, base + i) * inv * g_q[i] * g_k[i]);
}

constexpr int kGramTile = 64;
constexpr int kGramK = 32;

// G = W^T W / rows for W = [rows, d] (the key weights stacked over heads):
// a 64 x 64 tile of G per block, 256 threads with 4 x 4 outputs each, the
// contraction over rows staged through shared memory 32 rows at a time.
template <typename T>
__global__ void __launch_bounds__(256) gram_kernel(int rows, int d, const T* w, float* g) {
  __shared__ float a_s[kGramK][kGramTile];
  __shared__ float b_s[kGramK][kGramTile];
  const int i0 = blockIdx.y * kGramTile, j0 = blockIdx.x * kGramTile;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int r0 = 0; r0 < rows; r0 += kGramK) {
    for (int e = threadIdx.x; e < kGramK * kGramTile; e += 256) {
      const int rr = e / kGramTile, cc = e % kGramTile;
      const int r = r0 + rr;
      a_s[rr][cc] = (r < rows && i0 + cc < d) ? ld_f(w, (size_t)r * d + i0 + cc) : 0.f;
      b_s[rr][cc] = (r < rows && j0 + cc < d) ? ld_f(w, (size_t)r * d + j0 + cc) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < kGramK; ++k) {
      float av[4], bv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        av[u] = a_s[k][ty * 4 + u];
        bv[u] = b_s[k][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
    }
    __syncthreads();
  }
  const float inv_rows = 1.f / (float)rows;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int i = i0 + ty * 4 + u, j = j0 + tx * 4 + v;
      if (i < d && j < d) g[(size_t)i * d + j] = acc[u][v] * inv_rows;
    }
}

bool dims_valid(const mla_dims_t* d) {
  return d && d->H > 0 && d->d_c > 0 && d->d_n > 0 &&
         (d->dtype == MLA_BF16 || d->dtype == MLA_F32);
}

}  // namespace

extern "C" mla_status_t mla_qknorm_query(const mla_dims_t* dims, int32_t n_rows,
                                         const void* q_nope, const float* g_q, const float* g_k,
                                         float eps, void* q_out, mla_stream_t stream) {
  if (!dims_valid(dims) || n_rows < 0 || !(eps >= 0.f)) return MLA_ERR_INVALID_ARG;
  if (n_rows == 0) return MLA_OK;
  if (!q_nope || !g_q || !g_k || !q_out) return MLA_ERR_INVALID_ARG;
  const long long n = (long long)dims->H * dims->d_n;
  if (n > (1 << 30)) return MLA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16)
    qknorm_query_kernel<__nv_bfloat16><<<n_rows, kNormThreads, 0, st>>>(
        (int)n, static_cast<const __nv_bfloat16*>(q_nope), g_q, g_k, eps,
        static_cast<__nv_bfloat16*>(q_out));
  else
    qknorm_query_kernel<float><<<n_rows, kNormThreads, 0, st>>>(
        (int)n, static_cast<const float*>(q_nope), g_q, g_k, eps, static_cast<float*>(q_out));
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

extern "C" mla_status_t mla_qknorm_key_gram(const mla_dims_t* dims, const void* w_uk, float* gram,
                                            mla_stream_t stream) {
  if (!dims_valid(dims) || !w_uk || !gram) return MLA_ERR_INVALID_ARG;
  const long long rows = (long long)dims->H * dims->d_n;
  if (rows > (1 << 30)) return MLA_ERR_UNSUPPORTED;
  const int t = (dims->d_c + kGramTile - 1) / kGramTile;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16)
    gram_kernel<__nv_bfloat16><<<dim3(t, t), 256, 0, st>>>(
        (int)rows, dims->d_c, static_cast<const __nv_bfloat16*>(w_uk), gram);
  else
    gram_kernel<float><<<dim3(t, t), 256, 0, st>>>((int)rows, dims->d_c,
                                                   static_cast<const float*>(w_uk), gram);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
