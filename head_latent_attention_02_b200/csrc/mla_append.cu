// mla_append.cu -- the cache writer: new tokens into the paged latent cache.
//
// What it computes (Day 27 tutorial "Multi-Head Latent Attention", section
// "Position Rotations Complicate the Absorption": the decoupled rotary key is
// kept in the cache beside the latent; RedKnot-MLA abstract: a document is
// cached at canonical positions 0, 1, ... and relocated on the query side).
// Entry i of a call becomes the cache row of logical row row[i] of sequence
// seq[i] -- page block_table[seq][row / 64], slot row % 64 --
//     [ c_new[i] | R(cache_pos[i]) k_rope_raw[i] ],
// R rotating each adjacent feature pair (2j, 2j + 1) by
// cache_pos * base^(-2j / d_r), the angle in double precision and the
// rotation rounded to the storage type, as mla_absorb_q rotates queries.
//
// QK-normed caches ("QK-Normed MLA" abstract) also keep one statistic per
// row: with the key Gram matrix G = U_K^T U_K / (H d_n) given, the writer
// computes the inverse key RMS inv = 1 / sqrt(c^T G c + eps) of the row,
// stores it at key_inv_rms[page * 64 + slot] and stores the rotary key
// multiplied by 1 / inv, so that the decode's full 576-wide score times inv
// is the normalised content score plus the plain rotary score.
//
// HBM-bound: one warp per entry copies the latent in 16-byte chunks and
// rotates the rotary pairs lane by lane (c^T G c reads G from L2 once per
// row: d_c^2 multiply-adds per row).  This file is its own translation
// unit, hence its own module with its own status word, which mla_get_status
// reads together with the decode module's.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "mla.h"

namespace mla {
namespace {

constexpr int kRowsPerPage = 64;
constexpr int kAppendThreads = 256;

__device__ int g_append_status;

struct AppendArgs {
  int n_new, B, d_c, d_r, max_pages;
  long long n_pages;
  double rope_base;
  const void* c_new;
  const void* k_raw;
  const int32_t* cache_pos;
  const int32_t* seq;
  const int32_t* row;
  void* cache;
  const int32_t* block_table;
  const float* gram;   // [d_c, d_c] or null: plain rows
  float eps;
  float* key_inv;      // [n_pages * 64] when gram is given
};

__device__ __forceinline__ double load_d(const float* p, int i) { return p[i]; }
__device__ __forceinline__ double load_d(const __nv_bfloat16* p, int i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_f(float* p, int i, float x) { p[i] = x; }
__device__ __forceinline__ void store_f(__nv_bfloat16* p, int i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

template <typename T>
__global__ void __launch_bounds__(kAppendThreads) append_rows_kernel(AppendArgs a) {
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= a.n_new) return;
  const int i = (int)gw;
  const int b = a.seq[i], r = a.row[i];
  int page = -1;
  if (b >= 0 && b < a.B && r >= 0 && r / kRowsPerPage < a.max_pages)
    page = a.block_table[(size_t)b * a.max_pages + r / kRowsPerPage];
  if (page < 0 || page >= a.n_pages) {
    if (lane == 0) atomicCAS(&g_append_status, 0, (int)MLA_ERR_BAD_INDEX);
    return;
  }
  const int width = a.d_c + a.d_r;
  T* dst = static_cast<T*>(a.cache) + ((size_t)page * kRowsPerPage + r % kRowsPerPage) * width;
  const T* c = static_cast<const T*>(a.c_new) + (size_t)i * a.d_c;
  const size_t c_bytes = (size_t)a.d_c * sizeof(T);
  if (c_bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(c) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
    const uint4* s4 = reinterpret_cast<const uint4*>(c);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    for (size_t j = lane; j < c_bytes / 16; j += 32) d4[j] = s4[j];
  } else {
    for (int j = lane; j < a.d_c; j += 32) dst[j] = c[j];
  }
  // QK-normed rows: c^T G c, lanes splitting each row of G (coalesced)
  double kscale = 1.0;
  if (a.gram) {
    float part = 0.f;
    for (int r0 = 0; r0 < a.d_c; ++r0) {
      float dot = 0.f;
      for (int j = lane; j < a.d_c; j += 32)
        dot = fmaf(__ldg(a.gram + (size_t)r0 * a.d_c + j), (float)load_d(c, j), dot);
      part = fmaf((float)load_d(c, r0), dot, part);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    const float ms = fmaxf(part, 0.f) + a.eps;
    const float inv = rsqrtf(ms);
    kscale = sqrt((double)ms);
    if (lane == 0) a.key_inv[(size_t)page * kRowsPerPage + r % kRowsPerPage] = inv;
  }
  const T* k = static_cast<const T*>(a.k_raw) + (size_t)i * a.d_r;
  T* kd = dst + a.d_c;
  const double pos = (double)a.cache_pos[i];
  for (int j = lane; j < a.d_r / 2; j += 32) {
    const double theta = pow(a.rope_base, -2.0 * j / a.d_r);
    double sn, cs;
    sincos(pos * theta, &sn, &cs);
    const double x0 = load_d(k, 2 * j), x1 = load_d(k, 2 * j + 1);
    store_f(kd, 2 * j, (float)((x0 * cs - x1 * sn) * kscale));
    store_f(kd, 2 * j + 1, (float)((x0 * sn + x1 * cs) * kscale));
  }
}

}  // namespace

// Reads and clears this module's status word (mla_get_status calls it after
// synchronising the stream).
int append_take_status() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_append_status, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_append_status, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  return v;
}

}  // namespace mla

extern "C" mla_status_t mla_append_rows(const mla_dims_t* dims, int32_t n_new, const void* c_new,
                                        const void* k_rope_raw, const int32_t* cache_pos,
                                        const int32_t* seq, const int32_t* row, int32_t B,
                                        void* cache, int64_t n_pages, const int32_t* block_table,
                                        int32_t max_pages, const float* key_gram,
                                        float qk_eps, float* key_inv_rms, mla_stream_t stream) {
  if (!dims || dims->d_c <= 0 || dims->d_r < 0 || dims->d_r % 2 != 0 ||
      (dims->dtype != MLA_F32 && dims->dtype != MLA_BF16) || !(dims->rope_base > 0.0) ||
      n_new < 0 || B < 1 || n_pages < 1 || max_pages < 1)
    return MLA_ERR_INVALID_ARG;
  if (dims->page_size != mla::kRowsPerPage) return MLA_ERR_UNSUPPORTED;
  if (n_new == 0) return MLA_OK;
  if (!c_new || !k_rope_raw || !cache_pos || !seq || !row || !cache || !block_table)
    return MLA_ERR_INVALID_ARG;
  if ((key_gram == nullptr) != (key_inv_rms == nullptr) || (key_gram && !(qk_eps >= 0.f)))
    return MLA_ERR_INVALID_ARG;
  const size_t es = dims->dtype == MLA_BF16 ? 2 : 4;
  if ((reinterpret_cast<uintptr_t>(cache) % es) || (reinterpret_cast<uintptr_t>(c_new) % es) ||
      (reinterpret_cast<uintptr_t>(k_rope_raw) % es))
    return MLA_ERR_INVALID_ARG;
  mla::AppendArgs a;
  a.n_new = n_new;
  a.B = B;
  a.d_c = dims->d_c;
  a.d_r = dims->d_r;
  a.max_pages = max_pages;
  a.n_pages = n_pages;
  a.rope_base = dims->rope_base;
  a.c_new = c_new;
  a.k_raw = k_rope_raw;
  a.cache_pos = cache_pos;
  a.seq = seq;
  a.row = row;
  a.cache = cache;
  a.block_table = block_table;
  a.gram = key_gram;
  a.eps = qk_eps;
  a.key_inv = key_inv_rms;
  const long long threads = (long long)n_new * 32;
  const unsigned blocks = (unsigned)((threads + mla::kAppendThreads - 1) / mla::kAppendThreads);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16)
    mla::append_rows_kernel<__nv_bfloat16><<<blocks, mla::kAppendThreads, 0, st>>>(a);
  else
    mla::append_rows_kernel<float><<<blocks, mla::kAppendThreads, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
