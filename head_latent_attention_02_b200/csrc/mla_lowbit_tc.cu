// mla_lowbit_tc.cu -- the tensor-core route of the low-bit latent cache
// (QuantMLA abstract: content and rotary caches kept as INT4 / INT4 or
// INT2 / INT4 codes with one static scale per channel).
//
// A pre-pass dequantises the packed rows into a pool of dtype rows,
//     out[r][k] = code_k(r) * scale_k      (the product in fp32, then rounded),
// and the decode is mla_decode over that pool, so the scores and the
// weighted sum run on the tcgen05 path instead of the SIMT kernel of the
// fused low-bit decode.  The pre-pass reads the packed bytes once and writes
// the dequantised rows once; for pools of up to ~100 MB the decode then
// reads them back from L2.
//
// Packed row layout (the one mla_pack_rows writes): d_c content codes of
// bits_c bits, then d_r rotary codes of bits_r bits, code k of a segment in
// bits [bits * k mod 32, ...) of 32-bit word bits * k / 32 of the segment,
// two's complement.
//
// This file is its own translation unit; its only kernel has no failure
// mode of its own (every index is in range by construction), and the
// decode it chains to records its errors in the decode module's status.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "mla.h"

namespace mla {
namespace {

// The codes of one word as exact floats.  XOR with the sign bit of every
// field turns code c into c + 2^(B-1) in [0, 2^B); masking puts one field in
// each byte; a byte permute then builds the float 2^23 + (c + 2^(B-1))
// (0x4B0000 in the upper bytes, the field in the lowest), and one exact
// subtraction leaves c.  Per code: one PRMT and one FADD, no int-to-float
// conversion.
template <int B>
struct Codes;

template <>
struct Codes<4> {   // code j in bits [4j, 4j + 4): byte b holds codes 2b, 2b + 1
  __device__ static void get(uint32_t w, float* f) {
    w ^= 0x88888888u;
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      f[2 * b] = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7540u + b)) - 8388616.0f;
      f[2 * b + 1] = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7540u + b)) - 8388616.0f;
    }
  }
};

template <>
struct Codes<2> {   // code j in bits [2j, 2j + 2): byte b holds codes 4b .. 4b + 3
  __device__ static void get(uint32_t w, float* f) {
    w ^= 0xAAAAAAAAu;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint32_t q = (w >> (2 * s)) & 0x03030303u;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        f[4 * b + s] = __uint_as_float(__byte_perm(q, 0x4B000000u, 0x7540u + b)) - 8388610.0f;
    }
  }
};

__device__ __forceinline__ void put8(__nv_bfloat16* dst, const float* v) {
  uint4 o;
  uint32_t* h = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    h[j] = *reinterpret_cast<const uint32_t*>(&t);
  }
  *reinterpret_cast<uint4*>(dst) = o;
}

__device__ __forceinline__ void put8(float* dst, const float* v) {
  *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// Rows in passes of R (= blockDim.x / row_words) rows per block: thread t
// owns word w = t mod row_words of row t / row_words of each pass, so its
// 32 / B channels -- and their scales, held in registers -- never change.
// A block reads R consecutive packed rows (consecutive threads, consecutive
// words) and writes R consecutive output rows; kDqUnroll passes' loads are
// issued before any is decoded.
constexpr int kDqUnroll = 4;

template <typename T, int B>
__device__ __forceinline__ void dequant_slot(const uint32_t* packed, T* out, long long n_rows,
                                             int row_words, int width, int w, int k0,
                                             long long r0, long long step, const float* sv) {
  for (long long r = r0; r < n_rows; r += kDqUnroll * step) {
    uint32_t x[kDqUnroll];
#pragma unroll
    for (int u = 0; u < kDqUnroll; ++u) {
      const long long ru = r + u * step;
      x[u] = ru < n_rows ? __ldg(packed + ru * row_words + w) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kDqUnroll; ++u) {
      const long long ru = r + u * step;
      if (ru < n_rows) {
        float f[32 / B];
        Codes<B>::get(x[u], f);
#pragma unroll
        for (int j = 0; j < 32 / B; ++j) f[j] *= sv[j];
#pragma unroll
        for (int j0 = 0; j0 < 32 / B; j0 += 8) put8(out + ru * width + k0 + j0, f + j0);
      }
    }
  }
}

template <typename T, int BC, int BR>
__global__ void __launch_bounds__(1024) dequant_rows_kernel(long long n_rows, int d_c, int d_r,
                                                            const uint32_t* packed,
                                                            const float* scale_c,
                                                            const float* scale_r, T* out) {
  const int cwords = d_c * BC / 32, row_words = cwords + d_r * BR / 32;
  const int rows_per_pass = blockDim.x / row_words;
  const int t = threadIdx.x;
  if (t >= rows_per_pass * row_words) return;
  const int q = t / row_words, w = t - q * row_words;
  const long long r0 = (long long)blockIdx.x * rows_per_pass + q;
  const long long step = (long long)gridDim.x * rows_per_pass;
  const int width = d_c + d_r;
  if (w < cwords) {
    float sv[32 / BC];
#pragma unroll
    for (int j = 0; j < 32 / BC; ++j) sv[j] = scale_c[w * (32 / BC) + j];
    dequant_slot<T, BC>(packed, out, n_rows, row_words, width, w, w * (32 / BC), r0, step, sv);
  } else {
    const int k0 = (w - cwords) * (32 / BR);
    float sv[32 / BR];
#pragma unroll
    for (int j = 0; j < 32 / BR; ++j) sv[j] = scale_r[k0 + j];
    dequant_slot<T, BR>(packed, out, n_rows, row_words, width, w, d_c + k0, r0, step, sv);
  }
}

bool pair_ok(const mla_dims_t* d, int bits_c, int bits_r) {
  return ((bits_c == 4 && bits_r == 4) || (bits_c == 2 && bits_r == 4)) && d->d_c > 0 &&
         d->d_r >= 0 && (d->d_c * bits_c) % 32 == 0 && (d->d_r * bits_r) % 32 == 0 &&
         (d->dtype == MLA_BF16 || d->dtype == MLA_F32);
}

bool aligned_to(const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

template <typename T>
cudaError_t launch(int bits_c, long long n_rows, const mla_dims_t* d, const void* packed,
                   const float* sc, const float* sr, void* out, cudaStream_t st) {
  static int n_sm = 0;
  if (n_sm == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return cudaErrorUnknown;
  }
  // rows per pass: the fewest that fill whole warps (32 / gcd(row_words,
  // 32)), repeated up to ~512 threads; when those rows need more than 1024
  // threads, as many rows as 1024 threads hold (the last warp then partial)
  const int row_words = (d->d_c * bits_c + d->d_r * 4) / 32;
  int g = row_words, b = 32;
  while (b) { const int t = g % b; g = b; b = t; }
  int rows = 32 / g;
  if (rows * row_words > 1024) rows = 1024 / row_words > 0 ? 1024 / row_words : 1;
  else rows *= (512 / (rows * row_words) > 1 ? 512 / (rows * row_words) : 1);
  const int threads = rows * row_words;
  const long long need = (n_rows + (long long)rows * kDqUnroll - 1) / ((long long)rows * kDqUnroll);
  const long long cap = (long long)n_sm * (2048 / threads > 0 ? 2048 / threads : 1);
  const unsigned blocks = (unsigned)(need < cap ? need : cap);
  const uint32_t* src = static_cast<const uint32_t*>(packed);
  if (bits_c == 4)
    dequant_rows_kernel<T, 4, 4><<<blocks, threads, 0, st>>>(n_rows, d->d_c, d->d_r, src, sc, sr,
                                                              static_cast<T*>(out));
  else
    dequant_rows_kernel<T, 2, 4><<<blocks, threads, 0, st>>>(n_rows, d->d_c, d->d_r, src, sc, sr,
                                                              static_cast<T*>(out));
  return cudaGetLastError();
}

}  // namespace
}  // namespace mla

extern "C" {

size_t mla_lowbit_dequant_bytes(const mla_dims_t* dims, int64_t n_pages) {
  if (!dims || n_pages < 0 || dims->page_size < 1 || dims->d_c < 1 || dims->d_r < 0) return 0;
  const size_t es = dims->dtype == MLA_BF16 ? 2 : 4;
  return (size_t)n_pages * dims->page_size * (dims->d_c + dims->d_r) * es;
}

mla_status_t mla_dequant_rows(const mla_dims_t* dims, int32_t bits_c, int32_t bits_r,
                              int64_t n_rows, const void* packed, const float* scale_c,
                              const float* scale_r, void* out, mla_stream_t stream) {
  if (!dims || n_rows < 0) return MLA_ERR_INVALID_ARG;
  if (!mla::pair_ok(dims, bits_c, bits_r)) return MLA_ERR_UNSUPPORTED;
  if (n_rows == 0) return MLA_OK;
  if (!packed || !scale_c || !scale_r || !out || !mla::aligned_to(packed, 4) ||
      !mla::aligned_to(out, 16))
    return MLA_ERR_INVALID_ARG;
  // one thread per packed word of a row: at most 1024 words per row
  if ((dims->d_c * bits_c + dims->d_r * bits_r) / 32 > 1024) return MLA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e =
      dims->dtype == MLA_BF16
          ? mla::launch<__nv_bfloat16>(bits_c, n_rows, dims, packed, scale_c, scale_r, out, st)
          : mla::launch<float>(bits_c, n_rows, dims, packed, scale_c, scale_r, out, st);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status_t mla_decode_lowbit_tc(const mla_dims_t* dims, int32_t bits_c, int32_t bits_r,
                                  int32_t B, int32_t s_q, const void* q_abs, int32_t n_ver,
                                  const int32_t* head_ids, int32_t n_h, const void* cache,
                                  const float* scale_c, const float* scale_r, int64_t n_pages,
                                  const int32_t* block_table, int32_t max_pages,
                                  const mla_seg_t* segs, int32_t max_segs,
                                  const int32_t* gather_rows, const int32_t* n_gather,
                                  int32_t max_gather, const int32_t* q_pos, float* o_lat,
                                  float* lse, void* dequant, size_t dequant_bytes,
                                  void* workspace, size_t ws_bytes, mla_stream_t stream) {
  if (!dims || B < 0 || n_pages < 1) return MLA_ERR_INVALID_ARG;
  if (!mla::pair_ok(dims, bits_c, bits_r)) return MLA_ERR_UNSUPPORTED;
  if (B == 0) return MLA_OK;
  if (!dequant || dequant_bytes < mla_lowbit_dequant_bytes(dims, n_pages))
    return MLA_ERR_WORKSPACE;
  // every check of the decode, before the pre-pass writes the pool: the
  // argument shapes (mla_decode with B = 0 stops after them), then pointers,
  // alignments (the decode's tensor maps want the pool 256-byte aligned) and
  // the workspace
  const mla_status_t shape =
      mla_decode(dims, 0, s_q, q_abs, n_ver, head_ids, n_h, dequant, n_pages, block_table,
                 max_pages, segs, max_segs, gather_rows, n_gather, max_gather, q_pos, o_lat, lse,
                 workspace, ws_bytes, stream);
  if (shape != MLA_OK) return shape;
  if (!q_abs || !cache || !block_table || !segs || !q_pos || !o_lat || !lse ||
      !mla::aligned_to(dequant, 256) || !mla::aligned_to(q_abs, 16) ||
      !mla::aligned_to(o_lat, 16) || !mla::aligned_to(lse, 4))
    return MLA_ERR_INVALID_ARG;
  const size_t need = mla_decode_workspace_size(dims, B, s_q, n_ver, n_h);
  if (need == 0 || !workspace || ws_bytes < need) return MLA_ERR_WORKSPACE;
  const mla_status_t s = mla_dequant_rows(dims, bits_c, bits_r, n_pages * dims->page_size, cache,
                                          scale_c, scale_r, dequant, stream);
  if (s != MLA_OK) return s;
  return mla_decode(dims, B, s_q, q_abs, n_ver, head_ids, n_h, dequant, n_pages, block_table,
                    max_pages, segs, max_segs, gather_rows, n_gather, max_gather, q_pos, o_lat,
                    lse, workspace, ws_bytes, stream);
}

}  // extern "C"
