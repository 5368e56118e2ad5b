// common.cuh -- shared definitions of libmla's kernels (single translation unit).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mla.h"

namespace mla {

// Device status word: the first error a kernel meets while it runs.
__device__ int g_status;

__device__ __forceinline__ void set_status(int code) { atomicCAS(&g_status, 0, code); }

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Round a float to the nearest bfloat16 and back (the precision an operand
// has inside a bf16 tensor-core product).
__device__ __forceinline__ float round_bf16(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

constexpr int kPage = 64;
constexpr int kMaxVersions = 8;
constexpr float kNegInf = -__builtin_huge_valf();

// Description of one mla_decode call as the kernels see it.
struct DecodeArgs {
  int B, s_q, n_q, H, n_h, d_c, d_r, n_ver;
  int qH;                       // heads per query row of the q_abs the kernels read
  const int32_t* head_ids;      // [n_h] output head of each decoded head, or null = 0..n_h-1
  const float* key_inv;         // QK-normed decode: [n_pages * 64] inverse key RMS per cache row
  int max_pages, max_segs, max_gather;
  long long n_pages;
  float scale;
  const void* q_abs;
  const void* cache;
  const int32_t* block_table;
  const mla_seg_t* segs;
  const int32_t* gather_rows;   // may be null
  const int32_t* n_gather;      // null when gather_rows is null
  const int32_t* q_pos;
  float* o_lat;
  float* lse;
};

// Output head of the k-th decoded head: head_ids[k], or k when the call gives
// no list.  An id outside [0, H) records MLA_ERR_BAD_INDEX and yields -1 (the
// head's results are not written).
__device__ __forceinline__ int head_of(const DecodeArgs& a, int k) {
  if (!a.head_ids) return k;
  const int h = __ldg(a.head_ids + k);
  if (h < 0 || h >= a.H) {
    set_status(MLA_ERR_BAD_INDEX);
    return -1;
  }
  return h;
}

// Cache row of attended index `i` of sequence b (page mode: i-th row of the
// concatenated segments; gather mode: gather_rows[b][i]).  Returns false when
// the row cannot be located (bad gather row or page id), after recording
// MLA_ERR_BAD_INDEX.  On success fills the physical row (page*64+slot), the
// row's request position and its query version.
__device__ __forceinline__ bool locate_row(const DecodeArgs& a, int b, int i, long long* phys,
                                           int* kpos, int* ver) {
  const mla_seg_t* sg = a.segs + (size_t)b * a.max_segs;
  int row = -1, s_hit = -1;
  if (a.gather_rows) {
    row = a.gather_rows[(size_t)b * a.max_gather + i];
    for (int s = 0; s < a.max_segs; ++s) {
      if (row >= sg[s].row_begin && row < sg[s].row_end) { s_hit = s; break; }
    }
  } else {
    int rem = i;
    for (int s = 0; s < a.max_segs; ++s) {
      const int len = sg[s].row_end - sg[s].row_begin;
      if (len <= 0) continue;
      if (rem < len) { s_hit = s; row = sg[s].row_begin + rem; break; }
      rem -= len;
    }
  }
  if (s_hit < 0 || row < 0 || row / kPage >= a.max_pages) {
    set_status(MLA_ERR_BAD_INDEX);
    return false;
  }
  const int page = a.block_table[(size_t)b * a.max_pages + row / kPage];
  const int v = sg[s_hit].q_version;
  if (page < 0 || page >= a.n_pages || v < 0 || v >= a.n_ver) {
    set_status(MLA_ERR_BAD_INDEX);
    return false;
  }
  *phys = (long long)page * kPage + (row % kPage);
  *kpos = sg[s_hit].key_pos_base + (row - sg[s_hit].row_begin);
  *ver = v;
  return true;
}

// Number of attended rows of sequence b.
__device__ __forceinline__ int attended_rows(const DecodeArgs& a, int b) {
  if (a.gather_rows) return a.n_gather[b];
  const mla_seg_t* sg = a.segs + (size_t)b * a.max_segs;
  int n = 0;
  for (int s = 0; s < a.max_segs; ++s) n += max(0, sg[s].row_end - sg[s].row_begin);
  return n;
}

}  // namespace mla
