// mla_static_ws.cu -- mla_decode_static_ws: mla_decode with its scratch taken
// from a fixed device array of this library instead of a caller workspace.
//
// Who needs it: callers that cannot allocate device memory when they decode.
// A serving host that reserves all free device memory for its KV page pool up
// front has no room left to carve the split-merge scratch (about 39 MB on a
// 148-SM device) out of at decode time, and a plain-C host that only holds
// device pointers has no allocator of its own to take a workspace from.
//
// The array sits in its own translation unit, hence its own CUDA module: with
// the runtime's lazy module loading its memory is reserved only in contexts
// that call this entry point, not by every user of the library.
#include <cuda_runtime.h>

#include "mla.h"

namespace {

// Scratch shared by every call on a device.  It keeps the previous call's
// contents; nothing in it has to start at zero, because the planning kernel
// writes the plan header and every stream offset before the decode kernel
// reads them, and every split partial the merge kernel reads is written
// earlier in the same call.  Two calls that overlap on the GPU (other streams,
// or other host threads) use the same bytes and race.
static __device__ __align__(256) unsigned char g_decode_scratch[MLA_DECODE_STATIC_WS_BYTES];

// The device address of the array in the current context.  The lookup runs
// on every call: it is a table read once the module is loaded, and it stays
// right across a device reset or a change of context, which a cached pointer
// would not.
mla_status_t scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
    cudaGetLastError();   // clear the error the failed lookup recorded
    return MLA_ERR_CUDA;
  }
  *out = p;
  return MLA_OK;
}

}  // namespace

extern "C" mla_status_t mla_decode_static_ws_init(void) {
  void* p = nullptr;
  return scratch_address(&p);
}

extern "C" mla_status_t mla_decode_static_ws(
    const mla_dims_t* dims, int32_t B, int32_t s_q, const void* q_abs, int32_t n_ver,
    const int32_t* head_ids, int32_t n_h, const void* cache, int64_t n_pages,
    const int32_t* block_table, int32_t max_pages, const mla_seg_t* segs, int32_t max_segs,
    const int32_t* gather_rows, const int32_t* n_gather, int32_t max_gather, const int32_t* q_pos,
    float* o_lat, float* lse, mla_stream_t stream) {
  // the size query answers 0 both for invalid sizes and for a device that
  // cannot be queried: tell the two apart before trusting it
  if (!dims || B < 0 || s_q < 1 || n_ver < 1 || n_h < 1 || n_h > dims->H)
    return MLA_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  const size_t need = mla_decode_workspace_size(dims, B, s_q, n_ver, n_h);
  if (need == 0) return MLA_ERR_INVALID_ARG;
  if (need > MLA_DECODE_STATIC_WS_BYTES) return MLA_ERR_WORKSPACE;
  void* ws = nullptr;
  const mla_status_t st = scratch_address(&ws);
  if (st != MLA_OK) return st;
  return mla_decode(dims, B, s_q, q_abs, n_ver, head_ids, n_h, cache, n_pages, block_table,
                    max_pages, segs, max_segs, gather_rows, n_gather, max_gather, q_pos, o_lat,
                    lse, ws, MLA_DECODE_STATIC_WS_BYTES, stream);
}
