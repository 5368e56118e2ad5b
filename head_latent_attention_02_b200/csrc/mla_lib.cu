// mla_lib.cu -- the C ABI of libmla (include/mla.h): argument validation,
// TMA descriptor set-up and kernel launches.  Single translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "mla.h"
#include "common.cuh"
#include "ptx.cuh"
#include "kernels_simt.cuh"
#include "kernels_lowbit.cuh"
#include "decode_tc.cuh"
#include "wgemm.cuh"

namespace mla {
int append_take_status();   // the cache writer's module (mla_append.cu)
}
using namespace mla;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  bool tc_attr_set = false;
  bool wg_attr_set = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

// The tensor-core kernels take nearly all of an SM's shared memory.  The
// small kernels between them ask for the same split of the unified L1/shared
// storage, so consecutive launches never make an SM switch configuration.
mla_status_t prefer_max_shared() {
  const int carveout = cudaSharedmemCarveoutMaxShared;
  const void* small[] = {
      reinterpret_cast<const void*>(&tc::plan_kernel<false>),
      reinterpret_cast<const void*>(&tc::plan_kernel<true>),
      reinterpret_cast<const void*>(&tc::combine_kernel),
      reinterpret_cast<const void*>(&merge_lse_kernel),
      reinterpret_cast<const void*>(&absorb_kernel<float>),
      reinterpret_cast<const void*>(&absorb_kernel<__nv_bfloat16>),
      reinterpret_cast<const void*>(&decode_simt_kernel<float>),
      reinterpret_cast<const void*>(&decode_simt_kernel<__nv_bfloat16>),
      reinterpret_cast<const void*>(&vproj_simt_kernel<float>),
      reinterpret_cast<const void*>(&vproj_simt_kernel<__nv_bfloat16>),
      reinterpret_cast<const void*>(&oproj_simt_kernel<float>),
      reinterpret_cast<const void*>(&oproj_simt_kernel<__nv_bfloat16>)};
  for (const void* f : small)
    if (cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, carveout) !=
        cudaSuccess)
      return MLA_ERR_CUDA;
  return MLA_OK;
}

mla_status_t device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MLA_ERR_CUDA;
    if (prefer_max_shared() != MLA_OK) return MLA_ERR_CUDA;
    d.ready = true;
  }
  *out = &d;
  return MLA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool dims_ok(const mla_dims_t* d) {
  return d && d->H > 0 && d->d_c > 0 && d->d_r >= 0 && d->d_r % 2 == 0 && d->d_n > 0 &&
         d->d_v > 0 && d->d_model >= 0 && (d->dtype == MLA_F32 || d->dtype == MLA_BF16) &&
         std::isfinite(d->scale) && d->rope_base > 0.0;
}

size_t elem_size(const mla_dims_t* d) { return d->dtype == MLA_BF16 ? 2 : 4; }

bool tc_eligible(const mla_dims_t* d) {
  return d->dtype == MLA_BF16 && d->d_c == tc::kDc && d->d_r == tc::kDr;
}

// cuTensorMapEncodeTiled, fetched from the driver at run time so that the
// library loads on machines without a driver.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map over a [rows, 576] bf16 matrix (row pitch 1152 B) with 64-column
// boxes and 128-byte swizzle.  rank 2: (col, row), box {64, h}.  rank 3:
// (col, row, 64-column panel), box {64, h, panels}: each box row is 128 *
// panels contiguous bytes, landing as `panels` planes of h x 128 bytes.
bool make_map_576(CUtensorMap* m, const void* base, uint64_t rows, int rank, uint32_t h,
                  uint32_t panels = 9) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)rows, 9};
  cuuint64_t strides[2] = {(cuuint64_t)tc::kRow * 2, 128};
  cuuint32_t box[3] = {64, h, panels};
  if (rank == 2) dims[0] = tc::kRow;
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 store map for decode outputs: (column, row[, plane]) over rows of 512
// floats, box {32, 32[, 1]}, 128-byte swizzle.  rank 3: rows are heads
// (extent n_rows) and planes are query rows (stride plane_stride floats).
bool make_map_out(CUtensorMap* m, float* base, uint64_t n_rows, uint64_t n_planes,
                  uint64_t plane_stride, int rank) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)tc::kDc, (cuuint64_t)n_rows, (cuuint64_t)n_planes};
  cuuint64_t strides[2] = {(cuuint64_t)tc::kDc * 4, (cuuint64_t)plane_stride * 4};
  cuuint32_t box[3] = {(cuuint32_t)tc::kStoreCols, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (cuuint32_t)rank, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over a row-major [rows, cols] matrix seen as (64-column
// offset, row, 64-column panel), box {64, box_rows, box_panels}, 128-byte
// swizzle: a box is box_panels panels of box_rows x 128 bytes, and each row of
// it is 128 * box_panels contiguous bytes of the matrix.
bool make_map_panels(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                     uint32_t box_rows, uint32_t box_panels) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_panels};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Panels per weight unit: long contiguous row runs for the TMA engine, but
// at least three ring stages in shared memory, and K a whole number of units.
int wgemm_panels(int K, int n_pad) {
  int P = n_pad <= 32 ? 4 : 2;
  while (P > 1 && K % (wg::kKP * P) != 0) P /= 2;
  return P;
}

// Launch one weight-streaming product, one launch per 128 query rows.  W is
// the bf16 weight as a row-major [w_rows, w_cols] matrix (absorb: W_UK seen as
// [H d_n, d_c], read M-major; otherwise [M rows, K cols]).  `split_k` lets a
// CTA's run of units start and end inside an m-tile (the output product,
// which adds into a zeroed `out`), otherwise runs are whole m-tiles.  `x_bf16`
// (absorb) is the bf16 activation matrix [n_total, x_cols] read by TMA.
mla_status_t launch_wgemm(wg::Params p, const void* w, uint64_t w_rows, uint64_t w_cols,
                          int groups, int m_tiles, int K, bool split_k, const void* x_bf16,
                          uint64_t x_cols, cudaStream_t st) {
  DeviceInfo* d = nullptr;
  if (device_info(&d) != MLA_OK) return MLA_ERR_CUDA;
  if (!d->wg_attr_set) {
    if (cudaFuncSetAttribute(wg::wgemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             wg::kSmemMax) != cudaSuccess)
      return MLA_ERR_CUDA;
    d->wg_attr_set = true;
  }
  const bool absorb = p.mode == wg::kAbsorb;
  const int total_n = p.n;
  float* zero = p.zero;
  for (int q0 = 0; q0 < total_n; q0 += 128) {
    p.q0 = q0;
    p.n = std::min(128, total_n - q0);
    p.n_pad = (p.n + 15) / 16 * 16;
    p.P = wgemm_panels(K, p.n_pad);
    p.groups = groups;
    p.m_tiles = m_tiles;
    p.k_stages = K / (wg::kKP * p.P);
    const int units = groups * m_tiles * p.k_stages;
    int grid, chunk;
    if (split_k) {
      grid = std::min(d->num_sms, units);
      chunk = (units + grid - 1) / grid;
      grid = (units + chunk - 1) / chunk;
    } else {
      const int tiles = groups * m_tiles;
      grid = std::min(d->num_sms, tiles);
      const int per = (tiles + grid - 1) / grid;
      chunk = per * p.k_stages;
      grid = (tiles + per - 1) / per;
    }
    p.chunk = chunk;
    const int stage_bytes = p.P * (wg::kWPanel + p.n_pad * 128);
    p.stages = std::min(wg::kMaxStages, (wg::kSmemMax - wg::kSmemFixed) / stage_bytes);
    if (p.stages < 2) return MLA_ERR_UNSUPPORTED;
    const int smem = p.stages * stage_bytes + wg::kSmemFixed;
    p.zero = q0 == 0 ? zero : nullptr;
    CUtensorMap tw, tx;
    std::memset(&tx, 0, sizeof(tx));
    if (!make_map_panels(&tw, w, w_cols, w_rows, absorb ? wg::kKP * p.P : wg::kMT,
                         absorb ? 2 : p.P))
      return MLA_ERR_CUDA;
    if (x_bf16 && !make_map_panels(&tx, x_bf16, x_cols, (uint64_t)p.n_total, (uint32_t)p.n_pad,
                                   (uint32_t)p.P))
      return MLA_ERR_CUDA;
    // The split-K output product is a programmatic dependent of the value
    // launch before it: its W_O stream starts at once, and only the threads
    // that read v or add into `out` wait for the value launch on device.
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(wg::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = split_k ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, wg::wgemm_kernel, p, tw, tx) != cudaSuccess) return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

struct WsLayout {
  size_t off_plan, off_streams, off_bad, off_pairs, off_partial, off_plse, off_qpack, off_opack,
      off_lpack, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Bytes of the packed queries of a call with a head list (tensor-core path).
size_t q_pack_bytes(const mla_dims_t* dims, int B, int s_q, int n_ver, int n_h) {
  return align256((size_t)n_ver * B * s_q * n_h * (dims->d_c + dims->d_r) * elem_size(dims));
}

// q_pack_bytes: room for the listed heads' packed queries (mla_decode with a
// head list); o_rows: rows (query x head) of the packed whole-stream outputs
// of a head list.
WsLayout ws_layout(int n_streams, int G, size_t q_pack_bytes, size_t o_rows) {
  WsLayout w;
  w.off_plan = 0;
  w.off_streams = align256(sizeof(tc::PlanHeader));
  w.off_bad = w.off_streams + align256(sizeof(int) * (size_t)(n_streams + 1));
  // split partials: two slots per CTA pair, 128 rows of o each, then their lse
  w.off_pairs = w.off_bad + align256(sizeof(int) * (size_t)n_streams);
  w.off_partial = w.off_pairs + align256(sizeof(int) * (size_t)G);
  w.off_plse = w.off_partial + sizeof(float) * (size_t)tc::kDc * tc::kM * 2 * (size_t)G;
  w.off_qpack = align256(w.off_plse + sizeof(float) * (size_t)tc::kM * 2 * (size_t)G);
  w.off_opack = align256(w.off_qpack + q_pack_bytes);
  w.off_lpack = w.off_opack + sizeof(float) * (size_t)tc::kDc * o_rows;
  w.total = align256(w.off_lpack + sizeof(float) * o_rows);
  return w;
}

mla_status_t launch_ok() {
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

extern "C" {

int32_t mla_abi_version(void) { return MLA_ABI_VERSION; }

const char* mla_status_str(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
    case MLA_ERR_BAD_INDEX: return "MLA_ERR_BAD_INDEX";
  }
  return "MLA_ERR_UNKNOWN";
}

mla_status_t mla_get_status(mla_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  const int va = mla::append_take_status();
  return static_cast<mla_status_t>(v ? v : va);
}

mla_status_t mla_absorb_q(const mla_dims_t* dims, int32_t n_q, const void* q_nope,
                          const void* q_rope, const int32_t* q_pos, const int32_t* delta,
                          int32_t n_ver, const void* w_uk, void* q_abs, mla_stream_t stream) {
  if (!dims_ok(dims) || n_q < 0 || n_ver < 1 || n_ver > kMaxVersions || !delta)
    return MLA_ERR_INVALID_ARG;
  if (n_q == 0) return MLA_OK;
  if (!q_nope || !q_rope || !q_pos || !w_uk || !q_abs) return MLA_ERR_INVALID_ARG;
  AbsorbArgs a;
  a.n_q = n_q;
  a.H = dims->H;
  a.d_c = dims->d_c;
  a.d_r = dims->d_r;
  a.d_n = dims->d_n;
  a.n_ver = n_ver;
  a.rope_base = dims->rope_base;
  for (int i = 0; i < kMaxVersions; ++i) a.delta[i] = i < n_ver ? delta[i] : 0;
  a.q_nope = q_nope;
  a.q_rope = q_rope;
  a.q_pos = q_pos;
  a.w_uk = w_uk;
  a.q_abs = q_abs;
  cudaStream_t st0 = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16 && dims->d_c % wg::kMT == 0 && dims->d_n % wg::kKP == 0 &&
      aligned(q_nope, 16) && aligned(q_abs, 4)) {
    wg::Params p{};
    p.mode = wg::kAbsorb;
    p.n = n_q;
    p.n_total = n_q;
    p.H = dims->H;
    p.d_c = dims->d_c;
    p.d_r = dims->d_r;
    p.d_n = dims->d_n;
    p.d_v = dims->d_v;
    p.d_model = dims->d_model;
    p.out = q_abs;
    p.n_ver = n_ver;
    for (int i = 0; i < kMaxVersions; ++i) p.delta[i] = i < n_ver ? delta[i] : 0;
    p.rope_base = dims->rope_base;
    p.q_rope = q_rope;
    p.q_pos = q_pos;
    return launch_wgemm(p, w_uk, (uint64_t)dims->H * dims->d_n, dims->d_c, dims->H,
                        dims->d_c / wg::kMT, dims->d_n, false, q_nope,
                        (uint64_t)dims->H * dims->d_n, st0);
  }
  dim3 grid(dims->H, (n_q + kAbsQ - 1) / kAbsQ);
  const size_t smem = sizeof(float) * kAbsQ * dims->d_n;
  if (smem > 48 * 1024) return MLA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16)
    absorb_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(a);
  else
    absorb_kernel<float><<<grid, 256, smem, st>>>(a);
  return launch_ok();
}

size_t mla_decode_workspace_size(const mla_dims_t* dims, int32_t B, int32_t s_q, int32_t n_ver,
                                 int32_t n_h) {
  if (!dims_ok(dims) || B < 0 || s_q < 1 || n_ver < 1 || n_ver > kMaxVersions || n_h < 1 ||
      n_h > dims->H)
    return 0;
  if (!tc_eligible(dims)) return 256;   // the generic kernel needs no scratch
  DeviceInfo* d = nullptr;
  if (device_info(&d) != MLA_OK) return 0;
  const int n_hb = (n_h + tc::kM - 1) / tc::kM;
  return ws_layout(B * s_q * n_hb, d->num_sms / 2, q_pack_bytes(dims, B, s_q, n_ver, n_h),
                   (size_t)B * s_q * n_h).total;
}

}  // extern "C"

namespace {

// mla_decode and mla_decode_qknorm: key_inv (or null) is the per-row inverse
// key RMS of the QK-normed scores.
mla_status_t decode_impl(const mla_dims_t* dims, int32_t B, int32_t s_q, const void* q_abs,
                         int32_t n_ver, const int32_t* head_ids, int32_t n_h, const void* cache,
                         int64_t n_pages, const int32_t* block_table, int32_t max_pages,
                         const mla_seg_t* segs, int32_t max_segs, const int32_t* gather_rows,
                         const int32_t* n_gather, int32_t max_gather, const int32_t* q_pos,
                         float* o_lat, float* lse, void* workspace, size_t ws_bytes,
                         mla_stream_t stream, const float* key_inv) {
  if (!dims_ok(dims) || B < 0 || s_q < 1 || n_ver < 1 || n_h < 1 || n_h > dims->H ||
      n_pages < 1 || max_pages < 1 || max_segs < 1)
    return MLA_ERR_INVALID_ARG;
  if (dims->page_size != kPage || n_ver > kMaxVersions) return MLA_ERR_UNSUPPORTED;
  if (gather_rows && (!n_gather || max_gather < 1)) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!q_abs || !cache || !block_table || !segs || !q_pos || !o_lat || !lse)
    return MLA_ERR_INVALID_ARG;
  // cache rows, logical rows and q_abs rows are 32-bit indices on the device
  if (n_pages * kPage + 2 * kPage > INT32_MAX) return MLA_ERR_UNSUPPORTED;
  if ((long long)max_pages * kPage > INT32_MAX ||
      (long long)n_ver * B * s_q * dims->H > INT32_MAX)
    return MLA_ERR_UNSUPPORTED;
  const size_t es = elem_size(dims);
  if (!aligned(cache, 256) || !aligned(q_abs, 16) || !aligned(o_lat, 16) || !aligned(lse, 4) ||
      !aligned(key_inv, 16))
    return MLA_ERR_INVALID_ARG;
  // the per-row factors are read per page: gathered rows have no page run
  if (key_inv && gather_rows) return MLA_ERR_UNSUPPORTED;

  DecodeArgs a;
  a.B = B;
  a.s_q = s_q;
  a.n_q = B * s_q;
  a.H = dims->H;
  a.qH = dims->H;
  a.head_ids = head_ids;
  a.key_inv = key_inv;
  a.n_h = n_h;
  a.d_c = dims->d_c;
  a.d_r = dims->d_r;
  a.n_ver = n_ver;
  a.max_pages = max_pages;
  a.max_segs = max_segs;
  a.max_gather = gather_rows ? max_gather : 0;
  a.n_pages = n_pages;
  a.scale = dims->scale;
  a.q_abs = q_abs;
  a.cache = cache;
  a.block_table = block_table;
  a.segs = segs;
  a.gather_rows = gather_rows;
  a.n_gather = gather_rows ? n_gather : nullptr;
  a.q_pos = q_pos;
  a.o_lat = o_lat;
  a.lse = lse;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  if (!tc_eligible(dims)) {
    const int row = dims->d_c + dims->d_r;
    const size_t smem = sizeof(float) * ((size_t)n_ver * row + dims->d_c + 128 + 4) +
                        sizeof(long long) * 128 + 64;
    if (smem > 48 * 1024) return MLA_ERR_UNSUPPORTED;
    dim3 grid(n_h, B * s_q);
    if (dims->dtype == MLA_BF16)
      decode_simt_kernel<__nv_bfloat16><<<grid, 128, smem, st>>>(a);
    else
      decode_simt_kernel<float><<<grid, 128, smem, st>>>(a);
    (void)es;
    return launch_ok();
  }

  DeviceInfo* dev = nullptr;
  if (device_info(&dev) != MLA_OK) return MLA_ERR_CUDA;
  const int G = dev->num_sms / 2;
  const int n_hb = (n_h + tc::kM - 1) / tc::kM;
  const int n_streams = B * s_q * n_hb;
  const WsLayout wl = ws_layout(n_streams, G, q_pack_bytes(dims, B, s_q, n_ver, n_h),
                                (size_t)B * s_q * n_h);
  if (!workspace || ws_bytes < wl.total) return MLA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return MLA_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  // A head list is resolved on the device: the listed heads' queries are
  // packed densely, and the kernels write each result to its listed head.
  const void* q_src = q_abs;
  if (head_ids) {
    const int rows_out = n_ver * B * s_q * n_h;
    pack_heads_kernel<<<(rows_out + 7) / 8, 256, 0, st>>>(
        rows_out, n_h, dims->H, (int)(tc::kRow * es), head_ids,
        static_cast<const uint8_t*>(q_abs), ws + wl.off_qpack);
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    q_src = ws + wl.off_qpack;
    a.qH = n_h;
  }

  tc::Maps maps;
  const uint64_t cache_rows = (uint64_t)n_pages * kPage;
  const uint64_t q_rows = (uint64_t)n_ver * B * s_q * a.qH;
  if (!make_map_576(&maps.q3, q_src, q_rows, 3, tc::kM, tc::kStagePanels) ||
      !make_map_576(&maps.qr, q_src, q_rows, 2, tc::kM) ||
      !make_map_576(&maps.k3, cache, cache_rows, 3, tc::kT, tc::kStagePanels) ||
      !make_map_576(&maps.kp, cache, cache_rows, 2, tc::kPg) ||
      !make_map_576(&maps.vp, cache, cache_rows, 3, tc::kVRows, 8) ||
      !make_map_576(&maps.g4, cache, cache_rows, 2, 1))
    return MLA_ERR_CUDA;
  for (int i = 0; i < tc::kNumBoxHeights; ++i)
    if (!make_map_576(&maps.row[i], cache, cache_rows, 2, (uint32_t)(32 >> i)))
      return MLA_ERR_CUDA;

  if (!dev->tc_attr_set) {
    if (cudaFuncSetAttribute(tc::decode_tc_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             tc::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(tc::decode_tc_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             tc::kSmemBytes) != cudaSuccess)
      return MLA_ERR_CUDA;
    dev->tc_attr_set = true;
  }
  // page mode and gathered-row mode are separate instantiations
  const bool gather = gather_rows != nullptr;
  tc::PlanHeader* plan = reinterpret_cast<tc::PlanHeader*>(ws + wl.off_plan);
  int* stream_off = reinterpret_cast<int*>(ws + wl.off_streams);
  int* stream_bad = reinterpret_cast<int*>(ws + wl.off_bad);
  int* pair_stream = reinterpret_cast<int*>(ws + wl.off_pairs);
  float* partial = reinterpret_cast<float*>(ws + wl.off_partial);
  float* partial_lse = reinterpret_cast<float*>(ws + wl.off_plse);
  // whole-stream outputs: straight to o_lat, or packed by list position
  float* o_pack = head_ids ? reinterpret_cast<float*>(ws + wl.off_opack) : nullptr;
  float* lse_pack = head_ids ? reinterpret_cast<float*>(ws + wl.off_lpack) : nullptr;
  if (!make_map_out(&maps.o, head_ids ? o_pack : o_lat, (uint64_t)n_h, (uint64_t)B * s_q,
                    (uint64_t)(head_ids ? n_h : dims->H) * tc::kDc, 3) ||
      !make_map_out(&maps.part, partial, (uint64_t)tc::kM * 2 * G, 1, 0, 2))
    return MLA_ERR_CUDA;
  if (gather)
    tc::plan_kernel<true><<<1, tc::kPlanThreads, 0, st>>>(a, n_hb, G, plan, stream_off,
                                                          stream_bad, pair_stream);
  else
    tc::plan_kernel<false><<<1, tc::kPlanThreads, 0, st>>>(a, n_hb, G, plan, stream_off,
                                                           stream_bad, pair_stream);
  if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;

  tc::Params p;
  p.a = a;
  p.n_hb = n_hb;
  p.G = G;
  p.plan = plan;
  p.stream_off = stream_off;
  p.pair_stream = pair_stream;
  p.partial = partial;
  p.partial_lse = partial_lse;
  p.lse_pack = lse_pack;
  p.scale_log2 = dims->scale * tc::kLog2e;
  // The attention and merge kernels are programmatic dependents of the
  // kernel before them: each may start its set-up early and waits on device
  // (griddepcontrol.wait) before it reads its predecessor's results.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * G);
  cfg.blockDim = dim3(tc::kThreads);
  cfg.dynamicSmemBytes = tc::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if ((gather ? cudaLaunchKernelEx(&cfg, tc::decode_tc_kernel<true>, p, maps)
              : cudaLaunchKernelEx(&cfg, tc::decode_tc_kernel<false>, p, maps)) != cudaSuccess)
    return MLA_ERR_CUDA;

  cfg.gridDim = dim3(n_streams, tc::kM / 4);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  if (cudaLaunchKernelEx(&cfg, tc::combine_kernel, a, n_hb, static_cast<const tc::PlanHeader*>(plan),
                         static_cast<const int*>(stream_off), static_cast<const int*>(stream_bad),
                         static_cast<const float*>(partial),
                         static_cast<const float*>(partial_lse),
                         static_cast<const float*>(o_pack),
                         static_cast<const float*>(lse_pack)) != cudaSuccess)
    return MLA_ERR_CUDA;
  return launch_ok();
}

}  // namespace

extern "C" {

mla_status_t mla_decode(const mla_dims_t* dims, int32_t B, int32_t s_q, const void* q_abs,
                        int32_t n_ver, const int32_t* head_ids, int32_t n_h, const void* cache,
                        int64_t n_pages, const int32_t* block_table, int32_t max_pages,
                        const mla_seg_t* segs, int32_t max_segs, const int32_t* gather_rows,
                        const int32_t* n_gather, int32_t max_gather, const int32_t* q_pos,
                        float* o_lat, float* lse, void* workspace, size_t ws_bytes,
                        mla_stream_t stream) {
  return decode_impl(dims, B, s_q, q_abs, n_ver, head_ids, n_h, cache, n_pages, block_table,
                     max_pages, segs, max_segs, gather_rows, n_gather, max_gather, q_pos, o_lat,
                     lse, workspace, ws_bytes, stream, nullptr);
}

mla_status_t mla_decode_qknorm(const mla_dims_t* dims, int32_t B, int32_t s_q, const void* q_abs,
                               int32_t n_ver, const int32_t* head_ids, int32_t n_h,
                               const void* cache, const float* key_inv_rms, int64_t n_pages,
                               const int32_t* block_table, int32_t max_pages,
                               const mla_seg_t* segs, int32_t max_segs, const int32_t* q_pos,
                               float* o_lat, float* lse, void* workspace, size_t ws_bytes,
                               mla_stream_t stream) {
  if (!key_inv_rms) return MLA_ERR_INVALID_ARG;
  return decode_impl(dims, B, s_q, q_abs, n_ver, head_ids, n_h, cache, n_pages, block_table,
                     max_pages, segs, max_segs, nullptr, nullptr, 0, q_pos, o_lat, lse,
                     workspace, ws_bytes, stream, key_inv_rms);
}

}  // extern "C"

namespace {

bool lowbit_ok(const mla_dims_t* dims, int bits_c, int bits_r) {
  return ((bits_c == 4 && bits_r == 4) || (bits_c == 2 && bits_r == 4)) &&
         (dims->d_c * bits_c) % 32 == 0 && (dims->d_r * bits_r) % 32 == 0;
}

template <typename T>
void launch_pack(int bits_c, int n, const mla_dims_t* d, const void* rows, const float* sc,
                 const float* sr, void* out, cudaStream_t st) {
  const unsigned blocks = (unsigned)((n + 7) / 8);
  if (bits_c == 4)
    pack_rows_kernel<T, 4, 4><<<blocks, 256, 0, st>>>(n, d->d_c, d->d_r,
                                                      static_cast<const T*>(rows), sc, sr,
                                                      static_cast<uint8_t*>(out));
  else
    pack_rows_kernel<T, 2, 4><<<blocks, 256, 0, st>>>(n, d->d_c, d->d_r,
                                                      static_cast<const T*>(rows), sc, sr,
                                                      static_cast<uint8_t*>(out));
}

template <typename T>
void launch_lowbit(int bits_c, dim3 grid, size_t smem, const DecodeArgs& a, const float* sc,
                   const float* sr, cudaStream_t st) {
  if (bits_c == 4)
    decode_lowbit_kernel<T, 4, 4><<<grid, 128, smem, st>>>(a, sc, sr);
  else
    decode_lowbit_kernel<T, 2, 4><<<grid, 128, smem, st>>>(a, sc, sr);
}

}  // namespace

extern "C" {

mla_status_t mla_pack_rows(const mla_dims_t* dims, int32_t bits_c, int32_t bits_r, int64_t n_rows,
                           const void* rows, const float* scale_c, const float* scale_r,
                           void* packed, mla_stream_t stream) {
  if (!dims_ok(dims) || n_rows < 0) return MLA_ERR_INVALID_ARG;
  if (!lowbit_ok(dims, bits_c, bits_r)) return MLA_ERR_UNSUPPORTED;
  if (n_rows == 0) return MLA_OK;
  if (!rows || !scale_c || !scale_r || !packed || !aligned(packed, 4)) return MLA_ERR_INVALID_ARG;
  if (n_rows > (int64_t)INT32_MAX - 8) return MLA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16)
    launch_pack<__nv_bfloat16>(bits_c, (int)n_rows, dims, rows, scale_c, scale_r, packed, st);
  else
    launch_pack<float>(bits_c, (int)n_rows, dims, rows, scale_c, scale_r, packed, st);
  return launch_ok();
}

mla_status_t mla_decode_lowbit(const mla_dims_t* dims, int32_t bits_c, int32_t bits_r, int32_t B,
                               int32_t s_q, const void* q_abs, int32_t n_ver,
                               const int32_t* head_ids, int32_t n_h, const void* cache,
                               const float* scale_c, const float* scale_r, int64_t n_pages,
                               const int32_t* block_table, int32_t max_pages,
                               const mla_seg_t* segs, int32_t max_segs,
                               const int32_t* gather_rows, const int32_t* n_gather,
                               int32_t max_gather, const int32_t* q_pos, float* o_lat, float* lse,
                               mla_stream_t stream) {
  if (!dims_ok(dims) || B < 0 || s_q < 1 || n_ver < 1 || n_h < 1 || n_h > dims->H ||
      n_pages < 1 || max_pages < 1 || max_segs < 1)
    return MLA_ERR_INVALID_ARG;
  if (!lowbit_ok(dims, bits_c, bits_r)) return MLA_ERR_UNSUPPORTED;
  if (dims->page_size != kPage || n_ver > kMaxVersions) return MLA_ERR_UNSUPPORTED;
  if (gather_rows && (!n_gather || max_gather < 1)) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!q_abs || !cache || !scale_c || !scale_r || !block_table || !segs || !q_pos || !o_lat ||
      !lse || !aligned(cache, 4))
    return MLA_ERR_INVALID_ARG;
  if (n_pages * kPage + 2 * kPage > INT32_MAX || (long long)max_pages * kPage > INT32_MAX ||
      (long long)n_ver * B * s_q * dims->H > INT32_MAX)
    return MLA_ERR_UNSUPPORTED;
  DecodeArgs a;
  a.B = B;
  a.s_q = s_q;
  a.n_q = B * s_q;
  a.H = dims->H;
  a.qH = dims->H;
  a.head_ids = head_ids;
  a.key_inv = nullptr;
  a.n_h = n_h;
  a.d_c = dims->d_c;
  a.d_r = dims->d_r;
  a.n_ver = n_ver;
  a.max_pages = max_pages;
  a.max_segs = max_segs;
  a.max_gather = gather_rows ? max_gather : 0;
  a.n_pages = n_pages;
  a.scale = dims->scale;
  a.q_abs = q_abs;
  a.cache = cache;
  a.block_table = block_table;
  a.segs = segs;
  a.gather_rows = gather_rows;
  a.n_gather = gather_rows ? n_gather : nullptr;
  a.q_pos = q_pos;
  a.o_lat = o_lat;
  a.lse = lse;
  const int row = dims->d_c + dims->d_r;
  const size_t smem = sizeof(float) * ((size_t)n_ver * row + dims->d_c + 128 + 4) +
                      sizeof(long long) * 128 + 64;
  if (smem > 48 * 1024) return MLA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(n_h, B * s_q);
  if (dims->dtype == MLA_BF16)
    launch_lowbit<__nv_bfloat16>(bits_c, grid, smem, a, scale_c, scale_r, st);
  else
    launch_lowbit<float>(bits_c, grid, smem, a, scale_c, scale_r, st);
  return launch_ok();
}

mla_status_t mla_debug_wait_probe(int64_t limit_ns, int32_t* waited_us, mla_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 100000000 || !waited_us || !aligned(waited_us, 4))
    return MLA_ERR_INVALID_ARG;
  tc::wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (uint64_t)limit_ns, waited_us);
  return launch_ok();
}

mla_status_t mla_merge_lse(int32_t n_q, int32_t H, const int32_t* head_ids, int32_t n_h,
                           int32_t d, const float* o_a, const float* lse_a, const float* o_b,
                           const float* lse_b, float* o, float* lse, mla_stream_t stream) {
  if (n_q < 0 || H < 1 || n_h < 1 || n_h > H || d < 1) return MLA_ERR_INVALID_ARG;
  if (n_q == 0) return MLA_OK;
  if (!o_a || !lse_a || !o_b || !lse_b || !o || !lse) return MLA_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev) != MLA_OK) return MLA_ERR_CUDA;
  const long long rows = (long long)n_q * n_h;
  const long long blocks = (rows + 7) / 8;
  if (blocks > INT32_MAX) return MLA_ERR_INVALID_ARG;
  merge_lse_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      n_q, H, head_ids, n_h, d, o_a, lse_a, o_b, lse_b, o, lse);
  return launch_ok();
}

mla_status_t mla_out_proj(const mla_dims_t* dims, int32_t n_q, const float* o_lat,
                          const void* w_uv, const void* w_o, float* v, float* out,
                          mla_stream_t stream) {
  if (!dims_ok(dims) || n_q < 0) return MLA_ERR_INVALID_ARG;
  if (n_q == 0) return MLA_OK;
  if (!o_lat || !w_uv || !v || (w_o && (!out || dims->d_model < 1))) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int H = dims->H, d_c = dims->d_c, d_v = dims->d_v;
  if (dims->dtype == MLA_BF16 && d_v % wg::kMT == 0 && d_c % wg::kKP == 0 &&
      (!w_o || dims->d_model % wg::kMT == 0) && aligned(o_lat, 16) && aligned(v, 16)) {
    wg::Params p{};
    p.mode = wg::kValue;
    p.n = n_q;
    p.n_total = n_q;
    p.H = H;
    p.d_c = d_c;
    p.d_r = dims->d_r;
    p.d_n = dims->d_n;
    p.d_v = d_v;
    p.d_model = dims->d_model;
    p.x = o_lat;
    p.x_row_stride = (long long)H * d_c;
    p.x_head_stride = d_c;
    p.out = v;
    if (w_o) {   // the value launch zeroes `out` for the split-K output product
      p.zero = out;
      p.zero_n = (long long)n_q * dims->d_model;
    }
    mla_status_t rc = launch_wgemm(p, w_uv, (uint64_t)H * d_v, d_c, H, d_v / wg::kMT, d_c, false,
                                   nullptr, 0, st);
    if (rc != MLA_OK || !w_o) return rc;
    p.mode = wg::kOutput;
    p.n = n_q;
    p.x = v;
    p.x_row_stride = (long long)H * d_v;
    p.x_head_stride = 0;
    p.out = out;
    p.zero = nullptr;
    p.zero_n = 0;
    return launch_wgemm(p, w_o, dims->d_model, (uint64_t)H * d_v, 1, dims->d_model / wg::kMT,
                        H * d_v, true, nullptr, 0, st);
  }
  dim3 g1(H, (d_v + 7) / 8);
  if (dims->dtype == MLA_BF16)
    vproj_simt_kernel<__nv_bfloat16><<<g1, 256, 0, st>>>(
        n_q, H, d_c, d_v, o_lat, static_cast<const __nv_bfloat16*>(w_uv), v);
  else
    vproj_simt_kernel<float><<<g1, 256, 0, st>>>(n_q, H, d_c, d_v, o_lat,
                                                 static_cast<const float*>(w_uv), v);
  if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
  if (!w_o) return MLA_OK;
  const int K = H * d_v;
  dim3 g2((dims->d_model + 7) / 8);
  if (dims->dtype == MLA_BF16)
    oproj_simt_kernel<__nv_bfloat16><<<g2, 256, 0, st>>>(
        n_q, K, dims->d_model, v, static_cast<const __nv_bfloat16*>(w_o), out);
  else
    oproj_simt_kernel<float><<<g2, 256, 0, st>>>(n_q, K, dims->d_model, v,
                                                 static_cast<const float*>(w_o), out);
  return launch_ok();
}

}  // extern "C"
