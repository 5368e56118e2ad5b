// wgemm.cuh -- weight-streaming skinny GEMMs on sm_100a tensor cores.
//
// The three weight products of one decode step all read a large bf16 weight
// once and apply it to a handful of query rows:
//   absorb  q_abs[v, q, h, c] = sum_n W_UK[h][n][c] q_nope[q, h, n]
//           (Day 27 tutorial, "Move the Key Projection Into the Query"),
//           with the rotary part R(q_pos - delta_v) q_rope written alongside
//           (RedKnot-MLA abstract: query-side RoPE relocation);
//   value   v[q, h, d] = sum_c W_UV[h][d][c] o_lat[q, h, c]
//           ("Move the Value Expansion After the Weighted Sum");
//   output  out[q, m] = sum_j W_O[m][j] v[q, j]  (the shared projection).
// Each is computed transposed, D[m, n] = sum_k W[m, k] X[n, k], so the weight
// rows fill the 128-row MMA tile and the query rows are the (padded) N
// dimension.  One CTA owns 128 weight rows and a K range: its X slice is
// converted to bf16 into shared memory once, the weight streams through a
// 4-stage TMA ring, one thread issues tcgen05.mma (fp32 accumulator in TMEM),
// and the epilogue writes D transposed.  The output product splits K over
// CTAs and adds partial sums with fp32 atomics (the value kernel zeroes
// `out` first).
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace wg {

constexpr int kMT = 128;                 // weight rows per CTA
constexpr int kKP = 64;                  // K per panel (128 B of bf16)
constexpr int kWStage = kMT * kKP * 2;   // 16 KB
constexpr int kStages = 4;
constexpr int kXBytesMax = 32 * 1024;    // bf16 X slice (N_pad rows x K range)
constexpr int kSmemBytes = kStages * kWStage + kXBytesMax + 256 + 1024;
constexpr int kThreads = 128;

enum Mode : int { kAbsorb = 0, kValue = 1, kOutput = 2 };

struct Params {
  int mode;
  int n;          // query rows of this launch (q0 .. q0 + n - 1)
  int q0;         // first query row
  int n_total;    // query rows of the whole call (layout of q_abs)
  int n_pad;      // n padded to a multiple of 16 (<= 128)
  int K;          // reduction length of one product
  int k_chunk;    // K range of one CTA (multiple of 64)
  int H, d_c, d_r, d_n, d_v, d_model;
  const void* x;  // activations: bf16 (absorb) or fp32
  long long x_row_stride;   // elements between query rows of X
  long long x_head_stride;  // elements between heads of X
  void* out;
  // absorb only
  int n_ver;
  int delta[kMaxVersions];
  double rope_base;
  const void* q_rope;
  const int32_t* q_pos;
};

// Weight tile: absorb reads W_UK[h] ([d_n rows, d_c cols], the M dimension
// contiguous) as two 64-column boxes of 64 rows; the others read 128 weight
// rows x 64 K as one box.  Both land in the canonical 128-byte-swizzled
// layout the MMA descriptors below describe.
__global__ void __launch_bounds__(kThreads) wgemm_kernel(const __grid_constant__ Params p,
                                                         const __grid_constant__ CUtensorMap tw) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = smem;
  uint8_t* sX = smem + kStages * kWStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(sX + kXBytesMax);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kMT;           // first weight row (within a head)
  const int h = blockIdx.y;                  // head (absorb / value), 0 for output
  const int k0 = blockIdx.z * p.k_chunk;
  const int kc = min(p.k_chunk, p.K - k0);
  const int n_panels = kc / kKP;
  const uint32_t ncols = p.n_pad <= 32 ? 32 : (p.n_pad <= 64 ? 64 : (p.n_pad <= 128 ? 128 : 256));

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // weight ring: thread 0 starts the first loads before X is staged
  auto load_w = [&](int i) {
    const int s = i % kStages;
    uint8_t* dst = sW + s * kWStage;
    mbar_arrive_expect_tx(&full[s], kWStage);
    const int kk = k0 + i * kKP;
    if (p.mode == kAbsorb) {
      // rows kk..kk+63 of W_UK[h] (global row h*d_n + kk), columns m0..m0+127
      tma_load_2d(dst, &tw, &full[s], m0, h * p.d_n + kk);
      tma_load_2d(dst + kWStage / 2, &tw, &full[s], m0 + 64, h * p.d_n + kk);
    } else {
      const int row = (p.mode == kValue ? h * p.d_v : 0) + m0;
      tma_load_2d(dst, &tw, &full[s], kk, row);
    }
  };
  bool ok = true;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tw);
    for (int i = 0; i < kStages && i < n_panels; ++i) load_w(i);
  }

  // X slice -> bf16, K-major, 128-byte swizzle: panel j holds K [64 j, 64 j + 64)
  // of all n_pad rows (rows >= n are zero)
  const int chunks = p.n_pad * n_panels * 8;            // 16-byte chunks
  for (int e = threadIdx.x; e < chunks; e += kThreads) {
    const int c = e & 7;
    const int r = (e >> 3) % p.n_pad;
    const int j = (e >> 3) / p.n_pad;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < p.n) {
      const long long base = (long long)(p.q0 + r) * p.x_row_stride + (long long)h * p.x_head_stride +
                             k0 + j * kKP + c * 8;
      if (p.mode == kAbsorb) {
        val = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.x) + base);
      } else {
        const float* xf = static_cast<const float*>(p.x) + base;
        const float4 a = *reinterpret_cast<const float4*>(xf);
        const float4 b = *reinterpret_cast<const float4*>(xf + 4);
        __nv_bfloat162 t0 = __floats2bfloat162_rn(a.x, a.y), t1 = __floats2bfloat162_rn(a.z, a.w);
        __nv_bfloat162 t2 = __floats2bfloat162_rn(b.x, b.y), t3 = __floats2bfloat162_rn(b.z, b.w);
        val = make_uint4(*reinterpret_cast<uint32_t*>(&t0), *reinterpret_cast<uint32_t*>(&t1),
                         *reinterpret_cast<uint32_t*>(&t2), *reinterpret_cast<uint32_t*>(&t3));
      }
    }
    *reinterpret_cast<uint4*>(sX + j * p.n_pad * 128 + r * 128 + ((c ^ (r & 7)) << 4)) = val;
  }
  fence_proxy_async();
  __syncthreads();

  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_bf16_f32(kMT, p.n_pad, p.mode == kAbsorb, false);
    for (int i = 0; i < n_panels && ok; ++i) {
      const int s = i % kStages;
      if (!mbar_wait(&full[s], (i / kStages) & 1)) { set_status(MLA_ERR_TIMEOUT); ok = false; break; }
      tc_fence_after();
      const uint32_t wa = smem_u32(sW + s * kWStage);
      const uint32_t xb = smem_u32(sX + i * p.n_pad * 128);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        // absorb: W tile is M-major (two 64-column blocks 8 KB apart, 16 K
        // rows per step); otherwise K-major (16 K = 32 bytes per step)
        const uint64_t ad = (p.mode == kAbsorb)
                                ? smem_desc_sw128(wa + ks * 2048, kWStage / 2, 1024)
                                : smem_desc_sw128(wa + ks * 32, 16, 1024);
        const uint64_t bd = smem_desc_sw128(xb + ks * 32, 16, 1024);
        mma_bf16_ss(tmem, ad, bd, idesc, (i | ks) ? 1u : 0u);
      }
      mma_commit(&empty[s]);
      if (i + kStages < n_panels) {
        if (!mbar_wait(&empty[s], (i / kStages) & 1)) { set_status(MLA_ERR_TIMEOUT); ok = false; break; }
        load_w(i + kStages);
      }
    }
    mma_commit(done);
  }
  __syncwarp();
  const bool done_ok = __all_sync(0xffffffffu, mbar_wait(done, 0));
  if (!done_ok && lane == 0) set_status(MLA_ERR_TIMEOUT);
  tc_fence_after();

  // epilogue: lane = weight row m0 + 32 warp + lane, columns = query rows
  const int m = m0 + warp * 32 + lane;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  for (int c0 = 0; c0 < p.n_pad; c0 += 32) {
    float d[32];
    tmem_ld32(trow + c0, d);
    tmem_wait_ld();
    if (!done_ok) continue;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (c0 + i >= p.n) continue;
      const int q = p.q0 + c0 + i;
      if (p.mode == kOutput) {
        atomicAdd(static_cast<float*>(p.out) + (size_t)q * p.d_model + m, d[i]);
      } else if (p.mode == kValue) {
        static_cast<float*>(p.out)[((size_t)q * p.H + h) * p.d_v + m] = d[i];
      } else {
        const int row = p.d_c + p.d_r;
        for (int v = 0; v < p.n_ver; ++v)
          static_cast<__nv_bfloat16*>(p.out)[(((size_t)v * p.n_total + q) * p.H + h) * row + m] =
              __float2bfloat16_rn(d[i]);
      }
    }
  }

  // absorb: the rotary part of this head, once (by the CTA with m0 == 0):
  // pair i rotated by (q_pos - delta_v) * base^(-2i/d_r), angles in double
  if (p.mode == kAbsorb && blockIdx.x == 0) {
    const int half = p.d_r / 2, row = p.d_c + p.d_r;
    const __nv_bfloat16* qr = static_cast<const __nv_bfloat16*>(p.q_rope);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    for (int t = threadIdx.x; t < p.n * p.n_ver * half; t += kThreads) {
      const int i = t % half, v = (t / half) % p.n_ver, q = p.q0 + t / (half * p.n_ver);
      const double theta = pow(p.rope_base, -2.0 * i / p.d_r);
      double sn, cs;
      sincos((double)(p.q_pos[q] - p.delta[v]) * theta, &sn, &cs);
      const size_t src = ((size_t)q * p.H + h) * p.d_r + 2 * i;
      const double x0 = __bfloat162float(qr[src]), x1 = __bfloat162float(qr[src + 1]);
      const size_t dst = (((size_t)v * p.n_total + q) * p.H + h) * row + p.d_c + 2 * i;
      out[dst] = __float2bfloat16_rn((float)(x0 * cs - x1 * sn));
      out[dst + 1] = __float2bfloat16_rn((float)(x0 * sn + x1 * cs));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// out[q, :] = 0 before the split-K output product adds into it.
__global__ void zero_kernel(float* out, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = 0.f;
}

}  // namespace wg
}  // namespace mla
