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
// Each is computed transposed, D[m, n] = sum_k W[m, k] X[n, k], so 128 weight
// rows fill the MMA's M and the query rows are its (padded) N.
//
// The weight is cut into units of 128 rows x 64P K (P = 1, 2 or 4 panels of
// 64 K, one 3-D TMA box of 16P KB whose rows are 128P contiguous bytes -- the
// TMA engine moves long row runs much faster than 128-byte ones); a group
// (head) x m-tile x k-stage walk orders them with K fastest.  Each CTA
// is persistent on one SM and takes a contiguous run of units -- whole
// m-tiles for absorb/value (their outputs are written once), any run for the
// output product (partial sums are added with fp32 atomics into `out`, which
// the value launch zeroes).  Roles per CTA (320 threads):
//   warp 0     TMA producer: weight stages (and the bf16 query panel of the
//              absorb product) into a ring of up to 16 stages;
//   warp 1     MMA issuer (one thread): tcgen05.mma into one of two TMEM
//              accumulators, so the epilogue of one m-tile overlaps the next;
//   warps 2-5  epilogue: TMEM -> registers -> global (stores or atomics);
//   warps 6-9  convert the fp32 activation panel of each stage to bf16 in
//              the 128-byte-swizzled K-major layout, two warps per stage
//              (value/output), or apply the rotary relocation (absorb).
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace wg {

constexpr int kMT = 128;                 // weight rows per unit (MMA M)
constexpr int kKP = 64;                  // K per panel (128 bytes of bf16)
constexpr int kWPanel = kMT * kKP * 2;   // 16 KB: 128 rows x one panel
constexpr int kMaxStages = 16;
constexpr int kSmemMax = 232448;         // dynamic shared memory per CTA
constexpr int kSmemFixed = 512 + 1024;   // barriers + alignment slack
constexpr int kThreads = 320;

enum Mode : int { kAbsorb = 0, kValue = 1, kOutput = 2 };

struct Params {
  int mode;
  int n;          // query rows of this launch (q0 .. q0 + n - 1), <= 128
  int q0;         // first query row
  int n_total;    // query rows of the whole call (layout of q_abs)
  int n_pad;      // n padded to a multiple of 16
  int stages;     // ring depth
  int P;          // 64-K panels per unit
  int groups, m_tiles, k_stages;   // units = groups x m_tiles x k_stages
  int chunk;      // units per CTA
  int H, d_c, d_r, d_n, d_v, d_model;
  const void* x;  // activations: fp32 (value/output); absorb reads them by TMA
  long long x_row_stride;   // elements between query rows of X
  long long x_head_stride;  // elements between groups of X
  void* out;
  float* zero;    // value: `out` of the following output product, zeroed here
  long long zero_n;
  // absorb only
  int n_ver;
  int delta[kMaxVersions];
  double rope_base;
  const void* q_rope;
  const int32_t* q_pos;
};

struct Unit {
  int g, mt, ks;
};
__device__ __forceinline__ Unit unit_of(const Params& p, int u) {
  Unit r;
  r.ks = u % p.k_stages;
  const int t = u / p.k_stages;
  r.mt = t % p.m_tiles;
  r.g = t / p.m_tiles;
  return r;
}

__device__ __forceinline__ uint32_t acc_cols(int n_pad) {
  return n_pad <= 32 ? 32u : (n_pad <= 64 ? 64u : 128u);
}

// Weight unit in the canonical 128-byte-swizzled layouts.  Absorb reads
// W_UK[h] ([d_n, d_c], M contiguous) as 64P K rows x two 64-column M panels
// (M-major operand, panels 64P x 128 bytes apart); the others read 128 rows x
// P K panels (K-major, panels 16 KB apart).  The activation panel of a stage
// holds P panels of n_pad rows x 128 bytes.
__global__ void __launch_bounds__(kThreads, 1)
wgemm_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tw,
             const __grid_constant__ CUtensorMap tx) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  const int x_panel = p.n_pad * 128;
  const int x_stage = p.P * x_panel;
  const int w_stage = p.P * kWPanel;
  uint8_t* sW = smem;
  uint8_t* sX = smem + S * w_stage;
  uint64_t* full = reinterpret_cast<uint64_t*>(sX + S * x_stage);
  uint64_t* empty = full + kMaxStages;
  uint64_t* acc_full = empty + kMaxStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool absorb = p.mode == kAbsorb;
  const uint32_t ncols = acc_cols(p.n_pad);
  const int U = p.groups * p.m_tiles * p.k_stages;
  const int u0 = min(U, (int)blockIdx.x * p.chunk);
  const int u1 = min(U, u0 + p.chunk);

  // A launch that follows may start streaming its weights now; whatever it
  // reads of this launch's results waits for completion (griddepcontrol.wait)
  asm volatile("griddepcontrol.launch_dependents;");
  if (p.zero) {
    for (long long i = (long long)blockIdx.x * kThreads + threadIdx.x; i < p.zero_n;
         i += (long long)gridDim.x * kThreads)
      p.zero[i] = 0.f;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], absorb ? 1 : 3);   // TMA bytes (+ the two converter warps)
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 2 * ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      prefetch_tmap(&tw);
      if (absorb) prefetch_tmap(&tx);
      const uint32_t bytes = w_stage + (absorb ? x_stage : 0);
      for (int u = u0, i = 0; u < u1; ++u, ++i) {
        const int slot = i % S;
        if (!mbar_wait(&empty[slot], ((i / S) & 1) ^ 1)) { set_status(MLA_ERR_TIMEOUT); break; }
        const Unit w = unit_of(p, u);
        uint8_t* dst = sW + slot * w_stage;
        mbar_arrive_expect_tx(&full[slot], bytes);
        if (absorb) {
          // K rows 64P ks .. of W_UK[g] (global row g d_n + 64P ks), M panels
          // 2 mt and 2 mt + 1; the query panels: q_nope[q0.., g, same K]
          const int krow = w.g * p.d_n + w.ks * kKP * p.P;
          tma_load_3d(dst, &tw, &full[slot], 0, krow, 2 * w.mt);
          tma_load_3d(sX + slot * x_stage, &tx, &full[slot], 0, p.q0, krow / kKP);
        } else {
          const int row = (p.mode == kValue ? w.g * p.d_v : 0) + w.mt * kMT;
          tma_load_3d(dst, &tw, &full[slot], 0, row, w.ks * p.P);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kMT, p.n_pad, absorb, false);
      int seg = 0;
      for (int u = u0, i = 0; u < u1; ++u, ++i) {
        const int ks = u % p.k_stages;
        const bool first = ks == 0 || u == u0;
        const bool last = ks == p.k_stages - 1 || u == u1 - 1;
        const int ab = seg & 1;
        if (first && !mbar_wait(&acc_empty[ab], ((seg >> 1) & 1) ^ 1)) {
          set_status(MLA_ERR_TIMEOUT);
          break;
        }
        const int slot = i % S;
        if (!mbar_wait(&full[slot], (i / S) & 1)) { set_status(MLA_ERR_TIMEOUT); break; }
        tc_fence_after();
        const uint32_t wa = smem_u32(sW + slot * w_stage);
        const uint32_t xb = smem_u32(sX + slot * x_stage);
        for (int k = 0; k < 4 * p.P; ++k) {
          // absorb: W is M-major (16 K rows = 2 KB per step, the two M panels
          // 64P x 128 bytes apart); otherwise K-major (16 K = 32 bytes per
          // step inside a panel, panels 16 KB apart)
          const uint64_t ad =
              absorb ? smem_desc_sw128(wa + k * 2048, p.P * kKP * 128, 1024)
                     : smem_desc_sw128(wa + (k >> 2) * kWPanel + (k & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(xb + (k >> 2) * x_panel + (k & 3) * 32, 16, 1024);
          mma_bf16_ss(tmem + ab * ncols, ad, bd, idesc, (first && k == 0) ? 0u : 1u);
        }
        mma_commit(&empty[slot]);
        if (last) {
          mma_commit(&acc_full[ab]);
          ++seg;
        }
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    asm volatile("griddepcontrol.wait;" ::: "memory");   // `out` was zeroed by the value launch
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    int seg = 0;
    for (int u = u0; u < u1; ++u) {
      const int ks = u % p.k_stages;
      if (!(ks == p.k_stages - 1 || u == u1 - 1)) continue;
      const Unit w = unit_of(p, u);
      const int ab = seg & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[ab], (seg >> 1) & 1))) {
        if (lane == 0) set_status(MLA_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int m = w.mt * kMT + quad * 32 + lane;     // weight row of this lane
#pragma unroll 1
      for (int c0 = 0; c0 < p.n_pad; c0 += 16) {
        float d[16];
        tmem_ld16_sync(trow + ab * ncols + c0, d);
        const int nq = min(16, p.n - c0);
        if (p.mode == kOutput) {
          float* o = static_cast<float*>(p.out) + (size_t)(p.q0 + c0) * p.d_model + m;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (i < nq) atomicAdd(o + (size_t)i * p.d_model, d[i]);
        } else if (p.mode == kValue) {
          float* o = static_cast<float*>(p.out) + ((size_t)(p.q0 + c0) * p.H + w.g) * p.d_v + m;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (i < nq) o[(size_t)i * p.H * p.d_v] = d[i];
        } else {
          const int row = p.d_c + p.d_r;
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out);
          for (int v = 0; v < p.n_ver; ++v) {
            __nv_bfloat16* ov = o + (((size_t)v * p.n_total + p.q0 + c0) * p.H + w.g) * row + m;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (i < nq) ov[(size_t)i * p.H * row] = __float2bfloat16_rn(d[i]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      ++seg;
    }
  } else if (!absorb) {
    // ------------------------------------------------------------ X panels
    // Stage i is converted by the warp pair 2 (i mod 2), 2 (i mod 2) + 1 of
    // warps 6-9: rows q0 .. q0 + n_pad - 1 (zero past n) x K [64P ks, +64P)
    // of group g, fp32 -> bf16; in panel j, 16-byte chunk c of row r is
    // stored at chunk c ^ (r mod 8) of the row.  Each thread issues all its
    // loads of a stage before converting (one L2 round trip per stage), and
    // the two pairs work on alternate stages.  Two pairs <= S stages: a pair
    // that finished stage i - 2 has seen the slot of stage i freed at least
    // up to its previous use but one, so its parity wait on that slot is
    // never two phases behind.
    const int cw = warp - 6, pair = cw >> 1;
    const int t = (cw & 1) * 32 + lane;
    const float* xf = static_cast<const float*>(p.x);
    // the activations are the previous launch's results (the output product
    // is launched as its programmatic dependent; a no-op otherwise)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int per_panel = p.n_pad * 8;              // 16-byte chunks per panel
    const int total = per_panel * p.P;
    for (int u = u0, i = 0; u < u1; ++u, ++i) {
      if ((i & 1) != pair) continue;
      const int slot = i % S;
      if (!__all_sync(0xffffffffu, mbar_wait(&empty[slot], ((i / S) & 1) ^ 1))) {
        if (lane == 0) set_status(MLA_ERR_TIMEOUT);
        break;
      }
      const Unit w = unit_of(p, u);
      const float* src = xf + (long long)p.q0 * p.x_row_stride + (long long)w.g * p.x_head_stride +
                         w.ks * kKP * p.P;
      uint8_t* dst = sX + slot * x_stage;
      for (int e0 = t; e0 < total; e0 += 8 * 64) {
        float4 lo[8], hi[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int e = e0 + 64 * j, pn = e / per_panel, r = (e % per_panel) >> 3, c = e & 7;
          lo[j] = hi[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (e < total && r < p.n) {
            const float* s = src + (long long)r * p.x_row_stride + pn * kKP + c * 8;
            lo[j] = *reinterpret_cast<const float4*>(s);
            hi[j] = *reinterpret_cast<const float4*>(s + 4);
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int e = e0 + 64 * j, pn = e / per_panel, r = (e % per_panel) >> 3, c = e & 7;
          if (e >= total) continue;
          const __nv_bfloat162 t0 = __floats2bfloat162_rn(lo[j].x, lo[j].y);
          const __nv_bfloat162 t1 = __floats2bfloat162_rn(lo[j].z, lo[j].w);
          const __nv_bfloat162 t2 = __floats2bfloat162_rn(hi[j].x, hi[j].y);
          const __nv_bfloat162 t3 = __floats2bfloat162_rn(hi[j].z, hi[j].w);
          *reinterpret_cast<uint4*>(dst + pn * x_panel + r * 128 + ((c ^ (r & 7)) << 4)) =
              make_uint4(*reinterpret_cast<const uint32_t*>(&t0),
                         *reinterpret_cast<const uint32_t*>(&t1),
                         *reinterpret_cast<const uint32_t*>(&t2),
                         *reinterpret_cast<const uint32_t*>(&t3));
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[slot]);
    }
  } else {
    // ------------------------------------------------------------ rotary part
    // Rows (q, h) of this launch are shared out over the CTAs; a warp takes
    // every fourth row of its CTA's share, a lane the rotary pairs i = lane +
    // 32 k, rotated by (q_pos - delta_v) * base^(-2i/d_r) with the angle in
    // double.  The rows of a CTA share few query tokens, so sine and cosine
    // are recomputed only when the token changes.
    const int cw = warp - 6;
    const int rows = p.n * p.H;
    const int per = (rows + gridDim.x - 1) / gridDim.x;
    const int r0 = blockIdx.x * per, r1 = min(rows, r0 + per);
    const int half = p.d_r / 2, row = p.d_c + p.d_r;
    const __nv_bfloat16* qr = static_cast<const __nv_bfloat16*>(p.q_rope);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    for (int i = lane; i < half; i += 32) {
      const double theta = pow(p.rope_base, -2.0 * i / p.d_r);
      for (int v = 0; v < p.n_ver; ++v) {
        int q_prev = -1;
        double sn = 0.0, cs = 1.0;
        for (int r = r0 + cw; r < r1; r += 4) {
          const int q = p.q0 + r / p.H, h = r % p.H;
          if (q != q_prev) {
            sincos((double)(p.q_pos[q] - p.delta[v]) * theta, &sn, &cs);
            q_prev = q;
          }
          const size_t src = ((size_t)q * p.H + h) * p.d_r + 2 * i;
          const double x0 = __bfloat162float(qr[src]), x1 = __bfloat162float(qr[src + 1]);
          const size_t dst = (((size_t)v * p.n_total + q) * p.H + h) * row + p.d_c + 2 * i;
          __nv_bfloat162 y;
          y.x = __float2bfloat16_rn((float)(x0 * cs - x1 * sn));
          y.y = __float2bfloat16_rn((float)(x0 * sn + x1 * cs));
          *reinterpret_cast<__nv_bfloat162*>(out + dst) = y;
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * ncols);
  }
}

}  // namespace wg
}  // namespace mla
