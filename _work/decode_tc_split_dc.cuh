// decode_tc.cuh -- absorbed MLA decode on sm_100a tensor cores.
//
// What it computes (Day 27 tutorial "Multi-Head Latent Attention", sections
// "Move the Key Projection Into the Query", "Position Rotations Complicate
// the Absorption", "Move the Value Expansion After the Weighted Sum"): for a
// tile of up to 128 query rows (one query token x up to 128 heads) and every
// cached row t of the sequence,
//     S[m, t] = scale * (q_abs[m, :512] . c_t + q_abs[m, 512:] . k_rope_t)
//     P = online-softmax(S masked by key_pos(t) <= q_pos),  O[m, :] = sum_t P[m,t] c_t
// with the latent row [c_t | k_rope_t] (576 bf16) read once from HBM.
//
// Decomposition.  A 128-row fp32 accumulator over d_c = 512 fills all 512
// TMEM columns of an SM, so the work of one tile is split across a cluster of
// two CTAs along d_c: CTA 0 owns latent columns [0, 256) plus the 64 rotary
// columns, CTA 1 owns latent columns [256, 512).  Each CTA streams only its
// columns of every 64-row page (TMA, 128-byte swizzle), so every cache byte
// crosses HBM once.  Each CTA computes a partial score over its columns
// (tcgen05.mma, M=128 N=64, fp32 in TMEM), the two partials are exchanged
// through distributed shared memory and added in the same order on both
// sides, both CTAs run the identical online softmax, and each accumulates its
// half of O = P . c (tcgen05.mma, M=128 N=256, fp32 in TMEM columns 0-255).
//
// Roles per CTA (192 threads): warp 0 loads (TMA), warp 1 issues tcgen05.mma,
// warps 2-5 hold one query row per thread for softmax and the epilogue.
// Long sequences are split over CTA pairs; each pair gets a contiguous run of
// (sequence, row tile, page) units and writes either the final output or a
// normalised partial (o, lse) that the combine kernel merges.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace tc {

constexpr int kDc = 512, kDr = 64, kRow = kDc + kDr;
constexpr int kM = 128;                       // query rows per tile
constexpr int kN = 64;                        // cache rows per tile (one page)
constexpr int kPanelKV = kN * 128;            // one 64-column panel of a page: 8 KB
constexpr int kPanelQ = kM * 128;             // one 64-column panel of Q: 16 KB
constexpr int kMaxPanels = 5;                 // CTA 0: 4 latent + 1 rotary panel
constexpr int kStages = 2;
constexpr int kStageBytes = kMaxPanels * kPanelKV;   // 40 KB
constexpr int kQBytes = kMaxPanels * kPanelQ;        // 80 KB
constexpr int kPBytes = kM * 128;                    // 16 KB (128 x 64 bf16)
constexpr int kXBytes = kM * kN * 4;                 // 32 KB partial scores
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;
constexpr int kOffP = kOffKV + kStages * kStageBytes;
constexpr int kOffX = kOffP + 2 * kPBytes;
constexpr int kOffBar = kOffX + kXBytes;
constexpr int kBarBytes = 256;
constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;   // + alignment slack
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kColO = 0, kColS = 256;
constexpr int kMinChunk = 4;
constexpr int kNumBoxHeights = 7;             // 64, 32, 16, 8, 4, 2, 1 rows
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;     // log2 units: lazy rescale margin

// Partial slot: 128 rows x 512 fp32 + 128 lse.
constexpr size_t kSlotFloats = (size_t)kM * kDc + kM;

struct PlanHeader {
  int U;          // total (sequence, row tile, page) units
  int C;          // units per worker
  int G;          // workers (CTA pairs)
  int n_streams;  // (sequence, row tile) streams
};

struct Params {
  DecodeArgs a;
  int n_hb;                 // head blocks of <= 128 heads
  int G;
  const PlanHeader* plan;
  const int* stream_off;    // [n_streams + 1]
  float* partial;           // [2G][kSlotFloats]
  float scale_log2;
};

// ----------------------------------------------------------------- tiles
struct Tile {
  int n_valid;        // rows of the tile that exist (0..64)
  int ver;            // query version of the tile (gather: of its first row)
  long long phys0;    // physical row of row 0 (page mode)
  int kpos0;          // request position of row 0 (page mode)
  bool gather;
};

// Describe tile k of sequence b.  Page mode: the k-th page of the
// concatenated segments (segments start on page boundaries, so a page holds
// rows of one segment).  Gather mode: gathered rows [64k, 64k + 64).
// Deterministic: every role computes the same description.
__device__ __forceinline__ Tile describe(const DecodeArgs& a, int b, int k) {
  Tile t;
  t.gather = a.gather_rows != nullptr;
  t.n_valid = 0;
  t.ver = 0;
  t.phys0 = 0;
  t.kpos0 = 0;
  const mla_seg_t* sg = a.segs + (size_t)b * a.max_segs;
  if (t.gather) {
    const int ng = a.n_gather[b];
    t.n_valid = min(kN, ng - k * kN);
    const int r0 = a.gather_rows[(size_t)b * a.max_gather + k * kN];
    for (int s = 0; s < a.max_segs; ++s)
      if (r0 >= sg[s].row_begin && r0 < sg[s].row_end) { t.ver = sg[s].q_version; break; }
    return t;
  }
  int rem = k;
  for (int s = 0; s < a.max_segs; ++s) {
    const int len = sg[s].row_end - sg[s].row_begin;
    if (len <= 0) continue;
    const int np = (len + kN - 1) / kN;
    if (rem < np) {
      const int row0 = sg[s].row_begin + rem * kN;
      const int page = a.block_table[(size_t)b * a.max_pages + row0 / kN];
      t.ver = sg[s].q_version;
      t.kpos0 = sg[s].key_pos_base + (row0 - sg[s].row_begin);
      if (page >= 0 && page < a.n_pages) {
        t.n_valid = min(kN, sg[s].row_end - row0);
        t.phys0 = (long long)page * kN;
      } else {
        set_status(MLA_ERR_BAD_INDEX);   // the page's rows are left out, never read
      }
      return t;
    }
    rem -= np;
  }
  return t;
}

// Walk of one worker's units in (stream, page) order.
struct Walk {
  int s, k, u, u1;
};

__device__ __forceinline__ int stream_tiles(const Params& p, int s) {
  return p.stream_off[s + 1] - p.stream_off[s];
}

__device__ __forceinline__ bool walk_begin(const Params& p, int g, Walk& w) {
  const int U = p.plan->U, C = p.plan->C;
  const long long u0 = (long long)g * C;
  if (u0 >= U) return false;
  w.u = (int)u0;
  w.u1 = (int)min((long long)U, u0 + C);
  int lo = 0, hi = p.plan->n_streams - 1;   // last stream with off <= u0
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.stream_off[mid] <= w.u) lo = mid; else hi = mid - 1;
  }
  w.s = lo;
  while (stream_tiles(p, w.s) == 0) ++w.s;
  w.k = w.u - p.stream_off[w.s];
  return true;
}

__device__ __forceinline__ void walk_next(const Params& p, Walk& w) {
  ++w.u;
  ++w.k;
  if (w.u < w.u1 && w.k >= stream_tiles(p, w.s)) {
    ++w.s;
    while (stream_tiles(p, w.s) == 0) ++w.s;
    w.k = 0;
  }
}

struct StreamPos {
  int b, j, hb;
};
__device__ __forceinline__ StreamPos stream_pos(const Params& p, int s) {
  StreamPos r;
  r.hb = s % p.n_hb;
  const int bj = s / p.n_hb;
  r.j = bj % p.a.s_q;
  r.b = bj / p.a.s_q;
  return r;
}

// ----------------------------------------------------------------- barriers
struct Bars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_done, o_free;
  uint64_t x_full, x_empty;
  uint64_t mma_drain;
  uint32_t tmem_base;
};
static_assert(sizeof(Bars) <= kBarBytes, "barrier block too large");

__device__ __forceinline__ void fail(bool& ok) {
  if (ok) set_status(MLA_ERR_TIMEOUT);
  ok = false;
}

// ----------------------------------------------------------------- kernel
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ Params p,
                 const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_kv0,
                 const __grid_constant__ CUtensorMap tm_kv1,
                 const __grid_constant__ CUtensorMap tm_kv2,
                 const __grid_constant__ CUtensorMap tm_kv3,
                 const __grid_constant__ CUtensorMap tm_kv4,
                 const __grid_constant__ CUtensorMap tm_kv5,
                 const __grid_constant__ CUtensorMap tm_kv6) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sKV = smem + kOffKV;
  uint8_t* sP = smem + kOffP;
  float* sX = reinterpret_cast<float*>(smem + kOffX);
  Bars* bar = reinterpret_cast<Bars*>(smem + kOffBar);

  const DecodeArgs& a = p.a;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int g = blockIdx.x >> 1;
  const int panels = (rank == 0) ? 5 : 4;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar->kv_full[i], 1);
      mbar_init(&bar->kv_empty[i], 1);
    }
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar->s_full[i], 1);
      mbar_init(&bar->s_empty[i], 4);
      mbar_init(&bar->p_full[i], 4);
      mbar_init(&bar->p_empty[i], 1);
    }
    mbar_init(&bar->o_done, 1);
    mbar_init(&bar->o_free, 4);
    mbar_init(&bar->x_full, kM);
    mbar_init(&bar->x_empty, kM);
    mbar_init(&bar->mma_drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();   // peer barriers initialised before any remote arrive
  const uint32_t tmem = bar->tmem_base;

  Walk w;
  const bool has_work = walk_begin(p, g, w);
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_kv0);
    }
    const CUtensorMap* kvmaps[kNumBoxHeights] = {&tm_kv0, &tm_kv1, &tm_kv2, &tm_kv3,
                                                 &tm_kv4, &tm_kv5, &tm_kv6};
    int it = 0, n_qload = 0, cur_s = -1, cur_v = -1;
    for (bool more = has_work; more && ok; more = (w.u < w.u1)) {
      const StreamPos sp = stream_pos(p, w.s);
      const Tile t = describe(a, sp.b, w.k);
      if (w.s != cur_s || t.ver != cur_v) {
        if (n_qload > 0 && !mbar_wait(&bar->q_empty, (n_qload - 1) & 1)) { fail(ok); break; }
        if (lane == 0) {
          const int qi = sp.b * a.s_q + sp.j;
          const int y = (t.ver * a.n_q + qi) * a.H + a.h0 + sp.hb * kM;
          mbar_arrive_expect_tx(&bar->q_full, panels * kPanelQ);
          for (int pn = 0; pn < panels; ++pn) {
            const int x = (pn == 4) ? kDc : (int)rank * 256 + pn * 64;
            tma_load_2d(sQ + pn * kPanelQ, &tm_q, &bar->q_full, x, y);
          }
        }
        ++n_qload;
        cur_s = w.s;
        cur_v = t.ver;
      }
      const int st = it % kStages;
      if (!mbar_wait(&bar->kv_empty[st], ((it / kStages) & 1) ^ 1)) { fail(ok); break; }
      uint8_t* stage = sKV + st * kStageBytes;
      if (t.n_valid < kN) {
        // rows without data must read as zero in the P.c product
        const int zrows = kN - t.n_valid;
        for (int e = lane; e < panels * zrows * 8; e += 32) {
          const int pn = e / (zrows * 8);
          const int rr = t.n_valid + (e / 8) % zrows;
          const int ch = e % 8;
          *reinterpret_cast<uint4*>(stage + pn * kPanelKV + rr * 128 + ch * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();
        __syncwarp();
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar->kv_full[st], t.n_valid * panels * 128);
        if (!t.gather) {
          int row = 0;
          for (int hb = 0; hb < kNumBoxHeights; ++hb) {
            const int h = kN >> hb;
            if (t.n_valid & h) {
              for (int pn = 0; pn < panels; ++pn) {
                const int x = (pn == 4) ? kDc : (int)rank * 256 + pn * 64;
                tma_load_2d(stage + pn * kPanelKV + row * 128, kvmaps[hb], &bar->kv_full[st],
                            x, (int)(t.phys0 + row));
              }
              row += h;
            }
          }
        }
      }
      if (t.gather) {
        // one row per box; lanes split the rows, lane 0 already armed the barrier
        __syncwarp();
        for (int i = lane; i < t.n_valid; i += 32) {
          long long phys;
          int kpos, ver;
          if (!locate_row(a, sp.b, w.k * kN + i, &phys, &kpos, &ver)) phys = -1;
          for (int pn = 0; pn < panels; ++pn) {
            const int x = (pn == 4) ? kDc : (int)rank * 256 + pn * 64;
            if (phys >= 0) {
              tma_load_2d(stage + pn * kPanelKV + i * 128, kvmaps[kNumBoxHeights - 1],
                          &bar->kv_full[st], x, (int)phys);
            } else {
              // unlocatable row: zero it and account its bytes as arrived
              for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4*>(stage + pn * kPanelKV + i * 128 + ch * 16) =
                    make_uint4(0, 0, 0, 0);
            }
          }
          if (phys < 0) {
            fence_proxy_async();
            asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;"
                         ::"r"(smem_u32(&bar->kv_full[st])), "r"(panels * 128) : "memory");
          }
        }
      }
      ++it;
      walk_next(p, w);
    }
    // drain: every load issued by this warp has landed before the CTA exits
    for (int d = 1; d <= kStages && d <= it; ++d) {
      const int n = it - d;
      if (!mbar_wait(&bar->kv_full[n % kStages], (n / kStages) & 1)) { fail(ok); break; }
    }
    if (n_qload > 0 && !mbar_wait(&bar->q_full, (n_qload - 1) & 1)) fail(ok);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kM, kN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kM, 256, false, true);
      int it = 0, n_q = 0, cur_s = -1, cur_v = -1, n_streams = 0;
      int prev_first = 0, prev_stream_idx = 0;
      auto issue_pv = [&](int t, int first, int stream_idx) -> bool {
        const int pb = t & 1;
        if (!mbar_wait(&bar->p_full[pb], (t >> 1) & 1)) return false;
        if (first && stream_idx > 0 && !mbar_wait(&bar->o_free, (stream_idx - 1) & 1))
          return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(sP + pb * kPBytes);
        const uint32_t vb = smem_u32(sKV + (t % kStages) * kStageBytes);
#pragma unroll
        for (int ks = 0; ks < kN / 16; ++ks) {
          const uint64_t ad = smem_desc_sw128(pa + ks * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(vb + ks * 16 * 128, kPanelKV, 1024);
          mma_bf16_ss(tmem + kColO, ad, bd, idesc_pv, (first && ks == 0) ? 0u : 1u);
        }
        mma_commit(&bar->kv_empty[t % kStages]);
        mma_commit(&bar->p_empty[pb]);
        mma_commit(&bar->o_done);
        return true;
      };
      for (bool more = has_work; more && ok; more = (w.u < w.u1)) {
        const StreamPos sp = stream_pos(p, w.s);
        const Tile t = describe(a, sp.b, w.k);
        const bool first = (w.s != cur_s);
        if (first) ++n_streams;
        if (first || t.ver != cur_v) {
          if (!mbar_wait(&bar->q_full, n_q & 1)) { fail(ok); break; }
          ++n_q;
          cur_s = w.s;
          cur_v = t.ver;
        }
        const int st = it % kStages;
        if (!mbar_wait(&bar->kv_full[st], (it / kStages) & 1)) { fail(ok); break; }
        const int sb = it & 1;
        if (!mbar_wait(&bar->s_empty[sb], ((it >> 1) & 1) ^ 1)) { fail(ok); break; }
        tc_fence_after();
        const uint32_t qa = smem_u32(sQ);
        const uint32_t kb = smem_u32(sKV + st * kStageBytes);
        for (int pn = 0; pn < panels; ++pn) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = smem_desc_sw128(qa + pn * kPanelQ + ks * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(kb + pn * kPanelKV + ks * 32, 16, 1024);
            mma_bf16_ss(tmem + kColS + sb * kN, ad, bd, idesc_qk, (pn | ks) ? 1u : 0u);
          }
        }
        mma_commit(&bar->s_full[sb]);
        // does the next unit of this worker need another Q?
        Walk nx = w;
        walk_next(p, nx);
        if (nx.u < nx.u1) {
          const Tile tn = describe(a, stream_pos(p, nx.s).b, nx.k);
          if (nx.s != w.s || tn.ver != t.ver) mma_commit(&bar->q_empty);
        }
        if (it > 0 && !issue_pv(it - 1, prev_first, prev_stream_idx)) { fail(ok); break; }
        prev_first = first;
        prev_stream_idx = n_streams - 1;
        ++it;
        w = nx;
      }
      if (ok && it > 0 && !issue_pv(it - 1, prev_first, prev_stream_idx)) fail(ok);
      // every tcgen05 op issued here completes before TMEM is released
      mma_commit(&bar->mma_drain);
      if (!mbar_wait(&bar->mma_drain, 0)) fail(ok);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;
    const int m = quad * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t x_own = smem_u32(sX);
    const uint32_t x_peer = mapa(x_own, peer);
    const uint32_t xfull_peer = mapa(smem_u32(&bar->x_full), peer);
    const uint32_t xempty_peer = mapa(smem_u32(&bar->x_empty), peer);
    int it = 0, n_streams_done = 0;
    while (has_work && ok && w.u < w.u1) {
      const int s = w.s;
      const StreamPos sp = stream_pos(p, s);
      const int qi = sp.b * a.s_q + sp.j;
      const int qp = a.q_pos[qi];
      const int hrow = sp.hb * kM + m;          // head index within [h0, h0 + n_h)
      const bool row_valid = hrow < a.n_h;
      const int T = stream_tiles(p, s);
      float m_run = -INFINITY, l_run = 0.f;
      bool have_o = false;
      while (ok && w.u < w.u1 && w.s == s) {
        const Tile t = describe(a, sp.b, w.k);
        const int sb = it & 1;
        if (!mbar_wait(&bar->s_full[sb], (it >> 1) & 1)) { fail(ok); break; }
        tc_fence_after();
        float sv[64];
        {
          float tmp[32];
          tmem_ld32(trow + kColS + sb * kN, tmp);
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[i] = tmp[i];
          tmem_ld32(trow + kColS + sb * kN + 32, tmp);
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[32 + i] = tmp[i];
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->s_empty[sb]);

        // exchange partial scores with the peer CTA
        if (!mbar_wait_cluster(&bar->x_empty, (it & 1) ^ 1)) { fail(ok); break; }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t off = m * 256 + ((c ^ (m & 15)) << 4);
          st_cluster_v4(x_peer + off, sv[4 * c], sv[4 * c + 1], sv[4 * c + 2], sv[4 * c + 3]);
        }
        mbar_arrive_remote(xfull_peer);
        if (!mbar_wait_cluster(&bar->x_full, it & 1)) { fail(ok); break; }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float4 o = *reinterpret_cast<const float4*>(
              reinterpret_cast<const uint8_t*>(sX) + m * 256 + ((c ^ (m & 15)) << 4));
          // both CTAs add (own + peer) in an order-independent way: a + b == b + a
          sv[4 * c] += o.x;
          sv[4 * c + 1] += o.y;
          sv[4 * c + 2] += o.z;
          sv[4 * c + 3] += o.w;
        }
        mbar_arrive_remote(xempty_peer);

        // mask, scale (log2 domain), online softmax with lazy rescaling
        float mt = -INFINITY;
        if (t.gather) {
          const int i0 = w.k * kN + lane, i1 = i0 + 32;
          int kp0 = INT32_MAX, kp1 = INT32_MAX;
          long long ph;
          int vv;
          if (lane < t.n_valid && !locate_row(a, sp.b, i0, &ph, &kp0, &vv)) kp0 = INT32_MAX;
          if (lane + 32 < t.n_valid && !locate_row(a, sp.b, i1, &ph, &kp1, &vv)) kp1 = INT32_MAX;
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const int kp = __shfl_sync(0xffffffffu, (i < 32) ? kp0 : kp1, i & 31);
            const bool vis = (i < t.n_valid) && (kp <= qp);
            sv[i] = vis ? sv[i] * p.scale_log2 : -INFINITY;
            mt = fmaxf(mt, sv[i]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const bool vis = (i < t.n_valid) && (t.kpos0 + i <= qp);
            sv[i] = vis ? sv[i] * p.scale_log2 : -INFINITY;
            mt = fmaxf(mt, sv[i]);
          }
        }
        const bool need = mt > m_run + kRescaleThreshold;
        const float m_new = need ? mt : m_run;
        const float factor = need ? exp2f(m_run - m_new) : 1.f;   // exp2(-inf) = 0
        uint32_t pk[32];
        float lsum = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = (m_new == -INFINITY) ? 0.f : exp2f(sv[2 * i] - m_new);
          const float p1 = (m_new == -INFINITY) ? 0.f : exp2f(sv[2 * i + 1] - m_new);
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          lsum += __low2float(h2) + __high2float(h2);
          pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        l_run = l_run * factor + lsum;
        m_run = m_new;

        // correct O when this row's reference max moved (warp-uniform TMEM access)
        if (have_o && __any_sync(0xffffffffu, need)) {
          if (!mbar_wait(&bar->o_done, (it - 1) & 1)) { fail(ok); break; }
          tc_fence_after();
          const float f = need ? factor : 1.f;
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            float ov[32];
            tmem_ld32(trow + kColO + c, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= f;
            tmem_st32(trow + kColO + c, ov);
          }
          tmem_wait_st();
        }

        // P (bf16, 128-byte swizzled K-major rows) for the P.c product
        const int pb = it & 1;
        if (!mbar_wait(&bar->p_empty[pb], ((it >> 1) & 1) ^ 1)) { fail(ok); break; }
        uint8_t* prow = sP + pb * kPBytes + m * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          *reinterpret_cast<uint4*>(prow + ((c ^ (m & 7)) << 4)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->p_full[pb]);
        have_o = true;
        ++it;
        walk_next(p, w);
      }
      if (!ok) break;

      // epilogue: O is complete once the last P.c product of the stream is done
      if (!mbar_wait(&bar->o_done, (it - 1) & 1)) { fail(ok); break; }
      tc_fence_after();
      const int off_s = p.stream_off[s];
      const int range_u0 = g * p.plan->C;
      const bool whole = (off_s >= range_u0) && (off_s + T <= w.u1);
      const bool empty = !(l_run > 0.f);
      const float inv = empty ? 0.f : 1.f / l_run;
      const float lse = empty ? -INFINITY : (m_run + log2f(l_run)) * 0.6931471805599453f;
      float* dst;
      size_t lse_idx;
      float* lse_base;
      if (whole) {
        const size_t orow = (size_t)qi * a.H + a.h0 + hrow;
        dst = a.o_lat + orow * kDc + rank * 256;
        lse_base = a.lse;
        lse_idx = orow;
      } else {
        const int slot = 2 * g + ((off_s <= range_u0) ? 0 : 1);
        float* sl = p.partial + (size_t)slot * kSlotFloats;
        dst = sl + (size_t)m * kDc + rank * 256;
        lse_base = sl + (size_t)kM * kDc;
        lse_idx = m;
      }
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        float ov[32];
        tmem_ld32(trow + kColO + c, ov);
        tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            *reinterpret_cast<float4*>(dst + c + i) =
                make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
          }
        }
      }
      if (row_valid && rank == 0) lse_base[lse_idx] = lse;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->o_free);
      ++n_streams_done;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no CTA leaves while its peer may still touch its shared memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------- planner
// One CTA: per-sequence tile counts, validation, stream offsets, chunk size.
__global__ void plan_kernel(DecodeArgs a, int n_hb, int G, PlanHeader* plan, int* stream_off,
                            int* stream_bad) {
  const int n_rt = a.s_q * n_hb;
  const int n_streams = a.B * n_rt;
  __shared__ int s_total;
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
    int tiles = 0;
    bool bad = false;
    const mla_seg_t* sg = a.segs + (size_t)b * a.max_segs;
    int prev_end = 0;
    for (int s = 0; s < a.max_segs; ++s) {
      const int rb = sg[s].row_begin, re = sg[s].row_end;
      if (re == rb) continue;
      if (rb < prev_end || re < rb || rb % kN != 0 || re > a.max_pages * kN ||
          sg[s].q_version < 0 || sg[s].q_version >= a.n_ver) {
        bad = true;
        break;
      }
      prev_end = re;
      tiles += (re - rb + kN - 1) / kN;
    }
    if (a.gather_rows) {
      const int ng = a.n_gather[b];
      if (ng < 0 || ng > a.max_gather) bad = true;
      tiles = bad ? 0 : (ng + kN - 1) / kN;
      // every tile of gathered rows must share one query version
      for (int k = 0; !bad && k < tiles; ++k) {
        int v0 = -1;
        for (int i = k * kN; i < min(ng, k * kN + kN); ++i) {
          const int r = a.gather_rows[(size_t)b * a.max_gather + i];
          int v = -1;
          for (int s = 0; s < a.max_segs; ++s)
            if (r >= sg[s].row_begin && r < sg[s].row_end) { v = sg[s].q_version; break; }
          if (v < 0 || (v0 >= 0 && v != v0)) { bad = true; break; }
          v0 = v;
        }
      }
    }
    if (bad) {
      set_status(MLA_ERR_BAD_INDEX);
      tiles = 0;
    }
    for (int r = 0; r < n_rt; ++r) {
      stream_off[b * n_rt + r] = tiles;     // counts for now
      stream_bad[b * n_rt + r] = bad ? 1 : 0;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int s = 0; s < n_streams; ++s) {
      const int c = stream_off[s];
      stream_off[s] = acc;
      acc += c;
    }
    stream_off[n_streams] = acc;
    s_total = acc;
    plan->U = acc;
    plan->G = G;
    plan->n_streams = n_streams;
    plan->C = max(kMinChunk, (acc + G - 1) / max(G, 1));
  }
}

// ----------------------------------------------------------------- combine
// One CTA per stream: merge the split partials by log-sum-exp, or write the
// empty result for streams with no tiles (NaN when the sequence was invalid).
__global__ void __launch_bounds__(256) combine_kernel(DecodeArgs a, int n_hb,
                                                      const PlanHeader* plan,
                                                      const int* stream_off,
                                                      const int* stream_bad,
                                                      const float* partial) {
  const int s = blockIdx.x;
  const int hb = s % n_hb;
  const int qi = s / n_hb;             // (b * s_q + j)
  const int rows = min(kM, a.n_h - hb * kM);
  const int T = stream_off[s + 1] - stream_off[s];
  const int C = plan->C;
  __shared__ int slot_s[8];
  if (T == 0) {
    const float fill = stream_bad[s] ? __int_as_float(0x7fc00000) : 0.f;
    const float lfill = stream_bad[s] ? __int_as_float(0x7fc00000) : -INFINITY;
    for (int e = threadIdx.x; e < rows * kDc; e += blockDim.x) {
      const int m = e / kDc, c = e % kDc;
      a.o_lat[((size_t)qi * a.H + a.h0 + hb * kM + m) * kDc + c] = fill;
    }
    for (int m = threadIdx.x; m < rows; m += blockDim.x)
      a.lse[(size_t)qi * a.H + a.h0 + hb * kM + m] = lfill;
    return;
  }
  const int off = stream_off[s];
  const int g0 = off / C, g1 = (off + T - 1) / C;
  if (g0 == g1) return;   // a single worker covered the stream and wrote it
  const int ns = g1 - g0 + 1;
  // merge in groups of up to 8 splits (running log-sum-exp across groups)
  for (int m = 0; m < rows; ++m) {
    const size_t orow = (size_t)qi * a.H + a.h0 + hb * kM + m;
    float run_l = -INFINITY;
    for (int gb = 0; gb < ns; gb += 8) {
      const int cnt = min(8, ns - gb);
      __syncthreads();
      if (threadIdx.x < cnt) {
        const int gg = g0 + gb + threadIdx.x;
        slot_s[threadIdx.x] = 2 * gg + ((off <= gg * C) ? 0 : 1);
      }
      __syncthreads();
      float l_i[8];
      float lmax = run_l;
      for (int i = 0; i < cnt; ++i) {
        l_i[i] = partial[(size_t)slot_s[i] * kSlotFloats + (size_t)kM * kDc + m];
        lmax = fmaxf(lmax, l_i[i]);
      }
      float wrun = 0.f, wi[8], tot = 0.f;
      if (lmax != -INFINITY) {
        wrun = (run_l == -INFINITY) ? 0.f : __expf(run_l - lmax);
        tot = wrun;
        for (int i = 0; i < cnt; ++i) {
          wi[i] = (l_i[i] == -INFINITY) ? 0.f : __expf(l_i[i] - lmax);
          tot += wi[i];
        }
      } else {
        for (int i = 0; i < cnt; ++i) wi[i] = 0.f;
      }
      const float inv = (tot > 0.f) ? 1.f / tot : 0.f;
      for (int c = threadIdx.x; c < kDc; c += blockDim.x) {
        float acc = (gb == 0) ? 0.f : a.o_lat[orow * kDc + c] * wrun;
        for (int i = 0; i < cnt; ++i) {
          if (wi[i] != 0.f) acc += wi[i] * partial[(size_t)slot_s[i] * kSlotFloats + (size_t)m * kDc + c];
        }
        a.o_lat[orow * kDc + c] = acc * inv;
      }
      run_l = (tot > 0.f) ? lmax + logf(tot) : -INFINITY;
    }
    if (threadIdx.x == 0) a.lse[orow] = run_l;
  }
}

}  // namespace tc
}  // namespace mla
