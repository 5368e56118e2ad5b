// decode_tc.cuh -- absorbed MLA decode on sm_100a tensor cores (CTA pairs).
//
// What it computes (Day 27 tutorial "Multi-Head Latent Attention", sections
// "Move the Key Projection Into the Query", "Position Rotations Complicate
// the Absorption", "Move the Value Expansion After the Weighted Sum"): for
// 128 query rows (one query token x up to 128 heads) and every cached row t,
//     S[m, t] = scale * (q_abs[m, :512] . c_t + q_abs[m, 512:] . k_rope_t)
//     P = online-softmax(S masked by key_pos(t) <= q_pos),  O[m, :] = sum_t P[m,t] c_t
// reading each 576-element latent row [c_t | k_rope_t] from HBM once.
//
// Decomposition.  A cluster of two CTAs on two SMs shares one tcgen05 MMA
// (cta_group::2): CTA r holds the query rows of heads [64r, 64r + 64) and the
// cache rows of page 2k + r of a 128-row tile; the pair computes the full
// 128 x 128 score tile (N=128 MMAs accumulated over two column stages of the
// pages), each CTA receiving its 64 head rows in TMEM (tokens 0-63 in lanes
// 0-63, tokens 64-127 in lanes 64-127 of the same columns).  The softmax of
// a head row is shared by lanes t and t + 64 (the row max is combined
// through shared memory).  P . c runs as M=128 x N=256 pair MMAs; in MMA nb
// CTA r supplies latent columns [256 r + 128 nb, +128) for all 128 rows
// (re-read through L2), so each CTA's value columns are one contiguous half
// and O for its 64 heads lies in 256 TMEM columns with latent [0, 256) in
// lanes 0-63 and [256, 512) in lanes 64-127.  No scores or probabilities
// cross between the SMs: only the MMA operands do, inside the pair
// instruction.
//
// Loads.  Full rows are fetched with multi-dimensional TMA boxes so that each
// request covers long contiguous row runs: a score stage is one box of 64
// cache rows x 5 or 4 64-column panels (640/512-byte runs), a value stage
// one box of 32 rows x this CTA's four latent panels (512-byte runs, 16 KB),
// Q one box of 64 rows x 9 panels.  Partial pages and gathered rows use
// per-panel boxes of power-of-two heights, and rows without data come from
// boxes placed past the end of the cache, which the hardware fills with
// zeros.  The own-page rows of the next two tiles are prefetched into L2.
//
// Roles per CTA (224 threads): warp 0 streams Q and the score stages, warp 6
// the value stages (TMA), warp 1 of CTA 0 issues every MMA of the pair from
// per-tile flags precomputed in shared memory, warps 2-5 own one TMEM lane
// each for softmax and the epilogue (each CTA forwards one softmax-done
// arrival per tile to the issuer).  Work is split over CTA pairs as
// contiguous runs of (sequence, head block, tile) units -- runs that never
// straddle two sequences when all have the same length; a pair writes the
// final result of a sequence it covers entirely, else a normalised partial
// (o, lse) that the combine kernel merges.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace tc {

constexpr int kDc = 512, kDr = 64, kRow = kDc + kDr;
constexpr int kM = 128;                  // query rows of the pair
constexpr int kMh = 64;                  // query rows per CTA
constexpr int kT = 128;                  // cache rows per tile (two pages)
constexpr int kPg = 64;                  // rows per page
constexpr int kR = 32;                   // cache rows per value stage
constexpr int kQPanels = 9;              // 8 latent + 1 rotary 64-column panels
constexpr int kQPanel = kMh * 128;       // 64 rows x 128 B = 8 KB
constexpr int kSPanel = kR * 128;        // 32 rows x 128 B = 4 KB
constexpr int kKPanel = kPg * 128;       // 64 rows x 128 B = 8 KB
// Score stages split a page's rows by columns: stage 0 holds panels 0-4 and
// stage 1 panels 5-8 of all 64 rows, so each score MMA spans the page (N=128
// for the pair) and the two stages of a tile alternate between fixed slots.
constexpr int kKSplit = 5;                              // panels in stage 0
constexpr int kKStage0 = kKSplit * kKPanel;             // 40 KB
constexpr int kKStage1 = (kQPanels - kKSplit) * kKPanel;  // 32 KB
constexpr int kVStage = 4 * kSPanel;          // 16 KB: 32 rows x this CTA's 4 latent panels
constexpr int kKStages = 2, kVStages = 3;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQPanels * kQPanel;
constexpr int kOffV = kOffK + kKStage0 + kKStage1;
constexpr int kOffP = kOffV + kVStages * kVStage;
constexpr int kPBuf = 2 * kQPanel;       // 64 rows x 128 tokens bf16 (two 64-token panels)
constexpr int kOffMisc = kOffP + 2 * kPBuf;
constexpr int kMiscBytes = 1536;
constexpr int kOffBar = kOffMisc + kMiscBytes;
constexpr int kBarBytes = 512;
constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;   // + alignment slack
constexpr int kThreads = 224;
constexpr int kTmemCols = 512;
constexpr int kColO = 0, kColS = 256;
constexpr int kMinChunk = 2;
constexpr int kPlanThreads = 1024;       // planner block (one CTA)
constexpr int kPrefetchTiles = 2;        // tiles of own-page rows requested into L2 ahead
constexpr int kFlagTiles = 256;          // per-tile issue flags precomputed in shared memory
constexpr int kNumBoxHeights = 6;        // 32, 16, 8, 4, 2, 1 rows
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: lazy rescale margin
constexpr int kStoreCols = 32;           // fp32 columns per output store box (128 B)
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct PlanHeader {
  int U, C, G, n_streams;
};

// TMA descriptors (all 64 columns wide, 128-byte swizzle):
//   q   3-D (col, q_abs row, panel): 64 rows x 9 panels of one head block
//   k0  3-D (col, cache row, panel): 64 rows x panels 0-4 (score stage 0)
//   k1  3-D (col, cache row, panel): 64 rows x panels 5-8 (score stage 1)
//   v   3-D (col, cache row, panel): 32 rows x 4 panels (one latent half)
//   row 2-D (col, cache row): boxes of 32 >> i rows (i = 0..5) for partial
//       pages, gathered rows and zero rows past the end of the cache
// and two fp32 store maps (32 columns x 32 rows, 128-byte swizzle):
//   o   3-D (col, head - h0, query row) over o_lat: heads past n_h are
//       clipped by the map, so a store never reaches another head range
//   part 2-D (col, slot row) over the split partials [2G x 128, 512]
struct Maps {
  CUtensorMap q, k0, k1, v;
  CUtensorMap row[kNumBoxHeights];
  CUtensorMap o, part;
};

struct Params {
  DecodeArgs a;
  int n_hb;
  int G;
  const PlanHeader* plan;
  const int* stream_off;
  const int* pair_stream;  // stream holding the first unit of each pair's run
  float* partial_lse;     // [2G x 128] (the rows live behind the part map)
  float scale_log2;
};

// ----------------------------------------------------------------- tiles
struct Tile {
  int ver;
  bool gather;
  int g0;              // gather: index of the tile's first gathered row
  int n_rows;          // gather: gathered rows in the tile (1..128)
  long long phys0, phys1;   // page mode: physical row of each page's row 0
  int nv0, nv1;             // page mode: valid rows of each page (0 = absent)
  int kpos0, kpos1;         // page mode: request position of each page's row 0
};

// Number of 128-row tiles of a segment of len rows (pages are paired inside
// a segment, so a tile never mixes relocation versions).
__device__ __forceinline__ int seg_tiles(int len) {
  const int np = (len + kPg - 1) / kPg;
  return (np + 1) / 2;
}

// kGather: the call attends gathered rows (gather_rows != null).  The kernels
// are instantiated per mode, so the page-mode instantiation carries no code
// for gathered rows.
template <bool kGather>
__device__ __forceinline__ Tile describe(const DecodeArgs& a, int b, int k) {
  Tile t;
  t.gather = kGather;
  t.ver = 0;
  t.g0 = 0;
  t.n_rows = 0;
  t.phys0 = t.phys1 = 0;
  t.nv0 = t.nv1 = 0;
  t.kpos0 = t.kpos1 = 0;
  const mla_seg_t* sg = a.segs + (size_t)b * a.max_segs;
  if constexpr (kGather) {
    const int ng = a.n_gather[b];
    t.g0 = k * kT;
    t.n_rows = min(kT, ng - t.g0);
    const int r0 = a.gather_rows[(size_t)b * a.max_gather + t.g0];
    for (int s = 0; s < a.max_segs; ++s)
      if (r0 >= sg[s].row_begin && r0 < sg[s].row_end) { t.ver = sg[s].q_version; break; }
    return t;
  }
  int rem = k;
  for (int s = 0; s < a.max_segs; ++s) {
    const int len = sg[s].row_end - sg[s].row_begin;
    if (len <= 0) continue;
    const int nt = seg_tiles(len);
    if (rem < nt) {
      t.ver = sg[s].q_version;
      const int np = (len + kPg - 1) / kPg;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int pi = 2 * rem + i;
        if (pi >= np) break;
        const int row0 = sg[s].row_begin + pi * kPg;
        const int page = a.block_table[(size_t)b * a.max_pages + row0 / kPg];
        const int kp = sg[s].key_pos_base + (row0 - sg[s].row_begin);
        int nv = 0;
        long long ph = 0;
        if (page >= 0 && page < a.n_pages) {
          nv = min(kPg, sg[s].row_end - row0);
          ph = (long long)page * kPg;
        } else {
          set_status(MLA_ERR_BAD_INDEX);   // the page's rows are left out, never read
        }
        if (i == 0) { t.kpos0 = kp; t.nv0 = nv; t.phys0 = ph; }
        else        { t.kpos1 = kp; t.nv1 = nv; t.phys1 = ph; }
      }
      return t;
    }
    rem -= nt;
  }
  return t;
}

// Relocation version of tile k of sequence b, from the segment table alone
// (no block-table read: the MMA issuer only needs to know when the query
// panel changes).  0 if the tile lies in no segment, as in describe(): the
// loader and the issuer must take the same query-reload decisions.
template <bool kGather>
__device__ __forceinline__ int tile_version(const DecodeArgs& a, int b, int k) {
  const mla_seg_t* sg = a.segs + (size_t)b * a.max_segs;
  if constexpr (kGather) {
    const int r0 = a.gather_rows[(size_t)b * a.max_gather + k * kT];
    for (int s = 0; s < a.max_segs; ++s)
      if (r0 >= sg[s].row_begin && r0 < sg[s].row_end) return sg[s].q_version;
    return 0;
  }
  int rem = k;
  for (int s = 0; s < a.max_segs; ++s) {
    const int len = sg[s].row_end - sg[s].row_begin;
    if (len <= 0) continue;
    const int nt = seg_tiles(len);
    if (rem < nt) return sg[s].q_version;
    rem -= nt;
  }
  return 0;
}

// rows of tile half i (tile rows [64 i, 64 i + 64)) that hold data
__device__ __forceinline__ int half_rows(const Tile& t, int i) {
  if (t.gather) return max(0, min(kPg, t.n_rows - kPg * i));
  return i ? t.nv1 : t.nv0;
}
__device__ __forceinline__ long long half_phys(const Tile& t, int i) { return i ? t.phys1 : t.phys0; }
__device__ __forceinline__ int half_kpos(const Tile& t, int i) { return i ? t.kpos1 : t.kpos0; }

struct Walk {
  int s, k, u, u1;
};

__device__ __forceinline__ int stream_tiles(const Params& p, int s) {
  return p.stream_off[s + 1] - p.stream_off[s];
}

// The stream holding unit u: the last stream whose offset is <= u (streams
// without tiles share their successor's offset, so this is never one).
__device__ __forceinline__ int stream_of(const int* stream_off, int n_streams, int u, int lo) {
  int hi = n_streams - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (stream_off[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ bool walk_begin(const Params& p, int g, Walk& w) {
  const int U = p.plan->U, C = p.plan->C;
  const long long u0 = (long long)g * C;
  if (u0 >= U) return false;
  w.u = (int)u0;
  w.u1 = (int)min((long long)U, u0 + C);
  w.s = p.pair_stream[g];
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

// Issue flags of unit u of a pair's run starting at u0: bit 0, the unit opens
// a stream; bit 1, it needs another query panel (new stream or relocation
// version).  The same decisions as the query loader's.
template <bool kGather>
__device__ __forceinline__ uint32_t unit_flags(const Params& p, int u, int u0, int s_lo) {
  const int n_streams = p.plan->n_streams;
  const int s = stream_of(p.stream_off, n_streams, u, s_lo);
  const int ver = tile_version<kGather>(p.a, stream_pos(p, s).b, u - p.stream_off[s]);
  if (u == u0) return 3u;
  const int sp = stream_of(p.stream_off, n_streams, u - 1, s_lo);
  if (sp != s) return 3u;
  return tile_version<kGather>(p.a, stream_pos(p, sp).b, u - 1 - p.stream_off[sp]) != ver ? 2u
                                                                                       : 0u;
}

// ----------------------------------------------------------------- barriers
struct Bars {
  uint64_t kfull[kKStages], kempty[kKStages];
  uint64_t vfull[kVStages], vempty[kVStages];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_empty[2];
  // softmax of tile t done (S read, P written) in both CTAs: one arrival per
  // CTA, forwarded after the CTA's four softmax warps met on sm_local
  uint64_t sp_done[2], sm_local[2];
  uint64_t o_done[2], o_free;       // o_done[t & 1]: P.c of tile t complete
  uint64_t mma_drain;
  uint64_t k_started;               // this CTA's first query and score loads are issued
  uint64_t row_sync[2], l_sync;     // the 128 softmax threads of one CTA
  uint32_t tmem_base;
  uint8_t tflags[kFlagTiles];       // unit_flags of the pair's tiles (runs <= kFlagTiles)
};
static_assert(sizeof(Bars) <= kBarBytes, "barrier block too large");

__device__ __forceinline__ void fail(bool& ok) {
  if (ok) set_status(MLA_ERR_TIMEOUT);
  ok = false;
}

// Bounded waits whose outcome is the same for every lane of the warp, so a
// timeout makes the whole warp leave together.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}
__device__ __forceinline__ bool wait_warp_cluster(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait_cluster(bar, parity));
}

// Arrive on a barrier of the pair's rank-0 CTA (local or remote).
__device__ __forceinline__ void arrive_leader(uint64_t* bar, uint32_t rank) {
  if (rank == 0) mbar_arrive(bar);
  else mbar_arrive_cluster_addr(mapa(smem_u32(bar), 0));
}

// Fill smem rows [r0, r0 + n) (pitch 128 B, n <= 64) of one 64-column panel
// from cache rows starting at y, as power-of-two boxes.  A y at or past the end of
// the cache (oob) makes the hardware fill the rows with zeros, so rows
// without data read as 0 in the P.c product without any generic-proxy store.
__device__ __forceinline__ void load_rows(uint8_t* dst, const Maps& mp, uint32_t bar, int x,
                                          long long y, int r0, int n) {
  int r = r0;
  for (; n - (r - r0) > kR; r += kR)   // n <= 64: at most one leading full box
    tma_load_2d_pair(dst + r * 128, &mp.row[0], bar, x, (int)(y + (r - r0)));
  n -= r - r0;
#pragma unroll 1
  for (int hb = 0; hb < kNumBoxHeights; ++hb) {
    const int h = kR >> hb;
    if (n & h) {
      tma_load_2d_pair(dst + r * 128, &mp.row[hb], bar, x, (int)(y + (r - r0)));
      r += h;
    }
  }
}

// Gathered rows i0 + 32 k (k < N; those at or past n are absent) of sequence
// b: physical cache row (y_oob when absent or unlocatable) and request
// position (INT32_MAX likewise).  Every index, segment and block-table load of
// the N rows is issued before any result is used, so a lane pays about one
// dependent-load latency per tile rather than one per row and panel.  The
// planner has already checked that every gathered row of a live stream lies
// in a segment; a bad page id records MLA_ERR_BAD_INDEX and reads as zeros.
// Not inlined: only gathered tiles call it, and the loader loop of page tiles
// stays as compact as it is without it.
template <int N>
__device__ __noinline__ void locate_gathered(const DecodeArgs& a, int b, int i0, int n,
                                                long long y_oob, long long* phys, int* kpos) {
  const mla_seg_t* sg = a.segs + (size_t)b * a.max_segs;
  int row[N], seg[N], page[N];
  bool in[N];
#pragma unroll
  for (int k = 0; k < N; ++k) {
    row[k] = i0 + 32 * k < n ? a.gather_rows[(size_t)b * a.max_gather + i0 + 32 * k] : 0;
    seg[k] = -1;
  }
  for (int s = 0; s < a.max_segs; ++s) {
    const int rb = sg[s].row_begin, re = sg[s].row_end;
#pragma unroll
    for (int k = 0; k < N; ++k)
      if (seg[k] < 0 && row[k] >= rb && row[k] < re) seg[k] = s;
  }
#pragma unroll
  for (int k = 0; k < N; ++k) {
    const bool present = i0 + 32 * k < n;
    in[k] = present && seg[k] >= 0 && row[k] / kPage < a.max_pages;
    page[k] = in[k] ? a.block_table[(size_t)b * a.max_pages + row[k] / kPage] : -1;
    if (present && !in[k]) set_status(MLA_ERR_BAD_INDEX);
  }
#pragma unroll
  for (int k = 0; k < N; ++k) {
    phys[k] = y_oob;
    kpos[k] = INT32_MAX;
    if (in[k] && page[k] >= 0 && page[k] < a.n_pages) {
      phys[k] = (long long)page[k] * kPage + row[k] % kPage;
      kpos[k] = sg[seg[k]].key_pos_base + (row[k] - sg[seg[k]].row_begin);
    } else if (in[k]) {
      set_status(MLA_ERR_BAD_INDEX);
    }
  }
}

// Visibility of the 64 tile rows [64 half, +64) of tile t for a query at q_pos
// qp, as a bitmask (bit i: row 64 half + i exists and key_pos <= qp).  Page
// rows have consecutive key positions, so the mask is a prefix; gathered rows
// are located two per lane and combined by ballot.
__device__ __noinline__ uint64_t gather_visible(const DecodeArgs& a, const Tile& t, int b, int half,
                                               int qp, int lane) {
  long long ph[2];
  int kp[2];
  locate_gathered<2>(a, b, t.g0 + kPg * half + lane, t.g0 + t.n_rows, 0, ph, kp);
  const uint32_t lo = __ballot_sync(0xffffffffu, kp[0] <= qp);
  const uint32_t hi = __ballot_sync(0xffffffffu, kp[1] <= qp);
  return (uint64_t)lo | ((uint64_t)hi << 32);
}

template <bool kGather>
__device__ __forceinline__ uint64_t visible_rows(const DecodeArgs& a, const Tile& t, int b,
                                                 int half, int qp, int lane) {
  if constexpr (kGather) return gather_visible(a, t, b, half, qp, lane);
  const int n = min(half_rows(t, half), max(0, qp - half_kpos(t, half) + 1));
  return n >= 64 ? ~0ull : ((1ull << n) - 1ull);
}

// Rescale this warp's 32 TMEM lanes of O (256 columns) by f.
__device__ __noinline__ void scale_o(uint32_t taddr, float f) {
#pragma unroll 1
  for (int c = 0; c < 256; c += 32) {
    float ov[32];
    tmem_ld32(taddr + c, ov);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) ov[i] *= f;
    tmem_st32(taddr + c, ov);
  }
  tmem_wait_st();
}

// ----------------------------------------------------------------- kernel
template <bool kGather>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ Params p, const __grid_constant__ Maps mp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sK = smem + kOffK;
  uint8_t* sV = smem + kOffV;
  uint8_t* sP = smem + kOffP;
  float* sMax = reinterpret_cast<float*>(smem + kOffMisc);         // [2][128]
  float* sL = sMax + 2 * kM;                                       // [128]
  Bars* bar = reinterpret_cast<Bars*>(smem + kOffBar);

  const DecodeArgs& a = p.a;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int g = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&bar->kfull[i], 1);    // rank 0 arms both CTAs' bytes
      mbar_init(&bar->kempty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&bar->vfull[i], 1);
      mbar_init(&bar->vempty[i], 1);
    }
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar->s_full[i], 1);
      mbar_init(&bar->sp_done[i], 2);
      mbar_init(&bar->sm_local[i], 4);
      mbar_init(&bar->p_empty[i], 1);
    }
    mbar_init(&bar->o_done[0], 1);
    mbar_init(&bar->o_done[1], 1);
    mbar_init(&bar->o_free, 8);
    mbar_init(&bar->mma_drain, 1);
    mbar_init(&bar->k_started, 1);
    mbar_init(&bar->row_sync[0], kM);
    mbar_init(&bar->row_sync[1], kM);
    mbar_init(&bar->l_sync, kM);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&bar->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();     // both CTAs' barriers and TMEM exist before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  // Launched as a programmatic dependent of the planner: everything above
  // overlaps it; its plan and stream offsets are read only after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  Walk w;
  const bool has_work = walk_begin(p, g, w);
  bool ok = true;
  const int n_tiles = has_work ? w.u1 - w.u : 0;
  if (warp == 1 && rank == 0 && n_tiles <= kFlagTiles) {
    for (int i = lane; i < n_tiles; i += 32)
      bar->tflags[i] = (uint8_t)unit_flags<kGather>(p, w.u + i, w.u, w.s);
    __syncwarp();
  }

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------ loads
    // Every stage lands the same byte count in each CTA, all by TMA (rows
    // without data come from out-of-bounds boxes, which read as zero), so
    // rank 0 arms each stage with both CTAs' bytes and rank 1 never signals.
    const long long y_oob = a.n_pages * kPg;   // first row past the cache
    int nk = 0, nv = 0, n_qload = 0, cur_s = -1, cur_v = -1;
    if (lane == 0) {
      prefetch_tmap(&mp.q);
      prefetch_tmap(&mp.k0);
      prefetch_tmap(&mp.k1);
      prefetch_tmap(&mp.v);
      for (int i = 0; i < kNumBoxHeights; ++i) prefetch_tmap(&mp.row[i]);
    }
    // rows [0, n) of one panel, row 32 k + lane from physical row ph[k] (one
    // box per row; rows that could not be located are past the cache: zeros)
    auto gather_panel = [&](uint8_t* dst, uint32_t fb, const long long* ph, int n, int x) {
      for (int k = 0; 32 * k + lane < n; ++k)
        tma_load_2d_pair(dst + (32 * k + lane) * 128, &mp.row[kNumBoxHeights - 1], fb, x,
                         (int)ph[k]);
    };
    // physical rows of the current gathered tile: the score loader's rows
    // 64 rank + lane + 32 k (k < 2), the value loader's lane + 32 k (k < 4)
    long long gph[4];
    int gkp[4];
    // score stage j of tile t: all 64 rows of this CTA's page, panels
    // [5 j, 5 j + 5) (stage 0) or [5, 9) (stage 1), in slot j
    auto load_k = [&](const Tile& t, int b, int j) -> bool {
      if (!wait_warp(&bar->kempty[j], ((nk / kKStages) & 1) ^ 1)) return false;
      uint8_t* dst = sK + (j ? kKStage0 : 0);
      const int p0 = j ? kKSplit : 0, p1 = j ? kQPanels : kKSplit;
      const uint32_t fb = mapa(smem_u32(&bar->kfull[j]), 0);
      if (rank == 0 && lane == 0)
        mbar_arrive_expect_tx(&bar->kfull[j], 2 * (j ? kKStage1 : kKStage0));
      const int rows = half_rows(t, (int)rank);
      if constexpr (kGather) {
        for (int pn = p0; pn < p1; ++pn)
          gather_panel(dst + (pn - p0) * kKPanel, fb, gph, rows, 64 * pn);
      }
      if (lane == 0) {
        if (!kGather && rows == kPg) {
          tma_load_3d_pair(dst, j ? &mp.k1 : &mp.k0, fb, 0, (int)half_phys(t, (int)rank), p0);
        } else {
          for (int pn = p0; pn < p1; ++pn) {
            if (!kGather)
              load_rows(dst + (pn - p0) * kKPanel, mp, fb, 64 * pn, half_phys(t, (int)rank), 0, rows);
            load_rows(dst + (pn - p0) * kKPanel, mp, fb, 64 * pn, y_oob, rows, kPg - rows);
          }
        }
      }
      __syncwarp();
      ++nk;
      return true;
    };
    // value stage kc of tile t: tile rows [32 kc, +32), this CTA's latent
    // columns [256 rank, +256) (4 panels)
    auto load_v = [&](const Tile& t, int b) -> bool {
      for (int kc = 0; kc < 4; ++kc) {
        const int slot = nv % kVStages;
        if (!wait_warp(&bar->vempty[slot], ((nv / kVStages) & 1) ^ 1)) return false;
        uint8_t* dst = sV + slot * kVStage;
        const uint32_t fb = mapa(smem_u32(&bar->vfull[slot]), 0);
        if (rank == 0 && lane == 0) mbar_arrive_expect_tx(&bar->vfull[slot], 2 * kVStage);
        const int hi = kc >> 1, r0 = kR * (kc & 1);
        const int rows = max(0, min(kR, half_rows(t, hi) - r0));
        if constexpr (kGather) {
          for (int q = 0; q < 4; ++q)
            gather_panel(dst + q * kSPanel, fb, gph + kc, rows, 256 * (int)rank + 64 * q);
        }
        if (lane == 0) {
          if (!kGather && rows == kR) {
            tma_load_3d_pair(dst, &mp.v, fb, 0, (int)(half_phys(t, hi) + r0), 4 * (int)rank);
          } else {
            for (int q = 0; q < 4; ++q) {
              const int x = 256 * (int)rank + 64 * q;
              if (!kGather) load_rows(dst + q * kSPanel, mp, fb, x, half_phys(t, hi) + r0, 0, rows);
              load_rows(dst + q * kSPanel, mp, fb, x, y_oob, rows, kR - rows);
            }
          }
        }
        __syncwarp();
        ++nv;
      }
      return true;
    };
    const bool vwarp = (warp == 6);
    // L2 prefetch walker: the own-page rows of the next kPrefetchTiles tiles
    // are requested into L2 while the ring is still full, so that the stage
    // loads (and the peer's value loads of this page) hit L2.
    Walk pw = w;
    int n_tile = 0, n_pref = 2;      // the walker starts at the third tile
    if (has_work) {
      walk_next(p, pw);
      walk_next(p, pw);
    }
    for (bool more = has_work; more && ok; more = (w.u < w.u1)) {
      const StreamPos sp = stream_pos(p, w.s);
      const Tile t = describe<kGather>(a, sp.b, w.k);
      if (vwarp) {
        // the first value loads queue behind the query and score loads, which
        // the first MMAs need long before any value stage
        if (n_tile++ == 0 && !wait_warp(&bar->k_started, 0)) { fail(ok); break; }
        if constexpr (kGather) locate_gathered<4>(a, sp.b, t.g0 + lane, t.g0 + t.n_rows, y_oob, gph, gkp);
        if (!load_v(t, sp.b)) { fail(ok); break; }
        walk_next(p, w);
        continue;
      }
      if (w.s != cur_s || t.ver != cur_v) {
        if (n_qload > 0 && !wait_warp(&bar->q_empty, (n_qload - 1) & 1)) { fail(ok); break; }
        if (lane == 0) {
          const int qi = sp.b * a.s_q + sp.j;
          const int y = (t.ver * a.n_q + qi) * a.H + a.h0 + sp.hb * kM + kMh * (int)rank;
          const uint32_t qb = mapa(smem_u32(&bar->q_full), 0);
          if (rank == 0) mbar_arrive_expect_tx(&bar->q_full, 2 * kQPanels * kQPanel);
          tma_load_3d_pair(sQ, &mp.q, qb, 0, y, 0);
        }
        __syncwarp();
        ++n_qload;
        cur_s = w.s;
        cur_v = t.ver;
      }
      if constexpr (kGather)
        locate_gathered<2>(a, sp.b, t.g0 + kPg * (int)rank + lane, t.g0 + t.n_rows, y_oob, gph,
                           gkp);
      if (!load_k(t, sp.b, 0) || !load_k(t, sp.b, 1)) { fail(ok); break; }
      if (n_tile == 0 && lane == 0) mbar_arrive(&bar->k_started);
      // (not before the second tile: at start every CTA's first query and
      // score loads already fill HBM, and prefetches would only delay them)
      for (; lane == 0 && n_tile > 0 && n_pref <= n_tile + kPrefetchTiles && pw.u < pw.u1;
           ++n_pref) {
        const Tile tp = describe<kGather>(a, stream_pos(p, pw.s).b, pw.k);
        const int rows = half_rows(tp, (int)rank);
        if (!kGather && rows > 0) {
          const int y = (int)half_phys(tp, (int)rank);
          tma_prefetch_l2_3d(&mp.k0, 0, y, 0);
          tma_prefetch_l2_3d(&mp.k1, 0, y, kKSplit);
        }
        walk_next(p, pw);
      }
      __syncwarp();
      ++n_tile;
      walk_next(p, w);
    }
    // drain: every load issued here has landed before the CTA exits (the
    // stage barriers live in rank 0, which waits on them for both CTAs)
    if (rank == 0) {
      for (int d = 1; d <= kKStages && d <= nk && ok; ++d) {
        const int n = nk - d;
        if (!wait_warp(&bar->kfull[n % kKStages], (n / kKStages) & 1)) fail(ok);
      }
      for (int d = 1; d <= kVStages && d <= nv && ok; ++d) {
        const int n = nv - d;
        if (!wait_warp(&bar->vfull[n % kVStages], (n / kVStages) & 1)) fail(ok);
      }
      if (ok && !vwarp && n_qload > 0 && !wait_warp(&bar->q_full, (n_qload - 1) & 1)) fail(ok);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA (rank 0)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kM, 2 * kPg, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kM, 256, false, true);
      int it = 0, nk = 0, nv = 0, n_q = 0, n_streams = 0;
      int prev_first = 0, prev_stream_idx = 0;
      auto issue_pv = [&](int t, int first, int stream_idx) -> bool {
        const int pb = t & 1;
        if (!mbar_wait_cluster(&bar->sp_done[pb], (t >> 1) & 1)) return false;
        if (first && stream_idx > 0 && !mbar_wait_cluster(&bar->o_free, (stream_idx - 1) & 1))
          return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(sP + pb * kPBuf);
        for (int kc = 0; kc < 4; ++kc) {
          const int slot = nv % kVStages;
          if (!mbar_wait(&bar->vfull[slot], (nv / kVStages) & 1)) return false;
          tc_fence_after();
          const uint32_t vb = smem_u32(sV + slot * kVStage);
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int ks = 2 * kc + j;     // 16-row step of the 128-row tile
              const uint64_t ad =
                  smem_desc_sw128(pa + (ks >> 2) * kQPanel + (ks & 3) * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(vb + nb * 2 * kSPanel + j * 2048, kSPanel, 1024);
              mma_pair_bf16_ss(tmem + kColO + nb * 128, ad, bd, idesc_pv,
                               (first && ks == 0) ? 0u : 1u);
            }
          }
          mma_pair_commit_both(&bar->vempty[slot]);
          ++nv;
        }
        mma_pair_commit_both(&bar->p_empty[pb]);
        mma_pair_commit_both(&bar->o_done[pb]);
        return true;
      };
      // per-tile flags: from shared memory, or computed here for long runs
      auto flags_of = [&](int i) -> uint32_t {
        return n_tiles <= kFlagTiles ? bar->tflags[i]
                                     : unit_flags<kGather>(p, w.u + i, w.u, w.s);
      };
      uint32_t f = n_tiles > 0 ? flags_of(0) : 0u;
      for (; it < n_tiles && ok; ++it) {
        const bool first = f & 1u;
        if (first) ++n_streams;
        if (f & 2u) {
          if (!mbar_wait(&bar->q_full, n_q & 1)) { fail(ok); break; }
          ++n_q;
        }
        const int sb = it & 1;
        if (!mbar_wait_cluster(&bar->sp_done[sb], ((it >> 1) & 1) ^ 1)) { fail(ok); break; }
        tc_fence_after();
        const uint32_t qa = smem_u32(sQ);
        // S (64 columns: page 0 rows in lanes 0-63, page 1 rows in lanes
        // 64-127) accumulates over the two column stages of the tile
        for (int j = 0; j < 2 && ok; ++j) {
          if (!mbar_wait(&bar->kfull[j], (nk / kKStages) & 1)) { fail(ok); break; }
          tc_fence_after();
          const uint32_t kb = smem_u32(sK + (j ? kKStage0 : 0));
          const int p0 = j ? kKSplit : 0, p1 = j ? kQPanels : kKSplit;
          for (int pn = p0; pn < p1; ++pn) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t ad = smem_desc_sw128(qa + pn * kQPanel + ks * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(kb + (pn - p0) * kKPanel + ks * 32, 16, 1024);
              mma_pair_bf16_ss(tmem + kColS + sb * 64, ad, bd, idesc_qk, (pn | ks) ? 1u : 0u);
            }
          }
          mma_pair_commit_both(&bar->kempty[j]);
          ++nk;
        }
        if (!ok) break;
        mma_pair_commit_both(&bar->s_full[sb]);
        const uint32_t fn = it + 1 < n_tiles ? flags_of(it + 1) : 0u;
        if (fn & 2u) mma_pair_commit_both(&bar->q_empty);   // the next tile reloads Q
        if (it > 0 && !issue_pv(it - 1, prev_first, prev_stream_idx)) { fail(ok); break; }
        prev_first = first;
        prev_stream_idx = n_streams - 1;
        f = fn;
      }
      if (ok && it > 0 && !issue_pv(it - 1, prev_first, prev_stream_idx)) fail(ok);
      mma_pair_commit_own(&bar->mma_drain);
      if (!mbar_wait(&bar->mma_drain, 0)) fail(ok);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;
    const int t = quad * 32 + lane;           // TMEM lane
    const int half = t >> 6;                  // tile rows [64 half, +64)
    const int hl = t & 63;                    // head row of this CTA
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    int it = 0, n_epi = 0;
    // P.c of tile t is complete.  o_done[t & 1] completes once per two tiles;
    // the P buffer waits (p_empty) already ordered every earlier product of
    // the same parity, so the barrier is never a phase ahead or behind.
    auto wait_o_done = [&](int t) -> bool {
      return wait_warp(&bar->o_done[t & 1], (t >> 1) & 1);
    };
    while (has_work && ok && w.u < w.u1) {
      const int s = w.s;
      const StreamPos sp = stream_pos(p, s);
      const int qi = sp.b * a.s_q + sp.j;
      const int qp = a.q_pos[qi];
      const int hrow = sp.hb * kM + kMh * (int)rank + hl;   // head within [h0, h0 + n_h)
      const bool row_valid = hrow < a.n_h;
      const int T = stream_tiles(p, s);
      float m_run = -INFINITY, l_run = 0.f;
      bool have_o = false;
      while (ok && w.u < w.u1 && w.s == s) {
        const Tile tl = describe<kGather>(a, sp.b, w.k);
        const int sb = it & 1;
        const uint64_t vis = visible_rows<kGather>(a, tl, sp.b, half, qp, lane);
        if (!wait_warp(&bar->s_full[sb], (it >> 1) & 1)) { fail(ok); break; }
        tc_fence_after();
        const uint32_t s_col = trow + kColS + sb * 64;

        // pass 1: max of the visible scores of this lane's 64 rows
        float mh = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < 64; c += 16) {
          float x[16];
          tmem_ld16(s_col + c, x);
          tmem_wait_ld();
          const uint32_t bits = (uint32_t)(vis >> c);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (bits & (1u << i)) mh = fmaxf(mh, x[i]);
        }
        mh *= p.scale_log2;                   // scale > 0: max commutes, -inf stays
        // the two lanes of a head row agree on the tile max
        sMax[(it & 1) * kM + t] = mh;
        mbar_arrive(&bar->row_sync[it & 1]);
        if (!wait_warp(&bar->row_sync[it & 1], (it >> 1) & 1)) { fail(ok); break; }
        const float mt = fmaxf(mh, sMax[(it & 1) * kM + (t ^ 64)]);

        // lazy rescaling: keep the reference max unless it grows by > 2^8
        const bool need = mt > m_run + kRescaleThreshold;
        const float m_new = need ? mt : m_run;
        const float factor = need ? exp2f(m_run - m_new) : 1.f;   // exp2(-inf) = 0
        if (have_o && __any_sync(0xffffffffu, need)) {
          if (!wait_o_done(it - 1)) { fail(ok); break; }
          tc_fence_after();
          scale_o(trow + kColO, need ? factor : 1.f);
        }

        // pass 2: P = 2^(scale*S - m_new) on visible rows, bf16, 128-byte
        // swizzled K-major rows of the P.c operand
        const int pb = it & 1;
        if (!wait_warp(&bar->p_empty[pb], ((it >> 1) & 1) ^ 1)) { fail(ok); break; }
        uint8_t* prow = sP + pb * kPBuf + half * kQPanel + hl * 128;
        float lsum = 0.f;
        const bool any = (m_new != -INFINITY);
#pragma unroll 1
        for (int c = 0; c < 64; c += 16) {
          float x[16];
          tmem_ld16(s_col + c, x);
          tmem_wait_ld();
          const uint32_t bits = any ? (uint32_t)(vis >> c) : 0u;
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const float p0 = (bits & (1u << i)) ? ex2_approx(fmaf(x[i], p.scale_log2, -m_new)) : 0.f;
            const float p1 =
                (bits & (2u << i)) ? ex2_approx(fmaf(x[i + 1], p.scale_log2, -m_new)) : 0.f;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            lsum += __low2float(h2) + __high2float(h2);
            pk[i >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          const int ch = c >> 3;
          *reinterpret_cast<uint4*>(prow + ((ch ^ (hl & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(prow + (((ch + 1) ^ (hl & 7)) << 4)) =
              make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        l_run = l_run * factor + lsum;
        m_run = m_new;
        tc_fence_before();
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->sm_local[pb]);
        // one arrival per CTA reaches the leader: the pair's MMA traffic
        // shares the path a remote arrival takes, so fewer of them land sooner
        if (quad == 0) {
          if (!wait_warp(&bar->sm_local[pb], (it >> 1) & 1)) { fail(ok); break; }
          if (lane == 0) arrive_leader(&bar->sp_done[pb], rank);
        }
        have_o = true;
        ++it;
        walk_next(p, w);
      }
      if (!ok) break;

      // epilogue: O of the stream is complete once its last P.c is done
      if (!wait_o_done(it - 1)) { fail(ok); break; }
      tc_fence_after();
      sL[t] = l_run;
      mbar_arrive(&bar->l_sync);
      if (!wait_warp(&bar->l_sync, n_epi & 1)) { fail(ok); break; }
      ++n_epi;
      const float l_tot = l_run + sL[t ^ 64];
      const int off_s = p.stream_off[s];
      const int range_u0 = g * p.plan->C;
      const bool whole = (off_s >= range_u0) && (off_s + T <= w.u1);
      const bool empty = !(l_tot > 0.f);
      const float inv = empty ? 0.f : 1.f / l_tot;
      const float lse = empty ? -INFINITY : (m_run + log2f(l_tot)) * 0.6931471805599453f;
      // O rows go out through the P buffers (idle here: the last P.c is done
      // and this warp writes no new P before the next tile's pass 2).  Each
      // warp stages its own 32 rows x 32 columns per step in an 8 KB slice
      // (two 4 KB halves, alternating) and lane 0 stores the box by TMA, so
      // no cross-warp barrier is involved.
      const int slot = 2 * g + ((off_s <= range_u0) ? 0 : 1);
      const int row0 = kMh * (int)rank + 32 * (quad & 1);   // first head row of this warp
      const bool store = !whole || sp.hb * kM + row0 < a.n_h;
#pragma unroll 1
      for (int c = 0; c < 256; c += kStoreCols) {
        const int k = c / kStoreCols;
        uint8_t* stage = sP + quad * 8192 + (k & 1) * 4096;
        if (k >= 2) {
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
        }
        float ov[kStoreCols];
        tmem_ld32(trow + kColO + c, ov);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kStoreCols; i += 4)
          *reinterpret_cast<float4*>(stage + lane * 128 + (((i >> 2) ^ (lane & 7)) << 4)) =
              make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
        fence_proxy_async();
        __syncwarp();
        if (lane == 0 && store) {
          const int lat = 256 * half + c;
          if (whole) tma_store_3d(&mp.o, stage, lat, sp.hb * kM + row0, qi);
          else tma_store_2d(&mp.part, stage, lat, slot * kM + row0);
          bulk_commit();
        }
      }
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      if (row_valid && half == 0) {
        if (whole) a.lse[(size_t)qi * a.H + a.h0 + hrow] = lse;
        else p.partial_lse[(size_t)slot * kM + kMh * (int)rank + hl] = lse;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(&bar->o_free, rank);
    }
  }

  if (warp >= 2 && warp < 6 && lane == 0) bulk_wait_all();   // epilogue stores have landed
  asm volatile("griddepcontrol.launch_dependents;");            // the merge may be scheduled
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no CTA leaves while its peer may still touch its memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------- planner
// One CTA: per-sequence tile counts, validation, stream offsets, chunk size.
template <bool kGather>
__global__ void plan_kernel(DecodeArgs a, int n_hb, int G, PlanHeader* plan, int* stream_off,
                            int* stream_bad, int* pair_stream) {
  // let the decode kernel start its set-up now (it waits for our results)
  asm volatile("griddepcontrol.launch_dependents;");
  const int n_rt = a.s_q * n_hb;
  const int n_streams = a.B * n_rt;
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
    int tiles = 0;
    bool bad = false;
    const mla_seg_t* sg = a.segs + (size_t)b * a.max_segs;
    int prev_end = 0;
    for (int s = 0; s < a.max_segs; ++s) {
      const int rb = sg[s].row_begin, re = sg[s].row_end;
      if (re == rb) continue;
      if (rb < prev_end || re < rb || rb % kPg != 0 || re > a.max_pages * kPg ||
          sg[s].q_version < 0 || sg[s].q_version >= a.n_ver) {
        bad = true;
        break;
      }
      prev_end = re;
      tiles += seg_tiles(re - rb);
    }
    if (kGather && !bad) {
      const int ng = a.n_gather[b];
      if (ng < 0 || ng > a.max_gather) bad = true;
      tiles = bad ? 0 : (ng + kT - 1) / kT;
    }
    if (bad) {
      set_status(MLA_ERR_BAD_INDEX);
      tiles = 0;
    }
    for (int r = 0; r < n_rt; ++r) {
      stream_off[b * n_rt + r] = tiles;
      stream_bad[b * n_rt + r] = bad ? 1 : 0;
    }
  }
  __syncthreads();
  if constexpr (kGather) {
    // Every gathered row must lie in a segment, and the rows of one tile
    // (entries [128 k, 128 k + 128)) in segments of one relocation version.
    // One thread per entry, all sequences at once; a failing sequence is
    // marked 2 in its first stream's flag, then every stream of it is
    // emptied and flagged.
    const long long n_entries = (long long)a.B * a.max_gather;
    for (long long f = threadIdx.x; f < n_entries; f += blockDim.x) {
      const int b = (int)(f / a.max_gather), i = (int)(f % a.max_gather);
      const int ng = a.n_gather[b];
      if (ng < 0 || ng > a.max_gather || i >= ng) continue;
      const int32_t* gr = a.gather_rows + (size_t)b * a.max_gather;
      const int r = gr[i], r0 = gr[i - i % kT];
      const mla_seg_t* sg = a.segs + (size_t)b * a.max_segs;
      int v = -1, v0 = -1;
      for (int s = 0; s < a.max_segs; ++s) {
        const int rb = sg[s].row_begin, re = sg[s].row_end, q = sg[s].q_version;
        if (v < 0 && r >= rb && r < re) v = q;
        if (v0 < 0 && r0 >= rb && r0 < re) v0 = q;
      }
      if (v < 0 || v != v0) stream_bad[b * n_rt] = 2;
    }
    __syncthreads();
    for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
      if (stream_bad[b * n_rt] != 2) continue;
      set_status(MLA_ERR_BAD_INDEX);
      for (int r = 0; r < n_rt; ++r) {
        stream_off[b * n_rt + r] = 0;
        stream_bad[b * n_rt + r] = 1;
      }
    }
    __syncthreads();
  }
  // Exclusive prefix sum of the per-stream tile counts, one block-wide pass
  // per blockDim.x streams (warp scans, then a scan of the warp totals), and
  // whether every stream has the same count as stream 0.
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, n_warps = blockDim.x >> 5;
  const int T0 = n_streams > 0 ? stream_off[0] : 0;
  bool same = true;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n_streams; base += blockDim.x) {
    const int s = base + threadIdx.x;
    const int c = s < n_streams ? stream_off[s] : 0;
    if (s < n_streams) same = same && c == T0;
    int x = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, d);
      if (lane >= d) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int t = lane < n_warps ? warp_tot[lane] : 0;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, d);
        if (lane >= d) t += y;
      }
      if (lane < n_warps) warp_tot[lane] = t;
    }
    __syncthreads();
    const int incl = carry + (wid > 0 ? warp_tot[wid - 1] : 0) + x;
    if (s < n_streams) stream_off[s] = incl - c;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = incl;
    __syncthreads();
  }
  const bool uniform = __syncthreads_and(same) && T0 > 0;
  if (threadIdx.x == 0) {
    const int acc = carry;
    stream_off[n_streams] = acc;
    plan->U = acc;
    plan->G = G;
    plan->n_streams = n_streams;
    int C = max(kMinChunk, (acc + G - 1) / max(G, 1));
    // When every stream has the same T0 tiles, a chunk that divides T0 (or is
    // a multiple of it) never straddles two streams: no pair then pays a
    // second epilogue and query reload.  Taken when it costs at most a
    // quarter more tiles per pair than the even split.
    if (uniform && G > 0) {
      int Ca = 0;
      if (n_streams > G) {
        Ca = T0 * ((n_streams + G - 1) / G);
      } else {
        for (int parts = min(T0, G / n_streams); parts >= 1 && Ca == 0; --parts)
          if (T0 % parts == 0) Ca = T0 / parts;
      }
      if (Ca >= kMinChunk && 4 * Ca <= 5 * C) C = Ca;
    }
    plan->C = C;
  }
  __syncthreads();
  // the stream holding each pair's first unit (walk start without a search)
  const int U = plan->U, C = plan->C;
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    const long long u = (long long)g * C;
    pair_stream[g] = u < U ? stream_of(stream_off, n_streams, (int)u, 0) : 0;
  }
}

// ----------------------------------------------------------------- combine
// grid (n_streams, kM / 4), a warp per query row.  Streams covered by one
// pair were written directly; split streams are merged here by log-sum-exp
// (all parts' loads are independent of one another, so they overlap);
// streams without tiles get the empty result (NaN for an invalid sequence).
__global__ void __launch_bounds__(128) combine_kernel(DecodeArgs a, int n_hb,
                                                      const PlanHeader* plan,
                                                      const int* stream_off,
                                                      const int* stream_bad,
                                                      const float* partial,
                                                      const float* partial_lse) {
  // a programmatic dependent of the decode kernel: its outputs are complete
  // and visible only after this wait
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int s = blockIdx.x;
  const int m = blockIdx.y * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int hb = s % n_hb;
  const int qi = s / n_hb;
  const int rows = min(kM, a.n_h - hb * kM);
  if (m >= rows) return;
  const int T = stream_off[s + 1] - stream_off[s];
  const size_t orow = (size_t)qi * a.H + a.h0 + hb * kM + m;
  float* o = a.o_lat + orow * kDc;
  if (T == 0) {
    const float fill = stream_bad[s] ? __int_as_float(0x7fc00000) : 0.f;
    for (int c = lane; c < kDc; c += 32) o[c] = fill;
    if (lane == 0) a.lse[orow] = stream_bad[s] ? __int_as_float(0x7fc00000) : -INFINITY;
    return;
  }
  const int C = plan->C;
  const int off = stream_off[s];
  const int g0 = off / C, g1 = (off + T - 1) / C;
  if (g0 == g1) return;   // one pair covered the stream and wrote it
  auto slot_of = [&](int gg) { return 2 * gg + ((off <= gg * C) ? 0 : 1); };
  float lmax = -INFINITY;
  for (int gg = g0 + lane; gg <= g1; gg += 32)
    lmax = fmaxf(lmax, partial_lse[(size_t)slot_of(gg) * kM + m]);
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, d));
  float4 acc[kDc / 128];
#pragma unroll
  for (int i = 0; i < kDc / 128; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  float tot = 0.f;
  if (lmax != -INFINITY) {
#pragma unroll 4
    for (int gg = g0; gg <= g1; ++gg) {
      const int sl = slot_of(gg);
      const float li = partial_lse[(size_t)sl * kM + m];
      const float wgt = (li == -INFINITY) ? 0.f : __expf(li - lmax);
      tot += wgt;
      const float4* src =
          reinterpret_cast<const float4*>(partial + ((size_t)sl * kM + m) * kDc);
#pragma unroll
      for (int i = 0; i < kDc / 128; ++i) {
        const float4 v = src[lane + 32 * i];
        acc[i].x = fmaf(wgt, v.x, acc[i].x);
        acc[i].y = fmaf(wgt, v.y, acc[i].y);
        acc[i].z = fmaf(wgt, v.z, acc[i].z);
        acc[i].w = fmaf(wgt, v.w, acc[i].w);
      }
    }
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  float4* dst = reinterpret_cast<float4*>(o);
#pragma unroll
  for (int i = 0; i < kDc / 128; ++i)
    dst[lane + 32 * i] = make_float4(acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv);
  if (lane == 0) a.lse[orow] = tot > 0.f ? lmax + logf(tot) : -INFINITY;
}

}  // namespace tc
}  // namespace mla
