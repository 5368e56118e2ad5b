// decode_tc.cuh -- absorbed MLA decode on sm_100a tensor cores.
//
// What it computes (Day 27 tutorial "Multi-Head Latent Attention", sections
// "Move the Key Projection Into the Query", "Position Rotations Complicate
// the Absorption", "Move the Value Expansion After the Weighted Sum"): for
// the (up to) 128 head rows of one query token and every cached row t,
//     S[h, t] = scale * (q_abs[h, :512] . c_t + q_abs[h, 512:] . k_rope_t)
//     P = online-softmax(S masked by key_pos(t) <= q_pos),  O[h, :] = sum_t P[h,t] c_t
// reading each 576-element latent row [c_t | k_rope_t] from HBM once.
//
// Decomposition.  Every tensor-core product runs with 128 rows per SM, the
// shape at which tcgen05 reaches its full rate (64 rows per SM run at half
// rate), and the two products live on the two CTAs of a cluster:
//   - the score CTA (rank 0) holds the 128 heads' absorbed queries: the 512
//     latent columns in tensor memory (the A operand of the score MMAs, copied
//     in by tcgen05.cp) and the 64 rotary columns in shared memory.  It
//     streams each 128-row tile of cache rows through a ring of 64-column
//     panels and computes S = Q . [c | k_rope]^T as M=128 x N=128 MMAs into a
//     double-buffered accumulator.  Its softmax threads own one head row each
//     (lane = head; two warps split a row's 128 columns and exchange only
//     the row max).  They store P in bf16, with the per-row rescale factors,
//     straight into the value CTA's shared memory, then make those writes
//     visible to its tensor core with a cluster-scope async-proxy fence and
//     a release arrival on its barrier.
//   - the value CTA (rank 1) holds O = P . c for the 128 heads in all 512
//     tensor-memory columns.  It streams the same tile's latent columns again
//     (an L2 hit: the score CTA fetched them moments before) 16 rows at a
//     time and issues M=128 x N=256 MMAs with P as the A operand.  Its
//     epilogue warps apply the occasional rescale of O and write the result.
// Work is split over clusters as contiguous runs of (sequence, query token,
// head block, tile) units; a cluster writes the final result of a stream it
// covers entirely, else a normalised partial (o, lse) that the combine kernel
// merges.
//
// Loads.  The score MMA needs both pages of a tile in each 64-column panel
// (N = 128 rows; 64-row MMAs issue no faster than 128-row ones), so a score
// stage is three such panels.  When the two pages sit next to each other in
// the pool the stage is one 3-D box; otherwise each page-panel is its own box,
// which the TMA unit serves at about half the rate (a fixed cost per box).
// A value slot is 16 rows' 8 latent panels (one 3-D box of 16 KB); the
// eight slots hold a tile, each refilled as soon as its two MMAs finish.  Rows without
// data (past a sequence's end, behind a bad page id) come from boxes placed
// past the end of the cache, which the hardware fills with zeros, so NaN in
// unused rows never reaches a product.  Gathered rows (attended through a
// gather list) arrive as four-row gather boxes.
//
// Every wait is bounded and records MLA_ERR_TIMEOUT when it gives up.
#pragma once
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace tc {

constexpr int kDc = 512, kDr = 64, kRow = kDc + kDr;
constexpr int kM = 128;                  // head rows of a stream (MMA M)
constexpr int kT = 128;                  // cache rows per tile (two pages; score MMA N)
constexpr int kPg = 64;                  // rows per page
constexpr int kPanels = 9;               // 64-column panels of a row: 8 latent + 1 rotary
constexpr int kSlot = kT * 128;          // score panel: 128 rows x 128 B = 16 KB
constexpr int kStagePanels = 3;          // score ring stage: three panels (one 3-D box when
constexpr int kStage = kStagePanels * kSlot;   //   both pages of the tile are adjacent)
constexpr int kNStages = 4;              // score-side ring stages (192 KB)
constexpr int kVRows = 16;               // value slot: 16 rows of a page, 8 latent panels
constexpr int kVSlot = 8 * kVRows * 128; //   = 16 KB
constexpr int kNV = 8;                   // value-side ring slots (128 KB)
constexpr int kVPerTile = kT / kVRows;   // value slots per tile
constexpr int kPBuf = 2 * kM * 128;      // P: 128 rows x 128 tokens bf16, two 64-token panels
constexpr int kHdrFlag = 512;            // header after P: rescale factor per row (512 B),
constexpr int kMsgStride = 33 * 1024;    //   then one flag word per softmax warp
constexpr int kEndBytes = 1536;          // per stream end: row sums of both halves, row max
constexpr int kEpiWarps = 4;             // value CTA: rescale / epilogue warps (4 or 8)
constexpr int kEpiCols = kDc * 4 / kEpiWarps;   // O columns per epilogue warp
constexpr int kStoreCols = 32;           // epilogue: O columns per TMA store box
constexpr int kStageWarp = 32 * kStoreCols * 4;   // staging: 32 rows x 32 floats per warp
// score CTA
constexpr int kOffRing = 0;
constexpr int kOffQr = kOffRing + kNStages * kStage;           // rotary query panel
constexpr int kOffMax = kOffQr + kSlot;                        // row-max exchange [2][2][128]
constexpr int kEndScore = kOffMax + 2 * 2 * kM * 4;
// value CTA
constexpr int kOffVal = 0;
constexpr int kOffMsg = kOffVal + kNV * kVSlot;                // two incoming P messages
constexpr int kOffEnd = kOffMsg + 2 * kMsgStride;
constexpr int kOffStage = kOffEnd + 2 * kEndBytes;
constexpr int kEndValue = kOffStage + kEpiWarps * kStageWarp;
// unit descriptors, then barriers, at the same offsets in both CTAs (commits
// multicast to both)
constexpr int kOffDesc = kEndScore > kEndValue ? kEndScore : kEndValue;
constexpr int kOffBar = kOffDesc + 64 * 32;
constexpr int kBarBytes = 1024;
constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;   // + alignment slack
// warp 0 loads, warp 1 issues MMAs; score CTA: warps 2-9 run the softmax (two
// per TMEM lane quarter, one 64-column half of the tile each); value CTA:
// warps 2 .. 1 + kEpiWarps rescale O and write it out (kEpiCols columns
// each); warp 10 of both computes the unit descriptors
constexpr int kThreads = 352;
constexpr int kProducerWarp = 10;
constexpr int kSoftWarps = 8;
constexpr int kTmemCols = 512;
constexpr int kColQ = 0, kColS = 256;    // score CTA: Q latent (256 columns), S double buffer
constexpr int kMinChunk = 1;
constexpr int kPlanThreads = 1024;       // planner block (one CTA)
constexpr int kNumBoxHeights = 6;        // 32, 16, 8, 4, 2, 1 rows
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: lazy rescale margin
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffMsg % 1024 == 0 && kMsgStride % 1024 == 0 && kSlot % 1024 == 0 &&
              kVSlot % 1024 == 0 && kPBuf + kHdrFlag + 4 * kSoftWarps <= kMsgStride &&
              kVRows % 16 == 0 && kPg % kVRows == 0,
              "swizzle alignment and message size");

struct PlanHeader {
  int U, C, G, n_streams;
};

// TMA descriptors (64 columns wide, 128-byte swizzle):
//   q3   3-D (col, q_abs row, panel), box {64, 128, 3}: three panels of a head block
//   qr   2-D (col, q_abs row), box {64, 128}: the rotary panel of a head block
//   k3   3-D (col, cache row, panel), box {64, 128, 3}: three panels of two
//        physically adjacent pages (one score stage)
//   kp   2-D (col, cache row), box {64, 64}: one panel of a page
//   row  2-D (col, cache row), boxes of 32 >> i rows (i = 0..5) for partial
//        pages and zero rows past the end of the cache
//   vp   3-D (col, cache row, panel), box {64, 16, 8}: 16 rows' latent panels
//   g4   2-D (col, cache row), box {64, 1}: four-row gathers
//   o    3-D fp32 (col, head, query row) over the whole-stream outputs (o_lat,
//        or the packed output of a head list), box {32, 32, 1}: heads past
//        n_h fall outside the map and are not written
//   part 2-D fp32 (col, partial row), box {32, 32}: split partials
struct Maps {
  CUtensorMap q3, qr, k3, kp;
  CUtensorMap row[kNumBoxHeights];
  CUtensorMap vp, g4;
  CUtensorMap o, part;
};

struct Params {
  DecodeArgs a;
  int n_hb;
  int G;
  const PlanHeader* plan;
  const int* stream_off;
  const int* pair_stream;  // stream holding the first unit of each cluster's run
  float* partial;          // [2G x 128, 512] normalised split partials
  float* partial_lse;      // [2G x 128]
  float* lse_pack;         // head list: [n_q, n_h] lse of whole streams (else null)
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

// Gathered rows i0 + kStride k (k < N; those at or past n are absent) of sequence
// b: physical cache row (y_oob when absent or unlocatable) and request
// position (INT32_MAX likewise).  Every index, segment and block-table load of
// the N rows is issued before any result is used, so a lane pays about one
// dependent-load latency per tile rather than one per row and panel.  The
// planner has already checked that every gathered row of a live stream lies
// in a segment; a bad page id records MLA_ERR_BAD_INDEX and reads as zeros.
// Not inlined: only gathered tiles call it, and the loader loop of page tiles
// stays as compact as it is without it.
template <int N, int kStride>
__device__ __noinline__ void locate_gathered(const DecodeArgs& a, int b, int i0, int n,
                                                long long y_oob, long long* phys, int* kpos) {
  const mla_seg_t* sg = a.segs + (size_t)b * a.max_segs;
  int row[N], seg[N], page[N];
  bool in[N];
#pragma unroll
  for (int k = 0; k < N; ++k) {
    row[k] = i0 + kStride * k < n ? a.gather_rows[(size_t)b * a.max_gather + i0 + kStride * k] : 0;
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
    const bool present = i0 + kStride * k < n;
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

// ----------------------------------------------------------------- unit descriptors
// Everything a role needs about one unit (stream, tile) of a cluster's run,
// computed ahead of time by the producer warp so that no role waits on a chain
// of global loads (stream offsets, segments, block table, query position) in
// its per-tile loop.
constexpr uint32_t kFirst = 1, kLast = 2, kNewQ = 4, kWhole = 8, kSlot1 = 16;
struct Desc {
  int s, k;            // stream, tile within the stream
  int phys0, phys1;    // page mode: physical row of each page's row 0
  int kpos0, kpos1;    // page mode: request position of each page's row 0
  int qp;              // the stream's query position
  uint8_t nv0, nv1;    // page mode: valid rows of each page; gather mode: nv0 = rows in the tile
  uint8_t ver;         // relocation version (selects the query panel)
  uint8_t flags;       // kFirst / kLast: first / last tile of its stream in this run;
                       // kNewQ: needs another query panel; kWhole: the run covers the
                       // whole stream; kSlot1: the partial goes to the run's second slot
};
static_assert(sizeof(Desc) == 32, "descriptor size");
constexpr int kDescRing = 64;            // entries, filled in batches of 32 (one per lane)

// ----------------------------------------------------------------- barriers
struct Bars {
  // score CTA
  uint64_t ring_full[kNStages], ring_empty[kNStages];
  uint64_t qr_full, qr_empty, q_drain;
  uint64_t s_full[2], s_empty[2];
  uint64_t end_empty[2];              // stream-end message slot free (4 remote arrivals)
  uint64_t row_sync[2][4];            // per lane quarter: both halves published the row max
  // both CTAs: P.c of tile t complete (in the score CTA: P buffer t & 1 free)
  uint64_t pv[2];
  // value CTA
  uint64_t v_full[kNV], v_empty[kNV];
  uint64_t p_full[2];                 // P message of tile t landed (8 arrivals + bytes)
  uint64_t o_ok[2];                   // tile t may start its P.c (rescale or epilogue done)
  uint64_t end_full[2];               // stream-end message landed (8 arrivals + bytes)
  // both CTAs: descriptor batches
  uint64_t d_full[2], d_empty[2];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int n_units;                        // units in this cluster's run
};
static_assert(sizeof(Bars) <= kBarBytes, "barrier block too large");

// A phase that never completes: one thread per warp waits on a barrier that
// nothing arrives on, with the given limit, through the decode's own bounded
// wait, then records the timeout the way the decode's roles do.  Nothing is
// in flight, so the block returns cleanly.  1 block of 32 threads.
__global__ void __launch_bounds__(32) wait_probe_kernel(uint64_t limit_ns, int* waited) {
  __shared__ uint64_t never;
  if (threadIdx.x == 0) {
    mbar_init(&never, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer();
    const bool ok = mbar_wait(&never, 0, limit_ns);
    *waited = (int)((globaltimer() - t0) / 1000);   // microseconds
    if (!ok) set_status(MLA_ERR_TIMEOUT);
  }
}

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

// Descriptor ring: unit `it` is entry it % 64.  A consumer waits for the batch
// holding it when it reaches the batch's first entry (batch 0 was waited for
// before the loop) and releases the batch after its last entry.
__device__ __forceinline__ bool desc_wait(Bars* bar, int it, bool warp_wide) {
  if (it == 0 || (it & 31) != 0) return true;
  const int bt = it >> 5;
  return warp_wide ? wait_warp(&bar->d_full[bt & 1], (bt >> 1) & 1)
                   : mbar_wait(&bar->d_full[bt & 1], (bt >> 1) & 1);
}
__device__ __forceinline__ void desc_done(Bars* bar, int it, int n, bool arrive) {
  if (arrive && ((it & 31) == 31 || it == n - 1)) mbar_arrive(&bar->d_empty[(it >> 5) & 1]);
}

// Fill smem rows [r0, r0 + n) (pitch 128 B, n <= 64) of one 64-column panel
// from cache rows starting at y, as power-of-two boxes.  A y at or past the
// end of the cache makes the hardware fill the rows with zeros.
__device__ __forceinline__ void load_rows(uint8_t* dst, const Maps& mp, uint64_t* bar, int x,
                                          long long y, int r0, int n) {
  int r = r0;
  for (; n - (r - r0) > 32; r += 32)     // n <= 64: at most one leading full box
    tma_load_2d(dst + r * 128, &mp.row[0], bar, x, (int)(y + (r - r0)));
  n -= r - r0;
#pragma unroll 1
  for (int hb = 0; hb < kNumBoxHeights; ++hb) {
    const int h = 32 >> hb;
    if (n & h) {
      tma_load_2d(dst + r * 128, &mp.row[hb], bar, x, (int)(y + (r - r0)));
      r += h;
    }
  }
}

// Visibility of 64 tile rows [64 hf, 64 hf + 64) for the unit's query (bit i:
// row 64 hf + i exists and key_pos <= qp).  Page rows have consecutive key
// positions, so each page's mask is a prefix; gathered rows are located one
// per lane and combined by ballot.
template <bool kGather>
__device__ __forceinline__ uint64_t visibility(const DecodeArgs& a, const Desc& d, int b, int hf,
                                               int lane) {
  if constexpr (kGather) {
    long long ph[2];
    int kp[2];
    const int g0 = d.k * kT;
    locate_gathered<2, 32>(a, b, g0 + kPg * hf + lane, g0 + d.nv0, 0, ph, kp);
    const uint32_t lo = __ballot_sync(0xffffffffu, kp[0] <= d.qp);
    const uint32_t hi = __ballot_sync(0xffffffffu, kp[1] <= d.qp);
    return (uint64_t)lo | ((uint64_t)hi << 32);
  } else {
    const int nv = hf ? d.nv1 : d.nv0, kp = hf ? d.kpos1 : d.kpos0;
    const int n = max(0, min(nv, d.qp - kp + 1));
    return n >= 64 ? ~0ull : ((1ull << n) - 1ull);
  }
}

// Rescale this warp's 32 lanes of O (all 512 columns) by f.
__device__ __noinline__ void scale_o(uint32_t taddr, float f) {
#pragma unroll 1
  for (int c = 0; c < kEpiCols; c += 32) {
    float ov[32];
    tmem_ld32_sync(taddr + c, ov);
#pragma unroll
    for (int i = 0; i < 32; ++i) ov[i] *= f;
    tmem_st32(taddr + c, ov);
  }
  tmem_wait_st();
}

// Producer: the descriptors of units u0 + base + lane (lane < cnt), one per
// lane, with the loads of the whole batch in flight together.  `cs` is the
// stream of the batch's first unit; `ps` / `pv` are the stream and version of
// the unit before the batch (-1 for none); all three carry to the next batch.
template <bool kGather>
__device__ __forceinline__ Desc produce(const Params& p, int u0, int u1, int base, int cnt,
                                        int& cs, int& ps, int& pv, int lane) {
  const DecodeArgs& a = p.a;
  const int n_streams = p.plan->n_streams;
  const int u = u0 + base + lane;
  const bool live = lane < cnt;
  // The stream holding u is the last stream whose offset is <= u.  Windows of
  // 32 offsets from cs on (overlapping by one); a lane is resolved once the
  // offset after its candidate is > u.
  int s = -1, off = 0, off_next = 0;
  for (int ws = cs, guard = 0; guard < (1 << 16); ws += 31, ++guard) {
    const int o = ws + lane <= n_streams ? p.stream_off[ws + lane] : INT_MAX;
    int le = 0;
#pragma unroll 8
    for (int j = 0; j < 32; ++j) le += (__shfl_sync(0xffffffffu, o, j) <= u) ? 1 : 0;
    const int jm = max(le - 1, 0);
    const int o_j = __shfl_sync(0xffffffffu, o, jm);
    const int o_n = __shfl_sync(0xffffffffu, o, min(jm + 1, 31));
    if (live && s < 0 && jm < 31 && o_n > u) {
      s = ws + jm;
      off = o_j;
      off_next = o_n;
    }
    if (__all_sync(0xffffffffu, !live || s >= 0)) break;
  }
  Desc d;
  d.s = max(s, 0);
  d.k = u - off;
  const StreamPos sp = stream_pos(p, d.s);
  const int qi = sp.b * a.s_q + sp.j;
  d.qp = live ? a.q_pos[qi] : 0;
  Tile t = {};
  if (live) t = describe<kGather>(a, sp.b, d.k);
  d.phys0 = (int)t.phys0;
  d.phys1 = (int)t.phys1;
  d.kpos0 = t.kpos0;
  d.kpos1 = t.kpos1;
  d.nv0 = (uint8_t)(kGather ? t.n_rows : t.nv0);
  d.nv1 = (uint8_t)t.nv1;
  d.ver = (uint8_t)t.ver;
  const int T = off_next - off;
  uint32_t f = 0;
  if (u == u0 || d.k == 0) f |= kFirst;
  if (u == u1 - 1 || d.k == T - 1) f |= kLast;
  int s_prev = __shfl_up_sync(0xffffffffu, d.s, 1);
  int v_prev = __shfl_up_sync(0xffffffffu, (int)d.ver, 1);
  if (lane == 0) {
    s_prev = ps;
    v_prev = pv;
  }
  if (d.s != s_prev || (int)d.ver != v_prev) f |= kNewQ;
  if (off >= u0 && off + T <= u1) f |= kWhole;
  if (off > u0) f |= kSlot1;
  d.flags = (uint8_t)f;
  // carry to the next batch: the last live unit's stream and version
  const int last = max(cnt - 1, 0);
  cs = __shfl_sync(0xffffffffu, d.s, last);
  ps = cs;
  pv = __shfl_sync(0xffffffffu, (int)d.ver, last);
  return d;
}

// ----------------------------------------------------------------- kernel
template <bool kGather>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ Params p, const __grid_constant__ Maps mp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bar = reinterpret_cast<Bars*>(smem + kOffBar);
  Desc* ring_d = reinterpret_cast<Desc*>(smem + kOffDesc);
  const DecodeArgs& a = p.a;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();   // 0: scores and softmax; 1: P.c and output
  const int g = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNStages; ++i) {
      mbar_init(&bar->ring_full[i], 1);
      mbar_init(&bar->ring_empty[i], 1);
    }
    for (int i = 0; i < kNV; ++i) {
      mbar_init(&bar->v_full[i], 1);
      mbar_init(&bar->v_empty[i], 1);
    }
    mbar_init(&bar->qr_full, 1);
    mbar_init(&bar->qr_empty, 1);
    mbar_init(&bar->q_drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar->s_full[i], 1);
      mbar_init(&bar->s_empty[i], kSoftWarps);
      mbar_init(&bar->end_empty[i], kEpiWarps);
      for (int q = 0; q < 4; ++q) mbar_init(&bar->row_sync[i][q], 2);
      mbar_init(&bar->pv[i], 1);
      mbar_init(&bar->p_full[i], kSoftWarps);
      mbar_init(&bar->o_ok[i], kEpiWarps);
      mbar_init(&bar->end_full[i], kSoftWarps);
      mbar_init(&bar->d_full[i], 1);
      // consumers of each descriptor batch: loader, MMA issuer, and the eight
      // softmax warps (score CTA) or four epilogue warps (value CTA)
      mbar_init(&bar->d_empty[i], rank == 0 ? 2 + kSoftWarps : 2 + kEpiWarps);
    }
    mbar_init(&bar->mma_drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();     // both CTAs' barriers exist before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  // Launched as a programmatic dependent of the planner: everything above
  // overlaps it; its plan and stream offsets are read only after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  bool ok = true;
  const long long y_oob = a.n_pages * kPg;   // first row past the cache: reads as zeros
  const uint32_t peer = mapa(smem_u32(smem), rank ^ 1u);   // the other CTA's shared memory
  // roles with a per-unit loop (the other warps of the value CTA have none)
  const bool consumer = warp < (rank == 0 ? 2 + kSoftWarps : 2 + kEpiWarps);

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ descriptors
    Walk w;
    const bool has_work = walk_begin(p, g, w);
    const int u0 = w.u, u1 = has_work ? w.u1 : w.u;
    const int n = u1 - u0;
    int cs = has_work ? w.s : 0, ps = -1, pv = -1;
    for (int bt = 0; bt == 0 || 32 * bt < n; ++bt) {
      if (!wait_warp(&bar->d_empty[bt & 1], ((bt >> 1) & 1) ^ 1)) { fail(ok); break; }
      const int base = 32 * bt, cnt = min(32, n - base);
      if (cnt > 0) {
        const Desc d = produce<kGather>(p, u0, u1, base, cnt, cs, ps, pv, lane);
        if (lane < cnt) ring_d[(base + lane) % kDescRing] = d;
      }
      if (bt == 0 && lane == 0) bar->n_units = n;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->d_full[bt & 1]);
    }
  } else if (consumer) {
    // the run's length is published with the first batch
    if (!wait_warp(&bar->d_full[0], 0)) fail(ok);
  }
  const int n_units = (ok && consumer) ? bar->n_units : 0;

  if (rank == 0) {
    // ================================================================ score CTA
    uint8_t* ring = smem + kOffRing;
    uint8_t* sQr = smem + kOffQr;
    if (warp == 0) {
      // ------------------------------------------------------------ loads
      if (lane == 0) {
        prefetch_tmap(&mp.q3);
        prefetch_tmap(&mp.qr);
        prefetch_tmap(&mp.k3);
        prefetch_tmap(&mp.kp);
        if (kGather) prefetch_tmap(&mp.g4);
      }
      int nst = 0, nq = 0;
      for (int it = 0; it < n_units && ok; ++it) {
        if (!desc_wait(bar, it, true)) { fail(ok); break; }
        const Desc d = ring_d[it % kDescRing];
        const StreamPos sp = stream_pos(p, d.s);
        if (d.flags & kNewQ) {
          // the head block's absorbed queries: the rotary panel into its own
          // buffer, the 8 latent panels through the ring as three stages
          // (panels 0-2, 3-5, 6-8; the copy to tensor memory skips panel 8)
          const int qrow = (d.ver * a.n_q + sp.b * a.s_q + sp.j) * a.qH + sp.hb * kM;
          if (!wait_warp(&bar->qr_empty, (nq & 1) ^ 1)) { fail(ok); break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(&bar->qr_full, kSlot);
            tma_load_2d(sQr, &mp.qr, &bar->qr_full, kDc, qrow);
          }
          for (int st = 0; st < 3 && ok; ++st, ++nst) {
            const int slot = nst % kNStages;
            if (!wait_warp(&bar->ring_empty[slot], ((nst / kNStages) & 1) ^ 1)) { fail(ok); break; }
            if (lane == 0) {
              mbar_arrive_expect_tx(&bar->ring_full[slot], kStage);
              tma_load_3d(ring + slot * kStage, &mp.q3, &bar->ring_full[slot], 0, qrow, 3 * st);
            }
          }
          if (!ok) break;
          ++nq;
        }
        long long gph[4];
        int gkp[4];
        if constexpr (kGather)
          locate_gathered<4, 1>(a, sp.b, d.k * kT + 4 * lane, d.k * kT + d.nv0, y_oob, gph, gkp);
        // both pages full and next to each other in the pool: one box per stage
        const bool adjacent = !kGather && d.nv0 == kPg && d.nv1 == kPg && d.phys1 == d.phys0 + kPg;
        for (int st = 0; st < 3 && ok; ++st, ++nst) {
          const int slot = nst % kNStages;
          if (!wait_warp(&bar->ring_empty[slot], ((nst / kNStages) & 1) ^ 1)) { fail(ok); break; }
          uint8_t* dst = ring + slot * kStage;
          uint64_t* fb = &bar->ring_full[slot];
          if (lane == 0) mbar_arrive_expect_tx(fb, kStage);
          __syncwarp();
          if constexpr (kGather) {
#pragma unroll
            for (int pn = 0; pn < kStagePanels; ++pn)
              tma_gather4(dst + pn * kSlot + 4 * lane * 128, &mp.g4, fb, 64 * (3 * st + pn),
                          (int)gph[0], (int)gph[1], (int)gph[2], (int)gph[3]);
          } else if (adjacent) {
            if (lane == 0) tma_load_3d(dst, &mp.k3, fb, 0, d.phys0, 3 * st);
          } else if (lane < 2) {
            const int rows = lane ? d.nv1 : d.nv0;
            const long long ph = lane ? d.phys1 : d.phys0;
            for (int pn = 0; pn < kStagePanels; ++pn) {
              uint8_t* hd = dst + pn * kSlot + lane * (kPg * 128);
              const int x = 64 * (3 * st + pn);
              if (rows == kPg) {
                tma_load_2d(hd, &mp.kp, fb, x, (int)ph);
              } else {
                load_rows(hd, mp, fb, x, ph, 0, rows);
                load_rows(hd, mp, fb, x, y_oob, rows, kPg - rows);
              }
            }
          }
          __syncwarp();
        }
        desc_done(bar, it, n_units, lane == 0);
      }
      // drain: every load issued here has landed before the CTA exits
      for (int dd = 1; dd <= kNStages && dd <= nst && ok; ++dd) {
        const int n = nst - dd;
        if (!wait_warp(&bar->ring_full[n % kNStages], (n / kNStages) & 1)) fail(ok);
      }
      if (ok && nq > 0 && !wait_warp(&bar->qr_full, (nq - 1) & 1)) fail(ok);
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA
      if (lane == 0) {
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kM, kT, false, false);
        const uint32_t ring0 = smem_u32(ring), qr0 = smem_u32(sQr);
        int nst = 0, nq = 0;
        for (int it = 0; it < n_units && ok; ++it) {
          if (!desc_wait(bar, it, false)) { fail(ok); break; }
          const uint32_t flags = ring_d[it % kDescRing].flags;
          desc_done(bar, it, n_units, true);
          if (flags & kNewQ) {
            if (nq > 0) {   // the earlier score MMAs are done reading Q and its rotary panel
              mma_commit(&bar->qr_empty);
              mma_commit(&bar->q_drain);
              if (!mbar_wait(&bar->q_drain, (nq - 1) & 1)) { fail(ok); break; }
            }
            if (!mbar_wait(&bar->qr_full, nq & 1)) { fail(ok); break; }
            for (int st = 0; st < 3 && ok; ++st, ++nst) {
              const int slot = nst % kNStages;
              if (!mbar_wait(&bar->ring_full[slot], (nst / kNStages) & 1)) { fail(ok); break; }
              tc_fence_after();
              for (int pn = 0; pn < kStagePanels && 3 * st + pn < 8; ++pn)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                  tmem_cp_128x256b(tmem + kColQ + 32 * (3 * st + pn) + 8 * ks,
                                   smem_desc_sw128(ring0 + slot * kStage + pn * kSlot + ks * 32, 16, 1024));
              mma_commit(&bar->ring_empty[slot]);
            }
            if (!ok) break;
            ++nq;
          }
          const int sb = it & 1;
          if (!mbar_wait(&bar->s_empty[sb], ((it >> 1) & 1) ^ 1)) { fail(ok); break; }
          tc_fence_after();
          const uint32_t dt = tmem + kColS + 128 * sb;
          for (int st = 0; st < 3 && ok; ++st, ++nst) {
            const int slot = nst % kNStages;
            if (!mbar_wait(&bar->ring_full[slot], (nst / kNStages) & 1)) { fail(ok); break; }
            tc_fence_after();
#pragma unroll
            for (int pn = 0; pn < kStagePanels; ++pn) {
              const int panel = 3 * st + pn;
              const uint32_t kb = ring0 + slot * kStage + pn * kSlot;
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint64_t bd = smem_desc_sw128(kb + ks * 32, 16, 1024);
                if (panel < 8)
                  mma_bf16_ts(dt, tmem + kColQ + 32 * panel + 8 * ks, bd, idesc_qk, (panel | ks) ? 1u : 0u);
                else
                  mma_bf16_ss(dt, smem_desc_sw128(qr0 + ks * 32, 16, 1024), bd, idesc_qk, 1u);
              }
            }
            mma_commit(&bar->ring_empty[slot]);
          }
          if (!ok) break;
          mma_commit(&bar->s_full[sb]);
        }
        if (ok && nq > 0) mma_commit(&bar->qr_empty);
        mma_commit(&bar->mma_drain);
        if (!mbar_wait(&bar->mma_drain, 0)) fail(ok);
      }
    } else if (warp < kProducerWarp) {
      // ------------------------------------------------------------ softmax
      // Two warps per TMEM lane quarter: warp 2 + 4 hf owns columns
      // [64 hf, 64 hf + 64) of the tile (page hf) for the quarter's 32 rows.
      const int quad = warp & 3;
      const int hf = (warp - 2) >> 2;
      const int h = quad * 32 + lane;            // head row of the block = TMEM lane
      const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16) + kColS + 64 * hf;
      float* sMax = reinterpret_cast<float*>(smem + kOffMax);   // [buffer][half][row]
      const uint32_t mbase = peer + kOffMsg, ebase = peer + kOffEnd;
      int n_str = 0;
      float m_run = -INFINITY, l_run = 0.f;      // l_run: this half's share of the row sum
      // P, the rescale factors and the flags travel as asynchronous remote
      // stores (st.async) whose bytes complete a transaction count on the value
      // CTA's barrier: the warp never waits for them.  Each warp announces its
      // share of the bytes with one remote arrival.
      const uint32_t p_bytes = 32 * 8 * 16 + (hf == 0 ? 4 * 32 : 0) + 4;
      const uint32_t e_bytes = 4 * 32 + (hf == 0 ? 4 * 32 : 0);
      for (int it = 0; it < n_units && ok; ++it) {
        if (!desc_wait(bar, it, true)) { fail(ok); break; }
        const Desc d = ring_d[it % kDescRing];
        const StreamPos sp = stream_pos(p, d.s);
        const bool valid = sp.hb * kM + h < a.n_h;
        if (d.flags & kFirst) {
          m_run = -INFINITY;
          l_run = 0.f;
        }
        const uint64_t vis = visibility<kGather>(a, d, sp.b, hf, lane);
        const uint32_t v0 = (uint32_t)vis, v1 = (uint32_t)(vis >> 32);
        const int sb = it & 1, pb = it & 1;
        // QK-normed scores: one factor per column, the key's inverse RMS,
        // read for this half's page before the wait so the loads overlap it
        float kf[64];
        if (!kGather && a.key_inv) {
          const float4* src = reinterpret_cast<const float4*>(a.key_inv + (hf ? d.phys1 : d.phys0));
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float4 f = __ldg(src + j);
            kf[4 * j] = f.x;
            kf[4 * j + 1] = f.y;
            kf[4 * j + 2] = f.z;
            kf[4 * j + 3] = f.w;
          }
        }
        if (!wait_warp(&bar->s_full[sb], (it >> 1) & 1)) { fail(ok); break; }
        tc_fence_after();
        float x[64];
        tmem_ld64_sync(trow + 128 * sb, *reinterpret_cast<float(*)[2][32]>(x));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->s_empty[sb]);
        if (!kGather && a.key_inv) {
#pragma unroll
          for (int c = 0; c < 64; ++c) x[c] *= kf[c];
        }

        // max of this half's visible scores (four independent chains), then
        // of the row, through the partner warp (log2 units)
        // (branch-free: a select per element keeps every element's work in one
        // basic block, so the scheduler can overlap their latencies)
        // (a half whose 64 rows are all visible takes the loops without the
        // mask selects: the common case, and fewer instructions beside the
        // single-thread load and MMA issuers that share these schedulers)
        const bool all_vis = (v0 & v1) == 0xffffffffu;
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (all_vis) {
#pragma unroll
          for (int c = 0; c < 64; ++c) mx[c & 3] = fmaxf(mx[c & 3], x[c]);
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const bool vb = ((c < 32 ? v0 : v1) >> (c & 31)) & 1u;
            mx[c & 3] = fmaxf(mx[c & 3], vb ? x[c] : -INFINITY);
          }
        }
        const float mh = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
        sMax[(sb * 2 + hf) * kM + h] = mh;       // scale > 0: max commutes, -inf stays
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->row_sync[sb][quad]);
        if (!wait_warp(&bar->row_sync[sb][quad], (it >> 1) & 1)) { fail(ok); break; }
        const float mt = fmaxf(mh, sMax[(sb * 2 + (hf ^ 1)) * kM + h]);
        // lazy rescaling: keep the reference max unless it grows by > 2^8
        const bool need = mt > m_run + kRescaleThreshold;
        const float m_new = need ? mt : m_run;
        const float factor = need ? exp2f(m_run - m_new) : 1.f;   // exp2(-inf) = 0
        const bool any = valid && (m_new != -INFINITY);

        // P = 2^(scale*S - m_new) on visible rows, bf16, into P panel hf of the
        // value CTA's message buffer (128-byte swizzled K-major rows) once the
        // value CTA is done with the tile that last used it
        if (!wait_warp_cluster(&bar->pv[pb], ((it >> 1) & 1) ^ 1)) { fail(ok); break; }
        const uint32_t msg = mbase + pb * kMsgStride;
        const uint32_t prow = msg + hf * (kM * 128) + h * 128;
        const uint32_t fbar = mapa(smem_u32(&bar->p_full[pb]), 1);
        if (lane == 0) mbar_arrive_expect_tx_cluster(fbar, p_bytes);
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
        auto p_pass = [&](auto masked) {
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              const int c0 = c + i, c1 = c + i + 1;
              // every element's exponential is taken; the mask only selects
              float p0 = ex2_approx(fmaf(x[c0], p.scale_log2, -m_new));
              float p1 = ex2_approx(fmaf(x[c1], p.scale_log2, -m_new));
              if constexpr (decltype(masked)::value) {
                const bool b0 = any && (((c0 < 32 ? v0 : v1) >> (c0 & 31)) & 1u);
                const bool b1 = any && (((c1 < 32 ? v0 : v1) >> (c1 & 31)) & 1u);
                p0 = b0 ? p0 : 0.f;
                p1 = b1 ? p1 : 0.f;
              }
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
              ls[(i >> 1) & 3] += __low2float(h2) + __high2float(h2);
              pk[i >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            st_async_v4(prow + ((((c >> 3)) ^ (h & 7)) << 4), make_uint4(pk[0], pk[1], pk[2], pk[3]),
                        fbar);
          }
        };
        if (all_vis && any) p_pass(std::false_type{});
        else p_pass(std::true_type{});
        l_run = l_run * factor + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
        m_run = m_new;
        if (hf == 0) st_async_b32(msg + kPBuf + 4 * h, __float_as_uint(valid ? factor : 1.f), fbar);
        // O needs a rescale before this tile's P.c when a live row's reference
        // max moved (never on a stream's first tile: that P.c overwrites O)
        const bool wf = __any_sync(0xffffffffu, valid && need && !(d.flags & kFirst));
        if (lane == 0) st_async_b32(msg + kPBuf + kHdrFlag + 4 * (warp - 2), wf ? 1u : 0u, fbar);
        if (d.flags & kLast) {
          // stream end: each half's row sums and the row max for the epilogue
          const int es = n_str & 1;
          if (!wait_warp_cluster(&bar->end_empty[es], ((n_str >> 1) & 1) ^ 1)) { fail(ok); break; }
          const uint32_t e = ebase + es * kEndBytes;
          const uint32_t ebar = mapa(smem_u32(&bar->end_full[es]), 1);
          if (lane == 0) mbar_arrive_expect_tx_cluster(ebar, e_bytes);
          st_async_b32(e + hf * (4 * kM) + 4 * h, __float_as_uint(l_run), ebar);
          if (hf == 0) st_async_b32(e + 8 * kM + 4 * h, __float_as_uint(m_run), ebar);
          ++n_str;
        }
        desc_done(bar, it, n_units, lane == 0);
      }
    }
  } else {
    // ================================================================ value CTA
    uint8_t* vbuf = smem + kOffVal;     // kNV slots: 8 latent panels of kVRows rows
    uint8_t* msg = smem + kOffMsg;      // two P messages: P, then factors and the flags
    const float* endm = reinterpret_cast<const float*>(smem + kOffEnd);
    if (warp == 0) {
      // ------------------------------------------------------------ loads
      if (lane == 0) {
        prefetch_tmap(&mp.vp);
        if (kGather) prefetch_tmap(&mp.g4);
      }
      int nv = 0;
      for (int it = 0; it < n_units && ok; ++it) {
        if (!desc_wait(bar, it, true)) { fail(ok); break; }
        const Desc d = ring_d[it % kDescRing];
        const int b = stream_pos(p, d.s).b;
        for (int hq = 0; hq < kVPerTile && ok; ++hq, ++nv) {
          const int slot = nv % kNV;
          if (!wait_warp(&bar->v_empty[slot], ((nv / kNV) & 1) ^ 1)) { fail(ok); break; }
          uint8_t* dst = vbuf + slot * kVSlot;
          uint64_t* fb = &bar->v_full[slot];
          if (lane == 0) mbar_arrive_expect_tx(fb, kVSlot);
          __syncwarp();
          if constexpr (kGather) {
            // kVRows / 4 four-row groups x 8 latent panels, spread over the lanes
            constexpr int kQuads = kVRows / 4, kPer = kQuads * 8 / 32;
            long long gph[4];
            int gkp[4];
            const int r4 = 4 * (lane % kQuads);
            locate_gathered<4, 1>(a, b, d.k * kT + kVRows * hq + r4, d.k * kT + d.nv0, y_oob, gph,
                                  gkp);
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
              const int q = lane / kQuads + (32 / kQuads) * k;
              tma_gather4(dst + q * (kVRows * 128) + r4 * 128, &mp.g4, fb, 64 * q, (int)gph[0],
                          (int)gph[1], (int)gph[2], (int)gph[3]);
            }
          } else if (lane == 0) {
            // rows [ro, ro + kVRows) of page hp of the tile
            const int hp = hq * kVRows / kPg, ro = hq * kVRows % kPg;
            const int rows = max(0, min(kVRows, (hp ? d.nv1 : d.nv0) - ro));
            const long long ph = (hp ? d.phys1 : d.phys0) + ro;
            if (rows == kVRows) {
              tma_load_3d(dst, &mp.vp, fb, 0, (int)ph, 0);
            } else {
              for (int q = 0; q < 8; ++q) {
                load_rows(dst + q * (kVRows * 128), mp, fb, 64 * q, ph, 0, rows);
                load_rows(dst + q * (kVRows * 128), mp, fb, 64 * q, y_oob, rows, kVRows - rows);
              }
            }
          }
          __syncwarp();
        }
        desc_done(bar, it, n_units, lane == 0);
      }
      for (int dd = 1; dd <= kNV && dd <= nv && ok; ++dd) {
        const int n = nv - dd;
        if (!wait_warp(&bar->v_full[n % kNV], (n / kNV) & 1)) fail(ok);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA
      if (lane == 0) {
        constexpr uint32_t idesc_pv = idesc_bf16_f32(kM, 256, false, true);
        const uint32_t v0 = smem_u32(vbuf), p0 = smem_u32(msg);
        int nv = 0;
        for (int it = 0; it < n_units && ok; ++it) {
          if (!desc_wait(bar, it, false)) { fail(ok); break; }
          const bool first = ring_d[it % kDescRing].flags & kFirst;
          desc_done(bar, it, n_units, true);
          const int pb = it & 1;
          if (!mbar_wait_cluster(&bar->p_full[pb], (it >> 1) & 1) ||
              !mbar_wait(&bar->o_ok[pb], (it >> 1) & 1)) { fail(ok); break; }
          // P arrived as generic-proxy stores: order them before the tensor
          // core's (async-proxy) reads of the buffer
          fence_proxy_async();
          tc_fence_after();
          const uint32_t pa = p0 + pb * kMsgStride;
          for (int hq = 0; hq < kVPerTile && ok; ++hq, ++nv) {
            const int slot = nv % kNV;
            if (!mbar_wait(&bar->v_full[slot], (nv / kNV) & 1)) { fail(ok); break; }
            tc_fence_after();
            const uint32_t vb = v0 + slot * kVSlot;
#pragma unroll
            for (int ks = 0; ks < kVRows / 16; ++ks) {
              // tokens [t, t + 16) of the tile: P panel t / 64, 16-token step
              // (t % 64) / 16 within it
              const int t = hq * kVRows + 16 * ks;
              const uint64_t ad =
                  smem_desc_sw128(pa + (t / kPg) * (kM * 128) + ((t % kPg) / 16) * 32, 16, 1024);
#pragma unroll
              for (int nb = 0; nb < 2; ++nb) {
                const uint64_t bd =
                    smem_desc_sw128(vb + nb * 4 * (kVRows * 128) + ks * 2048, kVRows * 128, 1024);
                mma_bf16_ss(tmem + 256 * nb, ad, bd, idesc_pv, (first && t == 0) ? 0u : 1u);
              }
            }
            mma_commit(&bar->v_empty[slot]);
          }
          if (!ok) break;
          mma_commit_mask(&bar->pv[pb], 0x3);    // this CTA's epilogue and the score CTA's P buffer
        }
        mma_commit(&bar->mma_drain);
        if (!mbar_wait(&bar->mma_drain, 0)) fail(ok);
      }
    } else if (warp < 2 + kEpiWarps) {
      // ------------------------------------------------------------ rescale and epilogue
      // warps 2-5 take columns [0, kEpiCols) of O (with eight warps, warps
      // 6-9 the rest); a warp's lane quarter (its rows) is warp & 3
      const int quad = warp & 3;
      const int ch = (warp - 2) >> 2;
      const int h = quad * 32 + lane;
      const int col0 = ch * kEpiCols;
      const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16) + col0;
      float4* stage = reinterpret_cast<float4*>(smem + kOffStage + (warp - 2) * kStageWarp);
      int n_str = 0;
      for (int it = 0; it < n_units && ok; ++it) {
        if (!desc_wait(bar, it, true)) { fail(ok); break; }
        const Desc d = ring_d[it % kDescRing];
        desc_done(bar, it, n_units, lane == 0);
        const int pb = it & 1;
        if (!(d.flags & kFirst)) {
          if (!wait_warp_cluster(&bar->p_full[pb], (it >> 1) & 1)) { fail(ok); break; }
          const uint8_t* hdr = msg + pb * kMsgStride + kPBuf;
          const volatile uint32_t* wfl = reinterpret_cast<const volatile uint32_t*>(hdr + kHdrFlag);
          uint32_t flag = 0;
#pragma unroll
          for (int i = 0; i < kSoftWarps; ++i) flag |= wfl[i];
          if (flag) {
            // O must hold every earlier tile's P.c before it is rescaled
            if (!wait_warp(&bar->pv[(it - 1) & 1], ((it - 1) >> 1) & 1)) { fail(ok); break; }
            tc_fence_after();
            const float f = reinterpret_cast<const float*>(hdr)[h];
            scale_o(trow, f);
            tc_fence_before();
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->o_ok[pb]);
        if (d.flags & kLast) {
          // the stream's O is complete once this tile's P.c is done
          const int es = n_str & 1;
          if (!wait_warp(&bar->pv[pb], (it >> 1) & 1) ||
              !wait_warp_cluster(&bar->end_full[es], (n_str >> 1) & 1)) { fail(ok); break; }
          tc_fence_after();
          const float l_tot = endm[es * (kEndBytes / 4) + h] + endm[es * (kEndBytes / 4) + kM + h];
          const float m_fin = endm[es * (kEndBytes / 4) + 2 * kM + h];
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_addr(mapa(smem_u32(&bar->end_empty[es]), 0));
          const StreamPos sp = stream_pos(p, d.s);
          const int qi = sp.b * a.s_q + sp.j;
          const bool whole = d.flags & kWhole;
          const int slot = 2 * g + ((d.flags & kSlot1) ? 1 : 0);
          const bool empty = !(l_tot > 0.f);
          const float inv = empty ? 0.f : 1.f / l_tot;
          const float lse = empty ? -INFINITY : (m_fin + log2f(l_tot)) * 0.6931471805599453f;
          // O leaves through a per-warp staging tile (32 rows x 32 floats,
          // 128-byte swizzled as the store map expects) by TMA tensor stores:
          // a whole stream's rows to its heads (the map clips heads past n_h),
          // a split's rows to the pair's partial slot.
          const int hrow0 = sp.hb * kM + quad * 32;
          // a lane quarter whose 32 head rows all lie past n_h has nothing
          // live to write (heads of a partly filled block, e.g. 8 Global
          // heads): neither its rows of o_lat nor its partial rows are read
          const int n_store = hrow0 < a.n_h ? kEpiCols : 0;
          // 64 columns per tensor-memory round trip (two loads, one wait):
          // the epilogue pays a load's latency, not its size
#pragma unroll 1
          for (int c0 = 0; c0 < n_store; c0 += 2 * kStoreCols) {
            float ov[2][32];
            tmem_ld64_sync(trow + c0, ov);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int c = c0 + k * kStoreCols;
              if (c > 0) {
                if (lane == 0) bulk_wait_read<0>();   // the staging tile is free again
                __syncwarp();
              }
#pragma unroll
              for (int j = 0; j < 8; ++j)
                stage[lane * 8 + (j ^ (lane & 7))] =
                    make_float4(ov[k][4 * j] * inv, ov[k][4 * j + 1] * inv,
                                ov[k][4 * j + 2] * inv, ov[k][4 * j + 3] * inv);
              fence_proxy_async();
              __syncwarp();
              if (lane == 0) {
                if (whole) tma_store_3d(&mp.o, stage, col0 + c, hrow0, qi);
                else tma_store_2d(&mp.part, stage, col0 + c, slot * kM + quad * 32);
                bulk_commit();
              }
            }
          }
          if (lane == 0) bulk_wait_all();   // the stores are complete before the merge reads them
          __syncwarp();
          tc_fence_before();
          if (ch == 0) {
            const int hr = sp.hb * kM + h;
            if (!whole) p.partial_lse[(size_t)slot * kM + h] = lse;
            else if (hr < a.n_h) {
              if (p.lse_pack) p.lse_pack[(size_t)qi * a.n_h + hr] = lse;
              else a.lse[(size_t)qi * a.H + hr] = lse;
            }
          }
          ++n_str;
        }
      }
    }
  }

  asm volatile("griddepcontrol.launch_dependents;");   // the merge may be scheduled
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no CTA leaves while its peer may still write its shared memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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
                                                      const float* partial_lse,
                                                      const float* o_pack,
                                                      const float* lse_pack) {
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
  const int head = head_of(a, hb * kM + m);
  if (head < 0) return;
  const size_t orow = (size_t)qi * a.H + head;
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
  if (g0 == g1) {
    // one pair covered the stream and wrote it: to o_lat directly, or (head
    // list) packed by list position, moved here to the listed head's row
    if (lse_pack) {
      const size_t prow = (size_t)qi * a.n_h + hb * kM + m;
      const float4* src = reinterpret_cast<const float4*>(o_pack + prow * kDc);
      float4* dst = reinterpret_cast<float4*>(o);
#pragma unroll
      for (int i = 0; i < kDc / 128; ++i) dst[lane + 32 * i] = src[lane + 32 * i];
      if (lane == 0) a.lse[orow] = lse_pack[prow];
    }
    return;
  }
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
