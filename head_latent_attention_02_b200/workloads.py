"""Seeded synthetic inputs for absorbed MLA decode over a paged latent cache.

This module only draws and lays out inputs; it holds none of the method's
arithmetic (no absorption, no RoPE, no softmax).  The oracle and the CUDA
path both consume what it returns, so it is the single source of inputs for
parity tests, the smoke check and the benchmark.

Recipe (shared by every workload):
  * each tensor has its own stream ``numpy.random.default_rng([seed, k])``
    with a fixed index ``k`` per tensor;
  * latents ``c_KV``, cached rotary keys ``k_rope``, ``q_nope`` and ``q_rope``
    are N(0, 1); weights are N(0, 1/fan_in);
  * values are drawn in fp32 and, for bf16 workloads, rounded to the nearest
    bf16 (ties to even), so host arrays hold exactly what the GPU stores;
  * the cached ``k_rope`` rows are drawn directly: an isotropic Gaussian key
    rotated by any angle is again an isotropic Gaussian, so the stored row has
    the distribution of a raw key rotated at its cache position;
  * rows past a sequence's end in its last page, and every page no block
    table references, are filled with NaN; unused block-table slots point at
    a dedicated all-NaN page, so a stray read shows up as NaN, never as an
    out-of-bounds access.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

PAGE = 64

# tensor stream indices (fixed so that every workload draws the same way)
_K_QNOPE, _K_QROPE, _K_WUK, _K_WUV, _K_WO, _K_CACHE, _K_LENS, _K_PERM, _K_PROT = range(9)


@dataclasses.dataclass
class Workload:
    """One decode configuration (sizes, dtype and structure)."""
    name: str
    dtype: str               # "f32" or "bf16": storage type of q, cache and weights
    B: int                   # sequences
    H: int                   # query heads
    d_c: int = 512           # content latent width
    d_r: int = 64            # decoupled rotary key width
    d_n: int = 128           # per-head no-position query/key width
    d_v: int = 128           # per-head value width
    d_model: int = 7168      # output width of the shared output projection
    s_q: int = 1             # query tokens per sequence (the last s_q cached rows)
    lengths: Optional[list] = None   # cached rows per sequence
    len_range: Optional[tuple] = None  # (lo, hi) inclusive uniform lengths
    scattered: bool = False  # block-table page ids drawn as a seeded permutation
    rope_base: float = 10000.0
    # offline/online (RedKnot-style) structure
    prefix: int = 0          # rows of request prefix (relocation offset 0)
    doc: int = 0             # rows of a document cached at canonical position 0
    n_local: int = 0         # Local heads (first n_local heads after permutation)
    protected: int = 0       # protected document rows recomputed online
    protected_mode: str = "sample"   # "sample" (seeded) or "first"
    head_perm: bool = False  # Local/Global assignment by a seeded permutation

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(d_n + d_r): the width of the expanded query/key."""
        return 1.0 / math.sqrt(self.d_n + self.d_r)

    @property
    def row(self) -> int:
        return self.d_c + self.d_r


WORKLOADS = {
    # parity config: every size small, fp32 end to end
    "tiny_f32": Workload("tiny_f32", "f32", B=1, H=8, d_c=32, d_r=16, d_n=16,
                         d_v=16, d_model=128, lengths=[256]),
    # the headline decode workload: B=16, 128 heads, 4K context
    "bf16_b16_4k": Workload("bf16_b16_4k", "bf16", B=16, H=128, lengths=[4096] * 16),
    "bf16_varlen_b64": Workload("bf16_varlen_b64", "bf16", B=64, H=64,
                                len_range=(1024, 32768), scattered=True),
    "redknot_56_8": Workload("redknot_56_8", "bf16", B=1, H=64, prefix=8192,
                             doc=16384, n_local=56, protected=256),
    "bf16_long_256k": Workload("bf16_long_256k", "bf16", B=2, H=128, s_q=2,
                               lengths=[262144, 262144]),
}


def query_positions(wl: Workload, rows: int) -> list:
    """Request positions of a sequence's query tokens given its cached rows.

    With s_q == 1 the query is the new token right after the cache (the tiny
    config caches positions 0..255 and queries at 256).  With s_q > 1 the
    query tokens are the last s_q cached rows (positions rows-s_q .. rows-1),
    so the causal rule key_pos <= q_pos masks the later ones from the earlier.
    """
    if wl.s_q == 1:
        return [rows]
    return [rows - wl.s_q + j for j in range(wl.s_q)]


def _rng(seed: int, k: int) -> np.random.Generator:
    return np.random.default_rng([seed, k])


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    nan = np.isnan(x)
    out = r.view(np.float32).copy()
    out[nan] = np.nan
    return out


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of fp32 values that are already bf16-exact."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u >> 16).astype(np.uint16)


def _normal(rng, shape, std, dtype):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return round_bf16(x) if dtype == "bf16" else x


@dataclasses.dataclass
class DecodeInputs:
    """Host arrays for one workload (fp32 values; bf16-exact for bf16)."""
    wl: Workload
    q_nope: np.ndarray        # [B*s_q, H, d_n]
    q_rope: np.ndarray        # [B*s_q, H, d_r]
    q_pos: np.ndarray         # [B*s_q] int32 request positions
    deltas: np.ndarray        # [n_ver] int32 relocation offsets
    w_uk: np.ndarray          # [H, d_n, d_c]  W_UK[h] maps c to a content key
    w_uv: np.ndarray          # [H, d_v, d_c]  W_UV[h] maps c to a value
    w_o: np.ndarray           # [d_model, H*d_v]
    pool: np.ndarray          # [n_pages, PAGE, d_c + d_r]
    block_table: np.ndarray   # [B, max_pages] int32
    segs: np.ndarray          # [B, max_segs, 4] int32 (row_begin, row_end, q_version, key_pos_base)
    n_rows: np.ndarray        # [B] logical rows per sequence (end of its last segment)
    gather_rows: Optional[np.ndarray] = None  # [B, max_gather] int32
    n_gather: Optional[np.ndarray] = None     # [B] int32
    head_order: Optional[np.ndarray] = None   # head ids, Local heads first (RedKnot)
    nan_page: int = -1

    @property
    def n_q(self) -> int:
        return self.q_pos.shape[0]


def _lengths(wl: Workload, seed: int) -> list:
    if wl.lengths is not None:
        return list(wl.lengths)
    if wl.len_range is not None:
        lo, hi = wl.len_range
        return [int(v) for v in _rng(seed, _K_LENS).integers(lo, hi + 1, size=wl.B)]
    if wl.prefix or wl.doc:
        return [wl.prefix + wl.doc] * wl.B
    raise ValueError("workload has no lengths")


def make_weights(wl: Workload, seed: int = 0):
    """W_UK [H,d_n,d_c], W_UV [H,d_v,d_c] ~ N(0,1/d_c); W_O [d_model,H*d_v] ~ N(0,1/(H*d_v))."""
    w_uk = _normal(_rng(seed, _K_WUK), (wl.H, wl.d_n, wl.d_c), 1.0 / math.sqrt(wl.d_c), wl.dtype)
    w_uv = _normal(_rng(seed, _K_WUV), (wl.H, wl.d_v, wl.d_c), 1.0 / math.sqrt(wl.d_c), wl.dtype)
    w_o = _normal(_rng(seed, _K_WO), (wl.d_model, wl.H * wl.d_v),
                  1.0 / math.sqrt(wl.H * wl.d_v), wl.dtype)
    return w_uk, w_uv, w_o


def make_inputs(wl: Workload, seed: int = 0, lengths: Optional[list] = None,
                poison: bool = True, with_weights: bool = True,
                draw_cache: bool = True) -> DecodeInputs:
    """Draw every input of one decode step for ``wl``.

    ``lengths`` overrides the per-sequence lengths (used by parity tests to
    build ragged variants of a workload at sizes the oracle finishes fast).
    ``draw_cache=False`` leaves the pool's values undrawn (an uninitialised
    array of the right shape) for callers that fill the cache on the device
    and compare nothing against the oracle (throughput runs).
    """
    L = list(lengths) if lengths is not None else _lengths(wl, seed)
    assert len(L) == wl.B
    rows = [int(l) for l in L]
    n_q = wl.B * wl.s_q
    q_nope = _normal(_rng(seed, _K_QNOPE), (n_q, wl.H, wl.d_n), 1.0, wl.dtype)
    q_rope = _normal(_rng(seed, _K_QROPE), (n_q, wl.H, wl.d_r), 1.0, wl.dtype)
    q_pos = np.empty(n_q, np.int32)
    for b in range(wl.B):
        q_pos[b * wl.s_q:(b + 1) * wl.s_q] = query_positions(wl, rows[b])

    pages_per_seq = [(r + PAGE - 1) // PAGE for r in rows]
    total_pages = sum(pages_per_seq)
    n_pages = total_pages + 1            # + one all-NaN page
    nan_page = total_pages
    max_pages = max(pages_per_seq) if pages_per_seq else 1
    if wl.scattered:
        ids = _rng(seed, _K_PERM).permutation(total_pages).astype(np.int32)
    else:
        ids = np.arange(total_pages, dtype=np.int32)
    block_table = np.full((wl.B, max(max_pages, 1)), nan_page, np.int32)
    off = 0
    for b in range(wl.B):
        block_table[b, :pages_per_seq[b]] = ids[off:off + pages_per_seq[b]]
        off += pages_per_seq[b]

    # one contiguous draw for all used rows, in (sequence, row) order
    if draw_cache:
        n_used = sum(rows)
        rng = _rng(seed, _K_CACHE)
        lat = _normal(rng, (n_used, wl.row), 1.0, wl.dtype)
        pool = np.full((n_pages, PAGE, wl.row), np.nan if poison else 0.0, np.float32)
        off = 0
        for b in range(wl.B):
            for p in range(pages_per_seq[b]):
                take = min(PAGE, rows[b] - p * PAGE)
                pool[block_table[b, p], :take] = lat[off:off + take]
                off += take
        del lat
    else:
        pool = np.empty((n_pages, PAGE, wl.row), np.float32)

    # segments: one per sequence, or prefix + document for the RedKnot layout
    if wl.doc:
        assert wl.prefix % PAGE == 0, "a cached document starts on a page boundary"
        segs = np.zeros((wl.B, 2, 4), np.int32)
        for b in range(wl.B):
            segs[b, 0] = (0, wl.prefix, 0, 0)
            segs[b, 1] = (wl.prefix, wl.prefix + wl.doc, 1, wl.prefix)
        deltas = np.array([0, wl.prefix], np.int32)
    else:
        segs = np.zeros((wl.B, 1, 4), np.int32)
        for b in range(wl.B):
            segs[b, 0] = (0, rows[b], 0, 0)
        deltas = np.array([0], np.int32)

    gather_rows = n_gather = None
    if wl.protected:
        g = np.zeros((wl.B, wl.protected), np.int32)
        for b in range(wl.B):
            if wl.protected_mode == "first":
                pr = np.arange(wl.protected)
            else:
                pr = np.sort(_rng(seed, _K_PROT).choice(wl.doc, size=wl.protected, replace=False))
            g[b] = wl.prefix + pr
        gather_rows = g
        n_gather = np.full(wl.B, wl.protected, np.int32)

    head_order = None
    if wl.head_perm:
        head_order = _rng(seed, _K_PERM + 100).permutation(wl.H).astype(np.int32)

    if with_weights:
        w_uk, w_uv, w_o = make_weights(wl, seed)
    else:
        w_uk = w_uv = w_o = None
    return DecodeInputs(wl, q_nope, q_rope, q_pos, deltas, w_uk, w_uv, w_o, pool,
                        block_table, segs, np.array(rows, np.int32), gather_rows,
                        n_gather, head_order, nan_page)
