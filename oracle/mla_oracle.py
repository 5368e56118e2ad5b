"""Plain fp64 CPU oracle for absorbed Multi-head Latent Attention decode.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
link this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  It shares no code with the CUDA path.

Everything here is written from the method's definitions, in float64, with
library primitives (matmul, exp, log, sin, cos) as single steps and no
blocking, fusion or reordering beyond what the definitions state:

* Day 27 tutorial "Multi-Head Latent Attention: How DeepSeek Compressed the
  Cache Further" (kgptalkie):
    - "Learn a Smaller Shared Representation": one latent ``c_t`` per token;
    - "The Direct Form Explains the Meaning": per-head content key
      ``k^C_t = U_K c_t``, scored by a dot product with the query;
    - "Move the Key Projection Into the Query": ``q . (U_K c) = (U_K^T q) . c``;
    - "Move the Value Expansion After the Weighted Sum":
      ``sum_t a_t U_V c_t = U_V sum_t a_t c_t``, and the value up-projection
      may combine with the output projection;
    - "Position Rotations Complicate the Absorption": score = content term +
      rotary term, then scaled, masked and softmaxed;
    - "Count the Cache That Is Actually Stored": L*T*B*(d_c + d_r)*b bytes.
* "RedKnot-MLA: Multi-Head Offline-Online Reuse for DeepSeek-V4 Long-Context
  Serving", abstract: documents cached at canonical position zero,
  query-side RoPE relocation to the request position, Local heads from an
  offline (MLA-Off) partial plus protected rows recomputed online, Global
  heads online, merged before one shared output projection.

"QK-Normed MLA" abstract: post-projection QK RMSNorm made compatible with
the latent path (``decode_qknorm``; the explicit form and the absorbed form
with one cached inverse-RMS scalar per token).

QuantMLA abstract: a low-bit latent cache (symmetric per-channel codes,
packed; ``dequantize_pool`` gives the cache the low-bit attention reads).

Upstream of the decode, ``cache_rows`` and ``append_rows`` state how new
tokens enter the paged cache (the latent as is, the rotary key rotated at its
cache position, each logical row in its block-table page and slot).

Readings where the pages are silent (each one is listed with its reason in
the design notes): softmax scale 1/sqrt(d_n + d_r); RoPE on adjacent pairs
(2i, 2i+1) with angle pos * base^(-2i/d_r); cached rotary keys stored already
rotated at their cache position; visibility ``key_pos <= q_pos``; natural-log
LSE over scaled scores; an empty visible set gives o = 0 and lse = -inf.
Parity of those readings is unpinned by the pages: they are declared here and
held fixed, not derived.
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# Cache accounting -- tutorial, "Count the Cache That Is Actually Stored"
# ---------------------------------------------------------------------------

def cache_bytes(L: int, T: int, B: int, d_c: int, d_r: int, b: int) -> int:
    """Bytes of a uniform-layer MLA cache: one shared latent (no factor of 2
    around d_c, since it serves both keys and values) plus one rotary key."""
    return L * T * B * (d_c + d_r) * b


def mha_cache_bytes(L: int, T: int, B: int, heads: int, d_k: int, d_v: int, b: int) -> int:
    """Ordinary multi-head attention cache: a key and a value per head
    (tutorial, "Start With What Ordinary Attention Saves")."""
    return L * T * B * heads * (d_k + d_v) * b


def head_row_ceiling(local_heads: int, global_heads: int, reusable_layers: int,
                     total_layers: int) -> float:
    """RedKnot-MLA abstract, analytic logical head-row ceiling: the share of
    (layer, head) rows that can come from the offline path -- the Local
    heads' share of the heads times the reusable layers' share of the layers."""
    return local_heads / (local_heads + global_heads) * reusable_layers / total_layers


# ---------------------------------------------------------------------------
# Content path -- tutorial, "The Direct Form" and "Move the Key Projection"
# ---------------------------------------------------------------------------

def content_keys(u_k: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Direct form: expand every latent row into a content key, k^C_t = U_K c_t.

    u_k: [d_n, d_c] (one head's key up-projection); c: [T, d_c] -> [T, d_n].
    """
    return np.asarray(c, np.float64) @ np.asarray(u_k, np.float64).T


def values(u_v: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Direct form: expand every latent row into a value, v_t = U_V c_t."""
    return np.asarray(c, np.float64) @ np.asarray(u_v, np.float64).T


def absorb_query(u_k: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Projection absorption: transform the query once, U_K^T q.

    u_k: [d_n, d_c]; q: [..., d_n] -> [..., d_c].
    """
    return np.asarray(q, np.float64) @ np.asarray(u_k, np.float64)


def weighted_latent(a: np.ndarray, c: np.ndarray) -> np.ndarray:
    """sum_t a_t c_t: mix the narrow latents before any expansion."""
    return np.asarray(a, np.float64) @ np.asarray(c, np.float64)


# ---------------------------------------------------------------------------
# Rotary path -- tutorial, "Position Rotations Complicate the Absorption";
# RedKnot-MLA abstract, query-side RoPE relocation
# ---------------------------------------------------------------------------

def rope_inv_freq(d_r: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/d_r) for the d_r/2 feature pairs."""
    i = np.arange(d_r // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d_r)


def rope_rotate(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate each adjacent feature pair (2i, 2i+1) by the angle pos*theta_i.

    x: [..., d_r]; pos broadcasts against x[..., 0].  Angles are fp64.
    """
    x = np.asarray(x, np.float64)
    ang = np.asarray(pos, np.float64)[..., None] * rope_inv_freq(x.shape[-1], base)
    cos, sin = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (x.shape[-1],)), np.float64)
    out[..., 0::2] = x0 * cos - x1 * sin
    out[..., 1::2] = x0 * sin + x1 * cos
    return out


# ---------------------------------------------------------------------------
# Softmax and log-sum-exp
# ---------------------------------------------------------------------------

def softmax_lse(s: np.ndarray):
    """Row softmax and natural-log LSE of scaled, masked scores (-inf = masked).

    Returns (weights, lse).  A row with every entry masked gets weights 0 and
    lse = -inf.
    """
    s = np.asarray(s, np.float64)
    m = np.max(s, axis=-1, keepdims=True) if s.shape[-1] else np.full(s.shape[:-1] + (1,), NEG_INF)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(s - m_safe)
    tot = np.sum(e, axis=-1, keepdims=True)
    with np.errstate(divide="ignore"):
        lse = np.where(empty, NEG_INF, m_safe + np.log(np.where(empty, 1.0, tot)))
    a = np.where(empty, 0.0, e / np.where(empty, 1.0, tot))
    return a, lse[..., 0]


def merge_lse(o_a, lse_a, o_b, lse_b):
    """Merge two partial attentions over disjoint key sets.

    (o_x, lse_x) is a normalised output and the LSE of its key set; the
    result is the attention over the union (RedKnot-MLA abstract: the offline
    and online paths are merged before the shared output projection).
    o_*: [..., d]; lse_*: [...].
    """
    lse_a = np.asarray(lse_a, np.float64)
    lse_b = np.asarray(lse_b, np.float64)
    lse = np.logaddexp(lse_a, lse_b)
    empty = ~np.isfinite(lse)
    ref = np.where(empty, 0.0, lse)
    w_a = np.where(empty, 0.0, np.exp(lse_a - ref))
    w_b = np.where(empty, 0.0, np.exp(lse_b - ref))
    o = w_a[..., None] * np.asarray(o_a, np.float64) + w_b[..., None] * np.asarray(o_b, np.float64)
    return o, lse


# ---------------------------------------------------------------------------
# Paged cache bookkeeping (row -> page, slot; segment -> key position)
# ---------------------------------------------------------------------------

def sequence_rows(segs_b: np.ndarray, gather_b=None):
    """Logical rows of one sequence with their key positions and query versions.

    segs_b: [n_seg, 4] of (row_begin, row_end, q_version, key_pos_base).
    Row r of segment s sits at request position key_pos_base + (r - row_begin)
    and was cached with its rotary key at that position minus the relocation
    offset of version q_version.  With ``gather_b`` the row set is that list.
    Returns (rows, key_pos, version) as int64 arrays.
    """
    rows, kpos, ver = [], [], []
    if gather_b is None:
        for rb, re, v, kb in segs_b:
            for r in range(int(rb), int(re)):
                rows.append(r)
                kpos.append(int(kb) + r - int(rb))
                ver.append(int(v))
    else:
        for r in gather_b:
            r = int(r)
            hit = [s for s in segs_b if int(s[0]) <= r < int(s[1])]
            if len(hit) != 1:
                raise ValueError(f"gathered row {r} is in {len(hit)} segments")
            rb, re, v, kb = (int(x) for x in hit[0])
            rows.append(r)
            kpos.append(kb + r - rb)
            ver.append(v)
    return (np.array(rows, np.int64), np.array(kpos, np.int64), np.array(ver, np.int64))


def gather_cache(pool: np.ndarray, block_table_b: np.ndarray, rows: np.ndarray,
                 page: int = 64) -> np.ndarray:
    """Cached rows [T, d_c + d_r] of one sequence, read through its block table."""
    pages = np.asarray(block_table_b)[rows // page]
    return np.asarray(pool[pages, rows % page], np.float64)


# ---------------------------------------------------------------------------
# Cache writer (upstream of the decode) -- tutorial, "Position Rotations
# Complicate the Absorption" (the decoupled rotary key is stored beside the
# latent); RedKnot-MLA abstract (a document is cached at canonical position
# zero and relocated on the query side)
# ---------------------------------------------------------------------------

def cache_rows(c, k_rope_raw, cache_pos, base: float) -> np.ndarray:
    """Rows as the cache stores them, [T, d_c + d_r]: the latent c_t as it is
    and the rotary key rotated at its cache position.

    A row's cache position is its request position minus the relocation
    offset it will be served with: a prefix row is cached at its request
    position, a document cached on its own at 0, 1, 2, ...
    """
    c = np.asarray(c, np.float64)
    k = rope_rotate(k_rope_raw, np.asarray(cache_pos, np.float64), base)
    return np.concatenate([c, k], axis=-1)


def append_rows(pool: np.ndarray, block_table_b: np.ndarray, row0: int, rows: np.ndarray,
                page: int = 64) -> np.ndarray:
    """Store ``rows`` as logical rows row0, row0 + 1, ... of one sequence.

    Logical row r lives in page block_table_b[r // page] at slot r % page.
    Returns a new fp64 pool; every slot not written keeps its old contents.
    """
    out = np.array(pool, dtype=np.float64, copy=True)
    bt = np.asarray(block_table_b)
    for i, row in enumerate(np.asarray(rows, np.float64)):
        r = int(row0) + i
        out[int(bt[r // page]), r % page] = row
    return out


# ---------------------------------------------------------------------------
# Attention for one sequence, one head
# ---------------------------------------------------------------------------

def attend_direct(q_nope, q_rope, q_pos, u_k, u_v, c, k_rope, key_pos, key_shift,
                  scale, base):
    """Direct (expanded-key) form for one head of one sequence.

    q_nope [S, d_n], q_rope [S, d_r], q_pos [S]; c [T, d_c]; k_rope [T, d_r]
    as cached (rotated at key_pos - key_shift); key_pos, key_shift [T].
    The cached rotary key is first restored to its request position by
    rotating it forward by key_shift (the key-side repair that query-side
    relocation avoids); the query is rotated at its own position.
    Returns (o_lat [S, d_c], o [S, d_v], lse [S]).
    """
    k_content = content_keys(u_k, c)                        # [T, d_n]
    v_full = values(u_v, c)                                 # [T, d_v]
    k_r = rope_rotate(k_rope, key_shift, base)              # [T, d_r]
    q_r = rope_rotate(q_rope, q_pos, base)                  # [S, d_r]
    s = scale * (np.asarray(q_nope, np.float64) @ k_content.T + q_r @ k_r.T)
    visible = np.asarray(key_pos)[None, :] <= np.asarray(q_pos)[:, None]
    s = np.where(visible, s, NEG_INF)
    a, lse = softmax_lse(s)
    return weighted_latent(a, c), a @ v_full, lse


def attend_absorbed(q_lat, q_r_by_row, c, k_rope, key_pos, q_pos, scale):
    """Absorbed form for one head of one sequence.

    q_lat [S, d_c] = U_K^T q_nope; q_r_by_row [S, T, d_r] is, for each key
    row, the query's rotary part rotated at q_pos - (that row's relocation
    offset).  Scores are taken directly against the cached c and k_rope.
    Returns (o_lat [S, d_c], lse [S]).
    """
    c = np.asarray(c, np.float64)
    s = scale * (np.asarray(q_lat, np.float64) @ c.T
                 + np.einsum("std,td->st", q_r_by_row, np.asarray(k_rope, np.float64)))
    visible = np.asarray(key_pos)[None, :] <= np.asarray(q_pos)[:, None]
    s = np.where(visible, s, NEG_INF)
    a, lse = softmax_lse(s)
    return weighted_latent(a, c), lse


# ---------------------------------------------------------------------------
# Whole decode over the paged cache
# ---------------------------------------------------------------------------

def decode(inp, heads=None, rows_override=None, form="direct", seqs=None):
    """Attention outputs for every (query token, head) of a decode step.

    ``inp`` is a workloads.DecodeInputs (plain arrays).  ``heads`` selects
    logical head ids (default all).  ``rows_override`` maps a sequence index
    to an explicit list of logical rows (a key subset, e.g. protected rows or
    the offline complement); otherwise the sequence's gather list, else all
    its segment rows.  ``seqs`` restricts the sequences computed.
    Returns o_lat [n_q, n_h, d_c], lse [n_q, n_h] (and o [n_q, n_h, d_v] for
    the direct form), NaN where a sequence was skipped.
    """
    wl = inp.wl
    heads = list(range(wl.H)) if heads is None else list(heads)
    n_h = len(heads)
    n_q = inp.n_q
    o_lat = np.full((n_q, n_h, wl.d_c), np.nan)
    lse = np.full((n_q, n_h), np.nan)
    o_val = np.full((n_q, n_h, wl.d_v), np.nan)
    seqs = range(wl.B) if seqs is None else seqs
    for b in seqs:
        if rows_override is not None and b in rows_override:
            rows, kpos, ver = sequence_rows(inp.segs[b], rows_override[b])
        elif inp.gather_rows is not None:
            g = inp.gather_rows[b, :int(inp.n_gather[b])]
            rows, kpos, ver = sequence_rows(inp.segs[b], g)
        else:
            rows, kpos, ver = sequence_rows(inp.segs[b])
        cache = gather_cache(inp.pool, inp.block_table[b], rows)
        c, k_rope = cache[:, :wl.d_c], cache[:, wl.d_c:]
        shift = np.asarray(inp.deltas, np.int64)[ver]
        qs = slice(b * wl.s_q, (b + 1) * wl.s_q)
        q_pos = np.asarray(inp.q_pos[qs], np.int64)
        for i, h in enumerate(heads):
            if form == "direct":
                ol, ov, ls = attend_direct(inp.q_nope[qs, h], inp.q_rope[qs, h], q_pos,
                                           inp.w_uk[h], inp.w_uv[h], c, k_rope, kpos,
                                           shift, wl.scale, wl.rope_base)
                o_val[qs, i] = ov
            else:
                q_lat = absorb_query(inp.w_uk[h], inp.q_nope[qs, h])
                rel = q_pos[:, None] - shift[None, :]              # [S, T]
                q_r = rope_rotate(np.asarray(inp.q_rope[qs, h], np.float64)[:, None, :],
                                  rel, wl.rope_base)               # [S, T, d_r]
                ol, ls = attend_absorbed(q_lat, q_r, c, k_rope, kpos, q_pos, wl.scale)
            o_lat[qs, i] = ol
            lse[qs, i] = ls
    if form == "direct":
        return o_lat, lse, o_val
    return o_lat, lse


def decode_absorbed_fast(inp, heads=None, seqs=None, rows_override=None):
    """Absorbed form, vectorised over heads (same definition as ``decode``
    with form="absorbed", grouped by relocation version so the rotary query
    is formed once per version rather than once per key row).  Used where the
    per-row form is too slow (long contexts) and as the timed CPU baseline.
    ``rows_override`` maps a sequence to an explicit row list, as in ``decode``.
    Returns o_lat [n_q, n_h, d_c], lse [n_q, n_h].
    """
    wl = inp.wl
    heads = np.arange(wl.H) if heads is None else np.asarray(list(heads))
    n_q = inp.n_q
    o_lat = np.full((n_q, len(heads), wl.d_c), np.nan)
    lse = np.full((n_q, len(heads)), np.nan)
    seqs = range(wl.B) if seqs is None else seqs
    w_uk = np.asarray(inp.w_uk[heads], np.float64)                    # [n_h, d_n, d_c]
    for b in seqs:
        if rows_override is not None and b in rows_override:
            rows, kpos, ver = sequence_rows(inp.segs[b], rows_override[b])
        elif inp.gather_rows is not None:
            rows, kpos, ver = sequence_rows(inp.segs[b], inp.gather_rows[b, :int(inp.n_gather[b])])
        else:
            rows, kpos, ver = sequence_rows(inp.segs[b])
        cache = gather_cache(inp.pool, inp.block_table[b], rows)
        c, k_rope = cache[:, :wl.d_c], cache[:, wl.d_c:]
        for j in range(wl.s_q):
            qi = b * wl.s_q + j
            p = int(inp.q_pos[qi])
            qn = np.asarray(inp.q_nope[qi, heads], np.float64)            # [n_h, d_n]
            q_lat = np.einsum("hn,hnc->hc", qn, w_uk)                    # U_K^T q per head
            s = q_lat @ c.T                                              # content term
            for v in np.unique(ver):
                sel = ver == v
                q_r = rope_rotate(np.asarray(inp.q_rope[qi, heads], np.float64),
                                  p - int(inp.deltas[v]), wl.rope_base)    # [n_h, d_r]
                s[:, sel] += q_r @ k_rope[sel].T                         # rotary term
            s = np.where((kpos <= p)[None, :], wl.scale * s, NEG_INF)
            a, ls = softmax_lse(s)
            o_lat[qi] = a @ c
            lse[qi] = ls
    return o_lat, lse


# ---------------------------------------------------------------------------
# QK-normed MLA -- "QK-Normed MLA" abstract: post-projection RMSNorm of the
# queries and keys; the static key-side weight folds into the absorbed query
# and the dynamic key statistic is one inverse-RMS scalar per token and KV
# group, so the latent decode path survives
# ---------------------------------------------------------------------------

QK_NORM_EPS = 1e-6


def rms_norm(x, weight, eps: float = QK_NORM_EPS) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * weight over the last axis."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(weight, np.float64)


def key_inv_rms(c, w_uk, eps: float = QK_NORM_EPS) -> np.ndarray:
    """The dynamic key statistic, one per token: 1 / rms of the token's content
    keys of every head of the group, concatenated (H * d_n values).

    c [T, d_c]; w_uk [H, d_n, d_c] -> [T].  Computable when the row is
    written, from the latent alone.
    """
    k = np.einsum("hnc,tc->thn", np.asarray(w_uk, np.float64), np.asarray(c, np.float64))
    k = k.reshape(k.shape[0], -1)
    return 1.0 / np.sqrt(np.mean(k * k, axis=-1) + eps)


def qknorm_scores_direct(q_nope, q_rope, q_pos, w_uk, c, k_rope, key_shift, g_q, g_k,
                         scale, base, eps: float = QK_NORM_EPS) -> np.ndarray:
    """Scaled scores [H, T] of one query token with explicit post-projection
    QK RMSNorm: the content query of all heads (H * d_n values) and each
    token's content keys of all heads are normalised with weights g_q, g_k;
    the rotary path is left as it is.  Keys are expanded (U_K c_t) and the
    cached rotary keys restored to their request positions, as in
    ``attend_direct``.  q_nope [H, d_n]; q_rope [H, d_r]; w_uk [H, d_n, d_c];
    c [T, d_c]; k_rope [T, d_r]; key_shift [T]; g_q, g_k [H * d_n].
    """
    H, d_n = np.asarray(q_nope).shape
    q_hat = rms_norm(np.asarray(q_nope, np.float64).reshape(-1), g_q, eps).reshape(H, d_n)
    k = np.einsum("hnc,tc->thn", np.asarray(w_uk, np.float64), np.asarray(c, np.float64))
    k_hat = rms_norm(k.reshape(k.shape[0], -1), g_k, eps).reshape(k.shape)
    k_r = rope_rotate(k_rope, key_shift, base)
    q_r = rope_rotate(q_rope, q_pos, base)
    return scale * (np.einsum("hn,thn->ht", q_hat, k_hat) + q_r @ k_r.T)


def qknorm_scores_absorbed(q_nope, q_rope, q_pos, w_uk, c, k_rope, key_shift, g_q, g_k,
                           scale, base, eps: float = QK_NORM_EPS) -> np.ndarray:
    """The same scores [H, T] through the latent path: the query is normalised
    and multiplied by the key weight, then absorbed, U_K^T (g_k * q_hat); the
    content score against the cached latent is multiplied by the token's
    inverse key RMS; the rotary query is relocated per row as in
    ``attend_absorbed``.
    """
    H, d_n = np.asarray(q_nope).shape
    q_hat = rms_norm(np.asarray(q_nope, np.float64).reshape(-1), g_q, eps).reshape(H, d_n)
    q_w = q_hat * np.asarray(g_k, np.float64).reshape(H, d_n)
    q_lat = np.einsum("hn,hnc->hc", q_w, np.asarray(w_uk, np.float64))      # [H, d_c]
    c = np.asarray(c, np.float64)
    content = (q_lat @ c.T) * key_inv_rms(c, w_uk, eps)[None, :]
    rel = np.asarray(q_pos, np.float64) - np.asarray(key_shift, np.float64)    # [T]
    q_r = rope_rotate(np.asarray(q_rope, np.float64)[:, None, :], rel[None, :], base)  # [H, T, d_r]
    rotary = np.einsum("htd,td->ht", q_r, np.asarray(k_rope, np.float64))
    return scale * (content + rotary)


def decode_qknorm(inp, g_q, g_k, form: str = "absorbed", eps: float = QK_NORM_EPS, seqs=None):
    """QK-normed attention of every query token over its sequence (all heads
    form one KV group).  Masking, softmax and the weighted latent are those of
    the plain decode.  Returns o_lat [n_q, H, d_c], lse [n_q, H]."""
    wl = inp.wl
    scores = qknorm_scores_absorbed if form == "absorbed" else qknorm_scores_direct
    o_lat = np.full((inp.n_q, wl.H, wl.d_c), np.nan)
    lse = np.full((inp.n_q, wl.H), np.nan)
    for b in (range(wl.B) if seqs is None else seqs):
        rows, kpos, ver = sequence_rows(inp.segs[b])
        cache = gather_cache(inp.pool, inp.block_table[b], rows)
        c, k_rope = cache[:, :wl.d_c], cache[:, wl.d_c:]
        shift = np.asarray(inp.deltas, np.int64)[ver]
        for j in range(wl.s_q):
            qi = b * wl.s_q + j
            p = int(inp.q_pos[qi])
            s = scores(inp.q_nope[qi], inp.q_rope[qi], p, inp.w_uk, c, k_rope, shift,
                       g_q, g_k, wl.scale, wl.rope_base, eps)
            s = np.where((kpos <= p)[None, :], s, NEG_INF)
            a, ls = softmax_lse(s)
            o_lat[qi] = a @ c
            lse[qi] = ls
    return o_lat, lse


# ---------------------------------------------------------------------------
# Low-bit latent cache -- QuantMLA abstract: the content and rotary caches
# stored as low-bit integers (INT4 and INT4, or INT2 content with an INT4
# rotary key), unpacked and dequantised inside the attention.  The learned,
# offline-fused transforms of the abstract are not modelled: the scales are
# inputs.
# ---------------------------------------------------------------------------

def quantize_symmetric(x, scale, bits: int) -> np.ndarray:
    """Signed codes round(x / scale), ties to even, clamped to
    [-2^(bits-1), 2^(bits-1) - 1]; ``scale`` broadcasts over the last axis
    (one static scale per channel).  Returns int64 codes."""
    lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    q = np.round(np.asarray(x, np.float64) / np.asarray(scale, np.float64))
    return np.clip(q, lo, hi).astype(np.int64)


def dequantize(codes, scale) -> np.ndarray:
    """The value a code stands for: code * its channel's scale."""
    return np.asarray(codes, np.float64) * np.asarray(scale, np.float64)


def pack_codes(codes, bits: int) -> np.ndarray:
    """Pack signed codes along the last axis into bytes, 8 / bits codes per
    byte, the first code in the lowest bits, each as a bits-wide two's
    complement field."""
    codes = np.asarray(codes, np.int64)
    per = 8 // bits
    n = codes.shape[-1]
    assert n % per == 0
    fields = (codes & ((1 << bits) - 1)).reshape(codes.shape[:-1] + (n // per, per))
    out = np.zeros(fields.shape[:-1], np.int64)
    for k in range(per):
        out |= fields[..., k] << (bits * k)
    return out.astype(np.uint8)


def unpack_codes(packed, bits: int) -> np.ndarray:
    """Inverse of ``pack_codes``: signed codes, 8 / bits per byte."""
    b = np.asarray(packed, np.int64)
    per = 8 // bits
    mask, sign = (1 << bits) - 1, 1 << (bits - 1)
    fields = np.stack([(b >> (bits * k)) & mask for k in range(per)], axis=-1)
    codes = np.where(fields >= sign, fields - (1 << bits), fields)
    return codes.reshape(b.shape[:-1] + (b.shape[-1] * per,))


def quantized_row_bytes(d_c: int, d_r: int, bits_c: int, bits_r: int) -> int:
    """Bytes of one packed cache row (content codes, then rotary codes)."""
    return (d_c * bits_c + d_r * bits_r) // 8


def dequantize_pool(pool, d_c: int, scale_c, scale_r, bits_c: int, bits_r: int) -> np.ndarray:
    """The cache the low-bit attention reads: every stored row quantised with
    its per-channel scales (content and rotary separately) and dequantised.
    NaN rows (never referenced) stay NaN."""
    pool = np.asarray(pool, np.float64)
    out = np.array(pool, copy=True)
    used = ~np.isnan(pool).any(axis=-1)
    rows = pool[used]
    out[used, :d_c] = dequantize(quantize_symmetric(rows[:, :d_c], scale_c, bits_c), scale_c)
    out[used, d_c:] = dequantize(quantize_symmetric(rows[:, d_c:], scale_r, bits_r), scale_r)
    return out


def out_proj(o_lat, w_uv, w_o):
    """Value up-projection per head, then the shared output projection.

    o_lat [n_q, H, d_c]; w_uv [H, d_v, d_c]; w_o [d_model, H*d_v].
    Returns v [n_q, H, d_v] and out [n_q, d_model] (tutorial, "Move the Value
    Expansion After the Weighted Sum": expand the one mixed latent, then the
    head's contribution joins the final output projection).
    """
    o_lat = np.asarray(o_lat, np.float64)
    v = np.einsum("hdc,qhc->qhd", np.asarray(w_uv, np.float64), o_lat)
    out = v.reshape(v.shape[0], -1) @ np.asarray(w_o, np.float64).T
    return v, out


def fold_value_into_output(w_uv, w_o) -> np.ndarray:
    """Each head's value up-projection folded into its slice of the output
    projection (tutorial, "Move the Value Expansion After the Weighted Sum"):
    W_fold[:, h*d_c:(h+1)*d_c] = W_O[:, h*d_v:(h+1)*d_v] W_UV[h].
    w_uv [H, d_v, d_c]; w_o [d_model, H*d_v] -> [d_model, H*d_c]."""
    w_uv = np.asarray(w_uv, np.float64)
    w_o = np.asarray(w_o, np.float64)
    H, d_v, _ = w_uv.shape
    return np.concatenate([w_o[:, h * d_v:(h + 1) * d_v] @ w_uv[h] for h in range(H)], axis=1)


def out_proj_folded(o_lat, w_fold) -> np.ndarray:
    """out = W_fold concat_h(o_lat_h): one product from the weighted latents."""
    o_lat = np.asarray(o_lat, np.float64)
    return o_lat.reshape(o_lat.shape[0], -1) @ np.asarray(w_fold, np.float64).T

