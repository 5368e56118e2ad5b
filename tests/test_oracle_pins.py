"""Pins of the fp64 oracle to facts fixed outside the oracle itself.

Each test ties a part of the oracle to a value the pages print, a closed
form, an invariant, or a special case that reduces to a library routine
(torch's scaled_dot_product_attention, Python's complex exponential), so
that a dropped term, a wrong sign or index, or a transposed operand fails.
CPU only.
"""
import cmath
import itertools
import copy
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import mla_oracle as O
from head_latent_attention_02_b200.workloads import Workload, make_inputs

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


# --------------------------------------------------------------- worked examples

def test_worked_absorption_example():
    g = GOLD["absorption"]
    u_k, c, q = np.array(g["u_k"]), np.array(g["c"]), np.array(g["q"])
    k = O.content_keys(u_k, c[None, :])[0]
    assert np.array_equal(k, g["content_key"])
    assert float(q @ k) == g["direct_score"]
    qa = O.absorb_query(u_k, q)
    assert np.array_equal(qa, g["absorbed_query"])
    assert float(qa @ c) == g["absorbed_score"]


def test_worked_value_example():
    g = GOLD["value"]
    c, a, u_v = np.array(g["c"]), np.array(g["weights"]), np.array(g["u_v"])
    lat = O.weighted_latent(a, c)
    assert np.allclose(lat, g["weighted_latent"], rtol=0, atol=1e-15)
    out = O.values(u_v, lat[None, :])[0]
    assert np.allclose(out, g["value_out"], rtol=0, atol=1e-15)
    # linearity: expanding each latent then mixing gives the same output
    per_row = O.values(u_v, c)
    assert np.allclose(a @ per_row, g["value_out"], rtol=0, atol=1e-15)


def test_cache_count_example():
    g = GOLD["cache_count"]
    assert O.cache_bytes(1, 1, 1, g["d_c"], g["d_r"], g["bytes_per_number"]) == g["mla_bytes_per_layer_token"]
    assert O.mha_cache_bytes(1, 1, 1, g["mha_heads"], g["mha_key"], g["mha_value"],
                             g["bytes_per_number"]) == g["mha_bytes_per_layer_token"]
    assert O.mha_cache_bytes(1, 1, 1, 2, 4, 4, 1) == g["mha_numbers_per_layer_token"]
    # the headline layout: 576 bf16 numbers = 1152 bytes per layer-token
    assert O.cache_bytes(1, 1, 1, 512, 64, 2) == 1152


# --------------------------------------------------------------------- RoPE

def _rope_complex(x, pos, base):
    """Pairs (2i, 2i+1) as complex numbers times exp(i*pos*theta_i)."""
    d = len(x)
    out = []
    for i in range(d // 2):
        th = base ** (-2.0 * i / d)
        z = complex(x[2 * i], x[2 * i + 1]) * cmath.exp(1j * pos * th)
        out += [z.real, z.imag]
    return np.array(out)


@pytest.mark.parametrize("pos", [0, 1, 7, 4095, 24575, 262143])
def test_rope_matches_complex_rotation(pos):
    rng = np.random.default_rng(pos)
    x = rng.standard_normal(64)
    got = O.rope_rotate(x, pos, 10000.0)
    ref = _rope_complex(x, pos, 10000.0)
    assert np.allclose(got, ref, rtol=0, atol=1e-9)
    assert math.isclose(np.linalg.norm(got), np.linalg.norm(x), rel_tol=1e-12)


def test_rope_position_zero_is_identity_and_composes():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 16))
    assert np.array_equal(O.rope_rotate(x, 0, 10000.0), x)
    a, b = 1234, 56789
    two = O.rope_rotate(O.rope_rotate(x, a, 10000.0), b, 10000.0)
    assert np.allclose(two, O.rope_rotate(x, a + b, 10000.0), rtol=0, atol=1e-9)


def _tiny(B=2, H=3, d_c=8, d_r=4, d_n=5, d_v=6, s_q=1, lengths=(13, 70), **kw):
    wl = Workload("t", "f32", B=B, H=H, d_c=d_c, d_r=d_r, d_n=d_n, d_v=d_v,
                  d_model=H * d_v, s_q=s_q, lengths=None if lengths is None else list(lengths), **kw)
    return make_inputs(wl, seed=3)


def _shift_positions(inp, delta_pos):
    """Every request position (queries and keys) moves by delta_pos; the cache
    rows, rotated at their cache positions, move with them."""
    out = copy.deepcopy(inp)
    wl = inp.wl
    out.q_pos = inp.q_pos + delta_pos
    out.segs = inp.segs.copy()
    out.segs[:, :, 3] += delta_pos
    used = ~np.isnan(inp.pool[:, :, 0])
    kr = inp.pool[:, :, wl.d_c:].astype(np.float64)
    rot = O.rope_rotate(kr, delta_pos, wl.rope_base)
    out.pool = inp.pool.astype(np.float64)
    out.pool[:, :, wl.d_c:] = np.where(used[..., None], rot, np.nan)
    return out


@pytest.mark.parametrize("dpos", [5, 1000, 250000])
def test_rope_relative_position_invariance(dpos):
    inp = _tiny()
    o1, l1, v1 = O.decode(inp)
    o2, l2, v2 = O.decode(_shift_positions(inp, dpos))
    assert np.allclose(o1, o2, rtol=0, atol=1e-9)
    assert np.allclose(l1, l2, rtol=0, atol=1e-9)


def test_relocation_offset_invariance():
    """A document whose rotary keys were cached at canonical positions gives the
    same result as the same document cached at its request positions with no
    relocation (query-side repair equals key-side repair)."""
    wl = Workload("t", "f32", B=1, H=2, d_c=8, d_r=4, d_n=5, d_v=6, d_model=12,
                  prefix=64, doc=128)
    inp = make_inputs(wl, seed=5)
    o_rel, l_rel, _ = O.decode(inp)
    flat = copy.deepcopy(inp)
    # rotate the document rows forward by the offset and drop the relocation
    doc_pages = inp.block_table[0, 1:3]
    flat.pool = inp.pool.astype(np.float64)
    flat.pool[doc_pages, :, wl.d_c:] = O.rope_rotate(inp.pool[doc_pages, :, wl.d_c:], 64, wl.rope_base)
    flat.deltas = np.array([0, 0], np.int32)
    o_flat, l_flat, _ = O.decode(flat)
    assert np.allclose(o_rel, o_flat, rtol=0, atol=1e-10)
    assert np.allclose(l_rel, l_flat, rtol=0, atol=1e-10)


# ------------------------------------------------ special case: library attention

def test_matches_torch_sdpa_with_expanded_keys():
    """With keys and values expanded explicitly and the rotation done by complex
    multiplication, the oracle equals torch's scaled_dot_product_attention."""
    inp = _tiny(s_q=2, lengths=(13, 70))
    wl = inp.wl
    o_lat, lse, o_val = O.decode(inp)
    for b in range(wl.B):
        rows = int(inp.n_rows[b])
        r = np.arange(rows)
        cache = inp.pool[inp.block_table[b, r // 64], r % 64].astype(np.float64)
        c, kr = cache[:, :wl.d_c], cache[:, wl.d_c:]
        qs = slice(b * wl.s_q, (b + 1) * wl.s_q)
        qp = inp.q_pos[qs]
        mask = torch.tensor(r[None, :] <= qp[:, None])
        for h in range(wl.H):
            k = np.concatenate([c @ inp.w_uk[h].astype(np.float64).T,
                                np.stack([_rope_complex(kr[t], 0, wl.rope_base) for t in r])], 1)
            q = np.concatenate([inp.q_nope[qs, h].astype(np.float64),
                                np.stack([_rope_complex(inp.q_rope[qs][j, h], qp[j], wl.rope_base)
                                          for j in range(wl.s_q)])], 1)
            v = c @ inp.w_uv[h].astype(np.float64).T
            T = torch.from_numpy
            ref = torch.nn.functional.scaled_dot_product_attention(
                T(q)[None], T(k)[None], T(v)[None], attn_mask=mask[None], scale=wl.scale)[0]
            ref_lat = torch.nn.functional.scaled_dot_product_attention(
                T(q)[None], T(k)[None], T(c)[None], attn_mask=mask[None], scale=wl.scale)[0]
            assert np.allclose(o_val[qs, h], ref.numpy(), rtol=0, atol=1e-12)
            assert np.allclose(o_lat[qs, h], ref_lat.numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------- softmax closed forms

def test_softmax_rows_sum_to_one_and_lse_closed_form():
    rng = np.random.default_rng(0)
    s = rng.standard_normal((4, 37)) * 5
    a, lse = O.softmax_lse(s)
    assert np.allclose(a.sum(-1), 1.0, rtol=0, atol=1e-14)
    same = np.full((2, 9), 0.7)
    a2, l2 = O.softmax_lse(same)
    assert np.allclose(a2, 1 / 9, rtol=0, atol=1e-15)
    assert np.allclose(l2, 0.7 + math.log(9), rtol=0, atol=1e-14)
    a3, l3 = O.softmax_lse(np.full((1, 3), -np.inf))
    assert np.all(a3 == 0) and np.all(l3 == -np.inf)


def test_single_row_returns_its_latent():
    inp = _tiny(lengths=(1, 1))
    o_lat, lse, _ = O.decode(inp)
    for b in range(2):
        c = inp.pool[inp.block_table[b, 0], 0, :inp.wl.d_c]
        assert np.array_equal(o_lat[b, :, :], np.broadcast_to(c, o_lat[b].shape))


def test_zero_query_gives_mean_of_visible_rows():
    inp = _tiny(s_q=2, lengths=(13, 70))
    inp.q_nope[:] = 0
    inp.q_rope[:] = 0
    o_lat, lse, _ = O.decode(inp)
    wl = inp.wl
    for b in range(wl.B):
        rows = int(inp.n_rows[b])
        for j in range(wl.s_q):
            qi = b * wl.s_q + j
            vis = np.arange(int(inp.q_pos[qi]) + 1)      # key_pos <= q_pos
            vis = vis[vis < rows]
            c = inp.pool[inp.block_table[b, vis // 64], vis % 64, :wl.d_c].astype(np.float64)
            assert np.allclose(o_lat[qi], c.mean(0), rtol=0, atol=1e-13)
            assert np.allclose(lse[qi], math.log(len(vis)), rtol=0, atol=1e-13)
    # the last query of a sequence sees one more row than the one before it
    assert int(inp.q_pos[1]) == int(inp.n_rows[0]) - 1


# -------------------------------------------------------------- merge and forms

def test_merge_of_any_split_equals_unsplit():
    inp = _tiny(lengths=(13, 70))
    full_lat, full_lse, _ = O.decode(inp)
    rng = np.random.default_rng(7)
    for b in range(2):
        rows = np.arange(int(inp.n_rows[b]))
        mask = rng.random(len(rows)) < 0.4
        mask[0], mask[-1] = True, False
        a_lat, a_lse, _ = O.decode(inp, rows_override={b: rows[mask]}, seqs=[b])
        b_lat, b_lse, _ = O.decode(inp, rows_override={b: rows[~mask]}, seqs=[b])
        m_lat, m_lse = O.merge_lse(a_lat[b], a_lse[b], b_lat[b], b_lse[b])
        assert np.allclose(m_lat, full_lat[b], rtol=0, atol=1e-12)
        assert np.allclose(m_lse, full_lse[b], rtol=0, atol=1e-12)


def test_merge_with_empty_is_identity():
    rng = np.random.default_rng(2)
    o, l = rng.standard_normal((3, 5)), rng.standard_normal(3)
    ninf = np.full(3, -np.inf)
    m, ml = O.merge_lse(o, l, np.zeros((3, 5)), ninf)
    assert np.array_equal(ml, l) and np.allclose(m, o, rtol=0, atol=0)
    m2, ml2 = O.merge_lse(np.zeros((3, 5)), ninf, np.zeros((3, 5)), ninf)
    assert np.all(ml2 == -np.inf) and np.all(m2 == 0)


@pytest.mark.parametrize("kw", [dict(), dict(s_q=2, lengths=(64, 129)),
                                dict(prefix=64, doc=128, B=1, lengths=None)])
def test_absorbed_equals_direct(kw):
    inp = _tiny(**kw)
    d_lat, d_lse, _ = O.decode(inp)
    a_lat, a_lse = O.decode(inp, form="absorbed")
    f_lat, f_lse = O.decode_absorbed_fast(inp)
    for lat, lse in ((a_lat, a_lse), (f_lat, f_lse)):
        assert np.allclose(lat, d_lat, rtol=1e-10, atol=1e-12)
        assert np.allclose(lse, d_lse, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- bookkeeping

def test_page_placement_and_poison_do_not_matter():
    a = _tiny(lengths=(13, 200))
    b = copy.deepcopy(a)
    perm = np.random.default_rng(9).permutation(a.pool.shape[0])
    inv = np.argsort(perm)
    b.pool = a.pool[perm]                       # page p moves to slot inv[p]
    b.block_table = inv[a.block_table].astype(np.int32)
    oa, la, _ = O.decode(a)
    ob, lb, _ = O.decode(b)
    assert np.isfinite(oa).all() and np.array_equal(oa, ob) and np.array_equal(la, lb)


def test_out_proj_fold_identity():
    """The value up-projection folds into the shared output projection:
    W_O . concat_h(W_UV[h] o_h) == sum_h (W_O[:, h] W_UV[h]) o_h."""
    rng = np.random.default_rng(4)
    H, d_v, d_c, d_model, n = 3, 4, 6, 5, 2
    w_uv = rng.standard_normal((H, d_v, d_c))
    w_o = rng.standard_normal((d_model, H * d_v))
    o = rng.standard_normal((n, H, d_c))
    v, out = O.out_proj(o, w_uv, w_o)
    folded = sum(o[:, h] @ (w_o[:, h * d_v:(h + 1) * d_v] @ w_uv[h]).T for h in range(H))
    assert np.allclose(out, folded, rtol=0, atol=1e-12)
    w_fold = O.fold_value_into_output(w_uv, w_o)
    assert w_fold.shape == (d_model, H * d_c)
    assert np.allclose(O.out_proj_folded(o, w_fold), out, rtol=0, atol=1e-12)
    # by hand: W_UV = [[1, 2], [3, 4]], W_O = [[5, 6]] fold to [5+18, 10+24] =
    # [23, 34]; o = [1, 1] gives 57 both ways (W_UV o = [3, 7]; 15 + 42)
    wf = O.fold_value_into_output(np.array([[[1.0, 2.0], [3.0, 4.0]]]), np.array([[5.0, 6.0]]))
    assert wf.tolist() == [[23.0, 34.0]]
    assert O.out_proj_folded(np.array([[[1.0, 1.0]]]), wf).tolist() == [[57.0]]
    assert O.out_proj(np.array([[[1.0, 1.0]]]), np.array([[[1.0, 2.0], [3.0, 4.0]]]),
                      np.array([[5.0, 6.0]]))[1].tolist() == [[57.0]]
    g = GOLD["value"]
    v1, _ = O.out_proj(np.array(g["weighted_latent"])[None, None, :],
                       np.array(g["u_v"])[None], np.eye(4))
    assert np.allclose(v1[0, 0], g["value_out"], rtol=0, atol=1e-15)


# ------------------------------------------------------------- cache writer

def _textbook_head(q_nope, q_rope, p, u_k, c, k_raw, req_pos, scale, base):
    """One head and one query from the definitions, with Python complex
    numbers: every visible row (request position <= p) scores
    scale * (q_nope . U_K c_t + <R(p) q_rope, R(P_t) k_t>), where the rotary
    dot product of two real vectors is the real part of sum_i z_q,i conj(z_k,i)
    over the feature pairs.  Returns (sum_t a_t c_t, lse)."""
    d_r = len(q_rope)
    s = []
    for t in range(len(c)):
        if req_pos[t] > p:
            continue
        content = float(np.dot(q_nope, np.asarray(u_k, np.float64) @ c[t]))
        rot = 0.0
        for i in range(d_r // 2):
            th = base ** (-2.0 * i / d_r)
            zq = complex(q_rope[2 * i], q_rope[2 * i + 1]) * cmath.exp(1j * p * th)
            zk = complex(k_raw[t][2 * i], k_raw[t][2 * i + 1]) * cmath.exp(1j * req_pos[t] * th)
            rot += (zq * zk.conjugate()).real
        s.append((t, scale * (content + rot)))
    m = max(v for _, v in s)
    tot = sum(math.exp(v - m) for _, v in s)
    o = sum(math.exp(v - m) / tot * c[t] for t, v in s)
    return o, m + math.log(tot)


def test_written_cache_serves_textbook_rope_attention():
    # prefix rows are cached at their request positions; a document is cached
    # on its own at canonical positions 0, 1, ... and served right behind the
    # prefix (relocation offset = prefix length)
    wl = Workload("w", "f32", B=1, H=2, d_c=8, d_r=8, d_n=4, d_v=4, d_model=8,
                  prefix=64, doc=37)
    inp = make_inputs(wl, seed=11)
    rows, kpos, ver = O.sequence_rows(inp.segs[0])
    assert list(rows) == list(range(101))
    rng = np.random.default_rng(12)
    c = rng.standard_normal((101, wl.d_c))
    k_raw = rng.standard_normal((101, wl.d_r))
    cache_pos = kpos - np.asarray(inp.deltas)[ver]
    assert list(cache_pos[:64]) == list(range(64)) and list(cache_pos[64:]) == list(range(37))
    inp.pool = O.append_rows(inp.pool, inp.block_table[0], 0,
                             O.cache_rows(c, k_raw, cache_pos, wl.rope_base))
    o_d, l_d, _ = O.decode(inp)
    o_a, l_a = O.decode_absorbed_fast(inp)
    p = int(inp.q_pos[0])
    for h in range(wl.H):
        o_ref, l_ref = _textbook_head(inp.q_nope[0, h], inp.q_rope[0, h], p, inp.w_uk[h], c,
                                      k_raw, kpos, wl.scale, wl.rope_base)
        for o, l in ((o_d, l_d), (o_a, l_a)):
            assert np.allclose(o[0, h], o_ref, rtol=0, atol=1e-10)
            assert abs(l[0, h] - l_ref) < 1e-10


def test_cache_rows_at_position_zero_store_the_raw_key():
    rng = np.random.default_rng(13)
    c, k = rng.standard_normal((3, 8)), rng.standard_normal((3, 6))
    got = O.cache_rows(c, k, [0, 0, 0], 10000.0)
    assert np.array_equal(got[:, :8], c) and np.array_equal(got[:, 8:], k)


def test_append_rows_lands_in_its_slots_only():
    pool = np.full((6, 64, 3), np.nan)
    bt = np.array([4, 1, 5, 0])
    rows = np.arange(300, dtype=np.float64).reshape(100, 3)
    out = O.append_rows(pool, bt, 50, rows)          # logical rows 50 .. 149
    # logical rows 50-63 are slots 50-63 of page 4, rows 64-127 all of page 1,
    # rows 128-149 slots 0-21 of page 5; nothing else changes
    assert np.array_equal(out[4, 50:], rows[0:14])
    assert np.array_equal(out[1], rows[14:78])
    assert np.array_equal(out[5, :22], rows[78:100])
    untouched = np.ones((6, 64), bool)
    untouched[4, 50:] = untouched[1] = untouched[5, :22] = False
    assert np.isnan(out[untouched]).all()
    assert np.isnan(pool).all()                      # the input pool is not modified


# ------------------------------------------------------------- QK-normed MLA

def _qk_weights(inp, seed=21):
    g = np.random.default_rng(seed)
    n = inp.wl.H * inp.wl.d_n
    return 1.0 + 0.2 * g.standard_normal(n), 1.0 + 0.2 * g.standard_normal(n)


@pytest.mark.parametrize("kw", [dict(s_q=2, lengths=(13, 70)),
                                dict(B=1, s_q=1, lengths=None, prefix=64, doc=45)])
def test_qknorm_absorbed_equals_explicit(kw):
    # "exactly equivalent to explicit post-projection QK RMSNorm in exact
    # arithmetic": the latent path with one inverse-RMS scalar per token
    inp = _tiny(**kw)
    g_q, g_k = _qk_weights(inp)
    o_a, l_a = O.decode_qknorm(inp, g_q, g_k, "absorbed")
    o_d, l_d = O.decode_qknorm(inp, g_q, g_k, "direct")
    assert np.allclose(o_a, o_d, rtol=0, atol=1e-12)
    assert np.allclose(l_a, l_d, rtol=0, atol=1e-12)


def test_qknorm_matches_torch_rms_norm_and_sdpa():
    """Keys expanded explicitly, normalised by torch's rms_norm over all heads'
    content keys of a token, rotary parts by complex multiplication, then
    torch's scaled_dot_product_attention with the latent as values."""
    inp = _tiny(s_q=2, lengths=(13, 70))
    wl = inp.wl
    g_q, g_k = _qk_weights(inp)
    eps = O.QK_NORM_EPS
    T = torch.from_numpy
    outs = [O.decode_qknorm(inp, g_q, g_k, form) for form in ("absorbed", "direct")]
    for b in range(wl.B):
        rows = int(inp.n_rows[b])
        r = np.arange(rows)
        cache = inp.pool[inp.block_table[b, r // 64], r % 64].astype(np.float64)
        c, kr = cache[:, :wl.d_c], cache[:, wl.d_c:]
        k_all = np.stack([c @ inp.w_uk[h].astype(np.float64).T for h in range(wl.H)], 1)
        k_hat = torch.nn.functional.rms_norm(T(k_all.reshape(rows, -1)), (wl.H * wl.d_n,),
                                             T(g_k), eps).numpy().reshape(rows, wl.H, wl.d_n)
        for j in range(wl.s_q):
            qi = b * wl.s_q + j
            qp = int(inp.q_pos[qi])
            q_hat = torch.nn.functional.rms_norm(
                T(inp.q_nope[qi].astype(np.float64).reshape(-1)), (wl.H * wl.d_n,), T(g_q),
                eps).numpy().reshape(wl.H, wl.d_n)
            mask = torch.tensor(r[None, :] <= qp)
            for h in range(wl.H):
                q = np.concatenate([q_hat[h], _rope_complex(inp.q_rope[qi, h], qp, wl.rope_base)])
                k = np.concatenate([k_hat[:, h], kr], 1)
                ref = torch.nn.functional.scaled_dot_product_attention(
                    T(q)[None, None], T(k)[None], T(c)[None], attn_mask=mask[None],
                    scale=wl.scale)[0, 0].numpy()
                for o, _ in outs:
                    assert np.allclose(o[qi, h], ref, rtol=0, atol=1e-12)


def test_qknorm_is_scale_invariant_in_query_and_latent():
    # with eps = 0 the normalised content keys ignore a common scale of the
    # latent (so o_lat scales with it), and the normalised query ignores a
    # scale of q_nope
    inp = _tiny(s_q=2, lengths=(13, 70))
    g_q, g_k = _qk_weights(inp)
    o1, l1 = O.decode_qknorm(inp, g_q, g_k, eps=0.0)
    big = copy.deepcopy(inp)
    big.pool = inp.pool.astype(np.float64)
    big.pool[:, :, :inp.wl.d_c] *= 3.5
    big.q_nope = inp.q_nope * 0.25
    o2, l2 = O.decode_qknorm(big, g_q, g_k, eps=0.0)
    assert np.allclose(o2, 3.5 * o1, rtol=0, atol=1e-11)
    assert np.allclose(l2, l1, rtol=0, atol=1e-11)


def test_qknorm_with_unit_rms_inputs_is_plain_attention():
    # unit weights, eps = 0, every token's content keys (all heads) and every
    # query's content part already of RMS 1: the norms are identities
    inp = _tiny(s_q=2, lengths=(13, 70))
    wl = inp.wl
    pool = inp.pool.astype(np.float64)
    for pg in range(pool.shape[0]):
        for sl in range(pool.shape[1]):
            c = pool[pg, sl, :wl.d_c]
            if np.isnan(c).any():
                continue
            k = np.concatenate([inp.w_uk[h].astype(np.float64) @ c for h in range(wl.H)])
            pool[pg, sl, :wl.d_c] = c / math.sqrt(float(np.mean(k * k)))
    inp.pool = pool
    qn = inp.q_nope.astype(np.float64)
    inp.q_nope = qn / np.sqrt(np.mean(qn.reshape(qn.shape[0], -1) ** 2, -1))[:, None, None]
    ones = np.ones(wl.H * wl.d_n)
    o_n, l_n = O.decode_qknorm(inp, ones, ones, eps=0.0)
    o_p, l_p = O.decode_absorbed_fast(inp)
    assert np.allclose(o_n, o_p, rtol=0, atol=1e-11)
    assert np.allclose(l_n, l_p, rtol=0, atol=1e-11)


# ------------------------------------------------------------- low-bit cache

def test_packed_code_bytes_worked_by_hand():
    # INT4, first code in the low nibble: 1 -> 0x1 and -2 -> 0xE make 0xE1;
    # 7 -> 0x7 and -8 -> 0x8 make 0x87.  INT2, fields from the low bits up:
    # 1 -> 01, -2 -> 10, 0 -> 00, -1 -> 11 make 0b11001001 = 0xC9.
    assert O.pack_codes(np.array([1, -2, 7, -8]), 4).tolist() == [0xE1, 0x87]
    assert O.pack_codes(np.array([1, -2, 0, -1]), 2).tolist() == [0xC9]


@pytest.mark.parametrize("bits", [2, 4])
def test_pack_unpack_round_trip_every_byte(bits):
    lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    per = 8 // bits
    codes = np.array(list(itertools.product(range(lo, hi + 1), repeat=per))).reshape(-1)
    packed = O.pack_codes(codes, bits)
    assert sorted(packed.tolist()) == list(range(256))     # each byte value once
    assert np.array_equal(O.unpack_codes(packed, bits), codes)


@pytest.mark.parametrize("bits", [2, 4])
def test_quantization_error_bound_and_saturation(bits):
    lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    scale = np.array([0.5, 0.25, 2.0])
    x = np.random.default_rng(bits).uniform(lo, hi, (1000, 3)) * scale
    err = np.abs(O.dequantize(O.quantize_symmetric(x, scale, bits), scale) - x)
    assert (err <= scale / 2 + 1e-15).all()
    far = np.array([[100.0, -100.0, 1e9]]) * scale
    assert O.quantize_symmetric(far, scale, bits).tolist() == [[hi, lo, hi]]


def test_quantization_ties_go_to_the_even_code():
    s = np.array([1.0])
    x = np.array([[0.5], [1.5], [2.5], [-0.5], [-1.5], [6.5]])
    assert O.quantize_symmetric(x, s, 4)[:, 0].tolist() == [0, 2, 2, 0, -2, 6]


@pytest.mark.parametrize("bits_c", [2, 4])
def test_grid_exact_cache_passes_through_unchanged(bits_c):
    # a cache whose values are already code * channel scale is stored
    # exactly, so the low-bit attention equals the plain one on it
    inp = _tiny(s_q=2, lengths=(13, 70))
    wl = inp.wl
    g = np.random.default_rng(31)
    sc, sr = g.uniform(0.2, 0.6, wl.d_c), g.uniform(0.2, 0.6, wl.d_r)
    pool = inp.pool.astype(np.float64)
    used = ~np.isnan(pool).any(-1)
    n = int(used.sum())
    pool[used, :wl.d_c] = g.integers(-(1 << (bits_c - 1)), 1 << (bits_c - 1), (n, wl.d_c)) * sc
    pool[used, wl.d_c:] = g.integers(-8, 8, (n, wl.d_r)) * sr
    deq = O.dequantize_pool(pool, wl.d_c, sc, sr, bits_c, 4)
    assert np.array_equal(deq, pool, equal_nan=True)
    inp.pool = pool
    o1, l1 = O.decode_absorbed_fast(inp)
    inp.pool = deq
    o2, l2 = O.decode_absorbed_fast(inp)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_quantized_row_bytes():
    # 512 content + 64 rotary values: 1152 bytes in bf16, 288 at INT4/INT4
    # (4x), 160 at INT2 content with an INT4 rotary key (7.2x)
    assert O.quantized_row_bytes(512, 64, 4, 4) == 288
    assert O.quantized_row_bytes(512, 64, 2, 4) == 160


# ------------------------------------- absorbed vs direct on the named configs

def test_absorbed_equals_direct_on_named_configs():
    # the absorbed form gives the large configs their full coverage; the
    # direct (expanded-key) form checks it on seeded samples of them
    from head_latent_attention_02_b200.workloads import WORKLOADS
    inp = make_inputs(WORKLOADS["tiny_f32"], seed=0)
    d_lat, d_lse, _ = O.decode(inp)
    f_lat, f_lse = O.decode_absorbed_fast(inp)
    assert np.allclose(f_lat, d_lat, rtol=1e-10, atol=1e-12)
    assert np.allclose(f_lse, d_lse, rtol=1e-10, atol=1e-12)
    # B=16 x 4096 rows: sequences 0 and 15, heads 0 and 127
    inp = make_inputs(WORKLOADS["bf16_b16_4k"], seed=0, with_weights=True)
    seqs, heads = [0, 15], [0, 127]
    d_lat, d_lse, _ = O.decode(inp, heads=heads, seqs=seqs)
    f_lat, f_lse = O.decode_absorbed_fast(inp, heads=heads, seqs=seqs)
    rows = np.array(seqs)
    assert np.allclose(f_lat[rows], d_lat[rows], rtol=1e-10, atol=1e-12)
    assert np.allclose(f_lse[rows], d_lse[rows], rtol=1e-10, atol=1e-12)
    # RedKnot: a head over all 24 576 rows (prefix + relocated document) and
    # a head over the 256 gathered protected rows
    inp = make_inputs(WORKLOADS["redknot_56_8"], seed=0)
    rows_all = {0: list(range(int(inp.n_rows[0])))}
    for ov in (rows_all, None):
        d_lat, d_lse, _ = O.decode(inp, heads=[3], rows_override=ov)
        f_lat, f_lse = O.decode_absorbed_fast(inp, heads=[3], rows_override=ov)
        assert np.allclose(f_lat, d_lat, rtol=1e-10, atol=1e-12)
        assert np.allclose(f_lse, d_lse, rtol=1e-10, atol=1e-12)


def test_redknot_head_row_ceilings():
    # informational: the printed percentages follow from the printed layer
    # and head counts with the inferred layer totals
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "redknot_head_rows.json")))
    for pr in g["profiles"]:
        c = O.head_row_ceiling(pr["local_heads"], pr["global_heads"], pr["reusable_layers"],
                               pr["total_layers"])
        assert round(100 * c, 2) == pr["ceiling_percent"], pr["name"]
    # the 56/8 split of the RedKnot config is the Flash profile's
    assert O.head_row_ceiling(56, 8, 1, 1) == 0.875


def test_channel_scales_fold_into_query_and_output():
    # with one scale per channel, attention over the dequantised cache equals
    # attention over the raw integer codes with the scales folded into the
    # absorbed query (content and rotary parts) and into the weighted latent
    inp = _tiny(s_q=2, lengths=(13, 70))
    wl = inp.wl
    g = np.random.default_rng(41)
    sc, sr = g.uniform(0.2, 0.6, wl.d_c), g.uniform(0.2, 0.6, wl.d_r)
    pool = inp.pool.astype(np.float64)
    used = ~np.isnan(pool).any(-1)
    codes = np.full_like(pool, np.nan)
    codes[used, :wl.d_c] = O.quantize_symmetric(pool[used, :wl.d_c], sc, 4)
    codes[used, wl.d_c:] = O.quantize_symmetric(pool[used, wl.d_c:], sr, 4)
    deq = np.full_like(pool, np.nan)
    deq[used, :wl.d_c] = codes[used, :wl.d_c] * sc
    deq[used, wl.d_c:] = codes[used, wl.d_c:] * sr
    inp.pool = deq
    o_ref, l_ref = O.decode_absorbed_fast(inp)
    # integer codes are exact in bf16 (|code| <= 8)
    assert np.array_equal(codes[used], np.round(codes[used])) and np.abs(codes[used]).max() <= 8
    for b in range(wl.B):
        rows, kpos, ver = O.sequence_rows(inp.segs[b])
        cc = O.gather_cache(codes, inp.block_table[b], rows)
        for j in range(wl.s_q):
            qi = b * wl.s_q + j
            p = int(inp.q_pos[qi])
            q_lat = np.einsum("hn,hnc->hc", inp.q_nope[qi].astype(np.float64),
                              inp.w_uk.astype(np.float64)) * sc          # scale into the query
            q_r = O.rope_rotate(inp.q_rope[qi].astype(np.float64), p, wl.rope_base) * sr
            s = wl.scale * (q_lat @ cc[:, :wl.d_c].T + q_r @ cc[:, wl.d_c:].T)
            s = np.where((kpos <= p)[None, :], s, -np.inf)
            a, lse = O.softmax_lse(s)
            o = (a @ cc[:, :wl.d_c]) * sc                                  # scale after the sum
            assert np.allclose(o, o_ref[qi], rtol=0, atol=1e-12)
            assert np.allclose(lse, l_ref[qi], rtol=0, atol=1e-12)


def test_qknorm_one_factor_per_column_with_prescaled_rotary_keys():
    # if the cache writer stores rms_t * k_rope_t, the QK-normed score is one
    # 576-wide product against the stored row times the token's inverse RMS:
    # scale * inv_t * (q_w . c_t + q_r . (rms_t k_rope_t))
    inp = _tiny(B=1, s_q=1, lengths=None, prefix=64, doc=45)
    wl = inp.wl
    g_q, g_k = _qk_weights(inp)
    rows, kpos, ver = O.sequence_rows(inp.segs[0])
    cache = O.gather_cache(inp.pool, inp.block_table[0], rows)
    c, k_rope = cache[:, :wl.d_c], cache[:, wl.d_c:]
    shift = np.asarray(inp.deltas, np.int64)[ver]
    p = int(inp.q_pos[0])
    ref = O.qknorm_scores_absorbed(inp.q_nope[0], inp.q_rope[0], p, inp.w_uk, c, k_rope, shift,
                                   g_q, g_k, wl.scale, wl.rope_base)
    inv = O.key_inv_rms(c, inp.w_uk)
    stored = np.concatenate([c, k_rope / inv[:, None]], 1)          # rms_t * k_rope_t
    q_hat = O.rms_norm(inp.q_nope[0].astype(np.float64).reshape(-1), g_q).reshape(wl.H, wl.d_n)
    q_lat = np.einsum("hn,hnc->hc", q_hat * g_k.reshape(wl.H, wl.d_n), inp.w_uk.astype(np.float64))
    q_r = O.rope_rotate(inp.q_rope[0].astype(np.float64)[:, None, :],
                        (p - shift)[None, :], wl.rope_base)           # [H, T, d_r]
    s = wl.scale * inv[None, :] * (q_lat @ stored[:, :wl.d_c].T
                                   + np.einsum("htd,td->ht", q_r, stored[:, wl.d_c:]))
    assert np.allclose(s, ref, rtol=0, atol=1e-11)
