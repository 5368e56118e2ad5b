"""GPU parity: the libmla path against the fp64 oracle on the same seeded inputs.

Tolerances (fixed by the method's precision contract): bf16 storage with fp32
accumulation -- relative L2 <= 1e-2 and max-abs <= 2e-2 on o_lat, v and out,
|delta lse| <= 1e-2; fp32 storage -- 1e-5 on each.  Page and row bookkeeping
is exact: poisoned (NaN) rows and pages must never reach a result.
"""
import math

import numpy as np
import pytest
import torch

from head_latent_attention_02_b200 import mla, runner
from head_latent_attention_02_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle import mla_oracle as O

pytestmark = pytest.mark.gpu

TOL = {"bf16": dict(rel=1e-2, abs=2e-2, lse=1e-2), "f32": dict(rel=1e-5, abs=1e-5, lse=1e-5)}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_02_b200 import build
    build.build()
    mla.lib()
    assert mla.get_status() == 0


def _cmp(got, ref, tol, what, lse=False):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if lse:
        both_inf = np.isneginf(got) & np.isneginf(ref)
        d = np.abs(np.where(both_inf, 0.0, got - ref))
        assert np.isfinite(d).all(), f"{what}: non-finite lse mismatch"
        assert d.max() <= tol["lse"], f"{what}: max |dlse| = {d.max():.3e}"
        return d.max()
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    diff = got - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(diff).max() if diff.size else 0.0
    assert rel <= tol["rel"], f"{what}: rel L2 {rel:.3e}"
    assert mx <= tol["abs"], f"{what}: max abs {mx:.3e}"
    return rel, mx


def _gpu(inp, **kw):
    p = runner.upload(inp, **kw)
    runner.run_step(p)
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    return p


def _gpu_status(inp, code):
    p = runner.upload(inp)
    runner.run_step(p, out_proj=False)
    torch.cuda.synchronize()
    assert mla.get_status() == code
    assert mla.get_status() == 0
    return p


def _oracle(inp, heads=None):
    o_lat, lse = O.decode_absorbed_fast(inp, heads=heads)
    return o_lat, lse


def _check_all(inp, p, tol, seqs=None):
    wl = inp.wl
    o_ref, l_ref = _oracle(inp)
    v_ref, out_ref = O.out_proj(o_ref, inp.w_uv, inp.w_o)
    _cmp(p.o_lat.cpu().numpy(), o_ref, tol, "o_lat")
    _cmp(p.lse.cpu().numpy(), l_ref, tol, "lse", lse=True)
    _cmp(p.v.cpu().numpy(), v_ref, tol, "v")
    _cmp(p.out.cpu().numpy(), out_ref, tol, "out")


# ----------------------------------------------------------------- configs

def test_tiny_f32_config_direct_form():
    inp = make_inputs(WORKLOADS["tiny_f32"], seed=0)
    p = _gpu(inp)
    o_ref, l_ref, v_ref = O.decode(inp)             # direct (expanded-key) form
    _, out_ref = O.out_proj(o_ref, inp.w_uv, inp.w_o)
    tol = TOL["f32"]
    _cmp(p.o_lat.cpu().numpy(), o_ref, tol, "o_lat")
    _cmp(p.lse.cpu().numpy(), l_ref, tol, "lse", lse=True)
    _cmp(p.v.cpu().numpy(), v_ref, tol, "v")
    _cmp(p.out.cpu().numpy(), out_ref, tol, "out")


def _bf16(name="t", **kw):
    base = dict(B=3, H=128, d_model=512, lengths=[1000, 337, 64])
    base.update(kw)
    return Workload(name, "bf16", **base)


def test_bf16_ragged_pages():
    inp = make_inputs(_bf16(), seed=1)
    p = _gpu(inp)
    _check_all(inp, p, TOL["bf16"])
    # the direct form too, on a few heads of the longest sequence
    o_d, l_d, v_d = O.decode(inp, heads=[0, 77, 127], seqs=[0])
    _cmp(p.o_lat.cpu().numpy()[0][[0, 77, 127]], o_d[0], TOL["bf16"], "o_lat direct")


def test_bf16_many_splits_and_partial_last_page():
    # long sequences so that every sequence is split over several CTA pairs
    inp = make_inputs(_bf16(B=2, lengths=[9000, 4097]), seed=2)
    p = _gpu(inp)
    _check_all(inp, p, TOL["bf16"])


@pytest.mark.parametrize("H", [64, 8, 56, 200])
def test_bf16_head_counts(H):
    inp = make_inputs(_bf16(H=H, B=4, lengths=[130, 64, 1, 700], scattered=True), seed=3)
    p = _gpu(inp)
    _check_all(inp, p, TOL["bf16"])


@pytest.mark.parametrize("B,rows", [(100, 128), (16, 896), (32, 1024)])
def test_bf16_equal_length_sequences(B, rows):
    # equal tile counts per stream: more streams than CTA pairs (each pair
    # takes whole streams), a prime tile count (7: no aligned chunk), and
    # streams split into equal aligned parts
    inp = make_inputs(_bf16(B=B, d_model=256, lengths=[rows] * B), seed=5)
    p = _gpu(inp)
    seqs = sorted({0, B // 2, B - 1})
    o_ref, l_ref = O.decode_absorbed_fast(inp, seqs=seqs)
    _cmp(p.o_lat.cpu().numpy()[seqs], o_ref[seqs], TOL["bf16"], "o_lat")
    _cmp(p.lse.cpu().numpy()[seqs], l_ref[seqs], TOL["bf16"], "lse", lse=True)
    assert np.isfinite(p.o_lat.cpu().numpy()).all()


def test_bf16_many_short_sequences():
    # more streams than one planner pass covers (300 > 256) with mixed
    # lengths, including empty-ish single rows: exercises the carried prefix
    lengths = [int(x) for x in np.random.default_rng(7).integers(1, 300, size=300)]
    inp = make_inputs(_bf16(B=300, H=64, d_model=256, lengths=lengths), seed=6)
    p = _gpu(inp)
    seqs = [0, 1, 150, 257, 299]
    o_ref, l_ref = O.decode_absorbed_fast(inp, seqs=seqs)
    _cmp(p.o_lat.cpu().numpy()[seqs], o_ref[seqs], TOL["bf16"], "o_lat")
    _cmp(p.lse.cpu().numpy()[seqs], l_ref[seqs], TOL["bf16"], "lse", lse=True)
    assert np.isfinite(p.o_lat.cpu().numpy()).all()


def test_bf16_two_query_tokens_causal():
    inp = make_inputs(_bf16(B=2, s_q=2, lengths=[700, 130]), seed=4)
    p = _gpu(inp)
    _check_all(inp, p, TOL["bf16"])
    # the first query token of a sequence must not see the last cached row
    assert int(inp.q_pos[0]) == 698


@pytest.mark.parametrize("mode,perm", [("sample", False), ("first", False), ("sample", True)])
def test_redknot_offline_online_merge(mode, perm):
    wl = Workload("rk", "bf16", B=1, H=64, d_model=512, prefix=128, doc=512, n_local=56,
                  protected=100, protected_mode=mode, head_perm=perm)
    inp = make_inputs(wl, seed=5)
    order = inp.head_order if perm else np.arange(wl.H)
    local = order[:wl.n_local]                   # logical ids of the Local heads
    doc = np.arange(wl.prefix, wl.prefix + wl.doc)
    prot = inp.gather_rows[0]
    k_off = np.setdiff1d(doc, prot)
    # offline partial of the Local heads over the document rows not protected
    inp_off = make_inputs(wl, seed=5)
    inp_off.gather_rows = None
    o_off, l_off = O.decode_absorbed_fast(inp_off, heads=local, rows_override={0: k_off})
    o_off_dev = np.zeros((inp.n_q, wl.H, wl.d_c), np.float32)
    l_off_dev = np.full((inp.n_q, wl.H), -np.inf, np.float32)
    o_off_dev[:, local] = o_off
    l_off_dev[:, local] = l_off
    # the weights stay in the workload's head order: the calls take id lists
    p = _gpu(inp, o_off=o_off_dev, lse_off=l_off_dev)
    # reference: Local heads attend the whole document (offline + protected),
    # Global heads attend prefix + document; then one shared projection
    inp_all = make_inputs(wl, seed=5)
    inp_all.gather_rows = None
    o_ref = np.zeros((inp.n_q, wl.H, wl.d_c))
    l_ref = np.zeros((inp.n_q, wl.H))
    ol, ll = O.decode_absorbed_fast(inp_all, heads=local, rows_override={0: doc})
    o_ref[:, local], l_ref[:, local] = ol, ll
    glob = order[wl.n_local:]
    og, lg = O.decode_absorbed_fast(inp_all, heads=glob)
    o_ref[:, glob], l_ref[:, glob] = og, lg
    _, out_ref = O.out_proj(o_ref, inp.w_uv, inp.w_o)
    tol = TOL["bf16"]
    _cmp(p.o_lat.cpu().numpy(), o_ref, tol, "o_lat")
    _cmp(p.lse.cpu().numpy(), l_ref, tol, "lse", lse=True)
    _cmp(p.out.cpu().numpy(), out_ref, tol, "out")


def _decode_heads(inp, heads):
    """mla_decode over a list of head ids into NaN-filled outputs."""
    p = runner.upload(inp, with_out_proj=False)
    mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs)
    p.o_lat.fill_(float("nan"))
    p.lse.fill_(float("nan"))
    ids = torch.tensor(np.asarray(heads, np.int32), device="cuda")
    mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, ids, len(heads), p.cache, p.block_table,
               p.segs, p.q_pos, p.o_lat, p.lse, p.workspace)
    torch.cuda.synchronize()
    return p


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_head_list_writes_listed_heads_only(dtype):
    # 40 scattered heads of 128 (bf16, tensor-core path; packed queries) or 5
    # of 8 (fp32 generic path): each result lands in its head's row and every
    # other row is left as it was
    if dtype == "bf16":
        inp = make_inputs(_bf16(B=3, lengths=[300, 1000, 77]), seed=12)
        heads = np.random.default_rng(12).permutation(128)[:40]
    else:
        inp = make_inputs(WORKLOADS["tiny_f32"], seed=12)
        heads = np.array([6, 0, 3, 7, 2])
    p = _decode_heads(inp, heads)
    assert mla.get_status() == 0
    o, l = p.o_lat.cpu().numpy(), p.lse.cpu().numpy()
    o_ref, l_ref = O.decode_absorbed_fast(inp, heads=heads)
    _cmp(o[:, heads], o_ref, TOL[dtype], "o_lat")
    _cmp(l[:, heads], l_ref, TOL[dtype], "lse", lse=True)
    rest = np.setdiff1d(np.arange(inp.wl.H), heads)
    assert np.isnan(o[:, rest]).all() and np.isnan(l[:, rest]).all()


def test_head_list_with_an_id_out_of_range_is_reported():
    inp = make_inputs(_bf16(B=2, lengths=[200, 500]), seed=13)
    p = _decode_heads(inp, [5, 700, 9, -1])
    assert mla.get_status() == 6                       # MLA_ERR_BAD_INDEX
    o, l = p.o_lat.cpu().numpy(), p.lse.cpu().numpy()
    o_ref, l_ref = O.decode_absorbed_fast(inp, heads=[5, 9])
    _cmp(o[:, [5, 9]], o_ref, TOL["bf16"], "o_lat")
    _cmp(l[:, [5, 9]], l_ref, TOL["bf16"], "lse", lse=True)
    rest = np.setdiff1d(np.arange(128), [5, 9])
    assert np.isnan(o[:, rest]).all()
    assert mla.get_status() == 0


def test_redknot_offline_partial_made_on_the_gpu():
    # the MLA-Off partial of the Local heads (document rows not protected) is
    # computed by the decode call itself, then merged with the online part
    wl = Workload("rk", "bf16", B=1, H=64, d_model=512, prefix=128, doc=512, n_local=56,
                  protected=100, head_perm=True)
    inp = make_inputs(wl, seed=15)
    local = inp.head_order[:wl.n_local]
    doc = np.arange(wl.prefix, wl.prefix + wl.doc)
    k_off = np.setdiff1d(doc, inp.gather_rows[0])
    p = runner.upload(inp, o_off=np.zeros((inp.n_q, wl.H, wl.d_c), np.float32),
                      lse_off=np.full((inp.n_q, wl.H), -np.inf, np.float32))
    mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs)
    runner.offline_partial(p, k_off[None, :])
    runner.run_decode(p)
    mla.out_proj(p.dims, p.o_lat, p.w_uv, p.w_o, p.v, p.out)
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    inp_all = make_inputs(wl, seed=15)
    inp_all.gather_rows = None
    o_off, l_off = O.decode_absorbed_fast(inp_all, heads=local, rows_override={0: k_off})
    _cmp(p.o_off.cpu().numpy()[:, local], o_off, TOL["bf16"], "o_off")
    _cmp(p.lse_off.cpu().numpy()[:, local], l_off, TOL["bf16"], "lse_off", lse=True)
    o_ref = np.zeros((inp.n_q, wl.H, wl.d_c))
    l_ref = np.zeros((inp.n_q, wl.H))
    o_ref[:, local], l_ref[:, local] = O.decode_absorbed_fast(inp_all, heads=local,
                                                              rows_override={0: doc})
    glob = inp.head_order[wl.n_local:]
    o_ref[:, glob], l_ref[:, glob] = O.decode_absorbed_fast(inp_all, heads=glob)
    _, out_ref = O.out_proj(o_ref, inp.w_uv, inp.w_o)
    _cmp(p.o_lat.cpu().numpy(), o_ref, TOL["bf16"], "o_lat")
    _cmp(p.lse.cpu().numpy(), l_ref, TOL["bf16"], "lse", lse=True)
    _cmp(p.out.cpu().numpy(), out_ref, TOL["bf16"], "out")


@pytest.mark.parametrize("s_q", [48, 130])
def test_prefill_chunk_causal(s_q):
    # a prefill chunk: the last s_q cached rows are the query tokens, each
    # sees the rows up to its own position (one stream per query token)
    inp = make_inputs(_bf16(B=2, s_q=s_q, lengths=[300, 1000], H=64), seed=16)
    p = _gpu(inp)
    _check_all(inp, p, TOL["bf16"])


# ----------------------------------------------------------------- edge cases

def test_empty_and_single_row_gathers():
    wl = Workload("g", "bf16", B=3, H=128, d_model=256, lengths=[200, 200, 200])
    inp = make_inputs(wl, seed=6)
    inp.gather_rows = np.array([[5, 0, 0], [7, 150, 199], [0, 0, 0]], np.int32)
    inp.n_gather = np.array([1, 3, 0], np.int32)
    p = _gpu(inp)
    o, l = p.o_lat.cpu().numpy(), p.lse.cpu().numpy()
    assert np.all(o[2] == 0) and np.all(np.isneginf(l[2]))
    o_ref, l_ref = O.decode_absorbed_fast(inp, seqs=[0, 1])
    _cmp(o[:2], o_ref[:2], TOL["bf16"], "o_lat")
    _cmp(l[:2], l_ref[:2], TOL["bf16"], "lse", lse=True)
    # one gathered row: the output is that row's latent exactly (weight 1)
    c5 = inp.pool[inp.block_table[0, 0], 5, :wl.d_c]
    assert np.array_equal(o[0], np.broadcast_to(c5, o[0].shape))


def test_gathered_rows_validated_per_sequence():
    # RedKnot layout: prefix rows 0-127 (version 0), document rows 128-383
    # (version 1); 130 gathered document rows per sequence, i.e. two tiles
    wl = Workload("gv", "bf16", B=3, H=128, d_model=256, prefix=128, doc=256, protected=130)
    inp = make_inputs(wl, seed=9)
    g = inp.gather_rows
    g[0, 128:130] = [3, 4]     # second tile wholly in the prefix: valid
    g[1, 5] = 7                # a prefix row inside a document tile: rejected
    g[2, 129] = 5000           # a row outside every segment: rejected
    p = _gpu_status(inp, 6)
    o, l = p.o_lat.cpu().numpy(), p.lse.cpu().numpy()
    assert np.isnan(o[1:]).all() and np.isnan(l[1:]).all()
    o_ref, l_ref = O.decode_absorbed_fast(inp, seqs=[0])
    _cmp(o[0], o_ref[0], TOL["bf16"], "o_lat")
    _cmp(l[0], l_ref[0], TOL["bf16"], "lse", lse=True)


def test_gathered_rows_many_sequences():
    # 12 x 300 gathered entries: more than one planner pass over the entries,
    # three tiles per sequence (the last one ragged)
    wl = Workload("gm", "bf16", B=12, H=64, d_model=256, prefix=64, doc=1024, protected=300)
    inp = make_inputs(wl, seed=10)
    p = _gpu(inp)
    o_ref, l_ref = O.decode_absorbed_fast(inp)
    _cmp(p.o_lat.cpu().numpy(), o_ref, TOL["bf16"], "o_lat")
    _cmp(p.lse.cpu().numpy(), l_ref, TOL["bf16"], "lse", lse=True)


def test_query_before_every_row_is_empty():
    inp = make_inputs(_bf16(B=1, lengths=[300]), seed=7)
    inp.q_pos[:] = -1
    p = _gpu(inp)
    assert np.all(p.o_lat.cpu().numpy() == 0)
    assert np.all(np.isneginf(p.lse.cpu().numpy()))


def test_bad_page_id_is_reported_not_read():
    inp = make_inputs(_bf16(B=2, lengths=[200, 200]), seed=8)
    p = runner.upload(inp)
    bt = p.block_table.clone()
    bt[1, 1] = 1 << 20                     # far outside the pool
    p.block_table = bt
    runner.run_step(p, out_proj=False)
    torch.cuda.synchronize()
    assert mla.get_status() == 6
    # the first sequence is unaffected
    o_ref, l_ref = O.decode_absorbed_fast(inp, seqs=[0])
    _cmp(p.o_lat.cpu().numpy()[0], o_ref[0], TOL["bf16"], "o_lat")
    assert mla.get_status() == 0


# ----------------------------------------------------------------- full sizes

def _full(name, seqs, heads=None):
    inp = make_inputs(WORKLOADS[name], seed=0)
    p = _gpu(inp)
    o = p.o_lat.cpu().numpy()
    l = p.lse.cpu().numpy()
    o_ref, l_ref = O.decode_absorbed_fast(inp, heads=heads, seqs=seqs)
    wl = inp.wl
    rows = np.concatenate([np.arange(b * wl.s_q, (b + 1) * wl.s_q) for b in seqs])
    hs = np.arange(wl.H) if heads is None else np.asarray(heads)
    _cmp(o[rows][:, hs], o_ref[rows], TOL["bf16"], f"{name} o_lat")
    _cmp(l[rows][:, hs], l_ref[rows], TOL["bf16"], f"{name} lse", lse=True)
    assert np.isfinite(o).all()
    return inp, p


def test_full_bf16_b16_4k_sampled():
    inp, p = _full("bf16_b16_4k", seqs=[0, 7, 15])
    o_ref, l_ref = O.decode_absorbed_fast(inp, seqs=[3])
    v_ref, out_ref = O.out_proj(o_ref[3:4], inp.w_uv, inp.w_o)
    _cmp(p.out.cpu().numpy()[3:4], out_ref, TOL["bf16"], "out")


def test_full_bf16_varlen_b64_sampled():
    _full("bf16_varlen_b64", seqs=[0, 1, 31, 63])


def test_full_redknot_56_8():
    wl = WORKLOADS["redknot_56_8"]
    inp = make_inputs(wl, seed=0)
    local = np.arange(wl.n_local)
    doc = np.arange(wl.prefix, wl.prefix + wl.doc)
    k_off = np.setdiff1d(doc, inp.gather_rows[0])
    inp_all = make_inputs(wl, seed=0)
    inp_all.gather_rows = None
    o_off, l_off = O.decode_absorbed_fast(inp_all, heads=local, rows_override={0: k_off})
    o_off_dev = np.zeros((inp.n_q, wl.H, wl.d_c), np.float32)
    l_off_dev = np.full((inp.n_q, wl.H), -np.inf, np.float32)
    o_off_dev[:, :wl.n_local], l_off_dev[:, :wl.n_local] = o_off, l_off
    p = _gpu(inp, o_off=o_off_dev, lse_off=l_off_dev)
    o_ref = np.zeros((inp.n_q, wl.H, wl.d_c))
    l_ref = np.zeros((inp.n_q, wl.H))
    o_ref[:, :56], l_ref[:, :56] = O.decode_absorbed_fast(inp_all, heads=local,
                                                          rows_override={0: doc})
    og, lg = O.decode_absorbed_fast(inp_all, heads=np.arange(56, 64))
    o_ref[:, 56:], l_ref[:, 56:] = og, lg
    _, out_ref = O.out_proj(o_ref, inp.w_uv, inp.w_o)
    _cmp(p.o_lat.cpu().numpy(), o_ref, TOL["bf16"], "o_lat")
    _cmp(p.lse.cpu().numpy(), l_ref, TOL["bf16"], "lse", lse=True)
    _cmp(p.out.cpu().numpy(), out_ref, TOL["bf16"], "out")


def test_full_bf16_long_256k_sampled():
    _full("bf16_long_256k", seqs=[1])


# ----------------------------------------------------------------- bounded waits

def test_bounded_wait_gives_up_with_timeout_status():
    # a barrier phase that never completes: the wait gives up after its limit,
    # the status word says MLA_ERR_TIMEOUT, and the context keeps working
    waited = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = mla.lib().mla_debug_wait_probe(2_000_000, waited.data_ptr(), None)
    assert rc == 0
    torch.cuda.synchronize()
    assert mla.STATUS[mla.get_status()] == "MLA_ERR_TIMEOUT"
    assert 2000 <= int(waited.item()) < 1_000_000
    assert mla.get_status() == 0
    inp = make_inputs(_bf16(B=1, lengths=[300]), seed=17)
    p = _gpu(inp)
    _check_all(inp, p, TOL["bf16"])


# ----------------------------------------------------------------- the timed step

def test_graph_captured_step_matches_oracle():
    # the bench times one CUDA graph per step (absorb_q, decode, out_proj);
    # replaying such a graph must give the oracle's results, as eager calls do
    inp = make_inputs(_bf16(B=2, lengths=[700, 130]), seed=18)
    p = runner.upload(inp)
    runner.run_step(p)                      # loads the kernels before capture
    torch.cuda.synchronize()
    p.o_lat.fill_(float("nan"))
    p.out.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        runner.run_step(p)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    _check_all(inp, p, TOL["bf16"])


def test_f32_generic_path_wide_score_range():
    # scores far from |s| ~ 1: the fp32 generic kernel's exponentials must keep
    # the 1e-5 bar when the softmax is sharp (queries scaled by 8)
    inp = make_inputs(WORKLOADS["tiny_f32"], seed=19)
    inp.q_nope = (inp.q_nope * 8).astype(np.float32)
    inp.q_rope = (inp.q_rope * 8).astype(np.float32)
    p = _gpu(inp)
    o_ref, l_ref, v_ref = O.decode(inp)
    _, out_ref = O.out_proj(o_ref, inp.w_uv, inp.w_o)
    tol = TOL["f32"]
    _cmp(p.o_lat.cpu().numpy(), o_ref, tol, "o_lat")
    _cmp(p.lse.cpu().numpy(), l_ref, tol, "lse", lse=True)
    _cmp(p.out.cpu().numpy(), out_ref, tol, "out")
