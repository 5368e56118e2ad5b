"""mla_decode_static_ws -- decode with the library's fixed scratch array --
against the fp64 oracle and against mla_decode with a caller workspace,
through the C ABI.

Three calls of the static-scratch entry point in a row on different problems:
each later call runs over whatever the earlier ones left in the shared array,
and the third plans more streams than the second, so the plan entries it
reads hold leftovers.  Tolerance is the bf16 parity bar of the decode tests
(relative L2 <= 1e-2, max-abs <= 2e-2, |delta lse| <= 1e-2).
"""
import ctypes

import numpy as np
import pytest
import torch

from head_latent_attention_02_b200 import mla, runner
from head_latent_attention_02_b200.workloads import Workload, make_inputs
from oracle import mla_oracle as O

pytestmark = pytest.mark.gpu

TOL = dict(rel=1e-2, abs=2e-2, lse=1e-2)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_02_b200 import build
    build.build()
    mla.lib()
    # reserve the array before anything else claims device memory
    mla.decode_static_ws_init()
    assert mla.get_status() == 0


def _np(x):
    return x.detach().cpu().double().numpy() if torch.is_tensor(x) else np.asarray(x, np.float64)


def _close(got, ref, what, lse=False):
    got, ref = _np(got), _np(ref)
    if lse:
        both = np.isneginf(got) & np.isneginf(ref)
        d = np.abs(np.where(both, 0.0, got) - np.where(both, 0.0, ref))
        assert np.isfinite(d).all(), f"{what}: non-finite lse mismatch"
        assert d.max() <= TOL["lse"], f"{what}: max |dlse| {d.max():.3e}"
        return
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    diff = got - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30)
    assert rel <= TOL["rel"], f"{what}: rel L2 {rel:.3e}"
    assert np.abs(diff).max() <= TOL["abs"], f"{what}: max abs {np.abs(diff).max():.3e}"


def _decode_both(wl: Workload, seed: int, head_ids=None):
    inp = make_inputs(wl, seed=seed)
    p = runner.upload(inp, with_out_proj=False)
    n_h = p.H if head_ids is None else len(head_ids)
    ids = None if head_ids is None else torch.tensor(head_ids, dtype=torch.int32, device="cuda")
    mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs)
    mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, ids, n_h, p.cache, p.block_table, p.segs,
               p.q_pos, p.o_lat, p.lse, p.workspace)
    o_s = torch.full_like(p.o_lat, float("nan"))
    lse_s = torch.full_like(p.lse, float("nan"))
    mla.decode_static_ws(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, ids, n_h, p.cache, p.block_table,
                         p.segs, p.q_pos, o_s, lse_s)
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    return inp, p, o_s, lse_s


def test_static_scratch_decode_matches_oracle_and_workspace_decode_three_calls():
    # call 1: many short sequences, two query tokens, 64 heads (10 streams)
    wl1 = Workload("mixed", "bf16", B=5, H=64, d_model=512, s_q=2,
                   lengths=[1000, 337, 64, 2500, 1], scattered=True)
    # call 2: two long sequences split over many CTA pairs (every partial
    # slot used, 2 streams)
    wl2 = Workload("split", "bf16", B=2, H=128, d_model=512, lengths=[9000, 4097])
    # call 3: more streams again, over a list of 100 scattered heads
    wl3 = Workload("many", "bf16", B=12, H=128, d_model=512, len_range=(100, 3000))
    heads3 = np.random.default_rng(23).permutation(128)[:100].astype(np.int32)
    for i, (wl, seed, heads) in enumerate([(wl1, 21, None), (wl2, 22, None),
                                          (wl3, 24, heads3)]):
        inp, p, o_s, lse_s = _decode_both(wl, seed, heads)
        hs = np.arange(wl.H) if heads is None else heads
        o_ref, l_ref = O.decode_absorbed_fast(inp, heads=hs)
        _close(_np(o_s)[:, hs], o_ref, f"call {i + 1} o_lat vs oracle")
        _close(_np(lse_s)[:, hs], l_ref, f"call {i + 1} lse vs oracle", lse=True)
        _close(_np(o_s)[:, hs], _np(p.o_lat)[:, hs], f"call {i + 1} o_lat vs mla_decode")
        _close(_np(lse_s)[:, hs], _np(p.lse)[:, hs], f"call {i + 1} lse vs mla_decode", lse=True)
        if heads is not None:
            # heads not listed are left as they were
            rest = np.setdiff1d(np.arange(wl.H), hs)
            assert np.isnan(_np(o_s)[:, rest]).all() and np.isnan(_np(lse_s)[:, rest]).all()


def test_static_scratch_rejects_sizes_beyond_the_array():
    wl = Workload("big", "bf16", B=1, H=128, d_model=512, lengths=[64])
    dims = mla.make_dims(wl)
    B = 1_000_000                     # far more streams than the array can plan
    assert mla.workspace_size(dims, B, 1, 128) > (48 << 20)
    rc = mla.lib().mla_decode_static_ws(ctypes.byref(dims), B, 1, None, 1, None, 128, None, 1,
                                        None, 1, None, 1, None, None, 0, None, None, None, None)
    assert mla.STATUS[rc] == "MLA_ERR_WORKSPACE"
    # invalid sizes are reported as such, before the size query
    rc = mla.lib().mla_decode_static_ws(ctypes.byref(dims), 1, 1, None, 1, None, 129, None, 1,
                                        None, 1, None, 1, None, None, 0, None, None, None, None)
    assert mla.STATUS[rc] == "MLA_ERR_INVALID_ARG"
