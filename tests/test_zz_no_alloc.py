"""mla_decode_static_ws -- decode with the library's fixed scratch array --
against mla_decode with a caller workspace, through the C ABI.

Two calls of the static-scratch entry point in a row on different problems:
the second runs over whatever the first left in the shared array.  Tolerance
is the bf16 parity bar of the decode tests (relative L2 <= 1e-2, max-abs <=
2e-2, |delta lse| <= 1e-2).
"""
import ctypes

import numpy as np
import pytest
import torch

from head_latent_attention_02_b200 import mla, runner
from head_latent_attention_02_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL = dict(rel=1e-2, abs=2e-2, lse=1e-2)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_02_b200 import build
    build.build()
    mla.lib()
    assert mla.get_status() == 0


def _close(got, ref, what, lse=False):
    got = got.detach().cpu().double().numpy()
    ref = ref.detach().cpu().double().numpy()
    if lse:
        both = np.isneginf(got) & np.isneginf(ref)
        d = np.abs(np.where(both, 0.0, got - ref))
        assert np.isfinite(d).all(), f"{what}: non-finite lse mismatch"
        assert d.max() <= TOL["lse"], f"{what}: max |dlse| {d.max():.3e}"
        return
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    diff = got - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30)
    assert rel <= TOL["rel"], f"{what}: rel L2 {rel:.3e}"
    assert np.abs(diff).max() <= TOL["abs"], f"{what}: max abs {np.abs(diff).max():.3e}"


def _decode_both(wl: Workload, seed: int):
    p = runner.upload(make_inputs(wl, seed=seed), with_out_proj=False)
    mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs)
    mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, 0, p.H, p.cache, p.block_table, p.segs,
               p.q_pos, p.o_lat, p.lse, p.workspace)
    o_s = torch.full_like(p.o_lat, float("nan"))
    lse_s = torch.full_like(p.lse, float("nan"))
    mla.decode_static_ws(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, 0, p.H, p.cache, p.block_table,
                         p.segs, p.q_pos, o_s, lse_s)
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    return p, o_s, lse_s


def test_static_scratch_decode_matches_workspace_decode_two_calls():
    # call 1: long sequences split over many CTA pairs (every partial slot used)
    wl1 = Workload("split", "bf16", B=2, H=128, d_model=512, lengths=[9000, 4097])
    # call 2: other sizes -- more, shorter sequences, two query tokens, 64 heads
    wl2 = Workload("mixed", "bf16", B=5, H=64, d_model=512, s_q=2,
                   lengths=[1000, 337, 64, 2500, 1], scattered=True)
    for i, (wl, seed) in enumerate([(wl1, 21), (wl2, 22)]):
        p, o_s, lse_s = _decode_both(wl, seed)
        _close(o_s, p.o_lat, f"call {i + 1} o_lat")
        _close(lse_s, p.lse, f"call {i + 1} lse", lse=True)


def test_static_scratch_rejects_sizes_beyond_the_array():
    wl = Workload("big", "bf16", B=1, H=128, d_model=512, lengths=[64])
    dims = mla.make_dims(wl)
    B = 1_000_000                     # far more streams than the array can plan
    assert mla.workspace_size(dims, B, 1, 128) > (40 << 20)
    rc = mla.lib().mla_decode_static_ws(ctypes.byref(dims), B, 1, None, 1, 0, 128, None, 1, None,
                                        1, None, 1, None, None, 0, None, None, None, None)
    assert mla.STATUS[rc] == "MLA_ERR_WORKSPACE"
