"""The decode planner's work list, read back from the workspace after a real
decode call and compared bit-exactly with a CPU recomputation of its rules.

The planner (one CTA before the attention kernel) turns the block table and
segments into the schedule every CTA pair walks:
  * per (sequence, query token, 128-head block) stream, its tile count --
    ceil(pages / 2) per segment in page mode, ceil(n_gather / 128) for
    gathered rows -- and whether the sequence is invalid (then 0 tiles);
  * the exclusive prefix sum of the counts (stream offsets, total U);
  * the chunk C of consecutive tiles per pair: ceil(U / G), at least 2, or,
    when every stream has the same count T0 > 0, a divisor of T0 (at most
    G / n_streams parts) or a multiple of it (more streams than pairs) when
    that costs at most a quarter more than the even split;
  * the stream holding each pair's first tile.
Workspace layout: header {U, C, G, n_streams} at 0, then 256-byte-aligned
arrays of stream offsets [n_streams + 1], invalid flags [n_streams] and
first streams [G].
"""
import numpy as np
import pytest
import torch

from head_latent_attention_02_b200 import mla, runner
from head_latent_attention_02_b200.workloads import Workload, make_inputs

from tests.plan_rules import cpu_plan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_02_b200 import build
    build.build()
    mla.lib()
    assert mla.get_status() == 0


def _align256(x):
    return (x + 255) & ~255


def _gpu_plan(p, n_h, G):
    n_streams = p.B * p.s_q * -(-n_h // 128)
    ws = p.workspace.cpu().numpy()
    hdr = ws[:16].view(np.int32)
    o_str = 256
    o_bad = o_str + _align256(4 * (n_streams + 1))
    o_first = o_bad + _align256(4 * n_streams)
    return dict(U=int(hdr[0]), C=int(hdr[1]), G=int(hdr[2]), n_streams=int(hdr[3]),
                off=ws[o_str:o_str + 4 * (n_streams + 1)].view(np.int32),
                bad=ws[o_bad:o_bad + 4 * n_streams].view(np.int32),
                first=ws[o_first:o_first + 4 * G].view(np.int32))


def _check(inp, status=0):
    p = runner.upload(inp)
    runner.run_step(p, out_proj=False)
    torch.cuda.synchronize()
    assert mla.get_status() == status
    G = torch.cuda.get_device_properties(0).multi_processor_count // 2
    got, ref = _gpu_plan(p, inp.wl.H, G), cpu_plan(inp, inp.wl.H, G)
    assert got["G"] == G
    for k in ("U", "C", "n_streams"):
        assert got[k] == ref[k], (k, got[k], ref[k])
    np.testing.assert_array_equal(got["off"], ref["off"])
    np.testing.assert_array_equal(got["bad"], ref["bad"])
    np.testing.assert_array_equal(got["first"], ref["first"])
    return ref


def test_plan_equal_lengths_aligned_chunk():
    # 16 x 32 tiles: the even split is 7 per pair, the aligned chunk 8 (4 per sequence)
    ref = _check(make_inputs(Workload("p1", "bf16", B=16, H=128, d_model=256,
                                      lengths=[4096] * 16), seed=0))
    assert ref["C"] == 8


def test_plan_more_streams_than_pairs():
    # 100 streams of 2 tiles: the multiple-of-T0 chunk (4) costs more than 5/4
    # of the even split (3), so the even split stays
    ref = _check(make_inputs(Workload("p2", "bf16", B=100, H=128, d_model=256,
                                      lengths=[256] * 100), seed=1))
    assert ref["C"] == 3


def test_plan_ragged_lengths_and_two_query_tokens():
    _check(make_inputs(Workload("p3", "bf16", B=20, H=64, d_model=256, s_q=2,
                                len_range=(100, 5000), scattered=True), seed=2))


def test_plan_prefix_and_document_segments():
    _check(make_inputs(Workload("p4", "bf16", B=2, H=128, d_model=256, prefix=640,
                                doc=1000), seed=3))


def test_plan_gathered_rows_with_rejected_sequences():
    wl = Workload("p5", "bf16", B=4, H=128, d_model=256, prefix=128, doc=512, protected=200)
    inp = make_inputs(wl, seed=4)
    inp.gather_rows[1, 130] = 5          # a prefix row in a document tile
    inp.gather_rows[3, 0] = 4000         # outside every segment
    inp.n_gather[2] = 77
    ref = _check(inp, status=6)
    assert list(ref["bad"]) == [0, 1, 0, 1]
