"""GPU parity of QK-normed MLA against the oracle's decode_qknorm.

The GPU path: mla_qknorm_key_gram (key Gram matrix from W_UK), the cache
writer with that matrix (inverse key RMS per row, rescaled rotary key),
mla_qknorm_query (normalised, weighted content query), mla_absorb_q and
mla_decode_qknorm (one factor per score column).  The oracle normalises the
expanded content keys and queries explicitly ("QK-Normed MLA" abstract) in
fp64.  Tolerances: the decode parity bar (bf16: relative L2 <= 1e-2, max-abs
<= 2e-2, |delta lse| <= 1e-2; fp32: 1e-5); the statistics within fp32
rounding of their fp64 values.
"""
import numpy as np
import pytest
import torch

from head_latent_attention_02_b200 import mla, runner
from head_latent_attention_02_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle import mla_oracle as O

pytestmark = pytest.mark.gpu

TOL = {"bf16": dict(rel=1e-2, abs=2e-2, lse=1e-2), "f32": dict(rel=1e-5, abs=1e-5, lse=1e-5)}
EPS = O.QK_NORM_EPS


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
    if lse:
        both = np.isneginf(got) & np.isneginf(ref)
        d = np.abs(np.where(both, 0.0, got) - np.where(both, 0.0, ref))
        assert np.isfinite(d).all() and d.max() <= tol["lse"], f"{what}: {d.max():.3e}"
        return
    assert np.isfinite(got).all(), what
    diff = got - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30)
    assert rel <= tol["rel"], f"{what}: rel L2 {rel:.3e}"
    assert np.abs(diff).max() <= tol["abs"], f"{what}: max abs {np.abs(diff).max():.3e}"


def _weights(wl, seed):
    g = np.random.default_rng(seed)
    n = wl.H * wl.d_n
    return (g.uniform(0.5, 1.5, n).astype(np.float32), g.uniform(0.5, 1.5, n).astype(np.float32))


def _qknorm_gpu(inp, g_q, g_k):
    """The whole QK-normed decode on the GPU from the workload's rows."""
    wl = inp.wl
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    p = runner.upload(inp, with_out_proj=False)
    dims = p.dims
    gram = torch.empty((wl.d_c, wl.d_c), dtype=torch.float32, device="cuda")
    mla.qknorm_key_gram(dims, p.w_uk, gram)
    # rewrite every used row through the writer: cache position 0 leaves the
    # cached rotary key as it is, apart from the QK-norm rescaling
    seq = np.concatenate([np.full(n, b, np.int32) for b, n in enumerate(inp.n_rows)])
    row = np.concatenate([np.arange(n, dtype=np.int32) for n in inp.n_rows])
    page = inp.block_table[seq, row // 64]
    rows = inp.pool[page, row % 64]
    key_inv = torch.full((inp.pool.shape[0] * 64,), float("nan"), device="cuda")
    dev = lambda x, t: torch.from_numpy(np.ascontiguousarray(x)).to("cuda", t)
    mla.append_rows(dims, dev(rows[:, :wl.d_c], dt), dev(rows[:, wl.d_c:], dt),
                    dev(np.zeros(len(seq), np.int32), torch.int32), dev(seq, torch.int32),
                    dev(row, torch.int32), p.cache, p.block_table, key_gram=gram, qk_eps=EPS,
                    key_inv_rms=key_inv)
    q_norm = torch.empty_like(p.q_nope)
    mla.qknorm_query(dims, p.q_nope, dev(g_q, torch.float32), dev(g_k, torch.float32), EPS,
                     q_norm)
    mla.absorb_q(dims, q_norm, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs)
    mla.decode_qknorm(dims, p.B, p.s_q, p.q_abs, p.n_ver, None, p.H, p.cache, key_inv,
                      p.block_table, p.segs, p.q_pos, p.o_lat, p.lse, p.workspace)
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    return p, gram, key_inv, q_norm, rows, page, row


@pytest.mark.parametrize("kind", ["bf16", "f32"])
def test_qknorm_decode_matches_oracle(kind):
    if kind == "bf16":
        wl = Workload("qk", "bf16", B=3, H=128, d_model=512, lengths=[1000, 337, 64])
    else:
        wl = WORKLOADS["tiny_f32"]
    inp = make_inputs(wl, seed=31)
    g_q, g_k = _weights(wl, 31)
    p, gram, key_inv, q_norm, rows, page, row = _qknorm_gpu(inp, g_q, g_k)
    # the statistics
    w = np.asarray(inp.w_uk, np.float64).reshape(-1, wl.d_c)
    _cmp(gram.cpu().numpy(), w.T @ w / w.shape[0], dict(rel=1e-5, abs=1e-5), "gram")
    inv_ref = O.key_inv_rms(rows[:, :wl.d_c], inp.w_uk, EPS)
    inv_got = key_inv.cpu().numpy()[page * 64 + row % 64]
    assert np.abs(inv_got / inv_ref - 1).max() <= 1e-5
    qn_ref = O.rms_norm(np.asarray(inp.q_nope, np.float64).reshape(inp.n_q, -1), g_q, EPS) * g_k
    tol_q = 2.0 ** -7 if kind == "bf16" else 1e-5
    qn_got = q_norm.float().cpu().numpy().reshape(inp.n_q, -1)
    assert (np.abs(qn_got - qn_ref) <= tol_q * np.abs(qn_ref) + 1e-6).all()
    # the decode
    o_ref, l_ref = O.decode_qknorm(inp, g_q, g_k, eps=EPS)
    _cmp(p.o_lat.cpu().numpy(), o_ref, TOL[kind], "o_lat")
    _cmp(p.lse.cpu().numpy(), l_ref, TOL[kind], "lse", lse=True)


def test_qknorm_decode_with_unit_statistics_is_the_plain_decode():
    # factors of exactly one and unscaled rows: mla_decode_qknorm must give
    # mla_decode's result bit for bit (the factor multiplies each score once)
    inp = make_inputs(Workload("qk1", "bf16", B=2, H=64, d_model=512, lengths=[700, 130]),
                      seed=32)
    p = runner.upload(inp, with_out_proj=False)
    mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs)
    mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, None, p.H, p.cache, p.block_table, p.segs,
               p.q_pos, p.o_lat, p.lse, p.workspace)
    ones = torch.ones(inp.pool.shape[0] * 64, device="cuda")
    o2, l2 = torch.empty_like(p.o_lat), torch.empty_like(p.lse)
    mla.decode_qknorm(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, None, p.H, p.cache, ones,
                      p.block_table, p.segs, p.q_pos, o2, l2, p.workspace)
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    assert torch.equal(o2, p.o_lat) and torch.equal(l2, p.lse)
