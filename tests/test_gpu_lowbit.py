"""GPU parity of the low-bit latent cache (QuantMLA abstract): the packer
against the oracle's code packing, and mla_decode_lowbit against the fp64
oracle's attention over the dequantised pool.

The packer's codes are decided in fp32 (the kernel's precision), so the
expected codes here round x / scale in fp32 as well; the bytes must match
bit for bit.  The decode reads codes packed by the oracle and is compared
with the decode parity bar (bf16 queries: relative L2 <= 1e-2, max-abs <=
2e-2, |delta lse| <= 1e-2; fp32: 1e-5).
"""
import numpy as np
import pytest
import torch

from head_latent_attention_02_b200 import mla, runner
from head_latent_attention_02_b200.workloads import WORKLOADS, Workload, make_inputs, round_bf16
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


def _scales(wl, bits_c, seed):
    g = np.random.default_rng(seed)
    lo, hi = (0.3, 0.6) if bits_c == 4 else (0.8, 1.2)
    return (g.uniform(lo, hi, wl.d_c).astype(np.float32),
            g.uniform(0.3, 0.6, wl.d_r).astype(np.float32))


def _packed_pool(inp, sc, sr, bits_c, bits_r):
    """The pool's rows as the oracle quantises and packs them (unused rows: 0)."""
    wl = inp.wl
    pool = np.asarray(inp.pool, np.float64)
    used = ~np.isnan(pool).any(-1)
    rows = np.where(used[..., None], pool, 0.0)
    cc = O.pack_codes(O.quantize_symmetric(rows[..., :wl.d_c], sc, bits_c), bits_c)
    cr = O.pack_codes(O.quantize_symmetric(rows[..., wl.d_c:], sr, bits_r), bits_r)
    return np.concatenate([cc, cr], axis=-1)


@pytest.mark.parametrize("bits_c,bits_r", [(4, 4), (2, 4)])
@pytest.mark.parametrize("kind", ["bf16", "f32"])
def test_lowbit_decode_matches_oracle_on_dequantised_pool(kind, bits_c, bits_r):
    if kind == "bf16":
        wl = Workload("lb", "bf16", B=3, H=128, d_model=512, lengths=[700, 130, 64], scattered=True)
    else:
        wl = WORKLOADS["tiny_f32"]
    inp = make_inputs(wl, seed=41)
    sc, sr = _scales(wl, bits_c, 41)
    packed = _packed_pool(inp, sc, sr, bits_c, bits_r)
    assert packed.shape[-1] == O.quantized_row_bytes(wl.d_c, wl.d_r, bits_c, bits_r)
    p = runner.upload(inp, with_out_proj=False)
    mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs)
    cache = torch.from_numpy(packed).cuda()
    dev = lambda x: torch.from_numpy(x).cuda()
    heads = np.arange(wl.H)[::-1].copy().astype(np.int32)       # a head list, reversed
    mla.decode_lowbit(p.dims, bits_c, bits_r, p.B, p.s_q, p.q_abs, p.n_ver, dev(heads), wl.H,
                      cache, dev(sc), dev(sr), p.block_table, p.segs, p.q_pos, p.o_lat, p.lse)
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    inp_d = make_inputs(wl, seed=41)
    inp_d.pool = O.dequantize_pool(inp.pool, wl.d_c, sc, sr, bits_c, bits_r)
    o_ref, l_ref = O.decode_absorbed_fast(inp_d)
    _cmp(p.o_lat.cpu().numpy(), o_ref, TOL[kind], "o_lat")
    _cmp(p.lse.cpu().numpy(), l_ref, TOL[kind], "lse", lse=True)


@pytest.mark.parametrize("bits_c,bits_r", [(4, 4), (2, 4)])
def test_pack_rows_matches_oracle_packing(bits_c, bits_r):
    wl = Workload("lb", "bf16", B=1, H=8, d_model=512, lengths=[64])
    g = np.random.default_rng(7)
    n = 300
    sc, sr = _scales(wl, bits_c, 7)
    x = round_bf16(g.standard_normal((n, wl.row)).astype(np.float32) * 1.5)
    # exact ties (bf16-exact multiples of the scale) and saturation
    sc[:4] = 0.5
    x[0, :4] = np.array([0.25, 0.75, -1.25, 100.0], np.float32)
    rows = torch.from_numpy(x).to("cuda", torch.bfloat16)
    assert torch.equal(rows.float().cpu(), torch.from_numpy(x))
    out = torch.empty((n, O.quantized_row_bytes(wl.d_c, wl.d_r, bits_c, bits_r)), dtype=torch.uint8,
                      device="cuda")
    mla.pack_rows(mla.make_dims(wl), bits_c, bits_r, rows, torch.from_numpy(sc).cuda(),
                  torch.from_numpy(sr).cuda(), out)
    torch.cuda.synchronize()
    # codes decided in fp32: x / scale rounded half to even, clamped
    def codes(v, s, bits):
        q = np.rint(v.astype(np.float32) / s.astype(np.float32))
        return np.clip(q, -(1 << (bits - 1)), (1 << (bits - 1)) - 1).astype(np.int64)
    exp = np.concatenate([O.pack_codes(codes(x[:, :wl.d_c], sc, bits_c), bits_c),
                          O.pack_codes(codes(x[:, wl.d_c:], sr, bits_r), bits_r)], axis=-1)
    assert np.array_equal(out.cpu().numpy(), exp)
    # ties went to the even code (then clamped to the range), and the far
    # value saturated
    lo, hi = -(1 << (bits_c - 1)), (1 << (bits_c - 1)) - 1
    assert O.unpack_codes(exp[0], bits_c)[:4].tolist() == [0, min(2, hi), max(-2, lo), hi]


@pytest.mark.parametrize("bits_c,bits_r", [(4, 4), (2, 4)])
@pytest.mark.parametrize("kind", ["bf16", "f32"])
def test_dequant_rows_is_code_times_scale(kind, bits_c, bits_r):
    # every code value of the range in every channel position; the product
    # taken in fp32 (the kernel's precision) and rounded to the pool's type
    wl = Workload("lb", kind, B=1, H=8, d_model=512, lengths=[64])
    g = np.random.default_rng(9)
    n = 257                                                     # 32 full blocks + a tail row
    cc = g.integers(-(1 << (bits_c - 1)), 1 << (bits_c - 1), (n, wl.d_c))
    cr = g.integers(-(1 << (bits_r - 1)), 1 << (bits_r - 1), (n, wl.d_r))
    cc[0] = -(1 << (bits_c - 1))
    cc[1] = (1 << (bits_c - 1)) - 1
    sc, sr = _scales(wl, bits_c, 9)
    packed = np.concatenate([O.pack_codes(cc, bits_c), O.pack_codes(cr, bits_r)], axis=-1)
    dims = mla.make_dims(wl)
    dt = torch.bfloat16 if kind == "bf16" else torch.float32
    out = torch.full((n, wl.row), float("nan"), dtype=dt, device="cuda")
    mla.dequant_rows(dims, bits_c, bits_r, torch.from_numpy(packed).cuda(),
                     torch.from_numpy(sc).cuda(), torch.from_numpy(sr).cuda(), out)
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    codes = np.concatenate([O.unpack_codes(packed[:, :packed.shape[1] - wl.d_r * bits_r // 8],
                                           bits_c),
                            O.unpack_codes(packed[:, packed.shape[1] - wl.d_r * bits_r // 8:],
                                           bits_r)], axis=-1)
    assert np.array_equal(codes, np.concatenate([cc, cr], axis=-1))
    exp = codes.astype(np.float32) * np.concatenate([sc, sr]).astype(np.float32)
    if kind == "bf16":
        exp = round_bf16(exp)
    assert np.array_equal(out.float().cpu().numpy(), exp)


@pytest.mark.parametrize("bits_c,bits_r", [(4, 4), (2, 4)])
@pytest.mark.parametrize("kind", ["bf16", "f32"])
def test_lowbit_tc_decode_matches_oracle_on_dequantised_pool(kind, bits_c, bits_r):
    # the tensor-core route: dequantise the packed pool, then mla_decode
    if kind == "bf16":
        wl = Workload("lb", "bf16", B=3, H=128, d_model=512, lengths=[700, 130, 64], scattered=True)
    else:
        wl = WORKLOADS["tiny_f32"]
    inp = make_inputs(wl, seed=43)
    sc, sr = _scales(wl, bits_c, 43)
    packed = _packed_pool(inp, sc, sr, bits_c, bits_r)
    p = runner.upload(inp, with_out_proj=False)
    mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs)
    cache = torch.from_numpy(packed).cuda()
    dev = lambda x: torch.from_numpy(x).cuda()
    dq = torch.empty(mla.lowbit_dequant_bytes(p.dims, cache.shape[0]), dtype=torch.uint8,
                     device="cuda")
    heads = np.arange(wl.H)[::-1].copy().astype(np.int32)
    mla.decode_lowbit_tc(p.dims, bits_c, bits_r, p.B, p.s_q, p.q_abs, p.n_ver, dev(heads), wl.H,
                         cache, dev(sc), dev(sr), p.block_table, p.segs, p.q_pos, p.o_lat,
                         p.lse, dq, p.workspace)
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    inp_d = make_inputs(wl, seed=43)
    inp_d.pool = O.dequantize_pool(inp.pool, wl.d_c, sc, sr, bits_c, bits_r)
    o_ref, l_ref = O.decode_absorbed_fast(inp_d)
    _cmp(p.o_lat.cpu().numpy(), o_ref, TOL[kind], "o_lat")
    _cmp(p.lse.cpu().numpy(), l_ref, TOL[kind], "lse", lse=True)


def test_lowbit_tc_refuses_a_small_scratch_pool_before_any_launch():
    wl = Workload("lb", "bf16", B=1, H=128, d_model=512, lengths=[100])
    inp = make_inputs(wl, seed=44)
    sc, sr = _scales(wl, 4, 44)
    p = runner.upload(inp, with_out_proj=False)
    cache = torch.from_numpy(_packed_pool(inp, sc, sr, 4, 4)).cuda()
    need = mla.lowbit_dequant_bytes(p.dims, cache.shape[0])
    assert need == cache.shape[0] * 64 * wl.row * 2
    dq = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError, match="WORKSPACE"):
        mla.decode_lowbit_tc(p.dims, 4, 4, p.B, p.s_q, p.q_abs, p.n_ver, None, wl.H, cache,
                             torch.from_numpy(sc).cuda(), torch.from_numpy(sr).cuda(),
                             p.block_table, p.segs, p.q_pos, p.o_lat, p.lse, dq, p.workspace)
    torch.cuda.synchronize()
    assert int(dq.count_nonzero()) == 0 and mla.get_status() == 0
