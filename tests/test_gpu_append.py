"""GPU parity of the cache writer (mla_append_rows) against the oracle's
cache_rows / append_rows: latents copied bit for bit, rotary keys within one
unit in the last place of the storage type of the fp64 rotation, every other
slot of the pool untouched (NaN-poisoned), bad entries reported and skipped."""
import numpy as np
import pytest
import torch

from head_latent_attention_02_b200 import mla
from oracle import mla_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_02_b200 import build
    build.build()
    mla.lib()
    assert mla.get_status() == 0


def _dims(dtype, d_c, d_r):
    return mla.Dims(8, d_c, d_r, 16, 16, 128, 64, dtype, 0.1, 10000.0)


def _entries():
    # sequence 0: logical rows 50..149 (three pages); sequence 2: rows 0..9;
    # sequence 1: row 319 (the last slot of its fifth page)
    seq = np.array([0] * 100 + [2] * 10 + [1], np.int32)
    row = np.array(list(range(50, 150)) + list(range(10)) + [319], np.int32)
    # prefix-like rows at their request positions, a document at canonical
    # positions, and a far position
    pos = np.array(list(range(50, 150)) + list(range(10)) + [262143], np.int32)
    return seq, row, pos


@pytest.mark.parametrize("dtype,d_c,d_r", [(mla.MLA_BF16, 512, 64), (mla.MLA_F32, 32, 16)])
def test_append_rows_matches_oracle_writer(dtype, d_c, d_r):
    g = np.random.default_rng(5)
    B, max_pages, n_pages = 3, 5, 16
    bt = g.permutation(n_pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    seq, row, pos = _entries()
    n = len(seq)
    tdt = torch.bfloat16 if dtype == mla.MLA_BF16 else torch.float32
    c = torch.randn(n, d_c, generator=torch.Generator().manual_seed(1)).to(tdt)
    k = torch.randn(n, d_r, generator=torch.Generator().manual_seed(2)).to(tdt)
    pool = torch.full((n_pages, 64, d_c + d_r), float("nan"), dtype=tdt)
    dev = lambda t: t.cuda().contiguous()
    cache = dev(pool)
    mla.append_rows(_dims(dtype, d_c, d_r), dev(c), dev(k), dev(torch.from_numpy(pos)),
                    dev(torch.from_numpy(seq)), dev(torch.from_numpy(row)), cache,
                    dev(torch.from_numpy(bt)))
    torch.cuda.synchronize()
    assert mla.get_status() == 0
    got = cache.float().cpu().numpy().astype(np.float64)
    exp = pool.float().numpy().astype(np.float64)
    rows64 = O.cache_rows(c.float().numpy(), k.float().numpy(), pos, 10000.0)
    for i in range(n):
        exp = O.append_rows(exp, bt[seq[i]], int(row[i]), rows64[i:i + 1])
    written = ~np.isnan(exp).any(-1)
    # untouched slots stay NaN, written ones hold no NaN
    assert np.array_equal(~np.isnan(got).any(-1), written)
    assert np.array_equal(got[written][:, :d_c], exp[written][:, :d_c])      # latent: exact
    ulp = 2.0 ** -7 if dtype == mla.MLA_BF16 else 2.0 ** -23   # one unit in the last place
    kr_got, kr_exp = got[written][:, d_c:], exp[written][:, d_c:]
    assert (np.abs(kr_got - kr_exp) <= ulp * np.abs(kr_exp) + 1e-30).all()


def test_append_rows_reports_and_skips_bad_entries():
    d_c, d_r = 32, 16
    bt = np.array([[3, 1], [0, -5]], np.int32)            # page id -5 is invalid
    seq = np.array([0, 1, 2, 0, 1], np.int32)             # sequence 2 does not exist
    row = np.array([5, 70, 0, 200, 3], np.int32)          # row 200 is past max_pages*64
    pos = np.zeros(5, np.int32)
    c = torch.arange(5 * d_c, dtype=torch.float32).reshape(5, d_c)
    k = torch.ones(5, d_r)
    cache = torch.full((4, 64, d_c + d_r), float("nan"), device="cuda")
    dev = lambda t: t.cuda().contiguous()
    mla.append_rows(_dims(mla.MLA_F32, d_c, d_r), dev(c), dev(k), dev(torch.from_numpy(pos)),
                    dev(torch.from_numpy(seq)), dev(torch.from_numpy(row)), cache,
                    dev(torch.from_numpy(bt)))
    torch.cuda.synchronize()
    assert mla.get_status() == 6
    assert mla.get_status() == 0
    got = cache.cpu().numpy()
    # entry 0 -> page 3 slot 5, entry 4 -> page 0 slot 3; nothing else written
    assert np.array_equal(got[3, 5, :d_c], c[0].numpy())
    assert np.array_equal(got[0, 3, :d_c], c[4].numpy())
    assert np.array_equal(got[3, 5, d_c:], np.ones(d_r))   # position 0: the raw key
    assert (~np.isnan(got).any(-1)).sum() == 2
