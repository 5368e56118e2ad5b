"""Host-side checks of the C ABI: the library loads without a GPU, exports
every entry point include/mla.h declares, and rejects bad arguments before
touching the device."""
import ctypes

import pytest

from head_latent_attention_02_b200 import build as B
from head_latent_attention_02_b200 import mla


@pytest.fixture(scope="module")
def L():
    B.build()
    return mla.lib()


def test_exports_every_header_symbol(L):
    names = mla.header_symbols()
    assert {"mla_absorb_q", "mla_decode", "mla_merge_lse", "mla_out_proj"} <= set(names)
    for n in names:
        assert hasattr(L, n), n
    assert set(mla._SIGS) >= set(names)


def test_version_and_status_strings(L):
    assert L.mla_abi_version() == 1
    for code, name in mla.STATUS.items():
        assert mla.status_str(code) == name
    assert mla.status_str(99) == "MLA_ERR_UNKNOWN"


def _dims(**kw):
    d = dict(H=128, d_c=512, d_r=64, d_n=128, d_v=128, d_model=7168, page_size=64,
             dtype=mla.MLA_BF16, scale=1 / 192 ** 0.5, rope_base=10000.0)
    d.update(kw)
    return mla.Dims(**d)


NULL = None
FAKE = 0x1000   # never dereferenced: every case below fails validation first


def _decode(d, B=1, s_q=1, n_ver=1, head_ids=NULL, n_h=None, n_pages=4, max_pages=4,
            max_segs=1, gather=NULL, n_gather=NULL, max_gather=0, ws_bytes=0):
    n_h = (d.H if d is not None else 8) if n_h is None else n_h
    return mla.lib().mla_decode(ctypes.byref(d) if d is not None else None, B, s_q, FAKE, n_ver,
                                head_ids, n_h, FAKE, n_pages, FAKE, max_pages, FAKE, max_segs, gather,
                                n_gather, max_gather, FAKE, FAKE, FAKE, FAKE, ws_bytes, None)


@pytest.mark.parametrize("case", [
    dict(d=None), dict(B=-1), dict(s_q=0), dict(n_ver=0), dict(n_h=0), dict(n_h=129),
    dict(head_ids=FAKE, n_h=129), dict(n_pages=0), dict(max_pages=0), dict(max_segs=0),
    dict(gather=FAKE, n_gather=NULL, max_gather=4), dict(gather=FAKE, n_gather=FAKE, max_gather=0),
])
def test_decode_rejects_bad_arguments(L, case):
    d = case.pop("d", _dims())
    assert _decode(d, **case) == 1   # MLA_ERR_INVALID_ARG


def test_decode_rejects_bad_dims(L):
    assert _decode(_dims(d_r=63)) == 1
    assert _decode(_dims(dtype=7)) == 1
    assert _decode(_dims(H=0), n_h=1) == 1
    assert _decode(_dims(page_size=32)) == 2          # MLA_ERR_UNSUPPORTED
    assert _decode(_dims(), n_ver=9) == 2


def test_decode_rejects_sizes_past_32_bit_indices(L):
    # logical rows (max_pages x 64) and q_abs rows (n_ver x B x s_q x H) are
    # 32-bit on the device: refused before anything is launched
    assert _decode(_dims(), max_pages=1 << 26) == 2
    assert _decode(_dims(), B=1 << 22, s_q=2, n_ver=2) == 2
    assert _decode(_dims(), n_pages=1 << 25) == 2


def test_decode_rejects_misaligned_cache(L):
    d = _dims()
    rc = mla.lib().mla_decode(ctypes.byref(d), 1, 1, FAKE, 1, None, 128, FAKE + 16, 4, FAKE, 4,
                              FAKE, 1, None, None, 0, FAKE, FAKE, FAKE, FAKE, 0, None)
    assert rc == 1


def test_absorb_merge_outproj_reject_bad_arguments(L):
    d = _dims()
    f = mla.lib()
    arr = (ctypes.c_int32 * 1)(0)
    assert f.mla_absorb_q(ctypes.byref(d), 4, FAKE, FAKE, FAKE, arr, 0, FAKE, FAKE, None) == 1
    assert f.mla_absorb_q(ctypes.byref(d), 4, FAKE, FAKE, FAKE, arr, 9, FAKE, FAKE, None) == 1
    assert f.mla_absorb_q(ctypes.byref(d), 4, FAKE, FAKE, FAKE, None, 1, FAKE, FAKE, None) == 1
    assert f.mla_absorb_q(ctypes.byref(d), -1, FAKE, FAKE, FAKE, arr, 1, FAKE, FAKE, None) == 1
    assert f.mla_absorb_q(ctypes.byref(d), 4, None, FAKE, FAKE, arr, 1, FAKE, FAKE, None) == 1
    assert f.mla_absorb_q(ctypes.byref(d), 0, None, None, None, arr, 1, None, None, None) == 0
    assert f.mla_merge_lse(2, 64, None, 65, 512, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f.mla_merge_lse(2, 64, FAKE, 0, 512, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f.mla_merge_lse(2, 64, None, 8, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f.mla_merge_lse(2, 64, None, 8, 512, None, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f.mla_merge_lse(0, 64, None, 8, 512, None, None, None, None, None, None, None) == 0
    assert f.mla_out_proj(ctypes.byref(d), 2, None, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f.mla_out_proj(ctypes.byref(d), 2, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert f.mla_out_proj(ctypes.byref(d), -1, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1


def test_workspace_size_rejects_bad_arguments(L):
    d = _dims()
    assert mla.lib().mla_decode_workspace_size(None, 1, 1, 1, 128) == 0
    assert mla.lib().mla_decode_workspace_size(ctypes.byref(d), 1, 0, 1, 128) == 0
    assert mla.lib().mla_decode_workspace_size(ctypes.byref(d), 1, 1, 0, 128) == 0
    assert mla.lib().mla_decode_workspace_size(ctypes.byref(d), 1, 1, 9, 128) == 0
    assert mla.lib().mla_decode_workspace_size(ctypes.byref(d), 1, 1, 1, 129) == 0
    # the generic (non-576-wide) kernel needs only a token workspace
    assert mla.lib().mla_decode_workspace_size(ctypes.byref(_dims(dtype=mla.MLA_F32)), 1, 1, 1,
                                               8) == 256


def test_append_rows_rejects_bad_arguments(L):
    f = mla.lib()
    d = _dims()
    args = lambda **kw: [kw.get(k, v) for k, v in dict(
        dims=ctypes.byref(d), n=4, c=FAKE, k=FAKE, pos=FAKE, seq=FAKE, row=FAKE, B=2, cache=FAKE,
        n_pages=4, bt=FAKE, max_pages=2, gram=None, eps=0.0, inv=None, stream=None).items()]
    assert f.mla_append_rows(*args(dims=None)) == 1
    assert f.mla_append_rows(*args(n=-1)) == 1
    assert f.mla_append_rows(*args(B=0)) == 1
    assert f.mla_append_rows(*args(n_pages=0)) == 1
    assert f.mla_append_rows(*args(max_pages=0)) == 1
    assert f.mla_append_rows(*args(c=None)) == 1
    assert f.mla_append_rows(*args(cache=FAKE + 1)) == 1            # misaligned bf16 pointer
    assert f.mla_append_rows(*args(dims=ctypes.byref(_dims(d_r=63)))) == 1
    assert f.mla_append_rows(*args(dims=ctypes.byref(_dims(page_size=32)))) == 2
    assert f.mla_append_rows(*args(gram=FAKE)) == 1                # key_inv_rms missing
    assert f.mla_append_rows(*args(inv=FAKE)) == 1                 # key_gram missing
    assert f.mla_append_rows(*args(gram=FAKE, inv=FAKE, eps=-1.0)) == 1
    assert f.mla_append_rows(*args(n=0, c=None, k=None, pos=None, seq=None, row=None,
                                   cache=None, bt=None)) == 0


def test_qknorm_calls_reject_bad_arguments(L):
    f = mla.lib()
    d = _dims()
    assert f.mla_qknorm_query(None, 2, FAKE, FAKE, FAKE, 1e-6, FAKE, None) == 1
    assert f.mla_qknorm_query(ctypes.byref(d), -1, FAKE, FAKE, FAKE, 1e-6, FAKE, None) == 1
    assert f.mla_qknorm_query(ctypes.byref(d), 2, FAKE, None, FAKE, 1e-6, FAKE, None) == 1
    assert f.mla_qknorm_query(ctypes.byref(d), 2, FAKE, FAKE, FAKE, -1.0, FAKE, None) == 1
    assert f.mla_qknorm_query(ctypes.byref(d), 0, None, None, None, 1e-6, None, None) == 0
    assert f.mla_qknorm_key_gram(ctypes.byref(d), None, FAKE, None) == 1
    assert f.mla_qknorm_key_gram(None, FAKE, FAKE, None) == 1
    qk = lambda **kw: f.mla_decode_qknorm(
        ctypes.byref(d), 1, 1, FAKE, 1, None, 128, FAKE, kw.get("inv", FAKE), 4, FAKE, 4, FAKE,
        1, FAKE, FAKE, FAKE, FAKE, 0, None)
    assert qk(inv=None) == 1
    assert qk(inv=FAKE + 4) == 1                                   # not 16-byte aligned


def test_lowbit_calls_reject_bad_arguments(L):
    f = mla.lib()
    d = _dims()
    assert f.mla_pack_rows(ctypes.byref(d), 3, 4, 4, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert f.mla_pack_rows(ctypes.byref(d), 4, 2, 4, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert f.mla_pack_rows(ctypes.byref(d), 4, 4, -1, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f.mla_pack_rows(ctypes.byref(d), 4, 4, 4, FAKE, None, FAKE, FAKE, None) == 1
    assert f.mla_pack_rows(ctypes.byref(d), 4, 4, 4, FAKE, FAKE, FAKE, FAKE + 2, None) == 1
    assert f.mla_pack_rows(ctypes.byref(d), 2, 4, 0, None, None, None, None, None) == 0
    lb = lambda bc=4, br=4, cache=FAKE, sc=FAKE, n_h=128: f.mla_decode_lowbit(
        ctypes.byref(d), bc, br, 1, 1, FAKE, 1, None, n_h, cache, sc, FAKE, 4, FAKE, 4, FAKE, 1,
        None, None, 0, FAKE, FAKE, FAKE, None)
    assert lb(bc=8) == 2 and lb(bc=2, br=2) == 2
    assert lb(cache=FAKE + 1) == 1 and lb(sc=None) == 1 and lb(n_h=129) == 1


def test_lowbit_tc_calls_reject_bad_arguments(L):
    f = mla.lib()
    d = _dims()
    # pool bytes: pages * 64 rows * 576 channels * 2 bytes (bf16 dims)
    assert f.mla_lowbit_dequant_bytes(ctypes.byref(d), 3) == 3 * 64 * 576 * 2
    assert f.mla_lowbit_dequant_bytes(ctypes.byref(d), -1) == 0
    assert f.mla_lowbit_dequant_bytes(None, 3) == 0
    dq = lambda bc=4, br=4, n=4, src=FAKE, sc=FAKE, out=FAKE: f.mla_dequant_rows(
        ctypes.byref(d), bc, br, n, src, sc, FAKE, out, None)
    assert dq(bc=3) == 2 and dq(br=2) == 2
    assert dq(n=-1) == 1 and dq(sc=None) == 1
    assert dq(src=FAKE + 2) == 1 and dq(out=FAKE + 8) == 1       # 4- and 16-byte alignment
    assert dq(n=0, src=None, sc=None, out=None) == 0
    big = 3 * 64 * 576 * 2
    tc = lambda bc=4, n_h=128, q=FAKE, dqp=FAKE, dqb=big: f.mla_decode_lowbit_tc(
        ctypes.byref(d), bc, 4, 1, 1, q, 1, None, n_h, FAKE, FAKE, FAKE, 3, FAKE, 4, FAKE, 1,
        None, None, 0, FAKE, FAKE, FAKE, dqp, dqb, FAKE, 0, None)
    assert tc(bc=8) == 2
    assert tc(dqp=None) == 3 and tc(dqb=big - 1) == 3           # scratch pool too small
    assert tc(n_h=129) == 1 and tc(q=None) == 1
    assert tc(dqp=FAKE + 16) == 1                                 # pool not 256-byte aligned
    # everything else valid: a zero-byte workspace is refused before any launch
    assert tc() == 3


def test_wait_probe_rejects_bad_arguments(L):
    f = mla.lib()
    assert f.mla_debug_wait_probe(10, FAKE, None) == 1             # below 1 us
    assert f.mla_debug_wait_probe(10 ** 9, FAKE, None) == 1        # above 100 ms
    assert f.mla_debug_wait_probe(10 ** 6, None, None) == 1
    assert f.mla_debug_wait_probe(10 ** 6, FAKE + 2, None) == 1
