"""Device-side driver of one decode step through the libmla C ABI.

Uploads a workloads.DecodeInputs to the GPU once, then runs the hot path --
absorb_q, decode (+ split merge), the offline/online merge when the
workload has Local heads, and out_proj -- entirely in libmla kernels.
"""
from __future__ import annotations

import contextlib
import dataclasses
from typing import Optional

import numpy as np
import torch

from . import mla
from .workloads import DecodeInputs


def _dev(x: np.ndarray, dtype: torch.dtype, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype)


def _device_normal(shape, dtype: torch.dtype, device, seed: int) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.empty(shape, dtype=dtype, device=device)
    t.normal_(generator=g)
    return t


@dataclasses.dataclass
class DeviceProblem:
    dims: mla.Dims
    B: int
    s_q: int
    n_q: int
    H: int
    n_local: int
    local_ids: Optional[torch.Tensor]    # [n_local] int32 head ids of the Local heads
    global_ids: Optional[torch.Tensor]   # [H - n_local] int32 head ids of the Global heads
    n_ver: int
    deltas: list
    q_nope: torch.Tensor
    q_rope: torch.Tensor
    q_pos: torch.Tensor
    w_uk: torch.Tensor
    w_uv: torch.Tensor
    w_o: Optional[torch.Tensor]
    cache: torch.Tensor
    block_table: torch.Tensor
    segs: torch.Tensor
    gather_rows: Optional[torch.Tensor]
    n_gather: Optional[torch.Tensor]
    # outputs and scratch
    q_abs: torch.Tensor
    o_lat: torch.Tensor
    lse: torch.Tensor
    o_on: Optional[torch.Tensor]
    lse_on: Optional[torch.Tensor]
    o_off: Optional[torch.Tensor]
    lse_off: Optional[torch.Tensor]
    v: torch.Tensor
    out: torch.Tensor
    workspace: torch.Tensor


def upload(inp: DecodeInputs, device="cuda", with_out_proj=True,
           o_off: Optional[np.ndarray] = None, lse_off: Optional[np.ndarray] = None,
           device_cache_seed: Optional[int] = None) -> DeviceProblem:
    """Copy a workload's inputs to the device and allocate outputs.

    Weights and queries keep the workload's head order.  With Local heads,
    their ids are the first n_local entries of ``inp.head_order`` (a seeded
    permutation) or 0 .. n_local-1, and the Global heads are the rest; the
    decode and merge calls take those id lists.  ``o_off``/``lse_off`` are
    the offline partials, indexed by head id ([n_q, H, d_c] / [n_q, H]; only
    the Local heads' rows are read).  With ``device_cache_seed`` the cache is
    not copied from ``inp.pool`` (only its shape is used) but drawn N(0, 1) on
    the device from that seed, every row of every page (throughput runs of
    inputs made with ``draw_cache=False``).
    """
    wl = inp.wl
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    w_o = None
    if with_out_proj and inp.w_o is not None:
        w_o = _dev(inp.w_o, dt, device)
    local_ids = global_ids = None
    if wl.n_local:
        order = np.arange(wl.H) if inp.head_order is None else np.asarray(inp.head_order)
        local_ids = _dev(order[:wl.n_local].astype(np.int32), torch.int32, device)
        global_ids = _dev(order[wl.n_local:].astype(np.int32), torch.int32, device)
    dims = mla.make_dims(wl)
    n_q = inp.n_q
    n_ver = len(inp.deltas)
    row = wl.d_c + wl.d_r
    ws = mla.workspace_size(dims, wl.B, wl.s_q, wl.H, n_ver)
    prob = DeviceProblem(
        dims=dims, B=wl.B, s_q=wl.s_q, n_q=n_q, H=wl.H, n_local=wl.n_local,
        local_ids=local_ids, global_ids=global_ids, n_ver=n_ver,
        deltas=[int(d) for d in inp.deltas],
        q_nope=_dev(inp.q_nope, dt, device), q_rope=_dev(inp.q_rope, dt, device),
        q_pos=_dev(inp.q_pos, torch.int32, device),
        w_uk=_dev(inp.w_uk, dt, device), w_uv=_dev(inp.w_uv, dt, device), w_o=w_o,
        cache=(_dev(inp.pool, dt, device) if device_cache_seed is None
               else _device_normal(inp.pool.shape, dt, device, device_cache_seed)),
        block_table=_dev(inp.block_table, torch.int32, device),
        segs=_dev(inp.segs, torch.int32, device),
        gather_rows=None if inp.gather_rows is None else _dev(inp.gather_rows, torch.int32, device),
        n_gather=None if inp.n_gather is None else _dev(inp.n_gather, torch.int32, device),
        q_abs=torch.empty((n_ver, n_q, wl.H, row), dtype=dt, device=device),
        o_lat=torch.empty((n_q, wl.H, wl.d_c), dtype=torch.float32, device=device),
        lse=torch.empty((n_q, wl.H), dtype=torch.float32, device=device),
        o_on=None, lse_on=None, o_off=None, lse_off=None,
        v=torch.empty((n_q, wl.H, wl.d_v), dtype=torch.float32, device=device),
        out=torch.empty((n_q, max(wl.d_model, 1)), dtype=torch.float32, device=device),
        workspace=torch.empty(max(ws, 256), dtype=torch.uint8, device=device),
    )
    if wl.n_local:
        prob.o_on = torch.empty_like(prob.o_lat)
        prob.lse_on = torch.empty_like(prob.lse)
        prob.o_off = _dev(o_off, torch.float32, device)
        prob.lse_off = _dev(lse_off, torch.float32, device)
    return prob


@contextlib.contextmanager
def _nvtx(name: str):
    """An NVTX range around one C-ABI call (seen by nsys/ncu timelines)."""
    torch.cuda.nvtx.range_push(name)
    try:
        yield
    finally:
        torch.cuda.nvtx.range_pop()


def run_step(p: DeviceProblem, stream=None, out_proj: bool = True):
    """One pass of the hot path on ``stream``; results land in p.o_lat,
    p.lse, p.v and p.out."""
    with _nvtx("mla_absorb_q"):
        mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs, stream)
    run_decode(p, stream)
    if out_proj:
        with _nvtx("mla_out_proj"):
            mla.out_proj(p.dims, p.o_lat, p.w_uv, p.w_o, p.v,
                         p.out if p.w_o is not None else None, stream)


def run_decode(p: DeviceProblem, stream=None):
    """The attention part of a step (q_abs must be current): one decode call,
    or for Local/Global head splits the Global decode, the Local gathered
    decode and the offline/online merge."""
    if p.n_local:
        # Global heads: online over every row (prefix and relocated document)
        if p.H > p.n_local:
            with _nvtx("mla_decode global heads"):
                mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, p.global_ids, p.H - p.n_local,
                           p.cache, p.block_table, p.segs, p.q_pos, p.o_lat, p.lse,
                           p.workspace, stream=stream)
        # Local heads: protected rows online, merged with the offline partial
        with _nvtx("mla_decode local heads"):
            mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, p.local_ids, p.n_local, p.cache,
                       p.block_table, p.segs, p.q_pos, p.o_on, p.lse_on, p.workspace,
                       gather_rows=p.gather_rows, n_gather=p.n_gather, stream=stream)
        with _nvtx("mla_merge_lse"):
            mla.merge_lse(p.n_q, p.H, p.local_ids, p.n_local, p.dims.d_c, p.o_off, p.lse_off,
                          p.o_on, p.lse_on, p.o_lat, p.lse, stream)
    else:
        with _nvtx("mla_decode"):
            _decode_all(p, stream)


def _decode_all(p: DeviceProblem, stream=None):
    mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, None, p.H, p.cache, p.block_table, p.segs,
               p.q_pos, p.o_lat, p.lse, p.workspace, gather_rows=p.gather_rows,
               n_gather=p.n_gather, stream=stream)


def offline_partial(p: DeviceProblem, k_off: np.ndarray, stream=None):
    """The Local heads' MLA-Off partial on the device: their attention over the
    document rows that are not protected (``k_off`` [B, n_off] logical rows,
    each sequence's list sorted), written to p.o_off / p.lse_off by head id.
    RedKnot-MLA keeps this partial from an offline pass over the document;
    here the same decode call computes it for the current query, so that the
    online step merges a GPU-made partial.  q_abs must be current."""
    k_off = np.ascontiguousarray(k_off, np.int32)
    rows = torch.from_numpy(k_off).to(p.cache.device)
    n = torch.full((p.B,), k_off.shape[1], dtype=torch.int32, device=p.cache.device)
    if p.o_off is None:
        p.o_off = torch.empty_like(p.o_lat)
        p.lse_off = torch.empty_like(p.lse)
    with _nvtx("mla_decode offline partial"):
        mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, p.local_ids, p.n_local, p.cache,
                   p.block_table, p.segs, p.q_pos, p.o_off, p.lse_off, p.workspace,
                   gather_rows=rows, n_gather=n, stream=stream)
