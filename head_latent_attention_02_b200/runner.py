"""Device-side driver of one decode step through the libmla C ABI.

Uploads a workloads.DecodeInputs to the GPU once, then runs the hot path --
absorb_q, decode (+ split merge), the offline/online merge when the
workload has Local heads, and out_proj -- entirely in libmla kernels.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from . import mla
from .workloads import DecodeInputs


def _dev(x: np.ndarray, dtype: torch.dtype, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype)


@dataclasses.dataclass
class DeviceProblem:
    dims: mla.Dims
    B: int
    s_q: int
    n_q: int
    H: int
    n_local: int
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


def upload(inp: DecodeInputs, device="cuda", head_order=None, with_out_proj=True,
           o_off: Optional[np.ndarray] = None, lse_off: Optional[np.ndarray] = None
           ) -> DeviceProblem:
    """Copy a workload's inputs to the device and allocate outputs.

    ``head_order`` (optional permutation) stores head ``i`` of the device
    problem as logical head ``head_order[i]`` (weights, queries and W_O
    columns are permuted together, which leaves ``out`` unchanged); this is
    how a scattered Local/Global assignment is laid out with Local heads first.
    ``o_off``/``lse_off`` are the offline partials of the Local heads, in the
    device head order ([n_q, H, d_c] / [n_q, H]).
    """
    wl = inp.wl
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    order = np.arange(wl.H) if head_order is None else np.asarray(head_order)
    q_nope = inp.q_nope[:, order]
    q_rope = inp.q_rope[:, order]
    w_uk = inp.w_uk[order]
    w_uv = inp.w_uv[order]
    w_o = None
    if with_out_proj and inp.w_o is not None:
        cols = (order[:, None] * wl.d_v + np.arange(wl.d_v)[None, :]).reshape(-1)
        w_o = _dev(inp.w_o[:, cols], dt, device)
    dims = mla.make_dims(wl)
    n_q = inp.n_q
    n_ver = len(inp.deltas)
    row = wl.d_c + wl.d_r
    ws = mla.workspace_size(dims, wl.B, wl.s_q, wl.H)
    prob = DeviceProblem(
        dims=dims, B=wl.B, s_q=wl.s_q, n_q=n_q, H=wl.H, n_local=wl.n_local, n_ver=n_ver,
        deltas=[int(d) for d in inp.deltas],
        q_nope=_dev(q_nope, dt, device), q_rope=_dev(q_rope, dt, device),
        q_pos=_dev(inp.q_pos, torch.int32, device),
        w_uk=_dev(w_uk, dt, device), w_uv=_dev(w_uv, dt, device), w_o=w_o,
        cache=_dev(inp.pool, dt, device),
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


def run_step(p: DeviceProblem, stream=None, out_proj: bool = True):
    """One pass of the hot path on ``stream``; results land in p.o_lat,
    p.lse, p.v and p.out."""
    mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs, stream)
    run_decode(p, stream)
    if out_proj:
        mla.out_proj(p.dims, p.o_lat, p.w_uv, p.w_o, p.v, p.out if p.w_o is not None else None,
                     stream)


def run_decode(p: DeviceProblem, stream=None):
    """The attention part of a step (q_abs must be current): one decode call,
    or for Local/Global head splits the Global decode, the Local gathered
    decode and the offline/online merge."""
    if p.n_local:
        # Global heads: online over every row (prefix and relocated document)
        mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, p.n_local, p.H - p.n_local, p.cache,
                   p.block_table, p.segs, p.q_pos, p.o_lat, p.lse, p.workspace, stream=stream)
        # Local heads: protected rows online, merged with the offline partial
        mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, 0, p.n_local, p.cache, p.block_table,
                   p.segs, p.q_pos, p.o_on, p.lse_on, p.workspace, gather_rows=p.gather_rows,
                   n_gather=p.n_gather, stream=stream)
        mla.merge_lse(p.n_q, p.H, 0, p.n_local, p.dims.d_c, p.o_off, p.lse_off, p.o_on,
                      p.lse_on, p.o_lat, p.lse, stream)
    else:
        mla.decode(p.dims, p.B, p.s_q, p.q_abs, p.n_ver, 0, p.H, p.cache, p.block_table, p.segs,
                   p.q_pos, p.o_lat, p.lse, p.workspace, gather_rows=p.gather_rows,
                   n_gather=p.n_gather, stream=stream)
