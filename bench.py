"""Benchmark of the absorbed-MLA decode on B200 (libmla).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]
                    [--workload NAME] [--no-workloads] [--no-cpu-baseline]

A step is one pass of the whole hot path over one batch: absorb_q (W_UK and
the rotary query), decode over the paged latent cache (plan, split-KV
attention, split merge) and out_proj (W_UV then W_O), each call one CUDA
graph replayed in that order.  The workload is the B=16, H=128, 4096-row
bf16 decode (d_c=512, d_r=64, d_n=d_v=128, d_model=7168); inputs are
synthetic and seeded.  The metric is the decode call's latent-cache GB/s:
the 75.5 MB of cache rows it reads over its time, the median over the K
timed steps of CUDA events around it inside each step.  The whole step's
time and the other calls' medians are reported beside it, and (on one GPU)
the decode of the other configurations under ``workloads``.

Between steps the cache rotates over copies whose total exceeds twice the
126 MB L2 (and every step also streams the 235 MB W_O), so each decode reads
its cache from HBM.  Under torchrun every rank runs its own batch of 16
sequences (weak scaling, no collective on the data path); times are the max
over ranks.  ``--gpus N`` with N > 1 outside torchrun starts N ranks under
torchrun.  ``--impl reference`` times the fp64 CPU oracle on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "bf16_b16_4k"
METRIC = ("absorbed-MLA decode call (plan + attention + split merge): latent-cache GB/s "
          "(% of HBM peak) and µs at B=16, 4K")


def _peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


DECODE_PROFILE = os.path.join(ROOT, "profiles", "decode_b16_4k.md")
DECODE_SOURCES = ["head_latent_attention_02_b200/csrc/decode_tc.cuh",
                  "head_latent_attention_02_b200/csrc/mla_lib.cu"]


def _sources_sha1():
    import hashlib
    h = hashlib.sha1()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def decode_traffic():
    """DRAM bytes of one decode call (plan + attention + split merge) from the
    committed ncu summary, or None if the kernel sources changed since."""
    try:
        fields = {}
        for line in open(DECODE_PROFILE):
            if ":" in line and line.strip().startswith(("traffic_bytes", "sources_sha1")):
                k, v = line.strip().split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
        if fields.get("sources_sha1") != _sources_sha1():
            return None
        return int(fields["traffic_bytes"])
    except Exception:
        return None


def _cache_bytes(wl, rows_per_seq):
    return int(sum(rows_per_seq)) * (wl.d_c + wl.d_r) * 2


def decode_flops(wl, n_rows, n_gather=None):
    """Attention FLOPs of one step's decode calls: 2 * s_q * heads * rows *
    (d_c + d_r + d_c) -- the score over the 576-wide row and the weighted sum
    over the latent.  Global heads (all heads without a Local/Global split)
    attend every row of their sequence; Local heads attend the gathered rows."""
    per_row = 2 * wl.s_q * (2 * wl.d_c + wl.d_r)
    rows = int(np.sum(n_rows))
    if not wl.n_local:
        return per_row * wl.H * rows
    gathered = int(np.sum(n_gather)) if n_gather is not None else 0
    return per_row * ((wl.H - wl.n_local) * rows + wl.n_local * gathered)


def decode_roofline(flops, cache_bytes, t_dec_ms, peaks, src, traffic, kernel):
    """Roofline object of the decode call: against HBM (cache bytes / time)
    unless its arithmetic intensity is above the measured ridge (bf16 peak /
    HBM copy rate), then against the bf16 tensor peak (FLOPs / time)."""
    t = t_dec_ms * 1e-3
    intensity = flops / cache_bytes
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if intensity > ridge:
        achieved, peak, unit, bound = flops / t / 1e12, peaks["bf16_tflops"], "TFLOP/s", "tensor"
    else:
        achieved, peak, unit, bound = cache_bytes / t / 1e9, peaks["hbm_gbs"], "GB/s", "hbm"
    out = {"bound": bound, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
           "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": kernel,
           "peak_source": src, "flop_per_byte": round(intensity, 1),
           "ridge_flop_per_byte": round(ridge, 1)}
    # the nominal figure the target is stated against (8 TB/s HBM3e), beside
    # the measured copy rate
    out["frac_of_nominal_8tbs_hbm"] = round(cache_bytes / t / 1e9 / 8000.0, 4)
    return out


# ---------------------------------------------------------------- multi-rank
def max_over_ranks(values, device, world):
    """Element-wise max of per-rank times over all ranks: the job is as slow
    as its slowest replica.  All ranks must call it (it is a collective)."""
    import torch
    if world == 1:
        return [float(v) for v in values]
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def graph_kernel_count(graph, default):
    """Kernel nodes in a captured torch CUDA graph (the launches of one
    replay), or `default` if the graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as rt
        raw = rt.cudaGraph_t(init_value=int(graph.raw_cuda_graph()))
        err, _, n = rt.cudaGraphGetNodes(raw, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return default
        err, nodes, n = rt.cudaGraphGetNodes(raw, n)
        if err != rt.cudaError_t.cudaSuccess:
            return default
        kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes[:n]]
        return sum(1 for k in kinds if k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:
        return default


def job_throughput(bytes_per_rank, world, ms_per_step):
    """Whole-job GB/s when every rank streams its own batch (weak scaling)."""
    return bytes_per_rank * world / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML in a thread."""

    def __init__(self, index: int, period: float = 0.005):
        self.index, self.period = index, period
        self.samples = []
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self.ok = False
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def count(self, t0, t1):
        return sum(1 for s in self.samples if t0 <= s[0] <= t1)

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        nv = self._nv
        win = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples[-3:]
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
        }
        seen = sorted({n for _, _, r in win for n, bit in names.items() if r & bit})
        return {"sm_mhz": statistics.median([m for _, m, _ in win]) if win else None,
                "sm_max_mhz": self.max_mhz, "reasons": seen, "samples": len(win)}


# ---------------------------------------------------------------- GPU arm
L2_BYTES = 126 * 2 ** 20
EXTRA_WORKLOADS = ["bf16_varlen_b64", "redknot_56_8", "bf16_long_256k"]


def n_cache_copies(cache_bytes):
    """Copies of the cache to rotate over so that consecutive decode calls
    never find their rows in the 126 MB L2 (at least 3, total >= 2 x L2)."""
    return max(3, -(-2 * L2_BYTES // max(cache_bytes, 1)) + 1)


class Problem:
    """One workload on the device: the uploaded problem, its rotating cache
    copies and one CUDA graph per call (decode: one per cache copy)."""

    def __init__(self, name, rank, dev, stream):
        import torch

        from head_latent_attention_02_b200 import mla, runner
        from head_latent_attention_02_b200.workloads import WORKLOADS, make_inputs
        self.name = name
        wl = self.wl = WORKLOADS[name]
        # the cache is drawn on the device (seeded); nothing here is compared
        # with the oracle
        inp = self.inp = make_inputs(wl, seed=rank, poison=False, draw_cache=False)
        o_off = lse_off = None
        if wl.n_local:
            # the Local heads' offline (MLA-Off) partial is an input of the
            # step: synthetic normalised rows and log-sum-exp values
            g = np.random.default_rng([rank, 99])
            o_off = g.standard_normal((inp.n_q, wl.H, wl.d_c)).astype(np.float32) * 0.1
            lse_off = (g.standard_normal((inp.n_q, wl.H)) + 8.0).astype(np.float32)
        p = self.p = runner.upload(inp, device=dev, o_off=o_off, lse_off=lse_off,
                                   device_cache_seed=1000 + rank)
        # cache rows the decode reads: every sequence's rows, plus the
        # protected rows the Local heads re-read
        self.n_read = int(sum(inp.n_rows)) + (int(np.sum(inp.n_gather))
                                              if inp.n_gather is not None else 0)
        self.cache_bytes = self.n_read * (wl.d_c + wl.d_r) * 2
        self.n_copies = n_cache_copies(p.cache.numel() * p.cache.element_size())
        self.caches = [p.cache] + [p.cache.clone() for _ in range(self.n_copies - 1)]
        self.stream = stream
        self.mla, self.runner = mla, runner

        def dec(c):
            p.cache = self.caches[c]
            runner.run_decode(p)

        def capture(fn):
            gr = torch.cuda.CUDAGraph(keep_graph=True)   # keep_graph: nodes stay countable
            with torch.cuda.graph(gr):
                fn()
            gr.instantiate()
            return gr

        # eager warm-up (loads the kernels, sets attributes) before capture
        for c in range(self.n_copies):
            p.cache = self.caches[c]
            runner.run_step(p, stream=stream)
        torch.cuda.synchronize(dev)
        assert mla.get_status(stream) == 0
        self.g_abs = capture(lambda: mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas,
                                                  p.w_uk, p.q_abs))
        self.g_dec = [capture(lambda c=c: dec(c)) for c in range(self.n_copies)]
        self.g_out = capture(lambda: mla.out_proj(p.dims, p.o_lat, p.w_uv, p.w_o, p.v, p.out))
        self.kernels = {"absorb_q": graph_kernel_count(self.g_abs, 1),
                        "decode": graph_kernel_count(self.g_dec[0], 3),
                        "out_proj": graph_kernel_count(self.g_out, 2)}

    def steps(self, n, events=None):
        """n whole steps (absorb_q, decode, out_proj), each call its own graph
        replay; with ``events`` (a list) record four CUDA events per step:
        before absorb, before decode, after decode, after out_proj."""
        import torch
        for i in range(n):
            ev = None
            if events is not None:
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
                events.append(ev)
                ev[0].record(self.stream)
            self.g_abs.replay()
            if ev:
                ev[1].record(self.stream)
            self.g_dec[i % self.n_copies].replay()
            if ev:
                ev[2].record(self.stream)
            self.g_out.replay()
            if ev:
                ev[3].record(self.stream)

    def step_graphs(self, n):
        """n one-step CUDA graphs (absorb_q, decode over cache copy i % copies,
        out_proj), each with its own four timing events recorded inside the
        graph around the calls: a call's time is then its kernels' span on the
        device, with no graph-launch gap in it."""
        import torch
        p, mla, runner = self.p, self.mla, self.runner
        graphs, events = [], []
        for i in range(n):
            ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                ev[0].record()
                mla.absorb_q(p.dims, p.q_nope, p.q_rope, p.q_pos, p.deltas, p.w_uk, p.q_abs)
                ev[1].record()
                p.cache = self.caches[i % self.n_copies]
                runner.run_decode(p)
                ev[2].record()
                mla.out_proj(p.dims, p.o_lat, p.w_uv, p.w_o, p.v, p.out)
                ev[3].record()
            graphs.append(g)
            events.append(ev)
        return graphs, events

    def per_call_us(self, events):
        """Median over steps of each call's time (µs), from steps' events."""
        a = [e[0].elapsed_time(e[1]) * 1e3 for e in events]
        d = [e[1].elapsed_time(e[2]) * 1e3 for e in events]
        o = [e[2].elapsed_time(e[3]) * 1e3 for e in events]
        return {"absorb_q": statistics.median(a), "decode": statistics.median(d),
                "out_proj": statistics.median(o), "decode_min": min(d), "decode_max": max(d),
                "n": len(events)}

    def roofline(self, t_dec_us, peaks, src, traffic):
        wl, inp = self.wl, self.inp
        return decode_roofline(
            decode_flops(wl, inp.n_rows, inp.n_gather), self.cache_bytes, t_dec_us * 1e-3,
            peaks, src, traffic,
            "decode calls of the step (plan + decode_tc + combine"
            + (", twice, + merge_lse)" if wl.n_local else ")"))

    def _median_us(self, graphs, reps):
        """Median µs of single replays (CUDA events around each), rotating
        over ``graphs``."""
        import torch
        for i in range(3):
            graphs[i % len(graphs)].replay()
        ts = []
        for i in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(self.stream)
            graphs[i % len(graphs)].replay()
            b.record(self.stream)
            ts.append((a, b))
        torch.cuda.synchronize()
        assert self.mla.get_status(self.stream) == 0
        return statistics.median(x.elapsed_time(y) * 1e3 for x, y in ts)

    def _capture(self, fn):
        import torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    def qknorm_overhead(self, reps=20):
        """mla_decode_qknorm (one inverse-RMS factor per score column, read
        per page) against mla_decode on the same rows, both as decode-only
        graphs over the rotating cache copies."""
        import torch
        p, mla = self.p, self.mla
        n_rows = p.cache.shape[0] * p.cache.shape[1]
        g = torch.Generator(device=p.cache.device)
        g.manual_seed(7)
        key_inv = torch.rand(n_rows, generator=g, device=p.cache.device) + 0.5
        qk = [self._capture(lambda c=c: mla.decode_qknorm(
            p.dims, p.B, p.s_q, p.q_abs, p.n_ver, None, p.H, self.caches[c], key_inv,
            p.block_table, p.segs, p.q_pos, p.o_lat, p.lse, p.workspace))
            for c in range(self.n_copies)]
        t_plain = self._median_us(self.g_dec, reps)
        t_qk = self._median_us(qk, reps)
        del qk
        return {"decode_us": round(t_plain, 2), "qknorm_decode_us": round(t_qk, 2),
                "overhead_pct": round(100.0 * (t_qk / t_plain - 1.0), 2), "repeats": reps,
                "how": "decode-only graph replays, median of single replays"}

    def lowbit(self, reps=10):
        """mla_decode_lowbit over the rows packed as INT4/INT4 (288 B) and
        INT2/INT4 (160 B): µs and GB/s of packed rows read."""
        import torch
        p, mla, wl = self.p, self.mla, self.wl
        out = {}
        g = torch.Generator(device=p.cache.device)
        g.manual_seed(11)
        for bits_c, bits_r in ((4, 4), (2, 4)):
            row_bytes = (wl.d_c * bits_c + wl.d_r * bits_r) // 8
            lo = 0.3 if bits_c == 4 else 0.8
            sc = torch.rand(wl.d_c, generator=g, device=p.cache.device) * 0.3 + lo
            sr = torch.rand(wl.d_r, generator=g, device=p.cache.device) * 0.3 + 0.3
            n_rows = p.cache.shape[0] * p.cache.shape[1]
            n_copies = n_cache_copies(n_rows * row_bytes)
            packed = []
            for c in range(n_copies):
                src = self.caches[c % self.n_copies].view(n_rows, wl.d_c + wl.d_r)
                dst = torch.empty((p.cache.shape[0], p.cache.shape[1], row_bytes),
                                  dtype=torch.uint8, device=p.cache.device)
                mla.pack_rows(p.dims, bits_c, bits_r, src, sc, sr, dst.view(n_rows, row_bytes))
                packed.append(dst)
            gr = [self._capture(lambda c=c: mla.decode_lowbit(
                p.dims, bits_c, bits_r, p.B, p.s_q, p.q_abs, p.n_ver, None, p.H, packed[c], sc,
                sr, p.block_table, p.segs, p.q_pos, p.o_lat, p.lse)) for c in range(n_copies)]
            t = self._median_us(gr, reps)
            del gr
            # the tensor-core route: dequantise the whole packed pool into one
            # bf16 scratch pool, then the tensor-core decode over it
            dq = torch.empty(mla.lowbit_dequant_bytes(p.dims, p.cache.shape[0]),
                             dtype=torch.uint8, device=p.cache.device)
            gt = [self._capture(lambda c=c: mla.decode_lowbit_tc(
                p.dims, bits_c, bits_r, p.B, p.s_q, p.q_abs, p.n_ver, None, p.H, packed[c], sc,
                sr, p.block_table, p.segs, p.q_pos, p.o_lat, p.lse, dq, p.workspace))
                for c in range(n_copies)]
            t_tc = self._median_us(gt, reps)
            del gt, dq
            nbytes = self.n_read * row_bytes
            pool_bytes = n_rows * row_bytes
            out[f"int{bits_c}_int{bits_r}"] = {
                "row_bytes": row_bytes, "decode_us": round(t, 2), "packed_bytes": nbytes,
                "GB_s": round(nbytes / (t * 1e-6) / 1e9, 1),
                "frac_of_hbm": round(nbytes / (t * 1e-6) / 1e9 / _peaks()[0]["hbm_gbs"], 4),
                "kernel": "decode_lowbit_kernel (SIMT, one CTA per head and query row)",
                "tc_route_us": round(t_tc, 2),
                "tc_route": "dequant_rows_kernel over the whole packed pool ({:.1f} MB) into a "
                            "bf16 scratch pool, then the tensor-core decode".format(
                                pool_bytes / 1e6),
                "repeats": reps}
            del packed
        torch.cuda.empty_cache()
        return out

    def fold_gemm(self, reps=10):
        """The folded output projection (W_UV folded into W_O, out = o_lat
        [n_q, H d_c] x W_fold^T with W_fold [d_model, H d_c]) as a plain
        cuBLAS bf16 GEMM, against this library's two-GEMM out_proj call on
        the same rows.  Evidence for the design choice, not a product path:
        the folded weights are H d_c / (H d_v) = 4x the bytes of W_O."""
        import torch
        p, wl = self.p, self.wl
        try:
            K = wl.H * wl.d_c
            n_q = self.inp.n_q
            g = torch.Generator(device=p.cache.device)
            g.manual_seed(12)
            a = torch.randn(n_q, K, generator=g, device=p.cache.device).to(torch.bfloat16)
            w = torch.empty(wl.d_model, K, dtype=torch.bfloat16, device=p.cache.device)
            w.normal_(0.0, 0.01, generator=g)
            out = torch.empty(n_q, wl.d_model, dtype=torch.bfloat16, device=p.cache.device)
            for _ in range(3):
                torch.matmul(a, w.t(), out=out)
            ts = []
            for _ in range(reps):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(self.stream)
                torch.matmul(a, w.t(), out=out)
                e1.record(self.stream)
                ts.append((e0, e1))
            torch.cuda.synchronize()
            t_fold = float(np.median([x.elapsed_time(y) * 1e3 for x, y in ts]))
            t_two = self._median_us([self.g_out], reps)
            w_fold = w.numel() * 2
            w_two = (p.w_uv.numel() + p.w_o.numel()) * 2
            del a, w, out
            torch.cuda.empty_cache()
            return {"folded_gemm_us": round(t_fold, 2), "out_proj_us": round(t_two, 2),
                    "folded_weight_bytes": w_fold, "two_gemm_weight_bytes": w_two,
                    "folded_GB_s": round(w_fold / (t_fold * 1e-6) / 1e9, 1),
                    "folded_gemm": "torch.matmul (cuBLAS) bf16, [n_q, H*d_c] x [H*d_c, d_model]",
                    "repeats": reps}
        except Exception as e:   # a measurement of an alternative; never fails the run
            torch.cuda.empty_cache()
            return {"error": f"{type(e).__name__}: {e}"[:200]}

    def release(self):
        import torch
        del self.g_abs, self.g_dec, self.g_out, self.caches, self.p
        torch.cuda.empty_cache()


def measure_workload(name, rank, dev, stream, peaks, src, reps=20, qknorm=False):
    """Decode µs (median of ``reps`` steps), cache GB/s and roofline of one
    more workload on this GPU (with ``qknorm``, also the QK-normed decode's
    overhead on it)."""
    import torch
    prob = Problem(name, rank, dev, stream)
    graphs, ev = prob.step_graphs(reps)
    for g in graphs[:3]:
        g.replay()
    for g in graphs:
        g.replay()
    torch.cuda.synchronize(dev)
    assert prob.mla.get_status(stream) == 0
    t = prob.per_call_us(ev)
    del graphs
    out = {"decode_us": round(t["decode"], 2), "decode_us_min": round(t["decode_min"], 2),
           "repeats": reps, "cache_bytes": prob.cache_bytes,
           "GB_s": round(prob.cache_bytes / (t["decode"] * 1e-6) / 1e9, 1),
           "roofline": prob.roofline(t["decode"], peaks, src, None),
           "config": {"B": prob.wl.B, "H": prob.wl.H, "s_q": prob.wl.s_q,
                      "rows_total": int(sum(prob.inp.n_rows)),
                      "n_local_heads": prob.wl.n_local, "cache_copies": prob.n_copies}}
    if qknorm:
        out["qknorm"] = prob.qknorm_overhead()
    prob.release()
    return out


def run_gpu(args):
    import torch
    import torch.distributed as dist

    from head_latent_attention_02_b200 import build as hb, mla

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if rank == 0 or world == 1:
        hb.build()
    if world > 1:
        dist.barrier()
    mla.lib()
    peaks, src = _peaks()
    stream = torch.cuda.current_stream(dev)

    # clocks are sampled over the whole GPU section: set-up, warm-up, the
    # timed steps, the end-to-end steps and the other workloads
    with ClockSampler(local) as clk:
        t_gpu0 = time.perf_counter()
        prob = Problem(args.workload, rank, dev, stream)
        p = prob.p
        prob.steps(args.warmup)
        torch.cuda.synchronize(dev)
        assert mla.get_status(stream) == 0

        # --- device-timed region: exactly K steps, inputs resident in HBM.
        # One graph per step (up to 64, replayed in turn), each with timing
        # events inside it around its three calls.
        n_g = min(max(args.steps, 10), 64)
        graphs, g_events = prob.step_graphs(n_g)
        for g in graphs[:3]:
            g.replay()
        torch.cuda.synchronize(dev)
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        start.record(stream)
        for i in range(args.steps):
            graphs[i % n_g].replay()
        stop.record(stream)
        torch.cuda.synchronize(dev)
        t1 = time.perf_counter()
        if world > 1:
            dist.barrier()
        assert mla.get_status(stream) == 0
        ms_total = start.elapsed_time(stop)
        if args.steps < n_g:
            # fewer than 10 timed steps: every graph runs once more, so each
            # holds a step's times for the per-call medians
            for g in graphs[args.steps:]:
                g.replay()
            torch.cuda.synchronize(dev)
        per_call = prob.per_call_us(g_events)
        del graphs

        # --- end-to-end through the public API with host buffers: each step
        # copies its queries in from pinned memory and reads `out` back
        pin_qn = p.q_nope.cpu().pin_memory()
        pin_qr = p.q_rope.cpu().pin_memory()
        pin_qp = p.q_pos.cpu().pin_memory()
        pin_out = torch.empty_like(p.out, device="cpu").pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (pin_qn, pin_qr, pin_qp))
        d2h = pin_out.numel() * pin_out.element_size()

        def e2e_steps(n):
            for i in range(n):
                p.q_nope.copy_(pin_qn, non_blocking=True)
                p.q_rope.copy_(pin_qr, non_blocking=True)
                p.q_pos.copy_(pin_qp, non_blocking=True)
                p.cache = prob.caches[i % prob.n_copies]
                prob.runner.run_step(p, stream=stream)
                pin_out.copy_(p.out, non_blocking=True)

        e2e_steps(args.warmup)
        torch.cuda.synchronize(dev)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        s2.record(stream)
        e2e_steps(args.steps)
        e2.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = s2.elapsed_time(e2)
        assert mla.get_status(stream) == 0
        cache_bytes, wl, inp, kernels = prob.cache_bytes, prob.wl, prob.inp, prob.kernels
        n_copies = prob.n_copies
        variants = {}
        if world == 1 and not args.no_workloads and args.workload == WORKLOAD:
            variants["qknorm"] = prob.qknorm_overhead()
            variants["lowbit"] = prob.lowbit()
            variants["fold_value_into_output"] = prob.fold_gemm()
        prob.release()

        # --- the other configurations, decode only, on this GPU
        workloads = {}
        if world == 1 and not args.no_workloads and args.workload == WORKLOAD:
            for name in EXTRA_WORKLOADS:
                workloads[name] = measure_workload(name, rank, dev, stream, peaks, src,
                                                   qknorm=(name == "bf16_long_256k"))
        t_gpu1 = time.perf_counter()
    clocks = clk.summary(t_gpu0, t_gpu1)
    clocks["timed_window_samples"] = clk.count(t0, t1)

    t_dec_ms, ms_total, ms_e2e = max_over_ranks(
        [per_call["decode"] * 1e-3, ms_total, ms_e2e], dev, world)
    if world > 1:
        dist.barrier()

    if rank == 0:
        ms_step = ms_total / args.steps
        value = job_throughput(cache_bytes, world, t_dec_ms)
        e2e_val = job_throughput(cache_bytes, world, ms_e2e / args.steps)
        per_step_kernels = sum(kernels.values())
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_dec_ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) latents/queries, N(0,1/fan_in) weights)",
            "config": {"workload": args.workload, "B": wl.B, "H": wl.H,
                       "cached_rows_total": int(sum(inp.n_rows)),
                       "rows_per_sequence": (int(inp.n_rows[0]) if len(set(inp.n_rows)) == 1
                                             else f"{min(inp.n_rows)}..{max(inp.n_rows)}"),
                       "d_c": wl.d_c, "d_r": wl.d_r, "d_n": wl.d_n, "d_v": wl.d_v,
                       "d_model": wl.d_model, "page": 64, "s_q": wl.s_q,
                       "n_local_heads": wl.n_local,
                       "cache_bytes_per_step": cache_bytes,
                       "l2": f"cache rotates over {n_copies} copies "
                             f"({n_copies * cache_bytes / 1e6:.0f} MB) and each step streams "
                             f"W_O ({wl.d_model * wl.H * wl.d_v * 2 / 1e6:.0f} MB)",
                       "parallelism": f"replica x{world} (independent batches)"},
            "timing": ("value and ms_per_step: the decode call (plan + attention + split "
                       "merge), median over the timed steps of CUDA events recorded inside each "
                       "step's graph around the call (one graph per step: absorb_q, decode, "
                       "out_proj); step_ms: K graph replays between two events, divided by K"),
            "step_ms": round(ms_step, 5),
            "step_GB_s": round(job_throughput(cache_bytes, world, ms_step), 2),
            "breakdown_us": {"absorb_q": round(per_call["absorb_q"], 2),
                             "decode": round(per_call["decode"], 2),
                             "out_proj": round(per_call["out_proj"], 2),
                             "decode_min": round(per_call["decode_min"], 2),
                             "decode_max": round(per_call["decode_max"], 2),
                             "repeats": per_call["n"], "how": "median per call over the steps"},
            "roofline": decode_roofline(
                decode_flops(wl, inp.n_rows, inp.n_gather), cache_bytes, t_dec_ms, peaks, src,
                decode_traffic() if args.workload == WORKLOAD else None,
                "decode calls of the step (plan + decode_tc + combine"
                + (", twice, + merge_lse)" if wl.n_local else ")")),
            "clocks": clocks,
            "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "how": "whole step through the public API (H2D queries, absorb, decode, "
                           "out_proj, D2H out), cache bytes over the step time"},
            "gpu_launches": per_step_kernels * args.steps,
            "gpu_launches_note": f"{per_step_kernels} kernel nodes per step ({kernels})",
        }
        if workloads:
            line["workloads"] = workloads
        if variants:
            line["variants"] = variants
        if world == 1 and not args.no_cpu_baseline and args.workload == WORKLOAD:
            line["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def relaunch_under_torchrun(n):
    """`--gpus N` (N > 1) outside torchrun: run this script again as N ranks."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + sys.argv[1:]
    os.execv(sys.executable, cmd)


# ---------------------------------------------------------------- CPU arm
def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_sample_step(inp, n_seq, heads):
    from oracle import mla_oracle as O
    O.decode_absorbed_fast(inp, heads=heads, seqs=range(n_seq))


def cpu_baseline(seconds: float = 15.0, n_seq: int = 1, n_heads: int = 128):
    """The fp64 oracle (absorbed form) on a bounded sample of the workload."""
    from head_latent_attention_02_b200.workloads import WORKLOADS, make_inputs
    wl = WORKLOADS[WORKLOAD]
    inp = make_inputs(wl, seed=0, poison=False)
    heads = np.arange(n_heads)
    frac = n_seq * n_heads / (wl.B * wl.H)
    full_bytes = _cache_bytes(wl, inp.n_rows)
    reps, t = 0, 0.0
    t0 = time.perf_counter()
    while t < seconds:
        cpu_sample_step(inp, n_seq, heads)
        reps += 1
        t = time.perf_counter() - t0
    per = t / reps
    return {"value": round(frac * full_bytes / per / 1e9, 4), "unit": "GB/s",
            "cores": _cpu_threads(), "kind": "oracle",
            "sample": f"{n_seq} of {wl.B} sequences x {n_heads} of {wl.H} heads, fp64 absorbed "
                      f"form, {reps} reps in {t:.1f} s; GB/s scaled by the sampled fraction "
                      f"({frac:.4f}) of the step's cache bytes"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from head_latent_attention_02_b200.workloads import WORKLOADS, make_inputs
    wl = WORKLOADS[WORKLOAD]
    inp = make_inputs(wl, seed=0, poison=False)
    # per step: one sequence x 8 heads, so that W + K steps end within minutes
    n_seq, heads = 1, np.arange(8)
    frac = n_seq * len(heads) / (wl.B * wl.H)
    full_bytes = _cache_bytes(wl, inp.n_rows)
    for _ in range(args.warmup):
        cpu_sample_step(inp, n_seq, heads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cpu_sample_step(inp, n_seq, heads)
    dt = time.perf_counter() - t0
    ms_step = dt / args.steps * 1e3
    value = frac * full_bytes / (ms_step * 1e-3) / 1e9
    sample = (f"per step {n_seq} of {wl.B} sequences x {len(heads)} of {wl.H} heads (fp64 "
              f"absorbed oracle); GB/s scaled by the sampled fraction {frac:.5f}")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": wl.B, "H": wl.H, "cached_rows": 4096},
            "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": _cpu_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--workload", default=WORKLOAD,
                    help="bf16_b16_4k (default, the headline), bf16_varlen_b64, redknot_56_8, "
                         "bf16_long_256k")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the decode timings of the other configurations")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        relaunch_under_torchrun(args.gpus)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
