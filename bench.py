#!/usr/bin/env python
"""Decode-attention benchmark over a cross-layer-compressed KV cache (one JSON line).

A step is one decode step of every layer for every sequence of the workload: for the
selective xKV workloads, landmark scoring, chunk selection and reconstruct+attend per
layer; for dense reconstruction, reconstruct+attend; for R-CLA, the leader update and
attention per layer.  Layers run in order (a layer's query depends on the previous
layer's output in a real model).  Inputs are synthetic, seeded, generated on the device
before timing; the cache (bases, matrices, landmarks, leader caches) stays resident.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl cuda|reference]

With N > 1 (torchrun, one process per GPU) every rank runs its own replica of the
workload (sequences are independent: no collective on the data path); value is the
aggregate over ranks, timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn tokens/s (batch×steps) at 32K ctx; HBM GB/s vs 8 TB/s peak"
DEFAULT_WORKLOAD = "llama8b_sr_32k"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=16)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--batch", type=int, default=0,
                   help="override the workload's batch (smaller cases for profiling)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--path", choices=["explicit", "reassociated"], default="explicit",
                   help="xKV attention: explicit reconstruction (the method as the pages "
                        "state it) or its rank-space reassociation")
    p.add_argument("--scoring", choices=["fused", "separate"], default=None,
                   help="selective xKV: one fused scoring + selection call per layer "
                        "(xkv_score_select) or xkv_score_landmarks + xkv_select_chunks "
                        "(default: separate, the faster of the two here; fused when "
                        "--value-reserve is given, since reserved chunks go through it)")
    p.add_argument("--value-reserve", type=int, default=0,
                   help="selective xKV: also keep the N chunks of largest value range per "
                        "(sequence, KV head) (value-range-aware selection; the statistic and "
                        "the reserved chunks are built once, at setup)")
    p.add_argument("--layers", type=int, default=0,
                   help="run only the first N layers of the workload (small cases for "
                        "profiling; the reported config says so)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-graph", action="store_true",
                   help="launch every call directly instead of replaying a captured step")
    a = p.parse_args()
    if a.scoring is None:
        a.scoring = "fused" if a.value_reserve > 0 else "separate"
    return a


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def measured_tflops_sustained():
    """Dense bf16 rate of a GEMM timed inside a long loop (the power-capped figure)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured sustained"
    except Exception:
        return 1400.0, "fallback sustained"


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """This GPU's SM clock and clock-event (throttle) reasons, polled through NVML (the
    source nvidia-smi reads) every ~2 ms on a thread while the timed region runs, so a
    region of a few milliseconds still gets samples."""

    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40}

    def __init__(self, device_index: int):
        import torch
        self.nvml = None
        self.handle = None
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nvml = pynvml
        except Exception:
            self.nvml = None

    def _poll(self):
        nv, h = self.nvml, self.handle
        while not self.done.is_set():
            try:
                self.sm.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                self.mask |= nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                pass
            self.done.wait(0.002)

    def start(self):
        import threading
        self.sm, self.mask = [], 0
        if self.nvml is None:
            return
        self.done = threading.Event()
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.done.set()
        self.thread.join(timeout=5)
        self.thread = None
        if not self.sm:
            return None
        try:
            mx = self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
        except Exception:
            mx = max(self.sm)
        reasons = sorted(n for n, bit in self.REASONS.items() if self.mask & bit)
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": mx,
                "samples": len(self.sm), "reasons": reasons, "source": "nvml"}


# ------------------------------------------------------------------------ workloads
def _ra_kernels(w, n_sel):
    """Kernels of one rank-space attention call, following the library's launch plan: q~,
    the attention kernel, then the split merge and the projection, as one kernel when a
    head has 32 or more splits (dense calls at small batch), else as two.  Dense calls
    here take the head-batched kernel: one span of whole 128-token tiles per SM (148 spans)
    over the batch; selective calls split each unit's rows into items of <= 256 rows."""
    if n_sel == 0:
        tiles = -(-w.ctx_len // 128)
        ns = max(1, min(148 // w.batch, tiles))
        tps = -(-tiles // ns)
        n_split = -(-tiles // tps)
    else:
        n_split = -(-(n_sel * w.chunk) // 256)
        per = -(-n_sel // n_split)
        n_split = -(-n_sel // per)
    return 3 if n_split >= 32 else 4


class IoOverlap:
    """The host<->device copies of one end-to-end step, on a copy stream, overlapped with
    the layers: every layer's queries are issued at the start (after the copy stream has
    waited for the compute stream, so no copy overwrites a buffer the previous step still
    uses), each layer waits only for its own queries, and each layer's output is copied
    back as soon as the layer has run.  join() makes the compute stream wait for the last
    copy, so a timed region that ends on the compute stream covers every copy."""

    def __init__(self, q_host, q_dev, out_host, out_dev, copy_stream):
        import torch
        self.torch = torch
        self.cur, self.cs = torch.cuda.current_stream(), copy_stream
        self.out_host, self.out_dev = out_host, out_dev
        start = torch.cuda.Event()
        start.record(self.cur)
        self.cs.wait_event(start)
        self.ins = []
        with torch.cuda.stream(self.cs):
            for l in range(q_dev.shape[0]):
                q_dev[l].copy_(q_host[l], non_blocking=True)
                e = torch.cuda.Event()
                e.record(self.cs)
                self.ins.append(e)

    def before(self, l):
        self.cur.wait_event(self.ins[l])

    def after(self, l):
        e = self.torch.cuda.Event()
        e.record(self.cur)
        self.cs.wait_event(e)
        with self.torch.cuda.stream(self.cs):
            self.out_host[l].copy_(self.out_dev[l], non_blocking=True)

    def join(self):
        e = self.torch.cuda.Event()
        e.record(self.cs)
        self.cur.wait_event(e)


class XkvStep:
    """Device-resident xKV workload (selective or dense) and its decode step."""

    def __init__(self, w, seed, dev, path="explicit", scoring="fused", value_reserve=0):
        import torch
        from cross_layer_compressed_b200 import synth
        from cross_layer_compressed_b200 import xkv
        self.w, self.dev, self.xkv = w, dev, xkv
        self.path = path
        self.scoring = scoring
        self.d = xkv.dims_of(w)
        self.cache = synth.torch_xkv_cache(w, seed, device=dev)
        dt = self.cache["Ak"].dtype
        self.dense = w.mode == "dense"
        self.lm = None
        if not self.dense:
            self.lm = torch.empty((w.n_layers, w.batch, w.n_kv_heads, w.n_chunks, w.head_dim),
                                  dtype=dt, device=dev)
            for l in range(w.n_layers):
                xkv.xkv_build_landmarks(self.d, self.cache["Ak"][l // w.window],
                                        self.cache["Bkt"][l], self.lm[l])
        self.qpool = synth.torch_queries(w, seed, self.cache, device=dev)   # [nq][N][B][Hq][hd]
        self.n_sel = 0 if self.dense else w.n_sel
        # value-range-aware selection: per layer the statistic and the reserved chunks,
        # built once (setup, timed apart from the step)
        self.reserved, self.n_res, self.setup_value_ms = None, 0, None
        if value_reserve and not self.dense:
            assert scoring == "fused", "reserved chunks go through the fused selection"
            self.n_res = xkv.xkv_n_reserved(w.n_chunks, value_reserve, w.n_sink, w.n_recent)
            rho = torch.empty((w.batch, w.n_kv_heads, w.n_chunks), dtype=torch.float32,
                              device=dev)
            self.reserved = torch.empty((w.n_layers, w.batch, w.n_kv_heads, self.n_res),
                                        dtype=torch.int32, device=dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for l in range(w.n_layers):
                xkv.xkv_build_value_ranges(self.d, self.cache["Av"][l // w.window],
                                           self.cache["Bvt"][l], rho)
                xkv.xkv_reserve_value_chunks(self.d, rho, value_reserve, w.n_sink, w.n_recent,
                                             self.reserved[l])
            e1.record()
            torch.cuda.synchronize()
            self.setup_value_ms = e0.elapsed_time(e1)
            base = xkv.xkv_n_selected(w.n_chunks, 0, w.n_sink, w.n_recent)
            self.n_sel = base + self.n_res + min(w.top_k, w.n_chunks - base - self.n_res)
        mode = xkv.XKV_MODE_DENSE if self.dense else xkv.XKV_MODE_SELECTIVE
        if path == "reassociated":
            mode = xkv.XKV_MODE_REASSOC
        self.ws = torch.empty(xkv.xkv_workspace_bytes(self.d, self.n_sel, mode),
                              dtype=torch.uint8, device=dev)
        self.attend = (xkv.xkv_reassociated_attend if path == "reassociated"
                       else xkv.xkv_reconstruct_attend)
        self.scores = torch.empty((w.batch, w.n_kv_heads, max(w.n_chunks, 1)),
                                  dtype=torch.float64, device=dev)
        self.ws_select = None
        if not self.dense and scoring == "fused":
            self.ws_select = torch.empty(xkv.xkv_score_select_workspace_bytes(self.d),
                                         dtype=torch.uint8, device=dev)
        self.sel = torch.empty((w.n_layers, w.batch, w.n_kv_heads, max(self.n_sel, 1)),
                               dtype=torch.int32, device=dev)
        self.out = torch.empty((w.n_layers, w.batch, w.n_q_heads, w.head_dim),
                               dtype=torch.float32, device=dev)
        self.q_in = torch.empty_like(self.qpool[0])   # e2e: per-step queries land here
        # our kernels per layer: the fused selection's key and selection grids (or score,
        # select), then status clear + attention + split merge (explicit) or q~ +
        # attention + merge-and-projection (reassociated; q~ clears the status word)
        n_sel_kernels = 0 if self.dense else 2
        n_attn = _ra_kernels(w, self.n_sel) if path == "reassociated" else 3
        self.launches_per_step = w.n_layers * (n_sel_kernels + n_attn)
        torch.cuda.synchronize()

    def resident_bytes(self):
        n = sum(t.numel() * t.element_size() for t in self.cache.values())
        if self.lm is not None:
            n += self.lm.numel() * self.lm.element_size()
        return n

    def step(self, slot=None, q=None, attend_events=None, select_events=None, io=None):
        """One decode step over all layers; io = (q_host, out_host, copy_stream) runs it
        from host buffers with the copies overlapped (IoOverlap)."""
        w, xkv, d = self.w, self.xkv, self.d
        ov = IoOverlap(io[0], self.q_in, io[1], self.out, io[2]) if io is not None else None
        qq = self.q_in if ov is not None else (self.qpool[slot] if q is None else q)
        for l in range(w.n_layers):
            win = l // w.window
            if ov is not None:
                ov.before(l)
            if not self.dense:
                if select_events is not None:
                    select_events[l][0].record()
                if self.scoring == "fused":
                    xkv.xkv_score_select(d, self.lm[l], qq[l], w.top_k, w.n_sink, w.n_recent,
                                         self.sel[l], self.ws_select,
                                         reserved=None if self.reserved is None
                                         else self.reserved[l], n_reserved=self.n_res)
                else:
                    xkv.xkv_score_landmarks(d, self.lm[l], qq[l], self.scores)
                    xkv.xkv_select_chunks(d, self.scores, w.top_k, w.n_sink, w.n_recent,
                                          self.sel[l])
                if select_events is not None:
                    select_events[l][1].record()
            if attend_events is not None:
                attend_events[l][0].record()
            self.attend(d, self.cache["Ak"][win], self.cache["Av"][win], self.cache["Bkt"][l],
                        self.cache["Bvt"][l], qq[l], None if self.dense else self.sel[l],
                        self.n_sel, self.out[l], self.ws)
            if attend_events is not None:
                attend_events[l][1].record()
            if ov is not None:
                ov.after(l)
        if ov is not None:
            ov.join()

    def attend_bytes(self, slots):
        """Algorithmic bytes of each reconstruct+attend launch (per layer), averaged over
        the query slots used: the union over KV heads of the selected rows of A^K and A^V
        per sequence, B_l (K and V), the selection, q and out."""
        import torch
        w = self.w
        e = self.cache["Ak"].element_size()
        per_launch = []
        for slot in slots:
            self.step(slot)                    # recompute this slot's selections (untimed)
            torch.cuda.synchronize()
            for l in range(w.n_layers):
                if self.dense:
                    rows = w.batch * w.ctx_len
                else:
                    mask = torch.zeros((w.batch, w.n_chunks), dtype=torch.bool, device=self.dev)
                    mask.scatter_(1, self.sel[l].reshape(w.batch, -1).long(), True)
                    rows = int(mask.sum().item()) * w.chunk
                nbytes = (rows * (w.rank_k + w.rank_v) * e
                          + w.batch * w.d_kv * (w.rank_k + w.rank_v) * e
                          + w.batch * w.n_q_heads * w.head_dim * (e + 4)
                          + (0 if self.dense else w.batch * w.n_kv_heads * self.n_sel * 4))
                per_launch.append(nbytes)
        return float(np.mean(per_launch))

    def attend_flops(self):
        """Tensor-core flops of one explicit attention launch: the two reconstruction
        GEMMs over the attended rows plus q.K_hat and p.V_hat (dense mode: every row)."""
        w = self.w
        rows = w.ctx_len if self.dense else self.n_sel * w.chunk
        return (2.0 * w.batch * w.n_kv_heads * rows * w.head_dim * (w.rank_k + w.rank_v)
                + 4.0 * w.batch * w.n_q_heads * rows * w.head_dim)

    def step_bytes(self, attend_bytes_per_launch):
        w = self.w
        e = self.cache["Ak"].element_size()
        lm = 0 if self.dense else w.batch * w.n_kv_heads * w.n_chunks * w.head_dim * e
        sc = 0 if self.dense else w.batch * w.n_kv_heads * w.n_chunks * 8 * 2
        return w.n_layers * (attend_bytes_per_launch + lm + sc)

    def io_bytes(self):
        w = self.w
        return (self.q_in.numel() * self.q_in.element_size(),
                self.out.numel() * self.out.element_size())


class RclaStep:
    """Device-resident R-CLA workload and its decode step (leaders append, then attend)."""

    def __init__(self, w, seed, dev):
        import torch
        from cross_layer_compressed_b200 import synth
        from cross_layer_compressed_b200 import xkv
        self.w, self.dev, self.xkv = w, dev, xkv
        self.d = xkv.dims(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.L_max, dtype=w.dtype)
        c = synth.torch_rcla_cache(w, seed, device=dev)
        self.K, self.V, self.kn, self.vn = c["K_lead"], c["V_lead"], c["k_new"], c["v_new"]
        self.S = synth.leader_set(w)
        self.lo = [max(s for s in self.S if s <= l) for l in range(w.n_layers)]
        self.qpool = synth.torch_queries(w, seed, None, device=dev)
        self.ws = torch.empty(xkv.xkv_workspace_bytes(self.d, 0, xkv.XKV_MODE_RCLA),
                              dtype=torch.uint8, device=dev)
        self.out = torch.empty((w.n_layers, w.batch, w.n_q_heads, w.head_dim),
                               dtype=torch.float32, device=dev)
        self.q_in = torch.empty_like(self.qpool[0])
        self.len = w.ctx_len
        self.launches_per_step = w.n_layers * 2
        self.step_index = 0
        torch.cuda.synchronize()

    def resident_bytes(self):
        return 2 * self.K.numel() * self.K.element_size()

    def step(self, slot=None, q=None, attend_events=None, select_events=None, io=None):
        w, xkv = self.w, self.xkv
        ov = IoOverlap(io[0], self.q_in, io[1], self.out, io[2]) if io is not None else None
        qq = self.q_in if ov is not None else (self.qpool[slot] if q is None else q)
        # cache length cycles within the capacity so every step does the same work
        length = w.ctx_len + (self.step_index % max(w.extra_rows, 1))
        self.step_index += 1
        ns = slot if slot is not None else 0
        for l in range(w.n_layers):
            leader = self.lo[l] == l
            si = self.S.index(self.lo[l])
            if ov is not None:
                ov.before(l)
            if attend_events is not None:
                attend_events[l][0].record()
            xkv.rcla_decode_attend(self.d, l, self.lo, self.K, self.V, w.L_max,
                                   length if leader else length + 1,
                                   self.kn[ns, si] if leader else None,
                                   self.vn[ns, si] if leader else None, qq[l], self.out[l],
                                   self.ws)
            if attend_events is not None:
                attend_events[l][1].record()
            if ov is not None:
                ov.after(l)
        if ov is not None:
            ov.join()

    def attend_bytes(self, slots):
        w = self.w
        e = self.K.element_size()
        rows = w.ctx_len + 1
        per_layer = []
        for l in range(w.n_layers):
            leader = self.lo[l] == l
            b = (w.batch * w.n_kv_heads * rows * w.head_dim * 2 * e
                 + w.batch * w.n_q_heads * w.head_dim * (e + 4)
                 + (w.batch * w.n_kv_heads * w.head_dim * 2 * e * 2 if leader else 0))
            per_layer.append(b)
        return float(np.mean(per_layer))

    def step_bytes(self, attend_bytes_per_launch):
        return self.w.n_layers * attend_bytes_per_launch

    def io_bytes(self):
        return (self.q_in.numel() * self.q_in.element_size(),
                self.out.numel() * self.out.element_size())


# --------------------------------------------------------------------- CPU baseline
def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def host_cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _run_units(fn, n_units, threads):
    """Runs fn(i) for i < n_units on `threads` host threads (the oracle's C calls release
    the interpreter lock, so the threads run on separate cores); returns the wall time."""
    from concurrent.futures import ThreadPoolExecutor
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fn, range(n_units)))
    return time.perf_counter() - t0


def cpu_baseline(w, seed, budget_s=20.0):
    """The oracle, as it stands, on a bounded sample of one decode step, run on every host
    core: independent (sequence, KV head) units of one layer go to a pool of one thread
    per core, and the step time is extrapolated from the units finished per second."""
    import torch
    import oracle
    from cross_layer_compressed_b200 import synth
    oracle.build()
    cores = host_cores()
    G = w.n_q_heads // w.n_kv_heads
    if w.mode == "rcla":
        wl = synth.reduced(w, batch=1, n_layers=1, ctx_len=w.ctx_len, extra_rows=1)
        x = synth.np_rcla_inputs(wl, seed, len_rows=w.ctx_len)
        K = x["K_lead"].view(torch.int16).numpy().view(np.uint16)
        V = x["V_lead"].view(torch.int16).numpy().view(np.uint16)
        heads = [(np.ascontiguousarray(K[:, :, g:g + 1]), np.ascontiguousarray(V[:, :, g:g + 1]),
                  x["k_new"][0][:, g:g + 1].contiguous(), x["v_new"][0][:, g:g + 1].contiguous(),
                  x["q"][0][:, g * G:(g + 1) * G].contiguous()) for g in range(w.n_kv_heads)]

        def unit(i):
            Kg, Vg, kn, vn, qg = heads[i % w.n_kv_heads]
            oracle.rcla_decode_attend(0, [0], Kg.copy(), Vg.copy(), w.ctx_len, kn, vn, qg)
        what = "leader update + attention of one (sequence, KV head)"
    else:
        rng = np.random.default_rng(seed)
        wl = synth.reduced(w, batch=1, n_layers=1, ctx_len=w.ctx_len, n_needles=0)
        Ak = synth.to_storage(synth.np_basis(wl, seed, 0, 0, "k")[None], w.dtype)
        Av = synth.to_storage(synth.np_basis(wl, seed, 0, 0, "v")[None], w.dtype)
        Bkt = synth.to_storage(synth.np_recon_t(wl, seed, 0, 0, "k")[None], w.dtype)
        Bvt = synth.to_storage(synth.np_recon_t(wl, seed, 0, 0, "v")[None], w.dtype)
        q = synth.to_storage(synth.np_queries(wl, seed, 0, 0), w.dtype)
        lm = synth.to_storage(rng.standard_normal((1, w.n_kv_heads, w.n_chunks, w.head_dim))
                              * 1e-2, w.dtype) if w.mode != "dense" else None

        def unit(i):
            g = i % w.n_kv_heads
            sel = None
            if lm is not None:
                s = oracle.score_landmarks(lm[:, g:g + 1].contiguous(),
                                           q[:, g * G:(g + 1) * G].contiguous())
                sel = np.zeros((1, w.n_kv_heads, w.n_sel), dtype=np.int32)
                sel[:, g:g + 1] = oracle.select_chunks(s, w.top_k, w.n_sink, w.n_recent)
            oracle.reconstruct_attend(Ak, Av, Bkt, Bvt, q, sel, w.chunk, units=[(0, g)])
        what = ("scoring + selection + reconstruct-attend of one (sequence, KV head)"
                if w.mode != "dense" else "dense reconstruct-attend of one (sequence, KV head)")
    # one unit alone sizes the sample: as many units per core as fit the budget
    t1 = _run_units(unit, 1, 1)
    per_core = max(1, min(32, int(budget_s / max(t1, 1e-3) / 2)))
    n_units = cores * per_core
    wall = _run_units(unit, n_units, cores) if t1 < budget_s else t1
    if t1 >= budget_s:
        n_units, used = 1, 1
    else:
        used = cores
    units_per_s = n_units / wall
    step_units = w.batch * w.n_layers * w.n_kv_heads
    step_s = step_units / units_per_s
    sample = (f"{n_units} units ({what}; full-size rows, one layer's factors) on {used} host "
              f"threads of {cores} cores ({host_cpu_model()}): {units_per_s:.3g} units/s, "
              f"extrapolated to the {step_units} units of a {w.batch}-sequence x "
              f"{w.n_layers}-layer step")
    return {"value": w.batch / step_s, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": sample, "sample_seconds": round(wall, 3), "host_cores": cores,
            "cpu_model": host_cpu_model()}


def reference_arm(args, w, rank, world):
    """--impl reference: the oracle on the host cores, one bounded sample per step."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    budget = max(0.5, min(10.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(w, args.seed, budget_s=budget)
    vals, secs = [], []
    for _ in range(args.steps):
        r = cpu_baseline(w, args.seed, budget_s=budget)
        vals.append(r["value"])
        secs.append(r["sample_seconds"])
    v = float(np.mean(vals))
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * w.batch / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "batch": w.batch, "ctx_len": w.ctx_len,
                       "n_layers": w.n_layers},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": r["cores"],
                             "kind": "oracle", "sample": r["sample"],
                             "cpu_model": r["cpu_model"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def profiled_traffic(workload: str, kernel: str, source: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and workload,
    or None when there is none or the kernel's source changed since the capture."""
    import glob
    import hashlib
    src = os.path.join(ROOT, "cross_layer_compressed_b200", "csrc", source)
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    for path in glob.glob(os.path.join(ROOT, "profiles", f"{kernel}_{workload}*.md")):
        fields = {}
        for line in open(path):
            if ":" in line and not line.startswith(" "):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
        key = f"traffic_bytes_per_launch_{workload}"
        if fields.get("source_sha256_prefix") == sha and key in fields:
            return float(fields[key])
    return None


def count_kernel_nodes(g):
    """Kernel nodes of a captured CUDA graph (every kernel one replay launches), or None
    when the graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as rt
        h = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(h, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(h, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kern = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
        return sum(1 for nd in nodes[:n] if rt.cudaGraphNodeGetType(nd)[1] == kern)
    except Exception:
        return None


# ------------------------------------------------------------------ rank aggregation
def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank number over all ranks (the timed region's length)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(batch_per_rank: int, steps: int, world: int,
                           max_elapsed_ms: float) -> float:
    """Whole-job throughput: every rank decodes its own batch (weak scaling)."""
    return world * batch_per_rank * steps / (max_elapsed_ms / 1e3)


# --------------------------------------------------------------------------- driver
# ------------------------------------------------- cross-layer factorization (prefill)
# One window of the Llama-3.1-8B-shaped 32K workload: W = 4 layers, 8 sequences, L =
# 32768, d_kv = 8 x 128, ranks 512 (K) and 768 (V), 2 power passes.  A step factorizes
# the window's K caches and its V caches for every sequence.
CLF_WORKLOAD = "llama8b_clf_32k"
CLF = dict(window=4, batch=8, ctx_len=32768, n_kv_heads=8, head_dim=128, rank_k=512,
           rank_v=768, n_iter=2, tau=128.0, gap=0.1)
CLF_METRIC = ("prefill cross-layer factorization tokens/s (window of 4 layers, K and V "
              "caches, 32K ctx)")
# The same window after 256 generated tokens: the tail folded back into the factors.
REFOLD_WORKLOAD = "llama8b_refold_32k"
REFOLD_TAIL = 256
REFOLD_METRIC = ("tail refold tokens/s (window of 4 layers, K and V caches, 32K compressed "
                 "+ 256 generated rows)")
# fp64 FMA peak of the CUDA cores: 148 SMs x 64 fp64 FMA per clock x 2 flop x 1.965 GHz
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12
TF32_OVER_BF16 = 1.1 / 2.25                      # nominal dense tf32 : bf16 ratio


def clf_work(c, r):
    """Work of one bf16 factorization call of rank r, by arithmetic unit, and its launch
    counts.  Passes of CholeskyQR: the first and intermediate bases one each, the final
    basis two; every pass is a Gram matrix (fp64), a blocked Cholesky and inverse, and a
    product with R^-1 (TF32)."""
    B, L, q, W = c["batch"], c["ctx_len"], c["n_iter"], c["window"]
    n = W * c["n_kv_heads"] * c["head_dim"]
    KB = (r + 63) // 64
    y_pass = 2 if q == 0 else 1 + q + 1          # passes over L-row bases
    z_pass = q                                   # passes over n-row bases
    pass_rows = y_pass * L + z_pass * n
    bf16 = 2 * B * L * r * n * (1 + 4 * q + 2)   # X products: test matrix 1 part, others hi+lo
    tf32 = 2 * B * r * r * pass_rows
    fp64 = B * r * (r + 1) * pass_rows           # Gram matrices: r(r+1)/2 dot products
    # products (the library's own GEMM kernel): X Omega, per iteration X^T Q and X Z, the
    # final X^T Q, and one product with R^-1 per CholeskyQR pass
    gemm = 1 + 2 * q + 1 + (y_pass + z_pass)
    own = (2 + 2 * q) + 2 + (y_pass + z_pass) * 4 * KB + gemm
    return {"bf16": bf16, "tf32": tf32, "fp64": fp64, "own_launches": own,
            "gemm_launches": gemm}


def clf_cpu_baseline(c, seed, rows=2048):
    """The oracle (LAPACK SVD in fp64, one BLAS thread) on one sequence's K window cut
    to `rows` tokens; tokens/s counts K and V (two factorizations per token)."""
    import oracle
    from cross_layer_compressed_b200 import synth
    from threadpoolctl import threadpool_limits
    dk = c["n_kv_heads"] * c["head_dim"]
    X, _ = synth.np_window_caches(c["window"], 1, rows, dk, c["rank_k"] + 64, c["rank_k"],
                                  c["tau"], c["gap"], seed)
    Xq = synth.to_storage(X, "bf16").double().numpy()
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        oracle.factorize_window(Xq, c["rank_k"])
        dt = time.perf_counter() - t0
    return {"value": rows / (2 * dt), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"1 sequence x {rows} tokens of the K window (W = {c['window']}, "
                      f"d_kv = {dk}, exact SVD), counted twice for K and V",
            "sample_seconds": round(dt, 3)}


def run_clf(args, rank, world):
    import torch
    import torch.distributed as dist
    from cross_layer_compressed_b200 import build, synth
    c = dict(CLF)
    if args.batch:
        c["batch"] = args.batch
    refold = args.workload == REFOLD_WORKLOAD
    T = REFOLD_TAIL if refold else 0
    name, metric = (REFOLD_WORKLOAD, REFOLD_METRIC) if refold else (CLF_WORKLOAD, CLF_METRIC)
    if args.impl == "reference":
        if rank != 0:
            return
        for _ in range(args.warmup):
            clf_cpu_baseline(c, args.seed, rows=512)
        vals = [clf_cpu_baseline(c, args.seed) for _ in range(args.steps)]
        v = float(np.mean([x["value"] for x in vals]))
        line = {"metric": metric, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * c["batch"] * c["ctx_len"] / v, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "impl": "reference", "config": {"workload": name, **c, "n_tail": T},
                "cpu_baseline": {**vals[-1], "value": v},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    assert args.warmup >= 3 or os.environ.get("XKV_BENCH_ALLOW_SHORT"), "need >= 3 warm-up steps"
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    dev = torch.device("cuda", torch.cuda.current_device())
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    build.build()
    from cross_layer_compressed_b200 import xkv
    W, B, L = c["window"], c["batch"], c["ctx_len"]
    dk = c["n_kv_heads"] * c["head_dim"]
    n = W * dk
    d = xkv.dims(B, c["n_kv_heads"], c["n_kv_heads"], c["head_dim"], L, dtype="bf16")
    seed = args.seed + 1000 * rank
    calls = []
    for which, r in (("k", c["rank_k"]), ("v", c["rank_v"])):
        X, _ = synth.torch_window_caches(W, B, L + T, dk, r + 64, r, c["tau"], c["gap"], "bf16",
                                         seed + (0 if which == "k" else 1), device=dev)
        om = torch.from_numpy(synth.np_test_matrix(n, r, seed)).to(dev)
        A = torch.empty((B, L + T, r), dtype=torch.bfloat16, device=dev)
        Bt = torch.empty((W, B, dk, r), dtype=torch.bfloat16, device=dev)
        k = dict(r=r, X=X, om=om, A=A, Bt=Bt)
        if refold:
            # the window as the decode loop holds it: L rows in factors, T generated rows
            k["X"] = X[:, :, :L].contiguous()
            k["tail"] = X[:, :, L:].contiguous()
            del X
            k["A0"] = torch.empty((B, L, r), dtype=torch.bfloat16, device=dev)
            k["Bt0"] = torch.empty((W, B, dk, r), dtype=torch.bfloat16, device=dev)
            wsf = torch.empty(xkv.xkv_factorize_workspace_bytes(d, W, r), dtype=torch.uint8,
                              device=dev)
            xkv.xkv_factorize_window(d, W, r, k["X"], om, c["n_iter"], k["A0"], k["Bt0"], wsf)
            torch.cuda.synchronize(dev)
            del wsf
        calls.append(k)
    ws = torch.empty(max(xkv.xkv_refold_workspace_bytes(d, W, k["r"], T) if refold else
                         xkv.xkv_factorize_workspace_bytes(d, W, k["r"]) for k in calls),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(events=None, only=None):
        for i, k in enumerate(calls):
            if only is not None and i != only:
                continue
            if events is not None:
                events[i][0].record(stream)
            torch.cuda.nvtx.range_push("xkv_factorize")    # lets a profiler skip the setup
            if refold:
                xkv.xkv_refold_window(d, W, k["r"], k["A0"], k["Bt0"], k["tail"], T, k["om"],
                                      c["n_iter"], k["A"], k["Bt"], ws)
            else:
                xkv.xkv_factorize_window(d, W, k["r"], k["X"], k["om"], c["n_iter"], k["A"],
                                         k["Bt"], ws)
            torch.cuda.nvtx.range_pop()
            if events is not None:
                events[i][1].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    clocks = ClockSampler(dev.index)
    barrier()
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    barrier()
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    # per call, CUDA events on the launching stream
    per_call = [[], []]
    for _ in range(args.steps):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in calls]
        step(ev)
        barrier()
        for i in range(len(calls)):
            per_call[i].append(ev[i][0].elapsed_time(ev[i][1]))
    call_ms = [float(np.mean(p)) for p in per_call]
    # end to end: the caches (refold: the generated rows) from pinned host memory, the
    # factors back to the host
    e2e = None
    src = "tail" if refold else "X"
    if not args.no_e2e:
        hx = [torch.empty(k[src].shape, dtype=k[src].dtype, pin_memory=True) for k in calls]
        for h, k in zip(hx, calls):
            h.copy_(k[src].cpu())
        ha = [torch.empty(k["A"].shape, dtype=k["A"].dtype, pin_memory=True) for k in calls]
        hb = [torch.empty(k["Bt"].shape, dtype=k["Bt"].dtype, pin_memory=True) for k in calls]

        copy_stream = torch.cuda.Stream(dev)

        def e2e_step():
            # both calls' inputs cross on a copy stream (the V caches while the K call
            # runs), each call waits only for its own, and its factors go back as soon as
            # it is done; the step ends joined to the copy stream
            start = torch.cuda.Event()
            start.record(stream)
            copy_stream.wait_event(start)
            ins = []
            with torch.cuda.stream(copy_stream):
                for h, k in zip(hx, calls):
                    k[src].copy_(h, non_blocking=True)
                    ins.append(torch.cuda.Event())
                    ins[-1].record(copy_stream)
            for i, (a, b, k) in enumerate(zip(ha, hb, calls)):
                stream.wait_event(ins[i])
                step(only=i)
                done = torch.cuda.Event()
                done.record(stream)
                copy_stream.wait_event(done)
                with torch.cuda.stream(copy_stream):
                    a.copy_(k["A"], non_blocking=True)
                    b.copy_(k["Bt"], non_blocking=True)
            end = torch.cuda.Event()
            end.record(copy_stream)
            stream.wait_event(end)
        for _ in range(args.warmup):
            e2e_step()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        h2d = sum(h.numel() * h.element_size() for h in hx)
        d2h = sum(a.numel() * a.element_size() + b.numel() * b.element_size()
                  for a, b in zip(ha, hb))
        e2e = {"value": B * (L + T) * world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "copies": "per call on a copy stream, overlapped with the other call"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = clf_cpu_baseline(c, args.seed)
    if rank == 0:
        # Roofline of the whole V call (rank 768, the larger): the time its work needs on
        # each unit at that unit's peak -- bf16 products at the measured sustained bf16
        # rate, TF32 products at the nominal fraction of it, the fp64 Gram matrices at the
        # fp64 peak derived from unit counts and clock -- against the measured time.
        wv = clf_work({**c, "ctx_len": L + T}, c["rank_v"])
        bf16_peak, bf16_kind = measured_tflops_sustained()
        t_ideal = (wv["bf16"] / (bf16_peak * 1e12) + wv["tf32"] / (bf16_peak * TF32_OVER_BF16 * 1e12)
                   + wv["fp64"] / (FP64_PEAK_TFLOPS * 1e12))
        flops = wv["bf16"] + wv["tf32"] + wv["fp64"]
        t_call = call_ms[1] / 1e3
        line = {
            "metric": metric, "value": B * (L + T) * world * args.steps / (elapsed_ms / 1e3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": name, **c, "n_tail": T, "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2: {2 * calls[0]['X'].numel() * 2 / 1e9:.1f} "
                             "GB of caches per step"},
            "roofline": {"bound": "alu", "kernel": "factorize_window (rank 768 call, whole)",
                         "achieved": flops / t_call / 1e12, "peak": flops / t_ideal / 1e12,
                         "peak_kind": f"composite: bf16 {bf16_kind} {bf16_peak}, tf32 x"
                                      f"{TF32_OVER_BF16:.2f} of it, fp64 derived "
                                      f"{FP64_PEAK_TFLOPS:.1f} (148 SMs x 64 FMA x 2 x 1.965 GHz)",
                         "unit": "TFLOP/s", "frac": t_ideal / t_call, "traffic": None,
                         "flops_bf16": wv["bf16"], "flops_tf32": wv["tf32"],
                         "flops_fp64": wv["fp64"], "avg_launch_ms": call_ms[1],
                         "rank_512_call_ms": call_ms[0]},
            "gpu_launches": sum(clf_work(c, k["r"])["own_launches"] for k in calls) * args.steps,
            "refold_reconstruct_flops": (2 * B * L * c["rank_v"] * n) if refold else 0,
            "library_gemm_calls": 0,
            "clocks": clk, "e2e": e2e, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in (CLF_WORKLOAD, REFOLD_WORKLOAD):
        run_clf(args, rank, world)
        return
    from cross_layer_compressed_b200 import synth
    w = synth.WORKLOADS[args.workload]
    import dataclasses
    if args.batch:
        w = dataclasses.replace(w, batch=args.batch)
    if args.layers:
        w = dataclasses.replace(w, n_layers=min(args.layers, w.n_layers))
    if args.impl == "reference":
        reference_arm(args, w, rank, world)
        return

    import torch
    import torch.distributed as dist
    assert args.warmup >= 3 or os.environ.get("XKV_BENCH_ALLOW_SHORT"), "need >= 3 warm-up steps"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    from cross_layer_compressed_b200 import build
    build.build()
    wl = RclaStep(w, args.seed + rank, dev) if w.mode == "rcla" else \
        XkvStep(w, args.seed + rank, dev, args.path, args.scoring, args.value_reserve)
    nq = wl.qpool.shape[0]
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # ---------------- capture: one CUDA graph per query slot (the xKV steps are
    # stateless; the R-CLA step advances its cache length, so it launches directly)
    use_graph = not args.no_graph and w.mode != "rcla"
    for s in range(args.warmup):                    # also initialises the library's caches
        wl.step(s % nq)
    torch.cuda.synchronize(dev)
    slots = sorted({s % nq for s in range(max(args.steps, args.warmup))})
    # end to end: every slot's queries in pinned host memory, the outputs back into pinned
    # host memory, the copies on a stream of their own (IoOverlap)
    io = {}
    if not args.no_e2e:
        q_host = torch.empty(wl.qpool.shape, dtype=wl.qpool.dtype, pin_memory=True)
        q_host.copy_(wl.qpool.cpu())
        out_host = torch.empty(wl.out.shape, dtype=wl.out.dtype, pin_memory=True)
        copy_stream = torch.cuda.Stream(dev)
        io = {slot: (q_host[slot], out_host, copy_stream) for slot in slots}
        for slot in slots:
            wl.step(io=io[slot])
        torch.cuda.synchronize(dev)
    graphs, e2e_graphs, graph_kernels = {}, {}, {}
    if use_graph:
        for slot in slots:
            g = torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(g):
                wl.step(slot)
            graph_kernels[slot] = count_kernel_nodes(g)
            g.instantiate()
            graphs[slot] = g
            if io:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    wl.step(io=io[slot])
                e2e_graphs[slot] = g
        torch.cuda.synchronize(dev)

    def run_step(s):
        if use_graph:
            graphs[s % nq].replay()
        else:
            wl.step(s % nq)

    def run_e2e_step(s):
        if e2e_graphs:
            e2e_graphs[s % nq].replay()
        else:
            wl.step(io=io[s % nq])

    # ---------------- device-resident timing (the reported value)
    for s in range(args.warmup):
        run_step(s)
    clocks = ClockSampler(local)
    barrier()
    clocks.start()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(args.steps):
        run_step(s)
    stop.record(stream)
    barrier()
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world, dev)

    # ---------------- per-launch time of the attention kernel: the same steps launched
    # directly, CUDA events around every attention call on the launching stream
    def events():
        return [[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
                for _ in range(w.n_layers)]
    ev_steps, sel_steps = [], []
    barrier()
    for s in range(args.steps):
        ev, sv = events(), events()
        wl.step(s % nq, attend_events=ev,
                select_events=sv if w.mode == "sr" else None)
        ev_steps.append(ev)
        sel_steps.append(sv)
    barrier()
    per_launch = [a.elapsed_time(b) for step in ev_steps for a, b in step]
    attend_avg_ms = float(np.mean(per_launch))
    select_avg_ms = (float(np.mean([a.elapsed_time(b) for step in sel_steps for a, b in step]))
                     if w.mode == "sr" else None)

    # ---------------- end to end through the public API with host buffers: every step
    # copies its queries in from pinned host memory and its outputs back, each layer's
    # copies overlapped with the other layers' work (IoOverlap)
    e2e = None
    if not args.no_e2e:
        for s in range(args.warmup):
            run_e2e_step(s)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(args.steps):
            run_e2e_step(s)
        e1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        h2d, d2h = wl.io_bytes()
        e2e = {"value": aggregate_tokens_per_s(w.batch, args.steps, world, e2e_ms),
               "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "launch": "cuda graph" if e2e_graphs else "direct calls",
               "copies": "per layer on a copy stream, overlapped with the other layers"}
        if e2e_graphs:
            # the same loop with every C-ABI call made directly from the host (argument
            # checks, tensor-map encoding and the ctypes calls inside the timed region)
            barrier()
            e0.record(stream)
            for s in range(args.steps):
                wl.step(io=io[s % nq])
            e1.record(stream)
            barrier()
            direct_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
            e2e["direct_calls_value"] = aggregate_tokens_per_s(w.batch, args.steps, world,
                                                               direct_ms)

    # ---------------- algorithmic bytes (untimed: selections recomputed per slot)
    slots = sorted({s % nq for s in range(args.steps)})[:4]
    bytes_launch = wl.attend_bytes(slots)
    step_bytes = wl.step_bytes(bytes_launch)
    hbm_peak, _, peak_kind = measured_peaks()
    achieved = bytes_launch / (attend_avg_ms / 1e3) / 1e9
    if w.mode == "rcla":
        traffic = profiled_traffic(w.name, "k_rcla_tc", "rcla_tc.cu")
    elif args.path == "reassociated":
        traffic = profiled_traffic(w.name, "k_xkv_ra_dense" if w.mode == "dense" else "k_xkv_ra",
                                   "attend_ra.cu")
    else:
        traffic = profiled_traffic(w.name, "k_xkv_tc", "attend_tc.cu")

    kernel = ("rcla_decode_attend" if w.mode == "rcla" else
              "reassociated_attend" if args.path == "reassociated" else "reconstruct_attend")
    roofline = {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": hbm_peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm_peak,
                "frac_of_8tbs": achieved / 8000.0, "traffic": traffic,
                "bytes_per_launch": bytes_launch, "avg_launch_ms": attend_avg_ms}
    if w.mode != "rcla" and args.path == "explicit":
        # the explicit reconstruction is also a tensor-core workload: its GEMM rate
        # against the sustained bf16 peak, alongside the HBM figures
        tf_peak, tf_kind = measured_tflops_sustained()
        tflops = wl.attend_flops() / (attend_avg_ms / 1e3) / 1e12
        roofline.update({"flops_per_launch": wl.attend_flops(), "tflops": tflops,
                         "tensor_peak": tf_peak, "tensor_frac": tflops / tf_peak})
    if w.mode == "dense" and args.path == "explicit":
        # explicit dense reconstruction is bound by the tensor cores, not by HBM: report
        # the GEMM rate against the sustained bf16 peak (the kernel runs inside a long
        # step), keeping the HBM figures alongside
        tf_peak, tf_kind = measured_tflops_sustained()
        tflops = wl.attend_flops() / (attend_avg_ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "kernel": kernel, "achieved": tflops, "peak": tf_peak,
                    "peak_kind": tf_kind, "unit": "TFLOP/s", "frac": tflops / tf_peak,
                    "traffic": traffic, "flops_per_launch": wl.attend_flops(),
                    "hbm_gbs": achieved, "hbm_frac": achieved / hbm_peak,
                    "bytes_per_launch": bytes_launch, "avg_launch_ms": attend_avg_ms}

    # this library's kernels launched in the timed region: counted in the replayed graphs
    # when the steps are graphs, else the launch plan
    planned = wl.launches_per_step * args.steps
    launches, launches_source = planned, "launch plan"
    if use_graph and all(graph_kernels.get(sl) is not None for sl in slots):
        launches = sum(graph_kernels[s % nq] for s in range(args.steps))
        launches_source = "kernel nodes of the replayed CUDA graphs"
        if launches != planned:
            launches_source += f" (launch plan: {planned})"
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.seed)
    if rank == 0:
        ms_step = elapsed_ms / args.steps
        value = aggregate_tokens_per_s(w.batch, args.steps, world, elapsed_ms)
        cfg = {"workload": w.name, "batch": w.batch, "ctx_len": w.ctx_len,
               "n_layers": w.n_layers, "heads_q_kv": [w.n_q_heads, w.n_kv_heads],
               "head_dim": w.head_dim, "parallelism": f"replicas x{world}",
               "l2": f"inputs larger than L2: {wl.resident_bytes() / 1e9:.1f} GB resident, "
                     f"{step_bytes / 1e9:.2f} GB algorithmic per step"}
        if w.mode != "rcla":
            cfg.update({"window": w.window, "ranks_k_v": [w.rank_k, w.rank_v], "chunk": w.chunk,
                        "mode": w.mode, "path": args.path})
        if w.mode == "sr":
            cfg.update({"top_k": w.top_k, "n_sink": w.n_sink, "n_recent": w.n_recent,
                        "n_sel": wl.n_sel, "scoring": args.scoring})
            if args.value_reserve:
                cfg.update({"value_reserve": args.value_reserve, "n_reserved": wl.n_res,
                            "setup_value_ranges_ms": wl.setup_value_ms})
        if args.layers:
            cfg["layers_run"] = f"first {w.n_layers} layers only (profiling case)"
        if w.mode == "rcla":
            cfg.update({"leaders": len(wl.S), "ctx_rows": f"{w.ctx_len}..{w.L_max}"})
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": cfg,
            "step_gbs": step_bytes / (ms_step / 1e3) / 1e9,
            "roofline": roofline,
            "gpu_launches": launches,
            "gpu_launches_source": launches_source,
            "score_select_avg_ms": select_avg_ms,
            "cuda_graph": use_graph,
            "clocks": clk, "e2e": e2e, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
