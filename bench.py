"""Benchmark of the compressed-KV MLA decode step (KV-Kaizen cache) on B200.

One step = the whole hot path over one batch: every anchor layer appends one token through
kvk_quant_write (quantise-on-write), then every layer runs kvk_mla_decode (split decode +
log-sum-exp merge) over its anchor's packed cache.  Workload: the 14B shape at the 4x
budget (48 layers, 40 heads, r = 512, d_R = 64, 32 sequences x 8192 tokens, seeded table),
synthetic seeded inputs generated on the device.

Prints one JSON line.  `value` is the compressed-cache bytes the decode reads per step
(algorithmic, sum over layers of batch * tokens * (row_bytes + 2)) per second of the whole
step, appends included.  Inputs are larger than L2 (the per-layer cache is ~300 MB).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvk|reference]
                  [--workload 14b_4x] [--no-graph]

Under torchrun (N > 1) every rank runs an independent replica (the path is data-parallel
over sequences with no exchange step); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

LOG2 = 0.6931471805599453


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="kvk", choices=["kvk", "reference"])
    p.add_argument("--workload", default="14b_4x")
    p.add_argument("--budget", type=int, default=None,
                   help="compression target of a budget-sweep workload (1, 2, 4, 8 or 16)")
    p.add_argument("--graph", action="store_true",
                   help="replay the step as a CUDA graph (the default; kept for compatibility)")
    p.add_argument("--no-graph", action="store_true",
                   help="issue every launch of every step from the host instead of a graph")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    return p.parse_args()


def dist_setup(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
        pg = dist
    return rank, world, local, pg


def max_over_ranks(x: float, pg, device) -> float:
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg, device=None):
    if pg is not None:
        if device is not None and device.type == "cuda":
            pg.barrier(device_ids=[device.index])
        else:
            pg.barrier()


# Sources whose code makes up the dominant decode kernel (the token-scale tensor-core kernel
# that 16-bit layers take, and the headers it includes); the traffic record is tied to a
# comment- and whitespace-insensitive hash.
KERNEL_SOURCES = ("compressed_decode_attention_kvk_b200/csrc/kvk_decode_tc_token.cu",
                  "compressed_decode_attention_kvk_b200/csrc/kvk_quant_common.cuh",
                  "compressed_decode_attention_kvk_b200/csrc/kvk_sm100.cuh",
                  "compressed_decode_attention_kvk_b200/csrc/kvk_decode_common.cuh",
                  "compressed_decode_attention_kvk_b200/csrc/kvk_internal.cuh",
                  "include/kvk.h")


def kernel_code_hash(root=None):
    """sha256 over KERNEL_SOURCES with comments removed and whitespace collapsed."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(root or ROOT, rel)) as f:
            s = f.read()
        s = re.sub(r"/\*.*?\*/", " ", s, flags=re.S)
        s = re.sub(r"//[^\n]*", " ", s)
        h.update(" ".join(s.split()).encode())
        h.update(b"\0")
    return h.hexdigest()


def decode_traffic():
    """DRAM bytes per full-size decode launch of the tensor-core kernel, from the committed ncu
    capture (profiles/decode_tc_traffic.json), or None when the kernel's code has changed
    since that capture (the record keeps kernel_code_hash())."""
    try:
        with open(os.path.join(ROOT, "profiles", "decode_tc_traffic.json")) as f:
            rec = json.load(f)
        if kernel_code_hash() != rec["code_sha256"]:
            return None
        return rec
    except Exception:
        return None


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def physical_gpu_index(local: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        parts = [x.strip() for x in vis.split(",") if x.strip()]
        if local < len(parts):
            return parts[local]
    return str(local)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# workload construction (device-side seeded generation)
# ---------------------------------------------------------------------------

class DecodeWorkload:
    def __init__(self, name, device, pkg, budget=None, time_prefill=False):
        self.w = w = workloads.WORKLOADS[name]
        self.t = t = workloads.table(name, budget)
        self.budget = budget if budget is not None else (w.budgets[0] if w.budgets else None)
        self.device = device
        self.pkg = pkg
        self.B, self.T, self.H = w.batch, w.tokens, w.n_heads
        self.lay = pkg.Layout(t["anchor"], t["d"], t["b"], w.r, w.d_rope, self.B, self.T,
                              device=device, scale_group=w.scale_group)
        self.anchors = [l for l in range(w.n_layers) if t["anchor"][l] == l]
        zero = torch.zeros(self.B, dtype=torch.int32, device=device)
        self.prefill = None
        if time_prefill:
            self.prefill = self._timed_prefill(zero)
        else:
            for l in self.anchors:            # prefill (not timed)
                c = workloads.latent(w, l, self.B, self.T, device=device)
                kr = workloads.rope_key(w, l, self.B, self.T, device=device)
                self.lay.quant_write(l, c, kr, zero)
                del c, kr
        torch.cuda.synchronize(device)
        # per-step inputs: one new token per anchor (written at the last position), queries
        self.app_pos = torch.full((self.B,), self.T - 1, dtype=torch.int32, device=device)
        self.app = {l: (workloads.latent(w, l, self.B, 1, device=device, kind="append"),
                        workloads.rope_key(w, l, self.B, 1, device=device, kind="append"))
                    for l in self.anchors}
        self.q = {l: workloads.queries(w, l, self.B, device=device) for l in range(w.n_layers)}
        self.lens = torch.full((self.B,), self.T, dtype=torch.int32, device=device)
        # eviction workloads: one sorted keep list per sequence, shared by all layers
        self.keep = self.keep_len = None
        self.n_read = self.T
        if w.keep:
            self.keep = workloads.keep_lists(w, self.B, self.T, w.keep, device=device)
            self.keep_len = torch.full((self.B,), w.keep, dtype=torch.int32, device=device)
            self.n_read = w.keep
        self.sigma = {l: workloads.softmax_scale(t["d"][t["anchor"][l]], w.d_rope)
                      for l in range(w.n_layers)}
        self.out = {l: torch.empty(self.B, self.H, t["d"][t["anchor"][l]], dtype=torch.float32,
                                   device=device) for l in range(w.n_layers)}
        ks = w.keep if w.keep else None
        wsb = max(self.lay.workspace_bytes(l, self.B, self.H, keep_stride=ks)
                  for l in range(w.n_layers))
        self.ws = torch.empty(wsb, dtype=torch.uint8, device=device)
        self.bytes_per_layer = []
        for l in range(w.n_layers):
            info = self.lay.layer_info(l)
            # rows read (the kept ones with a keep list) and their scales (none for an
            # uncompressed anchor, one per group in a group-scaled cache), plus 4 B per index
            sb = 0 if info["b"] == 0 else 2 * info["scales_per_token"]
            self.bytes_per_layer.append(self.B * self.n_read * (info["row_bytes"] + sb) +
                                        (4 * self.B * w.keep if w.keep else 0))
        self.decode_bytes = sum(self.bytes_per_layer)
        mx = max(self.bytes_per_layer)
        self.l2_note = ("inputs larger than L2 (per-layer cache > 126 MB)" if mx > 126e6 and not w.keep else
                        f"per-layer cache {mx / 1e6:.1f} MB < 126 MB L2: layers that inherit "
                        "the previous layer's anchor may find it in L2" if not w.keep else
                        f"kept rows {mx / 1e6:.1f} MB per layer (< 126 MB L2), gathered from a "
                        f"{self.B * self.T * max(self.lay.layer_info(l)['row_bytes'] + 2 for l in range(w.n_layers)) / 1e6:.0f} MB "
                        "cache: a layer that inherits the previous layer's anchor may find them in L2")
        # one append launch for every anchor; per layer split decode + merge, and with a keep
        # list on the tensor-core kernel the compaction of the kept rows
        per_layer = 2
        if w.keep and self.lay.decode_path_for(0, self.q[0][0].dtype, self.H, True) == 1:
            per_layer = 3
        self.launches_per_step = 1 + per_layer * w.n_layers

    def _timed_prefill(self, zero):
        """The quantise-on-write of the whole prompt (batch x tokens) for every anchor layer,
        one kvk_quant_write_layers launch per chunk of at most 64 anchors, inputs resident in
        HBM; timed with CUDA events (best of 3).  Algorithmic bytes: the bf16 inputs read plus
        the rows and scales written."""
        from compressed_decode_attention_kvk_b200 import kvk
        w = self.w
        ins = {l: (workloads.latent(w, l, self.B, self.T, device=self.device),
                   workloads.rope_key(w, l, self.B, self.T, device=self.device))
               for l in self.anchors}
        torch.cuda.synchronize(self.device)
        nbytes = 0
        for l in self.anchors:
            info = self.lay.layer_info(l)
            sb = 0 if info["b"] == 0 else 2 * info["scales_per_token"]
            nbytes += self.B * self.T * ((info["d"] + w.d_rope) * 2 + info["row_bytes"] + sb)
        best = None
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for k in range(0, len(self.anchors), 64):
                ls = self.anchors[k:k + 64]
                kvk.kvk_quant_write_layers(self.lay.handle, ls, [ins[l][0] for l in ls],
                                           [ins[l][1] for l in ls], zero)
            b.record()
            torch.cuda.synchronize(self.device)
            ms = a.elapsed_time(b)
            best = ms if best is None else min(best, ms)
        del ins
        torch.cuda.empty_cache()
        peak, kind = measured_peaks()
        gbs = nbytes / (best * 1e-3) / 1e9
        return {"ms": round(best, 4), "bytes": nbytes, "GBps": round(gbs, 1),
                "frac": round(gbs / peak, 4), "peak": peak, "peak_kind": kind,
                "tokens": self.B * self.T, "anchors": len(self.anchors),
                "kernel": "quant_write_layers_kernel (the prompt's quantise-on-write)"}

    def step(self, events=None):
        from compressed_decode_attention_kvk_b200 import kvk
        h = self.lay.handle
        # the new token of every anchor layer, quantised and written in one launch
        kvk.kvk_quant_write_layers(h, self.anchors, [self.app[l][0] for l in self.anchors],
                                   [self.app[l][1] for l in self.anchors], self.app_pos)
        for l in range(self.w.n_layers):
            ql, qr = self.q[l]
            if events is not None:
                events[l][0].record()
            kvk.kvk_mla_decode(h, l, ql, qr, self.lens, self.sigma[l], self.out[l], self.ws,
                               keep_idx=self.keep, keep_len=self.keep_len)
            if events is not None:
                events[l][1].record()


def run_kvk(args, rank, world, local, pg):
    import compressed_decode_attention_kvk_b200 as pkg
    from compressed_decode_attention_kvk_b200 import build as kb
    if rank == 0 or not os.path.exists(kb.LIB):
        kb.build()
    barrier(pg)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = DecodeWorkload(args.workload, device, pkg, budget=args.budget,
                        time_prefill=workloads.WORKLOADS[args.workload].prefill)
    L = wl.w.n_layers

    # ---- device-timed steps (inputs resident in HBM) -----------------------------------
    # The step is captured once as a CUDA graph (append + every layer's decode and merge) and
    # replayed; --no-graph issues every launch from the host instead, with a pair of timing
    # events around each layer's decode.
    graph = None
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(L)] for _ in range(args.steps)]
    if not args.no_graph:
        s = torch.cuda.Stream(device)
        s.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(s):
            for _ in range(2):
                wl.step()
        torch.cuda.current_stream(device).wait_stream(s)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            wl.step()
    for _ in range(args.warmup):
        graph.replay() if graph else wl.step()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(pg, device)
    torch.cuda.synchronize(device)
    with ClockSampler(physical_gpu_index(local)) as clk:
        start.record()
        for k in range(args.steps):
            if graph:
                graph.replay()
            else:
                wl.step(events=ev[k])
        stop.record()
        torch.cuda.synchronize(device)
    barrier(pg, device)
    t_ms = start.elapsed_time(stop)
    t_ms = max_over_ranks(t_ms, pg, device)
    clocks = clk.summary()
    ms_step = t_ms / args.steps

    # dominant kernel: the decode launches (split + merge per layer), timed by CUDA events on
    # the launching stream inside the timed region.  With the graph the timed region's events
    # bracket whole steps, so a launch pair's duration is the step time over the layers (it
    # includes the step's one append launch, 0.1 % of the step, and the gaps between launches;
    # timing events between the layers' launches would cost ~5 % of the step themselves).
    if graph:
        dec_ms = ms_step / L
    else:
        dec_ms = sum(ev[k][l][0].elapsed_time(ev[k][l][1]) for k in range(args.steps)
                     for l in range(L)) / (args.steps * L)
    peak, peak_kind = measured_peaks()
    total_bytes = wl.decode_bytes * args.steps * world
    value = total_bytes / (t_ms * 1e-3) / 1e9
    roof = None
    traffic = decode_traffic()
    if dec_ms:
        ach = (wl.decode_bytes / L) / (dec_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                "frac": round(ach / peak, 4), "traffic": None, "peak_kind": peak_kind,
                "kernel": "kvk_mla_decode (split decode + merge), mean over layers" +
                          (" (graph replay: step time / layers)" if graph else ""),
                "launch_ms": round(dec_ms, 5)}
        if traffic is not None:
            # DRAM bytes / algorithmic bytes of one captured launch, applied to the mean layer
            roof["traffic"] = int(traffic["dram_over_algorithmic"] * wl.decode_bytes / L)
            roof["traffic_note"] = traffic["note"]

    # ---- end to end through the C ABI with host buffers -------------------------------
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, wl, device, pg)

    # ---- CPU oracle baseline (rank 0, N = 1 only) ---------------------------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    if rank == 0:
        line = {
            "metric": "compressed-KV MLA decode: HBM GB/s (% of peak) and decode steps/s, 14B shape",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "steps_per_s": round(1000.0 / ms_step * world, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded, generated on device)",
            "config": {"workload": args.workload, "layers": L, "heads": wl.H, "r": wl.w.r,
                       "d_rope": wl.w.d_rope, "batch": wl.B, "tokens": wl.T,
                       "budget": wl.budget, "scale_group": wl.w.scale_group,
                       "bits_per_token": wl.lay.bits_per_token,
                       "compression_vs_bf16_c0": round(
                           2 * wl.w.n_kv * wl.w.d_h * 16 * L / wl.lay.bits_per_token, 3)
                       if wl.w.n_kv else None,
                       "decode_bytes_per_step": wl.decode_bytes,
                       "l2": wl.l2_note,
                       "graph": bool(graph), "parallelism": f"replicas x{world}"},
            "roofline": roof, "e2e": e2e, "cpu_baseline": cpu, "prefill": wl.prefill,
            "gpu_launches": wl.launches_per_step * args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    wl.lay.close()


def run_e2e(args, wl, device, pg):
    """Same metric through the public API with host buffers: every step copies the step's
    inputs (new tokens, all layers' queries) from pinned host memory and reads every
    layer's output back to pinned host memory.

    The copies overlap the decode: host-to-device copies run on one stream, device-to-host
    copies on another (the two directions of the link work at once), and per-layer events
    order them against the compute stream -- layer l's query is copied in once the previous
    step's decode of layer l has consumed the buffer, layer l decodes once its query has
    landed and the previous step's read-back of its output buffer has finished, and layer l's
    output is read back as soon as its decode is done."""
    from compressed_decode_attention_kvk_b200 import kvk
    L = wl.w.n_layers
    h_app = {l: (c.cpu().pin_memory(), k.cpu().pin_memory()) for l, (c, k) in wl.app.items()}
    h_q = {l: (a.cpu().pin_memory(), b.cpu().pin_memory()) for l, (a, b) in wl.q.items()}
    h_out = {l: torch.empty(o.shape, dtype=o.dtype).pin_memory() for l, o in wl.out.items()}
    d_app = {l: (torch.empty_like(c), torch.empty_like(k)) for l, (c, k) in wl.app.items()}
    d_q = {l: (torch.empty_like(a), torch.empty_like(b)) for l, (a, b) in wl.q.items()}
    h2d = sum(c.numel() * c.element_size() + k.numel() * k.element_size()
              for c, k in h_app.values()) + sum(a.numel() * a.element_size() +
                                                b.numel() * b.element_size()
                                                for a, b in h_q.values())
    d2h = sum(o.numel() * o.element_size() for o in h_out.values())
    # a keep list is a per-step input too (eviction decisions change from step to step)
    h_keep = d_keep = None
    if wl.keep is not None:
        h_keep = wl.keep.cpu().pin_memory()
        d_keep = torch.empty_like(wl.keep)
        h2d += h_keep.numel() * h_keep.element_size()

    comp = torch.cuda.current_stream(device)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    ev_app, ev_qw = ev(), ev()
    ev_q = [ev() for _ in range(L)]
    ev_dec = [ev() for _ in range(L)]
    ev_d2h = [ev() for _ in range(L)]
    first = [True]

    def step():
        # inputs: new tokens (and keep lists) once the previous step's write has read them
        with torch.cuda.stream(s_in):
            if not first[0]:
                s_in.wait_event(ev_qw)
            if h_keep is not None:
                if not first[0]:
                    s_in.wait_event(ev_dec[L - 1])
                d_keep.copy_(h_keep, non_blocking=True)
            for l in wl.anchors:
                dc, dk = d_app[l]
                dc.copy_(h_app[l][0], non_blocking=True)
                dk.copy_(h_app[l][1], non_blocking=True)
            ev_app.record(s_in)
            for l in range(L):
                if not first[0]:
                    s_in.wait_event(ev_dec[l])     # the previous step's decode of l is done
                qa, qb = d_q[l]
                qa.copy_(h_q[l][0], non_blocking=True)
                qb.copy_(h_q[l][1], non_blocking=True)
                ev_q[l].record(s_in)
        comp.wait_event(ev_app)
        kvk.kvk_quant_write_layers(wl.lay.handle, wl.anchors, [d_app[l][0] for l in wl.anchors],
                                   [d_app[l][1] for l in wl.anchors], wl.app_pos, stream=comp)
        ev_qw.record(comp)
        for l in range(L):
            comp.wait_event(ev_q[l])
            if not first[0]:
                comp.wait_event(ev_d2h[l])         # the previous step's read-back of out[l]
            qa, qb = d_q[l]
            kvk.kvk_mla_decode(wl.lay.handle, l, qa, qb, wl.lens, wl.sigma[l], wl.out[l], wl.ws,
                               keep_idx=d_keep, keep_len=wl.keep_len, stream=comp)
            ev_dec[l].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_dec[l])
                h_out[l].copy_(wl.out[l], non_blocking=True)
                ev_d2h[l].record(s_out)
        first[0] = False

    def finish():
        comp.wait_stream(s_out)
        comp.wait_stream(s_in)

    for _ in range(max(1, args.warmup)):
        step()
    finish()
    torch.cuda.synchronize(device)
    barrier(pg, device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    s_in.wait_stream(comp)                         # no copy of the timed steps starts before a
    s_out.wait_stream(comp)
    for _ in range(args.steps):
        step()
    finish()                                       # every output is back on the host
    b.record(comp)
    torch.cuda.synchronize(device)
    t_ms = max_over_ranks(a.elapsed_time(b), pg, device)
    world = 1 if pg is None else pg.get_world_size()
    v = wl.decode_bytes * args.steps * world / (t_ms * 1e-3) / 1e9
    return {"value": round(v, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(t_ms / args.steps, 4),
            "copies": "H2D and D2H on their own streams, overlapping the decode"}


# ---------------------------------------------------------------------------
# oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

class OracleSampler:
    """Walks the workload's (layer, sequence) decode units in order -- layer 0's sequences,
    then layer 1's, ... -- and times the CPU oracle's decode of each (dequantise + fp64
    attention over the whole sequence).  Preparing a unit (generating the seeded inputs and
    quantising them through the oracle) is not timed."""

    def __init__(self, wl_name, device="cpu"):
        from oracle import oracle
        oracle.build()
        self.oracle = oracle
        self.w = workloads.WORKLOADS[wl_name]
        self.t = workloads.table(wl_name)
        self.device = device
        self.layer, self.seq = 0, 0
        self._cached = None   # (anchor, latent, rope) of the current anchor
        self._keep = None     # keep lists of an eviction workload

    def _next_unit(self):
        w, t = self.w, self.t
        layer, seq = self.layer, self.seq
        a = t["anchor"][layer]
        d, b = t["d"][a], t["b"][a]
        if self._cached is None or self._cached[0] != a:
            c = workloads.latent(w, a, w.batch, w.tokens, device=self.device)
            kr = workloads.rope_key(w, a, w.batch, w.tokens, device=self.device)
            self._cached = (a, c, kr)
        _, c, kr = self._cached
        ql, qr = workloads.queries(w, layer, w.batch, device=self.device)
        rows, scales, codes = self.oracle.quantize_rows(c[seq].float().cpu().numpy(),
                                                        kr[seq].float().cpu().numpy(), d, b)
        qln = ql[seq].double().cpu().numpy()
        qrn = qr[seq].double().cpu().numpy()
        if w.keep and self._keep is None:
            self._keep = workloads.keep_lists(w, w.batch, w.tokens, w.keep).numpy()
        tok = self._keep[seq] if w.keep else None
        self.seq += 1
        if self.seq == w.batch:
            self.seq = 0
            self.layer = (self.layer + 1) % w.n_layers
        return layer, d, (qln, qrn, codes, scales, rows.shape[1], tok)

    def run(self, budget_s, min_units=1):
        """Decode units until `budget_s` seconds of timed oracle work (at least `min_units`).
        Returns (algorithmic bytes, seconds, units, layers touched)."""
        nbytes, dt, units, layers = 0, 0.0, 0, set()
        while dt < budget_s or units < min_units:
            layer, d, (ql, qr, codes, scales, row_bytes, tok) = self._next_unit()
            sigma = workloads.softmax_scale(d, self.w.d_rope)
            t0 = time.perf_counter()
            self.oracle.decode_sequence(ql, qr, codes, scales, d, sigma, tok)
            dt += time.perf_counter() - t0
            nbytes += (codes.shape[0] * (row_bytes + 2) if tok is None
                       else len(tok) * (row_bytes + 6))
            units += 1
            layers.add(layer)
        return nbytes, dt, units, layers


def cpu_baseline(wl):
    sampler = OracleSampler(wl.w.name, device=wl.device)
    nbytes, dt, units, layers = sampler.run(budget_s=12.0)
    return {"value": round(nbytes / dt / 1e9, 5), "unit": "GB/s",
            "cores": sampler.oracle.num_threads(), "kind": "oracle",
            "sample": f"{units} (layer, sequence) decode units of {wl.B * wl.w.n_layers} "
                      f"(layers {min(layers)}..{max(layers)}, {wl.T} tokens each; "
                      f"{dt:.1f} s of fp64 oracle decode, OpenMP over heads)"}


def run_reference(args, rank, world, local, pg):
    """Reference arm: the CPU oracle as it stands, on the host cores.  Each step is a
    bounded sample of the workload: (layer, sequence) decode units, in order, for about
    two seconds of oracle work; the value is algorithmic decode bytes per second."""
    if rank != 0:
        return
    sampler = OracleSampler(args.workload)
    w = sampler.w
    for _ in range(args.warmup):
        sampler.run(budget_s=2.0)
    tot_b, tot_t, tot_u = 0, 0.0, 0
    for _ in range(args.steps):
        nb, dt, nu, _ = sampler.run(budget_s=2.0)
        tot_b += nb
        tot_t += dt
        tot_u += nu
    v = tot_b / tot_t / 1e9
    sample = (f"{tot_u} (layer, sequence) decode units over {args.steps} steps (about 2 s of "
              f"oracle work per step) of {w.batch} sequences x {w.tokens} tokens x "
              f"{w.n_layers} layers")
    line = {
        "impl": "reference",
        "metric": "compressed-KV MLA decode: HBM GB/s (% of peak) and decode steps/s, 14B shape",
        "value": round(v, 5), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": args.workload, "layers": w.n_layers, "heads": w.n_heads,
                   "batch": w.batch, "tokens": w.tokens},
        "cpu_baseline": {"value": round(v, 5), "unit": "GB/s", "kind": "oracle",
                         "cores": sampler.oracle.num_threads(), "sample": sample},
        "e2e": {"value": round(v, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local, pg = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world, local, pg)
        else:
            run_kvk(args, rank, world, local, pg)
    finally:
        if pg is not None:
            pg.destroy_process_group()


if __name__ == "__main__":
    main()
