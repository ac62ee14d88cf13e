#!/usr/bin/env python3
"""Benchmark of the low-bit weight GEMV decode path on B200.

A "step" is one pass of the hot path over one synthetic batch:

* --workload block (default): one Llama-2-70B-shaped decoder block at batch 1,
  the seven linears q/k/v/o (8192->8192, 8192->1024 x2, 8192->8192) and
  gate/up/down (8192->28672 x2, 28672->8192), weights RTN INT4 with group 64
  and fp16 scale/zero, GEMV only.  Four independent block copies (4 x 481.6 MB,
  larger than the 126 MB L2) are rotated between steps.
* --workload sweep80: the 80-layer sweep with the mixed per-layer bit schedule
  (attention 5/6 bits, MLP 2/3 bits, group 32), 34 GB of packed weights.
* --workload binlr: the binary low-rank GEMV at 0.8 bits per weight on the four
  70B linear shapes, batch 1 (a step = one product per shape, rotated copies).

Metric: weight GB/s = algorithmic bytes (packed codes + scales/zeros +
activations in + outputs out) / device time, with steps/s alongside.  The step
is captured once into a CUDA graph and replayed; timing uses CUDA events on the
replay stream with a synchronize and a barrier on both sides, max over ranks.

--impl reference times the CPU oracle (oracle/, plain C, fp64) on a bounded
sample of the same workload on the host cores.  Under torchrun each rank runs
its own replica of the workload (the path is not sharded: replicas only).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_gemv_group_b200 import synth  # noqa: E402
from quantized_gemv_group_b200 import workloads as wl  # noqa: E402

METRIC = "low-bit GEMV weight GB/s (% of B200 HBM peak); 70B-shaped decode steps/s"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0

# dram__bytes_read.sum + dram__bytes_write.sum per launch of the step's kernel (mean over
# the step's launches), from the ncu captures summarised in
# profiles/k_gemv_group_ldg__llama2_70b_block_int4_g64_m1.md and
# profiles/k_binlr_ldg__gate_shape_r5088_m1.md (None: not captured for the current kernel
# version).
NCU_TRAFFIC = {"block": (481.705e6 + 0.314e6) / 4, "sweep80": None, "binlr": 55.545e6 / 8}


# ---------------------------------------------------------------- helpers
def _rank_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons in the background."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.samples = []
        self.proc = None
        self.marks = []
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            uuid = str(device_index)
        self.gpu = uuid

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1, window):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.samples:
            if not (t0 <= ts <= t1):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": window}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "window": window}


# ---------------------------------------------------------------- workloads
class BlockWorkload:
    """Config 1: one 70B decoder block, INT4 g64, batch 1, rotated copies.

    A step runs the block's seven GEMVs as a decode step would order them: four
    grouped launches [q,k,v] (one shared input), [o], [gate,up] (one shared input),
    [down], each a programmatic dependent of the previous one."""

    name = "block"
    bits, group, copies = 4, 64, 4
    LAUNCHES = (("q_proj", "k_proj", "v_proj"), ("o_proj",), ("gate_proj", "up_proj"), ("down_proj",))

    def __init__(self, dev, M=1):
        from quantized_gemv_group_b200 import lbq
        self.lbq = lbq
        self.dev = dev
        self.M = M
        self.linears = wl.block_linears()
        self.by_name = {l.name: i for i, l in enumerate(self.linears)}
        self.sets = []
        for c in range(self.copies):
            layer = []
            for p, l in enumerate(self.linears):
                W = synth.weight(l.d_out, l.d_in, seed=synth.tensor_seed(c, p), device=dev)
                codes, s, z = lbq.lbq_quantize_rtn(W, self.bits, self.group)
                del W
                packed = lbq.lbq_pack(codes, self.bits, lbq.LAYOUT_KERNEL)
                layer.append((packed, s, z, None))
                del codes
            self.sets.append(layer)
        # one input per launch group (shared by q/k/v and by gate/up)
        self.xg = [synth.activations(M, self.linears[self.by_name[grp[0]]].d_in, seed=900 + gi, device=dev)
                   for gi, grp in enumerate(self.LAUNCHES)]
        self.x = [None] * len(self.linears)
        for gi, grp in enumerate(self.LAUNCHES):
            for nm in grp:
                self.x[self.by_name[nm]] = self.xg[gi]
        self.y = [torch.empty(M, l.d_out, dtype=torch.float16, device=dev) for l in self.linears]
        need = 256
        for c in range(self.copies):
            for grp in self.LAUNCHES:
                need = max(need, lbq.lbq_gemv_group_multi_workspace_bytes(self._problems(c, grp, self.x), M))
        self.ws = torch.zeros(need, dtype=torch.uint8, device=dev)
        self.bytes_per_step = (sum(wl.group_packed_bytes(l.d_out, l.d_in, self.bits, self.group) + 2 * M * l.d_out
                                   for l in self.linears) + sum(2 * M * x.shape[1] for x in self.xg))
        self.launches_per_step = len(self.LAUNCHES)
        torch.cuda.synchronize()

    def _problems(self, c, grp, xs):
        out = []
        for nm in grp:
            p = self.by_name[nm]
            packed, s, z, _ = self.sets[c][p]
            l = self.linears[p]
            out.append((xs[p], packed, s, z, self.y[p], l.d_out, l.d_in))
        return out

    def run_copy(self, c, xs=None, ys=None):
        xs = xs or self.x
        for grp in self.LAUNCHES:
            self.lbq.lbq_gemv_group_multi(self._problems(c, grp, xs), self.bits, self.group, ws=self.ws)

    def config(self):
        return {"workload": "llama2-70b decoder block GEMVs (q,k,v,o,gate,up,down), INT4 RTN g64, batch 1",
                "shapes": [[l.d_out, l.d_in] for l in self.linears], "bits": self.bits, "group": self.group,
                "launches": [list(g) for g in self.LAUNCHES],
                "global_batch": self.M, "weight_copies_rotated": self.copies,
                "l2": "inputs larger than L2: 4 rotated weight copies of 481.6 MB each",
                "parallelism": "replicas"}

    def host_inputs(self):
        return [x.cpu().pin_memory() for x in self.xg], [torch.empty_like(y, device="cpu").pin_memory()
                                                       for y in self.y]

    def device_inputs(self, xd):
        """Per-linear input list for the device copies `xd` of the launch-group inputs."""
        xs = [None] * len(self.linears)
        for gi, grp in enumerate(self.LAUNCHES):
            for nm in grp:
                xs[self.by_name[nm]] = xd[gi]
        return xs


class Sweep80Workload:
    """Config 2: 80 layers x 7 linears, mixed bits (attention 5/6, MLP 2/3), g32, batch 1.

    Each layer runs the decode order [q,k,v] [o] [gate,up] [down] as grouped launches."""

    name = "sweep80"
    group, copies = 32, 1
    LAUNCHES = BlockWorkload.LAUNCHES

    def __init__(self, dev, n_layers=wl.N_LAYERS, M=1):
        from quantized_gemv_group_b200 import lbq
        self.lbq = lbq
        self.dev = dev
        self.M = M
        self.linears = wl.block_linears()
        self.by_name = {l.name: i for i, l in enumerate(self.linears)}
        self.n_layers = n_layers
        self.layers = []
        for layer in range(n_layers):
            lw = []
            for p, l in enumerate(self.linears):
                b = wl.schedule_bits(layer, l.name, wl.N_LAYERS)
                W = synth.weight(l.d_out, l.d_in, seed=synth.tensor_seed(layer, p), device=dev)
                codes, s, z = lbq.lbq_quantize_rtn(W, b, self.group)
                del W
                packed = lbq.lbq_pack(codes, b, lbq.LAYOUT_KERNEL)
                del codes
                lw.append((packed, s, z, b))
            self.layers.append(lw)
        self.xg = [synth.activations(M, self.linears[self.by_name[grp[0]]].d_in, seed=900 + gi, device=dev)
                   for gi, grp in enumerate(self.LAUNCHES)]
        self.x = [None] * len(self.linears)
        for gi, grp in enumerate(self.LAUNCHES):
            for nm in grp:
                self.x[self.by_name[nm]] = self.xg[gi]
        self.y = [torch.empty(M, l.d_out, dtype=torch.float16, device=dev) for l in self.linears]
        need = 256
        for grp in self.LAUNCHES:
            need = max(need, lbq.lbq_gemv_group_multi_workspace_bytes(self._problems(0, grp, self.x), M))
        self.ws = torch.zeros(need, dtype=torch.uint8, device=dev)
        self.bytes_per_step = (sum(
            wl.group_packed_bytes(l.d_out, l.d_in, wl.schedule_bits(ly, l.name, wl.N_LAYERS), self.group)
            + 2 * M * l.d_out for ly in range(n_layers) for l in self.linears)
            + n_layers * sum(2 * M * x.shape[1] for x in self.xg))
        self.launches_per_step = n_layers * len(self.LAUNCHES)
        torch.cuda.synchronize()

    def _problems(self, layer, grp, xs):
        out = []
        for nm in grp:
            p = self.by_name[nm]
            packed, s, z, _ = self.layers[layer][p]
            l = self.linears[p]
            out.append((xs[p], packed, s, z, self.y[p], l.d_out, l.d_in))
        return out

    def run_copy(self, c, xs=None, ys=None):
        xs = xs or self.x
        for layer in range(self.n_layers):
            for grp in self.LAUNCHES:
                b = self.layers[layer][self.by_name[grp[0]]][3]
                self.lbq.lbq_gemv_group_multi(self._problems(layer, grp, xs), b, self.group, ws=self.ws)

    def config(self):
        return {"workload": f"llama2-70b {self.n_layers}-layer decode weight sweep, mixed RTN bits "
                            "(attn 6/5, mlp 3/2), g32, batch 1",
                "layers": self.n_layers, "group": self.group, "global_batch": self.M,
                "code_bits_per_weight": wl.schedule_code_bits_per_weight(),
                "launches": [list(g) for g in self.LAUNCHES],
                "l2": "inputs larger than L2 (34 GB of packed weights)", "parallelism": "replicas"}

    def host_inputs(self):
        return [x.cpu().pin_memory() for x in self.xg], [torch.empty_like(y, device="cpu").pin_memory()
                                                       for y in self.y]

    def device_inputs(self, xd):
        xs = [None] * len(self.linears)
        for gi, grp in enumerate(self.LAUNCHES):
            for nm in grp:
                xs[self.by_name[nm]] = xd[gi]
        return xs


class BinlrWorkload:
    """Config 3: binary low-rank GEMV at 0.8 bpw on the four 70B shapes, batch 1."""

    name = "binlr"
    bpw, copies = 0.8, 8

    def __init__(self, dev, M=1):
        from quantized_gemv_group_b200 import lbq
        self.lbq = lbq
        self.M = M
        self.shapes = wl.BINLR_SHAPES
        self.ranks = [wl.binlr_rank(o, i, self.bpw) for o, i in self.shapes]
        self.sets = []
        for c in range(self.copies):
            cur = []
            for si, ((d_out, d_in), r) in enumerate(zip(self.shapes, self.ranks)):
                seed = 10000 + 100 * c + si
                U = lbq.lbq_repack_signs(synth.sign_words(d_out, r, seed, device=dev), d_out, r)
                Vt = lbq.lbq_repack_signs(synth.sign_words(r, d_in, seed + 1, device=dev), r, d_in)
                s1 = synth.channel_scales(d_out, seed + 2, device=dev)
                s2 = synth.channel_scales(d_in, seed + 3, device=dev)
                cur.append((U, Vt, s1, s2))
            self.sets.append(cur)
        self.x = [synth.activations(M, d_in, seed=950 + i, device=dev) for i, (_, d_in) in enumerate(self.shapes)]
        self.y = [torch.empty(M, d_out, dtype=torch.float16, device=dev) for d_out, _ in self.shapes]
        need = max(lbq.lbq_workspace_bytes(lbq.OP_GEMV_BINLR, M, o, i, r)
                   for (o, i), r in zip(self.shapes, self.ranks))
        self.ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
        self.bytes_per_step = sum(wl.binlr_algorithmic_bytes(o, i, r, M) for (o, i), r in zip(self.shapes, self.ranks))
        # two launches per product (the register-streaming path for M <= 4), else five
        self.launches_per_step = (2 if M <= 4 else 5) * len(self.shapes)
        torch.cuda.synchronize()

    def run_copy(self, c, xs=None, ys=None):
        xs = xs or self.x
        ys = ys or self.y
        for (U, Vt, s1, s2), (d_out, d_in), r, x, y in zip(self.sets[c], self.shapes, self.ranks, xs, ys):
            self.lbq.lbq_gemv_binlr(x, U, Vt, s1, s2, d_out, d_in, r, self.lbq.LAYOUT_KERNEL, y=y, ws=self.ws)

    def config(self):
        return {"workload": f"binary low-rank GEMV, {self.bpw} bpw, 70B shapes {self.shapes}, batch {self.M}",
                "ranks": self.ranks, "global_batch": self.M, "weight_copies_rotated": self.copies,
                "l2": "8 rotated copies (> L2)", "parallelism": "replicas"}

    def host_inputs(self):
        return [x.cpu().pin_memory() for x in self.x], [torch.empty_like(y, device="cpu").pin_memory()
                                                      for y in self.y]


WORKLOADS = {"block": BlockWorkload, "sweep80": Sweep80Workload, "binlr": BinlrWorkload}


# ---------------------------------------------------------------- CPU oracle legs
def _oracle_block_inputs(dev, stride, only=None):
    """Inputs of the oracle's sampled block GEMV, made by the oracle itself on the host: the
    seeded synthetic weights of copy 0 of every block linear (only every `stride`-th 16-row
    tile), quantized and packed by oracle/, and the seeded activations of its launch group.
    One row of each sampled tile is the sample: 1/(16 stride) of the output rows.  `only`
    restricts it to the named projections."""
    import oracle as orc
    out = []
    for p, l in enumerate(wl.block_linears()):
        if only is not None and l.name not in only:
            continue
        n, k = l.d_out, l.d_in
        gi = next(i for i, grp in enumerate(BlockWorkload.LAUNCHES) if l.name in grp)
        x = synth.activations(1, k, seed=900 + gi, device=dev)
        W = synth.weight(n, k, seed=synth.tensor_seed(0, p), device=dev)
        tiles = np.arange(0, n // 16, stride)
        idx = (tiles[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
        w_sub = synth.bits_u16(W[torch.from_numpy(idx).to(W.device)])
        del W
        codes, s_, z_ = orc.quantize_rtn(w_sub, BlockWorkload.bits, BlockWorkload.group)
        packed = orc.pack(codes, BlockWorkload.bits, layout=orc.LAYOUT_KERNEL)
        pick = np.arange(len(tiles)) % 16                      # the sampled row of each tile
        out.append({"p": p, "n_sub": len(idx), "k": k, "xh": synth.bits_u16(x), "packed": packed, "s": s_,
                    "z": z_, "rows": np.arange(len(tiles)) * 16 + pick, "rows_global": tiles * 16 + pick})
    return out


def _oracle_block_run(inputs, wk=None):
    """Oracle GEMV on the prepared samples: (algorithmic bytes of the sampled work, seconds,
    worst rel-L2 of the GPU outputs of copy 0 at the same rows if wk is given)."""
    import oracle as orc
    tot_bytes, tot_s, worst = 0, 0.0, 0.0
    bits, group = BlockWorkload.bits, BlockWorkload.group
    for d in inputs:
        t0 = time.perf_counter()
        ref = orc.gemv_group(d["xh"], d["packed"], d["s"], d["z"], d["n_sub"], d["k"], bits, group,
                             layout=orc.LAYOUT_KERNEL, rows=d["rows"])
        tot_s += time.perf_counter() - t0
        tot_bytes += wl.gemv_algorithmic_bytes(len(d["rows"]), d["k"], bits, group, 1)
        if wk is not None:
            worst = max(worst, orc.rel_l2(wk.y[d["p"]].float().cpu().numpy()[:, d["rows_global"]], ref))
    return tot_bytes, tot_s, worst


def _block_config():
    """The block workload's config dict, without building the workload."""
    from types import SimpleNamespace
    return BlockWorkload.config(SimpleNamespace(linears=wl.block_linears(), bits=BlockWorkload.bits,
                                                group=BlockWorkload.group, LAUNCHES=BlockWorkload.LAUNCHES,
                                                M=1, copies=BlockWorkload.copies))


def run_reference(args, dev):
    """--impl reference: the CPU oracle on a bounded sample of the block workload, on inputs
    the oracle quantizes and packs itself (no GPU code on this arm)."""
    import oracle as orc
    ws, rank, _ = _rank_info()
    if rank != 0:
        return
    stride = 8
    inputs = _oracle_block_inputs(dev, stride)
    cores = orc.num_threads()
    for _ in range(args.warmup):
        _oracle_block_run(inputs)
    secs, byts = [], 0
    for _ in range(args.steps):
        b, s, _ = _oracle_block_run(inputs)
        secs.append(s)
        byts = b
    total = sum(secs)
    value = byts * args.steps / total / 1e9
    sample = f"1/{16 * stride} of the output rows of each of the 7 block linears per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _block_config(),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def run_gpu(args, dev):
    world, rank, local = _rank_info()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    wk = WORKLOADS[args.workload](dev)
    stream = torch.cuda.Stream(device=dev)
    peak, peak_kind = _peaks()

    # capture one graph per weight copy
    graphs = []
    with torch.cuda.stream(stream):
        for c in range(wk.copies):
            wk.run_copy(c)            # eager warm-up of every kernel variant
        torch.cuda.synchronize()
        for c in range(wk.copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                wk.run_copy(c)
            graphs.append(g)
    torch.cuda.synchronize()

    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    time.sleep(0.3)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % wk.copies].replay()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        t_wall0 = time.time()
        e0.record(stream)
        for i in range(args.steps):
            graphs[i % wk.copies].replay()
        e1.record(stream)
        torch.cuda.synchronize()
        t_wall1 = time.time()
        barrier()
        ms = e0.elapsed_time(e1)
        window = "timed region"
        if t_wall1 - t_wall0 < 1.0:       # too short for 100 ms sampling: replay 1.5 s more
            t_wall0 = time.time()
            while time.time() - t_wall0 < 1.5:
                for i in range(50):
                    graphs[i % wk.copies].replay()
                torch.cuda.synchronize()
            t_wall1 = time.time()
            window = "1.5 s replay of the same step right after the timed region"
    time.sleep(0.2)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1, window)

    ms_max = ms
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_max = float(t.item())
    ms_per_step = ms_max / args.steps
    value = world * wk.bytes_per_step * args.steps / (ms_max * 1e-3) / 1e9
    achieved = wk.bytes_per_step / (ms / args.steps * 1e-3) / 1e9

    # end-to-end: the public calls with host buffers, copies inside the timed region
    xh, yh = wk.host_inputs()
    xd = [torch.empty_like(x, device=dev) for x in xh]
    xs_dev = wk.device_inputs(xd) if hasattr(wk, "device_inputs") else xd
    with torch.cuda.stream(stream):
        def e2e_step(i):
            for a, b in zip(xd, xh):
                a.copy_(b, non_blocking=True)
            wk.run_copy(i % wk.copies, xs=xs_dev)
            for a, b in zip(yh, wk.y):
                a.copy_(b, non_blocking=True)
        for i in range(max(3, args.warmup)):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        n_e2e = max(10, min(args.steps, 200))
        f0.record(stream)
        for i in range(n_e2e):
            e2e_step(i)
        f1.record(stream)
        torch.cuda.synchronize()
    e2e_ms = f0.elapsed_time(f1)
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_val = world * wk.bytes_per_step * n_e2e / (e2e_ms * 1e-3) / 1e9
    h2d = sum(x.numel() * x.element_size() for x in xh)
    d2h = sum(y.numel() * y.element_size() for y in yh)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "steps_per_s": 1e3 / ms_per_step,
            "hbm_frac_of_8tbs": value / world / 8000.0,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic (seeded N(0,0.02^2) weights with 0.1% x20 outlier columns, N(0,1) activations)",
            "config": wk.config(),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": NCU_TRAFFIC.get(wk.name),
                         "algorithmic_bytes_per_launch": wk.bytes_per_step / wk.launches_per_step,
                         "launches_per_step": wk.launches_per_step, "peak_kind": peak_kind,
                         "note": "every launch of the step is the same kernel: algorithmic bytes per launch / "
                                 "mean launch time (CUDA events over the timed replays); traffic per launch "
                                 "from ncu"},
            "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": wk.launches_per_step * args.steps,
            "clocks": clocks}

    if rank == 0 and world == 1 and args.workload == "block" and not args.no_cpu_baseline:
        import oracle as orc
        with torch.cuda.stream(stream):
            wk.run_copy(0)                # outputs of copy 0, the one the oracle samples
        torch.cuda.synchronize()
        b, s, worst = _oracle_block_run(_oracle_block_inputs(dev, 4), wk)
        line["cpu_baseline"] = {"value": b / s / 1e9, "unit": UNIT, "cores": orc.num_threads(), "kind": "oracle",
                                "sample": "1/64 of the output rows of each of the 7 block linears (copy 0)"}
        line["parity_sampled_rel_l2"] = worst
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del graphs
        dist.destroy_process_group()


def run_breakdown(args, dev):
    """Per-linear device time of the block workload (stderr; analysis aid, not the bench line)."""
    wk = WORKLOADS[args.workload](dev)
    stream = torch.cuda.Stream(device=dev)
    reps = 20
    with torch.cuda.stream(stream):
        for p, l in enumerate(wk.linears):
            graphs = []
            for c in range(wk.copies):
                packed, s, z, _ = wk.sets[c][p] if args.workload == "block" else (None, None, None, None)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for _ in range(reps):
                        wk.lbq.lbq_gemv_group(wk.x[p], packed, s, z, l.d_out, l.d_in, wk.bits, wk.group,
                                              wk.lbq.LAYOUT_KERNEL, y=wk.y[p], ws=wk.ws)
                graphs.append(g)
            for c in range(wk.copies):
                graphs[c].replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(8):
                graphs[i % wk.copies].replay()
            e1.record(stream)
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / (8 * reps)
            byts = wl.gemv_algorithmic_bytes(l.d_out, l.d_in, wk.bits, wk.group, 1)
            print(f"{l.name:10s} {l.d_out:6d}x{l.d_in:<6d} {us:8.2f} us  {byts / us / 1e3:8.1f} GB/s",
                  file=sys.stderr, flush=True)


def _tensor_peak():
    """Dense fp16/bf16 tensor-core TFLOP/s (kind::f16 runs fp16 at the bf16 rate)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def run_prefill(args, dev):
    """Prefill sweep: gate/up 8192->28672 and down 28672->8192 at M = 1..1024 tokens,
    INT4 g128 (bf16 activations) and binary low-rank 0.8 bpw.  GEMV kernels below 64
    tokens, tcgen05 GEMMs from 64.  One JSON line with every case against both the HBM
    and the tensor-core roofline."""
    from quantized_gemv_group_b200 import lbq
    hbm, hbm_kind = _peaks()
    tc, tc_kind = _tensor_peak()
    stream = torch.cuda.Stream(device=dev)
    Ms = [1, 4, 16, 64, 256, 1024]
    shapes = [("gate_up", 28672, 8192), ("down", 8192, 28672)]
    if args.prefill_m:
        Ms = [int(v) for v in args.prefill_m.split(",")]
    if args.prefill_shape:
        shapes = [sh for sh in shapes if sh[0] in args.prefill_shape.split(",")]
    reps = 8
    cases = []
    for name, n, k in shapes:
        # INT4 g128: two weight copies (> L2 together) alternate between calls
        copies = []
        for c in range(2):
            W = synth.weight(n, k, seed=synth.tensor_seed(c, 4 if name == "gate_up" else 6), device=dev)
            codes, s, z = lbq.lbq_quantize_rtn(W, 4, 128)
            del W
            copies.append((lbq.lbq_pack(codes, 4), s, z))
            del codes
        r = wl.binlr_rank(n, k, 0.8)
        bcopies = []
        for c in range(8):
            seed = 20000 + 10 * c
            bcopies.append((lbq.lbq_repack_signs(synth.sign_words(n, r, seed, device=dev), n, r),
                            lbq.lbq_repack_signs(synth.sign_words(r, k, seed + 1, device=dev), r, k),
                            synth.channel_scales(n, seed + 2, device=dev), synth.channel_scales(k, seed + 3, device=dev)))
        for M in Ms:
            x = synth.activations(M, k, seed=31 + M, device=dev, dtype=torch.bfloat16)
            y = torch.empty(M, n, dtype=torch.float16, device=dev)
            for fmt in ("int4_g128", "binary_0.8"):
                if fmt == "int4_g128":
                    ws = torch.zeros(lbq.lbq_workspace_bytes(lbq.OP_GEMM_GROUP, M, n, k), dtype=torch.uint8, device=dev)

                    def call(i):
                        pk, s, z = copies[i % 2]
                        lbq.lbq_gemm_group(x, pk, s, z, n, k, 4, 128, y=y, ws=ws)
                    byts = wl.gemv_algorithmic_bytes(n, k, 4, 128, M)
                    flops = 2.0 * M * n * k
                    path = "tcgen05 GEMM" if M >= 64 else "GEMV (16-token blocks)"
                else:
                    ws = torch.zeros(lbq.lbq_workspace_bytes(lbq.OP_GEMM_BINLR, M, n, k, r), dtype=torch.uint8,
                                     device=dev)

                    def call(i):
                        U, Vt, s1, s2 = bcopies[i % 8]
                        lbq.lbq_gemm_binlr(x, U, Vt, s1, s2, n, k, r, lbq.LAYOUT_KERNEL, y=y, ws=ws)
                    byts = wl.binlr_algorithmic_bytes(n, k, r, M)
                    flops = 2.0 * M * r * (n + k)
                    path = "tcgen05 GEMM x2" if M >= 64 else "GEMV (16-token blocks)"
                with torch.cuda.stream(stream):
                    for i in range(8):
                        call(i)
                    torch.cuda.synchronize()
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        for i in range(reps):
                            call(i)
                    for _ in range(3):
                        g.replay()
                    torch.cuda.synchronize()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    R = 5
                    e0.record(stream)
                    for _ in range(R):
                        g.replay()
                    e1.record(stream)
                    torch.cuda.synchronize()
                us = e0.elapsed_time(e1) * 1e3 / (R * reps)
                t_hbm, t_tc = byts / (hbm * 1e3), flops / (tc * 1e6)
                bound = "hbm" if t_hbm >= t_tc else "tensor"
                cases.append({"shape": name, "n": n, "k": k, "M": M, "format": fmt, "path": path,
                              "us": round(us, 2), "GB_per_s": round(byts / us / 1e3, 1),
                              "TFLOP_per_s": round(flops / us / 1e6, 1), "bound": bound,
                              "roofline_frac": round(max(t_hbm, t_tc) / us, 3)})
                print(f"{name:8s} M={M:5d} {fmt:10s} {us:9.2f} us {byts / us / 1e3:8.1f} GB/s "
                      f"{flops / us / 1e6:8.1f} TF/s  {bound} frac {max(t_hbm, t_tc) / us:.3f}",
                      file=sys.stderr, flush=True)
                del g
            del x, y
        del copies, bcopies
        torch.cuda.empty_cache()
    line = {"metric": "prefill sweep: us per call and fraction of max(HBM, tensor) roofline",
            "unit": "us", "n_gpus": 1, "higher_is_better": False, "data": "synthetic",
            "config": {"workload": "gate/up 8192->28672 and down 28672->8192, M = 1..1024, bf16 activations, "
                                   "INT4 g128 and binary 0.8 bpw",
                       "l2": "2 rotated INT4 copies, 8 rotated binary copies"},
            "peaks": {"hbm_gbs": hbm, "hbm_kind": hbm_kind, "tensor_tflops": tc, "tensor_kind": tc_kind},
            "cases": cases}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["lbq", "reference"], default="lbq")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["prefill"], default="block")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--breakdown", action="store_true", help="print per-linear device times to stderr and exit")
    ap.add_argument("--prefill-m", default="", help="prefill sweep: comma-separated token counts (default all)")
    ap.add_argument("--prefill-shape", default="", help="prefill sweep: gate_up and/or down (default both)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    _, _, local = _rank_info()
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    if dev.type == "cuda":
        torch.cuda.set_device(dev)
    if args.breakdown:
        run_breakdown(args, dev)
    elif args.workload == "prefill":
        run_prefill(args, dev)
    elif args.impl == "reference":
        run_reference(args, dev)
    else:
        if dev.type != "cuda":
            raise SystemExit("bench.py --impl lbq needs a CUDA device")
        run_gpu(args, dev)


if __name__ == "__main__":
    main()
