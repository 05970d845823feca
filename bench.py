"""Benchmark of the fused INT8 Conv3 + BN + shortcut Sum + ReLU (Res3.2, 1x1
128 -> 512, 28x28) on B200, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 3] [--impl x1cb|reference]

One step = one pass of the fused op over one batch (config 3: B=2048).
Timing: CUDA events on the launching stream around exactly K launches,
bracketed by a barrier and a device synchronise on both sides; the max over
ranks.  Inputs (1.85 GB per step at B=2048) are larger than the 126 MB L2,
so no flush is needed; smaller workloads rotate over enough input/output
sets to span three times the L2.  With N > 1 every rank runs its own batch
(weak scaling, batches are independent; no collective on the data path):
launched under torch.distributed.run (WORLD_SIZE = N) each process drives
its LOCAL_RANK GPU; started plainly with --gpus N, bench.py launches the N
ranks itself.  --dry-run runs the same rank logic on the CPU over gloo.

Prints one JSON line (rank 0).  The oracle (plain C on the host cores) is
timed on a bounded sample as the CPU baseline; ``--impl reference`` times it
as the reference arm.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from x1_conv_bn_b200 import synth  # noqa: E402

METRIC = "fused int8 conv TOPS and HBM GB/s (% of roofline) at Res3.2 Conv3, B=2048"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# Dense int8 tensor throughput is twice dense bf16 on B200 (4.5 vs 2.25 POPS
# nominal); the int8 peak is that ratio times the measured bf16 GEMM figure.
INT8_PER_BF16 = 2.0
L2_BYTES = 126 * 2 ** 20


def metric_for(cfg):
    """The headline metric string for config 3; the same metric on the named
    workload for the others."""
    if cfg == "3":
        return METRIC
    return "fused int8 conv TOPS and HBM GB/s (% of roofline) at " + synth.WORKLOAD_NAMES[cfg]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="3", choices=sorted(synth.CONFIGS))
    ap.add_argument("--impl", default="x1cb", choices=["x1cb", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target length of the CPU-oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-1thread", action="store_true",
                    help="also time the oracle sample on one host thread")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--fusion", action="store_true",
                    help="block workloads: run conv2 and conv3 as one fused launch "
                         "(the library's default is two launches)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--dry-run", action="store_true",
                    help="CPU only: run the rank/timing logic over gloo with a host stand-in "
                         "for the kernel (tests the multi-process path without a GPU)")
    return ap.parse_args(argv)


# ---- small helpers (also exercised by the CPU tests) ---------------------------------

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def roofline(ops, nbytes, seconds, hbm_gbs, bf16_tflops, kind):
    """Roofline of one launch: the bound is the larger of bytes / HBM bandwidth
    and ops / int8 dense peak; `frac` = achieved / peak in the bound's unit
    (= roofline time / measured time)."""
    int8_tops = INT8_PER_BF16 * bf16_tflops
    t_hbm = nbytes / (hbm_gbs * 1e9)
    t_tc = ops / (int8_tops * 1e12)
    gbs = nbytes / seconds / 1e9
    tops = ops / seconds / 1e12
    if t_hbm >= t_tc:
        r = {"bound": "hbm", "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s",
             "frac": gbs / hbm_gbs, "peak_source": f"{kind} copy bandwidth (hbm_gbs)"}
    else:
        r = {"bound": "tensor", "achieved": tops, "peak": int8_tops, "unit": "TOPS",
             "frac": tops / int8_tops,
             "peak_source": f"{INT8_PER_BF16:g} x {kind} dense bf16 GEMM (int8:bf16 = 2:1)"}
    r["roofline_time_us"] = max(t_hbm, t_tc) * 1e6
    r["hbm_time_us"] = t_hbm * 1e6
    r["int8_time_us"] = t_tc * 1e6
    r["int8_tensor"] = {"achieved_tops": tops, "peak_tops": int8_tops, "frac": tops / int8_tops,
                        "peak_source": f"{INT8_PER_BF16:g} x {kind} dense bf16 GEMM burst "
                                       f"({bf16_tflops:g} TFLOP/s), nominal int8:bf16 = 2:1"}
    r["hbm"] = {"achieved_gbs": gbs, "peak_gbs": hbm_gbs, "frac": gbs / hbm_gbs}
    return r


def rotation_sets(bytes_per_step, l2_bytes=L2_BYTES, cap=512):
    """Input/output sets to cycle through so that no launch finds its operands
    in L2: enough sets to span three times the L2 (1 when one step alone does)."""
    if bytes_per_step >= 3 * l2_bytes:
        return 1
    return int(min(cap, -(-3 * l2_bytes // max(1, bytes_per_step))))


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def aggregate(per_rank_ms, units_per_rank):
    """Whole-job throughput: units over all ranks / slowest rank's time."""
    t = max(per_rank_ms)
    return units_per_rank * len(per_rank_ms) / (t * 1e-3), t


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The slowest rank's value (all ranks take part; a no-op for one rank)."""
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(base: int, rank: int) -> int:
    """Each rank draws its own independent batch (weak scaling)."""
    return base + 7919 * rank


def workload_units(cfg):
    s = synth.CONFIGS[cfg]
    return s.ops(), s.bytes_moved()


def is_block(s):
    return isinstance(s, (synth.BlockShape, synth.ProjBlockShape))


def block_fused(s, fused=False):
    """Whether the library runs this bottleneck's conv2 and conv3 as one
    launch: fusion enabled and the fused form applies (Cmid = 128, Cout up
    to 1024, whole-row I/O)."""
    return (fused and isinstance(s, synth.BlockShape) and s.Cmid == 128 and s.Cin % 128 == 0
            and s.Cin <= 1024 and s.W + 2 <= 128 and (s.W % 4 == 0 or 4 * s.W <= 256))


def launches_per_step(cfg, fused=False):
    """Kernel launches of one step: three per block, two when the Res3.2
    block's conv2 and conv3 run fused (Cmid = 128)."""
    s = synth.CONFIGS[cfg]
    if isinstance(s, synth.BlockShape):
        return 2 if block_fused(s, fused) else 3
    return 3 if is_block(s) else 1


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def read_traffic(profile_name, src_sha):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", profile_name)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    if not m or not h or h.group(1) != src_sha:
        return None
    return float(m.group(1))


KERNEL_SOURCES = {
    # the files that define each kernel's device code and launch plan
    "conv": ("x1cb_conv.cu", "x1cb_epi.cuh", "x1cb_ptx.cuh", "x1cb_plan.h"),
    "chain": ("x1cb_chain.cu", "x1cb_epi.cuh", "x1cb_ptx.cuh", "x1cb_plan.h"),
}


def kernel_source_sha(kernel="conv"):
    """Short hash of one kernel's sources: a profile's counters are used only
    while the kernel they were taken on is unchanged."""
    import hashlib

    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "x1_conv_bn_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()[:12]


# ---- inputs on the device -----------------------------------------------------------

def device_inputs(cfg, dev, seed, n_sets=1):
    """Packed operands of one step on the device, plus (n_sets - 1) more copies
    of the streamed tensors (activations, shortcut, output) so that the timed
    loop can rotate over sets larger than the L2.  Returns (call, ins, out):
    call(i) launches the op on set i; ins/out are set 0's tensors."""
    import x1_conv_bn_b200 as X

    s = synth.CONFIGS[cfg]
    if isinstance(s, synth.ProjBlockShape):
        inp = synth.proj_block_inputs(s, seed, device=dev)
        x = X.x1cb_pack_act(inp.x)
        ws = [X.x1cb_pack_weight(w) for w in inp.w]
        wp = X.x1cb_pack_weight(inp.wp)
        work = torch.empty(X.bottleneck_proj_i8_workspace_size(s.B, s.H, s.W, s.Cmid),
                           dtype=torch.int8, device=dev)
        xs = [x] + [x.clone() for _ in range(n_sets - 1)]
        outs = [torch.empty((s.B, s.Cout // 32, s.Ho, s.Wo, 32), dtype=torch.int8, device=dev)
                for _ in range(n_sets)]
        del inp.x

        def call(i=0, x_=None, out_=None, stream=None):
            X.bottleneck_proj_i8(xs[i] if x_ is None else x_, ws[0], inp.bias[0], inp.m[0],
                                 ws[1], inp.bias[1], inp.m[1], ws[2], wp, inp.bias[2], inp.m[2],
                                 inp.S, out=outs[i] if out_ is None else out_, workspace=work,
                                 stream=stream)

        return call, {"x": x}, outs[0]
    if isinstance(s, synth.StemShape):
        # the image width-folded (the stem's layout step, not timed): each
        # pixel carries its filter row's 7 taps x 3 channels
        inp = synth.stem_inputs(s, seed, device=dev)
        x = X.x1cb_pack_stem(inp.x, R=s.R)
        w = X.x1cb_pack_stem_weight(inp.w)
        del inp.x
        xs = [x] + [x.clone() for _ in range(n_sets - 1)]
        outs = [torch.empty((s.B, s.Oc // 32, s.Hp, s.Wp, 32), dtype=torch.int8, device=dev)
                for _ in range(n_sets)]

        def call(i=0, x_=None, out_=None, stream=None):
            X.stem_conv_bn_relu_maxpool_i8(xs[i] if x_ is None else x_, w, inp.bias, inp.m,
                                           inp.S, R=s.R, out=outs[i] if out_ is None else out_,
                                           stream=stream)

        return call, {"x": x}, outs[0]
    if isinstance(s, synth.ConvShape) and s.R == 3:
        inp = synth.conv_inputs(s, seed, device=dev)
        x = X.x1cb_pack_act(inp.x)
        w = X.x1cb_pack_weight(inp.w)
        del inp.x
        xs = [x] + [x.clone() for _ in range(n_sets - 1)]
        outs = [torch.empty((s.B, s.Oc // 32, s.H, s.W, 32), dtype=torch.int8, device=dev)
                for _ in range(n_sets)]

        def call(i=0, x_=None, out_=None, stream=None):
            X.conv3x3_bn_relu_i8(xs[i] if x_ is None else x_, w, inp.bias, inp.m, inp.S,
                                 out=outs[i] if out_ is None else out_, stream=stream)

        return call, {"x": x}, outs[0]
    if isinstance(s, synth.BlockShape):
        inp = synth.block_inputs(s, seed, device=dev)
        x = X.x1cb_pack_act(inp.x)
        ws = [X.x1cb_pack_weight(w) for w in inp.w]
        ws_bytes = X.bottleneck_i8_workspace_size(s.B, s.H, s.W, s.Cmid)
        work = torch.empty(ws_bytes, dtype=torch.int8, device=dev)
        xs = [x] + [x.clone() for _ in range(n_sets - 1)]
        outs = [torch.empty_like(x) for _ in range(n_sets)]
        del inp.x

        def call(i=0, x_=None, out_=None, stream=None):
            X.bottleneck_i8(xs[i] if x_ is None else x_, ws[0], inp.bias[0], inp.m[0], ws[1],
                            inp.bias[1], inp.m[1], ws[2], inp.bias[2], inp.m[2], inp.m_r, inp.S,
                            out=outs[i] if out_ is None else out_, workspace=work,
                            stream=stream)

        return call, {"x": x}, outs[0]
    inp = synth.conv_inputs(s, seed, device=dev)
    x = X.x1cb_pack_act(inp.x)
    w = X.x1cb_pack_weight(inp.w)
    r = X.x1cb_pack_act(inp.r)
    del inp.x, inp.r
    xs = [x] + [x.clone() for _ in range(n_sets - 1)]
    rs = [r] + [r.clone() for _ in range(n_sets - 1)]
    outs = [torch.empty((s.B, s.Oc // 32, s.H, s.W, 32), dtype=torch.int8, device=dev)
            for _ in range(n_sets)]

    def call(i=0, x_=None, r_=None, out_=None, stream=None):
        X.conv1x1_bn_add_relu_i8(xs[i] if x_ is None else x_, w, inp.bias, inp.m, inp.m_r,
                                 inp.S, rs[i] if r_ is None else r_,
                                 out=outs[i] if out_ is None else out_, stream=stream)

    return call, {"x": x, "r": r}, outs[0]


# ---- CPU oracle (baseline / reference arm) ---------------------------------------------

class OracleSample:
    """The oracle, as it stands, evaluated on a bounded sample of the workload:
    the first n output pixels (all channels) of the batch, with n calibrated so
    that one evaluation takes about `seconds` on the host cores."""

    def __init__(self, cfg, seconds, seed=7):
        from oracle import oracle as O

        self.O = O
        self.cfg = cfg
        self.s = synth.CONFIGS[cfg]
        self.cores = O.set_threads(0)
        s = self.s
        # output pixels per image (the projection block halves the image; its
        # oracle runs whole images, so its sample is whole images)
        self.proj = isinstance(s, synth.ProjBlockShape)
        self.stem = isinstance(s, synth.StemShape)
        self.hw = s.Ho * s.Wo if self.proj else (s.Hp * s.Wp if self.stem else s.H * s.W)
        self._make(1, seed)
        t = self._run(self.hw)
        per_px = t / self.hw
        n = int(max(1, min(s.B * self.hw, seconds / max(per_px, 1e-9))))
        imgs = (n + self.hw - 1) // self.hw
        if self.proj or self.stem:  # whole images
            n = imgs * self.hw
        if imgs > 1:
            self._make(imgs, seed)
        self.n = n
        self.imgs = imgs

    def _make(self, imgs, seed):
        s = self.s
        if isinstance(s, synth.StemShape):
            import dataclasses

            self.inp = synth.stem_inputs(dataclasses.replace(s, B=imgs), seed)
        elif isinstance(s, synth.ProjBlockShape):
            self.inp = synth.proj_block_inputs(
                synth.ProjBlockShape(imgs, s.H, s.W, s.Cin, s.Cmid, s.Cout), seed)
        elif isinstance(s, synth.BlockShape):
            self.inp = synth.block_inputs(synth.BlockShape(imgs, s.H, s.W, s.Cin, s.Cmid), seed)
        else:
            self.inp = synth.conv_inputs(
                synth.ConvShape(imgs, s.H, s.W, s.Ic, s.Oc, s.R, s.has_res), seed)

    def _run(self, n):
        inp, O = self.inp, self.O
        pix = torch.arange(n, dtype=torch.int64)
        t0 = time.perf_counter()
        if self.stem:
            O.conv_pool(inp.x, inp.w, inp.bias, inp.m, inp.S, stride=self.s.stride)
        elif self.proj:
            O.bottleneck_proj(inp.x, inp.w, inp.wp, inp.bias, inp.m, inp.S)
        elif isinstance(self.s, synth.BlockShape):
            O.bottleneck_pixels(inp.x, inp.w, inp.bias, inp.m, inp.m_r, inp.S, pix)
        else:
            O.conv_pixels(inp.x, inp.w, inp.bias, inp.m, inp.S, pix, inp.r, inp.m_r)
        return time.perf_counter() - t0

    def ops(self):
        return synth.CONFIGS[self.cfg].ops() * self.n / (self.s.B * self.hw)

    def time(self):
        """(ops per second, seconds) of one evaluation of the sample."""
        dt = self._run(self.n)
        return self.ops() / dt, dt

    def describe(self):
        return (f"first {self.n} output pixels (all channels) of the {self.s.B}-image batch, "
                f"i.e. {self.n / (self.s.B * self.hw):.2e} of the workload; oracle with int64 "
                f"intermediates on {self.cores} host threads")


# ---- main ------------------------------------------------------------------------------

def free_port():
    import socket

    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    return port


def spawn_ranks(n, argv):
    """`--gpus N` (N > 1) started without a launcher: run N ranks, one process
    per GPU, through torch.distributed.run on this node and return its exit
    status.  Rank 0 prints the JSON line."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def clocks_verdict(summary):
    """A run is rejected when a slowdown other than the power cap was active,
    or when the SM clock sat well below its maximum with no reason given (a
    leftover clock lock)."""
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    reasons = set(summary.get("reasons") or [])
    sm, mx = summary.get("sm_mhz"), summary.get("sm_max_mhz")
    stuck = sm is not None and mx and sm < 0.8 * mx and not reasons
    return bool(reasons & bad) or bool(stuck)


def dry_run(a, rank, world):
    """The rank/timing logic of a GPU run, on the CPU over gloo: each rank
    times a host stand-in for its kernel, the slowest rank's time is taken,
    rank 0 prints the line (marked dry_run; not a measurement)."""
    import torch.distributed as dist

    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    dd = dist if world > 1 else None
    a_ = torch.randn(256, 256)
    for _ in range(max(3, a.warmup)):
        a_ @ a_
    if dd is not None:
        dd.barrier()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        a_ @ a_
    ms = (time.perf_counter() - t0) * 1e3 / max(1, a.steps)
    ms_max = max_over_ranks(ms, dd, "cpu")
    ops = 2 * 256 ** 3
    value, _ = aggregate([ms_max] * world, ops)
    if dd is not None:
        dd.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"metric": "dry run (host stand-in, not a measurement)",
                          "value": value / 1e12, "unit": "TOPS", "n_gpus": world,
                          "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms_max,
                          "dry_run": True, "scaling": "weak"}), flush=True)


def block_stage_calls(cfg, dev, seed, fusion=False):
    """For the block workloads: the three stages as separate calls on the same
    buffers (conv1 x -> y1, conv2 y1 -> y2, conv3 y2 (+x) -> out), for
    per-stage timing.  Returns (label, ops, bytes, call) per stage."""
    import x1_conv_bn_b200 as X

    s = synth.CONFIGS[cfg]
    if isinstance(s, synth.ProjBlockShape):
        inp = synth.proj_block_inputs(s, seed, device=dev)
        x = X.x1cb_pack_act(inp.x)
        ws = [X.x1cb_pack_weight(w) for w in inp.w]
        wp = X.x1cb_pack_weight(inp.wp)
        y1 = torch.empty((s.B, s.Cmid // 32, s.H, s.W, 32), dtype=torch.int8, device=dev)
        y2 = torch.empty((s.B, s.Cmid // 32, s.Ho, s.Wo, 32), dtype=torch.int8, device=dev)
        out = torch.empty((s.B, s.Cout // 32, s.Ho, s.Wo, 32), dtype=torch.int8, device=dev)
        c1 = synth.ConvShape(s.B, s.H, s.W, s.Cin, s.Cmid, 1, False)
        px = s.B * s.Ho * s.Wo
        return [
            ("1x1 %d->%d" % (s.Cin, s.Cmid), c1.ops(), c1.bytes_moved(),
             lambda stream: X.conv1x1_bn_add_relu_i8(x, ws[0], inp.bias[0], inp.m[0], 0, inp.S,
                                                     None, out=y1, stream=stream)),
            ("3x3/2 %d->%d" % (s.Cmid, s.Cmid), 2 * px * s.Cmid * 9 * s.Cmid,
             s.B * s.H * s.W * s.Cmid + px * s.Cmid + 9 * s.Cmid ** 2 + 8 * s.Cmid,
             lambda stream: X.conv3x3s2_bn_relu_i8(y1, ws[1], inp.bias[1], inp.m[1], inp.S,
                                                   out=y2, stream=stream)),
            ("1x1 %d->%d + proj %d/2" % (s.Cmid, s.Cout, s.Cin),
             2 * px * s.Cout * (s.Cmid + s.Cin),
             px * (s.Cmid + s.Cin + s.Cout) + s.Cout * (s.Cmid + s.Cin) + 8 * s.Cout,
             lambda stream: X.conv1x1_proj_bn_relu_i8(y2, ws[2], x, wp, inp.bias[2], inp.m[2],
                                                      inp.S, out=out, stream=stream)),
        ]
    inp = synth.block_inputs(s, seed, device=dev)
    x = X.x1cb_pack_act(inp.x)
    ws = [X.x1cb_pack_weight(w) for w in inp.w]
    y1 = torch.empty((s.B, s.Cmid // 32, s.H, s.W, 32), dtype=torch.int8, device=dev)
    y2 = torch.empty_like(y1)
    out = torch.empty_like(x)
    st = s.stages()
    fused = block_fused(s, fusion)

    def label(c):
        return f"{c.R}x{c.R} {c.Ic}->{c.Oc}" + (" +res" if c.has_res else "")

    conv1 = (label(st[0]), st[0].ops(), st[0].bytes_moved(),
             lambda stream: X.conv1x1_bn_add_relu_i8(x, ws[0], inp.bias[0], inp.m[0], 0, inp.S,
                                                     None, out=y1, stream=stream))
    if fused:
        # conv2 -> conv3 fused: y1 and the shortcut in, out out; no y2 round trip
        px = s.B * s.H * s.W
        return [conv1, ("3x3 %d->%d -> 1x1 %d->%d +res (fused)" % (s.Cmid, s.Cmid, s.Cmid, s.Cin),
                        st[1].ops() + st[2].ops(),
                        px * (s.Cmid + 2 * s.Cin) + 9 * s.Cmid ** 2 + s.Cin * s.Cmid
                        + 8 * (s.Cmid + s.Cin),
                        lambda stream: X.conv3x3_conv1x1_bn_add_relu_i8(
                            y1, ws[1], inp.bias[1], inp.m[1], ws[2], inp.bias[2], inp.m[2],
                            inp.m_r, inp.S, x, out=out, stream=stream))]
    return [
        conv1,
        (label(st[1]), st[1].ops(), st[1].bytes_moved(),
         lambda stream: X.conv3x3_bn_relu_i8(y1, ws[1], inp.bias[1], inp.m[1], inp.S, out=y2,
                                             stream=stream)),
        (label(st[2]), st[2].ops(), st[2].bytes_moved(),
         lambda stream: X.conv1x1_bn_add_relu_i8(y2, ws[2], inp.bias[2], inp.m[2], inp.m_r,
                                                 inp.S, x, out=out, stream=stream)),
    ]


def time_launches(fn, stream, n, warm=5):
    for _ in range(warm):
        fn(stream)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(n):
        fn(stream)
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / n


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    a = parse(argv)
    launched = "WORLD_SIZE" in os.environ
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if a.gpus > 1 and not launched:
        return spawn_ranks(a.gpus, argv)
    if launched and world != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but WORLD_SIZE={world}: launch one rank per GPU")
    if a.dry_run:
        return dry_run(a, rank, world)
    cfg = a.config
    if a.batch:
        import dataclasses

        synth.CONFIGS[cfg] = dataclasses.replace(synth.CONFIGS[cfg], B=a.batch)
        synth.WORKLOAD_NAMES[cfg] = re.sub(r"B=\d+", f"B={a.batch}", synth.WORKLOAD_NAMES[cfg])
    s = synth.CONFIGS[cfg]
    metric = metric_for(cfg)
    ops, nbytes = workload_units(cfg)
    n_sets = rotation_sets(nbytes)
    l2 = ("inputs larger than L2 (no flush): %.2f GB per step vs 126 MB" % (nbytes / 1e9)
          if n_sets == 1 else
          "rotating over %d input/output sets (%.0f MB in all, %.1f MB per step) so that no "
          "launch finds its operands in the 126 MB L2" % (n_sets, n_sets * nbytes / 2 ** 20,
                                                          nbytes / 2 ** 20))
    cfg_json = {"workload": synth.WORKLOAD_NAMES[cfg],
                "shape": {k: getattr(s, k) for k in s.__dataclass_fields__},
                "layout": "NC/32HW32 activations, blocked [O1,I1,O2,I2] weights",
                "l2": l2,
                "parallelism": (f"replicas x{world} (independent batches, one process per GPU)"
                                if world > 1 else "1 GPU")}

    if a.impl == "reference":
        if rank != 0:
            return 0
        per_step = min(5.0, max(0.05, 90.0 / max(1, a.steps + a.warmup)))
        smp = OracleSample(cfg, per_step)
        vals = []
        for i in range(a.warmup + a.steps):
            v, dt = smp.time()
            if i >= a.warmup:
                vals.append((v, dt))
        v = smp.ops() * len(vals) / sum(dt for _, dt in vals) / 1e12
        ms = 1e3 * sum(dt for _, dt in vals) / len(vals)
        line = {"metric": metric, "value": v, "unit": "TOPS", "impl": "reference",
                "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "int64", "data": "synthetic", "config": cfg_json,
                "cpu_baseline": {"value": v, "unit": "TOPS", "cores": smp.cores,
                                 "cpu_model": cpu_model(), "kind": "oracle",
                                 "sample": smp.describe() + ", per step"},
                "e2e": {"value": v, "unit": "TOPS", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import x1_conv_bn_b200 as X
    from x1_conv_bn_b200 import _build

    if not os.path.exists(X.LIB_PATH):
        _build.build()
    X.lib()
    X.x1cb_set_block_fusion(a.fusion)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    call, ins, out = device_inputs(cfg, dev, shard_seed(synth.CONFIG_SEEDS[cfg], rank), n_sets)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for k in range(max(3, a.warmup)):
            call(k % n_sets, stream=stream)
    torch.cuda.synchronize()
    st, bits = X.x1cb_last_device_error(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {bits:#x} during warm-up")
    forms = X.x1cb_last_epilogue_forms(clear=True)

    # ---- timed region (device time, CUDA events on the launching stream) ----
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for k in range(a.steps):
                call(k % n_sets, stream=stream)
            e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize()
    barrier()
    ms_step = e0.elapsed_time(e1) / a.steps
    st, bits = X.x1cb_last_device_error(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {bits:#x} in the timed region")
    ms_max = max_over_ranks(ms_step, dist, dev)
    value_ops, _ = aggregate([ms_max] * world, ops)
    tops = value_ops / 1e12

    # ---- per-stage times of the block (its dominant kernel gets the roofline) ----
    stages = None
    if is_block(s):
        stages = []
        with torch.cuda.stream(stream):
            for lab, s_ops, s_bytes, fn in block_stage_calls(
                    cfg, dev, shard_seed(synth.CONFIG_SEEDS[cfg], rank), a.fusion):
                t = time_launches(fn, stream, max(20, min(200, a.steps)))
                stages.append({"stage": lab, "us": t * 1e3, "ops": s_ops, "bytes": s_bytes})
        torch.cuda.synchronize()
        if X.x1cb_last_device_error(clear=True)[0] != 0:
            raise RuntimeError("device status set in the per-stage timing")
        for stg in stages:
            stg["us"] = max_over_ranks(stg["us"], dist, dev)

    # ---- end to end through the API with host buffers ----
    # Every step uploads its inputs from pinned host memory, runs the fused op
    # and reads its result back.  Steps are double-buffered over three streams
    # (upload, compute, read-back) so that step i+1's upload, step i's kernel
    # and step i-1's read-back overlap: PCIe is full duplex and the copy
    # engines run beside the SMs.  Events order each buffer's reuse.
    e2e = None
    if not a.no_e2e:
        host_in = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in ins.items()}
        for k in ins:
            host_in[k].copy_(ins[k])
        host_out = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
        dev_in = [{k: torch.empty_like(v) for k, v in ins.items()} for _ in range(2)]
        dev_out = [torch.empty_like(out) for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in host_in.values())
        d2h = host_out[0].numel() * host_out[0].element_size()
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        n_e2e = a.e2e_steps

        def e2e_run(n):
            done_in = [None, None]    # kernel of the buffer's last step has read its inputs
            done_out = [None, None]   # read-back of the buffer's last step has finished
            for i in range(n):
                b = i % 2
                with torch.cuda.stream(s_in):
                    if done_in[b] is not None:
                        s_in.wait_event(done_in[b])
                    for k in dev_in[b]:
                        dev_in[b][k].copy_(host_in[k], non_blocking=True)
                    ev_in = torch.cuda.Event()
                    ev_in.record(s_in)
                stream.wait_event(ev_in)
                if done_out[b] is not None:
                    stream.wait_event(done_out[b])
                if "r" in dev_in[b]:
                    call(0, x_=dev_in[b]["x"], r_=dev_in[b]["r"], out_=dev_out[b], stream=stream)
                else:
                    call(0, x_=dev_in[b]["x"], out_=dev_out[b], stream=stream)
                ev_k = torch.cuda.Event()
                ev_k.record(stream)
                done_in[b] = ev_k
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_k)
                    host_out[b].copy_(dev_out[b], non_blocking=True)
                    ev_o = torch.cuda.Event()
                    ev_o.record(s_out)
                done_out[b] = ev_o

        e2e_run(2)
        torch.cuda.synchronize()
        barrier()
        e0.record(s_in)
        e2e_run(n_e2e)
        e1.record(s_out)  # after the last read-back; e0 came before the first upload
        torch.cuda.synchronize()
        barrier()
        st, bits = X.x1cb_last_device_error(clear=True)
        if st != 0:
            raise RuntimeError(f"device status {bits:#x} in the end-to-end region")
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dist, dev)
        e2e_ops, _ = aggregate([e2e_ms] * world, ops)
        e2e = {"value": e2e_ops / 1e12, "unit": "TOPS", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": n_e2e,
               "how": "per step: pinned host -> device inputs, fused op, device -> pinned "
                      "host result; double-buffered over upload/compute/read-back streams"}

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    hbm, bf16, peak_kind = peaks()
    launches = launches_per_step(cfg, a.fusion)
    gbs = nbytes / (ms_max * 1e-3) / 1e9
    if stages is None:
        roof = roofline(ops, nbytes, ms_max * 1e-3, hbm, bf16, peak_kind)
        if isinstance(s, synth.StemShape):
            roof["kernel"] = ("conv_bn_act_kernel<0, true> (folded stem: seven filter-row "
                              "MMAs of K=32 over the width-folded image, two MMA-issuing "
                              "warps, + BN + ReLU + 3x3/2 max pool)")
            roof["note"] = ("ops count the image's 3 real channels; the kernel multiplies the "
                            "folded 32-channel block (21 used)")
            prof = f"stem_b{s.B}.md"
        elif s.R == 3:
            roof["kernel"] = "conv_bn_act_kernel<0, false> (3x3, halo form)"
            prof = f"conv3x3_{cfg}_b{s.B}.md"
        else:
            narrow = "stage_ch=2" in X.x1cb_describe_plan(s.B, s.H, s.W, s.Ic, s.Oc, 1, True)
            roof["kernel"] = (f"conv_bn_act_kernel<{2 if narrow else 1}, false> (1x1 with shortcut, "
                              f"{'8' if narrow else '16'} KB shortcut/result stages)")
            prof = (f"conv1x1_res32_b{s.B}.md" if cfg in ("2", "3")
                    else f"conv1x1_{cfg}_b{s.B}.md")
        roof["algorithmic_bytes_per_launch"] = nbytes
        roof["algorithmic_ops_per_launch"] = ops
    else:
        for stg in stages:
            stg["roofline"] = roofline(stg["ops"], stg["bytes"], stg["us"] * 1e-6, hbm, bf16,
                                       peak_kind)
        top = max(stages, key=lambda t: t["us"])
        roof = dict(top["roofline"])
        roof["kernel"] = "stage " + top["stage"] + " (the block's slowest launch)"
        roof["algorithmic_bytes_per_launch"] = top["bytes"]
        roof["algorithmic_ops_per_launch"] = top["ops"]
        prof = f"bottleneck_{cfg}_b{s.B}" + ("_fused" if block_fused(s, a.fusion) else "") + ".md"
    roof["traffic"] = read_traffic(prof, kernel_source_sha("chain" if stages and
                                                           "fused" in roof["kernel"] else "conv"))
    roof["traffic_source"] = (f"ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, "
                              f"profiles/{prof}, taken on this kernel source"
                              if roof["traffic"] is not None else
                              "no ncu capture of this kernel source")
    clocks = clk.summary()
    clocks["rejected"] = clocks_verdict(clocks)
    line = {"metric": metric, "value": tops, "unit": "TOPS", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": cfg_json, "hbm_gbs": gbs, "roofline": roof,
            "gpu_launches": a.steps * launches, "epilogue_forms": forms, "clocks": clocks,
            "e2e": e2e}
    if stages is not None:
        line["stages"] = stages
    if world == 1 and not a.no_cpu_baseline:
        smp = OracleSample(cfg, a.cpu_seconds)
        v, dt = smp.time()
        line["cpu_baseline"] = {"value": v / 1e12, "unit": "TOPS", "cores": smp.cores,
                                "cpu_model": cpu_model(), "kind": "oracle",
                                "sample": smp.describe(), "seconds": dt}
        if a.cpu_1thread:
            from oracle import oracle as O

            O.set_threads(1)
            v1, dt1 = smp.time()
            O.set_threads(smp.cores)
            line["cpu_baseline"]["one_thread"] = {"value": v1 / 1e12, "seconds": dt1}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
