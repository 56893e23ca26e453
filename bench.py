"""Benchmark of the MACaQ W4A4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one forward pass of the layer's hot path over one batch: the online per-channel
scale + FWHT-32 + MXFP4 quantisation of the bf16 activations feeding the block-scaled
MXFP4 GEMM (macaq_w4a4_linear), on the Qwen3-32B-shaped MLP down projection at prefill
(M=4096, K=25600, N=5120; the largest single-GPU workload) with seeded synthetic inputs
(workloads.py).  The weight fold is offline and timed separately.  Inputs rotate over copies
whose bytes each exceed the 126 MB L2, so every step streams from HBM.

Printed on rank 0: one JSON line with the whole-job TFLOP/s, the roofline of the dominant
kernel (the tcgen05 GEMM, timed live with CUDA events), the online-transform overhead over
plain MXFP4 (macaq_mxfp4_linear: plain quantisation + the same GEMM) and over the GEMM alone, an end-to-end
figure through the C ABI with host buffers, the oracle's CPU throughput on a bounded
sample (whose rows are also compared with the GPU's codes, scales and outputs), SM clocks
sampled during the timed region, the secondary workloads (the Llama-3-8B up projection,
decode, the 64-layer stack, grouped MoE linears) and, last, a compact summary of every
workload's figures.

--impl reference times the CPU oracle (the reference arm of this repository) on a bounded
sample of the same workload.  With N > 1 GPUs (torchrun), each rank runs an independent
replica of the layer (the path has no exchange step); value = all ranks' work / max time.
"""
from __future__ import annotations

import argparse
import hashlib
import statistics
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as wls  # noqa: E402

L2_BYTES = 126 * 2 ** 20
FP4_OVER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor throughput on B200 (9 : 2.25 PFLOP/s)
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "W4A4 linear TFLOP/s & % roofline; transform overhead % vs plain MXFP4 GEMM"


class Ranks:
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE), replicas of the layer:
    the process group serves only the barriers around the timed region and the max over ranks
    of the device time (no data-path collective).  `backend` is "nccl" on GPUs; tests use
    "gloo" on the CPU."""

    def __init__(self, world, rank, local, backend):
        self.world, self.rank, self.local = world, rank, local
        self.dist = None
        if backend == "nccl":
            torch.cuda.set_device(local)
            self.device = torch.device("cuda", local)
        else:
            self.device = torch.device("cpu")
        if world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": self.device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.dist = dist

    @classmethod
    def from_env(cls, backend):
        return cls(int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                   int(os.environ.get("LOCAL_RANK", "0")), backend)

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, v):
        """The largest of every rank's v (every rank gets it)."""
        if self.dist is None:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.destroy_process_group()
            self.dist = None


def whole_job_tflops(world, flops_per_rank, ms_max):
    """Throughput of the whole job: every rank's work over the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def linear_roofline(wl, ms, fp4_tflops, hbm_gbs):
    """The whole linear against its roofline: the slower of its FP4 flops at the tensor peak and
    its algorithmic bytes (bf16 x, MXFP4 weights, bf16 y, multipliers) at the HBM bandwidth."""
    t_tensor = wl.flops / (fp4_tflops * 1e12)
    t_hbm = wls.alg_bytes(wl) / (hbm_gbs * 1e9)
    t_roof = max(t_tensor, t_hbm)
    return {"bound": "tensor" if t_tensor >= t_hbm else "hbm", "roofline_us": t_roof * 1e6,
            "achieved_us": ms * 1e3, "frac": t_roof / (ms * 1e-3)}


def headline_config(wl, world, l2_note):
    return {"workload": wl.name, "M": wl.M, "K": wl.K, "N": wl.N, "parallelism": f"replicas{world}", "l2": l2_note}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d, "measured"
    d = dict(PEAKS_FALLBACK)
    d["_source"] = "fallback"
    return d, "fallback"


def file_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(kernel_key)
    if not ent:
        return None
    src = os.path.join(ROOT, "online_hadamard_b200", "csrc", ent.get("source", ""))
    if not os.path.exists(src) or file_hash(src) != ent.get("source_hash"):
        return None
    return ent.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampling while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- setup


class Layer:
    """Folded weights and rotating input copies of one linear on one device."""

    def __init__(self, mq, wl, device, copies=None):
        self.mq, self.wl, self.dev = mq, wl, device
        W = wls.make_w(wl)
        s = wls.make_s(wl, W)
        x = wls.make_x(wl)
        footprint = wl.M * wl.K * 2 + wl.N * wl.K * 0.53125 + wl.M * wl.N * 2 + wl.M * wl.K * 0.53125
        self.copies = copies or max(2, math.ceil(3 * L2_BYTES / footprint))
        Wd = W.to(device)
        sd = s.to(device)
        self.Wq, self.Ws, self.am, self.x, self.y, self.ws, self.Aq, self.As = [], [], [], [], [], [], [], []
        self.gws = []
        torch.cuda.synchronize(device)
        t0 = time.perf_counter()
        for _ in range(self.copies):
            Wq, Ws, am = mq.macaq_fold_weights(Wd, sd)
            self.Wq.append(Wq)
            self.Ws.append(Ws)
            self.am.append(am)
        torch.cuda.synchronize(device)
        self.fold_s = (time.perf_counter() - t0) / self.copies
        del Wd
        xd = x.to(device)
        for _ in range(self.copies):
            self.x.append(xd.clone())
            self.y.append(torch.empty(wl.M, wl.N, dtype=torch.bfloat16, device=device))
            self.ws.append(torch.empty(mq.linear_workspace_bytes(wl.M, wl.N, wl.K), dtype=torch.uint8, device=device))
            self.gws.append(torch.empty(max(mq.gemm_workspace_bytes(wl.M, wl.N, wl.K), 1), dtype=torch.uint8,
                                        device=device))
            Aq, As = mq.macaq_act_transform_quant(xd, self.am[0])
            self.Aq.append(Aq)
            self.As.append(As)
        self.x_host = x.contiguous().pin_memory()
        torch.cuda.synchronize(device)

    def linear(self, i):
        c = i % self.copies
        self.mq.macaq_w4a4_linear(self.x[c], self.am[c], self.Wq[c], self.Ws[c], self.wl.N, y=self.y[c],
                                  workspace=self.ws[c])

    def gemm(self, i):
        c = i % self.copies
        self.mq.macaq_mxfp4_gemm(self.Aq[c], self.As[c], self.Wq[c], self.Ws[c], self.wl.M, self.wl.N, self.wl.K,
                                 y=self.y[c], workspace=self.gws[c])

    def plain(self, i):
        """Pure MXFP4: the same kernels as linear() without the scale and the transform."""
        c = i % self.copies
        self.mq.macaq_mxfp4_linear(self.x[c], self.Wq[c], self.Ws[c], self.wl.N, y=self.y[c], workspace=self.ws[c])

    def transform_only(self, i):
        c = i % self.copies
        self.mq.macaq_act_transform_quant(self.x[c], self.am[c], Aq=self.Aq[c], As=self.As[c])

    def time_e2e(self, steps, warmup):
        """ms per step end to end through the public call with host buffers: every step copies its
        x from pinned host memory (H2D), runs the W4A4 linear and reads its y back into pinned host
        memory (D2H), all inside the timed region.  Three streams and two device buffers, as a
        serving loop runs them: step i + 1's H2D proceeds while step i computes and its y returns
        (PCIe is full duplex); a buffer is reused only after its previous step's linear has read x
        and its y has been read back (events)."""
        mq, wl, dev = self.mq, self.wl, self.dev
        nb = 2
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        y_host = [torch.empty(wl.M, wl.N, dtype=torch.bfloat16).pin_memory() for _ in range(nb)]
        copied = [torch.cuda.Event() for _ in range(nb)]    # x[b] holds this step's input
        computed = [torch.cuda.Event() for _ in range(nb)]  # y[b] written, x[b] read
        returned = [torch.cuda.Event() for _ in range(nb)]  # y[b] read back

        def run(first, n):
            cur = torch.cuda.current_stream(dev)
            for st in (s_in, s_cmp, s_out):
                st.wait_stream(cur)  # start after the work (and the timing event) before the run
            for i in range(first, first + n):
                b = i % nb
                if i >= nb:
                    s_in.wait_event(computed[b])
                with torch.cuda.stream(s_in):
                    self.x[b].copy_(self.x_host, non_blocking=True)
                    copied[b].record(s_in)
                s_cmp.wait_event(copied[b])
                if i >= nb:
                    s_cmp.wait_event(returned[b])
                mq.macaq_w4a4_linear(self.x[b], self.am[b], self.Wq[b], self.Ws[b], wl.N, y=self.y[b],
                                     workspace=self.ws[b], stream=s_cmp)
                computed[b].record(s_cmp)
                s_out.wait_event(computed[b])
                with torch.cuda.stream(s_out):
                    y_host[b].copy_(self.y[b], non_blocking=True)
                    returned[b].record(s_out)
            for st in (s_in, s_cmp, s_out):
                cur.wait_stream(st)

        run(0, warmup)
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        run(warmup, steps)
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps


class GraphLoop:
    """`steps` calls of fn(i) captured once into a CUDA graph, replayed as one launch, so the
    timed region holds only GPU work (no per-call host launch overhead)."""

    def __init__(self, fn, steps, warmup, device, offset=0):
        self.device = device
        for i in range(warmup):
            fn(offset + i)
        torch.cuda.synchronize(device)
        self.stream = torch.cuda.Stream(device)
        self.graph = torch.cuda.CUDAGraph()
        self.stream.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(self.stream):
            with torch.cuda.graph(self.graph, stream=self.stream):
                for i in range(steps):
                    fn(offset + warmup + i)
        torch.cuda.current_stream(device).wait_stream(self.stream)
        torch.cuda.synchronize(device)
        self.graph.replay()  # one untimed replay
        torch.cuda.synchronize(device)

    def time_ms(self):
        """Total time of one replay, by CUDA events on the replaying stream."""
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        self.graph.replay()
        e1.record()
        torch.cuda.synchronize(self.device)
        return e0.elapsed_time(e1)


def time_ab(fns, steps, warmup, device, rounds=7):
    """ms per call of each fn in `fns` (name -> fn), each captured as a graph of `steps` calls;
    the graphs are replayed in turn for `rounds` rounds, the order rotated every round so that no
    variant always follows the same one (the board's power state carries over from one replay to
    the next), and each fn's median is returned, so a drift of the clock or of the power state
    falls on every fn alike (the comparisons -- overhead against plain MXFP4 -- are differences of
    a few percent)."""
    loops = {name: GraphLoop(fn, steps, warmup, device) for name, fn in fns.items()}
    names = list(loops)
    times = {name: [] for name in fns}
    for r in range(rounds):
        for name in names[r % len(names):] + names[:r % len(names)]:
            times[name].append(loops[name].time_ms() / steps)
    del loops
    return {name: statistics.median(v) for name, v in times.items()}


# --------------------------------------------------------------------------- CPU baseline


def _scale_index(rows, K):
    """Offsets of (row, 32-block) in the library's E8M0 "MMA tile layout" (include/macaq.h)."""
    kbp = 8 * ((K + 255) // 256)
    r = np.asarray(rows, dtype=np.int64)[:, None]
    kb = np.arange(K // 32, dtype=np.int64)[None, :]
    return ((r // 128) * (kbp // 4) + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4


def _mx_diff(codes, scales, ref_codes, ref_scales, V):
    """Mismatching MXFP4 codes and E8M0 scales of the GPU against the oracle, and how many of
    them are exempt: the oracle's fp32 value within 1 ulp of a rounding boundary of the E2M1
    grid (or the block maximum within 1 ulp of a power of two, for a scale).  V (the oracle's
    fp32 values before rounding, or a callable giving them) is used only when something differs."""
    g = np.stack([codes & 0xF, codes >> 4], -1).reshape(codes.shape[0], -1)
    r = np.stack([ref_codes & 0xF, ref_codes >> 4], -1).reshape(codes.shape[0], -1)
    bad_c, bad_s = g != r, scales != ref_scales
    out = {"codes": int(g.size), "code_mismatch": int(bad_c.sum()), "scales": int(bad_s.size),
           "scale_mismatch": int(bad_s.sum()), "exempt": 0}
    if bad_c.any() or bad_s.any():
        a = np.abs((V() if callable(V) else V).astype(np.float32))
        lo = np.nextafter(a, np.float32(0)).astype(np.float64)
        hi = np.nextafter(a, np.float32(np.inf)).astype(np.float64)
        sc = np.exp2(np.repeat(ref_scales, 32, axis=1).astype(np.float64) - 127)
        near = np.zeros(a.shape, bool)
        for t in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
            near |= (lo <= t * sc) & (t * sc <= hi)
        amax = a.reshape(a.shape[0], -1, 32).max(-1)
        ex = lambda v: (v.view(np.uint32) >> 23) & 0xFF
        near_s = (ex(np.nextafter(amax, np.float32(np.inf))) != ex(amax)) | \
                 (ex(np.nextafter(amax, np.float32(0))) != ex(amax))
        out["exempt"] = int((bad_c & near).sum() + (bad_s & near_s).sum())
    return out


def cpu_baseline(wl, gpu, min_seconds=10.0, rows_per_pass=128, max_passes=64):
    """The oracle as it stands, on the host cores: transform + quantise a seeded sample of
    activation rows and contract them with the folded weights (fp64), one new sample of
    `rows_per_pass` rows per pass, until at least `min_seconds` of CPU work (the fold is
    offline and excluded).  The first sample's codes, scales and outputs are compared with the
    GPU's for the same rows (`gpu`: device tensors of the timed layer), and the GPU's weight
    fold with the oracle's: bit-exact codes and scales (near-boundary mismatches counted as
    exempt), y within a relative Frobenius error of 1e-3 of the bf16-rounded exact result."""
    import oracle
    W = wls.make_w(wl)
    s = wls.make_s(wl, W)
    x = wls.make_x(wl)
    Wf = W.numpy()
    del W
    Wq, Ws, a = oracle.fold_weights(Wf, s.numpy())
    xs = x.float().numpy()
    rpp = min(rows_per_pass, wl.M)
    perm = np.random.default_rng(4).permutation(wl.M)
    passes, dt, first = 0, 0.0, None
    while passes < max_passes and (passes == 0 or dt < min_seconds) and (passes + 1) * rpp <= wl.M:
        idx = np.sort(perm[passes * rpp:(passes + 1) * rpp])
        t0 = time.perf_counter()
        Aq, As = oracle.act_transform_quant(xs[idx], a)
        y = oracle.mx_gemm(Aq, As, Wq, Ws)
        dt += time.perf_counter() - t0
        if first is None:
            first = (idx, Aq, As, y)
        passes += 1
    flops = passes * 2.0 * rpp * wl.N * wl.K
    idx, Aq, As, y = first
    V = oracle.transform_f32(xs[idx], a)
    g_codes = gpu["Aq"][torch.as_tensor(idx, device=gpu["Aq"].device)].cpu().numpy()
    g_scales = gpu["As"].cpu().numpy()[_scale_index(idx, wl.K)]
    act = _mx_diff(g_codes, g_scales, Aq, As, V)
    w_scales = gpu["Ws"].cpu().numpy()[_scale_index(np.arange(wl.N), wl.K)]
    w = _mx_diff(gpu["Wq"].cpu().numpy(), w_scales, Wq, Ws,
                 lambda: oracle.transform_f32(Wf, oracle.multipliers(s.numpy())[1]))
    gy = gpu["y"][torch.as_tensor(idx, device=gpu["y"].device)].double().cpu().numpy()
    ref = torch.from_numpy(y).to(torch.float32).to(torch.bfloat16).double().numpy()
    rel = float(np.linalg.norm(gy - ref) / np.linalg.norm(ref))
    parity = {"rows": int(len(idx)), "activations": act, "weights": w, "y_rel_fro_vs_oracle": rel,
              "y_tolerance": 1e-3, "ok": bool(rel <= 1e-3 and all(d["code_mismatch"] + d["scale_mismatch"] == d["exempt"]
                                                                  for d in (act, w)))}
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{passes} sample(s) of {rpp} of the {wl.M} rows of {wl.name} "
                      f"(transform+quant+fp64 GEMM against all {wl.N} outputs), {dt:.1f} s",
            "seconds": dt, "parity": parity}


HEADLINE = wls.QWEN_DOWN  # the largest single-GPU workload


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = HEADLINE
    import oracle
    W = wls.make_w(wl)
    s = wls.make_s(wl, W)
    x = wls.make_x(wl)
    Wq, Ws, a = oracle.fold_weights(W.numpy(), s.numpy())
    xs_all = x.float().numpy()
    rows = 16
    rng = np.random.default_rng(1)
    times = []
    for i in range(args.warmup + args.steps):
        idx = np.sort(rng.choice(wl.M, rows, replace=False))
        t0 = time.perf_counter()
        Aq, As = oracle.act_transform_quant(xs_all[idx], a)
        oracle.mx_gemm(Aq, As, Wq, Ws)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    dt = sum(times) / len(times)
    val = 2.0 * rows * wl.N * wl.K / dt / 1e12
    out = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic",
           "config": headline_config(wl, int(os.environ.get("WORLD_SIZE", "1")), "oracle on the host cores"),
           "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                            "sample": f"{rows} rows of {wl.M} per step"},
           "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


# --------------------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--no-stack", action="store_true", help="skip the 64-layer stack sweep")
    ap.add_argument("--profile", default=None, metavar="WORKLOAD",
                    help="run each kernel of one workload three times (for ncu captures) and exit; "
                         "WORKLOAD is a name from workloads.py, optionally with _M<m>")
    args = ap.parse_args()
    if args.profile:
        profile_kernels(args.profile)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return

    ranks = Ranks.from_env("nccl")
    world, rank, local = ranks.world, ranks.rank, ranks.local
    device = ranks.device

    import online_hadamard_b200 as mq
    mq.load_library()
    peaks, peak_src = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16

    wl = HEADLINE
    layer = Layer(mq, wl, device)

    barrier = ranks.barrier
    max_over_ranks = ranks.max

    # ---- headline: the fused linear, K steps captured in one CUDA graph
    loop = GraphLoop(layer.linear, args.steps, args.warmup, device)
    torch.cuda.synchronize(device)
    barrier()
    torch.cuda.synchronize(device)
    clocks = ClockSampler(local)
    clocks.start()
    ms_total = loop.time_ms()
    torch.cuda.synchronize(device)
    barrier()
    torch.cuda.synchronize(device)
    # the timed replay lasts milliseconds, shorter than nvidia-smi's sampling period: keep the
    # same graph replaying (untimed) for ~0.4 s so the clock samples are taken under this load
    t_soak = time.perf_counter()
    soak = 0
    while time.perf_counter() - t_soak < 0.4:
        loop.graph.replay()
        soak += 1
        if soak % 4 == 0:
            torch.cuda.synchronize(device)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    clk["window"] = f"the timed replay and {soak} untimed replays of the same graph right after it"
    del loop
    ms = max_over_ranks(ms_total / args.steps)
    value = whole_job_tflops(world, wl.flops, ms)

    # ---- dominant kernel, the comparators and end to end (same rotation); the overhead
    # compares medians of alternating replays of the W4A4 and plain-MXFP4 linears
    head = prefill_leg(layer, args, peaks)
    e2e_steps = max(3, min(args.steps, 10))
    ms_e2e = max_over_ranks(layer.time_e2e(e2e_steps, 3))

    extra = {}
    if world > 1:
        extra["tensor_parallel"] = tp_leg(mq, ranks, device, args)
    if not args.no_extra:
        extra.update(secondary(mq, device, peaks, args))
    if not args.no_stack:
        extra["qwen3_32b_stack"] = stack_sweep(mq, device, peaks)
        extra["qwen3_moe_grouped"] = moe_sweep(mq, device, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        layer.linear(0)
        torch.cuda.synchronize(device)
        cpu = cpu_baseline(wl, {"Aq": layer.Aq[0], "As": layer.As[0], "Wq": layer.Wq[0], "Ws": layer.Ws[0],
                                "y": layer.y[0]})

    if rank == 0:
        out = {
            "metric": METRIC,
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "mxfp4 (e2m1 x e2m1, ue8m0 scales, fp32 accumulate, bf16 out)", "data": "synthetic",
            "config": headline_config(wl, world, f"inputs rotated over {layer.copies} copies, each > L2"),
            "roofline": head["roofline"],
            "linear_roofline": linear_roofline(wl, ms, fp4_peak, peaks["hbm_gbs"]),
            "overhead": head["overhead"],
            "e2e": {"value": whole_job_tflops(world, wl.flops, ms_e2e), "unit": "TFLOP/s", "ms_per_step": ms_e2e,
                    "h2d_bytes_per_step": wl.M * wl.K * 2, "d2h_bytes_per_step": wl.M * wl.N * 2,
                    "overlap": "H2D of step i+1 with the linear and D2H of step i (three streams)"},
            "gpu_launches": 2 * args.steps,
            "clocks": clk,
            "fold_ms": layer.fold_s * 1e3,
            "cpu_baseline": cpu,
            "parity": cpu["parity"] if cpu else None,
            "secondary": extra,
        }
        out["summary"] = summary(out)
        print(json.dumps(out))
    ranks.close()


def tp_leg(mq, ranks, device, args, wl=wls.QWEN_DOWN):
    """The down projection split over the ranks by output columns (online_hadamard_b200.tensor_parallel):
    each rank's W4A4 linear on its N / world weight rows, then the NCCL all-gather of the output
    columns.  Eager launches timed with CUDA events, max over ranks; every rank takes the same
    collective steps in warm-up and timing."""
    from online_hadamard_b200 import tensor_parallel as tp
    W = wls.make_w(wl)
    s = wls.make_s(wl, W)
    Wq, Ws, am = mq.macaq_fold_weights(W.to(device), s.to(device))
    del W
    q, sc, n = tp.shard_folded_weights(Wq, Ws, wl.N, wl.K, ranks.world, ranks.rank)
    x = wls.make_x(wl).to(device)
    ws = torch.empty(mq.linear_workspace_bytes(wl.M, max(n, 1), wl.K), dtype=torch.uint8, device=device)
    step = lambda: tp.tp_w4a4_linear(x, am, q, sc, wl.N, workspace=ws)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    ranks.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize(device)
    ms = ranks.max(e0.elapsed_time(e1) / args.steps)
    ranks.barrier()
    return {"workload": wl.name, "ranks": ranks.world, "rows_per_rank": n, "ms": ms,
            "tflops": wl.flops / (ms * 1e-3) / 1e12, "scaling": "strong (one layer split over the ranks)",
            "collective": "all-gather of the bf16 output columns"}


def prefill_leg(layer, args, peaks):
    """A prefill linear's dominant kernel (the 2-CTA GEMM, timed alone on the same rotation) and
    the transform's overhead against plain MXFP4 and the GEMM alone, from medians of alternating
    graph replays of the four variants."""
    wl, device = layer.wl, layer.dev
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    ab = time_ab({"linear": layer.linear, "plain": layer.plain, "gemm": layer.gemm,
                  "transform": layer.transform_only}, args.steps, args.warmup, device)
    ms_gemm, ms_plain, ms_xform, ms_lin = ab["gemm"], ab["plain"], ab["transform"], ab["linear"]
    gemm_tflops = wl.flops / (ms_gemm * 1e-3) / 1e12
    xform_bytes = wl.M * wl.K * 2 + wl.M * wl.K * (0.5 + 1 / 32) + wl.K * 4
    peak_src = peaks.get("_source", "measured")
    return {
        "roofline": {"bound": "tensor", "kernel": "mxf4_gemm_pair_kernel<5> (2-CTA 256x256 tiles, scale warps)",
                     "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak,
                     "traffic": recorded_traffic("mxf4_gemm_pair_256x256:" + wl.name),
                     "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} x {FP4_OVER_BF16} "
                                    "(fp4:bf16 nominal)",
                     "ms_per_launch": ms_gemm},
        "overhead": {"linear_ms": ms_lin, "plain_mxfp4_ms": ms_plain, "gemm_only_ms": ms_gemm,
                     "vs_plain_mxfp4_pct": 100.0 * (ms_lin / ms_plain - 1.0),
                     "vs_gemm_only_pct": 100.0 * (ms_lin / ms_gemm - 1.0),
                     "method": "medians of 7 rounds of alternating graph replays per variant, order rotated each round",
                     "transform_quant_ms": ms_xform,
                     "transform_quant_gbs": xform_bytes / (ms_xform * 1e-3) / 1e9},
    }


def summary(out):
    """Every workload's key figures, rounded, in a few hundred characters (the end of the line)."""
    r = lambda v, n=3: None if v is None else float(f"{v:.{n}g}")
    sm = {"cfg4_down_prefill": {"tflops": r(out["value"]), "linear_roof": r(out["linear_roofline"]["frac"]),
                                "gemm_roof": r(out["roofline"]["frac"]),
                                "ovh_plain_pct": r(out["overhead"]["vs_plain_mxfp4_pct"], 2),
                                "ovh_gemm_pct": r(out["overhead"]["vs_gemm_only_pct"], 2)}}
    sec = out.get("secondary") or {}
    for k, v in sec.items():
        if k.startswith("llama3_8b_up_prefill"):
            sm["cfg2_llama_up"] = {"tflops": r(v["tflops"]), "linear_roof": r(v["linear_roofline"]["frac"]),
                                   "gemm_roof": r(v["roofline"]["frac"]),
                                   "ovh_plain_pct": r(v["overhead"]["vs_plain_mxfp4_pct"], 2),
                                   "ovh_gemm_pct": r(v["overhead"]["vs_gemm_only_pct"], 2)}
        elif k.startswith("qwen3_32b_up_decode"):
            sm["cfg3_" + k.split("_")[-1]] = {"gbs": r(v["gbs"]), "linear_roof": r(v["linear_roofline"]["frac"]),
                                              "ovh_plain_pct": r(v["vs_plain_mxfp4_pct"], 2)}
    st = sec.get("qwen3_32b_stack") or {}
    for k, v in st.items():
        if k.startswith("M"):
            sm["cfg5_" + k] = {"ms": r(v["w4a4_ms"]), "roof": r(v["linear_roofline_frac"]),
                               "ovh_plain_pct": r(v["vs_plain_mxfp4_pct"], 2),
                               "unstacked_ms": r(v["w4a4_one_linear_at_a_time_ms"])}
    for k, v in (sec.get("qwen3_moe_grouped") or {}).items():
        if isinstance(v, dict):
            sm["moe_" + k] = {"us": r(v["ms"] * 1e3), "roof": r(v["linear_roofline_frac"]),
                              "ovh_plain_pct": r(v["vs_plain_mxfp4_pct"], 2)}
    fl = sec.get("flip_refinement")
    if fl:
        sm["flip_llama_up"] = {"ms": r(fl["hessian_ms"] + fl["refine_ms"]),
                               "err_rtn": r(fl["held_out_rel_err_rtn"]), "err_refined": r(fl["held_out_rel_err_refined"])}
    par = out.get("parity")
    if par:
        sm["parity_cfg4"] = {"ok": par["ok"], "exempt": par["activations"]["exempt"] + par["weights"]["exempt"],
                             "y_rel": r(par["y_rel_fro_vs_oracle"], 2)}
    return sm


def profile_stacked(name):
    """Launch sequence for ncu of a stacked call of the 64-layer stack's first layer
    ("qwen3_32b_stack_qkv_M<m>" or "qwen3_32b_stack_gateup_M<m>"): fold its layers into one stacked
    buffer, then 3 x macaq_w4a4_linear_multi (one quantiser and one stacked GEMM each)."""
    import online_hadamard_b200 as mq
    base, _, m = name.partition("_M")
    names = {"qwen3_32b_stack_qkv": ("q", "k", "v"), "qwen3_32b_stack_gateup": ("gate", "up")}[base]
    M = int(m)
    layers = [wls.stack_layer(0, n, M) for n in names]
    K, Ns = layers[0].K, [wl.N for wl in layers]
    folds = []
    for wl in layers:
        W = wls.make_w_device(wl, "cuda")
        s = mq.macaq_calibrate_scale(wls.make_x_device(wl, wls.CALIB_TOKENS, "cuda", tensor_id=2), W)
        folds.append(mq.macaq_fold_weights(W, s))
        del W
    Wq, Ws, am = torch.cat([f[0] for f in folds]), torch.cat([f[1] for f in folds]), torch.stack([f[2] for f in folds])
    x = wls.make_x_device(layers[0], M, "cuda")
    ws = torch.empty(mq.linear_multi_workspace_bytes(M, len(Ns), K), dtype=torch.uint8, device="cuda")
    y = torch.empty(M, sum(Ns), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        mq.macaq_w4a4_linear_multi(x, am, Wq, Ws, Ns, y=y, workspace=ws)
    torch.cuda.synchronize()
    print(f"profiled {base} M={M} K={K} N={'+'.join(map(str, Ns))}")


def profile_kernels(name):
    """Launch sequence for ncu: fold once, then 3 x (transform+quant, plain quant, GEMM)."""
    import online_hadamard_b200 as mq
    if name.startswith("qwen3_32b_stack_"):
        return profile_stacked(name)
    base, _, m = name.partition("_M")
    wl = next(w for w in wls.ALL if w.name == base)
    if m:
        wl = wl.with_m(int(m))
    W = wls.make_w(wl)
    s = wls.make_s(wl, W)
    x = wls.make_x(wl).cuda()
    Wq, Ws, am = mq.macaq_fold_weights(W.cuda(), s.cuda())
    Aq, As = mq.macaq_act_transform_quant(x, am)
    y = torch.empty(wl.M, wl.N, dtype=torch.bfloat16, device="cuda")
    gws = torch.empty(max(mq.gemm_workspace_bytes(wl.M, wl.N, wl.K), 1), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        mq.macaq_act_transform_quant(x, am, Aq=Aq, As=As)
        mq.macaq_act_quant_plain(x, Aq=Aq, As=As)
        mq.macaq_mxfp4_gemm(Aq, As, Wq, Ws, wl.M, wl.N, wl.K, y=y, workspace=gws)
    torch.cuda.synchronize()
    print(f"profiled {wl.name} M={wl.M} K={wl.K} N={wl.N}")


# Layers of a decoder block that read the same activations: run as one stacked call.
STACK_GROUPS = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))


def stack_sweep(mq, device, peaks, Ms=(1, 32, 512, 4096), steps=3, warmup=2):
    """The 64-layer Qwen3-32B-shaped linear stack (q, k, v, o, gate, up, down per layer): each
    linear's weights and calibration batch are drawn on the device, s is calibrated and W folded
    by the library, and the fp32 weights are freed before the next linear, so only the 16.6 GB
    of MXFP4 weights stay resident.  The layers reading the same activations (q, k, v; gate, up)
    are folded into slices of one stacked buffer each.  Per M, all 448 linears run back to back in
    one CUDA graph three ways: W4A4 with the shared-input layers stacked (macaq_w4a4_linear_multi:
    q/k/v and gate/up each one quantiser and one GEMM launch), plain MXFP4 stacked the same way
    (the overhead's baseline), and W4A4 one linear at a time."""
    dims = {name: (K, N) for name, K, N in wls.QWEN_STACK_LINEARS}
    groups = []  # per (layer, group): K, Ns, stacked Wq, Ws, act_mult [G, K]
    for layer in range(64):
        for names in STACK_GROUPS:
            K = dims[names[0]][0]
            Ns = [dims[n][1] for n in names]
            Wq = torch.empty(sum(Ns), K // 2, dtype=torch.uint8, device=device)
            sb = [mq.scale_bytes(N, K) for N in Ns]
            Ws = torch.empty(sum(sb), dtype=torch.uint8, device=device)
            am = torch.empty(len(names), K, dtype=torch.float32, device=device)
            n0 = b0 = 0
            for g, name in enumerate(names):
                wl = wls.stack_layer(layer, name, 1)
                W = wls.make_w_device(wl, device)
                s = mq.macaq_calibrate_scale(wls.make_x_device(wl, wls.CALIB_TOKENS, device, tensor_id=2), W)
                mq.macaq_fold_weights(W, s, Wq=Wq[n0:n0 + Ns[g]], Ws=Ws[b0:b0 + sb[g]], act_mult=am[g])
                del W
                n0 += Ns[g]
                b0 += sb[g]
            groups.append((K, Ns, Wq, Ws, am, sb))
    torch.cuda.empty_cache()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    res = {"layers": 64, "linears": sum(len(g[1]) for g in groups),
           "weights_gb": sum(q.numel() + t.numel() for _, _, q, t, _, _ in groups) / 1e9,
           "stacked": "+".join("/".join(n) for n in STACK_GROUPS)}
    for M in Ms:
        xs = {K: wls.make_x_device(wls.stack_layer(0, name, M), M, device)
              for name, K, _ in wls.QWEN_STACK_LINEARS}
        ys = {tuple(Ns): torch.empty(M, sum(Ns), dtype=torch.bfloat16, device=device) for _, Ns, *_ in groups}
        ws = torch.empty(max(max(mq.linear_multi_workspace_bytes(M, len(Ns), K) for K, Ns, *_ in groups),
                             max(mq.linear_workspace_bytes(M, N, K) for _, K, N in wls.QWEN_STACK_LINEARS)),
                         dtype=torch.uint8, device=device)
        # the one-linear-at-a-time variant's operands: views into the stacked buffers
        singles = []
        for K, Ns, Wq, Ws, am, sb in groups:
            n0 = b0 = 0
            for g, N in enumerate(Ns):
                singles.append((K, N, Wq[n0:n0 + N], Ws[b0:b0 + sb[g]], am[g]))
                n0 += N
                b0 += sb[g]
        y1 = {N: torch.empty(M, N, dtype=torch.bfloat16, device=device) for _, _, N in wls.QWEN_STACK_LINEARS}

        def w4a4(i):
            for K, Ns, Wq, Ws, am, _ in groups:
                mq.macaq_w4a4_linear_multi(xs[K], am, Wq, Ws, Ns, y=ys[tuple(Ns)], workspace=ws)

        def plain(i):
            for K, Ns, Wq, Ws, _, _ in groups:
                mq.macaq_w4a4_linear_multi(xs[K], None, Wq, Ws, Ns, y=ys[tuple(Ns)], workspace=ws)

        def unstacked(i):
            for K, N, Wq, Ws, am in singles:
                mq.macaq_w4a4_linear(xs[K], am, Wq, Ws, N, y=y1[N], workspace=ws)

        ab = time_ab({"w4a4": w4a4, "plain": plain, "unstacked": unstacked}, steps, warmup, device, rounds=5)
        ms, ms_plain = ab["w4a4"], ab["plain"]
        flops = sum(2.0 * M * K * N for K, Ns, *_ in groups for N in Ns)
        nbytes = sum(wls.alg_bytes(wls.Workload("", 5, M, K, N, "normal", 0.0, 1.0)) for K, Ns, *_ in groups
                     for N in Ns)
        t_roof = max(flops / (fp4_peak * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9))
        res[f"M{M}"] = {"w4a4_ms": ms, "plain_mxfp4_ms": ms_plain, "vs_plain_mxfp4_pct": 100.0 * (ms / ms_plain - 1.0),
                        "w4a4_one_linear_at_a_time_ms": ab["unstacked"],
                        "tflops": flops / (ms * 1e-3) / 1e12, "gbs": nbytes / (ms * 1e-3) / 1e9,
                        "linear_roofline_frac": t_roof / (ms * 1e-3)}
        del xs, ys, ws, singles, y1
        torch.cuda.empty_cache()
    del groups
    torch.cuda.empty_cache()
    return res


def moe_sweep(mq, device, peaks, token_counts=(16, 4096), steps=10, warmup=3):
    """Grouped (mixture-of-experts) linears, Qwen3-MoE-like: 128 experts, top-8 routing, the up
    (2048 -> 768) and down (768 -> 2048) projections; per expert its own calibrated scale and
    folded weights.  W4A4 against plain MXFP4, graph-timed; bytes = the weights of the experts
    that received tokens + bf16 x and y."""
    E = wls.MOE_EXPERTS
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    res = {"experts": E, "topk": wls.MOE_TOPK}
    for li, (name, K, N) in enumerate(wls.MOE_LINEARS):
        Wq, Ws, am = [], [], []
        for e in range(E):
            wl = wls.Workload(f"moe_{name}", 6, 1, K, N, "normal", 0.01, 50.0, layer=E * li + e)
            W = wls.make_w_device(wl, device)
            s = mq.macaq_calibrate_scale(wls.make_x_device(wl, wls.CALIB_TOKENS, device, tensor_id=2), W)
            q, sc, a = mq.macaq_fold_weights(W, s)
            Wq.append(q)
            Ws.append(sc)
            am.append(a)
            del W
        Wq, Ws, am = torch.stack(Wq), torch.cat(Ws), torch.stack(am)
        for T in token_counts:
            counts = wls.moe_counts(T)
            rows = sum(counts)
            x = wls.make_x_device(wls.Workload(f"moe_{name}_x", 6, 1, K, N, "normal", 0.01, 50.0,
                                               layer=E * li + E), rows, device)
            y = torch.empty(rows, N, dtype=torch.bfloat16, device=device)
            ws = torch.empty(max(mq.grouped_workspace_bytes(counts, N, K), 1), dtype=torch.uint8, device=device)
            counts_dev = torch.tensor(counts, dtype=torch.int32, device=device)
            ws_dev = torch.empty(mq.grouped_device_workspace_bytes(rows, E, N, K), dtype=torch.uint8, device=device)
            ab = time_ab({"w4a4": lambda i: mq.macaq_w4a4_grouped_linear(x, counts, am, Wq, Ws, N, y=y, workspace=ws),
                          "plain": lambda i: mq.macaq_w4a4_grouped_linear(x, counts, None, Wq, Ws, N, y=y,
                                                                          workspace=ws),
                          "device": lambda i: mq.macaq_w4a4_grouped_linear_device(x, counts_dev, am, Wq, Ws, N,
                                                                                  capacity=T, y=y, workspace=ws_dev)},
                         steps, warmup, device)
            ms, ms_plain = ab["w4a4"], ab["plain"]
            active = sum(1 for c in counts if c)
            flops = 2.0 * rows * K * N
            nbytes = active * N * K * (0.5 + 1 / 32) + 2.0 * rows * (K + N) + 4.0 * K * active
            t_roof = max(flops / (fp4_peak * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9))
            res[f"{name}_T{T}"] = {"routed_rows": rows, "active_experts": active, "max_rows": max(counts),
                                    "ms": ms, "plain_mxfp4_ms": ms_plain, "device_counts_ms": ab["device"],
                                    "vs_plain_mxfp4_pct": 100.0 * (ms / ms_plain - 1.0),
                                    "tflops": flops / (ms * 1e-3) / 1e12, "gbs": nbytes / (ms * 1e-3) / 1e9,
                                    "linear_roofline_frac": t_roof / (ms * 1e-3)}
            del x, y, ws, ws_dev, counts_dev
        del Wq, Ws, am
        torch.cuda.empty_cache()
    return res


def flip_leg(mq, device, wl=wls.LLAMA_UP, calib_tokens=128, max_moves=64, held_out=256):
    """Flip-Refinement (offline) of one layer: the Hessian of a calibration batch and the refinement of
    its round-to-nearest codes, timed with CUDA events; moves per row; and what it buys -- the W4A4
    linear's relative output error against the exact x W^T on held-out tokens (same distribution),
    round-to-nearest against refined codes."""
    W = wls.make_w(wl).to(device)
    s = wls.make_s(wl, W.cpu()).to(device)
    xcal = torch.cat([wls.make_xcal(wl), wls._draw_x(wl, calib_tokens - wls.CALIB_TOKENS, 7).to(torch.bfloat16)])
    xcal = xcal.to(device)
    Wq, Ws, am = mq.macaq_fold_weights(W, s)
    rtn = Wq.clone()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    torch.cuda.synchronize(device)
    e[0].record()
    Hs = mq.macaq_calib_hessian(xcal, am)
    e[1].record()
    moves = mq.macaq_flip_refine(W, s, Hs, Wq, Ws, max_moves)
    e[2].record()
    torch.cuda.synchronize(device)
    xh = wls._draw_x(wl, held_out, 11).to(torch.bfloat16).to(device)
    exact = xh.float() @ W.t()
    rel = lambda y: float((y.float() - exact).norm() / exact.norm())
    out = {"workload": wl.name, "calibration_tokens": calib_tokens, "max_moves_per_row": max_moves,
           "hessian_ms": e[0].elapsed_time(e[1]), "refine_ms": e[1].elapsed_time(e[2]),
           "moves_per_row": float(moves.float().mean()), "code_bytes_changed": float((Wq != rtn).float().mean()),
           "held_out_rel_err_rtn": rel(mq.macaq_w4a4_linear(xh, am, rtn, Ws, wl.N)),
           "held_out_rel_err_refined": rel(mq.macaq_w4a4_linear(xh, am, Wq, Ws, wl.N))}
    del W, Hs, Wq, rtn, Ws
    torch.cuda.empty_cache()
    return out


def secondary(mq, device, peaks, args):
    """The Llama-3-8B up projection (tensor-bound prefill), decode (HBM-bound) and Flip-Refinement."""
    res = {"flip_refinement": flip_leg(mq, device)}
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    wl = wls.LLAMA_UP
    layer = Layer(mq, wl, device)
    leg = prefill_leg(layer, args, peaks)
    ms = leg["overhead"]["linear_ms"]
    res[wl.name] = {"ms": ms, "tflops": wl.flops / (ms * 1e-3) / 1e12,
                    "linear_roofline": linear_roofline(wl, ms, fp4_peak, peaks["hbm_gbs"]), **leg}
    del layer
    torch.cuda.empty_cache()
    steps = max(10, args.steps // 2)
    for M in wls.QWEN_DECODE_M:
        wl = wls.QWEN_UP_DECODE.with_m(M)
        layer = Layer(mq, wl, device)
        ab = time_ab({"linear": layer.linear, "plain": layer.plain}, steps, args.warmup, device)
        ms, ms_plain = ab["linear"], ab["plain"]
        res[f"{wl.name}_M{M}"] = {"ms": ms, "gbs": wls.alg_bytes(wl) / (ms * 1e-3) / 1e9,
                                   "frac_hbm": wls.alg_bytes(wl) / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                   "linear_roofline": linear_roofline(wl, ms, peaks["bf16_tflops"] * FP4_OVER_BF16,
                                                                      peaks["hbm_gbs"]),
                                   "vs_plain_mxfp4_pct": 100.0 * (ms / ms_plain - 1.0)}
        del layer
        torch.cuda.empty_cache()
    return res


if __name__ == "__main__":
    main()
