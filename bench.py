#!/usr/bin/env python
"""Benchmark of the fused GRPO policy-loss hot path on B200.

One step = the whole hot path on one synthetic batch: the policy and reference
lm_head GEMMs with the logsumexp / target-logit epilogue, the clipped-ratio GRPO
loss with the KL term, the in-place dlogits pass, and the dX / dW GEMMs, all
through the C ABI (pl_fused_linear_grpo) with inputs resident in HBM.  The default
workload is batch 1 x T=1024, H=4096, V=128256, bf16 (the shape of the published
B200 table of "Add SM100 CuTe DSL GRPO fast path", Liger-Kernel PR #1363).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  Under torchrun each rank runs its own batch
(weak scaling, no data-path collective); the time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import torch  # noqa: E402

METRIC = "fused GRPO fwd+bwd tokens/s and % of B200 BF16 tensor peak; loss-only GB/s"
# Published CuTe-DSL latency at batch 1, T=1024, H=4096, V=128256, BF16 on B200
# ("Add SM100 CuTe DSL GRPO fast path", "B200 results" table).
PUBLISHED_MS = {1: 6.69, 2: 12.09, 4: 23.07, 8: 43.79}
# Used only when MEASURED_PEAKS.json is absent: an earlier measurement on B200s of
# this kind -- copy bandwidth 6.65 TB/s, bf16 GEMM 1.59 PFLOP/s in a burst, settling
# near 1.4 PFLOP/s (at about 1.3 GHz) when run for seconds under the 1 kW power cap.
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
EPS_LO, EPS_HI = 0.2, 0.28
GRPO = 1  # the reduction bit of the library's mode word
GEMM_SOURCES = ["rl_post_policy_b200/csrc/gemm_tc.cu", "rl_post_policy_b200/csrc/sm100.cuh",
                "rl_post_policy_b200/csrc/gemm.h"]
LOSS_SOURCES = ["rl_post_policy_b200/csrc/loss_kernel.cu", "rl_post_policy_b200/csrc/policy_math.cuh"]
RKL_SOURCES = ["rl_post_policy_b200/csrc/reverse_kl.cu"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=2, choices=[2, 3, 4, 5])
    ap.add_argument("--chunk-rows", type=int, default=1024,
                    help="rows per chunk (multiple of 128; the pages' 1024 by default); -1: the whole "
                         "batch in one chunk")
    ap.add_argument("--no-loss-only", action="store_true")
    ap.add_argument("--no-reverse-kl", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the temperature and selective log-prob measurements")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other fused workloads (3, 4a, 4b) and the loss-only variants")
    ap.add_argument("--config-steps", type=int, default=10, help="timed steps per other fused workload")
    ap.add_argument("--only", choices=["reverse_kl", "loss_only", "loss_matrix", "configs"], default=None,
                    help="run one side measurement alone and print its JSON (for profiling); loss_matrix: "
                         "the loss kernel's 24 variants at bs=16 x 1024 and its bandwidth sweep, L2 flushed; "
                         "configs: the other fused workloads and the loss-only variants")
    ap.add_argument("--reps", type=int, default=30, help="timed calls per side measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=256, help="rows in the oracle's timed sample")
    ap.add_argument("--ref-rows", type=int, default=4, help="rows per step of the reference (oracle) arm")
    return ap.parse_args()


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        return json.loads(p.read_text()), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def sources_sha(paths) -> str:
    h = hashlib.sha256()
    for rel in paths:
        h.update((ROOT / rel).read_bytes())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, paths):
    """Per-launch DRAM bytes (read + write) from an ncu capture, taken from
    profiles/traffic.txt lines `<kernel> <sources sha> <bytes per launch>`,
    and only if the capture was taken on the current sources."""
    f = ROOT / "profiles" / "traffic.txt"
    if not f.exists():
        return None
    sha = sources_sha(paths)
    for line in f.read_text().splitlines():
        parts = line.split()
        if len(parts) == 3 and parts[0] == kernel and parts[1] == sha:
            return float(parts[2])
    return None


# ------------------------------------------------------------------ distributed
def dist_init(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        # NCCL's communicator set-up lines (rank count, devices, channels) on stderr,
        # so a run's log shows how many ranks took part
        os.environ.setdefault("NCCL_DEBUG", "INFO")
        os.environ.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
        os.environ.setdefault("NCCL_DEBUG_FILE", "/dev/stderr")
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """The SM clock and the active clock-event reasons, read through NVML every
    2 ms on a background thread while the GPU works (nvidia-smi every 100 ms
    where NVML is not available).  stop() keeps the samples taken between
    mark_start() and mark_end(), so a timed region of tens of milliseconds still
    gets a median of many readings."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    SMI_FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int, period_s: float = 0.002):
        self.period = period_s
        self.samples = []  # (time.time(), sm MHz, reason bits)
        self.t0 = self.t1 = None
        self.thread = self.proc = self.nvml = None
        self.max_mhz = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.uuid = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = (pynvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid
                           else pynvml.nvmlDeviceGetHandleByIndex(device))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            get = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
            self.get_reasons = get or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            self.nvml = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def _loop(self):
        import threading  # noqa: F401
        nv, h = self.nvml, self.handle
        while not self._stop:
            try:
                self.samples.append((time.time(), float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                     int(self.get_reasons(h))))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        self.t0 = self.t1 = None
        self.samples = []
        if self.nvml is not None:
            import threading
            self._stop = False
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
            return
        cmd = ["nvidia-smi", f"--query-gpu={self.SMI_FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def _smi_samples(self):
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        import datetime
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                mhz = float(f[1])
                self.max_mhz = float(f[2])
            except ValueError:
                continue
            bits = 0
            for (name, bit), v in zip(self.REASONS, f[5:9]):
                if v.lower().startswith("active"):
                    bits |= bit
            self.samples.append((ts, mhz, bits))

    def stop(self) -> dict:
        if self.thread is not None:
            self._stop = True
            self.thread.join(timeout=5)
            self.thread = None
            source = f"NVML every {self.period * 1e3:.0f} ms"
        elif self.proc is not None:
            self._smi_samples()
            self.proc = None
            source = "nvidia-smi every 100 ms"
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"], "samples": 0}
        total = len(self.samples)
        win = [x for x in self.samples
               if (self.t0 is None or x[0] >= self.t0) and (self.t1 is None or x[0] <= self.t1)]
        sm = [x[1] for x in win]
        bits = 0
        for x in win:
            bits |= x[2]
        reasons = sorted(name for name, bit in self.REASONS if bits & bit)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(sm) if sm else None, "reasons": reasons, "samples": len(sm),
                "samples_total": total, "source": source}


def peak_for(peaks, peak_kind, timed_s, dtype, clk=None):
    """The dense tensor peak a GEMM is held to: the measured burst figure when the
    timed region was short (under 2 s) and, where the SM clock was sampled, ran at
    the maximum clock (median within 3% of it); the sustained figure otherwise --
    after a fraction of a second of dense work the 1 kW power cap pulls the clock
    down to where the sustained figure was measured.  fp16 takes the bf16 figure
    (nominal ratio 1:1)."""
    mhz, mx = (clk or {}).get("sm_mhz"), (clk or {}).get("sm_max_mhz")
    at_max = mhz is None or not mx or mhz >= 0.97 * mx
    sustained = timed_s >= 2.0 or not at_max
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    peak = float(peaks.get(key, peaks["bf16_tflops"]))
    why = (f"timed region {timed_s:.2f} s" + (f", median SM clock {mhz:.0f} of {mx:.0f} MHz" if mhz and mx else ""))
    regime = ("sustained" if sustained else "burst") + f" ({why})"
    note = f"{peak_kind} {key}" + (" x 1.0 (fp16 nominal ratio 1:1)" if dtype == torch.float16 else "")
    return peak, f"{note}; {regime}"


# ------------------------------------------------------------------ workload
def workload_desc(w: int) -> dict:
    import synth
    d = dict(synth.WORKLOADS[w])
    d["N"] = d["bs"] * d["T"]
    return d


def chunk_rows_for(N: int, chunk_rows: int) -> int:
    """Rows per chunk: -1 = one chunk covering the batch (up to 32640 rows), else a
    multiple of 128."""
    c = N if chunk_rows < 0 else chunk_rows
    return max(128, min(32640, (c + 127) // 128 * 128))


def chunk_mode(N: int, chunk_rows: int) -> int:
    """PL_CHUNK_ROWS bits for chunk_rows_for(N, chunk_rows)."""
    import rl_post_policy_b200 as pl
    c = chunk_rows_for(N, chunk_rows)
    return pl.PL_CHUNK_ROWS(c), c


def arm_config(d: dict, chunk_rows: int, ws_world: int) -> dict:
    """The workload named in both arms' JSON lines."""
    N = d["bs"] * d["T"]
    par = (f"dp{ws_world}: one batch of {ws_world} x {N} rows sharded by sequences, dW/dbias/loss all-reduced"
           if ws_world > 1 else "dp1")
    return {"workload": f"fused GRPO fwd+bwd, bs={d['bs']} x T={d['T']} (N={N}), H={d['H']}, V={d['V']}, "
                        f"beta={d['beta']}, GRPO, eps=0.2/0.28",
            "per_gpu_rows": N, "chunk_rows": chunk_rows,
            "l2": "inputs larger than L2 (W and Wref are 1 GB each); no flush",
            "parallelism": par}


def make_fused_inputs(w: int, rank: int, chunk_rows: int = -1, beta=None):
    """Synthetic inputs on the GPU; old_lp = policy log-prob (from a forward-only
    call of the same entry point) + N(0, 0.1).  `beta` overrides the workload's."""
    import rl_post_policy_b200 as pl
    import synth
    d = workload_desc(w)
    if beta is not None:
        d["beta"] = beta
    inp = synth.fused_inputs(d["bs"], d["T"], d["H"], d["V"], d["dtype"], synth.seed_for(w, rank),
                             bias=d.get("bias", False), len_lo=d["len_lo"], len_hi=d["len_hi"],
                             fully_masked_last=d.get("fully_masked_last", False), device="cuda")
    N, V, H, bs, T = d["N"], d["V"], d["H"], d["bs"], d["T"]
    cbits, d["chunk_rows"] = chunk_mode(N, chunk_rows)
    mode = pl.dtype_mode(d["dtype"]) | pl.PL_GRPO | cbits
    wsb = pl.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, 1, int(inp["bias"] is not None))
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    loss = torch.zeros(1, device="cuda")
    logp = torch.zeros(N, device="cuda")
    zeros = torch.zeros(N, device="cuda")
    pl.check(pl.pl_fused_linear_grpo(inp["X"], inp["W"], inp["bias"], inp["targets"], None, None, zeros,
                                     inp["adv"], inp["mask"], bs, T, H, V, EPS_LO, EPS_HI, 0.0, mode, loss,
                                     None, None, None, logp, None, None, ws, wsb), "forward for old_lp")
    torch.cuda.synchronize()
    inp["old_lp"] = (logp + inp["old_noise"]).contiguous()
    return d, inp, ws, wsb, mode


class FusedStep:
    def __init__(self, d, inp, ws, wsb, mode):
        import rl_post_policy_b200 as pl
        self.pl, self.d, self.inp, self.ws, self.wsb, self.mode = pl, d, inp, ws, wsb, mode
        N, H, V = d["N"], d["H"], d["V"]
        self.loss = torch.zeros(1, device="cuda")
        self.dX = torch.empty(N, H, dtype=d["dtype"], device="cuda")
        self.dW = torch.empty(V, H, dtype=d["dtype"], device="cuda")
        self.db = torch.empty(V, dtype=d["dtype"], device="cuda") if inp["bias"] is not None else None

    def __call__(self, X=None, Xref=None, targets=None, old_lp=None, adv=None, mask=None):
        i, d = self.inp, self.d
        rc = self.pl.pl_fused_linear_grpo(
            i["X"] if X is None else X, i["W"], i["bias"], i["targets"] if targets is None else targets,
            i["Xref"] if Xref is None else Xref, i["Wref"], i["old_lp"] if old_lp is None else old_lp,
            i["adv"] if adv is None else adv, i["mask"] if mask is None else mask, d["bs"], d["T"], d["H"],
            d["V"], EPS_LO, EPS_HI, d["beta"], self.mode, self.loss, self.dX, self.dW, self.db, None, None,
            None, self.ws, self.wsb)
        if rc != 0:
            raise RuntimeError(f"pl_fused_linear_grpo: {self.pl.pl_status_string(rc)}")


class DataParallelStep:
    """One data-parallel step of the fused path (the multi-GPU partitioning the
    path has): this rank's sequences of one global batch through
    parallel.dp_fused_linear_grpo -- the rank's fused forward + backward
    normalised by its own count, the all-reduce of the count, the rank's share
    applied on the device, and the all-reduce of the loss, dW and dbias.  `ops`
    replaces the library's per-rank operations (CPU tests)."""

    def __init__(self, d, inp, chunk_rows=None, ops=None, group=None):
        from rl_post_policy_b200 import parallel
        self.parallel, self.d, self.inp, self.ops, self.group = parallel, d, inp, ops, group
        self.chunk_rows = chunk_rows
        self.out = None

    def __call__(self):
        i, d = self.inp, self.d
        self.out = self.parallel.dp_fused_linear_grpo(
            i["X"], i["W"], i["bias"], i["targets"], i["Xref"] if d["beta"] else None,
            i["Wref"] if d["beta"] else None, i["old_lp"], i["adv"], i["mask"], eps_lo=EPS_LO, eps_hi=EPS_HI,
            beta=d["beta"], reduction=GRPO, chunk_rows=self.chunk_rows, group=self.group, ops=self.ops)
        return self.out


def broadcast_weights(inp, ws_world):
    """Rank 0's W, Wref and bias on every rank: the data-parallel step holds one
    replica of the weights per rank (each rank draws its own rows)."""
    if ws_world == 1:
        return
    import torch.distributed as dist
    for k in ("W", "Wref", "bias"):
        if inp.get(k) is not None:
            dist.broadcast(inp[k], src=0)


def time_steps(fn, steps, ws_world):
    s = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws_world)
    torch.cuda.synchronize()
    a.record(s)
    for _ in range(steps):
        fn()
    b.record(s)
    torch.cuda.synchronize()
    barrier(ws_world)
    return a.elapsed_time(b)


# ------------------------------------------------------------------ loss-only kernel
def loss_only(peaks, peak_kind):
    """Bandwidth of the single-launch loss kernel on a large bf16 batch (bs=16,
    seq=2^23: inputs ~1.2 GB, far larger than L2) and the latency at bs=16 x 1024."""
    import rl_post_policy_b200 as pl
    import synth
    res = {}
    for name, (bs, seq, reps) in {"sweep": (16, 1 << 23, 50), "small": (16, 1024, 200)}.items():
        inp = synth.loss_inputs(bs, seq, torch.bfloat16, synth.seed_for(1, 1), len_lo=min(64, seq),
                                len_hi=seq, device="cuda")
        g = torch.empty_like(inp["policy_lp"])
        loss = torch.zeros(1, device="cuda")
        wsb = pl.pl_loss_workspace_bytes(bs, seq)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        mode = pl.PL_BF16 | pl.PL_BNPO

        def call():
            pl.pl_loss_ex(inp["policy_lp"], inp["old_lp"], inp["ref_lp"], inp["adv"], inp["mask"], bs, seq,
                          EPS_LO, EPS_HI, 0.04, mode, loss, g, None, None, ws, wsb)

        for _ in range(10):
            call()
        torch.cuda.synchronize()
        pl.pl_debug_timing_read()
        pl.pl_debug_timing(True)
        for _ in range(reps):
            call()
        torch.cuda.synchronize()
        pl.pl_debug_timing(False)
        ms, n = pl.pl_debug_timing_read()
        per = ms[1] / max(n[1], 1)
        tokens = bs * seq
        bytes_ = 9 * tokens  # 3 bf16 reads + bf16 grad write + 1 mask byte
        gbs = bytes_ / (per * 1e-3) / 1e9
        res[name] = {"bs": bs, "seq": seq, "us_per_call": per * 1e3, "GB_per_s": gbs,
                     "tokens_per_s": tokens / (per * 1e-3), "algorithmic_bytes": bytes_}
        if name == "small":
            # the launch-bound case again, 20 calls replayed as one CUDA graph
            from rl_post_policy_b200.pipeline import GraphedCall
            gc = GraphedCall(lambda: [call() for _ in range(20)])
            for _ in range(3):
                gc.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(10):
                gc.replay()
            e1.record()
            torch.cuda.synchronize()
            res[name]["graph_us_per_call"] = e0.elapsed_time(e1) * 1e3 / 200
        del inp, g, ws
    peak = float(peaks["hbm_gbs"])
    sw = res["sweep"]
    return {
        "metric": "loss-only GB/s", "value": sw["GB_per_s"], "unit": "GB/s",
        "workload": "loss-only BNPO fwd+bwd, bf16, beta=0.04, bs=16 x seq=8388608 (inputs > L2)",
        "roofline": {"bound": "hbm", "achieved": sw["GB_per_s"], "peak": peak, "unit": "GB/s",
                     "frac": sw["GB_per_s"] / peak, "peak_source": f"{peak_kind} hbm_gbs",
                     "traffic": recorded_traffic("loss_kernel", LOSS_SOURCES)},
        "small_workload": {"workload": "bs=16 x seq=1024 (launch-latency bound)",
                           "us_per_call": res["small"]["us_per_call"],
                           "tokens_per_s": res["small"]["tokens_per_s"],
                           "graph_us_per_call": res["small"]["graph_us_per_call"]},
    }


def loss_matrix(peaks, peak_kind, reps=20, sweep=True):
    """The loss kernel over its variants: BNPO/GRPO x beta in {0.04, 0} x fwd+bwd / fwd-only x
    bf16/fp16/fp32 at bs=16 x seq=1024 (launch-latency bound: about 144 KB per call in bf16), and
    a bandwidth sweep of bf16 BNPO fwd+bwd, beta=0.04, bs=16 x seq=2^18 ... 2^23.  A 256 MB buffer
    is written between calls so every call starts with a cold L2; only the loss kernel's own
    launches are timed (CUDA events around each)."""
    import rl_post_policy_b200 as pl
    import synth
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    peak = float(peaks["hbm_gbs"])

    def time_call(call):
        for _ in range(3):
            flush.zero_()
            call()
        torch.cuda.synchronize()
        pl.pl_debug_timing_read()
        pl.pl_debug_timing(True)
        for _ in range(reps):
            flush.zero_()
            call()
        torch.cuda.synchronize()
        pl.pl_debug_timing(False)
        ms, n = pl.pl_debug_timing_read()
        return ms[1] / max(n[1], 1)

    def one(bs, seq, dt, red, beta, grad, inp32):
        lp, old, ref = (inp32[k].to(dt) for k in ("policy_lp", "old_lp", "ref_lp"))
        g = torch.empty_like(lp) if grad else None
        loss = torch.zeros(1, device="cuda")
        wsb = pl.pl_loss_workspace_bytes(bs, seq)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        mode = pl.dtype_mode(dt) | red

        def call():
            pl.pl_loss_ex(lp, old, ref if beta else None, inp32["adv"], inp32["mask"], bs, seq, EPS_LO, EPS_HI,
                          beta, mode, loss, g, None, None, ws, wsb)

        per = time_call(call)
        esz = lp.element_size()
        tokens = bs * seq
        bytes_ = tokens * ((2 + (1 if beta else 0) + (1 if grad else 0)) * esz + 1)
        return {"bs": bs, "seq": seq, "dtype": str(dt).split(".")[-1], "reduction": "grpo" if red else "bnpo",
                "beta": beta, "grad": grad, "us_per_call": per * 1e3, "tokens_per_s": tokens / (per * 1e-3),
                "algorithmic_bytes": bytes_, "GB_per_s": bytes_ / (per * 1e-3) / 1e9,
                "frac": bytes_ / (per * 1e-3) / 1e9 / peak}

    variants = []
    inp32 = synth.loss_inputs(16, 1024, torch.float32, synth.seed_for(1), device="cuda")
    for dt in (torch.bfloat16, torch.float16, torch.float32):
        for red in (pl.PL_BNPO, pl.PL_GRPO):
            for beta in (0.04, 0.0):
                for grad in (True, False):
                    variants.append(one(16, 1024, dt, red, beta, grad, inp32))
    sweep_pts = []
    for k in (range(18, 24) if sweep else ()):
        seq = 1 << k
        inp = synth.loss_inputs(16, seq, torch.float32, synth.seed_for(1, 1), len_lo=64, len_hi=seq, device="cuda")
        sweep_pts.append(one(16, seq, torch.bfloat16, pl.PL_BNPO, 0.04, True, inp))
        del inp
    out = {"metric": "loss kernel variants and bandwidth sweep", "peak_GB_per_s": peak,
           "peak_source": f"{peak_kind} hbm_gbs", "l2": "256 MB written between calls",
           "variants_bs16_seq1024": variants}
    if sweep:
        out["sweep_bf16_bnpo_beta0.04"] = sweep_pts
    return out


# ------------------------------------------------------------------ temperature, selective log-prob
def next_rows(d, inp, ws, wsb, mode, peaks, peak_kind, reps=20):
    """The fused step at temperature 0.7 (pl_fused_linear_grpo_temp) and the fused
    selective log-prob forward + backward with an external dL/dlogp
    (pl_fused_selective_logprob), on the benchmarked workload's tensors, CUDA
    events around each library launch."""
    import rl_post_policy_b200 as pl
    import synth
    N, H, V, bs, T = d["N"], d["H"], d["V"], d["bs"], d["T"]
    dt = d["dtype"]
    loss = torch.zeros(1, device="cuda")
    dX = torch.empty(N, H, dtype=dt, device="cuda")
    dW = torch.empty(V, H, dtype=dt, device="cuda")
    db = torch.empty(V, dtype=dt, device="cuda") if inp["bias"] is not None else None
    lp = torch.empty(N, device="cuda")

    def timed(call):
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        pl.pl_debug_timing_read()
        pl.pl_debug_timing(True)
        t0 = time.perf_counter()
        for _ in range(reps):
            call()
        torch.cuda.synchronize()
        span = time.perf_counter() - t0
        pl.pl_debug_timing(False)
        ms, _ = pl.pl_debug_timing_read()
        return sum(ms) / reps, span

    def temp_call():
        pl.check(pl.pl_fused_linear_grpo_temp(inp["X"], inp["W"], inp["bias"], inp["targets"], inp["Xref"],
                                              inp["Wref"], inp["old_lp"], inp["adv"], inp["mask"], bs, T, H, V,
                                              EPS_LO, EPS_HI, d["beta"], 0.7, mode, loss, dX, dW, db, None, None,
                                              None, ws, wsb), "pl_fused_linear_grpo_temp")

    t_ms, t_span = timed(temp_call)
    smode = pl.dtype_mode(dt) | (mode & (0xFF << pl.PL_CHUNK_SHIFT))
    swsb = pl.pl_fused_selective_logprob_workspace_bytes(N, H, V, smode, 1, int(db is not None))
    sws = torch.zeros(swsb, dtype=torch.uint8, device="cuda")
    g = synth.normal((N,), synth.seed_for(2, 7), std=1e-3, device="cuda")

    def sel_call():
        pl.check(pl.pl_fused_selective_logprob(inp["X"], inp["W"], inp["bias"], inp["targets"], N, H, V, smode, g,
                                               lp, dX, dW, db, sws, swsb), "pl_fused_selective_logprob")

    s_ms, s_span = timed(sel_call)
    del sws, dX, dW
    f_temp, f_sel = 8.0 * N * H * V, 6.0 * N * H * V
    t_peak, t_src = peak_for(peaks, peak_kind, t_span, dt)
    s_peak, s_src = peak_for(peaks, peak_kind, s_span, dt)
    return {
        "temperature": {"workload": f"fused GRPO fwd+bwd at temperature 0.7, N={N}, H={H}, V={V}",
                        "ms": t_ms, "tokens_per_s": N / (t_ms * 1e-3), "tflops": f_temp / (t_ms * 1e-3) / 1e12,
                        "frac_of_peak": f_temp / (t_ms * 1e-3) / 1e12 / t_peak, "peak": t_peak,
                        "peak_source": t_src},
        "selective_logprob": {"workload": f"fused selective log-prob fwd + bwd (dX, dW), N={N}, H={H}, V={V}",
                              "ms": s_ms, "tokens_per_s": N / (s_ms * 1e-3), "tflops": f_sel / (s_ms * 1e-3) / 1e12,
                              "frac_of_peak": f_sel / (s_ms * 1e-3) / 1e12 / s_peak, "peak": s_peak,
                              "peak_source": s_src},
    }


# ------------------------------------------------------------------ reverse KL
def reverse_kl(peaks, peak_kind, reps=30):
    """Reverse-KL self-distillation at the model card's example shape (bs=4,
    seq=256, V=248320, bf16, ~1 GB of logits per call, far larger than L2):
    forward+gradient and forward-only, CUDA events around each launch."""
    import rl_post_policy_b200 as pl
    import synth
    w = synth.RKL_WORKLOADS[1]
    bs, seq, V = w["bs"], w["seq"], w["V"]
    N = bs * seq
    inp = synth.reverse_kl_inputs(bs, seq, V, w["dtype"], synth.seed_for(46, 1), device="cuda")
    s, t, m = inp["student"], inp["teacher"], inp["mask"]
    n_valid = int(m.sum().item())
    g = torch.empty_like(s)
    loss = torch.zeros(1, device="cuda")
    wsb = pl.pl_reverse_kl_workspace_bytes(N, V)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    esz = s.element_size()
    res = {}
    for name, grad in (("fwd_bwd", g), ("fwd", None)):
        def call():
            pl.pl_reverse_kl(s, t, m, N, V, pl.PL_BF16, loss, grad, None, None, ws, wsb)

        for _ in range(min(3, reps)):
            call()
        torch.cuda.synchronize()
        pl.pl_debug_timing_read()
        pl.pl_debug_timing(True)
        for _ in range(reps):
            call()
        torch.cuda.synchronize()
        pl.pl_debug_timing(False)
        ms, n = pl.pl_debug_timing_read()
        per = ms[2] / max(n[2], 1)
        # valid rows: read student + teacher (+ write the gradient); masked rows: the zero
        # gradient only; plus the mask
        bytes_ = n_valid * V * esz * (3 if grad is not None else 2) + N
        if grad is not None:
            bytes_ += (N - n_valid) * V * esz
        res[name] = {"us_per_call": per * 1e3, "GB_per_s": bytes_ / (per * 1e-3) / 1e9,
                     "rows_per_s": N / (per * 1e-3), "algorithmic_bytes": bytes_}
    del s, t, g, inp
    peak = float(peaks["hbm_gbs"])
    fb = res["fwd_bwd"]
    return {
        "metric": "reverse-KL GB/s", "value": fb["GB_per_s"], "unit": "GB/s",
        "workload": f"reverse KL fwd+grad, bf16, bs={bs} x seq={seq}, V={V}, mask uniform>0.2 "
                    f"({n_valid} valid rows)",
        "roofline": {"bound": "hbm", "achieved": fb["GB_per_s"], "peak": peak, "unit": "GB/s",
                     "frac": fb["GB_per_s"] / peak, "peak_source": f"{peak_kind} hbm_gbs",
                     "traffic": recorded_traffic("reverse_kl_kernel_grad", RKL_SOURCES)},
        "us_per_call": fb["us_per_call"],
        "forward_only": {"us_per_call": res["fwd"]["us_per_call"], "GB_per_s": res["fwd"]["GB_per_s"],
                         "frac": res["fwd"]["GB_per_s"] / peak,
                         "traffic": recorded_traffic("reverse_kl_kernel_fwd", RKL_SOURCES)},
    }


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(inp, d, rows):
    """The fp64 oracle on the first `rows` rows of the batch (one sequence of
    `rows` tokens): policy + reference forward over the full vocabulary, the
    loss, and dX / dW / dbias for those rows.  Returns (seconds, threads)."""
    import oracle
    cpu = {k: (v[:rows].cpu() if k in ("X", "Xref", "targets", "old_lp") else v)
           for k, v in inp.items() if isinstance(v, torch.Tensor)}
    W = inp["W"].cpu()
    Wref = inp["Wref"].cpu() if inp.get("Wref") is not None else None
    bias = inp["bias"].cpu() if inp.get("bias") is not None else None
    mask = inp["mask"].reshape(-1)[:rows].reshape(1, rows).cpu()
    adv = inp["adv"][:1].cpu()
    t0 = time.perf_counter()
    oracle.fused_grpo(cpu["X"], W, bias, cpu["targets"], cpu.get("Xref"), Wref,
                      cpu["old_lp"].reshape(1, rows), adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI,
                      beta=d["beta"], reduction=oracle.GRPO)
    return time.perf_counter() - t0, oracle.threads()


# ------------------------------------------------------------------ arms
def run_reference(args):
    ws_world, rank = dist_init(args)
    if rank != 0:
        return
    d = workload_desc(args.workload)
    import oracle  # noqa: F401
    # Inputs: the same recipe, generated on the CPU (no GPU work on this arm).
    import synth
    rows = max(1, min(args.ref_rows, d["N"]))
    inp = synth.fused_inputs(1, rows, d["H"], d["V"], d["dtype"], synth.seed_for(args.workload),
                             bias=d.get("bias", False), len_lo=rows, len_hi=rows)
    import oracle as orc
    _, lp, _ = orc.lm_head_logprob(inp["X"], inp["W"], inp["bias"], inp["targets"])
    inp["old_lp"] = (torch.from_numpy(lp) + inp["old_noise"].double()).float()
    times = []
    for i in range(args.warmup + args.steps):
        t, cores = oracle_sample(inp, d, rows)
        if i >= args.warmup:
            times.append(t)
    per = sum(times) / len(times)
    val = rows / per
    sample = (f"{rows} rows (one sequence) of the workload per step, value = rows / time: policy+reference "
              f"forward over V={d['V']}, loss, dX/dW/dbias, fp64")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(d, chunk_rows_for(d["N"], args.chunk_rows), args.gpus),
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }), flush=True)


def fused_roofline(d, steps, kms, kn, ms_per_step, timed_s, peaks, peak_kind, clk=None):
    """Roofline of the dominant kernel (the tcgen05 GEMM) over a timed region:
    algorithmic flops per GEMM launch over the mean launch time (CUDA events on
    the launching stream), against the dense tensor peak for the region's length,
    with the fractions of both measured peaks beside it."""
    N, H, V = d["N"], d["H"], d["V"]
    flops_step = (8 if d["beta"] != 0 else 6) * N * H * V
    gemm_ms = kms[0] / max(kn[0], 1)
    gemm_flops_launch = flops_step * steps / max(kn[0], 1)
    achieved = gemm_flops_launch / (gemm_ms * 1e-3) / 1e12
    peak, src = peak_for(peaks, peak_kind, timed_s, d["dtype"], clk)
    step_tflops = flops_step / (ms_per_step * 1e-3) / 1e12
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": src, "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained,
            "kernel": "gemm_kernel (tcgen05 persistent GEMM)", "launch_ms": gemm_ms, "launches": kn[0],
            "flops_per_step": flops_step, "share_of_step": kms[0] / max(sum(kms), 1e-9),
            "step_tflops": step_tflops, "step_frac_of_peak": step_tflops / peak,
            "step_frac_of_burst": step_tflops / burst, "step_frac_of_sustained": step_tflops / sustained}


def measure_fused(w, chunk_rows, steps, warmup, peaks, peak_kind, beta=None):
    """One fused workload at one chunk size: `warmup` untimed steps, then `steps`
    timed with CUDA events (and the GEMM launches with their own events), with
    the SM clock sampled inside the timed region."""
    import rl_post_policy_b200 as pl
    d, inp, ws, wsb, mode = make_fused_inputs(w, 0, chunk_rows, beta)
    step = FusedStep(d, inp, ws, wsb, mode)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    pl.check(pl.pl_device_status(ws), "device status after warm-up")
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    pl.pl_debug_timing_read()
    pl.pl_debug_timing(True)
    clocks.mark_start()
    t0 = time.perf_counter()
    elapsed = time_steps(step, steps, 1)
    span = time.perf_counter() - t0
    clocks.mark_end()
    pl.pl_debug_timing(False)
    clk = clocks.stop()
    kms, kn = pl.pl_debug_timing_read()
    pl.check(pl.pl_device_status(ws), "device status after timing")
    ms = elapsed / steps
    N = d["N"]
    rl = fused_roofline(d, steps, kms, kn, ms, span, peaks, peak_kind, clk)
    out = {"chunk_rows": d["chunk_rows"], "chunks": (N + d["chunk_rows"] - 1) // d["chunk_rows"],
           "steps": steps, "ms": ms, "tokens_per_s": N / (ms * 1e-3), "tflops": rl["step_tflops"],
           "frac": rl["step_frac_of_peak"], "peak": rl["peak"], "peak_source": rl["peak_source"],
           "frac_of_burst": rl["step_frac_of_burst"], "frac_of_sustained": rl["step_frac_of_sustained"],
           "gemm_tflops": rl["achieved"], "gemm_frac": rl["frac"], "gemm_frac_of_burst": rl["frac_of_burst"],
           "gemm_ms_per_step": kms[0] / steps, "other_kernels_ms_per_step": (kms[1] + kms[2]) / steps,
           "clocks": clk}
    if clk.get("sm_mhz"):
        out["ms_x_sm_ghz"] = ms * clk["sm_mhz"] / 1e3
    del step, inp, ws
    torch.cuda.empty_cache()
    return out


# The other fused workloads: name -> (workload number, beta).  Numbers as in synth.WORKLOADS.
OTHER_CONFIGS = {
    "w3_fp16_bias_bs4_T1024_H4096_V128256_beta0.04": (3, 0.04),
    "w4a_bf16_bs8_T1024_H4096_V128256_beta0.04": (4, 0.04),
    "w4a_bf16_bs8_T1024_H4096_V128256_beta0": (4, 0.0),
    "w4b_bf16_bs8_T1024_H4000_V152064_beta0.04": (5, 0.04),
    "w4b_bf16_bs8_T1024_H4000_V152064_beta0": (5, 0.0),
}


def other_configs(peaks, peak_kind, steps):
    """Every other fused workload at the pages' 1024-row chunks and with one
    chunk spanning the batch, plus the loss-only kernel's 24 variants at
    bs=16 x 1024 (the launch-bound loss workload)."""
    import synth
    out = {}
    for name, (w, beta) in OTHER_CONFIGS.items():
        d = synth.WORKLOADS[w]
        N = d["bs"] * d["T"]
        out[name] = {"workload": f"fused GRPO fwd+bwd, bs={d['bs']} x T={d['T']} (N={N}), H={d['H']}, "
                                 f"V={d['V']}, {str(d['dtype']).split('.')[-1]}, beta={beta}"
                                 + (", policy bias" if d.get("bias") else "")
                                 + (", last sequence fully masked" if d.get("fully_masked_last") else ""),
                     "flops_per_step": (8 if beta else 6) * N * d["H"] * d["V"],
                     "chunked_1024": measure_fused(w, 1024, steps, 2, peaks, peak_kind, beta),
                     "whole_batch": measure_fused(w, -1, steps, 2, peaks, peak_kind, beta)}
    out["w1_loss_only_variants_bs16_seq1024"] = loss_matrix(peaks, peak_kind, sweep=False)
    return out


def run_ours(args):
    ws_world, rank = dist_init(args)
    import rl_post_policy_b200 as pl
    peaks, peak_kind = load_peaks()
    if args.only:
        if rank == 0:
            if args.only == "reverse_kl":
                out = reverse_kl(peaks, peak_kind, args.reps)
            elif args.only == "loss_matrix":
                out = loss_matrix(peaks, peak_kind)
            elif args.only == "configs":
                out = other_configs(peaks, peak_kind, args.config_steps)
            else:
                out = loss_only(peaks, peak_kind)
            print(json.dumps(out), flush=True)
        return
    d, inp, ws, wsb, mode = make_fused_inputs(args.workload, rank, args.chunk_rows)
    N, H, V = d["N"], d["H"], d["V"]
    single = FusedStep(d, inp, ws, wsb, mode)
    if ws_world > 1:
        # one global batch sharded by sequences: the same weights on every rank
        broadcast_weights(inp, ws_world)
        step = DataParallelStep(d, inp, chunk_rows=d["chunk_rows"])
    else:
        step = single
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    pl.check(pl.pl_device_status(ws), "device status after warm-up")

    # ---- device-resident timed region ----
    clocks = ClockSampler(torch.cuda.current_device())
    pl.pl_debug_timing_read()
    launches0 = pl.pl_debug_launch_count()
    clocks.start()
    pl.pl_debug_timing(True)
    clocks.mark_start()
    t0 = time.perf_counter()
    elapsed = time_steps(step, args.steps, ws_world)
    span = time.perf_counter() - t0
    clocks.mark_end()
    pl.pl_debug_timing(False)
    clk = clocks.stop()
    launches = pl.pl_debug_launch_count() - launches0
    kms, kn = pl.pl_debug_timing_read()
    pl.check(pl.pl_device_status(ws), "device status after timing")
    if ws_world > 1:
        from rl_post_policy_b200 import parallel
        for w in parallel._default_ops()._ws.values():
            pl.check(pl.pl_device_status(w), "device status of the data-parallel step")
    t_max = max_over_ranks(elapsed, ws_world)
    ms_per_step = t_max / args.steps
    total_tokens = sum_over_ranks(float(N * args.steps), ws_world)
    value = total_tokens / (t_max * 1e-3)
    roofline = fused_roofline(d, args.steps, kms, kn, ms_per_step, max_over_ranks(span, ws_world), peaks,
                              peak_kind, clk)
    roofline["traffic"] = recorded_traffic("gemm_kernel", GEMM_SOURCES)
    if clk.get("sm_mhz"):
        roofline["gemm_ms_x_sm_ghz"] = roofline["launch_ms"] * clk["sm_mhz"] / 1e3

    # ---- end to end through the C ABI from pinned host buffers ----
    # Every step copies its inputs from pinned host memory (on a copy stream, one
    # step ahead, so the copy of step i+1 overlaps step i; step 0's copy is inside
    # the timed region too) and reads the step's loss back to the host.
    from rl_post_policy_b200.pipeline import InputPrefetcher
    host = {k: inp[k].cpu().pin_memory() for k in ("X", "Xref", "targets", "old_lp", "adv", "mask")}
    pf = InputPrefetcher({k: inp[k] for k in host})
    loss_host = torch.zeros(1).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())

    def e2e_run(steps):
        pf.prefetch(host)
        for i in range(steps):
            dev = pf.next()
            if i + 1 < steps:
                pf.prefetch(host)
            if ws_world > 1:
                step.inp = dict(inp, **dev)
                step()
                loss_host.copy_(step.out["loss"], non_blocking=True)
            else:
                step(**dev)
                loss_host.copy_(step.loss, non_blocking=True)
            pf.release()
        pf.finish()

    e2e_run(2)
    e2e_ms = max_over_ranks(time_steps(lambda: e2e_run(args.steps), 1, ws_world), ws_world) / args.steps
    e2e_val = total_tokens / args.steps / (e2e_ms * 1e-3)
    if ws_world > 1:
        step.inp = inp

    extra = {}
    if ws_world > 1:
        # the same step with no collective: each rank's own batch (weak scaling, independent batches)
        for _ in range(2):
            single()
        ind = max_over_ranks(time_steps(single, args.steps, ws_world), ws_world)
        extra["independent_batches"] = {
            "what": "each rank runs its own batch, no collective", "ms_per_step": ind / args.steps,
            "value": total_tokens / (ind * 1e-3), "unit": "tokens/s"}

    def side(fn, *fargs):
        # The bandwidth-bound side measurements come after seconds of power-capped
        # GEMM work, which leaves the SM clock low for a while; they get an idle
        # pause first and carry the clocks sampled while they ran.
        torch.cuda.synchronize()
        time.sleep(2.0)
        cs = ClockSampler(torch.cuda.current_device())
        cs.start()
        out = fn(*fargs)
        torch.cuda.synchronize()
        out["clocks"] = cs.stop()
        return out

    if rank == 0 and ws_world == 1 and not args.no_loss_only:
        extra["loss_only"] = side(loss_only, peaks, peak_kind)
    if rank == 0 and ws_world == 1 and not args.no_reverse_kl:
        extra["reverse_kl"] = side(reverse_kl, peaks, peak_kind, args.reps)
    if rank == 0 and ws_world == 1 and not args.no_next_rows:
        extra.update(next_rows(d, inp, ws, wsb, mode, peaks, peak_kind))
    cpu = None
    if rank == 0 and ws_world == 1 and not args.no_cpu_baseline:
        rows = max(1, min(args.cpu_rows, N))
        secs, cores = oracle_sample(inp, d, rows)
        cpu = {"value": rows / secs, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"first {rows} rows of the batch as one sequence: policy+reference forward over "
                         f"V={V}, GRPO loss, dX/dW/dbias, fp64 ({secs:.1f} s)"}
    if rank == 0 and ws_world == 1 and not args.no_configs:
        del single, step, ws
        torch.cuda.empty_cache()
        extra["configs"] = other_configs(peaks, peak_kind, args.config_steps)

    if rank == 0:
        bsz = d["bs"]
        pub = PUBLISHED_MS.get(bsz) if (args.workload in (2, 4) and H == 4096 and V == 128256) else None
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": (value / ws_world) / (N / (pub * 1e-3)) if pub else None,
            "dtype": "bf16" if d["dtype"] == torch.bfloat16 else "fp16", "data": "synthetic",
            "config": arm_config(d, d["chunk_rows"], ws_world),
            "clocks": clk, "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                                   "d2h_bytes_per_step": 4, "ms_per_step": e2e_ms},
            "gpu_launches": launches, "roofline": roofline, "cpu_baseline": cpu,
            "kernel_ms_per_step": {"gemm": kms[0] / args.steps, "loss_kernel": kms[1] / args.steps,
                                   "other": kms[2] / args.steps},
        }
        line.update(extra)
        print(json.dumps(line), flush=True)
    if ws_world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
