"""Benchmark of the Slim attention decode step (K-only cache) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
                    [--no-extras]

One step = one slim_decode_step over the whole batch: append this step's k,
scores of q against the K cache, softmax, V = K·W_KV by the selected
ordering, output. The headline workload is the largest one that fits one GPU:
7B-style MHA decode, d=4096, H=32 (d_h=128), B=16 sequences with ragged
cached lengths uniform in [16384, 32768], bf16 K cache, fp32 accumulation.
Inputs are seeded synthetic data (X ~ N(0,1), W_K = orthogonal·diag(U[0.5,2]),
W_V ~ N(0,1/d)) from only_cache_exact_b200.synth; the K cache is filled by the
library's own prompt-phase kernel from prompt rows drawn on the device.

Timing: W untimed warm-up steps and one untimed replay of every captured CUDA
graph, then exactly K steps replayed from CUDA graphs, bracketed by a barrier
and a device synchronise, timed with CUDA events on the launching stream; the
max over ranks is reported. Between steps either the K cache alone exceeds
twice the 126 MB L2, or enough copies of the cache, W_KV and the step inputs
rotate to exceed it, or (tiny workloads) a 256 MB buffer is written before
each step, which is then timed alone; `config.l2` says which. Lengths are reset
before each measured region; each step appends one row, so the attended length
grows by one per step of the same buffer set and the byte counts follow the
actual lengths.

With one GPU the same line also carries one record per other workload
(`workloads`), each with its own step count, roofline and oracle baseline;
the ordering (a)/(b) sweep over T = 1K..128K at d=4096, H=32, B=1
(`sweep`); the prompt-phase projection (`prefill`); and ordering (a) on the
d=1024 workload (`variant_a`).

Multi-GPU: sequences are independent, so every rank runs its own batch
(weak scaling, no collective on the data path); value = all ranks' steps /
max-over-ranks time.

--impl reference times the float64 CPU oracle (standard MHA with explicit K
and V caches) on the host cores: a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "slim decode steps/s and achieved HBM GB/s vs B200 peak (K-only cache)"

WORKLOADS = {
    # name: d, H, B, T (cached rows before the first step), dtype, append, steps (sub-record step count)
    "d4096_h32_b16_t16k_32k": dict(d=4096, H=32, B=16, T=(16384, 32768), dtype="bf16", append=True, steps=20,
                                   desc="7B-style MHA decode, d=4096 H=32 d_h=128, B=16, ragged T in [16K,32K], "
                                        "bf16 K cache, fp32 accumulation"),
    "d256_h4_b1_t128_f32": dict(d=256, H=4, B=1, T=128, dtype="f32", append=True, steps=16,
                                desc="single MHA layer fp32, d=256 H=4 d_h=64, B=1, 128-token prompt then "
                                     "16 decode steps"),
    "d1024_h16_b8_t4096": dict(d=1024, H=16, B=8, T=4096, dtype="bf16", append=True, steps=64,
                               desc="decode step, d=1024 H=16 d_h=64, B=8, T=4096 bf16 K cache, fp32 accumulation"),
    "d1280_h20_b64_t1500_cross": dict(d=1280, H=20, B=64, T=1500, dtype="bf16", append=False, steps=448,
                                      desc="encoder-decoder cross-attention decode, d=1280 H=20 d_h=64, B=64, "
                                           "fixed 1500-row encoder K cache, 448 steps"),
    "d4096_h32_b1_t8192": dict(d=4096, H=32, B=1, T=8192, dtype="bf16", append=True, steps=64,
                               desc="long-context layer, d=4096 H=32, B=1: 64 decode steps after the "
                                    "8192-token prompt"),
    "d4096_h32_b1_t131072": dict(d=4096, H=32, B=1, T=131072 - 80, cap=131072, dtype="bf16", append=True,
                                 steps=64, desc="long-context decode, d=4096 H=32, B=1, 64 steps at the end of "
                                                "the 131072-row K cache"),
}
DEFAULT = "d4096_h32_b16_t16k_32k"
SUBRECORDS = ["d256_h4_b1_t128_f32", "d1024_h16_b8_t4096", "d1280_h20_b64_t1500_cross", "d4096_h32_b1_t8192",
              "d4096_h32_b1_t131072"]
KV_BASELINE = ["d1024_h16_b8_t4096", "d4096_h32_b16_t16k_32k", "d1280_h20_b64_t1500_cross", "d4096_h32_b1_t131072"]
FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT, choices=sorted(WORKLOADS))
    ap.add_argument("--rot", type=int, default=0, help="buffer sets rotated (0: automatic)")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling runs)")
    ap.add_argument("--no-extras", action="store_true", help="headline line only (no sub-records, sweep, CPU legs)")
    ap.add_argument("--ref-seconds", type=float, default=20.0, help="CPU time budget of --impl reference")
    ap.add_argument("--variant", default="auto", choices=["auto", "a", "b"],
                    help="ordering of the timed steps (auto: the measured table; profiling runs pin one)")
    ap.add_argument("--from-x", action="store_true",
                    help="time the step from its input rows (slim_decode_step_x: q and k formed on the device)")
    return ap.parse_args()


# ------------------------------------------------------------------------------------------ helpers
def dist_init(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    return rank, world, local, pg


def seq_lengths(w, seed=0):
    from only_cache_exact_b200 import synth
    T = w["T"]
    if isinstance(T, tuple):
        return synth.make_lengths(w["B"], T[0], T[1], seed)
    return np.full(w["B"], T, dtype=np.int32)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    def __init__(self, dev_index):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _names(self, mask):
        nv = self.nv
        table = {
            "sw_power_cap": getattr(nv, "nvmlClocksThrottleReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwPowerBrakeSlowdown", 0x80),
        }
        return [k for k, v in table.items() if mask & v]

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.005)

    def sample(self):
        if self.nv is None:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons.update(self._names(self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)))
        except Exception:
            pass

    def __enter__(self):
        self.sample()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self.t.join()
        self.sample()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def kernel_sources_sha():
    """Hash of the split kernel's sources; a stored ncu figure is used only while it matches."""
    h = hashlib.sha256()
    for f in ("decode_b_tc.cu", "split_plan.cuh", "ptx.cuh"):
        h.update(open(os.path.join(ROOT, "only_cache_exact_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profile_traffic(workload):
    """DRAM bytes per split-kernel launch from profiles/decode_b_tc_<workload>.json (an ncu capture),
    if the kernel sources are unchanged since it was taken; else None."""
    path = os.path.join(ROOT, "profiles", f"decode_b_tc_{workload}.json")
    if not os.path.exists(path):
        return None
    try:
        j = json.load(open(path))
        if j.get("source_sha256_16") != kernel_sources_sha():
            return None
        return float(j["dram_bytes_per_launch"])
    except (ValueError, KeyError, OSError):
        return None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def cpu_oracle_rate(w, budget_s=12.0):
    """Oracle step time on the host: float64 standard MHA with explicit K and V caches, one sequence
    at a time (sequences are independent), as many steps as fit in the budget, scaled to the batch."""
    from threadpoolctl import threadpool_info

    from oracle import slim_oracle as O
    d, H = w["d"], w["H"]
    lens = seq_lengths(w)
    T = int(np.max(lens)) + (1 if w["append"] else 0)
    rng = np.random.default_rng(0)
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    q = rng.standard_normal(d)
    O.mha_decode(q, K, V, H)  # warm
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s or n == 0:
        O.mha_decode(q, K, V, H)
        n += 1
    per_seq = (time.perf_counter() - t0) / n
    # one step = every sequence of the batch (ragged: scaled by the attended rows)
    step_s = per_seq * float(np.sum(lens + (1 if w["append"] else 0))) / T
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return 1.0 / step_s, threads, n, T


# ------------------------------------------------------------------------------------------ one workload
class Workload:
    """Device state of one workload: K cache(s) filled by the prompt-phase kernel, W_KV, step inputs."""

    def __init__(self, name, S, dev, rank=0, world=1, max_steps=256, rot=0, mha=False, batch=0, variant=None,
                 from_x=False):
        import torch

        from only_cache_exact_b200 import params, replicas, synth
        self.name, self.S, self.dev = name, S, dev
        w = self.w = dict(WORKLOADS[name])
        if batch:
            w["B"] = batch
        self.mha = mha  # standard MHA step over K and V caches (the baseline) instead of the Slim step
        d, H, B = w["d"], w["H"], w["B"]
        self.d, self.H, self.B = d, H, B
        self.append = w["append"]
        self.lens0 = seq_lengths(w)
        gids = replicas.global_sequence_ids(rank, world, B)  # this rank's own token streams
        self.tdt = torch.bfloat16 if w["dtype"] == "bf16" else torch.float32
        self.dt_code = S.SLIM_BF16 if w["dtype"] == "bf16" else S.SLIM_F32
        self.esz = 2 if w["dtype"] == "bf16" else 4
        set_bytes = int(np.sum(self.lens0)) * d * self.esz * (2 if mha else 1) + (0 if mha else d * d * self.esz)
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        if rot:
            self.rot = rot
        elif set_bytes >= 2 * l2:
            self.rot = 1
        else:
            self.rot = min(8, -(-2 * l2 // set_bytes) + 1)
        self.flush = self.rot * set_bytes < 2 * l2  # too small to rotate past L2: flush before each step
        if self.flush:
            self.rot = 1
        per_set_appends = -(-max_steps // self.rot) + 4 if self.append else 0
        self.cap = int(np.max(self.lens0)) + per_set_appends + 8
        if "cap" in w:
            self.cap = min(self.cap, int(w["cap"]))
            if self.append and self.cap < int(np.max(self.lens0)) + -(-max_steps // self.rot):
                raise ValueError(f"{name}: {max_steps} steps do not fit the {self.cap}-row cache")
        wts = synth.make_weights(d, 0, w["dtype"])
        self.W_K = synth.to_storage(wts.W_K, w["dtype"]).to(dev)
        W_KV0 = params.make_wkv(wts.W_K, wts.W_V, dtype=self.tdt, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        K0 = torch.zeros(B, self.cap, d, dtype=self.tdt, device=dev)
        V0 = torch.zeros(B, self.cap, d, dtype=self.tdt, device=dev) if mha else None
        W_V = synth.to_storage(synth.round_to(wts.W_V, w["dtype"]), w["dtype"]).to(dev) if mha else None
        lens_dev0 = torch.zeros(B, dtype=torch.int32, device=dev)
        lens_v = torch.zeros(B, dtype=torch.int32, device=dev)
        t = time.perf_counter()
        for b in range(B):
            n = int(self.lens0[b])
            for r0 in range(0, n, 8192):
                r1 = min(n, r0 + 8192)
                Xb = synth.make_tokens_device(r1 - r0, d, 1000 + r0 // 8192, gids[b], w["dtype"], device=dev)
                S.slim_prefill_k(Xb.view(1, r1 - r0, d), self.W_K, K0[b:b + 1], lens_dev0[b:b + 1], self.status)
                if mha:
                    S.slim_prefill_k(Xb.view(1, r1 - r0, d), W_V, V0[b:b + 1], lens_v[b:b + 1], self.status)
        torch.cuda.synchronize()
        self.fill_s = time.perf_counter() - t
        self.lens_dev0 = lens_dev0
        x_new = np.stack([synth.make_tokens(1, d, 0, gids[b], w["dtype"], part=2)[0] for b in range(B)])
        self.wts, self.x_new = wts, x_new
        self.q0 = torch.from_numpy(x_new @ wts.W_Q).float().to(dev)
        self.k0 = (synth.to_storage(synth.round_to(x_new @ wts.W_K, w["dtype"]), w["dtype"]).to(dev)
                   if self.append else None)
        self.v0 = (synth.to_storage(synth.round_to(x_new @ wts.W_V, w["dtype"]), w["dtype"]).to(dev)
                   if self.append and mha else None)
        self.sets = []
        for i in range(self.rot):
            st_ = dict(K=K0 if i == 0 else K0.clone(), lens=lens_dev0.clone(),
                       q=self.q0.clone(), k=None if self.k0 is None else self.k0.clone(),
                       out=torch.empty(B, d, dtype=torch.float32, device=dev))
            if mha:
                st_.update(V=V0 if i == 0 else V0.clone(), v=None if self.v0 is None else self.v0.clone(),
                           ws=S.alloc_mha_workspace(self.dt_code, B, d, H, self.cap, device=dev))
            else:
                st_.update(W_KV=W_KV0 if i == 0 else W_KV0.clone(),
                           ws=S.alloc_workspace(self.dt_code, B, d, H, self.cap, S.SLIM_AUTO, device=dev))
            self.sets.append(st_)
        self.t_hint = int(np.max(self.lens0))
        self.variant = S.SLIM_AUTO if variant is None else variant
        self.from_x = from_x and not mha
        if self.from_x:
            # the step's input rows and the stored W_Q: every timed step forms q (and k) itself
            self.W_Q = synth.to_storage(synth.round_to(wts.W_Q, w["dtype"]), w["dtype"]).to(dev)
            self.x = synth.to_storage(x_new, w["dtype"]).to(dev)
            nws = S.slim_decode_step_x_workspace_bytes(self.dt_code, B, d, H, self.cap, S.SLIM_AUTO)
            for st_ in self.sets:
                st_["ws_x"] = torch.empty(nws, dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.Stream(device=dev)
        self.flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if self.flush else None
        torch.cuda.synchronize()

    def step(self, i, variant=None):
        S = self.S
        s = self.sets[i % self.rot]
        if self.mha:
            S.slim_mha_decode_step(s["q"], s["k"], s["v"], s["K"], s["V"], s["lens"], self.H, s["out"], s["ws"],
                                   self.status)
            return
        v = self.variant if variant is None else variant
        if self.from_x:
            S.slim_decode_step_x(self.x, self.W_Q, self.W_K if self.append else None, s["K"], s["lens"], s["W_KV"],
                                 self.H, s["out"], s["ws_x"], self.status, variant=v, t_hint=self.t_hint)
            return
        S.slim_decode_step(s["q"], s["k"], s["K"], s["lens"], s["W_KV"], self.H, s["out"], s["ws"], self.status,
                           variant=v, t_hint=self.t_hint)

    def reset_lengths(self):
        import torch
        for st_ in self.sets:
            st_["lens"].copy_(self.lens_dev0)
        torch.cuda.synchronize()

    def rows_attended(self, nsteps):
        """Rows all sequences attend over in nsteps steps started from freshly reset lengths."""
        base = int(self.lens0.astype(np.int64).sum())
        return sum(base + (self.B * ((s_ // self.rot) + 1) if self.append else 0) for s_ in range(nsteps))

    def algorithmic_bytes(self, nsteps):
        """(split kernel bytes per launch, step bytes) averaged over nsteps steps: K rows attended
        (incl. the appended one) read once, q, k_new read and written; the step adds W_KV once and
        the output."""
        caches = 2 if self.mha else 1
        per_step_const = self.B * self.d * 4 + (2 * caches * self.B * self.d * self.esz if self.append else 0)
        kernel = caches * self.rows_attended(nsteps) * self.d * self.esz / nsteps + per_step_const
        return kernel, kernel + (0 if self.mha else self.d * self.d * self.esz) + self.B * self.d * 4

    def time_steps(self, K_steps, W_steps, pg=None, sample_clocks=None):
        """Device time of exactly K_steps steps after W_steps warm-up steps (ms)."""
        import torch
        stream = self.stream
        with torch.cuda.stream(stream):
            for i in range(W_steps):
                self.step(i)
        stream.synchronize()
        if self.flush:
            # tiny workload: every step runs after a write of 256 MB, timed alone
            self.reset_lengths()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(K_steps)]
            if pg:
                pg.barrier()
            torch.cuda.synchronize()
            with sample_clocks or _Null():
                with torch.cuda.stream(stream):
                    for i in range(K_steps):
                        self.flush_buf.fill_(i & 0xFF)
                        evs[i][0].record(stream)
                        self.step(i)
                        evs[i][1].record(stream)
                stream.synchronize()
            return sum(a.elapsed_time(b) for a, b in evs)
        G = max(self.rot, min(K_steps, 256) // self.rot * self.rot)
        full, rem = divmod(K_steps, G)

        def capture(nsteps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for j in range(nsteps):
                    self.step(j)
            return g

        g_full = capture(G) if full else None
        g_rem = capture(rem) if rem else None
        torch.cuda.synchronize()
        # one untimed replay of each graph (uploads it), then back to the starting lengths
        self.reset_lengths()
        with torch.cuda.stream(stream):
            for g in (g_full, g_rem):
                if g is not None:
                    g.replay()
        stream.synchronize()
        self.reset_lengths()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        with sample_clocks or _Null():
            ev0.record(stream)
            with torch.cuda.stream(stream):
                for _ in range(full):
                    g_full.replay()
                if g_rem is not None:
                    g_rem.replay()
            ev1.record(stream)
            ev1.synchronize()
        ms = ev0.elapsed_time(ev1)
        del g_full, g_rem
        return ms

    def split_kernel_ms(self, n):
        """Average duration of the split kernel (the one that streams the K cache) over n steps, from
        event pairs the library records around it on its stream; steps queued behind a spin kernel so
        the GPU never waits for the host."""
        import torch
        S = self.S
        self.reset_lengths()
        S.slim_timing_enable(n)
        with torch.cuda.stream(self.stream):
            torch.cuda._sleep(int(50e6))
            for j in range(n):
                if self.flush:
                    self.flush_buf.fill_(j & 0xFF)
                self.step(j)
        self.stream.synchronize()
        ms = S.slim_timing_read(n)
        S.slim_timing_enable(0)
        return float(np.mean(ms)) if ms else None

    def e2e_ms(self, nsteps, pg=None):
        """Per-step time through slim_decode_step_host: pinned q, k in and out back every step."""
        import torch

        from only_cache_exact_b200 import replicas
        S = self.S
        q_h = self.q0.cpu().pin_memory()
        k_h = self.k0.cpu().pin_memory() if self.k0 is not None else None
        out_h = torch.empty(self.B, self.d, dtype=torch.float32).pin_memory()
        self.reset_lengths()

        def host_step(i):
            s = self.sets[i % self.rot]
            S.slim_decode_step_host(q_h, k_h, s["K"], s["lens"], s["W_KV"], self.H, out_h, s["ws"], self.status,
                                    variant=S.SLIM_AUTO, t_hint=self.t_hint, stream=self.stream)

        for i in range(3):
            host_step(i)
        self.stream.synchronize()
        self.reset_lengths()
        if pg:
            pg.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for i in range(nsteps):
            host_step(i)
        e1.record(self.stream)
        e1.synchronize()
        assert np.all(np.isfinite(out_h.numpy()))
        return replicas.max_over_ranks(e0.elapsed_time(e1) / nsteps, pg, self.dev)

    def measure(self, K_steps, W_steps, pg=None, clocks=None, e2e=True):
        """Steps/s, roofline of the split kernel, e2e and footprint for this workload."""
        from only_cache_exact_b200 import replicas
        S = self.S
        ms = self.time_steps(K_steps, W_steps, pg, clocks)
        ms = replicas.max_over_ranks(ms, pg, self.dev)
        st = int(self.status.item())
        ms_step = ms / K_steps
        chosen = (self.variant if self.variant != S.SLIM_AUTO
                  else S.slim_select_variant(self.dt_code, self.B, self.d, self.H, self.t_hint))
        launches = S.slim_last_launch_count()
        n_live = min(max(K_steps, 8), 64)
        split_ms = None if self.mha else self.split_kernel_ms(n_live)
        kbytes, sbytes_live = self.algorithmic_bytes(n_live)
        _, sbytes = self.algorithmic_bytes(K_steps)
        hbm_peak, _, peak_src = peaks()
        achieved = kbytes / (split_ms * 1e-3) / 1e9 if split_ms else None
        r = dict(ms_step=ms_step, status=st, chosen=chosen, launches=launches, split_ms=split_ms,
                 kernel_bytes=int(kbytes), step_bytes=int(sbytes), achieved=achieved, hbm_peak=hbm_peak,
                 peak_src=peak_src)
        r["e2e_ms"] = self.e2e_ms(max(8, min(K_steps, 200)), pg) if e2e and not self.mha else None
        return r

    def front_end(self, n=20):
        """The step started from its input rows (slim_decode_step_x: q = x·W_Q and, with append,
        k = x·W_K formed on the device) against the step handed q and k (slim_decode_step): n steps
        of each behind a spin kernel, from the same starting lengths. None for workloads timed with
        an L2 flush per step."""
        import torch

        from only_cache_exact_b200 import synth
        if self.flush or self.mha:
            return None
        S, dt = self.S, self.w["dtype"]
        W_Q = synth.to_storage(synth.round_to(self.wts.W_Q, dt), dt).to(self.dev)
        W_K = self.W_K if self.append else None
        x = synth.to_storage(self.x_new, dt).to(self.dev)
        nws = S.slim_decode_step_x_workspace_bytes(self.dt_code, self.B, self.d, self.H, self.cap, S.SLIM_AUTO)
        ws_x = [torch.empty(nws, dtype=torch.uint8, device=self.dev) for _ in range(self.rot)]

        def plain(i):
            s = self.sets[i % self.rot]
            S.slim_decode_step(s["q"], s["k"], s["K"], s["lens"], s["W_KV"], self.H, s["out"], s["ws"], self.status,
                               variant=S.SLIM_AUTO, t_hint=self.t_hint)

        def from_x(i):
            s = self.sets[i % self.rot]
            S.slim_decode_step_x(x, W_Q, W_K, s["K"], s["lens"], s["W_KV"], self.H, s["out"], ws_x[i % self.rot],
                                 self.status, variant=S.SLIM_AUTO, t_hint=self.t_hint)

        def timed(fn):
            self.reset_lengths()
            for i in range(3):
                fn(i)
            self.stream.synchronize()
            self.reset_lengths()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(self.stream):
                torch.cuda._sleep(int(50e6))
                e0.record(self.stream)
                for i in range(n):
                    fn(i)
                e1.record(self.stream)
            e1.synchronize()
            return e0.elapsed_time(e1) / n

        ms_q = timed(plain)
        ms_x = timed(from_x)
        launches = S.slim_last_launch_count()
        del ws_x
        return {"steps": n, "ms_per_step_from_q": ms_q, "ms_per_step_from_x": ms_x,
                "front_end_ms": ms_x - ms_q, "launches_per_step_from_x": launches,
                "projections": "q and k" if self.append else "q only (cross-attention)"}

    def l2_note(self):
        if self.flush:
            return f"a {FLUSH_BYTES >> 20} MB buffer written before every step (each step timed alone)"
        if self.rot == 1:
            return "K cache of one step larger than 2x L2 (no rotation needed)"
        return f"{self.rot} rotating buffer sets (K cache, W_KV, q, k) > 2x L2"

    def footprint(self):
        return {"k_only_bytes": int(self.B * self.cap * self.d * self.esz),
                "k_plus_v_bytes": int(2 * self.B * self.cap * self.d * self.esz)}


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def roofline_record(name, r):
    return {"bound": "hbm", "achieved": r["achieved"], "peak": r["hbm_peak"], "unit": "GB/s",
            "frac": (r["achieved"] / r["hbm_peak"]) if r["achieved"] else None,
            "traffic": profile_traffic(name),
            "kernel": "split kernel (streams the K cache; decode_b_tc_kernel for bf16, decode_simt_kernel for fp32)",
            "bytes_per_launch": r["kernel_bytes"], "avg_launch_ms": r["split_ms"],
            "peak_source": r["peak_src"] + " (MEASURED_PEAKS.json hbm_gbs, burst copy)"}


def sub_record(name, S, dev, cpu_budget):
    """One other workload at its own step count: the same measurements as the headline."""
    import torch
    w = WORKLOADS[name]
    wl = Workload(name, S, dev, max_steps=max(w["steps"], 64) + 8)
    r = wl.measure(w["steps"], 3)
    front = wl.front_end()
    rate, threads, n, T = cpu_oracle_rate(w, budget_s=cpu_budget)
    rec = {"workload": w["desc"], "steps": w["steps"], "warmup": 3, "ms_per_step": r["ms_step"],
           "steps_per_s": 1e3 / r["ms_step"], "tokens_per_s": 1e3 / r["ms_step"] * w["B"],
           "step_hbm_gbs": r["step_bytes"] / (r["ms_step"] * 1e-3) / 1e9,
           "step_frac": r["step_bytes"] / (r["ms_step"] * 1e-3) / 1e9 / r["hbm_peak"],
           "ordering": {1: "a", 2: "b"}.get(r["chosen"], "?"), "launches_per_step": r["launches"],
           "roofline": roofline_record(name, r),
           "e2e": {"value": 1e3 / r["e2e_ms"], "unit": "steps/s"} if r["e2e_ms"] else None,
           "l2": wl.l2_note(), "footprint": wl.footprint(), "status": r["status"], "front_end": front,
           "cpu_baseline": {"value": rate, "unit": "steps/s", "cores": threads, "kind": "oracle",
                            "sample": f"{n} single-sequence float64 oracle steps at T={T}, scaled to the batch"}}
    del wl
    torch.cuda.empty_cache()
    return rec


def kv_record(name, S, dev, slim_ms):
    """The standard MHA step over explicit K and V caches (slim_mha_decode_step) on the same workload,
    against the Slim step's ms per step: the pages' claim (up to 2x when memory-bound) as a ratio."""
    import torch
    w = WORKLOADS[name]
    steps = min(w["steps"], 64)
    wl = Workload(name, S, dev, max_steps=steps + 8, mha=True)
    ms = wl.time_steps(steps, 3) / steps
    _, sbytes = wl.algorithmic_bytes(steps)
    hbm_peak, _, _ = peaks()
    rec = {"workload": w["desc"], "steps": steps, "ms_per_step": ms, "steps_per_s": 1e3 / ms,
           "step_hbm_gbs": sbytes / (ms * 1e-3) / 1e9, "step_frac": sbytes / (ms * 1e-3) / 1e9 / hbm_peak,
           "kv_cache_bytes": int(2 * wl.B * wl.cap * wl.d * wl.esz), "l2": wl.l2_note(),
           "slim_ms_per_step": slim_ms, "slim_speedup": ms / slim_ms if slim_ms else None,
           "status": int(wl.status.item())}
    del wl
    torch.cuda.empty_cache()
    return rec


def run_sweep(S, dev):
    """Ordering (a) vs (b) over attended lengths T = 1K..128K (d=4096, H=32, B=1, no append), K cache
    filled by the prompt-phase kernel; and the 8192 x 4096 x 4096 prompt projection. Each T is timed
    with CUDA events behind a spin kernel (the GPU never waits for the host); the result goes into
    the SLIM_AUTO table and the ordering SLIM_AUTO then picks is reported."""
    import torch

    from only_cache_exact_b200 import params, synth
    d, H, B = 4096, 32, 1
    Ts = [1024, 2048, 4096, 8192, 16384, 32768, 65536, 131072 - 64]
    cap = 131072
    wts = synth.make_weights(d, 0, "bf16")
    W_K = synth.to_storage(wts.W_K, "bf16").to(dev)
    W_KV = params.make_wkv(wts.W_K, wts.W_V, dtype=torch.bfloat16, device=dev)
    K = torch.zeros(B, cap, d, dtype=torch.bfloat16, device=dev)
    lens = torch.zeros(B, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    chunk = 8192
    X = synth.make_tokens_device(chunk, d, 1000, 0, "bf16", device=dev).view(1, chunk, d)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):
        lens.zero_()
        S.slim_prefill_k(X, W_K, K, lens, status)
    torch.cuda.synchronize()
    reps = 5
    tot = 0.0
    for _ in range(reps):
        lens.zero_()
        torch.cuda._sleep(int(5e6))
        e0.record()
        S.slim_prefill_k(X, W_K, K, lens, status)
        e1.record()
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    ms_p = tot / reps
    prefill = {"rows": chunk, "d": d, "ms": ms_p, "tflops": 2.0 * chunk * d * d / ms_p / 1e9}
    # the prompt's attention output over the K-only cache: V = K·W_KV once, then causal attention
    Qp = synth.make_tokens_device(chunk, d, 7, 0, "bf16", part=2, device=dev).view(1, chunk, d)
    outp = torch.empty(1, chunk, d, dtype=torch.float32, device=dev)
    wsp = torch.empty(S.slim_prefill_attention_workspace_bytes(S.SLIM_BF16, B, d, H, cap), dtype=torch.uint8,
                      device=dev)
    for _ in range(2):
        S.slim_prefill_attention(Qp, K, lens, W_KV, H, outp, wsp, status)
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(reps):
        torch.cuda._sleep(int(5e6))
        e0.record()
        S.slim_prefill_attention(Qp, K, lens, W_KV, H, outp, wsp, status)
        e1.record()
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    ms_att = tot / reps
    att_flops = 2.0 * chunk * chunk * d + 2.0 * chunk * d * d  # causal QK^T and PV, plus V = K·W_KV
    prefill["attention"] = {"queries": chunk, "ms": ms_att, "tflops": att_flops / ms_att / 1e9,
                            "flops_note": "2·n²·d (causal QK^T and PV) + 2·n·d² (V = K·W_KV)"}
    del wsp, outp
    for r0 in range(chunk, cap, chunk):
        Xr = synth.make_tokens_device(chunk, d, 1000 + r0 // chunk, 0, "bf16", device=dev).view(1, chunk, d)
        S.slim_prefill_k(Xr, W_K, K, lens, status)
    torch.cuda.synchronize()
    x_new = synth.make_tokens(1, d, 0, 0, "bf16", part=2)
    q = torch.from_numpy(x_new @ wts.W_Q).float().to(dev)
    out = torch.empty(B, d, dtype=torch.float32, device=dev)
    ws = S.alloc_workspace(S.SLIM_BF16, B, d, H, cap, S.SLIM_AUTO, device=dev)
    S.slim_tune_clear()
    rows = []
    for T in Ts:
        ms = {}
        for name, v in (("a", S.SLIM_VARIANT_A), ("b", S.SLIM_VARIANT_B)):
            lens.fill_(T)
            for _ in range(2):
                S.slim_decode_step(q, None, K, lens, W_KV, H, out, ws, status, variant=v)
            torch.cuda.synchronize()
            n = 20 if name == "b" else max(3, min(20, 20 * 8192 // T))
            torch.cuda._sleep(int(20e6))
            e0.record()
            for _ in range(n):
                S.slim_decode_step(q, None, K, lens, W_KV, H, out, ws, status, variant=v)
            e1.record()
            e1.synchronize()
            ms[name] = e0.elapsed_time(e1) / n
        S.slim_tune_record(S.SLIM_BF16, B, d, H, T, ms["a"], ms["b"])
        pick = S.slim_select_variant(S.SLIM_BF16, B, d, H, T)
        step_bytes = T * d * 2 + d * d * 2 + 2 * d * 4
        rows.append({"T": T, "ms_a": ms["a"], "ms_b": ms["b"], "a_over_b": ms["a"] / ms["b"],
                     "b_step_hbm_gbs": step_bytes / (ms["b"] * 1e-3) / 1e9,
                     "a_tflops": 2.0 * T * d * d / (ms["a"] * 1e-3) / 1e12,
                     "auto_picks": {1: "a", 2: "b"}[pick]})
    S.slim_tune_clear()
    st = int(status.item())
    del K, ws
    torch.cuda.empty_cache()
    return {"d": d, "H": H, "B": B, "points": rows, "status": st}, prefill


def run_prefill_d1024(S, dev):
    """Prompt-phase projection of 8 sequences x 4096 rows at d=1024 (K = X·W_K)."""
    import torch

    from only_cache_exact_b200 import synth
    B, n_rows, d = 8, 4096, 1024
    X = synth.make_tokens_device(B * n_rows, d, 7, 0, "bf16", device=dev).view(B, n_rows, d)
    W_K = synth.to_storage(synth.make_weights(d, 0, "bf16").W_K, "bf16").to(dev)
    Kp = torch.empty(B, n_rows + 8, d, dtype=torch.bfloat16, device=dev)
    lens = torch.zeros(B, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(2):
        lens.zero_()
        S.slim_prefill_k(X, W_K, Kp, lens, status)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tot, reps = 0.0, 5
    for _ in range(reps):
        lens.zero_()
        torch.cuda._sleep(int(5e6))
        e0.record()
        S.slim_prefill_k(X, W_K, Kp, lens, status)
        e1.record()
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    ms = tot / reps
    return {"rows": B * n_rows, "d": d, "ms": ms, "tflops": 2.0 * B * n_rows * d * d / ms / 1e9}


def run_variant_a(S, dev):
    """Ordering (a) on the d=1024, B=8, T=4096 workload (materialise V = K·W_KV, then softmax·V)."""
    import torch
    wl = Workload("d1024_h16_b8_t4096", S, dev, max_steps=64)
    n = 20
    for i in range(3):
        wl.step(i, S.SLIM_VARIANT_A)
    wl.stream.synchronize()
    wl.reset_lengths()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(wl.stream):
        torch.cuda._sleep(int(20e6))
        e0.record(wl.stream)
        for i in range(n):
            wl.step(i, S.SLIM_VARIANT_A)
        e1.record(wl.stream)
    e1.synchronize()
    ms_a = e0.elapsed_time(e1) / n
    rows = wl.rows_attended(n) / n
    flops = 2.0 * rows * wl.d * wl.d
    _, tc_peak, _ = peaks()
    del wl
    torch.cuda.empty_cache()
    return {"ms_per_step": ms_a, "steps_per_s": 1e3 / ms_a, "tflops": flops / (ms_a * 1e-3) / 1e12,
            "frac_of_bf16_peak": flops / (ms_a * 1e-3) / 1e12 / tc_peak}


def run_front_kernel(S, dev):
    """The front-end kernel alone (slim_project_qk) on the batch shapes of the decode workloads: it
    reads W_Q (and W_K) once, so its roofline is HBM at 2·d² bytes per projection plus the rows.
    Each call is timed alone after a 256 MB write (the weights would otherwise sit in L2)."""
    import torch
    hbm_peak, _, _ = peaks()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    out = {}
    for d, B, with_k in ((1024, 8, True), (4096, 16, True), (1280, 64, False), (4096, 1, True)):
        x = torch.randn(B, d, generator=g, device=dev).to(torch.bfloat16)
        W_Q = (torch.randn(d, d, generator=g, device=dev) / d ** 0.5).to(torch.bfloat16)
        W_K = (torch.randn(d, d, generator=g, device=dev) / d ** 0.5).to(torch.bfloat16) if with_k else None
        q = torch.empty(B, d, dtype=torch.float32, device=dev)
        k = torch.empty(B, d, dtype=torch.bfloat16, device=dev) if with_k else None
        for _ in range(3):
            S.slim_project_qk(x, W_Q, W_K, q, k, status)
        torch.cuda.synchronize()
        reps, tot = 10, 0.0
        for i in range(reps):
            flush.fill_(i & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            S.slim_project_qk(x, W_Q, W_K, q, k, status)
            e1.record()
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        ms = tot / reps
        nproj = 2 if with_k else 1
        nbytes = nproj * d * d * 2 + B * d * 2 + B * d * 4 + (B * d * 2 if with_k else 0)
        out[f"d{d}_b{B}_{'qk' if with_k else 'q'}"] = {
            "ms": ms, "bytes": nbytes, "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
            "frac": nbytes / (ms * 1e-3) / 1e9 / hbm_peak, "status": int(status.item())}
        del x, W_Q, W_K, q, k
    del flush
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------------------------------ main
def main():
    args = parse()
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; no process group, no GPU
        if int(os.environ.get("RANK", "0")) != 0:
            return
        rank, world, local, pg = 0, int(os.environ.get("WORLD_SIZE", "1")), 0, None
    else:
        rank, world, local, pg = dist_init(args.gpus)
    workload_cfg = {"workload": w["desc"], "name": args.workload, "d": w["d"], "H": w["H"], "B": w["B"],
                    "T": list(w["T"]) if isinstance(w["T"], tuple) else w["T"], "append": w["append"],
                    "parallelism": f"replicas x{world} (independent sequences)"}

    if args.impl == "reference":
        rate, threads, n, T = cpu_oracle_rate(w, budget_s=args.ref_seconds)
        line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": "steps/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / rate, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": workload_cfg,
                "cpu_baseline": {"value": rate, "unit": "steps/s", "cores": threads, "kind": "oracle",
                                 "sample": f"{n} single-sequence oracle steps at T={T}, scaled to the batch"},
                "e2e": {"value": rate, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch

    from only_cache_exact_b200 import replicas, slim as S
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    variant = {"auto": S.SLIM_AUTO, "a": S.SLIM_VARIANT_A, "b": S.SLIM_VARIANT_B}[args.variant]
    wl = Workload(args.workload, S, dev, rank, world, max_steps=max(args.steps, args.warmup, 64) + 8,
                  rot=args.rot, batch=args.batch, variant=variant, from_x=args.from_x)
    if args.batch:  # a reduced batch for profiling captures; the line says so
        w = wl.w
        workload_cfg["B"] = w["B"]
        workload_cfg["workload"] += f" (batch reduced to {w['B']})"
    if args.variant != "auto":
        workload_cfg["ordering"] = args.variant
    if args.from_x:
        workload_cfg["from_input_rows"] = True
    sampler = ClockSampler(local)
    r = wl.measure(args.steps, args.warmup, pg, sampler)
    cfg = dict(workload_cfg)
    cfg["l2"] = wl.l2_note()
    cfg["attended_T_range"] = [int(np.min(wl.lens0)) + (1 if wl.append else 0),
                               int(np.max(wl.lens0)) + (-(-args.steps // wl.rot) if wl.append else 0)]
    h2d = int(w["B"] * w["d"] * 4 + (w["B"] * w["d"] * wl.esz if wl.append else 0))
    d2h = int(w["B"] * w["d"] * 4)
    footprint = wl.footprint()
    front = wl.front_end() if not args.no_extras else None
    del wl
    torch.cuda.empty_cache()

    extras = {}
    if not args.no_extras and world == 1:
        extras["workloads"] = {n: sub_record(n, S, dev, 3.0) for n in SUBRECORDS if n != args.workload}
        slim_ms = {n: rec["ms_per_step"] for n, rec in extras["workloads"].items()}
        slim_ms[args.workload] = r["ms_step"]
        extras["kv_baseline"] = {n: kv_record(n, S, dev, slim_ms.get(n))
                                 for n in KV_BASELINE if WORKLOADS[n]["dtype"] == "bf16"}
        extras["sweep"], extras["prefill"] = run_sweep(S, dev)
        extras["prefill_d1024"] = run_prefill_d1024(S, dev)
        extras["variant_a"] = run_variant_a(S, dev)
        extras["front_end_kernel"] = run_front_kernel(S, dev)

    if rank != 0:
        if pg:
            pg.destroy_process_group()
        return
    steps_per_s = replicas.whole_job_rate(1, world, r["ms_step"])
    cpu = None
    if world == 1 and not args.no_extras:
        rate, threads, n, T = cpu_oracle_rate(w)
        cpu = {"value": rate, "unit": "steps/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} single-sequence float64 oracle steps at T={T} (explicit K and V), "
                         f"scaled to the B={w['B']} batch"}
    line = {"metric": METRIC, "value": steps_per_s, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w["dtype"] == "bf16" else "f32", "data": "synthetic",
            "config": cfg,
            "tokens_per_s": steps_per_s * w["B"],
            "step_hbm_gbs": r["step_bytes"] / (r["ms_step"] * 1e-3) / 1e9,
            "step_frac": r["step_bytes"] / (r["ms_step"] * 1e-3) / 1e9 / r["hbm_peak"],
            "ordering": {1: "a", 2: "b"}.get(r["chosen"], "?"),
            "roofline": roofline_record(args.workload, r),
            "cpu_baseline": cpu,
            "e2e": {"value": replicas.whole_job_rate(1, world, r["e2e_ms"]), "unit": "steps/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": r["launches"] * args.steps,
            "launches_per_step": r["launches"],
            "clocks": sampler.summary(),
            "footprint": footprint,
            "front_end": front,
            "status": r["status"]}
    line.update(extras)
    print(json.dumps(line))
    if pg:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
