"""Benchmark of the ring-chunked attention / Ulysses hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  seq2head(Q), seq2head(K), seq2head(V) (GQA copy of 4 KV heads to 8 ranks)
  -> causal ring-chunked attention over L = 131072 (8 virtual ranks x 16384 tokens,
     per-rank head group of 4 query heads, tcgen05 tensor cores)
  -> head2seq(O)
i.e. the Ulysses layer of "Метод контекстного параллелизма Ulysses" with the ring
attention of "Как работает sequence parallelism в контексте LLM?" as its local kernel.

value = attention FLOPs (4*B*H*L^2*D / 2, causal) of all ranks' steps / device time of
the steps (max over ranks), in TFLOP/s.  With --gpus N every rank runs its own replica
(weak scaling: the path has no data-path exchange between independent replicas).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload ulysses_e2e|ulysses_32k|usp_e2e|long_128k|long_128k_zigzag|long_128k_packed|
                              long_128k_bwd|long_128k_bwd_zigzag|long_128k_bwd_packed|
                              long_128k_bwd_det|llama8b_32k_bwd|
                              llama8b_32k|small_4k|merge_128k]

long_128k_bwd_det times the backward with ra_set_bwd_deterministic(1) (dQ from the
query-stationary kernel: bit-reproducible gradients).

merge_128k times the log-sum-exp merge alone (ra_lse_merge, B=1, H=8, L=131072, D=128,
fp32): one step = one merge of two partials, reported in GB/s of 3*D*4 + 12 bytes per row
against the measured HBM copy rate.
"""
from __future__ import annotations

import argparse
import faulthandler
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ring-chunked attention TFLOP/s & % BF16 tensor peak (1 B200); permute GB/s"
UNIT = "TFLOP/s"
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_HBM_GBS = 8000.0
# workload name suffix of each path kind
SUFFIX = {"attn_zigzag": "_zigzag", "attn_packed": "_packed", "attn_bwd": "_backward",
          "attn_bwd_zigzag": "_zigzag_backward", "attn_bwd_packed": "_packed_backward",
          "attn_bwd_det": "_deterministic_backward"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ workloads
def workloads():
    from sequence_parallelism_attn_b200 import synth
    return {
        "ulysses_e2e": ("ulysses", synth.ULYSSES_128K),
        "ulysses_32k": ("ulysses", synth.ULYSSES_32K),
        "usp_e2e": ("ulysses", synth.USP_128K),
        "long_128k": ("attn", synth.LONG_128K),
        "long_128k_zigzag": ("attn_zigzag", synth.LONG_128K),
        "long_128k_packed": ("attn_packed", synth.LONG_128K),
        "long_128k_bwd": ("attn_bwd", synth.LONG_128K),
        "long_128k_bwd_zigzag": ("attn_bwd_zigzag", synth.LONG_128K),
        "long_128k_bwd_packed": ("attn_bwd_packed", synth.LONG_128K),
        "long_128k_bwd_det": ("attn_bwd_det", synth.LONG_128K),
        "llama8b_32k": ("attn", synth.LLAMA8B_GQA),
        "llama8b_32k_bwd": ("attn_bwd", synth.LLAMA8B_GQA),
        "small_4k": ("attn", synth.SMALL_BF16),
        "merge_128k": ("merge", synth.MERGE_128K),
    }


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock, power and clock-event reasons every 100 ms through NVML."""

    BAD = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown"}
    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
             0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.samples = []
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            prop = torch.cuda.get_device_properties(device_index)
            # torch gives the PCI location as three integers; NVML wants the string form
            bus = "%08X:%02X:%02X.0" % (int(prop.pci_domain_id), int(prop.pci_bus_id),
                                        int(prop.pci_device_id))
            assert isinstance(bus, str)
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: fall back to nvidia-smi
            self._nv = None
            self.error = str(e)
            self._bus = locals().get("bus")

    def _run_smi(self):
        import subprocess
        q = "clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active"
        cmd = ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self._bus:
            cmd += ["-i", self._bus]
        try:
            proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, text=True)
        except Exception:
            return
        for line in proc.stdout:
            if self._stop.is_set():
                break
            try:
                sm, mx, pw, rs = [x.strip() for x in line.split(",")]
                self.max_mhz = float(mx)
                self.samples.append((float(sm), int(rs, 16), float(pw)))
            except Exception:
                pass
        proc.terminate()

    def _run(self):
        nv = self._nv
        if nv is None:
            return self._run_smi()
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                power = nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0
                self.samples.append((sm, reasons, power))
            except Exception:
                pass
            self._stop.wait(0.1)

    def __enter__(self):
        if True:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        sm = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= s[1]
        reasons = [n for b, n in self.NAMES.items() if bits & b and b != 0x1]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "power_w_max": max(s[2] for s in self.samples),
                "samples": len(sm)}

    def rejected(self) -> bool:
        if not self.samples:
            return False
        bits = 0
        for s in self.samples:
            bits |= s[1]
        if any(bits & b for b in self.BAD):
            return True
        med = statistics.median(s[0] for s in self.samples)
        no_reason = not (bits & ~0x1)
        return bool(self.max_mhz and no_reason and med < 0.6 * self.max_mhz)


# ------------------------------------------------------------------ our path
class Path:
    """Device buffers and the per-step launches of one workload."""

    def __init__(self, kind, w, device):
        import torch
        from sequence_parallelism_attn_b200 import ra, synth
        self.ra, self.kind, self.w, self.dev = ra, kind, w, device
        # shard layout of the plain attention workloads (zigzag: rank i holds segments i and
        # 2P-1-i of 2P segments of Lc/2 tokens)
        self.layout = "zigzag" if kind in ("attn_zigzag", "attn_bwd_zigzag") else "contiguous"
        if kind == "merge":
            self.a = w
            # two partials with LSE ~ 4 N(0,1), drawn on the device; each step merges b into
            # a in place (a valid merge every time: the LSEs only grow)
            g = torch.Generator(device=device)
            g.manual_seed(w.seed)
            shape_o, shape_l = (w.B, w.L, w.H, w.D), (w.B, w.H, w.L)
            self.oa = torch.randn(shape_o, generator=g, device=device)
            self.la = 4.0 * torch.randn(shape_l, generator=g, device=device)
            self.ob = torch.randn(shape_o, generator=g, device=device)
            self.lb = 4.0 * torch.randn(shape_l, generator=g, device=device)
            self.launches_per_step = 1
            self.bytes = w.bytes()
            self.flops = 0.0
            self.permute_bytes = 0
            self.in_bytes = sum(t.numel() * 4 for t in (self.oa, self.la, self.ob, self.lb))
            self.out_bytes = (self.oa.numel() + self.la.numel()) * 4
        elif kind == "ulysses":
            a = w.attn()
            self.a = a
            self.q, self.k, self.v = synth.ulysses_inputs(w, device=device)
            # head-sharded buffers: [G, B, L, heads / G, D] (G = P for Ulysses itself)
            self.qh = torch.empty((w.G, w.B, a.L, a.H_q, a.D), dtype=w.dtype, device=device)
            self.kh = torch.empty((w.G, w.B, a.L, a.H_kv, a.D), dtype=w.dtype, device=device)
            self.vh = torch.empty_like(self.kh)
            self.o = torch.empty((a.B, a.L, a.H_q, a.D), dtype=torch.bfloat16, device=device)
            self.lse = torch.empty((a.B, a.H_q, a.L), dtype=torch.float32, device=device)
            self.o_seq = torch.empty_like(self.q)
            kvv = lambda x: [x.view(a.B, a.P, a.Lc, a.H_kv, a.D)[:, j] for j in range(a.P)]
            self.k_chunks, self.v_chunks = kvv(self.kh), kvv(self.vh)
            self.qa = self.qh.view(a.B, a.L, a.H_q, a.D)
            self.launches_per_step = 5
            self.flops = a.flops()
            self.permute_bytes = w.permute_bytes()
            self.in_bytes = sum(t.numel() * t.element_size() for t in (self.q, self.k, self.v))
            self.out_bytes = self.o_seq.numel() * self.o_seq.element_size()
        else:
            self.a = w
            q, k, v = synth.attention_inputs(w, device=device)
            self.q, self.k, self.v = q, k, v
            self.o = torch.empty((w.B, w.L, w.H_q, w.D), dtype=torch.bfloat16, device=device)
            self.lse = torch.empty((w.B, w.H_q, w.L), dtype=torch.float32, device=device)
            self.launches_per_step = 1
            self.flops = w.flops()
            self.pid = None
            if kind in ("attn_packed", "attn_bwd_packed"):
                # documents of 512..32768 tokens (log-uniform, seeded) packed into each row;
                # the algorithmic work is each document's own causal attention
                lens = synth.packed_lengths(w.L, w.seed + 21, 512, 32768)
                self.pid = synth.position_ids_from_lengths([lens] * w.B).to(device)
                self.flops = sum(4.0 * w.B * w.H_q * float(n) ** 2 * w.D / 2 for n in lens)
                self.n_docs = len(lens)
            if kind.startswith("attn_bwd"):
                # the backward pass: dout drawn like the inputs; the forward's O and LSE are
                # produced once, outside the timed steps.  Algorithmic work: five matmuls
                # (S recomputed, dP, dV, dK, dQ) against the forward's two -> 2.5x.
                g = torch.Generator(device=device)
                g.manual_seed(w.seed + 2)
                self.dout = torch.randn(q.shape, generator=g, device=device).to(torch.bfloat16)
                ra.ring_attn_fwd(q, k, v, w.causal, w.scale, out=self.o, lse=self.lse,
                                 layout=self.layout, position_ids=self.pid)
                self.dq = torch.empty((w.B, w.L, w.H_q, w.D), dtype=torch.float32, device=device)
                self.dk = torch.empty(k.shape, dtype=torch.float32, device=device)
                self.dv = torch.empty_like(self.dk)
                self.ws = torch.empty((w.B, w.H_q, w.L), dtype=torch.float32, device=device)
                self.flops = 2.5 * self.flops
                self.launches_per_step = 2  # Delta (and dQ zeroing), then dQ / dK / dV
                # the deterministic mode: Delta, dK / dV, then dQ by the query-stationary
                # kernel (a process-wide switch of the library, set once here)
                det = kind == "attn_bwd_det"
                ra.ra_set_bwd_deterministic(det)
                if det:
                    self.launches_per_step = 3
            self.permute_bytes = 0
            self.in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
            self.out_bytes = self.o.numel() * self.o.element_size()

    def step(self, ev=None):
        """One pass of the path.  ev: optional dict of CUDA event pairs per stage."""
        ra = self.ra
        rec = (lambda name, i: ev[name][i].record()) if ev is not None else (lambda *_: None)
        if self.kind == "merge":
            rec("attn", 0)
            ra.ra_lse_merge(self.oa, self.la, self.ob, self.lb)
            rec("attn", 1)
        elif self.kind == "ulysses":
            w, a = self.w, self.a
            rec("permute_in", 0)
            ra.ra_ulysses_seq2head(self.q, w.H_q, out=self.qh, groups=w.G)
            ra.ra_ulysses_seq2head(self.k, w.H_kv_rep, out=self.kh, groups=w.G)
            ra.ra_ulysses_seq2head(self.v, w.H_kv_rep, out=self.vh, groups=w.G)
            rec("permute_in", 1)
            rec("attn", 0)
            ra.ring_attn_fwd(self.qa, self.k_chunks, self.v_chunks, True, a.scale,
                             out=self.o, lse=self.lse)
            rec("attn", 1)
            rec("permute_out", 0)
            ra.ra_ulysses_head2seq(self.o.view(w.G, w.B, a.L, a.H_q, a.D), out=self.o_seq, P=w.P)
            rec("permute_out", 1)
        elif self.kind.startswith("attn_bwd"):
            w = self.w
            rec("attn", 0)
            ra.ring_attn_bwd(self.q, self.k, self.v, self.o, self.lse, self.dout, w.causal,
                             w.scale, dq=self.dq, dk=self.dk, dv=self.dv, workspace=self.ws,
                             layout=self.layout, position_ids=self.pid)
            rec("attn", 1)
        else:
            w = self.w
            rec("attn", 0)
            ra.ring_attn_fwd(self.q, self.k, self.v, w.causal, w.scale, out=self.o, lse=self.lse,
                             layout=self.layout, position_ids=self.pid)
            rec("attn", 1)

    def result(self):
        if self.kind == "merge":
            return self.oa
        return self.o_seq if self.kind == "ulysses" else self.o

    def inputs(self):
        """The step's input tensors (what the end-to-end leg uploads every step)."""
        if self.kind == "merge":
            return (self.oa, self.la, self.ob, self.lb)
        return (self.q, self.k, self.v)


class DistUlyssesPath:
    """The Ulysses step across N GPUs, one process each, with real exchanges: this rank's
    sequence shard of Q, K, V (L/N tokens, every head) -> seq->head all-to-all (pack
    kernel, NCCL all-to-all, unpack) -> causal attention of its H_q/N query heads over the
    whole sequence (the attention kernel over the workload's chunk count) -> head->seq
    all-to-all of O.  The total problem is the one-GPU workload's (strong scaling)."""

    @staticmethod
    def splits(w, world) -> bool:
        """The workload's query heads and sequence divide over `world` ranks."""
        return w.H_q % world == 0 and (w.P * w.Lc) % world == 0 and w.G == w.P

    def __init__(self, w, device, rank, world, exchange="nccl"):
        import torch
        from sequence_parallelism_attn_b200 import dist as rd, ra
        self.ra, self.rd, self.kind, self.w, self.dev = ra, rd, "ulysses_dist", w, device
        self.exchange = exchange
        L = w.P * w.Lc
        if not self.splits(w, world):
            raise ValueError(f"{w.name} does not split over {world} ranks")
        self.world, self.Ls, self.L = world, L // world, L
        self.H_kv_rep = math.lcm(w.H_kv, world)
        g = torch.Generator(device=device)
        g.manual_seed(w.seed + 7919 * rank)
        draw = lambda h: torch.randn((w.B, self.Ls, h, w.D), generator=g,
                                     device=device).to(w.dtype)
        self.q, self.k, self.v = draw(w.H_q), draw(w.H_kv), draw(w.H_kv)
        self.Hq_l, self.Hkv_l = w.H_q // world, self.H_kv_rep // world
        self.chunks = w.P  # the attention walks the same chunk count as on one GPU
        self.o = torch.empty((w.B, L, self.Hq_l, w.D), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((w.B, self.Hq_l, L), dtype=torch.float32, device=device)
        if exchange != "p2p":
            self.o_seq = torch.empty((w.B, self.Ls, w.H_q, w.D), dtype=w.dtype, device=device)
        else:
            # the one-kernel exchange: every rank's scatter stores into these symmetric
            # buffers (the head blocks of Q, K, V and this rank's shard of O)
            pb = lambda *shape: rd.PeerBuffers(shape, w.dtype, device=device)
            self.pq = pb(w.B, L, self.Hq_l, w.D)
            self.pk, self.pv = pb(w.B, L, self.Hkv_l, w.D), pb(w.B, L, self.Hkv_l, w.D)
            self.po = pb(w.B, self.Ls, w.H_q, w.D)
            self.o_seq = self.po.buf
        self.scale = w.D ** -0.5
        self.flops = 4.0 * w.B * self.Hq_l * float(L) ** 2 * w.D / 2
        self.launches_per_step = 3 + 1 + (1 if w.B == 1 else 2) + (3 if w.B > 1 else 0)
        if exchange == "p2p":
            self.launches_per_step = 3 + 1 + 1  # Q, K, V scatters, attention, O scatter
        es = torch.tensor([], dtype=w.dtype).element_size()
        part = (world - 1) / world
        self.bytes_sent = int(es * w.B * self.Ls * w.D * part *
                              (2 * w.H_q + 2 * self.H_kv_rep))
        self.permute_bytes = 0
        self.in_bytes = sum(t.numel() * t.element_size() for t in (self.q, self.k, self.v))
        self.out_bytes = self.q.numel() * self.q.element_size()

    def step(self, ev=None):
        rd, w = self.rd, self.w
        rec = (lambda name, i: ev[name][i].record()) if ev is not None else (lambda *_: None)
        rec("permute_in", 0)
        if self.exchange == "p2p":
            qh, kh, vh = rd.ulysses_seq2head_p2p_many([(self.q, self.pq, w.H_q),
                                                       (self.k, self.pk, self.H_kv_rep),
                                                       (self.v, self.pv, self.H_kv_rep)])
        else:
            qh = rd.ulysses_seq2head_dist(self.q, w.H_q)
            kh = rd.ulysses_seq2head_dist(self.k, self.H_kv_rep)
            vh = rd.ulysses_seq2head_dist(self.v, self.H_kv_rep)
        rec("permute_in", 1)
        rec("attn", 0)
        C, Lc = self.chunks, self.L // self.chunks
        kv = lambda x: [x.view(w.B, C, Lc, self.Hkv_l, w.D)[:, j] for j in range(C)]
        self.ra.ring_attn_fwd(qh, kv(kh), kv(vh), True, self.scale, out=self.o, lse=self.lse)
        rec("attn", 1)
        rec("permute_out", 0)
        # into the same buffer every step: the end-to-end leg reads it on another stream
        if self.exchange == "p2p":
            rd.ulysses_head2seq_p2p(self.o, self.po)
        else:
            rd.ulysses_head2seq_dist(self.o, out=self.o_seq)
        rec("permute_out", 1)

    def result(self):
        return self.o_seq

    def inputs(self):
        return (self.q, self.k, self.v)


def time_region(path, steps, torch, dist, ev_stages):
    """Time exactly `steps` steps between barrier+synchronize; returns (ms_total, stage_ms)."""
    events = {k: [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
              for k in ev_stages}
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start.record()
    for i in range(steps):
        path.step({k: events[k][i] for k in ev_stages})
    end.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    total = start.elapsed_time(end)
    stage = {k: [events[k][i][0].elapsed_time(events[k][i][1]) for i in range(steps)]
             for k in ev_stages}
    return total, stage


def max_over_ranks(x, dist, torch, device):
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def any_over_ranks(flag: bool, dist, torch, device) -> bool:
    """True on every rank when it is True on any: a decision that changes which collectives
    follow (a retried timing region) must be the same on all ranks."""
    return max_over_ranks(1.0 if flag else 0.0, dist, torch, device) > 0.5


def e2e_region(paths, steps, torch, dist, device):
    """The step through the public API, end to end: every step copies its inputs from
    pinned host memory to the device and reads its result back to pinned host memory.
    Two device buffer sets pipeline the work the way a caller would: the inputs of step
    i+1 go up on one copy stream and the output of step i comes down on another while the
    compute stream runs.  Events order every reuse of a buffer; the first upload and the
    last download are not hidden.  Returns ms per step (max over ranks)."""
    comp = torch.cuda.current_stream()
    up = torch.cuda.Stream(device=device)
    down = torch.cuda.Stream(device=device)
    host_in = [t.cpu().pin_memory() for t in paths[0].inputs()]
    res = paths[0].result()
    host_out = [torch.empty(res.shape, dtype=res.dtype, pin_memory=True) for _ in range(2)]
    ev = lambda: [torch.cuda.Event() for _ in range(2)]
    up_done, comp_done, down_done = ev(), ev(), ev()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)

    def upload(i):
        s = i % 2
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(comp_done[s])  # step i-2 has finished reading set s
            for h, d in zip(host_in, paths[s].inputs()):
                d.copy_(h, non_blocking=True)
            up_done[s].record(up)

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(comp)
    up.wait_event(start)
    down.wait_event(start)
    upload(0)
    for i in range(steps):
        s = i % 2
        comp.wait_event(up_done[s])
        if i >= 2:
            comp.wait_event(down_done[s])  # step i-2's result has left set s
        paths[s].step()
        comp_done[s].record(comp)
        if i + 1 < steps:
            upload(i + 1)
        with torch.cuda.stream(down):
            down.wait_event(comp_done[s])
            host_out[s].copy_(paths[s].result(), non_blocking=True)
            down_done[s].record(down)
    comp.wait_stream(up)
    comp.wait_stream(down)
    end.record(comp)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    return max_over_ranks(ms, dist, torch, device)


def attn_traffic(path_kind, backward=False):
    """DRAM bytes per launch of the dominant kernel (the attention kernel, or the backward
    kernel) from the committed ncu summary, if it was taken on the current kernel source
    (else None)."""
    import hashlib
    name = "attn_bwd_sm100" if backward else "attn_sm100"
    src = os.path.join(ROOT, "sequence_parallelism_attn_b200", "csrc", name + ".cu")
    prof = os.path.join(ROOT, "profiles", name + "_traffic.json")
    if not os.path.exists(prof):
        return None
    with open(prof) as f:
        d = json.load(f)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if d.get("kernel_sha") != sha:
        return None
    return d.get("bytes_per_launch", {}).get(path_kind)


# ------------------------------------------------------------------ CPU baseline (oracle)
def oracle_sample(w_attn, n_rows, seed=4242):
    """A bounded sample of the attention workload for the oracle: n query rows of one
    (batch, kv-head) sequence of the same length and distribution, against all their keys."""
    import numpy as np
    import torch
    g = torch.Generator().manual_seed(seed)
    L, D = w_attn.L, w_attn.D
    k = torch.randn(1, L, 1, D, generator=g).to(w_attn.dtype).double().numpy()
    v = torch.randn(1, L, 1, D, generator=g).to(w_attn.dtype).double().numpy()
    rt = torch.randint(0, L, (n_rows,), generator=g).numpy().astype(np.int64)
    q = (torch.randn(n_rows, D, generator=g) * w_attn.q_mult).to(w_attn.dtype).double().numpy()
    vis = (rt + 1) if w_attn.causal else np.full(n_rows, L)
    flops = float(np.sum(4.0 * vis * D))
    return q, np.zeros(n_rows, np.int32), rt, np.zeros(n_rows, np.int32), k, v, flops


def run_oracle_sample(w_attn, target_s=15.0, max_rows=4096):
    """Time the oracle as it stands on a bounded sample; returns (TFLOP/s, rows, seconds)."""
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    n = 8 * cores
    while True:
        q, rb, rt, rh, k, v, flops = oracle_sample(w_attn, n)
        t0 = time.perf_counter()
        oracle.attention_rows(q, rb, rt, rh, k, v, 1, w_attn.scale, w_attn.causal)
        dt = time.perf_counter() - t0
        if dt >= target_s * 0.5 or n >= max_rows:
            return flops / dt / 1e12, n, dt, cores
        n = min(max_rows, max(n * 2, int(n * target_s / max(dt, 1e-3))))


def oracle_bwd_sample(w_attn, Ls, seed=4243):
    """A bounded sample of a backward workload for the oracle: one head's sequence of Ls
    tokens (same distribution, causal as the workload) with dO; algorithmic FLOPs as for
    the GPU line (2.5x the forward's)."""
    import torch
    g = torch.Generator().manual_seed(seed)
    D = w_attn.D
    draw = lambda mult=1.0: (torch.randn(1, Ls, 1, D, generator=g) * mult).to(
        w_attn.dtype).double().numpy()
    q, k, v, dout = draw(w_attn.q_mult), draw(), draw(), draw()
    flops = 2.5 * 4.0 * float(Ls) * Ls * D / (2 if w_attn.causal else 1)
    return q, k, v, dout, flops


def run_oracle_bwd_sample(w_attn, target_s=15.0):
    """Time the oracle's gradients as they stand on a bounded sample; returns
    (TFLOP/s, Ls, seconds, cores)."""
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    Ls = 256
    while True:
        q, k, v, dout, flops = oracle_bwd_sample(w_attn, Ls)
        t0 = time.perf_counter()
        oracle.attention_backward(q, k, v, dout, w_attn.scale, w_attn.causal)
        dt = time.perf_counter() - t0
        if dt >= target_s * 0.5 or Ls >= w_attn.L:
            return flops / dt / 1e12, Ls, dt, cores
        Ls = min(w_attn.L, Ls * 2)  # the cost grows about 4x per doubling


# ------------------------------------------------------------------ main
def main():
    faulthandler.enable()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="ulysses_e2e")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--exchange", choices=["nccl", "p2p"], default="nccl",
                    help="N > 1 Ulysses step: NCCL all-to-alls with pack / unpack kernels, "
                         "or one scatter kernel per rank into symmetric-memory buffers "
                         "(the end-to-end leg is then skipped)")
    ap.add_argument("--ref-step-seconds", type=float, default=None,
                    help="reference arm: target seconds of oracle work per step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    kind, w = workloads()[args.workload]
    w_attn = w.attn() if kind == "ulysses" else w
    if kind == "merge":
        return merge_main(args, w)

    if args.impl == "reference":
        return reference_arm(args, kind, w, w_attn, rank, world)

    import torch
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    peaks, peaks_src = load_peaks()

    if world > 1 and kind == "ulysses" and DistUlyssesPath.splits(w, world):
        # N GPUs: the Ulysses layer with real all-to-alls between the ranks
        path = DistUlyssesPath(w, device, rank, world, exchange=args.exchange)
    else:
        # one GPU, a workload without an exchange, or heads that do not split over N:
        # independent replicas
        path = Path(kind, w, device)
    for _ in range(args.warmup):
        path.step()
    torch.cuda.synchronize()
    stages = ["attn"] + (["permute_in", "permute_out"] if kind == "ulysses" else [])
    for attempt in range(2):
        with ClockSampler(local_rank) as clk:
            total_ms, stage_ms = time_region(path, args.steps, torch, dist, stages)
        # retaken on every rank or on none: the retry runs collectives (barrier, all-reduce)
        if not any_over_ranks(clk.rejected(), dist, torch, device):
            break
    st = path.ra.ra_sync_status()
    if st != 0:
        raise RuntimeError(f"kernel status {st}: {path.ra.ra_last_error()}")
    ms_step = max_over_ranks(total_ms / args.steps, dist, torch, device)
    attn_ms = max_over_ranks(statistics.mean(stage_ms["attn"]), dist, torch, device)
    value = path.flops * world / (ms_step * 1e-3) / 1e12
    attn_tflops = path.flops / (attn_ms * 1e-3) / 1e12
    dist_ulysses = path.kind == "ulysses_dist"
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "strong" if dist_ulysses else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name + SUFFIX.get(kind, ""),
                   "global_batch": w_attn.B * (1 if dist_ulysses else world),
                   "seq_len": w_attn.L,
                   "heads_q": w_attn.H_q, "heads_kv": w_attn.H_kv, "head_dim": w_attn.D,
                   "virtual_ranks": w_attn.P, "chunk_len": w_attn.Lc, "causal": w_attn.causal,
                   "parallelism": f"ulysses{world}" if dist_ulysses else f"replicas{world}",
                   "l2": "inputs larger than L2 (126 MB); no flush between steps"},
    }
    if dist_ulysses:
        out["config"].update({"global_batch": w.B, "seq_len": path.L, "heads_q": w.H_q,
                              "heads_kv": w.H_kv, "tokens_per_rank": path.Ls,
                              "heads_q_per_rank": path.Hq_l, "heads_kv_per_rank": path.Hkv_l,
                              "exchange": ("one scatter kernel per rank into the peers' "
                                           "symmetric-memory buffers, a barrier on each side"
                                           if args.exchange == "p2p" else
                                           "NCCL all-to-all between the ranks, pack/unpack "
                                           "kernels around it")})
    if kind == "ulysses":
        # Ulysses: P head groups; the ring x Ulysses hybrid: fewer, each with a ring
        out["config"]["head_groups"] = w.G
    if kind in ("attn_packed", "attn_bwd_packed"):
        out["config"]["packed_documents"] = path.n_docs
        out["config"]["document_lengths"] = "512..32768 tokens, log-uniform, seeded"
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    # DRAM bytes from the committed capture of the one-GPU launch (another launch shape
    # when the heads are split over several GPUs)
    traffic = None if dist_ulysses else attn_traffic(args.workload,
                                                       backward=kind.startswith("attn_bwd"))
    out["roofline"] = {"bound": "tensor", "achieved": round(attn_tflops, 2),
                       "peak": sustained, "unit": "TFLOP/s",
                       "frac": round(attn_tflops / sustained, 4),
                       "traffic": traffic,
                       "kernel": ("bwd_delta + bwd_sm100 (dK, dV) + bwd_dq_sm100 (dQ), D=128"
                                  if kind == "attn_bwd_det" else
                                  "bwd_delta + bwd_sm100 (dQ, dK, dV), D=128"
                                  if kind.startswith("attn_bwd") else "attn_fwd_sm100<128>"),
                       "peak_source": f"{peaks_src} bf16_tflops_sustained",
                       "frac_of_burst": round(attn_tflops / peaks.get("bf16_tflops", 1590.0), 4),
                       "frac_of_datasheet": round(attn_tflops / DATASHEET_BF16_TFLOPS, 4)}
    if dist_ulysses:
        ex_ms = max_over_ranks(statistics.mean(
            a + b for a, b in zip(stage_ms["permute_in"], stage_ms["permute_out"])),
            dist, torch, device)
        out["exchange"] = {"ms_per_step": round(ex_ms, 4),
                           "bytes_sent_per_rank": path.bytes_sent,
                           "gbs_per_rank": round(path.bytes_sent / (ex_ms * 1e-3) / 1e9, 1)}
    elif kind == "ulysses":
        perm_ms = max_over_ranks(statistics.mean(
            a + b for a, b in zip(stage_ms["permute_in"], stage_ms["permute_out"])),
            dist, torch, device)
        perm_gbs = path.permute_bytes / (perm_ms * 1e-3) / 1e9
        out["permute"] = {"gbs": round(perm_gbs, 1), "bytes_per_step": path.permute_bytes,
                          "ms_per_step": round(perm_ms, 4),
                          "frac_of_measured_hbm": round(perm_gbs / peaks.get("hbm_gbs", 6650.0), 4),
                          "frac_of_datasheet_hbm": round(perm_gbs / DATASHEET_HBM_GBS, 4)}
    out["gpu_launches"] = path.launches_per_step * args.steps
    out["clocks"] = clk.summary()
    if not args.no_e2e and kind.startswith("attn_bwd"):
        # the leg streams the forward's inputs and output; a backward step's inputs (q, k,
        # v, O, LSE, dO) and results (dq, dk, dv) are not what it moves, so no number
        out["e2e"] = None
        out["e2e_note"] = "not measured for backward workloads"
    elif not args.no_e2e and dist_ulysses and args.exchange == "p2p":
        # the peers store into this rank's output buffer during their next step, which the
        # pipelined leg's copy stream would race
        out["e2e"] = None
        out["e2e_note"] = "not measured with the one-kernel exchange (--exchange p2p)"
    elif not args.no_e2e:
        # second buffer set for the pipelined end-to-end leg
        path2 = DistUlyssesPath(w, device, rank, world) if dist_ulysses else Path(kind, w, device)
        e2e_ms = e2e_region([path, path2], args.steps, torch, dist, device)
        del path2
        out["e2e"] = {"value": round(path.flops * world / (e2e_ms * 1e-3) / 1e12, 2),
                      "unit": UNIT, "h2d_bytes_per_step": path.in_bytes,
                      "d2h_bytes_per_step": path.out_bytes, "ms_per_step": round(e2e_ms, 3),
                      "steps": args.steps,
                      "pipelined": "step i+1 inputs up and step i output down on two copy "
                                   "streams, overlapping compute; all copies timed"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if kind.startswith("attn_bwd"):
            tf, n, dt, cores = run_oracle_bwd_sample(w_attn)
            sample = (f"gradients of one head's {n}-token sequence (D={w_attn.D}, "
                      f"{'causal' if w_attn.causal else 'non-causal'}), fp64 oracle, {dt:.1f} s")
        else:
            tf, n, dt, cores = run_oracle_sample(w_attn)
            sample = (f"{n} query rows x all visible keys of one {w_attn.L}-token sequence "
                      f"(D={w_attn.D}), fp64 oracle, {dt:.1f} s")
        out["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": sample}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def merge_sample(w, n_rows, seed=4244):
    """A bounded sample of the merge workload for the oracle: n rows of two partials drawn
    like the GPU inputs (O ~ N(0,1), LSE ~ 4 N(0,1))."""
    import torch
    g = torch.Generator().manual_seed(seed)
    oa = torch.randn(1, n_rows, 1, w.D, generator=g).double().numpy()
    ob = torch.randn(1, n_rows, 1, w.D, generator=g).double().numpy()
    la = (4.0 * torch.randn(1, 1, n_rows, generator=g)).double().numpy()
    lb = (4.0 * torch.randn(1, 1, n_rows, generator=g)).double().numpy()
    return oa, la, ob, lb, n_rows * (3 * w.D * 4 + 12)


def run_oracle_merge(w, target_s=10.0):
    """Time the oracle's merge as it stands on a bounded sample of rows; returns
    (GB/s, rows, seconds, cores)."""
    import oracle
    oracle.build()
    n = 1 << 14
    while True:
        oa, la, ob, lb, nbytes = merge_sample(w, n)
        t0 = time.perf_counter()
        oracle.lse_merge(oa, la, ob, lb)
        dt = time.perf_counter() - t0
        if dt >= target_s * 0.5 or n >= w.B * w.H * w.L:
            return nbytes / dt / 1e9, n, dt, 1
        n = min(w.B * w.H * w.L, n * 4)


def merge_main(args, w):
    """The merge workload: ra_lse_merge alone, GB/s against the HBM copy rate."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    config = {"workload": w.name, "rows": w.B * w.H * w.L, "heads": w.H, "seq_len": w.L,
              "head_dim": w.D, "bytes_per_row": 3 * w.D * 4 + 12,
              "l2": "inputs larger than L2 (126 MB); no flush between steps"}
    if args.impl == "reference":
        if rank != 0:
            return
        per_step = args.ref_step_seconds or max(1.0, min(10.0, 120.0 / (args.steps + args.warmup)))
        _, n, _, cores = run_oracle_merge(w, target_s=per_step)
        oa, la, ob, lb, nbytes = merge_sample(w, n)
        import oracle
        times = []
        for _ in range(args.steps):
            t0 = time.perf_counter()
            oracle.lse_merge(oa, la, ob, lb)
            times.append(time.perf_counter() - t0)
        sec = sum(times) / len(times)
        value = nbytes / sec / 1e9
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(config, parallelism="cpu-oracle"),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"{n} rows per step, fp64 oracle merge"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return
    import torch
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    peaks, peaks_src = load_peaks()
    path = Path("merge", w, device)
    for _ in range(args.warmup):
        path.step()
    torch.cuda.synchronize()
    for attempt in range(2):
        with ClockSampler(local_rank) as clk:
            total_ms, stage_ms = time_region(path, args.steps, torch, dist, ["attn"])
        if not clk.rejected():
            break
    st = path.ra.ra_sync_status()
    if st != 0:
        raise RuntimeError(f"kernel status {st}: {path.ra.ra_last_error()}")
    ms_step = max_over_ranks(total_ms / args.steps, dist, torch, device)
    k_ms = max_over_ranks(statistics.mean(stage_ms["attn"]), dist, torch, device)
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    value = path.bytes * world / (ms_step * 1e-3) / 1e9
    achieved = path.bytes / (k_ms * 1e-3) / 1e9
    out = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
           "data": "synthetic", "config": dict(config, parallelism=f"replicas{world}"),
           "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                        "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": None,
                        "kernel": "lse_merge_kernel", "peak_source": f"{peaks_src} hbm_gbs",
                        "frac_of_datasheet": round(achieved / DATASHEET_HBM_GBS, 4)},
           "gpu_launches": path.launches_per_step * args.steps, "clocks": clk.summary()}
    if not args.no_e2e:
        path2 = Path("merge", w, device)
        e2e_ms = e2e_region([path, path2], args.steps, torch, dist, device)
        del path2
        out["e2e"] = {"value": round(path.bytes * world / (e2e_ms * 1e-3) / 1e9, 1),
                      "unit": "GB/s", "h2d_bytes_per_step": path.in_bytes,
                      "d2h_bytes_per_step": path.out_bytes, "ms_per_step": round(e2e_ms, 3),
                      "steps": args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, n, dt, cores = run_oracle_merge(w)
        out["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                               "sample": f"{n} rows of two partials (D={w.D}), fp64 oracle "
                                         f"merge, {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def reference_arm(args, kind, w, w_attn, rank, world):
    """The oracle timed on the host cores as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    # size one step's sample so that warmup + steps end within a few minutes
    per_step_s = args.ref_step_seconds or max(2.0, min(20.0, 150.0 / (args.steps + args.warmup)))
    bwd = kind.startswith("attn_bwd")
    if bwd:
        _, n, _, _ = run_oracle_bwd_sample(w_attn, target_s=per_step_s)
        bq, bk, bv, bdo, flops = oracle_bwd_sample(w_attn, n)
        one_step = lambda: oracle.attention_backward(bq, bk, bv, bdo, w_attn.scale, w_attn.causal)
        sample = (f"gradients of one head's {n}-token sequence per step (D={w_attn.D}), "
                  f"fp64 oracle")
    else:
        _, n, _, _ = run_oracle_sample(w_attn, target_s=per_step_s)
        q, rb, rt, rh, k, v, flops = oracle_sample(w_attn, n)
        one_step = lambda: oracle.attention_rows(q, rb, rt, rh, k, v, 1, w_attn.scale,
                                                 w_attn.causal)
        sample = (f"{n} query rows x all visible keys of one {w_attn.L}-token sequence per "
                  f"step, fp64 oracle")
    for _ in range(args.warmup):
        pass  # the oracle has no warm state; the calibration run above served as warm-up
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        one_step()
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = flops / sec / 1e12
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic",
           "config": {"workload": w.name + SUFFIX.get(kind, ""),
                      "seq_len": w_attn.L, "head_dim": w_attn.D,
                      "causal": w_attn.causal, "parallelism": "cpu-oracle"},
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
