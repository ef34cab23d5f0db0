#!/usr/bin/env python
"""Throughput of the CSA / HCA hot path on B200, one JSON line on rank 0.

Default workload: hybrid decode at 1,048,576-token context, batch 8 per GPU:
one CSA layer (lightning indexer + top-2048 over 262,144 compressed entries,
sparse MQA over an FP8/BF16 split cache + a 128-token window) then one HCA
layer (dense MQA over 8,192 heavily compressed entries + the window), 64 query
heads, qk dim 192, v dim 128.  A step is that whole pass for one new token of
every sequence; value = tokens (sequences x GPUs) per second.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own 8 sequences
(weak scaling, no collective on the data path); time = max over ranks.
``--impl reference`` times the float64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
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
sys.path.insert(1, os.path.join(ROOT, "tests"))  # parity.py: the comparison rules of the GPU tests

METRIC = "CSA/HCA attention tokens/s at 128K and 1M ctx; % of HBM / tensor-core peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="hybrid_decode_l1m")
    ap.add_argument("--cpu-sample-s", type=float, default=12.0, help="host seconds for the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--profile-reps", type=int, default=100, help="launches of the dominant kernel to average")
    ap.add_argument("--breakdown", action="store_true", help="also time each library call of the step (stderr)")
    ap.add_argument("--no-extras", action="store_true", help="skip timing the rows beyond the headline step")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def profile_traffic(kernel: str, source: str, workload: str):
    """DRAM bytes per launch from the committed ncu data table (profiles/ncu_traffic.tsv), if it was captured on
    this workload and the kernel source has not changed since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.tsv")
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(os.path.join(ROOT, source), "rb").read()).hexdigest()[:16]
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        f = line.rstrip("\n").split("\t")
        if len(f) >= 4 and f[0] == kernel and f[2] == sha and f[3] == workload:
            return float(f[1])
    return None


class ClockSampler:
    """SM clock / throttle-reason samples while a region runs.

    Polls NVML in a thread (every 5 ms) on the GPU that torch's device `dev` is (matched by UUID, then PCI bus
    id), and takes one more sample when `mark()` is called after the region's work is enqueued, so that even a
    region of a few milliseconds has a sample taken while the GPU is busy.  Without NVML it falls back to an
    `nvidia-smi -lms 50` child.  Only reads: no clock, power or mode setting is touched."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []  # (sm_mhz, max_mhz, set of reasons)
        self.nvml = None
        self.proc = None
        self.lines = []
        self.stop = threading.Event()
        self.source = "none"

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
        except Exception:
            pass
        try:
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def _sample_nvml(self):
        nv, h = self.nvml
        try:
            sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception:
            return
        reasons = {name for name, const in self.REASONS if bits & getattr(nv, const, 0)}
        self.samples.append((float(sm), float(mx), reasons))

    def _poll(self):
        while not self.stop.wait(0.005):
            self._sample_nvml()

    def __enter__(self):
        try:
            self.nvml = self._nvml_handle()
            self.source = "nvml"
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            self.source = "nvidia-smi"
            time.sleep(0.4)
        except OSError:
            self.proc = None
        self.t0 = time.time()
        return self

    def mark(self):
        """One sample now (call it after the region's work is enqueued, while the GPU runs it)."""
        if self.nvml is not None:
            self._sample_nvml()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def __exit__(self, *exc):
        self.t1 = time.time()
        self.stop.set()
        if self.nvml is not None:
            self.thread.join(timeout=1)
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def _smi_samples(self):
        names = [n for n, _ in self.REASONS]
        out = []
        for t, r in self.lines:
            if not (self.t0 <= t <= self.t1 + 0.06):
                continue
            parts = [x.strip() for x in r.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            out.append((sm, mx, {n for n, v in zip(names, parts[5:9]) if v.lower().startswith("active")}))
        return out

    def summary(self):
        rows = self.samples if self.nvml is not None else self._smi_samples()
        sm = [r[0] for r in rows]
        mx = rows[-1][1] if rows else None
        reasons = set().union(*[r[2] for r in rows]) if rows else set()
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


# ---------------------------------------------------------------------------
# decode workloads (CSA decode, hybrid CSA + HCA decode)
# ---------------------------------------------------------------------------
def packed(torch, tensors, device, pin=False):
    """One contiguous byte buffer holding copies of `tensors` in 256-byte aligned slots, and the views."""
    offs, total = [], 0
    for t in tensors:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    buf = torch.empty(total, dtype=torch.uint8, device=device, pin_memory=pin)
    views = []
    for t, o in zip(tensors, offs):
        v = buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
    return buf, views


class DecodeRun:
    # steps captured per graph launch: in a model the step is one layer's attention, chained with the other
    # layers in one launch, so the launch of a graph is amortised over several steps here too (every step
    # still runs all of its work; its inputs alone exceed L2)
    graph_steps = 8

    @staticmethod
    def hca_sms_for(wl):
        """SMs the HCA branch keeps to while the CSA indexer streams its keys beside it (0 = all).  With bf16
        indexer keys the scoring kernel streams for ~46 us, and a branch held to 80 SMs (10 CTAs of 7 tiles
        per row) finishes inside that window: step 77.6 -> 73.6 us.  E4M3 and E2M1 keys score in 30-35 us, and
        there the whole GPU is better (61.8 us against 64.8 us at 80 SMs)."""
        return 80 if wl.kind == "hybrid" and not (wl.indexer_fp8 or wl.indexer_fp4) else 0

    def __init__(self, wl, rank, dev):
        import torch
        import long_context_sparse_10_b200 as csa
        from long_context_sparse_10_b200 import synth
        self.torch, self.csa, self.wl, self.dev = torch, csa, wl, dev
        from long_context_sparse_10_b200 import replicas
        self.host = synth.decode_inputs(wl, seed=0, batch=replicas.shard(rank, wl.B))
        h = self.host
        d = {k: v.to(dev) for k, v in h.items()}
        self.d = d
        B, L, H, k, m = wl.B, wl.L, wl.H, wl.k, wl.m
        self.scale = 1.0 / math.sqrt(192)
        self.q_pos0 = L - 1
        self.cache = csa.KVCache(nope=d["nope"], rope=d["rope"], scale=d["scale"])
        self.win = csa.Window(k=d["win_k"], pos0=L - wl.win, length=wl.win)
        self.idx = torch.empty(B, 1, k, dtype=torch.int32, device=dev)
        self.ws_idx = torch.empty(max(1, csa.csa_indexer_topk_workspace_size(B, 1, wl.N, k)), dtype=torch.uint8,
                                  device=dev)
        nws = csa.csa_sparse_mqa_workspace_size(B, 1, H, k, wl.win)
        self.ws_attn = torch.empty(max(1, nws), dtype=torch.uint8, device=dev)
        self.out = torch.empty(B, 1, H, 128, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(B, 1, H, dtype=torch.float32, device=dev)
        self.hybrid = wl.kind == "hybrid"
        if self.hybrid:
            self.side = torch.cuda.Stream(device=dev)  # the HCA branch's stream
            self.hca_sms = self.hca_sms_for(wl)
            self.hcache = csa.KVCache(nope=d["hca_nope"], rope=d["hca_rope"], scale=d["hca_scale"])
            self.hwin = csa.Window(k=d["hca_win_k"], pos0=L - wl.win, length=wl.win)
            hws = csa.hca_dense_mqa_workspace_size(B, 1, H, wl.N_hca, wl.win)
            self.ws_hca = torch.empty(max(1, hws), dtype=torch.uint8, device=dev)
            self.hout = torch.empty(B, 1, H, 128, dtype=torch.bfloat16, device=dev)
            self.hlse = torch.empty(B, 1, H, dtype=torch.float32, device=dev)
        # end-to-end buffers: the per-step inputs (queries, indexer queries and head weights) live in one
        # device buffer filled by one copy from one pinned host buffer; the outputs likewise
        keys = ["q", "qI", "wI"] + (["hca_q"] if self.hybrid else [])
        self.dev_in, views = packed(torch, [d[k] for k in keys], dev)
        for k_, v in zip(keys, views):
            d[k_] = v
        self.host_in, _ = packed(torch, [h[k_] for k_ in keys], "cpu", pin=True)
        outs = [self.out] + ([self.hout] if self.hybrid else [])
        self.dev_out, views = packed(torch, outs, dev)
        self.out = views[0]
        if self.hybrid:
            self.hout = views[1]
        self.host_out = torch.empty(self.dev_out.numel(), dtype=torch.uint8, pin_memory=True)
        # a second buffer set, so that the end-to-end loop can copy one step's inputs in (and the previous
        # step's outputs out) while the other step computes
        self.in_keys = keys
        dev_in_b, in_b = packed(torch, [d[k_] for k_ in keys], dev)
        dev_out_b, out_b = packed(torch, outs, dev)
        self.sets = [dict(dev_in=self.dev_in, ins=[d[k_] for k_ in keys], dev_out=self.dev_out,
                          outs=[self.out] + ([self.hout] if self.hybrid else []), host_in=self.host_in,
                          host_out=self.host_out),
                     dict(dev_in=dev_in_b, ins=in_b, dev_out=dev_out_b, outs=out_b,
                          host_in=torch.empty_like(self.host_in).pin_memory().copy_(self.host_in),
                          host_out=torch.empty_like(self.host_out).pin_memory())]
        self.tokens = B

    def step_timed(self):
        self.step()

    def indexer(self):
        wl = self.wl
        if wl.indexer_fp8:
            self.csa.csa_indexer_topk_e4m3(self.d["qI"], self.d["wI"], self.d["kI_codes"], self.d["kI_scale"], wl.m,
                                           wl.k, q_pos0=self.q_pos0, idx=self.idx, workspace=self.ws_idx)
        elif wl.indexer_fp4:
            self.csa.csa_indexer_topk_e2m1(self.d["qI"], self.d["wI"], self.d["kI_codes"], self.d["kI_scale"], wl.m,
                                           wl.k, q_pos0=self.q_pos0, idx=self.idx, workspace=self.ws_idx)
        else:
            self.csa.csa_indexer_topk(self.d["qI"], self.d["wI"], self.d["kIc"], wl.m, wl.k, q_pos0=self.q_pos0,
                                      idx=self.idx, workspace=self.ws_idx)

    def step(self):
        """One decode step.  The HCA branch does not depend on the CSA branch's indexer, so it runs on a second
        stream forked from (and joined back into) the caller's: its latency-bound kernels fill the SMs that the
        top-k tail and the CSA attention leave idle."""
        wl, csa, torch = self.wl, self.csa, self.torch
        main = torch.cuda.current_stream()
        if self.hybrid:
            self.side.wait_stream(main)
        self.indexer()
        if self.hybrid:
            with torch.cuda.stream(self.side):
                csa.hca_dense_mqa(self.d["hca_q"], self.hcache, wl.m_hca, self.hwin, self.scale, q_pos0=self.q_pos0,
                                  out=self.hout, lse=self.hlse, workspace=self.ws_hca, max_sms=self.hca_sms)
        csa.csa_sparse_mqa(self.d["q"], self.cache, wl.m, self.idx, self.win, self.scale, q_pos0=self.q_pos0,
                           out=self.out, lse=self.lse, workspace=self.ws_attn)
        if self.hybrid:
            main.wait_stream(self.side)

    def parts(self):
        """The step's library calls, separately (for --breakdown)."""
        wl, csa = self.wl, self.csa
        out = [("csa_indexer_topk", self.indexer),
               ("csa_sparse_mqa", lambda: csa.csa_sparse_mqa(self.d["q"], self.cache, wl.m, self.idx, self.win,
                                                             self.scale, q_pos0=self.q_pos0, out=self.out,
                                                             lse=self.lse, workspace=self.ws_attn))]
        if self.hybrid:
            out.append(("hca_dense_mqa", lambda: csa.hca_dense_mqa(self.d["hca_q"], self.hcache, wl.m_hca, self.hwin,
                                                                   self.scale, q_pos0=self.q_pos0, out=self.hout,
                                                                   lse=self.hlse, workspace=self.ws_hca)))
        return out

    def e2e_step(self):
        self.dev_in.copy_(self.host_in, non_blocking=True)
        self.step()
        self.host_out.copy_(self.dev_out, non_blocking=True)

    def e2e_bytes(self):
        return self.host_in.numel(), self.host_out.numel()

    def _bind(self, st):
        for k_, v in zip(self.in_keys, st["ins"]):
            self.d[k_] = v
        self.out = st["outs"][0]
        if self.hybrid:
            self.hout = st["outs"][1]

    def e2e_pipeline(self, n):
        """Capture n end-to-end steps into one CUDA graph: step i computes on buffer set i % 2 while a copy
        stream brings in step i+1's inputs and takes out step i-1's outputs.  Returns the graph."""
        torch = self.torch
        s_copy = torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_done = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            main = torch.cuda.current_stream()
            s_copy.wait_stream(main)
            with torch.cuda.stream(s_copy):
                self.sets[0]["dev_in"].copy_(self.sets[0]["host_in"], non_blocking=True)
                ev_in[0].record(s_copy)
            for i in range(n):
                cur = self.sets[i % 2]
                main.wait_event(ev_in[i])
                if i >= 2:
                    main.wait_event(ev_out[i - 2])  # this set's previous outputs are on the host
                self._bind(cur)
                self.step()
                ev_done[i].record(main)
                with torch.cuda.stream(s_copy):
                    if i + 1 < n:
                        if i >= 1:
                            s_copy.wait_event(ev_done[i - 1])  # the next set's last reader has finished
                        nxt = self.sets[(i + 1) % 2]
                        nxt["dev_in"].copy_(nxt["host_in"], non_blocking=True)
                        ev_in[i + 1].record(s_copy)
                    s_copy.wait_event(ev_done[i])
                    cur["host_out"].copy_(cur["dev_out"], non_blocking=True)
                    ev_out[i].record(s_copy)
            main.wait_stream(s_copy)
        self._bind(self.sets[0])
        return g

    def dominant(self):
        """(name, source file, algorithmic bytes per launch, callable that launches it)."""
        wl = self.wl
        per_entry = self.key_bytes()
        b = wl.B * wl.N * per_entry + wl.B * 4 * 64 * 2 + wl.B * 4 * 4
        name = ("indexer_score_long_e4m3" if wl.indexer_fp8 else
                "indexer_score_long_e2m1" if wl.indexer_fp4 else "indexer_score_long")
        return name, "long_context_sparse_10_b200/csrc/indexer.cu", b, "hbm", self.indexer

    def step_bytes(self):
        """Algorithmic HBM bytes of one decode step: the indexer keys and queries, the gathered split-cache
        entries (128 e4m3 + 64 bf16 + fp32 scale = 260 B), the window keys, the queries, the selection and the
        outputs; plus, for the hybrid step, the HCA layer's whole cache, window, query and output."""
        wl = self.wl
        B, H, k = wl.B, wl.H, wl.k
        b = B * wl.N * self.key_bytes() + B * (4 * 64 * 2 + 4 * 4)
        b += B * k * 260 + B * wl.win * 192 * 2 + B * H * 192 * 2 + B * H * 128 * 2 + B * k * 4
        if self.hybrid:
            b += B * wl.N_hca * 260 + B * wl.win * 192 * 2 + B * H * 192 * 2 + B * H * 128 * 2
        return b

    def step_roofline(self, ms, pk):
        b = self.step_bytes()
        return {"bound": "hbm", "algorithmic_bytes": b, "achieved": b / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": b / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}

    def key_bytes(self):
        """Indexer key bytes per entry: E4M3 codes + scale, E2M1 codes + scale, or bf16."""
        wl = self.wl
        return (64 + 4) if wl.indexer_fp8 else (32 + 4) if wl.indexer_fp4 else 64 * 2

    def describe(self, world):
        wl = self.wl
        keys = ("e4m3 keys + per-entry scale" if wl.indexer_fp8 else
                "e2m1 (FP4) keys + per-entry scale" if wl.indexer_fp4 else "bf16")
        s = (f"{wl.name}: decode at context {wl.L}, batch {wl.B} per GPU, {wl.H} query heads, qk 192 / v 128; "
             f"CSA m={wl.m} (N={wl.N}, FP8-e4m3 nope + BF16 RoPE cache, indexer 4x64 {keys}, top-k={wl.k})")
        if self.hybrid:
            s += f" then HCA m'={wl.m_hca} (N'={wl.N_hca}, same split cache)"
        s += f", sliding window {wl.win}"
        if self.hybrid:
            sms = self.hca_sms_for(wl)
            s += "; HCA branch on a forked stream" + (f" held to {sms} SMs" if sms else "")
        return {"workload": s, "global_batch": wl.B * world, "seq_len": wl.L, "parallelism": f"dp{world} (replicas)",
                "l2": f"inputs larger than L2 (the step streams {self.step_bytes() / 1e6:.0f} MB > 126 MB L2)",
                "timing": f"CUDA graph replay, {self.graph_steps} whole steps captured per launch"}

    def _oracle_seq(self, b):
        """Float64 oracle of sequence b's whole decode step: (scores, idx, csa (O, lse), hca (O, lse) or None)."""
        import numpy as np
        from oracle import csa_ref as R
        h, wl = self.host, self.wl
        qI = h["qI"][b:b + 1].double().numpy()
        wI = h["wI"][b:b + 1].double().numpy()
        if wl.indexer_fp8:
            kI = R.e4m3_decode(h["kI_codes"][b:b + 1].numpy()) * h["kI_scale"][b:b + 1].double().numpy()[..., None]
        elif wl.indexer_fp4:
            kI = R.e2m1_unpack(h["kI_codes"][b:b + 1].numpy()) * h["kI_scale"][b:b + 1].double().numpy()[..., None]
        else:
            kI = h["kIc"][b:b + 1].double().numpy()
        q = h["q"][b:b + 1].double().numpy()
        wk = h["win_k"][b:b + 1].double().numpy()
        nope, rope, sc = h["nope"][b:b + 1].numpy(), h["rope"][b:b + 1].double().numpy(), h["scale"][b:b + 1].numpy()
        pos = np.array([wl.L - 1])
        s = R.indexer_scores(qI, wI, kI, pos, wl.m)
        idx = R.topk_set(s, wl.k)
        K, V = R.dequant_split(nope, rope, sc)
        csa_out = R.csa_sparse_mqa(q, pos, K, V, idx, wl.m, wk, wk[..., :128], wl.L - wl.win, wl.win, self.scale)
        hca_out = None
        if self.hybrid:
            hq = h["hca_q"][b:b + 1].double().numpy()
            hwk = h["hca_win_k"][b:b + 1].double().numpy()
            HK, HV = R.dequant_split(h["hca_nope"][b:b + 1].numpy(), h["hca_rope"][b:b + 1].double().numpy(),
                                     h["hca_scale"][b:b + 1].numpy())
            hca_out = R.hca_dense_mqa(hq, pos, HK, HV, wl.m_hca, hwk, hwk[..., :128], wl.L - wl.win, wl.win,
                                      self.scale)
        return s, idx, csa_out, hca_out, (q, pos, K, V, wk)

    def self_check(self):
        """Sequence 0 of the last step against the float64 oracle (parity rules of the GPU tests)."""
        import numpy as np
        from oracle import csa_ref as R
        from parity import assert_close, assert_lse, check_topk
        torch, wl = self.torch, self.wl
        torch.cuda.synchronize()
        got_idx = self.idx[0:1].cpu().numpy()
        got_o, got_l = self.out[0:1].double().cpu().numpy(), self.lse[0:1].double().cpu().numpy()
        s, idx, (O, L), hca, (q, pos, K, V, wk) = self._oracle_seq(0)
        same = check_topk(got_idx, s, idx, wl.k, "bench self-check: indexer")
        if not same.all():  # tie-band row: attention is compared on the GPU's own selection
            O, L = R.csa_sparse_mqa(q, pos, K, V, got_idx.astype(np.int64), wl.m, wk, wk[..., :128], wl.L - wl.win,
                                    wl.win, self.scale)
        ma, rl = assert_close(got_o, O, "bench self-check: csa attention")
        assert_lse(got_l, L, "bench self-check: csa lse")
        res = {"rows": 1, "topk_identical": float(same.mean()), "max_abs": ma, "rel_l2": rl}
        if hca is not None:
            hma, hrl = assert_close(self.hout[0:1].double().cpu().numpy(), hca[0], "bench self-check: hca attention")
            assert_lse(self.hlse[0:1].double().cpu().numpy(), hca[1], "bench self-check: hca lse")
            res.update(hca_max_abs=hma, hca_rel_l2=hrl)
        return res

    def oracle_sample(self, budget_s):
        """Time the float64 oracle on whole sequences of this workload (host cores)."""
        done, spent = 0, 0.0
        for b in range(self.wl.B):
            t0 = time.perf_counter()
            self._oracle_seq(b)
            spent += time.perf_counter() - t0
            done += 1
            if spent >= budget_s:
                break
        return done, spent, f"{done} of {self.wl.B} sequences of one rank's batch, whole decode step each"


# ---------------------------------------------------------------------------
# prefill workloads (CSA prefill, HCA prefill)
# ---------------------------------------------------------------------------
class PrefillRun:
    def __init__(self, wl, rank, dev):
        import torch
        import long_context_sparse_10_b200 as csa
        from long_context_sparse_10_b200 import synth
        self.torch, self.csa, self.wl, self.dev = torch, csa, wl, dev
        self.host = synth.prefill_inputs(wl, seed=rank)
        d = {k: v.to(dev) for k, v in self.host.items()}
        self.d = d
        B, T, H, m, N = wl.B, wl.T, wl.H, wl.m, wl.N
        self.scale = 1.0 / math.sqrt(192)
        self.Kc = torch.empty(B, N, 192, dtype=torch.bfloat16, device=dev)
        self.Vc = torch.empty(B, N, 128, dtype=torch.bfloat16, device=dev)
        self.out = torch.empty(B, T, H, 128, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(B, T, H, dtype=torch.float32, device=dev)
        self.csa_kind = wl.kind == "csa"
        if self.csa_kind:
            self.kIc = torch.empty(B, N, 64, dtype=torch.bfloat16, device=dev)
            self.idx = torch.empty(B, T, wl.k, dtype=torch.int32, device=dev)
            self.ws_idx = torch.empty(max(1, csa.csa_indexer_topk_workspace_size(B, T, N, wl.k)), dtype=torch.uint8,
                                      device=dev)
        self.h_in = {k: self.host[k].pin_memory() for k in self.host}
        self.h_out = [torch.empty_like(self.out, device="cpu").pin_memory()]
        self.tokens = B * T
        # timed steps rotate over copies of the inputs and outputs, so that one pass over the sets exceeds the
        # 126 MB L2 and no step finds its inputs left in L2 by the step before
        self.set_bytes, nsets = self.rotation()
        self.rot = [dict(d=dict(d), out=self.out, lse=self.lse)]
        for _ in range(nsets - 1):
            self.rot.append(dict(d={k_: v.clone() for k_, v in d.items()}, out=torch.empty_like(self.out),
                                 lse=torch.empty_like(self.lse)))
        self.graph_steps = nsets
        self._rot_i = 0

    def rotation(self):
        """(bytes of one step's inputs and outputs, number of sets the timed steps rotate over)."""
        wl = self.wl
        set_bytes = sum(v.numel() * v.element_size() for v in self.host.values()) + wl.B * wl.T * wl.H * (128 * 2 + 4)
        return set_bytes, (1 if set_bytes > 126e6 else min(16, math.ceil(1.5 * 126e6 / set_bytes)))

    def step_timed(self):
        """One step on the next input/output set of the rotation."""
        st = self.rot[self._rot_i]
        self._rot_i = (self._rot_i + 1) % len(self.rot)
        self.d, self.out, self.lse = dict(st["d"]), st["out"], st["lse"]
        self.step()

    def attention(self):
        wl, csa = self.wl, self.csa
        win = csa.Window(k=self.d["k"], v=self.d["v"], pos0=0, length=wl.win)
        if self.csa_kind:
            csa.csa_sparse_mqa(self.d["q"], csa.KVCache(k=self.Kc, v=self.Vc), wl.m, self.idx, win, self.scale,
                               out=self.out, lse=self.lse)
        else:
            csa.hca_dense_mqa(self.d["q"], csa.KVCache(k=self.Kc, v=self.Vc), wl.m, win, self.scale,
                              out=self.out, lse=self.lse)

    def step(self):
        wl, csa, d = self.wl, self.csa, self.d
        fn = csa.csa_compress if self.csa_kind else csa.hca_compress
        fn(d["k"], d["w_k"], d["b_k"], wl.m, out=self.Kc)
        fn(d["v"], d["w_v"], d["b_v"], wl.m, out=self.Vc)
        if self.csa_kind:
            fn(d["kI"], d["w_i"], d["b_i"], wl.m, out=self.kIc)
            csa.csa_indexer_topk(d["qI"], d["wI"], self.kIc, wl.m, wl.k, idx=self.idx, workspace=self.ws_idx)
        self.attention()

    def parts(self):
        wl, csa, d = self.wl, self.csa, self.d
        fn = csa.csa_compress if self.csa_kind else csa.hca_compress
        out = [("compress K", lambda: fn(d["k"], d["w_k"], d["b_k"], wl.m, out=self.Kc)),
               ("compress V", lambda: fn(d["v"], d["w_v"], d["b_v"], wl.m, out=self.Vc))]
        if self.csa_kind:
            out += [("compress kI", lambda: fn(d["kI"], d["w_i"], d["b_i"], wl.m, out=self.kIc)),
                    ("csa_indexer_topk", lambda: csa.csa_indexer_topk(d["qI"], d["wI"], self.kIc, wl.m, wl.k,
                                                                      idx=self.idx, workspace=self.ws_idx))]
        out.append(("attention", self.attention))
        return out

    def e2e_step(self):
        for k, v in self.h_in.items():
            self.d[k].copy_(v, non_blocking=True)
        self.step()
        self.h_out[0].copy_(self.out, non_blocking=True)

    def e2e_bytes(self):
        return (sum(v.numel() * v.element_size() for v in self.h_in.values()),
                sum(v.numel() * v.element_size() for v in self.h_out))

    def _bind(self, st):
        for k_, v in st["ins"].items():
            self.d[k_] = v
        self.out = st["out"]

    def e2e_pipeline(self, n):
        """Capture n end-to-end steps into one CUDA graph over two buffer sets: while step i computes on set
        i % 2, one copy stream brings step i+1's inputs in from pinned host memory and another takes step i-1's
        output out (the two directions of the link overlap).  Returns the graph."""
        torch = self.torch
        sets = [dict(ins={k_: self.d[k_] for k_ in self.h_in}, out=self.out, h_in=self.h_in, h_out=self.h_out[0]),
                dict(ins={k_: torch.empty_like(self.d[k_]) for k_ in self.h_in}, out=torch.empty_like(self.out),
                     h_in={k_: torch.empty_like(v).pin_memory().copy_(v) for k_, v in self.h_in.items()},
                     h_out=torch.empty_like(self.h_out[0]).pin_memory())]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_done = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]

        def copy_in(st):
            for k_, v in st["h_in"].items():
                st["ins"][k_].copy_(v, non_blocking=True)

        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            main = torch.cuda.current_stream()
            s_in.wait_stream(main)
            s_out.wait_stream(main)
            with torch.cuda.stream(s_in):
                copy_in(sets[0])
                ev_in[0].record(s_in)
            for i in range(n):
                cur = sets[i % 2]
                main.wait_event(ev_in[i])
                if i >= 2:
                    main.wait_event(ev_out[i - 2])  # this set's previous output is on the host
                self._bind(cur)
                self.step()
                ev_done[i].record(main)
                if i + 1 < n:
                    with torch.cuda.stream(s_in):
                        if i >= 1:
                            s_in.wait_event(ev_done[i - 1])  # the next set's last reader has finished
                        copy_in(sets[(i + 1) % 2])
                        ev_in[i + 1].record(s_in)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[i])
                    cur["h_out"].copy_(cur["out"], non_blocking=True)
                    ev_out[i].record(s_out)
            main.wait_stream(s_in)
            main.wait_stream(s_out)
        self._bind(sets[0])
        return g

    def attn_flops(self):
        wl = self.wl
        t = __import__("numpy").arange(wl.T)
        ent = (t + 1) // wl.m
        if self.csa_kind:
            ent = __import__("numpy").minimum(ent, wl.k)
        keys = ent + __import__("numpy").minimum(wl.win, t + 1)
        return float(wl.B * wl.H * 2 * (192 + 128) * keys.sum())

    def step_roofline(self, ms, pk):
        """Tensor work of the whole prefill step (attention + indexer scores, algorithmic) against bf16 peak."""
        import numpy as np
        wl = self.wl
        f = self.attn_flops()
        if self.csa_kind:
            t = np.arange(wl.T)
            f += float(wl.B * 2 * 4 * 64 * np.minimum((t + 1) // wl.m, wl.N).sum())
        return {"bound": "tensor", "algorithmic_flops": f, "achieved": f / (ms * 1e-3) / 1e12,
                "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                "frac": f / (ms * 1e-3) / 1e12 / pk["bf16_tflops_sustained"]}

    def dominant(self):
        return ("attention_prefill", "long_context_sparse_10_b200/csrc/attention.cu", self.attn_flops(), "tensor",
                self.attention)

    def describe(self, world):
        wl = self.wl
        set_bytes, nsets = self.rotation()
        s = (f"{wl.name}: {wl.kind.upper()} prefill, B={wl.B}, T={wl.T}, {wl.H} query heads, qk 192 / v 128, "
             f"stride {wl.m}" + (f", indexer 4x64, top-k={wl.k}" if self.csa_kind else "") + f", window {wl.win}")
        return {"workload": s, "global_batch": wl.B * world, "seq_len": wl.T, "parallelism": f"dp{world} (replicas)",
                "l2": (f"inputs and outputs larger than L2 ({set_bytes / 1e6:.0f} MB per step)" if nsets == 1 else
                       f"steps rotate over {nsets} input/output sets of {set_bytes / 1e6:.0f} MB "
                       f"({nsets * set_bytes / 1e6:.0f} MB > 126 MB L2)"),
                "timing": f"CUDA graph replay, {nsets} whole steps captured per launch"}

    def self_check(self):
        """Sampled query rows of sequence 0 of the last step against the float64 oracle: rows before the window
        fills and before top-k selection becomes partial, and a stride over the rest."""
        import numpy as np
        from oracle import csa_ref as R
        from parity import assert_close, assert_lse, check_topk
        torch, wl, h = self.torch, self.wl, self.host
        torch.cuda.synchronize()
        cw = 2 * wl.m if self.csa_kind else wl.m

        def bf16_cache(x, w, b):   # the oracle's entries, stored as bf16 like the GPU cache
            y = R.compress(x[:1].double().numpy(), w.double().numpy(), b.double().numpy(), wl.m, cw)
            return torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16).double().numpy()

        Kc, Vc = bf16_cache(h["k"], h["w_k"], h["b_k"]), bf16_cache(h["v"], h["w_v"], h["b_v"])
        res = {}
        ma, _ = assert_close(self.Kc[0:1].double().cpu().numpy(), Kc, "bench self-check: compressed K", max_abs=1.6e-2)
        T = wl.T
        rows = np.unique(np.concatenate([np.arange(0, min(T, 40), 3), np.linspace(0, T - 1, 24).astype(np.int64),
                                         [T - 1]]))
        q = h["q"][:1, rows].double().numpy()
        K, V = h["k"][:1].double().numpy(), h["v"][:1].double().numpy()
        if self.csa_kind:
            kIc = bf16_cache(h["kI"], h["w_i"], h["b_i"])
            s = R.indexer_scores(h["qI"][:1, rows].double().numpy(), h["wI"][:1, rows].double().numpy(), kIc, rows,
                                 wl.m)
            idx = R.topk_set(s, wl.k)
            got_idx = self.idx[0:1, rows].cpu().numpy()
            same = check_topk(got_idx, s, idx, wl.k, "bench self-check: indexer")
            use = np.where(same[None, :, None], idx, got_idx.astype(np.int64))
            O, L = R.csa_sparse_mqa(q, rows, Kc, Vc, use, wl.m, K, V, 0, wl.win, self.scale)
            res["topk_identical"] = float(same.mean())
        else:
            O, L = R.hca_dense_mqa(q, rows, Kc, Vc, wl.m, K, V, 0, wl.win, self.scale)
        ma, rl = assert_close(self.out[0:1, rows].double().cpu().numpy(), O, "bench self-check: attention")
        assert_lse(self.lse[0:1, rows].double().cpu().numpy(), L, "bench self-check: lse")
        res.update(rows=int(len(rows)), max_abs=ma, rel_l2=rl)
        return res

    def oracle_sample(self, budget_s):
        import numpy as np
        from oracle import csa_ref as R
        h, wl = self.host, self.wl
        t0 = time.perf_counter()
        cw = 2 * wl.m if self.csa_kind else wl.m
        K = h["k"][:1].double().numpy()
        V = h["v"][:1].double().numpy()
        Kc = R.compress(K, h["w_k"].double().numpy(), h["b_k"].double().numpy(), wl.m, cw)
        Vc = R.compress(V, h["w_v"].double().numpy(), h["b_v"].double().numpy(), wl.m, cw)
        if self.csa_kind:
            kIc = R.compress(h["kI"][:1].double().numpy(), h["w_i"].double().numpy(), h["b_i"].double().numpy(),
                             wl.m, cw)
        rows_done = 0
        rng = np.random.default_rng(0)
        order = rng.permutation(wl.T)
        for c in range(0, wl.T, 64):
            rows = np.sort(order[c:c + 64])
            q = h["q"][:1, rows].double().numpy()
            if self.csa_kind:
                s = R.indexer_scores(h["qI"][:1, rows].double().numpy(), h["wI"][:1, rows].double().numpy(), kIc,
                                     rows, wl.m)
                idx = R.topk_set(s, wl.k)
                R.csa_sparse_mqa(q, rows, Kc, Vc, idx, wl.m, K, V, 0, wl.win, self.scale)
            else:
                R.hca_dense_mqa(q, rows, Kc, Vc, wl.m, K, V, 0, wl.win, self.scale)
            rows_done += len(rows)
            if time.perf_counter() - t0 >= budget_s:
                break
        spent = time.perf_counter() - t0
        return rows_done, spent, (f"compression of sequence 0 plus {rows_done} random query rows of it "
                                  f"(tokens/s counts those rows)")


# ---------------------------------------------------------------------------
# the rows beyond the headline step, each timed on its own (CUDA events around
# graph replays of the library call) against its roofline
# ---------------------------------------------------------------------------
def _time_graph(torch, fn, reps=20, iters=5):
    """Median per-call milliseconds of `fn` captured `reps` times in one CUDA graph.  `fn` may be a list of
    callables over distinct buffers, used in turn, so that consecutive calls do not find their inputs in L2."""
    fns = fn if isinstance(fn, (list, tuple)) else [fn]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for f in fns:
            f()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for r in range(reps):
            fns[r % len(fns)]()
    g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / reps)
    del g
    return statistics.median(ts)


def extras(dev, pk):
    """Grouped output projection, decode-time cache append, packed prefill and the context-parallel merges."""
    import numpy as np
    import torch
    import long_context_sparse_10_b200 as csa
    from long_context_sparse_10_b200 import context_parallel as cp
    g = np.random.default_rng(0)
    res = {}

    def bf16(shape, std=1.0):
        return torch.from_numpy((g.standard_normal(shape) * std).astype(np.float32)).to(torch.bfloat16).to(dev)

    # compression of the 65,536-token prefill (CSA m = 4: K 192, V 128, indexer key 64) and of the HCA
    # prefill (m' = 128): algorithmic bytes = raw tokens read once + entries written
    for name, (T, d, m, kind) in {"csa_compress_k_t65536": (65536, 192, 4, "csa"),
                                  "csa_compress_ki_t65536": (65536, 64, 4, "csa"),
                                  "hca_compress_k_b2_t8192": (16384, 192, 128, "hca")}.items():
        B = 2 if kind == "hca" else 1
        cw = 2 * m if kind == "csa" else m
        wc = torch.from_numpy((g.standard_normal(d) * 0.02).astype(np.float32)).to(dev)
        bc = torch.from_numpy((g.standard_normal((cw, d)) * 0.1).astype(np.float32)).to(dev)
        fn = csa.csa_compress if kind == "csa" else csa.hca_compress
        nbuf = max(2, int(300e6 // (T * d * 2)))   # inputs of consecutive calls together exceed the 126 MB L2
        xs_ = [bf16((B, T // B, d)) for _ in range(nbuf)]
        ys_ = [torch.empty(B, -(-(T // B) // m), d, dtype=torch.bfloat16, device=dev) for _ in range(nbuf)]
        ms = _time_graph(torch, [lambda x=x, y=y: fn(x, wc, bc, m, out=y) for x, y in zip(xs_, ys_)])
        byts = xs_[0].numel() * 2 + ys_[0].numel() * 2
        del xs_, ys_
        res[name] = {"us": ms * 1e3, "bound": "hbm", "algorithmic_bytes": byts,
                     "achieved_gbs": byts / (ms * 1e-3) / 1e9, "frac": byts / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
    # grouped output projection (64 heads in 8 groups of 8, d_g = 1024)
    ws_ = [bf16((8, 1024, 1024), 0.02) for _ in range(12)]   # 12 x 16 MiB of weights: more than L2
    w = ws_[0]
    for name, rows in (("decode_rows8", 8), ("prefill_rows16384", 16384)):
        o = bf16((rows, 64, 128), 0.5)
        if rows <= 128:
            ms = _time_graph(torch, [lambda w_=w_: csa.grouped_out_proj(o, w_) for w_ in ws_], reps=24)
        else:
            ms = _time_graph(torch, lambda: csa.grouped_out_proj(o, w))
        flops = 2.0 * rows * 64 * 128 * 1024
        byts = w.numel() * 2 + o.numel() * 2 + rows * 8 * 1024 * 2
        if rows <= 128:
            res[f"grouped_out_proj_{name}"] = {"us": ms * 1e3, "bound": "hbm", "algorithmic_bytes": byts,
                                               "achieved_gbs": byts / (ms * 1e-3) / 1e9,
                                               "frac": byts / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
        else:
            res[f"grouped_out_proj_{name}"] = {"us": ms * 1e3, "bound": "tensor", "algorithmic_flops": flops,
                                               "achieved_tflops": flops / (ms * 1e-3) / 1e12,
                                               "frac": flops / (ms * 1e-3) / 1e12 / pk["bf16_tflops"]}
    # decode-time append of the entry the newest token completes (8 sequences, split FP8 cache, d 192)
    B, rows = 8, 256
    xs = bf16((B, rows, 192))
    ww = torch.from_numpy((g.standard_normal(192) * 0.02).astype(np.float32)).to(dev)
    bb = torch.from_numpy((g.standard_normal((8, 192)) * 0.1).astype(np.float32)).to(dev)
    cache = csa.KVCache(nope=torch.zeros(B, 4096, 128, dtype=torch.uint8, device=dev),
                        rope=torch.zeros(B, 4096, 64, dtype=torch.bfloat16, device=dev),
                        scale=torch.zeros(B, 4096, device=dev))
    t = 4 * 4000 + 3
    ms = _time_graph(torch, lambda: csa.csa_compress_append(xs, t + 1 - rows, t, ww, bb, 4, cache))
    res["csa_compress_append_b8"] = {"us": ms * 1e3, "bound": "latency", "note": "one entry per sequence"}
    # packed CSA prefill: 16 documents, 16,384 tokens, H 64, k 512
    lens = [int(x) for x in g.integers(64, 2048, 16)]
    lens[-1] += 16384 - sum(lens)
    pkd = csa.Packed(lens, 4)
    TT = pkd.total_tokens
    q, K, V, qI, kI = bf16((TT, 64, 192)), bf16((TT, 192)), bf16((TT, 128)), bf16((TT, 4, 64)), bf16((TT, 64))
    wI = torch.from_numpy(g.random((TT, 4)).astype(np.float32)).to(dev)
    wk, bk = ww, bb
    wv = torch.from_numpy((g.standard_normal(128) * 0.02).astype(np.float32)).to(dev)
    bv = torch.from_numpy((g.standard_normal((8, 128)) * 0.1).astype(np.float32)).to(dev)
    wi = torch.from_numpy((g.standard_normal(64) * 0.02).astype(np.float32)).to(dev)
    bi = torch.from_numpy((g.standard_normal((8, 64)) * 0.1).astype(np.float32)).to(dev)

    def packed_step():
        Kc = csa.csa_compress_packed(K, pkd, wk, bk, 4)
        Vc = csa.csa_compress_packed(V, pkd, wv, bv, 4)
        kIc = csa.csa_compress_packed(kI, pkd, wi, bi, 4)
        idx = csa.csa_indexer_topk_packed(qI, wI, kIc, pkd, 4, 512)
        csa.csa_sparse_mqa_packed(q, pkd, csa.KVCache(k=Kc, v=Vc), 4, idx, K, V, 128, 1 / math.sqrt(192))
    ms = _time_graph(torch, packed_step, reps=3, iters=3)
    res["packed_csa_prefill_16docs_t16384"] = {"us": ms * 1e3, "tokens_per_s": TT / (ms * 1e-3),
                                               "documents": len(lens)}
    # context-parallel merges for 8 ranks, 8 decode rows, k 2048, 64 heads
    ops = cp.KernelOps()
    cs = torch.from_numpy(g.standard_normal((8, 1, 8 * 2048)).astype(np.float32)).to(dev)
    ci = torch.arange(8 * 2048, dtype=torch.int32, device=dev).repeat(8, 1).reshape(8, 1, 8 * 2048).contiguous()
    ms = _time_graph(torch, lambda: ops.topk_merge(cs, ci, 2048))
    res["cp_topk_merge_g8_rows8_k2048"] = {"us": ms * 1e3, "bound": "latency"}
    outs = bf16((8, 8, 1, 64, 128))
    lses = torch.from_numpy(g.standard_normal((8, 8, 1, 64)).astype(np.float32)).to(dev)
    ms = _time_graph(torch, lambda: ops.attn_merge(outs, lses))
    res["cp_attn_merge_g8_rows8"] = {"us": ms * 1e3, "bound": "latency"}
    return res


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def make_run(name, rank, dev):
    from long_context_sparse_10_b200 import synth
    wl = synth.WORKLOADS[name]
    return (DecodeRun if isinstance(wl, synth.Decode) else PrefillRun)(wl, rank, dev)


def reference_arm(args):
    """The float64 CPU oracle, timed on the host cores (rank 0 only): W untimed then K timed steps, each step a
    bounded sample of the workload (whole sequences for decode, sampled query rows for prefill)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from long_context_sparse_10_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    cls = DecodeRun if isinstance(wl, synth.Decode) else PrefillRun
    run = cls.__new__(cls)   # the same inputs, without touching a GPU
    run.wl = wl
    run.scale = 1.0 / math.sqrt(192)
    if isinstance(wl, synth.Decode):
        run.host = synth.decode_inputs(wl, seed=0, batch=slice(0, wl.B))
        run.hybrid = wl.kind == "hybrid"
    else:
        run.host = synth.prefill_inputs(wl, seed=0)
        run.csa_kind = wl.kind == "csa"
    budget = min(240.0, max(5.0, args.cpu_sample_s * 20))
    warm, timed = args.warmup, max(1, args.steps)
    # a step is at least one unit of oracle work (a whole sequence for decode, 64 query rows for prefill):
    # the first unit (a warm-up step when W >= 1) gives its cost, and when W + K such steps would outrun
    # the budget, fewer steps are timed (one warm-up at most), as the line states
    _, unit_s, _ = run.oracle_sample(0.0)
    warm = max(0, warm - 1)
    fit = int(budget / max(unit_s, 1e-3))
    if warm + timed > fit:
        warm = min(warm, 1)
        timed = max(1, min(timed, fit - warm))
    per_step = budget / (warm + timed)
    for _ in range(warm):
        run.oracle_sample(per_step)
    total_n, total_s, sample = 0, 0.0, ""
    for _ in range(timed):
        n, spent, sample = run.oracle_sample(per_step)
        total_n += n
        total_s += spent
    value = total_n / total_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": timed, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / timed,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": run.describe(args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample + f"; each step a sample of about {per_step:.1f} s",
                             "host_cpus": os.cpu_count()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if timed != args.steps:
        line["steps_requested"] = args.steps
        line["cpu_baseline"]["sample"] += (f"; {timed} of the {args.steps} requested steps timed (each step is at "
                                           f"least one unit of {unit_s:.2f} s, the run is bounded to {budget:.0f} s)")
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
        return
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one rank per GPU: relaunch this command under torchrun with --gpus ranks
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr", "127.0.0.1", "--master-port", str(29500 + os.getpid() % 1000), os.path.abspath(__file__),
               *sys.argv[1:]]
        sys.exit(subprocess.call(cmd))
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but the launcher started {world} rank(s)", file=sys.stderr)
        sys.exit(2)
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import long_context_sparse_10_b200 as csa
    from long_context_sparse_10_b200 import _lib, replicas
    lib = _lib.load()

    def barrier():
        if world > 1:
            dist.barrier()

    run = make_run(args.workload, rank, dev)
    torch.cuda.synchronize()

    # warm-up outside the graph (per-device one-time set-up happens here), then capture the step
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            run.step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    # the outputs of the last warm-up step against the oracle (rank 0): no line is printed for a wrong result
    check, ok = None, 1
    if rank == 0:
        try:
            check = run.self_check()
        except AssertionError as exc:
            print(f"bench.py: self-check against the oracle failed: {exc}", file=sys.stderr)
            ok = 0
    if world > 1:
        flag = torch.tensor([ok], dtype=torch.int32, device=dev)
        dist.all_reduce(flag, op=dist.ReduceOp.MIN)
        ok = int(flag.item())
    if not ok:
        if world > 1:
            dist.destroy_process_group()
        sys.exit(3)
    # one graph of run.graph_steps steps (each on the next set of a rotation that exceeds L2, for workloads
    # whose inputs alone would fit), and one of the remainder, so that exactly K steps are timed
    gs = run.graph_steps
    graph = torch.cuda.CUDAGraph()
    n0 = csa.launch_count()
    with torch.cuda.graph(graph):
        for _ in range(gs):
            run.step_timed()
    launches_per_step = (csa.launch_count() - n0) // gs  # this library's kernels in one captured step
    rem = args.steps % gs
    graph_rem = None
    if rem:
        graph_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_rem):
            for _ in range(rem):
                run.step_timed()
    for _ in range(max(3, -(-args.warmup // gs))):
        graph.replay()
    torch.cuda.synchronize()

    # timed region: K steps (K // gs replays of the rotation graph, then the remainder)
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        ev0.record()
        for _ in range(args.steps // gs):
            graph.replay()
        if graph_rem is not None:
            graph_rem.replay()
        ev1.record()
        clocks.mark()
        torch.cuda.synchronize()
    barrier()
    ms = replicas.max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)

    # dominant kernel: average launch duration with events recorded around it by the library
    name, src, work, bound, launch = run.dominant()
    reps = max(1, args.profile_reps)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:          # torch creates the CUDA event on first record
        a.record()
        b.record()
    torch.cuda.synchronize()
    for i in range(reps):
        a, b = evs[i]
        assert lib.csa_profile_next_call(a.cuda_event, b.cuda_event) == 0
        launch()
    torch.cuda.synchronize()
    kms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    pk, pk_kind = peaks()
    if bound == "hbm":
        achieved = work / (kms * 1e-3) / 1e9
        peak = pk["hbm_gbs"]
        unit = "GB/s"
    else:
        achieved = work / (kms * 1e-3) / 1e12
        peak = pk["bf16_tflops"]
        unit = "TFLOP/s"
    traffic = profile_traffic(name, src, args.workload)
    roofline = {"kernel": name, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "peak_source": f"{pk_kind} ({'hbm_gbs' if bound == 'hbm' else 'bf16_tflops'})",
                "traffic": traffic, "algorithmic_per_launch": work, "launch_ms": kms}

    if args.breakdown and rank == 0:
        # each library call of the step captured alone (20 back-to-back calls per graph), so
        # the events bracket device work only
        for name_, fn_ in run.parts():
            g_ = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_):
                for _ in range(20):
                    fn_()
            g_.replay()
            torch.cuda.synchronize()
            ts = []
            for _ in range(10):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                g_.replay()
                b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b) * 1e3 / 20)
            ts.sort()
            print(f"breakdown {name_:20s} median {ts[5]:8.1f} us  min {ts[0]:8.1f} us (graph, L2 warm)",
                  file=sys.stderr)
            del g_

    # end to end through the public API: every step copies its inputs from pinned host memory, runs the
    # library calls and copies the outputs back; the sequence is captured once in a CUDA graph (as a
    # serving loop would, steps double-buffered so one step's copies overlap the other's compute)
    # and replayed, so the copies sit inside the timed region of every step
    e2e = None
    if not args.no_e2e:
        k2 = max(10, min(args.steps // 10, 500))
        side2 = torch.cuda.Stream()
        side2.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side2):
            for _ in range(3):
                run.e2e_step()
        torch.cuda.current_stream().wait_stream(side2)
        torch.cuda.synchronize()
        per_graph = 1
        if hasattr(run, "e2e_pipeline"):
            per_graph = 8
            g_e2e = run.e2e_pipeline(per_graph)
        else:
            g_e2e = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_e2e):
                run.e2e_step()
        for _ in range(3):
            g_e2e.replay()
        torch.cuda.synchronize()
        barrier()
        reps = max(1, k2 // per_graph)
        k2 = reps * per_graph
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g_e2e.replay()
        e1.record()
        torch.cuda.synchronize()
        barrier()
        del g_e2e
        ems = replicas.max_over_ranks(e0.elapsed_time(e1) / k2, dev)
        bi, bo = run.e2e_bytes()
        e2e = {"value": run.tokens * world / (ems * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": ems, "steps": k2}

    extra = None
    if rank == 0 and world == 1 and not args.no_extras:
        extra = extras(dev, pk)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, spent, sample = run.oracle_sample(args.cpu_sample_s)
        cpu = {"value": n / spent, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle", "sample": sample,
               "host_cpus": os.cpu_count(), "seconds": spent}

    if rank == 0:
        line = {"metric": METRIC, "value": run.tokens * world / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": run.describe(world), "roofline": roofline, "step_roofline": run.step_roofline(ms, pk),
                "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps, "clocks": clocks.summary(),
                "self_check": check, "extras": extra, "library": csa.version()}
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
