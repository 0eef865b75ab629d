#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill_2k|prefill_16k|decode_uniform|decode_shared_prefix]

A step is one call of the entry point on one batch of the workload:
  prefill_2k           attn_fwd, bf16 causal, B=4 H=16 N=2048 d=128   (default)
  prefill_16k          attn_fwd, bf16 causal, B=1 H=32 N=16384 d=128 (x0.5)
  decode_uniform       paged_attn_decode, 64 seqs, H=32, bs=16, L~U[128,4096]
  decode_shared_prefix paged_attn_decode, 256 seqs, bs=32, 8-seq shared 512-token prefix
  decode_gqa_g4/_g8    paged_attn_decode_gqa, decode_uniform with 32 query heads over 8 / 4 K/V heads
  kv_append            paged_kv_append, 64 seqs x 512 new tokens (H=32, d=128, bs=16)
  block_copy           paged_block_copy, 1024 block pairs (copy-on-write), 128 KiB per block
  prefill_fp8_2k / _16k the prefill workloads through the FP8 path: attn_quantize_fp8 of Q and K
                       (incoherent processing on) + attn_fwd_fp8 (e4m3 QK^T, bf16 P.V)
  prefill_paged_chunked paged_attn_prefill, 8 seqs x 2048 new tokens after U{0..6144} cached,
                       32 query heads over 8 K/V heads, d=128, bs=16
The default line reports prefill_2k TFLOP/s and carries, measured the same
way in the same run, the other workloads of the path under their own keys:
"decode" (decode_uniform), "prefill_16k" and "decode_shared_prefix", each
with its roofline, timing statistics, clocks, e2e and cpu_baseline.

Rates use algorithmic work: prefill FLOPs = 4 * B * H * d * (visible query-key
pairs) (causal: N(N+1)/2 per head); decode bytes = K/V bytes the sequences
attend over (sum_s L_s * 2 * H * d * 2; for the shared-prefix workload the
unique physical bytes, logical bytes reported beside).

Timing: W untimed warm-up steps; the K steps are captured once in a CUDA
graph; after an untimed soak the graph is replayed back to back, each replay
(exactly K steps) between its own CUDA events on the launching stream, until
the timed region lasts at least --region-s seconds (1 s), the region
bracketed by barrier + cuda.synchronize.  value = work of all timed steps /
region time; timing_stats gives the median per-step time over the replays
and its spread; the clocks are the nvidia-smi samples taken inside the
region.  The roofline divides the dominant kernel's mean launch time into
its algorithmic work, against the measured burst peak (tensor-bound) or the
measured copy bandwidth (HBM-bound).  --eager times K separate calls
instead.  Inputs rotate over copies whose total exceeds L2 (prefill) or
exceed it alone (decode pools of GB).  Multi-GPU (torchrun): every rank runs
its own replica (independent problems, weak scaling, no collective on the
data path); the time is the max over ranks.  Only rank 0 prints the JSON
line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "prefill attn TFLOP/s & paged-decode KV GB/s, as % of B200 roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal B200 figures, reported beside the measured-peak fractions
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


# ---------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, ws: int) -> float:
    """Max of a per-rank float over all ranks (identity at world size 1)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms from the
    warm-up through the timed region (the soak keeps the GPU loaded for a
    while first, so short timed regions still have loaded samples)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.25)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        """Median SM clock and the throttle reasons seen between t0 and t1
        (perf_counter seconds; default: every sample)."""
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, line in self.lines:
            if (t0 is not None and t < t0) or (t1 is not None and t > t1 + 0.15):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


KERNEL_SOURCES = {"prefill_bf16_kernel": ("prefill_sm100.cu", "softmax_math.cuh", "ptx.cuh", "launch.h"),
                  "decode_split_kernel": ("decode_paged.cu", "ptx.cuh", "launch.h"),
                  "decode_mma_kernel": ("decode_paged.cu", "ptx.cuh", "launch.h"),
                  "kv_append_kernel": ("kv_cache_ops.cu", "ptx.cuh", "launch.h"),
                  "block_copy_kernel": ("kv_cache_ops.cu", "ptx.cuh", "launch.h")}


def _code_only(text: str) -> str:
    """C/C++ source without comments, trailing blanks or empty lines (string
    and character literals kept as written)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (line.rstrip() for line in "".join(out).split("\n"))
    return "\n".join(line for line in lines if line)


def kernel_sources_hash(kernel: str) -> str:
    """Hash of the code (comments and blank lines left out) of the source
    files a kernel is built from: profiler counters are only reported while
    it is unchanged."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "online_softmax_paged_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, only while the
    kernel sources are unchanged since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kernel}:{workload}")
    if not e or e.get("sources") != kernel_sources_hash(kernel):
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------- workloads

def pipelined_e2e(device, steps, upload, call, download, nbuf=2):
    """End-to-end time per step through the library's public calls.  Step k
    copies its inputs from pinned host memory into device buffer set
    b = k % nbuf (upload(b), on a stream of its own), runs the library call
    on them (call(b), on the current stream) and copies its result back into
    pinned host memory (download(b), on a third stream), so that step k+1's
    upload overlaps step k's call and download, as a server streaming
    requests would.  Events order the reuse of each buffer set: an upload
    waits for the download of the step that last used its set (which itself
    waited for that step's call).  Two untimed steps, then `steps` steps
    between CUDA events; returns ms per step."""
    cur = torch.cuda.current_stream(device)
    up, dn = torch.cuda.Stream(device), torch.cuda.Stream(device)
    freed = [None] * nbuf

    def run(k):
        b = k % nbuf
        if freed[b] is not None:
            up.wait_event(freed[b])
        with torch.cuda.stream(up):
            upload(b)
        e_up = torch.cuda.Event()
        e_up.record(up)
        cur.wait_event(e_up)
        call(b)
        e_call = torch.cuda.Event()
        e_call.record(cur)
        dn.wait_event(e_call)
        with torch.cuda.stream(dn):
            download(b)
        e_dn = torch.cuda.Event()
        e_dn.record(dn)
        freed[b] = e_dn

    for k in range(2):
        run(k)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(up)
    for k in range(steps):
        run(k)
    cur.wait_stream(dn)
    e1.record(cur)
    torch.cuda.synchronize(device)
    return e0.elapsed_time(e1) / steps


class Prefill:
    def __init__(self, cfg, name, device, seed=0):
        self.name = name
        self.cfg = cfg
        self.B, self.H, self.N, self.d = cfg["B"], cfg["H"], cfg["N"], cfg["d"]
        self.causal = cfg["causal"]
        one = 3 * self.B * self.H * self.N * self.d * 2
        self.copies = max(1, math.ceil(3 * L2_BYTES / one))
        self.sets = [W.dense_inputs(self.B, self.H, self.N, self.d, dtype=cfg["dtype"], mult=cfg["mult"],
                                    seed=seed + i, device=device, causal=self.causal) for i in range(self.copies)]
        self.O = torch.empty_like(self.sets[0]["Q"])
        self.LSE = torch.empty((self.B, self.H, self.N), dtype=torch.float32, device=device)
        pairs = self.N * (self.N + 1) // 2 if self.causal else self.N * self.N
        self.work = 4.0 * self.B * self.H * self.d * pairs  # FLOP per step
        self.unit, self.scale_unit = "TFLOP/s", 1e12
        self.launches_per_step = 1
        self.kernel = "prefill_bf16_kernel"

    def step(self, i, osp):
        s = self.sets[i % self.copies]
        osp.attn_fwd(s["Q"], s["K"], s["V"], O=self.O, LSE=self.LSE, causal=self.causal, scale=s["scale"])

    def config(self):
        return {"workload": self.name, "B": self.B, "H": self.H, "N": self.N, "d": self.d,
                "causal": self.causal, "dtype": "bf16", "global_batch": self.B, "seq_len": self.N,
                "l2": f"inputs rotate over {self.copies} copies ({self.copies * 3 * self.B * self.H * self.N * self.d * 2 / 2**20:.0f} MiB > L2)"}

    def e2e(self, osp, steps, device):
        s = self.sets[0]
        hq, hk, hv = (s[k].cpu().pin_memory() for k in ("Q", "K", "V"))
        ho = [torch.empty_like(hq).pin_memory() for _ in range(2)]
        hl = [torch.empty(self.LSE.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        dev = [(torch.empty_like(s["Q"]), torch.empty_like(s["K"]), torch.empty_like(s["V"]),
                torch.empty_like(self.O), torch.empty_like(self.LSE)) for _ in range(2)]

        def upload(b):
            dq, dk, dv = dev[b][:3]
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)

        def call(b):
            dq, dk, dv, o, lse = dev[b]
            osp.attn_fwd(dq, dk, dv, O=o, LSE=lse, causal=self.causal, scale=s["scale"])

        def download(b):
            ho[b].copy_(dev[b][3], non_blocking=True)
            hl[b].copy_(dev[b][4], non_blocking=True)

        ms = pipelined_e2e(device, steps, upload, call, download)
        h2d = 3 * hq.numel() * hq.element_size()
        d2h = ho[0].numel() * ho[0].element_size() + hl[0].numel() * 4
        return ms, h2d, d2h

    def cpu_sample(self, budget_s):
        """The oracle on whole heads, one after another, until the budget."""
        import numpy as np
        import oracle
        s = self.sets[0]
        done, t0 = 0, time.perf_counter()
        heads = [(b, h) for b in range(self.B) for h in range(self.H)]
        for b, h in heads:
            q, k, v = (s[x][b, h].float().cpu().numpy().astype(np.float64) for x in ("Q", "K", "V"))
            oracle.attention_head(q, k, v, self.causal, s["scale"])
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        return self.work * done / len(heads), dt, f"{done} of {len(heads)} (b, h) heads of {self.name}, full rows"


class Decode:
    def __init__(self, name, device, seed=0):
        self.name = name
        if name == "decode_uniform":
            self.p = W.paged_uniform(device=device, seed=seed, **W.DECODE_UNIFORM)
        elif name in ("decode_gqa_g4", "decode_gqa_g8"):
            # the uniform decode workload with 32 query heads over 8 (or 4)
            # key/value heads: grouped-query attention
            Hkv = 8 if name == "decode_gqa_g4" else 4
            base = W.paged_uniform(device=device, seed=seed, **{**W.DECODE_UNIFORM, "H": Hkv})
            g = torch.Generator(device=device)
            g.manual_seed(seed + 1)
            q = torch.randn((base.num_seqs, 32, base.d), generator=g, device=device).to(torch.bfloat16)
            self.p = W.PagedInputs(q, base.k_cache, base.v_cache, base.block_table, base.seq_lens,
                                   base.block_size, base.scale)
        elif name == "decode_shared_prefix_small":
            # 48 sequences (6 groups) of the shared-prefix workload in a
            # 2400-block pool (1.3 GB of K/V, above L2): the case profiler
            # captures run on
            self.p = W.paged_shared_prefix(device=device, seed=seed, **{**W.DECODE_SHARED_PREFIX, "num_seqs": 48,
                                                                         "pool": 2400})
        elif name == "decode_uniform_small":
            # 16 sequences of the uniform workload in a 4000-block pool (1 GiB
            # of K/V, still above L2): the case profiler captures run on
            self.p = W.paged_uniform(device=device, seed=seed, **{**W.DECODE_UNIFORM, "num_seqs": 16,
                                                                   "pool": 4000})
        else:
            self.p = W.paged_shared_prefix(device=device, seed=seed, **W.DECODE_SHARED_PREFIX)
        self.gqa = self.p.k_cache.shape[1] != self.p.q.shape[1]
        kv = W.PagedInputs(self.p.q[:, :self.p.k_cache.shape[1]], self.p.k_cache, self.p.v_cache,
                           self.p.block_table, self.p.seq_lens, self.p.block_size, self.p.scale)
        self.logical = W.logical_kv_bytes(kv)   # K/V bytes of the key/value heads attended
        self.unique = W.unique_kv_bytes(kv)
        self.work = float(self.unique if name.startswith("decode_shared_prefix") else self.logical)  # bytes per step
        self.O = torch.empty_like(self.p.q)
        self.LSE = torch.empty(self.p.q.shape[:2], dtype=torch.float32, device=device)
        import online_softmax_paged_b200 as osp
        n = osp.paged_attn_decode_gqa_workspace_size(self.p.num_seqs, self.p.H, self.p.k_cache.shape[1], self.p.d,
                                                     self.p.max_blocks_per_seq, self.p.block_size)
        self.ws = torch.empty(n, dtype=torch.uint8, device=device)
        self.ws_bytes = n
        self.unit, self.scale_unit = "GB/s", 1e9
        # timed as a whole call (the events wrap every kernel of it); groups of
        # 4 and 8 run the tensor-core variant and a merge kernel after it
        G = self.p.q.shape[1] // self.p.k_cache.shape[1]
        self.kernel = "decode_mma_kernel" if G >= 4 else "decode_split_kernel"
        # (groups of 4 and more plan inside their kernel up to 4096 sequences:
        # that kernel and the merge; otherwise the plan kernel and one more)
        self.launches_per_step = 2 + (1 if G >= 4 and self.p.num_seqs > 4096 else 0)

    def step(self, i, osp):
        p = self.p
        fn = osp.paged_attn_decode_gqa if self.gqa else osp.paged_attn_decode
        fn(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.block_size, O=self.O, LSE=self.LSE,
           scale=p.scale, workspace=self.ws)

    def config(self):
        p = self.p
        c = {"workload": self.name, "num_seqs": p.num_seqs, "H": p.H, "H_kv": int(p.k_cache.shape[1]), "d": p.d,
             "block_size": p.block_size,
             "pool_blocks": p.num_blocks, "dtype": "bf16", "global_batch": p.num_seqs,
             "seq_len": int(p.seq_lens.max().item()), "kv_bytes_logical": self.logical,
             "kv_bytes_unique": self.unique,
             "l2": f"KV pool {2 * p.k_cache.numel() * 2 / 2**30:.1f} GiB > L2"}
        return c

    def e2e(self, osp, steps, device):
        p = self.p
        hq = p.q.cpu().pin_memory()
        ht = p.block_table.cpu().pin_memory()
        hs = p.seq_lens.cpu().pin_memory()
        ho = [torch.empty_like(hq).pin_memory() for _ in range(2)]
        hl = [torch.empty(self.LSE.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        dev = [(torch.empty_like(p.q), torch.empty_like(p.block_table), torch.empty_like(p.seq_lens),
                torch.empty_like(self.O), torch.empty_like(self.LSE)) for _ in range(2)]
        fn = osp.paged_attn_decode_gqa if self.gqa else osp.paged_attn_decode

        def upload(b):
            dq, dt, ds = dev[b][:3]
            dq.copy_(hq, non_blocking=True)
            dt.copy_(ht, non_blocking=True)
            ds.copy_(hs, non_blocking=True)

        def call(b):
            # calls run one after another on one stream, so they share the workspace
            dq, dt, ds, o, lse = dev[b]
            fn(dq, p.k_cache, p.v_cache, dt, ds, p.block_size, O=o, LSE=lse, scale=p.scale, workspace=self.ws)

        def download(b):
            ho[b].copy_(dev[b][3], non_blocking=True)
            hl[b].copy_(dev[b][4], non_blocking=True)

        ms = pipelined_e2e(device, steps, upload, call, download)
        h2d = hq.numel() * 2 + ht.numel() * 4 + hs.numel() * 4
        d2h = ho[0].numel() * 2 + hl[0].numel() * 4
        return ms, h2d, d2h

    def cpu_sample(self, budget_s):
        import numpy as np
        import oracle
        p = self.p
        sl = p.seq_lens.cpu().numpy()
        bt = p.block_table.cpu().numpy()
        q = p.q.float().cpu().numpy().astype(np.float64)

        class Lazy:
            def __init__(self, t):
                self.t, self.shape = t, tuple(t.shape)

            def __getitem__(self, i):
                return self.t[int(i)].float().cpu().numpy()

        kc, vc = Lazy(p.k_cache), Lazy(p.v_cache)
        done_bytes, n, t0 = 0, 0, time.perf_counter()
        for s in range(p.num_seqs):
            oracle.paged_decode(q, kc, vc, bt, sl, p.block_size, p.scale, seqs=[s])
            done_bytes += int(sl[s]) * 2 * p.H * p.d * 2
            n += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        return float(done_bytes), dt, f"{n} of {p.num_seqs} sequences of {self.name} (all heads)"


class KVAppend:
    """paged_kv_append of a prefill chunk: 64 sequences x 512 new tokens
    (H=32, d=128, bs=16) written into fresh blocks drawn from a 20000-block
    pool.  Work = bytes read + written (the copy-bandwidth convention)."""

    def __init__(self, name, device, seed=0):
        self.name = name
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        S, T, H, d, bs, pool = 64, 512, 32, 128, 16, 20000
        self.k_cache = torch.zeros((pool, H, bs, d), dtype=torch.bfloat16, device=device)
        self.v_cache = torch.zeros_like(self.k_cache)
        mb = T // bs
        self.table = torch.randperm(pool, generator=g, device=device)[:S * mb].view(S, mb).to(torch.int32).contiguous()
        self.seq_ids = torch.arange(S, device=device, dtype=torch.int32).repeat_interleave(T).contiguous()
        self.positions = torch.arange(T, device=device, dtype=torch.int32).repeat(S).contiguous()
        self.k_new = torch.randn((S * T, H, d), generator=g, device=device).to(torch.bfloat16)
        self.v_new = torch.randn((S * T, H, d), generator=g, device=device).to(torch.bfloat16)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.work = float(2 * 2 * self.k_new.numel() * 2)  # K and V, read and written
        self.unit, self.scale_unit = "GB/s", 1e9
        self.launches_per_step = 1
        self.kernel = "kv_append_kernel"
        self.cfg = dict(num_seqs=S, new_tokens_per_seq=T, H=H, d=d, block_size=bs, pool_blocks=pool)

    def step(self, i, osp):
        osp.paged_kv_append(self.k_new, self.v_new, self.seq_ids, self.positions, self.table, self.k_cache,
                            self.v_cache, err_flag=self.err)

    def config(self):
        return {"workload": self.name, **self.cfg, "dtype": "bf16", "global_batch": self.cfg["num_seqs"],
                "seq_len": self.cfg["new_tokens_per_seq"], "bytes_per_step": int(self.work),
                "l2": "2.1 GiB of new K/V per step > L2"}

    def e2e(self, osp, steps, device):
        hk, hv = self.k_new.cpu().pin_memory(), self.v_new.cpu().pin_memory()
        he = [torch.zeros(1, dtype=torch.int32).pin_memory() for _ in range(2)]
        dev = [(torch.empty_like(self.k_new), torch.empty_like(self.v_new), torch.zeros_like(self.err))
               for _ in range(2)]

        def upload(b):
            dev[b][0].copy_(hk, non_blocking=True)
            dev[b][1].copy_(hv, non_blocking=True)

        def call(b):
            dk, dv, err = dev[b]
            osp.paged_kv_append(dk, dv, self.seq_ids, self.positions, self.table, self.k_cache, self.v_cache,
                                err_flag=err)

        def download(b):
            he[b].copy_(dev[b][2], non_blocking=True)

        ms = pipelined_e2e(device, steps, upload, call, download)
        return ms, 2 * hk.numel() * 2, 4

    def cpu_sample(self, budget_s):
        import numpy as np
        import oracle
        S = self.cfg["num_seqs"]
        T = self.cfg["new_tokens_per_seq"]
        n = 4 * T  # four sequences' tokens
        t0 = time.perf_counter()
        kc = np.zeros((self.table[:4].numel() + 1, 32, 16, 128))
        tbl = torch.arange(4 * (T // 16), dtype=torch.int32).view(4, T // 16).numpy()
        oracle.kv_append(kc, kc, tbl, self.k_new[:n].float().cpu().numpy(), self.v_new[:n].float().cpu().numpy(),
                         self.seq_ids[:n].cpu().numpy(), self.positions[:n].cpu().numpy(), 16)
        dt = time.perf_counter() - t0
        return self.work * n / (S * T), dt, f"4 of {S} sequences' tokens"


class BlockCopy:
    """paged_block_copy of 1024 (src, dst) pairs in a 20000-block pool
    (H=32, d=128, bs=16: 128 KiB per block per cache).  Work = bytes read +
    written."""

    def __init__(self, name, device, seed=0):
        self.name = name
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        pool, H, bs, d, n = 20000, 32, 16, 128, 1024
        self.k_cache = torch.randn((pool, H, bs, d), generator=g, device=device).to(torch.bfloat16)
        self.v_cache = torch.randn((pool, H, bs, d), generator=g, device=device).to(torch.bfloat16)
        perm = torch.randperm(pool, generator=g, device=device).to(torch.int32)
        self.src, self.dst = perm[:n].contiguous(), perm[n:2 * n].contiguous()
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.work = float(n * 2 * H * bs * d * 2 * 2)
        self.unit, self.scale_unit = "GB/s", 1e9
        self.launches_per_step = 1
        self.kernel = "block_copy_kernel"
        self.cfg = dict(pairs=n, H=H, d=d, block_size=bs, pool_blocks=pool)

    def step(self, i, osp):
        osp.paged_block_copy(self.k_cache, self.v_cache, self.src, self.dst, err_flag=self.err)

    def config(self):
        return {"workload": self.name, **self.cfg, "dtype": "bf16", "global_batch": self.cfg["pairs"],
                "seq_len": self.cfg["block_size"], "bytes_per_step": int(self.work),
                "l2": "268 MiB read per step > L2"}

    def e2e(self, osp, steps, device):
        hs, hd = self.src.cpu().pin_memory(), self.dst.cpu().pin_memory()
        he = [torch.zeros(1, dtype=torch.int32).pin_memory() for _ in range(2)]
        dev = [(torch.empty_like(self.src), torch.empty_like(self.dst), torch.zeros_like(self.err))
               for _ in range(2)]

        def upload(b):
            dev[b][0].copy_(hs, non_blocking=True)
            dev[b][1].copy_(hd, non_blocking=True)

        def call(b):
            ds, dd, err = dev[b]
            osp.paged_block_copy(self.k_cache, self.v_cache, ds, dd, err_flag=err)

        def download(b):
            he[b].copy_(dev[b][2], non_blocking=True)

        ms = pipelined_e2e(device, steps, upload, call, download)
        return ms, 2 * hs.numel() * 4, 4

    def cpu_sample(self, budget_s):
        import oracle
        n = 16
        kc = self.k_cache[:0]
        src = self.src[:n].cpu().numpy()
        dst = self.dst[:n].cpu().numpy()
        idx = sorted(set(src.tolist()) | set(dst.tolist()))
        remap = {b: i for i, b in enumerate(idx)}
        sub_k = self.k_cache[idx].float().cpu().numpy()
        sub_v = self.v_cache[idx].float().cpu().numpy()
        t0 = time.perf_counter()
        oracle.block_copy(sub_k, sub_v, [remap[b] for b in src], [remap[b] for b in dst])
        dt = time.perf_counter() - t0
        return self.work * n / self.cfg["pairs"], dt, f"{n} of {self.cfg['pairs']} pairs"


class Fp8Prefill:
    """The causal prefill workloads through the FP8 path: one step =
    attn_quantize_fp8(Q), attn_quantize_fp8(K) (random-sign Hadamard
    incoherent processing), attn_fwd_fp8.  Work = the bf16 prefill's FLOPs.
    The roofline is that of the attention kernel alone, timed with its own
    events; its peak blends the two contractions: QK^T at the e4m3 rate
    (2x bf16, the nominal ratio) and P.V at the bf16 rate, i.e. a time at
    peak of 0.75 x that of an all-bf16 kernel."""

    def __init__(self, cfg, name, device, seed=0):
        self.name = name
        self.cfg = cfg
        self.B, self.H, self.N, self.d = cfg["B"], cfg["H"], cfg["N"], cfg["d"]
        one = 3 * self.B * self.H * self.N * self.d * 2
        self.copies = max(1, math.ceil(3 * L2_BYTES / one))
        self.sets = [W.dense_inputs(self.B, self.H, self.N, self.d, dtype=cfg["dtype"], mult=cfg["mult"],
                                    seed=seed + i, device=device, causal=True) for i in range(self.copies)]
        self.signs = W.hadamard_signs(self.d, seed=seed, device=device)
        nblk = -(-self.N // 128)
        shp = (self.B, self.H, self.N, self.d)
        self.q8 = torch.empty(shp, dtype=torch.uint8, device=device)
        self.k8 = torch.empty(shp, dtype=torch.uint8, device=device)
        self.qs = torch.empty((self.B, self.H, nblk), dtype=torch.float32, device=device)
        self.ks = torch.empty((self.B, self.H, nblk), dtype=torch.float32, device=device)
        self.O = torch.empty(shp, dtype=torch.bfloat16, device=device)
        self.LSE = torch.empty((self.B, self.H, self.N), dtype=torch.float32, device=device)
        self.work = 4.0 * self.B * self.H * self.d * (self.N * (self.N + 1) // 2)
        self.unit, self.scale_unit = "TFLOP/s", 1e12
        self.launches_per_step = 3
        self.kernel = "prefill_bf16_kernel"
        self.peak_factor = 1.0 / 0.75
        self.kernel_events = []
        self.record = False

    def step(self, i, osp):
        s = self.sets[i % self.copies]
        osp.attn_quantize_fp8(s["Q"], signs=self.signs, codes=self.q8, scales=self.qs)
        osp.attn_quantize_fp8(s["K"], signs=self.signs, codes=self.k8, scales=self.ks)
        if self.record:
            st = torch.cuda.current_stream()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
        osp.attn_fwd_fp8(self.q8, self.qs, self.k8, self.ks, s["V"], O=self.O, LSE=self.LSE, causal=True,
                         scale=s["scale"])
        if self.record:
            e1.record(st)
            self.kernel_events.append((e0, e1))

    def dominant(self, i, osp):
        """The attention launch alone (on the codes the last quantisation left)."""
        s = self.sets[i % self.copies]
        osp.attn_fwd_fp8(self.q8, self.qs, self.k8, self.ks, s["V"], O=self.O, LSE=self.LSE, causal=True,
                         scale=s["scale"])

    def config(self):
        return {"workload": self.name, "B": self.B, "H": self.H, "N": self.N, "d": self.d, "causal": True,
                "dtype": "e4m3 Q/K, bf16 V/P/O", "global_batch": self.B, "seq_len": self.N,
                "incoherent_processing": True,
                "l2": f"inputs rotate over {self.copies} copies "
                      f"({self.copies * 3 * self.B * self.H * self.N * self.d * 2 / 2**20:.0f} MiB > L2)"}

    def e2e(self, osp, steps, device):
        s = self.sets[0]
        hq, hk, hv = (s[k].cpu().pin_memory() for k in ("Q", "K", "V"))
        ho = [torch.empty_like(hq).pin_memory() for _ in range(2)]
        hl = [torch.empty(self.LSE.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        dev = [(torch.empty_like(s["Q"]), torch.empty_like(s["K"]), torch.empty_like(s["V"]),
                torch.empty_like(self.O), torch.empty_like(self.LSE)) for _ in range(2)]

        def upload(b):
            dq, dk, dv = dev[b][:3]
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)

        def call(b):
            # quantisation buffers are shared: the calls run one after another on one stream
            dq, dk, dv, o, lse = dev[b]
            osp.attn_quantize_fp8(dq, signs=self.signs, codes=self.q8, scales=self.qs)
            osp.attn_quantize_fp8(dk, signs=self.signs, codes=self.k8, scales=self.ks)
            osp.attn_fwd_fp8(self.q8, self.qs, self.k8, self.ks, dv, O=o, LSE=lse, causal=True, scale=s["scale"])

        def download(b):
            ho[b].copy_(dev[b][3], non_blocking=True)
            hl[b].copy_(dev[b][4], non_blocking=True)

        ms = pipelined_e2e(device, steps, upload, call, download)
        return ms, 3 * hq.numel() * 2, ho[0].numel() * 2 + hl[0].numel() * 4

    def cpu_sample(self, budget_s):
        """The oracle's quantisation of one (b, h) head's Q and K and exact
        attention on the dequantised operands, head after head, until the budget."""
        import numpy as np
        import oracle
        from oracle import fp8 as F
        s = self.sets[0]
        sg = self.signs.cpu().numpy()
        done, t0 = 0, time.perf_counter()
        heads = [(b, h) for b in range(self.B) for h in range(self.H)]
        for b, h in heads:
            q = F.dequantize_blocks(*F.quantize_blocks(s["Q"][b, h].float().cpu().numpy()[None], 128, signs=sg))[0]
            k = F.dequantize_blocks(*F.quantize_blocks(s["K"][b, h].float().cpu().numpy()[None], 128, signs=sg))[0]
            v = s["V"][b, h].float().cpu().numpy().astype(np.float64)
            oracle.attention_head(q, k, v, True, s["scale"])
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        return self.work * done / len(heads), dt, f"{done} of {len(heads)} (b, h) heads of {self.name}, full rows"


class PagedPrefill:
    """paged_attn_prefill on the chunked-prefill workload.  Work = 4 * d *
    H_q * (visible query-key pairs), new token i of sequence s seeing
    ctx_s + i + 1 keys."""

    def __init__(self, name, device, seed=0):
        self.name = name
        self.cfg = dict(W.PREFILL_PAGED_CHUNKED)
        self.copies = 2
        self.sets = [W.paged_chunked_prefill(device=device, seed=seed + 10 * i, **self.cfg)
                     for i in range(self.copies)]
        p = self.sets[0]
        self.O = torch.empty_like(p.q)
        self.LSE = torch.empty(p.q.shape[:2], dtype=torch.float32, device=device)
        self.max_q = self.cfg["chunk"]
        d, Hq = self.cfg["d"], self.cfg["Hq"]
        pairs = []
        for q in self.sets:
            sl, n = q.seq_lens.cpu().tolist(), q.n_new.tolist()
            pairs.append(sum(nn * (L - nn) + nn * (nn + 1) // 2 for L, nn in zip(sl, n)))
        self.work_per_set = [4.0 * d * Hq * x for x in pairs]
        self.work = statistics.mean(self.work_per_set)
        self.unit, self.scale_unit = "TFLOP/s", 1e12
        self.launches_per_step = 1
        self.kernel = "prefill_bf16_kernel"

    def step(self, i, osp):
        p = self.sets[i % self.copies]
        osp.paged_attn_prefill(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.cu_q, p.block_size,
                               max_q_per_seq=self.max_q, O=self.O, LSE=self.LSE, scale=p.scale)

    def config(self):
        c = self.cfg
        return {"workload": self.name, **c, "dtype": "bf16", "global_batch": c["num_seqs"], "seq_len": c["chunk"],
                "flop_per_step": self.work,
                "l2": f"inputs rotate over {self.copies} sets; K/V read per step ~{self._kv_mib():.0f} MiB > L2"}

    def _kv_mib(self):
        p = self.sets[0]
        return float(p.seq_lens.sum()) * 2 * self.cfg["Hkv"] * self.cfg["d"] * 2 / 2**20

    def e2e(self, osp, steps, device):
        p = self.sets[0]
        hq = p.q.cpu().pin_memory()
        meta = [t.cpu().pin_memory() for t in (p.block_table, p.seq_lens, p.cu_q)]
        ho = [torch.empty_like(hq).pin_memory() for _ in range(2)]
        hl = [torch.empty(self.LSE.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        dev = [(torch.empty_like(p.q), [torch.empty_like(t) for t in (p.block_table, p.seq_lens, p.cu_q)],
                torch.empty_like(self.O), torch.empty_like(self.LSE)) for _ in range(2)]

        def upload(b):
            dev[b][0].copy_(hq, non_blocking=True)
            for d_, h_ in zip(dev[b][1], meta):
                d_.copy_(h_, non_blocking=True)

        def call(b):
            dq, dmeta, o, lse = dev[b]
            osp.paged_attn_prefill(dq, p.k_cache, p.v_cache, dmeta[0], dmeta[1], dmeta[2], p.block_size,
                                   max_q_per_seq=self.max_q, O=o, LSE=lse, scale=p.scale)

        def download(b):
            ho[b].copy_(dev[b][2], non_blocking=True)
            hl[b].copy_(dev[b][3], non_blocking=True)

        ms = pipelined_e2e(device, steps, upload, call, download)
        h2d = hq.numel() * 2 + sum(t.numel() * 4 for t in meta)
        d2h = ho[0].numel() * 2 + hl[0].numel() * 4
        return ms * self.work / self.work_per_set[0], h2d, d2h

    def oracle_rows(self, s, h, rows):
        """The oracle on given new-token rows of (sequence s, query head h);
        returns the FLOPs those rows stand for."""
        import numpy as np
        import oracle
        p = self.sets[0]
        L = int(p.seq_lens[s])
        n = int(p.cu_q[s + 1] - p.cu_q[s])
        q0 = int(p.cu_q[s])
        G = self.cfg["Hq"] // self.cfg["Hkv"]

        class Lazy:
            def __init__(self, t):
                self.t, self.shape = t, tuple(t.shape)

            def __getitem__(self, i):
                return self.t[int(i)].double().cpu().numpy()

        tbl = p.block_table[s].cpu().numpy()
        K = oracle.gather_paged(Lazy(p.k_cache), tbl, L, p.block_size)[h // G]
        V = oracle.gather_paged(Lazy(p.v_cache), tbl, L, p.block_size)[h // G]
        work = 0.0
        for i in rows:
            pos = L - n + i
            q = p.q[q0 + i, h:h + 1].double().cpu().numpy()
            oracle.attention_head(q, K[:pos + 1], V[:pos + 1], False, p.scale)
            work += 4.0 * self.cfg["d"] * (pos + 1)
        return work

    def cpu_sample(self, budget_s):
        """The oracle on rows of (sequence 0, head 0), 64 at a time, until the budget."""
        t0 = time.perf_counter()
        work, done = 0.0, 0
        while time.perf_counter() - t0 < budget_s and done < self.cfg["chunk"]:
            work += self.oracle_rows(0, 0, range(done, min(done + 64, self.cfg["chunk"])))
            done = min(done + 64, self.cfg["chunk"])
        dt = time.perf_counter() - t0
        return work, dt, f"new-token rows 0..{done - 1} of sequence 0, query head 0 (K/V gathered per 64 rows)"


def make_workload(name, device, seed=0):
    if name == "prefill_2k":
        return Prefill(W.PREFILL_CAUSAL_2K, name, device, seed)
    if name == "prefill_16k":
        return Prefill(W.PREFILL_CAUSAL_16K, name, device, seed)
    if name in ("decode_uniform", "decode_shared_prefix", "decode_uniform_small", "decode_shared_prefix_small",
                "decode_gqa_g4", "decode_gqa_g8"):
        return Decode(name, device, seed)
    if name == "kv_append":
        return KVAppend(name, device, seed)
    if name == "block_copy":
        return BlockCopy(name, device, seed)
    if name == "prefill_paged_chunked":
        return PagedPrefill(name, device, seed)
    if name == "prefill_fp8_2k":
        return Fp8Prefill(W.PREFILL_CAUSAL_2K, name, device, seed)
    if name == "prefill_fp8_16k":
        return Fp8Prefill(W.PREFILL_CAUSAL_16K, name, device, seed)
    raise SystemExit(f"unknown workload {name}")


# ---------------------------------------------------------------- timing

def _region(graph, replays, st, device, ws):
    """``replays`` back-to-back replays of ``graph`` between barrier +
    synchronize on both sides, a pair of CUDA events around each on the
    launching stream.  Returns (per-replay ms, total ms from the first start
    event to the last end event, (t0, t1) perf_counter span)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(replays)]
    barrier(ws)
    torch.cuda.synchronize(device)
    t0 = time.perf_counter()
    for a, b in evs:
        a.record(st)
        graph.replay()
        b.record(st)
    torch.cuda.synchronize(device)
    barrier(ws)
    t1 = time.perf_counter()
    return [a.elapsed_time(b) for a, b in evs], evs[0][0].elapsed_time(evs[-1][1]), (t0, t1)


def time_steps_graph(wl, osp, steps, warmup, device, ws, soak_s=0.0, region_s=1.0):
    """The K timed steps captured once into a CUDA graph; the graph is
    replayed back to back, each replay (exactly K steps) between its own
    CUDA events, until the timed region lasts at least ``region_s`` seconds
    (every rank replays the same number of times).  Device time only, without
    the host's per-call launch cost (a serving loop replays its decode steps
    the same way).  Steps of several launches whose roofline is one kernel's
    also get a graph of that kernel alone, timed the same way after the
    region.  Returns a dict of the timings."""
    st = torch.cuda.current_stream(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            wl.step(warmup + i, osp)
    gk = None
    if hasattr(wl, "dominant"):
        gk = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gk):
            for i in range(steps):
                wl.dominant(warmup + i, osp)
    g.replay()  # the first replay uploads the graph
    if gk is not None:
        gk.replay()
    torch.cuda.synchronize(device)
    # one replay sizes the region
    one_ms = _region(g, 1, st, device, 1)[1]
    replays = max(3, math.ceil(region_s * 1e3 / max(one_ms, 1e-3))) if region_s > 0 else 1
    replays = int(max_over_ranks(float(replays), ws))
    # the soak replays the same graph right before the timed region, so the
    # region starts at the clocks a loaded GPU settles to (capturing left the
    # GPU idle)
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < soak_s:
        g.replay()
        torch.cuda.synchronize(device)
    rep, total_ms, span = _region(g, replays, st, device, ws)
    out = {"rep_ms": rep, "total_ms": total_ms, "span": span, "replays": replays, "steps": steps,
           "kernel_rep_ms": None, "timing": "graph"}
    if gk is not None:
        out["kernel_rep_ms"] = _region(gk, replays, st, device, ws)[0]
    del g, gk
    return out


def time_steps(wl, osp, steps, warmup, device, ws, soak_s=0.0, graph=False, region_s=1.0):
    """W warm-up steps, then the timed region: with ``graph``, replays of the
    K steps captured in a CUDA graph (time_steps_graph); otherwise K eager
    calls with CUDA events around every launch, after an optional untimed
    soak.  Returns a dict of the timings."""
    st = torch.cuda.current_stream(device)
    for i in range(warmup):
        wl.step(i, osp)
    torch.cuda.synchronize(device)
    if graph:
        try:
            return time_steps_graph(wl, osp, steps, warmup, device, ws, soak_s, region_s)
        except Exception as e:  # capture unsupported here: time eagerly
            print(f"CUDA graph capture failed ({e!r}); timing eagerly", file=sys.stderr)
            torch.cuda.synchronize(device)
    if soak_s > 0:
        t0, i = time.perf_counter(), 0
        while time.perf_counter() - t0 < soak_s:
            for _ in range(8):
                wl.step(i, osp)
                i += 1
            torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(ws)
    torch.cuda.synchronize(device)
    t_region0 = time.perf_counter()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    if hasattr(wl, "kernel_events"):  # steps of several launches time the dominant one too
        wl.kernel_events.clear()
        wl.record = True
    g0.record(st)
    for i in range(steps):
        evs[i][0].record(st)
        wl.step(warmup + i, osp)
        evs[i][1].record(st)
    g1.record(st)
    torch.cuda.synchronize(device)
    barrier(ws)
    span = (t_region0, time.perf_counter())
    per = [a.elapsed_time(b) for a, b in evs]
    kper = None
    if hasattr(wl, "kernel_events"):
        wl.record = False
        kper = [a.elapsed_time(b) for a, b in wl.kernel_events]
    # eager: every step is its own "replay" of one step
    return {"rep_ms": per, "total_ms": g0.elapsed_time(g1), "span": span, "replays": steps, "steps": 1,
            "kernel_rep_ms": kper, "timing": "eager"}


def timing_stats(tm):
    """Per-step statistics of a timed region: the median per-replay time over
    K, its spread, and the mean over the whole region."""
    per = sorted(r / tm["steps"] for r in tm["rep_ms"])
    n = len(per)

    def q(f):
        return per[min(n - 1, max(0, int(round(f * (n - 1)))))]

    med = statistics.median(per)
    return {"replays": tm["replays"], "steps_per_replay": tm["steps"], "steps_timed": tm["replays"] * tm["steps"],
            "region_s": round(tm["span"][1] - tm["span"][0], 3), "timing": tm["timing"],
            "per_step_ms": {"median": round(med, 5), "mean": round(tm["total_ms"] / (tm["replays"] * tm["steps"]), 5),
                            "min": round(per[0], 5), "p10": round(q(0.1), 5), "p90": round(q(0.9), 5),
                            "max": round(per[-1], 5)},
            "spread_p10_p90_pct": round(100.0 * (q(0.9) - q(0.1)) / med, 2) if med > 0 else None}


def roofline(wl, launch_ms, pk, pk_src, bound, clocks=None):
    """Roofline of the dominant kernel from its mean launch time over the
    timed region.  Tensor-bound kernels are compared with the measured burst
    bf16 peak (one fixed denominator, whatever the clocks did); the fraction
    of the measured sustained (power-capped) peak is reported beside it with
    the median SM clock of the region."""
    achieved = wl.work / (launch_ms * 1e-3) / wl.scale_unit
    extra = {}
    if bound == "tensor":
        burst = float(pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        sustained = float(pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        f = getattr(wl, "peak_factor", 1.0)  # FP8 QK^T: the blended e4m3 / bf16 peak
        burst, sustained = burst * f, sustained * f
        peak = burst
        extra = {"peak_kind": "burst bf16 (measured cuBLAS-class matmul)",
                 "frac_of_sustained": round(achieved / sustained, 4), "peak_sustained": round(sustained, 1)}
        if clocks and clocks.get("sm_mhz"):
            extra["sm_mhz_median_in_region"] = clocks["sm_mhz"]
        if f != 1.0:
            extra["peak_kind"] += "; bf16 peak x 4/3 (QK^T at the e4m3 rate, P.V at the bf16 rate)"
        unit = "TFLOP/s"
    else:
        peak = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        unit = "GB/s"
        extra = {"peak_kind": "copy bandwidth (measured)"}
    spec = SPEC_PEAKS["bf16_tflops"] * getattr(wl, "peak_factor", 1.0) if bound == "tensor" else SPEC_PEAKS["hbm_gbs"]
    extra["frac_of_spec"] = round(achieved / spec, 4)
    tr = recorded_traffic(wl.kernel, wl.name)
    return {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": tr, "peak_source": pk_src,
            "kernel": wl.kernel, "launch_ms": round(launch_ms, 5), "work_per_launch": wl.work, **extra}


BAD_CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def measure(wl, osp, args, device, ws, clocks, pk, pk_src, region_s):
    """Time one workload (its timed region re-measured once if the clocks
    sampled inside it show a hardware or thermal slowdown) and return its
    rate, roofline, statistics and clocks."""
    bound = "tensor" if isinstance(wl, (Prefill, PagedPrefill, Fp8Prefill)) else "hbm"
    remeasured = False
    for attempt in range(2):
        tm = time_steps(wl, osp, args.steps, args.warmup if attempt == 0 else 1, device, ws, soak_s=args.soak,
                        graph=not args.eager, region_s=region_s)
        clk = clocks.summary(*tm["span"])
        if not set(clk["reasons"]) & set(BAD_CLOCK_REASONS) or attempt == 1:
            break
        remeasured = True
    n_steps = tm["replays"] * tm["steps"]
    t_max = max_over_ranks(tm["total_ms"], ws)
    work_all = sum_over_ranks(wl.work * n_steps, ws)
    value = work_all / (t_max * 1e-3) / wl.scale_unit
    ms_step = t_max / n_steps
    if tm["kernel_rep_ms"] is not None:  # the dominant kernel timed on its own
        kn = len(tm["kernel_rep_ms"]) * tm["steps"] if tm["timing"] == "graph" else len(tm["kernel_rep_ms"])
        launch_ms = max_over_ranks(sum(tm["kernel_rep_ms"]) / kn, ws)
    else:
        launch_ms = ms_step  # one launch, or a call whose kernels the events wrap together
    stats = timing_stats(tm)
    if clk.get("sm_mhz"):
        stats["kcycles_per_step_at_median_mhz"] = round(ms_step * clk["sm_mhz"], 2)
    clk = {**clk, "window": "timed region only", "remeasured": remeasured,
           "rejected": bool(set(clk["reasons"]) & set(BAD_CLOCK_REASONS))}
    return {"value": value, "ms_per_step": ms_step, "steps_timed": n_steps, "timing": tm["timing"],
            "roofline": roofline(wl, launch_ms, pk, pk_src, bound, clk), "stats": stats, "clocks": clk,
            "gpu_launches": wl.launches_per_step * n_steps}


def cpu_leg(wl, budget_s):
    work, dt, sample = wl.cpu_sample(budget_s)
    return {"value": round(work / dt / wl.scale_unit, 6), "unit": wl.unit, "cores": _cpu_threads(),
            "kind": "oracle", "sample": sample, "seconds": round(dt, 2)}


def e2e_leg(wl, osp, steps, device, ws):
    e2e_ms, h2d, d2h = wl.e2e(osp, steps, device)
    e2e_ms = max_over_ranks(e2e_ms, ws)
    val = sum_over_ranks(wl.work, ws) / (e2e_ms * 1e-3) / wl.scale_unit
    return {"value": round(val, 3), "unit": wl.unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(e2e_ms, 5),
            "pipeline": "each step uploads its inputs from pinned host memory and reads its result back; step k+1's "
                        "upload overlaps step k's call and download (2 device buffer sets, 3 streams)"}


# the other workloads the default line carries, measured the same way in the
# same run: the long causal prefill and the two paged-decode workloads
DEFAULT_LEGS = ("decode_uniform", "prefill_16k", "decode_shared_prefix")


def run_ours(args):
    ws, rank, local = dist_env()
    if ws > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import online_softmax_paged_b200 as osp
    osp.load()
    pk, pk_src = peaks()
    e2e_steps = max(3, min(args.steps, 20))

    wl = make_workload(args.workload, device, seed=args.seed + rank)
    with ClockSampler(local) as clocks:
        m = measure(wl, osp, args, device, ws, clocks, pk, pk_src, args.region_s)
        e2e = e2e_leg(wl, osp, e2e_steps, device, ws)
        cpu = cpu_leg(wl, args.cpu_budget) if rank == 0 and ws == 1 and not args.no_cpu else None
        config = wl.config()
        del wl
        legs = {}
        if args.workload == "prefill_2k" and not args.no_decode:
            for name in DEFAULT_LEGS:
                torch.cuda.empty_cache()
                lw = make_workload(name, device, seed=args.seed + rank)
                lm = measure(lw, osp, args, device, ws, clocks, pk, pk_src, args.region_s)
                leg = {"workload": name, "value": round(lm["value"], 3), "unit": lw.unit,
                       "ms_per_step": round(lm["ms_per_step"], 5), "steps": args.steps,
                       "roofline": lm["roofline"], "timing_stats": lm["stats"], "clocks": lm["clocks"],
                       "e2e": e2e_leg(lw, osp, min(e2e_steps, 5), device, ws),
                       "cpu_baseline": (cpu_leg(lw, args.cpu_budget) if rank == 0 and ws == 1 and not args.no_cpu
                                        else None),
                       "config": {**lw.config(), "timing": lm["timing"]}, "gpu_launches": lm["gpu_launches"]}
                legs[name] = leg
                del lw
        # the first leg keeps its historical key
        extra = {("decode" if k == "decode_uniform" else k): v for k, v in legs.items()}

    if rank == 0:
        line = {"metric": METRIC, "value": round(m["value"], 3), "unit": m["roofline"]["unit"], "n_gpus": ws,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(m["ms_per_step"], 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "e4m3+bf16" if args.workload.startswith("prefill_fp8") else "bf16",
                "data": "synthetic (seeded N(0,1), bf16)",
                "config": {**config, "parallelism": f"replicas{ws}" if ws > 1 else "single", "timing": m["timing"]},
                "roofline": m["roofline"], "timing_stats": m["stats"], "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": m["gpu_launches"], "clocks": m["clocks"],
                "timed_wall_s": m["stats"]["region_s"], **extra}
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args):
    """The oracle (plain fp64 CPU code, as it stands) on the same workload,
    one bounded sample per step; rank 0 only."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    import numpy as np
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    name = args.workload
    if name == "prefill_paged_chunked":
        wl = PagedPrefill(name, dev, args.seed)
        unit, su = "TFLOP/s", 1e12
        S = wl.cfg["num_seqs"]

        def one(i):
            s, h = i % S, (7 * i) % wl.cfg["Hq"]
            return wl.oracle_rows(s, h, range(0, wl.cfg["chunk"], 128))

        sample = f"16 new-token rows of one (sequence, head) of {name} per step"
        config = wl.config()
    elif name.startswith("prefill_fp8"):
        from oracle import fp8 as F
        cfg = W.PREFILL_CAUSAL_2K if name.endswith("2k") else W.PREFILL_CAUSAL_16K
        B, H, N, d = cfg["B"], cfg["H"], cfg["N"], cfg["d"]
        per_head = 4.0 * d * (N * (N + 1) // 2)
        unit, su = "TFLOP/s", 1e12
        inp = W.dense_inputs(B, H, N, d, dtype=cfg["dtype"], mult=cfg["mult"], seed=args.seed, device=dev,
                             causal=True)
        sg = W.hadamard_signs(d, seed=args.seed).numpy()
        heads = [(b, h) for b in range(B) for h in range(H)]

        def one(i):
            b, h = heads[i % len(heads)]
            q = F.dequantize_blocks(*F.quantize_blocks(inp["Q"][b, h].float().cpu().numpy()[None], 128, signs=sg))[0]
            k = F.dequantize_blocks(*F.quantize_blocks(inp["K"][b, h].float().cpu().numpy()[None], 128, signs=sg))[0]
            oracle.attention_head(q, k, inp["V"][b, h].float().cpu().numpy().astype(np.float64), True, inp["scale"])
            return per_head

        sample = f"one (b, h) head of {name} per step (quantise Q, K; exact attention)"
        config = {"workload": name, "B": B, "H": H, "N": N, "d": d, "causal": True,
                  "dtype": "e4m3 Q/K, bf16 V/P/O", "global_batch": B, "seq_len": N}
    elif name.startswith("prefill"):
        cfg = W.PREFILL_CAUSAL_2K if name == "prefill_2k" else W.PREFILL_CAUSAL_16K
        B, H, N, d = cfg["B"], cfg["H"], cfg["N"], cfg["d"]
        pairs = N * (N + 1) // 2
        per_head = 4.0 * d * pairs
        unit, su = "TFLOP/s", 1e12
        inp = W.dense_inputs(B, H, N, d, dtype=cfg["dtype"], mult=cfg["mult"], seed=args.seed, device=dev,
                             causal=True)
        heads = [(b, h) for b in range(B) for h in range(H)]

        def one(i):
            b, h = heads[i % len(heads)]
            q, k, v = (inp[x][b, h].float().cpu().numpy().astype(np.float64) for x in ("Q", "K", "V"))
            oracle.attention_head(q, k, v, True, inp["scale"])
            return per_head

        sample = f"one (b, h) head of {name} per step"
        config = {"workload": name, "B": B, "H": H, "N": N, "d": d, "causal": True, "dtype": "bf16",
                  "global_batch": B, "seq_len": N}
    else:
        wl = Decode(name, dev, args.seed)
        p = wl.p
        sl = p.seq_lens.cpu().numpy()
        bt = p.block_table.cpu().numpy()
        q = p.q.float().cpu().numpy().astype(np.float64)
        unit, su = "GB/s", 1e9
        kc_t, vc_t = p.k_cache, p.v_cache

        class Lazy:
            def __init__(self, t):
                self.t, self.shape = t, tuple(t.shape)

            def __getitem__(self, i):
                return self.t[int(i)].float().cpu().numpy()

        def one(i):
            s = i % p.num_seqs
            oracle.paged_decode(q, Lazy(kc_t), Lazy(vc_t), bt, sl, p.block_size, p.scale, seqs=[s])
            return float(int(sl[s]) * 2 * p.H * p.d * 2)

        sample = f"one sequence of {name} per step (all heads)"
        config = wl.config()
    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    work = 0.0
    for i in range(args.steps):
        work += one(args.warmup + i)
    dt = time.perf_counter() - t0
    val = work / dt / su
    line = {"metric": METRIC, "value": round(val, 6), "unit": unit, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), bf16)",
            "impl": "reference", "config": config,
            "cpu_baseline": {"value": round(val, 6), "unit": unit, "cores": _cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(val, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_2k",
                    choices=["prefill_2k", "prefill_16k", "decode_uniform", "decode_shared_prefix",
                             "decode_uniform_small", "decode_shared_prefix_small", "kv_append", "block_copy", "decode_gqa_g4", "decode_gqa_g8",
                             "prefill_paged_chunked", "prefill_fp8_2k", "prefill_fp8_16k"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the extra legs of the default line (decode_uniform, prefill_16k, decode_shared_prefix)")
    ap.add_argument("--region-s", type=float, default=1.0,
                    help="minimum length of each timed region: the K-step graph is replayed until it lasts this "
                         "long (0: one replay)")
    ap.add_argument("--soak", type=float, default=1.0, help="seconds of untimed load before timing (clocks)")
    ap.add_argument("--eager", action="store_true",
                    help="time K eager calls instead of one replay of the K steps captured in a CUDA graph")
    args = ap.parse_args(argv)
    if args.impl == "ours":
        args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
