#!/usr/bin/env python
"""Benchmark of the memory-bounded KV decode step on B200.

Default workload: the Qwen3-8B-shaped layer decode step (B=32, Hq=32, Hkv=8,
d=128, budget M=4096 slots per kv head, beta = sigmoid(N(2, 1.5))). A step is
one decode token per sequence: budget enforcement + insertion
(kvb_evict_insert), then split-K retention-gated attention, with the merge of
the split states launched by the same call when there are several
(kvb_decode_attn). --config selects the workload:
  1  tiny decode step (B=1, Hq=8, Hkv=2, d=64, M=256)
  2  the Qwen3-8B-shaped layer above (default)
  3  long context: B=4, Hq=32, Hkv=8, d=128, 131072 positions kept in 8192 slots, 64 splits
  4  attention-state memory: 256 query tokens x 32 heads, self attention over a shared
     2048-token cache, then the lookup + merge against 4096 entries per head
  5  memento compaction: B=64 sawtooth caches, 9 x (Geom(1500) block + U[120,180] memento)

Prints ONE JSON line (rank 0). `value` is tokens/s of the whole job (one
attention layer) with inputs resident in HBM; `e2e` is the same metric through
the public API with the step's inputs copied from pinned host memory and the
output read back every step. The default workload reads > 126 MB (L2) of K/V
per step, so no L2 flush is needed; workloads that fit in L2 are timed step by
step after a flush (the JSON line's config says which).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1..5] [--impl kvb|reference]
  python bench.py --asm-crossover | --asm-build     (lookup and build measurements, 1 GPU)

For N > 1 launch with torch.distributed.run: every rank runs an independent
replica (the path shards into independent sequences; no collective on the
data path), timing is the max over ranks.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn tokens/s and KV-cache GB/s (% of B200 HBM peak) at budget M"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1000 * 1000      # B200 L2 (126 MB)

# ncu DRAM traffic (read + write bytes per launch) of the dominant kernel, keyed by
# (sha256 of the kernel's source file, config, num_splits). Reported only while the source is
# unchanged since the counters were taken.
MEASURED_TRAFFIC = {
    # decode_attn_tc_kernel<128,4,1>, Qwen3-8B-shaped layer, S=1: 545,628,416 read + 3,972,608 written
    ("f9553bcebbe325aa", 2, 1): 549601024,
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="kvb", choices=["kvb", "reference"])
    ap.add_argument("--splits", type=int, default=0, help="num_splits (0: the workload's default)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed steps one by one")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--asm-build", action="store_true",
                    help="time the offline memory build (cosine Lloyd iteration, aggregation) instead of a "
                         "decode step")
    ap.add_argument("--asm-crossover", action="store_true",
                    help="time the linear and the two-level memory lookups alone over query counts and memory "
                         "sizes (one GPU; L2 flushed between iterations) instead of a decode step")
    return ap.parse_args()


# ----------------------------------------------------------------------------------------------
# environment
# ----------------------------------------------------------------------------------------------

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest value over all ranks (timings are the slowest rank's); identity for one rank."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_value(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput of `world` independent replicas: all ranks' units over the slowest time."""
    return units_per_rank * world / (ms_max / 1e3)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def bf16_peak():
    """Dense bf16 tensor TFLOP/s for a kernel timed alone (burst figure), and where it comes from."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        if "bf16_tflops" in p:
            return float(p["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.device_id = None
        try:
            prop = torch.cuda.get_device_properties(device)
            self.device_id = f"{prop.pci_domain_id:08X}:{prop.pci_bus_id:02X}:{prop.pci_device_id:02X}.0"
        except Exception:
            self.device_id = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.device_id:
            cmd += ["-i", self.device_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.15)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 7]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def kernel_src_hash(name: str = "decode_attn_tc.cuh") -> str:
    """Hash of the dominant kernel's source: stored ncu traffic applies only to that exact source."""
    with open(os.path.join(ROOT, "memory_bounded_kv_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


# ----------------------------------------------------------------------------------------------
# decode workloads (tiny, Qwen3-8B-shaped, long context): evict+insert, then attention
# ----------------------------------------------------------------------------------------------

class DecodeBench:
    def __init__(self, cfg: int, splits: int, rank: int):
        from memory_bounded_kv_b200 import synth
        from memory_bounded_kv_b200.cache import BoundedKVCache
        import memory_bounded_kv_b200 as kvb
        self.cfg = cfg
        self.w = w = synth.decode_workload(cfg)
        self.S = splits or w.splits[-1]
        self.cache = BoundedKVCache.from_host(w.k, w.v, w.log_beta, w.pos, w.len, w.Hq, w.M, num_splits=self.S)
        if cfg == 3:   # stream positions cap .. 131071 through budget enforcement, then draw survivors' K/V
            blocks = (synth.CONFIG3_LOGICAL_T - w.cap) // synth.STREAM_BLOCK
            for blk in range(blocks):
                lbs = torch.from_numpy(synth.stream_log_beta(w, blk)).cuda()
                base = w.cap + blk * synth.STREAM_BLOCK
                ts = torch.arange(base, base + synth.STREAM_BLOCK, dtype=torch.int32, device="cuda")
                ts = ts[:, None].expand(-1, w.B).contiguous()
                for i in range(synth.STREAM_BLOCK):
                    kvb.kvb_evict_insert(self.cache.k, self.cache.v, self.cache.log_beta, self.cache.pos,
                                         self.cache.len, None, None, lbs[i], ts[i], w.M)
            k, v = synth.long_context_kv(w)
            self.cache.k.copy_(torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).cuda())
            self.cache.v.copy_(torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda())
            torch.cuda.synchronize()
        self.pool = min(w.steps, 1024)
        inp = [w.step_inputs(s) for s in range(self.pool)]

        def stack(key, dt):
            a = np.stack([x[key] for x in inp])
            t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
            return t.view(dt) if a.dtype == np.uint16 else t

        self.h_q = stack("q", torch.bfloat16).pin_memory()
        self.h_kn = stack("k_new", torch.bfloat16).pin_memory()
        self.h_vn = stack("v_new", torch.bfloat16).pin_memory()
        self.h_lb = stack("log_beta_new", torch.float32).pin_memory()
        self.d_q, self.d_kn, self.d_vn, self.d_lb = (x.cuda() for x in (self.h_q, self.h_kn, self.h_vn, self.h_lb))
        self.o = torch.zeros(w.B, w.Hq, w.d, device="cuda")
        self.lse = torch.zeros(w.B, w.Hq, device="cuda")
        self.tokens_per_step = w.B
        self.launches_per_step = 2 + (self.S > 1)   # evict/insert, attention (+ split merge)
        self.workload = w.name

    def t_of(self, i: int):
        return self.w.t0 + i

    def run_device(self, first: int, count: int, events=None):
        """Steps first .. first+count-1 with inputs resident in HBM."""
        c, t_all = self.cache, self.t_dev
        for i in range(first, first + count):
            p = i % self.pool
            t = t_all[i]
            c.insert(self.d_kn[p], self.d_vn[p], self.d_lb[p], t)
            if events is not None:
                events[i - first][0].record()
            c.attend(self.d_q[p], t, self.o, self.lse)
            if events is not None:
                events[i - first][1].record()

    def prepare(self, total_steps: int):
        self.t_dev = torch.tensor([[self.t_of(i)] * self.w.B for i in range(total_steps)], dtype=torch.int32,
                                  device="cuda")
        self.h_t = self.t_dev.cpu().pin_memory()
        self.s_q = torch.empty_like(self.d_q[0])
        self.s_kn = torch.empty_like(self.d_kn[0])
        self.s_vn = torch.empty_like(self.d_vn[0])
        self.s_lb = torch.empty_like(self.d_lb[0])
        self.s_t = torch.empty_like(self.t_dev[0])
        self.h_o = torch.empty(self.o.shape, dtype=torch.float32).pin_memory()
        self.h_lse = torch.empty(self.lse.shape, dtype=torch.float32).pin_memory()

    def run_e2e(self, first: int, count: int):
        """Steps through the public API from pinned host buffers; output read back every step."""
        c = self.cache
        for i in range(first, first + count):
            p = i % self.pool
            self.s_q.copy_(self.h_q[p], non_blocking=True)
            self.s_kn.copy_(self.h_kn[p], non_blocking=True)
            self.s_vn.copy_(self.h_vn[p], non_blocking=True)
            self.s_lb.copy_(self.h_lb[p], non_blocking=True)
            self.s_t.copy_(self.h_t[i], non_blocking=True)
            c.step(self.s_q, self.s_kn, self.s_vn, self.s_lb, self.s_t, self.o, self.lse)
            self.h_o.copy_(self.o, non_blocking=True)
            self.h_lse.copy_(self.lse, non_blocking=True)

    def e2e_bytes(self):
        h2d = sum(x[0].numel() * x.element_size() for x in (self.h_q, self.h_kn, self.h_vn, self.h_lb))
        h2d += self.w.B * 4
        d2h = self.o.numel() * 4 + self.lse.numel() * 4
        return h2d, d2h

    def attn_bytes(self):
        """Algorithmic bytes of one attention launch: K, V (+ log beta, pos) of the cached slots,
        q, len, t in; o (fp32), lse out."""
        w = self.w
        n = int(self.cache.len.sum().item())
        per_slot = 2 * w.d * 2 + 8
        return n * per_slot + w.B * w.Hq * w.d * 2 + w.B * w.Hkv * 4 + w.B * 4 + w.B * w.Hq * (w.d * 4 + 4)

    def evict_bytes(self):
        """Budget enforcement reads the attention's per-split candidates (16 B each) and writes the
        new row; the scan of log beta/pos happens inside the attention pass."""
        w = self.w
        return w.B * w.Hkv * (self.S * 16 + 2 * w.d * 2 + 4 + 4 + 4)

    def kernel_name(self):
        merge = " + merge_splits_kernel" if self.S > 1 else ""
        return (f"kvb_decode_attn = decode_attn_tc_kernel<d={self.w.d},G={self.w.Hq // self.w.Hkv},bias=1>"
                f"{merge}, S={self.S}")

    def flush_l2(self):
        return self.attn_bytes() < L2_BYTES

    def config(self):
        w = self.w
        l2 = (f"flushed before every timed step (256 MiB write): a step reads {self.attn_bytes() / 1e6:.2f} MB"
              if self.flush_l2() else
              f"no flush: every step reads {self.attn_bytes() / 1e6:.0f} MB of K/V (inputs larger than L2)")
        return {"workload": self.workload, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "budget_M": w.M,
                "num_splits": self.S, "beta": "sigmoid(N(2,1.5))", "l2": l2,
                "parallelism": "replicas (independent sequences per GPU)"}

    def oracle_sample(self, budget_s: float = 15.0):
        """The oracle as it stands on whole-batch decode steps from the prefill state; returns
        (tokens/s, description)."""
        import oracle
        w = self.w
        c = dict(k=w.k.copy(), v=w.v.copy(), log_beta=w.log_beta.copy(), pos=w.pos.copy(), len=w.len.copy())
        t0 = time.perf_counter()
        steps = 0
        while True:
            x = w.step_inputs(steps)
            oracle.evict_insert(c, x["k_new"], x["v_new"], x["log_beta_new"], x["t"], w.M)
            oracle.decode_attn(x["q"], c["k"], c["v"], c["log_beta"], c["pos"], c["len"], x["t"])
            steps += 1
            if time.perf_counter() - t0 > budget_s or steps >= 64:
                break
        dt = time.perf_counter() - t0
        return w.B * steps / dt, f"{steps} whole-batch decode steps (B={w.B}) from the prefill state"


# ----------------------------------------------------------------------------------------------
# attention-state-memory workload: self attention + lookup/merge per step
# ----------------------------------------------------------------------------------------------

def _dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


class ASMBench:
    """A step: the 256 query tokens' causal self attention over the shared 2048-token cache
    (kvb_decode_attn, batch stride 0) and the memory lookup + merge (kvb_asm_lookup_merge)."""

    KERNEL_SRC = "asm_lookup.cuh"

    def flush_l2(self):
        return True

    # the fp32 contraction runs as three exact bf16 products per element (q . hi + q . mid + q . lo)
    PEAK_NOTE = "{kind} dense bf16 {bf16:.0f} TFLOP/s (bf16_tflops, burst) / 3 bf16 products per fp32 product"

    def __init__(self, splits: int = 0):
        import memory_bounded_kv_b200 as kvb
        from memory_bounded_kv_b200 import synth
        self.kvb = kvb
        self.w = w = synth.asm_workload()
        self.S = splits or 4
        N, H, Hkv, d = w.N, w.H, w.Hkv, w.d
        self.k = _dev(w.k).expand(N, Hkv, w.L, d)
        self.v = _dev(w.v).expand(N, Hkv, w.L, d)
        self.pos = _dev(w.pos).expand(N, Hkv, w.L)
        self.len, self.t = _dev(w.len), _dev(w.t)
        self.h_q = torch.from_numpy(w.q.view(np.int16)).view(torch.bfloat16).pin_memory()
        self.q = self.h_q.cuda()
        self.qbar, self.abar, self.lz = _dev(w.qbar), _dev(w.abar), _dev(w.log_zbar)
        self.o_self = torch.zeros(N, H, d, device="cuda")
        self.l_self = torch.zeros(N, H, device="cuda")
        self.op, self.lp = kvb.decode_workspace(N, H, d, self.S)
        self.idx = torch.zeros(N, H, dtype=torch.int32, device="cuda")
        self.o = torch.zeros(N, H, d, device="cuda")
        self.lse = torch.zeros(N, H, device="cuda")
        self.ws = torch.empty(kvb.kvb_asm_workspace_bytes(N, H, w.K), dtype=torch.uint8, device="cuda")
        self.tokens_per_step = N
        self.launches_per_step = 4   # attention + split merge, lookup + state merge
        self.workload = "attention-state memory H32 K4096 d128, 256 queries, self attention over 2048"

    def prepare(self, total_steps):
        self.s_q = torch.empty_like(self.q)
        self.h_o = torch.empty(self.o.shape, dtype=torch.float32).pin_memory()
        self.h_idx = torch.empty(self.idx.shape, dtype=torch.int32).pin_memory()

    def _step(self, q, events=None, j=0):
        kvb = self.kvb
        kvb.kvb_decode_attn(q, self.k, self.v, None, self.pos, self.len, self.t, self.o_self, self.l_self,
                            num_splits=self.S, o_part=self.op, lse_part=self.lp)
        if events is not None:
            events[j][0].record()
        kvb.kvb_asm_lookup_merge(q, self.qbar, self.abar, self.lz, self.o_self, self.l_self, self.idx, self.o,
                                 self.lse, self.ws)
        if events is not None:
            events[j][1].record()

    def run_device(self, first, count, events=None):
        for j in range(count):
            self._step(self.q, events, j)

    def run_e2e(self, first, count):
        for _ in range(count):
            self.s_q.copy_(self.h_q, non_blocking=True)
            self._step(self.s_q)
            self.h_o.copy_(self.o, non_blocking=True)
            self.h_idx.copy_(self.idx, non_blocking=True)

    def e2e_bytes(self):
        return self.h_q.numel() * 2, self.o.numel() * 4 + self.idx.numel() * 4

    def attn_bytes(self):
        return 0

    def evict_bytes(self):
        w = self.w
        kv = int(w.len.sum()) * w.d * 2 * 2
        return kv + w.H * w.K * w.d * 4

    def flops(self):
        w = self.w
        return 2.0 * w.N * w.H * w.K * w.d

    def kernel_name(self):
        return "asm_score_umma_kernel + asm_merge_kernel (kvb_asm_lookup_merge)"

    def config(self):
        w = self.w
        return {"workload": self.workload, "N": w.N, "H": w.H, "Hkv": w.Hkv, "K": w.K, "d": w.d, "L": w.L,
                "self_attn_splits": self.S,
                "l2": "flushed before every timed step (256 MiB write): q̄ 64 MiB + ā 32 MiB + K/V 8 MiB fit in L2",
                "parallelism": "replicas"}


# ----------------------------------------------------------------------------------------------
# memento-style block compaction (sawtooth cache)
# ----------------------------------------------------------------------------------------------

class MementoBench:
    """A step: every active sequence decodes one token (append, attention); after the last
    token of a memento, the finished block's slots are removed in place (kvb_compact_blocks)."""

    SPLIT_LEN = 512

    def __init__(self, splits: int = 0):
        from memory_bounded_kv_b200 import synth
        from memory_bounded_kv_b200.cache import BoundedKVCache
        self.w = w = synth.memento_workload()
        self.S = -(-w.cap // self.SPLIT_LEN)
        self.cache = BoundedKVCache(w.B, w.Hq, w.Hkv, w.d, w.cap, w.cap, num_splits=self.S,
                                    split_len=self.SPLIT_LEN, with_beta=False)
        pool = [w.step_inputs(s) for s in range(w.pool)]
        self.q = [_dev(x["q"]) for x in pool]
        self.kn = [_dev(x["k_new"]) for x in pool]
        self.vn = [_dev(x["v_new"]) for x in pool]
        self.o = torch.zeros(w.B, w.Hq, w.d, device="cuda")
        self.lse = torch.zeros(w.B, w.Hq, device="cuda")
        self.comp = {}
        for s in w.compaction_steps().tolist():
            rs, rl = w.compaction(s)
            self.comp[s] = (_dev(rs), _dev(rl))
        self.active = np.array([(s < w.total).sum() for s in range(w.steps)], np.int64)
        self.lens = None
        self.tokens_per_step = None
        self.launches_per_step = None
        self.workload = "memento compaction B64 Hq32 Hkv8 d128, 9 x (Geom(1500) block + U[120,180] memento)"

    def flush_l2(self):
        return True

    def clamp_steps(self, K, W, KR):
        n = self.w.steps
        W = min(W, n // 8)
        KR = min(KR, n // 8)
        K = min(K, n - W - KR) if K > 0 else n - W - KR
        return K, W, KR

    def prepare(self, total_steps):
        w = self.w
        steps = np.arange(w.steps)
        self.t_dev = torch.from_numpy(np.where(steps[:, None] < w.total[None, :], steps[:, None], -1)
                                      .astype(np.int32)).cuda()

    def run_device(self, first, count, events=None):
        c, w = self.cache, self.w
        for j, i in enumerate(range(first, min(first + count, w.steps))):
            p = i % w.pool
            t = self.t_dev[i]
            c.insert(self.kn[p], self.vn[p], None, t)
            if events is not None:
                events[j][0].record()
            c.attend(self.q[p], t, self.o, self.lse)
            if events is not None:
                events[j][1].record()
            if i in self.comp:
                c.compact(*self.comp[i])

    def tokens(self, first, count):
        return int(self.active[first:first + count].sum())

    def launches(self, first, count):
        per = 2 + (self.S > 1)
        return per * count + sum(1 for i in range(first, first + count) if i in self.comp)

    def mean_kv_bytes(self, first, count):
        w = self.w
        tot = 0
        for i in range(first, first + count):
            tot += int(w.cache_len(i)[i < w.total].sum())
        return tot * w.Hkv * (2 * w.d * 2) / count

    def config(self):
        w = self.w
        return {"workload": self.workload, "B": w.B, "cap": w.cap, "split_len": self.SPLIT_LEN,
                "num_splits": self.S, "schedule_steps": w.steps, "parallelism": "replicas",
                "l2": "flushed before every timed step (256 MiB write): the live caches grow from "
                      "a few MB to ~350 MB over the timed steps"}


# ----------------------------------------------------------------------------------------------
# timing driver
# ----------------------------------------------------------------------------------------------

def time_flushed_steps(steps, flush, world):
    """Device time of the steps, each started with a cold L2 (flush written before it, outside
    its events): the sum of the per-step event times, after a barrier on both sides."""
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in steps]
    for (a, b), step in zip(ev, steps):
        flush.fill_(1)
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    return sum(a.elapsed_time(b) for a, b in ev)


def time_region(fn, world):
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    fn()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    return e0.elapsed_time(e1)


def run_kvb(args, world, rank, local):
    hbm_peak, peak_kind = peaks()
    if args.config in (1, 2, 3):
        bench = DecodeBench(args.config, args.splits, rank)
    elif args.config == 4:
        bench = ASMBench(args.splits)
    else:
        bench = MementoBench(args.splits)
    K, W = args.steps, args.warmup
    KR = min(K, 500)                               # steps of the kernel-timing region
    if hasattr(bench, "clamp_steps"):              # the memento schedule is finite
        K, W, KR = bench.clamp_steps(K, W, KR)
    bench.prepare(2 * (W + K) + KR + 2)

    # warm-up; the timed region (the K steps captured once as a CUDA graph -- every launch of
    # every step with the programmatic dependencies between them -- and replayed; no events
    # inside); then a region of KR steps with CUDA events around the dominant launch
    bench.run_device(0, W)
    torch.cuda.synchronize()
    # a workload whose step touches less than L2 holds is timed step by step with a cold L2:
    # each step is its own CUDA graph, replayed after a 256 MiB write, with events around the
    # replay only (the flush is not timed); otherwise the K steps are one graph
    flush_l2 = bench.flush_l2() if hasattr(bench, "flush_l2") else False
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if flush_l2 else None
    graph, step_graphs = None, None
    if not args.no_graph:
        if flush_l2:
            step_graphs = []
            for i in range(K):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    bench.run_device(W + i, 1)
                step_graphs.append(g)
        else:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                bench.run_device(W, K)
    clocks = ClockSampler(local)
    clocks.start()
    if step_graphs is not None:
        ms = time_flushed_steps([g.replay for g in step_graphs], flush, world)
    elif flush_l2:
        ms = time_flushed_steps([lambda i=i: bench.run_device(W + i, 1) for i in range(K)], flush, world)
    elif graph is not None:
        ms = time_region(graph.replay, world)
    else:
        ms = time_region(lambda: bench.run_device(W, K), world)
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(KR)]
    if flush_l2:
        def kernel_region():
            for j in range(KR):
                flush.fill_(1)
                bench.run_device(W + K + j, 1, events[j:j + 1])
        time_region(kernel_region, world)
    else:
        time_region(lambda: bench.run_device(W + K, KR, events), world)
    clk = clocks.stop()
    del step_graphs
    kern_ms = [a.elapsed_time(b) for a, b in events]
    ms = max_over_ranks(ms, world)
    kms = max_over_ranks(statistics.mean(kern_ms), world)
    tokens = bench.tokens(W, K) if hasattr(bench, "tokens") else bench.tokens_per_step * K
    launches = bench.launches(W, K) if hasattr(bench, "launches") else bench.launches_per_step * K
    value = replica_value(tokens, world, ms)
    src = kernel_src_hash(getattr(bench, "KERNEL_SRC", "decode_attn_tc.cuh"))
    if hasattr(bench, "flops"):      # attention-state-memory lookup: tensor bound (bf16 x 3)
        bf16_tf, bf16_kind = bf16_peak()
        peak_tf = bf16_tf / 3.0
        achieved = bench.flops() / (kms / 1e3) / 1e12
        roofline = {"bound": "tensor", "kernel": bench.kernel_name(), "achieved": achieved, "peak": peak_tf,
                    "unit": "TFLOP/s", "frac": achieved / peak_tf,
                    "peak_source": ASMBench.PEAK_NOTE.format(kind=bf16_kind, bf16=bf16_tf),
                    "traffic": None, "algorithmic_flops_per_launch": bench.flops(), "kernel_ms_avg": kms}
        step_bytes = bench.evict_bytes()
    else:
        attn_bytes = bench.mean_kv_bytes(W + K, KR) if hasattr(bench, "mean_kv_bytes") else bench.attn_bytes()
        achieved = attn_bytes / (kms / 1e3) / 1e9
        name = (bench.kernel_name() if hasattr(bench, "kernel_name")
                else "kvb_decode_attn = decode_attn_tc_kernel<128,4,plain> + merge_splits_kernel")
        roofline = {"bound": "hbm", "kernel": name, "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                    "frac": achieved / hbm_peak, "peak_source": f"{peak_kind} (hbm_gbs)",
                    "traffic": MEASURED_TRAFFIC.get((src, args.config, getattr(bench, "S", 0))),
                    "algorithmic_bytes_per_launch": attn_bytes, "kernel_ms_avg": kms}
        step_bytes = attn_bytes + (bench.evict_bytes() if hasattr(bench, "evict_bytes") else 0)
    kv_gbs = step_bytes * K / (ms / 1e3) / 1e9

    e2e = None
    if not args.no_e2e and hasattr(bench, "run_e2e"):
        first = W + K + KR
        bench.run_e2e(first, W)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(time_region(lambda: bench.run_e2e(first + W, K), world), world)
        h2d, d2h = bench.e2e_bytes()
        e2e = {"value": bench.tokens_per_step * K * world / (ms_e2e / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e / K}

    cfg = bench.config()
    cfg["timed_launches"] = "cuda graph replay" if graph is not None else "stream launches"
    out = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "storage_dtype": "bf16",
        "data": "synthetic (seeded; shapes and distributions of the workload)",
        "config": cfg,
        "kv_gbs": kv_gbs,
        "kv_frac_of_hbm_peak": kv_gbs / hbm_peak,
        "roofline": roofline,
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": launches,
        "kernel_src_sha256_16": src,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and hasattr(bench, "oracle_sample"):
        v, sample = bench.oracle_sample()
        out["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample}
    return out


def run_reference(args, world, rank):
    """The oracle as it stands, timed on the host cores, on the workload's metric (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    from memory_bounded_kv_b200 import synth
    w = synth.decode_workload(2 if args.config not in (1, 3) else args.config)
    nb = 1   # one sequence per step keeps --steps K --warmup W within minutes
    c = dict(k=w.k[:nb].copy(), v=w.v[:nb].copy(), log_beta=w.log_beta[:nb].copy(), pos=w.pos[:nb].copy(),
             len=w.len[:nb].copy())

    def step(s):
        x = w.step_inputs(s % w.steps)
        t = np.full(nb, w.t0 + s, np.int32)
        oracle.evict_insert(c, x["k_new"][:nb], x["v_new"][:nb], x["log_beta_new"][:nb], t, w.M)
        oracle.decode_attn(x["q"][:nb], c["k"], c["v"], c["log_beta"], c["pos"], c["len"], t)

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    for s in range(args.warmup, args.warmup + args.steps):
        step(s)
    dt = time.perf_counter() - t0
    value = nb * args.steps / dt
    sample = f"{nb} of {w.B} sequences per decode step (one attention layer), steps continue from t={w.t0}"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_asm_build(args) -> dict:
    """The offline memory build at 16384 calibration queries per head (4 per entry), 32 heads,
    K = 4096 entries, d = 128: one Lloyd iteration (mean update by kvb_asm_aggregate, cosine
    assignment by kvb_asm_lookup_merge without merge) and the final aggregation of the states
    (q 134 MB bf16, a 268 MB f32 in). Each replayed from a CUDA graph after an L2 flush."""
    import memory_bounded_kv_b200 as kvb
    from memory_bounded_kv_b200 import asm_build
    from memory_bounded_kv_b200.synth import normal_bf16, rng
    hbm_peak, peak_kind = peaks()
    bf16_tf, bf16_kind = bf16_peak()
    M, H, K, d = 16384, 32, 4096, 128
    g = rng(44, 0)
    q = _dev(normal_bf16(g, (M, H, d)))
    a = torch.randn(M, H, d, device="cuda")
    lse = torch.rand(M, H, device="cuda") * 8
    init = np.tile(np.arange(K), (H, 1))
    idx, cent = asm_build.asm_kmeans(q, init, iters=1)
    ws_agg = torch.empty(kvb.kvb_asm_aggregate_workspace_bytes(H, K), dtype=torch.uint8, device="cuda")
    ws_lk = torch.empty(kvb.kvb_asm_workspace_bytes(M, H, K), dtype=torch.uint8, device="cuda")
    qbar = torch.empty(H, K, d, device="cuda")
    abar = torch.empty(H, K, d, dtype=torch.bfloat16, device="cuda")
    lz = torch.empty(H, K, device="cuda")
    cnt = torch.empty(H, K, dtype=torch.int32, device="cuda")

    def update():
        kvb.kvb_asm_aggregate(q, None, None, idx, cent, None, None, None, ws_agg)

    def assign():
        kvb.kvb_asm_lookup_merge(q, cent, None, None, None, None, idx, None, None, ws_lk)

    def aggregate():
        kvb.kvb_asm_aggregate(q, a, lse, idx, qbar, abar, lz, cnt, ws_agg)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    iters = max(3, min(args.steps, 20))
    out = {}
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    for name, fn in (("update", update), ("assign", assign), ("aggregate", aggregate)):
        for _ in range(max(2, args.warmup)):
            fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fn()
        out[name] = time_flushed_steps([graph.replay] * iters, flush, 1) / iters
        del graph
    clk = clocks.stop()
    flops = 2.0 * M * H * K * d
    agg_bytes = M * H * (d * 2 + d * 4 + 4 + 4) + H * K * (d * 4 + d * 2 + 4 + 4)
    return {"metric": "ASM offline build: Lloyd iteration and aggregation time", "unit": "ms",
            "higher_is_better": False, "n_gpus": 1, "steps": iters, "warmup": max(2, args.warmup),
            "dtype": "f32 (bf16 x 3 products)", "data": "synthetic (random queries and states)",
            "config": {"workload": f"{M} calibration queries x {H} heads -> {K} entries, d {d}",
                       "l2": "flushed before every timed call (256 MiB write)"},
            "lloyd_iteration_ms": out["update"] + out["assign"], "update_ms": out["update"],
            "assign_ms": out["assign"], "aggregate_ms": out["aggregate"],
            "assign_roofline": {"bound": "tensor", "achieved": flops / (out["assign"] / 1e3) / 1e12,
                                "peak": bf16_tf / 3.0, "unit": "TFLOP/s",
                                "frac": flops / (out["assign"] / 1e3) / 1e12 / (bf16_tf / 3.0),
                                "peak_source": f"{bf16_kind} bf16_tflops / 3"},
            "aggregate_roofline": {"bound": "hbm", "achieved": agg_bytes / (out["aggregate"] / 1e3) / 1e9,
                                   "peak": hbm_peak, "unit": "GB/s",
                                   "frac": agg_bytes / (out["aggregate"] / 1e3) / 1e9 / hbm_peak,
                                   "algorithmic_bytes": agg_bytes, "peak_source": f"{peak_kind} (hbm_gbs)"},
            "clocks": clk}


def run_asm_crossover(args) -> dict:
    """Lookup + merge alone, linear (kvb_asm_lookup_merge) against two-level
    (kvb_asm_hier_lookup_merge, C = sqrt(K) clusters, top-16), on the clustered memory
    of synth.asm_index_workload: 32 heads, d = 128, N query tokens per call. Every
    timed call starts with a cold L2 (a 256 MiB buffer is written before it, outside
    the events), as in decoding, where the other layers evict the memory between
    lookups; the *_warm_us columns repeat the calls back to back without the flush. Each
    call is replayed from a CUDA graph, so that the host's launch latency is not timed.
    Recall = share of (query, head) whose two-level entry is the linear one."""
    import memory_bounded_kv_b200 as kvb
    from memory_bounded_kv_b200 import synth
    hbm_peak, peak_kind = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    iters, warm = max(5, min(args.steps, 200)), max(3, args.warmup)
    rows = []
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    for K in (4096, 16384):
        C = int(round(K ** 0.5))
        m = 16
        w = synth.asm_index_workload(N=256, H=32, K=K, C=C)
        g = {name: _dev(getattr(w, name)) for name in ("q", "qhat", "offsets", "members", "qbar", "abar",
                                                      "log_zbar", "o_self", "lse_self")}
        for N in (1, 8, 64, 256):
            q, o_self, l_self = g["q"][:N].contiguous(), g["o_self"][:N].contiguous(), g["lse_self"][:N].contiguous()
            H, d = w.H, w.d
            out = {}
            for kind in ("linear", "hier"):
                idx = torch.zeros(N, H, dtype=torch.int32, device="cuda")
                o = torch.zeros(N, H, d, device="cuda")
                lse = torch.zeros(N, H, device="cuda")
                if kind == "linear":
                    ws = torch.empty(kvb.kvb_asm_workspace_bytes(N, H, K), dtype=torch.uint8, device="cuda")
                    call = lambda: kvb.kvb_asm_lookup_merge(q, g["qbar"], g["abar"], g["log_zbar"], o_self, l_self,
                                                            idx, o, lse, ws)
                else:
                    ws = torch.empty(kvb.kvb_asm_hier_workspace_bytes(N, H, m), dtype=torch.uint8, device="cuda")
                    call = lambda: kvb.kvb_asm_hier_lookup_merge(q, g["qhat"], g["offsets"], g["members"], g["qbar"],
                                                                 g["abar"], g["log_zbar"], o_self, l_self, idx, o,
                                                                 lse, ws, m)
                ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(iters)]
                for _ in range(warm):
                    call()
                torch.cuda.synchronize()
                # replayed as a CUDA graph: the events time the GPU work, not the host's launches
                side = torch.cuda.Stream()
                side.wait_stream(torch.cuda.current_stream())
                with torch.cuda.stream(side):
                    call()
                torch.cuda.current_stream().wait_stream(side)
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    call()
                graph.replay()
                torch.cuda.synchronize()
                for a, b in ev:
                    flush.fill_(1)
                    a.record()
                    graph.replay()
                    b.record()
                torch.cuda.synchronize()
                ms = statistics.median(x.elapsed_time(y) for x, y in ev)
                reps = 20           # the same call back to back: memory and translations warm
                for a, b in ev:
                    a.record()
                    for _ in range(reps):
                        graph.replay()
                    b.record()
                torch.cuda.synchronize()
                warm_ms = statistics.median(x.elapsed_time(y) for x, y in ev) / reps
                del graph
                out[kind] = (ms, idx.cpu().numpy(), ws, warm_ms)
            # algorithmic bytes of the two-level lookup: the first level, the selected clusters' rows, the merge
            nhm = N * H * m
            sel = out["hier"][2][nhm * 8: nhm * 12].view(torch.int32).cpu().numpy().reshape(N, H, m)
            sizes = np.diff(w.offsets, axis=1)
            rows_read = sum(int(sizes[h][sel[n, h][sel[n, h] >= 0]].sum()) for n in range(N) for h in range(H))
            hier_bytes = (N * H * C + rows_read) * d * 4 + N * H * (d * 2 + d * 4 * 2 + d * 2)
            lin_bytes = H * K * d * 4 + N * H * (d * 2 + d * 4 * 2 + d * 2)
            rows.append({
                "K": K, "C": C, "m": m, "N": N,
                "linear_us": round(out["linear"][0] * 1e3, 2), "hier_us": round(out["hier"][0] * 1e3, 2),
                "linear_warm_us": round(out["linear"][3] * 1e3, 2), "hier_warm_us": round(out["hier"][3] * 1e3, 2),
                "speedup": round(out["linear"][0] / out["hier"][0], 2),
                "recall": round(float((out["linear"][1] == out["hier"][1]).mean()), 4),
                "hier_gbs": round(hier_bytes / (out["hier"][0] / 1e3) / 1e9, 1),
                "hier_frac": round(hier_bytes / (out["hier"][0] / 1e3) / 1e9 / hbm_peak, 3),
                "linear_gbs": round(lin_bytes / (out["linear"][0] / 1e3) / 1e9, 1),
            })
    clk = clocks.stop()
    return {"metric": "ASM lookup + merge latency, linear vs two-level (median of cold-L2 calls)",
            "unit": "us", "higher_is_better": False, "n_gpus": 1, "steps": iters, "warmup": warm,
            "dtype": "f32", "data": "synthetic clustered memory (synth.asm_index_workload)",
            "config": {"workload": "attention-state memory, 32 heads, d 128, top-16 of sqrt(K) clusters",
                       "l2": "flushed before every timed call (256 MiB write)"},
            "peak_gbs": hbm_peak, "peak_source": f"{peak_kind} (hbm_gbs)", "rows": rows, "clocks": clk}


def main():
    args = parse()
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if args.asm_crossover:
        print(json.dumps(run_asm_crossover(args)), flush=True)
        return
    if args.asm_build:
        print(json.dumps(run_asm_build(args)), flush=True)
        return
    world, rank, local = dist_init()
    try:
        out = run_kvb(args, world, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
