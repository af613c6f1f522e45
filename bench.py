#!/usr/bin/env python
"""Benchmark of the memory-bounded KV decode step on B200.

Headline workload: the Qwen3-8B-shaped layer decode step (B=32, Hq=32, Hkv=8,
d=128, budget M=4096 slots per kv head, beta = sigmoid(N(2, 1.5))). A step is
one decode token per sequence: budget enforcement + insertion
(kvb_evict_insert), then split-K retention-gated attention, with the merge of
the split states launched by the same call when there are several
(kvb_decode_attn). The other workloads are measured in the same run and
reported under "configs" on the same JSON line:
  1   tiny decode step (B=1, Hq=8, Hkv=2, d=64, M=256)
  2   the Qwen3-8B-shaped layer above (the headline)
  3   long context: B=4, Hq=32, Hkv=8, d=128, 131072 positions kept in 8192 slots, 64 splits
  3p  the same with beta = 1 (no log beta; eviction is first-in first-out)
  4   attention-state memory: 256 query tokens x 32 heads, self attention over a shared
      2048-token cache, then the lookup + merge against 4096 entries per head
  5   memento compaction: B=64 sawtooth caches, 9 x (Geom(1500) block + U[120,180] memento)
  5p  the same on the paged cache (pages of 64 slots from one pool sized to the schedule's peak)

Prints ONE JSON line (rank 0). `value` is tokens/s of the whole job (one
attention layer) with inputs resident in HBM; `e2e` is the same metric through
the public API with every step's inputs copied from pinned host memory (one
packed copy) and its outputs read back (one copy), each step replayed from a
CUDA graph. Workloads whose step reads more than the 126 MB L2 are timed as
graphs of many steps; the others step by step, each step after a 256 MiB
write that flushes L2 (outside the events). The roofline of the dominant
launch comes from events around that launch's own graph in a second region.
After timing, one more step is computed two ways on the GPU (the timed path and
an independent one: full eviction scan, other split counts, the per-row kernel)
and compared ("consistency"); parity with the CPU oracle is the tests' job.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1|2|3|4|5] [--plain] [--paged]
                  [--configs all|none|LIST] [--seed S] [--check sampled|full|off]
                  [--impl kvb|reference]
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
import platform
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
WORKLOADS = ("1", "2", "3", "3p", "4", "5", "5p")

# ncu DRAM traffic (read + write bytes per launch) of the dominant kernel, keyed by
# (sha256 of the kernel's source file, workload, num_splits). Reported only while the source is
# unchanged since the counters were taken.
MEASURED_TRAFFIC = {
    # the fused decode step (decode_attn_tc_kernel with the insertion) at the Qwen3-8B-shaped layer,
    # one split: 545,730,816 read + 3,399,424 written
    # (bench.py --profile c2 under ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum)
    ("2a67484ce58e6b51", "2", 1): 549130240,
    # the long-context fused step (136,465,408 + 3,846,144) and its 64-way merge (4,247,552 + 0)
    # (bench.py --profile c3, the same metrics over both launches)
    ("2a67484ce58e6b51", "3", 64): 144559104,
    # the lookup over the prepared memory (102,808,320 + 3,240,192) and its merge (6,999,040 + 0)
    # (bench.py --profile c4, the same metrics over both launches)
    ("efd6765f5e1aeb11", "4", 4): 113047552,
}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--plain", action="store_true", help="beta = 1 variant of the long-context workload")
    ap.add_argument("--configs", default="all",
                    help="other workloads measured in the same run and reported under 'configs': 'all', "
                         "'none' or a comma list of " + ",".join(WORKLOADS))
    ap.add_argument("--seed", type=int, default=None, help="replace the workloads' own seeds")
    ap.add_argument("--paged", action="store_true", help="paged-cache variant of the memento workload")
    ap.add_argument("--check", default="sampled", choices=["sampled", "full", "off"],
                    help="after timing, one more step computed two ways on the GPU (the timed path and an "
                         "independent one) and compared (sampled: cache bytes of a few sequences; full: all)")
    ap.add_argument("--dump-state", default=None, metavar="DIR",
                    help="write the cache state before the checked step and that step's inputs as raw files "
                         "under DIR/<workload> (decode and memento workloads)")
    ap.add_argument("--replay", default=None, metavar="DIR",
                    help="instead of timing, run the step dumped under DIR once and write its outputs and "
                         "the cache after it under DIR/replayed")
    ap.add_argument("--profile", default=None, choices=list(PROFILE_CASES),
                    help="instead of timing, run a few launches of one workload's dominant kernel at its shape "
                         "(for ncu captures: small device footprint, no schedule walk)")
    ap.add_argument("--impl", default="kvb", choices=["kvb", "reference"])
    ap.add_argument("--splits", type=int, default=0, help="num_splits of the headline workload (0: its default)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--asm-build", action="store_true",
                    help="time the offline memory build (cosine Lloyd iteration, aggregation) instead of a "
                         "decode step")
    ap.add_argument("--asm-crossover", action="store_true",
                    help="time the linear and the two-level memory lookups alone over query counts and memory "
                         "sizes (one GPU; L2 flushed between iterations) instead of a decode step")
    return ap.parse_args(argv)


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


def _peaks_file():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f)
    return None


def peaks():
    p = _peaks_file()
    if p is not None and "hbm_gbs" in p:
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def bf16_peak():
    """Dense bf16 tensor TFLOP/s for a kernel timed alone (burst figure), and where it comes from."""
    p = _peaks_file()
    if p is not None and "bf16_tflops" in p:
        return float(p["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


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


_T0 = time.perf_counter()


def log(msg: str):
    """Progress on stderr (the JSON line alone goes to stdout)."""
    print(f"[bench {time.perf_counter() - _T0:7.1f}s] {msg}", file=sys.stderr, flush=True)


def _dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


class Packed:
    """One device buffer holding several tensors (each at a 256-byte aligned offset), so that a
    step's inputs arrive with one host-to-device copy and its outputs leave with one copy."""

    def __init__(self, layout):
        self.offsets, off = {}, 0
        for name, shape, dt in layout:
            n = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
            self.offsets[name] = (off, n, tuple(shape), dt)
            off = (off + n + 255) // 256 * 256
        self.nbytes = off
        self.payload = sum(v[1] for v in self.offsets.values())
        self.dev = torch.zeros(self.nbytes, dtype=torch.uint8, device="cuda")
        self.views = {k: self.dev[o:o + n].view(dt).view(shape) for k, (o, n, shape, dt) in self.offsets.items()}

    def fill_host(self, row: torch.Tensor, arrays: dict):
        """Write numpy arrays into a host uint8 row laid out like the device buffer."""
        for k, a in arrays.items():
            o, n, _, _ = self.offsets[k]
            row[o:o + n] = torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1))


def capture(fn):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def _consistency(exact: dict, o, lse, o_ref, l_ref, what: str, dev_err: int) -> dict:
    """Two GPU computations of the same step: fields in `exact` compared bit for bit; o within
    max-abs 2e-2 and rel-L2 1e-3; lse within max(1e-4, 2^-22 |lse|) (the tolerances of the parity
    tests, which compare with the CPU oracle)."""
    ok = dev_err == 0
    res = {"checked": what, "device_error_bits": int(dev_err)}
    for k, (a, b) in exact.items():
        same = bool(np.array_equal(a, b))
        res[f"{k}_exact"] = same
        ok &= same
    o = np.asarray(o, np.float64)
    err = np.abs(o - o_ref)
    nref = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(o - o_ref) / nref) if nref > 0 else float(np.linalg.norm(o))
    fin = ~np.isneginf(l_ref)
    same_inf = bool(np.array_equal(np.isneginf(lse), ~fin))
    dl = np.abs(np.asarray(lse, np.float64)[fin] - l_ref[fin])
    tol = np.maximum(1e-4, 2.0 ** -22 * np.abs(l_ref[fin]))
    res.update(max_abs=float(err.max()) if err.size else 0.0, rel_l2=rel,
               lse_max_abs=float(dl.max()) if dl.size else 0.0)
    ok &= res["max_abs"] <= 2e-2 and rel <= 1e-3 and same_inf and bool(np.all(dl <= tol))
    res["ok"] = bool(ok)
    return res


# ----------------------------------------------------------------------------------------------
# workloads. Each one enqueues step i on the current stream in three parts: pre (budget
# enforcement + insertion, or the self attention), attn (the dominant launch), post (compaction)
# ----------------------------------------------------------------------------------------------

class DecodeBench:
    """Decode workloads 1 (tiny), 2 (Qwen3-8B-shaped) and 3 (long context), and 3's beta = 1 variant."""

    bound = "hbm"
    KERNEL_SRC = "decode_attn_tc.cuh"

    def __init__(self, cfg: int, splits: int, seed=None, plain: bool = False):
        import memory_bounded_kv_b200 as kvb
        from memory_bounded_kv_b200 import synth
        from memory_bounded_kv_b200.cache import BoundedKVCache
        self.cfg, self.plain = cfg, plain
        self.key = f"{cfg}{'p' if plain else ''}"
        self.w = w = synth.decode_workload(cfg, seed=seed)
        self.S = splits or w.splits[-1]
        if cfg == 3:
            self.cache = BoundedKVCache(w.B, w.Hq, w.Hkv, w.d, w.cap, w.M, num_splits=self.S, with_beta=not plain)
            if plain:   # first-in first-out keeps exactly the last M positions of the stream
                pos = np.broadcast_to(np.arange(synth.CONFIG3_LOGICAL_T - w.M, synth.CONFIG3_LOGICAL_T,
                                                dtype=np.int32), (w.B, w.Hkv, w.M))
                self.cache.pos.copy_(_dev(pos.copy()))
                self.cache.len.fill_(w.M)
            else:
                self.cache.log_beta.copy_(_dev(w.log_beta))
                self.cache.pos.copy_(_dev(w.pos))
                self.cache.len.copy_(_dev(w.len))
                self._stream_build(kvb, synth)
            k, v = synth.long_context_kv(w)
            self.cache.k.copy_(_dev(k))
            self.cache.v.copy_(_dev(v))
            self.cache.full = True   # every row holds its budget M after the stream
            torch.cuda.synchronize()
        else:
            self.cache = BoundedKVCache.from_host(w.k, w.v, None if plain else w.log_beta, w.pos, w.len, w.Hq, w.M,
                                                  num_splits=self.S)
        self.pool = min(w.steps, 1024)
        self.inp = [w.step_inputs(s) for s in range(self.pool)]

        def stack(key):
            return _dev(np.stack([x[key] for x in self.inp]))

        self.d_q, self.d_kn, self.d_vn, self.d_lb = stack("q"), stack("k_new"), stack("v_new"), stack("log_beta_new")
        layout = [("q", (w.B, w.Hq, w.d), torch.bfloat16), ("k_new", (w.B, w.Hkv, w.d), torch.bfloat16),
                  ("v_new", (w.B, w.Hkv, w.d), torch.bfloat16), ("t", (w.B,), torch.int32)]
        if not plain:
            layout.append(("log_beta_new", (w.B, w.Hkv), torch.float32))
        self.stage = Packed(layout)
        self.out = Packed([("o", (w.B, w.Hq, w.d), torch.float32), ("lse", (w.B, w.Hq), torch.float32)])
        self.o, self.lse = self.out.views["o"], self.out.views["lse"]
        self.workload = w.name + (" beta=1" if plain else "")
        self.flush_l2 = self.attn_bytes() < L2_BYTES

    def _stream_build(self, kvb, synth):
        """Stream positions cap .. 131071 through budget enforcement (log beta and pos only): one
        block of 4096 insertions captured as a CUDA graph, replayed per block with its log beta."""
        w, c = self.w, self.cache
        lbs = torch.empty(synth.STREAM_BLOCK, w.B, w.Hkv, device="cuda")
        ts = torch.empty(synth.STREAM_BLOCK, w.B, dtype=torch.int32, device="cuda")

        def block():
            for i in range(synth.STREAM_BLOCK):
                kvb.kvb_evict_insert(c.k, c.v, c.log_beta, c.pos, c.len, None, None, lbs[i], ts[i], w.M)

        blocks = (synth.CONFIG3_LOGICAL_T - w.cap) // synth.STREAM_BLOCK
        g = None
        for blk in range(blocks):
            lbs.copy_(torch.from_numpy(synth.stream_log_beta(w, blk)))
            base = w.cap + blk * synth.STREAM_BLOCK
            ts.copy_(torch.arange(base, base + synth.STREAM_BLOCK, dtype=torch.int32)[:, None].expand(-1, w.B))
            if g is None:
                torch.cuda.synchronize()
                g = capture(block)
            g.replay()
        torch.cuda.synchronize()
        del g

    def prepare(self, total_steps: int):
        self.t_dev = (self.w.t0 + torch.arange(total_steps, dtype=torch.int32, device="cuda"))[:, None].expand(
            -1, self.w.B).contiguous()

    def n_steps(self):
        return None   # positions continue past the workload's own step count

    def _in(self, i, x):
        if x is not None:
            return x["q"], x["k_new"], x["v_new"], x.get("log_beta_new"), x["t"]
        p = i % self.pool
        return self.d_q[p], self.d_kn[p], self.d_vn[p], None if self.plain else self.d_lb[p], self.t_dev[i]

    def pre(self, i, x=None):
        if self.cache.full:   # the step's one launch does the insertion (attn)
            return
        _, kn, vn, lb, t = self._in(i, x)
        self.cache.insert(kn, vn, lb, t)

    def attn(self, i, x=None):
        q, kn, vn, lb, t = self._in(i, x)
        o, lse = (x["o"], x["lse"]) if x is not None and "o" in x else (self.o, self.lse)
        if self.cache.full:
            # budget enforcement from the previous step's records, insertion and attention in one
            # launch (the first step after a set-up, with no records yet, runs as two)
            self.cache.step(q, kn, vn, lb, t, o, lse)
        else:
            self.cache.attend(q, t, o, lse)

    def post(self, i, x=None):
        pass

    def host_inputs(self, i):
        x = self.inp[i % self.pool]
        out = dict(q=x["q"], k_new=x["k_new"], v_new=x["v_new"], t=np.full(self.w.B, self.w.t0 + i, np.int32))
        if not self.plain:
            out["log_beta_new"] = x["log_beta_new"]
        return out

    def tokens(self, i):
        return self.w.B

    def launches(self, i):
        if self.cache.full:
            return 1 + (self.S > 1)   # the fused step (+ split merge)
        return 2 + (self.S > 1)   # evict/insert, attention (+ split merge)

    def attn_bytes(self, i=None):
        """Algorithmic bytes of one attention launch: K, V (+ log beta) and pos of the cached slots
        (pos feeds the eviction candidates), q, len, t in; o (fp32), lse out. With the insertion
        fused into it, also the step's records in, the new rows in and the victims' rows out."""
        w = self.w
        n = w.B * w.Hkv * w.M        # every (b, g) holds M slots in these workloads
        per_slot = 2 * w.d * 2 + 4 + (0 if self.plain else 4)
        b = n * per_slot + w.B * w.Hq * w.d * 2 + w.B * w.Hkv * 4 + w.B * 4 + w.B * w.Hq * (w.d * 4 + 4)
        if self.cache.full:
            meta = 4 + (0 if self.plain else 4)
            b += w.B * w.Hkv * (self.S * 16 + 2 * (2 * w.d * 2 + meta))
        return b

    def other_bytes(self, i=None):
        """Budget enforcement reads the attention's per-split candidates (16 B each) and writes the
        new row; the scan of log beta/pos happens inside the attention pass. None when the step's
        one launch does the insertion."""
        w = self.w
        if self.cache.full:
            return 0
        return w.B * w.Hkv * (self.S * 16 + 2 * w.d * 2 + 4 + 4 + 4)

    def kernel_name(self):
        merge = " + merge_splits_kernel" if self.S > 1 else ""
        if self.cache.full:
            return (f"kvb_decode_step = decode_attn_tc_kernel<d={self.w.d},G={self.w.Hq // self.w.Hkv},"
                    f"bias={0 if self.plain else 1},insertion>{merge}, S={self.S}")
        return (f"kvb_decode_attn = decode_attn_tc_kernel<d={self.w.d},G={self.w.Hq // self.w.Hkv},"
                f"bias={0 if self.plain else 1}>{merge}, S={self.S}")

    def config(self):
        w = self.w
        l2 = (f"flushed before every timed step (256 MiB write): a step reads {self.attn_bytes() / 1e6:.2f} MB"
              if self.flush_l2 else
              f"no flush: every step reads {self.attn_bytes() / 1e6:.0f} MB of K/V (inputs larger than L2)")
        return {"workload": self.workload, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "budget_M": w.M,
                "num_splits": self.S, "beta": "1" if self.plain else "sigmoid(N(2,1.5))", "seed": w.seed,
                "l2": l2, "parallelism": "replicas (independent sequences per GPU)"}

    def dump_step(self, i, path):
        """The cache before the step at position t0 + i and that step's inputs."""
        from memory_bounded_kv_b200.state import dump_step
        dump_step(path, self.cache, self.host_inputs(i), extra_meta={"workload": self.workload, "step": int(i)})

    def check(self, i, full: bool):
        """Consistency of one more step (position t0 + i) computed two ways on the GPU from the same
        cache: the timed path (eviction from the attention's candidates, the workload's splits) and
        a copy of the cache stepped through the full eviction scan and another split count."""
        from memory_bounded_kv_b200 import kvb_get_error
        from memory_bounded_kv_b200.cache import BoundedKVCache
        w, c = self.w, self.cache
        torch.cuda.synchronize()
        S2 = 4 if self.S == 1 else 1
        c2 = BoundedKVCache(w.B, w.Hq, w.Hkv, w.d, w.cap, w.M, num_splits=S2, with_beta=not self.plain)
        for name in ("k", "v", "pos", "len") + (() if self.plain else ("log_beta",)):
            getattr(c2, name).copy_(getattr(c, name))
        o2, l2 = torch.zeros_like(self.o), torch.zeros_like(self.lse)
        q, kn, vn, lb, t = self._in(i, None)
        self.pre(i)
        self.attn(i)
        c2.insert(kn, vn, lb, t)          # no candidates: the scan
        c2.attend(q, t, o2, l2)
        torch.cuda.synchronize()
        sel = list(range(w.B)) if full else sorted({0, w.B - 1})
        exact = dict(victims=(_np(c.victim), _np(c2.victim)), len=(_np(c.len), _np(c2.len)),
                     pos=(_np(c.pos[sel]), _np(c2.pos[sel])), k=(_np(c.k[sel]), _np(c2.k[sel])))
        return _consistency(exact, _np(self.o), _np(self.lse), _np(o2), _np(l2),
                            f"one step at t={w.t0 + i}: candidates + {self.S} split(s) against the full scan + "
                            f"{S2} split(s); cache bytes of sequences {'all' if full else sel}", kvb_get_error())

    def oracle_sample(self, oracle, nthreads: int, budget_s: float):
        """The oracle as it stands on whole-batch decode steps from the prefill state, the
        (sequence, kv head) units spread over `nthreads` threads; returns (tokens/s, steps)."""
        w = self.w
        c = dict(k=w.k.copy(), v=w.v.copy(), log_beta=None if self.plain else w.log_beta.copy(), pos=w.pos.copy(),
                 len=w.len.copy())
        t0 = time.perf_counter()
        steps = 0
        while True:
            x = w.step_inputs(steps)
            oracle.decode_steps_threads(c, x["q"][None], x["k_new"][None], x["v_new"][None],
                                        None if self.plain else x["log_beta_new"][None], x["t"][None], w.M, nthreads)
            steps += 1
            if time.perf_counter() - t0 > budget_s or steps >= 64:
                break
        return w.B * steps / (time.perf_counter() - t0), steps


class ASMBench:
    """A step: the 256 query tokens' causal self attention over the shared 2048-token cache
    (kvb_decode_attn, batch stride 0: the query-batched kernel) and the memory lookup + merge over
    the memory prepared once at set-up (kvb_asm_prepare, then kvb_asm_lookup_merge_planes)."""

    bound = "tensor"
    KERNEL_SRC = "asm_planes.cuh"
    flush_l2 = True
    # the fp32 contraction runs as three exact bf16 products per element (q . hi + q . mid + q . lo)
    PEAK_NOTE = "{kind} dense bf16 {bf16:.0f} TFLOP/s (bf16_tflops, burst) / 3 bf16 products per fp32 product"

    SPLIT_LEN = 512   # the self attention's splits: a fixed length shared by every query row

    def __init__(self, splits: int = 0, seed=None):
        import memory_bounded_kv_b200 as kvb
        from memory_bounded_kv_b200 import synth
        self.kvb = kvb
        self.key = "4"
        self.w = w = synth.asm_workload(seed=4 if seed is None else seed)
        self.S = splits or 4
        N, H, Hkv, d = w.N, w.H, w.Hkv, w.d
        self.k = _dev(w.k).expand(N, Hkv, w.L, d)
        self.v = _dev(w.v).expand(N, Hkv, w.L, d)
        self.pos = _dev(w.pos).expand(N, Hkv, w.L)
        self.len, self.t = _dev(w.len), _dev(w.t)
        self.q = _dev(w.q)
        self.qbar, self.abar, self.lz = _dev(w.qbar), _dev(w.abar), _dev(w.log_zbar)
        self.o_self = torch.zeros(N, H, d, device="cuda")
        self.l_self = torch.zeros(N, H, device="cuda")
        self.op, self.lp = kvb.decode_workspace(N, H, d, self.S)
        self.out = Packed([("o", (N, H, d), torch.float32), ("lse", (N, H), torch.float32),
                           ("idx", (N, H), torch.int32)])
        self.o, self.lse, self.idx = self.out.views["o"], self.out.views["lse"], self.out.views["idx"]
        self.stage = Packed([("q", (N, H, d), torch.bfloat16)])
        self.ws = torch.empty(kvb.kvb_asm_workspace_bytes(N, H, w.K), dtype=torch.uint8, device="cuda")
        self.planes = kvb.kvb_asm_prepare(self.qbar)   # the memory is static: prepared once, untimed
        self.workload = f"attention-state memory H{H} K{w.K} d{d}, {N} queries, self attention over {w.L}"

    def prepare(self, total_steps):
        pass

    def n_steps(self):
        return None

    def pre(self, i, x=None):
        q = self.q if x is None else x["q"]
        self.kvb.kvb_decode_attn(q, self.k, self.v, None, self.pos, self.len, self.t, self.o_self, self.l_self,
                                 num_splits=self.S, split_len=self.SPLIT_LEN, o_part=self.op, lse_part=self.lp)

    def attn(self, i, x=None):   # the dominant launch: the lookup + merge
        q = self.q if x is None else x["q"]
        w = self.w
        self.kvb.kvb_asm_lookup_merge_planes(q, self.planes, w.H, w.K, self.abar, self.lz, self.o_self, self.l_self,
                                             self.idx, self.o, self.lse, self.ws)

    def post(self, i, x=None):
        pass

    def host_inputs(self, i):
        return {"q": self.w.q}

    def tokens(self, i):
        return self.w.N

    def launches(self, i):
        return 4   # attention + split merge, lookup + state merge

    def attn_bytes(self, i=None):
        """The lookup reads every prepared centroid (three bf16 parts) once and per query its q,
        o_self and ā, and writes o."""
        w = self.w
        return w.H * w.K * w.d * 6 + w.N * w.H * (w.d * 2 + w.d * 4 * 2 + w.d * 2)

    def other_bytes(self, i=None):
        """The self attention reads the shared cache's K and V once, and q."""
        w = self.w
        return w.L * w.Hkv * w.d * 2 * 2 + w.N * w.H * w.d * 2

    def flops(self):
        w = self.w
        return 2.0 * w.N * w.H * w.K * w.d

    def kernel_name(self):
        return "asm_score_planes_kernel + asm_merge_kernel (kvb_asm_lookup_merge_planes)"

    def config(self):
        w = self.w
        return {"workload": self.workload, "N": w.N, "H": w.H, "Hkv": w.Hkv, "K": w.K, "d": w.d, "L": w.L,
                "self_attn_splits": self.S, "seed": w.seed,
                "l2": "flushed before every timed step (256 MiB write): q̄ 64 MiB + ā 32 MiB + K/V 8 MiB fit in L2",
                "parallelism": "replicas"}

    def check(self, i, full: bool):
        """Consistency of the step computed two ways on the GPU: the self attention through the
        query-batched kernel (the timed path) and through the per-row kernel (splits of
        ceil(len / 4) slots); the lookup over the prepared memory (the timed path) and over the
        fp32 centroids (indices compared exactly)."""
        from memory_bounded_kv_b200 import kvb_get_error
        w = self.w
        self.pre(i)
        self.attn(i)
        o_self2, l_self2 = torch.zeros_like(self.o_self), torch.zeros_like(self.l_self)
        self.kvb.kvb_decode_attn(self.q, self.k, self.v, None, self.pos, self.len, self.t, o_self2, l_self2,
                                 num_splits=self.S, split_len=0, o_part=self.op, lse_part=self.lp)
        idx2 = torch.zeros_like(self.idx)
        o2, l2 = torch.zeros_like(self.o), torch.zeros_like(self.lse)
        # the lookup over the fp32 centroids (normalised and split on the fly)
        self.kvb.kvb_asm_lookup_merge(self.q, self.qbar, self.abar, self.lz, o_self2, l_self2, idx2, o2, l2, self.ws)
        torch.cuda.synchronize()
        self_par = _consistency({}, _np(self.o_self), _np(self.l_self), _np(o_self2), _np(l_self2), "self attention", 0)
        res = _consistency(dict(idx=(_np(self.idx), _np(idx2))), _np(self.o), _np(self.lse), _np(o2), _np(l2),
                           "query-batched self attention against the per-row kernel, then the lookup + merge of "
                           "each", kvb_get_error())
        res["self_attention"] = {k: self_par[k] for k in ("max_abs", "rel_l2", "lse_max_abs", "ok")}
        res["ok"] = res["ok"] and self_par["ok"]
        return res


class MementoBench:
    """A step: every active sequence decodes one token (append, attention); after the last token
    of a memento, the finished block's slots are removed in place (kvb_compact_blocks). The
    schedule is finite: timed steps are a spread sample of it, the others run untimed."""

    bound = "hbm"
    KERNEL_SRC = "decode_attn_tc.cuh"
    flush_l2 = True
    # the attention's fixed split length (a multiple of the 64-slot page). Measured on this
    # workload: 256 -> 115 us, 512 -> 90.5 us, 768 -> 86.1 us, 1024 -> 86.7 us, 1536 -> 92.9 us per
    # step (1280: 125 us on a grid sharing a factor 7 with the 14 splits per row, 88.1 us since the
    # library takes a grid coprime with the split count)
    SPLIT_LEN = 768

    def __init__(self, splits: int = 0, seed=None, paged: bool = False):
        from memory_bounded_kv_b200 import synth, _lib
        from memory_bounded_kv_b200.cache import BoundedKVCache, PagedKVCache
        self.paged = paged
        self.key = "5p" if paged else "5"
        self.w = w = synth.memento_workload(seed=5 if seed is None else seed)
        self.S = -(-w.cap // self.SPLIT_LEN)
        if paged:
            self.page = _lib.PAGE_SLOTS
            self.num_pages = w.peak_pages(self.page)
            self.cache = PagedKVCache(w.B, w.Hq, w.Hkv, w.d, max_pages=-(-w.cap // self.page),
                                      num_pages=self.num_pages, M=w.cap, num_splits=self.S,
                                      split_len=self.SPLIT_LEN, with_beta=False)
        else:
            self.cache = BoundedKVCache(w.B, w.Hq, w.Hkv, w.d, w.cap, w.cap, num_splits=self.S,
                                        split_len=self.SPLIT_LEN, with_beta=False)
        self.pool_in = [w.step_inputs(s) for s in range(w.pool)]
        self.q = [_dev(x["q"]) for x in self.pool_in]
        self.kn = [_dev(x["k_new"]) for x in self.pool_in]
        self.vn = [_dev(x["v_new"]) for x in self.pool_in]
        self.out = Packed([("o", (w.B, w.Hq, w.d), torch.float32), ("lse", (w.B, w.Hq), torch.float32)])
        self.o, self.lse = self.out.views["o"], self.out.views["lse"]
        self.stage = Packed([("q", (w.B, w.Hq, w.d), torch.bfloat16), ("k_new", (w.B, w.Hkv, w.d), torch.bfloat16),
                             ("v_new", (w.B, w.Hkv, w.d), torch.bfloat16), ("t", (w.B,), torch.int32),
                             ("rm_start", (w.B,), torch.int32), ("rm_len", (w.B,), torch.int32)])
        self.comp = {}
        for s in w.compaction_steps().tolist():
            self.comp[s] = tuple(_dev(a) for a in w.compaction(s))
        self.active = np.array([(s < w.total).sum() for s in range(w.steps)], np.int64)
        steps = np.arange(w.steps)
        self.t_np = np.where(steps[:, None] < w.total[None, :], steps[:, None], -1).astype(np.int32)
        self.t_dev = torch.from_numpy(self.t_np).cuda()
        self._lens = {}
        self.workload = (f"memento compaction B{w.B} Hq{w.Hq} Hkv{w.Hkv} d{w.d}, 9 x (Geom(1500) block + "
                         f"U[120,180] memento){', paged cache' if paged else ''}")

    def prepare(self, total_steps):
        pass

    def n_steps(self):
        return self.w.steps

    def reset(self):
        if self.paged:
            self.cache.reset()
        else:
            self.cache.len.zero_()
        self.cache.cand_valid = False

    def pre(self, i, x=None):
        p = i % self.w.pool
        kn, vn, t = (self.kn[p], self.vn[p], self.t_dev[i]) if x is None else (x["k_new"], x["v_new"], x["t"])
        self.cache.cand_valid = False   # the cache never reaches its budget: insertion appends
        self.cache.insert(kn, vn, None, t)

    def attn(self, i, x=None):
        p = i % self.w.pool
        q, t = (self.q[p], self.t_dev[i]) if x is None else (x["q"], x["t"])
        self.cache.attend(q, t, self.o, self.lse)

    def post(self, i, x=None):
        if i in self.comp:
            rs, rl = self.comp[i] if x is None else (x["rm_start"], x["rm_len"])
            self.cache.compact(rs, rl)

    def host_inputs(self, i):
        x = self.pool_in[i % self.w.pool]
        rs, rl = self.w.compaction(i) if i in self.comp else (np.zeros(self.w.B, np.int32),) * 2
        return dict(q=x["q"], k_new=x["k_new"], v_new=x["v_new"], t=self.t_np[i], rm_start=rs, rm_len=rl)

    def tokens(self, i):
        return int(self.active[i])

    def launches(self, i):
        return 2 + (self.S > 1) + (1 if i in self.comp else 0)

    def _len(self, i):
        if i not in self._lens:
            self._lens[i] = self.w.cache_len(i)
        return self._lens[i]

    def attn_bytes(self, i=None):
        """K, V and pos of the live slots of step i (pos feeds the eviction candidates), q in,
        o and lse out for the active sequences."""
        w = self.w
        n = int(self._len(i)[i < w.total].sum())
        act = int(self.active[i])
        return n * w.Hkv * (2 * w.d * 2 + 4) + act * w.Hq * w.d * 2 + act * w.Hq * (w.d * 4 + 4)

    def other_bytes(self, i=None):
        """The appended rows, and at a compaction step the moved rows (read and written)."""
        w = self.w
        moved = 0
        if i in self.comp:
            rs, rl = w.compaction(i)
            ln = self._len(i)
            for b in np.nonzero(rl)[0]:
                moved += int(ln[b]) - int(rs[b]) - int(rl[b])
        return int(self.active[i]) * w.Hkv * (2 * w.d * 2 + 4) + moved * w.Hkv * 2 * (2 * w.d * 2 + 4)

    def kernel_name(self):
        entry, paged = ("kvb_paged_decode_attn", ",paged") if self.paged else ("kvb_decode_attn", "")
        return (f"{entry} = decode_attn_tc_kernel<d={self.w.d},G={self.w.Hq // self.w.Hkv},bias=0{paged}> + "
                f"merge_splits_kernel, split_len={self.SPLIT_LEN}")

    def peak_kv_ratio(self):
        """Peak KV slots of a cache that keeps every token over the compacted cache's peak."""
        w = self.w
        prev = np.concatenate([np.zeros((w.B, 1), np.int64), np.cumsum(w.mem, axis=1)[:, :-1]], axis=1)
        return int(w.total.max()) / int((prev + w.blk + w.mem).max())

    def memory(self):
        """Device bytes of K, V and pos: the flat cache reserves cap slots per (sequence, kv head); the
        paged pool holds the schedule's peak page count."""
        w = self.w
        row = 2 * w.d * 2 + 4
        flat = w.B * w.Hkv * w.cap * row
        out = {"flat_reserved_bytes": flat}
        if self.paged:
            out.update(pool_pages=self.num_pages, pool_bytes=self.num_pages * self.page * row,
                       flat_over_paged=round(flat / (self.num_pages * self.page * row), 3))
        return out

    def config(self):
        w = self.w
        return {"workload": self.workload, "B": w.B, "cap": w.cap, "split_len": self.SPLIT_LEN,
                "num_splits": self.S, "schedule_steps": w.steps, "seed": w.seed, "parallelism": "replicas",
                "timed_steps": "a spread sample of the schedule (every other step runs untimed, in order)",
                "peak_kv_full_over_compacted": round(self.peak_kv_ratio(), 3), "memory": self.memory(),
                "l2": "flushed before every timed step (256 MiB write): the live caches grow from "
                      "a few MB to ~350 MB over the schedule"}

    def dump_step(self, i, path):
        """The cache before schedule step i and its inputs (the compaction only at a compaction step)."""
        from memory_bounded_kv_b200.state import dump_step
        x = self.host_inputs(i)
        if i not in self.comp:
            x.pop("rm_start"), x.pop("rm_len")
        dump_step(path, self.cache, x, extra_meta={"workload": self.workload, "step": int(i)})

    def check(self, i, full: bool):
        """Consistency of schedule step i: the timed path (eviction candidates, splits of 512
        slots) against the same step on a copy of the cache with one split."""
        from memory_bounded_kv_b200 import kvb_get_error
        c = self.cache
        torch.cuda.synchronize()
        o2, l2 = torch.zeros_like(self.o), torch.zeros_like(self.lse)
        p = i % self.w.pool
        self.pre(i)
        self.attn(i)
        if self.paged:
            from memory_bounded_kv_b200 import kvb_paged_decode_attn
            kvb_paged_decode_attn(c.pool, self.q[p], self.t_dev[i], o2, l2, num_splits=1)
        else:
            from memory_bounded_kv_b200 import kvb_decode_attn
            kvb_decode_attn(self.q[p], c.k, c.v, None, c.pos, c.len, self.t_dev[i], o2, l2, num_splits=1)
        self.post(i)
        torch.cuda.synchronize()
        return _consistency({}, _np(self.o), _np(self.lse), _np(o2), _np(l2),
                            f"schedule step {i}: {self.S} splits of {self.SPLIT_LEN} slots against one split",
                            kvb_get_error())


def make_bench(key: str, splits: int, seed):
    if key in ("1", "2", "3", "3p"):
        return DecodeBench(int(key[0]), splits, seed, plain=key.endswith("p"))
    if key == "4":
        return ASMBench(splits, seed)
    return MementoBench(splits, seed, paged=key.endswith("p"))


# ----------------------------------------------------------------------------------------------
# timing driver
# ----------------------------------------------------------------------------------------------

def time_graphs(graphs, flush, world):
    """Per-graph device times (ms): each replay bracketed by events, after a 256 MiB write that
    flushes L2 (outside the events) when `flush` is given."""
    barrier(world)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in graphs]
    for (a, b), g in zip(ev, graphs):
        if flush is not None:
            flush.fill_(1)
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    barrier(world)
    return [a.elapsed_time(b) for a, b in ev]


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


def pct(xs):
    a = np.asarray(xs, np.float64)
    return {"p10": float(np.percentile(a, 10)), "p50": float(np.percentile(a, 50)),
            "p90": float(np.percentile(a, 90)), "n": int(a.size)}


def measure(bench, K, W, world, e2e: bool):
    """Times one workload: the main region (inputs resident in HBM), a region with events around
    the dominant launch's own graph, per-step times, and the e2e region (inputs from pinned host
    memory, outputs read back). Returns the times and which steps each region ran."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if bench.flush_l2 else None
    n = bench.n_steps()
    KR = min(K, 200)
    E = min(K, 200)
    P = 0 if bench.flush_l2 else min(K, 200)

    def full_step(i, x=None):
        bench.pre(i, x)
        bench.attn(i, x)
        bench.post(i, x)

    if n is None:
        # positions continue: warm-up, main, kernel, per-step, e2e warm-up and e2e regions follow
        # one another; `nxt` is the first position no region used
        bounds = np.cumsum([0, W, K, KR, P, E, E])
        main, kern, per_step, warm_e2e, e2e_steps = (list(range(bounds[j], bounds[j + 1])) for j in range(1, 6))
        nxt = int(bounds[-1])
        bench.prepare(nxt + 1)
        for i in range(W):
            full_step(i)
        torch.cuda.synchronize()
    else:
        # a finite schedule: a spread sample of its steps is timed in each pass, the rest run untimed
        stride = max(1, n // K)
        main = list(range(stride // 2, n, stride))[:K]
        kern, e2e_steps, warm_e2e, per_step = main[:KR], main[:E], [], []
        nxt = main[len(main) // 2]

    def schedule_pass(timed: dict):
        """Runs the whole schedule from an empty cache; at the steps in `timed` calls their timer."""
        log(f"{bench.key}: schedule pass of {n} steps")
        bench.reset()
        torch.cuda.synchronize()
        for i in range(n):
            if i in timed:
                timed[i]()
            else:
                full_step(i)
        torch.cuda.synchronize()

    # ---- main region: device-resident inputs
    log(f"{bench.key}: main region ({len(main)} steps)")
    step_ms = None
    if n is None:
        if bench.flush_l2:
            graphs = [capture(lambda i=i: full_step(i)) for i in main]
            step_ms = time_graphs(graphs, flush, world)
            ms = sum(step_ms)
        else:
            chunk = 500
            graphs = [capture(lambda c=main[j:j + chunk]: [full_step(i) for i in c])
                      for j in range(0, len(main), chunk)]
            ms = time_region(lambda: [g.replay() for g in graphs], world)
        del graphs
    else:
        graphs = {i: capture(lambda i=i: full_step(i)) for i in main}
        step_ms = []
        barrier(world)
        schedule_pass({i: (lambda g=graphs[i]: step_ms.extend(time_graphs([g], flush, 1))) for i in main})
        barrier(world)
        ms = sum(step_ms)
        del graphs

    # ---- kernel region: the dominant launch in its own graph, events around it
    log(f"{bench.key}: kernel region ({len(kern)} launches)")
    parts = {}
    for i in kern:   # captured in step order, so each step sees the cache bookkeeping of the one before
        parts[i] = (capture(lambda i=i: bench.pre(i)), capture(lambda i=i: bench.attn(i)),
                    capture(lambda i=i: bench.post(i)))
    kern_ms = []

    def kernel_step(i):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if flush is not None:
            flush.fill_(1)
        parts[i][0].replay()
        a.record()
        parts[i][1].replay()
        b.record()
        parts[i][2].replay()
        kern_ev.append((a, b))

    kern_ev = []
    barrier(world)
    if n is None:
        torch.cuda.synchronize()
        for i in kern:
            kernel_step(i)
        torch.cuda.synchronize()
    else:
        schedule_pass({i: (lambda i=i: kernel_step(i)) for i in kern})
    barrier(world)
    kern_ms = [a.elapsed_time(b) for a, b in kern_ev]
    del parts

    # ---- per-step times of a workload timed as one graph: each step its own graph
    if step_ms is None:
        graphs = [capture(lambda i=i: full_step(i)) for i in per_step]
        step_ms = time_graphs(graphs, None, world)
        del graphs

    # ---- e2e region: each step's inputs from pinned host memory (one packed copy), its outputs
    # read back (one copy), the step in between. A workload timed as one graph of many steps
    # (larger than L2) is timed the same way here: all steps in one graph, the copies on their own
    # streams and double-buffered, so that a step's copies overlap its neighbours' kernels; the
    # others are timed step by step, each step one graph after an L2 flush.
    e2e_ms = None
    if e2e and n is None and not bench.flush_l2:
        log(f"{bench.key}: e2e region ({len(e2e_steps)} steps, copies overlapped)")
        e2e_ms = e2e_pipelined(bench, warm_e2e, e2e_steps, world)
    elif e2e:
        log(f"{bench.key}: e2e region ({len(e2e_steps)} steps)")
        rows = warm_e2e + e2e_steps
        h_in = torch.empty(len(rows), bench.stage.nbytes, dtype=torch.uint8).pin_memory()
        for j, i in enumerate(rows):
            bench.stage.fill_host(h_in[j], bench.host_inputs(i))
        h_out = torch.empty(bench.out.nbytes, dtype=torch.uint8).pin_memory()
        row_of = {i: j for j, i in enumerate(rows)}

        def e2e_step(i):
            bench.stage.dev.copy_(h_in[row_of[i]], non_blocking=True)
            full_step(i, bench.stage.views)
            h_out.copy_(bench.out.dev, non_blocking=True)

        for i in warm_e2e:   # warm-up through the same path
            e2e_step(i)
        torch.cuda.synchronize()
        graphs = {i: capture(lambda i=i: e2e_step(i)) for i in e2e_steps}
        if n is None:
            if bench.flush_l2:
                e2e_ms = sum(time_graphs([graphs[i] for i in e2e_steps], flush, world))
            else:
                e2e_ms = time_region(lambda: [graphs[i].replay() for i in e2e_steps], world)
        else:
            acc = []
            barrier(world)
            schedule_pass({i: (lambda g=graphs[i]: acc.extend(time_graphs([g], flush, 1))) for i in e2e_steps})
            barrier(world)
            e2e_ms = sum(acc)
        del graphs
    if n is not None:   # leave the cache as it was just before `nxt`, for the parity check
        bench.reset()
        for i in range(nxt):
            full_step(i)
        torch.cuda.synchronize()
    return dict(main=main, ms=ms, step_ms=step_ms, kern=kern, kern_ms=kern_ms, e2e_steps=e2e_steps,
                e2e_ms=e2e_ms, next=nxt)


def e2e_pipelined(bench, warm, steps, world):
    """Device time of `steps` decode steps through the public calls, each with its inputs copied
    from pinned host memory and its outputs copied back, captured as one CUDA graph: copies in on
    one stream, the step on the capturing stream, copies out on a third; inputs and outputs
    double-buffered. Step j's copy in waits for step j - 2's kernels (its buffer), step j waits for
    its copy in and for step j - 2's copy out (its output buffer), the copy out waits for step j."""
    rows = warm + steps
    stage = [bench.stage, Packed([(k, v[2], v[3]) for k, v in bench.stage.offsets.items()])]
    outb = [bench.out, Packed([(k, v[2], v[3]) for k, v in bench.out.offsets.items()])]
    h_in = torch.empty(len(rows), bench.stage.nbytes, dtype=torch.uint8).pin_memory()
    for j, i in enumerate(rows):
        bench.stage.fill_host(h_in[j], bench.host_inputs(i))
    h_out = torch.empty(2, bench.out.nbytes, dtype=torch.uint8).pin_memory()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def views(j):
        v = dict(stage[j % 2].views)
        v.update(outb[j % 2].views)
        return v

    def run(idx):
        cap = torch.cuda.current_stream()
        s_in.wait_stream(cap)
        s_out.wait_stream(cap)
        ev_comp, ev_in, ev_out = {}, {}, {}
        for j, i in enumerate(idx):
            b = j % 2
            with torch.cuda.stream(s_in):
                if j >= 2:
                    s_in.wait_event(ev_comp[j - 2])
                stage[b].dev.copy_(h_in[rows.index(i)], non_blocking=True)
                ev_in[j] = torch.cuda.Event()
                ev_in[j].record(s_in)
            cap.wait_event(ev_in[j])
            if j >= 2:
                cap.wait_event(ev_out[j - 2])
            bench.pre(i, views(j))
            bench.attn(i, views(j))
            bench.post(i, views(j))
            ev_comp[j] = torch.cuda.Event()
            ev_comp[j].record(cap)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[j])
                h_out[b].copy_(outb[b].dev, non_blocking=True)
                ev_out[j] = torch.cuda.Event()
                ev_out[j].record(s_out)
        cap.wait_stream(s_in)
        cap.wait_stream(s_out)

    run(warm)                      # warm-up through the same path (not captured)
    torch.cuda.synchronize()
    g = capture(lambda: run(steps))
    ms = time_region(g.replay, world)
    del g
    return ms


def report(bench, m, world, hbm_peak, peak_kind):
    """The JSON fields of one workload from its measurement."""
    main, K = m["main"], len(m["main"])
    ms = max_over_ranks(m["ms"], world)
    kms = max_over_ranks(statistics.mean(m["kern_ms"]), world)
    value = replica_value(sum(bench.tokens(i) for i in main), world, ms)
    src = kernel_src_hash(bench.KERNEL_SRC)
    if bench.bound == "tensor":
        bf16_tf, bf16_kind = bf16_peak()
        peak_tf = bf16_tf / 3.0
        achieved = bench.flops() / (kms / 1e3) / 1e12
        roofline = {"bound": "tensor", "kernel": bench.kernel_name(), "achieved": achieved, "peak": peak_tf,
                    "unit": "TFLOP/s", "frac": achieved / peak_tf,
                    "peak_source": ASMBench.PEAK_NOTE.format(kind=bf16_kind, bf16=bf16_tf),
                    "traffic": MEASURED_TRAFFIC.get((src, bench.key, getattr(bench, "S", 0))),
                    "algorithmic_flops_per_launch": bench.flops(), "kernel_ms_avg": kms,
                    "launches_timed": len(m["kern_ms"])}
    else:
        # launches of a finite schedule differ in size: bytes over time summed over the same launches
        kb = [bench.attn_bytes(i) for i in m["kern"]]
        achieved = sum(kb) / (max_over_ranks(sum(m["kern_ms"]), world) / 1e3) / 1e9
        roofline = {"bound": "hbm", "kernel": bench.kernel_name(), "achieved": achieved, "peak": hbm_peak,
                    "unit": "GB/s", "frac": achieved / hbm_peak, "peak_source": f"{peak_kind} (hbm_gbs)",
                    "traffic": MEASURED_TRAFFIC.get((src, bench.key, getattr(bench, "S", 0))),
                    "algorithmic_bytes_per_launch": statistics.mean(kb), "kernel_ms_avg": kms,
                    "launches_timed": len(m["kern_ms"])}
    step_bytes = sum(bench.attn_bytes(i) + bench.other_bytes(i) for i in main)
    kv_gbs = step_bytes / (ms / 1e3) / 1e9
    out = {"value": value, "unit": "tokens/s", "steps": K, "ms_per_step": ms / K, "kv_gbs": kv_gbs,
           "kv_frac_of_hbm_peak": kv_gbs / hbm_peak, "roofline": roofline,
           "step_ms_percentiles": pct(m["step_ms"]) if m["step_ms"] else None,
           "gpu_launches": sum(bench.launches(i) for i in main), "kernel_src_sha256_16": src}
    if m["e2e_ms"] is not None:
        E = len(m["e2e_steps"])
        e2e_ms = max_over_ranks(m["e2e_ms"], world)
        out["e2e"] = {"value": replica_value(sum(bench.tokens(i) for i in m["e2e_steps"]), world, e2e_ms),
                      "unit": "tokens/s", "h2d_bytes_per_step": bench.stage.payload,
                      "d2h_bytes_per_step": bench.out.payload, "ms_per_step": e2e_ms / E, "steps": E,
                      "copies": ("one packed host-to-device copy of the step's inputs and one device-to-host copy "
                                 "of its outputs per step; all steps in one CUDA graph, the copies on their own "
                                 "streams, double-buffered, overlapping the neighbouring steps' kernels"
                                 if (bench.n_steps() is None and not bench.flush_l2) else
                                 "one packed host-to-device copy of the step's inputs and one device-to-host copy "
                                 "of its outputs per step, inside each step's CUDA graph, after an L2 flush")}
    return out


def oracle_baseline(bench, budget_s: float):
    """The oracle as it stands on a bounded sample of the workload: on every host core (its
    parallel driver over independent (sequence, kv head) units) and on one core."""
    import oracle
    oracle.build()
    cores = host_cores()
    v_all, n_all = bench.oracle_sample(oracle, cores, budget_s)
    v_one, n_one = bench.oracle_sample(oracle, 1, budget_s / 3)
    w = bench.w
    return {"value": v_all, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n_all} whole-batch decode steps (B={w.B}) from the prefill state, the (sequence, kv head) "
                      f"units spread over {cores} threads",
            "cpu_model": cpu_model(),
            "single_core": {"value": v_one, "unit": "tokens/s", "cores": 1,
                            "sample": f"{n_one} whole-batch decode steps from the prefill state"}}


def run_workload(key, splits, args, world, local, K, W, hbm_peak, peak_kind, cpu_baseline: bool):
    clocks = ClockSampler(local)
    clocks.start()
    log(f"{key}: set-up")
    bench = make_bench(key, splits, args.seed)
    m = measure(bench, K, W, world, not args.no_e2e)
    clk = clocks.stop()
    r = report(bench, m, world, hbm_peak, peak_kind)
    r["config"] = bench.config()
    r["config"]["timed_launches"] = "cuda graph replay"
    r["clocks"] = clk
    if args.dump_state and hasattr(bench, "dump_step"):
        path = os.path.join(args.dump_state, key)
        log(f"{key}: dumping the state before step {m['next']} to {path}")
        bench.dump_step(m["next"], path)
    if args.check != "off":
        log(f"{key}: consistency check")
        r["consistency"] = bench.check(m["next"], args.check == "full")
    if cpu_baseline and hasattr(bench, "oracle_sample"):
        log(f"{key}: oracle baseline")
        r["cpu_baseline"] = oracle_baseline(bench, 12.0)
    log(f"{key}: done")
    del bench
    torch.cuda.empty_cache()
    return r


# ----------------------------------------------------------------------------------------------
# profiling cases: the dominant launches of each workload at its shape, a few times
# ----------------------------------------------------------------------------------------------

def _profile_decode(B, Hq, Hkv, d, cap, lens, S, split_len, bias, reps=4, fused=False):
    """kvb_decode_attn over a filled cache (K, V ~ N(0, 1), log beta ~ U(-3, -0.01), positions 0..cap-1)
    with the given lengths, `reps` times. `fused` (a full cache): one attention that leaves the
    eviction records, then `reps` decode steps of kvb_decode_step (insertion inside the launch)."""
    import memory_bounded_kv_b200 as kvb
    from memory_bounded_kv_b200.cache import BoundedKVCache
    g = torch.Generator(device="cuda").manual_seed(0)
    c = BoundedKVCache(B, Hq, Hkv, d, cap, cap, num_splits=S, split_len=split_len, with_beta=bias)
    c.k.normal_(generator=g)
    c.v.normal_(generator=g)
    if bias:
        c.log_beta.uniform_(-3, -0.01, generator=g)
    c.pos.copy_(torch.arange(cap, dtype=torch.int32, device="cuda").expand(B, Hkv, cap))
    c.len.copy_(torch.as_tensor(lens, dtype=torch.int32, device="cuda"))
    q = torch.randn(B, Hq, d, device="cuda", generator=g).to(torch.bfloat16)
    t = torch.full((B,), cap + 1, dtype=torch.int32, device="cuda")
    o = torch.zeros(B, Hq, d, device="cuda")
    lse = torch.zeros(B, Hq, device="cuda")
    if fused:
        c.full = True
        kn = torch.randn(B, Hkv, d, device="cuda", generator=g).to(torch.bfloat16)
        vn = torch.randn(B, Hkv, d, device="cuda", generator=g).to(torch.bfloat16)
        lbn = torch.full((B, Hkv), -0.5, device="cuda") if bias else None
        c.attend(q, t, o, lse)
        for r in range(reps):
            c.step(q, kn, vn, lbn, t + 1 + r, o, lse)
    else:
        for _ in range(reps):
            c.attend(q, t, o, lse)
    torch.cuda.synchronize()
    return kvb.kvb_get_error()


def _profile_c2():
    """The Qwen3-8B-shaped layer: 32 x 8 rows of 4096 slots, one split; an attention, then fused
    decode steps (the bench's steady state)."""
    return _profile_decode(32, 32, 8, 128, 4096, np.full((32, 8), 4096), 1, 0, True, fused=True)


def _profile_c3():
    """The long-context workload: 4 x 8 rows of 8192 slots, 64 splits; an attention, then fused
    decode steps."""
    return _profile_decode(4, 32, 8, 128, 8192, np.full((4, 8), 8192), 64, 0, True, fused=True)


def _profile_c5():
    """A mid-schedule memento cache: 64 x 8 rows, ragged lengths U[300, 3000), splits of 768 slots."""
    lens = np.repeat(np.random.default_rng(0).integers(300, 3000, 64)[:, None], 8, axis=1)
    return _profile_decode(64, 32, 8, 128, 3072, lens, 4, 768, False)


def _profile_c4():
    """The attention-state-memory step: shared-prefix self attention (4 splits of 512) and the lookup
    over the prepared memory, four times."""
    import memory_bounded_kv_b200 as kvb
    from memory_bounded_kv_b200 import synth
    w = synth.asm_workload()
    N, H, Hkv, d = w.N, w.H, w.Hkv, w.d
    k, v, pos = _dev(w.k).expand(N, Hkv, w.L, d), _dev(w.v).expand(N, Hkv, w.L, d), _dev(w.pos).expand(N, Hkv, w.L)
    q, ln, t = _dev(w.q), _dev(w.len), _dev(w.t)
    o_self = torch.zeros(N, H, d, device="cuda")
    l_self = torch.zeros(N, H, device="cuda")
    op, lp = kvb.decode_workspace(N, H, d, 4)
    planes = kvb.kvb_asm_prepare(_dev(w.qbar))
    abar, lz = _dev(w.abar), _dev(w.log_zbar)
    idx = torch.zeros(N, H, dtype=torch.int32, device="cuda")
    o = torch.zeros(N, H, d, device="cuda")
    lse = torch.zeros(N, H, device="cuda")
    ws = torch.empty(kvb.kvb_asm_workspace_bytes(N, H, w.K), dtype=torch.uint8, device="cuda")
    for _ in range(4):
        kvb.kvb_decode_attn(q, k, v, None, pos, ln, t, o_self, l_self, num_splits=4, split_len=512, o_part=op,
                            lse_part=lp)
        kvb.kvb_asm_lookup_merge_planes(q, planes, H, w.K, abar, lz, o_self, l_self, idx, o, lse, ws)
    torch.cuda.synchronize()
    return kvb.kvb_get_error()


PROFILE_CASES = {"c2": _profile_c2, "c3": _profile_c3, "c4": _profile_c4, "c5": _profile_c5}


def run_profile(case):
    err = PROFILE_CASES[case]()
    return {"profile": case, "device_error": err}


def run_replay(path):
    """One dumped step through the library: its outputs and the cache after it go to
    path/replayed (same format), with the device error word."""
    from memory_bounded_kv_b200 import kvb_get_error
    from memory_bounded_kv_b200 import state
    cache, inputs, meta = state.load_step(path)
    o, lse = state.replay_step(cache, inputs)
    torch.cuda.synchronize()
    err = kvb_get_error()
    tensors, _ = state.cache_state(cache)
    tensors = dict(tensors, out_o=o, out_lse=lse)
    out = os.path.join(path, "replayed")
    state.save(out, tensors, dict(meta, device_error=err))
    return {"replay": path, "written": out, "device_error": err, "workload": meta.get("extra", {}).get("workload"),
            "o_finite": bool(torch.isfinite(o).all().item()), "lse_finite": bool(torch.isfinite(lse).all().item())}


def run_kvb(args, world, rank, local):
    hbm_peak, peak_kind = peaks()
    key = f"{args.config}{'p' if (args.plain and args.config == 3) or (args.paged and args.config == 5) else ''}"
    W = max(3, args.warmup)
    head = run_workload(key, args.splits, args, world, local, args.steps, W, hbm_peak, peak_kind,
                        rank == 0 and world == 1 and not args.no_cpu_baseline)
    out = {
        "metric": METRIC,
        "value": head.pop("value"),
        "unit": head.pop("unit"),
        "n_gpus": world,
        "steps": head.pop("steps"),
        "warmup": W,
        "ms_per_step": head.pop("ms_per_step"),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "storage_dtype": "bf16",
        "data": "synthetic (seeded; shapes and distributions of the workload)",
        "config": head.pop("config"),
    }
    out.update(head)
    spec = args.configs.strip().lower()
    subs = [] if spec == "none" else (list(WORKLOADS) if spec == "all" else [s.strip() for s in spec.split(",")])
    subs = [s for s in subs if s and s != key]
    if subs:
        out["configs"] = {}
        for sk in subs:
            out["configs"][sk] = run_workload(sk, 0, args, world, local, min(args.steps, 48), min(W, 8),
                                              hbm_peak, peak_kind, False)
    return out


def run_reference(args, world, rank):
    """The oracle as it stands, timed on the host cores, on the workload's metric (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    from memory_bounded_kv_b200 import synth
    w = synth.decode_workload(2 if args.config not in (1, 3) else args.config, seed=args.seed)
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
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample,
                         "cpu_model": cpu_model()},
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
        out[name] = sum(time_graphs([graph] * iters, flush, 1)) / iters
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
    if args.replay:
        print(json.dumps(run_replay(args.replay)), flush=True)
        return
    if args.profile:
        out = run_profile(args.profile)
        print(json.dumps(out), flush=True)
        if out["device_error"]:
            sys.exit(1)
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
