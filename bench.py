"""Benchmark of the B200 grouped-query attention forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one forward pass (gqa_attn_fwd through the C ABI) over one batch of the
workload, with the inputs already resident in HBM.  The default workload is the
largest single-GPU configuration, the Llama-3.1-8B-shaped causal prefill (llama:
B=4, Hq=32, Hkv=8, S=8192, D=128, bf16); others: encoder (B=64, Hq=48, Hkv=12,
S=512, D=64, non-causal), llama_stress (q x 4),
decode_b{1,16,64,128,256} (Sq=1, Sk=32768, split-KV), decode_paged_bN (the same
cache in shuffled pages of 256 keys, gqa_attn_kvcache), decode_fp8_bN (that cache in
e4m3), varlen (32 packed causal sequences of 128..8192 tokens), bigbird (the Llama
shape, non-causal, with a BigBird-style block pattern over 128-blocks,
gqa_attn_blocksparse), llama_bwd (the backward pass of the Llama shape: dQ, dK, dV,
gqa_attn_backward; llama_bwd_b1: one batch element of it).  Prefill workloads report TFLOP/s, decode GB/s.

Under torchrun every rank runs its own copy of the workload (independent batches,
no collective on the data path: weak scaling); the time is the max over ranks.
``--impl reference`` times the float64 CPU oracle on a bounded sample of the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import pathlib
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = pathlib.Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "GQA attn fwd TFLOP/s (prefill) & KV-read GB/s (decode), % roofline, 1×B200"
L2_BYTES = 126 * 2**20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 data-sheet figures: dense bf16 tensor peak (e4m3: twice that) and HBM3e bandwidth;
# the lines report their fraction of these beside the measured-peak fraction
SPEC_PEAKS = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}
_FWD_SOURCES = ("sm100_ptx.cuh", "prefill_sm100.cuh", "decode.cuh", "gqa_attn.cu")
# the sources each timed kernel is built from (its traffic line is keyed by their hash)
KERNEL_SOURCES = {"forward": _FWD_SOURCES,
                  "backward": _FWD_SOURCES + ("backward.cuh", "backward_host.cuh")}


# ----------------------------------------------------------------------------- helpers
def kernel_source_hash(kernel: str = "") -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES["backward" if kernel.startswith("bwd") else "forward"]:
        h.update((ROOT / "exact_attention_gqa_b200" / "csrc" / f).read_bytes())
    return h.hexdigest()[:12]


def fp8_decode_splits(units: int, nblk: int, slots: int) -> int:
    """Split count the library picks for the e4m3 decode: the n in [1, min(64, nblk / 4)]
    with the shortest estimated makespan, ceil(units * pieces / slots) * (blocks per
    split + 3), over two resident CTAs per SM (ties: fewer splits)."""
    best_n, best = 1, None
    for n in range(1, max(1, min(64, nblk // 4)) + 1):
        bps = -(-nblk // n)
        pieces = -(-nblk // bps)
        cost = -(-(units * pieces) // slots) * (bps + 3)
        if best is None or cost < best:
            best_n, best = n, cost
    return best_n


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if still current."""
    f = ROOT / "profiles" / "dram_traffic.txt"
    if not f.exists():
        return None
    src = kernel_source_hash(kernel)
    for line in f.read_text().splitlines():
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == workload \
                and parts[1] == kernel and parts[2] == src:
            return float(parts[3])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.tmp = False

    def __enter__(self):
        # the raw samples go to GQA_CLOCKS_DIR when set (kept for inspection), else to a
        # temporary file; the JSON line carries their summary either way
        out_dir = os.environ.get("GQA_CLOCKS_DIR")
        name = f"clocks_rank{os.environ.get('RANK', '0')}.csv"
        if out_dir:
            pathlib.Path(out_dir).mkdir(parents=True, exist_ok=True)
            self.path = pathlib.Path(out_dir) / name
        else:
            fd, tmp = tempfile.mkstemp(prefix="gqa_", suffix="_" + name)
            os.close(fd)
            self.path = pathlib.Path(tmp)
            self.tmp = True
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        text = self.path.read_text() if self.path and self.path.exists() else ""
        if self.tmp and self.path:
            self.path.unlink(missing_ok=True)
        if self.proc is None or not text:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        rows = []
        for line in text.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        loaded = [r for r in rows if r[2] > 300.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3][1:5])
                          if v.lower() in ("active", "1")})
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(loaded)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value of x over all ranks (the slowest rank decides the time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- workloads
def workload_by_name(name: str):
    if name == "encoder":
        return W.ENCODER
    if name == "llama":
        return W.LLAMA
    if name == "llama_stress":
        return W.LLAMA_STRESS
    if name == "llama_window":
        return W.LLAMA_WINDOW
    if name == "varlen":
        return W.VARLEN
    if name == "bigbird":
        return W.BIGBIRD
    if name == "bigbird_varlen":
        return W.BIGBIRD_VARLEN
    if name == "llama_fp8":
        return W.LLAMA_FP8
    if name == "llama_bwd":
        return W.LLAMA_BWD
    if name == "llama_bwd_b1":
        return W.LLAMA_BWD_B1
    if name.startswith("decode_b"):
        return W.decode(int(name[len("decode_b"):]), num_splits=0)
    if name.startswith("decode_paged_b"):
        return W.decode_paged(int(name[len("decode_paged_b"):]))
    if name.startswith("decode_fp8_b"):
        return W.decode_fp8(int(name[len("decode_fp8_b"):]))
    raise SystemExit(f"unknown workload {name}")


class Case:
    """Device tensors, the work accounting and a zero-argument step for one workload."""

    def __init__(self, w: W.Workload, device, rank: int):
        import exact_attention_gqa_b200 as G
        self.G = G
        self.w = w
        self.device = device
        self.decode = w.Sq == 1
        self.varlen = bool(w.varlen)
        self.paged = w.page_size > 0
        if self.decode:
            q = W.make_decode_q(w, device=device)
            # rotate several KV copies when one is not larger than L2
            kv_bytes = W.kv_cache_bytes(w.B, w.Sk, w.Hkv, w.D)
            n_copies = 1 if kv_bytes > 2 * L2_BYTES else 3
            self.kv = []
            if self.paged:
                self.table = W.page_table(w).to(device)
                self.lens = torch.full((w.B,), w.Sk, dtype=torch.int32, device=device)
            for c in range(n_copies):
                if self.paged:
                    self.kv.append(W.make_paged_kv(w, self.table, device=device))
                    continue
                k = torch.empty(w.B, w.Sk, w.Hkv, w.D, device=device,
                                dtype=torch.float8_e4m3fn if w.kv_fp8 else torch.bfloat16)
                v = torch.empty_like(k)
                W.fill_decode_kv(w, k, v)
                self.kv.append((k, v))
            self.q = q
            rc, kern, splits, pack = G.gqa_attn_plan(w.B, w.Hq, w.Hkv, 1, w.Sk, w.D,
                                                     num_splits=w.num_splits,
                                                     pack_gqa=w.pack_gqa)
            if w.kv_fp8 and w.num_splits == 0:
                # the e4m3 path's own automatic count (the library's rule, restated)
                sms = torch.cuda.get_device_properties(device).multi_processor_count
                splits = fp8_decode_splits(w.B * w.Hkv * (1 if pack else w.G),
                                           (w.Sk + 63) // 64, 2 * sms)
            self.splits, self.pack = splits, pack
            self.bytes = W.decode_bytes(w.B, w.Hq, w.Hkv, w.Sk, w.D,
                                        kv_elt=1 if w.kv_fp8 else 2)
            self.flops = W.attention_flops(w.B, w.Hq, 1, w.Sk, w.D, False)
            self.units, self.unit = self.bytes / 1e9, "GB/s"
            self.launches_per_step = 2 if splits > 1 else 1
            self.kernel = "decode_split_sm100"
        elif w.backward:
            q, k, v = W.make_qkv(w, device=device)
            self.q, self.kv = q, [(k, v)]
            self.do = W.make_dout(w, device=device)
            self.fwd_out, self.fwd_lse = G.gqa_attn(q, k, v, causal=w.causal)
            self.grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
            # the backward's five products against the forward's two
            self.flops = int(2.5 * W.attention_flops(w.B, w.Hq, w.Sq, w.Sk, w.D, w.causal))
            self.units, self.unit = self.flops / 1e12, "TFLOP/s"
            self.launches_per_step = 3
            self.kernel = "bwd_tc"
            self.splits, self.pack = 1, 0
        elif w.qkv_fp8:
            q8, k8, v8 = W.make_qkv_e4m3(w, device=device)
            self.q, self.kv = q8, [(k8, v8)]
            self.flops = W.attention_flops(w.B, w.Hq, w.Sq, w.Sk, w.D, w.causal)
            self.units, self.unit = self.flops / 1e12, "TFLOP/s"
            self.launches_per_step = 1
            self.kernel = "prefill_fwd_sm100"
            self.splits, self.pack = 1, 1
        elif w.block_sparse and self.varlen:
            lengths = W.varlen_lengths(w)
            q, k, v, cu = W.make_varlen(w, device=device, lengths=lengths)
            self.q, self.kv, self.cu = q, [(k, v)], cu.to(device)
            self.max_len = int(lengths.max())
            self.lengths = lengths
            rp, col = W.bigbird_pattern_varlen(lengths.tolist(), w.block_sparse,
                                               seed=w.seed + 101)
            self.rp, self.col = rp.to(device), col.to(device)
            self.plan = G.gqa_attn_blocksparse_varlen_plan(cu, rp, Hq=w.Hq, Hkv=w.Hkv,
                                                           max_seqlen=self.max_len,
                                                           device=device)
            self.flops = W.blocksparse_varlen_flops(lengths.tolist(), rp, col, w.Hq, w.D)
            self.units, self.unit = self.flops / 1e12, "TFLOP/s"
            self.launches_per_step = 1
            self.kernel = "prefill_fwd_sm100"
            self.splits, self.pack = 1, 1
        elif w.block_sparse:
            q, k, v = W.make_qkv(w, device=device)
            self.q, self.kv = q, [(k, v)]
            rp, col = W.bigbird_pattern(w)
            self.rp, self.col = rp.to(device), col.to(device)
            self.flops = W.blocksparse_flops(w, rp, col)
            self.units, self.unit = self.flops / 1e12, "TFLOP/s"
            self.launches_per_step = 1
            self.kernel = "prefill_fwd_sm100"
            self.splits, self.pack = 1, 1
        elif self.varlen:
            lengths = W.varlen_lengths(w)
            q, k, v, cu = W.make_varlen(w, device=device, lengths=lengths)
            self.q, self.kv, self.cu = q, [(k, v)], cu.to(device)
            self.max_len = int(lengths.max())
            self.lengths = lengths
            self.flops = W.varlen_flops(lengths.tolist(), w.Hq, w.D, True)
            self.units, self.unit = self.flops / 1e12, "TFLOP/s"
            self.launches_per_step = 1
            self.kernel = "prefill_fwd_sm100"
            self.splits, self.pack = 1, 1
        else:
            q, k, v = W.make_qkv(w, device=device)
            self.q, self.kv = q, [(k, v)]
            self.flops = W.attention_flops(w.B, w.Hq, w.Sq, w.Sk, w.D, w.causal, w.window)
            self.units, self.unit = self.flops / 1e12, "TFLOP/s"
            self.launches_per_step = 1
            self.kernel = "prefill_fwd_sm100"
            rc, kern, self.splits, self.pack = G.gqa_attn_plan(w.B, w.Hq, w.Hkv, w.Sq, w.Sk,
                                                               w.D, causal=w.causal,
                                                               pack_gqa=w.pack_gqa)
        self.out = torch.empty(self.q.shape, dtype=torch.bfloat16, device=device)
        if self.varlen:
            self.lse = torch.empty(w.Hq, self.q.shape[0], dtype=torch.float32, device=device)
        else:
            self.lse = torch.empty(self.q.shape[0], w.Hq, self.q.shape[1], dtype=torch.float32,
                                   device=device)
        self.i = 0

    def in_bytes(self):
        k, v = self.kv[0]
        b = (self.q.numel() * self.q.element_size() + k.numel() * k.element_size() +
             v.numel() * v.element_size())
        if self.w.backward:  # the forward's O and L, and dO
            b += (self.fwd_out.numel() * 2 + self.fwd_lse.numel() * 4 +
                  self.do.numel() * 2)
        return b

    def out_bytes(self):
        if self.w.backward:  # dQ, dK, dV
            return sum(t.numel() * 2 for t in self.grads)
        return self.out.numel() * 2 + self.lse.numel() * 4

    def step(self):
        k, v = self.kv[self.i % len(self.kv)]
        self.i += 1
        w = self.w
        if w.backward:
            dq, dk, dv = self.grads
            self.G.gqa_attn_backward(self.q, k, v, self.fwd_out, self.fwd_lse, self.do,
                                     causal=w.causal, dq=dq, dk=dk, dv=dv)
            return
        if w.qkv_fp8:
            sc = W.FP8_PREFILL_SCALE
            self.G.gqa_attn_fp8(self.q, k, v, q_scale=sc, k_scale=sc, v_scale=sc,
                                causal=w.causal, out=self.out, lse=self.lse)
            return
        if w.block_sparse and self.varlen:
            self.G.gqa_attn_blocksparse_varlen(self.q, k, v, self.cu, self.rp, self.col,
                                               max_seqlen=self.max_len, plan=self.plan,
                                               out=self.out, lse=self.lse)
            return
        if w.block_sparse:
            self.G.gqa_attn_blocksparse(self.q, k, v, self.rp, self.col, out=self.out,
                                        lse=self.lse)
            return
        if w.kv_fp8:
            self.G.gqa_attn_kvcache(self.q, k, v, k_scale=W.FP8_SCALE, v_scale=W.FP8_SCALE,
                                    num_splits=w.num_splits, pack_gqa=w.pack_gqa, out=self.out,
                                    lse=self.lse)
            return
        if self.paged:
            self.G.gqa_attn_kvcache(self.q, k, v, seqlens_k=self.lens, max_seqlen_k=w.Sk,
                                    block_table=self.table, num_splits=w.num_splits,
                                    pack_gqa=w.pack_gqa, out=self.out, lse=self.lse)
            return
        kw = dict(causal=w.causal, out=self.out, lse=self.lse, pack_gqa=w.pack_gqa)
        if w.window:
            kw["window"] = w.window
        if self.decode:
            kw["num_splits"] = w.num_splits
        if self.varlen:
            kw.update(cu_seqlens=self.cu, max_seqlen=self.max_len)
        self.G.gqa_attn(self.q, k, v, **kw)


def capture_steps(step, n, device):
    """A CUDA graph of n consecutive steps (the launches of n calls of the public API).

    Decode steps are tens of microseconds, shorter than the host-side cost of one
    Python call, so they are timed by replaying a captured graph: the device then
    runs the steps back to back, as a serving loop that captures its decode step does.
    """
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for _ in range(n):
                step()
    torch.cuda.current_stream(device).wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    return g


# ----------------------------------------------------------------------------- CPU oracle
_SAMPLE_INPUTS = {}


def _sample_inputs(w: W.Workload):
    """The workload's q, k, v widened to float32 numpy arrays (and cu_seqlens), built once
    per process: the oracle's own entry widens a torch tensor on every call, which would
    dominate a row sample's time, and the reference arm samples every step."""
    if w.name not in _SAMPLE_INPUTS:
        if w.varlen:
            q, k, v, cu = W.make_varlen(w, lengths=W.varlen_lengths(w))
            cu = cu.numpy()
        else:
            (q, k, v), cu = W.make_qkv(w), None
        _SAMPLE_INPUTS[w.name] = tuple(t.float().numpy() for t in (q, k, v)) + (cu,)
    return _SAMPLE_INPUTS[w.name]


def oracle_sample(w: W.Workload, target_s: float, max_s: float, seed: int = 0):
    """Time the float64 oracle on a bounded sample of workload w.

    Prefill: random query rows (b, h, i), doubling the count until target_s of CPU
    work; returns TFLOP/s of the sampled rows.  Decode: whole batch elements (all
    heads over the 32768-key cache); returns GB/s of their KV.
    Returns (value, sample description, threads used, seconds).
    """
    import oracle
    rng = np.random.default_rng(seed)
    cores = oracle.max_threads()
    if w.Sq == 1 and w.page_size > 0:
        import dataclasses
        w1 = dataclasses.replace(w, B=1)
        table = W.page_table(w1)
        kp, vp = W.make_paged_kv(w1, table)
        q = W.make_decode_q(w1)
        lens = np.full(1, w.Sk, dtype=np.int32)
        n, el = 0, 0.0
        while el < target_s and el < max_s:
            t0 = time.perf_counter()
            oracle.decode_kvcache(q, kp, vp, scale=w.scale, seqlens_k=lens, block_table=table)
            el += time.perf_counter() - t0
            n += 1
        gb = n * W.decode_bytes(1, w.Hq, w.Hkv, w.Sk, w.D) / 1e9
        return gb / el, (f"{n} x one sequence through its block table (all {w.Hq} heads, "
                         f"Sk={w.Sk}, pages of {w.page_size})"), cores, el
    if w.backward:
        # batch element 0, the query heads of K/V head 0, the first 2048 positions (with
        # the causal mask those queries see only those keys: a problem of its own)
        S = 2048
        q, k, v = W.make_qkv(w, B=1, Sq=S, Sk=S)
        q, k, v = q[:, :, : w.G].contiguous(), k[:, :, :1].contiguous(), v[:, :, :1].contiguous()
        do = torch.randn(1, S, w.G, w.D, generator=torch.Generator().manual_seed(7)).bfloat16()
        flops = int(2.5 * W.attention_flops(1, w.G, S, S, w.D, w.causal))
        n, el = 0, 0.0
        while el < target_s and el < max_s:
            t0 = time.perf_counter()
            oracle.attention_backward(q, k, v, do, scale=w.scale, causal=w.causal)
            el += time.perf_counter() - t0
            n += 1
        return (n * flops / 1e12 / el, f"{n} x the backward of batch element 0, the {w.G} "
                f"query heads of K/V head 0, positions 0..{S - 1}", cores, el)
    if w.qkv_fp8:
        S = 1024
        q8, k8, v8 = W.make_qkv_e4m3(w, B=1, Sq=S, Sk=S)
        q8, k8, v8 = q8[:, :, : w.G].contiguous(), k8[:, :, :1].contiguous(), \
            v8[:, :, :1].contiguous()
        sc = W.FP8_PREFILL_SCALE
        flops = W.attention_flops(1, w.G, S, S, w.D, w.causal)
        n, el = 0, 0.0
        while el < target_s and el < max_s:
            t0 = time.perf_counter()
            oracle.attention_e4m3(q8, k8, v8, q_scale=sc, k_scale=sc, v_scale=sc,
                                  scale=w.scale, causal=w.causal)
            el += time.perf_counter() - t0
            n += 1
        return (n * flops / 1e12 / el, f"{n} x the e4m3 forward of batch element 0, the "
                f"{w.G} query heads of K/V head 0, positions 0..{S - 1}", cores, el)
    if w.block_sparse and w.varlen:
        lengths = W.varlen_lengths(w).tolist()
        q, k, v, cu = W.make_varlen(w, lengths=lengths)
        rp, col = W.bigbird_pattern_varlen(lengths, w.block_sparse, seed=w.seed + 101)
        # sequence 0, the G query heads of K/V head 0, with its rows of the pattern
        n0, nb = lengths[0], -(-lengths[0] // 128)
        q, k, v = (t[: n0][None][:, :, : h].contiguous() for t, h in ((q, w.G), (k, 1), (v, 1)))
        sub_rp, sub_col = rp[: nb + 1], col[: int(rp[nb])]
        flops = W.blocksparse_varlen_flops([n0], sub_rp, sub_col, w.G, w.D)
        n, el = 0, 0.0
        while el < target_s and el < max_s:
            t0 = time.perf_counter()
            oracle.attention_blocksparse(q, k, v, sub_rp, sub_col, scale=w.scale, blk=128)
            el += time.perf_counter() - t0
            n += 1
        return (n * flops / 1e12 / el, f"{n} x packed sequence 0 ({n0} positions), the "
                f"{w.G} query heads of KV head 0", cores, el)
    if w.block_sparse:
        q, k, v = W.make_qkv(w, B=1)
        q, k, v = q[:, :, : w.G].contiguous(), k[:, :, :1].contiguous(), v[:, :, :1].contiguous()
        rp, col = W.bigbird_pattern(w)
        import dataclasses
        w1 = dataclasses.replace(w, B=1, Hq=w.G, Hkv=1)
        flops = W.blocksparse_flops(w1, rp, col)
        n, el = 0, 0.0
        while el < target_s and el < max_s:
            t0 = time.perf_counter()
            oracle.attention_blocksparse(q, k, v, rp, col, scale=w.scale, blk=128)
            el += time.perf_counter() - t0
            n += 1
        return (n * flops / 1e12 / el,
                f"{n} x batch element 0, the {w.G} query heads of KV head 0", cores, el)
    if w.Sq == 1 and w.kv_fp8:
        kb, vb = W.make_decode_kv_one(w, 0)
        k8 = (kb.float() / W.FP8_SCALE).to(torch.float8_e4m3fn)[None]
        v8 = (vb.float() / W.FP8_SCALE).to(torch.float8_e4m3fn)[None]
        q = W.make_decode_q(W.decode(1))
        n, el = 0, 0.0
        while el < target_s and el < max_s:
            t0 = time.perf_counter()
            oracle.decode_kvcache(q, k8, v8, scale=w.scale, k_scale=W.FP8_SCALE,
                                  v_scale=W.FP8_SCALE)
            el += time.perf_counter() - t0
            n += 1
        gb = n * W.decode_bytes(1, w.Hq, w.Hkv, w.Sk, w.D, kv_elt=1) / 1e9
        return gb / el, (f"{n} x one batch element of the e4m3 cache (all {w.Hq} heads, "
                         f"Sk={w.Sk})"), cores, el
    if w.Sq == 1:
        k, v = W.make_decode_kv_one(w, 0)
        q = W.make_decode_q(W.decode(1))
        n, el = 0, 0.0
        while el < target_s and el < max_s:
            t0 = time.perf_counter()
            oracle.attention(q, k[None], v[None], scale=w.scale, causal=False)
            el += time.perf_counter() - t0
            n += 1
        gb = n * W.decode_bytes(1, w.Hq, w.Hkv, w.Sk, w.D) / 1e9
        return gb / el, f"{n} x one batch element (all {w.Hq} heads, Sk={w.Sk})", cores, el
    if w.varlen:
        lengths = W.varlen_lengths(w)
        q, k, v, cu = _sample_inputs(w)
        lens = [int(x) for x in lengths]

        def rows_of(n):
            b = rng.integers(0, len(lens), n)
            i = np.array([rng.integers(0, lens[x]) for x in b])
            return np.stack([b, rng.integers(0, w.Hq, n), i], axis=1).astype(np.int32)

        def flops(rows):
            return sum(4 * w.D * (int(i) + 1) for _, _, i in rows)
    else:
        q, k, v, cu = _sample_inputs(w)

        def rows_of(n):
            return np.stack([rng.integers(0, w.B, n), rng.integers(0, w.Hq, n),
                             rng.integers(0, w.Sq, n)], axis=1).astype(np.int32)

        def flops(rows):
            if not w.causal:
                return len(rows) * 4 * w.D * w.Sk
            lim = w.window if w.window > 0 else w.Sk
            return sum(4 * w.D * max(0, min(lim, int(i) + w.Sk - w.Sq + 1))
                       for _, _, i in rows)
    n, el, done, nrows = 64, 0.0, 0, 0
    while el < target_s and el < max_s:
        rows = rows_of(n)
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, rows, scale=w.scale, causal=w.causal, cu_seqlens=cu,
                              window=w.window)
        el += time.perf_counter() - t0
        done += flops(rows)
        nrows += n
        n = min(n * 2, 1 << 16)
    return done / 1e12 / el, f"{nrows} random query rows (b, h, i) of the workload", cores, el


# ----------------------------------------------------------------------------- arms
def workload_config(w) -> dict:
    """The workload's own keys of the JSON line's config (both arms)."""
    cfg = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Sq": w.Sq, "Sk": w.Sk,
           "D": w.D, "causal": w.causal}
    if w.kv_fp8:
        cfg["kv_cache"] = f"e4m3 codes, k_scale = v_scale = {W.FP8_SCALE}"
    if w.qkv_fp8:
        cfg["inputs"] = f"e4m3 codes, q_scale = k_scale = v_scale = {W.FP8_PREFILL_SCALE}"
    if w.backward:
        cfg["pass"] = "backward: dQ, dK, dV for a seeded dO (O and L from the forward)"
        cfg["flops"] = "2.5 x the forward's (five products against two)"
    if w.page_size:
        cfg["page_size"] = w.page_size
        cfg["block_table"] = "seeded shuffle of the page pool"
    if w.window:
        cfg["window"] = w.window
        cfg["flops"] = "4 D per (query, key) pair inside the causal window"
    return cfg


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = workload_by_name(args.workload)
    unit = "GB/s" if w.Sq == 1 else "TFLOP/s"
    per_step = []
    desc, cores = "", 0
    steps = args.steps if args.steps > 0 else 5  # the oracle has no 2 s calibration
    for s in range(args.warmup + steps):
        v, desc, cores, el = oracle_sample(w, target_s=2.0, max_s=6.0, seed=s)
        if s >= args.warmup:
            per_step.append((v, el))
    value = statistics.median(v for v, _ in per_step)
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(e for _, e in per_step),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": f"each step: {desc}"},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    import exact_attention_gqa_b200 as G
    from exact_attention_gqa_b200 import build
    build.build()
    device = torch.device("cuda", local)
    w = workload_by_name(args.workload)
    case = Case(w, device, rank)
    stream = torch.cuda.current_stream(device)
    for _ in range(max(args.warmup, 3)):
        case.step()
    torch.cuda.synchronize()
    # calibrate the step count so the timed region lasts about 2 s unless given
    if args.steps <= 0:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(5):
            case.step()
        t1.record(stream)
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1) / 5
        steps = int(max(20, min(5000 if case.decode else 20000, 2000.0 / max(ms, 1e-3))))
        steps = int(max_over_ranks(steps, world))
    else:
        steps = args.steps
    graph = capture_steps(case.step, steps, device) if case.decode else None
    # ---- device-timed region: inputs resident, K steps
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        torch.cuda.synchronize()
        barrier(world)
        ev0.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for _ in range(steps):
                case.step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    del graph
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world)
    ms_step = ms_total / steps
    value = case.units * world / (ms_step / 1e3)
    if rank != 0:
        # the other ranks take part in the e2e timing below, then exit
        pass
    # ---- end to end through the public API with host buffers
    e2e_steps = max(3, min(steps, 20))
    k0, v0 = case.kv[0]
    hq = torch.empty(case.q.shape, dtype=case.q.dtype, pin_memory=True).copy_(case.q)
    hk = torch.empty(k0.shape, dtype=k0.dtype, pin_memory=True).copy_(k0)
    hv = torch.empty(v0.shape, dtype=v0.dtype, pin_memory=True).copy_(v0)
    ho = torch.empty(case.out.shape, dtype=case.out.dtype, pin_memory=True)
    hl = torch.empty(case.lse.shape, dtype=case.lse.dtype, pin_memory=True)
    dq, dk, dv = torch.empty_like(case.q), torch.empty_like(k0), torch.empty_like(v0)
    cu_h = case.cu.cpu().pin_memory() if case.varlen else None
    dcu = torch.empty_like(case.cu) if case.varlen else None

    if case.paged:
        ht = case.table.cpu().pin_memory()
        hs = case.lens.cpu().pin_memory()
        dt, ds = torch.empty_like(case.table), torch.empty_like(case.lens)

    if w.backward:
        hout, hlse = case.fwd_out.cpu().pin_memory(), case.fwd_lse.cpu().pin_memory()
        hdo = case.do.cpu().pin_memory()
        dout_d, dlse_d, ddo_d = (torch.empty_like(t) for t in (case.fwd_out, case.fwd_lse,
                                                               case.do))
        hgrads = tuple(torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in case.grads)
    if w.block_sparse:
        hrp, hcol = case.rp.cpu().pin_memory(), case.col.cpu().pin_memory()
        drp, dcol = torch.empty_like(case.rp), torch.empty_like(case.col)

    def e2e_step():
        if w.backward:
            for d, h in ((dq, hq), (dk, hk), (dv, hv), (dout_d, hout), (dlse_d, hlse),
                         (ddo_d, hdo)):
                d.copy_(h, non_blocking=True)
            gd = G.gqa_attn_backward(dq, dk, dv, dout_d, dlse_d, ddo_d, causal=w.causal,
                                     dq=case.grads[0], dk=case.grads[1], dv=case.grads[2])
            for h, d in zip(hgrads, gd):
                h.copy_(d, non_blocking=True)
            return
        if w.qkv_fp8:
            sc = W.FP8_PREFILL_SCALE
            for d, h in ((dq, hq), (dk, hk), (dv, hv)):
                d.copy_(h, non_blocking=True)
            G.gqa_attn_fp8(dq, dk, dv, q_scale=sc, k_scale=sc, v_scale=sc, causal=w.causal,
                           out=case.out, lse=case.lse)
            ho.copy_(case.out, non_blocking=True)
            hl.copy_(case.lse, non_blocking=True)
            return
        if w.block_sparse and case.varlen:
            # the schedule from the host copies of the offsets and the pattern, then the
            # inputs in, the attention, the results out
            plan = G.gqa_attn_blocksparse_varlen_plan(cu_h, hrp, Hq=w.Hq, Hkv=w.Hkv,
                                                      max_seqlen=case.max_len, device=dq.device)
            for d, h in ((dq, hq), (dk, hk), (dv, hv), (dcu, cu_h), (drp, hrp), (dcol, hcol)):
                d.copy_(h, non_blocking=True)
            G.gqa_attn_blocksparse_varlen(dq, dk, dv, dcu, drp, dcol, max_seqlen=case.max_len,
                                          plan=plan, out=case.out, lse=case.lse)
            ho.copy_(case.out, non_blocking=True)
            hl.copy_(case.lse, non_blocking=True)
            return
        if w.block_sparse:
            for d, h in ((dq, hq), (dk, hk), (dv, hv), (drp, hrp), (dcol, hcol)):
                d.copy_(h, non_blocking=True)
            G.gqa_attn_blocksparse(dq, dk, dv, drp, dcol, out=case.out, lse=case.lse)
            ho.copy_(case.out, non_blocking=True)
            hl.copy_(case.lse, non_blocking=True)
            return
        if w.kv_fp8:
            for d, h in ((dq, hq), (dk, hk), (dv, hv)):
                d.copy_(h, non_blocking=True)
            G.gqa_attn_kvcache(dq, dk, dv, k_scale=W.FP8_SCALE, v_scale=W.FP8_SCALE,
                               num_splits=w.num_splits, pack_gqa=w.pack_gqa, out=case.out,
                               lse=case.lse)
            ho.copy_(case.out, non_blocking=True)
            hl.copy_(case.lse, non_blocking=True)
            return
        if case.paged:
            # the public KV-cache call on inputs copied in from pinned host memory
            for d, h in ((dq, hq), (dk, hk), (dv, hv), (dt, ht), (ds, hs)):
                d.copy_(h, non_blocking=True)
            G.gqa_attn_kvcache(dq, dk, dv, seqlens_k=ds, max_seqlen_k=w.Sk, block_table=dt,
                               num_splits=w.num_splits, pack_gqa=w.pack_gqa, out=case.out,
                               lse=case.lse)
            ho.copy_(case.out, non_blocking=True)
            hl.copy_(case.lse, non_blocking=True)
            return
        if w.window:
            for d, h in ((dq, hq), (dk, hk), (dv, hv)):
                d.copy_(h, non_blocking=True)
            G.gqa_attn(dq, dk, dv, causal=True, window=w.window, out=case.out, lse=case.lse)
            ho.copy_(case.out, non_blocking=True)
            hl.copy_(case.lse, non_blocking=True)
            return
        if not case.varlen:
            # the public host-buffer entry point: batch chunks with copy in, attention and
            # copy out overlapped on the library's streams
            G.gqa_attn_host(hq, hk, hv, ho, hl, dq, dk, dv, case.out, case.lse,
                            causal=w.causal, num_splits=w.num_splits if case.decode else 1,
                            pack_gqa=w.pack_gqa)
            return
        dcu.copy_(cu_h, non_blocking=True)
        G.gqa_attn_host(hq, hk, hv, ho, hl, dq, dk, dv, case.out, case.lse, causal=w.causal,
                        pack_gqa=w.pack_gqa, cu_seqlens=(cu_h, dcu), max_seqlen=case.max_len)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    h2d = hq.numel() * hq.element_size() + hk.numel() * hk.element_size() + \
        hv.numel() * hv.element_size() + \
        (cu_h.numel() * 4 if cu_h is not None else 0) + \
        ((ht.numel() + hs.numel()) * 4 if case.paged else 0) + \
        ((hrp.numel() + hcol.numel()) * 4 if w.block_sparse else 0)
    d2h = ho.numel() * 2 + hl.numel() * 4
    if w.block_sparse and case.varlen:  # the plan's block offsets and tile order
        h2d += case.plan.blk_off.numel() * 4 + case.plan.n_order * 4
    if w.backward:
        h2d += hout.numel() * 2 + hlse.numel() * 4 + hdo.numel() * 2
        d2h = sum(t.numel() * 2 for t in hgrads)
    err = G.gqa_attn_get_device_error()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    # ---- roofline of the dominant kernel
    peaks, peak_kind = load_peaks()
    kernel_ms = ms_step  # one launch per step (decode: split kernel + combine)
    if case.decode:
        achieved = case.bytes / (kernel_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        # A timed region of a second or more runs under the power cap, like the
        # sustained GEMM loop; a short one like the burst figure.
        sustained = ms_total >= 1000.0 and "bf16_tflops_sustained" in peaks
        key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
        achieved = case.flops / (kernel_ms / 1e3) / 1e12
        # an e4m3 contraction: the measured bf16 figure times the nominal 2x of fp8
        ratio = 2.0 if w.qkv_fp8 else 1.0
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks[key] * ratio,
                "unit": "TFLOP/s",
                "frac_of_burst": achieved / (peaks["bf16_tflops"] * ratio)}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["frac_of_spec"] = roof["achieved"] / (
        SPEC_PEAKS["hbm_gbs"] if case.decode
        else SPEC_PEAKS["bf16_tflops"] * (2.0 if w.qkv_fp8 else 1.0))
    if case.decode:
        roof["peak_source"] = f"{peak_kind} (hbm_gbs, copy)"
    else:
        roof["peak_source"] = (f"{peak_kind} ({key}: timed region {ms_total / 1e3:.1f} s, "
                               f"{'sustained' if sustained else 'burst'})"
                               + (" x 2, the nominal e4m3 / bf16 ratio" if w.qkv_fp8 else ""))
    roof["kernel"] = case.kernel
    tr = load_traffic(w.name, case.kernel)
    roof["traffic"] = tr
    # algorithmic bytes of one launch: q, k, v read once, O and L written once
    roof["algorithmic_bytes"] = case.in_bytes() + case.out_bytes()
    if tr is not None:
        roof["traffic_per_algorithmic"] = tr / roof["algorithmic_bytes"]
    # ---- CPU baseline (oracle on a bounded sample, rank 0, N=1 only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v_cpu, desc, cores, el = oracle_sample(w, target_s=args.cpu_seconds, max_s=30.0)
        cpu = {"value": v_cpu, "unit": case.unit, "cores": cores, "kind": "oracle",
               "sample": f"{desc}; {el:.1f} s of float64 CPU work"}
    cfg = workload_config(w)
    cfg.update({"pack_gqa": case.pack, "num_splits": case.splits,
           "per_rank": "independent copy of the workload on every rank",
           "l2": ("inputs larger than L2 (%.0f MB per step)" % (case.in_bytes() / 1e6)
                  if case.in_bytes() > L2_BYTES or len(case.kv) > 1 else "inputs fit in L2"),
           "kv_copies_rotated": len(case.kv),
           "timing": ("CUDA graph of the K steps, replayed once" if case.decode
                      else "K back-to-back calls")})
    if case.varlen:
        cfg["total_tokens"] = int(case.q.shape[0])
    if w.block_sparse:
        every = (sum((-(-int(n) // 128)) ** 2 for n in case.lengths.tolist()) if case.varlen
                 else (case.rp.numel() - 1) * -(-w.Sk // 128))
        cfg["block_pattern"] = dict(w.block_sparse, block=128, blocks=int(case.col.numel()),
                                    of=int(every))
        if case.varlen:
            cfg["padding"] = "each sequence to whole 128-position blocks (minimum padding)"
            cfg["tile_order"] = "host schedule: longest first onto the least loaded CTA"
    line = {"metric": METRIC, "value": value, "unit": case.unit, "n_gpus": world,
            "steps": steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if w.qkv_fp8 else "bf16",
            "data": "synthetic (seeded N(0,1) bf16)" + (", as e4m3 codes" if w.qkv_fp8 else ""),
            "config": cfg, "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": case.units * world / (e2e_ms / 1e3), "unit": case.unit,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms,
                    "path": ("gqa_attn_backward after pinned host copies of q, k, v, O, L "
                             "and dO; dQ, dK, dV copied back" if w.backward else
                             "gqa_attn_fp8 after pinned host copies of the e4m3 q, k, v; "
                             "results copied back" if w.qkv_fp8 else
                             "gqa_attn_blocksparse_varlen_plan on the host offsets and "
                             "pattern, pinned host copies of q, k, v, cu_seqlens and the "
                             "pattern, gqa_attn_blocksparse_varlen; results copied back"
                             if w.block_sparse and case.varlen else
                             "gqa_attn_blocksparse after pinned host copies of q, k, v and "
                             "the block pattern; results copied back" if w.block_sparse else
                             "gqa_attn_kvcache on the e4m3 cache after pinned host copies "
                             "of q and the caches; results copied back" if w.kv_fp8 else
                             "gqa_attn(window=...) after pinned host copies of q, k, v; "
                             "results copied back" if w.window else
                             "gqa_attn_kvcache on the paged cache after pinned host "
                             "copies of q, the page pools, the block table and the lengths; "
                             "results copied back" if case.paged else
                             "gqa_attn_fwd_host" + ("_varlen: 8 chunks of whole sequences"
                                                    if case.varlen else
                                                    ": 8 chunks (batch elements, or ranges of "
                                                    "positions when the batch is smaller)")
                             + ", pinned host buffers, copy in / attention / copy out "
                               "overlapped")},
            "gpu_launches": steps * case.launches_per_step,
            "clocks": clocks.summary(), "device_error": err,
            "kernel_source": kernel_source_hash(case.kernel), "library": G.library_path()}
    print(json.dumps(line), flush=True)


def run_decode_sweep(args, local):
    """Every decode cell: B x num_splits (1, 2, 4, 8, auto) x pack_gqa (1, 0); one line each."""
    import exact_attention_gqa_b200 as G
    from exact_attention_gqa_b200 import build
    build.build()
    device = torch.device("cuda", local)
    stream = torch.cuda.current_stream(device)
    peaks, peak_kind = load_peaks()
    batches = [int(b) for b in args.batches.split(",")] if args.batches else list(W.DECODE_BATCHES)
    for B in batches:
        base = W.decode(B)
        kv_bytes = W.kv_cache_bytes(B, base.Sk, base.Hkv, base.D)
        copies = 1 if kv_bytes > 2 * L2_BYTES else 3
        q = W.make_decode_q(base, device=device)
        kvs = []
        for _ in range(copies):
            k = torch.empty(B, base.Sk, base.Hkv, base.D, dtype=torch.bfloat16, device=device)
            v = torch.empty_like(k)
            W.fill_decode_kv(base, k, v)
            kvs.append((k, v))
        out = torch.empty_like(q)
        lse = torch.empty(B, base.Hq, 1, dtype=torch.float32, device=device)
        nbytes = W.decode_bytes(B, base.Hq, base.Hkv, base.Sk, base.D)
        for splits in (1, 2, 4, 8, 0):
            for pack in (1, 0):
                rc, kern, eff_splits, eff_pack = G.gqa_attn_plan(B, base.Hq, base.Hkv, 1, base.Sk,
                                                                 base.D, num_splits=splits,
                                                                 pack_gqa=pack)
                idx = [0]

                def step():
                    k, v = kvs[idx[0] % copies]
                    idx[0] += 1
                    G.gqa_attn(q, k, v, num_splits=splits, pack_gqa=pack, out=out, lse=lse)

                for _ in range(max(args.warmup, 3)):
                    step()
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                step()
                e1.record(stream)
                torch.cuda.synchronize()
                one = max(e0.elapsed_time(e1), 1e-3)
                steps = int(max(10, min(2000, 150.0 / one)))
                graph = capture_steps(step, steps, device)
                e0.record(stream)
                graph.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                del graph
                ms = e0.elapsed_time(e1) / steps
                gbs = nbytes / (ms * 1e-3) / 1e9
                print(json.dumps({"metric": METRIC, "sweep": "decode", "B": B, "Sk": base.Sk,
                                  "num_splits": splits, "pack_gqa": pack,
                                  "effective_splits": eff_splits, "effective_pack": eff_pack,
                                  "value": gbs, "unit": "GB/s", "ms_per_step": ms,
                                  "steps": steps, "kv_copies_rotated": copies,
                                  "frac_of_measured_copy": gbs / peaks["hbm_gbs"],
                                  "peak_source": peak_kind,
                                  "timing": "CUDA graph of the steps, replayed once",
                                  "gpu_launches_per_step": 2 if eff_splits > 1 else 1}),
                      flush=True)
        del kvs, q, out, lse
        torch.cuda.empty_cache()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0: about 2 s)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--sweep", choices=["decode"], default=None,
                    help="print one line per decode cell instead of the bench line")
    ap.add_argument("--batches", default="", help="decode sweep batch sizes (comma list)")
    args = ap.parse_args(argv)
    world, rank, local = dist_setup(args)
    if args.sweep == "decode":
        run_decode_sweep(args, local)
        return
    if args.impl == "reference":
        if args.steps <= 0:
            args.steps = 3
        run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
