#!/usr/bin/env python
"""Benchmark of the MiniKV hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl minikv|reference]

Default workload (the one the decode-bandwidth target is stated on): a
Mistral-7B-shaped GQA decode -- 32 layers, 32 query heads over 8 KV heads,
head size 128, batch 16, a 32768-token context of which 20% (6553 tokens) is
kept and packed 2-bit (key group G=32, value group 128, fp16 residual R=128).
A step is one generated token for the whole batch through all 32 layers: per
layer one minikv_decode_attn call (append the new token, attend over the
packed + residual cache, flush a key group to 2 bits every G steps).  The
calls are made one per layer from Python (host-side state), or, with
`--launch graph` (the default for the ragged workload), the caches keep their
per-sequence state on the GPU and the 32 calls of a step are captured once in a
CUDA graph and replayed every step.  The
per-layer caches (2.5 GB per step) are walked in order, so the working set is
far larger than the 126 MB L2.  The same run also times the prompt rows of
the path on a LLaMA2-7B-shaped prefill (32 layers x 32 heads, 4096 tokens,
W=32, keep 15%): minikv_select_prefill, minikv_topk_evict, minikv_quant_pack.

Inputs are seeded synthetic N(0,1) fp16 with 4 outlier key channels x10 per
KV head (no dataset, no weights).  Under torchrun every rank runs its own
replica (weak scaling, no collective on the data path); the timed region is
bracketed by barriers and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
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

METRIC = "decode attn tokens/s and HBM GB/s (% of peak) over 2-bit KV; prefill select ms"

# Decode workloads (--workload); the first is the default bench line.  keep_pct
# "pyramid" is the layer-discriminative budget: 30% of the context at layer 0
# falling linearly to 5% at the last layer.
DECODE_PRESETS = {
    "mistral7b_gqa_decode": dict(workload="mistral7b_gqa_decode", layers=32, batch=16, q_heads=32, kv_heads=8,
                                 head_dim=128, context=32768, keep_pct=20, G=32, Gv=128, R=128),
    "llama2_13b_decode": dict(workload="llama2_13b_decode", layers=40, batch=8, q_heads=40, kv_heads=40,
                              head_dim=128, context=16384, keep_pct=15, G=32, Gv=128, R=128),
    "pyramid_44k_decode": dict(workload="pyramid_44k_decode", layers=32, batch=4, q_heads=32, kv_heads=32,
                               head_dim=128, context=44000, keep_pct="pyramid", G=32, Gv=128, R=128),
    # the pyramid decode at the largest batch that fits the free HBM (sized at run time)
    "pyramid_44k_maxbatch_decode": dict(workload="pyramid_44k_maxbatch_decode", layers=32, batch="max", q_heads=32,
                                        kv_heads=32, head_dim=128, context=44000, keep_pct="pyramid", G=32, Gv=128,
                                        R=128),
    # every token kept, only quantized (the KIVI-like point of the method): 32K context
    "quant_only_32k_decode": dict(workload="quant_only_32k_decode", layers=32, batch=16, q_heads=32, kv_heads=8,
                                  head_dim=128, context=32768, keep_pct=100, G=32, Gv=128, R=128),
    # ragged batch: the 16 prompts' contexts rise evenly from 4K to 32K tokens, 20 % kept of each
    "mistral7b_gqa_ragged_decode": dict(workload="mistral7b_gqa_ragged_decode", layers=32, batch=16, q_heads=32,
                                        kv_heads=8, head_dim=128, context="4096..32768 (even ramp over the batch)",
                                        contexts=[4096 + (32768 - 4096) * b // 15 for b in range(16)],
                                        keep_pct=20, G=32, Gv=128, R=128),
}
PREFILL_PRESETS = {
    "llama2_7b_prefill_select": dict(workload="llama2_7b_prefill_select", layers=32, batch=1, q_heads=32,
                                     kv_heads=32, head_dim=128, prompt=4096, W=32, keep_pct=15, G=32, Gv=128,
                                     R=128),
    "pyramid_44k_prefill_select": dict(workload="pyramid_44k_prefill_select", layers=32, batch=4, q_heads=32,
                                       kv_heads=32, head_dim=128, prompt=44000, W=32, keep_pct="pyramid", G=32,
                                       Gv=128, R=128),
}
DECODE = dict(DECODE_PRESETS["mistral7b_gqa_decode"])
PREFILL = dict(PREFILL_PRESETS["llama2_7b_prefill_select"])

BYTES_PER_PACKED = 84     # per token and KV head at D=128, G=32, Gv=128: 64 code + 16 key + 4 value scale/zero
BYTES_PER_RESIDUAL = 512  # fp16 K + V row


def keep_of(T, pct, layer=0, n_layers=32):
    """Kept tokens of a layer: pct % of T, or the pyramid budget (30% at layer 0
    down to 5% at the last layer, linear in the layer index, floor in integers)."""
    if pct == "pyramid":
        return (T * (30 * (n_layers - 1) - 25 * layer)) // (100 * (n_layers - 1))
    return T * pct // 100


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def recorded_traffic(kernel: str, sources):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the current sources of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        h = hashlib.sha256()
        for src in sources:
            h.update(open(src, "rb").read())
        sha = h.hexdigest()[:16]
        for line in open(path):
            f = line.split()
            if len(f) >= 4 and f[0] == kernel and f[1] == sha:
                return float(f[2]), f[3]
    except OSError:
        pass
    return None, None


# ------------------------------------------------------------ multi-rank

def max_over_ranks(x: float, device) -> float:
    """The largest of every rank's x (the job is as slow as its slowest rank);
    x itself when the job has one rank.  `device` is where the all-reduce
    tensor lives (the rank's GPU under NCCL, the CPU under gloo)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(batch: int, steps: int, world: int, ms: float) -> float:
    """Whole-job throughput: every rank generates `batch` tokens per step, and
    the job took `ms` (the slowest rank's time)."""
    return batch * steps * world / (ms * 1e-3)


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons sampled by NVML while the timed region runs."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
               0x10: "sync_boost", 0x1: "gpu_idle"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self.period = period_s
        self.samples, self.reasons = [], 0
        self._stop = threading.Event()

    def _reasons(self):
        f = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return f(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons())
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------ CPU oracle

def _oracle_unit(n_keep, g, seed):
    import torch
    from bit_quantized_evicted_b200 import synth
    from oracle import minikv_oracle as O
    k = synth.keys_fp16((n_keep, 128), synth.seed_of(77, seed, synth.T_K)).numpy()
    v = synth.normal_fp16((n_keep, 128), synth.seed_of(77, seed, synth.T_V)).numpy()
    cache = O.SliceCache.from_kept(k, v, DECODE["R"], DECODE["G"], DECODE["Gv"])
    q = synth.normal_fp16((g, 128), synth.seed_of(77, seed, synth.T_QDEC)).numpy()
    kn = synth.keys_fp16((128,), synth.seed_of(77, seed, synth.T_KNEW)).numpy()
    vn = synth.normal_fp16((128,), synth.seed_of(77, seed, synth.T_VNEW)).numpy()
    del torch
    return cache, q, kn, vn


def oracle_decode_rate(budget_s: float, threads: int):
    """Unit-steps per second of the CPU oracle's decode step (one (sequence,
    KV head) of one layer: append, attend over 6553 kept tokens with g = 4
    query heads in fp64, flush when due), run on `threads` host threads."""
    n_keep = keep_of(DECODE["context"], DECODE["keep_pct"])
    g = DECODE["q_heads"] // DECODE["kv_heads"]
    units = [_oracle_unit(n_keep, g, i) for i in range(threads)]
    tau = 1.0 / math.sqrt(128.0)
    counts = [0] * threads
    deadline = time.perf_counter() + budget_s

    def work(i):
        c, q, kn, vn = units[i]
        while time.perf_counter() < deadline:
            c.step(q, kn, vn, tau)
            counts[i] += 1

    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(threads)))
    dt = time.perf_counter() - t0
    return sum(counts) / dt, sum(counts), dt


def compression(step_bytes):
    L, B, Hkv = DECODE["layers"], DECODE["batch"], DECODE["kv_heads"]
    per_layer = step_bytes / L
    ctx_tokens = sum(DECODE["contexts"]) if "contexts" in DECODE else B * DECODE["context"]
    kept = sum(seq_keeps()) if "contexts" in DECODE else B * sum(decode_keeps()) / L
    fp16 = Hkv * 128 * 2 * 2   # K and V bytes per token
    return {"of_full_context_fp16": per_layer / (ctx_tokens * fp16), "of_kept_fp16": per_layer / (kept * fp16)}


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_tokens_per_s(rate):
    units_per_step = DECODE["layers"] * DECODE["batch"] * DECODE["kv_heads"]
    return rate * DECODE["batch"] / units_per_step


def seq_keeps():
    """Kept tokens per sequence of a ragged workload (None for uniform batches)."""
    if "contexts" not in DECODE:
        return None
    return [keep_of(t, DECODE["keep_pct"]) for t in DECODE["contexts"]]


def decode_keeps():
    """Kept tokens per layer (the longest sequence's, for a ragged batch)."""
    if "contexts" in DECODE:
        return [max(seq_keeps())] * DECODE["layers"]
    return [keep_of(DECODE["context"], DECODE["keep_pct"], l, DECODE["layers"]) for l in range(DECODE["layers"])]


def decode_config(extra=None, step_bytes=None):
    c = {k: v for k, v in DECODE.items() if k != "eager"}
    keeps = decode_keeps()
    c["keep"] = keeps[0] if len(set(keeps)) == 1 else f"{keeps[0]}..{keeps[-1]} (per layer)"
    if "contexts" in DECODE:
        sk = seq_keeps()
        c.pop("contexts")
        c["keep"] = f"{min(sk)}..{max(sk)} (per sequence, mean {sum(sk) / len(sk):.0f})"
    gb = (step_bytes or 0) / 1e9
    c["l2"] = (f"inputs larger than L2: {DECODE['layers']} distinct layer caches, {gb:.2f} GB read per step"
               if step_bytes else f"inputs larger than L2: {DECODE['layers']} distinct layer caches")
    if extra:
        c.update(extra)
    return c


def run_reference(args):
    """The oracle as the reference arm: rank 0 only, host cores."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    threads = os.cpu_count() or 1
    per_step = max(0.05, min(0.5, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_decode_rate(per_step, threads)
    rates, units, timed = [], 0, 0.0
    for _ in range(args.steps):
        r, n, dt = oracle_decode_rate(per_step, threads)
        rates.append(r)
        units += n
        timed += dt
    rate = statistics.median(rates)
    v = cpu_tokens_per_s(rate)
    per_full_step = DECODE["layers"] * DECODE["batch"] * DECODE["kv_heads"]
    sample = (f"{units} decode unit-steps (one sequence x KV head of one layer: 6553 kept tokens, 4 query heads, fp64) "
              f"over {args.steps} steps of {per_step:.2f} s on {threads} threads; tokens/s = unit-steps/s x batch / "
              f"(32 layers x 16 x 8 units)")
    # the same config object as the GPU arm's (same workload, same timed-step bytes)
    cfg = decode_config({"parallelism": f"replicas x{args.gpus}"},
                        step_bytes=timed_step_bytes(args.warmup, args.steps))
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * DECODE["batch"] / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg,
            # value and ms_per_step are rates scaled up from the timed sample: one full step is
            # per_full_step unit-steps, far more than the sample holds
            "extrapolated": {"value": True, "ms_per_step": True, "timed_seconds": timed, "unit_steps_timed": units,
                             "unit_steps_per_full_step": per_full_step,
                             "unit_steps_per_s": rate},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "cpu_model": cpu_model(),
                             "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- GPU arm

# The largest batch of the pyramid workload that fits the free device memory
# (the long-prompt workload's batch is raised until HBM is full).  Every sequence
# costs its 32 per-layer caches (sized for 512 decode steps of growth), its
# share of the decode workspace and its step inputs / outputs; a fixed reserve
# covers the transient of loading one sequence and the allocator's slack.
MAXBATCH_RESERVE = 6 << 30
MAX_SEQS = 256   # most sequences a device-state batch may hold


def max_batch(mk, free_bytes, preset=None, steps=512, pool=8):
    d = preset or DECODE
    L, Hq, Hkv, G, Gv, R = d["layers"], d["q_heads"], d["kv_heads"], d["G"], d["Gv"], d["R"]
    keeps = [keep_of(d["context"], d["keep_pct"], l, L) for l in range(L)]
    caps = [((n + steps + 8) // G + 2) * G for n in keeps]
    lib = mk.lib()
    per_seq = sum(int(lib.minikv_cache_bytes(1, Hkv, 128, G, Gv, R, cap)) for cap in caps)
    per_seq += mk.workspace_size(mk.OP_DECODE_ATTN, 1, Hq, Hkv, max(caps) + R + G)
    per_seq += (pool + 4) * L * (Hq + 2 * Hkv) * 128 * 2 + 4 * L * Hq * 128 * 2
    B = int((free_bytes - MAXBATCH_RESERVE) // per_seq)
    return max(1, min(MAX_SEQS, B)), per_seq


def make_decode_state(torch, mk, synth, device, warmup, steps):
    L, Hq, Hkv = DECODE["layers"], DECODE["q_heads"], DECODE["kv_heads"]
    G, Gv, R = DECODE["G"], DECODE["Gv"], DECODE["R"]
    if DECODE["batch"] == "max":
        free, _ = torch.cuda.mem_get_info(device)
        DECODE["batch"], per_seq = max_batch(mk, free, steps=max(512, warmup + 3 * steps + 2))
        DECODE["max_batch_rule"] = (f"largest batch that fits {free / 1e9:.1f} GB of free HBM at "
                                    f"{per_seq / 1e9:.3f} GB per sequence (caches sized for 512 steps)")
    B = DECODE["batch"]
    keeps = decode_keeps()
    total_steps = max(warmup + 3 * steps + 2, 512 if "max_batch_rule" in DECODE else 0)
    cap_max = ((max(keeps) + total_steps + 8) // G + 2) * G
    op = mk.OP_DECODE_ATTN_MASS if DECODE.get("mass") else mk.OP_DECODE_ATTN
    ws = torch.zeros(mk.workspace_size(op, B, Hq, Hkv, cap_max + R + G), dtype=torch.uint8, device=device)
    wid = 4 if DECODE["workload"] == "mistral7b_gqa_decode" else 40 + list(DECODE_PRESETS).index(DECODE["workload"])
    caches = []
    sk = seq_keeps()
    per_seq_load = sk is not None or "max_batch_rule" in DECODE
    for l in range(L):
        N = keeps[l]
        cap = ((N + total_steps + 8) // G + 2) * G
        c = mk.MiniKVCache(B, Hkv, cap, G=G, Gv=Gv, R=R, Hq=Hq, device=device, ws=ws)
        if not DECODE.get("eager"):
            c.set_device_state()   # per-sequence state on the GPU: steps replay from CUDA graphs
        elif per_seq_load:
            c.set_ragged()
        if per_seq_load:   # each sequence loaded into its own row (its own length for a ragged batch)
            for b in range(B):
                n = sk[b] if sk is not None else N
                kb = synth.keys_fp16((Hkv, n, 128), synth.seed_of(wid, l, synth.T_K, 0, b), device)
                vb = synth.normal_fp16((Hkv, n, 128), synth.seed_of(wid, l, synth.T_V, 0, b), device)
                mk.quant_pack_seq(c, b, kb, vb)
                del kb, vb
            k = v = None
        else:
            k = torch.empty((B, Hkv, N, 128), dtype=torch.float16, device=device)
            v = torch.empty_like(k)
            for b in range(B):
                k[b] = synth.keys_fp16((Hkv, N, 128), synth.seed_of(wid, l, synth.T_K, 0, b), device)
                v[b] = synth.normal_fp16((Hkv, N, 128), synth.seed_of(wid, l, synth.T_V, 0, b), device)
            mk.quant_pack(c, k, v)
        # H2O-style running attention mass per token (--mass)
        c.mass = torch.zeros((B, Hkv, cap + R + G), dtype=torch.float32, device=device) if DECODE.get("mass") else None
        caches.append(c)
        del k, v
    torch.cuda.synchronize()
    # one pool of step inputs, laid out contiguously so that e2e copies are single transfers
    P = 8
    qin = torch.empty((P, L, B, Hq, 128), dtype=torch.float16, device=device)
    knin = torch.empty((P, L, B, Hkv, 128), dtype=torch.float16, device=device)
    vnin = torch.empty_like(knin)
    for p in range(P):
        for l in range(L):
            qin[p, l] = synth.normal_fp16((B, Hq, 128), synth.seed_of(wid, l, synth.T_QDEC, p), device)
            knin[p, l] = synth.keys_fp16((B, Hkv, 128), synth.seed_of(wid, l, synth.T_KNEW, p), device)
            vnin[p, l] = synth.normal_fp16((B, Hkv, 128), synth.seed_of(wid, l, synth.T_VNEW, p), device)
    out = torch.empty((L, B, Hq, 128), dtype=torch.float16, device=device)
    return caches, ws, qin, knin, vnin, out


class LengthMirror:
    """Host copy of every layer's per-sequence (n_packed, n_res), advanced the
    way a decode step advances the cache (append; flush G tokens when the ring
    of R+G is full), so that the algorithmic bytes of each step are known
    without reading the GPU's state."""

    def __init__(self, layer_lengths, G, R):
        self.G, self.ring = G, R + G

        def split(N):
            if N < R:
                return [0, N]
            r = R + (N - R) % G
            return [N - r, r]
        self.st = [[split(N) for N in lens] for lens in layer_lengths]

    def layer_bytes(self, l, Hkv, mass):
        """Bytes one layer-step reads: per (sequence, KV head) unit its packed and
        residual tokens (and one fp32 running score read and written per token
        with --mass)."""
        total = 0
        for nq, nr in self.st[l]:
            n = BYTES_PER_PACKED * nq + BYTES_PER_RESIDUAL * (nr + 1)
            if mass:
                n += 8 * (nq + nr + 1)
            total += n * Hkv
        return total

    def advance(self):
        for layer in self.st:
            for s in layer:
                s[1] += 1
                if s[1] == self.ring:
                    s[0] += self.G
                    s[1] -= self.G


def mirror_for_preset():
    """A LengthMirror of the current decode workload's starting lengths."""
    sk = seq_keeps()
    B = DECODE["batch"]
    return LengthMirror([sk if sk is not None else [n] * B for n in decode_keeps()], DECODE["G"], DECODE["R"])


def timed_step_bytes(warmup, steps):
    """Algorithmic bytes per timed step of the current decode workload: the
    mean over the timed steps, after `warmup` steps (host bookkeeping only, so
    that the reference arm states the same config as the GPU arm)."""
    m = mirror_for_preset()
    L, Hkv, mass = DECODE["layers"], DECODE["kv_heads"], bool(DECODE.get("mass"))
    for _ in range(warmup):
        m.advance()
    tot = 0
    for _ in range(steps):
        tot += sum(m.layer_bytes(l, Hkv, mass) for l in range(L))
        m.advance()
    return tot / max(1, steps)


def decode_call(mk, c, q, kn, vn, out, ws, stream):
    if c.mass is not None:
        mk.decode_attn_mass(c, q, kn, vn, c.mass, out=out, ws=ws, stream=stream)
    else:
        mk.decode_attn(c, q, kn, vn, out=out, ws=ws, stream=stream)


def run_prefill(torch, mk, synth, device, pk):
    """Prompt rows of one prefill workload: per layer select_prefill, topk_evict
    and quant_pack, each timed with CUDA events (3 warm-up layers first).  A
    layer's q, k, v are generated (untimed) just before its calls."""
    L, B, H, T, W = PREFILL["layers"], PREFILL["batch"], PREFILL["q_heads"], PREFILL["prompt"], PREFILL["W"]
    keeps = [keep_of(T, PREFILL["keep_pct"], l, 32) for l in range(L)]
    wid = 2 if PREFILL["workload"] == "llama2_7b_prefill_select" else 50
    kmax = min(max(keeps), T)
    ws = torch.empty(mk.workspace_size(mk.OP_SELECT_PREFILL, B, H, H, T, 128, W), dtype=torch.uint8, device=device)
    q = torch.empty((B, H, T, 128), dtype=torch.float16, device=device)
    k, v, o = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    sc = torch.empty((B, H, T), dtype=torch.float32, device=device)
    idx_buf = torch.empty(B * H * kmax, dtype=torch.int32, device=device)
    kk_buf = torch.empty(B * H * kmax * 128, dtype=torch.float16, device=device)
    vk_buf = torch.empty_like(kk_buf)
    cap = ((kmax + 2 * PREFILL["G"]) // PREFILL["G"] + 1) * PREFILL["G"]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)   # twice the L2

    def layer(l, e=None):
        q.copy_(synth.normal_fp16((B, H, T, 128), synth.seed_of(wid, l, synth.T_Q), device))
        k.copy_(synth.keys_fp16((B, H, T, 128), synth.seed_of(wid, l, synth.T_K), device))
        v.copy_(synth.normal_fp16((B, H, T, 128), synth.seed_of(wid, l, synth.T_V), device))
        n = min(keeps[l], T)
        idx = idx_buf[:B * H * n].view(B, H, n)   # contiguous views of this layer's size
        kk = kk_buf[:B * H * n * 128].view(B, H, n, 128)
        vk = vk_buf[:B * H * n * 128].view(B, H, n, 128)
        cache = mk.MiniKVCache(B, H, cap, G=PREFILL["G"], Gv=PREFILL["Gv"], R=PREFILL["R"], device=device)
        cache2 = mk.MiniKVCache(B, H, cap, G=PREFILL["G"], Gv=PREFILL["Gv"], R=PREFILL["R"], device=device)
        flush.zero_()   # evict the freshly generated inputs from L2 before the timed calls
        torch.cuda.synchronize()
        if e is not None:
            e[0].record()
        mk.select_prefill(q, k, v, W, o=o, scores=sc, ws=ws)
        if e is not None:
            e[1].record()
        mk.topk_evict(sc, k, v, W, keeps[l], idx=idx, k_kept=kk, v_kept=vk)
        if e is not None:
            e[2].record()
        mk.quant_pack(cache, kk, vk)
        if e is not None:
            e[3].record()
        # the fused form of the last two calls (select -> pack with no fp16 copy of the kept rows)
        mk.evict_pack(cache2, sc, k, v, W, keeps[l], idx=idx)
        if e is not None:
            e[4].record()
        torch.cuda.synchronize()

    for l in range(3):
        layer(l)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(L)]
    for l in range(L):
        layer(l, ev[l])
    sel = sum(e[0].elapsed_time(e[1]) for e in ev)
    top = sum(e[1].elapsed_time(e[2]) for e in ev)
    pk_ms = sum(e[2].elapsed_time(e[3]) for e in ev)
    fused = sum(e[3].elapsed_time(e[4]) for e in ev)
    flops = L * (2.0 * T * T * 128 * H * B + 2.0 * W * T * 128 * H * B)    # causal QK^T + PV, plus the window pass
    tflops = flops / (sel * 1e-3) / 1e12
    del q, k, v, o
    return {"workload": PREFILL["workload"], "config": {**PREFILL, "keep": keeps[0] if len(set(keeps)) == 1 else
                                                        f"{keeps[0]}..{keeps[-1]} (per layer)"},
            "select_prefill_ms": sel, "select_prefill_ms_per_layer": sel / L,
            "select_prefill_tflops": tflops,
            # select_prefill per layer (flash-attention pass + window pass) against the dense bf16 peak
            # (fp16 tensor-core rate = bf16 rate); each layer is timed alone after an L2 flush: burst peak
            "roofline": {"bound": "tensor", "kernel": "fa_tc_kernel + window_score_kernel", "achieved": tflops,
                         "peak": pk["bf16"], "unit": "TFLOP/s", "frac": tflops / pk["bf16"], "traffic": None,
                         "algorithmic_flops_per_layer": flops / L, "peak_source": pk["src"] + " (bf16 burst)"},
            "topk_evict_ms": top, "quant_pack_ms": pk_ms, "evict_pack_ms": fused, "layers": L}


class GpuCtx:
    """One process's GPU, rank and barrier for the timed regions."""

    def __init__(self):
        import torch
        import torch.distributed as dist
        self.torch, self.dist = torch, dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(self.local)
        self.device = torch.device("cuda", self.local)
        if self.world > 1:
            import datetime
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=self.device)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()


def measure_decode(ctx, args, steps, warmup, with_e2e=True):
    """Run the current decode workload (DECODE): warm-up steps, then `steps`
    timed steps (barrier + synchronize on both sides, max over ranks), then the
    same number of end-to-end steps through the public API with the inputs
    copied from pinned host memory and the outputs copied back.  Returns the
    measurements (rank-independent fields only)."""
    torch, device = ctx.torch, ctx.device
    from bit_quantized_evicted_b200 import minikv as mk
    from bit_quantized_evicted_b200 import synth

    caches, ws, qin, knin, vnin, out = make_decode_state(torch, mk, synth, device, warmup, steps)
    L, B, Hkv = DECODE["layers"], DECODE["batch"], DECODE["kv_heads"]
    mirror = mirror_for_preset()
    with_mass = bool(DECODE.get("mass"))
    eager = bool(DECODE.get("eager"))
    P = qin.shape[0]

    def layer_calls(q_src, kn_src, vn_src, p, ev=None, o=None):
        """One decode step: the L layer calls, on the current stream (looked up
        once per step, not once per call: it is host time on every call)."""
        o = out if o is None else o
        cur = torch.cuda.current_stream()
        for l in range(L):
            if ev is not None:
                ev[l][0].record(cur)
            decode_call(mk, caches[l], q_src[p, l], kn_src[p, l], vn_src[p, l], o[l], ws, cur)
            if ev is not None:
                ev[l][1].record(cur)

    def step_bytes():
        return [mirror.layer_bytes(l, Hkv, with_mass) for l in range(L)]

    for s in range(warmup):
        layer_calls(qin, knin, vnin, s % P)
        mirror.advance()
    torch.cuda.synchronize()

    # Graph mode: the caches keep their state on the GPU, so one captured step
    # per input-pool slot replays correctly at every later step.  Timing events
    # are recorded between replays, not inside the graphs (event nodes inside a
    # graph would sit between the kernels and slow the step).
    graphs = []
    if not eager:
        for p in range(P):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                layer_calls(qin, knin, vnin, p)
            graphs.append(g)
        torch.cuda.synchronize()

    # ---- device-timed region
    stream = torch.cuda.current_stream(device)
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(L)] for _ in range(steps)]
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    nbytes = []     # per step and layer: algorithmic bytes of the timed steps
    nbytes_k = []   # the same for the steps whose launches are timed one by one (eager)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx.barrier()
    torch.cuda.synchronize()
    with ClockSampler(ctx.local) as clk:
        t0.record(stream)
        for s in range(steps):
            p = (warmup + s) % P
            nbytes.append(step_bytes())
            if eager:   # the step as a caller runs it: nothing between the layer calls
                layer_calls(qin, knin, vnin, p)
            else:
                sev[s][0].record(stream)
                graphs[p].replay()
                sev[s][1].record(stream)
            mirror.advance()
        t1.record(stream)
        torch.cuda.synchronize()
        ctx.barrier()
        if eager:
            # the kernel durations: the same steps again with an event pair around
            # every launch (the events sit between the kernels, so this pass is not
            # the one the step time comes from)
            for s in range(steps):
                p = (warmup + steps + s) % P
                nbytes_k.append(step_bytes())
                layer_calls(qin, knin, vnin, p, evs[s])
                mirror.advance()
            torch.cuda.synchronize()
            ctx.barrier()
    ms = t0.elapsed_time(t1)
    launch_bytes = [b for sb in (nbytes_k if eager else nbytes) for b in sb]
    if eager:
        kern_ms = [evs[s][l][0].elapsed_time(evs[s][l][1]) for s in range(steps) for l in range(L)]
    else:   # a replay runs the L layer launches back to back: its time / L per launch (gaps included)
        kern_ms = [sev[s][0].elapsed_time(sev[s][1]) / L for s in range(steps)]
    ms = max_over_ranks(ms, device)
    tok_s = job_tokens_per_s(B, steps, ctx.world, ms)
    alg_bytes = sum(sum(sb) for sb in nbytes)
    mean_launch_bytes = sum(launch_bytes) / len(launch_bytes)
    mean_launch_s = statistics.mean(kern_ms) * 1e-3
    res = {"value": tok_s, "ms_per_step": ms / steps, "step_bytes": alg_bytes / steps,
           "hbm_gbs": alg_bytes / (ms * 1e-3) / 1e9, "mean_launch_bytes": mean_launch_bytes,
           "mean_launch_us": mean_launch_s * 1e6, "achieved_gbs": mean_launch_bytes / mean_launch_s / 1e9,
           "clocks": clk.summary(), "launches": L * steps * (2 if with_mass else 1), "eager": eager}
    del graphs

    if with_e2e:
        # ---- end to end: inputs from pinned host memory, outputs back, each step.
        # Two buffer sets and two copy streams: while step s computes, one brings
        # step s+1's inputs in and the other takes step s-1's outputs out; events
        # keep each buffer's copies and its compute apart.
        hq = qin.cpu().pin_memory()
        hk = knin.cpu().pin_memory()
        hv = vnin.cpu().pin_memory()
        dq = [torch.empty_like(qin[:1]) for _ in range(2)]
        dk = [torch.empty_like(knin[:1]) for _ in range(2)]
        dv = [torch.empty_like(vnin[:1]) for _ in range(2)]
        dout = [torch.empty_like(out) for _ in range(2)]
        hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        h2d = (dq[0].numel() + dk[0].numel() + dv[0].numel()) * 2
        d2h = out.numel() * 2
        g_e2e = []
        if not eager:
            for i in range(2):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    layer_calls(dq[i], dk[i], dv[i], 0, o=dout[i])
                g_e2e.append(g)
        cin, cout = torch.cuda.Stream(device), torch.cuda.Stream(device)
        in_ready = [torch.cuda.Event() for _ in range(2)]   # buffer i's inputs have landed
        done = [torch.cuda.Event() for _ in range(2)]       # step on buffer i computed
        out_free = [torch.cuda.Event() for _ in range(2)]   # buffer i's outputs copied out
        torch.cuda.synchronize()
        ctx.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cin.wait_stream(stream)
        cout.wait_stream(stream)
        for s in range(steps):
            i, p = s % 2, s % P
            with torch.cuda.stream(cin):
                if s >= 2:
                    cin.wait_event(done[i])      # step s-2 has read this buffer's inputs
                dq[i].copy_(hq[p:p + 1], non_blocking=True)
                dk[i].copy_(hk[p:p + 1], non_blocking=True)
                dv[i].copy_(hv[p:p + 1], non_blocking=True)
                in_ready[i].record(cin)
            stream.wait_event(in_ready[i])
            if s >= 2:
                stream.wait_event(out_free[i])   # step s-2's outputs have left this buffer
            if eager:
                layer_calls(dq[i], dk[i], dv[i], 0, o=dout[i])
            else:
                g_e2e[i].replay()
            done[i].record(stream)
            with torch.cuda.stream(cout):
                cout.wait_event(done[i])
                hout[i].copy_(dout[i], non_blocking=True)
                out_free[i].record(cout)
        stream.wait_stream(cin)
        stream.wait_stream(cout)
        e1.record(stream)
        torch.cuda.synchronize()
        ctx.barrier()
        del g_e2e
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), device)
        res["e2e"] = {"value": job_tokens_per_s(B, steps, ctx.world, e2e_ms), "unit": "tokens/s",
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    status_bad = sum(sum(c.status()) for c in caches)
    if status_bad:
        raise RuntimeError(f"{status_bad} sequences hit the cache capacity")
    del caches, ws, qin, knin, vnin, out
    torch.cuda.empty_cache()
    return res


def launch_name(eager):
    return ("eager: one Python call per layer (step time from calls with nothing between them; kernel "
            "durations from a second pass with an event pair around each launch)" if eager else
            "one CUDA graph replay per step (all layer calls captured, state on the GPU)")


def select_preset(name, args):
    DECODE.clear()
    DECODE.update(DECODE_PRESETS[name])
    if args.layers is not None and name == args.workload:
        DECODE["layers"] = args.layers
    if args.mass and name == args.workload:
        DECODE["mass"] = True
    if args.launch == "eager" or (args.launch == "auto" and AUTO_EAGER):
        DECODE["eager"] = True


# Workloads measured as compact sub-lines of the default run (so that their
# numbers are driver-observed): LLaMA2-13B MHA decode and the pyramid (B = 4).
SUBLINE_WORKLOADS = ("llama2_13b_decode", "pyramid_44k_decode")
SUBLINE_STEPS = 16
# --launch auto: one Python call per layer, for uniform and ragged batches
# alike.  The host-planned kernel is faster than the device-state kernel a graph
# replays, the host stays ahead of the GPU, and back-to-back calls let each
# layer's launch overlap the previous one's drain (programmatic dependent launch).
AUTO_EAGER = True


def run_gpu(args):
    from bit_quantized_evicted_b200 import minikv as mk

    ctx = GpuCtx()
    torch = ctx.torch
    mk.lib()
    pk = peaks()
    main = measure_decode(ctx, args, args.steps, args.warmup)
    B, L = DECODE["batch"], DECODE["layers"]
    cfg_extra = {"parallelism": f"replicas x{ctx.world}"}
    main_cfg = decode_config(cfg_extra, step_bytes=main["step_bytes"])
    eager = main["eager"]

    prefill = run_prefill(torch, mk, __import__("bit_quantized_evicted_b200.synth", fromlist=["x"]), ctx.device, pk) \
        if not args.no_prefill else None
    if prefill:
        prefill["tensor_frac_of_bf16_peak"] = prefill["roofline"]["frac"]

    sublines = {}
    if args.workload == "mistral7b_gqa_decode" and not args.no_sublines and not args.mass and args.layers is None:
        for name in SUBLINE_WORKLOADS:
            select_preset(name, args)
            r = measure_decode(ctx, args, SUBLINE_STEPS, 3, with_e2e=False)
            sublines[name] = {"value": r["value"], "unit": "tokens/s", "ms_per_step": r["ms_per_step"],
                              "steps": SUBLINE_STEPS, "warmup": 3, "hbm_gbs": r["hbm_gbs"],
                              "roofline": {"bound": "hbm", "kernel": "decode_kernel", "achieved": r["achieved_gbs"],
                                           "peak": pk["hbm"], "unit": "GB/s", "frac": r["achieved_gbs"] / pk["hbm"],
                                           "mean_launch_us": r["mean_launch_us"]},
                              "launch": launch_name(r["eager"]),
                              "config": decode_config(cfg_extra, step_bytes=r["step_bytes"])}
        select_preset(args.workload, args)

    cpu = None
    if (ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline and args.workload == "mistral7b_gqa_decode"
            and not args.mass):
        threads = os.cpu_count() or 1
        rate, n, dt = oracle_decode_rate(args.cpu_seconds, threads)
        rate1, n1, dt1 = oracle_decode_rate(max(1.0, args.cpu_seconds / 4), 1)
        cpu = {"value": cpu_tokens_per_s(rate), "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "cpu_model": cpu_model(), "single_thread_value": cpu_tokens_per_s(rate1),
               "sample": f"{n} decode unit-steps (one sequence x KV head of one layer: 6553 kept tokens, 4 query "
                         f"heads, fp64) in {dt:.1f} s on {threads} threads, scaled to 32 layers x 16 x 8 units "
                         f"per step; single-thread value from {n1} unit-steps in {dt1:.1f} s on one thread"}

    csrc = os.path.join(ROOT, "bit_quantized_evicted_b200", "csrc")
    traffic, traffic_note = recorded_traffic(
        "decode_kernel", [os.path.join(csrc, "decode.cu"), os.path.join(csrc, "common.cuh")])
    if args.mass:
        traffic, traffic_note = None, "no capture of the attention-mass variant (decode_kernel<true> + mass_kernel)"
    if ctx.rank == 0:
        line = {
            "metric": METRIC, "value": main["value"], "unit": "tokens/s", "n_gpus": ctx.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": main["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "u2+f16 (2-bit codes, fp16 scales/residual, fp32 accumulate)", "data": "synthetic",
            "config": main_cfg, "launch": launch_name(eager),
            "hbm_gbs": main["hbm_gbs"], "hbm_frac_of_peak": main["hbm_gbs"] / pk["hbm"],
            # cache bytes a layer-step reads (packed codes, scales, zeros, fp16 residual) against the
            # same batch's K and V in fp16: the full context, and the kept tokens only
            "compression": compression(main["step_bytes"]),
            "roofline": {"bound": "hbm", "kernel": "decode_kernel", "achieved": main["achieved_gbs"],
                         "peak": pk["hbm"], "unit": "GB/s", "frac": main["achieved_gbs"] / pk["hbm"],
                         "traffic": traffic, "algorithmic_bytes_per_launch": main["mean_launch_bytes"],
                         "mean_launch_us": main["mean_launch_us"], "peak_source": pk["src"],
                         "traffic_source": traffic_note,
                         # back to back (no events between the launches) consecutive layer
                         # launches overlap their set-up and drain: the step's time per layer
                         "back_to_back_us_per_layer": main["ms_per_step"] * 1e3 / DECODE["layers"]},
            "cpu_baseline": cpu,
            "e2e": main["e2e"],
            "gpu_launches": main["launches"],
            "clocks": main["clocks"],
            "prefill": prefill,
            "sublines": sublines or None,
        }
        print(json.dumps(line), flush=True)
    if ctx.world > 1:
        ctx.dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="minikv", choices=["minikv", "reference"])
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--workload", default="mistral7b_gqa_decode", choices=list(DECODE_PRESETS),
                    help="decode workload (the default one carries the bench line's target)")
    ap.add_argument("--launch", default="auto", choices=["auto", "graph", "eager"],
                    help="graph: state on the GPU, one captured CUDA graph replayed per step; eager: one Python "
                         "call per layer, host-side state; auto: eager")
    ap.add_argument("--mass", action="store_true",
                    help="decode with minikv_decode_attn_mass (H2O-style running attention mass per token)")
    ap.add_argument("--prefill-workload", default="llama2_7b_prefill_select", choices=list(PREFILL_PRESETS))
    ap.add_argument("--layers", type=int, default=None,
                    help="decode layers (fewer only for small profiling runs; default: the workload's)")
    ap.add_argument("--prefill-layers", type=int, default=None,
                    help="prefill layers (fewer only for small profiling runs; default: the workload's)")
    ap.add_argument("--no-sublines", action="store_true",
                    help="skip the compact LLaMA2-13B and pyramid decode sub-lines of the default run")
    args = ap.parse_args()
    select_preset(args.workload, args)
    PREFILL.clear()
    PREFILL.update(PREFILL_PRESETS[args.prefill_workload])
    if args.prefill_layers is not None:
        PREFILL["layers"] = args.prefill_layers
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
