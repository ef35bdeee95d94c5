#!/usr/bin/env python
"""Decode-step benchmark of the persistent megakernel.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--mode mega|perop|perop-graph] [--impl mk|reference]

A *step* is one greedy decode step of the whole decoder (every layer, LM head
and argmax) for the workload's batch, i.e. one megakernel launch.  Inputs are
synthetic (seeded random-init weights and token ids, see
persistent_task_runtime_b200/synth.py).  Prints ONE JSON line on rank 0.

``--mode perop`` times the comparison build: the same task code launched once
per operator (embedding, 5 per layer, LM head) on one stream.
``--mode perop-graph`` replays those launches from a CUDA graph recorded once.

Workloads (default ``8b_b1_ctx512``):
  tiny_b1_p16        2-layer tiny decoder, batch 1, 16-token prompt
  1.5b_b1_ctx256     1.5B-shaped decoder, batch 1, context 256
  8b_b1_ctx512       8B-shaped decoder, batch 1, context 512
  8b_bB_ctx1024      8B-shaped decoder, batch B in {1,2,4,8,16}, context 1024
  8b_b16_ragged      8B-shaped decoder, batch 16, contexts log-uniform 32..8192

Multi-GPU (torchrun): every rank runs an independent replica on its own GPU
(sequences are independent; there is no collective in the data path).  Time is
the max over ranks of the device-timed region; ``value`` is the tokens all
ranks produced divided by that time.
"""

from __future__ import annotations

import argparse
import contextlib
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from persistent_task_runtime_b200 import synth  # noqa: E402

METRIC = "decode tokens/s (µs/step; achieved HBM GB/s vs peak)"
UNIT = "tokens/s"


def parse_workload(name: str) -> dict:
    if name == "tiny_b1_p16":
        return dict(model="tiny", batch=1, lengths=[16], prefill="decode")
    if name == "1.5b_b1_ctx256":
        return dict(model="1.5b", batch=1, lengths=[256], prefill="decode")
    if name == "8b_b1_ctx512":
        return dict(model="8b", batch=1, lengths=[512], prefill="decode")
    if name == "8b_w4_b1_ctx512":
        # the 8B shape with 4-bit (W4A16) projections, batch 1, context 512
        return dict(model="8b", batch=1, lengths=[512], prefill="decode", w4=True)
    if name == "8b4l_b1_ctx512":
        # profiling case: 8B-shaped layers, 4 of them, same kernel (not a bench line)
        return dict(model="8b", layers=4, batch=1, lengths=[512], prefill="synthetic")
    if name.startswith("8b4l_b") and name.endswith("_ctx1024"):
        # profiling case: 8B-shaped layers, 4 of them, batch B at context 1024
        B = int(name[len("8b4l_b"):-len("_ctx1024")])
        return dict(model="8b", layers=4, batch=B, lengths=[1024] * B, prefill="synthetic")
    if name.startswith("8b_b") and name.endswith("_ctx1024"):
        B = int(name[len("8b_b"):-len("_ctx1024")])
        return dict(model="8b", batch=B, lengths=[1024] * B, prefill="synthetic")
    if name == "8b_b16_ragged":
        return dict(model="8b", batch=16, lengths=synth.ragged_lengths(16, 32, 8192, seed=2),
                    prefill="synthetic")
    raise SystemExit(f"unknown workload {name}")


def model_config(wl: dict) -> dict:
    cfg = dict(synth.CONFIGS[wl["model"]])
    if "layers" in wl:
        cfg["n_layers"] = wl["layers"]
    return cfg


# C/C++ tokens that matter to the digest: string and character literals are
# kept whole, comments are dropped (so that a comment inside a literal, or a
# quote inside a comment, is read the way the compiler reads it).
_C_TOKENS = re.compile(r'"(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\'|//[^\n]*|/\*.*?\*/', re.S)


def code_text(src: str) -> str:
    """C/C++ source without its comments, whitespace runs outside literals
    collapsed to one space."""
    parts, at = [], 0
    for m in _C_TOKENS.finditer(src):
        parts.append(" ".join(src[at:m.start()].split()))
        tok = m.group(0)
        parts.append(tok if tok[0] in "\"'" else "")
        at = m.end()
    parts.append(" ".join(src[at:].split()))
    return " ".join(p for p in parts if p)


def source_digest() -> str:
    """sha256 over the code of the kernel and plan sources (the code a DRAM
    capture covers); comments and layout do not enter it."""
    h = hashlib.sha256()
    cdir = os.path.join(ROOT, "persistent_task_runtime_b200", "csrc")
    for name in sorted(os.listdir(cdir)):
        if name.endswith((".cu", ".h")):
            with open(os.path.join(cdir, name), encoding="utf-8") as f:
                h.update(name.encode() + b"\0" + code_text(f.read()).encode())
    with open(os.path.join(ROOT, "include", "mk.h"), encoding="utf-8") as f:
        h.update(code_text(f.read()).encode())
    return h.hexdigest()


def profiled_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary of this workload,
    or None when there is none or the kernel sources changed since."""
    path = os.path.join(ROOT, "profiles", f"mk_decode_step_{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if line.startswith("- ") and " = " in line:
                k, v = line[2:].split(" = ", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_sha256") != source_digest() or "dram_bytes_per_launch" not in vals:
        return None
    return int(vals["dram_bytes_per_launch"])


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest value of x over all ranks (x itself on one rank)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, batch: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job tokens/s: every rank decodes `batch` tokens per step (replicas)."""
    return world * batch * steps / (elapsed_ms / 1e3)


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(),
                                 f"mk_bench_clocks_gpu{gpu_index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, p in rows for i in range(4)
                          if p[5 + i].lower() == "active"})
        busy = [r[0] for r in rows]
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def kv_bytes_read(cfg: dict, positions) -> int:
    """KV bytes one step reads: (pos+1) tokens x layers x K,V x Hkv x d x bf16."""
    per_tok = cfg["n_layers"] * 2 * cfg["n_kv_heads"] * cfg["head_dim"] * 2
    return sum((int(p) + 1) * per_tok for p in positions)


# ---------------------------------------------------------------- our arm --


def run_mk(args, rank: int, world: int, local_rank: int) -> dict:
    from persistent_task_runtime_b200 import mk
    from persistent_task_runtime_b200.kvcache import PagedKVCache

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = parse_workload(args.workload)
    cfg = model_config(wl)
    B, lengths = wl["batch"], list(wl["lengths"])
    W, K = args.warmup, args.steps
    horizon = W + K + max(args.e2e_steps, 0) + 8
    weights = (synth.make_w4_weights(cfg, seed=0, device=dev) if wl.get("w4")
               else synth.make_weights(cfg, seed=0, device=dev))
    cap = [n + horizon for n in lengths]
    kv = PagedKVCache(cfg, B, cap, page=16, device=dev)
    plan = mk.Plan(cfg, weights, max_batch=B, page_size=16, max_seq_len=max(cap) + 16,
                   gemv_path=args.gemv_path, schedule=args.schedule, attn_path=args.attn_path)
    info = plan.info()
    ids = torch.zeros(B, dtype=torch.int32, device=dev)
    pos = torch.zeros(B, dtype=torch.int32, device=dev)
    nids, npos = torch.zeros_like(ids), torch.zeros_like(pos)
    mode = {"mega": mk.MODE_MEGAKERNEL, "perop": mk.MODE_PER_OP,
            "perop-graph": mk.MODE_PER_OP_GRAPH}[args.mode]
    if mode == mk.MODE_PER_OP_GRAPH:
        torch.cuda.set_stream(torch.cuda.Stream(dev))   # graph capture needs a created stream
    stream = torch.cuda.current_stream(dev)

    prefill_info = None
    if wl["prefill"] == "decode" and args.prompt_path == "chunks":
        # the prompt through prompt chunks of up to 16 tokens on a plan of its
        # own (multi-token tasks; the LM head runs on the last chunk only)
        pplan = mk.Plan(cfg, weights, max_batch=16, page_size=16, max_seq_len=max(cap) + 16,
                        prefill=True, attn_path=args.attn_path)
        prompt = synth.make_ids(cfg["vocab"], (B, lengths[0]), seed=1).to(dev).to(torch.int32)
        first = torch.zeros(1, dtype=torch.int32, device=dev)
        for b in range(B):   # warm the plan (and the cache pages) once
            pplan.prefill(prompt[b], b, kv.view, first)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for b in range(B):
            pplan.prefill(prompt[b], b, kv.view, nids[b:b + 1])
        e1.record(stream)
        torch.cuda.synchronize(dev)
        st = pplan.status()
        if st != mk.MK_OK:
            raise RuntimeError(f"prefill failed: {mk.ERROR_NAMES.get(st, st)}")
        ms = e0.elapsed_time(e1)
        prefill_info = {"tokens": B * lengths[0], "ms": round(ms, 3),
                        "tokens_per_s": round(B * lengths[0] / (ms / 1e3), 1),
                        "chunk": 16, "launches": B * ((lengths[0] + 15) // 16)}
        pplan.close()
        ids.copy_(nids)
        pos.fill_(lengths[0])
    elif wl["prefill"] == "decode":
        # teacher-forced prompt through the same decode step
        prompt = synth.make_ids(cfg["vocab"], (lengths[0], B), seed=1).to(dev)
        for t in range(lengths[0]):
            ids.copy_(prompt[t])
            pos.fill_(t)
            plan.step(ids, pos, kv.view, nids, out_pos=npos)
        ids.copy_(nids)
        pos.copy_(npos)
    else:
        hist = synth.make_kv_history(dict(cfg), lengths, seed=3, device=dev)
        kv.load_history(hist, lengths)
        del hist
        ids.copy_(synth.make_ids(cfg["vocab"], (B,), seed=1).to(dev))
        pos.copy_(torch.tensor(lengths, dtype=torch.int32))
    st = plan.status()
    if st != mk.MK_OK:
        raise RuntimeError(f"prefill failed: {mk.ERROR_NAMES.get(st, st)}")
    start_pos = [int(x) for x in pos.tolist()]

    def one(i_ids, i_pos, o_ids, o_pos):
        plan.step(i_ids, i_pos, kv.view, o_ids, out_pos=o_pos, mode=mode)

    for _ in range(W):
        one(ids, pos, nids, npos)
        ids, nids = nids, ids
        pos, npos = npos, pos
    torch.cuda.synchronize(dev)
    pos_timed0 = [int(x) for x in pos.tolist()]

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        t0.record(stream)
        for i in range(K):
            ev[i][0].record(stream)
            one(ids, pos, nids, npos)
            ev[i][1].record(stream)
            ids, nids = nids, ids
            pos, npos = npos, pos
        t1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    st = plan.status()
    if st != mk.MK_OK:
        raise RuntimeError(f"timed steps failed: {mk.ERROR_NAMES.get(st, st)}")
    elapsed_ms = t0.elapsed_time(t1)
    print(f"[bench] rank {rank}: {K} steps in {elapsed_ms:.3f} ms "
          f"({1e3 * elapsed_ms / K:.1f} us/step)", file=sys.stderr, flush=True)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)

    # algorithmic bytes of one step: weights (+ one embedding row per sequence)
    # + KV read over positions 0..pos of every sequence, averaged over the
    # timed steps
    kvb = statistics.mean(kv_bytes_read(cfg, [p + s for p in pos_timed0]) for s in range(K))
    step_bytes = info["weight_bytes"] + B * cfg["hidden"] * 2 + kvb
    mean_launch_ms = statistics.mean(launch_ms)

    # end to end through the host-buffer entry point: H2D of ids/pos from
    # pinned memory, the step, D2H of the argmax ids (+ the status word)
    e2e = None
    if mode == mk.MODE_MEGAKERNEL and args.e2e_steps > 0:
        h_ids = torch.tensor(ids.tolist(), dtype=torch.int32).pin_memory()
        h_pos = torch.tensor(pos.tolist(), dtype=torch.int32).pin_memory()
        h_out = torch.zeros(B, dtype=torch.int32).pin_memory()
        n = args.e2e_steps
        for _ in range(2):  # warm
            plan.step_host(h_ids, h_pos, kv.view, h_out)
            h_ids.copy_(h_out)
            h_pos += 1
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        w0 = time.perf_counter()
        for _ in range(n):
            rc = plan.step_host(h_ids, h_pos, kv.view, h_out)
            if rc != mk.MK_OK:
                raise RuntimeError(f"host step failed: {rc}")
            h_ids.copy_(h_out)
            h_pos += 1
        e2e_s = max_over_ranks(time.perf_counter() - w0, world, dev)
        e2e = {"value": world * B * n / e2e_s, "unit": UNIT,
               "h2d_bytes_per_step": 2 * 4 * B, "d2h_bytes_per_step": 4 * B + 4,
               "us_per_step": 1e6 * e2e_s / n, "steps": n}
    plan.close()
    return dict(elapsed_ms=elapsed_ms, mean_launch_ms=mean_launch_ms, step_bytes=step_bytes,
                launch_ms=launch_ms,
                kv_bytes=kvb, weight_bytes=info["weight_bytes"], info=info, clocks=clk.summary(),
                e2e=e2e, cfg=cfg, B=B, lengths=lengths, mode=args.mode, start_pos=start_pos,
                prefill=prefill_info,
                launches_per_step=(1 if mode == mk.MODE_MEGAKERNEL else
                                   2 + 5 * cfg["n_layers"]))


# ------------------------------------------------------ the oracle (CPU) --


def oracle_layer_timing(cfg: dict, B: int, lengths, weights_cpu, reps: int = 1):
    """Time the oracle on a bounded sample: single decoder layers of one decode
    step (layer time) and the embedding + final norm + LM head (head time)."""
    import numpy as np
    import oracle

    ocfg = oracle.DecoderConfig(**{k: cfg[k] for k in (
        "n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
        "rms_eps", "rope_theta", "qk_norm")})
    one = dict(cfg, n_layers=1)
    ocfg1 = oracle.DecoderConfig(**{k: one[k] for k in (
        "n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
        "rms_eps", "rope_theta", "qk_norm")})
    wcls = oracle.W4Weights if "w4" in weights_cpu["layers"][0] else oracle.Weights
    W = wcls(weights_cpu, keep_f64=False)
    hist = synth.make_kv_history(one, lengths, seed=3)
    cache = oracle.KVCache(ocfg1, B, max(lengths) + 2)
    for b, n in enumerate(lengths):
        cache.load_history(0, b, hist[0]["k"][b, :, :n].double().numpy(),
                           hist[0]["v"][b, :, :n].double().numpy())
    ids = [1] * B
    pos = list(lengths)
    # head: embedding rows + final norm + LM head (a zero-layer pass)
    t = time.perf_counter()
    oracle.decode_step(ocfg1, W, cache, ids, pos, layers=0)
    head_s = time.perf_counter() - t
    layer_s = []
    for _ in range(reps):
        t = time.perf_counter()
        oracle.decode_step(ocfg1, W, cache, ids, pos, layers=1)
        layer_s.append(time.perf_counter() - t - head_s)
    del np
    return head_s, max(1e-9, statistics.median(layer_s)), ocfg.n_layers


def cpu_weights_sample(cfg: dict, w4: bool = False) -> dict:
    """CPU copy of the weights the oracle sample touches (first layer + head),
    drawn by the same generator on the CPU (4-bit layers for a 4-bit workload)."""
    if w4:
        return synth.make_w4_weights(cfg, seed=0, device="cpu", layers=1)
    return synth.make_weights(cfg, seed=0, device="cpu", layers=1)


def cores_used() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_threads(n: int):
    """(context that limits the oracle's BLAS/OpenMP and torch threads to n,
    threads used); n <= 0 keeps the process's thread pools as they are and
    reports their size (torchrun, for one, sets OMP_NUM_THREADS=1)."""
    from threadpoolctl import threadpool_info, threadpool_limits
    if n <= 0:
        pools = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        return contextlib.nullcontext(), max(pools) if pools else cores_used()
    torch.set_num_threads(n)
    return threadpool_limits(limits=n), n


def run_reference(args) -> dict:
    wl = parse_workload(args.workload)
    cfg = model_config(wl)
    B, lengths = wl["batch"], list(wl["lengths"])
    w = cpu_weights_sample(cfg, bool(wl.get("w4")))
    head_s, _, L = oracle_layer_timing(cfg, B, lengths, w)
    per_step = []
    for i in range(args.warmup + args.steps):
        h, layer_s, _ = oracle_layer_timing(cfg, B, lengths, w)
        if i >= args.warmup:
            per_step.append(head_s + L * layer_s)
    step_s = statistics.median(per_step)
    return dict(step_s=step_s, head_s=head_s, L=L, B=B, cfg=cfg, lengths=lengths)


# --------------------------------------------------------------------- main --


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--workload", default="8b_b1_ctx512")
    ap.add_argument("--mode", choices=["mega", "perop", "perop-graph"], default="mega")
    ap.add_argument("--impl", choices=["mk", "reference"], default="mk")
    ap.add_argument("--e2e-steps", type=int, default=32)
    ap.add_argument("--gemv-path", type=int, default=0, choices=[0, 1, 2, 3],
                    help="projections: 0 automatic, 1 mma.sync pages, 2 tcgen05 tiles, "
                         "3 mma.sync pages staged in tensor memory")
    ap.add_argument("--attn-path", type=int, default=0, choices=[0, 1, 2],
                    help="attention: 0 automatic, 1 CUDA-core FMA, 2 mma.sync tiles")
    ap.add_argument("--prompt-path", choices=["chunks", "decode"], default="chunks",
                    help="how a workload's prompt fills the cache: prompt chunks of 16 tokens "
                         "(mk_prefill_chunk) or one decode step per token")
    ap.add_argument("--schedule", type=int, default=0, choices=[0, 1, 2],
                    help="0 automatic (solidified), 1 solidified per-CTA task lists, 2 dynamic queue")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-threads", type=int, default=0,
                    help="threads for the CPU oracle (0: the process's BLAS thread pool as set up)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = parse_workload(args.workload)
    cfg = model_config(wl)
    config = {"workload": args.workload, "model_shape": wl["model"], "batch": wl["batch"],
              "weights_format": "4-bit codes + bf16 scale per 128 columns (W4A16)"
              if wl.get("w4") else "bf16",
              "context": wl["lengths"] if len(set(wl["lengths"])) > 1 else wl["lengths"][0],
              "kv_page": 16, "weights": "random N(0,0.02) bf16", "ids": "uniform random",
              "prefill": (("prompt chunks of 16 tokens" if args.prompt_path == "chunks"
                           else "teacher-forced decode steps") if wl["prefill"] == "decode"
                          else "synthetic KV history"),
              "l2": "inputs larger than L2 (every step streams all weights)",
              "parallelism": f"replicas{world}"}

    if args.impl == "reference":
        if rank != 0:
            return
        ctx, cores = oracle_threads(args.oracle_threads)
        with ctx:
            r = run_reference(args)
        val = r["B"] / r["step_s"]
        sample = (f"per step: one decoder layer of one {wl['model']} decode step "
                  f"(batch {r['B']}) timed, x{r['L']} layers + embedding/final-norm/LM-head "
                  f"timed once")
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * r["step_s"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        torch.distributed.init_process_group(
            "nccl", timeout=__import__("datetime").timedelta(seconds=120))
    r = run_mk(args, rank, world, local_rank)
    K = args.steps
    ms_per_step = r["elapsed_ms"] / K
    value = job_throughput(world, r["B"], K, r["elapsed_ms"])
    peaks = measured_peaks()
    achieved = r["step_bytes"] / (r["mean_launch_ms"] / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": profiled_traffic(args.workload),
                "traffic_source": ("ncu DRAM bytes of one launch, read from the committed "
                                   f"profiles/mk_decode_step_{args.workload}.md, used only while "
                                   "the kernel sources hash to the digest recorded there"),
                "peak_source": peaks["source"],
                "bytes_per_step": int(r["step_bytes"]), "kernel_us": 1e3 * r["mean_launch_ms"],
                "vs_8tbs": round(achieved / 8000.0, 4)}
    line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "us_per_step": round(1e3 * ms_per_step, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config, "mode": r["mode"],
            "plan": {"gemv_path": r["info"]["gemv_path"], "schedule": r["info"]["schedule"],
                     "attn_path": r["info"]["attn_path"], "n_tasks": r["info"]["n_tasks"]},
            "step_us": {"mean": round(1e3 * statistics.mean(r["launch_ms"]), 1),
                        "p50": round(1e3 * statistics.median(r["launch_ms"]), 1),
                        "min": round(1e3 * min(r["launch_ms"]), 1),
                        "max": round(1e3 * max(r["launch_ms"]), 1),
                        "std": round(1e3 * (statistics.pstdev(r["launch_ms"])
                                            if len(r["launch_ms"]) > 1 else 0.0), 2)},
            "roofline": roofline, "clocks": r["clocks"], "e2e": r["e2e"],
            "prompt": r["prefill"],
            "gpu_launches": K * r["launches_per_step"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        w = cpu_weights_sample(cfg, bool(wl.get("w4")))
        ctx, cores = oracle_threads(args.oracle_threads)
        with ctx:
            head_s, layer_s, L = oracle_layer_timing(cfg, r["B"], r["lengths"], w)
        step_s = head_s + L * layer_s
        line["cpu_baseline"] = {
            "value": r["B"] / step_s, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": (f"one decoder layer + embedding/final-norm/LM-head of one decode step "
                       f"(batch {r['B']}), scaled to {L} layers")}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
