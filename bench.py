#!/usr/bin/env python
"""Benchmark of one Medusa draft-and-verify step on B200.

A step is one pass of the whole hot path over one batch of synthetic input:
md_medusa_heads (K heads + per-head top-k) -> md_tree_build -> md_tree_attention
(one layer of the verification pass) -> md_tree_accept. The default workload is
the Llama-3.3-70B-shaped one at B = 1 (d 8192, V 128256, K 4, 64-candidate tree
from top-10 heads, 64 q / 8 kv heads, dh 128, KV prefix 4096, greedy).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl medusa|reference]

Prints one JSON line (rank 0). With N > 1 (torchrun) every rank runs its own
replica on its own GPU (requests are independent: no collective on the data
path); the timed region is bracketed by barriers and the slowest rank's time
is used; `value` counts the steps of all ranks.

`--impl reference` times the CPU oracle (plain fp64 numpy, host cores) on a
bounded sample of the same workload: the vocabulary projection and the
residual block on a fraction of their output columns and the attention on the
same fraction of its rows, scaled back to a whole step; tree build and
acceptance run in full.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from seeded_inputs import gen, synth  # noqa: E402
from seeded_inputs.workloads import WORKLOADS  # noqa: E402

METRIC = "Medusa head+tree-verify steps/s at 70B shapes B=1; HBM GB/s vs B200 peak"
L2_BYTES = 126 * 1024 * 1024


# --------------------------------------------------------------------------- #
# Algorithmic byte and flop counts (what the method must move / compute).
# --------------------------------------------------------------------------- #
def heads_bytes(w):
    """Weights, hidden rows in, top-k out; sampled drafts also read one uniform
    and write one logit per (row, head, token)."""
    extra = 8 * w.M * w.K * w.V if w.mode == "rejection" else 0
    return w.head_weight_bytes() + 2 * w.M * w.d + 8 * w.M * w.K * w.kmax + extra


PROFILE_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles")
TRAFFIC_PROFILE = os.path.join(PROFILE_DIR, "heads_traffic_prof-8b-v32000.md")
# The kernel sources each heads path runs (a traffic capture is tied to them).
HEADS_SOURCES = {"stream": ("heads.cuh", "common.cuh"),
                 "weights-as-m": ("heads.cuh", "heads_skinny.cuh", "common.cuh"),
                 "row-tiles": ("heads.cuh", "heads_gemm.cuh", "heads_gemm2.cuh", "common.cuh")}


def heads_path(M: int) -> str:
    return "stream" if M == 1 else "weights-as-m" if M <= 32 else "row-tiles"


def hydra_levels(parent):
    """Nodes with children at each depth (per request): the head rows of
    each level of md_hydra_draft."""
    depth = [0] * len(parent)
    for j in range(1, len(parent)):
        depth[j] = depth[parent[j]] + 1
    with_children = set(parent[1:])
    return [sum(1 for p in with_children if depth[p] == lvl) for lvl in range(max(depth))]


def hydra_bytes(w, levels):
    """Per level: one head's weights, the h and E rows its inputs read, its top-k out."""
    head = 2 * (w.d * w.d + w.d + w.d * w.V)
    return sum(head + 2 * 2 * w.B * n * w.d + 8 * w.B * n * w.kmax for n in levels)


def hydra_flops(w, levels):
    return sum(2 * w.B * n * (w.d * w.d + w.d * w.V) for n in levels)


def heads_source_digest(path: str = "stream") -> str:
    """sha256 (first 16 hex digits) of the heads sources with comments and
    whitespace removed: a change of code invalidates a recorded capture, a
    change of wording does not."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in HEADS_SOURCES[path]:
        with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "medusa_draft_heads_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(re.sub(r"\s+", "", src).encode())
    return h.hexdigest()[:16]


def _traffic_record(path):
    """(bytes per call, ratio to the algorithmic bytes, digest) from a traffic
    profile, or None."""
    if not os.path.exists(path):
        return None
    rec = {}
    with open(path) as fh:
        for line in fh:
            for key in ("traffic_per_call_bytes", "traffic_per_algorithmic_byte", "heads_source_digest"):
                if line.startswith(key + ":"):
                    rec[key] = line.split(":")[1].split()[0]
    return rec


def measured_heads_traffic(w):
    """DRAM bytes of one heads call, from ncu captures recorded under
    profiles/: the capture of this very workload when there is one (its
    metrics take a single ncu pass, so full-size calls are captured directly),
    else, for one-row streaming calls, the ratio DRAM traffic / algorithmic
    bytes of the 8B-shaped V 32000 capture times this workload's algorithmic
    bytes. Returns (bytes, source), or (None, None) when there is no capture
    or the heads sources changed since it was taken."""
    digest = heads_source_digest(heads_path(w.M))
    own = _traffic_record(os.path.join(PROFILE_DIR, f"heads_traffic_{w.name}.md"))
    if own and own.get("heads_source_digest") == digest and "traffic_per_call_bytes" in own:
        return float(own["traffic_per_call_bytes"]), f"profiles/heads_traffic_{w.name}.md (this workload)"
    if w.M > 1:
        return None, None
    rec = _traffic_record(TRAFFIC_PROFILE)
    if rec and rec.get("heads_source_digest") == digest and "traffic_per_algorithmic_byte" in rec:
        return (float(rec["traffic_per_algorithmic_byte"]) * heads_bytes(w),
                "profiles/heads_traffic_prof-8b-v32000.md scaled by algorithmic bytes")
    return None, None


def slowest_rank_ms(ms: float, world: int, device=None) -> float:
    """Elapsed milliseconds of the slowest rank (all-reduce MAX; a no-op on one rank)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, steps: int, max_ms: float) -> float:
    """Whole-job steps/s: every rank ran `steps` steps within the slowest rank's time."""
    return world * steps / (max_ms / 1000.0)


def heads_flops(w):
    return 2 * w.M * w.K * w.d * (w.d + w.V)


def attention_bytes(w, P):
    kv = sum(2 * w.Hkv * (int(p) + w.T) * w.dh * 2 for p in P)
    return kv + w.B * w.T * w.Hq * w.dh * (2 + 4)


def attention_flops(w, P):
    return sum(4 * w.Hq * w.T * (int(p) + w.T) * w.dh for p in P)


def accept_bytes(w):
    """Greedy / typical / sampled rules scan every tree row. The rejection rule
    reads at most the K + 1 target rows on the accepted path and K head rows
    per request (an upper bound: the walk stops at the first full rejection)."""
    if w.mode == "rejection":
        return w.B * (2 * w.K + 1) * w.V * 4
    return w.B * w.T * w.V * 4


NOMINAL_HBM_GBS = 7700.0   # B200 HBM3e, HGX figure (context only)


def read_stream_gbs(dev, nbytes=1 << 32, reps=10):
    """A read-only denominator for the weight streams: GB/s of one plain
    read-and-fold pass over a 4 GiB buffer (md_stream_read, 16-byte
    non-allocating loads), timed with CUDA events on its stream. The measured
    copy bandwidth moves every byte twice (read and write), and a read-only
    stream can exceed it."""
    import torch

    import medusa_draft_heads_b200 as md
    t = torch.zeros(nbytes // 4, dtype=torch.int32, device=dev)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    st = torch.cuda.current_stream(dev)
    for _ in range(3):
        md.stream_read(t, sink, st)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(reps):
        md.stream_read(t, sink, st)
    e1.record(st)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / reps
    del t
    torch.cuda.empty_cache()
    return nbytes / (ms / 1000.0) / 1e9


def attention_launches(w) -> int:
    """The tcgen05 tree attention is one kernel (its KV splits merge through
    distributed shared memory); GQA groups that do not divide 128 rows take
    the CUDA-core kernel and its merge kernel."""
    return 1 if 128 % (w.Hq // w.Hkv) == 0 else 2


def step_launches(w) -> int:
    """This library's kernels in one step: heads 3 (residual block, projection
    with the top-k, merge), tree build 1, attention, acceptance 2 (row scan or
    per-row draw, then the walk; 1 for the rejection rule)."""
    return 3 + 1 + attention_launches(w) + (1 if w.mode == "rejection" else 2)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------------------- #
# Clock sampling during the timed region.
# --------------------------------------------------------------------------- #
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        self.path = os.path.join("/tmp", f"medusa_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3] not in ("", "[N/A]"))}


# --------------------------------------------------------------------------- #
# The oracle on a bounded sample (cpu_baseline leg and --impl reference).
# --------------------------------------------------------------------------- #
def _weight_columns(key, k, n_in, n_out, cols, sigma):
    """Rows 0 .. n_in-1 of head k's [n_in, n_out] weight at the columns `cols`
    (bf16 bits), drawn from the counter-based generator in row blocks so the
    index arrays stay small."""
    cols = np.asarray(cols, dtype=np.uint64)[None, :]
    out = np.empty((n_in, cols.shape[1]), dtype=np.uint16)
    step = max(1, (1 << 23) // cols.shape[1])
    for i0 in range(0, n_in, step):
        ii = np.arange(i0, min(n_in, i0 + step), dtype=np.uint64)[:, None]
        idx = (np.uint64(k) * np.uint64(n_in) + ii) * np.uint64(n_out) + cols
        out[i0:i0 + ii.shape[0]] = gen.normal_bf16_at(key, idx.ravel(), sigma).reshape(ii.shape[0], -1)
    return out


class OracleSampler:
    """Times the CPU oracle on a fraction `frac` of the step's column/row work
    and scales it back to one whole step. Inputs are drawn on the host from
    the same seeded generator."""

    def __init__(self, w, frac: float, seed_offset: int = 0):
        from oracle import tree as ot
        self.w = w
        self.frac = frac
        s = w.seed + seed_offset
        d, V, K = w.d, w.V, w.K
        rng = np.random.default_rng(1234)
        self.cols_o = np.sort(rng.choice(d, max(1, int(round(d * frac))), replace=False))
        self.cols_v = np.sort(rng.choice(V, max(1, int(round(V * frac))), replace=False))
        kw = [gen.stream_key(s, n) for n in ("W1", "Wv")]
        # W1[k, i, o] and Wv[k, i, v] at the sampled columns only (counter-based draws)
        self.W1 = np.stack([_weight_columns(kw[0], k, d, d, self.cols_o, w.w_sigma) for k in range(K)])
        self.Wv = np.stack([_weight_columns(kw[1], k, d, V, self.cols_v, w.w_sigma) for k in range(K)])
        self.b1 = gen.normal_bf16(s, "b1", (K, d), w.w_sigma)
        self.h = gen.normal_bf16(s, "h", (w.M, d), 1.0)
        self.root = synth.root_tokens(s, w.B, V)
        self.P = synth.prefix_lengths(s, w.B, *w.prefix)
        tups = ot.select_tree(w.k_per_head, w.accept, w.n_nodes)
        self.parent, self.rank, _ = ot.spec_from_tuples(tups)
        self.q = gen.normal_bf16(s, "q", (w.B, w.T, w.Hq, w.dh), 1.0)
        self.k = gen.normal_bf16(s, "k_cache", (w.B, w.Hkv, w.S_max, w.dh), 1.0)
        self.v = gen.normal_bf16(s, "v_cache", (w.B, w.Hkv, w.S_max, w.dh), 1.0)
        nrows = w.B * w.T * w.Hq
        pick = rng.choice(nrows, max(1, int(round(nrows * frac))), replace=False)
        self.rows = [(int(r // (w.T * w.Hq)), int((r // w.Hq) % w.T), int(r % w.Hq)) for r in pick]
        self.topk_ids = rng.integers(0, V, (w.M, K, w.kmax)).astype(np.int32)
        # z of the right shape for the sampled projection (its values do not change the work)
        self.z = np.repeat(self.h[:, None, :], K, axis=1)
        tokens = synth.synthetic_tree_tokens(s, w.B, self.parent, V, root_tokens=self.root)
        self.tokens = tokens
        self.logits = synth.planted_logits(s, self.parent, tokens, V, w.accept, sigma=w.logit_sigma, bump=w.bump)
        # uniforms of the sampled rules; the heads' logits the rejection rule
        # reads over the whole vocabulary (their values do not change the work)
        self.u = rng.random((3, w.B, w.T))
        if w.mode == "rejection":
            self.u_draft = rng.random((w.M, K, len(self.cols_v)))
            self.head_logits = rng.normal(0.0, w.logit_sigma, (w.M, K, V))

    def step(self):
        """Returns the estimated seconds of one whole oracle step."""
        from oracle import accept as oacc
        from oracle import attention as oa
        from oracle import heads as oh
        from oracle import rejection as orj
        from oracle import tree as ot
        w = self.w
        t0 = time.perf_counter()
        oh.residual_block_columns(self.h, self.W1, self.b1[:, self.cols_o], self.cols_o)
        t1 = time.perf_counter()
        logits = oh.vocab_logits(self.z, self.Wv)          # self.Wv holds the sampled columns only
        if w.mode == "rejection":
            orj.sampled_drafts(logits, w.k_per_head, w.kmax, w.temperature, self.u_draft)
        else:
            oh.heads_topk(logits, w.k_per_head, w.kmax)
        t2 = time.perf_counter()
        ot.tree_build(self.parent, self.rank, self.topk_ids, self.root, self.P)
        t3 = time.perf_counter()
        oa.tree_attention(self.q, self.k, self.v, self.P, self.parent, rows=self.rows)
        t4 = time.perf_counter()
        if w.mode == "greedy":
            oacc.greedy_accept(self.logits, self.tokens, self.parent, w.K)
        elif w.mode == "typical":
            oacc.typical_accept(self.logits, self.tokens, self.parent, w.K, w.temperature, w.eps, w.alpha)
        elif w.mode == "sample":
            oacc.sampled_accept(self.logits, self.tokens, self.parent, w.K, w.temperature, self.u[0])
        else:
            orj.rejection_accept(self.logits, self.tokens, self.parent, self.rank, w.K, w.temperature,
                                 self.head_logits, np.arange(w.B), w.temperature, self.u[1], self.u[2])
        t5 = time.perf_counter()
        return (t1 - t0) / self.frac + (t2 - t1) / self.frac + (t3 - t2) + (t4 - t3) / self.frac + (t5 - t4)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, w):
    """--impl reference: the CPU oracle, K sample steps after W warm-ups."""
    frac = args.ref_frac
    smp = OracleSampler(w, frac)
    for _ in range(args.warmup):
        smp.step()
    est = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        est.append(smp.step())
    wall = time.perf_counter() - t0
    sec = float(np.mean(est))
    value = 1.0 / sec
    sample = (f"per step: residual block and vocabulary projection on {frac:.4g} of their output columns, "
              f"attention on {frac:.4g} of its (token, head) rows, scaled by 1/{frac:.4g}; tree build and "
              f"acceptance in full; {args.steps} sample steps took {wall:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * sec, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w, synth.prefix_lengths(w.seed, w.B, *w.prefix)),
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": blas_threads(),
                             "host_cpus": os.cpu_count(), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_oracle_check(args, w):
    """One whole (unsampled) oracle step of the workload beside the sampled
    estimate that the cpu_baseline and reference legs report, so the 1/frac
    scaling of the sampled step can be checked against the real thing."""
    t0 = time.perf_counter()
    full = OracleSampler(w, 1.0)
    setup = time.perf_counter() - t0
    full_s = [full.step() for _ in range(args.oracle_check_steps)]
    del full
    smp = OracleSampler(w, args.cpu_frac)
    smp.step()
    est = [smp.step() for _ in range(5)]
    unsampled, sampled = float(np.median(full_s)), float(np.median(est))
    print(json.dumps({"oracle_check": w.name, "unsampled_step_s": unsampled, "unsampled_steps": full_s,
                      "sampled_estimate_s": sampled, "frac": args.cpu_frac, "estimate_over_unsampled":
                      sampled / unsampled, "setup_s": setup, "cores": blas_threads(),
                      "host_cpus": os.cpu_count()}), flush=True)


def config_dict(w, P):
    return {"workload": w.name, "B": w.B, "heads_rows": w.M, "d": w.d, "V": w.V, "K": w.K,
            "k_per_head": list(w.k_per_head), "tree_nodes": w.n_nodes, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv,
            "dh": w.dh, "prefix": list(w.prefix) if P is None else [int(p) for p in P], "accept": w.mode,
            "l2": "inputs larger than L2: 8.99 GB of head weights stream every step; attention and acceptance "
                  "inputs rotate over buffer sets totalling more than 2x L2"}


# --------------------------------------------------------------------------- #
# The CUDA arm.
# --------------------------------------------------------------------------- #
def seed_step_uniforms(step, seed):
    """Seeded uniforms for the rules that draw random numbers: one per tree row
    (sampled acceptance), or per (row, head, token) for the draws plus two per
    tree row for the tests and the bonus draw (rejection acceptance)."""
    import torch
    g = torch.Generator().manual_seed(seed)
    for t in (step.uniforms, step.u_draft, step.u_accept, step.u_residual):
        if t is not None:
            t.copy_(torch.rand(t.shape, generator=g).clamp_(1e-7, 1 - 1e-7))


def run_medusa(args, w):
    import torch
    import torch.distributed as dist

    import medusa_draft_heads_b200 as md
    from medusa_draft_heads_b200.step import MedusaStep
    from seeded_inputs import device as sdev

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    seed = w.seed + rank
    stream = torch.cuda.Stream(dev)

    # ---- resident inputs -------------------------------------------------
    bf = dict(dtype=torch.bfloat16, device=dev)
    W1 = sdev.fill_normal(torch.empty((w.K, w.d, w.d), **bf), seed, "W1", w.w_sigma)
    b1 = sdev.fill_normal(torch.empty((w.K, w.d), **bf), seed, "b1", w.w_sigma)
    Wv = sdev.fill_normal(torch.empty(((w.d, w.V) if w.shared_vocab else (w.K, w.d, w.V)), **bf), seed, "Wv",
                          w.w_sigma)
    h = sdev.fill_normal(torch.empty((w.M, w.d), **bf), seed, "h", 1.0)
    root = torch.from_numpy(synth.root_tokens(seed, w.B, w.V)).to(dev)
    P = synth.prefix_lengths(seed, w.B, *w.prefix)
    prefix = torch.from_numpy(P).to(dev)
    tups = md.select_tree(w.k_per_head, w.accept, w.n_nodes)
    step = MedusaStep(B=w.B, M=w.M, d=w.d, V=w.V, K=w.K, k_per_head=w.k_per_head, tree_tuples=tups, Hq=w.Hq,
                      Hkv=w.Hkv, dh=w.dh, S_max=w.S_max, mode=w.mode, temperature=w.temperature, eps=w.eps,
                      alpha=w.alpha, device=dev, shared_vocab=w.shared_vocab)
    seed_step_uniforms(step, w.seed)
    head_row = None
    if w.M != w.B:
        head_row = torch.arange(w.B, dtype=torch.int32, device=dev) * w.T

    # attention / acceptance inputs: buffer sets that together exceed 2x L2
    set_bytes = 2 * w.B * w.Hkv * w.S_max * w.dh * 2 + w.B * w.T * w.V * 4 + w.B * w.T * w.Hq * w.dh * 2
    nsets = max(2, -(-2 * L2_BYTES // set_bytes))
    with torch.cuda.stream(stream):
        step.heads(h, W1, b1, Wv)
        step.build(root, prefix, head_row)
    stream.synchronize()
    tokens = step.tokens.cpu().numpy()
    parent_np = np.array(step.tree.parent)
    logits_dev = synth.planted_logits_device(seed, parent_np, tokens, w.V, w.accept, sigma=w.logit_sigma,
                                             bump=w.bump, device=dev)
    sets = []
    for i in range(nsets):
        q = sdev.fill_normal(torch.empty((w.B, w.T, w.Hq, w.dh), **bf), seed + 7919 * i, "q", 1.0)
        kc = sdev.fill_normal(torch.empty((w.B, w.Hkv, w.S_max, w.dh), **bf), seed + 7919 * i, "k_cache", 1.0)
        vc = sdev.fill_normal(torch.empty((w.B, w.Hkv, w.S_max, w.dh), **bf), seed + 7919 * i, "v_cache", 1.0)
        sets.append((q, kc, vc, logits_dev.clone()))
    torch.cuda.synchronize()

    def one_step(i, ev=None):
        q, kc, vc, lg = sets[i % nsets]
        if ev is not None:
            ev[0].record(stream)
        step.heads(h, W1, b1, Wv)
        if ev is not None:
            ev[1].record(stream)
        step.build(root, prefix, head_row)
        if ev is not None:
            ev[2].record(stream)
        step.attention(q, kc, vc, prefix)
        if ev is not None:
            ev[3].record(stream)
        step.accept(lg)
        if ev is not None:
            ev[4].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            one_step(i)
    stream.synchronize()
    status = md.device_status(stream=stream)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        time.sleep(0.3)
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            start.record(stream)
            for i in range(args.steps):
                one_step(i, evs[i])
            end.record(stream)
        torch.cuda.synchronize()
        barrier()
    total_ms = start.elapsed_time(end)
    per_call = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])
    clk = clocks.summary()

    total_ms = slowest_rank_ms(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = job_value(world, args.steps, total_ms)

    # ---- the same step replayed from CUDA graphs (one per buffer set) -------
    graph_ms = None
    try:
        if world > 1:   # every rank must take the same collective steps: eager only
            raise RuntimeError("multi-rank run")
        graphs = []
        for i in range(nsets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                one_step(i)
            graphs.append(g)
        for i in range(args.warmup):
            graphs[i % nsets].replay()
        barrier()
        torch.cuda.synchronize()
        gs, ge = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            gs.record(stream)
            for i in range(args.steps):
                graphs[i % nsets].replay()
            ge.record(stream)
        torch.cuda.synchronize()
        barrier()
        graph_ms = slowest_rank_ms(gs.elapsed_time(ge), world, dev) / args.steps
        del graphs
    except Exception as exc:  # capture not possible here: report the eager number only
        print(f"cuda graph replay unavailable: {exc}", file=sys.stderr)
        torch.cuda.synchronize()

    # ---- end to end through the public API with host buffers ---------------
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, step, h, W1, b1, Wv, root, prefix, head_row, sets, stream, dev, world, barrier)

    if rank == 0:
        peaks = measured_peaks()
        hb = heads_bytes(w)
        hf = heads_flops(w)
        heads_ms = float(per_call[:, 0].mean())
        if w.M > 32:     # row-tile tensor-core GEMMs: bound by the bf16 tensor pipe
            roof = {"kernel": "md_medusa_heads (tcgen05 GEMMs: residual block, vocabulary projection + top-k; merge)",
                    "bound": "tensor", "achieved": hf / (heads_ms / 1000.0) / 1e12,
                    "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                    "algorithmic_flops": hf, "peak_note": "measured cuBLAS bf16, sustained (kernel inside a long step)"}
        else:
            rd = read_stream_gbs(dev)
            roof = {"kernel": ("md_medusa_heads (residual block + vocabulary stream + top-k merge)" if w.M == 1 else
                               "md_medusa_heads (tcgen05 weight stream, weights as the MMA's M; top-k merge)"),
                    "bound": "hbm", "achieved": hb / (heads_ms / 1000.0) / 1e9, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "algorithmic_bytes": hb,
                    "peak_note": "copy bandwidth (every byte read and written); a read-only stream can exceed it, "
                                 "so frac_read (one read-only pass over 4 GiB, md_stream_read, timed in this run) "
                                 "and frac_nominal are given too",
                    "read_peak": rd, "nominal_peak": NOMINAL_HBM_GBS}
            roof["frac_read"] = roof["achieved"] / rd
            roof["frac_nominal"] = roof["achieved"] / NOMINAL_HBM_GBS
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["above_peak"] = roof["frac"] > 1.0
        if args.traffic is not None:
            roof["traffic"], roof["traffic_source"] = args.traffic, "--traffic"
        else:
            roof["traffic"], roof["traffic_source"] = measured_heads_traffic(w)
        roof["avg_ms"] = heads_ms
        roof["peak_source"] = peaks["source"]
        ab = attention_bytes(w, P)
        af = attention_flops(w, P)
        attn_ms = float(per_call[:, 2].mean())
        acc_ms = float(per_call[:, 3].mean())
        step_bytes = hb + ab + accept_bytes(w)
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_baseline(w, args)
        line = {
            "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(w, P),
            "roofline": roof,
            "graph_replay": None if graph_ms is None else {
                "ms_per_step": graph_ms, "steps_per_s": job_value(world, 1, graph_ms),
                "note": "the same four calls captured once per buffer set in CUDA graphs and replayed"},
            "step_gbs": step_bytes / (ms_per_step / 1000.0) / 1e9 / 1.0,
            "step_gbs_frac": step_bytes / (ms_per_step / 1000.0) / 1e9 / peaks["hbm_gbs"],
            "per_call_ms": {"medusa_heads": heads_ms, "tree_build": float(per_call[:, 1].mean()),
                            "tree_attention": attn_ms, "tree_accept": acc_ms},
            "attention": {"bytes": ab, "flops": af, "gbs": ab / (attn_ms / 1000) / 1e9,
                          "tflops": af / (attn_ms / 1000) / 1e12},
            "accept": {"bytes": accept_bytes(w), "gbs": accept_bytes(w) / (acc_ms / 1000) / 1e9},
            "gpu_launches": step_launches(w) * args.steps,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "accepted_len_mean": float(step.accept_len.float().mean().item()),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_part(args, w):
    """Time one of the four calls alone on the workload's shapes (for profiling
    and per-kernel study); only that call's inputs are allocated."""
    import torch

    import medusa_draft_heads_b200 as md
    from medusa_draft_heads_b200.step import MedusaStep
    from seeded_inputs import device as sdev

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    bf = dict(dtype=torch.bfloat16, device=dev)
    seed = w.seed
    tups = md.select_tree(w.k_per_head, w.accept, w.n_nodes)
    step = MedusaStep(B=w.B, M=w.M, d=w.d, V=w.V, K=w.K, k_per_head=w.k_per_head, tree_tuples=tups, Hq=w.Hq,
                      Hkv=w.Hkv, dh=w.dh, S_max=w.S_max, mode=w.mode, temperature=w.temperature, eps=w.eps,
                      alpha=w.alpha, device=dev, shared_vocab=w.shared_vocab)
    seed_step_uniforms(step, w.seed)
    P = synth.prefix_lengths(seed, w.B, *w.prefix)
    prefix = torch.from_numpy(P).to(dev)
    if args.part == "heads":
        W1 = sdev.fill_normal(torch.empty((w.K, w.d, w.d), **bf), seed, "W1", w.w_sigma)
        b1 = sdev.fill_normal(torch.empty((w.K, w.d), **bf), seed, "b1", w.w_sigma)
        Wv = sdev.fill_normal(torch.empty(((w.d, w.V) if w.shared_vocab else (w.K, w.d, w.V)), **bf), seed, "Wv",
                              w.w_sigma)
        h = sdev.fill_normal(torch.empty((w.M, w.d), **bf), seed, "h", 1.0)
        call = lambda i: step.heads(h, W1, b1, Wv)                              # noqa: E731
        nbytes, nflops, launches = heads_bytes(w), heads_flops(w), 3
    elif args.part == "hydra":
        W1 = sdev.fill_normal(torch.empty((w.K, w.d, w.d), **bf), seed, "W1", w.w_sigma)
        b1 = sdev.fill_normal(torch.empty((w.K, w.d), **bf), seed, "b1", w.w_sigma)
        Wv = sdev.fill_normal(torch.empty((w.K, w.d, w.V), **bf), seed, "Wv", w.w_sigma)
        h = sdev.fill_normal(torch.empty((w.M, w.d), **bf), seed, "h", 1.0)
        E = sdev.fill_normal(torch.empty((w.V, w.d), **bf), seed, "E", 1.0)
        root = torch.from_numpy(synth.root_tokens(seed, w.B, w.V)).to(dev)
        ws_h = md.workspace(md.hydra_workspace_bytes(step.tree, w.B, w.d, w.V, w.kmax), dev)
        call = lambda i: md.hydra_draft(step.tree, h, E, W1, b1, Wv, root, prefix, step.tokens,  # noqa: E731
                                        step.parent, step.anc, step.pos, ws_h)
        levels = hydra_levels(step.tree.parent)
        nbytes, nflops, launches = hydra_bytes(w, levels), hydra_flops(w, levels), 4 * len(levels) + 1
    elif args.part == "attention":
        nsets = 8
        sets = [(sdev.fill_normal(torch.empty((w.B, w.T, w.Hq, w.dh), **bf), seed + i, "q", 1.0),
                 sdev.fill_normal(torch.empty((w.B, w.Hkv, w.S_max, w.dh), **bf), seed + i, "k_cache", 1.0),
                 sdev.fill_normal(torch.empty((w.B, w.Hkv, w.S_max, w.dh), **bf), seed + i, "v_cache", 1.0))
                for i in range(nsets)]
        call = lambda i: step.attention(*sets[i % nsets], prefix)                # noqa: E731
        nbytes, nflops, launches = attention_bytes(w, P), attention_flops(w, P), attention_launches(w)
    elif args.part == "commit":
        tokens = synth.synthetic_tree_tokens(seed, w.B, np.array(step.tree.parent), w.V)
        logits = synth.planted_logits_device(seed, np.array(step.tree.parent), tokens, w.V, w.accept,
                                             sigma=w.logit_sigma, bump=w.bump, device=dev)
        step.tokens.copy_(torch.from_numpy(tokens))
        step.accept(logits)
        kc = sdev.fill_normal(torch.empty((w.B, w.Hkv, w.S_max, w.dh), **bf), seed, "k_cache", 1.0)
        vc = sdev.fill_normal(torch.empty((w.B, w.Hkv, w.S_max, w.dh), **bf), seed, "v_cache", 1.0)
        call = lambda i: step.commit(kc, vc, prefix)                               # noqa: E731
        nbytes = int(2 * 2 * w.B * w.Hkv * (step.accept_len.sum().item() + w.B) * w.dh * 2)
        nflops, launches = 0, 1
    else:
        tokens = synth.synthetic_tree_tokens(seed, w.B, np.array(step.tree.parent), w.V)
        logits = synth.planted_logits(seed, np.array(step.tree.parent), tokens, w.V, w.accept,
                                      sigma=w.logit_sigma, bump=w.bump)
        step.tokens.copy_(torch.from_numpy(tokens))
        if step.logits_dbg is not None:    # rejection rule: the heads' logits (draft distributions)
            sdev.fill_normal(step.logits_dbg, seed, "head_logits", 1.0)
        nsets = max(2, -(-2 * L2_BYTES // logits.nbytes))
        lgs = [torch.from_numpy(logits).to(dev) for _ in range(nsets)]
        call = lambda i: step.accept(lgs[i % nsets])                              # noqa: E731
        nbytes, nflops, launches = accept_bytes(w), 0, (1 if w.mode == "rejection" else 2)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            call(i)
    stream.synchronize()
    def timed(fn):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            start.record(stream)
            fn()
            end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / args.steps

    def eager():
        for i in range(args.steps):
            call(i)

    ms = timed(eager)
    # The same calls replayed from CUDA graphs (no host launch overhead): one
    # graph per input buffer set, each holding one call, as in the step timing.
    graph_ms = None
    try:
        nbuf = {"attention": 8}.get(args.part, 1)
        if args.part == "accept":
            nbuf = nsets
        graphs = []
        for i in range(nbuf):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                call(i)
            graphs.append(g)
        for i in range(args.warmup):
            graphs[i % nbuf].replay()
        stream.synchronize()

        def replay():
            for i in range(args.steps):
                graphs[i % nbuf].replay()
        graph_ms = timed(replay)
        del graphs
    except Exception:
        torch.cuda.synchronize()
    status = md.device_status(stream=stream)
    peaks = measured_peaks()
    print(json.dumps({"part": args.part, "workload": w.name, "ms_per_call": ms, "calls": args.steps,
                      "graph_ms_per_call": graph_ms,
                      "gbs": nbytes / (ms / 1000) / 1e9, "hbm_frac": nbytes / (ms / 1000) / 1e9 / peaks["hbm_gbs"],
                      "tflops": nflops / (ms / 1000) / 1e12 if nflops else None,
                      "algorithmic_bytes": nbytes, "flops": nflops, "gpu_launches": launches * args.steps,
                      "device_status": status}), flush=True)


def run_sweep(args):
    """The 8B-shaped sweep: B x tree x KV prefix x acceptance rule, one JSON line
    per point with the per-call times (device, CUDA events, eager)."""
    import torch

    import medusa_draft_heads_b200 as md
    from medusa_draft_heads_b200.step import MedusaStep
    from seeded_inputs import device as sdev
    from seeded_inputs.workloads import sweep_8b

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    bf = dict(dtype=torch.bfloat16, device=dev)
    base = sweep_8b(1, "64", 1024)
    W1 = sdev.fill_normal(torch.empty((base.K, base.d, base.d), **bf), base.seed, "W1", base.w_sigma)
    b1 = sdev.fill_normal(torch.empty((base.K, base.d), **bf), base.seed, "b1", base.w_sigma)
    Wv = sdev.fill_normal(torch.empty((base.K, base.d, base.V), **bf), base.seed, "Wv", base.w_sigma)
    Bs = [int(x) for x in args.sweep_batches.split(",")]
    for mode in args.sweep_modes.split(","):
        for tree in ("chain", "16", "64"):
            for P in (1024, 8192, 32768):
                for B in Bs:
                    w = sweep_8b(B, tree, P, mode)
                    tups = md.select_tree(w.k_per_head, w.accept, w.n_nodes)
                    step = MedusaStep(B=w.B, M=w.M, d=w.d, V=w.V, K=w.K, k_per_head=w.k_per_head, tree_tuples=tups,
                                      Hq=w.Hq, Hkv=w.Hkv, dh=w.dh, S_max=w.S_max, mode=w.mode,
                                      temperature=w.temperature, eps=w.eps, alpha=w.alpha, device=dev)
                    h = sdev.fill_normal(torch.empty((w.M, w.d), **bf), w.seed + B, "h", 1.0)
                    root = torch.from_numpy(synth.root_tokens(w.seed + B, w.B, w.V)).to(dev)
                    prefix = torch.full((w.B,), P, dtype=torch.int32, device=dev)
                    q = sdev.fill_normal(torch.empty((w.B, w.T, w.Hq, w.dh), **bf), w.seed + B, "q", 1.0)
                    kc = sdev.fill_normal(torch.empty((w.B, w.Hkv, w.S_max, w.dh), **bf), w.seed + B, "k_cache", 1.0)
                    vc = sdev.fill_normal(torch.empty((w.B, w.Hkv, w.S_max, w.dh), **bf), w.seed + B, "v_cache", 1.0)
                    with torch.cuda.stream(stream):
                        step.heads(h, W1, b1, Wv)
                        step.build(root, prefix)
                    stream.synchronize()
                    lg = synth.planted_logits_device(w.seed + B, np.array(step.tree.parent), step.tokens.cpu().numpy(),
                                                     w.V, w.accept, sigma=w.logit_sigma, bump=w.bump, device=dev)
                    torch.cuda.synchronize()
                    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
                    with torch.cuda.stream(stream):
                        for i in range(args.warmup + args.steps):
                            ev = evs[i - args.warmup] if i >= args.warmup else None
                            if ev: ev[0].record(stream)
                            step.heads(h, W1, b1, Wv)
                            if ev: ev[1].record(stream)
                            step.build(root, prefix)
                            if ev: ev[2].record(stream)
                            step.attention(q, kc, vc, prefix)
                            if ev: ev[3].record(stream)
                            step.accept(lg)
                            if ev: ev[4].record(stream)
                    torch.cuda.synchronize()
                    status = md.device_status(stream=stream)
                    per = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])
                    tot = float(np.mean([e[0].elapsed_time(e[4]) for e in evs]))
                    print(json.dumps({"sweep": w.name, "B": B, "tree": tree, "prefix": P, "mode": mode,
                                      "heads_path": ("tcgen05-pair-gemm" if w.M > 128 else "tcgen05-gemm" if w.M > 32
                                                     else "tcgen05-weights-as-m" if w.M > 1 else "cuda-core-stream"),
                                      "steps_per_s": 1000.0 / tot, "ms_per_step": tot,
                                      "ms": {"heads": float(per[:, 0].mean()), "build": float(per[:, 1].mean()),
                                             "attention": float(per[:, 2].mean()),
                                             "accept": float(per[:, 3].mean())},
                                      "attention_tflops": attention_flops(w, [P] * B) / (per[:, 2].mean() / 1e3) / 1e12,
                                      "accept_len_mean": float(step.accept_len.float().mean().item()),
                                      "device_status": status}), flush=True)
                    del step, h, q, kc, vc, lg
                    torch.cuda.empty_cache()


def run_e2e(args, w, step, h, W1, b1, Wv, root, prefix, head_row, sets, stream, dev, world, barrier):
    """Same step through the public API, with this step's inputs copied from
    pinned host memory and the result read back every step."""
    import torch
    q0, kc0, vc0, lg0 = sets[0]
    Pn = prefix.cpu().numpy()
    host = {
        "h": h.cpu().pin_memory(), "root": root.cpu().pin_memory(), "prefix": prefix.cpu().pin_memory(),
        "q": q0.cpu().pin_memory(),
        "k_new": torch.stack([kc0[b, :, Pn[b]:Pn[b] + w.T].cpu() for b in range(w.B)]).pin_memory(),
        "v_new": torch.stack([vc0[b, :, Pn[b]:Pn[b] + w.T].cpu() for b in range(w.B)]).pin_memory(),
        "logits": lg0.cpu().pin_memory(),
    }
    # the rules that draw random numbers take this step's uniforms from the host
    for name in ("uniforms", "u_draft", "u_accept", "u_residual"):
        if getattr(step, name) is not None:
            host[name] = getattr(step, name).cpu().pin_memory()
    # accept_len, path and bonus live in one device buffer: one copy back
    out_host = {"result": torch.empty(step.result.shape, dtype=step.result.dtype).pin_memory()}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in out_host.values())
    steps = max(50, args.steps // 4)

    # The inputs the heads do not read (q, the tree K/V, the target logits:
    # nearly all of the bytes) are copied on a second stream while the heads
    # run; attention and acceptance wait for that copy.
    copy_stream = torch.cuda.Stream(dev)
    copied = torch.cuda.Event()

    def e2e_step():
        with torch.cuda.stream(copy_stream):
            q0.copy_(host["q"], non_blocking=True)
            for b in range(w.B):
                kc0[b, :, Pn[b]:Pn[b] + w.T].copy_(host["k_new"][b], non_blocking=True)
                vc0[b, :, Pn[b]:Pn[b] + w.T].copy_(host["v_new"][b], non_blocking=True)
            lg0.copy_(host["logits"], non_blocking=True)
            for name in ("uniforms", "u_accept", "u_residual"):
                if name in host:
                    getattr(step, name).copy_(host[name], non_blocking=True)
            copied.record(copy_stream)
        h.copy_(host["h"], non_blocking=True)
        if "u_draft" in host:          # the draws' uniforms feed the heads
            step.u_draft.copy_(host["u_draft"], non_blocking=True)
        root.copy_(host["root"], non_blocking=True)
        prefix.copy_(host["prefix"], non_blocking=True)
        step.heads(h, W1, b1, Wv)
        step.build(root, prefix, head_row)
        stream.wait_event(copied)
        step.attention(q0, kc0, vc0, prefix)
        step.accept(lg0)
        out_host["result"].copy_(step.result, non_blocking=True)
        stream.synchronize()
        copy_stream.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(3):
            e2e_step()
        barrier()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(steps):
            e2e_step()
        e.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = slowest_rank_ms(s.elapsed_time(e), world, dev)
    return {"value": job_value(world, steps, ms), "unit": "steps/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "note": "per step: h, root token, prefix lengths, q, the tree tokens' K/V and the target logits "
                    "copied in from pinned host memory (q, K/V and logits on a second stream, overlapping the "
                    "heads); accept_len, path and bonus copied out in one copy; both streams synchronised after "
                    "every step"}


def cpu_baseline(w, args):
    frac = args.cpu_frac
    smp = OracleSampler(w, frac)
    smp.step()
    est = []
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < args.cpu_seconds or len(est) < 2:
        est.append(smp.step())
    sec = float(np.median(est))
    return {"value": 1.0 / sec, "unit": "steps/s", "cores": blas_threads(), "host_cpus": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{len(est)} oracle sample steps in {time.perf_counter() - t0:.1f} s; each: residual block "
                      f"and vocabulary projection on {frac:.4g} of their output columns, attention on {frac:.4g} of "
                      f"its (token, head) rows, scaled by 1/{frac:.4g}; tree build and acceptance in full"}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["medusa", "reference"], default="medusa")
    ap.add_argument("--workload", default="llama3-70b", choices=sorted(WORKLOADS))
    ap.add_argument("--part", choices=["step", "heads", "hydra", "attention", "accept", "commit"], default="step",
                    help="time one call alone (profiling); the JSON line then reports that call only")
    ap.add_argument("--sweep", action="store_true",
                    help="run the 8B-shaped sweep (B x tree x prefix x rule), one JSON line per point")
    ap.add_argument("--sweep-batches", default="1,2,4,8,16,32")
    ap.add_argument("--sweep-modes", default="greedy,typical")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-frac", type=float, default=1 / 64)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-frac", type=float, default=1 / 512)
    ap.add_argument("--oracle-check", action="store_true",
                    help="time whole (unsampled) oracle steps beside the sampled estimate, then exit (CPU only)")
    ap.add_argument("--oracle-check-steps", type=int, default=2)
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per heads call from an ncu capture of the current kernels")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.oracle_check:
        run_oracle_check(args, w)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.part != "step":
        run_part(args, w)
        return
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        run_reference(args, w)
        return
    run_medusa(args, w)


if __name__ == "__main__":
    main()
