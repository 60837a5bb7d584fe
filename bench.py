#!/usr/bin/env python
"""Throughput of the exact-attention forward path on B200.

Default (N=1): the causal GQA prefill shaped like Llama-3.1-8B (B=1, Hq=32,
Hkv=8, S=2048, D=128) - one step is one attn_fwd over one batch - reported as
TFLOP/s over the unmasked (q, kv) pairs (4*D FLOPs each). Secondary lines
measure the other workloads: sliding window + softcap, packed documents with
ALiBi under a block mask (block-mask build timed separately), and the MQA
paged decode (HBM GB/s over the algorithmic bytes).

Timing: inputs are resident in HBM and rotated over enough replicas that the
working set exceeds the 126 MB L2; the K timed steps are replayed from a CUDA
graph on one stream and timed with CUDA events, bracketed by a barrier and a
device synchronize; multi-GPU runs take the max over ranks. SM clocks and
throttle reasons are sampled with nvidia-smi during the timed region.

--impl reference times the fp64 CPU oracle (a deliberately slow, plain
program) on a bounded sample of the same workload.

Multi-GPU: the path has no exchange step (batches, heads and query tiles are
independent), so each rank runs its own batch of the workload (weak scaling,
no data-path collective); NCCL is used only to take the max time over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "attention fwd TFLOP/s (prefill) and HBM GB/s (decode) vs B200 roofline, 1 GPU"
PRIMARY = "causal_gqa_llama8b_s2048"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- workload accounting (closed forms)

def unmasked_pairs(w: W.Prefill, doc_lens=None) -> int:
    """Allowed (q, kv) pairs summed over batch and query heads."""
    S = w.S
    if w.mask == W.MASK_NONE:
        per = S * S
    elif w.mask == W.MASK_CAUSAL:
        per = S * (S + 1) // 2
    elif w.mask == W.MASK_WINDOW:
        Wn = w.window_left + 1  # 0 <= q - kv <= left
        per = sum(min(i + 1, Wn) for i in range(S))
    else:
        per = sum(L * (L + 1) // 2 for L in doc_lens)
    return per * w.B * w.Hq


def prefill_bytes(w: W.Prefill) -> int:
    """Q, K, V read once, O and LSE written once."""
    return 2 * w.B * w.S * w.D * (2 * w.Hq + 2 * w.Hkv) + 4 * w.B * w.Hq * w.S


def decode_bytes(w: W.Decode, seqlens) -> int:
    kv = 2 * 2 * int(np.sum(seqlens)) * w.Hkv * w.D
    qo = 2 * 2 * w.B * w.Hq * w.D
    meta = 4 * w.B * w.Hq + 4 * w.B * ((w.kv_len + w.page_size - 1) // w.page_size) + 4 * w.B
    return kv + qo + meta


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.reader = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.reader.join(timeout=2)

    def summary(self, t0: float, t1: float):
        rows = []
        for ts, line in self.lines:
            if t0 - 0.1 <= ts <= t1 + 0.1:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def physical_gpu_index(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ---------------------------------------------------------------- device helpers

def to_dev(bits, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def graph_time(torch, step_fn, steps: int, stream, warmup: int, barrier=None):
    """Warm up, capture `steps` calls of step_fn(i) in CUDA graphs (chunks of
    at most 200), replay them once between events. Returns seconds."""
    with torch.cuda.stream(stream):
        for i in range(warmup):
            step_fn(i)
    torch.cuda.synchronize()
    graphs = []
    chunk = 200
    done = 0
    while done < steps:
        n = min(chunk, steps - done)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                step_fn(done + i)
        graphs.append(g)
        done += n
    # one untimed replay so the graphs are uploaded
    with torch.cuda.stream(stream):
        for g in graphs:
            g.replay()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for g in graphs:
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3, (t_wall0, t_wall1)


def replicas_for(bytes_per_set: int) -> int:
    return max(1, int(np.ceil(1.5 * L2_BYTES / max(bytes_per_set, 1))))


# ---------------------------------------------------------------- arms

def prefill_setup(torch, ea, w: W.Prefill, device, seed_shift: int):
    wr = W.Prefill(**{**w.__dict__, "seed": w.seed + seed_shift})
    d = W.make_prefill_inputs(wr)
    nrep = replicas_for(prefill_bytes(w))
    qs, ks, vs = [], [], []
    q0, k0, v0 = (to_dev(d[x], device) for x in ("q", "k", "v"))
    for r in range(nrep):
        qs.append(q0 if r == 0 else q0.clone())
        ks.append(k0 if r == 0 else k0.clone())
        vs.append(v0 if r == 0 else v0.clone())
    o = torch.empty_like(q0)
    lse = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device=device)
    kw = {}
    bm = None
    if w.mask == W.MASK_CAUSAL:
        kw["causal"] = True
    elif w.mask == W.MASK_WINDOW:
        kw["window"] = (w.window_left, w.window_right)
    if w.mask == W.MASK_DOCUMENT:
        kw["doc_id"] = torch.from_numpy(d["doc_id"]).to(device)
        bm = ea.attn_build_block_mask(w.S, w.S, doc_id=kw["doc_id"])
        kw["block_mask"] = bm
    if w.mod == W.MOD_SOFTCAP:
        kw["softcap"] = w.softcap
    if w.mod == W.MOD_ALIBI:
        kw["alibi_slopes"] = torch.from_numpy(d["alibi"]).to(device)
    pairs = unmasked_pairs(w, d["doc_lens"])

    def step(i):
        r = i % nrep
        ea.attn_fwd(qs[r], ks[r], vs[r], out=o, lse=lse, **kw)

    return dict(step=step, pairs=pairs, flops=4 * w.D * pairs, bytes=prefill_bytes(w), nrep=nrep, kw=kw, d=d,
                bm=bm, o=o, lse=lse)


def backward_setup(torch, ea, w: W.Prefill, device, seed_shift: int):
    """attn_bwd on a causal/window/no-mask prefill workload: the forward's O and
    LSE plus a seeded upstream gradient dO, rotated over enough replicas that
    the step's inputs exceed L2. Algorithmic FLOPs: the five products of the
    chain rule (S, dP, dV, dK, dQ), 2.5x the forward's 4*D per pair."""
    wr = W.Prefill(**{**w.__dict__, "seed": w.seed + seed_shift})
    d = W.make_prefill_inputs(wr)
    kw = {}
    if w.mask == W.MASK_CAUSAL:
        kw["causal"] = True
    elif w.mask == W.MASK_WINDOW:
        kw["window"] = (w.window_left, w.window_right)
    q0, k0, v0 = (to_dev(d[x], device) for x in ("q", "k", "v"))
    do0 = to_dev(W.normal_bf16(wr.seed + 0x200, (w.B, w.S, w.Hq, w.D)), device)
    per_set = 2 * (3 * q0.numel() + 3 * k0.numel())  # q, o, dO, dq + k, v, dk, dv (bf16)
    nrep = replicas_for(per_set)
    sets = []
    for r in range(nrep):
        q, k, v, do = (x if r == 0 else x.clone() for x in (q0, k0, v0, do0))
        o, lse = ea.attn_fwd(q, k, v, **kw)
        sets.append((q, k, v, o, lse, do))
    dq, dk, dv = torch.empty_like(q0), torch.empty_like(k0), torch.empty_like(v0)
    ws = torch.empty(ea.attn_bwd_workspace_bytes(q0, k0, v0, **kw), dtype=torch.uint8, device=device)
    pairs = unmasked_pairs(w, d["doc_lens"])

    def step(i):
        q, k, v, o, lse, do = sets[i % nrep]
        ea.attn_bwd(q, k, v, o, lse, do, dq=dq, dk=dk, dv=dv, workspace=ws, **kw)

    return dict(step=step, pairs=pairs, flops=10 * w.D * pairs, nrep=nrep)


def decode_setup(torch, ea, w: W.Decode, device, seed_shift: int):
    wr = W.Decode(**{**w.__dict__, "seed": w.seed + seed_shift})
    d = W.make_decode_inputs(wr)
    q = to_dev(d["q"], device)[:, 0]
    kc = to_dev(d["k_cache"], device)
    vc = to_dev(d["v_cache"], device)
    bt = torch.from_numpy(d["block_table"]).to(device)
    sl = torch.from_numpy(d["cache_seqlens"]).to(device)
    o = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=device)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=device)
    lib = ea.load_library()
    splits = lib.attn_decode_num_splits(w.B, w.Hq, w.Hkv, w.kv_len, 0)
    ws = torch.empty(lib.attn_decode_workspace_bytes(w.B, w.Hq, w.D, splits), dtype=torch.uint8, device=device)

    def step(i):
        ea.attn_decode(q, kc, vc, bt, sl, max_seqlen=w.kv_len, out=o, lse=lse, workspace=ws)

    nbytes = decode_bytes(w, d["cache_seqlens"])
    pairs = int(np.sum(d["cache_seqlens"])) * w.Hq
    return dict(step=step, bytes=nbytes, flops=4 * w.D * pairs, splits=splits, d=d)


def kvcache_setup(torch, ea, device, seed_shift: int, B=32, Hq=32, Hkv=8, D=128, T=4, kv_len=8192, page=256):
    """flash_attn_with_kvcache step (speculative-decoding shape): rotary on q and
    on T new keys, append of the new k/v into a paged cache (block table from
    a page permutation), causal decode of the T tokens over kv_len keys per
    sequence. Each step appends at the same positions, so steps are identical.
    Algorithmic bytes: the K and V rows read (kv_len + T per sequence), q, the
    new k/v written, O out."""
    seed = 0xA77E0400 + seed_shift
    pages_per_seq = (kv_len + T + page - 1) // page
    P = B * pages_per_seq
    kc = to_dev(W.normal_bf16(seed, (P, page, Hkv, D)), device)
    vc = to_dev(W.normal_bf16(seed + 1, (P, page, Hkv, D)), device)
    q = to_dev(W.normal_bf16(seed + 2, (B, T, Hq, D)), device)
    kn = to_dev(W.normal_bf16(seed + 3, (B, T, Hkv, D)), device)
    vn = to_dev(W.normal_bf16(seed + 4, (B, T, Hkv, D)), device)
    bt = torch.from_numpy(W.page_permutation(seed + 5, P).reshape(B, pages_per_seq)).to(device)
    sl = torch.full((B,), kv_len, dtype=torch.int32, device=device)
    j = np.arange(D // 2)
    ang = np.arange(kv_len + T)[:, None] * (10000.0 ** (-2.0 * j / D))[None, :]
    cos = torch.from_numpy(np.cos(ang).astype(np.float32)).to(device)
    sin = torch.from_numpy(np.sin(ang).astype(np.float32)).to(device)
    new_len = torch.empty_like(sl)
    q_rot = torch.empty_like(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, T, Hq), dtype=torch.float32, device=device)
    lib = ea.load_library()
    splits = lib.attn_decode_num_splits(B, Hq, Hkv, kv_len + T, 0)
    ws = torch.empty(lib.attn_decode_workspace_bytes(B, Hq * T, D, splits), dtype=torch.uint8, device=device)

    def step(i):
        ea.attn_kvcache_update(kc, vc, sl, q=q, q_out=q_rot, k=kn, v=vn, block_table=bt, rotary_cos=cos,
                               rotary_sin=sin, rotary_interleaved=False, seqlens_out=new_len)
        ea.attn_decode(q_rot, kc, vc, bt, new_len, max_seqlen=kv_len + T, out=o, lse=lse, workspace=ws, causal=True)

    nbytes = 2 * B * (kv_len + T) * Hkv * D * 2 + 2 * (2 * B * T * Hq * D) + 2 * (2 * B * T * Hkv * D)
    return dict(step=step, bytes=nbytes, splits=splits,
                name="with_kvcache_gqa_b%d_q%d_kv%d" % (B, T, kv_len))


def e2e_prefill(torch, ea, w: W.Prefill, setup, device, steps: int):
    """Same metric through the public API with host buffers: per step, pinned
    host -> device copies of Q, K, V, the forward, device -> host copies of O,
    LSE. Steps are pipelined over two buffer sets and three streams, as a
    serving loop would run them: step i+1's inputs go up and step i-1's
    results come down while step i computes (H2D and D2H use separate copy
    engines). Every step still moves all of its bytes inside the timed
    region."""
    d = setup["d"]
    hq, hk, hv = (torch.from_numpy(np.ascontiguousarray(d[x]).view(np.int16)).view(torch.bfloat16).pin_memory()
                  for x in ("q", "k", "v"))
    nb = 2
    dev_in = [tuple(torch.empty_like(x, device=device) for x in (hq, hk, hv)) for _ in range(nb)]
    dev_out = [(torch.empty(hq.shape, dtype=torch.bfloat16, device=device),
                torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device=device)) for _ in range(nb)]
    host_out = [(torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory(),
                 torch.empty((w.B, w.Hq, w.S), dtype=torch.float32).pin_memory()) for _ in range(nb)]
    kw = setup["kw"]
    main = torch.cuda.current_stream(device)
    s_up, s_comp, s_down = (torch.cuda.Stream(device) for _ in range(3))
    up_done = [torch.cuda.Event() for _ in range(nb)]
    comp_done = [torch.cuda.Event() for _ in range(nb)]
    down_done = [torch.cuda.Event() for _ in range(nb)]
    state = {"i": 0}

    def step():
        i = state["i"]
        b = i % nb
        dq, dk, dv = dev_in[b]
        o, lse = dev_out[b]
        ho, hl = host_out[b]
        with torch.cuda.stream(s_up):
            if i >= nb:
                s_up.wait_event(comp_done[b])  # the forward of step i-2 has read these inputs
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            up_done[b].record(s_up)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(up_done[b])
            if i >= nb:
                s_comp.wait_event(down_done[b])  # step i-2's results have left these buffers
            ea.attn_fwd(dq, dk, dv, out=o, lse=lse, **kw)  # on s_comp, the current stream here
            comp_done[b].record(s_comp)
        with torch.cuda.stream(s_down):
            s_down.wait_event(comp_done[b])
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
            down_done[b].record(s_down)
        state["i"] = i + 1

    def join():
        for st in (s_up, s_comp, s_down):
            main.wait_stream(st)

    for _ in range(3):
        step()
    join()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for st in (s_up, s_comp, s_down):
        st.wait_stream(main)
    for _ in range(steps):
        step()
    join()
    e1.record(main)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = host_out[0][0].numel() * 2 + host_out[0][1].numel() * 4
    return setup["flops"] * steps / t / 1e12, h2d, d2h


def cpu_baseline_prefill(w: W.Prefill, seconds: float = 12.0, d=None, first_rows: int = 64):
    """The oracle, as it stands, on a bounded sample of query rows of the
    workload (inputs d generated once by the caller when given)."""
    import oracle
    if d is None:
        d = W.make_prefill_inputs(w)
    kw = {}
    if w.mask == W.MASK_CAUSAL:
        kw = dict(mask=W.MASK_CAUSAL, window=(-1, 0))
    elif w.mask == W.MASK_WINDOW:
        kw = dict(mask=W.MASK_WINDOW, window=(w.window_left, w.window_right))
    elif w.mask == W.MASK_DOCUMENT:
        kw = dict(mask=W.MASK_DOCUMENT, doc_id=d["doc_id"])
    if w.mod == W.MOD_SOFTCAP:
        kw.update(mod=W.MOD_SOFTCAP, softcap=w.softcap)
    if w.mod == W.MOD_ALIBI:
        kw.update(mod=W.MOD_ALIBI, alibi=d["alibi"])
    threads = oracle.default_threads()
    rng = np.random.default_rng(0)
    n = first_rows
    total_flops, total_t, total_rows = 0, 0.0, 0
    while total_t < seconds:
        rows = np.stack([rng.integers(0, w.B, n), rng.integers(0, w.Hq, n), rng.integers(0, w.S, n)],
                        axis=1).astype(np.int32)
        t0 = time.perf_counter()
        oracle.attn(d["q"], d["k"], d["v"], rows=rows, nthreads=threads, **kw)
        dt = time.perf_counter() - t0
        total_t += dt
        total_rows += n
        total_flops += 4 * w.D * sum(_row_pairs(w, int(i), d) for i in rows[:, 2])
        if dt < seconds / 8:
            n *= 2
    return {"value": total_flops / total_t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": "%d random query rows of %s (fp64 C oracle, %d threads, %.1f s)" % (
                total_rows, w.name, threads, total_t)}


def _row_pairs(w: W.Prefill, i: int, d) -> int:
    if w.mask == W.MASK_NONE:
        return w.S
    if w.mask == W.MASK_CAUSAL:
        return i + 1
    if w.mask == W.MASK_WINDOW:
        return min(i + 1, w.window_left + 1)
    doc = d["doc_id"]
    return int(i - np.searchsorted(doc, doc[i]) + 1)


# ---------------------------------------------------------------- ranks

class RankGroup:
    """The ranks of one run. Each rank processes its own batch (weak scaling,
    no data-path collective); the group is used only for the barriers around
    the timed region and for the max of the per-rank times. NCCL on GPUs;
    the same calls work over gloo on CPU."""

    def __init__(self, world: int = 1, rank: int = 0, local: int = 0, dist=None, device=None):
        self.world, self.rank, self.local = world, rank, local
        self.dist, self.device = dist, device

    def barrier(self):
        if self.dist is None:
            return
        if self.device is not None and self.device.type == "cuda":
            self.dist.barrier(device_ids=[self.local])
        else:
            self.dist.barrier()

    def max(self, x: float) -> float:
        if self.dist is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def init_ranks(backend: str, device=None, timeout_s: int = 120) -> RankGroup:
    """Joins the process group described by RANK / LOCAL_RANK / WORLD_SIZE /
    MASTER_ADDR / MASTER_PORT (torchrun's variables); world size 1 needs none."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world == 1:
        return RankGroup(1, 0, local, None, device)
    import datetime
    import torch.distributed as dist
    kw = {"device_id": device} if backend == "nccl" else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return RankGroup(world, rank, local, dist, device)


def rank_seed_shift(rank: int) -> int:
    """Each rank draws its own batch of the workload (same shapes, other seeds)."""
    return 1000 * rank


def weak_scaling_value(work_per_rank: float, world: int, t_max: float) -> float:
    """Whole-job throughput: the work all ranks processed over the slowest rank's time."""
    return work_per_rank * world / t_max


def _free_port() -> int:
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def launch_plan(gpus: int, env) -> str:
    """How this process runs `--gpus N`: "single" (N == 1, no process group),
    "rank" (already one of torchrun's N ranks), or "spawn" (N > 1 and no
    torchrun around us: relaunch this command under torch.distributed.run).
    A WORLD_SIZE that disagrees with --gpus is an error."""
    world = env.get("WORLD_SIZE")
    if world is None:
        return "spawn" if gpus > 1 else "single"
    if int(world) != gpus:
        raise SystemExit("bench.py: --gpus %d but WORLD_SIZE=%s; run N ranks with --gpus N" % (gpus, world))
    return "rank" if gpus > 1 else "single"


def spawn_ranks(gpus: int, argv, timeout_s: int = 1800) -> int:
    """Re-runs this script as `gpus` ranks of one node (torch.distributed.run,
    rendezvous on 127.0.0.1) and returns the launcher's exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=%d" % gpus,
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.abspath(__file__)] + list(argv)
    try:
        return subprocess.run(cmd, timeout=timeout_s).returncode
    except subprocess.TimeoutExpired:
        sys.stderr.write("bench.py: ranks did not finish within %d s\n" % timeout_s)
        return 124


def plumbing_check(args) -> int:
    """CPU rehearsal of a multi-rank run (gloo): every rank draws its own
    batch of the workload, the barrier and the max over ranks run as in the
    GPU path, and rank 0 prints one JSON line with the world size, each rank's
    input digest and the slowest rank's (synthetic) time."""
    import hashlib
    group = init_ranks("gloo", timeout_s=120)
    w = W.WORKLOADS[args.workload]
    mine = W.Prefill(**{**w.__dict__, "seed": w.seed + rank_seed_shift(group.rank)})
    q = W.make_prefill_inputs(mine, S=128)["q"]
    digest = hashlib.sha256(q.tobytes()).hexdigest()[:16]
    group.barrier()
    t_max = group.max(1.0 + 0.25 * group.rank)
    digests = [digest]
    if group.dist is not None:
        digests = [None] * group.world
        group.dist.all_gather_object(digests, digest)
    world = group.world
    group.close()
    if group.rank == 0:
        print(json.dumps({"plumbing": True, "n_gpus": world, "gpus_flag": args.gpus, "rank_input_digests": digests,
                          "t_max": t_max, "value": weak_scaling_value(1.0, world, t_max)}), flush=True)
    return 0


# ---------------------------------------------------------------- main

def reference_arm(args):
    """Times the fp64 CPU oracle on bounded samples of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w = W.WORKLOADS[PRIMARY]
    oracle.build()
    d = W.make_prefill_inputs(w)
    # Each step is a bounded sample of query rows, sized so that the whole
    # run (warm-up included) takes about two minutes whatever K and W are.
    per_step = min(2.0, max(0.002, 120.0 / max(args.steps + args.warmup, 1)))
    rows = 64 if per_step >= 0.05 else 8
    for _ in range(args.warmup):
        cpu_baseline_prefill(w, seconds=per_step, d=d, first_rows=rows)
    t_steps = []
    vals = []
    total_rows = 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        cb = cpu_baseline_prefill(w, seconds=per_step, d=d, first_rows=rows)
        t_steps.append(time.perf_counter() - t0)
        vals.append(cb["value"])
        total_rows += int(cb["sample"].split()[0])
    value = float(np.mean(vals))
    sample = ("%d steps, each a bounded sample of random query rows of %s (about %.3f s of fp64 C oracle time "
              "on %d threads); %d rows in total" % (args.steps, w.name, per_step, cb["cores"], total_rows))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(t_steps)),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": PRIMARY, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S, "D": w.D,
                       "mask": "causal", "step": "bounded sample of query rows"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cb["cores"], "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=6000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--no-secondary", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=PRIMARY, choices=[k for k, v in W.WORKLOADS.items()
                                                          if isinstance(v, W.Prefill)])
    ap.add_argument("--secondary-steps", type=int, default=200)
    ap.add_argument("--profile", default=None, choices=list(W.WORKLOADS) + ["block_mask", "backward_" + PRIMARY, "with_kvcache"],
                    help="run --steps eager steps of one workload (for ncu captures); prints no JSON line")
    ap.add_argument("--plumbing-check", action="store_true",
                    help="CPU only: rehearse the N-rank launch, barrier and max over ranks over gloo")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus < 1:
        raise SystemExit("bench.py: --gpus must be at least 1")
    if args.impl == "reference":
        return reference_arm(args)
    if args.profile:
        return profile_arm(args)
    if launch_plan(args.gpus, os.environ) == "spawn":
        return spawn_ranks(args.gpus, sys.argv[1:])
    if args.plumbing_check:
        return plumbing_check(args)

    import torch
    import exact_attention_145_b200 as ea

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    ranks = init_ranks("nccl", device)
    world, rank = ranks.world, ranks.rank
    barrier, max_over_ranks = ranks.barrier, ranks.max

    peaks, peak_src = load_peaks()
    ea.load_library()
    stream = torch.cuda.Stream(device)
    w = W.WORKLOADS[args.workload]

    # ------------------------------------------------------------ primary: prefill
    setup = prefill_setup(torch, ea, w, device, seed_shift=rank_seed_shift(rank))
    sampler = ClockSampler(physical_gpu_index(local)) if rank == 0 else None
    if sampler:
        sampler.start()
    t, (tw0, tw1) = graph_time(torch, setup["step"], args.steps, stream, args.warmup, barrier)
    if sampler:
        sampler.stop()
    t_max = max_over_ranks(t)
    value = weak_scaling_value(setup["flops"] * args.steps, world, t_max) / 1e12
    launch_s = t / args.steps
    achieved = setup["flops"] / launch_s / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = _traffic_from_profiles(args.workload)

    # e2e_prefill returns this rank's TFLOP/s; the job's figure is the work of
    # all ranks over the slowest rank's time per unit of work.
    e2e_val, h2d, d2h = e2e_prefill(torch, ea, w, setup, device, steps=min(args.steps, 50))
    e2e_total = world / max_over_ranks(1.0 / e2e_val)

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * t_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S, "D": w.D,
                       "mask": {0: "none", 1: "causal", 2: "window", 3: "document"}[w.mask],
                       "pairs": setup["pairs"], "flops_per_step": setup["flops"],
                       "l2": "inputs rotated over %d replicas (%.0f MB > 126 MB L2), no flush" % (
                           setup["nrep"], setup["nrep"] * prefill_bytes(w) / 1e6),
                       "timing": "CUDA graph replay of the K steps on one stream, CUDA events",
                       "parallelism": "independent replicas per GPU (no data-path collective)"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": "attn_fwd_kernel<128, prefill, no score mod, no block mask>",
                         "peak_source": "%s bf16 burst (MEASURED_PEAKS.json)" % peak_src
                         if peak_src == "measured" else "fallback 1.59 PF/s"},
            "e2e": {"value": e2e_total, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps}
    if sampler:
        line["clocks"] = sampler.summary(tw0, tw1)

    # ------------------------------------------------------------ secondary workloads
    if not args.no_secondary:
        line["secondary"] = secondary(torch, ea, device, stream, peaks, rank, barrier, max_over_ranks, world,
                                      args.secondary_steps)
        line["gpu_launches"] += line["secondary"].pop("_launches", 0)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prefill(w)

    ranks.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def secondary(torch, ea, device, stream, peaks, rank, barrier, max_over_ranks, world, steps):
    out = {}
    launches = 0
    for name in ("window1024_softcap30_s8192", "packed_docs_alibi_s16384"):
        w = W.WORKLOADS[name]
        s = prefill_setup(torch, ea, w, device, seed_shift=rank_seed_shift(rank))
        t, _ = graph_time(torch, s["step"], steps, stream, 5, barrier)
        t = max_over_ranks(t)
        ach = s["flops"] / (t / steps) / 1e12
        out[name] = {"value": weak_scaling_value(s["flops"] * steps, world, t) / 1e12, "unit": "TFLOP/s", "ms_per_step": 1e3 * t / steps, "pairs": s["pairs"],
                     "roofline_frac": ach / float(peaks["bf16_tflops"])}
        launches += steps
        if s["bm"] is not None:
            doc = s["kw"]["doc_id"]
            bm = s["bm"]
            lib = ea.load_library()
            import ctypes
            from exact_attention_145_b200 import _lib
            spec = _lib.MaskSpec()
            spec.kind, spec.window_left, spec.window_right, spec.q_offset, spec.doc_id = 3, -1, -1, 0, doc.data_ptr()

            def bstep(i):
                _lib.check(lib.attn_build_block_mask(ctypes.byref(spec), ctypes.byref(bm.c),
                                                     torch.cuda.current_stream(device).cuda_stream), "build")

            tb, _ = graph_time(torch, bstep, 50, stream, 3, barrier)
            out[name]["block_mask_build_us"] = 1e6 * tb / 50
            launches += 50
    w = W.WORKLOADS[PRIMARY]
    s = backward_setup(torch, ea, w, device, seed_shift=rank_seed_shift(rank))
    bsteps = max(steps // 4, 10)
    t, _ = graph_time(torch, s["step"], bsteps, stream, 5, barrier)
    t = max_over_ranks(t)
    ach = s["flops"] / (t / bsteps) / 1e12
    out["backward_" + PRIMARY] = {
        "value": weak_scaling_value(s["flops"] * bsteps, world, t) / 1e12, "unit": "TFLOP/s",
        "ms_per_step": 1e3 * t / bsteps, "pairs": s["pairs"], "flops_per_step": s["flops"],
        "flops_rule": "10*D*pairs (S, dP, dV, dK, dQ products)",
        "roofline": {"bound": "tensor", "achieved": ach, "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                     "frac": ach / float(peaks["bf16_tflops"]), "traffic": None},
        "kernels": "delta_kernel, attn_bwd_dkdv_kernel<128>, attn_bwd_dkdv_reduce_kernel<128>, attn_bwd_dq_kernel<128>"}
    launches += 4 * bsteps  # delta (+ plan), dK/dV, dK/dV reduce (split tiles), dQ
    w = W.WORKLOADS["mqa_paged_decode_b32_kv32768"]
    s = decode_setup(torch, ea, w, device, seed_shift=rank_seed_shift(rank))
    t, _ = graph_time(torch, s["step"], steps, stream, 5, barrier)
    t = max_over_ranks(t)
    gbs = s["bytes"] / (t / steps) / 1e9
    out[w.name] = {"value": gbs * world, "unit": "GB/s", "ms_per_step": 1e3 * t / steps, "bytes": s["bytes"],
                   "splits": s["splits"], "roofline_frac": gbs / float(peaks["hbm_gbs"]),
                   "tflops": s["flops"] / (t / steps) / 1e12}
    launches += 2 * steps
    s = kvcache_setup(torch, ea, device, rank_seed_shift(rank))
    t, _ = graph_time(torch, s["step"], steps, stream, 5, barrier)
    t = max_over_ranks(t)
    gbs = s["bytes"] / (t / steps) / 1e9
    out[s["name"]] = {"value": gbs * world, "unit": "GB/s", "ms_per_step": 1e3 * t / steps, "bytes": s["bytes"],
                      "splits": s["splits"], "roofline_frac": gbs / float(peaks["hbm_gbs"]),
                      "kernels": "kvcache_update_kernel, attn_fwd_kernel<decode>, lse_combine_kernel"}
    launches += 3 * steps
    out["_launches"] = launches
    return out


def profile_arm(args):
    """Eager steps of one workload, for ncu captures (no timing, no JSON)."""
    import torch
    import exact_attention_145_b200 as ea
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    name = args.profile
    if name == "block_mask":
        w = W.WORKLOADS["packed_docs_alibi_s16384"]
        d = W.make_prefill_inputs(w)
        doc = torch.from_numpy(d["doc_id"]).to(device)
        step = lambda i: ea.attn_build_block_mask(w.S, w.S, doc_id=doc)  # noqa: E731
    elif name == "with_kvcache":
        step = kvcache_setup(torch, ea, device, 0)["step"]
    elif name.startswith("backward_"):
        step = backward_setup(torch, ea, W.WORKLOADS[name[len("backward_"):]], device, 0)["step"]
    elif isinstance(W.WORKLOADS[name], W.Decode):
        step = decode_setup(torch, ea, W.WORKLOADS[name], device, 0)["step"]
    else:
        step = prefill_setup(torch, ea, W.WORKLOADS[name], device, 0)["step"]
    for i in range(args.warmup + args.steps):
        step(i)
    torch.cuda.synchronize()
    print("profile run ok: %s, %d steps" % (name, args.warmup + args.steps))
    return 0


def code_digest(text: str) -> str:
    """sha256 (16 hex digits) of C++ source with comments and whitespace removed,
    so that editing a comment does not count as changing the kernel."""
    import hashlib
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = re.sub(r"\s+", "", text)
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def kernel_source_sha() -> str:
    """Digest of the prefill kernel's code (fwd_kernel.cuh + sm100.cuh)."""
    parts = []
    for f in ("exact_attention_145_b200/csrc/fwd_kernel.cuh", "exact_attention_145_b200/csrc/sm100.cuh"):
        with open(os.path.join(ROOT, f)) as fh:
            parts.append(fh.read())
    return code_digest("\n".join(parts))


def _traffic_from_profiles(workload: str):
    """DRAM bytes per launch of the prefill kernel from the committed ncu
    summary, or None when the kernel source changed since that capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(workload)
    if not d or d.get("kernel_source_sha") != kernel_source_sha():
        return None
    return d["dram_bytes_per_launch"]


if __name__ == "__main__":
    sys.exit(main())
