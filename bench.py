#!/usr/bin/env python
"""Throughput of the OneTrans hot path on B200: candidates scored per second
(Stage II over the KV cache) and users encoded per second (Stage I).

One step = auto-split tokenization of every candidate's NS features, Stage I
of every user's S tokens into the paged KV cache (the two are independent
and run on two streams at once), and Stage II scoring of every candidate
against its user's cache, all through the C ABI.  Workload
(default): 6 layers, d=256, 4 heads, FFN 1024, 12 NS tokens, L_S = 1178,
pyramid query counts 1190 -> 12 (linear), 16 users x 512 candidates, NS
features 512 wide, bf16 storage.  Other workloads: --workload append (non-
pyramid cross-request append of 16 events for 256 users, then 128
candidates each), s_forward / l_forward (one-pass forward).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun) every rank serves its own users: no data
moves between ranks, work per GPU is fixed (weak scaling), the device time
is the max over ranks.  `--impl reference` times the fp64 CPU oracle on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "candidates scored/sec (Stage II, KV-cached) and users/sec (Stage I) on 1 B200"
UNIT = "candidates/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="kv_serving",
                    choices=("kv_serving", "append", "s_forward", "l_forward", "train"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--users", type=int, default=0, help="override users per GPU (small profiling captures)")
    ap.add_argument("--cands", type=int, default=0, help="override candidates per user (small captures)")
    return ap.parse_args()


# ------------------------------------------------------------- dist utils

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def shard_users(n_users_per_rank: int, rank: int):
    """User ids served by `rank`: a contiguous block of n_users_per_rank.
    Every rank holds the same count (weak scaling) and no id repeats."""
    return list(range(rank * n_users_per_rank, (rank + 1) * n_users_per_rank))


def max_over_ranks(value: float, pg=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock, power and throttle reasons while the
    timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[3]) if v.lower() == "active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------- workload

# ------------------------------------------------- workload descriptions
# Shared by both arms, so that the reference arm's line names the same
# metric, unit and config as this arm's.

APPEND_METRIC = "users appended (dL=16 events) and their candidates scored per second on 1 B200"


def forward_metric(name: str) -> str:
    return f"samples/sec of the one-pass forward ({name}) on 1 B200"


def kv_serving_config(U: int, C: int, ws: int) -> dict:
    return {"workload": "kv_serving: auto-split + Stage I + Stage II; 6 layers d=256 4 heads FFN 1024, "
                        f"pyramid queries 1190->12 (linear), {U} users x 1178 S tokens, {C} "
                        "candidates/user, 12 NS tokens from 512 features", "users_per_gpu": U,
            "candidates_per_gpu": U * C, "parallelism": f"users sharded over {ws} GPU(s), no collective",
            "pipeline": "batch k+1's auto-split and Stage I (two side streams) are issued before batch k's "
                        "Stage II; two banks of KV cache and NS tokens; the timed span covers the fill "
                        "and the drain, so every batch counted is complete inside it",
            "l2": "inputs larger than L2: the timed loops cycle 8 distinct input sets of 17.6 MB (141 MB); "
                  "no flush between the overlapping steps"}


def append_config(U: int, C: int, dL: int, ws: int) -> dict:
    return {"workload": f"append: non-pyramid 6 layers d=256 4 heads FFN 1024, {U} users x 1178 cached "
                        f"S tokens, append dL={dL} events (64-wide, 3 behavior types), then "
                        f"{C} candidates/user (12 NS tokens from 512 features) scored over 1194 keys",
            "users_per_gpu": U, "candidates_per_gpu": U * C,
            "parallelism": f"users sharded over {ws} GPU(s), no collective",
            "pipeline": "batch k+1's append and auto-split (two side streams) are issued before batch k's "
                        "Stage II; the timed span covers the fill and the drain",
            "l2": "inputs larger than L2: every step reads its own 1.9 GB cache; no flush between the "
                  "overlapping steps"}


def forward_config(name: str, U: int, ws: int) -> dict:
    from onetrans_synth import WORKLOADS
    wl = WORKLOADS[name]
    sh = wl.shape
    return {"workload": f"{name}: {sh.n_layers} layers d={sh.d} {sh.n_heads} heads FFN {sh.d_ff}, "
                        f"{U} samples x ({wl.L_S} S + {sh.L_NS} NS tokens), pyramid "
                        f"{wl.pyramid[0]}->{wl.pyramid[-1]} (linear)",
            "samples_per_gpu": U, "parallelism": f"samples sharded over {ws} GPU(s), no collective",
            "l2": "512 MB buffer written between timed steps (not timed)"}


ALU_KERNELS = ("train_attn_rows",)   # kernel kinds that run on the CUDA cores' FMA pipes
TRAIN_METRIC = "samples/sec of the training step (forward + backward with recomputation) on 1 B200"
TRAIN_SAMPLES = 64


def train_config(U: int, ws: int) -> dict:
    from onetrans_synth import WORKLOADS
    wl = WORKLOADS["s_forward"]
    sh = wl.shape
    return {"workload": f"train: the s_forward model ({sh.n_layers} layers d={sh.d} {sh.n_heads} heads FFN "
                        f"{sh.d_ff}, pyramid {wl.pyramid[0]}->{wl.pyramid[-1]}), {U} samples x ({wl.L_S} S + "
                        f"{sh.L_NS} NS tokens): forward keeping each layer's input, attention output and "
                        "log-sum-exp, backward with the rest of each layer recomputed; bf16 operands, float32 "
                        "gradients of the input and of every weight",
            "samples_per_gpu": U, "parallelism": f"samples sharded over {ws} GPU(s), no collective",
            "l2": "512 MB buffer written between timed steps (not timed)"}


def workload_meta(name: str, ws: int):
    """(metric, unit, config, units per GPU per step) of a workload at its
    default size, without building it."""
    from onetrans_synth import WORKLOADS
    if name == "train":
        return TRAIN_METRIC, "samples/s", train_config(TRAIN_SAMPLES, ws), TRAIN_SAMPLES
    wl = WORKLOADS[name]
    if name == "kv_serving":
        return METRIC, UNIT, kv_serving_config(wl.users, wl.cands, ws), wl.users * wl.cands
    if name == "append":
        return APPEND_METRIC, "users/s", append_config(wl.users, wl.cands, wl.dL, ws), wl.users
    return forward_metric(name), "samples/s", forward_config(name, wl.users, ws), wl.users


class KVServing:
    """Auto-split + Stage I + Stage II for U users x C candidates, served as
    a pipeline: batch k's front (the candidates' auto-split on one side
    stream, Stage I on another) is issued before batch k-1's back (Stage II
    on the caller's stream), so Stage I's short, latency-bound launches run
    beside the previous batch's Stage II.  Two banks of KV cache and NS
    tokens alternate between batches; events order every reuse."""

    pipelined = True
    n_input_sets = 8      # distinct input buffers cycled by the timed loops (141 MB > 126 MB L2)

    def __init__(self, rank: int, wl_name: str = "kv_serving", users: int = 0, cands: int = 0):
        import torch
        import unified_transformer_recommender_b200 as ot
        from onetrans_synth import WORKLOADS, gen_normal, make_weights
        self.ot, self.torch = ot, torch
        wl = WORKLOADS[wl_name]
        self.wl, sh = wl, wl.shape
        self.U, self.C = users or wl.users, cands or wl.cands
        self.W = make_weights(sh, wl.seed_weights, wl.dtype)
        self.model = ot.model_from_arrays(sh, self.W, pyramid_q=list(wl.pyramid), mode=ot.BF16)
        seed = wl.seed_inputs + 7919 * rank     # each rank serves different users
        self.S_h = gen_normal(seed, (self.U, wl.L_S, sh.d), "bf16")
        self.F_h = gen_normal(seed + 100, (self.U * self.C, sh.ns_feat), "bf16")
        dev = torch.device("cuda")
        S0 = torch.from_numpy(self.S_h).to(dev, torch.bfloat16)
        F0 = torch.from_numpy(self.F_h).to(dev, torch.bfloat16)
        # further input sets: the same values rotated over users / candidates,
        # in buffers of their own
        self.S_sets = [S0] + [torch.roll(S0, i, 0).contiguous() for i in range(1, self.n_input_sets)]
        self.F_sets = [F0] + [torch.roll(F0, 37 * i, 0).contiguous() for i in range(1, self.n_input_sets)]
        self.S, self.F = S0, F0
        # pinned host copies for the end-to-end leg
        self.S_pin = torch.from_numpy(self.S_h).to(torch.bfloat16).pin_memory()
        self.F_pin = torch.from_numpy(self.F_h).to(torch.bfloat16).pin_memory()
        m = self.model
        self.ns = [torch.empty(self.U * self.C, sh.L_NS, sh.d, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.cache = [ot.Cache(m, self.U, wl.L_S) for _ in range(2)]
        self.out = torch.empty(self.U * self.C, sh.L_NS, sh.d, dtype=torch.float32, device=dev)
        self.out_pin = torch.empty(self.out.shape, dtype=torch.float32).pin_memory()
        self.ws_a = m.workspace(ot.OP_AUTOSPLIT, self.U * self.C)
        self.ws_1 = m.workspace(ot.OP_STAGE1, self.U, wl.L_S)
        self.ws_2 = m.workspace(ot.OP_STAGE2, self.U * self.C, wl.L_S)
        # default priority: the front's short launches fill the SMs that the
        # previous batch's Stage II leaves idle (a higher priority made them
        # hold back Stage II's CTAs and the step slower)
        self.s_front, self.s_tok = torch.cuda.Stream(), torch.cuda.Stream()
        ev = torch.cuda.Event
        self.ev_in, self.ev_tok = ev(), ev()
        self.ev_front, self.ev_back = [ev(), ev()], [ev(), ev()]
        self.front_spans = None   # list of (start, end) events around each front's Stage I, when set
        self.slots = list(range(self.U))
        self.offs = [u * self.C for u in range(self.U + 1)]
        self.units = self.U * self.C
        self.h2d = self.S_h.size * 2 + self.F_h.size * 2
        self.d2h = self.out.numel() * 4

    def set_inputs(self, i: int):
        self.S, self.F = self.S_sets[i % self.n_input_sets], self.F_sets[i % self.n_input_sets]

    def front(self, k: int, main, serial: bool = False):
        """Auto-split and Stage I of batch k into bank k % 2, on the side
        streams, after the inputs are ready on `main` and after Stage II of
        batch k-2 (the bank's last reader).  Returns the event that marks the
        front done (its inputs may then be overwritten).  serial: everything
        on `main` (the per-kernel timing pass)."""
        ot, m, b = self.ot, self.model, k & 1
        s_front, s_tok = (main, main) if serial else (self.s_front, self.s_tok)
        self.ev_in.record(main)
        for s in (s_front, s_tok):
            s.wait_event(self.ev_in)
            s.wait_event(self.ev_back[b])
        ot.onetrans_tokenize_autosplit(m, self.F, self.ns[b], self.ws_a, stream=s_tok)
        self.ev_tok.record(s_tok)
        if self.front_spans is not None:
            e = (self.torch.cuda.Event(enable_timing=True), self.torch.cuda.Event(enable_timing=True))
            e[0].record(s_front)
        ot.onetrans_stage1_encode(m, self.cache[b], self.slots, self.S, self.ws_1, stream=s_front)
        if self.front_spans is not None:
            e[1].record(s_front)
            self.front_spans.append(e)
        s_front.wait_event(self.ev_tok)
        self.ev_front[b].record(s_front)
        return self.ev_front[b]

    def back(self, k: int, main):
        """Stage II of batch k on `main` into self.out."""
        b = k & 1
        main.wait_event(self.ev_front[b])
        self.ot.onetrans_stage2_score(self.model, self.cache[b], self.slots, self.offs, self.ns[b], self.out,
                                      self.ws_2, stream=main)
        self.ev_back[b].record(main)

    metric, unit = METRIC, UNIT
    io_names = ("S", "F")       # per-step inputs, uploaded from pinned host copies in the end-to-end leg

    def config(self, ws):
        return kv_serving_config(self.U, self.C, ws)

    def prepare(self, n_steps: int):
        pass

    def oracle(self):
        return oracle_sample()


class Append:
    """Cross-request append for U users (non-pyramid 6 x 256, 1178 cached S
    tokens each): tokenize dL = 16 new events, append their K/V to every
    layer's cache, then auto-split and score C candidates per user against
    the extended cache.  Each step starts from a 1178-token cache: every step
    gets its own cache, encoded by Stage I before anything is timed (one
    cache is 1.9 GB at 256 users, so this workload caps its step counts:
    3 warm-up, 2 x 10 timed and 5 end-to-end steps hold 53 GB).  Served as a
    pipeline like KVServing: batch k+1's append runs beside batch k's
    Stage II."""

    pipelined = True

    max_steps, max_warmup = 10, 3
    io_names = ("ev", "F")

    metric, unit = APPEND_METRIC, "users/s"

    def __init__(self, rank: int, users: int = 0, cands: int = 0):
        import torch
        import unified_transformer_recommender_b200 as ot
        from onetrans_synth import WORKLOADS, gen_normal, make_weights, random_types
        self.ot, self.torch = ot, torch
        wl = WORKLOADS["append"]
        self.wl, sh = wl, wl.shape
        self.U, self.C, self.dL = users or wl.users, cands or wl.cands, wl.dL
        W = make_weights(sh, wl.seed_weights, wl.dtype, event_dim=wl.event_dim)
        self.model = ot.model_from_arrays(sh, W, pyramid_q=None, mode=ot.BF16, event_dim=wl.event_dim)
        seed = wl.seed_inputs + 7919 * rank
        dev = torch.device("cuda")
        self.S = torch.from_numpy(gen_normal(seed, (self.U, wl.L_S, sh.d), "bf16")).to(dev, torch.bfloat16)
        self.ev_h = gen_normal(seed + 200, (self.U, self.dL, wl.event_dim), "bf16")
        self.F_h = gen_normal(seed + 100, (self.U * self.C, sh.ns_feat), "bf16")
        self.ev = torch.from_numpy(self.ev_h).to(dev, torch.bfloat16)
        self.ty = torch.from_numpy(random_types(seed + 300, (self.U, self.dL), sh.n_types)).to(dev)
        self.F = torch.from_numpy(self.F_h).to(dev, torch.bfloat16)
        self.ev_pin = torch.from_numpy(self.ev_h).to(torch.bfloat16).pin_memory()
        self.F_pin = torch.from_numpy(self.F_h).to(torch.bfloat16).pin_memory()
        m = self.model
        self.caches, self.k = [], 0
        self.bank_cache = [None, None]
        # default priority: the front's short launches fill the SMs that the
        # previous batch's Stage II leaves idle (a higher priority made them
        # hold back Stage II's CTAs and the step slower)
        self.s_front, self.s_tok = torch.cuda.Stream(), torch.cuda.Stream()
        ev = torch.cuda.Event
        self.ev_in, self.ev_tok = ev(), ev()
        self.ev_front, self.ev_back = [ev(), ev()], [ev(), ev()]
        self.front_spans = None
        self.slots = list(range(self.U))
        self.offs = [u * self.C for u in range(self.U + 1)]
        self.ns = [torch.empty(self.U * self.C, sh.L_NS, sh.d, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.out = torch.empty(self.U * self.C, sh.L_NS, sh.d, dtype=torch.float32, device=dev)
        self.out_pin = torch.empty(self.out.shape, dtype=torch.float32).pin_memory()
        self.ws_1 = m.workspace(ot.OP_STAGE1, self.U, wl.L_S)
        self.ws_ap = m.workspace(ot.OP_APPEND, self.U, self.dL)
        self.ws_a = m.workspace(ot.OP_AUTOSPLIT, self.U * self.C)
        self.ws_2 = m.workspace(ot.OP_STAGE2, self.U * self.C, wl.L_S + self.dL)
        self.units = self.U
        self.h2d = self.ev_h.size * 2 + self.F_h.size * 2
        self.d2h = self.out.numel() * 4

    def config(self, ws):
        return append_config(self.U, self.C, self.dL, ws)

    def prepare(self, n_steps: int):
        """One Stage I-encoded cache per step to come (untimed)."""
        ot = self.ot
        for _ in range(n_steps):
            c = ot.Cache(self.model, self.U, self.wl.L_S + self.dL)
            ot.onetrans_stage1_encode(self.model, c, self.slots, self.S, self.ws_1)
            self.caches.append(c)
        self.torch.cuda.synchronize()

    def set_inputs(self, i: int):
        pass

    def front(self, k: int, main, serial: bool = False):
        """The append into the next prepared cache and the candidates'
        auto-split into NS bank k % 2, on two side streams, after the inputs
        are ready on `main` and after Stage II of batch k-2.  serial:
        everything on `main` (the per-kernel timing pass)."""
        ot, m, b = self.ot, self.model, k & 1
        s_front, s_tok = (main, main) if serial else (self.s_front, self.s_tok)
        cache = self.caches[self.k]
        self.k += 1
        self.bank_cache[b] = cache
        self.ev_in.record(main)
        for s in (s_front, s_tok):
            s.wait_event(self.ev_in)
            s.wait_event(self.ev_back[b])
        ot.onetrans_tokenize_autosplit(m, self.F, self.ns[b], self.ws_a, stream=s_tok)
        self.ev_tok.record(s_tok)
        if self.front_spans is not None:
            e = (self.torch.cuda.Event(enable_timing=True), self.torch.cuda.Event(enable_timing=True))
            e[0].record(s_front)
        ot.onetrans_cache_append(m, cache, self.slots, self.ev, self.ty, self.ws_ap, stream=s_front)
        if self.front_spans is not None:
            e[1].record(s_front)
            self.front_spans.append(e)
        s_front.wait_event(self.ev_tok)
        self.ev_front[b].record(s_front)
        return self.ev_front[b]

    def back(self, k: int, main):
        b = k & 1
        main.wait_event(self.ev_front[b])
        self.ot.onetrans_stage2_score(self.model, self.bank_cache[b], self.slots, self.offs, self.ns[b], self.out,
                                      self.ws_2, stream=main)
        self.ev_back[b].record(main)

    def oracle(self):
        return oracle_sample_append(self.U, self.C)


class Forward:
    """One-pass forward of B samples through the stack (onetrans_forward):
    s_forward = 6 x 256, 64 samples of 1178 + 12 tokens, pyramid 1190 -> 12;
    l_forward = 8 x 384, 256 samples of 2048 + 16 tokens, pyramid 2064 -> 16."""

    unit = "samples/s"
    io_names = ("X",)

    def __init__(self, name: str, rank: int, users: int = 0):
        import torch
        import unified_transformer_recommender_b200 as ot
        from onetrans_synth import WORKLOADS, gen_normal, make_weights
        self.ot, self.torch, self.name = ot, torch, name
        wl = WORKLOADS[name]
        self.wl, sh = wl, wl.shape
        self.U = users or wl.users
        self.metric = forward_metric(name)
        W = make_weights(sh, wl.seed_weights, wl.dtype)
        self.model = ot.model_from_arrays(sh, W, pyramid_q=list(wl.pyramid), mode=ot.BF16)
        dev = torch.device("cuda")
        self.X_h = gen_normal(wl.seed_inputs + 7919 * rank, (self.U, wl.L0, sh.d), "bf16")
        self.X = torch.from_numpy(self.X_h).to(dev, torch.bfloat16)
        self.X_pin = torch.from_numpy(self.X_h).to(torch.bfloat16).pin_memory()
        sched = self.model.schedule(wl.L_S)
        self.out = torch.empty(self.U, sched[-1], sh.d, dtype=torch.float32, device=dev)
        self.out_pin = torch.empty(self.out.shape, dtype=torch.float32).pin_memory()
        self.ws = self.model.workspace(ot.OP_FORWARD, self.U, wl.L_S)
        self.units = self.U
        self.h2d = self.X_h.size * 2
        self.d2h = self.out.numel() * 4

    def config(self, ws):
        return forward_config(self.name, self.U, ws)

    def prepare(self, n_steps: int):
        pass

    def step(self, ev_mid=None):
        self.ot.onetrans_forward(self.model, self.X, self.out, self.ws)

    def oracle(self):
        return oracle_sample_forward(self.name, self.U)


class Train:
    """Training step of the s_forward model (onetrans_forward_backward) on
    TRAIN_SAMPLES samples: an upstream gradient dY of the output in, the
    output, dX0 and every weight gradient out."""

    unit = "samples/s"
    io_names = ("X", "dY")

    def __init__(self, rank: int, users: int = 0):
        import torch
        import unified_transformer_recommender_b200 as ot
        from onetrans_synth import WORKLOADS, gen_normal, make_weights
        self.ot, self.torch = ot, torch
        wl = WORKLOADS["s_forward"]
        self.wl, sh = wl, wl.shape
        self.U = users or TRAIN_SAMPLES
        self.metric = TRAIN_METRIC
        self.W = make_weights(sh, wl.seed_weights, wl.dtype)
        self.model = ot.model_from_arrays(sh, self.W, pyramid_q=list(wl.pyramid), mode=ot.BF16)
        dev = torch.device("cuda")
        self.X_h = gen_normal(wl.seed_inputs + 7919 * rank, (self.U, wl.L0, sh.d), "bf16")
        self.dY_h = gen_normal(wl.seed_inputs + 17 + 7919 * rank, (self.U, sh.L_NS, sh.d), "fp32")
        self.X = torch.from_numpy(self.X_h).to(dev, torch.bfloat16)
        self.dY = torch.from_numpy(self.dY_h).to(dev)
        self.X_pin = torch.from_numpy(self.X_h).to(torch.bfloat16).pin_memory()
        self.dY_pin = torch.from_numpy(self.dY_h).pin_memory()
        self.out = torch.empty(self.U, sh.L_NS, sh.d, dtype=torch.float32, device=dev)
        self.out_pin = torch.empty(self.out.shape, dtype=torch.float32).pin_memory()
        self.dX = torch.empty(self.U, wl.L0, sh.d, dtype=torch.float32, device=dev)
        keys = ("g_attn", "g_ffn", "Wqkv_S", "Wqkv_NS", "Wo", "W1_S", "b1_S", "W2_S", "b2_S", "W1_NS", "b1_NS",
                "W2_NS", "b2_NS")
        self.grads = {k: [torch.empty(tuple(self.W[k][l].shape), dtype=torch.float32, device=dev)
                          for l in range(sh.n_layers)] for k in keys}
        self.ws = self.model.workspace(ot.OP_TRAIN, self.U, wl.L_S)
        self.units = self.U
        self.h2d = self.X_h.size * 2 + self.dY_h.size * 4
        self.d2h = self.out.numel() * 4

    def config(self, ws):
        return train_config(self.U, ws)

    def prepare(self, n_steps: int):
        pass

    def step(self, ev_mid=None):
        self.ot.onetrans_forward_backward(self.model, self.X, self.dY, self.out, self.dX, self.grads, self.ws)

    def oracle(self):
        return oracle_sample_train(self.U)


class E2EPipeline:
    """End-to-end leg: every step uploads its inputs from pinned host memory
    and downloads its result to pinned host memory, through the public API.
    Two device copies of the inputs and of the output let the upload of step
    i+1 and the download of step i-1 run on side streams while step i
    computes, as a serving loop would; event waits keep each buffer's reuse
    in order.  The timed span runs from the first upload to the last
    download."""

    def __init__(self, wk):
        import torch
        self.wk, self.torch = wk, torch
        self.din = [{n: getattr(wk, n) for n in wk.io_names},
                    {n: torch.empty_like(getattr(wk, n)) for n in wk.io_names}]
        self.dout = [wk.out, torch.empty_like(wk.out)]
        self.hout = [wk.out_pin, torch.empty(wk.out_pin.shape, dtype=wk.out_pin.dtype, pin_memory=True)]
        self.s_in, self.s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = torch.cuda.Event
        self.in_ready, self.in_free = [ev(), ev()], [ev(), ev()]
        self.done, self.out_free = [ev(), ev()], [ev(), ev()]

    def run(self, n: int, main, e0=None, e1=None):
        torch, wk = self.torch, self.wk
        start = torch.cuda.Event()
        if e0 is not None:
            e0.record(main)
        start.record(main)
        self.s_in.wait_event(start)
        self.s_out.wait_event(start)
        pipelined = getattr(wk, "pipelined", False)
        for i in range(n):
            b = i & 1
            if i >= 2:
                self.s_in.wait_event(self.in_free[b])
            with torch.cuda.stream(self.s_in):
                for name in wk.io_names:
                    self.din[b][name].copy_(getattr(wk, name + "_pin"), non_blocking=True)
                self.in_ready[b].record(self.s_in)
            main.wait_event(self.in_ready[b])
            for name in wk.io_names:
                setattr(wk, name, self.din[b][name])
            if pipelined:
                # batch i's front reads the inputs; batch i-1's Stage II
                # follows on `main`, its download on s_out
                self.in_free[b] = wk.front(i, main)
                if i >= 1:
                    self._back(i - 1, main)
            else:
                if i >= 2:
                    main.wait_event(self.out_free[b])
                wk.out = self.dout[b]
                wk.step()
                self.in_free[b].record(main)
                self._download(b, main)
        if pipelined:
            self._back(n - 1, main)
        main.wait_stream(self.s_in)
        main.wait_stream(self.s_out)
        if e1 is not None:
            e1.record(main)
        for name in wk.io_names:
            setattr(wk, name, self.din[0][name])
        wk.out = self.dout[0]

    def _back(self, j: int, main):
        bj = j & 1
        if j >= 2:
            main.wait_event(self.out_free[bj])
        self.wk.out = self.dout[bj]
        self.wk.back(j, main)
        self._download(bj, main)

    def _download(self, b: int, main):
        self.done[b].record(main)
        self.s_out.wait_event(self.done[b])
        with self.torch.cuda.stream(self.s_out):
            self.hout[b].copy_(self.dout[b], non_blocking=True)
            self.out_free[b].record(self.s_out)


def run_pipelined(wk, main, n: int, serial: bool = False):
    """n batches through a pipelined workload: front(i) is issued before
    back(i-1); the last back drains the pipeline.  serial: front(i) then
    back(i), every kernel on `main`, so each runs alone (the per-kernel
    timing pass)."""
    for i in range(n):
        wk.set_inputs(i)
        if serial:
            wk.front(i, main, serial=True)
            wk.back(i, main)
            continue
        wk.front(i, main)
        if i >= 1:
            wk.back(i - 1, main)
    if not serial:
        wk.back(n - 1, main)


def make_workload(name: str, rank: int, users: int = 0, cands: int = 0):
    if name == "kv_serving":
        return KVServing(rank, users=users, cands=cands)
    if name == "append":
        return Append(rank, users=users, cands=cands)
    if name == "train":
        return Train(rank, users=users)
    return Forward(name, rank, users=users)


# ------------------------------------------------------------- CPU oracle

def oracle_sample(n_cands: int = 160, seed_shift: int = 0):
    """Time the fp64 oracle on 1 user's Stage I plus n_cands candidates'
    auto-split and Stage II; returns (candidates/s of the full workload by
    linear extrapolation, sample description, threads used)."""
    from onetrans_synth import WORKLOADS, gen_normal, make_weights
    from oracle import onetrans as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count()
    wl = WORKLOADS["kv_serving"]
    sh = wl.shape
    W = make_weights(sh, wl.seed_weights, "bf16")
    S = gen_normal(wl.seed_inputs + seed_shift, (1, wl.L_S, sh.d), "bf16")
    F = gen_normal(wl.seed_inputs + 100 + seed_shift, (n_cands, sh.ns_feat), "bf16")
    t0 = time.perf_counter()
    kv = O.stage1(S[0], W, sh.L_NS, sh.n_heads, sh.eps, wl.pyramid)
    t1 = time.perf_counter()
    ns = O.autosplit(F, W, sh.L_NS)
    for c in range(n_cands):
        O.stage2(kv, ns[c], W, sh.n_heads, sh.eps)
    t2 = time.perf_counter()
    per_user, per_cand = t1 - t0, (t2 - t1) / n_cands
    step_s = wl.users * per_user + wl.users * wl.cands * per_cand
    desc = (f"oracle fp64: Stage I of 1 user ({per_user:.2f} s) + auto-split and Stage II of {n_cands} "
            f"candidates ({per_cand * 1e3:.1f} ms each), extrapolated linearly to {wl.users} users x "
            f"{wl.cands} candidates ({step_s:.0f} s per step)")
    return wl.users * wl.cands / step_s, desc, cores, t2 - t0


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def oracle_sample_append(users: int, cands: int, n_cands: int = 16):
    """fp64 oracle on 1 user's append (tokenize dL events, extend every
    layer's K/V) plus n_cands candidates' auto-split and Stage II, extrapolated
    linearly to users x cands; returns (users/s, description, threads, s)."""
    from onetrans_synth import WORKLOADS, gen_normal, make_weights, random_types
    from oracle import onetrans as O
    wl = WORKLOADS["append"]
    sh = wl.shape
    W = make_weights(sh, wl.seed_weights, "bf16", event_dim=wl.event_dim)
    S = gen_normal(wl.seed_inputs, (1, wl.L_S, sh.d), "bf16")
    ev = gen_normal(wl.seed_inputs + 200, (1, wl.dL, wl.event_dim), "bf16")
    ty = random_types(wl.seed_inputs + 300, (1, wl.dL), sh.n_types)
    F = gen_normal(wl.seed_inputs + 100, (n_cands, sh.ns_feat), "bf16")
    kv0 = O.stage1(S[0], W, sh.L_NS, sh.n_heads, sh.eps)
    t0 = time.perf_counter()
    kv = O.append(kv0, O.tokenize_events(ev[0], ty[0], W), W, sh.n_heads, sh.eps)
    t1 = time.perf_counter()
    ns = O.autosplit(F, W, sh.L_NS)
    for c in range(n_cands):
        O.stage2(kv, ns[c], W, sh.n_heads, sh.eps)
    t2 = time.perf_counter()
    per_user, per_cand = t1 - t0, (t2 - t1) / n_cands
    step_s = users * per_user + users * cands * per_cand
    desc = (f"oracle fp64: append of 1 user ({per_user:.2f} s) + auto-split and Stage II of {n_cands} candidates "
            f"({per_cand * 1e3:.1f} ms each), extrapolated linearly to {users} users x {cands} candidates")
    return users / step_s, desc, _oracle_threads(), t2 - t0


def oracle_sample_forward(name: str, samples: int):
    """fp64 oracle forward of 1 sample of the workload; returns (samples/s,
    description, threads, s)."""
    from onetrans_synth import WORKLOADS, gen_normal, make_weights
    from oracle import onetrans as O
    wl = WORKLOADS[name]
    sh = wl.shape
    W = make_weights(sh, wl.seed_weights, "bf16")
    X = gen_normal(wl.seed_inputs, (1, wl.L0, sh.d), "bf16")
    t0 = time.perf_counter()
    O.forward(X, W, sh.L_NS, sh.n_heads, sh.eps, list(wl.pyramid))
    t1 = time.perf_counter()
    desc = f"oracle fp64: forward of 1 sample ({t1 - t0:.2f} s); the batch of {samples} scales linearly"
    return 1.0 / (t1 - t0), desc, _oracle_threads(), t1 - t0


def oracle_sample_train(samples: int):
    """fp64 oracle training step (forward keeping each layer's input, backward
    with recomputation) of 1 sample of the train workload; returns (samples/s,
    description, threads, s)."""
    from onetrans_synth import WORKLOADS, gen_normal, make_weights
    from oracle import onetrans as O
    wl = WORKLOADS["s_forward"]
    sh = wl.shape
    W = make_weights(sh, wl.seed_weights, "bf16")
    X = gen_normal(wl.seed_inputs, (1, wl.L0, sh.d), "bf16")
    dY = gen_normal(wl.seed_inputs + 17, (1, sh.L_NS, sh.d), "fp32")
    t0 = time.perf_counter()
    O.forward_backward(X, W, sh.L_NS, sh.n_heads, sh.eps, list(wl.pyramid), dY)
    t1 = time.perf_counter()
    desc = (f"oracle fp64: training step of 1 sample ({t1 - t0:.2f} s); the batch of {samples} scales "
            "linearly")
    return 1.0 / (t1 - t0), desc, _oracle_threads(), t1 - t0


def run_reference(args, rank):
    """The oracle timed on the host cores, each step a bounded sample of the
    workload extrapolated to its full size; same metric, unit and config as
    this arm's line.  Rank 0 alone runs it."""
    if rank != 0:
        return
    from onetrans_synth import WORKLOADS
    metric, unit, config, units = workload_meta(args.workload, args.gpus)
    wl = WORKLOADS.get(args.workload)
    if args.workload == "kv_serving":
        def sample(i):
            return oracle_sample(n_cands=8, seed_shift=i)
    elif args.workload == "append":
        def sample(i):
            return oracle_sample_append(wl.users, wl.cands, n_cands=4)
    elif args.workload == "train":
        def sample(i):
            return oracle_sample_train(TRAIN_SAMPLES)
    else:
        def sample(i):
            return oracle_sample_forward(args.workload, wl.users)
    vals, samples, cores = [], None, 1
    for i in range(args.warmup + args.steps):
        v, desc, cores, secs = sample(i)
        if i >= args.warmup:
            vals.append(v)
            samples = desc
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * units / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": samples},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------------- main

def main():
    args = parse()
    ws, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank)
    import torch
    import torch.distributed as dist
    if ws > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    import unified_transformer_recommender_b200 as ot

    wk = make_workload(args.workload, rank, users=args.users, cands=args.cands)
    if hasattr(wk, "max_steps"):
        args.steps = min(args.steps, wk.max_steps)
        args.warmup = min(max(args.warmup, 3), wk.max_warmup)
    e2e_steps = max(3, args.steps // 4)
    wk.prepare(args.warmup + 2 * args.steps + 2 + e2e_steps)   # two timed passes
    mid = {"kv_serving": "stage1", "append": "append"}.get(args.workload)
    pipelined = getattr(wk, "pipelined", False)
    # L2 flush between the steps of the workloads that run one step at a time
    flush = None if pipelined else torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")  # > 126 MB L2
    st = torch.cuda.current_stream()

    if pipelined:
        run_pipelined(wk, st, args.warmup)
    else:
        for _ in range(args.warmup):
            wk.step()
    torch.cuda.synchronize()
    assert ot.onetrans_device_status() == 0

    # ---- device-timed region: inputs resident in HBM.  Pass 1 records CUDA
    # events between steps only (none between kernels, so each kernel's launch
    # overlaps its predecessor's drain); pass 2 repeats the same steps with an
    # event pair around every kernel of the library for the per-kernel times
    # of the roofline.  A pipelined workload's steps overlap: its pass 1 is one
    # span from the first front to the last Stage II, with the inputs cycled
    # through sets larger than L2, and its pass 2 runs the batches one after
    # another on one stream so that every kernel's time is its own; the
    # others flush L2 between timed steps.
    clocks = ClockSampler(torch.cuda.current_device())

    def timed_pass(profile):
        ot.onetrans_profile_enable(profile)
        barrier()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        if pipelined:
            wk.front_spans = []
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            run_pipelined(wk, st, args.steps, serial=profile)
            e1.record(st)
            torch.cuda.synchronize()
            total = e0.elapsed_time(e1)
            mid_ms = sum(a.elapsed_time(b) for a, b in wk.front_spans)
            wk.front_spans = None
        else:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for i in range(args.steps):
                flush.zero_()
                evs[i][0].record(st)
                wk.step()
                evs[i][1].record(st)
            torch.cuda.synchronize()
            total = sum(a.elapsed_time(b) for a, b in evs)
            mid_ms = None
        barrier()
        wall = time.perf_counter() - t0
        prof = ot.onetrans_profile_read() if profile else None
        ot.onetrans_profile_enable(False)
        return total, mid_ms, wall, prof

    clocks.start()
    total_local, mid_local, wall, _ = timed_pass(False)
    total_prof, _, _, prof = timed_pass(True)
    clk = clocks.stop()
    total_ms = max_over_ranks(total_local)
    total_ms_prof = max_over_ranks(total_prof)
    value = wk.units * args.steps * ws / (total_ms / 1e3)
    if mid:
        s1_total = max_over_ranks(mid_local)

    # ---- end to end through the public API, host buffers (uploads and
    # downloads pipelined with the neighbouring steps' compute)
    pipe = E2EPipeline(wk)
    pipe.run(2, st)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipe.run(e2e_steps, st, e0, e1)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = wk.units * e2e_steps * ws / (e2e_ms / 1e3)
    assert ot.onetrans_device_status() == 0

    # ---- roofline of the dominant kernel (largest device time in the timed region)
    pk = peaks()
    dom_name, dom = max(prof.items(), key=lambda kv: kv[1]["ms"])
    # DRAM bytes per launch come from ncu captures of single launches, which
    # this run does not make; the line's mean over Stage I and Stage II
    # launches has no captured counterpart
    traffic = None
    per_launch_ms = dom["ms"] / dom["launches"]
    # the per-kernel times are single launches of well under a millisecond,
    # timed one by one: the burst figure of the measured GEMM peak applies
    tensor_bound = dom["flops"] / max(dom["bytes"], 1.0) > pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)
    if dom_name in ALU_KERNELS:
        # CUDA-core float32 arithmetic: SMs x 128 FMA lanes x 2 FLOP x the SM
        # clock measured under load (median of the samples)
        sm_count = torch.cuda.get_device_properties(0).multi_processor_count
        mhz = clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0
        peak = sm_count * 128 * 2 * mhz * 1e6 / 1e12
        achieved = dom["flops"] / (dom["ms"] / 1e3) / 1e12
        roof = {"bound": "alu", "kernel": dom_name, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "peak_source": f"{sm_count} SMs x 128 fp32 FMA lanes x 2 FLOP x {mhz:.0f} MHz (measured clock)",
                "traffic": traffic, "flops_per_launch": dom["flops"] / dom["launches"],
                "ms_per_launch": per_launch_ms}
    elif tensor_bound:
        achieved = dom["flops"] / (dom["ms"] / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": dom_name, "achieved": achieved, "peak": pk["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                "peak_source": pk["source"] + " bf16 burst (single launches)", "traffic": traffic,
                "flops_per_launch": dom["flops"] / dom["launches"], "ms_per_launch": per_launch_ms}
    else:
        achieved = dom["bytes"] / (dom["ms"] / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": dom_name, "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "peak_source": pk["source"] + " copy", "traffic": traffic,
                "bytes_per_launch": dom["bytes"] / dom["launches"], "ms_per_launch": per_launch_ms}
    kernels = {k: {"launches": v["launches"], "ms": round(v["ms"], 3),
                   "share": round(v["ms"] / sum(x["ms"] for x in prof.values()), 4),
                   "TFLOP/s": round(v["flops"] / (v["ms"] / 1e3) / 1e12, 1) if v["flops"] else None,
                   "GB/s": round(v["bytes"] / (v["ms"] / 1e3) / 1e9, 1)}
               for k, v in sorted(prof.items(), key=lambda kv: -kv[1]["ms"])}

    line = {
        "metric": wk.metric, "value": value, "unit": wk.unit, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": wk.config(ws),
    }
    if args.workload == "kv_serving":
        line["users_per_s"] = wk.U * args.steps * ws / (total_ms / 1e3)
    if mid:
        # the front's span on its own stream, beside the previous batch's Stage II
        line[f"{mid}_ms_per_step"] = s1_total / args.steps
    line.update({
        "e2e": {"value": e2e_value, "unit": wk.unit, "h2d_bytes_per_step": wk.h2d, "d2h_bytes_per_step": wk.d2h,
                "steps": e2e_steps, "copies": "pinned host buffers; uploads and downloads on two side streams "
                                              "overlap the neighbouring steps' compute"},
        "gpu_launches": int(sum(v["launches"] for v in prof.values())),
        "roofline": roof,
        "kernels": kernels,
        "kernel_times": "second pass over the same steps with a CUDA event pair around every launch "
                        f"(on its stream){', batches one after another on one stream' if pipelined else ''}; "
                        f"that pass took {total_ms_prof / args.steps:.4f} ms per step",
        "clocks": clk,
        "wall_s_timed": wall,
    })
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and not (args.users or args.cands):
        v, desc, cores, secs = wk.oracle()
        line["cpu_baseline"] = {"value": v, "unit": wk.unit, "cores": cores, "kind": "oracle", "sample": desc,
                                "seconds": round(secs, 1)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
