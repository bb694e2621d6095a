#!/usr/bin/env python
"""Benchmark of the iS-KV hot path on B200.

Workload (one GPU): the decode step of a 32-layer GQA model (8 KV heads x head_dim 128, so
d = 1024) at which every layer's K and V pending queue fills at once -- 64 compressed histories at
n ~ 16384 rows, rank r = 256, fold block b = 64, bf16 factors. One timed step runs every row of the
hot path once:

  1. fold (Algorithm 2): one 64-row block into each of the 64 histories (one batched call);
  2. re-orthogonalisation (Section 4.4) of all 64 histories (one batched call);
  3. reconstruction (Algorithm 3 steps 7-8) of all 64 caches -- compressed rows plus 640 exact rows
     (512-token prompt kept exact, 128-row recent window), RoPE theta = 500000 on K;
  4. prompt-block selection (Algorithm 1 steps 2-4) on one layer's 65536-token post-RoPE prompt.

n grows by 64 rows per step; it starts so that the timed steps are centred on n = 16384. Inputs are
seeded synthetic low-rank-plus-noise rows (K spectrum i^-1.2, V i^-0.6, noise 0.02) standing in for
model traces. Everything a step reads is resident in HBM before timing starts; a step touches
~4 GB, far more than the 126 MB L2, so no flush is needed.

metric: block folds/s (64 folds per step); the line also reports reconstructed KV rows/s and, per
stage, device time and the achieved fraction of the measured HBM roofline.

--impl reference times the float64 CPU oracle on a bounded sample of the same step (one fold,
one reorth and one reconstruction at n = 16384, one selection) and extrapolates to a whole step.
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

METRIC = "block folds/s and reconstructed KV rows/s (n=16K,d=1024,r=256), % of roofline"
LAYERS, HEADS, HEAD_DIM = 32, 8, 128
D, R, BLK = HEADS * HEAD_DIM, 256, 64
N_MID = 16384
PROMPT, WINDOW = 512, 128
THETA = 500000.0
SEL_L = 65536
Q_HEADS = 32  # decode-attention query heads (grouped: 4 per KV head)
SPEC = {"K": 1.2, "V": 0.6}
NOISE = 0.02


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------------------------------------------
# Clock sampling during the timed region.

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, log_dir=None):
        self.idx = gpu_index
        self.proc = None
        self.path = os.path.join(log_dir or tempfile.gettempdir(), f"clocks_rank{gpu_index}.csv")

    def start(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------------
# Multi-rank plumbing: one process per GPU, independent histories (weak scaling). The only
# collectives are the start/stop barriers and this max over ranks of the device-timed duration.

def max_over_ranks(value: float, device) -> float:
    """Maximum of `value` over all ranks of the default process group (the value itself when
    running alone)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Seed of a rank's synthetic histories: every rank folds different data."""
    return 1000 + 100 * int(rank)


# ------------------------------------------------------------------------------------------------
# The B200 arm.

class Workload:
    """64 histories (32 layers x {K, V}) and every per-step input, resident on the device."""

    def __init__(self, kv, torch, dev, warmup: int, timed: int, extra: int, seed: int = 1000,
                 layers: int = LAYERS):
        import synth
        self.kv, self.torch, self.dev = kv, torch, dev
        # n after the fold of step t is n0 + 64 (t + 1); the timed steps are centred on N_MID.
        self.n0 = N_MID - BLK * (warmup + (timed + 1) // 2)
        self.n_cap = self.n0 + BLK * (warmup + timed + extra + 1)
        self.hists, self.kinds = [], []
        gen = torch.Generator(device=dev)
        for layer in range(layers):
            for kind in ("K", "V"):
                h = kv.LowRankHistory(D, R, self.n_cap, storage=torch.bfloat16, device=dev)
                sd = seed + 2 * layer + (kind == "V")
                U = synth.torch_orthonormal(self.n0, R, sd, device=dev)
                B = synth.torch_orthonormal(D, R, sd + 50000, device=dev)
                s = (self.n0 ** 0.5) * torch.arange(1, R + 1, device=dev,
                                                    dtype=torch.float32) ** (-SPEC[kind])
                h.U[:self.n0] = U.to(torch.bfloat16)
                h.B.copy_(B.to(torch.bfloat16))
                h.sigma.copy_(s)
                h.pos[:self.n0] = torch.arange(PROMPT, PROMPT + self.n0, dtype=torch.int32,
                                               device=dev)
                h.meta.copy_(torch.tensor([R, self.n0, 0, 0], dtype=torch.int64))
                self.hists.append(h)
                self.kinds.append(kind)
        # Pending blocks: rows in the history's subspace plus noise (4 rotating sets).
        self.F = []
        for sset in range(4):
            blocks = []
            for i, h in enumerate(self.hists):
                gen.manual_seed(seed + 7919 * sset + i)
                a = SPEC[self.kinds[i]]
                coef = torch.randn(BLK, R, generator=gen, device=dev) * (
                    torch.arange(1, R + 1, device=dev, dtype=torch.float32) ** (-a))
                rows = coef @ h.B.float().T + NOISE * torch.randn(BLK, D, generator=gen, device=dev)
                blocks.append(rows.to(torch.bfloat16).contiguous())
            self.F.append(blocks)
        # Exact rows per history: 512 prompt rows + 128 window rows.
        self.exact = []
        for i in range(len(self.hists)):
            gen.manual_seed(seed + 31337 + i)
            self.exact.append((torch.randn(PROMPT + WINDOW, D, generator=gen, device=dev)
                               ).to(torch.bfloat16).contiguous())
        self.rope = [k == "K" for k in self.kinds]
        self.n_total_max = PROMPT + self.n_cap + WINDOW
        self.outs = [torch.empty(self.n_total_max, D, dtype=torch.bfloat16, device=dev)
                     for _ in self.hists]
        # Prompt keys for the selection (post-RoPE, 5% outlier blocks per head).
        keys, _ = synth.outlier_prompt_keys(SEL_L, HEADS, HEAD_DIM, seed=4)
        self.keys = torch.as_tensor(keys, dtype=torch.float32).to(dev).to(torch.bfloat16)
        self.sel_out = None
        # Workspaces (sized once).
        cnt = len(self.hists)
        self.ws_fold = torch.empty(kv.fold_workspace_size(cnt, D, R, BLK) + 256,
                                   dtype=torch.uint8, device=dev)
        self.ws_reorth = torch.empty(kv.reorth_workspace_size(cnt, D, R, self.n_cap) + 256,
                                     dtype=torch.uint8, device=dev)
        self.ws_recon = torch.empty(kv.reconstruct_workspace_size(cnt, D, R) + 256,
                                    dtype=torch.uint8, device=dev)
        self.ws_sel = torch.empty(kv.select_workspace_size(SEL_L, HEADS, 8) + 256,
                                  dtype=torch.uint8, device=dev)
        # Per-step positions.
        self.step_idx = 0
        torch.cuda.synchronize(dev)

    @staticmethod
    def _aligned(buf):
        off = (-buf.data_ptr()) % 256
        return buf[off:]

    def n_after(self, t):
        return self.n0 + BLK * (t + 1)

    def positions(self, t):
        torch = self.torch
        n_before = self.n0 + BLK * t
        fpos = torch.arange(PROMPT + n_before, PROMPT + n_before + BLK, dtype=torch.int32,
                            device=self.dev)
        n = n_before + BLK
        epos = torch.cat([torch.arange(0, PROMPT, dtype=torch.int32, device=self.dev),
                          torch.arange(PROMPT + n, PROMPT + n + WINDOW, dtype=torch.int32,
                                       device=self.dev)])
        return fpos, epos, PROMPT + n + WINDOW

    def step(self, t, fpos, epos, n_total, F=None):
        kv = self.kv
        F = F if F is not None else self.F[t % 4]
        cnt = len(self.hists)
        kv.fold_block_batched(self.hists, F, [fpos] * cnt, ws=self._aligned(self.ws_fold))
        kv.reorth(self.hists, ws=self._aligned(self.ws_reorth))
        kv.reconstruct_batched(self.hists, self.exact, [epos] * cnt, n_total, HEADS, HEAD_DIM,
                               self.rope, THETA, outs=self.outs, ws=self._aligned(self.ws_recon))
        self.sel_out = kv.select_prompt_blocks(self.keys, 8, 128, 4, 32,
                                               ws=self._aligned(self.ws_sel), out=self.sel_out)


ROOFLINE_STAGE = "reconstruct.compressed"


def stage_bytes(n_mean: float, layers: int = LAYERS):
    """Algorithmic bytes per call of each stage for one whole step (2 histories per layer), bf16
    factors."""
    H = layers * 2
    n_tot = PROMPT + n_mean + WINDOW
    return {
        # U read + write over every history row (Algorithm 2 step 7).
        "fold.coord_rotate": H * (4.0 * n_mean * R),
        # per compressed row: U row (2r) + output row (2d) + position (4); plus the basis (2dr).
        "reconstruct.compressed": H * (n_mean * (2 * R + 2 * D + 4) + 2.0 * D * R),
        # per exact row: read (2d) + write (2d) + position.
        "reconstruct.exact": H * ((PROMPT + WINDOW) * (4.0 * D + 4)),
        # reorth: U read for the Gram (2nr) + U read/write in the rotation (4nr).
        "reorth.gram": H * (2.0 * n_mean * R + 2.0 * D * R),
        "reorth.coord_rotate": H * (4.0 * n_mean * R),
        # selection: every post-RoPE key once (bf16).
        "select": SEL_L * HEADS * HEAD_DIM * 2.0,
    }, H * n_tot


def time_attention(wl, kv, torch, dev, stream, reps: int = 10, warm: int = 3):
    """Decode attention over the compressed cache of every layer (K and V histories of the
    benchmark state, the same 640 exact rows per history, one float32 query of 32 heads per
    layer), timed on its own: it is the next row after the hot path, not part of the step."""
    layers = len(wl.hists) // 2
    n = int(wl.hists[0].status()[1])
    epos = torch.cat([torch.arange(0, PROMPT, dtype=torch.int32, device=dev),
                      torch.arange(PROMPT + n, PROMPT + n + WINDOW, dtype=torch.int32,
                                   device=dev)])
    n_total = PROMPT + n + WINDOW
    gen = torch.Generator(device=dev)
    gen.manual_seed(777)
    qs = [torch.randn(Q_HEADS, HEAD_DIM, generator=gen, device=dev) for _ in range(layers)]
    outs = [torch.empty(Q_HEADS, HEAD_DIM, dtype=torch.float32, device=dev) for _ in range(layers)]
    kh, vh = wl.hists[0::2], wl.hists[1::2]
    kex, vex = wl.exact[0::2], wl.exact[1::2]
    ws = torch.empty(kv.attention_workspace_size(layers, D, R, wl.n_cap, n_total, Q_HEADS) + 256,
                     dtype=torch.uint8, device=dev)
    wsa = Workload._aligned(ws)

    def call():
        kv.decode_attention_batched(kh, vh, kex, [epos] * layers, vex, [epos] * layers, n_total,
                                    qs, HEADS, HEAD_DIM, THETA, outs=outs, ws=wsa, stream=stream)

    for _ in range(warm):
        call()
    torch.cuda.synchronize(dev)
    kv.stage_times(reset=True)
    kv.stage_timing(True)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(reps):
        call()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    kv.stage_timing(False)
    st = kv.stage_times(reset=True)
    ms = ev0.elapsed_time(ev1) / reps
    status = [h.status()[3] for h in wl.hists]
    # Algorithmic bytes per call: both coordinate tables, both bases, the exact rows of both
    # caches and the positions (scores and partial sums are the kernels' own intermediates).
    byt = layers * (2 * n * R * 2 + 2 * D * R * 2 + 2 * (PROMPT + WINDOW) * D * 2 + 2 * n * 4)
    hbm, _, _ = peaks()
    gbs = byt / (ms / 1e3) / 1e9
    return {"ms_per_call": round(ms, 4), "layers": layers, "n": n, "n_total": n_total,
            "q_heads": Q_HEADS, "kv_heads": HEADS, "bytes_per_call": int(byt),
            "achieved_gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
            "stages": {k: round(v[0] / max(v[1], 1), 4) for k, v in st.items()
                       if k.startswith("attention") and v[1]},
            "status_clean": all(x == 0 for x in status)}


def run_diagnostics(wl, kv, torch, dev, stream):
    """Section 5.1 eq. (12) and factor orthogonality of every history after the timed steps:
    ||U^T U - I||_F, ||B^T B - I||_F, persistent bytes against the dense cache."""
    n = [int(h.status()[1]) for h in wl.hists]
    ne = [PROMPT + WINDOW] * len(wl.hists)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    kv.diagnostics(wl.hists, n_exact=ne, exact_bytes=2, stream=stream)  # warm-up
    ev0.record(stream)
    ou, ob, pb = kv.diagnostics(wl.hists, n_exact=ne, exact_bytes=2, stream=stream)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    dense = sum(2 * (x + PROMPT + WINDOW) * D for x in n)
    tot = int(pb.sum().item())
    return {"ms_per_call": round(ev0.elapsed_time(ev1), 4),
            "orth_u_max": float(ou.max().item()), "orth_b_max": float(ob.max().item()),
            "persistent_bytes": tot, "dense_bytes": int(dense),
            "compression": round(dense / max(tot, 1), 3)}


def time_cache_policy(wl, kv, torch, dev, stream):
    """The cache policy's decode step (Algorithm 3 steps 1-2 and 4-6) on the benchmark's 64 histories:
    each side's exact-row table holds its 512 protected prompt rows and its 128 window rows (W = 128,
    b = 64); 63 steps only store the new rows, the 64th folds the oldest 64 rows of every table and
    removes them from the tables. Run last: it folds one more block into every history."""
    cnt = len(wl.hists)
    tabs = []
    for i, h in enumerate(wl.hists):
        n = int(h.status()[1])
        t = kv.ExactTable(D, PROMPT + WINDOW + BLK, window=WINDOW, block=BLK, reorth_rows=0,
                          dtype=torch.bfloat16, device=dev)
        t.rows[:PROMPT + WINDOW].copy_(wl.exact[i])
        win = torch.arange(PROMPT + n, PROMPT + n + WINDOW, dtype=torch.int32, device=dev)
        t.pos[:PROMPT + WINDOW].copy_(torch.cat([torch.arange(PROMPT, dtype=torch.int32,
                                                              device=dev), win]))
        for j in range(WINDOW):
            t.live[j] = PROMPT + n + j
        t.t.n_prot, t.t.n_live, t.t.last, t.t.hist_rows = PROMPT, WINDOW, PROMPT + n + WINDOW - 1, n
        tabs.append(t)
    gen = torch.Generator(device=dev)
    gen.manual_seed(4242)
    rows = torch.randn(BLK, cnt, D, generator=gen, device=dev).to(torch.bfloat16)
    batch = kv.CacheBatch(tabs, wl.hists)
    torch.cuda.synchronize(dev)
    kv.stage_times(reset=True)
    kv.stage_timing(True)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record(stream)
    for j in range(BLK - 1):
        folded, _ = batch.step(rows[j], stream=stream)
        assert not any(folded)
    ev[1].record(stream)
    folded, _ = batch.step(rows[BLK - 1], stream=stream)
    ev[2].record(stream)
    torch.cuda.synchronize(dev)
    kv.stage_timing(False)
    st = kv.stage_times(reset=True)
    a_ms = ev[0].elapsed_time(ev[1]) / (BLK - 1)
    f_ms = ev[1].elapsed_time(ev[2])
    per = {k: round(v[0] / max(v[1], 1), 4) for k, v in st.items()
           if v[1] and (k.startswith("cache") or k.startswith("fold"))}
    ok = all(folded) and all(t.t.n_live == WINDOW for t in tabs) and \
        all(h.status()[3] == 0 for h in wl.hists)
    return {"tables": cnt, "window": WINDOW, "block": BLK,
            "store_step_ms": round(a_ms, 4), "fold_step_ms": round(f_ms, 4),
            "ms_per_token_amortised": round(((BLK - 1) * a_ms + f_ms) / BLK, 4),
            "kernel_ms": per, "status_ok": bool(ok),
            "note": "step times are CUDA events on the stream around each call, so a store-only "
                    "step includes the host's per-call overhead; kernel_ms are the library's "
                    "stage events"}


def run_b200(args):
    import torch
    import torch.distributed as dist

    import kv_cache_online_b200 as kv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(f"cuda:{local}"))
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    kv._lib.load()
    steps_total = args.warmup + args.steps
    e2e_steps = 0 if args.no_e2e else args.steps
    wl = Workload(kv, torch, dev, args.warmup, args.steps, e2e_steps, seed=rank_seed(rank),
                  layers=args.layers)
    pos = [wl.positions(t) for t in range(steps_total + e2e_steps)]
    stream = torch.cuda.current_stream(dev)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    # Warm-up.
    for t in range(args.warmup):
        wl.step(t, *pos[t])
    barrier()

    # Timed region (device events on the launching stream, stage events inside the library).
    sampler = ClockSampler(local, args.clock_log_dir)
    kv.stage_times(reset=True)
    kv.stage_timing(True)
    launches0 = kv.launch_count()
    sampler.start()
    time.sleep(0.3)
    barrier()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for t in range(args.warmup, steps_total):
        wl.step(t, *pos[t])
    ev1.record(stream)
    barrier()
    clocks = sampler.stop()
    launches = kv.launch_count() - launches0
    kv.stage_timing(False)
    st = kv.stage_times(reset=True)
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    ms_step = ms / args.steps
    folds_step = len(wl.hists)
    n_mean = sum(wl.n_after(t) for t in range(args.warmup, steps_total)) / args.steps
    value = world * folds_step * args.steps / (ms / 1e3)
    rows_step = len(wl.hists) * (PROMPT + n_mean + WINDOW)
    rows_per_s = world * rows_step * args.steps / (ms / 1e3)

    # Parity spot check of the benchmark state (one history, sampled rows) against the oracle.
    check = None
    if rank == 0 and not args.no_check:
        check = spot_check(wl, torch)

    # Stage rooflines.
    hbm, tc, peak_kind = peaks()
    sbytes, _ = stage_bytes(n_mean, args.layers)
    stages = {}
    for name, (tot_ms, calls) in st.items():
        if calls == 0:
            continue
        avg = tot_ms / calls
        ent = {"ms_per_call": round(avg, 4), "calls": int(calls),
               "share": round(tot_ms / max(ms, 1e-9), 4)}
        if name in sbytes:
            gbs = sbytes[name] / (avg / 1e3) / 1e9
            ent.update({"bytes_per_call": int(sbytes[name]), "achieved_gbs": round(gbs, 1),
                        "frac_hbm": round(gbs / hbm, 4)})
        stages[name] = ent
    dom = max(stages, key=lambda k: stages[k]["ms_per_call"] * stages[k]["calls"])
    # The roofline line reports the reconstruction kernel: the step's largest HBM-bound kernel
    # with an algorithmic byte count (the Jacobi stages have none independent of their sweeps).
    rl_name = ROOFLINE_STAGE if ROOFLINE_STAGE in stages else max(
        (k for k in stages if k in sbytes), key=lambda k: stages[k]["ms_per_call"])
    rl = stages[rl_name]
    traffic, earlier = load_traffic(rl_name)
    roofline = {"kernel": rl_name, "bound": "hbm", "achieved": rl["achieved_gbs"],
                "peak": hbm, "unit": "GB/s", "frac": rl["frac_hbm"],
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, burst copy)",
                "traffic": traffic, "dominant_stage": dom}
    if earlier is not None:
        roofline["traffic_earlier_capture"] = earlier

    # Diagnostics of the benchmark state (eq. 12 bytes, factor orthogonality).
    diag = None
    if not args.no_attention:
        diag = run_diagnostics(wl, kv, torch, dev, stream)

    # Decode attention over the compressed cache (the next row after the hot path), timed apart.
    attn = None
    if not args.no_attention:
        attn = time_attention(wl, kv, torch, dev, stream)

    # End-to-end through the C ABI with host buffers.
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(wl, kv, torch, dev, stream, pos, steps_total, e2e_steps, world)

    # The cache policy's decode step on the same histories (folds one more block into each).
    policy = None
    if not args.no_attention:
        policy = time_cache_policy(wl, kv, torch, dev, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(args.cpu_budget)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "folds/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "decode step, 32 layers x {K,V} histories at n~16K "
                                   "(fold b=64 + reorth + reconstruct with RoPE + one 64K-token "
                                   "prompt selection)",
                       "layers": args.layers, "histories_per_gpu": folds_step, "d": D, "r": R,
                       "b": BLK, "n_mean": n_mean, "kv_heads": HEADS, "head_dim": HEAD_DIM,
                       "exact_rows": PROMPT + WINDOW, "rope_theta": THETA,
                       "select_prompt_tokens": SEL_L, "storage": "bf16",
                       "parallelism": f"replicas x{world} (independent histories per GPU)",
                       "l2": "inputs > L2 (~4 GB touched per step), no flush"},
            "reconstructed_rows_per_s": round(rows_per_s, 1),
            "roofline": roofline,
            "stages": stages,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "clocks": clocks,
            "cpu_baseline": cpu,
            "parity_spot_check": check,
            "decode_attention": attn,
            "diagnostics": diag,
            "cache_policy": policy,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def load_traffic(stage: str):
    """(DRAM bytes per launch of `stage`, context) from the committed ncu summary
    (profiles/traffic.json). The bytes are None unless the capture was taken on the current kernel
    ("current": true); an older capture is returned only as context."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        j = json.load(f)
    ent = j.get(stage)
    if ent is None:
        return None, None
    if ent.get("current", False):
        return ent.get("dram_bytes_per_launch"), None
    return None, {"dram_bytes_per_launch": ent.get("dram_bytes_per_launch"),
                  "note": ent.get("note", "")}


def spot_check(wl, torch):
    """Oracle check of the benchmark's own state: the reconstruction of one K history (sampled
    rows, RoPE) against the float64 definition."""
    import numpy as np

    from oracle import fold as of
    from oracle import reconstruct as orec
    h = wl.hists[0]
    k, n, _, st = h.status()
    U = h.U[:n, :k].double().cpu().numpy()
    s = h.sigma[:k].double().cpu().numpy()
    B = h.B[:, :k].double().cpu().numpy()
    pos = h.pos[:n].cpu().numpy()
    rows = np.random.Generator(np.random.PCG64(0)).choice(n, 256, replace=False)
    out = wl.outs[0]
    ref = orec.reconstruct(U[rows], s, B, pos[rows], np.zeros((0, D)), np.zeros(0, dtype=int),
                           int(pos.max()) + 1, HEADS, HEAD_DIM, True, THETA)
    got = out[torch.as_tensor(pos[rows], dtype=torch.long, device=out.device)].double().cpu().numpy()
    err = of.rel_fro(got, ref[pos[rows]])
    return {"history": "layer0.K", "k": k, "n": n, "status_bits": st,
            "recon_rel_fro_sampled": float(err), "tol": 2e-2, "ok": bool(err < 2e-2 and st == 0)}


def run_e2e(wl, kv, torch, dev, stream, pos, first_step, steps, world):
    """Same step through the C ABI, with the step's inputs copied from pinned host memory and the
    step's result (every history's sigma and meta word, and the selection outputs) copied back.
    As a serving loop would, the inputs of step t+1 are copied on a second stream while step t
    computes (two device input buffers, ordered by events); every copy of every step, and the
    result read-back, lie inside the timed region."""
    cnt = len(wl.hists)
    hostF = [[f.cpu().pin_memory() for f in s] for s in wl.F]
    hostK = wl.keys.cpu().pin_memory()
    devF = [[torch.empty_like(f) for f in wl.F[0]] for _ in range(2)]
    devK = [torch.empty_like(wl.keys) for _ in range(2)]
    res_sig = torch.empty(cnt, R, dtype=torch.float32).pin_memory()
    res_meta = torch.empty(cnt, 4, dtype=torch.int64).pin_memory()
    res_cnt = torch.empty(2 + HEADS, dtype=torch.int64).pin_memory()
    res_pk = torch.empty(SEL_L, dtype=torch.int32).pin_memory()
    res_pv = torch.empty(SEL_L, dtype=torch.int32).pin_memory()
    h2d = sum(f.numel() * f.element_size() for f in hostF[0]) + hostK.numel() * hostK.element_size()
    d2h = (res_sig.numel() * 4 + res_meta.numel() * 8 + res_cnt.numel() * 8 + res_pk.numel() * 4
           + res_pv.numel() * 4)
    keys_dev = wl.keys
    copy_stream = torch.cuda.Stream(dev)
    ready = [torch.cuda.Event() for _ in range(2)]   # inputs of the buffer's step are on the device
    free = [torch.cuda.Event() for _ in range(2)]    # the buffer's last step has finished with it

    def copy_in(i):
        b = i % 2
        with torch.cuda.stream(copy_stream):
            if i >= 2:
                copy_stream.wait_event(free[b])
            hf = hostF[(first_step + i) % 4]
            for j in range(cnt):
                devF[b][j].copy_(hf[j], non_blocking=True)
            devK[b].copy_(hostK, non_blocking=True)
            ready[b].record(copy_stream)

    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    copy_stream.wait_event(ev0)
    t0 = time.perf_counter()
    copy_in(0)
    for i in range(steps):
        t = first_step + i
        b = i % 2
        if i + 1 < steps:
            copy_in(i + 1)
        stream.wait_event(ready[b])
        wl.keys = devK[b]
        wl.step(t, *pos[t], F=devF[b])
        free[b].record(stream)
        for j, h in enumerate(wl.hists):
            res_sig[j].copy_(h.sigma, non_blocking=True)
            res_meta[j].copy_(h.meta, non_blocking=True)
        res_cnt.copy_(wl.sel_out["counts"], non_blocking=True)
        res_pk.copy_(wl.sel_out["P_K"], non_blocking=True)
        res_pv.copy_(wl.sel_out["P_V"], non_blocking=True)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - t0
    ms = ev0.elapsed_time(ev1)
    wl.keys = keys_dev
    ok = bool(torch.all(res_meta[:, 3] == 0).item())
    ms = max_over_ranks(ms, dev)
    return {"value": round(world * cnt * steps / (ms / 1e3), 2), "unit": "folds/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms / steps, 4),
            "host_wall_ms_per_step": round(wall * 1e3 / steps, 4), "status_ok": ok,
            "copies": "inputs of step t+1 copied on a second stream during step t"}


# ------------------------------------------------------------------------------------------------
# CPU oracle legs (the baseline the task asks for; never a target).

_KEYS = {}


def _oracle_sample(seed=7):
    """Float64 oracle on one history of the step: fold, reorth and reconstruction at n = 16384,
    plus one prompt selection. Returns the seconds of each part."""
    import numpy as np

    import synth
    from oracle import fold as of
    from oracle import reconstruct as orec
    from oracle import reorth as oreo
    from oracle import select as osel
    g = np.random.Generator(np.random.PCG64(seed))
    n = N_MID
    U = np.linalg.qr(g.standard_normal((n, R)))[0]
    B = np.linalg.qr(g.standard_normal((D, R)))[0]
    s = np.sqrt(n) * np.arange(1, R + 1) ** -1.2
    F = (g.standard_normal((BLK, R)) * np.arange(1, R + 1) ** -1.2) @ B.T + NOISE * g.standard_normal((BLK, D))
    t = {}
    a = time.perf_counter()
    res = of.fold_block(U, s, B, F, R)
    t["fold"] = time.perf_counter() - a
    a = time.perf_counter()
    U2, s2, B2 = oreo.reorth(res.U, res.sigma, res.B)
    t["reorth"] = time.perf_counter() - a
    a = time.perf_counter()
    pos = np.arange(PROMPT, PROMPT + U2.shape[0])
    ex = g.standard_normal((PROMPT + WINDOW, D))
    epos = np.r_[np.arange(PROMPT), np.arange(PROMPT + U2.shape[0], PROMPT + U2.shape[0] + WINDOW)]
    orec.reconstruct(U2, s2, B2, pos, ex, epos, PROMPT + U2.shape[0] + WINDOW, HEADS, HEAD_DIM,
                     True, THETA)
    t["reconstruct"] = time.perf_counter() - a
    if "k" not in _KEYS:
        _KEYS["k"] = synth.outlier_prompt_keys(SEL_L, HEADS, HEAD_DIM, seed=4)[0]
    a = time.perf_counter()
    osel.select_prompt_blocks(_KEYS["k"], 8, 128, 4, 32)
    t["select"] = time.perf_counter() - a
    return t


def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(budget_s: float):
    reps, total, parts = 0, 0.0, None
    while reps == 0 or (total < budget_s and reps < 3):
        t = _oracle_sample(seed=7 + reps)
        parts = t if parts is None else {k: parts[k] + t[k] for k in t}
        total += sum(t.values())
        reps += 1
    parts = {k: v / reps for k, v in parts.items()}
    hist = LAYERS * 2
    step_s = hist * (parts["fold"] + parts["reorth"] + parts["reconstruct"]) + parts["select"]
    return {"value": round(hist / step_s, 4), "unit": "folds/s", "cores": _cpu_threads(),
            "kind": "oracle",
            "sample": (f"{reps} x (1 fold + 1 reorth + 1 reconstruction at n=16384, d=1024, r=256, "
                       f"+ 1 selection of a 65536-token prompt), float64 NumPy; a step = 64 x "
                       f"(fold+reorth+reconstruct) + 1 selection"),
            "seconds_per_part": {k: round(v, 4) for k, v in parts.items()}}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    _oracle_sample(seed=99)  # one untimed pass: imports, BLAS start-up, the prompt keys
    steps_s = []
    for i in range(args.steps):
        t = _oracle_sample(seed=100 + i)
        steps_s.append(LAYERS * 2 * (t["fold"] + t["reorth"] + t["reconstruct"]) + t["select"])
    step = sum(steps_s) / len(steps_s)
    value = LAYERS * 2 / step
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "folds/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(step * 1e3, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "decode step, 32 layers x {K,V} histories at n~16K (fold b=64 + "
                                   "reorth + reconstruct with RoPE + one 64K-token prompt selection)",
                       "d": D, "r": R, "b": BLK, "n": N_MID},
            "cpu_baseline": {"value": round(value, 4), "unit": "folds/s", "cores": _cpu_threads(),
                             "kind": "oracle",
                             "sample": "per step: 1 fold + 1 reorth + 1 reconstruction at n=16384 "
                                       "and 1 selection, extrapolated to 64 histories"},
            "e2e": {"value": round(value, 4), "unit": "folds/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-check", action="store_true")
    ap.add_argument("--no-attention", action="store_true",
                    help="skip the rows timed apart from the step: decode attention over the "
                         "compressed cache, the diagnostics and the cache-policy step")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--clock-log-dir", default=None,
                    help="folder for the nvidia-smi clock samples of the timed region "
                         "(default: the system's temporary folder)")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="model layers (2 histories each); the headline workload is 32")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "b200":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_b200(args)


if __name__ == "__main__":
    main()
