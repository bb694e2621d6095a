#!/usr/bin/env python
"""Benchmark of the iS-KV hot path on B200.

Workload (one GPU): the decode steps of a 32-layer GQA model (8 KV heads x head_dim 128, so
d = 1024) at which every layer's K and V pending queue fills at once -- 64 compressed histories at
n ~ 16384 rows, rank r = 256, fold block b = 64, bf16 factors. One timed step runs every row of the
hot path:

  1. fold (Algorithm 2): one 64-row block into each of the 64 histories (one batched call);
  2. re-orthogonalisation (Section 4.4) of all 64 histories, every 4th step: the pages' cadence of
     one re-orthogonalisation per 256 folded rows;
  3. reconstruction (Algorithm 3 steps 7-8) of all 64 caches -- compressed rows plus 640 exact rows
     (512-token prompt kept exact, 128-row recent window), RoPE theta = 500000 on K;
  4. prompt-block selection (Algorithm 1 steps 2-4) on one layer's 65536-token post-RoPE prompt.

Inputs: every history is built on the device by folding seeded synthetic rows from the start, and
the timed steps fold the rows that follow: per history, G diag(s) H(t)^T + 0.02 N(0, 1) with
s_j = j^-1.2 (keys) or j^-0.6 (values) and a dominant subspace H(t) that turns by 0.05 rad per
1024 rows (the decode-simulation workload), standing in for model traces. n starts so that the
timed steps are centred on n = 16384. Everything a step reads is resident in HBM before timing
starts; a step touches ~4 GB, far more than the 126 MB L2, so no flush is needed.

metric: block folds/s (64 folds per step); the line also reports reconstructed KV rows/s, per-stage
device time with its roofline fraction (HBM for the streaming kernels, the float32 CUDA-core peak
for the Jacobi core SVD), the core's sweep counts, rates at the sweep workload's cadence (one
re-orthogonalisation per 16 folds), and the eq. (14) factor drift of one K and one V history.

--impl reference times the float64 CPU oracle, one history's share of a step per timed step.
--gpus N runs N ranks (one process per GPU, launched through torch.distributed.run when the
caller did not); --dry-run exercises that plumbing on CPU processes without a GPU.
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
DRIFT_RAD_PER_1K = 0.05  # rotation of the rows' dominant subspace per 1024 rows
REORTH_EVERY = 4         # folds per re-orthogonalisation: 256 rows at b = 64, as on the pages
SWEEP_REORTH_EVERY = 16  # the cadence of the sweep workload
SMS, FP32_LANES = 148, 128  # B200: SMs, float32 FMA lanes per SM


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
    """64 histories (32 layers x {K, V}) built on the device from drifting synthetic rows, and
    every per-step input, resident on the device."""

    def __init__(self, kv, torch, dev, warmup: int, timed: int, extra: int, seed: int = 1000,
                 layers: int = LAYERS):
        import synth
        self.kv, self.torch, self.dev = kv, torch, dev
        # n after the fold of step t is n0 + 64 (t + 1); the timed steps are centred on N_MID.
        self.n0 = N_MID - BLK * (warmup + (timed + 1) // 2)
        self.n_cap = self.n0 + BLK * (warmup + timed + extra + 4)
        self.kinds = [kind for _ in range(layers) for kind in ("K", "V")]
        cnt = len(self.kinds)
        self.hists = [kv.LowRankHistory(D, R, self.n_cap, storage=torch.bfloat16, device=dev)
                      for _ in range(cnt)]
        # Workspaces (sized once).
        self.ws_fold = torch.empty(kv.fold_workspace_size(cnt, D, R, BLK) + 256,
                                   dtype=torch.uint8, device=dev)
        self.ws_reorth = torch.empty(kv.reorth_workspace_size(cnt, D, R, self.n_cap) + 256,
                                     dtype=torch.uint8, device=dev)
        self.ws_recon = torch.empty(kv.reconstruct_workspace_size(cnt, D, R) + 256,
                                    dtype=torch.uint8, device=dev)
        self.ws_sel = torch.empty(kv.select_workspace_size(SEL_L, HEADS, 8) + 256,
                                  dtype=torch.uint8, device=dev)
        # Build: fold the first n0 rows of every stream, re-orthogonalising on the step's cadence.
        # The rows of layer 0's K and V histories are kept for the factor-drift measurement.
        self.drift = synth.DriftingRows(cnt, D, [SPEC[k] for k in self.kinds], NOISE, seed, BLK,
                                        angle_per_1k=DRIFT_RAD_PER_1K, device=dev)
        self.kept = [torch.empty(self.n_cap, D, dtype=torch.bfloat16, device=dev)
                     for _ in range(2)]
        self.fpos = torch.arange(PROMPT, PROMPT + self.n_cap + BLK, dtype=torch.int32, device=dev)
        for g in range(self.n0 // BLK):
            F = self.drift.next_blocks().to(torch.bfloat16)
            for i in range(2):
                self.kept[i][g * BLK:(g + 1) * BLK].copy_(F[i])
            self._fold(g, F)
        # Pending blocks of every later step (warm-up, timed, end-to-end) and three more for the
        # cache policy's step (its window rows and its new rows), made before any timing.
        self.F = [self.drift.next_blocks().to(torch.bfloat16)
                  for _ in range(warmup + timed + extra + 3)]
        self.drift = None  # release the generator's d x d matrices
        # Exact rows per history: 512 prompt rows + 128 window rows.
        gen = torch.Generator(device=dev)
        self.exact = []
        for i in range(cnt):
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
        self.side = torch.cuda.Stream(dev)
        self.rec_stream = torch.cuda.Stream(dev)
        self.ev_start = torch.cuda.Event()
        self.ev_sel = torch.cuda.Event()
        self.ev_fold = torch.cuda.Event()
        self.ev_rec = torch.cuda.Event()
        self.rec_pending = False
        torch.cuda.synchronize(dev)

    def _fold(self, g, F, stream=None, factors_ready=None):
        """Fold block g (global block index; rows g*64 .. g*64+63 of every stream) and, when the
        cadence says so, re-orthogonalise. With `factors_ready` the fold's factor-writing stages
        wait for that event (the previous step's reconstruction)."""
        kv = self.kv
        fpos = self.fpos[g * BLK:(g + 1) * BLK]
        kv.fold_block_batched(self.hists, list(F), [fpos] * len(self.hists),
                              ws=self._aligned(self.ws_fold), stream=stream,
                              factors_ready=factors_ready)
        if (g + 1) % REORTH_EVERY == 0:
            kv.reorth(self.hists, ws=self._aligned(self.ws_reorth), stream=stream)

    @staticmethod
    def _aligned(buf):
        off = (-buf.data_ptr()) % 256
        return buf[off:]

    def folded_rows(self, i, steps):
        """Every row history i (0: layer 0's K, 1: its V) has folded after `steps` steps."""
        for t in range(steps):
            g = self.n0 // BLK + t
            self.kept[i][g * BLK:(g + 1) * BLK].copy_(self.F[t][i])
        return self.kept[i][:self.n0 + BLK * steps]

    def n_after(self, t):
        return self.n0 + BLK * (t + 1)

    def reorths_in(self, t0, t1):
        """Re-orthogonalisations run by steps t0 .. t1-1."""
        g0 = self.n0 // BLK
        return sum(1 for t in range(t0, t1) if (g0 + t + 1) % REORTH_EVERY == 0)

    def positions(self, t):
        torch = self.torch
        n = self.n_after(t)
        epos = torch.cat([torch.arange(0, PROMPT, dtype=torch.int32, device=self.dev),
                          torch.arange(PROMPT + n, PROMPT + n + WINDOW, dtype=torch.int32,
                                       device=self.dev)])
        return epos, PROMPT + n + WINDOW

    def step(self, t, epos, n_total, F=None, stream=None):
        """One decode step, pipelined over three streams. The prompt selection reads nothing the
        fold or the reconstruction writes, so it runs beside them. The step's reconstruction runs on
        its own stream after the fold (and reorth), and the next step's fold starts beside it: the
        fold's read-only stages (projection, residual QR, core SVD) overlap the reconstruction,
        and its rotations and write-back wait for it (iskv_fold_block_batched_after). The step
        ends when the fold and the selection have; `drain` waits for the last reconstruction."""
        kv, torch = self.kv, self.torch
        F = F if F is not None else self.F[t]
        main = stream if stream is not None else torch.cuda.current_stream(self.dev)
        self.ev_start.record(main)
        self.side.wait_event(self.ev_start)
        self.sel_out = kv.select_prompt_blocks(self.keys, 8, 128, 4, 32,
                                               ws=self._aligned(self.ws_sel), out=self.sel_out,
                                               stream=self.side)
        self.ev_sel.record(self.side)
        self._fold(self.n0 // BLK + t, F, stream=main,
                   factors_ready=self.ev_rec if self.rec_pending else None)
        self.ev_fold.record(main)
        self.rec_stream.wait_event(self.ev_fold)
        kv.reconstruct_batched(self.hists, self.exact, [epos] * len(self.hists), n_total, HEADS,
                               HEAD_DIM, self.rope, THETA, outs=self.outs,
                               ws=self._aligned(self.ws_recon), stream=self.rec_stream)
        self.ev_rec.record(self.rec_stream)
        self.rec_pending = True
        main.wait_event(self.ev_sel)

    def drain(self, stream=None):
        """Make `stream` wait for the last step's reconstruction."""
        main = stream if stream is not None else self.torch.cuda.current_stream(self.dev)
        if self.rec_pending:
            main.wait_event(self.ev_rec)


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
    each side's exact-row table holds its 512 protected prompt rows and its 128 window rows (the next
    rows of the history's stream; W = 128, b = 64); 63 steps only store the stream's following rows,
    the 64th folds the oldest 64 rows of every table and removes them from the tables. Run last: it
    folds one more block into every history."""
    cnt = len(wl.hists)
    tabs = []
    for i, h in enumerate(wl.hists):
        n = int(h.status()[1])
        t = kv.ExactTable(D, PROMPT + WINDOW + BLK, window=WINDOW, block=BLK, reorth_rows=0,
                          dtype=torch.bfloat16, device=dev)
        t.rows[:PROMPT].copy_(wl.exact[i][:PROMPT])
        t.rows[PROMPT:PROMPT + WINDOW].copy_(torch.cat([wl.F[-3][i], wl.F[-2][i]]))
        win = torch.arange(PROMPT + n, PROMPT + n + WINDOW, dtype=torch.int32, device=dev)
        t.pos[:PROMPT + WINDOW].copy_(torch.cat([torch.arange(PROMPT, dtype=torch.int32,
                                                              device=dev), win]))
        for j in range(WINDOW):
            t.live[j] = PROMPT + n + j
        t.t.n_prot, t.t.n_live, t.t.last, t.t.hist_rows = PROMPT, WINDOW, PROMPT + n + WINDOW - 1, n
        tabs.append(t)
    # The window holds the next 128 rows of each history's stream; the decode rows follow them.
    rows = wl.F[-1].transpose(0, 1).contiguous()
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


def workload_config(layers: int, world: int):
    """The workload's description, shared by both arms' JSON lines."""
    return {"workload": "decode steps, 32 layers x {K,V} histories at n~16K (fold b=64 every step, "
                        "reorth every 4 folds, reconstruct with RoPE + one 64K-token prompt "
                        "selection per step)",
            "layers": layers, "histories_per_gpu": 2 * layers, "d": D, "r": R, "b": BLK,
            "n_center": N_MID, "kv_heads": HEADS, "head_dim": HEAD_DIM,
            "exact_rows": PROMPT + WINDOW, "rope_theta": THETA, "select_prompt_tokens": SEL_L,
            "storage": "bf16", "reorth_every_folds": REORTH_EVERY,
            "inputs": f"rows G diag(s) H(t)^T + {NOISE} N(0,1), s_j = j^-1.2 (K) / j^-0.6 (V), "
                      f"subspace drift {DRIFT_RAD_PER_1K} rad per 1024 rows; histories built by "
                      f"folding the same streams from n = 0",
            "parallelism": f"replicas x{world} (independent histories per GPU)",
            "l2": "inputs > L2 (~4 GB touched per step), no flush"}


def fp32_peak_tflops(sm_mhz):
    """Float32 CUDA-core peak at the sampled SM clock: 148 SMs x 128 FMA lanes x 2 flop."""
    mhz = sm_mhz or 1965.0
    return SMS * FP32_LANES * 2 * mhz * 1e6 / 1e12


def core_roofline(stats, stage, peak_tflops):
    """Achieved float32 rate of the core SVD stage: the flops the kernel executed (counted on the
    device: pair inner products and applied rotations) over its measured time, and for comparison
    the usual estimate of about 7 (k + b)^3 flops per one-sided Jacobi sweep of a (k + b)-column
    core."""
    if not stats["cores"] or stage is None:
        return None
    ms = stage["ms_per_call"] * stage["calls"]
    tflops = stats["flops"] / (ms / 1e3) / 1e12
    return {"cores": stats["cores"], "sweeps_mean": round(stats["sweeps"] / stats["cores"], 3),
            "sweeps_max": stats["max_sweeps"],
            "rotations_per_core": round(stats["rotations"] / stats["cores"], 1),
            "flops_per_core": round(stats["flops"] / stats["cores"], 1),
            "achieved_tflops": round(tflops, 3), "peak_tflops": round(peak_tflops, 2),
            "frac_fp32": round(tflops / peak_tflops, 4),
            "peak_source": "148 SMs x 128 FP32 lanes x 2 flop x median sampled SM clock"}


def factor_drift(torch, X, h):
    """Eq. (14) of the pages' appendix: the relative error of the history's factors against the
    rows it folded, minus that of a fresh rank-r SVD of the same rows (float64, torch on the
    device; a measurement, not part of the path)."""
    k, n, _, _ = h.status()
    Xd = X[:n].double()
    inc = (h.U[:n, :k].double() * h.sigma[:k].double()) @ h.B[:, :k].double().T
    nx = torch.linalg.matrix_norm(Xd)
    e_inc = float(torch.linalg.matrix_norm(Xd - inc) / nx)
    S = torch.linalg.svdvals(Xd)
    e_svd = float(torch.sqrt(torch.sum(S[k:] ** 2)) / nx)
    return {"n": int(n), "k": int(k), "rel_err_incremental": round(e_inc, 6),
            "rel_err_fresh_svd": round(e_svd, 6), "factor_drift": round(e_inc - e_svd, 6)}


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
    t_setup = time.perf_counter()
    wl = Workload(kv, torch, dev, args.warmup, args.steps, e2e_steps, seed=rank_seed(rank),
                  layers=args.layers)
    setup_s = time.perf_counter() - t_setup
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
    kv.core_stats(reset=True)
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
    wl.drain(stream)
    ev1.record(stream)
    barrier()
    clocks = sampler.stop()
    launches = kv.launch_count() - launches0
    kv.stage_timing(False)
    st = kv.stage_times(reset=True)
    cstats = kv.core_stats(reset=True)
    status_ok = all(h.status()[3] == 0 for h in wl.hists)
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    ms_step = ms / args.steps
    folds_step = len(wl.hists)
    n_mean = sum(wl.n_after(t) for t in range(args.warmup, steps_total)) / args.steps
    value = world * folds_step * args.steps / (ms / 1e3)
    rows_step = len(wl.hists) * (PROMPT + n_mean + WINDOW)
    rows_per_s = world * rows_step * args.steps / (ms / 1e3)
    n_reorth = wl.reorths_in(args.warmup, steps_total)

    # Stage rooflines: HBM for the streaming stages, float32 CUDA cores for the core SVDs.
    hbm, tc, peak_kind = peaks()
    fp32 = fp32_peak_tflops(clocks.get("sm_mhz"))
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
    core = {"fold": core_roofline(cstats["fold"], stages.get("fold.core_svd"), fp32),
            "reorth": core_roofline(cstats["reorth"], stages.get("reorth.core_svd"), fp32)}
    dom = max(stages, key=lambda k: stages[k]["ms_per_call"] * stages[k]["calls"])
    traffic, earlier = load_traffic(ROOFLINE_STAGE)
    rl_hbm = {"kernel": ROOFLINE_STAGE, "bound": "hbm",
              "achieved": stages[ROOFLINE_STAGE]["achieved_gbs"], "peak": hbm, "unit": "GB/s",
              "frac": stages[ROOFLINE_STAGE]["frac_hbm"],
              "peak_source": ("MEASURED_PEAKS.json hbm_gbs (burst copy)" if peak_kind == "measured"
                              else "fallback 6650 GB/s (no MEASURED_PEAKS.json)"),
              "traffic": traffic}
    if earlier is not None:
        rl_hbm["traffic_earlier_capture"] = earlier
    rl_rot = None
    if "fold.coord_rotate" in stages:
        rr = stages["fold.coord_rotate"]
        rl_rot = {"kernel": "fold.coord_rotate", "bound": "hbm", "achieved": rr["achieved_gbs"],
                  "peak": hbm, "unit": "GB/s", "frac": rr["frac_hbm"],
                  "traffic": load_traffic("fold.coord_rotate")[0]}
    # The roofline line reports the dominant stage: the fold's core SVD (float32 ALU-bound) when
    # it dominates, else the largest HBM-bound stage.
    if dom in ("fold.core_svd", "reorth.core_svd") and core[dom.split(".")[0]] is not None:
        c = core[dom.split(".")[0]]
        roofline = {"kernel": f"{dom} (k_core)", "bound": "alu", "achieved": c["achieved_tflops"],
                    "peak": c["peak_tflops"], "unit": "TFLOP/s", "frac": c["frac_fp32"],
                    "peak_source": c["peak_source"], "traffic": load_traffic(dom)[0],
                    "dominant_stage": dom}
    else:
        roofline = dict(rl_hbm, dominant_stage=dom)

    # Rates at the sweep workload's cadence (one re-orthogonalisation per 16 folds), from the
    # measured stage times of this run.
    fold_ms = sum(v["ms_per_call"] * v["calls"] for k, v in stages.items()
                  if k.startswith("fold.")) / args.steps
    reorth_ms = (sum(v["ms_per_call"] * v["calls"] for k, v in stages.items()
                     if k.startswith("reorth.")) / max(n_reorth, 1))
    recon_ms = sum(v["ms_per_call"] for k, v in stages.items() if k.startswith("reconstruct."))
    cadence = {
        "fold_ms_per_call": round(fold_ms, 4), "reorth_ms_per_call": round(reorth_ms, 4),
        "reconstruct_ms_per_call": round(recon_ms, 4),
        "folds_per_s_fold_only": round(folds_step / (fold_ms / 1e3), 1),
        f"folds_per_s_reorth_every_{REORTH_EVERY}": round(
            folds_step / ((fold_ms + reorth_ms / REORTH_EVERY) / 1e3), 1),
        f"folds_per_s_reorth_every_{SWEEP_REORTH_EVERY}": round(
            folds_step / ((fold_ms + reorth_ms / SWEEP_REORTH_EVERY) / 1e3), 1),
        "reorths_per_s": round(folds_step / (reorth_ms / 1e3), 1),
        "note": "fold-only and cadence rates are sums of this run's stage times (CUDA events)"}

    # Eq. (14) factor drift of layer 0's K and V histories against the rows they folded.
    drift = None
    if not args.no_check:
        drift = {kind: factor_drift(torch, wl.folded_rows(i, steps_total), wl.hists[i])
                 for i, kind in enumerate(("K", "V"))}
        drift["pages_table5_fp16_factors"] = {"K": [0.0016, 0.0071], "V": [0.0160, 0.0207]}

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
            "config": dict(workload_config(args.layers, world), n_mean=n_mean),
            "reconstructed_rows_per_s": round(rows_per_s, 1),
            "roofline": roofline,
            "roofline_kernels": {"reconstruct.compressed": rl_hbm, "fold.coord_rotate": rl_rot},
            "core_svd": core,
            "stages": stages,
            "cadence_rates": cadence,
            "factor_drift_eq14": drift,
            "status_ok": status_ok,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "clocks": clocks,
            "cpu_baseline": cpu,
            "decode_attention": attn,
            "diagnostics": diag,
            "cache_policy": policy,
            "setup_s": round(setup_s, 2),
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


def run_e2e(wl, kv, torch, dev, stream, pos, first_step, steps, world):
    """Same steps through the C ABI, with each step's inputs (its 64 pending blocks and the prompt
    keys) copied from pinned host memory and the step's result (every history's sigma and meta
    word, and the selection outputs) copied back. As a serving loop would, the inputs of step t+1
    are copied on a second stream while step t computes (two device input buffers, ordered by
    events); every copy of every step, and the result read-back, lie inside the timed region."""
    cnt = len(wl.hists)
    hostF = [wl.F[first_step + i].cpu().pin_memory() for i in range(steps)]
    hostK = wl.keys.cpu().pin_memory()
    devF = [torch.empty_like(wl.F[0]) for _ in range(2)]
    devK = [torch.empty_like(wl.keys) for _ in range(2)]
    res_sig = torch.empty(cnt, R, dtype=torch.float32).pin_memory()
    res_meta = torch.empty(cnt, 4, dtype=torch.int64).pin_memory()
    # The histories' sigma and meta words are gathered on the device first, so each step reads
    # them back with two copies rather than two per history.
    dev_sig = torch.empty(cnt, R, dtype=torch.float32, device=dev)
    dev_meta = torch.empty(cnt, 4, dtype=torch.int64, device=dev)
    res_cnt = torch.empty(2 + HEADS, dtype=torch.int64).pin_memory()
    res_pk = torch.empty(SEL_L, dtype=torch.int32).pin_memory()
    res_pv = torch.empty(SEL_L, dtype=torch.int32).pin_memory()
    h2d = hostF[0].numel() * hostF[0].element_size() + hostK.numel() * hostK.element_size()
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
            devF[b].copy_(hostF[i], non_blocking=True)
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
        torch.stack([h.sigma for h in wl.hists], out=dev_sig)
        torch.stack([h.meta for h in wl.hists], out=dev_meta)
        res_sig.copy_(dev_sig, non_blocking=True)
        res_meta.copy_(dev_meta, non_blocking=True)
        res_cnt.copy_(wl.sel_out["counts"], non_blocking=True)
        res_pk.copy_(wl.sel_out["P_K"], non_blocking=True)
        res_pv.copy_(wl.sel_out["P_V"], non_blocking=True)
    wl.drain(stream)
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
# CPU oracle legs: the float64 oracle timed on the host cores, a reported baseline (never a target).

_KEYS = {}
SEL_SLICE = SEL_L // (2 * LAYERS)  # one history's share of the step's prompt selection


def _oracle_inputs(seed):
    import numpy as np
    g = np.random.Generator(np.random.PCG64(seed))
    n = N_MID
    U = np.linalg.qr(g.standard_normal((n, R)))[0]
    B = np.linalg.qr(g.standard_normal((D, R)))[0]
    s = np.sqrt(n) * np.arange(1, R + 1) ** -1.2
    F = ((g.standard_normal((BLK, R)) * np.arange(1, R + 1) ** -1.2) @ B.T
         + NOISE * g.standard_normal((BLK, D)))
    ex = g.standard_normal((PROMPT + WINDOW, D))
    return U, s, B, F, ex


def _oracle_sample(seed, reorth: bool):
    """One history's share of a step, on the float64 oracle: a fold at n = 16384, d = 1024,
    r = 256, b = 64, a re-orthogonalisation when the cadence has one, the reconstruction of the
    history's cache with RoPE, and the selection of a 1024-token prompt slice (1/64 of the step's
    65536-token selection). Returns the seconds of each part (inputs are drawn untimed)."""
    import synth
    from oracle import fold as of
    from oracle import reconstruct as orec
    from oracle import reorth as oreo
    from oracle import select as osel
    import numpy as np
    U, s, B, F, ex = _oracle_inputs(seed)
    if "k" not in _KEYS:
        _KEYS["k"] = synth.outlier_prompt_keys(SEL_SLICE, HEADS, HEAD_DIM, seed=4)[0]
    t = {}
    a = time.perf_counter()
    res = of.fold_block(U, s, B, F, R)
    t["fold"] = time.perf_counter() - a
    U2, s2, B2 = res.U, res.sigma, res.B
    t["reorth"] = 0.0
    if reorth:
        a = time.perf_counter()
        U2, s2, B2 = oreo.reorth(U2, s2, B2)
        t["reorth"] = time.perf_counter() - a
    n = U2.shape[0]
    a = time.perf_counter()
    pos = np.arange(PROMPT, PROMPT + n)
    epos = np.r_[np.arange(PROMPT), np.arange(PROMPT + n, PROMPT + n + WINDOW)]
    orec.reconstruct(U2, s2, B2, pos, ex, epos, PROMPT + n + WINDOW, HEADS, HEAD_DIM, True, THETA)
    t["reconstruct"] = time.perf_counter() - a
    a = time.perf_counter()
    osel.select_prompt_blocks(_KEYS["k"], 8, 128, 4, 32)
    t["select_slice"] = time.perf_counter() - a
    return t


def _host_cores():
    """Cores this process may run on, and the BLAS thread count."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    blas = None
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 1) for i in threadpool_info()), default=None)
    except Exception:
        pass
    return int(cores or 1), blas


ORACLE_SAMPLE = ("each step = one history's share of a B200 step on the float64 NumPy oracle: 1 "
                 "fold at n=16384, d=1024, r=256, b=64 + 1 reorth on every 4th step + 1 "
                 "reconstruction of 640 exact + ~16K compressed rows with RoPE + the selection of a "
                 "1024-token prompt slice (1/64 of the 65536-token selection)")


def cpu_baseline(budget_s: float):
    """The oracle timed on this host's cores on a bounded sample of the workload (about
    `budget_s` seconds of CPU work); folds/s = samples / their total time."""
    _oracle_sample(99, False)  # untimed: imports, BLAS start-up, the prompt keys
    reps, total, parts = 0, 0.0, {}
    while reps < REORTH_EVERY or (total < budget_s and reps < 4 * REORTH_EVERY):
        t = _oracle_sample(7 + reps, (reps + 1) % REORTH_EVERY == 0)
        for k, v in t.items():
            parts[k] = parts.get(k, 0.0) + v
        total += sum(t.values())
        reps += 1
    cores, blas = _host_cores()
    return {"value": round(reps / total, 4), "unit": "folds/s", "cores": cores,
            "blas_threads": blas, "kind": "oracle",
            "sample": f"{reps} steps, {round(total, 2)} s; " + ORACLE_SAMPLE,
            "seconds_per_part": {k: round(v / reps, 4) for k, v in parts.items()}}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for i in range(args.warmup):   # untimed: imports, BLAS start-up, the prompt keys
        _oracle_sample(99 + i, False)
    steps_s = []
    for i in range(args.steps):
        t = _oracle_sample(100 + i, (i + 1) % REORTH_EVERY == 0)
        steps_s.append(sum(t.values()))
    step = sum(steps_s) / len(steps_s)
    value = 1.0 / step
    cores, blas = _host_cores()
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "folds/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(step * 1e3, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.layers, world),
            "cpu_baseline": {"value": round(value, 4), "unit": "folds/s", "cores": cores,
                             "blas_threads": blas, "kind": "oracle",
                             "sample": ORACLE_SAMPLE, "extrapolated": False},
            "e2e": {"value": round(value, 4), "unit": "folds/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# ------------------------------------------------------------------------------------------------
# Launch: N ranks (torch.distributed.run) and a CPU dry run of the multi-rank plumbing.

def launch_ranks(argv, n):
    """Re-run this script as `n` ranks through torch.distributed.run on this node."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def run_dry(args):
    """The multi-rank plumbing without a GPU: gloo process group, a barrier-bracketed timed
    region of host work per rank, the max over ranks, and rank 0's JSON line."""
    import datetime

    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    for _ in range(args.warmup):
        torch.ones(64, 64) @ torch.ones(64, 64)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        torch.ones(64, 64) @ torch.ones(64, 64)
    ms = (time.perf_counter() - t0) * 1e3
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        dist.barrier()
    if rank == 0:
        print(json.dumps({"metric": METRIC, "dry_run": True, "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": round(ms / max(args.steps, 1), 6),
                          "ranks_timed": world}))
    if world > 1:
        dist.destroy_process_group()


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--dry-run", action="store_true",
                    help="exercise the multi-rank launch and timing plumbing on CPU (no GPU)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-check", action="store_true",
                    help="skip the factor-drift measurement")
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
    if args.warmup < 3 and args.impl == "b200" and not args.dry_run:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    world = int(os.environ.get("WORLD_SIZE", "0"))
    if args.gpus > 1 and world == 0:
        return launch_ranks(argv, args.gpus)
    if world and world != args.gpus:
        print(f"warning: --gpus {args.gpus} but {world} ranks were launched; reporting {world}",
              file=sys.stderr)
    if args.dry_run:
        run_dry(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_b200(args)
    return 0


if __name__ == "__main__":
    sys.exit(main())
