#!/usr/bin/env python
"""Benchmark of the CSA / HCA forward-pass hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input:
  * decode workloads: the compressed cache (entries, indexer keys, window) is
    resident in HBM; a step scores every visible entry of every sequence
    (indexer), selects the top k, and attends over the selected entries plus
    the window (csa_index_topk + csa_attend; hca_attend for HCA);
  * prefill workloads: csa_compress of the whole sequence, then index/top-k
    and attention for every token.
One process per GPU (torchrun for N > 1); each rank runs its own batch (weak
scaling, no data-path collective).  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_sparse_09_b200 import binding as bd  # noqa: E402
from long_context_sparse_09_b200 import dist as D  # noqa: E402
from long_context_sparse_09_b200 import synth  # noqa: E402
from long_context_sparse_09_b200.configs import DEFAULT_BENCH, WORKLOADS  # noqa: E402

METRIC = "CSA decode query-tok/s @1M ctx & prefill tok/s; % of HBM / tensor roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

L2_BYTES = 126 * 1000 * 1000  # B200 L2 capacity

# ncu DRAM traffic per launch of the dominant kernel, with the hash of the
# source file it was measured on (the value is dropped once the file changes).
NCU_TRAFFIC = {
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum on
    # pro_csa_decode_1m with 2 sequences (134.30 MB read + 3.38 MB written),
    # scaled by the units of a full launch (4 sequences)
    ("index_scores", "pro_csa_decode_1m"): (275.37e6, "266b1e616614"),
    # ncu --set full on flash_csa_prefill_32k cut to 8,192 tokens (565.12 MB
    # read + 484.08 MB written: the queries read and the outputs written once;
    # the gathered rows come from L2), scaled by the queries of a full launch
    # (32,768: traffic grows in proportion)
    ("attend", "flash_csa_prefill_32k"): (4196.78e6, "b8cd68c0a9a9"),
}


# ------------------------------------------------------------------ utils --
def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def _src_hash(fname):
    with open(os.path.join(ROOT, "long_context_sparse_09_b200", "csrc", fname), "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


class ClockSampler:
    """nvidia-smi clocks / throttle reasons of this GPU, sampled every 50 ms."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.lines = []
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, v in zip(self.NAMES, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    world, rank, local = D.world()
    torch.cuda.set_device(local)
    D.init("nccl")
    return world, rank, local


def _barrier(world):
    D.barrier()


def _max_over_ranks(x, world):
    return D.max_over_ranks(x, device="cuda")


# --------------------------------------------------------------- workloads --
class DecodeStep:
    """Resident cache + one query per sequence; a step = index/top-k + attend.
    With fp4, the indexer keys are held in MXFP4 (quantised once from the
    same bf16 keys; the cache is resident state) and the step scores them
    with csa_index_topk_mxfp4."""

    def __init__(self, wl, device, seed_offset=0, fp4=False):
        self.wl = wl
        self.fp4 = fp4
        self.p = bd.params_for(wl)
        inp = synth.decode_inputs(wl.with_(seed=wl.seed + D.seed_offset(seed_offset)),
                                  device=device)
        self.inp = inp
        B, N = wl.B, inp["N"]
        self.N = N
        if fp4:
            self.kcodes, self.kscales = bd.mxfp4_quantize(inp["kI"])
        self.out = torch.empty(B, wl.n_h, wl.c, dtype=torch.bfloat16, device=device)
        if wl.variant == "csa":
            self.idx = torch.empty(B, wl.topk, dtype=torch.int32, device=device)
            self.ws_i = torch.empty(max(bd.index_topk_workspace_bytes(self.p, B, 1, N), 1),
                                    dtype=torch.uint8, device=device)
        self.ws_a = torch.empty(max(bd.attend_workspace_bytes(self.p, B, 1, N), 1),
                                dtype=torch.uint8, device=device)

    def run(self, q=None, qI=None, w=None, q_pos=None, out=None):
        i, wl = self.inp, self.wl
        q = i["q"] if q is None else q
        out = self.out if out is None else out
        q_pos = i["q_pos"] if q_pos is None else q_pos
        if wl.variant == "csa":
            if self.fp4:
                bd.csa_index_topk_mxfp4(self.p, q_pos, i["qI"] if qI is None else qI,
                                        i["w"] if w is None else w, self.kcodes, self.kscales,
                                        self.idx, workspace=self.ws_i)
            else:
                bd.csa_index_topk(self.p, q_pos, i["qI"] if qI is None else qI,
                                  i["w"] if w is None else w, i["kI"], self.idx,
                                  workspace=self.ws_i)
            bd.csa_attend(self.p, q_pos, q, self.idx, i["ckv"], i["ckv_scale"], i["win"],
                          i["win_scale"], i["win_pos0"], i["sink"], out,
                          workspace=self.ws_a)
        else:
            bd.hca_attend(self.p, q_pos, q, i["ckv"], i["ckv_scale"], i["win"],
                          i["win_scale"], i["win_pos0"], i["sink"], out,
                          workspace=self.ws_a)

    # per-step host<->device traffic of the end-to-end leg
    def step_inputs(self):
        i = self.inp
        names = ["q", "q_pos"] + (["qI", "w"] if self.wl.variant == "csa" else [])
        return {k: i[k] for k in names}

    def units(self):
        return self.wl.B  # queries per step

    def time_append(self, steps, stream):
        """Device time of the decode-time compressor for the step's tokens
        (csa_decode_append / hca_decode_append at the workload's d; its own
        small caches; every token closes a block, the costliest case).  One
        graph holds one call per copy of the packed weights, the copies
        together twice the L2, so every call streams its weights from HBM
        and the graph launch is spread over many calls.  Returns (ms per
        call, weight bytes per call, {kernel kind: ms per call})."""
        wl, dev = self.wl, self.out.device
        B, d = wl.B, wl.d
        W = synth.weights(wl.with_(seed=wl.seed + 7), device=dev)
        packed0 = bd.csa_pack_weights(self.p, W)
        del W
        ncols = (4 * wl.c + 4 * wl.c_I) if wl.variant == "csa" else 2 * wl.c
        wbytes = ncols * d * 2
        ncopy = max(2, min(32, -(-2 * L2_BYTES // wbytes)))
        packs = [packed0] + [packed0.clone() for _ in range(ncopy - 1)]
        H = torch.randn(B, d, device=dev).to(torch.bfloat16)
        t = torch.full((B,), wl.m - 1, dtype=torch.int32, device=dev)
        tail = torch.zeros(bd.decode_tail_bytes(self.p, B, d) // 4, dtype=torch.float32,
                           device=dev)
        rb = synth.kv_record_bytes(wl)
        ckv = torch.empty(B, 1, rb, dtype=torch.uint8, device=dev)
        win = torch.empty(B, 1, rb, dtype=torch.uint8, device=dev)
        fp8 = wl.kv == "fp8mix"
        ckv_s = torch.empty(B, 1, device=dev) if fp8 else None
        win_s = torch.empty(B, 1, device=dev) if fp8 else None
        wp0 = torch.full((B,), wl.m - 1, dtype=torch.int32, device=dev)
        kI = torch.empty(B, 1, wl.c_I, dtype=torch.bfloat16, device=dev) if wl.variant == "csa" else None

        def call(packed):
            if wl.variant == "csa":
                bd.csa_decode_append(self.p, H, t, packed, tail, ckv, ckv_s, kI, win, win_s, wp0)
            else:
                bd.hca_decode_append(self.p, H, t, packed, tail, ckv, ckv_s, win, win_s, wp0)

        for pk in packs:
            call(pk)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for pk in packs:
                call(pk)
        for _ in range(3):
            g.replay()
        reps = max(1, steps // ncopy)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / (reps * ncopy)
        # per kernel: the same calls in a graph with the library's event pairs
        # (an eager pass first fills the event pool, so capture creates none)
        bd.profile_collect()
        bd.profile_enable(True)
        for pk in packs:
            call(pk)
        torch.cuda.synchronize()
        bd.profile_collect()
        gp = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gp):
            for pk in packs:
                call(pk)
        bd.profile_enable(False)
        gp.replay()
        torch.cuda.synchronize()
        split = {k: round(v[0] / ncopy, 5) for k, v in bd.profile_collect().items() if v[1]}
        assert bd.device_status() == 0, "device error word set by the decode append"
        del g, gp, packs
        return ms, wbytes, split

    def recall_vs_bf16(self):
        """Per query, the fraction of the bf16 indexer's selection that this
        step's MXFP4 selection also makes (KV recall, plain set arithmetic)."""
        i, wl = self.inp, self.wl
        self.run()
        got = self.idx.cpu().numpy()
        ref = torch.empty_like(self.idx)
        bd.csa_index_topk(self.p, i["q_pos"], i["qI"], i["w"], i["kI"], ref, workspace=self.ws_i)
        ref = ref.cpu().numpy()
        out = []
        for a, b in zip(got, ref):
            sb = set(int(x) for x in b if x >= 0)
            out.append(len(sb & set(int(x) for x in a if x >= 0)) / max(len(sb), 1))
        return out

    def time_query_proj(self, steps, stream):
        """Device time of csa_query_proj for the step's tokens at the
        workload's d, d_c and head shapes (random bf16 weights N(0, 1/fan_in);
        graph replays of one call per copy of the packed weights, the copies
        together at least twice the L2, so every call streams its weights from
        HBM).  Returns (ms per call, packed weight bytes)."""
        wl, dev = self.wl, self.out.device
        B, d, d_c = wl.B, wl.d, wl.d_c
        gen = torch.Generator(device=dev).manual_seed(wl.seed + 13)
        rnd = lambda *sh: (torch.randn(*sh, device=dev, generator=gen) / sh[0] ** 0.5).to(
            torch.bfloat16)
        packed0 = bd.query_proj_pack(self.p, rnd(d, d_c), rnd(d, wl.n_hI),
                                     rnd(d_c, wl.n_h * wl.c), rnd(d_c, wl.n_hI * wl.c_I))
        nbytes = packed0.numel()
        ncopy = max(2, min(16, -(-2 * L2_BYTES // nbytes)))
        packs = [packed0] + [packed0.clone() for _ in range(ncopy - 1)]
        H = torch.randn(B, d, device=dev, generator=gen).to(torch.bfloat16)
        pos = self.inp["q_pos"]
        cQ = torch.empty(B, d_c, dtype=torch.bfloat16, device=dev)
        q = torch.empty(B, wl.n_h, wl.c, dtype=torch.bfloat16, device=dev)
        qI = torch.empty(B, wl.n_hI, wl.c_I, dtype=torch.bfloat16, device=dev)
        w = torch.empty(B, wl.n_hI, device=dev)
        ws = torch.empty(bd.query_proj_workspace_bytes(self.p, B, d, d_c), dtype=torch.uint8,
                         device=dev)

        def call(pk):
            bd.csa_query_proj(self.p, H, pos, pk, d_c, cQ, q, qI, w, workspace=ws)

        for pk in packs:
            call(pk)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for pk in packs:
                call(pk)
        for _ in range(3):
            g.replay()
        reps = max(1, steps // ncopy)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        assert bd.device_status() == 0, "device error word set by the query projection"
        del g, packs
        return e0.elapsed_time(e1) / (reps * ncopy), nbytes

    def time_out_proj(self, steps, stream):
        """Device time of csa_out_proj on the step's attention output (the
        grouped output projection of the workload's g and d_g; graph replays,
        4 calls per graph; weights larger than the L2, streamed from HBM
        each call).  Returns (ms per call, packed weight bytes)."""
        wl, dev = self.wl, self.out.device
        g, d_g, d = wl.g_out, wl.d_g, wl.d
        Kg = wl.c * wl.n_h // g
        gen = torch.Generator(device=dev).manual_seed(wl.seed + 11)
        WG = (torch.randn(g, Kg, d_g, device=dev, generator=gen) / Kg ** 0.5).to(torch.bfloat16)
        WO = (torch.randn(g * d_g, d, device=dev, generator=gen) / (g * d_g) ** 0.5).to(
            torch.bfloat16)
        packed = bd.out_proj_pack(WG, WO)
        del WG, WO
        O = self.out.view(self.out.shape[0], wl.n_h, wl.c)
        res = torch.empty(O.shape[0], d, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(bd.out_proj_workspace_bytes(O.shape[0], wl.n_h, wl.c, g, d_g, d),
                         dtype=torch.uint8, device=dev)
        per_graph = 4
        for _ in range(2):
            bd.csa_out_proj(O, packed, g, d_g, res, workspace=ws)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for _ in range(per_graph):
                bd.csa_out_proj(O, packed, g, d_g, res, workspace=ws)
        gr.replay()
        reps = max(1, steps // per_graph)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            gr.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        assert bd.device_status() == 0, "device error word set by the output projection"
        nbytes = packed.numel()
        del gr, packed
        return e0.elapsed_time(e1) / (reps * per_graph), nbytes

    def step_work(self):
        """("hbm", algorithmic bytes of one step): every cache byte the step
        must read once (indexer keys, the selected entries, the window rows;
        all visible entries for HCA) plus the queries and the outputs."""
        wl, B, N = self.wl, self.wl.B, self.N
        row = synth.kv_record_bytes(wl) + (4 if wl.kv == "fp8mix" else 0)
        qo = 2 * wl.n_h * wl.c * 2 + 4
        key_row = (wl.c_I // 2 + wl.c_I // 32) if self.fp4 else wl.c_I * 2
        if wl.variant == "csa":
            per_q = (N * key_row + wl.n_hI * (wl.c_I * 2 + 4) + wl.topk * row
                     + wl.n_win * row + qo)
        else:
            per_q = (N + wl.n_win) * row + qo
        return "hbm", B * per_q

    def dominant(self):
        """(kernel kind, algorithmic bytes per launch, source file)."""
        wl, B, N = self.wl, self.wl.B, self.N
        if wl.variant == "csa":
            key_row = (wl.c_I // 2 + wl.c_I // 32) if self.fp4 else wl.c_I * 2
            nbytes = B * N * key_row + B * wl.n_hI * (wl.c_I * 2 + 4) + B * 4
            return "index_scores", nbytes, "index_fp4.cu" if self.fp4 else "index_tc.cu", "hbm"
        rb = synth.kv_record_bytes(wl)
        nbytes = B * (N + wl.n_win) * rb + 2 * B * wl.n_h * wl.c * 2
        return "attend", nbytes, "attend_tc.cu", "hbm"

    def cpu_baseline(self, max_queries=None):
        """Oracle (as it stands) on the queries of one step; returns
        (queries, seconds, sample description)."""
        import numpy as np
        import oracle
        from oracle import pipeline as P
        wl, i = self.wl, self.inp
        nq = wl.B if max_queries is None else min(wl.B, max_queries)
        host = getattr(self, "_cpu_host", {})  # host copies, made once
        self._cpu_host = host
        for b in range(nq):
            if b in host:
                continue
            h = {"q": i["q"][b:b + 1].double().cpu().numpy(),
                 "pos": i["q_pos"][b:b + 1].cpu().numpy(),
                 "win": P.cache_values(i["win"][b].cpu(), None if i["win_scale"] is None
                                       else i["win_scale"][b].cpu(), wl.kv, wl.c, wl.rope_dims),
                 "wp0": int(i["win_pos0"][b])}
            if wl.variant == "csa":
                h["qI"] = i["qI"][b:b + 1].double().cpu().numpy()
                h["w"] = i["w"][b:b + 1].double().cpu().numpy()
                h["kI"] = i["kI"][b].double().cpu().numpy()
            else:
                h["kv"] = P.cache_values(i["ckv"][b].cpu(), None, wl.kv, wl.c, wl.rope_dims)
            host[b] = h
        sink = i["sink"].double().cpu().numpy()
        t_total = 0.0
        for b in range(nq):
            h = host[b]
            t0 = time.perf_counter()
            if wl.variant == "csa":
                scores = oracle.index_scores(h["pos"], wl.m, h["qI"], h["w"], h["kI"])
                nv = np.array([oracle.nvis(int(h["pos"][0]), wl.m, self.N)], np.int32)
                idx, _ = oracle.topk(scores, nv, wl.topk)
                t_total += time.perf_counter() - t0
                # gather the selected rows (outside the timed part: a format
                # conversion, not the oracle's arithmetic)
                sel = idx[0][idx[0] >= 0]
                rows = P.cache_values(i["ckv"][b][torch.from_numpy(sel).long().to(i["ckv"].device)].cpu(),
                                      None if i["ckv_scale"] is None else
                                      i["ckv_scale"][b][torch.from_numpy(sel).long().to(i["ckv"].device)].cpu(),
                                      wl.kv, wl.c, wl.rope_dims)
                t0 = time.perf_counter()
                # entries renumbered 0..k-1, all visible at the query position
                oracle.attend(h["pos"], h["q"], np.arange(len(sel), dtype=np.int32)[None, :],
                              wl.m, rows, wl.n_win, h["win"], h["wp0"], sink, wl.rope_dims,
                              wl.rope_base, wl.softmax_scale)
            else:
                P.attend_wl(wl, h["pos"], h["q"], None, h["kv"], h["win"], h["wp0"], sink)
            t_total += time.perf_counter() - t0
        return nq, t_total, f"{nq} of the {wl.B} queries of one step (full context each)"


class PrefillStep:
    """One sequence of T tokens: compress (entries, indexer keys, window rows),
    then index/top-k and attention for every token."""

    def __init__(self, wl, device, seed_offset=0):
        self.wl = wl
        self.p = bd.params_for(wl)
        wl_s = wl.with_(seed=wl.seed + seed_offset)
        self.W = synth.weights(wl_s, device=device)
        self.inp = synth.prefill_inputs(wl_s, device=device)
        self.packed = bd.csa_pack_weights(self.p, self.W)
        B, T = wl.B, wl.T
        nE = T // wl.m
        self.nE = nE
        kvdt = torch.bfloat16 if wl.kv == "bf16" else torch.float32
        self.ckv = torch.empty(B, nE, wl.c, dtype=kvdt, device=device)
        self.win = torch.empty(B, T, wl.c, dtype=kvdt, device=device)
        self.kI = torch.empty(B, nE, wl.c_I, dtype=kvdt, device=device)
        self.idx = torch.empty(B * T, wl.topk, dtype=torch.int32, device=device)
        self.out = torch.empty(B * T, wl.n_h, wl.c, dtype=kvdt, device=device)
        self.win_pos0 = torch.zeros(B, dtype=torch.int32, device=device)
        self.ws_c = torch.empty(bd.compress_workspace_bytes(self.p, B, T, wl.d), dtype=torch.uint8,
                                device=device)
        self.ws_i = torch.empty(bd.index_topk_workspace_bytes(self.p, B, T, nE), dtype=torch.uint8,
                                device=device)
        self.ws_a = torch.empty(max(bd.attend_workspace_bytes(self.p, B, T, nE), 1),
                                dtype=torch.uint8, device=device)

    def run(self, H=None, q=None, qI=None, w=None, q_pos=None, out=None):
        i = self.inp
        H = i["H"] if H is None else H
        out = self.out if out is None else out
        q_pos = i["q_pos"] if q_pos is None else q_pos
        bd.csa_compress(self.p, H, self.packed, self.ckv, None, self.kI, self.win, None,
                        workspace=self.ws_c)
        bd.csa_index_topk(self.p, q_pos, i["qI"] if qI is None else qI,
                          i["w"] if w is None else w, self.kI, self.idx, workspace=self.ws_i)
        bd.csa_attend(self.p, q_pos, i["q"] if q is None else q, self.idx, self.ckv, None,
                      self.win, None, self.win_pos0, i["sink"], out, workspace=self.ws_a)

    def step_inputs(self):
        i = self.inp
        return {k: i[k] for k in ("H", "q", "qI", "w", "q_pos")}

    def cpu_baseline(self, max_queries=None, n_tok=1024, n_q=32):
        """Oracle (as it stands) on a bounded sample of the step: compression
        of the first n_tok tokens, and index / top-k / attention for n_q
        queries spread over the sequence (full-length synthetic caches);
        tokens/s is extrapolated from the time per token of the two parts.
        Returns (tokens, seconds, sample description)."""
        import numpy as np
        from oracle import pipeline as P
        wl, i = self.wl, self.inp
        T, nE = wl.T, self.nE
        W = {k: v.cpu() for k, v in self.W.items()}
        H = i["H"][0, :n_tok].cpu()
        t0 = time.perf_counter()
        P.compress_seq(wl, W, H)
        s_comp = time.perf_counter() - t0
        t_comp = s_comp / n_tok
        st = synth._Streams(wl.seed + 99, "cpu")
        kv = P.cache_values(*synth.cache_rows(wl, st, "bkv", (), nE), wl.kv, wl.c, wl.rope_dims)
        win = P.cache_values(*synth.cache_rows(wl, st, "bwin", (), T), wl.kv, wl.c, wl.rope_dims)
        kI = st.normal("bkI", (nE, wl.c_I), dtype=torch.float32).double().numpy()
        sel = np.linspace(0, T - 1, n_q).astype(np.int64)
        t0s = i["q_pos"][sel].cpu().numpy()
        qI = i["qI"][sel].double().cpu().numpy()
        w = i["w"][sel].double().cpu().numpy()
        q = i["q"][sel].double().cpu().numpy()
        sink = i["sink"].double().cpu().numpy()
        t0 = time.perf_counter()
        idx, _, _, _ = P.select(wl, t0s, qI, w, kI)
        P.attend_wl(wl, t0s, q, idx, kv, win, 0, sink)
        s_query = time.perf_counter() - t0
        t_query = s_query / n_q
        per_token = t_comp + t_query
        measured = s_comp + s_query
        # (tokens' worth of work measured, seconds measured): their ratio is
        # the extrapolated rate 1 / (t_comp + t_query)
        return measured / per_token, measured, (
            f"compression of {n_tok} tokens and index/top-k/attention of {n_q} queries spread "
            f"over {T}; tokens/s extrapolated from the time per token of the two parts")

    def units(self):
        return self.wl.B * self.wl.T  # tokens per step

    def flops(self):
        """Algorithmic FLOPs of one step (compress GEMM + indexer + attention)."""
        wl, T, m = self.wl, self.wl.T, self.wl.m
        ncols = 4 * wl.c + 4 * wl.c_I
        comp = 2.0 * T * wl.d * ncols
        pairs = sum(min(self.nE, (t + 1) // m) for t in range(T))
        index = 2.0 * pairs * wl.n_hI * wl.c_I
        keys = sum(min(wl.topk, min(self.nE, (t + 1) // m)) + min(wl.n_win, t + 1) for t in range(T))
        attn = 4.0 * keys * wl.n_h * wl.c
        return comp, index, attn

    def step_work(self):
        """("tensor", algorithmic FLOPs of one step)."""
        return "tensor", sum(self.flops())

    def dominant(self):
        comp, index, attn = self.flops()
        return "attend", attn, "attend_tc.cu", "tensor"


# --------------------------------------------------------------- measure --
# workloads measured after the default one, as sub-objects of its line
OTHER_WORKLOADS = ("flash_csa_prefill_32k", "hca_decode_1m", "flash_csa_decode_64k",
                   "pro_csa_decode_1m+mxfp4")


def time_step(step, steps, warmup, world, stream):
    """Device time of one step.  The timed step is a CUDA-graph replay of
    the library calls (launch overhead out of the way); `steps` replays sit
    between CUDA events on the launching stream, barriers and a synchronize
    on both sides, max over ranks.  A second graph of the same step carries
    the per-kernel event pairs of the library's profiler; it is replayed as
    many times right after the timed region and gives the kernel times (its
    event nodes would otherwise add to the step time)."""
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    assert bd.device_status() == 0, "device error word set during warm-up"
    l0 = bd.kernel_launches()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step.run()
    launches_per_step = bd.kernel_launches() - l0
    bd.profile_enable(True)
    step.run()
    torch.cuda.synchronize()
    bd.profile_collect()  # warms the event pool so capture creates no events
    graph_prof = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_prof):
        step.run()
    bd.profile_enable(False)
    for _ in range(warmup):
        graph.replay()
        graph_prof.replay()
    torch.cuda.synchronize()
    _barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    ms = e0.elapsed_time(e1) / steps
    e0.record(stream)
    for _ in range(steps):
        graph_prof.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    prof_ms = e0.elapsed_time(e1) / steps
    prof = bd.profile_collect()  # per-kernel device time of the last replay
    assert bd.device_status() == 0, "device error word set during the timed steps"
    del graph, graph_prof
    return {"ms": _max_over_ranks(ms, world), "prof_ms": prof_ms, "prof": prof,
            "launches_per_step": launches_per_step}


def rooflines(step, prof, ms):
    """(dominant-kernel roofline, per-kernel split, whole-step roofline)."""
    wl = step.wl
    kind, nbytes, src, bound = step.dominant()
    kms, kcnt = prof.get(kind, (0.0, 0))  # one replay: kcnt launches of the kernel
    hbm, tfl, peak_src = _peaks()
    roof = None
    if kcnt and bound == "hbm":
        per_launch_ms = kms / kcnt
        achieved = nbytes / (per_launch_ms / 1e3) / 1e9
        tr = NCU_TRAFFIC.get((kind, wl.name))
        traffic = tr[0] if tr and tr[1] == _src_hash(src) else None
        roof = {"bound": bound, "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": traffic, "kernel": kind,
                "algorithmic_bytes_per_launch": nbytes, "launch_ms": round(per_launch_ms, 5),
                "peak_source": peak_src}
    elif kcnt:
        per_launch_ms = kms / kcnt
        achieved = nbytes / (per_launch_ms / 1e3) / 1e12
        tr = NCU_TRAFFIC.get((kind, wl.name))
        traffic = tr[0] if tr and tr[1] == _src_hash(src) else None
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tfl, "unit": "TFLOP/s",
                "frac": round(achieved / tfl, 4), "traffic": traffic, "kernel": kind,
                "algorithmic_flops_per_launch": nbytes, "launch_ms": round(per_launch_ms, 5),
                "peak_source": peak_src}
    kernels = {k: {"ms_per_step": round(v[0], 5), "launches": v[1],
                   "share": round(v[0] / max(sum(x[0] for x in prof.values()), 1e-12), 4)}
               for k, v in prof.items() if v[1]}
    sbound, work = step.step_work()
    if sbound == "hbm":
        t_roof = work / (hbm * 1e9) * 1e3
        step_roof = {"bound": "hbm", "algorithmic_bytes_per_step": work, "peak": hbm,
                     "unit": "GB/s", "achieved": round(work / (ms / 1e3) / 1e9, 1)}
    else:
        t_roof = work / (tfl * 1e12) * 1e3
        step_roof = {"bound": "tensor", "algorithmic_flops_per_step": work, "peak": tfl,
                     "unit": "TFLOP/s", "achieved": round(work / (ms / 1e3) / 1e12, 1)}
    step_roof.update({"roofline_ms": round(t_roof, 5), "frac": round(t_roof / ms, 4),
                      "peak_source": peak_src})
    return roof, kernels, step_roof


def cpu_baseline(step, target_s):
    """The oracle as it stands on the host cores, on a bounded sample of the
    step (decode: the step's queries, repeated until about target_s of
    oracle time; prefill: the sample PrefillStep.cpu_baseline describes)."""
    import oracle
    wl = step.wl
    unit = "query-tok/s" if wl.mode == "decode" else "tok/s"
    if wl.mode == "decode":
        nq, secs, sample, passes = 0, 0.0, "", 0
        while secs < target_s and passes < 64:
            n1, s1, sample = step.cpu_baseline()
            nq, secs, passes = nq + n1, secs + s1, passes + 1
        sample = f"{sample}, {passes} passes"
    else:
        nq, secs, sample = step.cpu_baseline()
    return {"value": round(nq / secs, 4), "unit": unit, "cores": oracle.num_threads(),
            "kind": "oracle", "sample": sample, "seconds": round(secs, 4)}


def measure_other(wl, args, world, rank, dev, stream, fp4=False):
    """One more workload of the metric, timed like the default one (graph
    replays between CUDA events, per-kernel split, rooflines, clocks, the
    oracle on a bounded sample); returns its sub-object.  fp4: the decode
    step with MXFP4 indexer keys, plus its selection's recall of the bf16
    indexer's selection."""
    if wl.mode == "decode":
        step = DecodeStep(wl, dev, seed_offset=rank, fp4=fp4)
    else:
        step = PrefillStep(wl, dev, seed_offset=rank)
    steps = args.steps if wl.mode == "decode" else max(3, min(args.steps, 20))
    clocks = ClockSampler(dev)
    time.sleep(0.15)
    t = time_step(step, steps, max(3, args.warmup), world, stream)
    clk = clocks.stop()
    roof, kernels, step_roof = rooflines(step, t["prof"], t["ms"])
    unit = "query-tok/s" if wl.mode == "decode" else "tok/s"
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not fp4:
        cpu = cpu_baseline(step, 5.0)
    out = {"value": round(step.units() * world / (t["ms"] / 1e3), 2), "unit": unit,
           "ms_per_step": round(t["ms"], 5), "steps": steps,
           "config": {"batch_per_gpu": wl.B, "context": wl.T, "m": wl.m, "topk": wl.topk,
                      "n_h": wl.n_h, "c": wl.c, "kv_format": wl.kv, "n_win": wl.n_win,
                      "d": wl.d, "dtype": wl.act},
           "gpu_launches": t["launches_per_step"] * steps,
           "roofline": roof, "step_roofline": step_roof, "kernels": kernels,
           "ms_per_step_with_events": round(t["prof_ms"], 5),
           "cpu_baseline": cpu, "clocks": clk}
    if fp4:
        out["indexer_keys"] = "MXFP4 (E2M1 codes + E8M0 block scales, 68 B per entry)"
        out["recall_vs_bf16_topk"] = [round(r, 4) for r in step.recall_vs_bf16()]
    del step
    return out


# -------------------------------------------------------------------- main --
def run_ours(args, world, rank, local):
    from long_context_sparse_09_b200 import build
    if rank == 0 or world == 1:
        build.build_library()
    _barrier(world)
    wl = WORKLOADS[args.workload]
    if args.batch:
        wl = wl.with_(B=args.batch)
    if args.context:
        wl = wl.with_(T=args.context)
    dev = torch.device(f"cuda:{local}")
    torch.manual_seed(0)
    fp4_keys = args.fp4 and wl.mode == "decode" and wl.variant == "csa"
    if wl.mode == "decode":
        step = DecodeStep(wl, dev, seed_offset=rank, fp4=fp4_keys)
    else:
        step = PrefillStep(wl, dev, seed_offset=rank)
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(dev)
    time.sleep(0.15)
    t = time_step(step, args.steps, args.warmup, world, stream)
    clk = clocks.stop()
    ms, prof_ms, prof = t["ms"], t["prof_ms"], t["prof"]
    launches = t["launches_per_step"] * args.steps
    units = step.units() * world
    value = units / (ms / 1e3)

    # end to end through the public API: every step copies its inputs from
    # pinned host memory to the device, runs the library calls (a CUDA graph
    # of them per input buffer) and copies the result back to pinned host
    # memory.  The copies run on two
    # copy streams (in, out) with double buffers, so that step k+1's inputs
    # and step k's read-back overlap the compute, as a serving loop would;
    # every copy of every timed step lies inside the timed region.
    # the step's inputs sit in one pinned staging buffer (each at a 256-byte
    # offset), so that one copy per step carries them all
    inputs = step.step_inputs()
    offs, total = {}, 0
    for k, v in inputs.items():
        offs[k] = total
        total += (v.numel() * v.element_size() + 255) // 256 * 256

    def views(flat):
        return {k: flat[offs[k]:offs[k] + v.numel() * v.element_size()].view(v.dtype).view(v.shape)
                for k, v in inputs.items()}

    host_flat = torch.empty(total, dtype=torch.uint8).pin_memory()
    host_in = views(host_flat)
    for k, v in inputs.items():
        host_in[k].copy_(v.cpu())
    dev_flat = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]
    dev_in = [views(f) for f in dev_flat]
    dev_out = [torch.empty_like(step.out) for _ in range(2)]
    host_out = [torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory() for _ in range(2)]
    h2d = total  # bytes copied per step, padding included
    d2h = host_out[0].numel() * host_out[0].element_size()
    copy_stream = torch.cuda.Stream(device=dev)  # host -> device
    back_stream = torch.cuda.Stream(device=dev)  # device -> host
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b copied
    ev_used = [torch.cuda.Event() for _ in range(2)]   # step on buffer b computed
    ev_read = [torch.cuda.Event() for _ in range(2)]   # result of buffer b read back

    # the library calls of a step on buffer b, as a serving loop issues them:
    # captured once per buffer set into a CUDA graph (the calls take no
    # allocation and accept capture), replayed every step
    def step_kwargs(bsel):
        d = dev_in[bsel]
        kw = {"q": d["q"], "qI": d.get("qI"), "w": d.get("w"), "q_pos": d["q_pos"],
              "out": dev_out[bsel]}
        if "H" in d:
            kw["H"] = d["H"]
        return kw

    for bsel in range(2):
        dev_flat[bsel].copy_(host_flat)
        step.run(**step_kwargs(bsel))
    torch.cuda.synchronize()
    step_graphs = []
    for bsel in range(2):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step.run(**step_kwargs(bsel))
        step_graphs.append(g)

    def e2e_step(k):
        bsel = k & 1
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(ev_used[bsel])  # inputs of step k-2 no longer needed
            dev_flat[bsel].copy_(host_flat, non_blocking=True)
            ev_in[bsel].record(copy_stream)
        stream.wait_event(ev_in[bsel])
        stream.wait_event(ev_read[bsel])  # result of step k-2 read back
        step_graphs[bsel].replay()
        ev_used[bsel].record(stream)
        with torch.cuda.stream(back_stream):
            back_stream.wait_event(ev_used[bsel])
            host_out[bsel].copy_(dev_out[bsel], non_blocking=True)
            ev_read[bsel].record(back_stream)

    def arm():  # the events of both buffers start out complete
        for bsel in range(2):
            ev_used[bsel].record(stream)
            ev_read[bsel].record(stream)

    arm()
    for k in range(args.warmup):
        e2e_step(k)
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    arm()  # the first copies start inside the timed region
    for k in range(args.steps):
        e2e_step(k)
    for bsel in range(2):
        stream.wait_event(ev_read[bsel])  # the last results are on the host
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    assert bd.device_status() == 0, "device error word set during the timed steps"

    append = None
    if wl.mode == "decode":
        # the decode-time compressor, timed on its own (not part of `value`)
        a_ms, a_bytes, a_split = step.time_append(min(args.steps, 500), stream)
        hbm0, _, _ = _peaks()
        append = {"ms_per_call": round(a_ms, 5), "tokens": wl.B,
                  "weight_bytes": a_bytes, "hbm_frac": round(a_bytes / (a_ms / 1e3) / 1e9 / hbm0, 4),
                  "kernels_ms": a_split}

    out_proj = None
    if wl.mode == "decode" and wl.act == "bf16":
        # the grouped output projection after the step (timed on its own)
        o_ms, o_bytes = step.time_out_proj(min(args.steps, 200), stream)
        hbm0, _, _ = _peaks()
        out_proj = {"ms_per_call": round(o_ms, 5), "tokens": wl.B, "g": wl.g_out, "d_g": wl.d_g,
                    "weight_bytes": o_bytes,
                    "hbm_frac": round(o_bytes / (o_ms / 1e3) / 1e9 / hbm0, 4)}

    query_proj = None
    if wl.mode == "decode" and wl.variant == "csa" and wl.act == "bf16":
        # the query-side projections before the step (timed on their own)
        qp_ms, qp_bytes = step.time_query_proj(min(args.steps, 200), stream)
        hbm0, _, _ = _peaks()
        query_proj = {"ms_per_call": round(qp_ms, 5), "tokens": wl.B, "d_c": wl.d_c,
                      "weight_bytes": qp_bytes,
                      "hbm_frac": round(qp_bytes / (qp_ms / 1e3) / 1e9 / hbm0, 4)}

    roof, kernels, step_roof = rooflines(step, prof, ms)
    entries = getattr(step, "N", getattr(step, "nE", 0))
    unit = "query-tok/s" if wl.mode == "decode" else "tok/s"
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(step, 10.0)

    # the other workloads of the metric (prefill tokens/s, the HCA and the
    # V4-Flash decode), each timed the same way, as sub-objects of the line
    others = {}
    if args.workload == DEFAULT_BENCH and not args.batch and not args.context and \
            not args.no_others:
        del step, step_graphs, dev_flat, dev_in, dev_out
        torch.cuda.empty_cache()
        for name in OTHER_WORKLOADS:
            base, _, variant = name.partition("+")
            others[name] = measure_other(WORKLOADS[base], args, world, rank, dev, stream,
                                         fp4=variant == "mxfp4")
            torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "batch_per_gpu": wl.B, "context": wl.T,
                       "entries_per_seq": entries,
                       "m": wl.m, "topk": wl.topk,
                       "n_h": wl.n_h, "c": wl.c, "kv_format": wl.kv, "n_win": wl.n_win,
                       "indexer_keys": "mxfp4" if fp4_keys else "bf16",
                       "l2": "inputs larger than L2 (cache streamed every step)"},
            "e2e": {"value": round(units / (e2e_ms / 1e3), 2),
                    "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 5)},
            "gpu_launches": launches,
            "timing": ("CUDA-graph replays of the step; kernel times from the last of as many "
                       "replays of the same step with per-kernel CUDA events"),
            "ms_per_step_with_events": round(prof_ms, 5),
            "roofline": roof,
            "kernels": kernels,
            "step_roofline": step_roof,
            "decode_append": append,
            "out_proj": out_proj,
            "query_proj": query_proj,
            "cpu_baseline": cpu,
            "clocks": clk,
            "workloads": others,
        }
        print(json.dumps(line), flush=True)


def run_reference(args, world, rank, local):
    """The oracle as it stands on the host cores, same workload and metric.

    A step is one query of the workload.  When K + W full queries would take
    longer than about four minutes, every step takes the same query on the
    first N/D entries of its cache instead (its position moved to the end of
    that range, window unchanged) and counts as 1/D query; D is the smallest
    power of two that fits the run into the budget.  Top-k and attention do
    not shrink with D, so the sampled rate is, if anything, low."""
    if rank != 0:
        return
    import numpy as np
    import oracle
    from oracle import pipeline as P
    wl = WORKLOADS[args.workload]
    if wl.mode != "decode":
        raise SystemExit("the reference arm times decode workloads")
    dev = torch.device(f"cuda:{local}") if torch.cuda.is_available() else torch.device("cpu")
    inp = synth.decode_inputs(wl, device=dev)
    N = inp["N"]
    b = 0  # the first sequence of the batch
    qd = inp["q"][b:b + 1].double().cpu().numpy()
    win = P.cache_values(inp["win"][b].cpu(), None if inp["win_scale"] is None
                         else inp["win_scale"][b].cpu(), wl.kv, wl.c, wl.rope_dims)
    kvv = None
    if wl.variant == "csa":
        qI = inp["qI"][b:b + 1].double().cpu().numpy()
        w = inp["w"][b:b + 1].double().cpu().numpy()
        kI = inp["kI"][b].double().cpu().numpy()
    else:
        kvv = P.cache_values(inp["ckv"][b].cpu(), None, wl.kv, wl.c, wl.rope_dims)
    sink = inp["sink"].double().cpu().numpy()
    L = int(inp["q_pos"][b])

    def one(n_ent):
        """One query over the first n_ent entries; returns the oracle's seconds."""
        pos = np.array([min(L, wl.m * n_ent + wl.m - 1)], np.int32)
        wp0 = int(pos[0]) - wl.n_win + 1
        t0 = time.perf_counter()
        if wl.variant == "csa":
            scores = oracle.index_scores(pos, wl.m, qI, w, kI[:n_ent])
            nv = np.array([oracle.nvis(int(pos[0]), wl.m, n_ent)], np.int32)
            idx, _ = oracle.topk(scores, nv, wl.topk)
            dt = time.perf_counter() - t0
            sel = idx[0][idx[0] >= 0]
            st = torch.from_numpy(sel).long().to(inp["ckv"].device)
            rows = P.cache_values(inp["ckv"][b][st].cpu(), None if inp["ckv_scale"] is None
                                  else inp["ckv_scale"][b][st].cpu(), wl.kv, wl.c, wl.rope_dims)
            t0 = time.perf_counter()
            oracle.attend(pos, qd, np.arange(len(sel), dtype=np.int32)[None, :], wl.m, rows,
                          wl.n_win, win, wp0, sink, wl.rope_dims, wl.rope_base, wl.softmax_scale)
            return dt + time.perf_counter() - t0
        P.attend_wl(wl, pos, qd, None, kvv[:n_ent], win, wp0, sink)
        return time.perf_counter() - t0

    budget = 240.0
    t_full = one(N)  # probe (counts as the first warm-up step)
    D = 1
    while (args.steps + args.warmup) * t_full / D > budget and N // (2 * D) >= max(wl.topk, 1):
        D *= 2
    n_ent = N // D
    total_s = 0.0
    for s in range(1, args.warmup + args.steps):
        dt = one(n_ent)
        if s >= args.warmup:
            total_s += dt
    if args.warmup == 0:
        total_s += t_full if D == 1 else one(n_ent)
    units = args.steps / D
    v = units / total_s
    sample = (f"1 query per step (sequence 0, full {wl.T}-token context)" if D == 1 else
              f"1 query per step on the first 1/{D} of its {N} entries (counted as 1/{D} query)")
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "query-tok/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * total_s / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "batch_per_gpu": wl.B, "context": wl.T},
            "cpu_baseline": {"kind": "oracle", "cores": oracle.num_threads(), "value": round(v, 4),
                             "unit": "query-tok/s", "sample": sample},
            "e2e": {"value": round(v, 4), "unit": "query-tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_BENCH, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-others", action="store_true",
                    help="time the named workload only (no prefill / HCA / Flash sub-objects)")
    ap.add_argument("--batch", type=int, default=0, help="override sequences per GPU (profiling)")
    ap.add_argument("--context", type=int, default=0, help="override context length (profiling)")
    ap.add_argument("--fp4", action="store_true",
                    help="decode step with the MXFP4 indexer as the named workload (profiling)")
    args = ap.parse_args()
    if args.impl == "reference":
        # rank 0 alone times the oracle on the host; no process group
        world, rank, local = D.world()
        run_reference(args, world, rank, local)
        return
    world, rank, local = _dist()
    try:
        run_ours(args, world, rank, local)
    finally:
        D.finalize()


if __name__ == "__main__":
    main()
