"""Seeded synthetic inputs for the CSA / HCA forward pass.

Both the CUDA path and the CPU oracle are fed from here; this module holds
none of the method's arithmetic (no projection, normalisation, rotation,
softmax or quantisation rule), only random draws of the right shapes,
dtypes and distributions:

* activations H ~ N(0, 1); weights ~ N(0, 1/fan_in); position biases
  ~ N(0, 0.1) (0.1 read as the variance); sink logits ~ N(0, 1);
* projected queries q, indexer queries q^I and head weights w ~ N(0, 1) --
  the distribution the low-rank query path (c^Q = h W^DQ, q = c^Q W^UQ,
  q^I = c^Q W^IUQ, w = h W^w) yields for h ~ N(0, 1) and N(0, 1/fan_in)
  weights; RMSNorm leaves unit-RMS vectors (as N(0,1) rows nearly are);
* decode caches (compressed entries, indexer keys, window rows) ~ N(0, 1)
  rows; the FP8-mixed format draws an fp32 per-entry scale uniformly in
  [3.5, 5] / 448 and stores the E4M3 cast of x / scale (a library cast) with
  the last rope_dims kept as BF16.

Every tensor is produced on ``device`` from a ``torch.Generator`` seeded per
(workload seed, stream name), so the same call gives the same values.
"""
from __future__ import annotations

import zlib

import torch

from .configs import Workload

def _dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


class _Streams:
    def __init__(self, seed: int, device):
        self.seed = seed
        self.device = torch.device(device)

    def gen(self, name: str) -> torch.Generator:
        g = torch.Generator(device=self.device)
        g.manual_seed((self.seed * 1000003 + zlib.crc32(name.encode())) % (2 ** 63))
        return g

    def normal(self, name, shape, std=1.0, dtype=torch.float32):
        t = torch.randn(shape, generator=self.gen(name), device=self.device,
                        dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        return t.to(dtype)

    def uniform(self, name, shape, lo, hi):
        t = torch.rand(shape, generator=self.gen(name), device=self.device,
                       dtype=torch.float32)
        return t.mul_(hi - lo).add_(lo)


def kv_record_bytes(wl: Workload) -> int:
    """Bytes of one cache row in the main plane for the workload's format."""
    if wl.kv == "f32":
        return 4 * wl.c
    if wl.kv == "bf16":
        return 2 * wl.c
    return (wl.c - wl.rope_dims) + 2 * wl.rope_dims


def cache_rows(wl: Workload, st: _Streams, name: str, lead: tuple, rows: int):
    """A synthetic cache of `rows` rows per lead index in the workload's
    format: returns (record tensor, scale tensor or None)."""
    shape = lead + (rows, wl.c)
    if wl.kv in ("f32", "bf16"):
        return st.normal(name, shape, dtype=_dtype(wl.kv)), None
    nf = wl.c - wl.rope_dims
    x = st.normal(name + ".x", lead + (rows, nf))
    scale = st.uniform(name + ".scale", lead + (rows,), 3.5 / 448.0, 5.0 / 448.0)
    codes = (x / scale.unsqueeze(-1)).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn)
    del x
    rope = st.normal(name + ".rope", lead + (rows, wl.rope_dims), dtype=torch.bfloat16)
    rec = torch.cat([codes.view(torch.uint8), rope.view(torch.uint8)], dim=-1)
    return rec.contiguous(), scale.contiguous()


def weights(wl: Workload, device="cpu") -> dict:
    """Compressor weights [d][width] and position biases [m][width]."""
    st = _Streams(wl.seed, device)
    adt = _dtype(wl.act)
    std = wl.d ** -0.5
    bstd = 0.1 ** 0.5
    out = {}
    branches = ("a", "b") if wl.overlap else ("a",)
    for br in branches:
        out[f"Wkv_{br}"] = st.normal(f"Wkv_{br}", (wl.d, wl.c), std, adt)
        out[f"Wz_{br}"] = st.normal(f"Wz_{br}", (wl.d, wl.c), std, adt)
        out[f"B_{br}"] = st.normal(f"B_{br}", (wl.m, wl.c), bstd)
        if wl.variant == "csa":
            out[f"WIkv_{br}"] = st.normal(f"WIkv_{br}", (wl.d, wl.c_I), std, adt)
            out[f"WIz_{br}"] = st.normal(f"WIz_{br}", (wl.d, wl.c_I), std, adt)
            out[f"BI_{br}"] = st.normal(f"BI_{br}", (wl.m, wl.c_I), bstd)
    return out


def prefill_inputs(wl: Workload, device="cpu", T: int | None = None) -> dict:
    """Hidden states, projected queries and sinks of a prefill workload
    (all T queries of each sequence, positions 0..T-1)."""
    T = wl.T if T is None else T
    st = _Streams(wl.seed, device)
    adt = _dtype(wl.act)
    Q = wl.B * T
    out = {
        "H": st.normal("H", (wl.B, T, wl.d), dtype=adt),
        "q": st.normal("q", (Q, wl.n_h, wl.c), dtype=adt),
        "sink": st.normal("sink", (wl.n_h,)),
        "q_pos": torch.arange(T, dtype=torch.int32, device=device).repeat(wl.B),
    }
    if wl.variant == "csa":
        out["qI"] = st.normal("qI", (Q, wl.n_hI, wl.c_I), dtype=adt)
        out["w"] = st.normal("w", (Q, wl.n_hI))
    return out


def decode_inputs(wl: Workload, device="cpu", B: int | None = None,
                  L: int | None = None) -> dict:
    """A resident cache of context length L per sequence plus one new query
    per sequence at position L; the window holds tokens L-n_win+1..L."""
    B = wl.B if B is None else B
    L = wl.T if L is None else L
    N = L // wl.m
    st = _Streams(wl.seed, device)
    adt = _dtype(wl.act)
    ckv, ckv_scale = cache_rows(wl, st, "ckv", (B,), N)
    win, win_scale = cache_rows(wl, st, "win", (B,), wl.n_win)
    out = {
        "N": N,
        "ckv": ckv, "ckv_scale": ckv_scale,
        "win": win, "win_scale": win_scale,
        "q": st.normal("q", (B, wl.n_h, wl.c), dtype=adt),
        "sink": st.normal("sink", (wl.n_h,)),
        "q_pos": torch.full((B,), L, dtype=torch.int32, device=device),
        "win_pos0": torch.full((B,), L - wl.n_win + 1, dtype=torch.int32,
                               device=device),
    }
    if wl.variant == "csa":
        out["kI"] = st.normal("kI", (B, N, wl.c_I), dtype=adt)
        out["qI"] = st.normal("qI", (B, wl.n_hI, wl.c_I), dtype=adt)
        out["w"] = st.normal("w", (B, wl.n_hI))
    return out
