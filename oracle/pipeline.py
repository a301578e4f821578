"""Oracle compositions of the whole CSA / HCA forward pass (test
infrastructure only; see the package docstring).

The steps are taken in the order of the DeepSeek-V4 reading notes
("DeepSeekV4技术报告阅读笔记", 2.3-2.5): compress (eq. 9-12 or 20-23), RMSNorm +
partial RoPE of the entries and of the window rows, indexer scores (eq. 16),
top-k (eq. 17), shared-KV MQA with window and sink (eq. 19 / 26 / 27) and
the R_{-t} de-rotation of the output.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (attend, compress, fp8mix_decode, fp8mix_encode, index_scores,
               matmul, mxfp4_round, norm_rope_rows, nvis, rmsnorm, rope, round_bf16, topk,
               _f64)


def store(x: np.ndarray, fmt: str, rope_dims: int) -> np.ndarray:
    """Round fp64 values to a storage format and return the stored values:
    'f32' (nearest fp32), 'bf16' (nearest bf16), 'fp8mix' (E4M3 with a
    per-row scale on the non-RoPE dims, bf16 on the RoPE dims)."""
    if fmt == "f32":
        return x.astype(np.float32).astype(np.float64)
    if fmt == "bf16":
        return round_bf16(x)
    codes, rope, scale = fp8mix_encode(x, rope_dims)
    c = x.shape[-1]
    # rope holds bf16-exact values: the fp32 -> bf16 cast below is exact
    bits = torch.from_numpy(rope.astype(np.float32)).to(torch.bfloat16).view(torch.int16)
    bits = bits.numpy().view(np.uint16)
    return fp8mix_decode(codes, bits, scale, c, rope_dims)


def cache_values(rec, scale, fmt: str, c: int, rope_dims: int) -> np.ndarray:
    """fp64 values of a cache held in the library's layout: f32 / bf16 rows
    [.., rows, c], or fp8mix records [.., rows, (c-rope) + 2*rope bytes] with
    an fp32 scale per row."""
    if fmt in ("f32", "bf16"):
        return _f64(rec)
    rec = rec.detach().cpu()
    lead = rec.shape[:-1]
    nf = c - rope_dims
    r2 = rec.reshape(-1, rec.shape[-1])
    codes = r2[:, :nf].contiguous().numpy()
    bits = r2[:, nf:].contiguous().view(torch.int16).numpy().view(np.uint16)
    sc = scale.detach().cpu().reshape(-1).numpy().astype(np.float32)
    return fp8mix_decode(codes, bits, sc, c, rope_dims).reshape(*lead, c)


def compress_seq(wl, W: dict, H):
    """(kv [N][c], kI [N][c_I] or None, win [T][c]) of one sequence, each
    rounded to its storage format."""
    H = _f64(H)
    if wl.variant == "csa":
        raw = compress(H, wl.m, W["Wkv_a"], W["Wz_a"], W["B_a"],
                       W["Wkv_b"], W["Wz_b"], W["B_b"])
        kI = compress(H, wl.m, W["WIkv_a"], W["WIz_a"], W["BI_a"],
                      W["WIkv_b"], W["WIz_b"], W["BI_b"])
        kI = store(kI, wl.act, 0)
    else:
        raw = compress(H, wl.m, W["Wkv_a"], W["Wz_a"], W["B_a"])
        kI = None
    kv = norm_rope_rows(raw, wl.rope_dims, wl.rope_base, wl.rms_eps, 0.0, float(wl.m))
    kv = store(kv, wl.kv, wl.rope_dims)
    Ca = matmul(H, W["Wkv_a"])
    win = norm_rope_rows(Ca, wl.rope_dims, wl.rope_base, wl.rms_eps, 0.0, 1.0)
    win = store(win, wl.kv, wl.rope_dims)
    return kv, kI, win


def select(wl, t0s, qI, w, kI):
    """(idx [Q][k], scores [Q][N], nvis [Q], kth [Q]) of eq. 16-17."""
    N = kI.shape[0]
    scores = index_scores(t0s, wl.m, qI, w, kI)
    nv = np.array([nvis(t, wl.m, N) for t in t0s], dtype=np.int32)
    idx, kth = topk(scores, nv, wl.topk)
    return idx, scores, nv, kth


def attend_wl(wl, t0s, q, idx, kv, win, win_pos0, sink, rope_shift=0.0):
    return attend(t0s, q, idx, wl.m, kv, wl.n_win, win, win_pos0, sink,
                  wl.rope_dims, wl.rope_base, wl.softmax_scale, rope_shift)


def query_proj(H, pos, WDQ, WUQ, WIUQ, Ww, n_h: int, c: int, n_hI: int, c_I: int,
               rope_dims: int, base: float, eps: float, round_mid: bool = False):
    """The query side of the layer for tokens H [T][d] at positions pos [T]
    (the reading notes eq. 13-15 and 18; 2.5.1, 2.5.2):
        c^Q = h W^{DQ}                          (eq. 13, d -> d_c)
        q^I = c^Q W^{IUQ}, one c_I row per head (eq. 14)
        w   = h W^{w}                           (eq. 15)
        q   = c^Q W^{UQ}, one c row per head    (eq. 18)
    then every head of q is RMS-normalised (unit gain, 2.5.1) and rotated on
    its last rope_dims at its token's position (2.5.2).  Readings: no norm on
    c^Q and none and no rotation on q^I (the pages give neither; the
    indexer keys have neither either).  With round_mid, c^Q is rounded to
    bf16 (the activation dtype) before the two up-projections, as a
    stored low-rank latent is (reading: the latent between the products is
    stored in the activation dtype, like the group outputs of the output
    projection).  Returns (c^Q, q, q^I, w)."""
    H = _f64(H)
    T = H.shape[0]
    cQ = matmul(H, WDQ)
    if round_mid:
        cQ = round_bf16(cQ)
    qI = matmul(cQ, WIUQ).reshape(T, n_hI, c_I)
    w = matmul(H, Ww)
    q = matmul(cQ, WUQ).reshape(T, n_h, c)
    for t in range(T):
        for h in range(n_h):
            q[t, h] = rope(rmsnorm(q[t, h], eps), rope_dims, base, float(pos[t]))
    return cQ, q, qI, w


def index_scores_fp4(wl, t0s, qI, w, kI):
    """Index scores of eq. 16 with the QK path in MXFP4 and bf16 scores
    (PaperTrace 3.3): every head of q^I and every row of K^I is rounded to
    MXFP4 along c_I (blocks of 32); the products, ReLU and the w-weighted
    head sum are then exact, and the score is rounded to bf16 (-inf where
    the entry is not visible).  Readings: w stays fp32; the rounding to bf16
    is the score's only rounding after the inputs'."""
    s = index_scores(t0s, wl.m, mxfp4_round(qI), w, mxfp4_round(kI))
    return np.where(np.isfinite(s), round_bf16(np.where(np.isfinite(s), s, 0.0)), s)


def topk_recall(idx_a, idx_b) -> np.ndarray:
    """Per query, the fraction of idx_b's selected entries (-1 padding
    ignored) that idx_a also selects: the KV recall of a selection."""
    idx_a, idx_b = np.asarray(idx_a), np.asarray(idx_b)
    out = np.empty(idx_a.shape[0])
    for q in range(idx_a.shape[0]):
        b = set(int(i) for i in idx_b[q] if i >= 0)
        a = set(int(i) for i in idx_a[q] if i >= 0)
        out[q] = len(a & b) / len(b) if b else 1.0
    return out

