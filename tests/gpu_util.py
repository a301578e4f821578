"""Helpers shared by the GPU parity tests: buffer allocation in the library's
layouts, conversion of stored values to float64, and the comparison rules.

Comparison rules (what "parity" means here):
* fp outputs: bf16 / FP8 paths: max-abs <= 2e-2 and rel-L2 <= 5e-3 against
  the fp64 oracle; fp32 path: max-abs <= 1e-5.
* indexer scores: |gpu - oracle| <= tol, tol derived from fp32 accumulation
  of c_I products per head and n_hI heads: 4 (c_I + n_hI) 2^-24
  (sum_h |w_h| |q_h|) . |K_s| (factor 4 of margin over the first-order bound).
* top-k sets: equal, except at ties: an index selected by only one side must
  have an oracle score within 1e-6 relative of the oracle's k-th score;
  output ascending, -1 padded, visible.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle import pipeline as P

DEV = "cuda"
U32 = 2.0 ** -24


def row_bytes(wl) -> int:
    if wl.kv == "f32":
        return 4 * wl.c
    if wl.kv == "bf16":
        return 2 * wl.c
    return (wl.c - wl.rope_dims) + 2 * wl.rope_dims


def alloc_kv(wl, lead: tuple, rows: int, device=DEV):
    """Empty cache rows in the workload's KV format: (rec, scale or None)."""
    if wl.kv == "f32":
        return torch.empty(lead + (rows, wl.c), dtype=torch.float32, device=device), None
    if wl.kv == "bf16":
        return torch.empty(lead + (rows, wl.c), dtype=torch.bfloat16, device=device), None
    rec = torch.empty(lead + (rows, row_bytes(wl)), dtype=torch.uint8, device=device)
    return rec, torch.empty(lead + (rows,), dtype=torch.float32, device=device)


def kv_values(wl, rec, scale) -> np.ndarray:
    return P.cache_values(rec, scale, wl.kv, wl.c, wl.rope_dims)


def act_dtype(wl):
    return torch.float32 if wl.act == "f32" else torch.bfloat16


def to_dev(d: dict) -> dict:
    return {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in d.items()}


def assert_close(got, ref, fmt: str, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    if fmt == "f32":
        assert err.max() <= 1e-5, f"{what}: max-abs {err.max():.3g} > 1e-5"
    else:
        rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
        assert err.max() <= 2e-2, f"{what}: max-abs {err.max():.3g} > 2e-2"
        assert rel <= 5e-3, f"{what}: rel-L2 {rel:.3g} > 5e-3"


def score_tolerance(qI, w, kI) -> np.ndarray:
    """Per (query, entry) bound on the fp32 accumulation error of eq. 16."""
    qI = np.abs(np.asarray(qI, dtype=np.float64))
    w = np.abs(np.asarray(w, dtype=np.float64))
    K = np.abs(np.asarray(kI, dtype=np.float64))
    n_hI, c_I = qI.shape[1], qI.shape[2]
    comb = np.einsum("qh,qhe->qe", w, qI)
    return 4.0 * (c_I + n_hI) * U32 * (comb @ K.T) + 1e-30


def check_topk(idx_gpu, score_gpu, scores_ref, nv, k, tol, what=""):
    """Check GPU idx/scores of several queries against oracle scores."""
    idx_gpu = np.asarray(idx_gpu)
    for q in range(idx_gpu.shape[0]):
        n = int(nv[q])
        keep = min(k, n)
        row = idx_gpu[q]
        sel = row[:keep]
        assert np.all(row[keep:] == -1), f"{what} q{q}: padding"
        assert np.all(np.diff(sel) > 0), f"{what} q{q}: not ascending/unique"
        assert keep == 0 or (sel[0] >= 0 and sel[-1] < n), f"{what} q{q}: out of range"
        if score_gpu is not None and keep:
            sg = np.asarray(score_gpu[q][:keep], dtype=np.float64)
            bad = np.abs(sg - scores_ref[q, sel]) > tol[q, sel]
            assert not bad.any(), f"{what} q{q}: score mismatch at {sel[bad][:5]}"
        if keep == 0:
            continue
        ref_idx, kth = oracle.topk(scores_ref[q: q + 1], np.array([n], np.int32), k)
        ref_sel = ref_idx[0][:keep]
        only_g = np.setdiff1d(sel, ref_sel)
        only_o = np.setdiff1d(ref_sel, sel)
        assert len(only_g) == len(only_o)
        if len(only_g):
            # the stated bar: indices may differ only at ties within 1e-6
            # relative (oracle scores of the differing index and of the k-th)
            for s in np.concatenate([only_g, only_o]):
                gap = abs(scores_ref[q, s] - kth[0])
                lim = 1e-6 * max(abs(scores_ref[q, s]), abs(kth[0]))
                assert gap <= lim, (
                    f"{what} q{q}: index {s} differs, |I(s)-I(kth)| = {gap:.3g} "
                    f"> 1e-6 relative ({lim:.3g})")


# ------------------------------------------------------ FP8-mixed records --
# Relative deviation allowed between the GPU's fp32 row (the value it
# quantises) and the oracle's fp64 row, as a fraction of the row's largest
# FP8-dim magnitude.  Both sides compute the same row from the same stored
# inputs; they differ only by fp32 rounding in the GPU's sums (bf16 products
# accumulated in fp32 over d terms, the 2m-slot softmax, RMSNorm, RoPE), a few
# parts in 10^7 of max|x| on these inputs; 2^-16 = 1.5e-5 leaves a 30x margin.
FP8_SLACK = 2.0 ** -16

_E4M3 = None


def _e4m3_values() -> np.ndarray:
    global _E4M3
    if _E4M3 is None:
        _E4M3 = np.array([oracle.e4m3_decode(c) for c in range(256)])
    return _E4M3


def check_fp8_records(rec, scale, x_ref, wl, what, slack=FP8_SLACK):
    """Pin of the FP8-mixed storage rule on the GPU's records ("02 ·
    DeepSeek-V4: 压缩注意力撑起 1M 上下文" 2.5: RoPE dims in BF16, the others in
    FP8; the reading: per row scale = max|x| / 448 over the FP8 dims in
    fp32, E4M3 code = round-to-nearest-even, saturating, of x / scale).

    rec [.., rows, (c - rope) + 2 rope] uint8 and scale [.., rows] fp32 are
    the GPU's; x_ref [rows][c] is the oracle's unquantised fp64 row.
    * scale: equal to oracle.fp8mix_encode's scale within `slack` relative
      (a rule such as max|x| / 240 is off by 87%);
    * codes: the GPU quantises its own fp32 row, which lies within
      slack * max|x| of the oracle's, so its scaled value lies within
      y +- slack * (448 + |y|) of the oracle's y = x / scale.  Rounding to
      nearest is monotone, so the GPU's code must decode to a value between
      the oracle encoder's codes of those two extremes: the oracle's own code
      wherever the band holds no rounding boundary (nearly every element),
      its neighbour only where it does.  Truncation, a wrong scale or a
      wrong rounding mode fail on most elements;
    * RoPE dims: the GPU's bf16 value lies between the bf16 roundings of the
      two extremes x +- slack * max|x|."""
    r2 = rec.detach().cpu().contiguous().reshape(-1, rec.shape[-1]).numpy()
    sg = scale.detach().cpu().reshape(-1).numpy().astype(np.float64)
    x = np.asarray(x_ref, dtype=np.float64).reshape(-1, wl.c)
    assert r2.shape[0] == x.shape[0], (what, r2.shape, x.shape)
    nf = wl.c - wl.rope_dims
    codes_o, _, s_o = oracle.fp8mix_encode(x, wl.rope_dims)
    s_o = s_o.astype(np.float64)
    rel = np.abs(sg / s_o - 1.0)
    assert rel.max() <= slack, (
        f"{what}: scale differs from max|x|/448 by {rel.max():.3g} relative (> {slack:.3g}) "
        f"at row {int(rel.argmax())}")
    y = (x[:, :nf].astype(np.float32) / s_o[:, None].astype(np.float32)).astype(np.float64)
    band = slack * (448.0 + np.abs(y))
    enc = np.vectorize(oracle.e4m3_encode, otypes=[np.uint8])
    tab = _e4m3_values()
    v_lo = tab[enc(np.clip(y - band, -448.0, 448.0))]
    v_hi = tab[enc(np.clip(y + band, -448.0, 448.0))]
    cg = r2[:, :nf]
    v_g = tab[cg]
    bad = (v_g < v_lo) | (v_g > v_hi)
    n_diff = int(np.count_nonzero(cg != codes_o))
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} E4M3 codes outside the rounding band "
        f"(first at {np.argwhere(bad)[0].tolist()}: gpu {int(cg[bad][0]):#x}, oracle "
        f"{int(codes_o[bad][0]):#x}); {n_diff} codes differ in all")
    # RoPE dims: little-endian bf16 bit patterns after the codes
    bits = r2[:, nf:].copy().view(np.uint16).astype(np.uint32) << 16
    got_r = bits.view(np.float32).astype(np.float64)
    amax = (s_o * 448.0)[:, None]
    xr = x[:, nf:]
    r_lo = oracle.round_bf16(xr - slack * amax)
    r_hi = oracle.round_bf16(xr + slack * amax)
    bad_r = (got_r < r_lo) | (got_r > r_hi)
    assert not bad_r.any(), f"{what}: {int(bad_r.sum())} bf16 RoPE dims outside the rounding band"
    return n_diff
