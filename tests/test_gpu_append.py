"""Decode-time compressor (csa_decode_append / hca_decode_append) against
the oracle: appending the tokens of a sequence one at a time must give the
same entries, indexer keys and window rows as compressing the whole
sequence ("DeepSeekV4技术报告阅读笔记" eq. 9-12 / 20-23, 2.5.1-2.5.3), up to
the order of the softmax sums (a running maximum and rescaled sums)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline as P
from long_context_sparse_09_b200 import binding as bd, synth
from long_context_sparse_09_b200.configs import WORKLOADS
from gpu_util import (DEV, act_dtype, alloc_kv, assert_close, check_fp8_records, check_topk,
                      kv_values, score_tolerance, to_dev)

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["flash_csa_decode_64k"]

APPEND_CASES = [
    # name, variant, act, kv, B, T, d, c, rope, c_I, m
    ("csa_bf16", "csa", "bf16", "bf16", 2, 42, 256, 512, 64, 128, 4),
    ("csa_fp8", "csa", "bf16", "fp8mix", 2, 36, 128, 512, 64, 64, 4),
    ("csa_f32", "csa", "f32", "f32", 1, 33, 96, 128, 32, 32, 4),
    ("hca_bf16", "hca", "bf16", "bf16", 2, 50, 128, 128, 32, 0, 16),
    # more sequences than one projection launch takes (two launches)
    ("csa_b18", "csa", "bf16", "bf16", 18, 13, 64, 128, 32, 32, 4),
    # the heavy compression rate: entries span 128 tokens
    ("hca_m128", "hca", "bf16", "bf16", 1, 300, 64, 128, 32, 0, 128),
    # the bench's launch configurations: the 1M decode (4 sequences, d = 7168,
    # FP8-mixed; 20 tiles x 7 slices), the 64K decode (32 sequences: two
    # launches) and the HCA decode (16 sequences, m' = 128)
    ("pro_decode_shape", "csa", "bf16", "fp8mix", 4, 8, 7168, 512, 64, 128, 4),
    ("flash_decode_shape", "csa", "bf16", "bf16", 32, 8, 4096, 512, 64, 128, 4),
    ("hca_decode_shape", "hca", "bf16", "bf16", 16, 128, 4096, 512, 64, 0, 128),
]


@pytest.fixture(autouse=True)
def _clean_status(cuda_ok):
    bd.device_status()
    yield
    torch.cuda.synchronize()
    assert bd.device_status() == 0


@pytest.mark.parametrize("case", APPEND_CASES, ids=[c[0] for c in APPEND_CASES])
def test_append_matches_whole_sequence(case):
    name, variant, act, kv, B, T, d, c, rd, ci, m = case
    wl = BASE.with_(variant=variant, act=act, kv=kv, d=d, c=c, rope_dims=rd, c_I=ci,
                    n_hI=4 if ci else 0, m=m, T=T, B=B, seed=len(name) + 23)
    p = bd.params_for(wl)
    W = synth.weights(wl)
    H = synth.prefill_inputs(wl)["H"]  # [B][T][d]
    packed = bd.csa_pack_weights(p, to_dev(W))
    nE = T // m
    ckv, ckv_s = alloc_kv(wl, (B,), nE)
    win, win_s = alloc_kv(wl, (B,), T)
    kI = torch.empty(B, nE, ci, dtype=act_dtype(wl), device=DEV) if variant == "csa" else None
    # the state needs no initialisation: every slot restarts at its entry's
    # first token, so NaN left in it must never reach a result
    tail = torch.full((bd.decode_tail_bytes(p, B, d) // 4,), float("nan"), device=DEV)
    win_pos0 = torch.zeros(B, dtype=torch.int32, device=DEV)
    Hd = H.to(DEV)
    for t in range(T):
        h = Hd[:, t, :].contiguous()
        tt = torch.full((B,), t, dtype=torch.int32, device=DEV)
        if variant == "csa":
            bd.csa_decode_append(p, h, tt, packed, tail, ckv, ckv_s, kI, win, win_s, win_pos0)
        else:
            bd.hca_decode_append(p, h, tt, packed, tail, ckv, ckv_s, win, win_s, win_pos0)
    torch.cuda.synchronize()
    got_kv = kv_values(wl, ckv, ckv_s)
    got_win = kv_values(wl, win, win_s)
    for b in range(B):
        ref_kv, ref_kI, ref_win = P.compress_seq(wl, W, H[b])
        if kv == "fp8mix":
            raw = oracle.norm_rope_rows(
                oracle.compress(H[b], m, W["Wkv_a"], W["Wz_a"], W["B_a"], W["Wkv_b"], W["Wz_b"],
                                W["B_b"]), rd, wl.rope_base, wl.rms_eps, 0.0, float(m))
            check_fp8_records(ckv[b], ckv_s[b], raw, wl, f"{name} kv")
            raw_w = oracle.norm_rope_rows(oracle.matmul(H[b], W["Wkv_a"]), rd, wl.rope_base,
                                          wl.rms_eps, 0.0, 1.0)
            check_fp8_records(win[b], win_s[b], raw_w, wl, f"{name} win")
        else:
            fmt = wl.act if kv != "bf16" else "bf16"
            assert_close(got_kv[b], ref_kv, fmt, f"{name} kv")
            assert_close(got_win[b], ref_win, fmt, f"{name} win")
        if kI is not None:
            assert_close(kI[b].double().cpu().numpy(), ref_kI, wl.act, f"{name} kI")


def test_append_flags_out_of_range_rows():
    """An entry past the cache or a window row outside it is skipped and
    reported in the device error word."""
    wl = BASE.with_(d=64, c=128, rope_dims=32, c_I=32, n_hI=4, m=4, T=8, B=1)
    p = bd.params_for(wl)
    W = synth.weights(wl)
    packed = bd.csa_pack_weights(p, to_dev(W))
    ckv = torch.zeros(1, 1, 128, dtype=torch.bfloat16, device=DEV)
    kI = torch.zeros(1, 1, 32, dtype=torch.bfloat16, device=DEV)
    win = torch.zeros(1, 2, 128, dtype=torch.bfloat16, device=DEV)
    tail = torch.zeros(bd.decode_tail_bytes(p, 1, 64) // 4, dtype=torch.float32, device=DEV)
    h = torch.randn(1, 64, device=DEV).to(torch.bfloat16)
    # token 7 closes block 1, but the cache holds one entry; window rows 0..1
    tt = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    bd.csa_decode_append(p, h, tt, packed, tail, ckv, None, kI, win, None,
                         torch.zeros(1, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    flags = bd.device_status()
    assert flags & 0x1 and flags & 0x2
    assert bd.device_status() == 0


@pytest.mark.parametrize("variant", ["csa", "hca"])
def test_incremental_decode_rolls_the_window(variant):
    """The self-contained decode step: append token t, then select and
    attend for the query at t.  The window holds 2 n_win rows and rolls
    several times; after each checked step the rows of positions
    t-n_win+1..t equal the oracle's window rows, and the attention output
    over the step's caches equals the oracle's."""
    nwin, m = 6, 4
    wl = BASE.with_(variant=variant, act="bf16", kv="bf16", d=64, c=128, rope_dims=32,
                    c_I=32 if variant == "csa" else 0, n_hI=4 if variant == "csa" else 0,
                    n_h=4, m=m, topk=4 if variant == "csa" else 0, n_win=nwin, T=44, B=2,
                    seed=71)
    p = bd.params_for(wl)
    B, T, d = wl.B, wl.T, wl.d
    W = synth.weights(wl)
    H = synth.prefill_inputs(wl)["H"]
    packed = bd.csa_pack_weights(p, to_dev(W))
    nE = T // m
    Wrows = 2 * nwin
    ckv, _ = alloc_kv(wl, (B,), nE)
    win, _ = alloc_kv(wl, (B,), Wrows)
    ckv.zero_()
    win.zero_()
    kI = torch.zeros(B, nE, wl.c_I, dtype=torch.bfloat16, device=DEV) if variant == "csa" else None
    tail = torch.full((bd.decode_tail_bytes(p, B, d) // 4,), float("nan"), device=DEV)
    win_pos0 = torch.zeros(B, dtype=torch.int32, device=DEV)
    g = torch.Generator().manual_seed(5)
    q = torch.randn(T, B, wl.n_h, wl.c, generator=g).to(torch.bfloat16)
    sink = torch.randn(wl.n_h, generator=g)
    if variant == "csa":
        qI = torch.randn(T, B, wl.n_hI, wl.c_I, generator=g).to(torch.bfloat16)
        w = torch.randn(T, B, wl.n_hI, generator=g)
    ref = [P.compress_seq(wl, W, H[b]) for b in range(B)]  # (kv, kI, win) per sequence
    Hd = H.to(DEV)
    checked = {0, 3, 5, 11, 12, 13, 19, 30, 31, 43}
    for t in range(T):
        tt = torch.full((B,), t, dtype=torch.int32, device=DEV)
        h = Hd[:, t, :].contiguous()
        if variant == "csa":
            bd.csa_decode_append(p, h, tt, packed, tail, ckv, None, kI, win, None, win_pos0)
        else:
            bd.hca_decode_append(p, h, tt, packed, tail, ckv, None, win, None, win_pos0)
        if t not in checked:
            continue
        out = torch.empty(B, wl.n_h, wl.c, dtype=torch.bfloat16, device=DEV)
        qd = q[t].to(DEV)
        if variant == "csa":
            idx = torch.empty(B, wl.topk, dtype=torch.int32, device=DEV)
            sco = torch.empty(B, wl.topk, device=DEV)
            bd.csa_index_topk(p, tt, qI[t].to(DEV), w[t].to(DEV), kI, idx, sco)
            bd.csa_attend(p, tt, qd, idx, ckv, None, win, None, win_pos0, sink.to(DEV), out)
        else:
            bd.hca_attend(p, tt, qd, ckv, None, win, None, win_pos0, sink.to(DEV), out)
        torch.cuda.synchronize()
        wp0 = win_pos0.cpu().numpy()
        for b in range(B):
            lo = max(0, t - nwin + 1)
            assert wp0[b] <= lo and t - wp0[b] < Wrows, (t, b, wp0[b])
            got_w = kv_values(wl, win[b].cpu(), None)
            assert_close(got_w[lo - wp0[b]: t - wp0[b] + 1], ref[b][2][lo: t + 1], "bf16",
                         f"{variant} t{t} b{b} window")
            kv_b = kv_values(wl, ckv[b].cpu(), None)
            pos = np.array([t], dtype=np.int32)
            if variant == "csa":
                kIb = kI[b].cpu()
                sref = oracle.index_scores(pos, m, qI[t, b:b + 1], w[t, b:b + 1], kIb)
                tol = score_tolerance(qI[t, b:b + 1].double().numpy(), w[t, b:b + 1].numpy(),
                                      kIb.double().numpy())
                nv = np.array([oracle.nvis(t, m, nE)])
                ig = idx[b:b + 1].cpu().numpy()
                check_topk(ig, sco[b:b + 1].cpu().numpy(), sref, nv, wl.topk, tol,
                           f"t{t} b{b}")
                sel = ig[0][ig[0] >= 0]
                oref, _ = oracle.attend(pos, q[t, b:b + 1], np.arange(len(sel), dtype=np.int32)[None],
                                        m, kv_b[sel], nwin, got_w, int(wp0[b]), sink,
                                        wl.rope_dims, wl.rope_base, wl.softmax_scale)
            else:
                oref, _ = P.attend_wl(wl, pos, q[t, b:b + 1], None, kv_b, got_w, int(wp0[b]), sink)
            assert_close(out[b:b + 1].double().cpu().numpy(), oref, "bf16", f"{variant} t{t} b{b} out")
