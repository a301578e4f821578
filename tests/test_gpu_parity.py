"""GPU parity of every step of the CSA / HCA forward pass against the fp64
CPU oracle, through the C ABI (binding -> libcsa.so).  Stage-isolated: each
GPU stage and the oracle get the same upstream tensors, so rounding in one
stage cannot flip a later decision.  Sizes span several tiles and ragged
tails; edge cases cover empty visibility, fewer visible entries than k,
split and unsplit attention, and every KV format."""
import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline as P
from long_context_sparse_09_b200 import binding as bd
from long_context_sparse_09_b200 import synth
from long_context_sparse_09_b200.configs import WORKLOADS
from gpu_util import (DEV, act_dtype, alloc_kv, assert_close, check_fp8_records, check_topk,
                      kv_values, score_tolerance, to_dev)

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["flash_csa_decode_64k"]


@pytest.fixture(autouse=True)
def _clean_status(cuda_ok):
    bd.device_status()
    yield
    torch.cuda.synchronize()
    assert bd.device_status() == 0


def _gen(seed):
    return torch.Generator().manual_seed(seed)


# ------------------------------------------------------------ index/top-k --

INDEX_CASES = [
    # name, act, B, Q, N, n_hI, c_I, k, positions
    ("f32_small", "f32", 2, 5, 1037, 4, 32, 16, "decode"),
    ("bf16_ragged", "bf16", 2, 3, 3001, 64, 128, 512, "decode"),
    ("bf16_causal", "bf16", 1, 300, 300, 64, 128, 32, "prefill"),
    ("bf16_few_visible", "bf16", 3, 4, 200, 8, 64, 128, "prefill"),
    ("bf16_h16_groups", "bf16", 2, 8, 900, 16, 64, 40, "prefill"),
    ("bf16_h32_decode", "bf16", 5, 2, 2500, 32, 64, 64, "decode"),
    ("bf16_multi_cta_topk", "bf16", 3, 1, 50000, 64, 128, 1024, "decode"),
    ("bf16_multi_cta_ragged", "bf16", 2, 2, 9001, 64, 128, 300, "prefill"),
]


@pytest.mark.parametrize("case", INDEX_CASES, ids=[c[0] for c in INDEX_CASES])
def test_index_topk_parity(case):
    name, act, B, Q, N, nh, ci, k, mode = case
    wl = BASE.with_(act=act, n_hI=nh, c_I=ci, topk=k)
    p = bd.params_for(wl)
    g = _gen(sum(map(ord, name)))
    dt = act_dtype(wl)
    qI = torch.randn(B * Q, nh, ci, generator=g).to(dt)
    w = torch.randn(B * Q, nh, generator=g)
    kI = torch.randn(B, N, ci, generator=g).to(dt)
    if mode == "decode":
        pos = torch.full((B * Q,), wl.m * N, dtype=torch.int32)
    else:  # causal prefill positions including t0 < m-1 (nothing visible)
        pos = torch.randint(0, wl.m * N + 8, (B * Q,), generator=g, dtype=torch.int32)
        pos[0] = 0
        pos[-1] = wl.m * N - 1
    idx = torch.empty(B * Q, k, dtype=torch.int32, device=DEV)
    sco = torch.empty(B * Q, k, dtype=torch.float32, device=DEV)
    bd.csa_index_topk(p, pos.to(DEV), qI.to(DEV), w.to(DEV), kI.to(DEV), idx, sco)
    torch.cuda.synchronize()
    for b in range(B):
        rows = slice(b * Q, (b + 1) * Q)
        sref = oracle.index_scores(pos[rows].numpy(), wl.m, qI[rows], w[rows], kI[b])
        nv = np.array([oracle.nvis(t, wl.m, N) for t in pos[rows].numpy()])
        tol = score_tolerance(qI[rows].double().numpy(), w[rows].numpy(), kI[b].double().numpy())
        check_topk(idx[rows].cpu().numpy(), sco[rows].cpu().numpy(), sref, nv, k, tol, name)


@pytest.mark.parametrize("nh,N", [(8, 1000), (8, 3000), (64, 20000)])
def test_index_topk_all_ties_take_lowest_indices(nh, N):
    """w = 0: every score is 0, the selection is 0..k-1 (lower index wins);
    the long case overflows the multi-CTA candidate list on purpose."""
    wl = BASE.with_(n_hI=nh, c_I=64, topk=100)
    p = bd.params_for(wl)
    qI = torch.randn(2, nh, 64).to(torch.bfloat16).to(DEV)
    w = torch.zeros(2, nh, device=DEV)
    kI = torch.randn(2, N, 64).to(torch.bfloat16).to(DEV)
    pos = torch.full((2,), 4 * N, dtype=torch.int32, device=DEV)
    idx = torch.empty(2, 100, dtype=torch.int32, device=DEV)
    bd.csa_index_topk(p, pos, qI, w, kI, idx)
    assert torch.equal(idx.cpu(), torch.arange(100, dtype=torch.int32).repeat(2, 1))


@pytest.mark.parametrize("B,Q,N,k", [(1, 200, 2000, 64), (2, 1, 20000, 300)])
def test_index_topk_integer_scores_exact(B, Q, N, k):
    """Small-integer q^I, K^I and w: every score is exact in fp32, so many
    scores tie at the k-th value and the selection must equal the oracle's
    (ties to the lower index) element for element.  Covers the per-query
    and the multi-CTA top-k."""
    wl = BASE.with_(n_hI=16, c_I=64, topk=k)
    p = bd.params_for(wl)
    g = _gen(B * 1000 + N)
    qI = torch.randint(0, 2, (B * Q, 16, 64), generator=g).to(torch.bfloat16)
    kI = torch.randint(-2, 3, (B, N, 64), generator=g).to(torch.bfloat16)
    w = torch.randint(1, 3, (B * Q, 16), generator=g).float() * 0.5
    pos = torch.full((B * Q,), 4 * N, dtype=torch.int32)
    if Q > 1:
        pos = torch.randint(4 * k, 4 * N, (B * Q,), generator=g, dtype=torch.int32)
    idx = torch.empty(B * Q, k, dtype=torch.int32, device=DEV)
    sco = torch.empty(B * Q, k, dtype=torch.float32, device=DEV)
    bd.csa_index_topk(p, pos.to(DEV), qI.to(DEV), w.to(DEV), kI.to(DEV), idx, sco)
    torch.cuda.synchronize()
    for b in range(B):
        rows = slice(b * Q, (b + 1) * Q)
        sref = oracle.index_scores(pos[rows].numpy(), wl.m, qI[rows], w[rows], kI[b])
        nv = np.array([oracle.nvis(t, wl.m, N) for t in pos[rows].numpy()], np.int32)
        ref_idx, _ = oracle.topk(sref, nv, k)
        assert np.array_equal(idx[rows].cpu().numpy(), ref_idx), f"b{b}: selection differs"
        got = sco[rows].cpu().numpy()
        exp = np.take_along_axis(sref, np.maximum(ref_idx, 0), axis=1)
        assert np.array_equal(got[ref_idx >= 0], exp[ref_idx >= 0]), f"b{b}: scores differ"


# ---------------------------------------------------------------- attend --

def _rand_idx(g, pos, m, N, k):
    rows = []
    for t in pos.tolist():
        nv = min(N, (t + 1) // m) if t >= 0 else 0
        if nv <= k:
            r = list(range(nv)) + [-1] * (k - nv)
        else:
            r = sorted(torch.randperm(nv, generator=g)[:k].tolist())
        rows.append(r)
    return torch.tensor(rows, dtype=torch.int32)


ATTN_CASES = [
    # name, variant, act, kv, B, Q, N, n_h, c, rope, m, k, n_win, mode
    ("csa_bf16_decode_split", "csa", "bf16", "bf16", 3, 1, 2000, 16, 512, 64, 4, 64, 128, "decode"),
    ("csa_fp8_decode", "csa", "bf16", "fp8mix", 2, 1, 1500, 32, 512, 64, 4, 96, 128, "decode"),
    ("csa_f32_prefill", "csa", "f32", "f32", 1, 200, 64, 8, 128, 32, 4, 16, 16, "prefill"),
    ("csa_bf16_prefill_many", "csa", "bf16", "bf16", 1, 700, 300, 16, 512, 64, 4, 32, 128, "prefill"),
    # many queries, one key slice each (keys on M): several 72-key tiles with
    # a ragged last one, 64 and 2 x 64 heads, dense HCA rows by TMA boxes
    ("csa_bf16_prefill_h64_tiles", "csa", "bf16", "bf16", 1, 300, 400, 64, 512, 64, 4, 200, 128, "prefill"),
    ("csa_bf16_prefill_h128_2seq", "csa", "bf16", "bf16", 2, 100, 300, 128, 512, 64, 4, 96, 128, "prefill"),
    # FP8-mixed rows (64-key tiles) over more single-slice queries than SMs
    ("csa_fp8_prefill_many", "csa", "bf16", "fp8mix", 1, 300, 400, 64, 512, 64, 4, 96, 128, "prefill"),
    ("hca_bf16_prefill_many", "hca", "bf16", "bf16", 1, 200, 300, 32, 512, 64, 4, 0, 128, "prefill"),
    # no window: queries before the first complete entry have no key at all
    # (all weight on the sink), interleaved with the others in each CTA's
    # walk over more queries than SMs
    ("hca_bf16_prefill_nowin", "hca", "bf16", "bf16", 1, 400, 24, 16, 512, 64, 4, 0, 0, "prefill"),
    # few queries at random positions: key slices of a cluster that hold no keys
    ("csa_bf16_split_ragged", "csa", "bf16", "bf16", 2, 3, 600, 16, 512, 64, 4, 64, 128, "prefill"),
    ("csa_fp8_split_ragged", "csa", "bf16", "fp8mix", 1, 5, 900, 64, 512, 64, 4, 128, 128, "prefill"),
    # two head blocks of 64 (bf16 48-key tiles, clusters of slices)
    ("csa_bf16_h128_decode", "csa", "bf16", "bf16", 2, 1, 3000, 128, 512, 64, 4, 256, 128, "decode"),
    ("hca_bf16_decode", "hca", "bf16", "bf16", 2, 1, 300, 16, 512, 64, 128, 0, 128, "decode"),
    ("hca_f32_prefill", "hca", "f32", "f32", 1, 150, 20, 4, 128, 32, 8, 0, 16, "prefill"),
    ("hca_fp8_decode", "hca", "bf16", "fp8mix", 2, 1, 260, 16, 512, 64, 128, 0, 128, "decode"),
]


@pytest.mark.parametrize("case", ATTN_CASES, ids=[c[0] for c in ATTN_CASES])
def test_attend_parity(case):
    name, variant, act, kv, B, Q, N, nh, c, rd, m, k, nwin, mode = case
    wl = BASE.with_(variant=variant, act=act, kv=kv, n_h=nh, c=c, rope_dims=rd, m=m,
                    topk=k, n_win=nwin, n_hI=0 if variant == "hca" else 8,
                    c_I=0 if variant == "hca" else 32, seed=len(name))
    p = bd.params_for(wl)
    g = _gen(len(name) * 7)
    st = synth._Streams(wl.seed, "cpu")
    ckv, ckv_s = synth.cache_rows(wl, st, "ckv", (B,), N)
    if mode == "decode":
        L = m * N + (m - 1)
        pos = torch.full((B * Q,), L, dtype=torch.int32)
        W = nwin
        win_pos0 = torch.full((B,), L - nwin + 1, dtype=torch.int32)
    else:
        T = m * N + 5
        pos = torch.randint(0, T, (B * Q,), generator=g, dtype=torch.int32)
        pos[0] = 0
        pos[1] = min(T - 1, m - 1)
        W = T
        win_pos0 = torch.zeros(B, dtype=torch.int32)
    win, win_s = synth.cache_rows(wl, st, "win", (B,), W)
    q = torch.randn(B * Q, nh, c, generator=g).to(act_dtype(wl))
    sink = torch.randn(nh, generator=g)
    out = torch.empty(B * Q, nh, c, dtype=act_dtype(wl), device=DEV)
    dv = lambda t: None if t is None else t.to(DEV)
    if variant == "csa":
        idx = _rand_idx(g, pos, m, N, k)
        bd.csa_attend(p, dv(pos), dv(q), dv(idx), dv(ckv), dv(ckv_s), dv(win), dv(win_s),
                      dv(win_pos0), dv(sink), out)
    else:
        idx = None
        bd.hca_attend(p, dv(pos), dv(q), dv(ckv), dv(ckv_s), dv(win), dv(win_s), dv(win_pos0),
                      dv(sink), out)
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    kvv = kv_values(wl, ckv, ckv_s)
    wv = kv_values(wl, win, win_s)
    for b in range(B):
        rows = slice(b * Q, (b + 1) * Q)
        ref, mass = P.attend_wl(wl, pos[rows].numpy(), q[rows], None if idx is None else idx[rows],
                                kvv[b], wv[b], int(win_pos0[b]), sink)
        assert_close(got[rows], ref, wl.act, f"{name} b{b}")


def test_attend_flags_out_of_range_index():
    """An index >= the visible entries is skipped and reported in the device
    error word (never dereferenced)."""
    wl = BASE.with_(n_h=16, topk=8)
    p = bd.params_for(wl)
    N = 64
    ckv = torch.randn(1, N, 512).to(torch.bfloat16).to(DEV)
    win = torch.randn(1, 128, 512).to(torch.bfloat16).to(DEV)
    q = torch.randn(1, 16, 512).to(torch.bfloat16).to(DEV)
    pos = torch.tensor([4 * N - 1], dtype=torch.int32, device=DEV)
    idx = torch.tensor([[0, 1, 2, 3, 4, 5, 6, 10_000]], dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    bd.csa_attend(p, pos, q, idx, ckv, None, win,
                  None, torch.tensor([4 * N - 128], dtype=torch.int32, device=DEV),
                  torch.zeros(16, device=DEV), out)
    assert bd.device_status() & bd.DEV_BAD_INDEX


# -------------------------------------------------------------- compress --

COMP_CASES = [
    # name, variant, act, kv, B, T, d, c, rope, c_I, m
    ("csa_f32", "csa", "f32", "f32", 1, 259, 96, 128, 32, 32, 4),
    ("csa_bf16", "csa", "bf16", "bf16", 2, 130, 256, 512, 64, 128, 4),
    ("csa_fp8", "csa", "bf16", "fp8mix", 1, 64, 128, 512, 64, 64, 4),
    ("hca_bf16", "hca", "bf16", "bf16", 2, 100, 128, 128, 32, 0, 16),
    ("hca_f32", "hca", "f32", "f32", 1, 77, 64, 64, 16, 0, 8),
    # the GEMM with the fold epilogue: overlapping row tiles across two
    # sequences with ragged ends, m = 8 (15 entries a tile), HCA m' = 128
    ("csa_fp8_two_seq", "csa", "bf16", "fp8mix", 2, 250, 192, 512, 64, 128, 4),
    ("csa_m8_bf16", "csa", "bf16", "bf16", 1, 200, 128, 256, 64, 64, 8),
    ("hca_m128_bf16", "hca", "bf16", "bf16", 2, 300, 128, 256, 64, 0, 128),
]


@pytest.mark.parametrize("case", COMP_CASES, ids=[c[0] for c in COMP_CASES])
def test_compress_parity(case):
    name, variant, act, kv, B, T, d, c, rd, ci, m = case
    wl = BASE.with_(variant=variant, act=act, kv=kv, d=d, c=c, rope_dims=rd, c_I=ci,
                    n_hI=4 if ci else 0, m=m, T=T, B=B, seed=len(name) + 11)
    p = bd.params_for(wl)
    W = synth.weights(wl)
    H = synth.prefill_inputs(wl)["H"]
    Wd = to_dev(W)
    packed = bd.csa_pack_weights(p, Wd)
    nE = T // m
    ckv, ckv_s = alloc_kv(wl, (B,), nE)
    win, win_s = alloc_kv(wl, (B,), T)
    if variant == "csa":
        kI = torch.empty(B, nE, ci, dtype=act_dtype(wl), device=DEV)
        bd.csa_compress(p, H.to(DEV), packed, ckv, ckv_s, kI, win, win_s)
    else:
        kI = None
        bd.hca_compress(p, H.to(DEV), packed, ckv, ckv_s, win, win_s)
    torch.cuda.synchronize()
    got_kv = kv_values(wl, ckv, ckv_s)
    got_win = kv_values(wl, win, win_s)
    for b in range(B):
        ref_kv, ref_kI, ref_win = P.compress_seq(wl, W, H[b])
        if wl.kv == "fp8mix":
            # the stored records against the oracle's encoding of its own
            # unquantised rows: scale and E4M3 codes exact up to the rounding
            # band of the two sides' fp32 / fp64 rows
            raw = (oracle.norm_rope_rows(_raw_entries(wl, W, H[b]), rd, wl.rope_base, wl.rms_eps,
                                         0.0, float(m)))
            check_fp8_records(ckv[b], ckv_s[b], raw, wl, f"{name} kv")
            raw_w = oracle.norm_rope_rows(oracle.matmul(H[b], W["Wkv_a"]), rd, wl.rope_base,
                                          wl.rms_eps, 0.0, 1.0)
            check_fp8_records(win[b], win_s[b], raw_w, wl, f"{name} win")
        else:
            assert_close(got_kv[b], ref_kv, wl.act if wl.kv != "bf16" else "bf16", f"{name} kv")
            assert_close(got_win[b], ref_win, wl.act if wl.kv != "bf16" else "bf16", f"{name} win")
        if kI is not None:
            assert_close(kI[b].double().cpu().numpy(), ref_kI, wl.act, f"{name} kI")


def _raw_entries(wl, W, H):
    return oracle.compress(H, wl.m, W["Wkv_a"], W["Wz_a"], W["B_a"], W.get("Wkv_b"),
                           W.get("Wz_b"), W.get("B_b"))


# ------------------------------------------------- end to end, fp32 tiny --

def test_e2e_tiny_prefill_f32():
    """The fp32 workload end to end: compress -> index/top-k -> attend on the
    GPU against the oracle pipeline (tolerance 1e-5)."""
    wl = WORKLOADS["tiny_csa_prefill_f32"]
    p = bd.params_for(wl)
    W = synth.weights(wl)
    inp = synth.prefill_inputs(wl)
    d = to_dev(inp)
    packed = bd.csa_pack_weights(p, to_dev(W))
    T, nE = wl.T, wl.T // wl.m
    ckv, _ = alloc_kv(wl, (1,), nE)
    win, _ = alloc_kv(wl, (1,), T)
    kI = torch.empty(1, nE, wl.c_I, device=DEV)
    bd.csa_compress(p, d["H"], packed, ckv, None, kI, win, None)
    idx = torch.empty(T, wl.topk, dtype=torch.int32, device=DEV)
    sco = torch.empty(T, wl.topk, device=DEV)
    bd.csa_index_topk(p, d["q_pos"], d["qI"], d["w"], kI, idx, sco)
    out = torch.empty(T, wl.n_h, wl.c, device=DEV)
    bd.csa_attend(p, d["q_pos"], d["q"], idx, ckv, None, win, None,
                  torch.zeros(1, dtype=torch.int32, device=DEV), d["sink"], out)
    torch.cuda.synchronize()
    ref_kv, ref_kI, ref_win = P.compress_seq(wl, W, inp["H"][0])
    assert_close(ckv[0].double().cpu().numpy(), ref_kv, "f32", "kv")
    assert_close(kI[0].double().cpu().numpy(), ref_kI, "f32", "kI")
    assert_close(win[0].double().cpu().numpy(), ref_win, "f32", "win")
    t0s = inp["q_pos"].numpy()
    # top-k, stage-isolated: oracle scores on the GPU's stored keys
    kI_g = kI[0].double().cpu().numpy()
    sref = oracle.index_scores(t0s, wl.m, inp["qI"], inp["w"], kI_g)
    nv = np.array([oracle.nvis(t, wl.m, nE) for t in t0s])
    tol = score_tolerance(inp["qI"].numpy(), inp["w"].numpy(), kI_g)
    check_topk(idx.cpu().numpy(), sco.cpu().numpy(), sref, nv, wl.topk, tol, "e2e")
    # attention with the GPU's (validated) selection
    ref_out, _ = P.attend_wl(wl, t0s, inp["q"], idx.cpu().numpy(), ref_kv, ref_win, 0, inp["sink"])
    assert_close(out.double().cpu().numpy(), ref_out, "f32", "out")
