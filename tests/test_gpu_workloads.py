"""The benchmark workloads at their full sizes, in the launch configuration
bench.py times, checked against the oracle on sampled outputs it can compute
one by one (whole sequences for decode, sampled entries / tokens / queries
for the 32K prefill)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline as P
from long_context_sparse_09_b200 import binding as bd
from long_context_sparse_09_b200 import synth
from long_context_sparse_09_b200.configs import WORKLOADS
from gpu_util import (DEV, act_dtype, alloc_kv, assert_close, check_topk, kv_values,
                      score_tolerance, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status(cuda_ok):
    bd.device_status()
    yield
    torch.cuda.synchronize()
    assert bd.device_status() == 0


def _rows(t, b, idx=None):
    x = t[b] if idx is None else t[b][idx]
    return x.cpu()


@pytest.mark.parametrize("name", ["flash_csa_decode_64k", "pro_csa_decode_1m"])
def test_csa_decode_full_size(name):
    wl = WORKLOADS[name]
    p = bd.params_for(wl)
    inp = synth.decode_inputs(wl, device=DEV)
    B, N = wl.B, inp["N"]
    idx = torch.empty(B, wl.topk, dtype=torch.int32, device=DEV)
    sco = torch.empty(B, wl.topk, device=DEV)
    out = torch.empty(B, wl.n_h, wl.c, dtype=torch.bfloat16, device=DEV)
    bd.csa_index_topk(p, inp["q_pos"], inp["qI"], inp["w"], inp["kI"], idx, sco)
    bd.csa_attend(p, inp["q_pos"], inp["q"], idx, inp["ckv"], inp["ckv_scale"], inp["win"],
                  inp["win_scale"], inp["win_pos0"], inp["sink"], out)
    torch.cuda.synchronize()
    sink = inp["sink"].cpu()
    for b in (0, B - 1):
        pos = inp["q_pos"][b:b + 1].cpu().numpy()
        qI = inp["qI"][b:b + 1].cpu()
        w = inp["w"][b:b + 1].cpu()
        kI = inp["kI"][b].cpu()
        sref = oracle.index_scores(pos, wl.m, qI, w, kI)
        tol = score_tolerance(qI.double().numpy(), w.numpy(), kI.double().numpy())
        nv = np.array([oracle.nvis(int(pos[0]), wl.m, N)])
        ig = idx[b:b + 1].cpu().numpy()
        check_topk(ig, sco[b:b + 1].cpu().numpy(), sref, nv, wl.topk, tol, f"{name} b{b}")
        sel = torch.from_numpy(ig[0][ig[0] >= 0]).long()
        rows = kv_values(wl, _rows(inp["ckv"], b, sel.to(DEV)),
                         None if inp["ckv_scale"] is None else _rows(inp["ckv_scale"], b, sel.to(DEV)))
        win = kv_values(wl, _rows(inp["win"], b),
                        None if inp["win_scale"] is None else _rows(inp["win_scale"], b))
        ref, _ = oracle.attend(pos, inp["q"][b:b + 1].cpu(), np.arange(len(sel), dtype=np.int32)[None],
                               wl.m, rows, wl.n_win, win, int(inp["win_pos0"][b]), sink,
                               wl.rope_dims, wl.rope_base, wl.softmax_scale)
        assert_close(out[b:b + 1].double().cpu().numpy(), ref, "bf16", f"{name} out b{b}")


def test_hca_decode_full_size():
    wl = WORKLOADS["hca_decode_1m"]
    p = bd.params_for(wl)
    inp = synth.decode_inputs(wl, device=DEV)
    out = torch.empty(wl.B, wl.n_h, wl.c, dtype=torch.bfloat16, device=DEV)
    bd.hca_attend(p, inp["q_pos"], inp["q"], inp["ckv"], None, inp["win"], None,
                  inp["win_pos0"], inp["sink"], out)
    torch.cuda.synchronize()
    for b in (0, wl.B - 1):
        ref, _ = P.attend_wl(wl, inp["q_pos"][b:b + 1].cpu().numpy(), inp["q"][b:b + 1].cpu(), None,
                             inp["ckv"][b].cpu(), inp["win"][b].cpu(), int(inp["win_pos0"][b]),
                             inp["sink"].cpu())
        assert_close(out[b:b + 1].double().cpu().numpy(), ref, "bf16", f"hca b{b}")


def test_csa_prefill_32k_full_size():
    """compress -> index/top-k -> attend over 32,768 tokens; sampled entries,
    window rows and queries against the oracle, stage-isolated."""
    wl = WORKLOADS["flash_csa_prefill_32k"]
    p = bd.params_for(wl)
    W = synth.weights(wl, device=DEV)
    inp = synth.prefill_inputs(wl, device=DEV)
    T, nE = wl.T, wl.T // wl.m
    packed = bd.csa_pack_weights(p, W)
    ckv, _ = alloc_kv(wl, (1,), nE)
    win, _ = alloc_kv(wl, (1,), T)
    kI = torch.empty(1, nE, wl.c_I, dtype=torch.bfloat16, device=DEV)
    bd.csa_compress(p, inp["H"], packed, ckv, None, kI, win, None)
    idx = torch.empty(T, wl.topk, dtype=torch.int32, device=DEV)
    sco = torch.empty(T, wl.topk, device=DEV)
    bd.csa_index_topk(p, inp["q_pos"], inp["qI"], inp["w"], kI, idx, sco)
    out = torch.empty(T, wl.n_h, wl.c, dtype=torch.bfloat16, device=DEV)
    bd.csa_attend(p, inp["q_pos"], inp["q"], idx, ckv, None, win, None,
                  torch.zeros(1, dtype=torch.int32, device=DEV), inp["sink"], out)
    torch.cuda.synchronize()
    Wc = {k: v.cpu() for k, v in W.items()}
    H = inp["H"][0]
    m = wl.m
    # compression: sampled entries (each needs its 2m tokens only)
    for i in (0, 1, 2, 4095, nE - 1):
        lo = max(0, m * (i - 1))
        Hs = H[lo: m * (i + 1)].cpu()
        li = i - lo // m
        raw = oracle.compress(Hs, m, Wc["Wkv_a"], Wc["Wz_a"], Wc["B_a"], Wc["Wkv_b"], Wc["Wz_b"],
                              Wc["B_b"], i0=li, i1=li + 1)
        ref = oracle.norm_rope_rows(raw, wl.rope_dims, wl.rope_base, wl.rms_eps, m * i, m)
        assert_close(ckv[0, i:i + 1].double().cpu().numpy(), ref, "bf16", f"entry {i}")
        rawI = oracle.compress(Hs, m, Wc["WIkv_a"], Wc["WIz_a"], Wc["BI_a"], Wc["WIkv_b"],
                               Wc["WIz_b"], Wc["BI_b"], i0=li, i1=li + 1)
        assert_close(kI[0, i:i + 1].double().cpu().numpy(), rawI, "bf16", f"kI {i}")
    for j in (0, 1, 2047, T - 1):
        ca = oracle.matmul(H[j:j + 1].cpu(), Wc["Wkv_a"])
        ref = oracle.norm_rope_rows(ca, wl.rope_dims, wl.rope_base, wl.rms_eps, j, 1)
        assert_close(win[0, j:j + 1].double().cpu().numpy(), ref, "bf16", f"win {j}")
    # index / top-k on the GPU's keys, attention on the GPU's cache
    qs = np.array([0, 3, 4, 1000, 2047, 16383, T - 2, T - 1])
    kI_h = kI[0].cpu()
    sref = oracle.index_scores(qs, m, inp["qI"][qs].cpu(), inp["w"][qs].cpu(), kI_h)
    tol = score_tolerance(inp["qI"][qs].cpu().double().numpy(), inp["w"][qs].cpu().numpy(),
                          kI_h.double().numpy())
    nv = np.array([oracle.nvis(int(t), m, nE) for t in qs])
    check_topk(idx[qs].cpu().numpy(), sco[qs].cpu().numpy(), sref, nv, wl.topk, tol, "prefill")
    kv_h = ckv[0].cpu()
    win_h = win[0].cpu()
    ref, _ = P.attend_wl(wl, qs, inp["q"][qs].cpu(), idx[qs].cpu().numpy(), kv_h, win_h, 0,
                         inp["sink"].cpu())
    assert_close(out[qs].double().cpu().numpy(), ref, "bf16", "prefill out")
