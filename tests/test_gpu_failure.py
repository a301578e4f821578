"""Failure detection on the GPU without a fault: the bounded mbarrier wait
every kernel of the library uses is made to run out (a barrier no thread
arrives at, a 1 ms limit, nothing asynchronous in flight); the kernel must
return, report CSA_DEV_TIMEOUT in the device error word, release its TMEM,
and leave the context usable -- the next library call is clean and matches
the oracle."""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_09_b200 import binding as bd
from long_context_sparse_09_b200.configs import WORKLOADS
from gpu_util import DEV, check_topk, score_tolerance

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports(cuda_ok):
    bd.device_status()
    waited = torch.zeros(1, dtype=torch.int64, device=DEV)
    bd.diag_bounded_wait(1_000_000, arrive=False, waited=waited)  # 1 ms, nobody arrives
    torch.cuda.synchronize()
    assert bd.device_status() == bd.DEV_TIMEOUT
    ns = int(waited.item())
    assert 1_000_000 <= ns < 1_000_000_000, ns
    # twice in a row: the TMEM of the first probe was released
    bd.diag_bounded_wait(1_000_000, arrive=False)
    torch.cuda.synchronize()
    assert bd.device_status() == bd.DEV_TIMEOUT


def test_bounded_wait_that_completes_reports_nothing(cuda_ok):
    bd.device_status()
    waited = torch.zeros(1, dtype=torch.int64, device=DEV)
    bd.diag_bounded_wait(200_000_000, arrive=True, waited=waited)  # arrival after 20 ms
    torch.cuda.synchronize()
    assert bd.device_status() == 0
    assert int(waited.item()) < 200_000_000


def test_library_is_usable_after_a_timeout(cuda_ok):
    bd.diag_bounded_wait(1_000_000, arrive=False)
    torch.cuda.synchronize()
    assert bd.device_status() == bd.DEV_TIMEOUT
    wl = WORKLOADS["flash_csa_decode_64k"].with_(n_hI=64, c_I=128, topk=64)
    p = bd.params_for(wl)
    g = torch.Generator().manual_seed(5)
    B, N = 2, 3000
    qI = torch.randn(B, 64, 128, generator=g).to(torch.bfloat16)
    w = torch.randn(B, 64, generator=g)
    kI = torch.randn(B, N, 128, generator=g).to(torch.bfloat16)
    pos = torch.full((B,), 4 * N, dtype=torch.int32)
    idx = torch.empty(B, 64, dtype=torch.int32, device=DEV)
    sco = torch.empty(B, 64, device=DEV)
    bd.csa_index_topk(p, pos.to(DEV), qI.to(DEV), w.to(DEV), kI.to(DEV), idx, sco)
    torch.cuda.synchronize()
    assert bd.device_status() == 0
    for b in range(B):
        sref = oracle.index_scores(pos[b:b + 1].numpy(), wl.m, qI[b:b + 1], w[b:b + 1], kI[b])
        tol = score_tolerance(qI[b:b + 1].double().numpy(), w[b:b + 1].numpy(),
                              kI[b].double().numpy())
        check_topk(idx[b:b + 1].cpu().numpy(), sco[b:b + 1].cpu().numpy(), sref,
                   np.array([N]), 64, tol, f"after timeout b{b}")


def test_bounded_wait_rejects_bad_limits():
    assert bd.lib().csa_diag_bounded_wait(0, 0, None, None) == 1
    assert bd.lib().csa_diag_bounded_wait(3_000_000_000, 0, None, None) == 1
    assert bd.lib().csa_diag_bounded_wait(1000, 2, None, None) == 1
