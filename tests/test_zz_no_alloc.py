"""csa_index_topk_noalloc, the indexer + top-k entry point for callers that
cannot allocate device memory (a host framework that owns all device memory
and offers its plugins no workspace, or a loop where an allocation would
synchronise the device).  It must give what csa_index_topk gives, call after
call, while taking its scratch from the library's fixed array.

This file is collected last on purpose: a run that stops at the first
failure has then already run every other test."""
import ctypes as C

import numpy as np
import pytest
import torch

from long_context_sparse_09_b200 import binding as bd
from long_context_sparse_09_b200.configs import WORKLOADS
from gpu_util import DEV, score_tolerance

pytestmark = pytest.mark.gpu


def _case(seed, B, Q, N, nh, ci, k, causal):
    g = torch.Generator().manual_seed(seed)
    qI = torch.randn(B * Q, nh, ci, generator=g).to(torch.bfloat16)
    w = torch.randn(B * Q, nh, generator=g)
    kI = torch.randn(B, N, ci, generator=g).to(torch.bfloat16)
    if causal:
        pos = torch.randint(0, 4 * N + 4, (B * Q,), generator=g, dtype=torch.int32)
    else:
        pos = torch.full((B * Q,), 4 * N, dtype=torch.int32)
    return pos, qI, w, kI


@pytest.mark.parametrize("causal", [False, True])
def test_noalloc_matches_allocating_entry_point_twice(cuda_ok, causal):
    base = WORKLOADS["flash_csa_decode_64k"]
    B, Q, N, nh, ci, k = (2, 3, 3001, 64, 128, 512) if not causal else (1, 64, 700, 16, 64, 48)
    p = bd.params_for(base.with_(n_hI=nh, c_I=ci, topk=k))
    bd.device_status()
    for call in range(2):  # two calls in a row, different inputs each time
        pos, qI, w, kI = _case(100 * call + int(causal), B, Q, N, nh, ci, k, causal)
        d = [t.to(DEV) for t in (pos, qI, w, kI)]
        idx_ref = torch.empty(B * Q, k, dtype=torch.int32, device=DEV)
        sco_ref = torch.empty(B * Q, k, device=DEV)
        bd.csa_index_topk(p, *d, idx_ref, sco_ref)
        idx = torch.full((B * Q, k), -7, dtype=torch.int32, device=DEV)
        sco = torch.full((B * Q, k), float("nan"), device=DEV)
        bd.csa_index_topk_noalloc(p, *d, idx, sco)
        torch.cuda.synchronize()
        assert bd.device_status() == 0
        assert torch.equal(idx.cpu(), idx_ref.cpu()), f"call {call}: indices differ"
        # scores within the fp32 accumulation tolerance the parity tests use
        s, s_ref = sco.cpu().double().numpy(), sco_ref.cpu().double().numpy()
        valid = idx_ref.cpu().numpy() >= 0
        for b in range(B):
            rows = slice(b * Q, (b + 1) * Q)
            tol = score_tolerance(qI[rows].double().numpy(), w[rows].numpy(),
                                  kI[b].double().numpy())
            sel = np.where(valid[rows], idx_ref[rows].cpu().numpy(), 0)
            t = np.take_along_axis(tol, sel, axis=1)
            vr = valid[rows]
            diff = np.abs(s[rows][vr] - s_ref[rows][vr])
            assert np.all(diff <= t[vr]), f"call {call}: scores differ"
            # padded slots (fewer visible entries than k) hold the same value
            # in both outputs (the no-alloc output starts as NaN)
            assert np.array_equal(s[rows][~vr], s_ref[rows][~vr]), f"call {call}: padding"


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_ok):
    base = WORKLOADS["pro_csa_decode_1m"]
    p = bd.params_for(base)
    fake = C.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    # 32 sequences x 262,144 entries of fp32 scores = 32 MiB > 16 MiB
    st = bd.lib().csa_index_topk_noalloc(C.byref(p), 32, 1, fake, fake, fake, fake, 262144,
                                         fake, None, None)
    assert st == 8  # CSA_ERR_WORKSPACE
