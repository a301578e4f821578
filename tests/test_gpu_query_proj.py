"""Query-side projections (csa_query_proj) against the oracle
("DeepSeekV4技术报告阅读笔记" eq. 13-15 and 18, 2.5.1-2.5.2): the latent c^Q
and the head weights w from h, then q^I and the normalised, rotated q from
the GPU's own (bf16) c^Q -- stage-isolated through the oracle with W^{DQ}
the identity -- then end to end against the oracle with the latent rounded
to bf16.  Several tiles, ragged feature counts (zero-padded weight rows),
one and two chunks of 16 tokens, and the V4-Flash and V4-Pro shapes at the
bench's token counts."""
import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline as P
from long_context_sparse_09_b200 import binding as bd
from long_context_sparse_09_b200.configs import WORKLOADS
from gpu_util import DEV, U32, assert_close

pytestmark = pytest.mark.gpu

CASES = [
    # name, R, d, d_c, n_h, c, rope, n_hI, c_I
    ("small", 5, 256, 128, 4, 128, 32, 4, 64),
    ("two_chunks_ragged", 17, 512, 192, 6, 64, 16, 8, 32),
    ("flash_decode_shape", 32, 4096, 1024, 64, 512, 64, 64, 128),
    ("pro_decode_shape", 4, 7168, 1536, 128, 512, 64, 64, 128),
]


@pytest.fixture(autouse=True)
def _clean_status(cuda_ok):
    bd.device_status()
    yield
    torch.cuda.synchronize()
    assert bd.device_status() == 0


def _bf(x):
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_query_proj_matches_oracle(case):
    name, R, d, d_c, n_h, c, rd, n_hI, c_I = case
    wl = WORKLOADS["flash_csa_decode_64k"].with_(d=d, d_c=d_c, n_h=n_h, c=c, rope_dims=rd,
                                                 n_hI=n_hI, c_I=c_I)
    p = bd.params_for(wl)
    g = torch.Generator().manual_seed(R * 7919 + d)
    H = _bf(torch.randn(R, d, generator=g))
    WDQ = _bf(torch.randn(d, d_c, generator=g) / d ** 0.5)
    Ww = _bf(torch.randn(d, n_hI, generator=g) / d ** 0.5)
    WUQ = _bf(torch.randn(d_c, n_h * c, generator=g) / d_c ** 0.5)
    WIUQ = _bf(torch.randn(d_c, n_hI * c_I, generator=g) / d_c ** 0.5)
    pos = torch.randint(0, 1 << 20, (R,), generator=g, dtype=torch.int32)
    packed = bd.query_proj_pack(p, WDQ.to(DEV), Ww.to(DEV), WUQ.to(DEV), WIUQ.to(DEV))
    cQ = torch.empty(R, d_c, dtype=torch.bfloat16, device=DEV)
    q = torch.empty(R, n_h, c, dtype=torch.bfloat16, device=DEV)
    qI = torch.empty(R, n_hI, c_I, dtype=torch.bfloat16, device=DEV)
    w = torch.empty(R, n_hI, device=DEV)
    bd.csa_query_proj(p, H.to(DEV), pos.to(DEV), packed, d_c, cQ, q, qI, w)
    torch.cuda.synchronize()
    Hd = H.double().numpy()
    cQ_ref, _, _, w_ref = P.query_proj(Hd, pos.numpy(), WDQ, WUQ, WIUQ, Ww, n_h, c, n_hI,
                                       c_I, rd, wl.rope_base, wl.rms_eps)
    # stage 1: the latent (stored bf16) and the head weights (fp32, within
    # the first-order bound of fp32 accumulation of d products, 4x margin)
    assert_close(cQ.double().cpu().numpy(), cQ_ref, "bf16", f"{name} cQ")
    w_tol = 4.0 * d * U32 * (np.abs(Hd) @ np.abs(Ww.double().numpy())) + 1e-30
    w_err = np.abs(w.double().cpu().numpy() - w_ref)
    assert np.all(w_err <= w_tol), f"{name} w: {w_err.max():.3g}"
    # stage 2 from the GPU's own latent: W^{DQ} = I makes the oracle's c^Q
    # exactly the GPU's
    cQ_g = cQ.double().cpu().numpy()
    _, q_ref, qI_ref, _ = P.query_proj(cQ_g, pos.numpy(), np.eye(d_c), WUQ, WIUQ,
                                       np.zeros((d_c, n_hI)), n_h, c, n_hI, c_I, rd,
                                       wl.rope_base, wl.rms_eps)
    assert_close(qI.double().cpu().numpy(), qI_ref, "bf16", f"{name} qI")
    assert_close(q.double().cpu().numpy(), q_ref, "bf16", f"{name} q")
    # end to end, the oracle rounding its latent as the GPU stores it
    _, q_e, qI_e, _ = P.query_proj(Hd, pos.numpy(), WDQ, WUQ, WIUQ, Ww, n_h, c, n_hI, c_I, rd,
                                   wl.rope_base, wl.rms_eps, round_mid=True)
    assert_close(q.double().cpu().numpy(), q_e, "bf16", f"{name} q end to end")
    assert_close(qI.double().cpu().numpy(), qI_e, "bf16", f"{name} qI end to end")
    # the heads are unit-RMS after the norm (RoPE keeps it), to bf16 rounding
    ms = (q.double().cpu().numpy() ** 2).mean(axis=2)
    assert np.all(np.abs(ms - 1.0) <= 1e-2), f"{name}: head mean squares {ms.min()}..{ms.max()}"
