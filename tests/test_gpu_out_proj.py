"""Grouped output projection (csa_out_proj) against the oracle
("DeepSeekV4技术报告阅读笔记" 2.3.3; PaperTrace 2.2): the group outputs Y
(bf16) stage by stage, then the layer output from the GPU's own Y, then end
to end; several tiles, ragged feature and token counts, one and two chunks of
16 tokens, and the V4-Flash and V4-Pro shapes."""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_09_b200 import binding as bd
from gpu_util import DEV, assert_close

pytestmark = pytest.mark.gpu

CASES = [
    # name, R, n_h, c, g, d_g, d
    ("small", 3, 8, 64, 2, 128, 200),
    ("two_chunks", 17, 16, 64, 4, 256, 96),
    ("one_group", 5, 4, 64, 1, 128, 136),
    ("flash", 2, 64, 512, 8, 1024, 4096),
    ("pro", 1, 128, 512, 16, 1024, 7168),
    # the bench's launch configurations: 4 tokens of V4-Pro, 32 of V4-Flash
    ("pro_decode_shape", 4, 128, 512, 16, 1024, 7168),
    ("flash_decode_shape", 32, 64, 512, 8, 1024, 4096),
]


@pytest.fixture(autouse=True)
def _clean_status(cuda_ok):
    bd.device_status()
    yield
    torch.cuda.synchronize()
    assert bd.device_status() == 0


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_out_proj_matches_oracle(case):
    name, R, n_h, c, g, d_g, d = case
    gen = torch.Generator().manual_seed(R * 1000 + d)
    Kg = c * n_h // g
    O = torch.randn(R, n_h, c, generator=gen).to(torch.bfloat16)
    WG = (torch.randn(g, Kg, d_g, generator=gen) / Kg ** 0.5).to(torch.bfloat16)
    WO = (torch.randn(g * d_g, d, generator=gen) / (g * d_g) ** 0.5).to(torch.bfloat16)
    packed = bd.out_proj_pack(WG.to(DEV), WO.to(DEV))
    ws = torch.empty(bd.out_proj_workspace_bytes(R, n_h, c, g, d_g, d), dtype=torch.uint8,
                     device=DEV)
    out = torch.empty(R, d, dtype=torch.bfloat16, device=DEV)
    bd.csa_out_proj(O.to(DEV), packed, g, d_g, out, workspace=ws)
    torch.cuda.synchronize()
    Y_gpu = ws[:R * g * d_g * 2].view(torch.bfloat16).view(R, g * d_g).double().cpu().numpy()
    Y_ref, out_ref = oracle.group_out_proj(O, WG, WO, round_mid=True)
    assert_close(Y_gpu, Y_ref, "bf16", f"{name} Y")
    # stage-isolated: the output projection of the GPU's own Y
    assert_close(out.double().cpu().numpy(), Y_gpu @ WO.double().numpy(), "bf16", f"{name} out")
    assert_close(out.double().cpu().numpy(), out_ref, "bf16", f"{name} end to end")
