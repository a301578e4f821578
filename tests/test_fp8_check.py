"""The FP8-mixed record check of the GPU tests (gpu_util.check_fp8_records)
run on the CPU against records written by the oracle's own encoder: it must
accept them when the encoded rows differ from the reference rows by fp32
rounding only, and reject each planted mistake (codes truncated instead of
rounded to nearest, a scale of max|x| / 240 instead of / 448, a scale off by
a factor 1 + 1e-3, RoPE dims truncated to bf16)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_09_b200.configs import WORKLOADS
from gpu_util import check_fp8_records

WL = WORKLOADS["pro_csa_decode_1m"]  # c = 512, 64 RoPE dims


def _rows(seed, n=24):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, WL.c))
    return x / np.sqrt(np.mean(x * x, axis=1, keepdims=True))


def _records(codes, rope_vals, scale):
    rope = torch.from_numpy(np.ascontiguousarray(rope_vals)).to(torch.bfloat16)
    rb = rope.view(torch.uint8).reshape(codes.shape[0], -1)
    rec = torch.cat([torch.from_numpy(np.ascontiguousarray(codes)), rb], dim=1)
    return rec, torch.from_numpy(np.ascontiguousarray(scale, dtype=np.float32))


def _encode_fp32_like(x, seed):
    """The oracle's encoding of a row carrying fp32-sized deviations."""
    rng = np.random.default_rng(seed)
    xg = x * (1.0 + 2.0 ** -24 * rng.standard_normal(x.shape))
    return oracle.fp8mix_encode(xg, WL.rope_dims)


def test_accepts_the_rule_applied_to_an_fp32_row():
    x = _rows(1)
    codes, rope, sc = _encode_fp32_like(x, 2)
    rec, s = _records(codes, rope, sc)
    check_fp8_records(rec, s, x, WL, "exact")


def test_rejects_truncated_codes():
    x = _rows(3)
    nf = WL.c - WL.rope_dims
    codes, rope, sc = oracle.fp8mix_encode(x, WL.rope_dims)
    y = x[:, :nf].astype(np.float32) / sc[:, None]
    tab = np.array([oracle.e4m3_decode(c) for c in range(128)])
    trunc = np.empty_like(codes)
    for i, j in np.ndindex(y.shape):  # largest magnitude not above |y|
        mag = int(np.searchsorted(tab[:127], abs(float(y[i, j])), side="right")) - 1
        trunc[i, j] = mag | (0x80 if y[i, j] < 0 else 0)
    assert np.count_nonzero(trunc != codes) > 0
    rec, s = _records(trunc, rope, sc)
    with pytest.raises(AssertionError, match="E4M3 codes outside"):
        check_fp8_records(rec, s, x, WL, "truncated")


@pytest.mark.parametrize("factor", [448.0 / 240.0, 1.0 + 1e-3])
def test_rejects_a_wrong_scale(factor):
    x = _rows(4)
    nf = WL.c - WL.rope_dims
    _, rope, sc = oracle.fp8mix_encode(x, WL.rope_dims)
    sc2 = (sc * factor).astype(np.float32)
    codes = np.array([[oracle.e4m3_encode(float(np.float32(v) / s)) for v in row[:nf]]
                      for row, s in zip(x, sc2)], dtype=np.uint8)
    rec, s = _records(codes, rope, sc2)
    with pytest.raises(AssertionError, match="scale differs"):
        check_fp8_records(rec, s, x, WL, "scale")


def test_rejects_truncated_rope_dims():
    x = _rows(5)
    nf = WL.c - WL.rope_dims
    codes, _, sc = oracle.fp8mix_encode(x, WL.rope_dims)
    bits = torch.from_numpy(x[:, nf:].astype(np.float32)).view(torch.int32) & ~0xFFFF
    rope_t = bits.view(torch.float32).double().numpy()  # toward zero
    assert np.count_nonzero(rope_t != oracle.round_bf16(x[:, nf:])) > 0
    rec, s = _records(codes, rope_t, sc)
    with pytest.raises(AssertionError, match="RoPE dims"):
        check_fp8_records(rec, s, x, WL, "rope")
