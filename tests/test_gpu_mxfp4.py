"""The MXFP4 indexer ("02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文" 3.3: the
indexer's QK path in FP4, scores in bf16) against the oracle:

* the quantiser (csa_mxfp4_quantize) byte for byte against the oracle's
  MXFP4 encoder, ties, saturation and all-zero blocks included;
* the scores of csa_index_topk_mxfp4 (every visible entry, read back by
  asking for k >= the visible count) against the oracle's exact score of the
  MXFP4-rounded q^I and K^I: each GPU score must be the bf16 rounding of a
  value within the fp32 head-sum bound of the exact one;
* the selection against the oracle's top-k of the GPU's own bf16 scores
  (stage-isolated, element for element: ties to the lower index), and
  against the oracle end to end on integer inputs, where every score is
  exact;
* the 1M-context decode shape (4 x 262,144 entries, k = 1024), with its
  recall of the bf16 indexer's selection reported;
* a block exponent outside the exact range is reported (CSA_DEV_RANGE)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline as P
from long_context_sparse_09_b200 import binding as bd
from long_context_sparse_09_b200.configs import WORKLOADS
from gpu_util import DEV, score_tolerance

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["pro_csa_decode_1m"]


@pytest.fixture(autouse=True)
def _clean_status(cuda_ok):
    bd.device_status()
    yield
    torch.cuda.synchronize()
    assert bd.device_status() == 0


def oracle_pack(x):
    """The oracle's MXFP4 encoding of rows x [rows][width] in the library's
    layout: (codes [rows][width/2], scales [rows][width/32])."""
    x = np.asarray(x, dtype=np.float64)
    rows, width = x.shape
    codes = np.empty((rows, width // 2), np.uint8)
    scales = np.empty((rows, width // 32), np.uint8)
    for r in range(rows):
        c, e = oracle.mxfp4_encode(x[r])
        codes[r] = c[0::2] | (c[1::2] << 4)
        scales[r] = (e + 127).astype(np.uint8)
    return codes, scales


def _special_rows():
    """Blocks of 32 that exercise the rounding rule: every E2M1 midpoint
    (ties to the even mantissa), values above 6 (saturation), negative
    values rounding to zero, an all-zero block, tiny and large scales."""
    rows = []
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 7.5, 6.5, 0.1, 4.0]
    blk = np.array((mids + [-m for m in mids] + [0.0] * 8)[:32])  # amax 7.5: scale 2^0
    rows.append(np.concatenate([blk, blk * 2.0 ** -5, blk * 2.0 ** 9, np.zeros(32)]))
    rows.append(np.concatenate([blk * 0.5, -blk, blk * 2.0 ** -20, blk * 2.0 ** 12]))
    return np.array(rows)


def test_quantize_matches_oracle_bytes():
    g = torch.Generator().manual_seed(11)
    x = torch.randn(300, 128, generator=g) * torch.exp(torch.randn(300, 1, generator=g))
    x = torch.cat([x, torch.from_numpy(_special_rows()).float()]).to(torch.bfloat16)
    codes, scales = bd.mxfp4_quantize(x.to(DEV))
    torch.cuda.synchronize()
    c_ref, s_ref = oracle_pack(x.double().numpy())
    assert np.array_equal(scales.cpu().numpy(), s_ref), "scale bytes differ"
    got = codes.cpu().numpy()
    bad = np.argwhere(got != c_ref)
    assert bad.size == 0, f"code bytes differ at {bad[:5].tolist()}"


def _setup(seed, B, Q, N, nh, k, mode):
    wl = BASE.with_(n_hI=nh, c_I=128, topk=k)
    g = torch.Generator().manual_seed(seed)
    qI = torch.randn(B * Q, nh, 128, generator=g).to(torch.bfloat16)
    w = torch.randn(B * Q, nh, generator=g)
    kI = torch.randn(B, N, 128, generator=g).to(torch.bfloat16)
    if mode == "decode":
        pos = torch.full((B * Q,), wl.m * N, dtype=torch.int32)
    else:
        pos = torch.randint(0, wl.m * N + 8, (B * Q,), generator=g, dtype=torch.int32)
        pos[0] = 0
        pos[-1] = wl.m * N - 1
    return wl, qI, w, kI, pos


def _gpu_scores_all(wl, pos, qI, w, codes, scales, N):
    """Every visible GPU score: the call with k = N returns all visible
    entries in index order with their scores."""
    R = qI.shape[0]
    p = bd.params_for(wl.with_(topk=N))
    idx = torch.empty(R, N, dtype=torch.int32, device=DEV)
    sco = torch.empty(R, N, device=DEV)
    bd.csa_index_topk_mxfp4(p, pos.to(DEV), qI.to(DEV), w.to(DEV), codes, scales, idx, sco)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sco.double().cpu().numpy()


def _check_scores(got_all, idx_all, pos, wl, qI, w, kI_b, what):
    """GPU bf16 scores against the bf16 rounding of the oracle's exact
    score of the MXFP4-rounded inputs, within the fp32 head-sum bound."""
    qr = oracle.mxfp4_round(qI.double().numpy())
    kr = oracle.mxfp4_round(kI_b.double().numpy())
    exact = oracle.index_scores(pos.numpy(), wl.m, qr, w, kr)
    tol = score_tolerance(qr, w.numpy(), kr)
    N = kI_b.shape[0]
    for q in range(got_all.shape[0]):
        nv = oracle.nvis(int(pos[q]), wl.m, N)
        assert np.array_equal(idx_all[q, :nv], np.arange(nv)), f"{what} q{q}: all-visible order"
        if nv == 0:
            continue
        ex, t = exact[q, :nv], tol[q, :nv]
        lo, hi = oracle.round_bf16(ex - t), oracle.round_bf16(ex + t)
        g = got_all[q, :nv]
        bad = (g < lo) | (g > hi)
        assert not bad.any(), (f"{what} q{q}: {int(bad.sum())} scores off, first at "
                               f"{int(np.argmax(bad))}: gpu {g[bad][0]}, exact {ex[bad][0]}")
        assert np.array_equal(g, oracle.round_bf16(g)), f"{what} q{q}: not bf16 values"


MX_CASES = [
    # name, B, Q, N, n_hI, k, positions
    ("decode_ragged", 2, 1, 3001, 64, 512, "decode"),
    ("causal_many", 1, 70, 900, 64, 40, "prefill"),
    ("heads32", 3, 2, 1500, 32, 100, "prefill"),
    ("multi_cta_topk", 2, 1, 40000, 64, 1024, "decode"),
]


@pytest.mark.parametrize("case", MX_CASES, ids=[c[0] for c in MX_CASES])
def test_index_topk_mxfp4_matches_oracle(case):
    name, B, Q, N, nh, k, mode = case
    wl, qI, w, kI, pos = _setup(sum(map(ord, name)), B, Q, N, nh, k, mode)
    codes, scales = bd.mxfp4_quantize(kI.to(DEV))
    idx_all, got_all = _gpu_scores_all(wl, pos, qI, w, codes, scales, N)
    p = bd.params_for(wl)
    idx = torch.empty(B * Q, k, dtype=torch.int32, device=DEV)
    sco = torch.empty(B * Q, k, device=DEV)
    bd.csa_index_topk_mxfp4(p, pos.to(DEV), qI.to(DEV), w.to(DEV), codes, scales, idx, sco)
    torch.cuda.synchronize()
    idx, sco = idx.cpu().numpy(), sco.double().cpu().numpy()
    for b in range(B):
        rows = slice(b * Q, (b + 1) * Q)
        _check_scores(got_all[rows], idx_all[rows], pos[rows], wl, qI[rows], w[rows], kI[b],
                      f"{name} b{b}")
        # the selection: the oracle's top-k of the GPU's own scores, exactly
        nv = np.array([oracle.nvis(int(t), wl.m, N) for t in pos[rows]], np.int32)
        s_gpu = np.where(np.arange(N)[None, :] < nv[:, None], got_all[rows], -np.inf)
        ref_idx, _ = oracle.topk(s_gpu, nv, k)
        assert np.array_equal(idx[rows], ref_idx), f"{name} b{b}: selection differs"
        sel = np.maximum(ref_idx, 0)
        ok = ref_idx >= 0
        assert np.array_equal(sco[rows][ok], np.take_along_axis(s_gpu, sel, 1)[ok])


@pytest.mark.parametrize("B,Q,N,k", [(1, 120, 1200, 64), (2, 1, 20000, 300)])
def test_index_topk_mxfp4_integer_inputs_exact(B, Q, N, k):
    """Integer q^I in {0, 1}, K^I in {-2..2} and w in {0.5, 1}: every value is
    exact in MXFP4 and every score exact in fp32, so the bf16 scores and the
    selection (many ties, lower index first) must equal the oracle's end to
    end, element for element."""
    wl = BASE.with_(n_hI=32, c_I=128, topk=k)
    g = torch.Generator().manual_seed(B * 100 + N)
    qI = torch.randint(0, 2, (B * Q, 32, 128), generator=g).to(torch.bfloat16)
    kI = torch.randint(-2, 3, (B, N, 128), generator=g).to(torch.bfloat16)
    w = torch.randint(1, 3, (B * Q, 32), generator=g).float() * 0.5
    pos = torch.full((B * Q,), 4 * N, dtype=torch.int32)
    if Q > 1:
        pos = torch.randint(4 * k, 4 * N, (B * Q,), generator=g, dtype=torch.int32)
    codes, scales = bd.mxfp4_quantize(kI.to(DEV))
    p = bd.params_for(wl)
    idx = torch.empty(B * Q, k, dtype=torch.int32, device=DEV)
    sco = torch.empty(B * Q, k, device=DEV)
    bd.csa_index_topk_mxfp4(p, pos.to(DEV), qI.to(DEV), w.to(DEV), codes, scales, idx, sco)
    torch.cuda.synchronize()
    for b in range(B):
        rows = slice(b * Q, (b + 1) * Q)
        sref = P.index_scores_fp4(wl, pos[rows].numpy(), qI[rows], w[rows], kI[b])
        nv = np.array([oracle.nvis(int(t), wl.m, N) for t in pos[rows]], np.int32)
        ref_idx, _ = oracle.topk(sref, nv, k)
        assert np.array_equal(idx[rows].cpu().numpy(), ref_idx), f"b{b}: selection differs"
        got = sco[rows].cpu().double().numpy()
        exp = np.take_along_axis(sref, np.maximum(ref_idx, 0), axis=1)
        assert np.array_equal(got[ref_idx >= 0], exp[ref_idx >= 0]), f"b{b}: scores differ"


def test_index_topk_mxfp4_decode_1m_shape():
    """The bench's launch configuration: 4 sequences of 262,144 entries,
    k = 1024.  Scores of 4,096 sampled entries per query against the oracle
    one by one; the selection against the oracle's top-k of the GPU's scores;
    the recall of the bf16 indexer's selection is reported."""
    wl = BASE
    B, N, k = wl.B, wl.T // wl.m, wl.topk
    g = torch.Generator(device=DEV).manual_seed(3)
    qI = torch.randn(B, 64, 128, device=DEV, generator=g).to(torch.bfloat16)
    w = torch.randn(B, 64, device=DEV, generator=g)
    kI = torch.randn(B, N, 128, device=DEV, generator=g).to(torch.bfloat16)
    pos = torch.full((B,), wl.m * N, dtype=torch.int32, device=DEV)
    codes, scales = bd.mxfp4_quantize(kI)
    idx_all, got_all = _gpu_scores_all(wl, pos.cpu(), qI.cpu(), w.cpu(), codes, scales, N)
    p = bd.params_for(wl)
    idx = torch.empty(B, k, dtype=torch.int32, device=DEV)
    bd.csa_index_topk_mxfp4(p, pos, qI, w, codes, scales, idx)
    idx_bf = torch.empty(B, k, dtype=torch.int32, device=DEV)
    bd.csa_index_topk(p, pos, qI, w, kI, idx_bf)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    for b in range(B):
        assert np.array_equal(idx_all[b], np.arange(N))
        smp = np.sort(rng.choice(N, 4096, replace=False))
        kb = kI[b][torch.from_numpy(smp).to(DEV)].cpu()
        pos_s = torch.tensor([wl.m * len(smp)], dtype=torch.int32)
        _check_scores(got_all[b:b + 1, smp], np.arange(len(smp))[None, :], pos_s, wl,
                      qI[b:b + 1].cpu(), w[b:b + 1].cpu(), kb, f"1M b{b}")
        ref_idx, _ = oracle.topk(got_all[b:b + 1], np.array([N], np.int32), k)
        assert np.array_equal(idx[b:b + 1].cpu().numpy(), ref_idx), f"1M b{b}: selection"
    recall = P.topk_recall(idx.cpu().numpy(), idx_bf.cpu().numpy())
    print(f"MXFP4 selection recall of the bf16 top-{k}: {recall.round(4).tolist()}")
    assert recall.min() > 0.5, recall  # a broken path selects near-random entries


def test_index_topk_mxfp4_flags_out_of_range_blocks():
    wl = BASE.with_(n_hI=16, c_I=128, topk=8)
    p = bd.params_for(wl)
    N = 256
    kI = torch.randn(1, N, 128)
    kI[0, 3, 0] = 2.0 ** 17  # block exponent 15 > 13
    codes, scales = bd.mxfp4_quantize(kI.to(torch.bfloat16).to(DEV))
    qI = torch.randn(1, 16, 128).to(torch.bfloat16).to(DEV)
    w = torch.rand(1, 16, device=DEV)
    idx = torch.empty(1, 8, dtype=torch.int32, device=DEV)
    bd.csa_index_topk_mxfp4(p, torch.tensor([4 * N], dtype=torch.int32, device=DEV), qI, w,
                            codes, scales, idx)
    assert bd.device_status() & bd.DEV_RANGE
