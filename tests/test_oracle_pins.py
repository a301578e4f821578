"""Pins of the CPU oracle against facts other than its own code: the OCP E4M3
and bf16 definitions as implemented by torch's casts, closed forms, invariants
the DeepSeek-V4 pages state, special cases that reduce to library routines
(numpy matmul / complex arithmetic / sort, torch SDPA) and brute force on tiny
inputs.  Each test names the passage it follows."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline as P
from long_context_sparse_09_b200.configs import WORKLOADS


def rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- formats ---

def test_e4m3_decode_all_codes_match_torch():
    """OCP E4M3 (PaperTrace 2.5: the non-RoPE dims are FP8): every code."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if math.isnan(ref[c]):
            assert math.isnan(v), c
        else:
            assert v == ref[c], (c, v, ref[c])


def test_e4m3_encode_matches_torch_cast_in_range():
    r = rng(1)
    reps = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(
        torch.float8_e4m3fn).float().numpy()
    reps = np.unique(reps[np.isfinite(reps)])
    mids = (reps[1:] + reps[:-1]) / 2  # exact ties in fp32
    xs = np.concatenate([reps, mids, r.normal(0, 40, 4000), r.normal(0, 0.01, 2000),
                         r.uniform(-448, 448, 2000)]).astype(np.float32)
    xs = xs[np.abs(xs) <= 448]
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(x)) for x in xs], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    # -0.0 / +0.0 may differ only in the sign bit of a zero
    bad = [i for i in bad if not (xs[i] == 0 or (got[i] & 0x7F) == 0 == (ref[i] & 0x7F))]
    assert not bad, [(float(xs[i]), got[i], ref[i]) for i in bad[:5]]


def test_e4m3_encode_saturates():
    assert oracle.e4m3_encode(1e6) == 0x7E and oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_encode(-470.0) == 0xFE


def test_bf16_round_matches_torch():
    r = rng(2)
    x = np.concatenate([r.normal(0, 1, 5000), r.normal(0, 1e-30, 100),
                        r.normal(0, 1e30, 100)]).astype(np.float32)
    # exact ties: a bf16 value plus half its ulp
    base = torch.from_numpy(r.normal(0, 1, 500).astype(np.float32)).to(torch.bfloat16).float().numpy()
    ulp = np.array([np.spacing(np.float32(abs(b))) * 2 ** 16 for b in base], dtype=np.float32)
    ties = (base + np.sign(base) * ulp / 2).astype(np.float32)
    x = np.concatenate([x, ties]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    got = oracle.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_fp8mix_roundtrip_error_bound():
    """Quantise -> dequantise error <= half an E4M3 ulp times the scale; the
    largest magnitude maps to 448 exactly; RoPE dims are bf16."""
    r = rng(3)
    x = r.normal(0, 1, (64, 128))
    x[5, :96] = 0.0  # all-zero FP8 part: scale 1
    codes, rope, scale = oracle.fp8mix_encode(x, 32)
    bits = torch.from_numpy(rope.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    y = oracle.fp8mix_decode(codes, bits, scale, 128, 32)
    assert scale[5] == 1.0
    for i in range(64):
        xs = (x[i, :96].astype(np.float32) / scale[i]).astype(np.float64)
        if i != 5:
            assert np.max(np.abs([oracle.e4m3_decode(c) for c in codes[i]])) == 448.0
        q = y[i, :96] / scale[i]
        # E4M3 spacing at |v|: 2^(floor(log2|v|)-3), 2^-9 below 2^-6
        e = np.floor(np.log2(np.maximum(np.abs(xs), 2.0 ** -6)))
        half_ulp = 2.0 ** (e - 3) / 2
        assert np.all(np.abs(q - xs) <= half_ulp * (1 + 1e-6)), i
    np.testing.assert_array_equal(y[:, 96:], oracle.round_bf16(x[:, 96:]))


# ------------------------------------------------------------- RoPE / norm --

def test_rope_is_complex_rotation():
    """Notes 2.5.2: R_n rotates 2-D sub-spaces; pair p as a complex number
    times exp(i * pos * base^(-2p/r))."""
    r = rng(4)
    x = r.normal(0, 1, 64)
    for pos in (0.0, 1.0, 17.0, 1048576.0, -3.0):
        y = oracle.rope(x, 64, 10000.0, pos)
        z = x[0::2] + 1j * x[1::2]
        th = 10000.0 ** (-2.0 * np.arange(32) / 64)
        w = z * np.exp(1j * pos * th)
        np.testing.assert_allclose(y[0::2], w.real, atol=1e-12)
        np.testing.assert_allclose(y[1::2], w.imag, atol=1e-12)


def test_rope_group_properties():
    """Notes 2.5.2: R_n^T = R_{-n}, R_m R_n = R_{m+n}; only the last dims move."""
    r = rng(5)
    x = r.normal(0, 1, 96)
    y = oracle.rope(oracle.rope(x, 32, 10000.0, 37.0), 32, 10000.0, 100.0)
    np.testing.assert_allclose(y, oracle.rope(x, 32, 10000.0, 137.0), atol=1e-12)
    np.testing.assert_allclose(oracle.rope(oracle.rope(x, 32, 1e4, 5.0), 32, 1e4, -5.0), x, atol=1e-13)
    np.testing.assert_array_equal(oracle.rope(x, 32, 1e4, 9.0)[:64], x[:64])


def test_rmsnorm_invariant():
    """Notes 2.5.1: RMSNorm(x) = x / RMS(x) (gain 1): a positive multiple of x
    whose mean square is ms / (ms + eps)."""
    r = rng(6)
    x = r.normal(0, 3, 200)
    for eps in (0.0, 1e-6, 0.5):
        y = oracle.rmsnorm(x, eps)
        ms = np.mean(x ** 2)
        assert np.mean(y ** 2) == pytest.approx(ms / (ms + eps), rel=1e-12)
        ratio = y / x
        assert np.all(ratio > 0) and np.ptp(ratio) < 1e-12


# ------------------------------------------------------------- compression --

def _comp_case(T=24, d=16, width=8, m=4, seed=7, zero_z=False):
    r = rng(seed)
    H = r.normal(0, 1, (T, d))
    W = {k: r.normal(0, d ** -0.5, (d, width)) for k in ("Wkv_a", "Wkv_b", "Wz_a", "Wz_b")}
    B = {k: r.normal(0, 0.3, (m, width)) for k in ("B_a", "B_b")}
    if zero_z:
        W["Wz_a"][:] = 0
        W["Wz_b"][:] = 0
        B["B_a"][:] = 0
        B["B_b"][:] = 0
    return H, W, B


def test_compress_weights_sum_to_one():
    """Notes eq. 11: each column of the 2m x c weight block sums to 1; for
    i = 0 the b rows drop out (weight 0).  HCA (eq. 22): m slots only."""
    H, W, B = _comp_case()
    out, S = oracle.compress(H, 4, W["Wkv_a"], W["Wz_a"], B["B_a"], W["Wkv_b"],
                             W["Wz_b"], B["B_b"], want_S=True)
    np.testing.assert_allclose(S.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(S[0, 4:] == 0) and np.all(S[1:, 4:] > 0)
    out, S = oracle.compress(H, 4, W["Wkv_a"], W["Wz_a"], B["B_a"], want_S=True)
    np.testing.assert_allclose(S.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(S[:, 4:] == 0)


def test_compress_uniform_weights_give_block_means():
    """Eq. 11-12 with Z = 0 and B = 0: the softmax is uniform, so entry i is
    the mean of the m a-rows and m b-rows (only the a-rows for i = 0)."""
    m = 4
    H, W, B = _comp_case(zero_z=True)
    out = oracle.compress(H, m, W["Wkv_a"], W["Wz_a"], B["B_a"], W["Wkv_b"],
                          W["Wz_b"], B["B_b"])
    Ca, Cb = H @ W["Wkv_a"], H @ W["Wkv_b"]
    for i in range(H.shape[0] // m):
        a = Ca[m * i: m * i + m]
        if i == 0:
            ref = a.mean(axis=0)
        else:
            ref = np.concatenate([a, Cb[m * i - m: m * i]]).mean(axis=0)
        np.testing.assert_allclose(out[i], ref, atol=1e-12)


@pytest.mark.parametrize("branch,slot", [("a", 0), ("a", 3), ("b", 1), ("b", 2)])
def test_compress_dominant_slot_selects_token(branch, slot):
    """Eq. 11-12 / PaperTrace 2.1: entry i takes tokens 4i..4i+3 as C^a and
    4i-4..4i-1 as C^b.  A huge bias on one slot makes the entry equal to that
    token's row (pins the token-to-slot map and the b-branch shift)."""
    m = 4
    H, W, B = _comp_case(m=m)
    B["B_a"][:] = 0
    B["B_b"][:] = 0
    B[f"B_{branch}"][slot, :] = 200.0
    out = oracle.compress(H, m, W["Wkv_a"], W["Wz_a"], B["B_a"], W["Wkv_b"],
                          W["Wz_b"], B["B_b"])
    Ca, Cb = H @ W["Wkv_a"], H @ W["Wkv_b"]
    for i in range(1, H.shape[0] // m):
        ref = Ca[m * i + slot] if branch == "a" else Cb[m * (i - 1) + slot]
        np.testing.assert_allclose(out[i], ref, atol=1e-9)


def test_compress_each_token_in_two_entries():
    """PaperTrace 2.1: every token enters exactly two CSA entries (its own
    block as C^a, the next as C^b); HCA blocks do not overlap."""
    m = 4
    H, W, B = _comp_case(T=32, m=m)
    base = oracle.compress(H, m, W["Wkv_a"], W["Wz_a"], B["B_a"], W["Wkv_b"], W["Wz_b"], B["B_b"])
    base_h = oracle.compress(H, m, W["Wkv_a"], W["Wz_a"], B["B_a"])
    for j in (0, 5, 11, 27):
        H2 = H.copy()
        H2[j] += 1.0
        out = oracle.compress(H2, m, W["Wkv_a"], W["Wz_a"], B["B_a"], W["Wkv_b"], W["Wz_b"], B["B_b"])
        changed = set(np.nonzero(np.any(out != base, axis=1))[0])
        want = {j // m, j // m + 1} & set(range(len(base)))
        assert changed == want, (j, changed)
        out_h = oracle.compress(H2, m, W["Wkv_a"], W["Wz_a"], B["B_a"])
        assert set(np.nonzero(np.any(out_h != base_h, axis=1))[0]) == {j // m}


def test_hca_group_of_one_is_identity():
    """Eq. 22-23 with m' = 1: softmax over one slot is 1, so C^Comp = C = H W."""
    H, W, B = _comp_case()
    out = oracle.compress(H, 1, W["Wkv_a"], W["Wz_a"], B["B_a"][:1])
    np.testing.assert_allclose(out, H @ W["Wkv_a"], atol=1e-12)


def test_compress_entry_range_matches_full():
    H, W, B = _comp_case(T=40)
    full = oracle.compress(H, 4, W["Wkv_a"], W["Wz_a"], B["B_a"], W["Wkv_b"], W["Wz_b"], B["B_b"])
    part = oracle.compress(H, 4, W["Wkv_a"], W["Wz_a"], B["B_a"], W["Wkv_b"], W["Wz_b"], B["B_b"], i0=3, i1=7)
    np.testing.assert_array_equal(part, full[3:7])


# ------------------------------------------------------------------ index --

def test_nvis_is_complete_blocks():
    """Notes 2.3.2 / PaperTrace 2.4: only complete blocks are visible.  Brute
    force: entry s is visible iff every token of its a-window is <= t0."""
    for m in (1, 4, 128):
        for t0 in range(0, 3 * m + 2):
            brute = sum(1 for s in range(10) if all(tok <= t0 for tok in range(m * s, m * s + m)))
            assert oracle.nvis(t0, m, 10) == min(brute, 10)


def test_index_scores_closed_forms():
    """Eq. 16: since ReLU(x) - ReLU(-x) = x and ReLU(x) + ReLU(-x) = |x|,
    I(q) - I(-q) = (sum_h w_h q_h) . K_s and I(q) + I(-q) = sum_h w_h |q_h.K_s|;
    with one head and w = 1, I = ReLU(q . K_s)."""
    r = rng(8)
    Q, nh, cI, N, m = 3, 5, 16, 40, 4
    qI = r.normal(0, 1, (Q, nh, cI))
    w = r.normal(0, 1, (Q, nh))
    K = r.normal(0, 1, (N, cI))
    t0 = [1000, 1000, 1000]
    Ip = oracle.index_scores(t0, m, qI, w, K)
    Im = oracle.index_scores(t0, m, -qI, w, K)
    lin = np.einsum("qh,qhe->qe", w, qI) @ K.T
    np.testing.assert_allclose(Ip - Im, lin, atol=1e-11)
    absd = np.einsum("qh,qhs->qs", w, np.abs(np.einsum("qhe,se->qhs", qI, K)))
    np.testing.assert_allclose(Ip + Im, absd, atol=1e-11)
    one = oracle.index_scores(t0, m, qI[:, :1], np.ones((Q, 1)), K)
    np.testing.assert_allclose(one, np.maximum(qI[:, 0] @ K.T, 0), atol=1e-12)


def test_index_scores_mask_invisible():
    r = rng(9)
    qI, w, K = r.normal(0, 1, (3, 2, 8)), r.normal(0, 1, (3, 2)), r.normal(0, 1, (10, 8))
    sc = oracle.index_scores([2, 3, 13], 4, qI, w, K)
    assert np.all(np.isneginf(sc[0])) and np.isfinite(sc[1, 0]) and np.all(np.isneginf(sc[1, 1:]))
    assert np.all(np.isfinite(sc[2, :3])) and np.all(np.isneginf(sc[2, 3:]))


# ------------------------------------------------------------------ top-k --

def test_topk_matches_full_sort():
    """Eq. 17 by brute force: a stable sort by (-score, index)."""
    r = rng(10)
    Q, N, k = 6, 300, 17
    sc = np.round(r.normal(0, 1, (Q, N)), 1)  # many exact ties
    nv = np.array([300, 250, 17, 5, 0, 100], dtype=np.int32)
    idx, kth = oracle.topk(sc, nv, k)
    for q in range(Q):
        order = np.lexsort((np.arange(nv[q]), -sc[q, : nv[q]]))[:k]
        want = np.sort(order)
        got = idx[q][idx[q] >= 0]
        np.testing.assert_array_equal(got, want)
        assert np.all(idx[q][len(want):] == -1)
        if len(want):
            assert kth[q] == sc[q, order[-1]]


def test_topk_zero_weights_take_lowest_indices():
    """All scores equal (w = 0): the tie rule keeps indices 0..k-1."""
    sc = oracle.index_scores([10 ** 6], 4, np.ones((1, 2, 4)), np.zeros((1, 2)), np.ones((50, 4)))
    idx, _ = oracle.topk(sc, np.array([50], np.int32), 8)
    np.testing.assert_array_equal(idx[0], np.arange(8))


# -------------------------------------------------------------- attention --

def _sdpa_with_sink(q, keys, sink, scale):
    """torch SDPA (fp64, CPU) over [keys, sink column]: the sink is a key with
    logit z'_h (added through the mask) and a zero value."""
    Qn, nh, c = q.shape
    outs = []
    for i in range(Qn):
        K = torch.from_numpy(keys[i])  # [n, c]
        n = K.shape[0]
        Kx = torch.cat([K, torch.zeros(1, c, dtype=torch.float64)])
        Vx = Kx.clone()
        qq = torch.from_numpy(q[i]).unsqueeze(1)  # [nh, 1, c]
        mask = torch.zeros(nh, 1, n + 1, dtype=torch.float64)
        mask[:, 0, n] = torch.from_numpy(sink)
        o = torch.nn.functional.scaled_dot_product_attention(
            qq, Kx.expand(nh, n + 1, c), Vx.expand(nh, n + 1, c), attn_mask=mask, scale=scale)
        outs.append(o[:, 0].numpy())
    return np.stack(outs)


def test_attend_matches_sdpa_with_sink_column():
    """Eq. 19 + eq. 27 with no RoPE dims: shared-KV MQA over selected entries
    and window rows, the sink adding exp(z'_h) to the denominator -- the same
    as textbook attention with one extra zero-valued key of logit z'_h."""
    r = rng(11)
    Q, nh, c, N, m, nwin = 4, 3, 16, 20, 4, 5
    q = r.normal(0, 1, (Q, nh, c))
    kv = r.normal(0, 1, (N, c))
    win = r.normal(0, 1, (40, c))
    sink = r.normal(0, 1, nh)
    t0 = np.array([3, 20, 39, 70], np.int32)
    win_pos0 = 0
    win_full = r.normal(0, 1, (80, c))
    idx = np.array([[-1, -1, -1], [0, 2, 4], [1, 5, 9], [3, 7, 16]], np.int32)
    scale = 0.37
    out, mass = oracle.attend(t0, q, idx, m, kv, nwin, win_full, win_pos0, sink, 0, 1e4, scale)
    keys = []
    for i in range(Q):
        sel = [kv[s] for s in idx[i] if s >= 0]
        lo = max(0, t0[i] - nwin + 1)
        keys.append(np.array(sel + [win_full[t] for t in range(lo, t0[i] + 1)]))
    ref = _sdpa_with_sink(q, keys, sink, scale)
    np.testing.assert_allclose(out, ref, atol=1e-12)
    np.testing.assert_allclose(mass, 1.0, atol=1e-12)
    # HCA: all visible entries (floor((t0+1)/m)) and the window
    out_d, _ = oracle.attend(t0, q, None, m, kv, nwin, win_full, win_pos0, sink, 0, 1e4, scale)
    keys = []
    for i in range(Q):
        nv = min(N, (t0[i] + 1) // m)
        lo = max(0, t0[i] - nwin + 1)
        keys.append(np.array([kv[s] for s in range(nv)] + [win_full[t] for t in range(lo, t0[i] + 1)]))
    np.testing.assert_allclose(out_d, _sdpa_with_sink(q, keys, sink, scale), atol=1e-12)


def test_attend_sink_limits():
    """Eq. 27: z' -> -inf gives plain softmax attention; z' -> +inf drives
    every weight, hence the output, to 0 (PaperTrace 2.4)."""
    r = rng(12)
    q, kv, win = r.normal(0, 1, (2, 2, 8)), r.normal(0, 1, (6, 8)), r.normal(0, 1, (30, 8))
    t0 = np.array([23, 25], np.int32)
    out_hi, _ = oracle.attend(t0, q, None, 4, kv, 3, win, 0, np.array([60.0, 60.0]), 0, 1e4, 0.3)
    assert np.max(np.abs(out_hi)) < 1e-20
    out_lo, _ = oracle.attend(t0, q, None, 4, kv, 3, win, 0, np.array([-1e300, -1e300]), 0, 1e4, 0.3)
    keys = [np.concatenate([kv, win[21:24]]), np.concatenate([kv, win[23:26]])]
    ref = []
    for i in range(2):
        z = 0.3 * q[i] @ keys[i].T
        p = np.exp(z - z.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        ref.append(p @ keys[i])
    np.testing.assert_allclose(out_lo, np.stack(ref), atol=1e-12)


def test_attend_derotation_undoes_the_key_rotation():
    """Notes 2.5.2: o~_t = R_{-t} o_t.  A single key -- the window row of token
    t0 itself, stored as R_{t0} u -- gets weight 1, so the output is u."""
    r = rng(13)
    c, rd = 32, 16
    u = r.normal(0, 1, c)
    t0 = 1000
    row = oracle.rope(u, rd, 1e4, float(t0))
    win = np.zeros((5, c))
    win[4] = row
    q = r.normal(0, 1, (1, 2, c))
    out, _ = oracle.attend(np.array([t0], np.int32), q, None, 4, np.zeros((0, c)), 1, win,
                           t0 - 4, np.array([-1e300] * 2), rd, 1e4, 0.1)
    np.testing.assert_allclose(out[0, 0], u, atol=1e-10)
    np.testing.assert_allclose(out[0, 1], u, atol=1e-10)


def test_attend_rejects_invisible_selection():
    r = rng(14)
    with pytest.raises(ValueError):
        oracle.attend(np.array([7], np.int32), r.normal(0, 1, (1, 1, 8)),
                      np.array([[2]], np.int32), 4, r.normal(0, 1, (9, 8)), 0, None, 0,
                      np.zeros(1), 0, 1e4, 0.3)


# ------------------------------------------------------ end-to-end (oracle) --

TINY = WORKLOADS["tiny_csa_prefill_f32"].with_(T=64, d=48, c=32, rope_dims=8, n_h=3,
                                                n_hI=2, c_I=8, topk=4, n_win=6)


def _tiny_inputs(wl, seed=0):
    from long_context_sparse_09_b200 import synth
    wl = wl.with_(seed=seed)
    return wl, synth.weights(wl), synth.prefill_inputs(wl)


def _e2e(wl, W, inp, q_override=None, rope_shift=0.0, H_override=None):
    H = inp["H"][0] if H_override is None else H_override
    kv, kI, win = P.compress_seq(wl, W, H)
    t0s = inp["q_pos"].numpy()
    q = inp["q"] if q_override is None else q_override
    if wl.variant == "csa":
        idx, *_ = P.select(wl, t0s, inp["qI"], inp["w"], kI)
    else:
        idx = None
    out, mass = P.attend_wl(wl, t0s, q, idx, kv, win, 0, inp["sink"], rope_shift)
    return out, idx, mass


def test_e2e_causality():
    """Notes 2.3.2: a query never sees a later token.  Perturbing tokens
    after t0 leaves O[t0] and the top-k of t0 bit-identical."""
    wl, W, inp = _tiny_inputs(TINY)
    out0, idx0, mass = _e2e(wl, W, inp)
    np.testing.assert_allclose(mass, 1.0, atol=1e-12)
    t0 = 37
    H2 = inp["H"][0].clone()
    H2[t0 + 1:] += torch.randn(H2[t0 + 1:].shape, generator=torch.Generator().manual_seed(5))
    out1, idx1, _ = _e2e(wl, W, inp, H_override=H2)
    np.testing.assert_array_equal(out1[: t0 + 1], out0[: t0 + 1])
    np.testing.assert_array_equal(idx1[: t0 + 1], idx0[: t0 + 1])
    assert np.any(out1[t0 + 1:] != out0[t0 + 1:])


def test_e2e_dense_when_k_covers_all_entries():
    """With k >= the number of visible entries, CSA attends every visible
    entry: the same as dense (HCA-style) attention over the same cache."""
    wl, W, inp = _tiny_inputs(TINY.with_(topk=64))
    H = inp["H"][0]
    kv, kI, win = P.compress_seq(wl, W, H)
    t0s = inp["q_pos"].numpy()
    idx, *_ = P.select(wl, t0s, inp["qI"], inp["w"], kI)
    sparse, _ = P.attend_wl(wl, t0s, inp["q"], idx, kv, win, 0, inp["sink"])
    dense, _ = P.attend_wl(wl, t0s, inp["q"], None, kv, win, 0, inp["sink"])
    np.testing.assert_allclose(sparse, dense, atol=1e-13)


@pytest.mark.parametrize("variant", ["csa", "hca"])
def test_e2e_rope_shift_invariance(variant):
    """Notes 2.5.2: with q and keys rotated at their positions and the output
    de-rotated by R_{-t}, O depends on relative positions only: shifting every
    RoPE position by the same amount leaves O unchanged."""
    wl = TINY if variant == "csa" else TINY.with_(variant="hca", m=8, n_hI=0, c_I=0, topk=0)
    wl, W, inp = _tiny_inputs(wl, seed=3)
    u = inp["q"].double().numpy()
    t0s = inp["q_pos"].numpy()
    outs = []
    for shift in (0.0, 4096.0):
        q = np.stack([[oracle.rope(u[i, h], wl.rope_dims, wl.rope_base, t0s[i] + shift)
                       for h in range(wl.n_h)] for i in range(len(t0s))])
        H = inp["H"][0]
        raw_kv, kI, _ = None, None, None
        if wl.variant == "csa":
            raw = oracle.compress(H, wl.m, W["Wkv_a"], W["Wz_a"], W["B_a"], W["Wkv_b"], W["Wz_b"], W["B_b"])
            kI = oracle.compress(H, wl.m, W["WIkv_a"], W["WIz_a"], W["BI_a"], W["WIkv_b"], W["WIz_b"], W["BI_b"])
        else:
            raw = oracle.compress(H, wl.m, W["Wkv_a"], W["Wz_a"], W["B_a"])
        kv = oracle.norm_rope_rows(raw, wl.rope_dims, wl.rope_base, wl.rms_eps, shift, wl.m)
        win = oracle.norm_rope_rows(oracle.matmul(H, W["Wkv_a"]), wl.rope_dims, wl.rope_base,
                                    wl.rms_eps, shift, 1.0)
        idx = P.select(wl, t0s, inp["qI"], inp["w"], kI)[0] if wl.variant == "csa" else None
        out, _ = P.attend_wl(wl, t0s, q, idx, kv, win, 0, inp["sink"], rope_shift=shift)
        outs.append(out)
    np.testing.assert_allclose(outs[0], outs[1], atol=1e-9)


# ------------------------------------------------ grouped output projection ---
# "DeepSeekV4技术报告阅读笔记" 2.3.3 (Grouped Output Projection); PaperTrace 2.2.

def _gop_inputs(Q=3, n_h=8, c=6, g=4, d_g=5, d=7, seed=41):
    r = rng(seed)
    O = r.standard_normal((Q, n_h, c))
    WG = r.standard_normal((g, c * n_h // g, d_g))
    WO = r.standard_normal((g * d_g, d))
    return O, WG, WO


def test_group_out_proj_one_group_is_two_matmuls():
    O, WG, WO = _gop_inputs(g=1)
    Y, out = oracle.group_out_proj(O, WG, WO, round_mid=False)
    flat = O.reshape(O.shape[0], -1)
    np.testing.assert_allclose(Y, flat @ WG[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out, (flat @ WG[0]) @ WO, rtol=1e-12, atol=1e-12)


def test_group_out_proj_is_a_block_diagonal_projection():
    """The notes' one-line summary: R^{c n_h} -> R^{d_g g} by a block-diagonal
    matrix (one block per group of consecutive heads), then -> R^d."""
    import scipy.linalg
    O, WG, WO = _gop_inputs()
    Y, out = oracle.group_out_proj(O, WG, WO, round_mid=False)
    W_eff = scipy.linalg.block_diag(*WG) @ WO
    flat = O.reshape(O.shape[0], -1)
    np.testing.assert_allclose(Y, flat @ scipy.linalg.block_diag(*WG), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out, flat @ W_eff, rtol=1e-10, atol=1e-10)


def test_group_out_proj_groups_are_independent():
    O, WG, WO = _gop_inputs()
    g, d_g = WG.shape[0], WG.shape[2]
    hpg = O.shape[1] // g
    Y0, _ = oracle.group_out_proj(O, WG, WO, round_mid=False)
    O2 = O.copy()
    O2[:, 2 * hpg:3 * hpg] += 1.0  # the heads of group 2 only
    Y1, _ = oracle.group_out_proj(O2, WG, WO, round_mid=False)
    changed = np.any(Y0 != Y1, axis=0).reshape(g, d_g).any(axis=1)
    assert changed.tolist() == [False, False, True, False]


def test_group_out_proj_rounds_the_group_outputs():
    O, WG, WO = _gop_inputs()
    Yx, _ = oracle.group_out_proj(O, WG, WO, round_mid=False)
    Y, out = oracle.group_out_proj(O, WG, WO, round_mid=True)
    np.testing.assert_array_equal(Y, torch.from_numpy(Yx).to(torch.bfloat16).double().numpy())
    np.testing.assert_allclose(out, Y @ WO, rtol=1e-12, atol=1e-12)


def test_group_out_proj_parameter_counts_of_the_pages():
    """PaperTrace 2.2: with V4-Pro's shapes (c = 512, n_h = 128, g = 16,
    d_g = 1024, d = 7168) the grouped projection has about 180 million
    parameters and a direct one about 470 million; the notes 2.3.3 count
    c n_h d_g + d_g g d multiplications.  The oracle accepts exactly these
    operand shapes."""
    c, n_h, g, d_g, d = 512, 128, 16, 1024, 7168
    grouped = g * (c * n_h // g) * d_g + (g * d_g) * d
    assert grouped == c * n_h * d_g + d_g * g * d
    assert abs(grouped / 1.8e8 - 1) < 0.03
    assert abs(c * n_h * d / 4.7e8 - 1) < 0.01
    O = np.zeros((1, 4, 2))
    with pytest.raises(ValueError):
        oracle.group_out_proj(O, np.zeros((2, 3, 5)), np.zeros((10, 3)))  # c n_h / g = 4


# ------------------------------------------------------ query projections ---
# "DeepSeekV4技术报告阅读笔记" eq. 13-15, 18 and 2.5.1-2.5.2.

def _qp_inputs(T=5, d=24, d_c=12, n_h=3, c=16, n_hI=2, c_I=8, seed=53):
    r = rng(seed)
    return dict(H=r.standard_normal((T, d)), WDQ=r.standard_normal((d, d_c)) / d ** 0.5,
                WUQ=r.standard_normal((d_c, n_h * c)) / d_c ** 0.5,
                WIUQ=r.standard_normal((d_c, n_hI * c_I)) / d_c ** 0.5,
                Ww=r.standard_normal((d, n_hI)) / d ** 0.5,
                n_h=n_h, c=c, n_hI=n_hI, c_I=c_I)


def _qp(x, pos, rope_dims=8, eps=1e-6, **over):
    a = dict(x)
    a.update(over)
    return P.query_proj(a["H"], pos, a["WDQ"], a["WUQ"], a["WIUQ"], a["Ww"], a["n_h"], a["c"],
                        a["n_hI"], a["c_I"], rope_dims, 10000.0, eps)


def test_query_proj_low_rank_chain_is_two_matmuls():
    x = _qp_inputs()
    pos = np.arange(5)
    cQ, q, qI, w = _qp(x, pos)
    np.testing.assert_allclose(cQ, x["H"] @ x["WDQ"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(qI.reshape(5, -1), (x["H"] @ x["WDQ"]) @ x["WIUQ"],
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(w, x["H"] @ x["Ww"], rtol=1e-12, atol=1e-12)


def test_query_heads_are_unit_rms_and_scale_free():
    """Each q head has mean square 1 after the norm (the rotation keeps it),
    and scaling h leaves q unchanged while q^I and w scale with it: the norm
    applies to q only."""
    x = _qp_inputs()
    pos = np.array([0, 3, 17, 250, 4095])
    _, q, qI, w = _qp(x, pos, eps=0.0)
    np.testing.assert_allclose((q ** 2).mean(axis=2), 1.0, rtol=1e-12)
    _, q2, qI2, w2 = _qp(x, pos, eps=0.0, H=3.0 * x["H"])
    np.testing.assert_allclose(q2, q, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(qI2, 3.0 * qI, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(w2, 3.0 * w, rtol=1e-12, atol=1e-12)


def test_query_rotation_uses_the_token_position():
    """q(t) . R_s k depends on t - s only (2.5.2): shifting the query's and
    the key's positions together leaves the score; position 0 is unrotated."""
    x = _qp_inputs(T=1)
    k = rng(7).standard_normal(16)
    _, q0, _, _ = _qp(x, np.array([0]))
    _, qn, _, _ = _qp(x, np.array([0]), rope_dims=0)
    np.testing.assert_allclose(q0, qn, rtol=1e-12, atol=1e-12)
    for t, s, shift in [(9, 4, 100), (1000, 3, 77)]:
        _, qa, _, _ = _qp(x, np.array([t]))
        _, qb, _, _ = _qp(x, np.array([t + shift]))
        ka, kb = oracle.rope(k, 8, 10000.0, s), oracle.rope(k, 8, 10000.0, s + shift)
        np.testing.assert_allclose(qa[0] @ ka, qb[0] @ kb, rtol=1e-9, atol=1e-9)
        _, qc, _, _ = _qp(x, np.array([t + 1]))
        assert not np.allclose(qc[0] @ ka, qa[0] @ ka)


def test_query_latent_rounding_is_the_only_change():
    """round_mid rounds c^Q to bf16 before the up-projections and nothing
    else: with W^DQ the identity and bf16-representable h, c^Q is already a
    bf16 value and all four outputs are bit-identical; with h off the bf16
    grid they differ, and equal the chain run on bf16(h W^DQ) by matmuls."""
    x = _qp_inputs(d=12, d_c=12)
    x["WDQ"] = np.eye(12)
    pos = np.array([1, 5, 9, 70, 300])
    x["H"] = oracle.round_bf16(x["H"])
    a = _qp(x, pos)
    b = P.query_proj(x["H"], pos, x["WDQ"], x["WUQ"], x["WIUQ"], x["Ww"], 3, 16, 2, 8, 8,
                     10000.0, 1e-6, round_mid=True)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    x2 = _qp_inputs()
    c = P.query_proj(x2["H"], pos, x2["WDQ"], x2["WUQ"], x2["WIUQ"], x2["Ww"], 3, 16, 2, 8, 8,
                     10000.0, 1e-6, round_mid=True)
    d = _qp(x2, pos)
    assert not np.array_equal(c[2], d[2])
    cq = oracle.round_bf16(x2["H"] @ x2["WDQ"])
    np.testing.assert_array_equal(c[0], cq)
    np.testing.assert_allclose(c[2].reshape(5, -1), cq @ x2["WIUQ"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(c[3], d[3], rtol=0, atol=0)  # w does not see the latent


# ------------------------------------------------------------------ MXFP4 ---
# The indexer's QK path in MXFP4 ("02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文"
# 3.3); the format is the OCP Microscaling one (tests/golden/e2m1_values.txt).

def _golden_e2m1():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "e2m1_values.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    return {int(r[0]): float(r[-1]) for r in rows}


def test_e2m1_decode_matches_the_spec_table():
    for code, v in _golden_e2m1().items():
        got = oracle.e2m1_decode(code)
        assert got == v and math.copysign(1.0, got) == math.copysign(1.0, v), code


def _nearest_e2m1(v):
    """Brute force: the E2M1 magnitude nearest to |v| (ties to the even
    mantissa, i.e. the even code), saturating at 6."""
    grid = [(abs(val), code) for code, val in _golden_e2m1().items() if code < 8]
    a = min(abs(v), 6.0)
    best = min(grid, key=lambda g: (abs(g[0] - a), g[1] & 1))
    return math.copysign(best[0], v) if best[0] else 0.0


def test_mxfp4_elements_are_the_nearest_e2m1_values():
    r = rng(61)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.9]
    for trial in range(50):
        x = r.uniform(-8, 8, 32)
        x[0] = 7.5 if trial % 2 else -7.5  # block maximum in [4, 8): scale 2^0
        x[1:1 + len(mids)] = mids
        codes, exps = oracle.mxfp4_encode(x)
        assert exps.tolist() == [0]
        got = oracle.mxfp4_decode(codes, exps)
        want = np.array([_nearest_e2m1(v) for v in x])
        np.testing.assert_array_equal(np.abs(got), np.abs(want))


def test_mxfp4_block_scale_and_error_bound():
    r = rng(62)
    for _ in range(40):
        x = r.standard_normal(96) * 10.0 ** r.uniform(-3, 3)
        codes, exps = oracle.mxfp4_encode(x)
        y = oracle.mxfp4_decode(codes, exps)
        for b in range(3):
            blk, e = x[32 * b:32 * b + 32], int(exps[b])
            amax = np.abs(blk).max()
            assert 4.0 * 2.0 ** e <= amax < 8.0 * 2.0 ** e   # the top binade holds the max
            err = np.abs(y[32 * b:32 * b + 32] - blk)
            # half a grid step (at most 1 scale unit) below 6, saturation above
            assert np.all(err <= np.maximum(2.0 ** e, np.abs(blk) - 6.0 * 2.0 ** e) + 1e-300)


def test_mxfp4_power_of_two_equivariance():
    x = rng(63).standard_normal(64)
    c0, e0 = oracle.mxfp4_encode(x)
    c1, e1 = oracle.mxfp4_encode(x * 2.0 ** 5)
    np.testing.assert_array_equal(c0, c1)
    np.testing.assert_array_equal(e1, e0 + 5)


def test_fp4_index_scores_on_representable_inputs():
    """Inputs already in MXFP4 pass unchanged: the FP4 scores are the exact
    scores rounded to bf16; a top-k on them keeps full recall of itself."""
    wl = WORKLOADS["tiny_csa_prefill_f32"]
    r = rng(64)
    n_hI, c_I, N = wl.n_hI, wl.c_I, 40
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    kI = r.choice(grid, (N, c_I)) * r.choice([-1, 1], (N, c_I)) * 2.0 ** -3
    kI[:, ::32] = 6.0 * 2.0 ** -3  # every block holds its top value
    qI = r.choice(grid, (2, n_hI, c_I)) * 2.0 ** -2
    qI[:, :, ::32] = 4.0 * 2.0 ** -2
    w = r.standard_normal((2, n_hI))
    t0s = np.array([N * wl.m - 1, 17])
    np.testing.assert_array_equal(oracle.mxfp4_round(kI), kI)
    s4 = P.index_scores_fp4(wl, t0s, qI, w, kI)
    ref = oracle.index_scores(t0s, wl.m, qI, w, kI)
    fin = np.isfinite(ref)
    np.testing.assert_array_equal(np.isfinite(s4), fin)
    np.testing.assert_array_equal(s4[fin], oracle.round_bf16(ref[fin]))
    idx, _ = oracle.topk(s4, np.array([oracle.nvis(int(t), wl.m, N) for t in t0s]), 8)
    assert P.topk_recall(idx, idx).tolist() == [1.0, 1.0]


# ------------------------------------------------- cache size per token ---
# The compressed cache per token and layer that "02 · DeepSeek-V4: 压缩注意力
# 撑起 1M 上下文" section 2.5 works out for V4-Pro (tests/golden/
# kv_elements_per_token.txt).

def _golden_kv_elements():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "kv_elements_per_token.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    return {r[0]: int(r[1]) for r in rows}


def _compress_weights(wl, d, r):
    W = {}
    for k, width in (("Wkv_a", wl.c), ("Wz_a", wl.c), ("Wkv_b", wl.c), ("Wz_b", wl.c),
                     ("WIkv_a", wl.c_I), ("WIz_a", wl.c_I), ("WIkv_b", wl.c_I),
                     ("WIz_b", wl.c_I)):
        if width:
            W[k] = r.normal(0, d ** -0.5, (d, width))
    for k, width in (("B_a", wl.c), ("B_b", wl.c), ("BI_a", wl.c_I), ("BI_b", wl.c_I)):
        if width:
            W[k] = r.normal(0, 0.3, (wl.m, width))
    return W


def test_cache_elements_per_token_match_the_worked_example():
    """The oracle's whole-sequence compressor stores c/m + c_I/m elements per
    token for a CSA layer and c/m' for an HCA layer: the page's 160 and 4 at
    the V4-Pro widths, and about 4,900 over its 30 CSA and 31 HCA layers."""
    gold = _golden_kv_elements()
    r = rng(11)
    d, T = 16, 256
    pro = WORKLOADS["pro_csa_decode_1m"]
    hca = WORKLOADS["hca_decode_1m"].with_(c=pro.c)
    assert (pro.c, pro.c_I, pro.m, hca.m) == (512, 128, 4, 128)
    kv, kI, win = P.compress_seq(pro, _compress_weights(pro, d, r), r.normal(0, 1, (T, d)))
    assert kv.shape == (T // pro.m, pro.c) and kI.shape == (T // pro.m, pro.c_I)
    assert win.shape == (T, pro.c)  # the window side output, one row per token
    csa = (kv.size + kI.size) / T
    kv_h, kI_h, _ = P.compress_seq(hca, _compress_weights(hca, d, r), r.normal(0, 1, (T, d)))
    assert kI_h is None and kv_h.shape == (T // hca.m, hca.c)
    hca_el = kv_h.size / T
    assert csa == gold["csa_layer_elements_per_token"]
    assert hca_el == gold["hca_layer_elements_per_token"]
    total = gold["pro_csa_layers"] * csa + gold["pro_hca_layers"] * hca_el
    assert abs(total - gold["pro_elements_per_token_about"]) <= 0.01 * gold[
        "pro_elements_per_token_about"]
