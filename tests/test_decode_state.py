"""The decode-time compressor's state machine, on the CPU: the running
softmax that csa_decode_append / hca_decode_append keep for each open entry
(largest logit, rescaled denominator and weighted sum, an entry's slot
restarted by its first token, the b window of block j feeding entry j + 1),
and the window roll.  A numpy model of both is run token by token and checked
against the oracle's whole-sequence compression ("DeepSeekV4技术报告阅读笔记"
eq. 11-12 and 22-23) and against the window the attention must see
(§2.5.3): the readings the CUDA kernels implement, pinned without a GPU."""
import numpy as np
import pytest

import oracle


def _state_machine(Ca, Za, Ba, Cb, Zb, Bb, m, b_entry_shift=1):
    """Entries folded one token at a time with S = 2 slots (overlap) or 1.
    The state starts as NaN: every slot must be restarted before use.  The b
    window of block j feeds entry j + b_entry_shift (1 is the method)."""
    T, c = Ca.shape
    overlap = Cb is not None
    S = 2 if overlap else 1
    mx = np.full((S, c), np.nan)
    den = np.full((S, c), np.nan)
    num = np.full((S, c), np.nan)

    def add(slot, C, z, fresh):
        if fresh:
            mx[slot], den[slot], num[slot] = z, 1.0, C
            return
        m1 = np.maximum(mx[slot], z)
        s0, s1 = np.exp(mx[slot] - m1), np.exp(z - m1)
        mx[slot], den[slot], num[slot] = m1, den[slot] * s0 + s1, num[slot] * s0 + s1 * C

    out = []
    for t in range(T):
        j, r = divmod(t, m)
        add(j % S, Ca[t], Za[t] + Ba[r], r == 0 and (not overlap or j == 0))
        if overlap:
            add((j + b_entry_shift) % S, Cb[t], Zb[t] + Bb[r], r == 0 and b_entry_shift == 1)
        if r == m - 1:
            out.append(num[j % S] / den[j % S])
    return np.array(out)


@pytest.mark.parametrize("overlap,m,T", [(True, 4, 37), (True, 1, 9), (False, 16, 70),
                                         (False, 128, 300)])
def test_running_softmax_equals_the_fold(overlap, m, T):
    rng = np.random.default_rng(11 + m)
    d, c = 24, 10
    H = rng.standard_normal((T, d))
    W = {k: rng.standard_normal((d, c)) / np.sqrt(d) for k in ("Wkv_a", "Wz_a", "Wkv_b", "Wz_b")}
    # large position biases make the running maximum move often
    B_a, B_b = 3.0 * rng.standard_normal((m, c)), 3.0 * rng.standard_normal((m, c))
    Ca, Za = H @ W["Wkv_a"], H @ W["Wz_a"]
    Cb, Zb = (H @ W["Wkv_b"], H @ W["Wz_b"]) if overlap else (None, None)
    got = _state_machine(Ca, Za, B_a, Cb, Zb, B_b if overlap else None, m)
    if overlap:
        ref = oracle.compress(H, m, W["Wkv_a"], W["Wz_a"], B_a, W["Wkv_b"], W["Wz_b"], B_b)
    else:
        ref = oracle.compress(H, m, W["Wkv_a"], W["Wz_a"], B_a)
    assert got.shape == ref.shape == (T // m, c)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_running_softmax_catches_a_wrong_slot():
    """A state machine that folds the b window of block j into entry j (a
    plausible slip) disagrees with the fold: the test above has teeth."""
    rng = np.random.default_rng(3)
    T, d, c, m = 24, 8, 4, 4
    H = rng.standard_normal((T, d))
    Wa, Wza, Wb, Wzb = (rng.standard_normal((d, c)) for _ in range(4))
    B_a, B_b = rng.standard_normal((m, c)), rng.standard_normal((m, c))
    ref = oracle.compress(H, m, Wa, Wza, B_a, Wb, Wzb, B_b)
    wrong = _state_machine(H @ Wa, H @ Wza, B_a, H @ Wb, H @ Wzb, B_b, m, b_entry_shift=0)
    assert not np.allclose(wrong, ref, rtol=1e-6, atol=1e-6)


def _roll_model(T, n_win, W):
    """Positions held by the W window rows after each token, as the append
    writes and rolls them; returns the list of (win_pos0, rows) per step."""
    keep = max(n_win - 1, 0)
    rows = np.full(W, -1)
    wp0 = 0
    states = []
    for t in range(T):
        wr = t - wp0
        if wr == W and W >= 2 * keep and W > 0:
            rows[:keep] = rows[W - keep:W].copy()
            wp0 = t - keep
            wr = keep
        assert 0 <= wr < W, (t, wr)
        rows[wr] = t
        states.append((wp0, rows.copy()))
    return states


@pytest.mark.parametrize("n_win,W", [(6, 12), (6, 10), (128, 256), (1, 1), (2, 2)])
def test_window_roll_keeps_the_last_n_win_tokens(n_win, W):
    T = 5 * W + 3
    for t, (wp0, rows) in enumerate(_roll_model(T, n_win, W)):
        for pos in range(max(0, t - n_win + 1), t + 1):
            r = pos - wp0
            assert 0 <= r < W and rows[r] == pos, (t, pos, wp0)
