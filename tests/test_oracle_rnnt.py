"""Pins of the oracle's RNNT head: the LSTM cell (gate order, both biases), the
joint network and the greedy decoding loop (emission / advance rules, the
per-frame symbol cap, the predictor advancing only on emitted symbols)."""
import numpy as np
import pytest

import oracle
import oracle.rnnt as orn
from conftest import read_golden_rows


def _cell_case(row, P=3, split_bias=True):
    _, c_in, gates, c_out, h_out = row
    b = np.repeat(np.array([float(v) for v in gates.split()]), P)
    b_ih, b_hh = (b / 2, b / 2) if split_bias else (b, np.zeros(4 * P))
    z = np.zeros((4 * P, P))
    h, c = orn.lstm_step(np.zeros(P), np.zeros(P), np.full(P, float(c_in)), z, z, b_ih, b_hh)
    return h, c, float(c_out), float(h_out)


def _lstm_pins_hold():
    for row in read_golden_rows("lstm.txt"):
        h, c, c_ref, h_ref = _cell_case(row)
        if not (np.allclose(c, c_ref, rtol=0, atol=1e-12) and np.allclose(h, h_ref, rtol=0, atol=1e-12)):
            return False
    return True


def test_lstm_cell_hand_cases():
    """Zero weights: c' = c/2, h' = tanh(c/2)/2.  Saturated gates i = 1, f = 0,
    o = 1 with candidate bias 0.5: c' = tanh(0.5), h' = tanh(tanh(0.5)).  The two
    biases are split half and half, so a dropped bias changes the result."""
    assert _lstm_pins_hold()


def test_lstm_cell_matches_explicit_loops():
    rng = np.random.default_rng(0)
    P, I = 4, 3
    w_ih, w_hh = rng.normal(size=(4 * P, I)), rng.normal(size=(4 * P, P))
    b_ih, b_hh = rng.normal(size=4 * P), rng.normal(size=4 * P)
    x, h, c = rng.normal(size=I), rng.normal(size=P), rng.normal(size=P)
    h2, c2 = orn.lstm_step(x, h, c, w_ih, w_hh, b_ih, b_hh)
    for j in range(P):
        pre = []
        for gate in range(4):
            r = gate * P + j
            pre.append(sum(w_ih[r, k] * x[k] for k in range(I)) + sum(w_hh[r, k] * h[k] for k in range(P))
                       + b_ih[r] + b_hh[r])
        sg = [1 / (1 + np.exp(-v)) for v in pre]
        cj = sg[1] * c[j] + sg[0] * np.tanh(pre[2])
        assert c2[j] == pytest.approx(cj, abs=1e-12)
        assert h2[j] == pytest.approx(sg[3] * np.tanh(cj), abs=1e-12)


def _swap_i_f(x, h, c, w_ih, w_hh, b_ih, b_hh):
    P = h.shape[0]
    perm = np.r_[P:2 * P, 0:P, 2 * P:4 * P]
    return _ORIG_LSTM(x, h, c, w_ih[perm], w_hh[perm], b_ih[perm], b_hh[perm])


def _swap_g_o(x, h, c, w_ih, w_hh, b_ih, b_hh):
    P = h.shape[0]
    perm = np.r_[0:2 * P, 3 * P:4 * P, 2 * P:3 * P]
    return _ORIG_LSTM(x, h, c, w_ih[perm], w_hh[perm], b_ih[perm], b_hh[perm])


def _drop_hh_bias(x, h, c, w_ih, w_hh, b_ih, b_hh):
    return _ORIG_LSTM(x, h, c, w_ih, w_hh, b_ih, np.zeros_like(b_hh))


_ORIG_LSTM = orn.lstm_step


@pytest.mark.parametrize("mutant", [_swap_i_f, _swap_g_o, _drop_hh_bias], ids=["swap_i_f", "swap_g_o", "one_bias"])
def test_lstm_pins_catch_gate_order_and_bias_mistakes(monkeypatch, mutant):
    monkeypatch.setattr(orn, "lstm_step", mutant)
    assert not _lstm_pins_hold()


def test_joint_closed_form():
    """enc / pred projections = I, zero biases, out = I: logits = act(f + g)."""
    d = 4
    W = {"rnnt.joint.enc.weight": np.eye(d), "rnnt.joint.enc.bias": np.zeros(d),
         "rnnt.joint.pred.weight": np.eye(d), "rnnt.joint.pred.bias": np.zeros(d),
         "rnnt.joint.out.weight": np.eye(d), "rnnt.joint.out.bias": np.array([0.0, 0.0, 0.0, 0.5])}
    f, g = np.array([1.0, -2.0, 0.5, 0.0]), np.array([0.5, 1.0, -1.0, -1.0])
    np.testing.assert_allclose(orn.rnnt_joint(f, g, W, "relu"), [1.5, 0.0, 0.0, 0.5])
    np.testing.assert_allclose(orn.rnnt_joint(f, g, W, "tanh"),
                               [np.tanh(1.5), np.tanh(-1.0), np.tanh(-0.5), np.tanh(-1.0) + 0.5])


def _scripted(monkeypatch, decisions, C):
    """Replace the joint by a script: each call returns one-hot logits of the next
    decision; record the predictor inputs."""
    calls = {"n": 0, "inputs": []}
    queue = list(decisions)

    def joint(f_t, g, W, act="relu", dtype=np.float64):
        k = queue[calls["n"]]
        calls["n"] += 1
        z = np.zeros(C)
        z[k] = 1.0
        return z

    def lstm(x, h, c, *w):
        calls["inputs"].append(x.copy())
        return _ORIG_LSTM(x, h, c, *w)

    monkeypatch.setattr(orn, "rnnt_joint", joint)
    monkeypatch.setattr(orn, "lstm_step", lstm)
    return calls, queue


def _tiny_weights(C, P=3, d=2):
    rng = np.random.default_rng(1)
    return {"rnnt.embed.weight": rng.normal(size=(C, P)), "rnnt.lstm.weight_ih_l0": rng.normal(size=(4 * P, P)),
            "rnnt.lstm.weight_hh_l0": rng.normal(size=(4 * P, P)), "rnnt.lstm.bias_ih_l0": np.zeros(4 * P),
            "rnnt.lstm.bias_hh_l0": np.zeros(4 * P)}


def test_greedy_loop_rules(monkeypatch):
    """Frame 0 emits 2 then 3 then blank; frame 1 blank; frame 2 emits 1 until
    the cap (max_symbols = 3) -- the joint is not asked again there; frame 3
    emits 0 then blank.  The predictor starts from a zero input and then takes
    the embedding of each emitted symbol, in order."""
    C, blank, M = 5, 4, 3
    decisions = [2, 3, blank, blank, 1, 1, 1, 0, blank]
    calls, queue = _scripted(monkeypatch, decisions, C)
    W = _tiny_weights(C)
    sym, frames, gap = orn.rnnt_greedy_clip(np.zeros((4, 2)), W, C, max_symbols=M)
    assert sym == [2, 3, 1, 1, 1, 0]
    assert frames == [0, 0, 2, 2, 2, 3]
    assert calls["n"] == len(decisions)
    emb = W["rnnt.embed.weight"]
    assert np.all(calls["inputs"][0] == 0)
    for x, k in zip(calls["inputs"][1:], sym):
        np.testing.assert_array_equal(x, emb[k])
    assert len(calls["inputs"]) == 1 + len(sym)
    assert gap == 1.0


def test_greedy_first_index_on_ties(monkeypatch):
    C = 4

    def joint(f_t, g, W, act="relu", dtype=np.float64):
        return np.array([0.0, 1.0, 1.0, 1.0]) if joint.n == 0 else np.array([0.0, 0.0, 0.0, 1.0])
    joint.n = 0

    def counting(*a, **k):
        out = joint(*a, **k)
        joint.n += 1
        return out

    monkeypatch.setattr(orn, "rnnt_joint", counting)
    sym, frames, gap = orn.rnnt_greedy_clip(np.zeros((1, 2)), _tiny_weights(C), C)
    assert sym == [1] and frames == [0] and gap == 0.0


def test_reexported_by_package():
    assert oracle.rnnt_greedy_clip is orn.rnnt_greedy_clip or callable(oracle.rnnt_greedy_clip)
