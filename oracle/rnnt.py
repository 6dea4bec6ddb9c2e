"""Plain NumPy definition of the RNNT head and its greedy decoding (oracle).

TEST INFRASTRUCTURE ONLY -- see the package docstring.  One clip at a time, in
the order the decoding takes its steps; nothing is batched or tuned.

Sources (page title, section):
  [MLX-trap]  "GigaAM on MLX: the transcripts matched, but the model was broken":
              "What we're porting" (the head is a single-layer LSTM of size 320
              plus a joint network), "Trap 4" (PyTorch LSTM weights weight_ih /
              weight_hh with two biases that add up).
  [RNNT-card] "GigaAM v3 RNNT -- MLX (Apple Silicon)": character model of 33
              letters + blank, "sequential greedy decode"; "Notes for other
              runtimes": the LSTM bias is bias_ih + bias_hh, blank =
              len(vocabulary).
  [v3-MLX]    "GigaAM v3 MLX": "Architecture details" (RNNT predictor, RNNT
              joint, greedy RNNT; 1025 output classes, blank 1024),
              "Performance" (joint and greedy loop dominate the runtime).

Readings where the pages are silent (each also listed in the design notes):
  R17 LSTM gate order i, f, g, o (PyTorch's layout of weight_ih_l0 /
      weight_hh_l0, the tensors [MLX-trap] "Trap 4" names); c' = f c + i g,
      h' = o tanh(c'), sigmoid gates, tanh candidate.
  R18 predictor input: the embedding of the last emitted symbol; before the
      first symbol the input is the zero vector and the state is zero.
  R19 joint: a = act(W_enc f_t + b_enc + W_pred g + b_pred), logits = W_out a +
      b_out, with joint width 320 ("size 320" of the head) and act = ReLU (tanh
      selectable); the predictor output g is the LSTM hidden state.
  R20 greedy: at frame t, repeat {argmax (lowest index) of the logits; blank ->
      next frame; else emit the symbol, advance the predictor with it} with at
      most max_symbols emissions per frame (10), then the next frame.
"""
from __future__ import annotations

from typing import Dict, List, Tuple

import numpy as np

__all__ = ["sigmoid", "lstm_step", "rnnt_joint", "rnnt_greedy_clip"]


def sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def lstm_step(x, h, c, w_ih, w_hh, b_ih, b_hh):
    """One step of a single-layer LSTM (R17).  x [I], h, c [P]; w_ih [4P, I],
    w_hh [4P, P]; both biases are added ([RNNT-card] "Notes for other runtimes")."""
    P = h.shape[0]
    z = w_ih @ x + b_ih + w_hh @ h + b_hh
    i = sigmoid(z[0:P])
    f = sigmoid(z[P:2 * P])
    g = np.tanh(z[2 * P:3 * P])
    o = sigmoid(z[3 * P:4 * P])
    c2 = f * c + i * g
    h2 = o * np.tanh(c2)
    return h2, c2


def rnnt_joint(f_t, g, W: Dict[str, np.ndarray], act: str = "relu", dtype=np.float64):
    """Joint network logits for encoder frame f_t [d] and predictor output g [P] (R19)."""
    a = (W["rnnt.joint.enc.weight"].astype(dtype) @ f_t + W["rnnt.joint.enc.bias"].astype(dtype)
         + W["rnnt.joint.pred.weight"].astype(dtype) @ g + W["rnnt.joint.pred.bias"].astype(dtype))
    a = np.maximum(a, 0.0) if act == "relu" else np.tanh(a)
    return W["rnnt.joint.out.weight"].astype(dtype) @ a + W["rnnt.joint.out.bias"].astype(dtype)


def rnnt_greedy_clip(enc: np.ndarray, W: Dict[str, np.ndarray], n_classes: int, max_symbols: int = 10,
                     act: str = "relu", dtype=np.float64) -> Tuple[List[int], List[int], float]:
    """Greedy RNNT decoding of one clip's valid encoder frames enc [T, d] (R18, R20).

    Returns (symbols, the frame index of each symbol, the smallest gap between the
    best and second-best logit over every decision taken): the gap tells how close
    the path came to a tie."""
    blank = n_classes - 1
    emb = W["rnnt.embed.weight"].astype(dtype)
    w_ih = W["rnnt.lstm.weight_ih_l0"].astype(dtype)
    w_hh = W["rnnt.lstm.weight_hh_l0"].astype(dtype)
    b_ih = W["rnnt.lstm.bias_ih_l0"].astype(dtype)
    b_hh = W["rnnt.lstm.bias_hh_l0"].astype(dtype)
    P = w_hh.shape[1]
    h = np.zeros(P, dtype)
    c = np.zeros(P, dtype)
    g, state = lstm_step(np.zeros(emb.shape[1], dtype), h, c, w_ih, w_hh, b_ih, b_hh)
    h, c = g, state
    symbols: List[int] = []
    frames: List[int] = []
    min_gap = np.inf
    enc = np.asarray(enc, dtype)
    for t in range(enc.shape[0]):
        emitted = 0
        while emitted < max_symbols:
            z = rnnt_joint(enc[t], h, W, act, dtype)
            k = int(np.argmax(z))
            top2 = np.partition(z, -2)[-2:]
            min_gap = min(min_gap, float(top2[1] - top2[0]))
            if k == blank:
                break
            symbols.append(k)
            frames.append(t)
            h, c = lstm_step(emb[k], h, c, w_ih, w_hh, b_ih, b_hh)
            emitted += 1
    return symbols, frames, float(min_gap)
