"""Work split across GPUs and long-form chunking around the C ABI (host logic).

Nothing here computes any step of the recognition path; every step runs in
``libgam.so``.  This module decides which clips each rank decodes, cuts long
recordings into overlapping chunks, gathers the per-rank transcripts and joins
the transcripts of overlapping chunks.

* Batch sharding.  Clips are independent (each valid encoder frame sees only
  its own clip's samples), so a batch splits across ranks with no exchange on
  the data path.  ``partition`` balances the ranks' work by the clips'
  encoder cost (GEMM work grows with the frame count L', attention with L'^2),
  largest clip first onto the least loaded rank.  ``gather_transcripts`` is
  the one exchange: every rank's (clip index, tokens) to every rank, through
  torch.distributed (NCCL between GPUs, gloo on CPU).
* Long-form chunks.  "GigaAM v3 MLX", "Long-form transcription", recommends
  20 s chunks with 0-2 s of overlap for long audio.  ``chunk_long_audio`` cuts
  them; ``merge_overlapped`` keeps each token from the chunk that owns its
  time, splitting every overlap at its midpoint, so a token seen by two chunks
  is kept once.  A token's time is the centre of its encoder frame's input
  span: encoder frame t reads mel frames 4t - 6 .. 4t + 6 (two stride-2,
  kernel-5 convolutions), centred on mel frame 4t, whose samples start at
  160 * 4t; the centre is 640 t + 160 samples after the chunk's start.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np

SAMPLES_PER_ENCODER_FRAME = 640
FRAME_CENTRE_OFFSET = 160


def encoder_frames(n_samples: int) -> int:
    """Valid encoder frames L' of a clip of n samples (window 320, hop 160,
    L = floor((T - 1) / 2) after each stride-2 conv)."""
    if n_samples < 320:
        return 0
    F = 1 + (n_samples - 320) // 160
    L1 = max((F - 1) // 2, 0)
    return max((L1 - 1) // 2, 0)


def clip_cost(n_samples: int, cfg: dict) -> float:
    """Encoder work of one clip in FLOPs: the block GEMMs per frame plus attention."""
    L = encoder_frames(int(n_samples))
    d, f, nl = cfg["d_model"], cfg["ffn_dim"], cfg["n_layers"]
    gemm = 2.0 * (4 * d * f + 4 * d * d + 3 * d * d)
    return nl * (L * gemm + 4.0 * L * L * d)


def partition(lengths: Sequence[int], world: int, cfg: dict) -> List[List[int]]:
    """Clip indices per rank: longest-processing-time-first over the clips' costs
    (each clip to the currently least loaded rank, ties to the lower rank); each
    rank's indices in increasing order.  The largest load is at most 4/3 of the
    best possible split plus one clip."""
    costs = [clip_cost(n, cfg) for n in lengths]
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    load = [0.0] * world
    parts: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        parts[r].append(i)
        load[r] += costs[i]
    return [sorted(p) for p in parts]


def gather_transcripts(indices: Sequence[int], tokens: Sequence[Sequence[int]], n_clips: int,
                       group=None) -> List[List[int]]:
    """Every rank's transcripts to every rank, in clip order.  indices[j] is the
    batch position of this rank's j-th clip and tokens[j] its token ids."""
    import torch.distributed as td
    mine = [(int(i), [int(t) for t in tok]) for i, tok in zip(indices, tokens)]
    world = td.get_world_size(group)
    got: List[object] = [None] * world
    td.all_gather_object(got, mine, group=group)
    out: List[List[int]] = [[] for _ in range(n_clips)]
    seen = set()
    for part in got:
        for i, tok in part:
            if i in seen:
                raise ValueError(f"clip {i} decoded by two ranks")
            seen.add(i)
            out[i] = tok
    if len(seen) != n_clips:
        raise ValueError(f"{n_clips - len(seen)} clips were not decoded by any rank")
    return out


def chunk_long_audio(x: np.ndarray, chunk_samples: int, overlap_samples: int
                     ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Cut one recording into chunks of chunk_samples that start every
    chunk_samples - overlap_samples samples (the last one shorter).  Returns
    (chunks [n, chunk_samples] float32, zero padded; lengths [n] int32; starts [n])."""
    x = np.asarray(x, dtype=np.float32)
    if not 0 <= overlap_samples < chunk_samples:
        raise ValueError("need 0 <= overlap < chunk")
    step = chunk_samples - overlap_samples
    starts = [0]
    while starts[-1] + chunk_samples < len(x):
        starts.append(starts[-1] + step)
    chunks = np.zeros((len(starts), chunk_samples), np.float32)
    lens = np.zeros(len(starts), np.int32)
    for k, s in enumerate(starts):
        seg = x[s:s + chunk_samples]
        chunks[k, :len(seg)] = seg
        lens[k] = len(seg)
    return chunks, lens, np.asarray(starts, np.int64)


def token_times(starts: Sequence[int], frames: Sequence[Sequence[int]]) -> List[List[int]]:
    """Sample position of every token: chunk start + 640 t + 160 for encoder frame t."""
    return [[int(s) + SAMPLES_PER_ENCODER_FRAME * int(t) + FRAME_CENTRE_OFFSET for t in fr]
            for s, fr in zip(starts, frames)]


def merge_overlapped(tokens: Sequence[Sequence[int]], frames: Sequence[Sequence[int]], starts: Sequence[int],
                     lengths: Sequence[int]) -> Tuple[List[int], List[int]]:
    """Join the transcripts of consecutive overlapping chunks: chunk k keeps the
    tokens whose time lies in [b_(k-1), b_k), b_k the midpoint of the overlap of
    chunks k and k+1 (the first chunk from the start, the last to the end).
    Returns (tokens, their sample positions)."""
    n = len(starts)
    times = token_times(starts, frames)
    bounds = []
    for k in range(n - 1):
        end_k = int(starts[k]) + int(lengths[k])
        bounds.append((int(starts[k + 1]) + end_k) / 2.0)
    out_tok: List[int] = []
    out_time: List[int] = []
    for k in range(n):
        lo = bounds[k - 1] if k > 0 else -np.inf
        hi = bounds[k] if k < n - 1 else np.inf
        for tok, tm in zip(tokens[k], times[k]):
            if lo <= tm < hi:
                out_tok.append(int(tok))
                out_time.append(tm)
    return out_tok, out_time
