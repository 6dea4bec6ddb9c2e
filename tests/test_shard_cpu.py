"""Batch sharding across ranks and long-form chunk merging (host logic, CPU):
the length-balanced partition, the transcript gather over gloo with world
size 2, and the join of overlapping chunks ("GigaAM v3 MLX", "Long-form
transcription": 20 s chunks with 0-2 s of overlap)."""
import itertools
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from conformer_speech_recognition_b200 import shard, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_encoder_frames_match_plan():
    import oracle
    cfg = synth.workload_config("c2_varlen_b32_d768")
    for n in (1279, 1280, 16000, 320000, 480000, 37123):
        assert shard.encoder_frames(n) == oracle.clip_lengths_plan(n, cfg)["L2"]


def test_partition_covers_each_clip_once_and_balances():
    cfg = synth.workload_config("c2_varlen_b32_d768")
    lens = synth.clip_lengths("c2_varlen_b32_d768")
    for world in (1, 2, 3, 4, 8):
        parts = shard.partition(lens, world, cfg)
        assert sorted(itertools.chain(*parts)) == list(range(len(lens)))
        loads = [sum(shard.clip_cost(lens[i], cfg) for i in p) for p in parts]
        total = sum(loads)
        biggest = max(shard.clip_cost(n, cfg) for n in lens)
        # LPT bound: max load <= 4/3 of the best split, which is >= total / world
        assert max(loads) <= (4.0 / 3.0) * max(total / world, biggest) + 1e-6
    # exhaustive check on a tiny case: LPT is within 4/3 of the optimum
    small = [48000, 16000, 32000, 80000, 64000, 20000]
    parts = shard.partition(small, 2, cfg)
    costs = [shard.clip_cost(n, cfg) for n in small]
    best = min(max(sum(c for c, m in zip(costs, mask) if m), sum(c for c, m in zip(costs, mask) if not m))
               for mask in itertools.product([0, 1], repeat=len(small)))
    got = max(sum(costs[i] for i in p) for p in parts)
    assert got <= (4.0 / 3.0) * best + 1e-6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gather_worker(rank, world, port, out):
    import datetime
    import torch.distributed as td
    sys.path.insert(0, ROOT)
    from conformer_speech_recognition_b200 import shard as sh
    td.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                          timeout=datetime.timedelta(seconds=60))
    try:
        cfg = synth.workload_config("c2_varlen_b32_d768")
        lens = synth.clip_lengths("c2_varlen_b32_d768")
        mine = sh.partition(lens, world, cfg)[rank]
        tokens = [[i % 7] * (i % 5) for i in mine]  # stand-in transcripts: clip i -> (i % 5) x (i % 7)
        out[rank] = (mine, sh.gather_transcripts(mine, tokens, len(lens)))
    finally:
        td.destroy_process_group()


def test_gather_transcripts_gloo_world_2():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_gather_worker, args=(world, port, out), nprocs=world, join=True)
    n = len(synth.clip_lengths("c2_varlen_b32_d768"))
    expected = [[i % 7] * (i % 5) for i in range(n)]
    assert sorted(out[0][0] + out[1][0]) == list(range(n)) and not set(out[0][0]) & set(out[1][0])
    for r in range(world):
        assert out[r][1] == expected


def test_chunking_covers_the_recording():
    x = np.arange(100_000, dtype=np.float32)
    chunks, lens, starts = shard.chunk_long_audio(x, 32000, 4000)
    assert list(starts) == [0, 28000, 56000, 84000]
    assert list(lens) == [32000, 32000, 32000, 16000]
    for c, n, s in zip(chunks, lens, starts):
        np.testing.assert_array_equal(c[:n], x[s:s + n])
        assert np.all(c[n:] == 0)
    _, lens0, starts0 = shard.chunk_long_audio(x, 50000, 0)
    assert list(starts0) == [0, 50000] and list(lens0) == [50000, 50000]


@pytest.mark.parametrize("overlap", [0, 16000, 32000])
def test_merge_overlapped_recovers_a_timeline(overlap):
    """A known token timeline (one token per encoder-frame slot on a grid); each
    chunk 'decodes' exactly the tokens whose time falls inside it, at the frame
    the time maps to; the merge returns the timeline once, in order."""
    total = 60 * 16000
    chunk = 20 * 16000
    rng = np.random.default_rng(overlap)
    slots = np.sort(rng.choice(total // 640, size=400, replace=False))
    times = slots * 640 + 160
    toks = rng.integers(0, 33, size=len(times))
    _, lens, starts = shard.chunk_long_audio(np.zeros(total, np.float32), chunk, overlap)
    tok_c, frm_c = [], []
    for s, n in zip(starts, lens):
        inside = (times >= s) & (times < s + n) & ((times - s - 160) % 640 == 0)
        tok_c.append(toks[inside].tolist())
        frm_c.append(((times[inside] - s - 160) // 640).tolist())
    merged, mt = shard.merge_overlapped(tok_c, frm_c, starts, lens)
    assert merged == toks.tolist()
    assert mt == times.tolist()
