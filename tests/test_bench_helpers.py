"""Host logic of bench.py that needs no GPU: the share of work the paired kernel takes."""
import os
import sys
import types

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def fake(blocks, nb, cnt):
    return types.SimpleNamespace(key_rows=lambda *a, **k: (torch.tensor(blocks, dtype=torch.int32),
                                                           torch.tensor(nb, dtype=torch.int32), None,
                                                           torch.tensor(cnt, dtype=torch.int32)))


def problem(layout, seqlens_q=None, S1=0, topk=3, block_size=16):
    return types.SimpleNamespace(indices=None, k=None, q=None, q_rope=None, block_size=block_size, layout=layout,
                                 sparse_mode=3, seqlens_q=seqlens_q, seqlens_kv=seqlens_q, S1=S1, topk=topk)


def test_pairs_need_identical_live_blocks_in_one_sequence():
    # rows 0 / 1: same live blocks (entries past the count differ); rows 2 / 3: a different block
    blocks = [[1, 2, -7], [1, 2, 5], [3, 4, 0], [3, 9, 0], [1, 0, 0]]
    nb, cnt = [2, 2, 2, 2, 1], [32, 32, 32, 32, 16]
    S = fake(blocks, nb, cnt)
    assert bench.paired_work_fraction(problem("TND", np.array([4, 5])), S) == 64 / 144
    # the same rows split across two sequences (TND cumulative ends): no pair
    assert bench.paired_work_fraction(problem("TND", np.array([1, 5])), S) == 0.0
    # BSND: sequences of S1 = 2 rows, rows 0 / 1 in batch 0
    assert bench.paired_work_fraction(problem("BSND", S1=2), S) == 64 / 144


def test_empty_rows_never_pair():
    S = fake([[0], [0]], [0, 0], [0, 0])
    assert bench.paired_work_fraction(problem("BSND", S1=2, topk=1), S) == 0.0


def test_smaller_workload5_case_keeps_each_rows_share():
    """`bench.py --workload 5 --seqs S` (profiling captures): S1 = S2 = S and topk scaled with S, so
    row t still selects min(t + 1, topk) distinct causal keys, padded with -1 — the full workload's
    recipe at a quarter (or any fraction) of its size."""
    from workloads import make_device_problem
    S = 1024
    p = make_device_problem(5, device="cpu", seqs=[S])
    topk = 8192 * S // 32768
    assert p.layout == "BSND" and p.block_size == 1 and not p.deterministic
    assert tuple(p.indices.shape) == (1, S, 1, topk) and tuple(p.q.shape) == (1, S, 128, 512)
    idx = p.indices.reshape(S, topk)
    for t in (0, 1, topk - 2, topk - 1, topk, S // 2, S - 1):
        row = idx[t]
        live = row[row >= 0]
        assert live.numel() == min(t + 1, topk), t
        assert bool((row[live.numel():] == -1).all()), t
        assert int(live.max()) <= t and live.unique().numel() == live.numel(), t
