"""Host side of the query-row sharded backward, without a GPU: the work-balanced
row partition, the identity it relies on (the oracle's key-side sums over disjoint
row sets add up to the whole; dQuery rows are independent), and the two-rank
orchestration over torch.distributed (gloo, world size 2) with the device calls
replaced by stand-ins."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_attention_backward_sfa_b200.shard import balanced_row_ranges
from workloads import tiny_problem
from parity import oracle_backward, oracle_forward


def test_balanced_row_ranges_properties():
    rng = np.random.default_rng(5)
    for trial in range(200):
        n = int(rng.integers(0, 60))
        parts = int(rng.integers(1, 9))
        w = rng.integers(0, 50, size=n).astype(np.float64)
        for align in (1, 2):
            r = balanced_row_ranges(w, parts, align=align)
            assert len(r) == parts
            assert r[0][0] == 0 and r[-1][1] == n
            assert all(a <= b for a, b in r) and all(r[i][1] == r[i + 1][0] for i in range(parts - 1))
            # inner boundaries on multiples of `align` (pairs of rows 2m, 2m + 1 stay together)
            assert all(b % align == 0 or b == n for _, b in r[:-1])
            if n and w.sum() > 0:
                sums = np.array([w[a:b].sum() for a, b in r])
                assert sums.sum() == w.sum()
                # every boundary sits at the row edge nearest its target, then moves at most align - 1
                # rows to its multiple of `align`: no share is off by more than 2 * align - 1 rows
                assert np.abs(sums - w.sum() / parts).max() <= (2 * align - 1) * w.max() + 1e-9


def test_balanced_row_ranges_edges():
    assert balanced_row_ranges([], 3) == [(0, 0)] * 3
    assert balanced_row_ranges([0, 0, 0, 0], 2) == [(0, 2), (2, 4)]
    assert balanced_row_ranges([3, 1], 1) == [(0, 2)]
    assert balanced_row_ranges([1, 1, 1, 1, 4], 2) == [(0, 4), (4, 5)]
    assert balanced_row_ranges([1, 1, 1, 1, 1, 1], 2, align=1) == [(0, 3), (3, 6)]
    assert balanced_row_ranges([1, 1, 1, 1, 1, 1], 2) in ([(0, 2), (2, 6)], [(0, 4), (4, 6)])
    with pytest.raises(ValueError):
        balanced_row_ranges([1, -1], 2)
    with pytest.raises(ValueError):
        balanced_row_ranges([1, 1], 0)


def _problem():
    return tiny_problem(901, layout="TND", seqlens_q=[5, 7], seqlens_kv=[9, 12], N1=2, D=8, Dr=4, topk=4,
                        block_size=2, sparse_mode=3, index_mode="causal")


def test_oracle_row_shards_add_up():
    """Key-side sums over disjoint query-row ranges add up to the full sums; dQuery rows are unchanged."""
    p = _problem()
    out, m, l = oracle_forward(p)
    full = oracle_backward(p, out, m, l)
    ranges = balanced_row_ranges(np.ones(p.T1), 3)
    parts = [oracle_backward(p, out, m, l, tokens=list(range(a, b))) for a, b in ranges if b > a]
    for i in (1, 2, 4):  # dKey, dValue, dKeyRope
        np.testing.assert_allclose(sum(pt[i] for pt in parts), full[i], rtol=1e-12, atol=1e-14)
    for i in (0, 3):  # dQuery, dQueryRope: rows of each range, in order
        np.testing.assert_array_equal(np.concatenate([pt[i] for pt in parts]), full[i])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # (1) the reduction step on the oracle's partial sums: rank r's rows, all-reduced
        p = _problem()
        out, m, l = oracle_forward(p)
        rb, re_ = balanced_row_ranges(np.ones(p.T1), world)[rank]
        part = oracle_backward(p, out, m, l, tokens=list(range(rb, re_)))
        acc = torch.from_numpy(np.concatenate([part[1], part[4], part[2]], axis=1).copy())  # [T2, D | Dr | D]
        dist.all_reduce(acc)
        full = oracle_backward(p, out, m, l)
        ref = np.concatenate([full[1], full[4], full[2]], axis=1)
        ok1 = bool(np.allclose(acc.numpy(), ref, rtol=1e-12, atol=1e-14))

        # (2) sfa_grad_sharded's orchestration with the device calls replaced by stand-ins
        import sparse_attention_backward_sfa_b200.ops as ops
        from sparse_attention_backward_sfa_b200.shard import sfa_grad_sharded
        T1, T2 = 10, 10
        work = torch.tensor([1, 1, 1, 1, 1, 5, 5, 1, 1, 1], dtype=torch.int32)
        calls = []
        ops.compact_indices = lambda *a, **k: (None, None, work.clone())
        ops.sfa_dkv_accumulator = lambda *a, **k: torch.zeros(T2, 3, dtype=torch.int64)

        seen_dmax = []

        def fake_rows(*a, row_begin, row_end, dkv_accum, d_query, d_query_rope, dout_absmax=None, **k):
            calls.append((row_begin, row_end))
            seen_dmax.append(None if dout_absmax is None else float(dout_absmax))
            dkv_accum[row_begin:row_end] += 1      # each row "contributes" to the key row of the same index
            d_query[row_begin:row_end] = rank + 1
            return d_query, d_query_rope

        # each rank's own max|dOut| differs; the grid must use the max over ranks
        ops.dout_absmax = lambda *a, **k: torch.tensor([float(rank + 3)])
        ops.sfa_grad_rows = fake_rows
        ops.sfa_dkv_finalize = lambda acc, *a, **k: (acc.clone(), acc.clone(), acc.clone())
        q = torch.zeros(T1, 2)
        dq, dk, dv, dqr, dkr, rng_ = sfa_grad_sharded(q, None, None, None, None, None, None, None, torch.zeros(T1, 1),
                                                       None, scale=1.0, sparse_block_size=1, layout="TND",
                                                       sparse_mode=0, deterministic=True)
        expect = balanced_row_ranges(work.numpy(), world)[rank]
        ok2 = (calls == [expect] and rng_ == expect and bool((dk == 1).all()) and seen_dmax == [float(world + 2)]
               and bool((dq[expect[0]:expect[1]] == rank + 1).all())
               and bool((dq[:expect[0]] == 0).all()) and bool((dq[expect[1]:] == 0).all()))
        results[rank] = (ok1, ok2)
    finally:
        dist.destroy_process_group()


def test_sharded_reduction_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        mp.start_processes(_worker, args=(2, port, results), nprocs=2, join=True, start_method="spawn")
        assert dict(results) == {0: (True, True), 1: (True, True)}
