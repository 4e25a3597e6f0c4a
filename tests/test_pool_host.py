"""Host block pool and continuous-batching planner (include/deltakv_pool.h), on the CPU.

The pool hands out the physical blocks of the paged cache; the planner turns queued requests into the compress
and decode batches of each serving step.  Both are host C++ in libdeltakv.so and need no GPU.  The tests check
the pool's bookkeeping against a plain model under random operations, and drive the planner through serving
loops (with preemption under block pressure) while checking every plan against the request-level accounting
the header defines.
"""
import numpy as np
import pytest

from residual_kv_cache_delta_b200 import deltakv as D
from residual_kv_cache_delta_b200 import pool as P


def _ceil(a, b):
    return -(-a // b)


def test_pool_exports_and_status_name():
    lib = D.load_library()
    for name in P.EXPORTED:
        assert hasattr(lib, name), name
    assert D.status_string(P.DKV_ERR_OUT_OF_BLOCKS) == "block pool exhausted"


def test_pool_in_order_placement_and_tables():
    p = P.BlockPool(num_blocks=10, block_tokens=16, max_seqs=4, max_blocks_per_seq=6)
    a, b = p.open(), p.open()
    p.grow(a, 33)                   # 3 blocks
    p.grow(b, 16)                   # 1 block
    p.grow(a, 40)                   # still 3 blocks
    assert p.info(a) == (40, 3) and p.info(b) == (16, 1)
    t = p.block_tables([a, b], 5)
    assert t.tolist() == [[0, 1, 2, -1, -1], [3, -1, -1, -1, -1]]
    assert p.num_free() == 6
    with pytest.raises(D.DeltaKVError):
        p.block_tables([a], 2)      # a holds 3 blocks
    with pytest.raises(D.DeltaKVError):
        p.grow(a, 39)               # sequences only grow
    p.close(a)
    assert p.num_free() == 9
    c = p.open()
    p.grow(c, 1)
    assert p.block_tables([c], 1)[0, 0] == 0  # freed blocks are reused first, first block first


def test_pool_reservation_is_all_or_nothing():
    p = P.BlockPool(num_blocks=5, block_tokens=16, max_seqs=3, max_blocks_per_seq=4)
    a, b = p.open(), p.open()
    p.grow(a, 48)
    with pytest.raises(P.OutOfBlocks):
        p.grow(b, 48)               # needs 3, 2 free
    assert p.info(b) == (0, 0) and p.num_free() == 2
    with pytest.raises(P.OutOfBlocks):
        p.grow(a, 80)               # 5 blocks > max_blocks_per_seq
    assert p.info(a) == (48, 3)
    p.open()
    with pytest.raises(P.OutOfBlocks):
        p.open()                    # max_seqs open


def test_pool_seeded_placement_is_a_permutation():
    n = 257
    p = P.BlockPool(num_blocks=n, block_tokens=16, max_seqs=1, max_blocks_per_seq=n, seed=12345)
    s = p.open()
    p.grow(s, n * 16)
    ids = p.block_tables([s], n)[0]
    assert sorted(ids.tolist()) == list(range(n))
    assert ids.tolist() != list(range(n))
    q = P.BlockPool(num_blocks=n, block_tokens=16, max_seqs=1, max_blocks_per_seq=n, seed=12345)
    s2 = q.open()
    q.grow(s2, n * 16)
    assert np.array_equal(q.block_tables([s2], n)[0], ids)  # seeded: reproducible


def test_pool_random_operations_keep_blocks_disjoint_and_conserved():
    rng = np.random.default_rng(0)
    nb, R, ms, mbps = 64, 16, 8, 20
    p = P.BlockPool(nb, R, ms, mbps, seed=7)
    model = {}  # seq -> length
    for _ in range(3000):
        op = rng.integers(3)
        if op == 0:
            try:
                s = p.open()
                assert s not in model
                model[s] = 0
            except P.OutOfBlocks:
                assert len(model) == ms
        elif op == 1 and model:
            s = int(rng.choice(list(model)))
            new_len = model[s] + int(rng.integers(0, 70))
            held = sum(_ceil(L, R) for L in model.values())
            need = _ceil(new_len, R) - _ceil(model[s], R)
            try:
                p.grow(s, new_len)
                model[s] = new_len
            except P.OutOfBlocks:
                assert _ceil(new_len, R) > mbps or need > nb - held
        elif op == 2 and model:
            s = int(rng.choice(list(model)))
            p.close(s)
            del model[s]
        seqs = sorted(model)
        held = sum(_ceil(L, R) for L in model.values())
        assert p.num_free() == nb - held
        if seqs:
            t = p.block_tables(seqs, mbps)
            used = t[t >= 0]
            assert len(used) == held and len(np.unique(used)) == held and (held == 0 or used.max() < nb)
            for i, s in enumerate(seqs):
                assert p.info(s) == (model[s], _ceil(model[s], R))
                assert np.all(t[i, :_ceil(model[s], R)] >= 0) and np.all(t[i, _ceil(model[s], R):] == -1)


def _serve(nb, R, max_batch, max_prefill, reqs, seed=0, max_steps=10000):
    """Drives the planner to completion, checking each plan; returns (steps, preemptions, finish order)."""
    pool = P.BlockPool(nb, R, max_batch, nb, seed=seed)
    bat = P.Batcher(pool, max_prefill, max_batch)
    info = {}
    for rid, (prompt, new) in enumerate(reqs):
        bat.submit(rid, prompt, new)
        info[rid] = dict(prompt=prompt, new=new, gen=0, cached=0, admitted_at=None)
    order, preempt = [], 0
    submitted = list(range(len(reqs)))
    for step in range(max_steps):
        w, r, f = bat.counts()
        if w == 0 and r == 0:
            break
        plan = bat.plan()
        preempt += plan.num_preempted
        assert len(plan.comp_req) == len(plan.dec_req) <= max_batch
        assert plan.cu_new[0] == 0 and np.all(np.diff(plan.cu_new) >= 1)
        prefill_rows = 0
        for i, rid in enumerate(plan.comp_req):
            st = info[int(rid)]
            n = int(plan.cu_new[i + 1] - plan.cu_new[i])
            if plan.comp_from[i] == 0:           # (re)admitted: the whole prefix, prompt + generated so far
                assert n == st["prompt"] + st["gen"] and plan.start_pos[i] == 0
                st["cached"] = 0
                prefill_rows += n
            else:                                # running: the token generated by the previous step
                assert n == 1 and plan.start_pos[i] == st["cached"] == plan.comp_from[i]
            st["cached"] += n
        nfresh = int(np.sum(plan.comp_from == 0))
        assert nfresh <= 1 or prefill_rows <= max_prefill
        assert plan.dec_req.tolist() == plan.comp_req.tolist()
        for i, rid in enumerate(plan.dec_req):
            st = info[int(rid)]
            assert plan.context_len[i] == st["cached"] == st["prompt"] + st["gen"]
        # the pool holds every block of every running sequence, and no block twice
        t = pool.block_tables(plan.dec_seq, nb)
        for i in range(len(plan.dec_seq)):
            nblk = _ceil(int(plan.context_len[i]), R)
            assert np.all(t[i, :nblk] >= 0) and np.all(t[i, nblk:] == -1)
        used = t[t >= 0]
        assert len(np.unique(used)) == len(used)
        fin = bat.commit()
        for rid in plan.dec_req:
            info[int(rid)]["gen"] += 1
        for rid in fin:
            assert info[rid]["gen"] == info[rid]["new"]
            order.append(rid)
    assert sorted(order) == submitted, "every request finishes"
    assert pool.num_free() == nb
    return step, preempt, order


def test_batcher_serves_everything_in_fifo_order_without_pressure():
    reqs = [(40 + 13 * i, 3 + (i % 4)) for i in range(12)]
    steps, preempt, order = _serve(nb=400, R=16, max_batch=16, max_prefill=4096, reqs=reqs)
    assert preempt == 0


def test_batcher_prefill_budget_limits_admission_per_step():
    reqs = [(100, 2)] * 6
    pool = P.BlockPool(1000, 16, 8, 1000)
    bat = P.Batcher(pool, 250, 8)
    for i, (a, b) in enumerate(reqs):
        bat.submit(i, a, b)
    plan = bat.plan()
    assert plan.comp_req.tolist() == [0, 1]          # 200 rows; a third prompt would exceed 250
    bat.commit()
    plan = bat.plan()
    assert plan.comp_req.tolist() == [0, 1, 2, 3]    # appends of 0, 1 and two new prompts


def test_batcher_preempts_under_block_pressure_and_recomputes():
    rng = np.random.default_rng(3)
    reqs = [(int(rng.integers(20, 120)), int(rng.integers(5, 60))) for _ in range(30)]
    steps, preempt, order = _serve(nb=24, R=16, max_batch=8, max_prefill=512, reqs=reqs, seed=99)
    assert preempt > 0


def test_batcher_rejects_requests_the_pool_can_never_hold():
    pool = P.BlockPool(8, 16, 4, 8)
    bat = P.Batcher(pool, 1000, 4)
    with pytest.raises(D.DeltaKVError):
        bat.submit(0, 16 * 8, 2)                     # 129 tokens at the last decode: 9 blocks > 8
    bat.submit(1, 16 * 8, 1)
    with pytest.raises(D.DeltaKVError):
        bat.submit(1, 10, 1)                         # duplicate id
    with pytest.raises(D.DeltaKVError):
        bat.commit()                                 # nothing planned
