"""The sink / local / update-buffer bookkeeping (ReindexPlan) on the CPU.

The plan decides, step by step, which dense-tail tokens move into the index
and when; DecodeCache executes its actions on the GPU.  Here the actions are
applied to a plain model of token positions, and after every step:
  * the index holds exactly the positions [sink, z) and the tail [z, T) (no
    token lost, none in both);
  * the tail never drops to `local` or below and never passes its capacity;
  * in line, a batch of `update` oldest tail tokens moves at once when the
    tail is full;
  * asynchronously, a batch is staged as consecutive pieces from the tail's
    start, in order, `pieces` of them, and published `publish_lag` steps after
    its last piece -- then exactly the staged tokens leave the tail.
"""
import pytest

from kv_cache_top_b200.decode_cache import ReindexPlan


@pytest.mark.parametrize("local,update,async_reindex,pieces,lag", [
    (64, 32, False, 4, 1),
    (64, 32, True, 4, 1),
    (512, 512, True, 4, 1),
    (512, 512, False, 1, 1),
    (16, 8, True, 1, 1),
    (16, 8, True, 3, 2),
    (16, 5, True, 9, 1),        # more pieces than the batch allows: clamped to update - lag
    (16, 2, True, 4, 5),        # the shortest asynchronous batch: one piece, lag 1
    (100, 37, True, 6, 3),
])
def test_plan_keeps_every_token_in_index_or_tail(local, update, async_reindex, pieces, lag):
    sink, T0, steps = 4, 1000, 3000
    plan = ReindexPlan(local, update, async_reindex, pieces, lag)
    z = T0 - local                     # zone end: index = [sink, z), tail = [z, T)
    T = T0
    staged = []                        # tail offsets staged for the current batch
    pieces_seen, last_piece_step = 0, None
    batches = 0
    lag = max(1, min(lag, update - 1))               # the plan keeps pieces + lag <= update
    eff_pieces = max(1, min(pieces, update - lag))
    for t in range(steps):
        acts = plan.before_token()
        for a in acts:
            if a[0] == "reindex":
                assert not async_reindex
                assert a[1] == T - z == local + update          # the tail was full
                z += update
                batches += 1
            elif a[0] == "stage":
                assert async_reindex
                first, count, tail_seen = a[1], a[2], a[3]
                assert count >= 1
                assert first == len(staged)                     # consecutive, from the tail's start
                assert (tail_seen is not None) == (first == 0)  # the first piece copies the tail
                if tail_seen is not None:
                    assert tail_seen == T - z >= local + update
                staged.extend(range(first, first + count))
                assert first + count <= T - z                   # only tokens already in the tail
                pieces_seen += 1
                last_piece_step = t
            else:
                assert async_reindex and a[0] == "publish"
                assert staged == list(range(update))            # exactly the oldest `update` tokens
                assert pieces_seen == eff_pieces
                assert t - last_piece_step == lag
                z += update
                batches += 1
                staged, pieces_seen = [], 0
        assert len(acts) <= 1
        plan.add_token()
        T += 1
        # the plan's view agrees with the model
        assert plan.tail == T - z
        assert plan.published == z - (T0 - local)
        assert plan.reindexed == batches
        assert local < plan.tail <= plan.max_tail
        assert plan.staging == (len(staged) > 0 or (async_reindex and plan.staged_for >= 0))
    # batches move at the rate tokens arrive
    assert abs(batches * update - (steps - update)) <= update + eff_pieces + lag


def test_plan_bounds_the_staging_cycle():
    # more pieces than the batch allows: clamped so a batch drains as fast as tokens arrive
    plan = ReindexPlan(16, 5, True, 9, 1)
    assert plan.pieces + plan.lag <= plan.update
    with pytest.raises(ValueError):
        ReindexPlan(16, 1, True, 1, 1)


def test_plan_capacity_is_checked():
    plan = ReindexPlan(8, 4, True, 2, 1)
    plan.tail = plan.max_tail
    with pytest.raises(RuntimeError):
        plan.add_token()
