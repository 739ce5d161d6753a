"""Expert parallelism on two gloo ranks (CPU): the exchange of candidates, slots, rows and
expert outputs around the owner's capacity selection and FFN, with every compute step done by
the oracle.  Each rank's outputs and routing must equal the single-batch oracle layer's on the
union of both ranks' tokens, bit for bit ("Expert Networks > Worked Example: Expert
Specialization": the experts run concurrently on separate hardware; the capacity, drop priority and
slots are those of the whole batch)."""
import math

import pytest
import torch.multiprocessing as mp

from tests import ep_worker


@pytest.mark.parametrize("cfg", [
    (48, 16, 24, 8, 2, 1.0, "f32", 0, 1),        # drops at the experts' owners
    (40, 16, 24, 4, 1, 0.5, "f32", 0, 2),        # top-1, half the pairs dropped
    (32, 8, 12, 6, 3, 0.75, "f32", 2, 3),        # arrival order
    (32, 8, 12, 6, 3, 1.0, "f32", 1, 4),         # renormalised weights
    (24, 16, 32, 4, 2, math.inf, "bf16", 0, 5),  # dropless, bf16 values
    (16, 8, 8, 2, 2, 0.5, "f32", 0, 6)])         # one expert per rank, k = E
def test_expert_parallel_matches_single_batch(cfg):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = 29600 + cfg[-1]
    mp.start_processes(ep_worker.cpu_rank, args=(2, port, cfg, out), nprocs=2,
                       start_method="spawn")
    assert out[0] == [] and out[1] == [], (out[0], out[1])


@pytest.mark.parametrize("cfg", [
    (16, 16, 24, 8, 2, 0.75, "f32", 0, 11),      # two experts per rank, drops
    (12, 8, 16, 4, 2, 1.0, "bf16", 2, 12)])      # one expert per rank, arrival order
def test_expert_parallel_four_ranks(cfg):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = 29640 + cfg[-1]
    mp.start_processes(ep_worker.cpu_rank, args=(4, port, cfg, out), nprocs=4,
                       start_method="spawn")
    assert all(out[r] == [] for r in range(4)), dict(out)


def test_group_order_is_a_stable_sort_by_destination():
    """The exchange groups pairs by owner with a counting sort; it must equal a stable sort."""
    import torch
    from expert_ffn_layer_router_b200 import ep
    g = torch.Generator().manual_seed(1)
    for world in (1, 2, 3, 8, 64):
        for P in (0, 1, 31, 5000):
            dest = torch.randint(0, world, (P,), generator=g)
            order, counts = ep._group_order(dest, world)
            assert torch.equal(order, torch.argsort(dest, stable=True))
            assert torch.equal(counts, torch.bincount(dest, minlength=world))
