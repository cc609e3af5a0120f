"""KV parallelism across ranks (long_context_decode_helix_b200.kvp), host side, no GPU: the
placement and ownership rules against the oracle's layout, and two gloo ranks running the exchange
with the oracle standing in for the partial and combine kernels (the kernels themselves are tested
on the GPU)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from long_context_decode_helix_b200 import kvp


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_token_rank_and_local_positions_follow_the_round_robin_layout(world):
    S = 1000
    sets = oracle.shard_tokens(S, world, "rr", 16)
    for r in range(world):
        assert np.array_equal(kvp.local_positions(S, r, world).numpy(), sets[r])
    for t in range(S):
        assert kvp.token_rank(t, world) == oracle.rr_place(t, world, 16)[0]


def test_append_valid_marks_the_owner_of_each_new_token():
    world, pos = 4, [0, 15, 16, 47, 64, 1000]
    for r in range(world):
        nv = kvp.append_valid(pos, r, world).tolist()
        assert nv == [1 if oracle.rr_place(t, world, 16)[0] == r else 0 for t in pos]
    # every new token has exactly one owner
    assert sum(kvp.append_valid(pos, r, world) for r in range(world)).tolist() == [1] * len(pos)


@pytest.mark.parametrize("world", [2, 3, 8])
def test_decode_loop_appends_build_each_ranks_shard(world):
    """Token by token, each rank appends exactly the new tokens ``append_valid`` gives it; after S
    steps its history is its shard of the layout, for requests of different lengths."""
    lens0, S = [0, 37], 300
    held = [[[] for _ in lens0] for _ in range(world)]
    for step in range(S):
        pos = [L + step for L in lens0]
        for r in range(world):
            for b, v in enumerate(kvp.append_valid(pos, r, world).tolist()):
                if v:
                    held[r][b].append(pos[b])
    for r in range(world):
        for b, L0 in enumerate(lens0):
            want = [t for t in kvp.local_positions(L0 + S, r, world).tolist() if t >= L0]
            assert held[r][b] == want


@pytest.mark.parametrize("world,Hq", [(1, 128), (2, 128), (3, 128), (8, 128), (4, 6), (16, 16)])
def test_owned_heads_partition_the_heads(world, Hq):
    ranges = [kvp.owned_heads(r, world, Hq) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == Hq
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0
    sizes = [h1 - h0 for h0, h1 in ranges]
    assert max(sizes) - min(sizes) <= 1


def _oracle_combine(o_parts, lses, h0, h1, out=None, lse_out=None, out_dtype=None):
    """The oracle's LSE combine over the sources' heads [h0, h1), in the kernel's calling form."""
    O_s = np.stack([o[:, h0:h1].numpy() for o in o_parts])
    L_s = np.stack([l[:, h0:h1].numpy() for l in lses])
    O, L = oracle.combine(O_s, L_s)
    return torch.from_numpy(O), torch.from_numpy(L)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q, K, V, lens, scale, errors):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        B, Hq, _ = q.shape
        dv = V.shape[-1]
        ex = kvp.KVPExchange(B, Hq, dv, "cpu", mode="gather", combine_fn=_oracle_combine)
        # this rank's partial over its own tokens of every request (stand-in for the kernel)
        for b in range(B):
            idx = kvp.local_positions(lens[b], rank, world).numpy()
            for h in range(Hq):
                o, l = oracle.attend(q[b, h : h + 1], K[b, idx], V[b, idx], scale)
                ex.o_partial[0, b, h] = torch.from_numpy(o[0])
                ex.lse[0, b, h] = float(l[0])
        for _ in range(2):  # twice: the exchange is reusable step after step
            O, L = ex.combine()
        h0, h1 = kvp.owned_heads(rank, world, Hq)
        assert tuple(O.shape) == (B, h1 - h0, dv) and tuple(L.shape) == (B, h1 - h0)
        # the partials travel in fp32 (the kernels' buffers): agreement to fp32 rounding
        for b in range(B):
            Oref, Lref = oracle.attend(q[b, h0:h1], K[b, : lens[b]], V[b, : lens[b]], scale)
            np.testing.assert_allclose(O[b].double().numpy(), Oref, rtol=1e-5, atol=1e-6)
            np.testing.assert_allclose(L[b].double().numpy(), Lref, rtol=1e-6, atol=1e-6)
        ex.close()
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        errors.put(f"rank {rank}: {type(e).__name__}: {e}")


@pytest.mark.parametrize("world,Hq", [(2, 6), (3, 6), (3, 2)])
def test_gather_exchange_equals_unsharded_attention(world, Hq):
    """Every rank ends with the unsharded attention of the heads it owns (none, when there are
    more ranks than heads), to the fp32 rounding of the exchanged partials."""
    rng = np.random.default_rng(5)
    B, d, dv = 2, 16, 8
    lens = [70, 3]  # the second request has no token on some ranks: empty partials
    S = max(lens)
    q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, S, d))
    V = rng.standard_normal((B, S, dv))
    ctx = mp.get_context("spawn")
    errors = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, K, V, lens, 0.25, errors))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    msgs = []
    while not errors.empty():
        msgs.append(errors.get())
    assert not msgs, "\n".join(msgs)
    assert all(p.exitcode == 0 for p in procs)


def _decode_rank_main(rank, world, port, q, K, V, lens0, steps, scale, errors):
    """One rank of a KV-parallel decode loop (``kvp.KVPDecodeRank``, as ``bench.py --kvp-ranks``
    drives it) with the oracle standing in for the append, partial and combine kernels."""
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        B, Hq, _ = q.shape
        dv = V.shape[-1]
        # the rank's local history: its tokens of every request's prefill
        held = [[int(t) for t in kvp.local_positions(L, rank, world)] for L in lens0]

        def append_fn(rows, n_valid):
            for b, v in enumerate(n_valid.tolist()):
                if v:
                    held[b].append(rows["pos"][b])

        def partial_fn(q_, o_part, lse):
            for b in range(B):
                idx = np.array(held[b], dtype=np.int64)
                for h in range(Hq):
                    if len(idx) == 0:  # an empty shard: O_s = 0, lse_s = -inf
                        o_part[0, b, h] = 0.0
                        lse[0, b, h] = float("-inf")
                        continue
                    o, l = oracle.attend(q_[b, h:h + 1], K[b, idx], V[b, idx], scale)
                    o_part[0, b, h] = torch.from_numpy(o[0])
                    lse[0, b, h] = float(l[0])

        ex = kvp.KVPExchange(B, Hq, dv, "cpu", mode="gather", combine_fn=_oracle_combine)
        dec = kvp.KVPDecodeRank(ex, append_fn, partial_fn, lens0)
        assert dec.owned_counts() == [len(h) for h in held]
        for s in range(steps):
            pos = [L + s for L in lens0]
            O, L = dec.step({"pos": pos}, q)
        assert dec.owned_counts() == [len(h) for h in held]
        h0, h1 = kvp.owned_heads(rank, world, Hq)
        for b in range(B):
            S = lens0[b] + steps
            Oref, Lref = oracle.attend(q[b, h0:h1], K[b, :S], V[b, :S], scale)
            np.testing.assert_allclose(O[b].double().numpy(), Oref, rtol=1e-5, atol=1e-6)
            np.testing.assert_allclose(L[b].double().numpy(), Lref, rtol=1e-6, atol=1e-6)
        ex.close()
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        errors.put(f"rank {rank}: {type(e).__name__}: {e}")


@pytest.mark.parametrize("world", [2])
def test_decode_loop_over_ranks_equals_unsharded_attention(world):
    """Prefill, then 40 decode steps: every new token lands on exactly one rank, and after the last
    step each rank's owned heads equal unsharded attention over the whole history."""
    rng = np.random.default_rng(9)
    B, Hq, d, dv, steps = 2, 4, 16, 8, 40
    lens0 = [33, 5]
    S = max(lens0) + steps
    q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, S, d))
    V = rng.standard_normal((B, S, dv))
    ctx = mp.get_context("spawn")
    errors = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_decode_rank_main,
                         args=(r, world, port, q, K, V, lens0, steps, 0.25, errors))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
    msgs = []
    while not errors.empty():
        msgs.append(errors.get())
    assert not msgs, "\n".join(msgs)
    assert all(p.exitcode == 0 for p in procs)
