"""The combine over separate source buffers (helix_attn_combine_sources), and the KV-parallel
exchange across processes (long_context_decode_helix_b200.kvp) with the library's own partial and
combine kernels: two processes share one GPU, each holding one KVP shard of every request in a
kvp = 1 cache, and the owner's combine reads the other process's partials through a CUDA IPC
mapping. Only host barriers order the processes; no kernel waits on another."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads as wl
import _gpu

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("kind", ["gqa", "mla"])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_combine_sources_equals_combine(kind, out_dtype):
    """Per-shard views of one partial as separate sources: bit-identical to helix_attn_combine on
    every head range, and to the oracle."""
    if kind == "gqa":
        w, lens = wl.WORKLOADS["gqa_s128k"].with_(B=3, Hq=32, Hkv=2, S=2000, kvp=4), [2000, 5, 900]
    else:
        w, lens = wl.WORKLOADS["mla_s1m"].with_(B=2, S=1500, kvp=3), [1500, 100]
    hx = _gpu.hx()
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens)
    q = wl.query(w, "cuda")
    o_part, lse = hx.partial(cache, q, w.softmax_scale)
    full, full_lse = hx.combine(o_part, lse, out_dtype=out_dtype)
    srcs_o = [o_part[s] for s in range(w.kvp)]
    srcs_l = [lse[s] for s in range(w.kvp)]
    for h0, h1 in [(0, w.Hq), (0, 1), (5, 17), (w.Hq - 3, w.Hq)]:
        out, lse_out = hx.combine_sources(srcs_o, srcs_l, h0, h1, out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert torch.equal(out, full[:, h0:h1]) and torch.equal(lse_out, full_lse[:, h0:h1])
    # the sources in another order give the same merge up to the order of the sum
    out_r, lse_r = hx.combine_sources(srcs_o[::-1], srcs_l[::-1], 0, w.Hq, out_dtype=torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_allclose(out_r.cpu().numpy(), full.float().cpu().numpy(), atol=1e-2)
    np.testing.assert_allclose(lse_r.cpu().numpy(), full_lse.cpu().numpy(), atol=1e-5)
    for b in range(w.B):
        for h in range(0, w.Hkv if kind == "gqa" else 1):
            O, L, _, _ = _gpu.oracle_head_group(w, q, b, h, lens[b])
            hs = slice(h * w.G, (h + 1) * w.G)
            _gpu.assert_close_O(out_r[b, hs].cpu().numpy(), O, f"{kind} O b={b} h={h}")
            _gpu.assert_close_lse(lse_r[b, hs].cpu().numpy(), L, f"{kind} LSE b={b} h={h}")


def test_combine_sources_rejects_bad_arguments():
    hx = _gpu.hx()
    o = torch.zeros(2, 4, 8, device="cuda")
    l = torch.zeros(2, 4, device="cuda")
    with pytest.raises(hx.HelixError):
        hx.combine_sources([o], [l], 3, 3)  # empty head range
    with pytest.raises(hx.HelixError):
        hx.combine_sources([o], [l], 0, 5)  # past the last head
    with pytest.raises(hx.HelixError):
        hx.combine_sources([o] * 17, [l] * 17, 0, 4)  # more sources than the limit


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _kvp_rank(rank, world, port, mode, errors):
    try:
        sys.path.insert(0, HERE)
        sys.path.insert(0, os.path.dirname(HERE))
        import torch.distributed as dist

        import _gpu as g
        import workloads as w_
        from long_context_decode_helix_b200 import kvp

        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        torch.cuda.set_device(0)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        hx = g.hx()
        full = w_.WORKLOADS["gqa_s128k"].with_(B=2, Hq=16, Hkv=2, S=3000, kvp=world)
        lens = [3000, 1100]
        # this rank's shard of every request, as a kvp = 1 cache in increasing position order
        idx = [kvp.local_positions(L, rank, world) for L in lens]
        n_loc = [len(i) for i in idx]
        loc = full.with_(kvp=1, S=max(n_loc))
        cache = g.make_cache(loc)
        rows = w_.append_rows(full, 0, full.S, "cuda")
        k_loc = torch.zeros(full.B, max(n_loc), full.Hkv, full.d, dtype=torch.bfloat16,
                            device="cuda")
        v_loc = torch.zeros_like(k_loc)
        for b in range(full.B):
            k_loc[b, : n_loc[b]] = rows["k_new"][b, idx[b].cuda()]
            v_loc[b, : n_loc[b]] = rows["v_new"][b, idx[b].cuda()]
        hx.append(cache, k_loc, v_loc, n_valid=torch.tensor(n_loc, dtype=torch.int32,
                                                            device="cuda"))
        q = w_.query(full, "cuda")
        ex = kvp.KVPExchange(full.B, full.Hq, full.dv, "cuda", mode=mode)
        for _ in range(2):  # two steps: the exchange and its mappings are reusable
            hx.partial(cache, q, full.softmax_scale, ex.o_partial, ex.lse)
            O, L = ex.combine(out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert cache.err_bits() == 0
        h0, h1 = kvp.owned_heads(rank, world, full.Hq)
        O, L = O.cpu().numpy(), L.cpu().numpy()
        for b in range(full.B):
            for h in range(h0, h1):
                K, V = g.oracle_kv(full, b, h // full.G, lens[b])
                Oref, Lref = oracle.attend(oracle.attention._f64(q[b, h : h + 1]), K, V,
                                           full.softmax_scale)
                g.assert_close_O(O[b, h - h0][None], Oref, f"rank {rank} O b={b} h={h}")
                g.assert_close_lse(L[b, h - h0][None], Lref, f"rank {rank} LSE b={b} h={h}")
        ex.close()
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        import traceback

        errors.put(f"rank {rank}: {type(e).__name__}: {e}\n{traceback.format_exc()}")


@pytest.mark.parametrize("mode", ["peer", "gather"])
def test_kvp_exchange_two_processes(mode):
    """Two processes, one KVP shard each: the owned heads equal the unsharded attention."""
    world = 2
    ctx = mp.get_context("spawn")
    errors = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_kvp_rank, args=(r, world, port, mode, errors))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=600)
    for p in procs:
        if p.is_alive():
            p.kill()
    msgs = []
    while not errors.empty():
        msgs.append(errors.get())
    assert not msgs, "\n".join(msgs)
    assert all(p.exitcode == 0 for p in procs)
