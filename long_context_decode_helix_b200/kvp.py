"""KV parallelism across GPUs: one KVP shard per rank, and the exchange of the partials.

Paper summary, paragraph on KV parallelism, and the paper review's "The Secret Weapon" prompt: the
KV history of every request is split over the KVP ranks; each rank attends over its own slice and
produces, per query head, a partial output normalised over that slice and its log-sum-exp; an
all-to-all then brings the partials of every head group to the rank that owns the group, which
rescales and sums them (the LSE combine).

Here rank r of a process group of N ranks is KVP shard r. It keeps shard r of every request's
history (the tokens the round-robin rule places on shard r) in a cache with kvp = 1, runs the
partial kernel over it for every head, and the exchange gives each rank the N partials of the
heads it owns (``owned_heads``). Two forms of the exchange, both ending in the library's own
combine kernel (``combine_sources``):

* ``"peer"``: every rank maps the other ranks' partial buffers into its address space once (CUDA
  IPC, through torch's sharing of CUDA tensors); each step, after a barrier that says every rank's
  partial is written, the owner's combine reads its heads' rows of all N partials straight from the
  other GPUs' memory with plain loads over NVLink: the exchange and the merge are one kernel. A
  second barrier keeps a rank from overwriting its partial while the others may still read it.
* ``"gather"``: an all-gather of the partials into local buffers (NCCL, or gloo for CPU tests),
  then the same combine. It moves N times the bytes the owner needs and maps no memory.

The host side (placement of new tokens, head ownership, the barriers and the collective) is plain
Python over ``torch.distributed``; every step of the attention arithmetic runs in the library's
kernels.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def owned_heads(rank: int, world: int, num_q_heads: int) -> tuple[int, int]:
    """Head range [h0, h1) whose combine rank ``rank`` performs: contiguous, sizes differ by at
    most one."""
    base, rem = divmod(num_q_heads, world)
    h0 = rank * base + min(rank, rem)
    return h0, h0 + base + (1 if rank < rem else 0)


def token_rank(t: int, world: int, rr_block: int = 16) -> int:
    """The KVP rank that stores history position t under round-robin placement: blocks of
    ``rr_block`` consecutive tokens go to the ranks in turn, starting with rank 0."""
    return (t // rr_block) % world


def append_valid(positions, rank: int, world: int, rr_block: int = 16, device="cpu"):
    """For a one-token append at history positions ``positions[b]`` (the request's current length),
    the ``n_valid`` row of this rank: 1 where the new token belongs to it, else 0."""
    return torch.tensor([1 if token_rank(int(t), world, rr_block) == rank else 0 for t in positions],
                        dtype=torch.int32, device=device)


def owned_count(L: int, rank: int, world: int, rr_block: int = 16) -> int:
    """How many of the history positions t < L rank ``rank`` stores: whole rounds of the rotation
    give rr_block tokens each, then the rank's part of the last, partial round."""
    full, rem = divmod(int(L), rr_block * world)
    return full * rr_block + min(max(rem - rank * rr_block, 0), rr_block)


def local_positions(S: int, rank: int, world: int, rr_block: int = 16) -> torch.Tensor:
    """The history positions t < S that rank ``rank`` stores, in increasing order (its local
    history, as a kvp = 1 cache holds it)."""
    t = torch.arange(S, dtype=torch.int64)
    return t[(t // rr_block) % world == rank]


class KVPExchange:
    """The exchange and combine of one decode step on one rank.

    ``o_partial`` [1][B][Hq][dv] and ``lse`` [1][B][Hq] (fp32) are this rank's partial buffers: the
    partial kernel writes them (pass them to ``helix.partial`` of the rank's kvp = 1 cache), then
    ``combine()`` returns (O, LSE) for the heads ``owned_heads(rank, world, Hq)``: O [B][h1 - h0][dv].
    Every rank must call ``combine()`` the same number of times (it holds collectives).
    ``combine_fn`` replaces the library's combine (same signature as ``combine_sources``), for tests
    of the host logic on machines without a GPU.
    """

    def __init__(self, batch: int, num_q_heads: int, v_dim: int, device, mode: str = "peer",
                 group=None, combine_fn=None):
        if mode not in ("peer", "gather"):
            raise ValueError("mode is 'peer' or 'gather'")
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if self.world > 16:
            raise ValueError("at most 16 KVP ranks (the combine's source limit)")
        self.mode = mode
        self.B, self.Hq, self.dv = batch, num_q_heads, v_dim
        self.h0, self.h1 = owned_heads(self.rank, self.world, num_q_heads)
        self.device = torch.device(device)
        self.o_partial = torch.zeros(1, batch, num_q_heads, v_dim, dtype=torch.float32,
                                     device=self.device)
        self.lse = torch.full((1, batch, num_q_heads), float("-inf"), dtype=torch.float32,
                              device=self.device)
        if combine_fn is None:
            from . import combine_sources as combine_fn
        self._combine = combine_fn
        self._peers = None
        if mode == "peer":
            if self.device.type != "cuda":
                raise ValueError("the peer exchange maps CUDA buffers")
            from torch.multiprocessing.reductions import reduce_tensor

            mine = (reduce_tensor(self.o_partial), reduce_tensor(self.lse))
            shared = [None] * self.world
            dist.all_gather_object(shared, mine, group=group)
            peers = []
            for r, ((fo, ao), (fl, al)) in enumerate(shared):
                if r == self.rank:
                    peers.append((self.o_partial, self.lse))
                else:  # another process's buffers, mapped into this one
                    peers.append((fo(*ao), fl(*al)))
            self._peers = peers
        else:
            self._all_o = torch.empty(self.world, batch, num_q_heads, v_dim, dtype=torch.float32,
                                      device=self.device)
            self._all_lse = torch.empty(self.world, batch, num_q_heads, dtype=torch.float32,
                                        device=self.device)

    def _sync(self):
        if self.device.type == "cuda":
            torch.cuda.current_stream(self.device).synchronize()
        dist.barrier(group=self.group)

    def _merge(self, o_parts, lses, out, lse_out, out_dtype):
        if self.h1 == self.h0:  # more ranks than heads: this rank owns none
            return (torch.empty(self.B, 0, self.dv, dtype=out_dtype, device=self.device),
                    torch.empty(self.B, 0, dtype=torch.float32, device=self.device))
        return self._combine(o_parts, lses, self.h0, self.h1, out=out, lse_out=lse_out,
                             out_dtype=out_dtype)

    def combine(self, out=None, lse_out=None, out_dtype=torch.bfloat16):
        """Exchange the partials and merge the owned heads; returns (O, LSE)."""
        if self.mode == "peer":
            self._sync()  # every rank's partial is written
            o_parts = [o[0] for o, _ in self._peers]
            lses = [l[0] for _, l in self._peers]
            res = self._merge(o_parts, lses, out, lse_out, out_dtype)
            self._sync()  # nobody reads a partial any more: it may be overwritten
            return res
        dist.all_gather_into_tensor(self._all_o, self.o_partial, group=self.group)
        dist.all_gather_into_tensor(self._all_lse, self.lse, group=self.group)
        return self._merge(list(self._all_o), list(self._all_lse), out, lse_out, out_dtype)

    def close(self):
        """Drop the mappings of the other ranks' buffers (every rank calls it)."""
        self._peers = None
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)


class KVPDecodeRank:
    """One rank's side of a KV-parallel decode step, as a decode loop runs it.

    Per step: the new token of every request is appended on the rank that owns its history
    position (``append_valid``), every rank runs the partial attention over its local shard for all
    heads into the exchange's buffers, and ``exchange.combine()`` returns the LSE-combined output of
    the heads this rank owns.

    ``append_fn(rows, n_valid)`` appends one new row per request where ``n_valid[b]`` is 1 (for the
    library: ``helix.append(cache, **rows, n_valid=n_valid)`` on the rank's kvp = 1 cache);
    ``partial_fn(q, o_partial, lse)`` writes this rank's partials (``helix.partial``). Both are
    arguments so the loop's host logic can be exercised without a GPU.
    """

    def __init__(self, exchange: KVPExchange, append_fn, partial_fn, lengths, rr_block: int = 16):
        self.ex = exchange
        self.append_fn = append_fn
        self.partial_fn = partial_fn
        self.rr_block = rr_block
        self.lengths = [int(L) for L in lengths]  # every request's global history length

    def owned_counts(self):
        """How many tokens of each request's current history this rank stores."""
        return [owned_count(L, self.ex.rank, self.ex.world, self.rr_block) for L in self.lengths]

    def append(self, rows):
        """Append the step's new token of every request (on its owner only)."""
        nv = append_valid(self.lengths, self.ex.rank, self.ex.world, self.rr_block,
                          device=self.ex.device)
        self.append_fn(rows, nv)
        self.lengths = [L + 1 for L in self.lengths]

    def attend(self, q, out=None, lse_out=None, out_dtype=torch.bfloat16):
        """Partial attention over the local shard, then the exchange and combine."""
        self.partial_fn(q, self.ex.o_partial, self.ex.lse)
        return self.ex.combine(out=out, lse_out=lse_out, out_dtype=out_dtype)

    def step(self, rows, q, out=None, lse_out=None, out_dtype=torch.bfloat16):
        """One decode step: append, partial, exchange + combine; returns (O, LSE) of the owned
        heads."""
        self.append(rows)
        return self.attend(q, out, lse_out, out_dtype)

