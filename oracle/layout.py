"""Token -> (KVP shard, local index, page, slot) placement rules, written out directly.

TEST INFRASTRUCTURE (see the package docstring).

Round-robin rule. Sources: paper summary (fdeinterviews.com), paragraph on the Helix layouts (new KV
entries rotate across the KVP ranks every 16 tokens, so memory fills evenly); NVIDIA technical blog,
Korean edition (open-lab.net), KV-cache section, worked example (tokens 1-16 on KVP 0, tokens 17-32
on KVP 1, counted from 1).

Readings where the pages are silent:
* positions are counted from 0, so token t belongs to block floor(t / 16), and block j goes to
  shard j mod P;
* the whole history is placed as if appended token by token (the pages describe only new entries);
* inside a shard, tokens keep increasing global order, so the local index of t is the number of
  earlier tokens of the same shard: floor(j / P) * 16 + t mod 16.

Contiguous rule (used by the tiny configuration): shard s holds [s*C, (s+1)*C) for a chunk C.

Paging: local index l lives on the shard's page floor(l / page_tokens) at slot l mod page_tokens.
"""

from __future__ import annotations

import numpy as np


def rr_place(t: int, P: int, block: int = 16):
    """Round-robin placement of global position t over P shards: returns (shard, local index)."""
    j, r = divmod(int(t), block)
    return j % P, (j // P) * block + r


def contig_place(t: int, C: int):
    """Contiguous placement with C tokens per shard: returns (shard, local index)."""
    return divmod(int(t), C)


def place(t: int, P: int, layout: str, block: int = 16, chunk: int | None = None):
    if layout == "rr":
        return rr_place(t, P, block)
    if layout == "contig":
        return contig_place(t, chunk)
    raise ValueError(layout)


def shard_tokens(S: int, P: int, layout: str, block: int = 16, chunk: int | None = None):
    """Global positions held by each shard, in local-index order: a list of P int64 arrays.

    Built by placing t = 0, 1, ..., S-1 one at a time, exactly as an append loop would.
    """
    out = [[] for _ in range(P)]
    for t in range(S):
        s, l_ = place(t, P, layout, block, chunk)
        assert l_ == len(out[s]), "local index must equal the count of earlier tokens in the shard"
        out[s].append(t)
    return [np.asarray(x, dtype=np.int64) for x in out]


def shard_lens(S: int, P: int, layout: str, block: int = 16, chunk: int | None = None):
    """Number of tokens each shard holds after S tokens have been placed."""
    n = [0] * P
    for t in range(S):
        n[place(t, P, layout, block, chunk)[0]] += 1
    return n


def page_slot(l_: int, page_tokens: int = 64):
    """(page index within the shard, slot within the page) of local index l."""
    return divmod(int(l_), page_tokens)
