"""Plain, slow, fp64 CPU oracle for KV-parallel (sequence-sharded) decode attention.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or call anything in this
package.  The CUDA library never imports it and shares no code, header, table or helper with it.

Sources (each function names the passage it follows):

* "Helix Parallelism: Rethinking Sharding Strategies for Interactive Multi-Million-Token LLM
  Decoding" -- paper summary page (fdeinterviews.com), paragraph on KV parallelism: every KVP shard
  attends over its slice of the history and returns a partial output and a log-sum-exp; combining
  them gives the exact full-context result (the Flash-Decoding identity).
* Same page, paragraph on the Helix layouts: new KV entries rotate across KVP ranks every 16 tokens.
* Paper review (jaehun.me), "Prompt 1.3.2 -- The Secret Weapon": the boxed LSE-rescaling equation
  for merging partial outputs (its LaTeX is garbled on the page; the reading used here is the
  normalised-partials form, see ``attention.combine``).
* NVIDIA technical blog, Korean edition (open-lab.net), KV-cache section: the worked round-robin
  example (the first block of 16 tokens goes to KVP rank 0, the next 16 to rank 1).
* NVFP4 decode follows the public OCP Microscaling (MX) v1.0 FP4 E2M1 element definition and the
  OCP 8-bit floating point (OFP8) E4M3 definition; the pages say only "FP4".

Parity status: attention, combine, layout and NVFP4 decode are pinned by tests under ``tests/``
(closed forms, invariances, brute force, library special cases, published format tables and the
pages' round-robin example).  No function here is "parity unpinned".
"""

from .attention import attend, decode, partial, combine  # noqa: F401
from .layout import rr_place, contig_place, shard_tokens, shard_lens, page_slot  # noqa: F401
from .nvfp4 import e2m1_value, e4m3_value, nvfp4_dequant, nvfp4_encode  # noqa: F401
