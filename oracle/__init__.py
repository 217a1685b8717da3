"""Plain, slow, fp64 CPU oracle for the Kara window-compression path and LaCache's ladder.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or execute this
package: only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm use it. It shares no code, tables or constants with the CUDA library; both sides
take their inputs from the seeded generators in ``decode_kv_cache_kara_b200.synth``.

Sources (the five web pages on Kara and LaCache):

* "Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache Compression"
  (shd-paper.top summary; English abstract, key points, method details).
* The gist.science explainers of the same paper (German and Japanese): the two-way attention
  score, the Token2Chunk analogy and the every-100-steps schedule.
* "LaCache: Ladder-Shaped KV Caching for Efficient Long-Context Modeling of Large Language
  Models" (papercache.org summary): ladder pattern, span S, overlap O, iterative compaction.

Modules:

* ``kara``    - window scoring, top-k selection, Token2Chunk, paged compaction.
* ``decode``  - paged GQA decode attention over the (compressed) cache.
* ``lacache`` - the ladder keep map and ladder compaction.
* ``decode_loop`` - the decode loop around them: block allocation for new slots, the fused
  append + attention step, the tail-W trigger checked periodically, the window-query ring.

Parity status of every function is stated in its module header.
"""

from . import kara, decode, lacache, decode_loop  # noqa: F401
