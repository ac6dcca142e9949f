"""CPU oracle for the streaming-frame step: 3D RoPE, dual-stream paged KV retention, attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or link this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the CUDA path
(``rope_paged_kv_02_b200``) and imports nothing from it.

Everything here is plain numpy in float64, written for a reader to check against the
source pages by eye.  The pages are five articles about the lingbot-map project; they are
cited by title and section:

* [3DRoPE-KV]  "How 3D RoPE Positional Encoding Works with the Paged KV Cache in LingBot-Map"
* [VideoRoPE]  "Video RoPE Positional Encoding: 3D Rotary Embeddings for Long-Sequence Video
               in Ling-Bot-Map"
* [RealTime3D] "How LingBot-Map Achieves Real-Time 3D Reconstruction: Streaming Transformers
               and KV Caching"
* [KVBenefits] "KV Caching Benefits in Ling Bot-Map: 7 Advantages for Streaming Vision Models"
* [RoPERange]  "How to Handle Sequences Exceeding the RoPE Training Range in LingBot-Map"

Modules:

* ``rope3d``     per-axis frequency tables, token positions, rotation (fp64).
* ``rope2d``     the 2D (y, x) variant: halves of the features per axis, base frequency
                 100, tables sized from the token count.
* ``retention``  the page table / free list / deferred-eviction state machine, plus the
                 closed form of the retained set.
* ``attention``  explicit masked softmax attention over the whole history, and over the
                 retained keys only.
* ``stream``     drives a whole stream of frames through the three parts above.

Pins (tests under ``tests/test_oracle_*.py``, marker ``not gpu``) tie every function to
something other than itself: the pages' printed shapes and the 80 % storage figure, a
library 1D-RoPE frequency routine, a complex-number rotation, norm and relative-offset
invariants, closed forms of the retained set, torch's SDPA on CPU in float64, and
brute-force loops on tiny inputs.  Parity with the real lingbot-map code is unpinned for
the conventions the pages leave open (pair layout, special-token positions, free-list
order, special page size): those are stated readings, self-consistent across oracle and
CUDA path.
"""

from . import rope3d, rope2d, retention, attention, stream  # noqa: F401
