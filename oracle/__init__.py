"""CPU oracle for the LatentIndex decode indexer.

TEST INFRASTRUCTURE.  This package is the plain, slow, obviously correct
statement of what the indexer computes: NumPy float64 (BLAS for the matrix
products), a pure-Python brute force for tiny inputs, the cache element codecs
written from their format definitions, and the closed-form counters printed in
the LatentIndex summary.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it.  The library never calls
it and shares no code with it: the CUDA path must fail loudly when its
extension is missing instead of falling back here.

Pins (tests/test_oracle.py): a hand-computed worked example
(tests/golden/hand_example.json), the storage and positions-scored numbers
printed in the summary (tests/golden/printed_numbers.json), an independent
pure-Python brute force that reconstructs every key explicitly, the method's
invariants (absorption exactness, HS with B >= L equals full selection, a
one-layer group with an identity decoder is DSA-style scoring), and the
codecs against torch's bf16 / float8_e4m3fn conversions.  The two-branch
latent (rope.py: rotary rotation, LayerNorm, native rotated keys) is pinned
by plane geometry, the rotation group laws, torch's float64 layer_norm and
the exactness of absorbing frequency-wise complex decoders into post-RoPE
queries (tests/test_oracle_rope.py).  The selection-quality metrics
(recall.py: attention-mass recall per head and of the head average, the
IndexCache comparator) are pinned by a hand-computed example, a brute force
over all size-K sets and scipy's softmax (tests/test_oracle_recall.py).  The pages print no
score values of their own, so the score arithmetic is pinned by hand
arithmetic and brute force rather than by a published example.
"""
from . import bruteforce, codecs, counters, indexer, recall, rope

__all__ = ["codecs", "counters", "indexer", "bruteforce", "recall", "rope"]
