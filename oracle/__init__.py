"""fp64 CPU oracle for the MTLA hot path — TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it: the only common module is the seeded input generator
(``mtla_synth``), which holds none of the method's arithmetic.

Everything here is plain numpy in float64, written to be read against the
pages that define Multi-head Temporal Latent Attention (MTLA, Deng & Woodland,
NeurIPS 2025).  Sources cited in the docstrings:

* "Notes": the paper-notes page *Multi-head Temporal Latent Attention*
  (NeurIPS 2025 notes), sections *Overall framework*, *Key designs*
  (hyper-network temporal merging; stride-aware causal mask; decoupled RoPE
  with temporal compression) and *Loss / training strategy*.
* "Figure 1" / "Figure 2": the figure captions on the sciencestack abstract
  page of arXiv 2505.13544 (Fig. 1: absorption of the latent-to-KV maps into
  the query/output layers; Fig. 2: incremental inference (a), pre-downsampling
  (b), stride-aware training mask (c)).
* "News": the machine-translated news article on MTLA (its s = 2 walk-through
  of the cache length, and the remark that a very large s keeps about one
  cache entry).

Pins (tests/test_oracle_pins.py) tie every function to something other than
itself.  The hyper-network parameterisation (which Linear sees which input,
biases, the sinusoid and the RoPE form) is fixed by convention because the
pages do not spell it out; see ``merge_weight`` and ``rope``.
"""
from .mtla_oracle import *  # noqa: F401,F403
