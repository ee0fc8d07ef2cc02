"""CPU oracle of the CSA/HCA compressed attention operator -- TEST INFRASTRUCTURE ONLY.

This package is the executable definition the CUDA path is checked against.
It is plain numpy in float64 over the exact values of the stored bytes, with
no blocking, fusion or reordering beyond what each step's definition states.
Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import it; the operator itself never calls it, and it shares no code with the
CUDA path (it has its own format decoders and encoders, its own rotary
tables and its own selection).

Every function cites the passage of the source pages it follows.  The pages
are five explainer pages on DeepSeek-V4 (cited by page title and section):

* "DeepSeek-V4, explained." (vibeengines.com): numbered list "For one query,
  an attention layer that compresses and then selects works like this" and
  its notation glossary.
* "Decoding DeepSeek-V4" (bibekananda.in): "Compressing the past".
* "DeepSeek-V4" (sghael.github.io): "Compressing features versus compressing
  time", "Compress, then select", "A coarse overview alongside local detail".
* "DeepSeek-V4 Explained: Compressed Sparse Attention and 1M Context at 10%
  KV" (researchpapers.dev): "The attention stack, and why it is two
  mechanisms".
* "DeepSeek-V4: Making a Million Tokens Affordable" (hyan-yao.github.io):
  "Two ways to shrink attention, interleaved".

Where the pages leave a step open the reading taken is stated in the
function's docstring.  Parity status: every function here is pinned by the
CPU tests (closed forms, invariants, library routines, brute force and the
pages' worked counts) except one open question that is "parity unpinned" by
design: whether this gate/indexer parameterisation is DeepSeek's own, which
the pages do not give.
"""
