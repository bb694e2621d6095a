"""Float64 CPU oracle for the iS-KV hot path.

TEST INFRASTRUCTURE ONLY. This package states, in plain NumPy float64, what the CUDA library must
compute: the block-incremental SVD fold, re-orthogonalisation, reconstruction with RoPE, and the
prompt-block protection score and selection. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import it. The CUDA library never calls into it and
it never calls into the CUDA library; the two share no code.

Sources (cited by page title and section throughout):

* "iS-KV reading notes" -- the zhongzhuzhou.org blog notes on *iS-KV: Online Low-Rank KV Cache
  Compression via Block-Incremental SVD* (arXiv 2610.02815 v1). Primary authority. Its inline
  formulas were lost in extraction; where a formula had to be rebuilt from the prose, the function
  that uses it says so.
* "ai4snews digest" -- the English abstract digest with the caption of the paper's Fig. 2.

Pins: every function here is checked by ``tests/test_oracle_*.py`` against closed forms, worked
examples printed on the pages (``tests/golden``), invariants and brute force. No function is
"parity unpinned".

Modules
-------
fold        Algorithm 2 (block fold) and the plain truncated-SVD definition it must reach.
reorth      Section 4.4 re-orthogonalisation.
rope        rotate-half rotary position embedding used on reconstructed keys.
reconstruct per-step reconstruction (Algorithm 3 steps 7-8).
select      Algorithm 1 steps 2-4 (block outlier score, lowest-128 per head, union, value radius).
accounting  Section 5.1 persistent-storage arithmetic (eq. 12 and its consequences).
drift       Section 2.3 coordinate drift and the appendix factor-drift measure (eq. 14).
attention   decode attention over the compressed cache (Algorithm 3 steps 7-9).
policy      the cache policy: protected rows, recent window, pending FIFO and the fold schedule
            (Algorithm 1 steps 5-8, Algorithm 3 steps 1-6).
"""

from . import accounting, attention, drift, fold, policy, reconstruct, reorth, rope, select  # noqa: F401

__all__ = ["accounting", "attention", "drift", "fold", "policy", "reconstruct", "reorth", "rope",
           "select"]
