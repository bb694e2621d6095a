"""Oracle: prompt-block protection score and selection (iS-KV reading notes, Section 3.1,
Algorithm 1 steps 2-4).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Definition (Section 3.1): the prompt is cut into blocks of 8 tokens; the last 4 blocks and the
partial tail form a local suffix. For each KV head, a block's score is the minimum, over its tokens,
of the cosine between the token's **post-RoPE** key and the block-mean key. Each head picks its 128
lowest-scoring blocks (all of them if there are fewer). The union of the picked positions over heads,
plus the suffix, is the protected key set ``P_K``; a picked position keeps the whole row across all
heads. ``P_V`` is every prompt position within 32 tokens of a position in ``P_K``.

Readings where the pages are silent:

* candidates are the full blocks before the 4-block suffix; the suffix is added unconditionally;
* ties are broken by ascending block index (order on ``(score, block)``);
* ``cos = dot / max(|k| |m|, 1e-30)``, so a zero key or a zero mean scores 0;
* "within 32 tokens" is inclusive: ``|p - q| <= 32``, clipped to ``[0, L)``.
"""

from __future__ import annotations

import numpy as np

COS_FLOOR = 1e-30


def block_scores(keys, block: int = 8, n_blocks: int | None = None) -> np.ndarray:
    """Scores ``(H, n_blocks)`` in float64 for full blocks ``0 .. n_blocks-1``.

    ``keys`` is ``(L, H, hd)`` post-RoPE. ``n_blocks`` defaults to ``L // block``.
    """
    K = np.asarray(keys, dtype=np.float64)
    L, H, hd = K.shape
    nb = L // block if n_blocks is None else int(n_blocks)
    if nb <= 0:
        return np.zeros((H, 0))
    Kb = K[: nb * block].reshape(nb, block, H, hd)            # (nb, block, H, hd)
    mean = Kb.mean(axis=1)                                    # (nb, H, hd)
    dots = np.einsum("jthd,jhd->jth", Kb, mean)
    kn = np.sqrt(np.einsum("jthd,jthd->jth", Kb, Kb))
    mn = np.sqrt(np.einsum("jhd,jhd->jh", mean, mean))[:, None, :]
    cos = dots / np.maximum(kn * mn, COS_FLOOR)
    return cos.min(axis=1).T.copy()                           # (H, nb)


def select_prompt_blocks(keys, block: int = 8, per_head: int = 128, suffix_blocks: int = 4,
                         v_radius: int = 32):
    """Algorithm 1 steps 2-4. Returns a dict with

    ``scores`` (H, n_cand) float64, ``head_blocks`` list of ascending int arrays (picked blocks per
    head), ``P_K`` and ``P_V`` ascending int64 token positions, ``n_cand``, ``suffix_start``.
    """
    K = np.asarray(keys)
    L, H, _ = K.shape
    nb = L // block
    n_cand = max(nb - int(suffix_blocks), 0)
    suffix_start = n_cand * block                    # first token of the suffix
    scores = block_scores(K, block, n_cand)
    head_blocks = []
    protected = np.zeros(L, dtype=bool)
    protected[suffix_start:] = True
    for h in range(H):
        order = np.lexsort((np.arange(n_cand), scores[h]))  # by score, then block index
        picked = np.sort(order[: min(int(per_head), n_cand)])
        head_blocks.append(picked.astype(np.int64))
        for j in picked:
            protected[j * block:(j + 1) * block] = True
    P_K = np.flatnonzero(protected).astype(np.int64)
    near = np.zeros(L, dtype=bool)
    for p in P_K:
        near[max(0, p - v_radius):min(L, p + v_radius + 1)] = True
    P_V = np.flatnonzero(near).astype(np.int64)
    return {"scores": scores, "head_blocks": head_blocks, "P_K": P_K, "P_V": P_V,
            "n_cand": n_cand, "suffix_start": suffix_start}
