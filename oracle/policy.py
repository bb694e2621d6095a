"""Oracle: the cache policy -- which rows stay exact and when pending rows are folded (iS-KV reading
notes, Section 3.1, Section 3.2, Algorithm 1 steps 5-9 and Algorithm 3 steps 1-6).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

One side ``X`` (keys or values) of one (sequence, layer) keeps three kinds of exact rows:

* protected rows ``P_X`` (Algorithm 1 steps 2-4; fixed for the whole decode),
* the recent window: the rows at the ``W`` most recent positions (Algorithm 1 step 5 starts it empty
  for keys and with the last ``min(W, L)`` prompt positions for values),
* the pending FIFO: unprotected rows that have left the window and wait for a full block.

Everything else of the prompt is compressed at prefill (Algorithm 1 step 7); during decode a block
of the ``b`` oldest pending rows is folded as soon as ``b`` are pending (Algorithm 3 step 4), its
positions join the compressed position table and its exact copies go away (step 6). After every
``reorth_rows`` rows merged by folds the history is re-orthogonalised (step 5).

Readings where the pages leave a step open:

* the window is the set of the ``W`` most recent positions; a protected position inside it is stored
  once (as protected) and stays exact when it leaves; an unprotected one moves to the FIFO;
* a decode row is never protected (the protected set is fixed at prefill);
* the initial window is no longer than ``W`` (``init_window <= W``), so at most one row joins the FIFO
  per decode step and a fold (a refit) takes exactly the ``b`` (``r_V``) rows that are pending;
* re-orthogonalisation runs in the step whose fold brings the count to ``reorth_rows``; the count
  then restarts from zero;
* the value side's first refit (Algorithm 3 step 3, ``refit_rows`` = r_V > 0): the FIFO grows until
  ``refit_rows`` rows are pending; those rows, appended to the rows the history represents, are
  re-factored by a rank-r truncated SVD; regular ``block`` folds follow. The refit's rows do not
  count toward ``reorth_rows`` (Section 4.4 excludes the value side's first refactorisation).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import fold as _fold
from . import reorth as _reorth


def prefill_partition(L: int, protected, init_window: int):
    """Algorithm 1 steps 5-7 for one side: split the prompt positions ``0 .. L-1`` into

    ``prot``  = ``P_X`` (ascending),
    ``live``  = ``W_X \\ P_X`` with ``W_X`` the last ``min(init_window, L)`` positions (ascending),
    ``comp``  = every other position (ascending): the rows the prompt SVD compresses.
    """
    L = int(L)
    P = sorted(int(p) for p in protected)
    if len(set(P)) != len(P) or any(p < 0 or p >= L for p in P):
        raise ValueError("protected positions must be unique and inside the prompt")
    w = min(int(init_window), L)
    pset = set(P)
    live = [p for p in range(L - w, L) if p not in pset]
    comp = [p for p in range(L - w) if p not in pset]
    return P, live, comp


@dataclass
class Side:
    """The position bookkeeping of one side (no row data)."""

    window: int
    block: int
    reorth_rows: int
    prot: list
    live: list                 # unprotected exact rows, ascending: the FIFO, then the window part
    last: int                  # last stored position
    fold_rows: int = 0
    compressed: list = field(default_factory=list)   # positions merged by decode-time folds
    refit_rows: int = 0        # r_V for the value side's first refit; 0 = none
    refit_done: bool = True

    def pending(self):
        """The FIFO: live rows whose position has left the window ``(last - W, last]``."""
        edge = self.last - self.window
        return [p for p in self.live if p <= edge]


def new_side(L: int, protected, init_window: int, window: int, block: int, reorth_rows: int,
             refit_rows: int = 0):
    """State after Algorithm 1 (steps 5-9) and the positions the prompt SVD compresses."""
    if not 0 <= int(init_window) <= int(window):
        raise ValueError("need 0 <= init_window <= window")
    prot, live, comp = prefill_partition(L, protected, init_window)
    side = Side(int(window), int(block), int(reorth_rows), prot, live, int(L) - 1,
                refit_rows=int(refit_rows), refit_done=int(refit_rows) == 0)
    return side, comp


def append(side: Side, position: int):
    """Algorithm 3 steps 1-2 and the scheduling of steps 3-5 for one new row at ``position``.

    Returns the actions of this step: ``("refit", positions)`` for the value side's first refit,
    ``("fold", positions)`` for the block to merge and ``("reorth",)`` when the merged-row count
    reaches ``reorth_rows``.
    """
    if position != side.last + 1:
        raise ValueError("decode rows arrive one position at a time")
    side.last = position
    side.live.append(position)
    actions = []
    pend = side.pending()
    if not side.refit_done:
        if len(pend) >= side.refit_rows:
            blk = pend[: side.refit_rows]
            side.live = side.live[side.refit_rows:]
            side.compressed.extend(blk)
            side.refit_done = True
            actions.append(("refit", blk))
        return actions
    if len(pend) >= side.block:
        blk = pend[: side.block]
        side.live = side.live[side.block:]
        side.compressed.extend(blk)
        actions.append(("fold", blk))
        side.fold_rows += side.block
        if side.reorth_rows > 0 and side.fold_rows >= side.reorth_rows:
            side.fold_rows = 0
            actions.append(("reorth",))
    return actions


def exact_positions(side: Side):
    """Positions whose exact row is kept: protected rows first, then the live rows (both ascending);
    the order of the exact-row table."""
    return list(side.prot) + list(side.live)


def refit(U, sigma, B, F, r: int):
    """Algorithm 3 step 3: the rank-``r`` truncated SVD of the rows the history represents followed
    by the rows ``F``. Returns ``(U, sigma, B)``."""
    F = np.asarray(F, dtype=np.float64)
    X = np.concatenate([_fold.low_rank_product(U, sigma, B), F]) if np.size(U) else F
    return _fold.truncated_svd(X, r)


def run_decode(prompt_rows, decode_rows, protected, init_window: int, window: int, block: int,
               r: int, reorth_rows: int, tau_rel: float = 0.0, init_history=None,
               refit_rows: int = 0):
    """Algorithm 1 then Algorithm 3 steps 1-6 for one side, with the row data.

    ``init_history`` = ``(U, sigma, B)`` for the compressed prompt rows (in ``comp`` order); when
    ``None`` it is the rank-``r`` truncated SVD of those rows (Algorithm 1 step 7). Returns a dict with
    the final side, the history ``(U, sigma, B, pos)``, the exact table ``(rows, positions)`` and the
    actions of every decode step.
    """
    Xp = np.asarray(prompt_rows, dtype=np.float64)
    Xd = np.asarray(decode_rows, dtype=np.float64)
    L, d = Xp.shape
    side, comp = new_side(L, protected, init_window, window, block, reorth_rows, refit_rows)
    if init_history is None:
        if comp:
            U, sigma, B = _fold.truncated_svd(Xp[comp], r)
        else:
            U, sigma, B = _fold.empty_history(d)
    else:
        U, sigma, B = (np.asarray(a, dtype=np.float64) for a in init_history)
    hpos = list(comp)
    rows = {p: Xp[p] for p in side.prot + side.live}
    steps = []
    for i in range(Xd.shape[0]):
        t = L + i
        rows[t] = Xd[i]
        acts = append(side, t)
        for a in acts:
            if a[0] in ("fold", "refit"):
                F = np.stack([rows[p] for p in a[1]])
                if a[0] == "fold":
                    res = _fold.fold_block(U, sigma, B, F, r, tau_rel)
                    U, sigma, B = res.U, res.sigma, res.B
                else:
                    U, sigma, B = refit(U, sigma, B, F, r)
                hpos.extend(a[1])
                for p in a[1]:
                    del rows[p]
            else:
                U, sigma, B = _reorth.reorth(U, sigma, B)
        steps.append(acts)
    ex = exact_positions(side)
    return {"side": side, "history": (U, sigma, B, np.asarray(hpos, dtype=np.int64)),
            "exact": (np.stack([rows[p] for p in ex]) if ex else np.zeros((0, d)),
                      np.asarray(ex, dtype=np.int64)),
            "steps": steps, "comp": np.asarray(comp, dtype=np.int64)}
