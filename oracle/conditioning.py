"""Router-margin conditioning of synthetic inputs -- TEST INFRASTRUCTURE ONLY.

The expert indices chosen by the router are an integer decision taken from floating-point logits.
The CUDA router accumulates in fp32, the oracle in fp64; on random data a token whose top logits
are nearly equal could be ordered differently by the two. To compare indices bit for bit, the test
inputs move such tokens away from near-ties: a token whose sorted top-(k+1) logits (top-k when
k = E) have any adjacent gap below ``margin`` gets a fresh x row, drawn by the caller's
``redraw(b, t, attempt)``, until the gaps clear the margin. The fp32 accumulation error of a
D-term dot product of N(0,1) inputs with N(0,1/D) weights is of order 1e-6, far below the default
margin of 1e-3, so with these inputs fp32 and fp64 logits always give the same decision.
"""
from __future__ import annotations

import numpy as np

from .swimba_oracle import block_branches, router_logits


def near_tie_mask(logits: np.ndarray, k: int, margin: float) -> np.ndarray:
    """True where the top-(k+1) sorted logits have an adjacent gap below ``margin``."""
    E = logits.shape[-1]
    m = min(k + 1, E)
    if m < 2:
        return np.zeros(logits.shape[:-1], dtype=bool)
    top = -np.sort(-logits, axis=-1)[..., :m]
    gaps = top[..., :-1] - top[..., 1:]
    return np.any(gaps < margin, axis=-1)


def condition_router_margin(x_store, widen, W_r, k, redraw, margin=1e-3, max_attempts=64):
    """Redraw the x rows [B, L, D] (storage form, modified in place) that sit near a router tie.

    ``widen(stored) -> fp64`` gives the exact value of stored rows; ``redraw(b, t, attempt)``
    returns a new stored row. Returns the number of rows redrawn.
    """
    Bsz, L, D = x_store.shape
    W_r64 = np.asarray(W_r, dtype=np.float64)
    redrawn = 0
    for b in range(Bsz):
        logits = router_logits(widen(x_store[b]), W_r64)
        for t in np.nonzero(near_tie_mask(logits, k, margin))[0]:
            for attempt in range(max_attempts):
                row = redraw(b, int(t), attempt)
                lg = router_logits(widen(row[None, :]), W_r64)
                if not near_tie_mask(lg, k, margin)[0]:
                    x_store[b, t] = row
                    redrawn += 1
                    break
            else:
                raise RuntimeError(f"token ({b},{t}) stays within {margin} of a router tie")
    return redrawn


def condition_block_router_margin(u_store, widen, BW, k, io, redraw, conv_state=None, margin=2e-3,
                                  max_rounds=64):
    """The same conditioning for the Swimba block, whose router sees x = SiLU(conv(u W_in)): while
    a token (b, t) of x sits near a router tie, its block input row u[b, t] (storage form, modified
    in place) is redrawn with ``redraw(b, t, attempt)``. A new row changes x at t .. t+W-1, so the
    check repeats over the whole input until no near tie is left. Returns the rows redrawn."""
    attempts = {}
    for _ in range(max_rounds):
        _, _, x, _ = block_branches(widen(u_store), BW, conv_state, io)
        logits = router_logits(x, BW["W_r"])
        ties = np.argwhere(near_tie_mask(logits, k, margin))
        if ties.size == 0:
            return sum(attempts.values())
        for b, t in ties:
            a = attempts.get((int(b), int(t)), 0)
            u_store[b, t] = redraw(int(b), int(t), a)
            attempts[(int(b), int(t))] = a + 1
    raise RuntimeError(f"block input keeps a token within {margin} of a router tie")
