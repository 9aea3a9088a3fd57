"""fp64 CPU oracle for the LoopSpec acceptance step (test infrastructure only).

TEST INFRASTRUCTURE ONLY: the tests and the smoke check use this module; the
product library never imports it and shares no code with it.

What it computes (LoopSpec article, rit.work: sections on the second branch and
on the final check).  A looped model drafts the next token from an early loop
depth (the first proposal x1, drawn from the draft distribution q1) and, when a
deeper intermediate state has lowered its confidence in x1, prepares a fallback
proposal x2 from the deeper distribution's remainder after the first proposal.
The final distribution p (all R loops) then decides, in this order:

  1. accept x1 with probability min(1, p(x1) / q1(x1));
  2. else, if there is a fallback, accept x2 with probability
     min(1, p1(x2) / q2(x2)), where p1 = norm((p - q1)+) is what p still has to
     give after step 1 and q2 = norm((qf - q1)+) the fallback's distribution;
  3. else restart: draw from norm((p1 - q2)+) (from p1 when there was no fallback).

Readings where the article is silent (each listed in the design notes):
  * "lowered its confidence in x1": qf(x1) < q1(x1), both at temperature 1.
  * "remainder after the first proposal": q2 = norm((qf - q1)+).
  * Greedy decoding (temperature 0): every distribution is the one-hot of its
    argmax (lowest index on ties); the fallback is the deeper state's best token
    other than x1, so the emitted token is always argmax p.
  * A block of k draft positions is checked position by position; the first
    position whose x1 is rejected ends the block (its token is the fallback or the
    restart draw, and later drafts, built on x1, are void).
  * A draw from a distribution w with a uniform u in [0, 1) is the smallest token
    v with w(0) + ... + w(v) > u * (w(0) + ... + w(V-1)).
  * A remainder with no mass (p <= q1 everywhere, which rounding alone can
    produce) is replaced by the distribution it was taken from.

Each step is the textbook speculative-sampling rejection test applied to what the
target still has to give, so the emitted token is distributed exactly as p;
`output_distribution` writes that marginal out so the tests can check it.
"""
from __future__ import annotations

import numpy as np

ALL_ACCEPTED, FALLBACK, RESTART = 0, 1, 2


def softmax(z: np.ndarray, temperature: float) -> np.ndarray:
    """Distribution of logits z at the temperature; 0 gives the argmax one-hot."""
    z = np.asarray(z, dtype=np.float64)
    if temperature == 0:
        out = np.zeros_like(z)
        out[int(np.argmax(z))] = 1.0
        return out
    y = z / temperature
    e = np.exp(y - y.max())
    return e / e.sum()


def residual(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """norm((a - b)+); all zeros when a <= b everywhere."""
    r = np.maximum(a - b, 0.0)
    s = r.sum()
    return r / s if s > 0 else r


def draw(w: np.ndarray, u: float) -> int:
    """Smallest v with cumsum(w)[v] > u * sum(w) (inverse CDF)."""
    c = np.cumsum(w)
    return int(np.searchsorted(c, u * c[-1], side="right"))


def fallback_gate(zq: np.ndarray, zf: np.ndarray, x1: int) -> bool:
    """The deeper state lowered its confidence in x1 (probabilities at temperature 1)."""
    return softmax(zf, 1.0)[x1] < softmax(zq, 1.0)[x1]


def fallback_distribution(zq, zf, temperature):
    """q2: the fallback's distribution (greedy: one-hot of the best token other than x1
    is taken by `fallback_token`)."""
    return residual(softmax(zf, temperature), softmax(zq, temperature))


def fallback_token(zq, zf, x1: int, temperature: float, u: float) -> int:
    """The fallback proposal: a draw from q2 (greedy: argmax of zf without x1)."""
    if temperature == 0:
        z = np.asarray(zf, dtype=np.float64).copy()
        z[x1] = -np.inf
        return int(np.argmax(z))
    return draw(fallback_distribution(zq, zf, temperature), u)


def accept_position(zp, zq, zf, x1: int, x2: int, u, temperature: float):
    """One position.  u = (u_accept_x1, u_accept_x2, u_restart).  Returns
    (accepted x1, token emitted if x1 was rejected, path)."""
    p = softmax(zp, temperature)
    q1 = softmax(zq, temperature)
    gate = zf is not None and fallback_gate(zq, zf, x1)
    if temperature == 0:
        best = int(np.argmax(zp))
        if x1 == best:
            return True, -1, ALL_ACCEPTED
        if gate and x2 == best:
            return False, x2, FALLBACK
        return False, best, RESTART
    if u[0] * q1[x1] < p[x1]:
        return True, -1, ALL_ACCEPTED
    p1 = residual(p, q1)
    if p1.sum() == 0:
        p1 = p
    if gate:
        q2 = fallback_distribution(zq, zf, temperature)
        if q2.sum() > 0:
            if u[1] * q2[x2] < p1[x2]:
                return False, x2, FALLBACK
            r2 = residual(p1, q2)
            return False, draw(r2 if r2.sum() > 0 else p1, u[2]), RESTART
    return False, draw(p1, u[2]), RESTART


def accept_block(zp, zq, zf, x1, x2, u, temperature: float):
    """k positions of one sequence: (number of accepted drafts, emitted token or -1,
    path of the last position checked)."""
    k = len(x1)
    for j in range(k):
        ok, tok, path = accept_position(zp[j], zq[j], None if zf is None else zf[j], int(x1[j]), int(x2[j]),
                                        u[j], temperature)
        if not ok:
            return j, tok, path
    return k, -1, ALL_ACCEPTED


def output_distribution(zp, zq, zf, temperature: float) -> np.ndarray:
    """The marginal distribution of the token one position emits (x1 if accepted,
    else the fallback or restart token), over x1 ~ q1, x2 ~ q2 and the uniforms,
    written out term by term for sampling temperatures."""
    p = softmax(zp, temperature)
    q1 = softmax(zq, temperature)
    V = len(p)
    p1 = residual(p, q1)
    q2 = None if zf is None else fallback_distribution(zq, zf, temperature)
    out = np.zeros(V)
    for x1 in range(V):
        if q1[x1] == 0:
            continue
        a1 = min(1.0, p[x1] / q1[x1])
        out[x1] += q1[x1] * a1
        rej = q1[x1] * (1.0 - a1)
        if rej == 0:
            continue
        if zf is not None and fallback_gate(zq, zf, x1) and q2.sum() > 0:
            r2 = residual(p1, q2)
            for x2 in range(V):
                if q2[x2] == 0:
                    continue
                a2 = min(1.0, p1[x2] / q2[x2])
                out[x2] += rej * q2[x2] * a2
                out += rej * q2[x2] * (1.0 - a2) * r2
        else:
            out += rej * p1
    return out
