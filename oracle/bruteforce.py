"""Exact-rational brute force of the recurrence for tiny heads.

TEST INFRASTRUCTURE ONLY (same rules as ``sketchssm_oracle``).  Pure-Python
``fractions.Fraction`` arithmetic with explicit dk x dk transition matrices,
composed densely.  It shares no code with the fp64 oracle: where the oracle
applies M_t by its action (a x - ...), this module builds the matrix M_t
entry by entry and multiplies matrices, so a wrong sign, a transposed factor
or a dropped term in either one shows up as a disagreement.

Definitions (project page, "01 / The idea": S_t = M_t S_{t-1} + B_t, read
o_t = S_t^T q_t; family forms as in the oracle's reading P1):
    Mamba-2  M = a I
    GDN      M = a (I - b k k^T)
    KDA      M = (I - b k k^T) Diag(a)
    all      B = b k v^T
With dyadic inputs every quantity is an exact rational.
"""
from __future__ import annotations

from fractions import Fraction

MAMBA2, GDN, KDA = 0, 1, 2


def _zeros(n, m):
    return [[Fraction(0)] * m for _ in range(n)]


def _eye(n):
    M = _zeros(n, n)
    for i in range(n):
        M[i][i] = Fraction(1)
    return M


def _matmul(A, B):
    n, m, p = len(A), len(B), len(B[0])
    return [[sum((A[i][t] * B[t][j] for t in range(m)), Fraction(0)) for j in range(p)]
            for i in range(n)]


def _add(A, B):
    return [[A[i][j] + B[i][j] for j in range(len(A[0]))] for i in range(len(A))]


def _transpose(A):
    return [list(r) for r in zip(*A)]


def _col(x):
    return [[xi] for xi in x]


def transition_matrix(family, k, a, b):
    """The dk x dk matrix M_t, built entry by entry."""
    n = len(k)
    if family == MAMBA2:
        return [[(a if i == j else Fraction(0)) for j in range(n)] for i in range(n)]
    erase = [[(Fraction(1) if i == j else Fraction(0)) - b * k[i] * k[j] for j in range(n)]
             for i in range(n)]
    if family == GDN:
        return [[a * erase[i][j] for j in range(n)] for i in range(n)]
    if family == KDA:
        return [[erase[i][j] * a[j] for j in range(n)] for i in range(n)]   # erase @ Diag(a)
    raise ValueError(family)


def update_matrix(k, v, b):
    """B_t = b k v^T."""
    return [[b * k[i] * v[j] for j in range(len(v))] for i in range(len(k))]


def recurrence(family, S0, tokens, queries):
    """Run S_t = M_t S_{t-1} + B_t over the tokens; return (states, outputs).

    tokens: list of (k, v, a, b); queries: list of q (or None) per token.
    """
    S = [list(r) for r in S0]
    states, outs = [], []
    for (k, v, a, b), q in zip(tokens, queries):
        S = _add(_matmul(transition_matrix(family, k, a, b), S), update_matrix(k, v, b))
        states.append(S)
        outs.append(None if q is None else [r[0] for r in _matmul(_transpose(S), _col(q))])
    return states, outs


def window_decomposition(family, tokens, q):
    """(q~, o_buf) from dense products.

    With Phi_j = M_tau ... M_{j+1} (identity for j = tau), the state after
    tau updates is Phi_0 S0 + sum_j Phi_j B_j, so
        S_tau^T q = S0^T (Phi_0^T q) + sum_j B_j^T Phi_j^T q.
    """
    n = len(tokens[0][0])
    tau = len(tokens)
    Phi = [None] * (tau + 1)
    Phi[tau] = _eye(n)
    for j in range(tau, 0, -1):
        k, v, a, b = tokens[j - 1]
        Phi[j - 1] = _matmul(Phi[j], transition_matrix(family, k, a, b))
    q_tilde = [r[0] for r in _matmul(_transpose(Phi[0]), _col(q))]
    dv = len(tokens[0][1])
    o_buf = [Fraction(0)] * dv
    for j in range(1, tau + 1):
        k, v, a, b = tokens[j - 1]
        term = _matmul(_transpose(_matmul(Phi[j], update_matrix(k, v, b))), _col(q))
        o_buf = [o_buf[i] + term[i][0] for i in range(dv)]
    return q_tilde, o_buf
