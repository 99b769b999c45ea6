"""CPU oracle for the Gated DeltaNet state recurrence -- TEST INFRASTRUCTURE ONLY.

The recurrent half of the hybrid model is the gated delta rule.  The pages
describe its mechanism without a formula: every write overwrites the state
along the current key direction, so the state behaves as a continuously
overwritten register rather than an accumulator; injected noise stays at a
flat plateau and a state impulse is forgotten within hundreds of steps
(bayesiansapien wiki, "The four-part mechanism study", part 3; nefut
abstract, third mechanism; aimodeling, "Why the recurrent half survives").
The formula is the published gated delta rule, restated here:

    S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t

with S_t in R^{d_v x d_k}, k_t of unit length, alpha_t = exp(g_t) in (0, 1]
(g from the decay gate of the in-projection epilogue) and beta_t in (0, 1)
(the write strength, a sigmoid).  Everything is float64.

Two forms:
  gdn_recurrence_seq      -- the definition, one token at a time;
  gdn_recurrence_chunked  -- the chunkwise algorithm a GPU kernel runs (each
                             chunk solves for the values it writes with one
                             unit-lower-triangular system), derived from the
                             definition as follows.  With u_t = beta_t (v_t -
                             alpha_t S_{t-1} k_t) the step is S_t = alpha_t
                             S_{t-1} + u_t k_t^T, so inside a chunk that starts
                             from S_0, with gamma_t = prod_{i<=t} alpha_i,
                               S_t = gamma_t S_0 + sum_{j<=t} (gamma_t/gamma_j) u_j k_j^T,
                               (I + A) U = diag(beta) V - diag(beta gamma) K S_0^T,
                               A_tj = beta_t (gamma_t/gamma_j) (k_t . k_j)  (j < t),
                               O = diag(gamma) Q S_0^T + (M o (Q K^T)) U,
                               M_tj = gamma_t/gamma_j  (j <= t),
                               S_C = gamma_C S_0 + U^T diag(gamma_C/gamma) K.

Noise model (error e_t = quantised state minus exact state, noise eta_t
injected at each write): e_t = alpha_t e_{t-1} (I - beta_t k_t k_t^T) + eta_t.
For a unit key (I - b k k^T)^2 = I - (2b - b^2) k k^T, so
||e (I - b k k^T)||_F^2 = ||e||_F^2 - (2b - b^2) ||e k||^2, and for keys
uniform on the sphere E||e k||^2 = ||e||_F^2 / d_k.  Hence, at constant
alpha, beta, the per-step contraction of the mean squared error is
    rho = alpha^2 (1 - (2 beta - beta^2) / d_k),
the impulse decays as rho^t, and the noise plateau is sigma^2 / (1 - rho)
(sigma^2 = E||eta||_F^2) -- where an additive state S_t = S_{t-1} + v_t k_t^T
accumulates t sigma^2.  gdn_error_contraction / gdn_noise_plateau give these
closed forms; tests check them against simulated recurrences.

Pinning status: gdn_recurrence_seq -- exact overwrite along k (beta = 1),
decay-only action orthogonal to k, alpha = 1 beta = 0 identity, brute-force
unrolled small case; gdn_recurrence_chunked -- equals the sequential form;
the closed forms -- statistical agreement with simulation.
"""
from __future__ import annotations

import numpy as np


def gdn_recurrence_seq(q, k, v, g, beta, S0=None):
    """The gated delta rule, token by token (float64).

    q, k: [T, d_k] (k rows of unit length); v: [T, d_v]; g: [T] (log decay,
    <= 0); beta: [T].  Returns (O [T, d_v], S_T [d_v, d_k]).
    """
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    g, beta = np.asarray(g, np.float64), np.asarray(beta, np.float64)
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, np.float64)
    O = np.empty((T, dv))
    eye = np.eye(dk)
    for t in range(T):
        alpha = np.exp(g[t])
        S = alpha * S @ (eye - beta[t] * np.outer(k[t], k[t])) + beta[t] * np.outer(v[t], k[t])
        O[t] = S @ q[t]
    return O, S


def gdn_recurrence_chunked(q, k, v, g, beta, chunk=64, S0=None):
    """The same recurrence computed chunk by chunk (see the module docstring)."""
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    g, beta = np.asarray(g, np.float64), np.asarray(beta, np.float64)
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, np.float64)
    O = np.empty((T, dv))
    for c0 in range(0, T, chunk):
        sl = slice(c0, min(T, c0 + chunk))
        Q, K, V, b = q[sl], k[sl], v[sl], beta[sl]
        C = K.shape[0]
        G = np.cumsum(g[sl])                       # log gamma_t
        ratio = np.exp(G[:, None] - G[None, :])    # gamma_t / gamma_j
        KK = K @ K.T
        A = np.tril(b[:, None] * ratio * KK, -1)
        rhs = b[:, None] * V - (b * np.exp(G))[:, None] * (K @ S.T)
        U = np.linalg.solve(np.eye(C) + A, rhs)
        M = np.tril(ratio)
        O[sl] = np.exp(G)[:, None] * (Q @ S.T) + (M * (Q @ K.T)) @ U
        S = np.exp(G[-1]) * S + U.T @ (np.exp(G[-1] - G)[:, None] * K)
    return O, S


def gdn_error_contraction(alpha: float, beta: float, dk: int) -> float:
    """rho: per-step factor of E||e||_F^2 for keys uniform on the unit sphere."""
    return alpha ** 2 * (1.0 - (2.0 * beta - beta ** 2) / dk)


def gdn_noise_plateau(sigma2: float, alpha: float, beta: float, dk: int) -> float:
    """Steady-state E||e||_F^2 when noise of mean square sigma2 enters every step."""
    return sigma2 / (1.0 - gdn_error_contraction(alpha, beta, dk))


def gdn_error_trace(keys, beta, alpha, noise, e0=None):
    """||e_t||_F^2 of the error recurrence e_t = alpha e_{t-1} (I - beta k k^T) + noise_t.

    keys: [T, d_k] unit rows; noise: [T, d_v, d_k] (or None: no injection);
    e0: initial error [d_v, d_k].  Returns [T] squared Frobenius norms.
    """
    keys = np.asarray(keys, np.float64)
    T, dk = keys.shape
    dv = noise.shape[1] if noise is not None else np.asarray(e0).shape[0]
    e = np.zeros((dv, dk)) if e0 is None else np.array(e0, np.float64)
    out = np.empty(T)
    for t in range(T):
        kt = keys[t]
        e = alpha * (e - beta * np.outer(e @ kt, kt))
        if noise is not None:
            e = e + noise[t]
        out[t] = np.sum(e * e)
    return out
