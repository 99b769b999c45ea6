"""GPU parity: the chunked gated delta rule kernel vs the CPU oracle.

The oracle (oracle/gdn.py, token by token in float64) is pinned on CPU by
properties of the mechanism the pages describe (each write overwrites the
state along its key direction: bayesiansapien wiki, "The four-part mechanism
study", part 3).  Here the fp32 kernel must match it on ragged chunk counts,
grouped heads and a non-zero initial state; at the GDN in-projection's size
(8192 tokens, 48 value heads over 16 key heads) on sampled heads; and the
mechanism itself must show on the GPU: the output error caused by noise
injected into the values stays flat along the sequence.
"""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_quantizer_b200 as nv

pytestmark = pytest.mark.gpu

D = 128


def inputs(T, Hv, group, seed, state_scale=0.5):
    rng = np.random.default_rng(seed)
    Hk = Hv // group
    q = rng.standard_normal((T, Hk, D)).astype(np.float32)
    k = rng.standard_normal((T, Hk, D))
    k = (k / np.linalg.norm(k, axis=2, keepdims=True)).astype(np.float32)
    v = rng.standard_normal((T, Hv, D)).astype(np.float32)
    # the decay gate's range: -exp(A_log) softplus(.), A_log in (-1, 1.5)
    g = (-np.exp(rng.uniform(-1, 1.5, Hv))[None, :] *
         np.log1p(np.exp(rng.normal(-2, 1, (T, Hv))))).astype(np.float32)
    beta = (1 / (1 + np.exp(-rng.normal(0, 1.5, (T, Hv))))).astype(np.float32)
    S0 = (rng.standard_normal((Hv, D, D)) * state_scale).astype(np.float32)
    return q, k, v, g, beta, S0


def run_gpu(q, k, v, g, beta, S0, group):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    state = t(S0)
    o, state = nv.nvfp4_gdn_recurrence(t(q), t(k), t(v), t(g), t(beta), group=group, state=state)
    assert nv.nvfp4_last_device_error()[0] == 0
    return o.cpu().numpy(), state.cpu().numpy()


def check_head(o, S, q, k, v, g, beta, S0, group, h):
    hk = h // group
    ref_o, ref_S = oracle.gdn_recurrence_seq(q[:, hk], k[:, hk], v[:, h], g[:, h], beta[:, h],
                                             S0=S0[h].astype(np.float64))
    so, ss = np.abs(ref_o).max(), np.abs(ref_S).max()
    assert np.abs(o[:, h] - ref_o).max() <= 2e-5 * so + 1e-6, f"head {h} output"
    assert np.abs(S[h] - ref_S).max() <= 2e-5 * ss + 1e-6, f"head {h} state"


@pytest.mark.parametrize("T", [1, 63, 64, 65, 300])
def test_matches_the_oracle(T):
    Hv, group = 6, 3
    q, k, v, g, beta, S0 = inputs(T, Hv, group, seed=T)
    o, S = run_gpu(q, k, v, g, beta, S0, group)
    for h in range(Hv):
        check_head(o, S, q, k, v, g, beta, S0, group, h)


@pytest.mark.slow
def test_gdn_inproj_size_on_sampled_heads():
    T, Hv, group = 8192, 48, 3
    q, k, v, g, beta, S0 = inputs(T, Hv, group, seed=1, state_scale=0.0)
    o, S = run_gpu(q, k, v, g, beta, S0, group)
    for h in (0, 17, 47):
        check_head(o, S, q, k, v, g, beta, S0, group, h)


def test_injected_noise_plateaus():
    """Outputs of a clean run and of a run whose values carry small noise:
    their difference holds a flat level along 8192 tokens (no decay, so only
    the overwrite can hold it) instead of growing with position."""
    T, Hv, group = 8192, 4, 1
    q, k, v, g, beta, S0 = inputs(T, Hv, group, seed=5, state_scale=0.0)
    g[:] = 0.0                                   # no decay: the overwrite alone bounds the error
    beta[:] = 0.5
    noisy = v + np.random.default_rng(9).standard_normal(v.shape).astype(np.float32) * 1e-2
    o1, _ = run_gpu(q, k, v, g, beta, S0, group)
    o2, _ = run_gpu(q, k, noisy, g, beta, S0, group)
    err = np.sqrt(np.mean((o2 - o1) ** 2, axis=(1, 2)))          # per token
    q2, q4 = err[T // 4: T // 2].mean(), err[3 * T // 4:].mean()
    assert abs(q4 / q2 - 1.0) < 0.1
