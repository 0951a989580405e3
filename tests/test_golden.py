"""The hand-derived worked example in tests/golden/worked_example_d2.txt (a derivation from the
update rule of "Exact Flow Linear Attention", technical summary, Methodology 3, with every value an
exact short fraction): the oracle must reproduce it to rounding, and the GPU paths that take these
sizes (the SIMT chunk forward and the decode step, fp32) to fp32 accuracy."""
import os

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


def load():
    rows = []
    for line in open(os.path.join(HERE, "golden", "worked_example_d2.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        parts = [p.split() for p in line.split("|")]
        rows.append([float(x) for x in parts[0]] + [float(x) for x in parts[1]] +
                    [float(x) for x in parts[2]] + [float(x) for x in parts[3]])
    a = np.array(rows)
    L = a.shape[0]
    k = a[:, 0:2].reshape(1, 1, L, 2)
    v = a[:, 2:4].reshape(1, 1, L, 2)
    beta = a[:, 4].reshape(1, 1, L)
    q = a[:, 5:7].reshape(1, 1, L, 2)
    alpha = a[:, 7].reshape(1, 1, L)
    o = a[:, 8:10].reshape(1, 1, L, 2)
    S = a[:, 10:14].reshape(L, 2, 2)
    return q, k, v, beta, alpha, o, S


def test_fixture_is_consistent_with_its_alpha_column():
    """The betas were chosen so that a_t is an exact fraction: check that choice, in fp64."""
    _, k, _, beta, alpha, _, _ = load()
    lam = (k * k).sum(-1)
    a = np.where(lam > 0, -np.expm1(-beta * lam) / np.where(lam > 0, lam, 1.0), beta)
    np.testing.assert_allclose(a, alpha, rtol=0, atol=1e-15)


def test_oracle_reproduces_the_worked_example(oracle_mod):
    q, k, v, beta, alpha, o, S = load()
    lam = (k * k).sum(-1)
    for t in range(q.shape[2]):
        assert abs(oracle_mod.alpha(float(lam[0, 0, t]), float(beta[0, 0, t])) - alpha[0, 0, t]) <= 1e-15
    o_got, S_got = oracle_mod.fwd(q, k, v, beta, None, nthreads=1)
    np.testing.assert_allclose(o_got, o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(S_got[0, 0], S[-1], rtol=0, atol=1e-14)
    for t in range(q.shape[2]):  # every prefix ends in the listed state
        _, St = oracle_mod.fwd(q[:, :, :t + 1], k[:, :, :t + 1], v[:, :, :t + 1],
                               beta[:, :, :t + 1], None, nthreads=1)
        np.testing.assert_allclose(St[0, 0], S[t], rtol=0, atol=1e-14)


@pytest.mark.gpu
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_gpu_chunk_forward_reproduces_the_worked_example(chunk):
    from delta_rule_linear_efla_b200 import efla

    q, k, v, beta, _, o, S = load()
    t = lambda x: torch.tensor(x, dtype=torch.float32, device="cuda")
    o_got, S_got = efla.chunk_fwd(t(q), t(k), t(v), t(beta), None, chunk=chunk)
    torch.cuda.synchronize()
    np.testing.assert_allclose(o_got.cpu().numpy(), o, rtol=0, atol=1e-6)
    np.testing.assert_allclose(S_got.cpu().numpy()[0, 0], S[-1], rtol=0, atol=1e-6)


@pytest.mark.gpu
def test_gpu_decode_steps_reproduce_the_worked_example():
    from delta_rule_linear_efla_b200 import efla

    q, k, v, beta, _, o, S = load()
    t = lambda x: torch.tensor(x, dtype=torch.float32, device="cuda")
    state = torch.zeros(1, 1, 2, 2, dtype=torch.float32, device="cuda")
    for i in range(q.shape[2]):
        o_i = efla.recurrent_step(t(q[:, :, i]), t(k[:, :, i]), t(v[:, :, i]), t(beta[:, :, i]), state)
        torch.cuda.synchronize()
        np.testing.assert_allclose(o_i.cpu().numpy().reshape(2), o[0, 0, i], rtol=0, atol=1e-6)
        np.testing.assert_allclose(state.cpu().numpy()[0, 0], S[i], rtol=0, atol=1e-6)
