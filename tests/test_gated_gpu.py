"""GPU parity of the gated form, S_t = g_t (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T
(efla_chunk_fwd_gated, efla_recurrent_step_gated), against the oracle's gated form, element by
element on the same seeded inputs, with the parity bounds of every other test (max |delta| /
RMS <= 1e-4 for fp32 inputs, 2e-2 for bf16).  Gates are drawn as sigmoid(N(2, 1)) per token
(mean decay about 0.86, some tokens near 0.5), in the input dtype, so both sides see the same
rounded values.
"""
import numpy as np
import pytest
import torch

from conftest import rel_err
from delta_rule_linear_efla_b200 import efla, inputs

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _gate(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.sigmoid(2.0 + torch.randn(shape, generator=g)).to(dtype)


def _dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _unit_keys(x):
    k = x["k"].double()
    x["k"] = (k / k.norm(dim=-1, keepdim=True).clamp_min(1e-30)).to(x["k"].dtype)
    return x


@pytest.mark.parametrize("wid,kw", [(1, {}), (2, {}), (3, {}), (4, {}),
                                    (2, dict(B=1, H=2, L=77, dk=40, dv=24)),
                                    (5, dict(B=1, H=2, L=2000))])
def test_gated_chunk_forward_matches_oracle(oracle_mod, wid, kw):
    w = inputs.workload(wid, **kw)
    x = inputs.make_inputs(w, seed=300 + wid)
    x["g"] = _gate(x["beta"].shape, x["beta"].dtype, 400 + wid)
    d = _dev(x)
    o, S = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=w.chunk, g=d["g"])
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    o_ref, S_ref = oracle_mod.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], g=x["g"])
    tol = TOL[w.dtype]
    assert rel_err(o.cpu().numpy(), o_ref) <= tol
    assert rel_err(S.cpu().numpy(), S_ref) <= tol


def test_gated_delta_rule_matches_oracle(oracle_mod):
    """Under the Euler rule (alpha = beta) the gated form is Gated DeltaNet's update; unit-norm
    keys, where the delta rule is stable."""
    w = inputs.workload(2, B=2, H=2, L=300)
    x = _unit_keys(inputs.make_inputs(w, seed=31))
    x["g"] = _gate(x["beta"].shape, x["beta"].dtype, 32)
    d = _dev(x)
    o, S = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64, g=d["g"], rule="euler")
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_mod.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], g=x["g"], rule="euler")
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["bf16"]


def test_gate_of_one_is_the_ungated_forward_bit_for_bit():
    """fp32 inputs take the SIMT path either way; a gate of exactly 1 makes every decay factor
    e^0 = 1, so the gated call must reproduce the ungated one bit for bit."""
    w = inputs.workload(2, B=1, H=3, L=200, dk=64, dv=48, dtype="fp32")
    x = _dev(inputs.make_inputs(w, seed=33))
    one = torch.ones_like(x["beta"])
    o1, S1 = efla.chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], chunk=32)
    o2, S2 = efla.chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], chunk=32, g=one)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (40, 24)])
def test_gated_decode_step_matches_oracle(oracle_mod, dtype, dk, dv):
    w = inputs.workload(4, B=8, H=4, L=1, dk=dk, dv=dv, dtype=dtype)
    x = inputs.make_inputs(w, seed=34)
    g = _gate((w.B, w.H), x["beta"].dtype, 35)
    gen = torch.Generator().manual_seed(36)
    S = torch.randn((w.B, w.H, dk, dv), generator=gen) * 0.3
    q, k, v, beta = (x[n][:, :, 0].contiguous() for n in ("q", "k", "v", "beta"))
    Sd = S.cuda()
    o = efla.recurrent_step(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), Sd, g=g.cuda())
    torch.cuda.synchronize()
    o_ref = np.zeros((w.B, w.H, dv))
    S_ref = np.zeros((w.B, w.H, dk, dv))
    for b in range(w.B):
        for h in range(w.H):
            S_ref[b, h], o_ref[b, h], _ = oracle_mod.step(S[b, h], q[b, h], k[b, h], v[b, h],
                                                          float(beta[b, h]), g=float(g[b, h]))
    tol = TOL[dtype]
    assert rel_err(o.cpu().numpy(), o_ref) <= tol
    assert rel_err(Sd.cpu().numpy(), S_ref) <= tol


def test_gated_segments_match_oracle(oracle_mod):
    """Few heads and a long sequence: the gated form on the sequence-segment path (each
    segment's affine map, S_out = P S_in + H, carries the decays too), stiff inputs."""
    w = inputs.workload(5, B=1, H=2, L=8192 + 37)
    assert efla.chunk_fwd_path(w.B, w.H, w.L, w.dk, w.dv, 64, torch.bfloat16) == "tcgen05-segments"
    x = inputs.make_inputs(w, seed=41)
    x["g"] = _gate(x["beta"].shape, x["beta"].dtype, 42)
    d = _dev(x)
    o, S = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64, g=d["g"])
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    o_ref, S_ref = oracle_mod.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], g=x["g"])
    assert rel_err(o.cpu().numpy(), o_ref) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["bf16"]


@pytest.mark.parametrize("lo,hi", [(0.005, 0.05), (0.3, 0.6), (0.999, 1.0)])
def test_gated_strong_and_weak_decays(oracle_mod, lo, hi):
    """Decays from near 0 (the chunk's cumulative decay underflows: every factor the kernels
    apply must stay a decay of at most 1) to near 1, with a nonzero starting state and a
    ragged tail, bf16 output too."""
    w = inputs.workload(2, B=1, H=3, L=700, dk=128, dv=64, s0_std=0.3)
    x = inputs.make_inputs(w, seed=43)
    gen = torch.Generator().manual_seed(44)
    x["g"] = (lo + (hi - lo) * torch.rand(x["beta"].shape, generator=gen)).to(x["beta"].dtype)
    d = _dev(x)
    o_ref, S_ref = oracle_mod.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], g=x["g"])
    for odt in (torch.float32, torch.bfloat16):
        o, S = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64, g=d["g"], o_dtype=odt)
        torch.cuda.synchronize()
        assert efla.last_device_error() == 0
        assert np.isfinite(o.float().cpu().numpy()).all()
        tol = TOL["bf16"] + (2.0 ** -8 * np.abs(o_ref).max() / np.sqrt((o_ref ** 2).mean())
                             if odt == torch.bfloat16 else 0.0)
        assert rel_err(o.float().cpu().numpy(), o_ref) <= tol
        assert rel_err(S.cpu().numpy(), S_ref) <= TOL["bf16"]


def test_gate_of_one_on_the_tensor_cores_matches_the_ungated_forward(oracle_mod):
    """bf16 at the tensor-core sizes: with g = 1 every decay factor is exactly 1, so the gated
    kernels compute the ungated forward; they take the intra-chunk output term at higher
    precision (fp16 hi + lo factors), so against the oracle their error is at most the ungated
    kernels' (plus rounding noise), and the two results agree within the bf16 bound."""
    w = inputs.workload(4, B=1, H=4, L=1000)
    x = inputs.make_inputs(w, seed=45)
    d = _dev(x)
    one = torch.ones_like(d["beta"])
    o1, S1 = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64)
    o2, S2 = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64, g=one)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_mod.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"])
    e1, e2 = rel_err(o1.cpu().numpy(), o_ref), rel_err(o2.cpu().numpy(), o_ref)
    assert e2 <= e1 * 1.1 + 1e-4, (e1, e2)
    assert rel_err(S2.cpu().numpy(), S_ref) <= TOL["bf16"]
    assert rel_err(o2.cpu().numpy(), o1.cpu().numpy()) <= TOL["bf16"]
