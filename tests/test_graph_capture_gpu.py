"""CUDA-graph capture of the forward paths: every kernel of a call is enqueued on the caller's
stream with no host synchronisation, so a captured call replays to the eager call's results bit
for bit.  Covered: the tensor-core chunk forward in one pass and cut into sequence segments, the
keeping forward of a training step, and a decode step (its in-place state carry included)."""
import pytest
import torch

from delta_rule_linear_efla_b200 import efla, inputs

pytestmark = pytest.mark.gpu


def _inputs(wid, **kw):
    x = inputs.make_inputs(inputs.workload(wid, **kw), seed=13)
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _capture(fn):
    """Warm up on a side stream, capture one call, replay it once; returns its outputs."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = fn()
    graph.replay()
    torch.cuda.synchronize()
    return graph, out


@pytest.mark.parametrize("wid,kw", [(4, dict(B=1, H=3, L=300)),      # one pass, ragged tail
                                    (3, dict(B=1, H=2, L=4096))])    # sequence segments
def test_chunk_forward_replays_bit_for_bit(wid, kw):
    d = _inputs(wid, **kw)
    args = (d["q"], d["k"], d["v"], d["beta"], d["S0"])
    ref = efla.chunk_fwd(*args, o_dtype=torch.bfloat16)
    graph, got = _capture(lambda: efla.chunk_fwd(*args, o_dtype=torch.bfloat16))
    assert efla.last_device_error() == 0
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    del graph


def test_keeping_forward_replays_bit_for_bit():
    d = _inputs(4, B=1, H=2, L=200)
    args = (d["q"], d["k"], d["v"], d["beta"], d["S0"])
    ref = efla.chunk_fwd_keep(*args)
    graph, got = _capture(lambda: efla.chunk_fwd_keep(*args))
    assert efla.last_device_error() == 0
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    del graph


def test_decode_step_replays_with_its_state_carry():
    """Two replays of a captured decode step advance the state twice, as two eager steps do."""
    g = torch.Generator().manual_seed(3)
    B, H, dk, dv = 4, 8, 128, 128
    q, k = (torch.randn(B, H, dk, generator=g).to(torch.bfloat16).cuda() for _ in range(2))
    v = torch.randn(B, H, dv, generator=g).to(torch.bfloat16).cuda()
    beta = torch.sigmoid(torch.randn(B, H, generator=g)).to(torch.bfloat16).cuda()
    S0 = (torch.randn(B, H, dk, dv, generator=g) * 0.1).cuda()
    S_ref = S0.clone()
    o_ref = [efla.recurrent_step(q, k, v, beta, S_ref) for _ in range(2)]
    S = S0.clone()
    o = torch.empty(B, H, dv, device="cuda")
    graph, _ = _capture(lambda: efla.recurrent_step(q, k, v, beta, S, o=o))
    # the warm-up and the capture's replay have advanced S twice; start again from S0
    S.copy_(S0)
    outs = []
    for _ in range(2):
        graph.replay()
        torch.cuda.synchronize()
        outs.append(o.clone())
    assert efla.last_device_error() == 0
    assert torch.equal(S, S_ref)
    for a, b in zip(outs, o_ref):
        assert torch.equal(a, b)
