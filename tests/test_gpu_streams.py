"""Streams and CUDA graphs: a plan shared by calls running at once on two
streams (each launch takes its own work counter from the plan's pool), and the
forward and backward captured once in a CUDA graph and replayed on new
inputs.  Both must give the same bits as plain calls on one stream."""
import dataclasses

import pytest
import torch

import sta_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sta():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import sparse_attention_video_sta_b200 as s
    return s


def _inputs(w, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    shape = (w.batch, w.heads, w.tokens, w.head_dim)
    return [torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16) for _ in range(4)]


def test_two_streams_share_a_plan(sta):
    """Four input sets, forward and backward issued alternately on two
    streams with no ordering between them, against the same calls made one
    after another."""
    w = sta_inputs.WORKLOADS[2]
    w = dataclasses.replace(w, heads=4, name=w.name + "_heads4")
    plan = sta.sta_plan(w.latent, w.tile, w.batch, w.heads, sta_inputs.windows(w).tolist())
    sets = [_inputs(w, 100 + i) for i in range(4)]
    ref = []
    for q, k, v, do in sets:
        o, lse = sta.sta_attention(q, k, v, plan, w.softmax_scale)
        ref.append((o, lse) + sta.sta_attention_backward(q, k, v, o, lse, do, plan, w.softmax_scale))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    cur = torch.cuda.current_stream()
    for s in streams:
        s.wait_stream(cur)
    got = [None] * len(sets)
    for i, (q, k, v, do) in enumerate(sets):
        s = streams[i % 2]
        with torch.cuda.stream(s):
            o, lse = sta.sta_attention(q, k, v, plan, w.softmax_scale)
            got[i] = (o, lse) + sta.sta_attention_backward(q, k, v, o, lse, do, plan, w.softmax_scale)
    for s in streams:
        cur.wait_stream(s)
    torch.cuda.synchronize()
    assert sta.sta_last_device_status(plan) == 0
    for i in range(len(sets)):
        for a, b in zip(got[i], ref[i]):
            assert torch.equal(a, b), i


def test_graph_capture_replays_forward_and_backward(sta):
    """The fused forward and backward captured in one CUDA graph; new inputs
    copied into the captured buffers, replayed twice, equal plain calls."""
    w = sta_inputs.WORKLOADS[1]
    plan = sta.sta_plan(w.latent, w.tile, w.batch, w.heads, sta_inputs.windows(w).tolist())
    q, k, v, do = (x.clone() for x in _inputs(w, 7))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture (first-call set-up)
        o, lse = sta.sta_attention(q, k, v, plan, w.softmax_scale)
        sta.sta_attention_backward(q, k, v, o, lse, do, plan, w.softmax_scale)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        o_g, lse_g = sta.sta_attention(q, k, v, plan, w.softmax_scale)
        dq_g, dk_g, dv_g = sta.sta_attention_backward(q, k, v, o_g, lse_g, do, plan, w.softmax_scale)
    for seed in (8, 9):
        for dst, src in zip((q, k, v, do), _inputs(w, seed)):
            dst.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        o, lse = sta.sta_attention(q, k, v, plan, w.softmax_scale)
        dq, dk, dv = sta.sta_attention_backward(q, k, v, o, lse, do, plan, w.softmax_scale)
        assert sta.sta_last_device_status(plan) == 0
        for a, b in ((o_g, o), (lse_g, lse), (dq_g, dq), (dk_g, dk), (dv_g, dv)):
            assert torch.equal(a, b), seed
    del graph


def test_tensors_on_another_device_than_the_plan_are_rejected(sta):
    """The binding runs every call on the device of its tensors and its plan,
    and refuses a mismatch before any launch (checked here by marking the plan
    as another device's: nothing reaches the library or that device)."""
    w = sta_inputs.WORKLOADS[1]
    plan = sta.sta_plan(w.latent, w.tile, w.batch, w.heads, sta_inputs.windows(w).tolist())
    assert plan.device == torch.cuda.current_device()
    q, k, v, do = _inputs(w, 3)
    o, lse = sta.sta_attention(q, k, v, plan, w.softmax_scale)
    real = plan.device
    plan.device = real + 1
    try:
        for call in (lambda: sta.sta_attention(q, k, v, plan, w.softmax_scale),
                     lambda: sta.sta_attention(q, k, v, plan, w.softmax_scale, fused=False),
                     lambda: sta.sta_attention_backward(q, k, v, o, lse, do, plan, w.softmax_scale)):
            with pytest.raises(ValueError, match="one CUDA device"):
                call()
    finally:
        plan.device = real
    assert sta.sta_last_device_status(plan) == 0
