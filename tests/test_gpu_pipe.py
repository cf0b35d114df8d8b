"""The host-memory pipeline (sta_pipe_*) gives the same bits as the fused
forward on device tensors, across more calls than it has buffer slots (so
slots are reused while earlier calls are still copying out)."""
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


@pytest.mark.parametrize("depth", [1, 2, 3])
def test_pipe_matches_forward(sta, depth):
    w = sta_inputs.WORKLOADS[1]
    wins = sta_inputs.windows(w).tolist()
    plan = sta.sta_plan(w.latent, w.tile, w.batch, w.heads, wins)
    pipe = sta.sta_pipe_create(plan, w.head_dim, w.softmax_scale, depth=depth)
    calls = 5
    g = torch.Generator().manual_seed(depth)
    ins = [[torch.randn(w.batch, w.heads, w.tokens, w.head_dim, generator=g).to(torch.bfloat16).pin_memory()
            for _ in range(3)] for _ in range(calls)]
    outs = [(torch.empty(w.batch, w.heads, w.tokens, w.head_dim, dtype=torch.bfloat16).pin_memory(),
             torch.empty(w.batch, w.heads, w.tokens, dtype=torch.float32).pin_memory()) for _ in range(calls)]
    for (q, k, v), (o, l) in zip(ins, outs):
        pipe.submit(q, k, v, o, l)
    pipe.wait()
    for (q, k, v), (o, l) in zip(ins, outs):
        od, ld = sta.sta_attention(q.cuda(), k.cuda(), v.cuda(), plan, w.softmax_scale)
        assert torch.equal(o, od.cpu()) and torch.equal(l, ld.cpu())
    pipe.destroy()
    assert sta.sta_last_device_status(plan) == 0


def test_pipe_rejects_pageable_and_wrong_shapes(sta):
    w = sta_inputs.WORKLOADS[1]
    plan = sta.sta_plan(w.latent, w.tile, w.batch, w.heads, sta_inputs.windows(w).tolist())
    pipe = sta.sta_pipe_create(plan, w.head_dim, w.softmax_scale)
    x = torch.zeros(w.batch, w.heads, w.tokens, w.head_dim, dtype=torch.bfloat16)
    l = torch.zeros(w.batch, w.heads, w.tokens, dtype=torch.float32).pin_memory()
    with pytest.raises(ValueError):
        pipe.submit(x, x, x, x, l)  # pageable
    xp = x.pin_memory()
    with pytest.raises(ValueError):
        pipe.submit(xp, xp, xp, xp[:, :, :-1].contiguous().pin_memory(), l)
    pipe.destroy()
