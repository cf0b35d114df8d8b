"""Pins of the oracle's STA gradients (dQ, dK, dV) against facts other than
the backward code itself.

- Finite differences of the forward oracle (already pinned on its own) on
  inputs whose perturbed values are exact in bf16: a fourth-order central
  difference of L = sum(O * G) must equal <G-weighted gradient> from the
  backward oracle.  A dropped D term, a missing scale, a transposed operand
  or a wrong key set all move the gradient by O(1) and fail here.
- Dense special case: with a window covering the volume, the gradients equal
  those of torch autograd on dense softmax attention in fp64 (library routine).
- Masked case: torch autograd on attention masked with the brute-force
  nearest-centre mask from the forward pins.
- Invariants of softmax attention: the rows of dS sum to zero, so dK summed
  over keys is zero; the rows of P sum to one, so dV summed over keys equals
  dO summed over queries; with every v_j equal, dP does not depend on j and
  dQ = dK = 0.
"""
import numpy as np
import pytest
import torch

import oracle
from test_oracle_pins import brute_mask


def grid_bf16(rng, shape, k_max=160):
    """bf16 values k * 2^-7 with |k| <= k_max: x +- 2^-7 and x +- 2^-6 stay exact."""
    k = rng.integers(-k_max, k_max + 1, size=shape)
    return torch.from_numpy((k * 2.0 ** -7).astype(np.float32)).to(torch.bfloat16)


def loss(q, k, v, g, latent, tile, windows, scale):
    o, _ = oracle.sta_attention(q, k, v, latent, tile, windows, scale, nthreads=4)
    return float(np.sum(o * g.to(torch.float64).numpy()))


TINY = dict(latent=(4, 4, 6), tile=(2, 2, 2), windows=[[2, 4, 2], [4, 2, 6]], B=1, d=8)


def tiny_inputs(seed):
    rng = np.random.default_rng(seed)
    c = TINY
    N = c["latent"][0] * c["latent"][1] * c["latent"][2]
    H = len(c["windows"])
    shape = (c["B"], H, N, c["d"])
    q, k, v = (grid_bf16(rng, shape) for _ in range(3))
    g = grid_bf16(rng, shape, k_max=128)
    return q, k, v, g


def test_finite_differences():
    c = TINY
    q, k, v, g = tiny_inputs(7)
    scale = 0.5
    dq, dk, dv = oracle.sta_backward(q, k, v, g, c["latent"], c["tile"], c["windows"], scale, nthreads=4)
    grads = {"q": dq, "k": dk, "v": dv}
    h = 2.0 ** -7
    rng = np.random.default_rng(11)
    N = q.shape[2]
    for name in ("q", "k", "v"):
        for _ in range(10):
            idx = (0, int(rng.integers(0, 2)), int(rng.integers(0, N)), int(rng.integers(0, c["d"])))
            vals = {}
            for step in (-2, -1, 1, 2):
                t = {"q": q.clone(), "k": k.clone(), "v": v.clone()}
                x = float(t[name][idx])
                t[name][idx] = x + step * h
                assert float(t[name][idx]) == x + step * h  # exact in bf16
                vals[step] = loss(t["q"], t["k"], t["v"], g, c["latent"], c["tile"], c["windows"], scale)
            fd = (8.0 * (vals[1] - vals[-1]) - (vals[2] - vals[-2])) / (12.0 * h)
            an = grads[name][idx]
            assert abs(fd - an) <= 1e-7 + 1e-6 * abs(an), (name, idx, fd, an)


def autograd_reference(q, k, v, g, mask, scale):
    """fp64 gradients of masked softmax attention via torch autograd."""
    qd, kd, vd = (x.to(torch.float64).requires_grad_(True) for x in (q, k, v))
    s = torch.einsum("bhnd,bhmd->bhnm", qd, kd) * scale
    s = s.masked_fill(~mask, float("-inf"))
    o = torch.softmax(s, dim=-1) @ vd
    (o * g.to(torch.float64)).sum().backward()
    return qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy()


def test_dense_window_matches_autograd():
    latent, tile, d = (4, 6, 6), (2, 2, 2), 16
    N = 4 * 6 * 6
    torch.manual_seed(3)
    q, k, v, g = (torch.randn(1, 2, N, d).to(torch.bfloat16) for _ in range(4))
    windows = [[8, 12, 12], [4, 6, 6]]  # both cover the whole volume
    scale = float(np.float32(1.0 / np.sqrt(d)))
    dq, dk, dv = oracle.sta_backward(q, k, v, g, latent, tile, windows, scale, nthreads=4)
    mask = torch.ones(1, 2, N, N, dtype=torch.bool)
    rq, rk, rv = autograd_reference(q, k, v, g, mask, scale)
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.max(np.abs(a - b)) <= 1e-11 * max(1.0, np.max(np.abs(b)))


@pytest.mark.parametrize("latent,tile,windows", [
    ((6, 8, 8), (2, 4, 4), [[2, 4, 4], [4, 8, 4], [6, 4, 8]]),
    ((4, 8, 12), (2, 4, 4), [[2, 8, 8], [4, 4, 4], [2, 4, 12]]),
])
def test_masked_matches_autograd(latent, tile, windows):
    d = 8
    N = latent[0] * latent[1] * latent[2]
    H = len(windows)
    torch.manual_seed(5)
    q, k, v, g = (torch.randn(2, H, N, d).to(torch.bfloat16) for _ in range(4))
    scale = 0.37
    dq, dk, dv = oracle.sta_backward(q, k, v, g, latent, tile, windows, scale, nthreads=4)
    mask = torch.stack([torch.from_numpy(brute_mask(latent, tile, w)) for w in windows])
    mask = mask.unsqueeze(0).expand(2, H, N, N)
    rq, rk, rv = autograd_reference(q, k, v, g, mask, float(np.float32(scale)))
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.max(np.abs(a - b)) <= 1e-11 * max(1.0, np.max(np.abs(b)))


def test_sum_invariants():
    latent, tile, d = (6, 8, 8), (2, 4, 4), 16
    N = 6 * 8 * 8
    windows = [[2, 4, 4], [4, 8, 8]]
    torch.manual_seed(9)
    q, k, v, g = (torch.randn(1, 2, N, d).to(torch.bfloat16) for _ in range(4))
    dq, dk, dv = oracle.sta_backward(q, k, v, g, latent, tile, windows, 0.25, nthreads=4)
    scale_k = np.max(np.abs(dk))
    assert np.max(np.abs(dk.sum(axis=2))) <= 1e-11 * N * scale_k
    g64 = g.to(torch.float64).numpy()
    np.testing.assert_allclose(dv.sum(axis=2), g64.sum(axis=2), rtol=0, atol=1e-10)


def test_constant_values_give_zero_dq_dk():
    latent, tile, d = (4, 4, 4), (2, 2, 2), 8
    N = 64
    torch.manual_seed(13)
    q, k, g = (torch.randn(1, 1, N, d).to(torch.bfloat16) for _ in range(3))
    v = torch.randn(1, 1, 1, d).to(torch.bfloat16).expand(1, 1, N, d).contiguous()
    dq, dk, dv = oracle.sta_backward(q, k, v, g, latent, tile, [[2, 2, 2]], 0.5, nthreads=2)
    assert np.max(np.abs(dq)) < 1e-13
    assert np.max(np.abs(dk)) < 1e-13
    assert np.max(np.abs(dv)) > 0.1


def test_sampled_rows_equal_full():
    c = TINY
    q, k, v, g = tiny_inputs(21)
    dq, dk, dv = oracle.sta_backward(q, k, v, g, c["latent"], c["tile"], c["windows"], 0.3, nthreads=3)
    rows = np.array([[0, 0], [1, 5], [1, 95], [0, 40]], dtype=np.int64)
    sq = oracle.sta_backward_dq(q, k, v, g, c["latent"], c["tile"], c["windows"], 0.3, rows=rows)
    sk, sv = oracle.sta_backward_dkdv(q, k, v, g, c["latent"], c["tile"], c["windows"], 0.3, keys=rows)
    for i, (bh, t) in enumerate(rows):
        np.testing.assert_array_equal(sq[i], dq[0, bh, t])
        np.testing.assert_array_equal(sk[i], dk[0, bh, t])
        np.testing.assert_array_equal(sv[i], dv[0, bh, t])
