"""Pins for the oracle's sharded AdamW update.

"Sharded Training: FSDP2, DTensor, Tensor and Pipeline Parallelism": the
optimizer is built after sharding, so its state is sharded (fully_shard
paragraph); Fence 4 compares fully_shard + AdamW with plain AdamW to 1e-6.
"Introduction to PyTorch FSDP2 Backend Features", Working Principle: the
update state steps the sharded parameters with the gradient slices.

Pins: torch.optim.AdamW(foreach=False) on the unsharded parameter with the
averaged gradient (a library routine), within 1e-6 * (1 + |x|); the closed
form of the first step; a zero gradient leaves p * (1 - lr * wd); padding
stays +0 through several steps.
"""
import numpy as np
import pytest
import torch

from fully_sharded_shard_b200 import workloads as W

HP = dict(W.ADAMW_DEFAULTS)


def _close(got, want, tol=1e-6):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    return np.all(np.abs(got - want) <= tol * (1.0 + np.abs(want)))


def _unshard(p, buf, i):
    parts = []
    for j in range(p.N):
        lo = j * p.S + int(p.shard_off[i])
        parts.append(buf[lo:lo + p.valid_rows(i, j) * int(p.cols[i])])
    return np.concatenate(parts)


@pytest.mark.parametrize("shapes,N", [
    ([(32, 16), (32,), (4, 32), (4,)], 2),
    ([(7, 3), (5,), (1, 32), (1,), (13, 9)], 4),
    ([(33, 17), (6,)], 8),
])
def test_sharded_adamw_matches_torch_adamw(oracle, shapes, N):
    gen = torch.Generator().manual_seed(21)
    params = [torch.nn.Parameter(torch.empty(s).uniform_(-0.25, 0.25, generator=gen))
              for s in shapes]
    opt = torch.optim.AdamW(params, lr=HP["lr"], betas=(HP["beta1"], HP["beta2"]),
                            eps=HP["eps"], weight_decay=HP["weight_decay"],
                            foreach=False, fused=False)
    p = oracle.plan(shapes, N)
    arena = np.zeros(p.P_arena, np.float32)
    for i, x in enumerate(params):
        arena[p.arena_off[i]:p.arena_off[i] + x.numel()] = x.detach().reshape(-1).numpy()
    master = oracle.shard(p, arena)
    m = np.zeros_like(master)
    v = np.zeros_like(master)
    for step in range(1, 4):
        # the averaged gradient, as the reduce-scatter leaves it
        gfull = [torch.randn(s, generator=gen) for s in shapes]
        garena = np.zeros(p.P_arena, np.float32)
        for i, x in enumerate(params):
            x.grad = gfull[i].clone()
            garena[p.arena_off[i]:p.arena_off[i] + x.numel()] = gfull[i].reshape(-1).numpy()
        gshard = oracle.shard(p, garena)
        opt.step()
        oracle.adamw(master, m, v, gshard, step=step, **HP)
        for i, x in enumerate(params):
            st = opt.state[x]
            assert _close(_unshard(p, master, i), x.detach().reshape(-1).numpy())
            assert _close(_unshard(p, m, i), st["exp_avg"].reshape(-1).numpy())
            assert _close(_unshard(p, v, i), st["exp_avg_sq"].reshape(-1).numpy())
    # padding stays exactly +0 in parameters and both moments
    for buf in (master, m, v):
        for j in range(N):
            for i in range(p.n):
                lo = j * p.S + int(p.shard_off[i]) + p.valid_rows(i, j) * int(p.cols[i])
                hi = j * p.S + int(p.shard_off[i]) + int(p.shard_size[i])
                assert np.all(buf[lo:hi].view(np.uint32) == 0)


def test_first_step_closed_form(oracle):
    rng = np.random.default_rng(1)
    p0 = rng.normal(0, 0.02, 4096).astype(np.float32)
    g = rng.normal(0, 1e-3, 4096).astype(np.float32)
    master, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    oracle.adamw(master, m, v, g, step=1, **HP)
    lr, wd, eps = HP["lr"], HP["weight_decay"], HP["eps"]
    gd = g.astype(np.float64)
    # m = (1 - b1) g, v = (1 - b2) g^2, m_hat = g, sqrt(v_hat) = |g|
    want_p = p0.astype(np.float64) * (1 - lr * wd) - lr * gd / (np.abs(gd) + eps)
    assert np.all(np.abs(master - want_p) <= 2 ** -23 * np.abs(want_p) + 1e-12)
    assert np.all(np.abs(m - (1 - HP["beta1"]) * gd) <= 2 ** -23 * np.abs(m))
    assert np.all(np.abs(v - (1 - HP["beta2"]) * gd * gd) <= 2 ** -23 * np.abs(v))


def test_zero_gradient_only_decays(oracle):
    p0 = np.linspace(-1, 1, 1001, dtype=np.float32)
    master, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for step in (1, 2, 3):
        before = master.copy()
        oracle.adamw(master, m, v, np.zeros_like(p0), step=step, **HP)
        want = (before.astype(np.float64) * (1 - HP["lr"] * HP["weight_decay"])).astype(np.float32)
        assert np.array_equal(master, want)
        assert np.all(m == 0) and np.all(v == 0)


def test_update_magnitude_is_about_lr(oracle):
    """Adam is scale-invariant apart from eps and weight decay: doubling the
    gradient barely moves the result (the reason a 2x AVG bug hid)."""
    rng = np.random.default_rng(2)
    p0 = rng.normal(0, 0.02, 2048).astype(np.float32)
    g = rng.normal(0, 1e-3, 2048).astype(np.float32)
    a = [p0.copy(), np.zeros_like(p0), np.zeros_like(p0)]
    b = [p0.copy(), np.zeros_like(p0), np.zeros_like(p0)]
    oracle.adamw(*a, g, step=1, **HP)
    oracle.adamw(*b, 2 * g, step=1, **HP)
    big = np.abs(g) > 1e-4          # where eps is negligible against |g|
    d = np.abs(a[0].astype(np.float64) - b[0])[big]
    assert d.max() < 3e-8
    step = np.abs(a[0].astype(np.float64) - p0 * (1 - HP["lr"] * HP["weight_decay"]))[big]
    assert np.allclose(step, HP["lr"], rtol=1e-3)
