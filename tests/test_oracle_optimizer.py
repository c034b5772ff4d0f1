"""Pins of the oracle's optimizer step (clip -> AdamW -> clamp) to facts outside it.

The pages fix the recipe (P5 §6.2 clip_grad_norm_ with max_norm 1.0; P1's AdamW with lr
1e-3, betas (0.9, 0.95), weight decay 0.01, eps 1e-6; P1's clamp of the latent weight to
[-1, 1]) and call
torch's routines for it, so torch's own clip_grad_norm_ + AdamW + clamp_ in float64
is an independent pin; the first step and the clip coefficient also have closed forms.
"""
import numpy as np
import pytest
import torch

HP = dict(lr=1e-3, betas=(0.9, 0.95), eps=1e-6, weight_decay=0.01)
# large lr * wd and eps: the order of decay and update, and where eps enters, show up
HP_LOUD = dict(lr=5e-2, betas=(0.8, 0.9), eps=1e-3, weight_decay=0.3)


def _ulp(a, b):
    ai = np.asarray(a, dtype=np.float32).view(np.int32).astype(np.int64)
    bi = np.asarray(b, dtype=np.float32).view(np.int32).astype(np.int64)
    # map the sign-magnitude order onto integers so that -0.0 and +0.0 are neighbours
    ai = np.where(ai < 0, -(ai & 0x7FFFFFFF), ai)
    bi = np.where(bi < 0, -(bi & 0x7FFFFFFF), bi)
    return np.abs(ai - bi)


def _torch_step(W, dW, m, v, t, max_norm, hp):
    """One float64 step with torch's routines from the given fp32 state."""
    p = torch.nn.Parameter(torch.from_numpy(W.astype(np.float64)))
    p.grad = torch.from_numpy(dW.astype(np.float64))
    opt = torch.optim.AdamW([p], foreach=False, **hp)
    if t > 1:
        opt.state[p]["step"] = torch.tensor(float(t - 1), dtype=torch.float64)
        opt.state[p]["exp_avg"] = torch.from_numpy(m.astype(np.float64))
        opt.state[p]["exp_avg_sq"] = torch.from_numpy(v.astype(np.float64))
    if max_norm > 0:
        torch.nn.utils.clip_grad_norm_([p], max_norm)
    opt.step()
    with torch.no_grad():
        p.clamp_(-1.0, 1.0)
    st = opt.state[p]
    return p.detach().numpy(), st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()


@pytest.mark.parametrize("max_norm,hp", [(1.0, HP), (0.0, HP), (1e3, HP), (1.0, HP_LOUD), (0.0, HP_LOUD)])
def test_optimizer_matches_torch_adamw(ora, max_norm, hp):
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.3, size=(24, 40)).astype(np.float32)
    W[0, :4] = [0.9995, -0.9995, 1.0, -1.0]           # near / at the clamp
    m = np.zeros_like(W)
    v = np.zeros_like(W)
    for t in range(1, 5):
        dW = (rng.normal(0, 0.05, size=W.shape) * (1 + 3 * t)).astype(np.float32)
        dW[0, :2] = [-0.2, 0.2]                       # drives the planted weights past +-1
        W2, m2, v2, c = ora.optimizer_step(W, dW, m, v, t, max_norm=max_norm, **hp)
        tw, tm, tv = _torch_step(W, dW, m, v, t, max_norm, hp)
        assert _ulp(W2, tw.astype(np.float32)).max() <= 1
        assert _ulp(m2, tm.astype(np.float32)).max() <= 1
        assert _ulp(v2, tv.astype(np.float32)).max() <= 1
        W, m, v = W2, m2, v2
    assert W.max() <= 1.0 and W.min() >= -1.0
    assert W[0, 0] == 1.0 and W[0, 1] == -1.0          # clamped, not beyond


def test_optimizer_first_step_closed_form(ora):
    """t = 1 from zero moments: the bias corrections cancel, so without clipping
    W1 = W0 (1 - lr wd) - lr g / (|g| + eps)."""
    rng = np.random.default_rng(5)
    W = rng.normal(0, 0.2, size=(8, 64)).astype(np.float32)
    g = rng.normal(0, 1e-3, size=W.shape).astype(np.float32)
    z = np.zeros_like(W)
    W1, m1, v1, c = ora.optimizer_step(W, g, z, z, 1, max_norm=0.0, **HP)
    lr, wd, eps = HP["lr"], HP["weight_decay"], HP["eps"]
    gd = g.astype(np.float64)
    ref = W.astype(np.float64) * (1 - lr * wd) - lr * gd / (np.abs(gd) + eps)
    assert c == 1.0
    assert _ulp(W1, np.clip(ref, -1, 1).astype(np.float32)).max() <= 1
    assert _ulp(m1, (0.1 * gd).astype(np.float32)).max() <= 1
    assert _ulp(v1, (0.05 * gd * gd).astype(np.float32)).max() <= 1


def test_optimizer_clip_coefficient(ora):
    W = np.zeros((4, 8), dtype=np.float32)
    z = np.zeros_like(W)
    g = np.zeros_like(W)
    g[0, 0], g[1, 1] = 6.0, 8.0                        # norm exactly 10
    _, m1, _, c = ora.optimizer_step(W, g, z, z, 1, max_norm=1.0, **HP)
    assert c == pytest.approx(1.0 / (10.0 + 1e-6), rel=1e-15)
    assert m1[0, 0] == np.float32(0.1 * 6.0 * c)
    _, _, _, c2 = ora.optimizer_step(W, g * np.float32(0.05), z, z, 1, max_norm=1.0, **HP)
    assert c2 == 1.0                                   # norm 0.5 < max_norm: untouched
    _, _, _, c3 = ora.optimizer_step(W, z, z, z, 1, max_norm=1.0, **HP)
    assert c3 == 1.0                                   # zero gradient: coefficient capped at 1
