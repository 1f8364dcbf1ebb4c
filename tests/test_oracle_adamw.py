"""Pins of the oracle's shard update (unscale, AdamW on fp32 state, fp16 write).

- first step from zero moments has a closed form: p1 = p0(1 - lr wd) - lr g/(|g| + eps);
- zero gradients leave the moments at exactly zero and only decay the weights;
- with one rank and loss scale 1 the update is torch.optim.AdamW (fp32, CPU);
- non-finite ring sums are counted per bucket and propagate.
"""
import numpy as np
import torch

import oracle
from oracle.layout import make_layout


def _one_rank_case(n, seed, warm=False):
    rng = np.random.default_rng(seed)
    g16 = (rng.standard_normal((1, n)) * 1e-2).astype(np.float16)
    master = (rng.standard_normal(n) * 0.02).astype(np.float32)
    if warm:
        m = (rng.standard_normal(n) * 1e-3).astype(np.float32)
        v = np.abs(rng.standard_normal(n) * 1e-5).astype(np.float32)
    else:
        m = np.zeros(n, np.float32)
        v = np.zeros(n, np.float32)
    return g16, master, m, v


def test_first_step_closed_form():
    n, N, L = 4096, 4, 512.0
    rng = np.random.default_rng(3)
    g16 = (rng.standard_normal((N, n)) * 0.5).astype(np.float16)
    master = (rng.standard_normal(n) * 0.02).astype(np.float32)
    hp = oracle.Hyper(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=L)
    lay = make_layout([n], N, 1000, 128)
    res = oracle.run_steps(lay, 1, g16.view(np.uint16).copy(), master,
                           np.zeros(n, np.float32), np.zeros(n, np.float32), hp, 1)
    g = g16.astype(np.float64).sum(axis=0) / (N * L)
    decayed = master.astype(np.float64) * (1 - hp.lr * hp.weight_decay)
    stepped = hp.lr * g / (np.abs(g) + hp.eps)
    # relative to the size of the two terms (p1 itself can cancel to ~0)
    rel = np.abs(res.master - (decayed - stepped)) / (np.abs(decayed) + np.abs(stepped))
    assert rel.max() < 1e-6
    assert np.allclose(res.m, 0.1 * g, rtol=1e-6, atol=0)
    assert np.allclose(res.v, 0.001 * g * g, rtol=1e-5, atol=0)


def test_zero_gradient_only_decays():
    n, steps = 1000, 7
    lay = make_layout([n - 13], 3, 256, 8)
    P = lay.padded
    master = np.zeros(P, np.float32)
    master[: n - 13] = np.linspace(-1, 1, n - 13, dtype=np.float32)
    hp = oracle.Hyper(lr=1e-2, weight_decay=0.1, loss_scale=8.0)
    res = oracle.run_steps(lay, 2, np.zeros((3, P), np.uint16), master,
                           np.zeros(P, np.float32), np.zeros(P, np.float32), hp, steps)
    assert np.all(res.m == 0) and np.all(res.v == 0)
    expect = master.astype(np.float64) * (1 - 1e-2 * 0.1) ** steps
    assert np.all(np.abs(res.master - expect) <= steps * 2.0 ** -24 * np.abs(expect) + 0)
    assert np.all(res.master[n - 13:] == 0) and np.all(res.p16_full[n - 13:] == 0)
    assert np.all(np.abs(res.master) <= np.abs(master))


def test_matches_torch_adamw_single_rank():
    n, steps = 5000, 6
    for warm in (False, True):
        g16, master, m, v = _one_rank_case(n, 5, warm)
        hp = oracle.Hyper(lr=3e-3, beta1=0.85, beta2=0.99, eps=1e-8, weight_decay=0.05, loss_scale=1.0)
        lay = make_layout([n], 1, 999, 8)
        P = lay.padded
        pad = lambda a: np.concatenate([a, np.zeros(P - n, a.dtype)])
        res = oracle.run_steps(lay, 1, np.ascontiguousarray(pad(g16[0].view(np.uint16))[None]),
                               pad(master), pad(m), pad(v), hp, steps)
        p = torch.tensor(master.copy(), requires_grad=True)
        opt = torch.optim.AdamW([p], lr=hp.lr, betas=(hp.beta1, hp.beta2), eps=hp.eps,
                                weight_decay=hp.weight_decay, foreach=False)
        if warm:   # torch keeps its moments in its state dict: seed them with step 0
            opt.state[p]["step"] = torch.tensor(0.0)
            opt.state[p]["exp_avg"] = torch.tensor(m.copy())
            opt.state[p]["exp_avg_sq"] = torch.tensor(v.copy())
        gt = torch.tensor(g16[0].astype(np.float32))
        for _ in range(steps):
            p.grad = gt.clone()
            opt.step()
        tp = p.detach().numpy()
        tm = opt.state[p]["exp_avg"].numpy()
        tv = opt.state[p]["exp_avg_sq"].numpy()
        # relative to |p| + steps*lr, the most the steps can move p (p can pass through 0)
        assert np.max(np.abs(res.master[:n] - tp) / (np.abs(tp) + steps * hp.lr)) < 1e-6
        # m mixes old m and g with opposite signs: measure against |m| + |g|;
        # v sums positive terms, so plain relative error applies
        gmag = np.abs(g16[0].astype(np.float64))
        assert np.max(np.abs(res.m[:n] - tm) / (np.abs(tm) + gmag)) < 1e-6
        assert np.max(np.abs(res.v[:n] - tv) / np.abs(tv)) < 1e-5
        f16 = tp.astype(np.float16).view(np.uint16).astype(np.int32)
        assert np.max(np.abs(res.p16_full[:n].astype(np.int32) - f16)) <= 1


def test_nonfinite_counted_per_bucket_and_propagated():
    N, n = 4, 3000
    lay = make_layout([n], N, 700, 16)
    P = lay.padded
    g = np.zeros((N, P), np.uint16)
    marks = {5: 0x7C00, 1500: 0xFC00, 1501: 0x7E00, 2999: 0x7C00}   # +inf, -inf, nan, +inf
    for i, bits in marks.items():
        g[1, i] = bits
    g[2, 2999] = 0xFC00                                             # inf + -inf = nan
    res = oracle.run_steps(lay, 2, g, np.zeros(P, np.float32), np.zeros(P, np.float32),
                           np.zeros(P, np.float32), oracle.Hyper(), 1)
    want = [sum(1 for i in marks if lo <= i < hi) for lo, hi in lay.buckets]
    assert list(res.nonfinite) == want
    assert np.isinf(res.reduced[5]) and np.isnan(res.reduced[2999]) and np.isnan(res.reduced[1501])
    assert np.isnan(res.master[5]) or np.isinf(res.master[5])
