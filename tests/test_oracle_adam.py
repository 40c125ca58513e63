"""Oracle step pinned against independent references.

- Adam / AdamW against torch.optim in float64 (an independent implementation
  of Kingma-Ba Adam and Loshchilov-Hutter decoupled weight decay), within
  1e-6 relative. [P2] "Where We Were" names Adam/AdamW; the equations are the
  textbook ones.
- step-1 closed forms, and a zero gradient leaving the weights untouched.
- the rank-ordered binary32 gradient sum against numpy's sequential float32
  accumulation.
- ZeRO stage 1/2/3 results bit-identical to the plain data-parallel result for
  every Nd in 1..9 and Psi in 1..40 ([P2] "The Breakthrough": ZeRO leaves the
  training math untouched; [P1] "The replication nobody questioned").
- the overflow skip: state and t unchanged, and a skipped step followed by a
  good one equals the good one alone.
"""
import numpy as np
import pytest
import torch

from oracle import zero_ref as Z

F16_MAX = 65504.0


def _grads(rng, nd, n, sigma=1.0, scale=1.0):
    g = (rng.standard_normal((nd, n)) * sigma * scale).clip(-F16_MAX, F16_MAX)
    return [np.ascontiguousarray(row.astype(np.float16).view(np.uint16)) for row in g]


def _torch_run(w0, unscaled_grads_per_step, hp, adamw):
    p = torch.nn.Parameter(torch.from_numpy(w0.astype(np.float64)))
    kw = dict(lr=float(np.float32(hp.lr)), betas=(float(np.float32(hp.beta1)),
                                                   float(np.float32(hp.beta2))),
              eps=float(np.float32(hp.eps)), foreach=False)
    if adamw:
        opt = torch.optim.AdamW([p], weight_decay=float(np.float32(hp.weight_decay)), **kw)
    else:
        opt = torch.optim.Adam([p], weight_decay=0.0, **kw)
    for g in unscaled_grads_per_step:
        p.grad = torch.from_numpy(g.astype(np.float64))
        opt.step()
    st = opt.state[p]
    return p.detach().numpy(), st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()


def _rel_close(a, b, rel):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = np.maximum(np.abs(b), np.abs(b).max() * 1e-3 + 1e-30)
    return np.max(np.abs(a - b) / scale) <= rel


@pytest.mark.parametrize("adamw", [False, True])
def test_adam_matches_torch_fp64(adamw):
    rng = np.random.default_rng(7 + adamw)
    n, nd, steps, scale = 257, 4, 5, 1024.0
    hp = Z.hyper(lr=1e-3, weight_decay=0.01 if adamw else 0.0)
    w = rng.uniform(-0.1, 0.1, n).astype(np.float32)
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    p16 = np.zeros(n, np.uint16)
    w0 = w.copy()
    t = 0
    unscaled = []
    gmax = np.zeros(n)
    for _ in range(steps):
        gs = _grads(rng, nd, n, sigma=1e-3, scale=scale)
        # the reduced, unscaled gradient exactly as binary32 arithmetic makes it
        s = Z.f32_from_f16(gs[0])
        for g in gs[1:]:
            s = (s + Z.f32_from_f16(g)).astype(np.float32)
        # unscaled independently of the oracle: scale is a power of two, so
        # dividing in float64 is exact
        unscaled.append(s.astype(np.float64) / scale)
        gmax = np.maximum(gmax, np.abs(unscaled[-1]))
        sk, t = Z.dp_step(gs, w, m, v, p16, scale, hp, t)
        assert not sk
    assert t == steps
    tw, tm, tv = _torch_run(w0, unscaled, hp, adamw)
    assert _rel_close(w, tw, 1e-6)
    assert _rel_close(v, tv, 1e-6)
    # m is a signed running average and cancels; its rounding error is relative
    # to the size of the terms it sums, (1 - beta1) |g|, not to |m| itself
    assert np.max(np.abs(m - tm) / ((1 - 0.9) * gmax)) <= 1e-6
    assert (p16 == Z.f16_from_f32(w)).all()


def test_inv_scale():
    for k in range(-20, 40):
        assert Z.inv_scale(2.0**k) == np.float32(2.0 ** (-k))
    # non powers of two: one rounding of the exact reciprocal
    for x in (3.0, 1000.0, 65535.0, 1e-3):
        r = Z.inv_scale(x)
        assert abs(float(r) - 1.0 / float(np.float32(x))) <= 0.5 * float(np.spacing(r))


def test_step1_closed_form():
    rng = np.random.default_rng(3)
    n = 1000
    hp = Z.hyper(lr=1e-3)
    w = rng.uniform(-0.1, 0.1, n).astype(np.float32)
    w0 = w.astype(np.float64)
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    p16 = np.zeros(n, np.uint16)
    gs = _grads(rng, 1, n, sigma=0.5)
    g = Z.f32_from_f16(gs[0]).astype(np.float64)
    sk, t = Z.dp_step(gs, w, m, v, p16, 1.0, hp, 0)
    assert not sk and t == 1
    b1, b2 = 0.9, 0.999
    assert np.allclose(m, (1 - np.float32(b1)) * g, rtol=1e-6, atol=0)
    assert np.allclose(v, (1 - np.float32(b2)) * g * g, rtol=1e-6, atol=0)
    expect = w0 - np.float32(1e-3) * g / (np.abs(g) + np.float32(1e-8))
    # within a few roundings of the operands' size: the subtraction rounds at
    # the scale of max(|w0|, |w1|), and lr * u rounds at the scale of lr
    mag = np.maximum(np.maximum(np.abs(w0), np.abs(w)), 1e-3).astype(np.float32)
    assert (np.abs(w - expect) <= 2 * np.spacing(mag)).all()
    # the step moves each weight by lr against the sign of its gradient
    nz = g != 0
    assert np.allclose((w0 - w)[nz], 1e-3 * np.sign(g[nz]), rtol=1e-4)


def test_zero_gradient_leaves_weights():
    rng = np.random.default_rng(4)
    n = 513
    w = rng.uniform(-3, 3, n).astype(np.float32)
    w[:4] = [0.0, -0.0, 1e-40, -1e-40]
    w_before = w.copy()
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    p16 = np.zeros(n, np.uint16)
    zeros = [np.zeros(n, np.uint16) for _ in range(3)]
    sk, t = Z.dp_step(zeros, w, m, v, p16, 8.0, Z.hyper(), 0)
    assert not sk and t == 1
    assert (w.view(np.uint32) == w_before.view(np.uint32)).all()


def test_reduction_is_rank_ordered_fp32():
    # values chosen so that the order of the fp32 additions matters: 0.001 is
    # below half a binary32 spacing of 65504, so it is lost if added to it first
    g = np.array([[65504.0], [0.001], [-65504.0]], np.float16)
    gs = [np.ascontiguousarray(r.view(np.uint16)) for r in g]
    w = np.zeros(1, np.float32)
    m = np.zeros(1, np.float32)
    v = np.zeros(1, np.float32)
    p16 = np.zeros(1, np.uint16)
    Z.dp_step(gs, w, m, v, p16, 1.0, Z.hyper(beta1=0.0, beta2=0.0), 0)
    # beta1 = 0 makes m the reduced gradient itself
    f = g.astype(np.float32)[:, 0]
    seq = np.add.accumulate(f, dtype=np.float32)[-1]
    assert m[0] == seq == np.float32(0.0)
    assert (f[0] + f[2]) + f[1] != 0.0  # another order keeps it
    rng = np.random.default_rng(5)
    for nd in (2, 3, 8, 17):
        gs = _grads(rng, nd, 300, sigma=300.0)
        w = np.zeros(300, np.float32)
        m = np.zeros(300, np.float32)
        v = np.zeros(300, np.float32)
        Z.dp_step(gs, w, m, v, np.zeros(300, np.uint16), 1.0, Z.hyper(beta1=0.0, beta2=0.0), 0)
        stack = np.stack([Z.f32_from_f16(x) for x in gs])
        assert (m.view(np.uint32) == np.add.accumulate(stack, axis=0, dtype=np.float32)[-1]
                .view(np.uint32)).all()


def _zero12_run(psi, nd, steps, rng, hp, scale, inject=None):
    w0 = rng.uniform(-1, 1, psi).astype(np.float32)
    parts = [Z.partition(psi, nd, r) for r in range(nd)]
    w_sh = [w0[b:e].copy() for b, e in parts]
    m_sh = [np.zeros(e - b, np.float32) for b, e in parts]
    v_sh = [np.zeros(e - b, np.float32) for b, e in parts]
    rep = [Z.f16_from_f32(w0) for _ in range(nd)]
    dw, dm, dv = w0.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32)
    dp16 = Z.f16_from_f32(w0)
    t_z = t_d = 0
    for s in range(steps):
        gs = _grads(rng, nd, psi, sigma=0.1, scale=scale)
        if inject is not None and s == inject[0]:
            gs[inject[1]][inject[2]] = 0x7C00
        sk_z, t_z = Z.zero12_step(psi, gs, w_sh, m_sh, v_sh, rep, scale, hp, t_z)
        sk_d, t_d = Z.dp_step(gs, dw, dm, dv, dp16, scale, hp, t_d)
        assert sk_z == sk_d and t_z == t_d
    return (np.concatenate(w_sh), np.concatenate(m_sh), np.concatenate(v_sh), rep,
            dw, dm, dv, dp16, t_z)


@pytest.mark.parametrize("nd", range(1, 10))
def test_zero12_equals_dp_bitwise(nd):
    rng = np.random.default_rng(100 + nd)
    hp = Z.hyper(lr=1e-2, weight_decay=0.01)
    for psi in range(1, 41):
        zw, zm, zv, rep, dw, dm, dv, dp16, _ = _zero12_run(psi, nd, 3, rng, hp, 64.0)
        assert (zw.view(np.uint32) == dw.view(np.uint32)).all()
        assert (zm.view(np.uint32) == dm.view(np.uint32)).all()
        assert (zv.view(np.uint32) == dv.view(np.uint32)).all()
        for r in rep:
            assert (r == dp16).all()


def _zero3_run(numel, nd, steps, rng, hp, scale, inject=None):
    psi = sum(numel)
    w0 = rng.uniform(-1, 1, psi).astype(np.float32)
    offs = np.concatenate([[0], np.cumsum(numel)])
    w_sh, p_sh = [], []
    for r in range(nd):
        pieces = []
        for ti, n in enumerate(numel):
            b, e = Z.chunk(n, nd, r)
            pieces.append(w0[offs[ti] + b: offs[ti] + e])
        w_sh.append(np.concatenate(pieces).astype(np.float32) if pieces else np.zeros(0, np.float32))
        p_sh.append(Z.f16_from_f32(w_sh[-1]))
    m_sh = [np.zeros_like(x) for x in w_sh]
    v_sh = [np.zeros_like(x) for x in w_sh]
    dw, dm, dv = w0.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32)
    dp16 = Z.f16_from_f32(w0)
    t_z = t_d = 0
    for s in range(steps):
        gs = _grads(rng, nd, psi, sigma=0.1, scale=scale)
        if inject is not None and s == inject[0]:
            gs[inject[1]][inject[2]] = 0xFC00
        sk_z, t_z = Z.zero3_step(numel, gs, w_sh, m_sh, v_sh, p_sh, scale, hp, t_z)
        sk_d, t_d = Z.dp_step(gs, dw, dm, dv, dp16, scale, hp, t_d)
        assert sk_z == sk_d and t_z == t_d
    return w_sh, m_sh, v_sh, p_sh, dw, dm, dv, dp16, offs


def _assemble(numel, nd, sh, offs, dtype):
    out = np.zeros(sum(numel), dtype)
    for r in range(nd):
        q = 0
        for ti, n in enumerate(numel):
            b, e = Z.chunk(n, nd, r)
            out[offs[ti] + b: offs[ti] + e] = sh[r][q: q + e - b]
            q += e - b
    return out


@pytest.mark.parametrize("nd", range(1, 10))
def test_zero3_equals_dp_bitwise(nd):
    rng = np.random.default_rng(200 + nd)
    hp = Z.hyper(lr=1e-2)
    for trial in range(12):
        numel = [int(x) for x in rng.integers(1, 14, size=rng.integers(1, 5))]
        w_sh, m_sh, v_sh, p_sh, dw, dm, dv, dp16, offs = _zero3_run(numel, nd, 3, rng, hp, 16.0)
        for sh, ref in ((w_sh, dw), (m_sh, dm), (v_sh, dv)):
            got = _assemble(numel, nd, sh, offs, np.float32)
            assert (got.view(np.uint32) == ref.view(np.uint32)).all()
        assert (_assemble(numel, nd, p_sh, offs, np.uint16) == dp16).all()
        # the layer gather rebuilds each unit from the shards
        units = list(np.sort(rng.integers(0, 3, size=len(numel))))
        for u in sorted(set(units)):
            got = Z.zero3_gather(numel, units, nd, u, p_sh)
            want = np.concatenate([dp16[offs[i]:offs[i + 1]] for i in range(len(numel))
                                   if units[i] == u])
            assert (got == want).all()


def test_skip_leaves_state_and_t():
    rng = np.random.default_rng(9)
    psi, nd = 37, 4
    hp = Z.hyper()
    # clean 3-step run vs the same run with an inf injected at step index 1,
    # on rank 3, in partition 0 (owned by rank 0): the flag is global.
    clean = _zero12_run(psi, nd, 3, np.random.default_rng(1), hp, 1024.0)
    skip = _zero12_run(psi, nd, 3, np.random.default_rng(1), hp, 1024.0, inject=(1, 3, 0))
    assert clean[-1] == 3 and skip[-1] == 2
    # the skipped run equals a run of steps 0 and 2 only
    rng2 = np.random.default_rng(1)
    w0 = rng2.uniform(-1, 1, psi).astype(np.float32)
    g_steps = [_grads(rng2, nd, psi, sigma=0.1, scale=1024.0) for _ in range(3)]
    w, m, v = w0.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32)
    p16 = Z.f16_from_f32(w0)
    t = 0
    for s in (0, 2):
        _, t = Z.dp_step(g_steps[s], w, m, v, p16, 1024.0, hp, t)
    assert (skip[0].view(np.uint32) == w.view(np.uint32)).all()
    assert (skip[1].view(np.uint32) == m.view(np.uint32)).all()
    assert (skip[2].view(np.uint32) == v.view(np.uint32)).all()
    for r in skip[3]:
        assert (r == p16).all()


def test_skip_on_nan_and_on_overflowing_unscale():
    n = 16
    w = np.linspace(-1, 1, n).astype(np.float32)
    m = np.full(n, 0.5, np.float32)
    v = np.full(n, 0.25, np.float32)
    p16 = Z.f16_from_f32(w)
    snap = [a.copy() for a in (w, m, v, p16)]
    g = [np.zeros(n, np.uint16) for _ in range(2)]
    g[1][n - 1] = 0x7E00  # NaN
    sk, t = Z.dp_step(g, w, m, v, p16, 1.0, Z.hyper(), 5)
    assert sk and t == 5
    for a, b in zip((w, m, v, p16), snap):
        assert (a.view(np.uint8) == b.view(np.uint8)).all()
    # finite fp16 gradients whose unscaled sum overflows binary32
    g = [np.full(n, 0x7BFF, np.uint16) for _ in range(2)]  # 65504 each
    sk, t = Z.dp_step(g, w, m, v, p16, 1e-36, Z.hyper(), 5)
    assert sk and t == 5


def test_stage3_skip_is_global():
    rng = np.random.default_rng(11)
    numel = [9, 4, 13]
    # inf on rank 2 in tensor 0's chunk owned by rank 0
    res = _zero3_run(numel, 3, 2, rng, Z.hyper(), 4.0, inject=(0, 2, 0))
    assert res is not None


# ---- per-tensor weight-decay exclusion -------------------------------------
# Decoupled weight decay (Loshchilov and Hutter) applied to some tensors only:
# an excluded tensor takes the Adam update with weight decay 0.

def _mask_case(seed, n_tensors=7):
    rng = np.random.default_rng(seed)
    numel = rng.integers(1, 60, n_tensors)
    no_decay = [bool(i % 2) for i in range(n_tensors)]
    return rng, [int(x) for x in numel], no_decay


def test_masked_decay_matches_torch_param_groups():
    """Against torch.optim.AdamW in float64 with two parameter groups (weight
    decay on the decayed tensors, 0 on the excluded ones)."""
    rng, numel, no_decay = _mask_case(11)
    n, nd, steps, scale = sum(numel), 4, 4, 1024.0
    hp = Z.hyper(lr=1e-3, weight_decay=0.1)
    mask = Z.decay_mask(numel, no_decay)
    w = rng.uniform(-0.5, 0.5, n).astype(np.float32)
    w0 = w.copy()
    m, v, p16 = np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.uint16)
    t, unscaled, gmax = 0, [], np.zeros(n)
    for _ in range(steps):
        gs = _grads(rng, nd, n, sigma=1e-3, scale=scale)
        s = Z.f32_from_f16(gs[0])
        for g in gs[1:]:
            s = (s + Z.f32_from_f16(g)).astype(np.float32)
        unscaled.append(s.astype(np.float64) / scale)
        gmax = np.maximum(gmax, np.abs(unscaled[-1]))
        sk, t = Z.dp_step(gs, w, m, v, p16, scale, hp, t, decay=mask)
        assert not sk
    # torch: one parameter per tensor, grouped by exclusion
    offs = np.concatenate([[0], np.cumsum(numel)])
    params = [torch.nn.Parameter(torch.from_numpy(w0[offs[i]:offs[i + 1]].astype(np.float64)))
              for i in range(len(numel))]
    groups = [{"params": [p for p, x in zip(params, no_decay) if not x],
               "weight_decay": float(np.float32(hp.weight_decay))},
              {"params": [p for p, x in zip(params, no_decay) if x], "weight_decay": 0.0}]
    opt = torch.optim.AdamW(groups, lr=float(np.float32(hp.lr)),
                            betas=(float(np.float32(0.9)), float(np.float32(0.999))),
                            eps=float(np.float32(1e-8)), foreach=False)
    for g in unscaled:
        for i, p in enumerate(params):
            p.grad = torch.from_numpy(g[offs[i]:offs[i + 1]].copy())
        opt.step()
    tw = np.concatenate([p.detach().numpy() for p in params])
    assert _rel_close(w, tw, 1e-6)
    # the excluded tensors really differ from a run that decays everything
    w_all = w0.copy()
    rng2, _, _ = _mask_case(11)
    rng2.uniform(-0.5, 0.5, n)
    m2, v2, t2 = np.zeros(n, np.float32), np.zeros(n, np.float32), 0
    for _ in range(steps):
        gs = _grads(rng2, nd, n, sigma=1e-3, scale=scale)
        _, t2 = Z.dp_step(gs, w_all, m2, v2, p16.copy(), scale, hp, t2)
    excl = mask == 0
    assert (w_all[excl] != w[excl]).any()
    assert (w_all[~excl].view(np.uint32) == w[~excl].view(np.uint32)).all()


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_masked_decay_is_elementwise_selection(seed):
    """Elements are independent: a masked step equals, element by element, the
    unmasked step with the weight decay or with weight decay 0, bit for bit;
    an all-ones mask equals no mask."""
    rng, numel, no_decay = _mask_case(seed, n_tensors=9)
    n, nd = sum(numel), 3
    mask = Z.decay_mask(numel, no_decay)
    w0 = rng.uniform(-2, 2, n).astype(np.float32)
    m0 = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    v0 = (rng.uniform(0, 1e-6, n)).astype(np.float32)
    gs = _grads(rng, nd, n, sigma=1e-3, scale=256.0)
    hp = Z.hyper(lr=1e-2, weight_decay=0.05)
    hp0 = Z.hyper(lr=1e-2, weight_decay=0.0)
    out = {}
    for name, h, dm in (("masked", hp, mask), ("ones", hp, np.ones(n, np.uint8)),
                        ("wd", hp, None), ("nowd", hp0, None)):
        w, m, v, p = w0.copy(), m0.copy(), v0.copy(), np.zeros(n, np.uint16)
        sk, t = Z.dp_step(gs, w, m, v, p, 256.0, h, 2, decay=dm)
        assert not sk and t == 3
        out[name] = (w, m, v, p)
    sel = mask != 0
    for k in range(4):
        expect = np.where(sel, out["wd"][k], out["nowd"][k])
        assert (out["masked"][k].view(np.uint8) == expect.view(np.uint8)).all()
        assert (out["ones"][k].view(np.uint8) == out["wd"][k].view(np.uint8)).all()
    assert (out["wd"][0] != out["nowd"][0]).any()


# ---- ZeRO == DP on random sizes (beyond the brute-force grid) ---------------
from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=40, deadline=None, derandomize=True)
@given(psi=st.integers(1, 5000), nd=st.integers(1, 64), n_t=st.integers(1, 6), seed=st.integers(0, 10**6))
def test_zero_stages_equal_dp_random(psi, nd, n_t, seed):
    """Stage 1/2 and stage 3 (random tensor split) are bit-identical to the
    plain data-parallel step, including empty partitions and chunks."""
    rng = np.random.default_rng(seed)
    n_t = min(n_t, psi)
    cuts = np.sort(rng.choice(np.arange(1, psi), size=n_t - 1, replace=False)) if n_t > 1 else []
    numel = [int(x) for x in np.diff(np.concatenate([[0], cuts, [psi]]))]
    w0 = rng.uniform(-1, 1, psi).astype(np.float32)
    gs = _grads(rng, nd, psi, sigma=1e-3, scale=256.0)
    hp = Z.hyper(lr=1e-2, weight_decay=0.01)
    w, m, v, p = w0.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32), np.zeros(psi, np.uint16)
    _, t = Z.dp_step(gs, w, m, v, p, 256.0, hp, 0)
    # stage 1/2
    parts = [Z.partition(psi, nd, r) for r in range(nd)]
    ws = [w0[b:e].copy() for b, e in parts]
    ms = [np.zeros(e - b, np.float32) for b, e in parts]
    vs = [np.zeros(e - b, np.float32) for b, e in parts]
    reps = [np.zeros(psi, np.uint16) for _ in range(nd)]
    _, t12 = Z.zero12_step(psi, gs, ws, ms, vs, reps, 256.0, hp, 0)
    assert t12 == t
    assert (np.concatenate(ws).view(np.uint32) == w.view(np.uint32)).all()
    assert all((r == p).all() for r in reps)
    # stage 3
    offs = np.concatenate([[0], np.cumsum(numel)])
    w3 = [np.concatenate([w0[offs[i] + b: offs[i] + e] for i, n in enumerate(numel)
                          for b, e in [Z.chunk(n, nd, r)]]).astype(np.float32) for r in range(nd)]
    m3 = [np.zeros_like(x) for x in w3]
    v3 = [np.zeros_like(x) for x in w3]
    p3 = [np.zeros(x.size, np.uint16) for x in w3]
    _, t3 = Z.zero3_step(numel, gs, w3, m3, v3, p3, 256.0, hp, 0)
    assert t3 == t
    units = list(range(len(numel)))
    for u in units:
        got = Z.zero3_gather(numel, units, nd, u, p3)
        assert (got == p[offs[u]:offs[u + 1]]).all()
