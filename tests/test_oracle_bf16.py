"""Oracle pins for the BF16 setup without fp32 master weights ([P3] "Why
parameter count is not training memory": not every BF16 setup keeps master
weights; [P2] "The Mathematics": model-state memory (2 + 2 + K) Psi, here
K = 8, the two Adam moments).

- bfloat16 decoding of all 2^16 patterns and rounding over a sweep of binary32
  patterns, against torch's bfloat16 conversion (round to nearest even).
- the step against float64 torch.optim.AdamW restarted from the stored
  bfloat16 parameter every step: moments within 1e-6, the new parameter
  within one bfloat16 spacing.
- what dropping the master costs ([P1] "Why you can't just delete the fp32
  copies": updates below half a spacing are lost): with |w| in [1, 2) and
  lr = 1e-3 every bfloat16 parameter stays put while the fp32-master step
  moves every one.
- the skip leaves parameters, moments and t unchanged.
"""
import numpy as np
import pytest
import torch

from oracle import zero_ref as Z


def _bits_to_bf16_f32(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16).float().numpy()


def test_bf16_decode_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = Z.f32_from_bf16(bits)
    want = _bits_to_bf16_f32(bits)
    nan = np.isnan(want)
    assert (np.isnan(got) == nan).all()
    assert (got[~nan].view(np.uint32) == want[~nan].view(np.uint32)).all()


def test_bf16_round_sweep():
    hi = np.arange(0, 1 << 16, dtype=np.uint32) << 16
    lows = np.array([0, 1, 0x3FFF, 0x7FFF, 0x8000, 0x8001, 0xBFFF, 0xFFFF], np.uint32)
    bits = (hi[:, None] | lows[None, :]).ravel()
    x = bits.view(np.float32)
    x = np.ascontiguousarray(x[~np.isnan(x)])
    got = Z.bf16_from_f32(x)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (got == want).all(), int((got != want).sum())
    # the hand-derived edges: the largest finite value, the overflow midpoint,
    # the smallest subnormal and its half
    assert Z.bf16_from_f64_scalar((2 - 2**-7) * 2.0**127) == 0x7F7F
    assert Z.bf16_from_f64_scalar((2 - 2**-8) * 2.0**127) == 0x7F80
    assert Z.bf16_from_f64_scalar(2.0**-133) == 0x0001
    assert Z.bf16_from_f64_scalar(2.0**-134) == 0x0000  # a tie, to even
    assert Z.bf16_from_f64_scalar(1.5 * 2.0**-134) == 0x0001
    assert Z.bf16_from_f64_scalar(1 + 2**-8) == 0x3F80  # tie to even
    assert Z.bf16_from_f64_scalar(1 + 3 * 2**-8) == 0x3F82


def _bf16_grads(rng, nd, n, sigma):
    return [Z.bf16_from_f32((rng.standard_normal(n) * sigma).astype(np.float32)) for _ in range(nd)]


@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_bf16_step_matches_torch_restarted_from_bf16(wd):
    rng = np.random.default_rng(5)
    n, nd, scale = 513, 4, 8.0
    hp = Z.hyper(lr=1e-2, weight_decay=wd)
    w16 = Z.bf16_from_f32(rng.uniform(-2, 2, n).astype(np.float32))
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    tm = torch.zeros(n, dtype=torch.float64)
    tv = torch.zeros(n, dtype=torch.float64)
    t = 0
    f32 = lambda x: float(np.float32(x))  # noqa: E731
    for step in range(5):
        gs = _bf16_grads(rng, nd, n, 1e-2 * scale)
        s = Z.f32_from_bf16(gs[0])
        for g in gs[1:]:
            s = (s + Z.f32_from_bf16(g)).astype(np.float32)
        g64 = s.astype(np.float64) / scale  # scale is a power of two: exact
        p = torch.nn.Parameter(torch.from_numpy(Z.f32_from_bf16(w16).astype(np.float64)))
        opt = torch.optim.AdamW([p], lr=f32(1e-2), betas=(f32(0.9), f32(0.999)), eps=f32(1e-8),
                                weight_decay=f32(wd), foreach=False)
        p.grad = torch.from_numpy(g64)
        opt.step()  # initialises the state; replace it with the running moments and redo
        st = opt.state[p]
        p.data = torch.from_numpy(Z.f32_from_bf16(w16).astype(np.float64))
        st["exp_avg"] = tm.clone()
        st["exp_avg_sq"] = tv.clone()
        st["step"] = torch.tensor(float(t))
        opt.step()
        tm, tv = st["exp_avg"].clone(), st["exp_avg_sq"].clone()
        sk, t = Z.bf16_step(gs, w16, m, v, scale, hp, t)
        assert not sk and t == step + 1
        gmax = np.abs(g64).max()
        assert np.max(np.abs(m - tm.numpy()) / ((1 - 0.9) * gmax)) <= 1e-6
        assert np.max(np.abs(v - tv.numpy()) / np.maximum(tv.numpy(), 1e-30)) <= 1e-6
        w_new = p.detach().numpy()
        got = Z.f32_from_bf16(w16).astype(np.float64)
        # within one bfloat16 spacing of the float64 result (2^(e-7) in binade 2^e)
        spacing = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(w_new), 2.0**-126))) - 7)
        assert (np.abs(got - w_new) <= spacing).all()


def test_dropping_the_master_loses_small_updates():
    rng = np.random.default_rng(9)
    n, nd = 4096, 2
    w0 = rng.uniform(1.0, 2.0, n).astype(np.float32) * np.where(rng.random(n) < 0.5, -1, 1)
    w16 = Z.bf16_from_f32(w0)
    start = w16.copy()
    m, v = np.zeros(n, np.float32), np.zeros(n, np.float32)
    # the fp32-master step on the same parameters, as fp16 gradients
    wm = Z.f32_from_bf16(w16)
    mm, vm, p16 = np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.uint16)
    w_master0 = wm.copy()
    hp = Z.hyper(lr=1e-3)
    t = tm = 0
    for step in range(3):
        # gradients exact in both formats: 8-bit integers times 2^-10
        q = rng.integers(1, 256, size=(nd, n))
        g32 = (q * 2.0**-10).astype(np.float32)
        g32[:, :] = np.abs(g32) * np.sign(w0)  # push every weight the same way every step
        gs16 = [Z.bf16_from_f32(r) for r in g32]
        assert all((Z.f32_from_bf16(g) == r).all() for g, r in zip(gs16, g32))
        _, t = Z.bf16_step(gs16, w16, m, v, 1.0, hp, t)
        _, tm = Z.dp_step([Z.f16_from_f32(r) for r in g32], wm, mm, vm, p16, 1.0, hp, tm)
    # |lr * update| ~ 1e-3 < 2^-8 (half a spacing in [1, 2)): every update lost
    assert (w16 == start).all()
    assert (wm != w_master0).all()
    assert np.abs(wm - w_master0).max() == pytest.approx(3e-3, rel=0.05)


def test_bf16_skip_leaves_everything():
    rng = np.random.default_rng(2)
    n = 300
    w16 = Z.bf16_from_f32(rng.uniform(-1, 1, n).astype(np.float32))
    m = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    v = rng.uniform(0, 1e-6, n).astype(np.float32)
    before = (w16.copy(), m.copy(), v.copy())
    gs = _bf16_grads(rng, 3, n, 1e-3)
    gs[2][n - 1] = 0x7F80  # +inf
    sk, t = Z.bf16_step(gs, w16, m, v, 1.0, Z.hyper(), 4)
    assert sk and t == 4
    for a, b in zip((w16, m, v), before):
        assert (a.view(np.uint8) == b.view(np.uint8)).all()
