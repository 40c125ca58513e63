"""Checkpoint / resume through zero_set_state, and the PyTorch-facing
ZeroAdam object, on the GPU against the oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200 import synth as S

from gpu_common import compare_f16, compare_f32, host_f32, host_u16, hyper

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

from test_gpu_parity import VARIANTS, Case  # noqa: E402


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("stage", [1, 3])
def test_resume_continues_bit_identically(stage, variant):
    nd = 4
    tensors = [(8 * nd * 300, 0), (1001, 1), (8 * nd * 700, 1)] if stage == 3 else None
    psi = sum(n for n, _ in tensors) if tensors else 50_003
    a = Case(psi, nd, stage, variant, tensors=tensors, hp=dict(weight_decay=0.01))
    for s in range(3):
        a.step(a.grads(s))
    a.check("after 3 steps")
    # save: the live arrays and t
    wp, mp, vp, t = A.zero_current_state(a.h)
    n = a.L.state_elems
    base = a.ws.ptr()
    saved = [a.ws.full[a.ws.g + p - base: a.ws.g + p - base + 4 * n].view(torch.float32).clone()
             for p in (wp, mp, vp)]
    # a fresh handle with different initial weights, restored from the save
    b = Case(psi, nd, stage, variant, tensors=tensors, hp=dict(weight_decay=0.01), seed=7)
    A.zero_set_state(b.h, saved[0].data_ptr(), saved[1].data_ptr(), saved[2].data_ptr(), t, b.stream)
    for s in range(3, 5):
        gs = a.grads(s)
        a.step(gs)
        b.upload(gs)
        assert A.zero_step(b.h, [g.data_ptr() for g in b.g_dev], b.loss_scale, hyper(**b.hp),
                           b.stream) == A.ZERO_OK
    a.check("after 5 steps")
    wa, ma, va, ta = A.zero_current_state(a.h)
    wb, mb, vb, tb = A.zero_current_state(b.h)
    assert ta == tb == 5
    for pa, pb, name in ((wa, wb, "master"), (ma, mb, "m"), (va, vb, "v")):
        ga = host_f32(a.ws.full[a.ws.g + pa - a.ws.ptr(): a.ws.g + pa - a.ws.ptr() + 4 * n].view(torch.float32))
        gb = host_f32(b.ws.full[b.ws.g + pb - b.ws.ptr(): b.ws.g + pb - b.ws.ptr() + 4 * n].view(torch.float32))
        compare_f32(gb, ga, f"resumed {name}")
    if stage <= 2:
        for ra, rb in zip(a.bufs, b.bufs):
            compare_f16(rb.bits(), ra.bits(), "resumed replica")
    else:
        compare_f16(b.ws.u16(b.L.off_shard16, n), a.ws.u16(a.L.off_shard16, n), "resumed shards")
    a.close()
    b.close()


def test_zero_adam_object_matches_oracle_and_round_trips():
    from zero_partitioned_mixed_02_b200 import ZeroAdam
    psi, nd = 30_011, 4
    w0 = S.host_f32(psi, 0, S.key(0, S.STREAM_MASTER, 0, 0), S.uniform(-0.1, 0.1))
    reps = [torch.zeros(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    opt = ZeroAdam(psi, nd, 2, torch.from_numpy(w0.copy()).cuda(), reps)
    w, m, v = w0.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32)
    p16 = np.zeros(psi, np.uint16)
    t = 0
    grads = [torch.empty(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    for s in range(3):
        gs = [S.host_f16_bits(psi, 0, S.key(0, S.STREAM_GRAD, s, k), S.normal(1e-3, 512.0))
              for k in range(nd)]
        for g, x in zip(grads, gs):
            g.copy_(torch.from_numpy(x.view(np.int16)))
        assert opt.step(grads, 512.0, weight_decay=0.01) is False
        sk, t = Z.dp_step(gs, w, m, v, p16, 512.0, Z.hyper(weight_decay=0.01), t)
    gw, gm, gv = opt.state()
    compare_f32(host_f32(gw), w, "master")
    compare_f32(host_f32(gm), m, "m")
    compare_f32(host_f32(gv), v, "v")
    for r in reps:
        compare_f16(host_u16(r), p16, "replica")
    sd = opt.state_dict()
    assert sd["t"] == 3
    opt.load_state_dict(sd)  # restoring the live state is a no-op
    gw2, _, _ = opt.state()
    compare_f32(host_f32(gw2), w, "master after load")
    opt.close()


@pytest.mark.parametrize("variant", [A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_FUSED_TMA])
def test_prefetched_gathers_match_oracle(variant):
    from zero_partitioned_mixed_02_b200.prefetch import LayerPrefetcher
    nd = 4
    sizes = [8 * nd * 900, 8 * nd * 40, 8 * nd * 1500, 8 * nd * 300, 777]
    units = [0, 1, 1, 2, 2]
    c = Case(sum(sizes), nd, 3, variant, tensors=list(zip(sizes, units)))
    c.step(c.grads(0))
    pf = LayerPrefetcher(c.h, c.L, torch.cuda.current_stream())
    assert pf.peak_bytes == 2 * c.L.transient_bytes
    order = [0, 1, 2, 2, 1, 0]  # forward, then backward
    seen = []
    for u, w in pf.walk(order, unit_numel=lambda u: A.zero_unit_range(c.cfg, u)[1]):
        want = Z.zero3_gather(c.numel, c.units, nd, u, c.p_sh)
        compare_f16(host_u16(w), want, f"prefetched unit {u}")
        seen.append(u)
    assert seen == order
    c.close()


def test_offload_object_equals_device_object():
    """ZeroOffloadAdam (host state, host Adam) and ZeroAdam (device) on the same
    inputs: identical masters, moments and fp16 replicas after three steps and
    a skipped one; state_dict / load_state_dict round trip on the host."""
    from zero_partitioned_mixed_02_b200 import ZeroAdam, ZeroOffloadAdam
    psi, nd = 40_003, 4
    tensors = [(25_000, 0), (15_003, 0, A.ZERO_TENSOR_NO_DECAY)]
    w0 = S.host_f32(psi, 0, S.key(2, S.STREAM_MASTER, 0, 0), S.uniform(-0.5, 0.5))
    reps_d = [torch.zeros(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    reps_o = [torch.zeros(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    dev = ZeroAdam(psi, nd, 2, torch.from_numpy(w0.copy()).cuda(), reps_d, tensors=tensors)
    off = ZeroOffloadAdam(psi, nd, 2, w0, reps_o, tensors=tensors, chunk_elems=8192, threads=3)
    grads = [torch.empty(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    for s in range(4):
        gs = [S.host_f16_bits(psi, 0, S.key(2, S.STREAM_GRAD, s, k), S.normal(1e-3, 256.0)) for k in range(nd)]
        if s == 2:
            gs[1][77] = 0x7C00
        for g, x in zip(grads, gs):
            g.copy_(torch.from_numpy(x.view(np.int16)))
        assert dev.step(grads, 256.0, weight_decay=0.05) == off.step(grads, 256.0, weight_decay=0.05) == (s == 2)
    torch.cuda.synchronize()
    for a, b, what in zip(dev.state(), off.state(), ("master", "m", "v")):
        compare_f32(b.numpy(), host_f32(a), what)
    for r_d, r_o in zip(reps_d, reps_o):
        compare_f16(host_u16(r_o), host_u16(r_d), "replica")
    assert off.t == dev.t == 3
    sd = off.state_dict()
    off.load_state_dict(sd)
    torch.cuda.synchronize()
    compare_f32(off.state()[0].numpy(), host_f32(dev.state()[0]), "master after load")
    dev.close()
    off.close()


def test_zero_adam_bf16_object():
    """ZeroAdam with precision=bf16 and the default variant runs the fused TMA
    step (stage 2, Nd = 4: the last replica is its roll-back copy); its state
    has no master; three steps equal the oracle. Where no second replica
    exists (one rank) the default becomes the two-pass TMA step."""
    from zero_partitioned_mixed_02_b200 import ZeroAdam
    psi, nd = 20_000, 4
    w0 = S.host_f32(psi, 0, S.key(3, S.STREAM_MASTER, 0, 0), S.uniform(-1.0, 1.0))
    reps = [torch.zeros(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    opt = ZeroAdam(psi, nd, 2, torch.from_numpy(w0.copy()).cuda(), reps, precision=A.ZERO_PRECISION_BF16)
    assert opt.cfg.c.variant == A.ZERO_VARIANT_FUSED_TMA
    one = ZeroAdam(64, 1, 2, torch.zeros(64, dtype=torch.float32, device="cuda"),
                   [torch.zeros(64, dtype=torch.int16, device="cuda")], precision=A.ZERO_PRECISION_BF16)
    assert one.cfg.c.variant == A.ZERO_VARIANT_TWO_PASS_TMA
    one.close()
    w16 = Z.bf16_from_f32(w0)
    m, v, t = np.zeros(psi, np.float32), np.zeros(psi, np.float32), 0
    grads = [torch.empty(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    for s in range(3):
        gs = [Z.bf16_from_f32(S.host_f32(psi, 0, S.key(3, S.STREAM_GRAD, s, k), S.normal(1e-3, 1.0)))
              for k in range(nd)]
        for g, x in zip(grads, gs):
            g.copy_(torch.from_numpy(x.view(np.int16)))
        assert opt.step(grads, 1.0, weight_decay=0.01) is False
        _, t = Z.bf16_step(gs, w16, m, v, 1.0, Z.hyper(weight_decay=0.01), t)
    gw, gm, gv = opt.state()
    assert gw is None
    compare_f32(host_f32(gm), m, "m")
    compare_f32(host_f32(gv), v, "v")
    for r in reps:
        compare_f16(host_u16(r), w16, "bf16 replica")
    sd = opt.state_dict()
    assert sd["master"] is None and sd["t"] == 3
    opt.load_state_dict(sd)
    opt.close()


@pytest.mark.parametrize("precision", [A.ZERO_PRECISION_FP16, A.ZERO_PRECISION_BF16])
def test_partial_update_is_reported_and_restored(precision):
    """The two-pass TMA step updates in place. A bounded wait of its update
    pass that gives up (a tile left unarmed by the test hook: no fault) leaves
    the state partly updated; ZeroAdam raises ZeroPartialUpdateError, the state
    saved before the step restores master/m/v, t and the parameters exactly,
    and the same step run again equals the oracle's."""
    from zero_partitioned_mixed_02_b200 import ZeroAdam
    from zero_partitioned_mixed_02_b200.optimizer import ZeroPartialUpdateError
    bf16 = precision == A.ZERO_PRECISION_BF16
    psi, nd = 200_000, 4
    w0 = S.host_f32(psi, 0, S.key(5, S.STREAM_MASTER, 0, 0), S.uniform(-1.0, 1.0))
    reps = [torch.zeros(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    opt = ZeroAdam(psi, nd, 2, torch.from_numpy(w0.copy()).cuda(), reps,
                   variant=A.ZERO_VARIANT_TWO_PASS_TMA, precision=precision)
    assert A.zero_uses_tma(opt.h)
    hp = Z.hyper(weight_decay=0.01)
    if bf16:
        w16, w = Z.bf16_from_f32(w0), None
    else:
        w, w16 = w0.copy(), Z.f16_from_f32(w0)
    m, v, t = np.zeros(psi, np.float32), np.zeros(psi, np.float32), 0
    grads = [torch.empty(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]

    def grads_of(s):
        if bf16:
            gs = [Z.bf16_from_f32(S.host_f32(psi, 0, S.key(5, S.STREAM_GRAD, s, k), S.normal(1e-3, 1.0)))
                  for k in range(nd)]
        else:
            gs = [S.host_f16_bits(psi, 0, S.key(5, S.STREAM_GRAD, s, k), S.normal(1e-3, 1024.0))
                  for k in range(nd)]
        for g, x in zip(grads, gs):
            g.copy_(torch.from_numpy(x.view(np.int16)))
        return gs

    scale = 1.0 if bf16 else 1024.0

    def oracle_step(gs):
        nonlocal t
        if bf16:
            _, t = Z.bf16_step(gs, w16, m, v, scale, hp, t)
        else:
            _, t = Z.dp_step(gs, w, m, v, w16, scale, hp, t)

    def check(what):
        gw, gm, gv = opt.state()
        if not bf16:
            compare_f32(host_f32(gw), w, f"master, {what}")
        compare_f32(host_f32(gm), m, f"m, {what}")
        compare_f32(host_f32(gv), v, f"v, {what}")
        for r in reps:
            compare_f16(host_u16(r), w16, f"parameters, {what}")
        assert opt.t == t

    gs = grads_of(0)
    assert opt.step(grads, scale, weight_decay=0.01) is False
    oracle_step(gs)
    check("after step 0")
    sd = opt.state_dict()

    gs = grads_of(1)
    A.zero_test_hold_update_tile(opt.h, 3, 1 << 14)
    with pytest.raises(ZeroPartialUpdateError) as ei:
        opt.step(grads, scale, weight_decay=0.01)
    assert ei.value.code == A.ZERO_ERR_PARTIAL
    assert opt.t == 1  # t did not advance
    _, gm, _ = opt.state()
    changed = int((host_f32(gm).view(np.uint32) != m.view(np.uint32)).sum())
    assert 0 < changed < psi  # the other tiles were updated in place, the held one not

    opt.load_state_dict(sd)
    check("restored")
    assert opt.step(grads, scale, weight_decay=0.01) is False
    oracle_step(gs)
    check("after the step run again")
    opt.close()


def test_update_hold_hook_refuses_other_variants():
    psi, nd = 10_000, 2
    for variant in (A.ZERO_VARIANT_FUSED_TMA, A.ZERO_VARIANT_TWO_PASS):
        c = Case(psi, nd, 2, variant)
        with pytest.raises(A.ZeroError) as ei:
            A.zero_test_hold_update_tile(c.h, 0, 1 << 10)
        assert ei.value.code == A.ZERO_ERR_ARG
        c.close()
