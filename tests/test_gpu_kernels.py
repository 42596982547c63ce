"""GPU parity of each kernel family against the fp64 oracle, through the C ABI.

Sizes span several tiles and a ragged tail (rows or columns that are not a
multiple of the 128 x 256 GEMM tile, or of the 64 x 64 transpose tile), and
include the degenerate cases: empty tensors, 0-D scalars, zero gradients and
rank-deficient directions.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import synth
import adamw_hybrid_optimizer_muon_b200 as ma
from gpu_helpers import (TOL_BF16, TOL_F32, bf16_round, check_muon, check_state, dev_f32, dev_grad, f32, host,
                         hp32, momentum_terms, oracle_muon)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    ma.ma_device_status(reset=True)
    yield
    assert ma.ma_device_status(reset=True) == ma.MA_OK


# ------------------------------------------------------------------------------------------ AdamW

@pytest.mark.parametrize("gdt", ["bf16", "f32"])
def test_adamw_parity_two_steps(gdt):
    sizes = [0, 1, 3, 4, 5, 1023, 8192, 8193, 65537, 300000]
    r = np.random.default_rng(100)
    P0 = [(r.standard_normal(n) * 0.02).astype(np.float32) for n in sizes]
    Pd = [dev_f32(p) for p in P0]
    Md = [torch.zeros_like(p) for p in Pd]
    Vd = [torch.zeros_like(p) for p in Pd]
    # one misaligned view exercises the scalar path
    big = dev_f32(np.zeros(5001, np.float32))
    Pd.append(big[1:])
    P0.append(np.zeros(5000, np.float32))
    Md.append(torch.zeros(5001, device="cuda")[1:])
    Vd.append(torch.zeros(5001, device="cuda")[1:])
    lr, b1, b2, eps, wd = (f32(x) for x in (0.02, 0.9, 0.95, 1e-8, 0.01))
    for step in (1, 2):
        G = [bf16_round(r.standard_normal(p.numel()) * 1e-3) for p in Pd]
        Gd = [dev_grad(g, gdt) for g in G]
        before = [(host(p), host(m), host(v)) for p, m, v in zip(Pd, Md, Vd)]
        ma.adamw_step_fused(Pd, Gd, Md, Vd, ma.adamw_hparams(lr, b1, b2, eps, wd, step))
        torch.cuda.synchronize()
        for (p0, m0, v0), g, p, m, v in zip(before, G, Pd, Md, Vd):
            rp, rm, rv = oracle.adamw_update(p0, g, m0, v0, step, lr, b1, b2, eps, wd)
            tp, tm, tv = oracle.adamw_term_magnitudes(p0, g, m0, v0, step, lr, b1, b2, eps, wd)
            check_state(host(p), rp, tp, what="param")
            check_state(host(m), rm, tm, what="exp_avg")
            check_state(host(v), rv, tv, what="exp_avg_sq")
        for g, gd in zip(G, Gd):  # gradients are preserved bit for bit
            assert np.array_equal(host(gd).astype(np.float32), g.astype(np.float32))


def test_adamw_many_tensors_multiple_launches():
    # more tensors than one parameter block holds (320): the call splits its launches
    n = 700
    r = np.random.default_rng(101)
    P = [dev_f32(r.standard_normal(37) * 0.02) for _ in range(n)]
    G = [bf16_round(r.standard_normal(37) * 1e-3) for _ in range(n)]
    M = [torch.zeros_like(p) for p in P]
    V = [torch.zeros_like(p) for p in P]
    P0 = [host(p) for p in P]
    ma.adamw_step_fused(P, [dev_grad(g, "bf16") for g in G], M, V, ma.adamw_hparams(step=1))
    torch.cuda.synchronize()
    hpv = [f32(x) for x in (0.02, 0.9, 0.95, 1e-8, 0.01)]
    for p0, g, p in zip(P0, G, P):
        rp, _, _ = oracle.adamw_update(p0, g, 0 * p0, 0 * p0, 1, *hpv)
        tp, _, _ = oracle.adamw_term_magnitudes(p0, g, 0 * p0, 0 * p0, 1, *hpv)
        check_state(host(p), rp, tp)


# ------------------------------------------------------------------------------------------ Newton-Schulz alone

def _ns_case(batch, m, n, seed):
    r = np.random.default_rng(seed)
    X = r.standard_normal((batch, m, n))
    X /= np.linalg.norm(X, axis=(1, 2), keepdims=True)  # spectral norm <= 1
    return bf16_round(X)


@pytest.mark.parametrize("m,n", [(128, 256), (256, 512), (96, 640), (384, 1024), (128, 128), (200, 328),
                                 (1280, 1280)])
@pytest.mark.parametrize("steps", [1, 5])
def test_ns_iterate_bf16_matches_oracle(m, n, steps):
    batch = 3
    X = _ns_case(batch, m, n, seed=m * 7 + n)
    Xd = dev_grad(X, "bf16").reshape(batch, m, n)
    out = torch.empty_like(Xd)
    ws = torch.empty(ma.ns_iterate_workspace_bytes(batch, m, n), dtype=torch.uint8, device="cuda")
    ma.ns_iterate_bf16(Xd, out, [oracle.CUBIC], steps, ws)
    torch.cuda.synchronize()
    got = host(out)
    for b in range(batch):
        ref = oracle.ns_iterate(X[b].astype(np.float64), [oracle.CUBIC], steps)
        err = np.linalg.norm(got[b] - ref) / np.linalg.norm(ref)
        assert err <= TOL_BF16, f"batch {b}: relative error {err:.3e}"


@pytest.mark.parametrize("m,n", [(128, 256), (160, 392)])
def test_ns_iterate_bf16_quintic_schedule(m, n):
    # a per-iteration schedule with c != 0 exercises the A^2 GEMM
    coeffs = [(2.0, -1.5, 0.5), (1.5, -0.5, 0.0), (1.875, -1.25, 0.375)]
    X = _ns_case(2, m, n, seed=5)
    Xd = dev_grad(X, "bf16").reshape(2, m, n)
    out = torch.empty_like(Xd)
    ws = torch.empty(ma.ns_iterate_workspace_bytes(2, m, n), dtype=torch.uint8, device="cuda")
    ma.ns_iterate_bf16(Xd, out, coeffs, 3, ws)
    torch.cuda.synchronize()
    got = host(out)
    for b in range(2):
        ref = oracle.ns_iterate(X[b].astype(np.float64), coeffs, 3)
        assert np.linalg.norm(got[b] - ref) / np.linalg.norm(ref) <= TOL_BF16


# ------------------------------------------------------------------------------------------ Muon step

MUON_CASES = [
    # (R, C, heads, nesterov, scale_mode, coeffs)
    ((256, 512), 1, True, 0, (oracle.CUBIC,)),
    ((512, 256), 1, True, 0, (oracle.CUBIC,)),      # tall: transpose path, s = sqrt(2)
    ((200, 136), 1, False, 1, (oracle.CUBIC,)),     # ragged tall, plain momentum
    ((136, 392), 1, True, 2, (oracle.CUBIC,)),      # ragged wide
    ((256, 512), 4, True, 0, (oracle.CUBIC,)),      # per-head, wide slices 64 x 512
    ((512, 128), 2, True, 0, (oracle.CUBIC,)),      # per-head, tall slices 256 x 128
    ((128, 384), 1, True, 0, ((2.0, -1.5, 0.5), (1.5, -0.5, 0.0))),  # c != 0 schedule
    ((96, 200), 1, True, 0, (oracle.CUBIC,)),       # ragged, m < 128 (single-CTA tiles)
    ((384, 120), 1, True, 0, ((2.0, -1.5, 0.5), (1.5, -0.5, 0.0))),  # tall, m = 120, c != 0
]


def _muon_run(shape, heads, nesterov, mode, coeffs, precision, gdt, batch=2, steps=2, seed=0, cautious=False,
              wd=0.01):
    R, C = shape
    hp = hp32(synth.MuonHP(nesterov=nesterov, scale_mode=mode, heads=heads, precision=precision,
                           coeffs=tuple(coeffs), ns_steps=len(coeffs) if len(coeffs) > 1 else 5, cautious=cautious,
                           weight_decay=wd))
    r = np.random.default_rng(seed)
    W = [(r.standard_normal(shape) * 0.02).astype(np.float32) for _ in range(batch)]
    Wd = [dev_f32(w) for w in W]
    Md = [torch.zeros(shape, device="cuda") for _ in range(batch)]
    mhp = ma.muon_hparams(hp.lr, hp.beta, hp.weight_decay, hp.eps, hp.nesterov, hp.ns_steps, hp.coeffs,
                          hp.scale_mode, hp.heads, hp.precision, hp.cautious)
    ws = torch.empty(ma.muon_workspace_bytes(batch, R, C, mhp), dtype=torch.uint8, device="cuda")
    errs = []
    for step in range(steps):
        G = [bf16_round(r.standard_normal(shape) * 1e-3) for _ in range(batch)]
        Gd = [dev_grad(g, gdt) for g in G]
        before = [(host(w), host(m)) for w, m in zip(Wd, Md)]
        ma.muon_step_batched(Wd, Gd, Md, mhp, ws)
        torch.cuda.synchronize()
        for (w0, m0), g, w, m in zip(before, G, Wd, Md):
            rw, rm = oracle_muon(w0, g, m0, hp)
            check_state(host(m), rm, momentum_terms(m0, g, hp.beta), what="momentum")
            errs.append(check_muon(w0, host(w), rw, hp.lr, hp.weight_decay,
                                   TOL_F32 if precision else TOL_BF16))
        for g, gd in zip(G, Gd):
            assert np.array_equal(host(gd).astype(np.float32), g.astype(np.float32))
    return errs


@pytest.mark.parametrize("case", MUON_CASES, ids=lambda c: f"{c[0][0]}x{c[0][1]}h{c[1]}")
def test_muon_fp32_mode_parity(case):
    _muon_run(*case, precision=1, gdt="f32")


@pytest.mark.parametrize("case", MUON_CASES, ids=lambda c: f"{c[0][0]}x{c[0][1]}h{c[1]}")
@pytest.mark.parametrize("gdt", ["bf16", "f32"])
def test_muon_bf16_parity(case, gdt):
    _muon_run(*case, precision=0, gdt=gdt)


@pytest.mark.parametrize("shape", [(256, 512), (512, 256), (200, 136)])
@pytest.mark.parametrize("precision", [0, 1])
def test_muon_cautious_decay(shape, precision):
    # The decay mask (O*W > 0) is decided in floating point, so where O is near
    # zero the GPU and the fp64 oracle may decide differently. The test reads
    # the GPU's decision back, requires it to match the oracle wherever |O| is
    # not small, and checks values under the GPU's own decision. A large decay
    # makes the two candidate values of every element far apart.
    R, C = shape
    lr, beta, wd, eps = f32(0.02), f32(0.95), f32(5.0), f32(1e-7)
    r = np.random.default_rng(40)
    W0 = (r.standard_normal(shape) * 0.02).astype(np.float32).astype(np.float64)
    g = bf16_round(r.standard_normal(shape) * 1e-3)
    hp = ma.muon_hparams(lr=lr, beta=beta, weight_decay=wd, eps=eps, precision=precision, cautious=True)
    Wd, Md = [dev_f32(W0)], [torch.zeros(shape, device="cuda")]
    ws = torch.empty(ma.muon_workspace_bytes(1, R, C, hp), dtype=torch.uint8, device="cuda")
    ma.muon_step_batched(Wd, [dev_grad(g, "bf16")], Md, hp, ws)
    torch.cuda.synchronize()
    got = host(Wd[0])
    W_nodecay, _ = oracle.muon_update(W0, g, np.zeros(shape), lr, beta, 0.0, eps=eps)
    O = (W0 - W_nodecay) / lr                       # scaled orthogonalised update
    decayed = (1 - lr * wd) * W0 - lr * O
    kept = W0 - lr * O
    gpu_mask = np.abs(got - decayed) < np.abs(got - kept)
    ref_mask = O * W0 > 0
    # the decision is clear where neither factor is near zero; where W0 is tiny
    # the two candidates are closer than the update's rounding and either is fine
    clear = (np.abs(O) > 0.05 * np.sqrt(np.mean(O * O))) & (np.abs(W0) > 0.05 * np.sqrt(np.mean(W0 * W0)))
    assert np.array_equal(gpu_mask[clear], ref_mask[clear])
    check_muon(W0, got, np.where(gpu_mask, decayed, kept), lr, wd, TOL_F32 if precision else TOL_BF16)


@pytest.mark.parametrize("precision", [0, 1])
def test_muon_zero_gradient_only_decays(precision):
    shape = (128, 256)
    W0 = (np.random.default_rng(3).standard_normal(shape) * 0.02).astype(np.float32)
    Wd = [dev_f32(W0)]
    Md = [torch.zeros(shape, device="cuda")]
    Gd = [torch.zeros(shape, device="cuda", dtype=torch.bfloat16)]
    hp = ma.muon_hparams(precision=precision)
    ws = torch.empty(ma.muon_workspace_bytes(1, *shape, hp), dtype=torch.uint8, device="cuda")
    ma.muon_step_batched(Wd, Gd, Md, hp, ws)
    torch.cuda.synchronize()
    # one fp32 rounding of the decay factor and one of the product
    assert np.allclose(host(Wd[0]), W0.astype(np.float64) * (1 - f32(0.02) * f32(0.01)), rtol=2.5e-7, atol=0)


def test_muon_rank_one_direction_is_kept():
    # a rank-1 gradient is not zeroed: after normalisation it is a fixed point of the cubic
    R, C = 128, 256
    r = np.random.default_rng(4)
    g = bf16_round(np.outer(r.standard_normal(R), r.standard_normal(C)) * 1e-3)
    W0 = np.zeros((R, C), np.float32)
    Wd, Md = [dev_f32(W0)], [torch.zeros((R, C), device="cuda")]
    hp = ma.muon_hparams(precision=0)
    ws = torch.empty(ma.muon_workspace_bytes(1, R, C, hp), dtype=torch.uint8, device="cuda")
    ma.muon_step_batched(Wd, [dev_grad(g, "bf16")], Md, hp, ws)
    torch.cuda.synchronize()
    got = host(Wd[0])
    ref, _ = oracle.muon_update(W0, g, np.zeros_like(g), f32(0.02), f32(0.95), f32(0.01), eps=f32(1e-7))
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < TOL_BF16
    assert np.linalg.norm(ref) == pytest.approx(0.02, rel=1e-3)  # ||lr * O||_F = lr * 1


def test_failed_call_changes_nothing_and_determinism():
    shape = (256, 512)
    r = np.random.default_rng(5)
    W0 = (r.standard_normal(shape) * 0.02).astype(np.float32)
    g = bf16_round(r.standard_normal(shape) * 1e-3)
    hp = ma.muon_hparams()
    need = ma.muon_workspace_bytes(1, *shape, hp)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    Wd, Md, Gd = [dev_f32(W0)], [torch.zeros(shape, device="cuda")], [dev_grad(g, "bf16")]
    with pytest.raises(ma.MAError) as e:
        ma.muon_step_batched(Wd, Gd, Md, hp, ws, ws_bytes=need - 1)
    assert e.value.code == ma.MA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert np.array_equal(host(Wd[0]), W0.astype(np.float64)) and float(Md[0].abs().sum()) == 0.0
    outs = []
    for _ in range(2):
        W2, M2 = [dev_f32(W0)], [torch.zeros(shape, device="cuda")]
        ma.muon_step_batched(W2, Gd, M2, hp, ws)
        ma.muon_step_batched(W2, Gd, M2, hp, ws)
        torch.cuda.synchronize()
        outs.append((W2[0].clone(), M2[0].clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_bounded_wait_times_out_and_context_survives():
    ma.ma_selftest_wait_timeout(20_000_000)  # 20 ms; nothing ever completes the barrier
    assert ma.ma_device_status(reset=True) == ma.MA_ERR_TIMEOUT
    assert ma.ma_device_status(reset=True) == ma.MA_OK
    # the context is still usable afterwards
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0
    _muon_run((128, 256), 1, True, 0, (oracle.CUBIC,), precision=0, gdt="bf16", batch=1, steps=1)


@pytest.mark.parametrize("heads", [1, 32])
def test_newton_schulz_wait_timeout_winds_down_and_context_survives(heads):
    """A wait limit far below one tile's main loop makes the bounded waits
    inside real Newton-Schulz launches run out: 4096 x 4096 matrices on the
    CTA-pair kernel (heads = 1) and their 128-row head slices on the
    single-CTA kernel (heads = 32). Every launch of the step must record
    MA_ERR_TIMEOUT, wind down (the leader drains the issued MMAs and the bulk
    loads in flight, then both CTAs release TMEM) and return; with the default
    limit back, ordinary steps on the same context, on both kernels, match the
    oracle."""
    shape, batch = (4096, 4096), 2
    hp = ma.muon_hparams(heads=heads)
    W = [torch.zeros(shape, device="cuda") for _ in range(batch)]
    M = [torch.zeros(shape, device="cuda") for _ in range(batch)]
    g = torch.Generator(device="cuda").manual_seed(3)
    G = [(torch.randn(shape, device="cuda", generator=g) * 1e-3).bfloat16() for _ in range(batch)]
    ws = torch.empty(ma.muon_workspace_bytes(batch, *shape, hp), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    ma.ma_device_status(reset=True)
    try:
        ma.ma_set_wait_limit_ns(2_000)  # 2 us: a 256 x 256 tile's main loop takes tens of microseconds
        ma.muon_step_batched(W, G, M, hp, ws)
        torch.cuda.synchronize()
    finally:
        ma.ma_set_wait_limit_ns(2_000_000_000)  # the library's default
    assert ma.ma_device_status(reset=True) == ma.MA_ERR_TIMEOUT
    assert ma.ma_device_status(reset=True) == ma.MA_OK
    # the context, the kernels' TMEM and the workspace are usable again
    _muon_run((512, 1024), 1, True, 0, (oracle.CUBIC,), precision=0, gdt="bf16", batch=2, steps=1)
    _muon_run((2048, 128), 4, True, 0, (oracle.CUBIC,), precision=0, gdt="bf16", batch=1, steps=1)
