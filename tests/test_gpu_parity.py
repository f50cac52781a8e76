"""GPU parity: every libmhc entry point against the fp64 oracle, element by
element, on the same seeded inputs.

Tolerances (norm-wise, per output tensor: max|gpu - ref| / max|ref|):
  fp32 I/O  1e-5
  bf16 I/O  2e-2   (bf16 inputs widen exactly on both sides; the gap is fp32
                    accumulation, bf16 rounding of the outputs and, for the
                    tensor-core projection, bf16 operands)
Standalone Sinkhorn and depth gain (fp32): 1e-5.
"""
import numpy as np
import pytest
import torch

from conftest import assert_close, close_errs, rel_err

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}


@pytest.fixture(scope="module")
def mhc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from manifold_constrained_hyper_token_b200 import build
    build.build()
    import manifold_constrained_hyper_token_b200 as m
    return m


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _inputs(T, n, C, dtype, seed=0, alpha=0.01):
    from manifold_constrained_hyper_token_b200 import synth
    d = synth.layer_inputs(T, n, C, seed=seed, dtype=dtype, backward=True)
    d["alpha"] = torch.tensor([alpha], dtype=torch.float32)
    return d


def _dev(d):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in d.items()}


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


# --------------------------------------------------------------- Sinkhorn
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("iters", [0, 1, 20])
@pytest.mark.parametrize("B", [1, 1000, 1003])
def test_sinkhorn_parity(mhc, oracle_mod, n, iters, B):
    from manifold_constrained_hyper_token_b200 import synth
    lg = synth.sinkhorn_logits(B, n, seed=n * 7 + iters)
    st = _status()
    out = mhc.mhc_sinkhorn_knopp(lg.cuda(), iters, dev_status=st)
    ref = oracle_mod.sinkhorn(lg, iters)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close(_np(out), ref, 1e-5)


@pytest.mark.parametrize("n", [4, 8, 16])
def test_sinkhorn_full_batch(mhc, oracle_mod, n):
    """2^22 matrices, logits N(0, 2), 20 iterations: sampled parity plus the
    column sums of every matrix (exact after the closing column pass)."""
    from manifold_constrained_hyper_token_b200 import synth
    B = 1 << 22
    lg = synth.sinkhorn_logits(B, n, seed=100 + n)
    out = mhc.mhc_sinkhorn_knopp(lg.cuda(), 20)
    idx = synth.token_sample(B, 2048, seed=n)
    ref = oracle_mod.sinkhorn(lg[idx], 20)
    assert_close(_np(out[idx.cuda()]), ref, 1e-5)
    assert float(out.min()) >= 0.0
    assert float((out.sum(dim=1) - 1).abs().max()) < 1e-5
    del out


def test_sinkhorn_nonfinite_status(mhc):
    lg = torch.zeros(64, 4, 4)
    lg[5, 1, 2] = float("inf")
    st = _status()
    mhc.mhc_sinkhorn_knopp(lg.cuda(), 20, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4


# ------------------------------------------------------------ depth gain
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("L", [0, 1, 64])
def test_depth_amax_parity(mhc, oracle_mod, n, L):
    from manifold_constrained_hyper_token_b200 import synth
    T = 301
    lg = synth.sinkhorn_logits(T * max(L, 1), n, seed=200 + n + L)
    H = oracle_mod.sinkhorn(lg, 20).reshape(T, max(L, 1), n, n)[:, :L]
    Ht = torch.from_numpy(np.ascontiguousarray(H)).float()
    gf, gb = mhc.mhc_depth_amax(Ht.cuda() if L > 0 else torch.empty(T, 0, n, n, device="cuda"))
    rf, rb = oracle_mod.depth_amax(Ht)
    assert_close(_np(gf), rf, 1e-5)
    assert_close(_np(gb), rb, 1e-5)


def test_depth_amax_non_doubly_stochastic(mhc, oracle_mod):
    H = torch.randn(257, 8, 4, 4, generator=torch.Generator().manual_seed(5)) * 0.7
    gf, gb = mhc.mhc_depth_amax(H.cuda())
    rf, rb = oracle_mod.depth_amax(H)
    assert_close(_np(gf), rf, 1e-5)
    assert_close(_np(gb), rb, 1e-5)


def test_depth_amax_sinkhorn_batch(mhc, oracle_mod):
    """2^16 tokens x 64 layers of 20-iteration Sinkhorn outputs (N(0,2) logits)."""
    from manifold_constrained_hyper_token_b200 import synth
    T, L, n = 1 << 16, 64, 4
    lg = synth.sinkhorn_logits(T * L, n, seed=300)
    H = mhc.mhc_sinkhorn_knopp(lg.cuda(), 20).view(T, L, n, n)
    gf, gb = mhc.mhc_depth_amax(H)
    idx = synth.token_sample(T, 1024, seed=3)
    rf, rb = oracle_mod.depth_amax(H[idx.cuda()].cpu())
    assert_close(_np(gf[idx.cuda()]), rf, 1e-5)
    assert_close(_np(gb[idx.cuda()]), rb, 1e-5)
    print(f"Amax gain over {T} tokens x {L} layers: fwd max {float(gf.max()):.6f} "
          f"bwd max {float(gb.max()):.6f}")


# ----------------------------------------------------------------- post
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("T,C", [(1, 8), (67, 24), (130, 256)])
def test_post_parity(mhc, oracle_mod, dtype, n, T, C):
    d = _inputs(T, n, C, dtype, seed=T + C)
    g = torch.Generator().manual_seed(T * 3 + n)
    Hpost = torch.rand(T, n, generator=g) * 2
    Hres = torch.rand(T, n, n, generator=g)
    out = mhc.mhc_post(d["x"].cuda(), d["f_out"].cuda(), Hpost.cuda(), Hres.cuda())
    ref = oracle_mod.post(d["x"], d["f_out"], Hpost, Hres)
    assert_close(_np(out), ref, TOL[dtype])


def test_post_standard_residual_exact(mhc):
    x = torch.randn(33, 1, 64)
    f = torch.randn(33, 64)
    out = mhc.mhc_post(x.cuda(), f.cuda(), torch.ones(33, 1).cuda(), torch.ones(33, 1, 1).cuda())
    assert torch.equal(out.cpu()[:, 0], x[:, 0] + f)


# ------------------------------------------------------------------ pre
def _check_pre(mhc, oracle_mod, d, iters, dtype, eps=1e-6):
    dd = _dev(d)
    st = _status()
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"], t_max=iters,
                                          eps=eps, dev_status=st)
    ref = oracle_mod.pre(d["x"], d["phi"], d["b"], float(d["alpha"][0]), iters=iters, eps=eps)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    tol = TOL[dtype]
    errs = {}
    for k, got in (("H_pre", Hpre), ("H_post", Hpost), ("H_res", Hres), ("h_in", h_in)):
        errs[k] = max(assert_close(_np(got), ref[k], tol, k))
    return errs


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("T,C", [(1, 8), (65, 24), (130, 256)])
@pytest.mark.parametrize("iters", [0, 1, 20])
def test_pre_parity(mhc, oracle_mod, dtype, n, T, C, iters):
    d = _inputs(T, n, C, dtype, seed=T * 11 + C + n)
    _check_pre(mhc, oracle_mod, d, iters, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_pre_large_alpha_parity(mhc, oracle_mod, dtype):
    """alpha = 1 so that the projection, not the bias, dominates the logits."""
    d = _inputs(200, 4, 512, dtype, seed=9, alpha=1.0)
    errs = _check_pre(mhc, oracle_mod, d, 20, dtype)
    if dtype == torch.bfloat16:
        # the gates and Sinkhorn run in fp32 on an fp32 projection: far inside 2e-2
        assert max(errs["H_pre"], errs["H_post"], errs["H_res"]) < 1e-4, errs


def test_pre_nonfinite_status(mhc):
    d = _dev(_inputs(70, 4, 64, torch.bfloat16, seed=1))
    d["x"][3, 1, 5] = float("nan")
    st = _status()
    mhc.mhc_pre(d["x"], d["phi"], d["b"], d["alpha"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4


def test_tiny_forward_with_linear_F(mhc, oracle_mod):
    """T=64, n=4, C=256 fp32, F = fixed random linear map W [256, 256]."""
    from manifold_constrained_hyper_token_b200 import synth
    d = synth.tiny_forward(0)
    dd = _dev(d)
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"])
    f_out = (h_in.double() @ dd["W"].double().T).float().contiguous()
    x_next = mhc.mhc_post(dd["x"], f_out, Hpost, Hres)
    ref = oracle_mod.pre(d["x"], d["phi"], d["b"], float(d["alpha"][0]))
    f_ref = ref["h_in"] @ _np(d["W"]).T
    xn_ref = oracle_mod.post(d["x"], f_ref, ref["H_post"], ref["H_res"])
    assert_close(_np(h_in), ref["h_in"], 1e-5)
    assert_close(_np(f_out), f_ref, 1e-5)
    assert_close(_np(x_next), xn_ref, 1e-5)


# -------------------------------------------------------------- backward
def _alpha_err(ga, ref_total, per_token):
    """grad_alpha = sum_t alpha-scaled dz_t . y_t / r_t is a scalar sum over tokens whose
    terms cancel: in these cases |sum_t term_t| is up to 300 times smaller than
    sum_t |term_t| (n = 1, T = 130, C = 256, t_max = 1).  The rounding error of a
    floating-point sum is bounded in proportion to sum_t |term_t| (the forward error
    bound of recursive summation), not to |sum|, so the tolerance is applied to
    |gpu - ref| / max(|ref|, sum_t |term_t|)."""
    scale = max(abs(ref_total), float(np.sum(np.abs(per_token))))
    return abs(float(_np(ga).reshape(-1)[0]) - ref_total) / scale if scale > 0 else 0.0


def _alpha_terms(oracle_mod, call, T):
    """Per-token grad_alpha terms from the oracle, one token per call."""
    return np.array([call(slice(t, t + 1))["grad_alpha"] for t in range(T)])


def _check_bwd(mhc, oracle_mod, d, iters, dtype, eps=1e-6, idx=None, chunk=None):
    dd = _dev(d)
    st = _status()
    gx, gphi, gb, ga, gf = mhc.mhc_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"], dd["f_out"],
                                            dd["grad_x_next"], dd["grad_h_in"], t_max=iters,
                                            eps=eps, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle_mod.backward(d["x"], d["phi"], d["b"], float(d["alpha"][0]), d["f_out"],
                              d["grad_x_next"], d["grad_h_in"], iters=iters, eps=eps, chunk=chunk)
    tol = TOL[dtype]
    errs = {}
    for k, got in (("grad_x", gx), ("grad_f_out", gf), ("grad_phi", gphi), ("grad_b", gb)):
        errs[k] = max(assert_close(_np(got), ref[k], tol, k))
    a = float(d["alpha"][0])
    terms = _alpha_terms(oracle_mod, lambda sl: oracle_mod.backward(
        d["x"][sl], d["phi"], d["b"], a, d["f_out"][sl], d["grad_x_next"][sl],
        d["grad_h_in"][sl], iters=iters, eps=eps), d["x"].shape[0])
    errs["grad_alpha"] = _alpha_err(ga, ref["grad_alpha"], terms)
    assert errs["grad_alpha"] < tol, errs
    return errs, (gx, gphi, gb, ga, gf)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("T,C", [(1, 8), (65, 24), (130, 256)])
@pytest.mark.parametrize("iters", [0, 1, 20])
def test_backward_parity(mhc, oracle_mod, dtype, n, T, C, iters):
    d = _inputs(T, n, C, dtype, seed=T * 13 + C + n + iters)
    _check_bwd(mhc, oracle_mod, d, iters, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_backward_large_alpha_parity(mhc, oracle_mod, dtype):
    d = _inputs(150, 4, 512, dtype, seed=19, alpha=1.0)
    _check_bwd(mhc, oracle_mod, d, 20, dtype)


# ---------------------------- cross-layer fusion: post(l) + mapping(l+1)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("n,T,C", [(1, 33, 24), (2, 70, 64), (4, 300, 520), (4, 1, 8), (4, 129, 4096),
                                   (8, 65, 136), (16, 33, 64)])
def test_post_fused_parity(mhc, oracle_mod, dtype, n, T, C):
    """x_next and layer l+1's maps against the oracle's post then pre, and bit for bit
    against the unfused mhc_post -> mhc_pre (the fused kernel maps the stored x_next)."""
    from manifold_constrained_hyper_token_b200 import synth
    d = _inputs(T, n, C, dtype, seed=5 * T + C + n)
    a = float(d["alpha"][0])
    fwd = oracle_mod.pre(d["x"], d["phi"], d["b"], a)
    hp = torch.from_numpy(fwd["H_post"]).float()
    hr = torch.from_numpy(fwd["H_res"]).float()
    nxt = synth.layer_params(n, C, seed=1000 + n)
    dd, dn = _dev(d), _dev(nxt)
    st = _status()
    xn, hpre, hpost, hres = mhc.mhc_post_fused(dd["x"], dd["f_out"], hp.cuda(), hr.cuda(),
                                               dn["phi"], dn["b"], dn["alpha"], dev_status=st)
    xn_u = mhc.mhc_post(dd["x"], dd["f_out"], hp.cuda(), hr.cuda())
    _, hpre_u, hpost_u, hres_u = mhc.mhc_pre(xn_u, dn["phi"], dn["b"], dn["alpha"])
    h_in = mhc.mhc_layer_input(xn, hpre)
    h_in_u = mhc.mhc_pre(xn_u, dn["phi"], dn["b"], dn["alpha"])[0]
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref_xn = oracle_mod.post(d["x"], d["f_out"], hp, hr)
    ref = oracle_mod.pre(ref_xn, nxt["phi"], nxt["b"], float(nxt["alpha"][0]))
    tol = TOL[dtype]
    assert_close(_np(xn), ref_xn, tol)
    for got, k in ((hpre, "H_pre"), (hpost, "H_post"), (hres, "H_res")):
        assert_close(_np(got), ref[k], tol, k)
    assert torch.equal(xn, xn_u)
    assert torch.equal(hpre, hpre_u) and torch.equal(hpost, hpost_u) and torch.equal(hres, hres_u)
    assert torch.equal(h_in, h_in_u)


# ------------------------------------- the backward in training order (split)
def _hpost(T, n, seed):
    """Forward-style H_post values in (0, 2), float32, shared by both sides."""
    g = torch.Generator().manual_seed(seed)
    return (2.0 * torch.rand(T, n, generator=g)).float()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("n,T,C", [(1, 33, 24), (2, 70, 64), (4, 300, 520), (4, 1, 8), (8, 65, 136),
                                   (16, 40, 64)])
def test_post_backward_parity(mhc, oracle_mod, dtype, n, T, C):
    """grad_f_out within the I/O tolerance; red (fp32 sums over C of exact products)
    within 1e-5."""
    d = _inputs(T, n, C, dtype, seed=T + 7 * C + n)
    hp = _hpost(T, n, seed=T + n)
    dd = _dev(d)
    gf, red = mhc.mhc_post_backward(dd["x"], dd["f_out"], hp.cuda(), dd["grad_x_next"])
    ref = oracle_mod.post_backward(d["x"], d["f_out"], hp, d["grad_x_next"])
    assert_close(_np(gf), ref["grad_f_out"], TOL[dtype])
    assert_close(_np(red), ref["red"], 1e-5)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("n,T,C", [(1, 33, 24), (2, 70, 64), (4, 300, 520), (4, 1, 8), (8, 65, 136),
                                   (16, 40, 64)])
@pytest.mark.parametrize("iters", [1, 20])
def test_pre_backward_parity(mhc, oracle_mod, dtype, n, T, C, iters):
    """The pre half on the same red as the oracle (the oracle's post-half red,
    rounded to float32, fed to both sides)."""
    d = _inputs(T, n, C, dtype, seed=3 * T + C + n + iters)
    a = float(d["alpha"][0])
    fwd = oracle_mod.pre(d["x"], d["phi"], d["b"], a, iters=iters)
    red = torch.from_numpy(oracle_mod.post_backward(d["x"], d["f_out"], fwd["H_post"],
                                                    d["grad_x_next"])["red"]).float()
    dd = _dev(d)
    gx, gphi, gb, ga = mhc.mhc_pre_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"],
                                            dd["grad_x_next"], dd["grad_h_in"], red.cuda(),
                                            t_max=iters)
    ref = oracle_mod.pre_backward(d["x"], d["phi"], d["b"], a, d["grad_x_next"], d["grad_h_in"],
                                  red, iters=iters)
    tol = TOL[dtype]
    terms = _alpha_terms(oracle_mod, lambda sl: oracle_mod.pre_backward(
        d["x"][sl], d["phi"], d["b"], a, d["grad_x_next"][sl], d["grad_h_in"][sl], red[sl],
        iters=iters), T)
    for k, got in (("grad_x", gx), ("grad_phi", gphi), ("grad_b", gb)):
        assert_close(_np(got), ref[k], tol, k)
    assert _alpha_err(ga, ref["grad_alpha"], terms) < tol


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_split_backward_chain(mhc, oracle_mod, dtype):
    """GPU forward, then post half -> pre half on the GPU, against the oracle's one-call
    backward and against the GPU's one-call backward."""
    T, n, C = 260, 4, 1000
    d = _inputs(T, n, C, dtype, seed=77)
    dd = _dev(d)
    _, _, Hpost, _ = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"])
    gf, red = mhc.mhc_post_backward(dd["x"], dd["f_out"], Hpost, dd["grad_x_next"])
    gx, gphi, gb, ga = mhc.mhc_pre_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"],
                                            dd["grad_x_next"], dd["grad_h_in"], red)
    whole = mhc.mhc_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"], dd["f_out"],
                             dd["grad_x_next"], dd["grad_h_in"])
    ref = oracle_mod.backward(d["x"], d["phi"], d["b"], float(d["alpha"][0]), d["f_out"],
                              d["grad_x_next"], d["grad_h_in"])
    tol = TOL[dtype]
    for got, w, r in ((gx, whole[0], ref["grad_x"]), (gphi, whole[1], ref["grad_phi"]),
                      (gb, whole[2], ref["grad_b"]), (gf, whole[4], ref["grad_f_out"])):
        assert_close(_np(got), r, tol)
        assert_close(_np(got), _np(w), tol)
    a = float(d["alpha"][0])
    terms = _alpha_terms(oracle_mod, lambda sl: oracle_mod.backward(
        d["x"][sl], d["phi"], d["b"], a, d["f_out"][sl], d["grad_x_next"][sl],
        d["grad_h_in"][sl]), T)
    assert _alpha_err(ga, ref["grad_alpha"], terms) < tol


# ------------------------------------------ per-group alpha (pre, post, res)
ALPHA3 = [0.02, -0.015, 0.03]


def _alpha3_errs(ga, ref_ga, per_token):
    """Each group's grad_alpha is a token sum that can cancel: measured against the
    sum of its per-token magnitudes (as _alpha_err for one alpha)."""
    got = _np(ga).reshape(-1)
    out = []
    for g in range(3):
        scale = max(abs(ref_ga[g]), float(np.sum(np.abs(per_token[:, g]))))
        out.append(abs(got[g] - ref_ga[g]) / scale if scale > 0 else 0.0)
    return out


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("n,T,C", [(4, 130, 520), (2, 65, 24), (16, 33, 64)])
def test_pre_per_group_alpha(mhc, oracle_mod, dtype, n, T, C):
    d = _inputs(T, n, C, dtype, seed=11 * T + n)
    d["alpha"] = torch.tensor(ALPHA3, dtype=torch.float32)
    dd = _dev(d)
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"])
    ref = oracle_mod.pre(d["x"], d["phi"], d["b"], np.array(ALPHA3))
    for got, k in ((h_in, "h_in"), (Hpre, "H_pre"), (Hpost, "H_post"), (Hres, "H_res")):
        assert_close(_np(got), ref[k], TOL[dtype], k)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("n,T,C", [(4, 130, 520), (2, 65, 24), (8, 33, 136), (16, 33, 64)])
def test_backward_per_group_alpha(mhc, oracle_mod, dtype, n, T, C):
    d = _inputs(T, n, C, dtype, seed=13 * T + n)
    d["alpha"] = torch.tensor(ALPHA3, dtype=torch.float32)
    a3 = np.array(ALPHA3)
    dd = _dev(d)
    gx, gphi, gb, ga, gf = mhc.mhc_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"], dd["f_out"],
                                            dd["grad_x_next"], dd["grad_h_in"])
    assert ga.numel() == 3
    ref = oracle_mod.backward(d["x"], d["phi"], d["b"], a3, d["f_out"], d["grad_x_next"],
                              d["grad_h_in"])
    tol = TOL[dtype]
    for got, k in ((gx, "grad_x"), (gphi, "grad_phi"), (gb, "grad_b"), (gf, "grad_f_out")):
        assert_close(_np(got), ref[k], tol, k)
    terms = np.array([oracle_mod.backward(d["x"][t:t + 1], d["phi"], d["b"], a3, d["f_out"][t:t + 1],
                                          d["grad_x_next"][t:t + 1], d["grad_h_in"][t:t + 1])["grad_alpha"]
                      for t in range(T)])
    assert max(_alpha3_errs(ga, ref["grad_alpha"], terms)) < tol


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_split_backward_per_group_alpha(mhc, oracle_mod, dtype):
    T, n, C = 130, 4, 520
    d = _inputs(T, n, C, dtype, seed=99)
    d["alpha"] = torch.tensor(ALPHA3, dtype=torch.float32)
    a3 = np.array(ALPHA3)
    dd = _dev(d)
    _, _, Hpost, _ = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"])
    gf, red = mhc.mhc_post_backward(dd["x"], dd["f_out"], Hpost, dd["grad_x_next"])
    gx, gphi, gb, ga = mhc.mhc_pre_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"],
                                            dd["grad_x_next"], dd["grad_h_in"], red)
    ref = oracle_mod.backward(d["x"], d["phi"], d["b"], a3, d["f_out"], d["grad_x_next"],
                              d["grad_h_in"])
    tol = TOL[dtype]
    for got, k in ((gx, "grad_x"), (gphi, "grad_phi"), (gb, "grad_b"), (gf, "grad_f_out")):
        assert_close(_np(got), ref[k], tol, k)
    terms = np.array([oracle_mod.backward(d["x"][t:t + 1], d["phi"], d["b"], a3, d["f_out"][t:t + 1],
                                          d["grad_x_next"][t:t + 1], d["grad_h_in"][t:t + 1])["grad_alpha"]
                      for t in range(T)])
    assert max(_alpha3_errs(ga, ref["grad_alpha"], terms)) < tol


def test_pre_backward_small_workspace_rejected(mhc):
    d = _dev(_inputs(64, 4, 256, torch.bfloat16, seed=5))
    red = torch.zeros(64, 20, dtype=torch.float32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(mhc.MhcError) as e:
        mhc.mhc_pre_backward(d["x"], d["phi"], d["b"], d["alpha"], d["grad_x_next"],
                             d["grad_h_in"], red, workspace=ws)
    assert e.value.status == 6


def test_backward_is_deterministic(mhc):
    d = _dev(_inputs(300, 4, 512, torch.bfloat16, seed=4))
    a = mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"], d["grad_x_next"],
                         d["grad_h_in"])
    b = mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"], d["grad_x_next"],
                         d["grad_h_in"])
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_wide_backward_is_deterministic(mhc, dtype):
    """n = 16 runs its own kernels (k_wide.cu): fixed-order sums there too."""
    d = _dev(_inputs(100, 16, 136, dtype, seed=6))
    a = mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"], d["grad_x_next"],
                         d["grad_h_in"])
    b = mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"], d["grad_x_next"],
                         d["grad_h_in"])
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("T,C", [(1000, 1024), (2048, 7168)])
def test_n8_backward_is_deterministic(mhc, T, C):
    """n = 8 with bf16 runs the tensor-core kernels, whose grad_phi is split over
    persistent CTAs (shared blocks added in CTA order) and whose Sinkhorn sums run
    as butterflies over 8 lanes: repeated calls give identical bits."""
    d = _dev(_inputs(T, 8, C, torch.bfloat16, seed=10))
    a = mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"], d["grad_x_next"],
                         d["grad_h_in"])
    b = mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"], d["grad_x_next"],
                         d["grad_h_in"])
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_backward_small_workspace_rejected(mhc):
    d = _dev(_inputs(64, 4, 64, torch.bfloat16))
    need = mhc.mhc_backward_workspace_size(4, 64, 64, torch.bfloat16)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(mhc.MhcError) as e:
        mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"], d["grad_x_next"],
                         d["grad_h_in"], workspace=ws)
    assert e.value.status == 6


# ------------------------------------------------------ full-size configs
@pytest.mark.slow
def test_forward_bf16_full_size(mhc, oracle_mod):
    """T=8192, n=4, C=4096 bf16 forward (pre + post with a supplied f_out):
    a seeded sample of tokens against the oracle."""
    from manifold_constrained_hyper_token_b200 import synth
    T, n, C = 8192, 4, 4096
    d = synth.layer_inputs(T, n, C, seed=0, dtype=torch.bfloat16, backward=False)
    dd = _dev(d)
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"])
    x_next = mhc.mhc_post(dd["x"], dd["f_out"], Hpost, Hres)
    idx = synth.token_sample(T, 256, seed=1)
    ref = oracle_mod.pre(d["x"][idx], d["phi"], d["b"], float(d["alpha"][0]))
    xn = oracle_mod.post(d["x"][idx], d["f_out"][idx], ref["H_post"], ref["H_res"])
    ic = idx.cuda()
    for got, r in ((h_in[ic], ref["h_in"]), (Hpre[ic], ref["H_pre"]), (Hpost[ic], ref["H_post"]),
                   (Hres[ic], ref["H_res"]), (x_next[ic], xn)):
        assert_close(_np(got), r, 2e-2)


@pytest.mark.slow
def test_forward_backward_full_size(mhc, oracle_mod):
    """T=16384, n=4, C=7168 bf16 forward + backward: per-token outputs on a seeded
    sample of tokens; grad_phi / grad_b / grad_alpha against the full-T oracle."""
    from manifold_constrained_hyper_token_b200 import synth
    T, n, C = 16384, 4, 7168
    d = synth.layer_inputs(T, n, C, seed=0, dtype=torch.bfloat16, backward=True)
    dd = _dev(d)
    alpha = float(d["alpha"][0])
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"])
    x_next = mhc.mhc_post(dd["x"], dd["f_out"], Hpost, Hres)
    gx, gphi, gb, ga, gf = mhc.mhc_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"], dd["f_out"],
                                            dd["grad_x_next"], dd["grad_h_in"])
    torch.cuda.synchronize()
    idx = synth.token_sample(T, 256, seed=2)
    ic = idx.cuda()
    ref = oracle_mod.pre(d["x"][idx], d["phi"], d["b"], alpha)
    xn = oracle_mod.post(d["x"][idx], d["f_out"][idx], ref["H_post"], ref["H_res"])
    for got, r in ((h_in[ic], ref["h_in"]), (Hres[ic], ref["H_res"]), (x_next[ic], xn)):
        assert_close(_np(got), r, 2e-2)
    rs = oracle_mod.backward(d["x"][idx], d["phi"], d["b"], alpha, d["f_out"][idx],
                             d["grad_x_next"][idx], d["grad_h_in"][idx])
    assert_close(_np(gx[ic]), rs["grad_x"], 2e-2)
    assert_close(_np(gf[ic]), rs["grad_f_out"], 2e-2)
    full = oracle_mod.backward(d["x"], d["phi"], d["b"], alpha, d["f_out"], d["grad_x_next"],
                               d["grad_h_in"], chunk=1024)
    assert_close(_np(gphi), full["grad_phi"], 2e-2)
    assert_close(_np(gb), full["grad_b"], 2e-2)
    assert_close(_np(ga), np.array([full["grad_alpha"]]), 2e-2)


# ------------- bf16 n = 8 on the tensor cores: several 128-token tiles with a
# ragged last one, several 256-channel phi u blocks and 128-channel grad_phi
# blocks with a ragged last one, and C % 16 == 8 (a half-filled last block of
# the tiled phi copy)
N8_SHAPES = [(300, 520), (129, 4104), (1000, 1024)]


@pytest.mark.parametrize("T,C", N8_SHAPES)
def test_n8_tensor_core_pre(mhc, oracle_mod, T, C):
    d = _inputs(T, 8, C, torch.bfloat16, seed=11 * T + C)
    dd = _dev(d)
    st = _status()
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle_mod.pre(d["x"], d["phi"], d["b"], float(d["alpha"][0]))
    for k, got in (("h_in", h_in), ("H_pre", Hpre), ("H_post", Hpost), ("H_res", Hres)):
        assert_close(_np(got), ref[k], 2e-2, k)


@pytest.mark.parametrize("T,C", N8_SHAPES)
def test_n8_tensor_core_backward(mhc, oracle_mod, T, C):
    d = _inputs(T, 8, C, torch.bfloat16, seed=13 * T + C)
    _check_bwd(mhc, oracle_mod, d, 20, torch.bfloat16)


@pytest.mark.slow
def test_n8_forward_backward_large(mhc, oracle_mod):
    """T=4096, n=8, C=7168 bf16 forward + backward (the n = 8 bench layer at a
    quarter of its tokens): per-token outputs on a seeded sample of tokens;
    grad_phi / grad_b / grad_alpha against the full-T oracle."""
    from manifold_constrained_hyper_token_b200 import synth
    T, n, C = 4096, 8, 7168
    d = synth.layer_inputs(T, n, C, seed=3, dtype=torch.bfloat16, backward=True)
    dd = _dev(d)
    alpha = float(d["alpha"][0])
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"])
    gx, gphi, gb, ga, gf = mhc.mhc_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"], dd["f_out"],
                                            dd["grad_x_next"], dd["grad_h_in"])
    torch.cuda.synchronize()
    idx = synth.token_sample(T, 128, seed=4)
    ic = idx.cuda()
    ref = oracle_mod.pre(d["x"][idx], d["phi"], d["b"], alpha)
    for got, r in ((h_in[ic], ref["h_in"]), (Hres[ic], ref["H_res"]), (Hpre[ic], ref["H_pre"])):
        assert_close(_np(got), r, 2e-2)
    rs = oracle_mod.backward(d["x"][idx], d["phi"], d["b"], alpha, d["f_out"][idx],
                             d["grad_x_next"][idx], d["grad_h_in"][idx])
    assert_close(_np(gx[ic]), rs["grad_x"], 2e-2)
    assert_close(_np(gf[ic]), rs["grad_f_out"], 2e-2)
    full = oracle_mod.backward(d["x"], d["phi"], d["b"], alpha, d["f_out"], d["grad_x_next"],
                               d["grad_h_in"], chunk=512)
    assert_close(_np(gphi), full["grad_phi"], 2e-2)
    assert_close(_np(gb), full["grad_b"], 2e-2)
    assert_close(_np(ga), np.array([full["grad_alpha"]]), 2e-2)


@pytest.mark.slow
def test_n16_forward_backward_large(mhc, oracle_mod):
    """T=200, n=16, C=7168 bf16 forward + backward: the n = 16 tensor-core kernels at
    the bench's channel count (112 projection chunks, 28 phi u channel blocks, 56
    grad_phi blocks, C-reduction slabs of 8 tokens) and a ragged second token tile,
    every output against the oracle."""
    from manifold_constrained_hyper_token_b200 import synth
    T, n, C = 200, 16, 7168
    d = synth.layer_inputs(T, n, C, seed=6, dtype=torch.bfloat16, backward=True)
    dd = _dev(d)
    alpha = float(d["alpha"][0])
    st = _status()
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"], dev_status=st)
    gx, gphi, gb, ga, gf = mhc.mhc_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"], dd["f_out"],
                                            dd["grad_x_next"], dd["grad_h_in"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle_mod.pre(d["x"], d["phi"], d["b"], alpha)
    for k, got in (("h_in", h_in), ("H_pre", Hpre), ("H_post", Hpost), ("H_res", Hres)):
        assert_close(_np(got), ref[k], 2e-2, k)
    rb = oracle_mod.backward(d["x"], d["phi"], d["b"], alpha, d["f_out"], d["grad_x_next"],
                             d["grad_h_in"])
    for k, got in (("grad_x", gx), ("grad_f_out", gf), ("grad_phi", gphi), ("grad_b", gb)):
        assert_close(_np(got), rb[k], 2e-2, k)
    assert_close(_np(ga), np.array([rb["grad_alpha"]]), 2e-2, "grad_alpha")


# ------------- bf16 n = 4 mapping with each 128-token tile cut into channel
# parts (one CTA each, records added by the tile's last part in part order)
# whenever one CTA per tile would leave SMs idle.  (T, C): several parts per
# tile, a ragged last chunk (C % 32 != 0), a ragged last tile, and the 16-part
# limit per tile.
SPLIT_SHAPES = [(1000, 1024), (300, 7168), (777, 1000), (4096, 7168), (129, 4104)]


@pytest.mark.parametrize("T,C", SPLIT_SHAPES)
def test_channel_split_mapping_pre(mhc, oracle_mod, T, C):
    d = _inputs(T, 4, C, torch.bfloat16, seed=T + 3 * C)
    idx = np.unique(np.concatenate([np.arange(0, T, max(1, T // 200)), [T - 1]]))
    dd = _dev(d)
    st = _status()
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle_mod.pre(d["x"][idx], d["phi"], d["b"], float(d["alpha"][0]))
    ic = torch.from_numpy(idx).cuda()
    for k, got in (("h_in", h_in), ("H_pre", Hpre), ("H_post", Hpost), ("H_res", Hres)):
        assert_close(_np(got[ic]), ref[k], 2e-2, k)


@pytest.mark.parametrize("T,C", SPLIT_SHAPES[:3] + SPLIT_SHAPES[4:])
def test_channel_split_mapping_backward(mhc, oracle_mod, T, C):
    d = _inputs(T, 4, C, torch.bfloat16, seed=2 * T + C)
    _check_bwd(mhc, oracle_mod, d, 20, torch.bfloat16)


@pytest.mark.parametrize("T,C", [(1000, 1024), (300, 7168)])
def test_channel_split_mapping_pre_backward(mhc, oracle_mod, T, C):
    d = _inputs(T, 4, C, torch.bfloat16, seed=5 * T + C)
    a = float(d["alpha"][0])
    fwd = oracle_mod.pre(d["x"], d["phi"], d["b"], a)
    red = torch.from_numpy(oracle_mod.post_backward(d["x"], d["f_out"], fwd["H_post"],
                                                    d["grad_x_next"])["red"]).float()
    dd = _dev(d)
    gx, gphi, gb, ga = mhc.mhc_pre_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"],
                                            dd["grad_x_next"], dd["grad_h_in"], red.cuda())
    ref = oracle_mod.pre_backward(d["x"], d["phi"], d["b"], a, d["grad_x_next"], d["grad_h_in"],
                                  red)
    for k, got in (("grad_x", gx), ("grad_phi", gphi), ("grad_b", gb)):
        assert_close(_np(got), ref[k], 2e-2, k)


def test_channel_split_mapping_is_deterministic(mhc):
    """Parts of a tile are added in part order: repeated calls give identical bits."""
    d = _dev(_inputs(4096, 4, 7168, torch.bfloat16, seed=8))
    outs = [mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"], d["grad_x_next"],
                             d["grad_h_in"]) for _ in range(2)]
    for u, v in zip(*outs):
        assert torch.equal(u, v)
    pre = [mhc.mhc_pre(d["x"], d["phi"], d["b"], d["alpha"]) for _ in range(2)]
    for u, v in zip(*pre):
        assert torch.equal(u, v)
