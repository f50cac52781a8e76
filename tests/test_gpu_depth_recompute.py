"""DepthStack on the GPU: L = 24 mHC layers, n = 4, C = 7168, bf16 streams,
F_l(h) = s_l h, backward in training order (mhc_post_backward, then F's
backward, then mhc_pre_backward) with block recompute (reportify.cn mHC
summary, [21] recompute, [22] memory-optimal recompute block).

* Recompute changes no bit: blocks of 1, 4 (the plan's) and 24 layers give
  identical x_L, grad_x_0 and per-layer grad_phi / grad_b / grad_alpha at
  T = 4096 (every kernel reduces in a fixed order).
* The allocator follows the plan's cost: for each block size the peak device
  memory over forward + backward, less the memory held before the forward, is
  R(B) C T 2 bytes (R from mhc_recompute_plan's cost, in units of C bf16 elements
  per token) plus a term that every block size shares: the gradient pair,
  the F temporaries and the workspaces.  That shared term agrees across the
  three block sizes to within two units and is at most 12 units + 64 MB.
* Against the oracle: on 64 sampled tokens the oracle runs its own fp64 chain
  through the 24 layers (pre, F, post; then post_backward, F's backward,
  pre_backward).  The GPU's x_L and grad_x_0 at T = 4096 are compared on those
  tokens, with the depth-scaled bf16 bound (2e-2 plus one bf16 unit roundoff per
  stored tensor on the path).  A DepthStack run on just those 64 tokens then gives
  per-layer parameter gradients, compared with the oracle chain's sums over them.
  grad_alpha is a sum over tokens whose terms cancel (the sum can be far smaller
  than the terms), so its error is taken against max(|sum|, sum of |terms|), the
  scale that the chained inputs' error and fp32 accumulation act on; the oracle
  gives the per-token terms one token at a time.
"""
import math

import numpy as np
import pytest
import torch

from conftest import rel_err

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

L, T, N, C = 24, 4096, 4, 7168
SAMPLE = 64
TOL = 2e-2
U_BF16 = 2.0 ** -9
UNIT = C * T * 2          # one C-wide bf16 row per token


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


def _R(B):
    return N * (math.ceil(L / B) - 1) + (N + 2) * B


@pytest.fixture(scope="module")
def setup(mhc):
    from manifold_constrained_hyper_token_b200 import synth
    prms = [synth.layer_params(N, C, seed=l) for l in range(L)]
    gains = [synth.depth_gain(l) for l in range(L)]
    d = synth.depth_stack_chunk(T, N, C, chunk=0)
    return prms, gains, d


def _stack(mhc, prms, gains, block):
    from manifold_constrained_hyper_token_b200.depth import DepthStack
    dprm = [{k: v.cuda() for k, v in p.items()} for p in prms]

    def F(l, h):
        return (h.float() * gains[l]).to(torch.bfloat16)

    def F_backward(l, h, f, gf):
        return (gf.float() * gains[l]).to(torch.bfloat16)

    return DepthStack(dprm, F, F_backward, n=N, block=block)


def _run(mhc, setup, block):
    prms, gains, d = setup
    st = _stack(mhc, prms, gains, block)
    x0, G = d["x0"].cuda(), d["G_last"].cuda()
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    xL = st.forward(x0)
    gx0, grads = st.backward(G)
    torch.cuda.synchronize()
    peak = torch.cuda.max_memory_allocated() - base
    return st.block, xL, gx0, grads, peak


@pytest.fixture(scope="module")
def runs(mhc, setup):
    out = {}
    for block in (None, 1, L):
        B, xL, gx0, grads, peak = _run(mhc, setup, block)
        out[B] = dict(xL=xL.cpu(), gx0=gx0.cpu(),
                      grads=[tuple(g.cpu() for g in gl) for gl in grads], peak=peak)
        del xL, gx0, grads
        torch.cuda.empty_cache()
    return out


def test_plan_block(mhc, runs):
    assert mhc.mhc_recompute_plan(N, L) == (4, _R(4))
    assert sorted(runs) == [1, 4, L]


def test_recompute_is_bit_identical(runs):
    ref = runs[1]
    for B in (4, L):
        r = runs[B]
        assert torch.equal(r["xL"], ref["xL"]), B
        assert torch.equal(r["gx0"], ref["gx0"]), B
        for l in range(L):
            for a, b in zip(r["grads"][l], ref["grads"][l]):
                assert torch.equal(a, b), (B, l)


def test_memory_follows_plan(runs):
    shared = {B: runs[B]["peak"] - _R(B) * UNIT for B in runs}
    print({B: (runs[B]["peak"] / UNIT, _R(B), shared[B] / UNIT) for B in runs})
    assert runs[4]["peak"] < runs[1]["peak"] < runs[L]["peak"]
    for B, s in shared.items():
        assert 0 <= s <= 12 * UNIT + (64 << 20), (B, s / UNIT)
    assert max(shared.values()) - min(shared.values()) <= 2 * UNIT


def _oracle_chain(o, prms, gains, x0, G):
    xs, fs, rs = [x0], [], []
    for l in range(L):
        a = float(prms[l]["alpha"][0])
        r = o.pre(xs[l], prms[l]["phi"], prms[l]["b"], a)
        f = gains[l] * r["h_in"]
        fs.append(f)
        rs.append(r)
        xs.append(o.post(xs[l], f, r["H_post"], r["H_res"]))
    grads = [None] * L
    alpha_scale = [0.0] * L
    for l in reversed(range(L)):
        a = float(prms[l]["alpha"][0])
        pb = o.post_backward(xs[l], fs[l], rs[l]["H_post"], G)
        gh = gains[l] * pb["grad_f_out"]
        rb = o.pre_backward(xs[l], prms[l]["phi"], prms[l]["b"], a, G, gh, pb["red"])
        grads[l] = (rb["grad_phi"], rb["grad_b"], rb["grad_alpha"])
        terms = [o.pre_backward(xs[l][t:t + 1], prms[l]["phi"], prms[l]["b"], a, G[t:t + 1],
                                gh[t:t + 1], pb["red"][t:t + 1])["grad_alpha"]
                 for t in range(xs[l].shape[0])]
        alpha_scale[l] = max(abs(rb["grad_alpha"]), float(np.sum(np.abs(terms))))
        G = rb["grad_x"]
    return xs[L], G, grads, alpha_scale


def test_chained_against_oracle(mhc, setup, runs, oracle_mod):
    from manifold_constrained_hyper_token_b200 import synth
    prms, gains, d = setup
    idx = synth.token_sample(T, SAMPLE, seed=0)
    xL_o, gx0_o, grads_o, alpha_scale = _oracle_chain(oracle_mod, prms, gains,
                                                      _np(d["x0"][idx]), _np(d["G_last"][idx]))
    r = runs[4]
    e_x = rel_err(_np(r["xL"][idx]), xL_o)
    e_g = rel_err(_np(r["gx0"][idx]), gx0_o)
    print(f"x_L {e_x:.2e}  grad_x_0 {e_g:.2e}")
    assert e_x < TOL + L * U_BF16
    assert e_g < TOL + (2 * L - 1) * U_BF16

    # the same 64 tokens as a stack of their own: per-layer parameter gradients
    st = _stack(mhc, prms, gains, None)
    xs = d["x0"][idx].contiguous().cuda()
    Gs = d["G_last"][idx].contiguous().cuda()
    st.forward(xs)
    _, grads = st.backward(Gs)
    bound = TOL + 2 * L * U_BF16
    worst = [0.0, 0.0, 0.0]
    for l in range(L):
        for k in range(2):
            e = rel_err(_np(grads[l][k]), grads_o[l][k])
            worst[k] = max(worst[k], e)
            assert e < bound, (l, ("grad_phi", "grad_b")[k], e)
        e = abs(float(_np(grads[l][2]).reshape(-1)[0]) - grads_o[l][2]) / alpha_scale[l]
        worst[2] = max(worst[2], e)
        assert e < bound, (l, "grad_alpha", e)
    print("worst per-layer grad_phi, grad_b, grad_alpha:", worst)
