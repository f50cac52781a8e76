"""Depth stack on the GPU against the fp64 oracle: L = 24 mHC layers over
T = 65536 tokens, n = 4, C = 7168, bf16 activations, per-layer phi (seed l) and
F_l(h) = s_l * h, forward and backward through the whole stack.

The GPU runs the full stack in 16384-token chunks (tokens are independent in
every per-token output; only grad_phi / grad_b / grad_alpha sum over tokens).
Three checks:

* per layer: on sampled tokens, every one of the 24 layers against the oracle
  fed the bf16 inputs that the GPU layer saw (x_l, f_out_l, grad_x_{l+1},
  grad_h_in_l), at the single-layer bf16 tolerance 2e-2;
* chained: on the same tokens the oracle runs its own fp64 chain through all 24
  layers (forward x_1..x_24, then backward grad_x_23..grad_x_0).  The GPU
  stores every stream and gradient in bf16 (unit roundoff u = 2^-9), and each
  stored tensor on the path adds up to one such rounding, so after k stored
  tensors the bound is 2e-2 + k u: k = l for x_l, k = L + (L - 1 - l) for
  grad_x_l (the forward streams plus the gradients from above);
* full layers: the first and the last layer on every token with the oracle fed
  the GPU layer's inputs, and grad_phi / grad_b / grad_alpha against the oracle
  summed over all 65536 tokens.

F's backward is outside the layer: with f_out = s_l h_in,
grad_h_in = s_l grad_f_out, and grad_f_out does not depend on grad_h_in, so each
layer runs the library backward once with grad_h_in = 0 to read grad_f_out,
scales it, and runs it again.  The oracle takes the same two steps.
"""
import numpy as np
import pytest
import torch

from conftest import rel_err

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

L, T, N, C = 24, 65536, 4, 7168
TC = 16384          # tokens per GPU chunk
SUB = 4096          # tokens per oracle call in the full-layer check
SAMPLE = 64         # chained tokens per chunk
FULL_LAYERS = (0, L - 1)
TOL = 2e-2
U_BF16 = 2.0 ** -9


@pytest.fixture(scope="module")
def mhc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from manifold_constrained_hyper_token_b200 import build
    build.build()
    import manifold_constrained_hyper_token_b200 as m
    return m


class _Err:
    """Norm-wise relative error of one tensor accumulated over token chunks."""

    def __init__(self):
        self.num = 0.0
        self.den = 0.0

    def add(self, got, ref):
        got = np.asarray(got, dtype=np.float64)
        self.num = max(self.num, float(np.max(np.abs(got - ref))))
        self.den = max(self.den, float(np.max(np.abs(ref))))

    def value(self):
        return self.num / self.den if self.den > 0 else self.num


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _oracle_layer_backward(o, x, prm, f, G, s_l):
    """The oracle's two-step layer backward (grad_h_in = s_l * grad_f_out)."""
    a = float(prm["alpha"][0])
    zero = np.zeros((x.shape[0], x.shape[2]))
    gf = o.backward(x, prm["phi"], prm["b"], a, f, G, zero)["grad_f_out"]
    g = s_l * gf
    return o.backward(x, prm["phi"], prm["b"], a, f, G, g), g


def test_depth_stack_24_layers(mhc, oracle_mod):
    from manifold_constrained_hyper_token_b200 import synth
    o = oracle_mod
    prms = [synth.layer_params(N, C, seed=l) for l in range(L)]
    gains = [synth.depth_gain(l) for l in range(L)]
    dprm = [{k: v.cuda() for k, v in p.items()} for p in prms]

    chain_x = [_Err() for _ in range(L + 1)]      # x_l, l = 1..L
    chain_gx = [_Err() for _ in range(L)]         # grad_x_l, l = 0..L-1
    layer = [{k: _Err() for k in ("H_res", "x_next", "grad_x", "grad_f_out")} for _ in range(L)]
    full = {l: {k: _Err() for k in ("h_in", "H_pre", "H_post", "H_res", "x_next", "grad_x",
                                    "grad_f_out")} for l in FULL_LAYERS}
    gpu_par = {l: [0.0, 0.0, 0.0] for l in FULL_LAYERS}   # grad_phi, grad_b, grad_alpha sums
    ref_par = {l: [0.0, 0.0, 0.0] for l in FULL_LAYERS}

    for c in range(T // TC):
        d = synth.depth_stack_chunk(TC, N, C, chunk=c)
        idx = synth.token_sample(TC, SAMPLE, seed=c)
        ic = idx.cuda()

        # ---------------------------------------------------- GPU forward
        xs = [d["x0"].cuda()]
        fs, Hs = [], []
        for l in range(L):
            h_in, Hpre, Hpost, Hres = mhc.mhc_pre(xs[l], dprm[l]["phi"], dprm[l]["b"],
                                                  dprm[l]["alpha"])
            f = (h_in.float() * gains[l]).to(torch.bfloat16)
            fs.append(f)
            Hs.append((h_in, Hpre, Hpost, Hres))
            xs.append(mhc.mhc_post(xs[l], f, Hpost, Hres))

        # --------------------------------------------------- GPU backward
        G = d["G_last"].cuda()
        gxs = [None] * L
        gs = [None] * L
        Gin = [None] * L     # sampled grad_x_next rows fed to layer l
        gfs = [None] * L
        outs = {}
        for l in reversed(range(L)):
            p = dprm[l]
            zero = torch.zeros_like(fs[l])
            gf = mhc.mhc_backward(xs[l], p["phi"], p["b"], p["alpha"], fs[l], G, zero)[4]
            g = (gf.float() * gains[l]).to(torch.bfloat16)
            gx, gphi, gb, ga, gf2 = mhc.mhc_backward(xs[l], p["phi"], p["b"], p["alpha"], fs[l],
                                                     G, g)
            gs[l] = g
            Gin[l] = G[ic].clone()
            gfs[l] = gf2[ic].clone()
            if l in FULL_LAYERS:
                outs[l] = dict(G=G, grad_x=gx, grad_f_out=gf2)
                for k, v in enumerate((gphi, gb, ga)):
                    gpu_par[l][k] = gpu_par[l][k] + _np(v)
            gxs[l] = gx[ic].clone()
            G = gx
        torch.cuda.synchronize()

        # ------------------- every layer on sampled tokens, GPU layer inputs
        for l in range(L):
            a = float(prms[l]["alpha"][0])
            x, f = xs[l][ic].cpu(), fs[l][ic].cpu()
            r = o.pre(x, prms[l]["phi"], prms[l]["b"], a)
            layer[l]["H_res"].add(_np(Hs[l][3][ic]), r["H_res"])
            layer[l]["x_next"].add(_np(xs[l + 1][ic]), o.post(x, f, r["H_post"], r["H_res"]))
            rb = o.backward(x, prms[l]["phi"], prms[l]["b"], a, f, Gin[l].cpu(), gs[l][ic].cpu())
            layer[l]["grad_x"].add(_np(gxs[l]), rb["grad_x"])
            layer[l]["grad_f_out"].add(_np(gfs[l]), rb["grad_f_out"])

        # ------------------------------- chained oracle on sampled tokens
        xo = _np(d["x0"][idx])
        xo_l = [xo]
        fo_l = []
        for l in range(L):
            a = float(prms[l]["alpha"][0])
            r = o.pre(xo_l[l], prms[l]["phi"], prms[l]["b"], a)
            fo = gains[l] * r["h_in"]
            fo_l.append(fo)
            xo_l.append(o.post(xo_l[l], fo, r["H_post"], r["H_res"]))
            chain_x[l + 1].add(_np(xs[l + 1][ic]), xo_l[l + 1])
        Go = _np(d["G_last"][idx])
        for l in reversed(range(L)):
            rb, _ = _oracle_layer_backward(o, xo_l[l], prms[l], fo_l[l], Go, gains[l])
            chain_gx[l].add(_np(gxs[l]), rb["grad_x"])
            Go = rb["grad_x"]

        # ------------------------- full layers on the GPU layer's own inputs
        for l in FULL_LAYERS:
            a = float(prms[l]["alpha"][0])
            h_in, Hpre, Hpost, Hres = Hs[l]
            for t0 in range(0, TC, SUB):
                sl = slice(t0, t0 + SUB)
                x = xs[l][sl].cpu()
                f = fs[l][sl].cpu()
                r = o.pre(x, prms[l]["phi"], prms[l]["b"], a)
                for k, got in (("h_in", h_in), ("H_pre", Hpre), ("H_post", Hpost),
                               ("H_res", Hres)):
                    full[l][k].add(_np(got[sl]), r[k])
                full[l]["x_next"].add(_np(xs[l + 1][sl]), o.post(x, f, r["H_post"], r["H_res"]))
                rb = o.backward(x, prms[l]["phi"], prms[l]["b"], a, f, outs[l]["G"][sl].cpu(),
                                gs[l][sl].cpu())
                full[l]["grad_x"].add(_np(outs[l]["grad_x"][sl]), rb["grad_x"])
                full[l]["grad_f_out"].add(_np(outs[l]["grad_f_out"][sl]), rb["grad_f_out"])
                ref_par[l][0] = ref_par[l][0] + rb["grad_phi"]
                ref_par[l][1] = ref_par[l][1] + rb["grad_b"]
                ref_par[l][2] = ref_par[l][2] + rb["grad_alpha"]
        del xs, fs, Hs, outs, G, gxs, gs, Gin, gfs
        torch.cuda.empty_cache()

    print("layer  per-layer(x_next, grad_x)   chained(x_{l+1}, grad_x_l)  chained bounds")
    for l in range(L):
        kx, kg = l + 1, L + (L - 1 - l)
        print(f"{l:5d}  {layer[l]['x_next'].value():.2e} {layer[l]['grad_x'].value():.2e}"
              f"        {chain_x[l + 1].value():.2e} {chain_gx[l].value():.2e}"
              f"        {TOL + kx * U_BF16:.2e} {TOL + kg * U_BF16:.2e}")
    for l in FULL_LAYERS:
        print(f"full layer {l}: " + ", ".join(f"{k} {e.value():.2e}" for k, e in full[l].items()) +
              f", grad_phi {rel_err(gpu_par[l][0], ref_par[l][0]):.2e}"
              f", grad_b {rel_err(gpu_par[l][1], ref_par[l][1]):.2e}")
    for l in range(L):
        for k, e in layer[l].items():
            assert e.value() < TOL, ("per-layer", l, k, e.value())
    for l in range(L):
        assert chain_x[l + 1].value() < TOL + (l + 1) * U_BF16, ("chained x", l + 1)
        assert chain_gx[l].value() < TOL + (L + (L - 1 - l)) * U_BF16, ("chained grad_x", l)
    for l in FULL_LAYERS:
        for k, e in full[l].items():
            assert e.value() < TOL, (l, k, e.value())
        assert rel_err(gpu_par[l][0], ref_par[l][0]) < TOL
        assert rel_err(gpu_par[l][1], ref_par[l][1]) < TOL
        assert rel_err(np.atleast_1d(gpu_par[l][2]), np.atleast_1d(ref_par[l][2])) < TOL
