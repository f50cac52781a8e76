"""Host-side argument checks of the Python binding (no GPU).

Every entry point of the binding checks each tensor it hands to the library
against the problem's sizes before any launch: the element type the kernels
read or write, at least as many elements as they touch, and the device of x.
A mis-sized argument must raise ValueError naming it, never reach a kernel.

The tests build the arguments on the CPU.  A call whose arguments all pass the
checks stops at the last guard, which turns tensors into device pointers and
accepts CUDA tensors only; so "reaches the device guard" means "every size,
type and device check passed".  Each entry point is called that way for every
stream count, both activation types and both alpha forms, in the same
argument forms the GPU tests and the benchmark use; then one argument at a
time is made too short, of the wrong type or on another device.
"""
import pytest
import torch

from manifold_constrained_hyper_token_b200 import build, synth

F32, BF16 = torch.float32, torch.bfloat16
DEVICE_GUARD = "CUDA tensors only"
T, C = 5, 16


@pytest.fixture(scope="module")
def mhc():
    build.build()
    import manifold_constrained_hyper_token_b200 as m
    return m


def _args(n, dtype, ag):
    d = synth.layer_inputs(T, n, C, seed=1, dtype=dtype, backward=True)
    if ag == 3:
        d["alpha"] = torch.tensor([0.01, 0.02, 0.03], dtype=F32)
    d["H_pre"] = torch.zeros(T, n)
    d["H_post"] = torch.zeros(T, n)
    d["H_res"] = torch.zeros(T, n, n)
    d["red"] = torch.zeros(T, n * n + n)
    d["ws"] = torch.zeros(256, dtype=torch.uint8)
    d["st"] = torch.zeros(1, dtype=torch.int32)
    return d


def _outs(d, ag):
    """Caller-owned outputs of the backward, in the library's order."""
    x = d["x"]
    n = x.shape[1]
    M = n * n + 2 * n
    return (torch.empty_like(x), torch.empty(n * C, M), torch.empty(M),
            torch.empty(3 if ag == 3 else 1), torch.empty(T, C, dtype=x.dtype))


def _calls(mhc, d, ag):
    """Every tensor-taking entry point with well-formed arguments, by name; each
    entry takes the argument dict so that a test can alter one argument."""
    return {
        "pre": lambda a: mhc.mhc_pre(a["x"], a["phi"], a["b"], a["alpha"], dev_status=a["st"]),
        "pre_out": lambda a: mhc.mhc_pre(
            a["x"], a["phi"], a["b"], a["alpha"],
            out=(torch.empty(T, C, dtype=a["x"].dtype), a["H_pre"], a["H_post"], a["H_res"]),
            workspace=a["ws"]),
        "post": lambda a: mhc.mhc_post(a["x"], a["f_out"], a["H_post"], a["H_res"],
                                       dev_status=a["st"]),
        "backward": lambda a: mhc.mhc_backward(a["x"], a["phi"], a["b"], a["alpha"], a["f_out"],
                                               a["grad_x_next"], a["grad_h_in"],
                                               dev_status=a["st"]),
        "backward_noalloc": lambda a: mhc.mhc_backward_noalloc(
            a["x"], a["phi"], a["b"], a["alpha"], a["f_out"], a["grad_x_next"], a["grad_h_in"]),
        "post_fused": lambda a: mhc.mhc_post_fused(a["x"], a["f_out"], a["H_post"], a["H_res"],
                                                   a["phi"], a["b"], a["alpha"]),
        "layer_input": lambda a: mhc.mhc_layer_input(a["x"], a["H_pre"]),
        "post_backward": lambda a: mhc.mhc_post_backward(a["x"], a["f_out"], a["H_post"],
                                                         a["grad_x_next"]),
        "pre_backward": lambda a: mhc.mhc_pre_backward(a["x"], a["phi"], a["b"], a["alpha"],
                                                       a["grad_x_next"], a["grad_h_in"],
                                                       a["red"]),
        "backward_map": lambda a: mhc.mhc_backward_map(a["x"], a["phi"], a["b"], a["alpha"],
                                                       a["f_out"], a["grad_x_next"],
                                                       a["grad_h_in"], a["ws"]),
        "backward_apply": lambda a: mhc.mhc_backward_apply(a["x"], a["phi"], a["grad_x_next"],
                                                           a["grad_h_in"], a["ws"],
                                                           alpha_groups=ag),
        # the caller-owned output forms (the benchmark's and the no-alloc caller's)
        "post_out": lambda a: mhc.mhc_post(a["x"], a["f_out"], a["H_post"], a["H_res"],
                                           out=torch.empty_like(a["x"])),
        "post_fused_out": lambda a: mhc.mhc_post_fused(
            a["x"], a["f_out"], a["H_post"], a["H_res"], a["phi"], a["b"], a["alpha"],
            out=(torch.empty_like(a["x"]), torch.empty_like(a["H_pre"]),
                 torch.empty_like(a["H_post"]), torch.empty_like(a["H_res"])),
            workspace=a["ws"]),
        "layer_input_out": lambda a: mhc.mhc_layer_input(
            a["x"], a["H_pre"], out=torch.empty(T, C, dtype=a["x"].dtype)),
        "backward_out": lambda a: mhc.mhc_backward(
            a["x"], a["phi"], a["b"], a["alpha"], a["f_out"], a["grad_x_next"], a["grad_h_in"],
            out=_outs(a, ag), workspace=a["ws"]),
        "backward_noalloc_out": lambda a: mhc.mhc_backward_noalloc(
            a["x"], a["phi"], a["b"], a["alpha"], a["f_out"], a["grad_x_next"], a["grad_h_in"],
            out=_outs(a, ag), dev_status=a["st"]),
        "backward_apply_out": lambda a: mhc.mhc_backward_apply(
            a["x"], a["phi"], a["grad_x_next"], a["grad_h_in"], a["ws"], alpha_groups=ag,
            out=_outs(a, ag)),
        "post_backward_out": lambda a: mhc.mhc_post_backward(
            a["x"], a["f_out"], a["H_post"], a["grad_x_next"],
            out=(torch.empty_like(a["f_out"]), torch.empty_like(a["red"]))),
        "pre_backward_out": lambda a: mhc.mhc_pre_backward(
            a["x"], a["phi"], a["b"], a["alpha"], a["grad_x_next"], a["grad_h_in"], a["red"],
            out=_outs(a, ag)[:4], workspace=a["ws"]),
    }


@pytest.mark.parametrize("ag", [1, 3], ids=["alpha1", "alpha3"])
@pytest.mark.parametrize("dtype", [F32, BF16], ids=["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_well_formed_calls_pass_every_check(mhc, n, dtype, ag):
    d = _args(n, dtype, ag)
    for name, call in _calls(mhc, d, ag).items():
        with pytest.raises(ValueError, match=DEVICE_GUARD):
            call(d)


def test_well_formed_sinkhorn_and_depth_gain(mhc):
    lg = synth.sinkhorn_logits(7, 4)
    with pytest.raises(ValueError, match=DEVICE_GUARD):
        mhc.mhc_sinkhorn_knopp(lg, 20, out=torch.empty_like(lg))
    with pytest.raises(ValueError, match=DEVICE_GUARD):
        mhc.mhc_depth_amax(torch.zeros(6, 3, 4, 4), out=(torch.empty(6), torch.empty(6)))
    with pytest.raises(ValueError, match=DEVICE_GUARD):
        mhc.mhc_depth_amax(torch.empty(6, 0, 4, 4))


def _short(t):
    """The same tensor one element short."""
    return t.reshape(-1)[:-1].clone()


def _retyped(t):
    return t.to(BF16 if t.dtype == F32 else F32)


# (entry point, argument, how it is spoiled, the name the error gives)
SPOILED = [
    ("pre", "phi", _short, "phi"),
    ("pre", "phi", _retyped, "phi"),
    ("pre", "b", _short, "b"),
    ("pre", "alpha", lambda t: torch.empty(0, dtype=F32), "alpha"),
    ("pre", "st", lambda t: torch.zeros(1, dtype=torch.int64), "dev_status"),
    ("post", "f_out", _short, "f_out"),
    ("post", "f_out", _retyped, "f_out"),
    ("post", "H_post", _short, "H_post"),
    ("post", "H_res", _short, "H_res"),
    ("post", "H_res", _retyped, "H_res"),
    ("backward", "grad_x_next", _short, "grad_x_next"),
    ("backward", "grad_h_in", _retyped, "grad_h_in"),
    ("backward", "f_out", _short, "f_out"),
    ("backward_noalloc", "grad_h_in", _short, "grad_h_in"),
    ("post_fused", "H_res", _short, "H_res"),
    ("post_fused", "phi", _short, "phi"),
    ("layer_input", "H_pre", _short, "H_pre"),
    ("post_backward", "grad_x_next", _short, "grad_x_next"),
    ("post_backward", "H_post", _retyped, "H_post"),
    ("pre_backward", "red", _short, "red"),
    ("pre_backward", "grad_h_in", _short, "grad_h_in"),
    ("backward_map", "grad_x_next", _retyped, "grad_x_next"),
    ("backward_apply", "phi", _short, "phi"),
    ("backward_apply", "grad_h_in", _short, "grad_h_in"),
]


@pytest.mark.parametrize("dtype", [F32, BF16], ids=["f32", "bf16"])
@pytest.mark.parametrize("call,arg,spoil,name", SPOILED,
                         ids=[f"{c}-{a}-{s.__name__}" for c, a, s, _ in SPOILED])
def test_spoiled_argument_is_named(mhc, dtype, call, arg, spoil, name):
    d = _args(4, dtype, 1)
    d[arg] = spoil(d[arg])
    with pytest.raises(ValueError, match=rf"^{name}: "):
        _calls(mhc, d, 1)[call](d)


def test_argument_on_another_device_is_named(mhc):
    d = _args(4, BF16, 1)
    d["f_out"] = torch.empty(T, C, dtype=BF16, device="meta")
    with pytest.raises(ValueError, match=r"^f_out: on meta"):
        _calls(mhc, d, 1)["post"](d)
    d = _args(4, BF16, 1)
    d["ws"] = torch.empty(256, dtype=torch.uint8, device="meta")
    with pytest.raises(ValueError, match=r"^workspace: on meta"):
        _calls(mhc, d, 1)["pre_out"](d)


@pytest.mark.parametrize("which", ["grad_x", "grad_phi", "grad_b", "grad_alpha", "grad_f_out"])
def test_short_backward_outputs_are_named(mhc, which):
    n, ag = 4, 3
    d = _args(n, BF16, ag)
    M = n * n + 2 * n
    out = dict(grad_x=torch.empty(T, n, C, dtype=BF16), grad_phi=torch.empty(n * C, M),
               grad_b=torch.empty(M), grad_alpha=torch.empty(3),
               grad_f_out=torch.empty(T, C, dtype=BF16))
    out[which] = _short(out[which])
    order = ("grad_x", "grad_phi", "grad_b", "grad_alpha", "grad_f_out")
    with pytest.raises(ValueError, match=rf"^{which}: "):
        mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"], d["grad_x_next"],
                         d["grad_h_in"], out=tuple(out[k] for k in order))
    with pytest.raises(ValueError, match=rf"^{which}: "):
        mhc.mhc_backward_apply(d["x"], d["phi"], d["grad_x_next"], d["grad_h_in"], d["ws"],
                               alpha_groups=ag, out=tuple(out[k] for k in order))


def test_sinkhorn_and_depth_gain_reject_other_types_and_short_outputs(mhc):
    lg = synth.sinkhorn_logits(7, 4)
    with pytest.raises(ValueError, match=r"^logits: dtype"):
        mhc.mhc_sinkhorn_knopp(lg.to(BF16), 20)
    with pytest.raises(ValueError, match=r"^out: "):
        mhc.mhc_sinkhorn_knopp(lg, 20, out=_short(lg))
    H = torch.zeros(6, 3, 4, 4)
    with pytest.raises(ValueError, match=r"^H: dtype"):
        mhc.mhc_depth_amax(H.double())
    with pytest.raises(ValueError, match=r"^gain_bwd: "):
        mhc.mhc_depth_amax(H, out=(torch.empty(6), torch.empty(5)))
