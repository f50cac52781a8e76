"""A stack of mHC layers with block recompute, backward in training order.

Layer l maps the stream x_l [T,n,C] to x_{l+1} through the library's calls:

    h_in_l, H_pre, H_post, H_res = mhc_pre(x_l, phi_l, b_l, alpha_l)
    f_out_l = F(l, h_in_l)                              (the wrapped layer)
    x_{l+1} = mhc_post(x_l, f_out_l, H_post, H_res)

and back, in the order the chain rule needs (G = grad of x_{l+1}):

    grad_f_out, red = mhc_post_backward(x_l, f_out_l, H_post, G)
    grad_h_in = F_backward(l, h_in_l, f_out_l, grad_f_out)
    grad_x_l, grad_phi_l, grad_b_l, grad_alpha_l =
        mhc_pre_backward(x_l, phi_l, b_l, alpha_l, G, grad_h_in, red)

Recompute (reportify.cn mHC summary, [21]): the forward keeps only the input
stream of each block of consecutive layers and drops every other
intermediate; the backward rebuilds one block at a time, last block first.
The block size comes from ``mhc_recompute_plan`` ([22]: the block that makes
the total memory smallest; the cost it minimises is stated in include/mhc.h).

The schedule is a plain list of steps (``schedule``) that ``DepthStack``
executes; a test replays the same list to count resident memory.  All
arithmetic of the mHC layer runs in libmhc.so; F and F_backward are the
caller's.
"""
from __future__ import annotations

from typing import Callable, Sequence

from .api import mhc_post, mhc_post_backward, mhc_pre, mhc_pre_backward, mhc_recompute_plan


def recompute_blocks(L: int, block: int) -> list[tuple[int, int]]:
    """Cut layers 0..L-1 into [l0, l1) blocks of at most ``block`` layers.  The first
    block takes the remainder, so the last block (rebuilt while every other block's
    input is still held) is a full one."""
    if L < 1 or block < 1:
        raise ValueError("L and block must be >= 1")
    block = min(block, L)
    first = L % block or block
    bounds = [(0, first)]
    while bounds[-1][1] < L:
        l0 = bounds[-1][1]
        bounds.append((l0, l0 + block))
    return bounds


def schedule(L: int, block: int) -> tuple[list[tuple], list[tuple]]:
    """(forward steps, backward steps) of an L-layer stack with the given block size.

    forward : ("forward", l, keep) -- run layer l; keep its input x_l when it starts a block
    backward: ("recompute", l, nxt) -- rerun layer l of the block being rebuilt, holding
                                       h_in_l, f_out_l and H_post_l, and x_{l+1} when nxt
                                       (l + 1 lies inside the block)
              ("backward", l)      -- layer l's backward; drops what recompute l held
              ("release", l0)      -- drop the kept input of the block that starts at l0
    """
    blocks = recompute_blocks(L, block)
    starts = {l0 for l0, _ in blocks}
    fwd = [("forward", l, l in starts) for l in range(L)]
    bwd: list[tuple] = []
    for l0, l1 in reversed(blocks):
        bwd += [("recompute", l, l + 1 < l1) for l in range(l0, l1)]
        bwd += [("backward", l) for l in reversed(range(l0, l1))]
        bwd.append(("release", l0))
    return fwd, bwd


class DepthStack:
    """L mHC layers around caller-supplied layer functions.

    layers     : per layer a dict with CUDA tensors ``phi`` [nC, n^2+2n] fp32, ``b``
                 [n^2+2n] fp32 and ``alpha`` [1] or [3] fp32
    F          : F(l, h_in [T,C]) -> f_out [T,C]; it is called again for the layers
                 being rebuilt and must give the same result both times
    F_backward : F_backward(l, h_in, f_out, grad_f_out) -> grad_h_in [T,C]
    block      : recompute block size; None takes ``mhc_recompute_plan``'s
    """

    def __init__(self, layers: Sequence[dict], F: Callable, F_backward: Callable,
                 n: int, block: int | None = None, t_max: int = 20, eps: float = 1e-6):
        self.layers = list(layers)
        self.L = len(self.layers)
        self.F, self.F_backward = F, F_backward
        self.t_max, self.eps = t_max, eps
        self.block = mhc_recompute_plan(n, self.L)[0] if block is None else int(block)
        self.fwd_steps, self.bwd_steps = schedule(self.L, self.block)
        self.kept: dict[int, object] = {}

    def _pre(self, l, x):
        p = self.layers[l]
        return mhc_pre(x, p["phi"], p["b"], p["alpha"], t_max=self.t_max, eps=self.eps)

    def forward(self, x0):
        """x_L.  Keeps the input stream of every block for ``backward``."""
        self.kept = {}
        x = x0
        for _, l, keep in self.fwd_steps:
            if keep:
                self.kept[l] = x
            h_in, _, H_post, H_res = self._pre(l, x)
            f_out = self.F(l, h_in)
            x = mhc_post(x, f_out, H_post, H_res)
        return x

    def backward(self, grad_xL):
        """(grad_x0, [(grad_phi_l, grad_b_l, grad_alpha_l) for l in 0..L-1]).  Needs the
        inputs kept by the last ``forward``; releases them as it goes."""
        if len(self.kept) != len(recompute_blocks(self.L, self.block)):
            raise RuntimeError("DepthStack.backward needs a forward first")
        grads: list = [None] * self.L
        xs: dict[int, object] = {}
        held: dict[int, tuple] = {}
        G = grad_xL
        for step in self.bwd_steps:
            kind, l = step[0], step[1]
            if kind == "recompute":
                x = self.kept[l] if l in self.kept else xs[l]
                xs[l] = x
                h_in, _, H_post, H_res = self._pre(l, x)
                f_out = self.F(l, h_in)
                held[l] = (h_in, f_out, H_post)
                if step[2]:
                    xs[l + 1] = mhc_post(x, f_out, H_post, H_res)
            elif kind == "backward":
                h_in, f_out, H_post = held.pop(l)
                x = xs.pop(l)
                p = self.layers[l]
                grad_f_out, red = mhc_post_backward(x, f_out, H_post, G)
                grad_h_in = self.F_backward(l, h_in, f_out, grad_f_out)
                gx, gphi, gb, ga = mhc_pre_backward(x, p["phi"], p["b"], p["alpha"], G,
                                                    grad_h_in, red, t_max=self.t_max,
                                                    eps=self.eps)
                grads[l] = (gphi, gb, ga)
                del h_in, f_out, H_post, x, grad_f_out, red, grad_h_in
                G = gx
            else:
                del self.kept[l]
        return G, grads
