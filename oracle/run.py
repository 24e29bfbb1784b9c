"""Runs a seeded synthetic workload through the fp64 oracle.  TEST
INFRASTRUCTURE (tests/, smoke() and bench.py's CPU-baseline leg only).

Inputs come from ``synth`` (storage-rounded draws) and are widened exactly to
fp64; nothing is rounded after that.
"""
from __future__ import annotations

import numpy as np

import synth
from . import vit_ref as R


def layer_f64(inputs, i):
    """Layer i's parameters of a ``synth.Inputs`` widened to fp64."""
    dt = inputs.workload.dtype
    return {k: synth.to_f64(v, dt) for k, v in inputs.layers[i].items()}


def sequence_args(wl):
    cu, pos = R.positions_from_grids(wl.grids)
    return cu, (pos if wl.rope else None)


class _LazyLayers:
    """Layers ``[0, n)`` of a workload's inputs, each widened to fp64 only
    when the stack reaches it (27 fp64 layers of the 1152-wide model would
    hold 3.3 GB at once)."""

    def __init__(self, inputs, n):
        self.inputs, self.n = inputs, n

    def __len__(self):
        return self.n

    def __getitem__(self, i):
        if not 0 <= i < self.n:
            raise IndexError(i)
        return layer_f64(self.inputs, i)


def run_layers(inputs, x=None, n_layers=None):
    """The layer stack of a workload (``vit_ref.encoder_forward``) on its
    seeded inputs, or on ``x``."""
    wl = inputs.workload
    cu, pos = sequence_args(wl)
    y = synth.to_f64(inputs.x, wl.dtype) if x is None else np.asarray(x, np.float64)
    pkv = None if inputs.prefix_kv is None else synth.to_f64(inputs.prefix_kv, wl.dtype)
    n = len(inputs.layers) if n_layers is None else n_layers
    return R.encoder_forward(y, _LazyLayers(inputs, n), cu, pos, wl.heads, wl.head_dim,
                             wl.ln_eps, wl.rope_theta, pkv, wl.attn_only)


def run_workload(inputs, n_layers=None):
    """Stack, then the 2x2 merge where the workload has one."""
    y = run_layers(inputs, n_layers=n_layers)
    if inputs.workload.merge:
        y = R.spatial_merge_2x2(y, inputs.workload.grids)
    return y
