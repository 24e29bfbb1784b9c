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


def run_layers(inputs, x=None, n_layers=None):
    """The layer stack of a workload on its seeded inputs (or on ``x``)."""
    wl = inputs.workload
    cu, pos = sequence_args(wl)
    y = synth.to_f64(inputs.x, wl.dtype) if x is None else np.asarray(x, np.float64)
    pkv = None if inputs.prefix_kv is None else synth.to_f64(inputs.prefix_kv, wl.dtype)
    n = len(inputs.layers) if n_layers is None else n_layers
    for i in range(n):
        y = R.layer_forward(y, layer_f64(inputs, i), cu, pos, wl.heads, wl.head_dim,
                            wl.ln_eps, wl.rope_theta, pkv, wl.attn_only)
    return y


def run_workload(inputs, n_layers=None):
    """Stack, then the 2x2 merge where the workload has one."""
    y = run_layers(inputs, n_layers=n_layers)
    if inputs.workload.merge:
        y = R.spatial_merge_2x2(y, inputs.workload.grids)
    return y
