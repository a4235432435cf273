"""GPU parity at the workloads' full sizes (one layer or sampled units), in the same
launch configuration the library picks automatically.

rho4-prefill  T=4, 24 layers, H=16, d=128, r_k=96, r_v=160 (rho = 4), B=32, N=4096
deep-T32      T=32 loops, 8 layers, r 96/160 (rho = 32), B=16, N=4096
lla2d         LLA-2D: heads folded into one latent, T=4, 24 layers, r 64/128, B=16, N=4096
capacity      768 sequences x 4096 tokens x 24 layers resident (~116 GB of latents)
longctx       B=8, contexts uniform in [8192, 16384], 24 layers
"""
import numpy as np
import pytest
import torch

import decode_attention_12_b200 as lla
import lla_synth as S
from gpu_util import (assert_attn_close, oracle_decode, oracle_decode_units, run_decode, sample_units)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_rho4_layer_all_loops_fused():
    w = S.WORKLOADS["rho4-prefill"]
    layer = 7
    p = S.decode_inputs(w, layer, DEV)
    out, lse, st = run_decode(p, w, layer, 0, 4, 1.0)
    assert st == 0
    units = sample_units(w.B, w.H, 96, seed=1)
    o_ref, l_ref = oracle_decode_units(p, w, layer, 0, 4, 1.0, units)
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("Tq,t0", [(32, 0), (1, 0), (1, 31), (5, 11)])
def test_deep_recurrence_T32(Tq, t0):
    w = S.WORKLOADS["deep-T32"]
    layer = 3
    p = S.decode_inputs(w, layer, DEV, Tq=Tq)
    out, lse, st = run_decode(p, w, layer, t0, Tq, 1.0)
    assert st == 0
    units = sample_units(w.B, w.H, 24, seed=2)
    o_ref, l_ref = oracle_decode_units(p, w, layer, t0, Tq, 1.0, units)
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("Tq,t0", [(4, 0), (1, 2), (2, 1), (3, 1)])
def test_lla2d_folded_heads(Tq, t0):
    w = S.WORKLOADS["lla2d"]
    layer = 23
    p = S.decode_inputs(w, layer, DEV, Tq=Tq)
    out, lse, st = run_decode(p, w, layer, t0, Tq, 1.0)
    assert st == 0
    units = sample_units(w.B, w.H, 64, seed=3)
    o_ref, l_ref = oracle_decode_units(p, w, layer, t0, Tq, 1.0, units)
    assert_attn_close(out, lse, o_ref, l_ref)


def test_capacity_116GB_resident_first_and_last_layer():
    """All 24 layers of 768 x 4096 tokens resident; layers 0 and 23 hold drawn latents
    (the last one sits past 100 GB of planes, exercising 64-bit offsets)."""
    w = S.WORKLOADS["capacity-768x4k"]
    lat, _, _, _ = lla.cache_bytes(lla.make_dims(w.T, w.L, w.H, w.d, w.r_k, w.r_v), [4096] * 768)
    assert lat == 115_964_116_992
    p = S.decode_inputs(w, [0, w.L - 1], DEV)
    assert p["k"].numel() * 2 + p["v"].numel() * 2 == lat
    units = sample_units(w.B, w.H, 48, seed=4)
    for layer in (0, w.L - 1):
        out, lse, st = run_decode(p, w, layer, 0, 4, 1.0)
        assert st == 0
        o_ref, l_ref = oracle_decode_units(p, w, layer, 0, 4, 1.0, units)
        assert_attn_close(out, lse, o_ref, l_ref)


def test_long_context_8x16k_full_layer():
    w = S.WORKLOADS["longctx-8x16k"]
    layer = 11
    p = S.decode_inputs(w, layer, DEV)
    out, lse, st = run_decode(p, w, layer, 0, 4, 1.0)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, layer, 0, 4, 1.0)
    assert_attn_close(out, lse, o_ref, l_ref)


LLA2D_EDGE_LENS = [0, 1, 31, 64, 65, 255, 256, 257, 383, 384, 385, 1000, 4096]


@pytest.mark.parametrize("Tq,t0", [(4, 0), (1, 3)])
def test_lla2d_ragged_and_empty_contexts(Tq, t0):
    """LLA-2D with ragged contexts (empty, one token, tile and share boundaries +-1):
    every head of every sequence against the oracle; an empty context gives out = 0 and
    lse = -inf."""
    w = S.shrink(S.WORKLOADS["lla2d"], name="lla2d-edge", L=2, B=len(LLA2D_EDGE_LENS))
    layer = 1
    p = S.decode_inputs(w, layer, DEV, Tq=Tq, lens=LLA2D_EDGE_LENS, gap=3)
    out, lse, st = run_decode(p, w, layer, t0, Tq, 1.0)
    assert st == 0
    units = [(b, h) for b in range(w.B) for h in range(w.H)]
    o_ref, l_ref = oracle_decode_units(p, w, layer, t0, Tq, 1.0, units)
    assert_attn_close(out, lse, o_ref, l_ref)
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))
