"""GPU parity: the reconstruct-on-read decode (K_hat, V_hat rebuilt per tile on tensor
cores) against the fp64 oracle's reconstruct form, and against the absorbed form."""
import numpy as np
import pytest
import torch

import decode_attention_12_b200 as lla
import lla_synth as S
from gpu_util import assert_attn_close, attn_errors, oracle_decode, oracle_decode_units, run_decode

pytestmark = pytest.mark.gpu
DEV = "cuda"
REC = lla.RECONSTRUCT


def test_reconstruct_ouro_layer_all_loops():
    w = S.WORKLOADS["ouro1.4b-layer"]
    p = S.decode_inputs(w, 0, DEV)
    out, lse, st = run_decode(p, w, 0, 0, 4, 1.0, variant=REC)
    assert st == 0
    units = [(b, h) for b in range(0, 64, 3) for h in range(16)]
    o_ref, l_ref = oracle_decode_units(p, w, 0, 0, 4, 1.0, units, variant="reconstruct")
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("Tq,t0", [(4, 0), (1, 3), (2, 1)])
def test_reconstruct_equals_absorb_on_gpu(Tq, t0):
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name="rec-abs", B=8, len_lo=100, len_hi=3000)
    p = S.decode_inputs(w, 0, DEV, Tq=Tq, perturb=0.2)
    a = run_decode(p, w, 0, t0, Tq, 1.0, variant=lla.ABSORB)
    r = run_decode(p, w, 0, t0, Tq, 1.0, variant=REC)
    assert a[2] == 0 and r[2] == 0
    o_ref, l_ref = oracle_decode(p, w, 0, t0, Tq, 1.0, variant="reconstruct")
    assert_attn_close(r[0], r[1], o_ref, l_ref)
    max_abs, rel = attn_errors(r[0], a[0].double().cpu().numpy())
    assert max_abs <= 1e-2 and rel <= 5e-3


def test_reconstruct_ragged_edges_match_oracle():
    lens = [0, 1, 2, 31, 255, 257, 1000, 4097]
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name="rec-edge2", B=len(lens))
    p = S.decode_inputs(w, 0, DEV, lens=lens, gap=3)
    out, lse, st = run_decode(p, w, 0, 0, 4, 1.0, variant=REC)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 4, 1.0, variant="reconstruct")
    assert_attn_close(out, lse, o_ref, l_ref)
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


@pytest.mark.parametrize("variant", [lla.ABSORB, lla.RECONSTRUCT])
def test_lla2d_small_rank_both_variants(variant):
    w = S.shrink(S.WORKLOADS["lla2d"], name="2d-small", L=1, H=4, r_k=16, r_v=32, B=5,
                 len_lo=50, len_hi=1500)
    p = S.decode_inputs(w, 0, DEV)
    out, lse, st = run_decode(p, w, 0, 0, 4, 1.0, variant=variant)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 4, 1.0, variant="reconstruct")
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("Tq,t0", [(6, 1), (5, 0)])
def test_reconstruct_more_loop_queries_than_one_latent_pass(Tq, t0):
    """Eight loops: a call with 5 or 6 loop queries reads the latents in two passes (4 + the
    rest); both passes' records meet in the one combine."""
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name="rec-T8", T=8, B=6, len_lo=200, len_hi=2500)
    p = S.decode_inputs(w, 0, DEV, Tq=Tq, perturb=0.1)
    out, lse, st = run_decode(p, w, 0, t0, Tq, 1.0, variant=REC)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, t0, Tq, 1.0, variant="reconstruct")
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("rk,rv", [(16, 32), (32, 32), (16, 16)])
def test_reconstruct_large_logits_and_ranks(rk, rv):
    """Softmax scale 30: sharp rows stress the running max and the precision of the rebuilt
    keys (W_up enters the tensor cores as bf16 hi + lo parts)."""
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name=f"rec-big-{rk}-{rv}", r_k=rk, r_v=rv, B=5,
                 len_lo=130, len_hi=2100)
    p = S.decode_inputs(w, 0, DEV)
    out, lse, st = run_decode(p, w, 0, 0, 4, 30.0, variant=REC)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 4, 30.0, variant="reconstruct")
    assert_attn_close(out, lse, o_ref, l_ref)
