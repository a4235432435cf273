"""GPU parity of the absorbed read with a decoupled rotary sub-key beside the latent (LLA
paper, Pith verdict record, desk-editor letter) against the fp64 oracle, which rebuilds
the keys instead of absorbing them.  The stored sub-keys are rotated on the host (fp64,
RoFormer's complex form) before upload; the library rotates the queries' rotary parts.

Cases: sub-key widths 32 and 64, both pairings, ragged contexts (empty, one token, tile
edges), query positions after and far past the context, a single loop query, fixed
split counts, and a full decode-step layer on sampled units.
"""
import numpy as np
import pytest

import decode_attention_12_b200 as lla
import lla_synth as S
from gpu_util import assert_attn_close, oracle_decode_units, run_decode_decoupled, stored_subkeys

pytestmark = pytest.mark.gpu
DEV = "cuda"
CTX_LENS = [0, 1, 31, 129, 700, 2048, 3000, 64]


def _case(w, lens, d_r, base, style, Tq, t0, q_pos, units_per_seq=3, num_splits=0, scale=1.0):
    layer = 1 if w.L > 1 else 0
    p = S.decode_inputs(w, layer, DEV, Tq=Tq, lens=lens, gap=3)
    raw = S.rope_subkeys(w, layer, p["slots"], d_r, DEV)
    k_rope = stored_subkeys(raw.cpu().numpy(), p["starts"], p["lens"], base, style, w.torch_dtype).to(DEV)
    plane = k_rope.new_zeros((w.L,) + tuple(k_rope.shape))
    plane[layer] = k_rope
    q_rope = S.rope_queries(w, len(lens), Tq, d_r, DEV)
    out, lse, st = run_decode_decoupled(p, w, layer, t0, Tq, scale, plane, q_rope, q_pos, base, style,
                                        num_splits=num_splits)
    assert st == 0
    heads = np.linspace(0, w.H - 1, units_per_seq).astype(int)
    units = [(b, int(h)) for b in range(len(lens)) for h in heads]
    o_ref, l_ref = oracle_decode_units(p, w, layer, t0, Tq, scale, units,
                                       decoupled=(k_rope.cpu(), q_rope.cpu(), np.asarray(q_pos), base, style))
    assert_attn_close(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("d_r,style", [(64, lla.ROPE_HALF), (32, lla.ROPE_INTERLEAVED)])
def test_decoupled_ragged(d_r, style):
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], L=2, B=len(CTX_LENS))
    _case(w, CTX_LENS, d_r, 10000.0, style, Tq=4, t0=0, q_pos=CTX_LENS)


@pytest.mark.parametrize("Tq,t0,ns", [(1, 2, 0), (3, 1, 5)])
def test_decoupled_loop_ranges_and_splits(Tq, t0, ns):
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], L=2, B=len(CTX_LENS))
    _case(w, CTX_LENS, 64, 500000.0, lla.ROPE_INTERLEAVED, Tq=Tq, t0=t0,
          q_pos=[n + 20000 for n in CTX_LENS], num_splits=ns, scale=0.7)


def test_decoupled_full_layer_sampled():
    w = S.WORKLOADS["ouro1.4b-layer"]
    lens = S.context_lengths(w)
    _case(w, lens, 64, 10000.0, lla.ROPE_HALF, Tq=4, t0=0, q_pos=lens, units_per_seq=1)


def test_decoupled_more_than_eight_loop_queries():
    """T = 12 loops, all 12 loop queries in one pass: the fragment rows g + 8 carry queries
    (the kernel's 16-row variant)."""
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name="dec-T12", T=12, L=2, B=len(CTX_LENS))
    _case(w, CTX_LENS, 32, 10000.0, lla.ROPE_HALF, Tq=12, t0=0, q_pos=CTX_LENS, units_per_seq=2)
