"""Failure detection on the GPU without a fault: a kernel's bounded wait on a barrier that
nothing completes gives up, the status word reports LLA_ERR_DEVICE_TIMEOUT to the host, and
the context stays usable (a decode runs and matches the oracle afterwards)."""
import time

import pytest
import torch

import decode_attention_12_b200 as lla
import lla_synth as S
from gpu_util import assert_attn_close, oracle_decode, run_decode

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    lla.selftest_wait_timeout(ws)
    status = lla.status_fetch(ws)            # synchronises the stream
    waited = time.perf_counter() - t0
    assert status == lla.LLA_ERR_DEVICE_TIMEOUT
    assert 1.0 < waited < 30.0
    assert lla.status_fetch(ws) == 0         # fetched and cleared
    w = S.shrink(S.WORKLOADS["ouro1.4b-layer"], name="after-timeout", B=2, len_lo=50, len_hi=200)
    p = S.decode_inputs(w, 0, "cuda")
    out, lse, st = run_decode(p, w, 0, 0, 4, 1.0)
    assert st == 0
    o_ref, l_ref = oracle_decode(p, w, 0, 0, 4, 1.0)
    assert_attn_close(out, lse, o_ref, l_ref)
