"""GPU parity of the codec fit (SVD initialisation; LLA review page, What carries the
argument) against the fp64 oracle (numpy SVD) on the same stored calibration tokens.

Compared: mu (fp32 store), the r leading singular values, and every column of W_up (fp32)
and W_down (bf16 store) under the shared sign convention.  Eigenvector sensitivity is
about eps * lambda_max / gap, so each column's bound adds 1e-12 * lambda_max / gap_j to the
fp32 rounding (lambda = sigma^2, gap_j = distance to the nearest other eigenvalue).
Cases: per-head ranks 16/32 and 96/160 (two layers), LLA-2D (W = 8192), and a small
calibration set (n = 64).
"""
import numpy as np
import pytest
import torch

import decode_attention_12_b200 as lla
import lla_synth as S
import oracle
from gpu_util import dims_of, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fit(w, layer0, n_layers, n_cal):
    layers = list(range(layer0, layer0 + n_layers))
    dims = dims_of(w)
    Hs, Dp = w.heads_stored, w.d * (w.H if w.fold2d else 1)
    xs = {ax: torch.stack([S.draw_encode_tokens(w, l, ax, n_cal, DEV, seed_tag="calib") for l in layers])
          for ax in ("k", "v")}
    out = {}
    for ax, r in (("k", w.r_k), ("v", w.r_v)):
        out[f"W_down_{ax}"] = torch.full((w.L, Hs, r, w.W), float("nan"), dtype=w.torch_dtype, device=DEV)
        out[f"W_up_{ax}"] = torch.full((w.L, Hs, w.T, r, Dp), float("nan"), device=DEV)
        out[f"mu_{ax}"] = torch.full((w.L, Hs, w.T, Dp), float("nan"), device=DEV)
        out[f"sigma_{ax}"] = torch.full((n_layers, Hs, n_cal), float("nan"), device=DEV)
    codec = lla.make_codec(W_down_k=out["W_down_k"], W_down_v=out["W_down_v"], W_up_k=out["W_up_k"],
                           W_up_v=out["W_up_v"], mu_k=out["mu_k"], mu_v=out["mu_v"])
    wsb = lla.codec_fit_workspace_bytes(dims, n_layers, n_cal)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=DEV)
    lla.codec_fit(dims, layer0, n_layers, xs["k"], xs["v"], n_cal, codec, ws, wsb,
                  sigma_k=out["sigma_k"], sigma_v=out["sigma_v"])
    torch.cuda.synchronize()
    assert lla.status_fetch(ws) == 0, "Jacobi sweeps did not converge"
    for li, l in enumerate(layers):
        for ax, r in (("k", w.r_k), ("v", w.r_v)):
            x = to64(xs[ax][li])
            for hs in range(Hs):
                xr = x.reshape(n_cal, -1) if w.fold2d else x[:, :, hs, :].reshape(n_cal, -1)
                mu, Wd, Wu, sigma = oracle.codec_fit(xr, r, w.T)
                np.testing.assert_allclose(to64(out[f"mu_{ax}"][l, hs]).reshape(-1), mu, rtol=1e-6,
                                           atol=1e-6 * np.abs(mu).max())
                s_gpu = to64(out[f"sigma_{ax}"][li, hs])
                np.testing.assert_allclose(s_gpu[:r], sigma[:r], rtol=2e-6)
                lam = sigma ** 2
                gap = np.array([min(lam[j - 1] - lam[j] if j > 0 else np.inf, lam[j] - lam[j + 1])
                                for j in range(r)])
                tol = 2e-6 + 1e-12 * lam[0] / gap                       # per column
                wu = to64(out[f"W_up_{ax}"][l, hs])                      # [T, r, Dp]
                err_up = np.abs(wu - Wu).max(axis=(0, 2))
                assert np.all(err_up <= tol), f"W_up column errors {err_up[err_up > tol]} > {tol[err_up > tol]}"
                wd = to64(out[f"W_down_{ax}"][l, hs])                    # [r, W]
                if w.dtype == "bf16":  # stored in bf16: one rounding of the reference
                    ref = to64(torch.as_tensor(Wd.T).to(torch.bfloat16))
                    err_dn = np.abs(wd - ref).max(axis=1)
                    assert np.all(err_dn <= 2.0 ** -8 * np.abs(Wd.T).max(axis=1) + tol)
                else:
                    assert np.all(np.abs(wd - Wd.T).max(axis=1) <= tol)


def test_fit_per_head_small_ranks():
    _fit(S.WORKLOADS["ouro1.4b-layer"], 0, 1, 256)


def test_fit_per_head_large_ranks_two_layers():
    _fit(S.shrink(S.WORKLOADS["rho4-prefill"], L=4), 2, 2, 256)


def test_fit_lla2d_wide_stack():
    _fit(S.shrink(S.WORKLOADS["lla2d"], L=2), 1, 1, 256)


def test_fit_small_calibration_set():
    _fit(S.WORKLOADS["ouro1.4b-layer"], 0, 1, 64)


def test_fit_fp32_storage():
    """fp32 tokens and W_down (the tiny workload: T = 4, H = 2, d = 64, ranks 8/16)."""
    _fit(S.WORKLOADS["tiny-fp32"], 0, 1, 128)
