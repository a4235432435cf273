"""Seeded synthetic inputs for the LLA decode/encode path (shared by tests, bench, oracle checks).

This module draws inputs only.  It computes none of the path's arithmetic: no
encode, no reconstruction, no attention.  Both the CUDA path and the CPU oracle
receive the arrays it produces; neither imports the other.

Recipe (stand-in for the teacher activations of the pages' Ouro/Huginn models,
whose weights are not available):

* K/V trajectories ("Looped Latent Attention ...", Pith review page, Core claim
  and Figure 2: one direction carries about 60 % of the cross-loop energy):
  for each (workload, layer, head-or-fold, axis) a stacked token vector
  ``x = mu_gen + sum_j z_j a_j + 0.1 * eps`` in R^W (W = T*d, or T*H*d for
  LLA-2D), with J = 16 orthonormal directions u_j (QR of a seeded Gaussian),
  energy fractions e_1 = 0.60 and e_j proportional to 2^-(j-2) (j >= 2) summing to
  0.40, a_j = sqrt(e_j * W) u_j (mean per-element signal variance 1),
  mu_gen ~ N(0, 1) per element, z ~ N(0, 1), eps ~ N(0, 1) (noise variance 0.01).
* Codec initialisation (same page, "What carries the argument": the codec is
  initialised from the top right singular vectors of teacher activations):
  256 calibration tokens from the same model; mu = their mean; W_down = top-r
  right singular vectors of the centred calibration matrix; W_up,t = transpose of
  the loop-t row block of W_down; mu_t = loop-t slice of mu.  A numpy SVD is the
  one library step.  Optionally the up-projections are perturbed, because a
  distilled codec need not have W_up equal to W_down^T.
* Decode-time cache contents: the cached latents are drawn directly with the
  statistics an SVD codec gives to fresh trajectory tokens: independent
  N(0, sigma_j^2 / n_cal) per latent dimension j (sigma_j = calibration singular
  values).  Queries q ~ N(0, 1) / sqrt(d).  Context lengths uniform inclusive.
* Encode inputs: trajectory tokens laid out [n_tok][T][H][d] (loop-major, as a
  looped model produces them loop by loop).
* Decoupled rotary sub-keys (LLA paper, Pith verdict record, desk-editor letter):
  raw sub-keys N(0, 1) per (layer, head, slot) and rotary query parts N(0, 1) / sqrt(d),
  drawn here unrotated; the tests rotate the stored sub-keys at their positions.
* Hybrid-window inputs ("Hybrid Latent Attention for Looped Language Models",
  abstract: exact keys and values of the most recent tokens): fresh trajectory
  tokens of the same model, drawn as encode inputs and laid out per window row,
  [B][H][T][w_max][d] per layer and axis; rows in use per sequence uniform in
  [0, w_max] unless given.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Optional

import numpy as np
import torch

N_DIRECTIONS = 16
TOP_ENERGY = 0.60
NOISE_STD = 0.1
N_CALIB = 256


# ---------------------------------------------------------------------------
# Workloads (shapes of the pages' Ouro/Huginn settings; all synthetic)
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    L: int
    H: int
    d: int
    r_k: int
    r_v: int
    B: int
    len_lo: int
    len_hi: int
    dtype: str = "bf16"          # storage type of latents, queries, outputs
    fold2d: bool = False         # LLA-2D: heads folded into one latent

    @property
    def W(self) -> int:
        """Width of one stacked (token, head-or-fold) vector."""
        return self.T * self.d * (self.H if self.fold2d else 1)

    @property
    def heads_stored(self) -> int:
        return 1 if self.fold2d else self.H

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny-fp32", T=4, L=1, H=2, d=64, r_k=8, r_v=16, B=1,
                 len_lo=64, len_hi=64, dtype="f32"),
        Workload("ouro1.4b-layer", T=4, L=1, H=16, d=128, r_k=16, r_v=32, B=64,
                 len_lo=2048, len_hi=4096),
        Workload("rho4-prefill", T=4, L=24, H=16, d=128, r_k=96, r_v=160, B=32,
                 len_lo=4096, len_hi=4096),
        Workload("capacity-768x4k", T=4, L=24, H=16, d=128, r_k=16, r_v=32, B=768,
                 len_lo=4096, len_hi=4096),
        Workload("longctx-8x16k", T=4, L=24, H=16, d=128, r_k=16, r_v=32, B=8,
                 len_lo=8192, len_hi=16384),
        Workload("deep-T32", T=32, L=8, H=16, d=128, r_k=96, r_v=160, B=16,
                 len_lo=4096, len_hi=4096),
        Workload("lla2d", T=4, L=24, H=16, d=128, r_k=64, r_v=128, B=16,
                 len_lo=4096, len_hi=4096, fold2d=True),
    ]
}


def shrink(w: Workload, **kw) -> Workload:
    """Copy of a workload with some fields replaced (smaller test cases)."""
    return dataclasses.replace(w, **kw)


# ---------------------------------------------------------------------------
# Seeds
# ---------------------------------------------------------------------------
def seed_of(*parts) -> int:
    """Stable 63-bit seed from any tuple of names and integers."""
    h = hashlib.blake2b("/".join(str(p) for p in parts).encode(), digest_size=8)
    return int.from_bytes(h.digest(), "little") & ((1 << 63) - 1)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


# ---------------------------------------------------------------------------
# Trajectory model and SVD codec initialisation
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class TrajectoryModel:
    A: np.ndarray        # [J, W] scaled directions a_j
    mu_gen: np.ndarray   # [W]

    @property
    def W(self) -> int:
        return self.A.shape[1]


def energy_fractions(J: int = N_DIRECTIONS) -> np.ndarray:
    tail = np.array([2.0 ** -(j - 2) for j in range(2, J + 1)])
    tail = tail / tail.sum() * (1.0 - TOP_ENERGY)
    return np.concatenate([[TOP_ENERGY], tail])


def trajectory_model(seed: int, W: int, J: int = N_DIRECTIONS) -> TrajectoryModel:
    rng = np.random.default_rng(seed)
    G = rng.standard_normal((W, J))
    Q, _ = np.linalg.qr(G)
    e = energy_fractions(J)
    A = (np.sqrt(e * W)[:, None] * Q.T)
    mu_gen = rng.standard_normal(W)
    return TrajectoryModel(A=A, mu_gen=mu_gen)


def draw_tokens_np(model: TrajectoryModel, n: int, seed: int) -> np.ndarray:
    """n stacked token vectors in fp64 (host)."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((n, model.A.shape[0]))
    eps = rng.standard_normal((n, model.W))
    return model.mu_gen[None, :] + z @ model.A + NOISE_STD * eps


@dataclasses.dataclass
class Codec:
    """SVD-initialised codec of one (layer, head-or-fold, axis)."""
    W_down: np.ndarray   # [W, r]
    mu: np.ndarray       # [W]
    sigma: np.ndarray    # calibration singular values (all of them)
    W_up: np.ndarray     # [T, r, W/T]  per-loop up-projections
    T: int

    @property
    def r(self) -> int:
        return self.W_down.shape[1]

    def mu_t(self) -> np.ndarray:
        return self.mu.reshape(self.T, -1)

    def latent_std(self, n_cal: int = N_CALIB) -> np.ndarray:
        return self.sigma[: self.r] / math.sqrt(n_cal)


def fit_codec(x_cal: np.ndarray, r: int, T: int, perturb: float = 0.0,
              seed: Optional[int] = None) -> Codec:
    """SVD initialisation from calibration tokens x_cal [n_cal, W] (fp64)."""
    mu = x_cal.mean(axis=0)
    _, S, Vt = np.linalg.svd(x_cal - mu[None, :], full_matrices=False)
    if r > Vt.shape[0]:
        raise ValueError("rank exceeds the calibration rank")
    W_down = Vt[:r].T.copy()
    W = W_down.shape[0]
    W_up = W_down.reshape(T, W // T, r).transpose(0, 2, 1).copy()
    if perturb:
        rng = np.random.default_rng(seed)
        W_up = W_up + perturb * rng.standard_normal(W_up.shape) / math.sqrt(r)
    return Codec(W_down=W_down, mu=mu, sigma=S, W_up=W_up, T=T)


def orthonormal_codec(W: int, T: int, seed: int, mu_scale: float = 1.0) -> Codec:
    """Full-rank codec: random orthonormal W_down (r = W), W_up,t its loop blocks^T."""
    rng = np.random.default_rng(seed)
    Q, _ = np.linalg.qr(rng.standard_normal((W, W)))
    mu = mu_scale * rng.standard_normal(W)
    W_up = Q.reshape(T, W // T, W).transpose(0, 2, 1).copy()
    return Codec(W_down=Q, mu=mu, sigma=np.ones(W), W_up=W_up, T=T)


def layer_codecs(w: Workload, layer: int, perturb: float = 0.0):
    """Codecs of one layer: list over stored heads of (codec_K, codec_V)."""
    out = []
    for h in range(w.heads_stored):
        pair = []
        for axis, r in (("K", w.r_k), ("V", w.r_v)):
            s = seed_of(w.name, layer, h, axis)
            model = trajectory_model(s, w.W)
            x_cal = draw_tokens_np(model, N_CALIB, seed_of(w.name, layer, h, axis, "calib"))
            pair.append(fit_codec(x_cal, r, w.T, perturb=perturb,
                                  seed=seed_of(w.name, layer, h, axis, "perturb")))
        out.append(tuple(pair))
    return out


# ---------------------------------------------------------------------------
# Device-layout codec tensors of one layer (what the library receives)
# ---------------------------------------------------------------------------
def codec_tensors(w: Workload, codecs, device) -> dict:
    """Stack the per-head codecs of one layer into the library's layouts.

    W_down_{k,v}: [H', r, W]      (W_down transposed; storage dtype bf16 or f32)
    W_up_{k,v}:   per-head [H, T, r, d];  LLA-2D [T, r, H*d]   (fp32)
    mu_{k,v}:     per-head [H, T, d];     LLA-2D [T, H*d]      (fp32)
    """
    Wd_dtype = torch.float32 if w.dtype == "f32" else torch.bfloat16
    res = {}
    for ai, ax in enumerate(("k", "v")):
        Wd = np.stack([c[ai].W_down.T for c in codecs])          # [H', r, W]
        Wu = np.stack([c[ai].W_up for c in codecs])              # [H', T, r, W/T]
        mu = np.stack([c[ai].mu_t() for c in codecs])            # [H', T, W/T]
        if w.fold2d:
            Wu, mu = Wu[0], mu[0]
        res[f"W_down_{ax}"] = torch.from_numpy(Wd).to(Wd_dtype).to(device).contiguous()
        res[f"W_up_{ax}"] = torch.from_numpy(Wu).float().to(device).contiguous()
        res[f"mu_{ax}"] = torch.from_numpy(mu).float().to(device).contiguous()
    return res


# ---------------------------------------------------------------------------
# Decode-time inputs: lengths, latent planes, queries
# ---------------------------------------------------------------------------
def context_lengths(w: Workload, seed_tag="lens") -> np.ndarray:
    rng = np.random.default_rng(seed_of(w.name, seed_tag))
    return rng.integers(w.len_lo, w.len_hi + 1, size=w.B).astype(np.int32)


def slot_starts(lens: np.ndarray, gap: int = 0) -> np.ndarray:
    """Exclusive prefix sum of lengths (+ optional unused gap between sequences)."""
    starts = np.zeros(len(lens), dtype=np.int64)
    if len(lens) > 1:
        starts[1:] = np.cumsum(lens[:-1].astype(np.int64) + gap)
    return starts


def draw_latents(n_slots: int, std: np.ndarray, seed: int, device, dtype) -> torch.Tensor:
    """[n_slots, r] latents, dimension j ~ N(0, std_j^2), rounded to ``dtype``."""
    g = _gen(device, seed)
    z = torch.randn(n_slots, len(std), generator=g, device=device, dtype=torch.float32)
    s = torch.as_tensor(np.asarray(std, dtype=np.float32), device=device)
    return (z * s).to(dtype)


def draw_queries(B: int, Tq: int, H: int, d: int, seed: int, device, dtype) -> torch.Tensor:
    g = _gen(device, seed)
    q = torch.randn(B, Tq, H, d, generator=g, device=device, dtype=torch.float32)
    return (q / math.sqrt(d)).to(dtype)


def draw_layer_cache(w: Workload, layer: int, codecs, n_slots: int, device,
                     out_k: Optional[torch.Tensor] = None,
                     out_v: Optional[torch.Tensor] = None):
    """Latent planes of one layer: k [H', n_slots, r_k], v [H', n_slots, r_v]."""
    Hs = w.heads_stored
    if out_k is None:
        out_k = torch.empty(Hs, n_slots, w.r_k, dtype=w.torch_dtype, device=device)
    if out_v is None:
        out_v = torch.empty(Hs, n_slots, w.r_v, dtype=w.torch_dtype, device=device)
    for h in range(Hs):
        ck, cv = codecs[h]
        out_k[h].copy_(draw_latents(n_slots, ck.latent_std(), seed_of(w.name, layer, h, "cK"),
                                    device, w.torch_dtype))
        out_v[h].copy_(draw_latents(n_slots, cv.latent_std(), seed_of(w.name, layer, h, "cV"),
                                    device, w.torch_dtype))
    return out_k, out_v


# ---------------------------------------------------------------------------
# Encode inputs: trajectory tokens in the [n_tok, T, H, d] layout
# ---------------------------------------------------------------------------
def draw_encode_tokens(w: Workload, layer: int, axis: str, n_tok: int, device,
                       seed_tag="tokens", chunk: int = 1 << 16) -> torch.Tensor:
    """Trajectory tokens of one layer and axis, [n_tok, T, H, d] in ``w.dtype``.

    Per head (or for the fold) the stacked vector is mu_gen + z A + 0.1 eps,
    computed in fp64 on ``device`` and rounded once to the storage type.
    """
    T, H, d = w.T, w.H, w.d
    out = torch.empty(n_tok, T, H, d, dtype=w.torch_dtype, device=device)
    for hs in range(w.heads_stored):
        model = trajectory_model(seed_of(w.name, layer, hs, axis.upper()), w.W)
        A = torch.from_numpy(model.A).to(device)
        mu = torch.from_numpy(model.mu_gen).to(device)
        g = _gen(device, seed_of(w.name, layer, hs, axis.upper(), seed_tag))
        for a in range(0, n_tok, chunk):
            b = min(n_tok, a + chunk)
            z = torch.randn(b - a, A.shape[0], generator=g, device=device, dtype=torch.float64)
            eps = torch.randn(b - a, w.W, generator=g, device=device, dtype=torch.float64)
            x = mu[None, :] + z @ A + NOISE_STD * eps
            if w.fold2d:
                out[a:b] = x.view(b - a, T, H, d).to(w.torch_dtype)
            else:
                out[a:b, :, hs, :] = x.view(b - a, T, d).to(w.torch_dtype)
    return out


# ---------------------------------------------------------------------------
# Everything one decode call needs, in the library's device layouts
# ---------------------------------------------------------------------------
def decode_inputs(w: Workload, layers, device, Tq: Optional[int] = None, lens=None, gap: int = 0,
                  perturb: float = 0.0, q_tag="q") -> dict:
    """Draw the latent cache, codec and queries for ``layers`` of workload ``w``.

    Returns device tensors in the library layouts (see include/lla.h):
      k, v        [L][H'][slots][r]      latents (layers not listed stay zero)
      W_up_k/v    [L][H'][T][r][D']      fp32;  mu_k/v [L][H'][T][D'] fp32
      W_down_k/v  [L][H'][r][W]          storage dtype
      seq_start   int64 [B], ctx_lens int32 [B]
      q           [B][Tq][H][d]          storage dtype
    plus host copies ``lens`` / ``starts`` and the fitted ``codecs`` per layer.
    """
    if isinstance(layers, int):
        layers = [layers]
    Tq = w.T if Tq is None else Tq
    lens = context_lengths(w) if lens is None else np.asarray(lens, dtype=np.int32)
    starts = slot_starts(lens, gap)
    slots = int(starts[-1] + lens[-1] + gap) if len(lens) else 1
    slots = max(slots, 1)
    Hs, T, Dp = w.heads_stored, w.T, w.d * (w.H if w.fold2d else 1)
    dt = w.torch_dtype
    out = {
        "k": torch.zeros(w.L, Hs, slots, w.r_k, dtype=dt, device=device),
        "v": torch.zeros(w.L, Hs, slots, w.r_v, dtype=dt, device=device),
        "W_up_k": torch.zeros(w.L, Hs, T, w.r_k, Dp, dtype=torch.float32, device=device),
        "W_up_v": torch.zeros(w.L, Hs, T, w.r_v, Dp, dtype=torch.float32, device=device),
        "mu_k": torch.zeros(w.L, Hs, T, Dp, dtype=torch.float32, device=device),
        "mu_v": torch.zeros(w.L, Hs, T, Dp, dtype=torch.float32, device=device),
        "W_down_k": torch.zeros(w.L, Hs, w.r_k, w.W, dtype=dt, device=device),
        "W_down_v": torch.zeros(w.L, Hs, w.r_v, w.W, dtype=dt, device=device),
        "seq_start": torch.as_tensor(starts, dtype=torch.int64, device=device),
        "ctx_lens": torch.as_tensor(lens, dtype=torch.int32, device=device),
        "lens": lens, "starts": starts, "slots": slots, "codecs": {},
    }
    for layer in layers:
        codecs = layer_codecs(w, layer, perturb=perturb)
        out["codecs"][layer] = codecs
        ct = codec_tensors(w, codecs, device)
        for name in ("W_up_k", "W_up_v", "mu_k", "mu_v", "W_down_k", "W_down_v"):
            src = ct[name]
            if w.fold2d and name.startswith(("W_up", "mu")):
                src = src.unsqueeze(0)
            out[name][layer].copy_(src)
        draw_layer_cache(w, layer, codecs, slots, device, out_k=out["k"][layer], out_v=out["v"][layer])
    out["q"] = draw_queries(w.B, Tq, w.H, w.d, seed_of(w.name, q_tag, Tq), device, dt)
    return out


# ---------------------------------------------------------------------------
# Hybrid form: exact window rows of every sequence
# ---------------------------------------------------------------------------
def window_lengths(B: int, w_max: int, seed_tag="win_len") -> np.ndarray:
    rng = np.random.default_rng(seed_of("window", B, w_max, seed_tag))
    return rng.integers(0, w_max + 1, size=B).astype(np.int32)


def window_inputs(w: Workload, layers, B: int, w_max: int, device, win_lens=None,
                  seed_tag="window") -> dict:
    """Exact window keys / values in the library layout [L][B][H][T][w_max][d].

    Rows of a layer are trajectory tokens of that layer's K (V) model (the tokens a
    looped model would emit), one token per (sequence, row); layers not listed stay
    zero.  Returns device tensors ``win_k``, ``win_v``, ``win_len`` (int32 [B]) and the
    host copy ``win_lens``.
    """
    if isinstance(layers, int):
        layers = [layers]
    win_lens = window_lengths(B, w_max) if win_lens is None else np.asarray(win_lens, dtype=np.int32)
    shape = (w.L, B, w.H, w.T, w_max, w.d)
    out = {"win_k": torch.zeros(shape, dtype=w.torch_dtype, device=device),
           "win_v": torch.zeros(shape, dtype=w.torch_dtype, device=device),
           "win_len": torch.as_tensor(win_lens, dtype=torch.int32, device=device),
           "win_lens": win_lens, "w_max": w_max}
    if B * w_max == 0:
        return out
    for layer in layers:
        for axis, name in (("k", "win_k"), ("v", "win_v")):
            tok = draw_encode_tokens(w, layer, axis, B * w_max, device, seed_tag=seed_tag)
            # [B*w_max, T, H, d] -> [B, H, T, w_max, d]
            out[name][layer].copy_(tok.view(B, w_max, w.T, w.H, w.d).permute(0, 3, 2, 1, 4))
    return out


# ---------------------------------------------------------------------------
# Decoupled rotary sub-keys beside the latents (drawn unrotated)
# ---------------------------------------------------------------------------
def rope_subkeys(w: Workload, layer: int, n_slots: int, d_rope: int, device) -> torch.Tensor:
    """Raw sub-keys [H', n_slots, d_rope], N(0, 1), float32."""
    g = _gen(device, seed_of(w.name, layer, "k_rope", d_rope))
    return torch.randn(w.heads_stored, n_slots, d_rope, generator=g, device=device, dtype=torch.float32)


def rope_queries(w: Workload, B: int, Tq: int, d_rope: int, device) -> torch.Tensor:
    """Rotary query parts [B, Tq, H, d_rope], N(0, 1) / sqrt(d), in the storage type."""
    g = _gen(device, seed_of(w.name, "q_rope", B, Tq, d_rope))
    q = torch.randn(B, Tq, w.H, d_rope, generator=g, device=device, dtype=torch.float32)
    return (q / math.sqrt(w.d)).to(w.torch_dtype)
