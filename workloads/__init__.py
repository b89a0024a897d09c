"""Seeded synthetic inputs for the KroQuant online activation quantizer.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark. It draws random numbers and shapes them like DiT activations; it
holds none of the quantizer's arithmetic (no transform, no scale rule, no
rounding to E2M1).

Recipe (the same for every consumer):

* Each case has a seed ``1000 * config_index + sub`` where ``sub`` indexes the
  hidden-size variant (and, for the FLUX-shaped case, the outlier gain).
* Three independent numpy ``default_rng`` streams are derived from the seed:
  ``[seed, 0, chunk]`` draws activation rows in chunks of ``ROW_CHUNK`` rows,
  ``[seed, 1]`` draws per-channel quantities (outlier channel set, AdaLN-style
  channel gain), ``[seed, 2]`` draws the transform parameters.  Separate
  streams make any row prefix of a case identical to the same rows of the
  full-size case, so reduced-size parity cases are prefixes of the full ones.
* Activations are drawn in float64, multiplied by the channel gains, rounded
  to float32 and then to bfloat16 (round-to-nearest-even both times).
* Transform parameters per 32-channel block and Kronecker factor k=1..5:
  ``a, c ~ U(-1, 1)`` and ``b = 2**U(-1, 1)`` (so ``b`` is never zero), stored
  as float32 ``[d/32, 5, 3]`` in the order ``(a, b, c)``.
* The SmoothQuant comparator's reciprocal channel scale is synthesised as
  ``inv_s[c] = 1 / sqrt(max_t |x[t, c]|)`` (migration strength 0.5 against a
  unit weight range), computed in float64 and rounded once to float32; a
  channel whose maximum is zero gets ``inv_s = 1``.

Shapes follow the DiT workloads of the KroQuant paper (PixArt-Sigma, SANA,
FLUX.1-schnell; arXiv 2607.21446, section 4.1) and a bandwidth stress case.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os
from typing import Optional

import numpy as np
import torch

ROW_CHUNK = 1024
BLOCK = 32

# name -> recipe.  "dist": row distribution; "frac": share of outlier channels;
# "gains": outlier multiplier per sub-case (several only for the FLUX shape).
CONFIGS = {
    "tiny": dict(index=0, M=256, d=(1152,), dist="normal", frac=0.01, gains=(50.0,)),
    "pixart_sigma": dict(index=1, M=2 * 4096, d=(1152, 4608), dist="adaln", frac=0.01, gains=(50.0,)),
    "sana": dict(index=2, M=4 * 1024, d=(2240, 5600), dist="t4", frac=0.005, gains=(80.0,)),
    "flux_schnell": dict(index=3, M=4096 + 512, d=(3072, 12288), dist="normal", frac=0.01,
                         gains=(5.0, 20.0, 100.0)),
    "stress": dict(index=4, M=16384, d=(12288,), dist="t3", frac=0.005, gains=(100.0,)),
}


@dataclasses.dataclass
class Case:
    """One seeded input: bf16 activations plus the per-block parameters."""

    name: str
    M: int
    d: int
    seed: int
    gain: float
    x: torch.Tensor          # bfloat16 [M, d], CPU
    params: np.ndarray       # float32 [d/32, 5, 3] = (a, b, c) per factor
    inv_s: np.ndarray        # float32 [d], SmoothQuant comparator input

    @property
    def nb(self) -> int:
        return self.d // BLOCK

    def x_bits(self) -> np.ndarray:
        """The activations as raw bfloat16 bit patterns (uint16 [M, d])."""
        return self.x.view(torch.int16).numpy().view(np.uint16)


def case_seed(name: str, d_idx: int = 0, gain_idx: int = 0) -> int:
    cfg = CONFIGS[name]
    sub = d_idx * len(cfg["gains"]) + gain_idx
    return 1000 * cfg["index"] + sub


def _draw_rows(dist: str, seed: int, chunk: int, rows: int, d: int) -> np.ndarray:
    rng = np.random.default_rng([seed, 0, chunk])
    if dist in ("normal", "adaln"):
        return rng.standard_normal((rows, d))
    if dist == "t4":
        return rng.standard_t(4.0, (rows, d))
    if dist == "t3":
        return rng.standard_t(3.0, (rows, d))
    raise ValueError(f"unknown distribution {dist!r}")


def channel_gain(name: str, d: int, seed: int, gain: float) -> np.ndarray:
    """Per-channel multiplier: outlier channels times ``gain`` (and AdaLN-style
    ``1 + s_c`` with ``s_c ~ N(0, 0.5)`` for the PixArt-shaped case)."""
    cfg = CONFIGS[name]
    rng = np.random.default_rng([seed, 1])
    g = np.ones(d)
    if cfg["dist"] == "adaln":
        g = g * (1.0 + rng.normal(0.0, 0.5, d))
    n_out = int(round(cfg["frac"] * d))
    chans = rng.choice(d, size=n_out, replace=False)
    g[chans] *= gain
    return g


def draw_params(d: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng([seed, 2])
    nb = d // BLOCK
    a = rng.uniform(-1.0, 1.0, (nb, 5))
    b = 2.0 ** rng.uniform(-1.0, 1.0, (nb, 5))
    c = rng.uniform(-1.0, 1.0, (nb, 5))
    return np.stack([a, b, c], axis=-1).astype(np.float32)


def draw_params16(d: int, seed: int) -> np.ndarray:
    """Parameters of the 16-element-block variant: ``[d/16, 4, 3]`` float32,
    same distribution as ``draw_params``, from the stream ``[seed, 3]``."""
    rng = np.random.default_rng([seed, 3])
    nb = d // 16
    a = rng.uniform(-1.0, 1.0, (nb, 4))
    b = 2.0 ** rng.uniform(-1.0, 1.0, (nb, 4))
    c = rng.uniform(-1.0, 1.0, (nb, 4))
    return np.stack([a, b, c], axis=-1).astype(np.float32)


def draw_weight(N: int, d: int, seed: int) -> torch.Tensor:
    """Synthetic bf16 weight matrix ``[N, d]`` of a linear layer (row = output
    channel): ``N(0, 1/d)`` entries from the stream ``[seed, 4]``, rounded to
    float32 and then bf16."""
    rng = np.random.default_rng([seed, 4])
    v = rng.standard_normal((N, d)) / np.sqrt(d)
    return torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)


# Tokens per sample of each DiT-shaped config: PixArt-Sigma 1024^2 (64 x 64
# latent patches, batch 2), SANA 1024^2 (32 x 32, batch 4), FLUX.1-schnell
# (4096 image + 512 text tokens, batch 1), the stress case 4 x 4096.
TOKENS_PER_SAMPLE = {"tiny": 128, "pixart_sigma": 4096, "sana": 1024,
                     "flux_schnell": 4608, "stress": 4096}


def draw_adaln(B: int, d: int, seed: int):
    """AdaLN modulation of B samples as a bf16 modulation MLP would emit it:
    ``shift ~ N(0, 0.5)``, ``scale ~ N(0, 0.5)`` with 1 % of the channels
    amplified (scale ``~ U(5, 30)``, channels drawn per sample), from the stream
    ``[seed, 5]``.  Returns (shift, scale) as bf16 ``[B, d]``."""
    rng = np.random.default_rng([seed, 5])
    shift = rng.normal(0.0, 0.5, (B, d))
    scale = rng.normal(0.0, 0.5, (B, d))
    n_amp = max(1, int(round(0.01 * d)))
    for b in range(B):
        ch = rng.choice(d, size=n_amp, replace=False)
        scale[b, ch] = rng.uniform(5.0, 30.0, n_amp)
    cast = lambda v: torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)
    return cast(shift), cast(scale)


def synth_inv_s(x: torch.Tensor) -> np.ndarray:
    """Reciprocal SmoothQuant channel scale for migration strength 0.5 and a
    unit weight range, from the column maxima of ``x`` (bf16 [M, d])."""
    amax = np.zeros(x.shape[1], dtype=np.float64)
    for r0 in range(0, x.shape[0], 4 * ROW_CHUNK):
        blk = x[r0:r0 + 4 * ROW_CHUNK].float().abs().amax(dim=0).double().numpy()
        amax = np.maximum(amax, blk)
    s = np.sqrt(amax)
    s[s == 0] = 1.0
    return (1.0 / s).astype(np.float32)


def make_case(name: str, d_idx: int = 0, gain_idx: int = 0, M: Optional[int] = None,
              threads: Optional[int] = None, row0: int = 0) -> Case:
    """Build a seeded case; ``M`` (default: the config's token count) keeps a
    row prefix of the full-size case.  ``row0`` (a multiple of ``ROW_CHUNK``)
    starts the rows further down the same stream, so that several shards of
    one larger batch can be drawn independently."""
    if row0 % ROW_CHUNK:
        raise ValueError("row0 must be a multiple of ROW_CHUNK")
    cfg = CONFIGS[name]
    d = cfg["d"][d_idx]
    gain = cfg["gains"][gain_idx]
    M = cfg["M"] if M is None else int(M)
    seed = case_seed(name, d_idx, gain_idx)
    g = channel_gain(name, d, seed, gain)
    x = torch.empty((M, d), dtype=torch.bfloat16)

    def fill(chunk: int) -> None:
        r0 = chunk * ROW_CHUNK
        rows = min(ROW_CHUNK, M - r0)
        v = _draw_rows(cfg["dist"], seed, chunk + row0 // ROW_CHUNK, ROW_CHUNK, d)[:rows] * g
        x[r0:r0 + rows] = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)

    n_chunks = (M + ROW_CHUNK - 1) // ROW_CHUNK
    workers = threads or min(8, os.cpu_count() or 1)
    if n_chunks > 1 and workers > 1:
        with _cf.ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, range(n_chunks)))
    else:
        for ch in range(n_chunks):
            fill(ch)
    params = draw_params(d, seed)
    return Case(name=name, M=M, d=d, seed=seed, gain=gain, x=x, params=params,
                inv_s=synth_inv_s(x))


def all_case_keys():
    """(name, d_idx, gain_idx) for every seeded input of every config."""
    out = []
    for name, cfg in CONFIGS.items():
        for di in range(len(cfg["d"])):
            for gi in range(len(cfg["gains"])):
                out.append((name, di, gi))
    return out


def random_bf16(shape, seed: int, scale: float = 1.0) -> torch.Tensor:
    """Plain N(0, scale^2) bf16 tensor for edge-case tests."""
    rng = np.random.default_rng([seed, 9])
    v = rng.standard_normal(shape) * scale
    return torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)


def device_randn_bf16(shape, seed: int, device) -> torch.Tensor:
    """N(0, 1) bf16 drawn on the device by torch's seeded generator, for
    inputs too large to draw on the host (large-offset tests)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    rows = max(1, (1 << 26) // max(1, shape[1]))
    for r0 in range(0, shape[0], rows):
        blk = torch.randn((min(rows, shape[0] - r0), shape[1]), generator=gen, device=device)
        out[r0:r0 + blk.shape[0]] = blk.to(torch.bfloat16)
    return out


def bf16_from_float(values) -> torch.Tensor:
    """bf16 tensor from values that are exactly representable in bf16."""
    t = torch.as_tensor(np.asarray(values, dtype=np.float32))
    b = t.to(torch.bfloat16)
    if not torch.equal(b.float(), t):
        raise ValueError("values are not exactly representable in bfloat16")
    return b


def algorithmic_bytes(M: int, d: int) -> float:
    """Bytes one quantizer pass must move: bf16 in (2 B), packed E2M1 out
    (0.5 B) and one E8M0 scale byte per 32 elements."""
    return M * d * (2.0 + 0.5 + 1.0 / BLOCK)


__all__ = ["CONFIGS", "Case", "make_case", "case_seed", "all_case_keys", "random_bf16",
           "bf16_from_float", "device_randn_bf16", "draw_params", "draw_params16", "draw_weight", "draw_adaln", "TOKENS_PER_SAMPLE", "channel_gain", "synth_inv_s", "algorithmic_bytes",
           "ROW_CHUNK", "BLOCK"]
