"""Workload presets and seeded synthetic inputs.

This module holds shapes and random numbers only: no step of the attention
method is computed here.  Both the CUDA path (through the binding) and the
CPU oracle receive the arrays produced below, so the two sides always see
identical, already dtype-rounded values.

Shapes follow the Wan2.1-1.3B layer the VideoMLA pages build on
(d_model 1536, 12 heads of 128, content latent 192, positional key 32;
ai-papers.net "VideoMLA" article, architecture paragraph under Figure 1).
Value distributions: x ~ N(0, 1), every weight ~ N(0, 1/fan_in).

Seeding: every tensor draws from its own numpy PCG64 stream keyed by
``SeedSequence([seed, tensor_id, chunk, step, layer, sample])`` so that any
single tensor (one chunk of one sample, one layer's weights) can be
regenerated without drawing the others.  Draws are float32 normals, rounded
once to the workload dtype (bf16 with round-to-nearest-even, via torch's CPU
conversion) and returned as float32 arrays holding exactly representable
values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import numpy as np

# tensor ids for the seed sequence
TID_X = 1
TID_W_DKV = 2
TID_W_KR = 3
TID_W_DQ = 4
TID_W_UQ = 5
TID_W_UK = 6
TID_W_UV = 7
TID_W_QR = 8
TID_W_O = 9
TID_Q = 10          # absorbed queries drawn directly (tests of a single call)
TID_LATENT = 11     # chunk latents drawn directly
TID_GRAD = 12       # upstream gradients


@dataclasses.dataclass(frozen=True)
class MLAConfig:
    """One workload: layer shape, frame geometry, rollout schedule."""

    name: str
    dtype: str                     # "fp32" or "bf16"
    d_model: int
    n_heads: int
    d_head: int
    d_c: int                       # content latent width
    d_rope: int                    # decoupled positional key width
    d_cq: int                      # query latent width
    rope_pairs: Tuple[int, int, int]   # rotary pairs on the (t, h, w) axes
    rope_base: float
    frame_h: int
    frame_w: int
    chunk_frames: int
    window_frames: int
    batch: int
    n_chunks: int                  # chunks in the rollout
    measured_chunk: int            # chunk whose attention is the headline call
    n_layers: int = 1
    n_steps: int = 1               # denoising steps per chunk (frozen cache)
    seed: int = 0

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_head + self.d_rope)

    @property
    def tokens_per_frame(self) -> int:
        return self.frame_h * self.frame_w

    @property
    def n_q(self) -> int:
        """Query tokens per sample in one chunk."""
        return self.chunk_frames * self.tokens_per_frame

    @property
    def d_latent(self) -> int:
        """Cached scalars per token: content latent plus positional key."""
        return self.d_c + self.d_rope

    def first_frame(self, chunk: int) -> int:
        return chunk * self.chunk_frames

    def valid_frames(self, chunk: int) -> int:
        """Cached frames a chunk attends to (all earlier frames, up to the window)."""
        return min(self.first_frame(chunk), self.window_frames)

    def keys_per_query(self, chunk: int) -> int:
        return (self.valid_frames(chunk) + self.chunk_frames) * self.tokens_per_frame

    def attention_flops(self, chunk: int) -> float:
        """Latent-space attention work of one call: 2*(D + d_c) flop per
        (query row, valid key, head), D = d_c + d_rope."""
        return (2.0 * (self.d_latent + self.d_c) * self.n_q * self.keys_per_query(chunk)
                * self.n_heads * self.batch)


WAN = dict(d_model=1536, n_heads=12, d_head=128, d_c=192, d_rope=32, d_cq=512,
           rope_pairs=(4, 6, 6), rope_base=10000.0, frame_h=30, frame_w=52)

CONFIGS: Dict[int, MLAConfig] = {
    0: MLAConfig(name="toy_fp32", dtype="fp32", d_model=64, n_heads=2, d_head=16, d_c=16,
                 d_rope=8, d_cq=32, rope_pairs=(2, 1, 1), rope_base=10000.0, frame_h=4,
                 frame_w=4, chunk_frames=1, window_frames=2, batch=1, n_chunks=4,
                 measured_chunk=3),
    1: MLAConfig(name="wan1.3b_b1_w6_c3", dtype="bf16", chunk_frames=3, window_frames=6,
                 batch=1, n_chunks=3, measured_chunk=2, **WAN),
    2: MLAConfig(name="wan1.3b_b1_w21_c3_rollout80", dtype="bf16", chunk_frames=3,
                 window_frames=21, batch=1, n_chunks=80, measured_chunk=79, **WAN),
    3: MLAConfig(name="wan1.3b_b8_w9_c3", dtype="bf16", chunk_frames=3, window_frames=9,
                 batch=8, n_chunks=4, measured_chunk=3, **WAN),
    4: MLAConfig(name="wan1.3b_30layer_b2_w12_c3", dtype="bf16", chunk_frames=3,
                 window_frames=12, batch=2, n_chunks=10, measured_chunk=9, n_layers=30,
                 n_steps=4, **WAN),
}


def small_bf16_config() -> MLAConfig:
    """A bf16 case the oracle finishes in well under a second that still spans
    several 128-row tiles with ragged tails (tokens per frame 6*10 = 60, chunk 3
    frames = 180 queries, window 4 frames) while keeping the Wan layer widths
    that the tensor-core path is built for."""
    return MLAConfig(name="wan_layer_small_frames", dtype="bf16", chunk_frames=3,
                     window_frames=4, batch=2, n_chunks=4, measured_chunk=3,
                     **{**WAN, "frame_h": 6, "frame_w": 10})


def rope_pairs_for(d_rope: int) -> Tuple[int, int, int]:
    """Rotary pairs per (t, h, w) axis for a positional width: a quarter of the pairs on the
    temporal axis, the rest split evenly between rows and columns (Wan: 32 -> (4, 6, 6))."""
    n = d_rope // 2
    pt = n // 4
    ph = (n - pt) // 2
    return pt, ph, n - pt - ph


def with_latent_shape(cfg: MLAConfig, d_c: int, d_rope: int) -> MLAConfig:
    """The same workload with another content-latent and positional-key width (the latent-size
    ablation shapes); the name records the shape."""
    if (d_c, d_rope) == (cfg.d_c, cfg.d_rope):
        return cfg
    return dataclasses.replace(cfg, d_c=d_c, d_rope=d_rope, rope_pairs=rope_pairs_for(d_rope),
                               name=f"{cfg.name}_dc{d_c}_dr{d_rope}")


# --------------------------------------------------------------------------
# rounding helpers (dtype plumbing, not method arithmetic)

def round_to_dtype(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round a float32 array to the workload dtype; returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "fp32":
        return a
    if dtype == "bf16":
        import torch
        return torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(f"unknown dtype {dtype!r}")


def _rng(cfg: MLAConfig, tid: int, chunk: int = 0, step: int = 0, layer: int = 0,
         sample: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence([cfg.seed, tid, chunk, step, layer, sample])
    return np.random.Generator(np.random.PCG64(ss))


def _normal(cfg: MLAConfig, shape, std: float, tid: int, **key) -> np.ndarray:
    z = _rng(cfg, tid, **key).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        z *= np.float32(std)
    return round_to_dtype(z, cfg.dtype)


# --------------------------------------------------------------------------
# weights

@dataclasses.dataclass
class LayerWeights:
    """One attention layer's projections, in the pages' roles.

    w_dkv [d_c, d_model]      joint KV down-projection (content latent)
    w_kr  [d_rope, d_model]   head-shared positional key projection
    w_dq  [d_cq, d_model]     query down-projection (query latent)
    w_uq  [H, d_head, d_cq]   per-head content-query up-projection
    w_uk  [H, d_head, d_c]    per-head key up-projection
    w_uv  [H, d_head, d_c]    per-head value up-projection
    w_qr  [H, d_rope, d_cq]   per-head positional query projection
    w_o   [d_model, H*d_head] output projection
    """

    w_dkv: np.ndarray
    w_kr: np.ndarray
    w_dq: np.ndarray
    w_uq: np.ndarray
    w_uk: np.ndarray
    w_uv: np.ndarray
    w_qr: np.ndarray
    w_o: np.ndarray


def layer_weights(cfg: MLAConfig, layer: int = 0) -> LayerWeights:
    H, dh, dc, dr, dq, dm = (cfg.n_heads, cfg.d_head, cfg.d_c, cfg.d_rope, cfg.d_cq,
                             cfg.d_model)
    s = lambda fan: 1.0 / math.sqrt(fan)
    return LayerWeights(
        w_dkv=_normal(cfg, (dc, dm), s(dm), TID_W_DKV, layer=layer),
        w_kr=_normal(cfg, (dr, dm), s(dm), TID_W_KR, layer=layer),
        w_dq=_normal(cfg, (dq, dm), s(dm), TID_W_DQ, layer=layer),
        w_uq=_normal(cfg, (H, dh, dq), s(dq), TID_W_UQ, layer=layer),
        w_uk=_normal(cfg, (H, dh, dc), s(dc), TID_W_UK, layer=layer),
        w_uv=_normal(cfg, (H, dh, dc), s(dc), TID_W_UV, layer=layer),
        w_qr=_normal(cfg, (H, dr, dq), s(dq), TID_W_QR, layer=layer),
        w_o=_normal(cfg, (dm, H * dh), s(H * dh), TID_W_O, layer=layer),
    )


# --------------------------------------------------------------------------
# activations

def chunk_x(cfg: MLAConfig, chunk: int, step: int = 0, layer: int = 0,
            samples: Optional[range] = None) -> np.ndarray:
    """Video latent tokens of one chunk: [B, n_q, d_model], row-major tokens
    (frame, then row h, then column w)."""
    samples = range(cfg.batch) if samples is None else samples
    return np.stack([_normal(cfg, (cfg.n_q, cfg.d_model), 1.0, TID_X, chunk=chunk, step=step,
                             layer=layer, sample=b) for b in samples])


def direct_queries(cfg: MLAConfig, chunk: int, std: float = 0.5, samples=None) -> np.ndarray:
    """Absorbed queries [B, n_q, H, d_c + d_rope] drawn directly (not projected from x), for
    tests that feed one call its inputs."""
    samples = range(cfg.batch) if samples is None else samples
    return np.stack([_normal(cfg, (cfg.n_q, cfg.n_heads, cfg.d_latent), std, TID_Q, chunk=chunk,
                             sample=b) for b in samples])


def direct_latents(cfg: MLAConfig, chunk: int, samples=None) -> np.ndarray:
    """Chunk latents [B, n_q, d_c + d_rope] ([c_KV || unrotated k_R]) drawn directly, N(0, 1)."""
    samples = range(cfg.batch) if samples is None else samples
    return np.stack([_normal(cfg, (cfg.n_q, cfg.d_latent), 1.0, TID_LATENT, chunk=chunk, sample=b)
                     for b in samples])


def upstream_gradient(cfg: MLAConfig, chunk: int, width: int, std: float = 1.0,
                      samples=None) -> np.ndarray:
    """A synthetic upstream gradient [B, n_q, H, width] (training-use tests)."""
    samples = range(cfg.batch) if samples is None else samples
    return np.stack([_normal(cfg, (cfg.n_q, cfg.n_heads, width), std, TID_GRAD, chunk=chunk,
                             sample=b) for b in samples])


def sample_rows(n: int, k: int, seed: int = 0, tag: int = 0) -> np.ndarray:
    """A seeded, sorted sample of k distinct row indices in [0, n), always
    including the first and last row (the ragged tail)."""
    if k >= n:
        return np.arange(n)
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0xA11, tag, n])))
    pick = rng.choice(n - 2, size=k - 2, replace=False) + 1
    return np.sort(np.concatenate([[0, n - 1], pick]))
