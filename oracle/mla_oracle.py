"""Plain, slow, float64 CPU oracle for VideoMLA latent-KV attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` do.  It shares no code, table or helper with the CUDA library.

What it computes is the *non-absorbed* definition of the attention layer
described on the VideoMLA pages:

* hyper.ai summary of VideoMLA (English edition), section "Method"; the same
  paragraph appears in the Chinese edition, section "方法".  Every token x_t is
  compressed by a joint down-projection into a content latent c_KV (written to
  the cache); one positional key k_R = W_R^K x_t, common to all heads, is kept
  unrotated and rotated by 3D-RoPE only when attention runs; per-head keys and
  values are rebuilt from c_KV by per-head up-projections; the query side has a
  query latent c_Q from x_t and per-head positional queries computed from c_Q
  and rotated; the score of head h adds the content term q_nope . k_nope and
  the positional term q_rope . k_rope; the cache holds d_c + d_rope scalars per
  token instead of 2 n_h d_h.
* ai-papers.net article "VideoMLAとは？", paragraph after Figure 1: the base
  model is Wan2.1-1.3B, the content latent is 192 wide, and a token's cached
  state shrinks from 3,072 to 224 scalars.
* chatpaper abstract (English): long rollouts keep a sliding window of fixed
  size as their KV cache; with the latent layout each layer's cache needs
  92.7% less memory per token.

Where the pages are silent the oracle takes the plainest reading (each one is
listed with its reason in the design notes):

1. q_nope_h = W_UQ_h c_Q (the pages name q_nope but not its projection).
2. No normalisation of c_Q, c_KV, q or k.
3. softmax scale 1/sqrt(d_head + d_rope).
4. 3D-RoPE: axis a in (t, h, w) owns n_a adjacent channel pairs; pair i of
   axis a turns by pos_a * base**(-i / n_a); bands ordered t, h, w; the pair
   (x0, x1) maps to (x0 cos - x1 sin, x0 sin + x1 cos).  This convention is
   PARITY UNPINNED by the pages (they only say "3D-RoPE"); what is pinned is
   that it is a rotation, relative in position and identity at the origin.
5. Positions: t = absolute latent-frame index since the rollout began, (h, w)
   = the token's row and column inside its frame; tokens are row-major.
6. A chunk attends to every token of the (at most W) most recent earlier
   frames still in the window, and to every token of its own chunk
   (bidirectionally); nothing else.  The chunk enters the window after its
   attention.
7. The primary output is the concatenation of the per-head outputs; the
   output projection W_O is applied only as a secondary product.

Dtype: every input is the already-rounded array the GPU receives, promoted to
float64; all arithmetic is float64.
"""
from __future__ import annotations

import collections
import dataclasses
import math
from typing import Deque, Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "Dims", "dims_from", "token_positions", "rope3d_angles", "rope3d",
    "down_project", "query_latent", "query_heads", "key_value_heads",
    "attention_probabilities", "attend", "FrameRecord", "SlidingWindow",
    "chunk_step", "absorbed_query", "up_project_output",
    "output_projection", "dense_scalars_per_token", "latent_scalars_per_token",
    "kv_reduction", "softmax_backward", "rope3d_adjoint", "latent_attention_backward",
    "layer_backward_nonabsorbed",
]


@dataclasses.dataclass(frozen=True)
class Dims:
    """Layer shape and frame geometry, restated for the oracle's own use."""

    d_model: int
    n_heads: int
    d_head: int
    d_c: int
    d_rope: int
    d_cq: int
    pairs_t: int
    pairs_h: int
    pairs_w: int
    rope_base: float
    frame_h: int
    frame_w: int
    chunk_frames: int
    window_frames: int

    @property
    def softmax_scale(self) -> float:
        # reading 3: 1/sqrt(d_head + d_rope)
        return 1.0 / math.sqrt(self.d_head + self.d_rope)

    @property
    def tokens_per_frame(self) -> int:
        return self.frame_h * self.frame_w


def dims_from(obj) -> Dims:
    """Build Dims from any object with the same field names (duck-typed)."""
    pt, ph, pw = obj.rope_pairs
    return Dims(d_model=obj.d_model, n_heads=obj.n_heads, d_head=obj.d_head, d_c=obj.d_c,
                d_rope=obj.d_rope, d_cq=obj.d_cq, pairs_t=pt, pairs_h=ph, pairs_w=pw,
                rope_base=float(obj.rope_base), frame_h=obj.frame_h, frame_w=obj.frame_w,
                chunk_frames=obj.chunk_frames, window_frames=obj.window_frames)


# ---------------------------------------------------------------------------
# cache size (hyper.ai summary, Method: 2 n_h d_h -> d_c + d_h^rope scalars)

def dense_scalars_per_token(d: Dims) -> int:
    """Per-token, per-layer scalars of a dense per-head K/V cache: 2 n_h d_h."""
    return 2 * d.n_heads * d.d_head


def latent_scalars_per_token(d: Dims) -> int:
    """Per-token, per-layer scalars of the latent cache: d_c + d_rope."""
    return d.d_c + d.d_rope


def kv_reduction(d: Dims) -> float:
    """Fractional per-token KV memory cut of the latent layout."""
    return 1.0 - latent_scalars_per_token(d) / dense_scalars_per_token(d)


# ---------------------------------------------------------------------------
# positions and 3D-RoPE (hyper.ai summary, Method: k_R stays unrotated in the
# cache and gets its 3D-RoPE rotation when attention runs; so does the query's
# positional part)

def token_positions(frames: Sequence[int], d: Dims) -> np.ndarray:
    """(t, h, w) of every token of the given frames, frames in the order given,
    tokens row-major inside a frame (reading 5).  int64 [len(frames)*tpf, 3]."""
    out = []
    for t in frames:
        for r in range(d.frame_h):
            for c in range(d.frame_w):
                out.append((int(t), r, c))
    return np.asarray(out, dtype=np.int64).reshape(-1, 3)


def rope3d_angles(pos: np.ndarray, d: Dims) -> np.ndarray:
    """Rotation angle of every channel pair: [N, pairs_t + pairs_h + pairs_w]
    (reading 4)."""
    pos = np.asarray(pos, dtype=np.float64)
    bands = []
    for axis, n_pairs in enumerate((d.pairs_t, d.pairs_h, d.pairs_w)):
        inv_freq = d.rope_base ** (-np.arange(n_pairs, dtype=np.float64) / n_pairs)
        bands.append(pos[:, axis:axis + 1] * inv_freq[None, :])
    return np.concatenate(bands, axis=1)


def rope3d(vec: np.ndarray, pos: np.ndarray, d: Dims) -> np.ndarray:
    """Rotate the last axis (d_rope channels, adjacent pairs) of vec [N, ..., d_rope]
    by the angles of positions pos [N, 3]."""
    vec = np.asarray(vec, dtype=np.float64)
    assert vec.shape[-1] == d.d_rope == 2 * (d.pairs_t + d.pairs_h + d.pairs_w)
    ang = rope3d_angles(pos, d)                        # [N, P]
    ang = ang.reshape(ang.shape[:1] + (1,) * (vec.ndim - 2) + ang.shape[1:])
    x0 = vec[..., 0::2]
    x1 = vec[..., 1::2]
    cos, sin = np.cos(ang), np.sin(ang)
    out = np.empty_like(vec)
    out[..., 0::2] = x0 * cos - x1 * sin
    out[..., 1::2] = x0 * sin + x1 * cos
    return out


# ---------------------------------------------------------------------------
# projections (hyper.ai summary, Method)

def down_project(x: np.ndarray, w_dkv: np.ndarray, w_kr: np.ndarray):
    """c_KV = W_down^KV x and k_R = W_R^K x for every token x [N, d_model]."""
    x = np.asarray(x, dtype=np.float64)
    return x @ np.asarray(w_dkv, np.float64).T, x @ np.asarray(w_kr, np.float64).T


def query_latent(x: np.ndarray, w_dq: np.ndarray) -> np.ndarray:
    """c_Q = W_down^Q x: [N, d_cq]."""
    return np.asarray(x, np.float64) @ np.asarray(w_dq, np.float64).T


def query_heads(c_q: np.ndarray, w_uq: np.ndarray, w_qr: np.ndarray):
    """Per-head content query q_nope_h = W_UQ_h c_Q (reading 1) and unrotated
    positional query q_R_h = W_QR_h c_Q: [N, H, d_head], [N, H, d_rope]."""
    c_q = np.asarray(c_q, np.float64)
    q_nope = np.einsum("hdk,nk->nhd", np.asarray(w_uq, np.float64), c_q)
    q_r = np.einsum("hdk,nk->nhd", np.asarray(w_qr, np.float64), c_q)
    return q_nope, q_r


def key_value_heads(c_kv: np.ndarray, w_uk: np.ndarray, w_uv: np.ndarray):
    """Per-head keys and values rebuilt from the shared latent:
    k_nope_h = W_UK_h c_KV, v_h = W_UV_h c_KV: [M, H, d_head] each."""
    c_kv = np.asarray(c_kv, np.float64)
    k = np.einsum("hdc,mc->mhd", np.asarray(w_uk, np.float64), c_kv)
    v = np.einsum("hdc,mc->mhd", np.asarray(w_uv, np.float64), c_kv)
    return k, v


# ---------------------------------------------------------------------------
# attention (hyper.ai summary, Method: score of head h = content term + positional term)

def attention_probabilities(q_nope, q_rope, k_nope, k_rope, scale: float):
    """Full softmax over all keys for one head.

    q_nope [N, dh], q_rope [N, dr], k_nope [M, dh], k_rope [M, dr].
    Returns (p [N, M], lse [N]) with lse the natural log of the softmax
    denominator of the scaled scores.
    """
    s = (q_nope @ k_nope.T + q_rope @ k_rope.T) * scale
    row_max = s.max(axis=1, keepdims=True)
    e = np.exp(s - row_max)
    denom = e.sum(axis=1, keepdims=True)
    return e / denom, (row_max + np.log(denom))[:, 0]


def attend(q_nope, q_rope, k_nope, k_rope, v, scale: float, c_keys=None, keep_p=False):
    """Multi-head attention with one head-shared positional key.

    q_nope [N, H, dh], q_rope [N, H, dr], k_nope [M, H, dh], k_rope [M, dr],
    v [M, H, dh].  Heads are evaluated one after another.  Returns a dict with
    o [N, H*dh] (heads concatenated in head order), lse [H, N], and when
    ``c_keys`` [M, d_c] is given the latent output o_lat [N, H, d_c]
    (sum_m p c_KV[m]); p [H, N, M] only when ``keep_p``.
    """
    n, n_heads, dh = q_nope.shape
    o = np.empty((n, n_heads, dh))
    lse = np.empty((n_heads, n))
    o_lat = None if c_keys is None else np.empty((n, n_heads, c_keys.shape[1]))
    ps = [] if keep_p else None
    for h in range(n_heads):
        p, lse[h] = attention_probabilities(q_nope[:, h], q_rope[:, h], k_nope[:, h], k_rope,
                                            scale)
        o[:, h] = p @ v[:, h]
        if c_keys is not None:
            o_lat[:, h] = p @ c_keys
        if keep_p:
            ps.append(p)
    out = dict(o=o.reshape(n, n_heads * dh), lse=lse)
    if o_lat is not None:
        out["o_lat"] = o_lat
    if keep_p:
        out["p"] = np.stack(ps)
    return out


# ---------------------------------------------------------------------------
# sliding window of past frames (chatpaper abstract: fixed-size sliding-window
# KV cache; hyper.ai summary, Introduction: rolling key-value cache)

@dataclasses.dataclass
class FrameRecord:
    """What the latent cache keeps for one latent frame: its absolute frame
    index, the content latents and the unrotated positional keys of its tokens."""

    t: int
    c_kv: np.ndarray      # [tpf, d_c]
    k_r: np.ndarray       # [tpf, d_rope]


class SlidingWindow:
    """The most recent W frames, oldest first (a deque, no slot arithmetic)."""

    def __init__(self, d: Dims):
        self.d = d
        self.frames: Deque[FrameRecord] = collections.deque(maxlen=d.window_frames)

    def append_chunk(self, first_frame: int, c_kv: np.ndarray, k_r: np.ndarray) -> None:
        tpf = self.d.tokens_per_frame
        n_frames = c_kv.shape[0] // tpf
        for f in range(n_frames):
            self.frames.append(FrameRecord(first_frame + f, c_kv[f * tpf:(f + 1) * tpf].copy(),
                                           k_r[f * tpf:(f + 1) * tpf].copy()))

    def frame_indices(self) -> List[int]:
        return [r.t for r in self.frames]

    def keys(self):
        """Concatenated (c_kv [M, d_c], k_r [M, d_rope], pos [M, 3]) of the window."""
        if not self.frames:
            d = self.d
            return (np.zeros((0, d.d_c)), np.zeros((0, d.d_rope)),
                    np.zeros((0, 3), dtype=np.int64))
        c = np.concatenate([r.c_kv for r in self.frames])
        k = np.concatenate([r.k_r for r in self.frames])
        return c, k, token_positions(self.frame_indices(), self.d)


# ---------------------------------------------------------------------------
# one chunk of a rollout, end to end

def chunk_step(d: Dims, w, x: np.ndarray, window: SlidingWindow, first_frame: int,
               rows: Optional[np.ndarray] = None, append: bool = True,
               keep_p: bool = False) -> Dict[str, np.ndarray]:
    """Attention of one chunk of one sample against the window, then the window update.

    x [Nq, d_model] are the chunk's tokens (frames first_frame .. +C-1).  The
    keys are every token of the window's frames followed by every token of the
    chunk (reading 6).  ``rows`` selects the query rows whose outputs are
    evaluated (all by default); rows are independent given the keys, and every
    evaluated row takes its softmax over all of its keys at once.  When
    ``append`` is set the chunk's latents enter the window afterwards.

    Returns the chunk latents (c_kv, k_r), the selected rows' c_q, q_nope, q_r,
    q_rope and positions, every key's latent, positional key and position, the
    output o [n, H*d_head], the latent output o_lat [n, H, d_c], lse [H, n],
    and (``keep_p``) the probabilities p [H, n, M].
    """
    tpf = d.tokens_per_frame
    n_q = x.shape[0]
    assert n_q == d.chunk_frames * tpf
    rows = np.arange(n_q) if rows is None else np.asarray(rows)

    c_kv_chunk, k_r_chunk = down_project(x, w.w_dkv, w.w_kr)
    pos_chunk = token_positions(range(first_frame, first_frame + d.chunk_frames), d)

    c_win, k_win, pos_win = window.keys()
    c_all = np.concatenate([c_win, c_kv_chunk])
    k_r_all = np.concatenate([k_win, k_r_chunk])
    pos_all = np.concatenate([pos_win, pos_chunk])

    k_nope, v = key_value_heads(c_all, w.w_uk, w.w_uv)
    k_rope = rope3d(k_r_all, pos_all, d)

    c_q = query_latent(x[rows], w.w_dq)
    q_nope, q_r = query_heads(c_q, w.w_uq, w.w_qr)
    q_rope = rope3d(q_r, pos_chunk[rows], d)

    att = attend(q_nope, q_rope, k_nope, k_rope, v, d.softmax_scale, c_keys=c_all,
                 keep_p=keep_p)

    out = dict(c_kv=c_kv_chunk, k_r=k_r_chunk, c_q=c_q, q_nope=q_nope, q_r=q_r,
               q_rope=q_rope, pos_q=pos_chunk[rows], pos_k=pos_all, c_keys=c_all,
               k_r_keys=k_r_all, k_rope=k_rope, rows=rows,
               window_frames=np.asarray(window.frame_indices(), dtype=np.int64), **att)
    if append:
        window.append_chunk(first_frame, c_kv_chunk, k_r_chunk)
    return out


# ---------------------------------------------------------------------------
# absorbed-form intermediates.  Absorption is exact algebra: the content score
# q_nope_h . (W_UK_h c) equals (W_UK_h^T q_nope_h) . c, and the head output
# W_UV_h sum p c equals sum p (W_UV_h c).  These functions compute the
# intermediates that a latent-space kernel produces, so that each stage of the
# CUDA path can be checked on its own.

def absorbed_query(c_q: np.ndarray, w_uq, w_uk, w_qr, pos_q: np.ndarray, d: Dims) -> np.ndarray:
    """Q' [N, H, d_c + d_rope] = [W_UK_h^T W_UQ_h c_Q || RoPE3D(W_QR_h c_Q)] (unscaled)."""
    q_nope, q_r = query_heads(c_q, w_uq, w_qr)
    q_lat = np.einsum("hdc,nhd->nhc", np.asarray(w_uk, np.float64), q_nope)
    return np.concatenate([q_lat, rope3d(q_r, pos_q, d)], axis=2)


def up_project_output(o_lat: np.ndarray, w_uv) -> np.ndarray:
    """o[n] = concat_h W_UV_h O_lat[n, h]: [N, H*d_head]."""
    o = np.einsum("hdc,nhc->nhd", np.asarray(w_uv, np.float64), o_lat)
    return o.reshape(o.shape[0], -1)


def output_projection(o: np.ndarray, w_o) -> np.ndarray:
    """y = W_O o (reading 7: secondary product)."""
    return np.asarray(o, np.float64) @ np.asarray(w_o, np.float64).T


# ---------------------------------------------------------------------------
# gradients of the attention layer (training use: the pages train the latent students with
# teacher forcing and distillation through these layers; hyper.ai summary, "Method").  With an
# upstream gradient g of the output, L = sum g * output; the derivatives below are the
# textbook ones of softmax attention, taken one step of the forward at a time, in reverse.

def softmax_backward(p: np.ndarray, d_p: np.ndarray) -> np.ndarray:
    """dL/ds for p = softmax over the last axis of s, given dL/dp:
    p * (d_p - sum_j p_j d_p_j)."""
    return p * (d_p - (p * d_p).sum(axis=-1, keepdims=True))


def rope3d_adjoint(vec: np.ndarray, pos: np.ndarray, d: Dims) -> np.ndarray:
    """Transpose of the 3D-RoPE map at positions pos: each pair's rotation by a is orthogonal,
    so its transpose is the rotation by -a, i.e. the map at the negated positions."""
    return rope3d(vec, -np.asarray(pos), d)


def latent_attention_backward(q: np.ndarray, c_keys: np.ndarray, k_r_keys: np.ndarray,
                              pos_k: np.ndarray, d_o_lat: np.ndarray, d: Dims):
    """Gradients of the latent-space attention call.

    Forward (what the attention kernel computes): for head h and query n,
      K'_m = [c_m || RoPE3D(k_R,m, pos_m)],  s = scale * q[n, h] . K'_m,
      p = softmax over m,  O_lat[n, h] = sum_m p_m c_m.
    q [N, H, d_c + d_rope] (positional part already rotated), c_keys [M, d_c], k_r_keys
    [M, d_rope] (unrotated), pos_k [M, 3], d_o_lat [N, H, d_c] = dL/dO_lat.

    Returns o_lat, lse [H, N], d_q [N, H, D] (w.r.t. q as given), d_c [M, d_c] and d_k_r
    [M, d_rope] (w.r.t. the unrotated positional keys).  The value of a key is its content
    latent, so d_c collects both the value gradient and the content part of the key gradient.
    """
    q = np.asarray(q, np.float64)
    c_keys = np.asarray(c_keys, np.float64)
    d_o_lat = np.asarray(d_o_lat, np.float64)
    n, n_heads, width = q.shape
    scale = d.softmax_scale
    k_full = np.concatenate([c_keys, rope3d(k_r_keys, pos_k, d)], axis=1)     # K' [M, D]
    o_lat = np.empty((n, n_heads, d.d_c))
    lse = np.empty((n_heads, n))
    d_q = np.empty_like(q)
    d_k_full = np.zeros_like(k_full)
    d_v = np.zeros_like(c_keys)
    for h in range(n_heads):
        s = (q[:, h] @ k_full.T) * scale
        row_max = s.max(axis=1, keepdims=True)
        e = np.exp(s - row_max)
        p = e / e.sum(axis=1, keepdims=True)
        lse[h] = (row_max + np.log(e.sum(axis=1, keepdims=True)))[:, 0]
        o_lat[:, h] = p @ c_keys
        # O_lat = p V (V = c_keys)
        d_p = d_o_lat[:, h] @ c_keys.T
        d_v += p.T @ d_o_lat[:, h]
        # p = softmax(s)
        d_s = softmax_backward(p, d_p)
        # s = scale q K'^T
        d_q[:, h] = scale * (d_s @ k_full)
        d_k_full += scale * (d_s.T @ q[:, h])
    d_c = d_v + d_k_full[:, :d.d_c]
    d_k_r = rope3d_adjoint(d_k_full[:, d.d_c:], pos_k, d)
    return dict(o_lat=o_lat, lse=lse, d_q=d_q, d_c=d_c, d_k_r=d_k_r)


def layer_backward_nonabsorbed(d: Dims, w, c_q: np.ndarray, pos_q: np.ndarray,
                               c_keys: np.ndarray, k_r_keys: np.ndarray, pos_k: np.ndarray,
                               d_o: np.ndarray):
    """Gradients of the non-absorbed layer (per-head keys and values rebuilt from c_KV) w.r.t.
    the query latent c_Q [N, d_cq], the key latents c_keys [M, d_c] and the unrotated positional
    keys k_r_keys [M, d_rope], for the upstream gradient d_o [N, H, d_head] of the per-head
    outputs o_h = sum_m p_m v_m,h.  Returns d_c_q, d_c, d_k_r and o [N, H, d_head]."""
    scale = d.softmax_scale
    q_nope, q_r = query_heads(c_q, w.w_uq, w.w_qr)
    q_rope = rope3d(q_r, pos_q, d)
    k_nope, v = key_value_heads(c_keys, w.w_uk, w.w_uv)
    k_rope = rope3d(k_r_keys, pos_k, d)
    n, n_heads, dh = q_nope.shape
    d_o = np.asarray(d_o, np.float64)
    o = np.empty((n, n_heads, dh))
    d_q_nope = np.empty_like(q_nope)
    d_q_rope = np.empty_like(q_rope)
    d_k_nope = np.zeros_like(k_nope)
    d_v = np.zeros_like(v)
    d_k_rope = np.zeros_like(k_rope)
    for h in range(n_heads):
        p, _ = attention_probabilities(q_nope[:, h], q_rope[:, h], k_nope[:, h], k_rope, scale)
        o[:, h] = p @ v[:, h]
        d_p = d_o[:, h] @ v[:, h].T
        d_v[:, h] = p.T @ d_o[:, h]
        d_s = softmax_backward(p, d_p)
        d_q_nope[:, h] = scale * (d_s @ k_nope[:, h])
        d_q_rope[:, h] = scale * (d_s @ k_rope)
        d_k_nope[:, h] = scale * (d_s.T @ q_nope[:, h])
        d_k_rope += scale * (d_s.T @ q_rope[:, h])
    w_uq, w_uk = np.asarray(w.w_uq, np.float64), np.asarray(w.w_uk, np.float64)
    w_uv, w_qr = np.asarray(w.w_uv, np.float64), np.asarray(w.w_qr, np.float64)
    # k_nope_h = W_UK_h c, v_h = W_UV_h c, k_rope = RoPE(k_R)
    d_c = (np.einsum("hdc,mhd->mc", w_uk, d_k_nope) + np.einsum("hdc,mhd->mc", w_uv, d_v))
    d_k_r = rope3d_adjoint(d_k_rope, pos_k, d)
    # q_nope_h = W_UQ_h c_Q, q_rope_h = RoPE(W_QR_h c_Q)
    d_q_r = rope3d_adjoint(d_q_rope, pos_q, d)
    d_c_q = (np.einsum("hdk,nhd->nk", w_uq, d_q_nope) + np.einsum("hdk,nhd->nk", w_qr, d_q_r))
    return dict(d_c_q=d_c_q, d_c=d_c, d_k_r=d_k_r, o=o)
