"""Python binding of the C ABI: the same entry points, taking torch tensors.

Every function here only marshals arguments (shape/dtype checks, raw device pointers, the
current CUDA stream) and calls the library; all arithmetic runs in the CUDA kernels.  A non-zero
status raises MLAError with the library's message.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import (MLA_APPEND, MLA_BF16, MLA_FP32, MLA_PATH_AUTO, MLA_PATH_SIMT,
                   MLA_PATH_TC_PAIR, MLA_PATH_TC_SINGLE, MLA_PROJECT, MLA_PROJECT_AND_APPEND, MLAConfigC, MLAError)

__all__ = [
    "make_config", "torch_dtype", "mla_config_check", "mla_cache_append", "mla_rope3d",
    "mla_key_positions", "mla_compose_query_weights", "mla_query_proj", "mla_project_chunk",
    "mla_attention_workspace_bytes", "mla_attention_fwd", "mla_attention_fwd_static_scratch",
    "mla_project_latents", "mla_project_latents_rotated", "mla_attention_fwd_from_cq",
    "mla_rotate_ring_keys", "mla_attention_fwd_cached_ring", "mla_attention_uses_tensor_cores",
    "mla_attention_bwd_workspace_bytes", "mla_attention_bwd",
    "mla_out_proj", "MLAError",
    "MLA_PROJECT", "MLA_APPEND", "MLA_PROJECT_AND_APPEND", "MLA_PATH_AUTO", "MLA_PATH_SIMT",
    "MLA_PATH_TC_SINGLE", "MLA_PATH_TC_PAIR",
]


def make_config(cfg, kernel_path: int = MLA_PATH_AUTO, batch: Optional[int] = None) -> MLAConfigC:
    """struct mla_config from a workload preset (mla_latent_kv_attn_b200.inputs.MLAConfig)."""
    pt, ph, pw = cfg.rope_pairs
    return MLAConfigC(
        d_model=cfg.d_model, n_heads=cfg.n_heads, d_head=cfg.d_head, d_c=cfg.d_c,
        d_rope=cfg.d_rope, d_cq=cfg.d_cq, rope_pairs_t=pt, rope_pairs_h=ph, rope_pairs_w=pw,
        rope_base=cfg.rope_base, softmax_scale=cfg.softmax_scale, frame_h=cfg.frame_h,
        frame_w=cfg.frame_w, chunk_frames=cfg.chunk_frames, window_frames=cfg.window_frames,
        batch=cfg.batch if batch is None else batch,
        dtype=MLA_FP32 if cfg.dtype == "fp32" else MLA_BF16, kernel_path=kernel_path)


def torch_dtype(c: MLAConfigC) -> torch.dtype:
    return torch.float32 if c.dtype == MLA_FP32 else torch.bfloat16


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, shape=None) -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _geom(c: MLAConfigC):
    tpf = c.frame_h * c.frame_w
    return tpf, c.chunk_frames * tpf, c.d_c + c.d_rope


def mla_config_check(c: MLAConfigC) -> None:
    _lib.check("mla_config_check", _lib.lib().mla_config_check(ctypes.byref(c)))


def mla_cache_append(c: MLAConfigC, x, w_dkv_kr, chunk_lat, cache, slot_frame, first_frame: int,
                     mode: int, stream=None) -> None:
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B = c.batch
    st = _lib.lib().mla_cache_append(
        ctypes.byref(c), _ptr(x, "x", dt, (B, n_q, c.d_model)),
        _ptr(w_dkv_kr, "w_dkv_kr", dt, (D, c.d_model)), _ptr(chunk_lat, "chunk_lat", dt, (B, n_q, D)),
        _ptr(cache, "cache", dt, (B, c.window_frames * tpf, D)),
        _ptr(slot_frame, "slot_frame", torch.int32, (B, c.window_frames)), first_frame, mode,
        _stream(stream))
    _lib.check("mla_cache_append", st)


def mla_rope3d(c: MLAConfigC, data, n_vec: int, col_offset: int, vec_stride: int,
               frame_table=None, first_frame: int = 0, stream=None) -> None:
    """Rotates data [n_samples, rows, row_width] in place (see include/mla.h)."""
    if data.dim() != 3:
        raise ValueError("data must be [n_samples, rows, row_width]")
    n_s, rows, width = data.shape
    fstride = frame_table.shape[1] if frame_table is not None else 0
    st = _lib.lib().mla_rope3d(
        ctypes.byref(c), _ptr(data, "data", torch_dtype(c)), n_s, rows, width, col_offset, n_vec,
        vec_stride, _ptr(frame_table, "frame_table", torch.int32), fstride, first_frame,
        _stream(stream))
    _lib.check("mla_rope3d", st)


def mla_key_positions(c: MLAConfigC, slot_frame, n_valid_frames: int, first_frame: int,
                      pos_out, stream=None) -> None:
    tpf, n_q, _ = _geom(c)
    n_keys = n_valid_frames * tpf + n_q
    st = _lib.lib().mla_key_positions(
        ctypes.byref(c), _ptr(slot_frame, "slot_frame", torch.int32, (c.batch, c.window_frames)),
        n_valid_frames, first_frame, _ptr(pos_out, "pos_out", torch.int32, (c.batch, n_keys, 3)),
        _stream(stream))
    _lib.check("mla_key_positions", st)


def mla_compose_query_weights(c: MLAConfigC, w_uq, w_uk, w_qr, w_qcat, stream=None) -> None:
    dt = torch_dtype(c)
    H, D = c.n_heads, c.d_c + c.d_rope
    st = _lib.lib().mla_compose_query_weights(
        ctypes.byref(c), _ptr(w_uq, "w_uq", dt, (H, c.d_head, c.d_cq)),
        _ptr(w_uk, "w_uk", dt, (H, c.d_head, c.d_c)), _ptr(w_qr, "w_qr", dt, (H, c.d_rope, c.d_cq)),
        _ptr(w_qcat, "w_qcat", dt, (H, D, c.d_cq)), _stream(stream))
    _lib.check("mla_compose_query_weights", st)


def mla_query_proj(c: MLAConfigC, x, w_dq, w_qcat, c_q, q, first_frame: int, stream=None) -> None:
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B, H = c.batch, c.n_heads
    st = _lib.lib().mla_query_proj(
        ctypes.byref(c), _ptr(x, "x", dt, (B, n_q, c.d_model)),
        _ptr(w_dq, "w_dq", dt, (c.d_cq, c.d_model)), _ptr(w_qcat, "w_qcat", dt, (H, D, c.d_cq)),
        _ptr(c_q, "c_q", dt, (B, n_q, c.d_cq)), _ptr(q, "q", dt, (B, n_q, H, D)), first_frame,
        _stream(stream))
    _lib.check("mla_query_proj", st)


def mla_project_chunk(c: MLAConfigC, x, w_x, w_qcat, c_q, q, chunk_lat, first_frame: int,
                      stream=None) -> None:
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B, H = c.batch, c.n_heads
    st = _lib.lib().mla_project_chunk(
        ctypes.byref(c), _ptr(x, "x", dt, (B, n_q, c.d_model)),
        _ptr(w_x, "w_x", dt, (c.d_cq + D, c.d_model)), _ptr(w_qcat, "w_qcat", dt, (H, D, c.d_cq)),
        _ptr(c_q, "c_q", dt, (B, n_q, c.d_cq)), _ptr(q, "q", dt, (B, n_q, H, D)),
        _ptr(chunk_lat, "chunk_lat", dt, (B, n_q, D)), first_frame, _stream(stream))
    _lib.check("mla_project_chunk", st)


def mla_project_latents(c: MLAConfigC, x, w_x, c_q, chunk_lat, stream=None) -> None:
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B = c.batch
    st = _lib.lib().mla_project_latents(
        ctypes.byref(c), _ptr(x, "x", dt, (B, n_q, c.d_model)),
        _ptr(w_x, "w_x", dt, (c.d_cq + D, c.d_model)), _ptr(c_q, "c_q", dt, (B, n_q, c.d_cq)),
        _ptr(chunk_lat, "chunk_lat", dt, (B, n_q, D)), _stream(stream))
    _lib.check("mla_project_latents", st)


def mla_project_latents_rotated(c: MLAConfigC, x, w_x, c_q, chunk_lat, cache, slot_frame,
                                n_valid_frames: int, first_frame: int, workspace,
                                rotate_ring: bool = True, dev_status=None, stream=None) -> None:
    """mla_project_latents that also writes the chunk attention's rotated positional keys into
    `workspace` (the ring's too with rotate_ring), for mla_attention_fwd_from_cq(...,
    prerotated=True)."""
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B = c.batch
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = _lib.lib().mla_project_latents_rotated(
        ctypes.byref(c), _ptr(x, "x", dt, (B, n_q, c.d_model)),
        _ptr(w_x, "w_x", dt, (c.d_cq + D, c.d_model)), _ptr(c_q, "c_q", dt, (B, n_q, c.d_cq)),
        _ptr(chunk_lat, "chunk_lat", dt, (B, n_q, D)),
        _ptr(cache, "cache", dt, (B, c.window_frames * tpf, D)),
        _ptr(slot_frame, "slot_frame", torch.int32, (B, c.window_frames)), n_valid_frames,
        first_frame, 1 if rotate_ring else 0, _ptr(workspace, "workspace"), ws_bytes,
        _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _lib.check("mla_project_latents_rotated", st)


def mla_attention_uses_tensor_cores(c: MLAConfigC, with_w_uv: bool = True) -> bool:
    r = int(_lib.lib().mla_attention_uses_tensor_cores(ctypes.byref(c), 1 if with_w_uv else 0))
    if r < 0:
        raise MLAError("mla_attention_uses_tensor_cores", _lib.MLA_ERR_INVALID_ARG, _lib.last_error())
    return bool(r)


def mla_attention_workspace_bytes(c: MLAConfigC, n_valid_frames: int) -> int:
    return int(_lib.lib().mla_attention_workspace_bytes(ctypes.byref(c), n_valid_frames))


def _attention(fn_name: str, c: MLAConfigC, q, chunk_lat, cache, slot_frame, n_valid_frames: int,
               first_frame: int, w_uv, out, lse, workspace, dev_status, stream) -> None:
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B, H = c.batch, c.n_heads
    out_shape = (B, n_q, H * c.d_head) if w_uv is not None else (B, n_q, H, c.d_c)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = getattr(_lib.lib(), fn_name)(
        ctypes.byref(c), _ptr(q, "q", dt, (B, n_q, H, D)), _ptr(chunk_lat, "chunk_lat", dt, (B, n_q, D)),
        _ptr(cache, "cache", dt, (B, c.window_frames * tpf, D)),
        _ptr(slot_frame, "slot_frame", torch.int32, (B, c.window_frames)), n_valid_frames,
        first_frame, _ptr(w_uv, "w_uv", dt, (H, c.d_head, c.d_c)), _ptr(out, "out", dt, out_shape),
        _ptr(lse, "lse", torch.float32, (B, H, n_q)), _ptr(workspace, "workspace"), ws_bytes,
        _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _lib.check(fn_name, st)


def mla_attention_fwd(c: MLAConfigC, q, chunk_lat, cache, slot_frame, n_valid_frames: int,
                      first_frame: int, w_uv, out, lse=None, workspace=None, dev_status=None,
                      stream=None) -> None:
    _attention("mla_attention_fwd", c, q, chunk_lat, cache, slot_frame, n_valid_frames,
               first_frame, w_uv, out, lse, workspace, dev_status, stream)


def mla_attention_fwd_from_cq(c: MLAConfigC, c_q, w_qcat, chunk_lat, cache, slot_frame,
                              n_valid_frames: int, first_frame: int, w_uv, out, lse=None,
                              workspace=None, dev_status=None, stream=None,
                              cached_ring: bool = False, prerotated: bool = False) -> None:
    """mla_attention_fwd with the query heads (and their 3D-RoPE) formed inside the attention
    kernel from the query latent c_q and the composed weights w_qcat.  cached_ring: the
    workspace already holds the ring's rotated keys (mla_rotate_ring_keys); prerotated: it holds
    every rotated key of the call (mla_project_latents_rotated), so no rotation pass runs."""
    if cached_ring and prerotated:
        raise ValueError("cached_ring and prerotated are exclusive")
    fn = ("mla_attention_fwd_from_cq_prerotated" if prerotated else
          "mla_attention_fwd_from_cq_cached_ring" if cached_ring else "mla_attention_fwd_from_cq")
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B, H = c.batch, c.n_heads
    out_shape = (B, n_q, H * c.d_head) if w_uv is not None else (B, n_q, H, c.d_c)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = getattr(_lib.lib(), fn)(
        ctypes.byref(c), _ptr(c_q, "c_q", dt, (B, n_q, c.d_cq)),
        _ptr(w_qcat, "w_qcat", dt, (H, D, c.d_cq)), _ptr(chunk_lat, "chunk_lat", dt, (B, n_q, D)),
        _ptr(cache, "cache", dt, (B, c.window_frames * tpf, D)),
        _ptr(slot_frame, "slot_frame", torch.int32, (B, c.window_frames)), n_valid_frames,
        first_frame, _ptr(w_uv, "w_uv", dt, (H, c.d_head, c.d_c)), _ptr(out, "out", dt, out_shape),
        _ptr(lse, "lse", torch.float32, (B, H, n_q)), _ptr(workspace, "workspace"), ws_bytes,
        _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _lib.check(fn, st)


def mla_attention_fwd_cached_ring(c: MLAConfigC, q, chunk_lat, cache, slot_frame,
                                  n_valid_frames: int, first_frame: int, w_uv, out, lse=None,
                                  workspace=None, dev_status=None, stream=None) -> None:
    """mla_attention_fwd for a workspace whose ring part mla_rotate_ring_keys has filled for the
    same (unchanged) ring; only the chunk's positional keys are rotated."""
    _attention("mla_attention_fwd_cached_ring", c, q, chunk_lat, cache, slot_frame,
               n_valid_frames, first_frame, w_uv, out, lse, workspace, dev_status, stream)


def mla_rotate_ring_keys(c: MLAConfigC, cache, slot_frame, n_valid_frames: int, workspace,
                         stream=None) -> None:
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B = c.batch
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = _lib.lib().mla_rotate_ring_keys(
        ctypes.byref(c), _ptr(cache, "cache", dt, (B, c.window_frames * tpf, D)),
        _ptr(slot_frame, "slot_frame", torch.int32, (B, c.window_frames)), n_valid_frames,
        _ptr(workspace, "workspace"), ws_bytes, _stream(stream))
    _lib.check("mla_rotate_ring_keys", st)


def mla_attention_bwd_workspace_bytes(c: MLAConfigC, n_valid_frames: int) -> int:
    return int(_lib.lib().mla_attention_bwd_workspace_bytes(ctypes.byref(c), n_valid_frames))


def mla_attention_bwd(c: MLAConfigC, q, chunk_lat, cache, slot_frame, n_valid_frames: int,
                      first_frame: int, o_lat, lse, d_o_lat, d_q, d_chunk_lat, d_cache, workspace,
                      dev_status=None, stream=None) -> None:
    """Gradients of the latent attention call (see include/mla.h)."""
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B, H = c.batch, c.n_heads
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = _lib.lib().mla_attention_bwd(
        ctypes.byref(c), _ptr(q, "q", dt, (B, n_q, H, D)), _ptr(chunk_lat, "chunk_lat", dt, (B, n_q, D)),
        _ptr(cache, "cache", dt, (B, c.window_frames * tpf, D)),
        _ptr(slot_frame, "slot_frame", torch.int32, (B, c.window_frames)), n_valid_frames,
        first_frame, _ptr(o_lat, "o_lat", dt, (B, n_q, H, c.d_c)),
        _ptr(lse, "lse", torch.float32, (B, H, n_q)), _ptr(d_o_lat, "d_o_lat", dt, (B, n_q, H, c.d_c)),
        _ptr(d_q, "d_q", dt, (B, n_q, H, D)), _ptr(d_chunk_lat, "d_chunk_lat", dt, (B, n_q, D)),
        _ptr(d_cache, "d_cache", dt, (B, c.window_frames * tpf, D)), _ptr(workspace, "workspace"),
        ws_bytes, _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _lib.check("mla_attention_bwd", st)


def mla_out_proj(c: MLAConfigC, o_lat, w_uv, o, w_o=None, y=None, stream=None) -> None:
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B, H = c.batch, c.n_heads
    st = _lib.lib().mla_out_proj(
        ctypes.byref(c), _ptr(o_lat, "o_lat", dt, (B, n_q, H, c.d_c)),
        _ptr(w_uv, "w_uv", dt, (H, c.d_head, c.d_c)), _ptr(w_o, "w_o", dt, (c.d_model, H * c.d_head)),
        _ptr(o, "o", dt, (B, n_q, H * c.d_head)), _ptr(y, "y", dt, (B, n_q, c.d_model)),
        _stream(stream))
    _lib.check("mla_out_proj", st)


def mla_attention_fwd_static_scratch(c: MLAConfigC, q, chunk_lat, cache, slot_frame,
                                     n_valid_frames: int, first_frame: int, w_uv, out, lse=None,
                                     dev_status=None, stream=None) -> None:
    """mla_attention_fwd for callers that cannot allocate: the scratch lives in the library's
    built-in 16 MiB device array (one per device, shared by all calls; order calls on one
    stream).  The first call on a device should come before any stream capture."""
    tpf, n_q, D = _geom(c)
    dt = torch_dtype(c)
    B, H = c.batch, c.n_heads
    out_shape = (B, n_q, H * c.d_head) if w_uv is not None else (B, n_q, H, c.d_c)
    st = _lib.lib().mla_attention_fwd_static_scratch(
        ctypes.byref(c), _ptr(q, "q", dt, (B, n_q, H, D)), _ptr(chunk_lat, "chunk_lat", dt, (B, n_q, D)),
        _ptr(cache, "cache", dt, (B, c.window_frames * tpf, D)),
        _ptr(slot_frame, "slot_frame", torch.int32, (B, c.window_frames)), n_valid_frames,
        first_frame, _ptr(w_uv, "w_uv", dt, (H, c.d_head, c.d_c)), _ptr(out, "out", dt, out_shape),
        _ptr(lse, "lse", torch.float32, (B, H, n_q)), _ptr(dev_status, "dev_status", torch.int32),
        _stream(stream))
    _lib.check("mla_attention_fwd_static_scratch", st)
