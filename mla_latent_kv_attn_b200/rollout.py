"""Host-side driver of a chunked rollout: the schedule, the ring state and the per-chunk calls.

A rollout generates chunk after chunk of ``chunk_frames`` latent frames.  Chunk c covers frames
c*C .. c*C + C - 1; it attends to the frames still in the window (at most W earlier frames) and
to itself, then its latents enter the ring (hyper.ai summary of VideoMLA, "Introduction":
streaming students generate frames with a rolling key-value cache; chatpaper abstract: the
window has a fixed size).

The ring stores frame f in slot f mod W.  Frames are appended in order from frame 0, so the
first min(frames so far, W) slots are exactly the filled ones and attention walks slots
0 .. n_valid*tpf - 1 (the softmax does not depend on key order).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import torch

from . import api
from .api import MLA_APPEND, MLA_PROJECT, MLA_PROJECT_AND_APPEND


def chunk_schedule(chunk_frames: int, window_frames: int, chunk: int) -> Tuple[int, int]:
    """(first_frame, n_valid_frames) of a chunk."""
    first = chunk * chunk_frames
    return first, min(first, window_frames)


@dataclasses.dataclass
class DeviceWeights:
    """One layer's weights on the device, in the layouts the C ABI takes."""

    w_dkv_kr: torch.Tensor   # [d_c + d_rope, d_model]
    w_dq: torch.Tensor       # [d_cq, d_model]
    w_x: torch.Tensor        # [d_cq + d_c + d_rope, d_model]: W_down^Q, W_down^KV, W_R^K stacked
    w_qcat: torch.Tensor     # [H, d_c + d_rope, d_cq]  (composed on the device)
    w_uv: torch.Tensor       # [H, d_head, d_c]
    w_o: torch.Tensor        # [d_model, H*d_head]


def upload_weights(c, lw, device="cuda", stream=None) -> DeviceWeights:
    """Copies a layer's weights (numpy, already dtype-rounded) and composes the absorbed query
    weights on the device."""
    dt = api.torch_dtype(c)
    t = lambda a: torch.from_numpy(a).to(device=device, dtype=dt).contiguous()
    import numpy as np
    w_uq, w_uk, w_qr = t(lw.w_uq), t(lw.w_uk), t(lw.w_qr)
    w_qcat = torch.empty((c.n_heads, c.d_c + c.d_rope, c.d_cq), device=device, dtype=dt)
    api.mla_compose_query_weights(c, w_uq, w_uk, w_qr, w_qcat, stream=stream)
    w_x = t(np.concatenate([lw.w_dq, lw.w_dkv, lw.w_kr], 0))
    return DeviceWeights(w_dkv_kr=w_x[c.d_cq:], w_dq=w_x[:c.d_cq], w_x=w_x, w_qcat=w_qcat,
                         w_uv=t(lw.w_uv), w_o=t(lw.w_o))


class Ring:
    """The latent cache of one layer for B samples: cache [B, W*tpf, D] and slot_frame [B, W]."""

    def __init__(self, c, device="cuda"):
        tpf = c.frame_h * c.frame_w
        self.c = c
        self.cache = torch.zeros((c.batch, c.window_frames * tpf, c.d_c + c.d_rope),
                                 device=device, dtype=api.torch_dtype(c))
        self.slot_frame = torch.full((c.batch, c.window_frames), -1, device=device,
                                     dtype=torch.int32)

    def state_dict(self):
        return {"cache": self.cache.clone(), "slot_frame": self.slot_frame.clone()}

    def load_state_dict(self, sd):
        self.cache.copy_(sd["cache"])
        self.slot_frame.copy_(sd["slot_frame"])


class ChunkBuffers:
    """Per-chunk activations and scratch, allocated once per workload."""

    def __init__(self, c, device="cuda", fuse_uv: bool = True):
        tpf = c.frame_h * c.frame_w
        n_q = c.chunk_frames * tpf
        D = c.d_c + c.d_rope
        dt = api.torch_dtype(c)
        B, H = c.batch, c.n_heads
        self.x = torch.empty((B, n_q, c.d_model), device=device, dtype=dt)
        self.c_q = torch.empty((B, n_q, c.d_cq), device=device, dtype=dt)
        self.q = torch.empty((B, n_q, H, D), device=device, dtype=dt)
        self.chunk_lat = torch.empty((B, n_q, D), device=device, dtype=dt)
        self.o = torch.empty((B, n_q, H * c.d_head), device=device, dtype=dt)
        self.o_lat = torch.empty((B, n_q, H, c.d_c), device=device, dtype=dt)
        self.lse = torch.empty((B, H, n_q), device=device, dtype=torch.float32)
        ws = api.mla_attention_workspace_bytes(c, c.window_frames)
        self.workspace = torch.empty((max(ws, 256),), device=device, dtype=torch.uint8)
        self.dev_status = torch.zeros((1,), device=device, dtype=torch.int32)


def fused_query_supported(c) -> bool:
    """Whether mla_attention_fwd_from_cq (query heads formed inside the attention kernel) serves
    this configuration."""
    return (c.dtype == api.MLA_BF16 and c.kernel_path != api.MLA_PATH_SIMT
            and c.d_c in (128, 192) and c.d_rope in (16, 32, 64) and c.d_c + c.d_rope <= 256
            and c.d_cq % 64 == 0 and c.d_head == 128)


def _use_fused_q(c, fused_q: Optional[bool]) -> bool:
    """fused_q as given, or (None) the fused form wherever the configuration allows it."""
    return fused_query_supported(c) if fused_q is None else bool(fused_q)


def attend_chunk(c, w: DeviceWeights, ring: Ring, buf: ChunkBuffers, chunk: int,
                 fuse_uv: bool = True, stream=None, fused_q: Optional[bool] = None) -> torch.Tensor:
    """Query path, chunk latents and attention of one chunk (buf.x holds its tokens).
    Returns buf.o (fused W_UV) or buf.o_lat (latent output).  With fused_q the x-projection also
    writes every rotated positional key of the call and the attention kernel forms the query
    heads itself from c_Q (buf.q is then not written): two launches.  fused_q=None picks the
    fused form wherever the configuration allows it."""
    first, n_valid = chunk_schedule(c.chunk_frames, c.window_frames, chunk)
    out = buf.o if fuse_uv else buf.o_lat
    if _use_fused_q(c, fused_q):
        _attend_from_cq(c, w, ring, buf, buf.x, n_valid, first, out, fuse_uv, buf.workspace,
                        rotate_ring=True, stream=stream)
        return out
    api.mla_project_chunk(c, buf.x, w.w_x, w.w_qcat, buf.c_q, buf.q, buf.chunk_lat, first,
                          stream=stream)
    api.mla_attention_fwd(c, buf.q, buf.chunk_lat, ring.cache, ring.slot_frame, n_valid, first,
                          w.w_uv if fuse_uv else None, out, buf.lse, buf.workspace,
                          buf.dev_status, stream=stream)
    return out


def _attend_from_cq(c, w: DeviceWeights, ring: Ring, buf: ChunkBuffers, x, n_valid: int,
                    first: int, out, fuse_uv: bool, workspace, rotate_ring: bool,
                    stream=None) -> None:
    """The two calls of a chunk's attention with the query heads formed in the attention kernel:
    the x-projection with the rotated keys (mla_project_latents_rotated) and the attention with
    no rotation pass."""
    api.mla_project_latents_rotated(c, x, w.w_x, buf.c_q, buf.chunk_lat, ring.cache,
                                    ring.slot_frame, n_valid, first, workspace,
                                    rotate_ring=rotate_ring, dev_status=buf.dev_status,
                                    stream=stream)
    api.mla_attention_fwd_from_cq(c, buf.c_q, w.w_qcat, buf.chunk_lat, ring.cache,
                                  ring.slot_frame, n_valid, first, w.w_uv if fuse_uv else None,
                                  out, buf.lse, workspace, buf.dev_status, stream=stream,
                                  prerotated=True)


def append_chunk(c, ring: Ring, buf: ChunkBuffers, chunk: int, stream=None) -> None:
    """Moves the chunk's latents (buf.chunk_lat) into the ring, after its attention."""
    first, _ = chunk_schedule(c.chunk_frames, c.window_frames, chunk)
    api.mla_cache_append(c, None, None, buf.chunk_lat, ring.cache, ring.slot_frame, first,
                         MLA_APPEND, stream=stream)


def prefill_chunk(c, w: DeviceWeights, ring: Ring, buf: ChunkBuffers, chunk: int,
                  stream=None) -> None:
    """Projects buf.x and appends it to the ring without attending (cache warm-up)."""
    first, _ = chunk_schedule(c.chunk_frames, c.window_frames, chunk)
    api.mla_cache_append(c, buf.x, w.w_dkv_kr, buf.chunk_lat, ring.cache, ring.slot_frame, first,
                         MLA_PROJECT_AND_APPEND, stream=stream)


def run_chunk(c, w: DeviceWeights, ring: Ring, buf: ChunkBuffers, chunk: int,
              fuse_uv: bool = True, stream=None, fused_q: Optional[bool] = None) -> torch.Tensor:
    """One whole chunk: attend, then append."""
    out = attend_chunk(c, w, ring, buf, chunk, fuse_uv=fuse_uv, stream=stream, fused_q=fused_q)
    append_chunk(c, ring, buf, chunk, stream=stream)
    return out


def check_device_status(buf: ChunkBuffers) -> None:
    """Raises if a kernel reported a bounded wait that ran out (reads one int; synchronises)."""
    v = int(buf.dev_status.item())
    if v != 0:
        raise api.MLAError("device", v, "a kernel's bounded wait ran out")


class HostStreamer:
    """Drives chunks whose tokens are in pinned host memory and whose outputs go back to pinned
    host memory, with the copies overlapped with the device work of neighbouring chunks.

    Two device buffer sets alternate.  Chunk n's tokens travel host -> device on one copy stream
    while chunk n-1 computes; chunk n's output travels device -> host on a second copy stream
    while chunk n+1 computes.  CUDA events order every reuse of a buffer:
      - the copy into buffer set k waits until the chunk that last used set k has finished;
      - the compute of a chunk waits for its tokens and for the copy-out of the output that
        used the same buffer set two chunks earlier.
    Chunks still compute strictly in order on the compute stream, so the ring sees exactly the
    append order of run_chunk.  Nothing here synchronises the host.
    """

    def __init__(self, c, w: DeviceWeights, ring: Ring, device="cuda", compute_stream=None):
        self.c, self.w, self.ring = c, w, ring
        self.bufs = [ChunkBuffers(c, device=device), ChunkBuffers(c, device=device)]
        self.compute = compute_stream or torch.cuda.current_stream(device)
        self.h2d = torch.cuda.Stream(device=device)
        self.d2h = torch.cuda.Stream(device=device)
        self.x_free = [None, None]   # event: the compute that last read bufs[k] is done
        self.o_free = [None, None]   # event: the copy-out of bufs[k].o is done
        self.n = 0

    def begin(self, event: torch.cuda.Event) -> None:
        """Makes both copy streams wait for `event` (e.g. the start of a timed region)."""
        self.h2d.wait_event(event)
        self.d2h.wait_event(event)

    def submit(self, chunk: int, x_host: torch.Tensor, o_host: torch.Tensor,
               fuse_uv: bool = True, fused_q: Optional[bool] = None,
               ring: Optional[Ring] = None) -> None:
        """Enqueues chunk `chunk`: copy-in of x_host, attention, append, copy-out into o_host.
        `ring` (default: the streamer's own) lets one streamer serve several independent
        rollouts, each with its ring; chunks of one ring still run in submission order."""
        ring = self.ring if ring is None else ring
        k = self.n % 2
        b = self.bufs[k]
        with torch.cuda.stream(self.h2d):
            if self.x_free[k] is not None:
                self.h2d.wait_event(self.x_free[k])
            b.x.copy_(x_host, non_blocking=True)
            x_ready = torch.cuda.Event()
            x_ready.record(self.h2d)
        self.compute.wait_event(x_ready)
        if self.o_free[k] is not None:
            self.compute.wait_event(self.o_free[k])
        out = run_chunk(self.c, self.w, ring, b, chunk, fuse_uv=fuse_uv, stream=self.compute,
                        fused_q=fused_q)
        done = torch.cuda.Event()
        done.record(self.compute)
        self.x_free[k] = done
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(done)
            o_host.copy_(out, non_blocking=True)
            o_done = torch.cuda.Event()
            o_done.record(self.d2h)
        self.o_free[k] = o_done
        self.n += 1

    def finish(self) -> None:
        """Makes the compute stream wait for every copy issued so far."""
        for e in self.o_free:
            if e is not None:
                self.compute.wait_event(e)

    def check_device_status(self) -> None:
        for b in self.bufs:
            check_device_status(b)


class ChunkGraph:
    """One chunk's whole path (projections, attention, append) captured as a CUDA graph.

    A chunk's kernels depend on its index only through launch parameters (first frame, valid
    frames, ring slots), so each chunk index gets its own graph; capturing is host-side work
    that can run ahead of the device, and a replay launches the chunk's kernels back to back
    without per-kernel host overhead.  Buffers, ring and weights are bound at capture time and
    must stay alive and in place while the graph is used.  `events=True` also records timing
    events inside the graph around each of the chunk's three calls: the projections
    (proj_start .. attn_start), the attention call (attn_start .. attn_end) and the append
    (attn_end .. append_end).
    """

    def __init__(self, c, w: DeviceWeights, ring: Ring, buf: ChunkBuffers, chunk: int,
                 x: Optional[torch.Tensor] = None, events: bool = False, fuse_uv: bool = True,
                 fused_q: Optional[bool] = None):
        self.chunk = chunk
        fused_q = _use_fused_q(c, fused_q)
        first, n_valid = chunk_schedule(c.chunk_frames, c.window_frames, chunk)
        x = buf.x if x is None else x
        # external events: recorded by the graph at replay time (a plain event recorded during
        # capture only orders the graph's nodes and cannot be timed)
        mk = lambda: torch.cuda.Event(enable_timing=True, external=True) if events else None
        self.proj_start, self.attn_start, self.attn_end, self.append_end = mk(), mk(), mk(), mk()
        self.graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(self.graph, stream=side, capture_error_mode="relaxed"):
            if events:
                self.proj_start.record()
            if fused_q:
                api.mla_project_latents_rotated(c, x, w.w_x, buf.c_q, buf.chunk_lat, ring.cache,
                                                ring.slot_frame, n_valid, first, buf.workspace,
                                                dev_status=buf.dev_status)
            else:
                api.mla_project_chunk(c, x, w.w_x, w.w_qcat, buf.c_q, buf.q, buf.chunk_lat, first)
            if events:
                self.attn_start.record()
            out = buf.o if fuse_uv else buf.o_lat
            if fused_q:
                api.mla_attention_fwd_from_cq(c, buf.c_q, w.w_qcat, buf.chunk_lat, ring.cache,
                                              ring.slot_frame, n_valid, first,
                                              w.w_uv if fuse_uv else None, out, buf.lse,
                                              buf.workspace, buf.dev_status, prerotated=True)
            else:
                api.mla_attention_fwd(c, buf.q, buf.chunk_lat, ring.cache, ring.slot_frame,
                                      n_valid, first, w.w_uv if fuse_uv else None, out, buf.lse,
                                      buf.workspace, buf.dev_status)
            if events:
                self.attn_end.record()
            api.mla_cache_append(c, None, None, buf.chunk_lat, ring.cache, ring.slot_frame,
                                 first, MLA_APPEND)
            if events:
                self.append_end.record()
        torch.cuda.current_stream().wait_stream(side)
        self.out = out

    def replay(self) -> torch.Tensor:
        self.graph.replay()
        return self.out

    def attention_ms(self) -> float:
        return self.attn_start.elapsed_time(self.attn_end)

    def projection_ms(self) -> float:
        return self.proj_start.elapsed_time(self.attn_start)

    def append_ms(self) -> float:
        return self.attn_end.elapsed_time(self.append_end)


class LayerStack:
    """A stack of attention layers, each with its own weights and ring, driven through a chunked
    rollout with several denoising steps per chunk.

    Every step of a chunk runs every layer's attention against that layer's ring, which stays
    frozen until the chunk is finished (hyper.ai summary of VideoMLA, "Introduction": the cache
    rolls forward chunk by chunk).  So the positional keys of each ring are rotated once per
    chunk (mla_rotate_ring_keys into the layer's own workspace) and every step only rotates the
    chunk's keys: in the x-projection's epilogue with the fused query heads
    (mla_project_latents_rotated with rotate_ring=False, then the attention with no rotation
    pass), else in mla_attention_fwd_cached_ring.  At the last step each layer
    appends the chunk's latents to its ring right after its attention.

    One set of chunk activations (buf) is shared by all layers: a call's outputs are valid until
    the next call.  capture_chunk() records a whole chunk (rotations, every step and layer,
    appends) as one CUDA graph, with the step/layer inputs bound at capture time.
    """

    def __init__(self, c, weights, device="cuda", fuse_uv: bool = True,
                 fused_q: Optional[bool] = None):
        self.c = c
        # the query heads formed inside the attention kernel where the configuration allows
        self.fused_q = fused_query_supported(c) if fused_q is None else fused_q
        self.w = list(weights)
        self.rings = [Ring(c, device=device) for _ in self.w]
        ws = max(api.mla_attention_workspace_bytes(c, c.window_frames), 256)
        self.ws = [torch.empty((ws,), device=device, dtype=torch.uint8) for _ in self.w]
        self.buf = ChunkBuffers(c, device=device)
        self.fuse_uv = fuse_uv

    @property
    def n_layers(self) -> int:
        return len(self.w)

    def begin_chunk(self, chunk: int, stream=None) -> None:
        """Rotates every layer's ring keys for this chunk's (frozen) ring state."""
        _, n_valid = chunk_schedule(self.c.chunk_frames, self.c.window_frames, chunk)
        for l in range(self.n_layers):
            api.mla_rotate_ring_keys(self.c, self.rings[l].cache, self.rings[l].slot_frame,
                                     n_valid, self.ws[l], stream=stream)

    def attend(self, chunk: int, layer: int, x: torch.Tensor, append: bool = False,
               stream=None) -> torch.Tensor:
        """One layer's projections and attention for one step of the chunk (x: [B, n_q, d_model]
        on the device); with append=True (the chunk's last step) the layer's ring takes the
        chunk's latents afterwards.  Returns buf.o (or buf.o_lat without the W_UV epilogue)."""
        c, b, w, ring = self.c, self.buf, self.w[layer], self.rings[layer]
        first, n_valid = chunk_schedule(c.chunk_frames, c.window_frames, chunk)
        out = b.o if self.fuse_uv else b.o_lat
        if self.fused_q:
            # the ring part of the layer's workspace was rotated by begin_chunk; the projection
            # writes the chunk's rotated keys next to it
            _attend_from_cq(c, w, ring, b, x, n_valid, first, out, self.fuse_uv, self.ws[layer],
                            rotate_ring=False, stream=stream)
        else:
            api.mla_project_chunk(c, x, w.w_x, w.w_qcat, b.c_q, b.q, b.chunk_lat, first,
                                  stream=stream)
            api.mla_attention_fwd_cached_ring(c, b.q, b.chunk_lat, ring.cache, ring.slot_frame,
                                              n_valid, first, w.w_uv if self.fuse_uv else None,
                                              out, b.lse, self.ws[layer], b.dev_status,
                                              stream=stream)
        if append:
            api.mla_cache_append(c, None, None, b.chunk_lat, ring.cache, ring.slot_frame, first,
                                 MLA_APPEND, stream=stream)
        return out

    def run_chunk(self, chunk: int, n_steps: int, x_of, stream=None) -> None:
        """A whole chunk: n_steps steps through every layer; x_of(step, layer) gives the device
        input of each call."""
        self.begin_chunk(chunk, stream=stream)
        for s in range(n_steps):
            for l in range(self.n_layers):
                self.attend(chunk, l, x_of(s, l), append=(s == n_steps - 1), stream=stream)

    def capture_chunk(self, chunk: int, n_steps: int, x_of) -> torch.cuda.CUDAGraph:
        """run_chunk recorded as one CUDA graph (inputs x_of(step, layer) bound at capture)."""
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
            self.run_chunk(chunk, n_steps, x_of)
        torch.cuda.current_stream().wait_stream(side)
        return g
