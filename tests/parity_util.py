"""Shared harness of the GPU parity tests: run a rollout through the C ABI and the same rollout
through the CPU oracle on identical seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mla_latent_kv_attn_b200 import api, inputs, rollout

# Tolerances against the float64 oracle.
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
FP32_MAX_ABS = 1e-4


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare(name: str, got, ref, dtype: str, report: dict | None = None):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{name}: shape {got.shape} vs {ref.shape}"
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    err = got - ref
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)) if err.size else 0.0
    if report is not None:
        report[name] = (max_abs, rel)
    if dtype == "fp32":
        assert max_abs <= FP32_MAX_ABS, f"{name}: max-abs {max_abs:.3e} > {FP32_MAX_ABS}"
    else:
        assert max_abs <= BF16_MAX_ABS, f"{name}: max-abs {max_abs:.3e} > {BF16_MAX_ABS}"
        assert rel <= BF16_REL_L2, f"{name}: rel-L2 {rel:.3e} > {BF16_REL_L2}"
    return max_abs, rel


class GpuRun:
    """One layer's rollout through the C ABI."""

    def __init__(self, cfg, path=api.MLA_PATH_AUTO, layer=0, weights=None):
        self.cfg = cfg
        self.c = api.make_config(cfg, kernel_path=path)
        self.lw = weights if weights is not None else inputs.layer_weights(cfg, layer)
        self.w = rollout.upload_weights(self.c, self.lw)
        self.ring = rollout.Ring(self.c)
        self.buf = rollout.ChunkBuffers(self.c)
        self.dt = api.torch_dtype(self.c)

    def load_x(self, x: np.ndarray):
        self.buf.x.copy_(torch.from_numpy(x).to(self.dt))

    def prefill(self, chunk: int, x: np.ndarray):
        self.load_x(x)
        rollout.prefill_chunk(self.c, self.w, self.ring, self.buf, chunk)

    def attend(self, chunk: int, x: np.ndarray, want_latent=True, fused_q=False):
        """Runs the chunk's attention (fused W_UV and, optionally, latent output); returns numpy
        copies of every intermediate.  Does not append.  With fused_q the attention kernel forms
        the query heads itself (no q in the result)."""
        self.load_x(x)
        self.buf.dev_status.zero_()
        o = rollout.attend_chunk(self.c, self.w, self.ring, self.buf, chunk, fuse_uv=True,
                                 fused_q=fused_q)
        res = dict(o=to_np(o), lse=to_np(self.buf.lse), c_q=to_np(self.buf.c_q),
                   chunk_lat=to_np(self.buf.chunk_lat))
        if not fused_q:
            res["q"] = to_np(self.buf.q)
        if want_latent:
            first, n_valid = rollout.chunk_schedule(self.cfg.chunk_frames, self.cfg.window_frames,
                                                    chunk)
            if fused_q:
                api.mla_attention_fwd_from_cq(self.c, self.buf.c_q, self.w.w_qcat,
                                              self.buf.chunk_lat, self.ring.cache,
                                              self.ring.slot_frame, n_valid, first, None,
                                              self.buf.o_lat, None, self.buf.workspace,
                                              self.buf.dev_status)
            else:
                api.mla_attention_fwd(self.c, self.buf.q, self.buf.chunk_lat, self.ring.cache,
                                      self.ring.slot_frame, n_valid, first, None, self.buf.o_lat,
                                      None, self.buf.workspace, self.buf.dev_status)
            res["o_lat"] = to_np(self.buf.o_lat)
        torch.cuda.synchronize()
        rollout.check_device_status(self.buf)
        return res

    def key_positions(self, chunk: int) -> np.ndarray:
        first, n_valid = rollout.chunk_schedule(self.cfg.chunk_frames, self.cfg.window_frames, chunk)
        n_keys = n_valid * self.cfg.tokens_per_frame + self.cfg.n_q
        pos = torch.empty((self.cfg.batch, n_keys, 3), device="cuda", dtype=torch.int32)
        api.mla_key_positions(self.c, self.ring.slot_frame, n_valid, first, pos)
        return pos.cpu().numpy()

    def append(self, chunk: int):
        rollout.append_chunk(self.c, self.ring, self.buf, chunk)


class OracleRun:
    """The same rollout on the CPU oracle, one window per sample."""

    def __init__(self, cfg, lw):
        self.cfg = cfg
        self.d = oracle.dims_from(cfg)
        self.lw = lw
        self.windows = [oracle.SlidingWindow(self.d) for _ in range(cfg.batch)]

    def prefill(self, chunk: int, x: np.ndarray):
        first = chunk * self.cfg.chunk_frames
        for b in range(self.cfg.batch):
            c_kv, k_r = oracle.down_project(x[b], self.lw.w_dkv, self.lw.w_kr)
            self.windows[b].append_chunk(first, c_kv, k_r)

    def step(self, chunk: int, x: np.ndarray, rows, samples=None, append=True):
        first = chunk * self.cfg.chunk_frames
        out = []
        for b in range(self.cfg.batch):
            if samples is not None and b not in samples:
                if append:
                    c_kv, k_r = oracle.down_project(x[b], self.lw.w_dkv, self.lw.w_kr)
                    self.windows[b].append_chunk(first, c_kv, k_r)
                out.append(None)
                continue
            r = oracle.chunk_step(self.d, self.lw, x[b], self.windows[b], first, rows=rows,
                                  append=append)
            r["q_abs"] = oracle.absorbed_query(r["c_q"], self.lw.w_uq, self.lw.w_uk, self.lw.w_qr,
                                               r["pos_q"], self.d)
            out.append(r)
        return out


def check_chunk(name, cfg, g, o_res, rows, report=None, samples=None):
    """Compares the GPU intermediates of one chunk with the oracle's, for every sample."""
    dt = cfg.dtype
    for b, r in enumerate(o_res):
        if r is None:
            continue
        tag = f"{name}[b{b}]"
        lat_ref = np.concatenate([r["c_kv"], r["k_r"]], axis=1)
        compare(tag + ".chunk_lat", g["chunk_lat"][b], lat_ref, dt, report)
        compare(tag + ".c_q", g["c_q"][b][rows], r["c_q"], dt, report)
        if "q" in g:
            compare(tag + ".q", g["q"][b][rows], r["q_abs"], dt, report)
        compare(tag + ".o", g["o"][b][rows], r["o"], dt, report)
        if "o_lat" in g:
            compare(tag + ".o_lat", g["o_lat"][b][rows], r["o_lat"], dt, report)
        lse_tol = "fp32" if dt == "fp32" else "bf16"
        compare(tag + ".lse", g["lse"][b][:, rows], r["lse"], lse_tol, report)


def expected_slot_frame(cfg, window: oracle.SlidingWindow) -> np.ndarray:
    sf = np.full(cfg.window_frames, -1, dtype=np.int64)
    for t in window.frame_indices():
        sf[t % cfg.window_frames] = t
    return sf


def check_ring(cfg, gpu: GpuRun, orc: OracleRun, report=None):
    """Ring contents after an append: slot_frame bit-exact, cached latents within tolerance."""
    sf = gpu.ring.slot_frame.cpu().numpy()
    cache = to_np(gpu.ring.cache)
    tpf = cfg.tokens_per_frame
    for b in range(cfg.batch):
        exp = expected_slot_frame(cfg, orc.windows[b])
        np.testing.assert_array_equal(sf[b], exp)
        recs = {r.t: r for r in orc.windows[b].frames}
        for s, t in enumerate(sf[b]):
            if t < 0:
                continue
            ref = np.concatenate([recs[t].c_kv, recs[t].k_r], axis=1)
            compare(f"ring[b{b}].slot{s}", cache[b, s * tpf:(s + 1) * tpf], ref, cfg.dtype, report)


def expected_key_positions(cfg, window: oracle.SlidingWindow, first: int) -> np.ndarray:
    """Keys in the walk order of the kernels: ring slots 0..n_valid-1, then the chunk."""
    d = oracle.dims_from(cfg)
    frames = window.frame_indices()
    by_slot = sorted(frames, key=lambda t: t % cfg.window_frames)
    return np.concatenate([oracle.token_positions(by_slot, d),
                           oracle.token_positions(range(first, first + cfg.chunk_frames), d)])
