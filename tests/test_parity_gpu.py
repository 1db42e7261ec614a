"""GPU parity: the CUDA path through the C ABI against the float64 CPU oracle, element by
element, on identical seeded inputs.

Floating point: bf16 workloads within max-abs 2e-2 and rel-L2 5e-3, fp32 within max-abs 1e-4,
for every intermediate the ABI exposes (chunk latents, query latent, absorbed query, latent
output, output, lse).  Integer work (key positions, ring slots) is bit-exact.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_attn_b200 import api, inputs, rollout
from parity_util import (GpuRun, OracleRun, check_chunk, check_ring, compare,
                         expected_key_positions, to_np)

pytestmark = pytest.mark.gpu

# "tc": the default path (tensor cores, one CTA per head and query tile); "pair": the CTA-pair
# attention kernel; "simt": CUDA cores
PATHS = {"tc": api.MLA_PATH_AUTO, "pair": api.MLA_PATH_TC_PAIR, "simt": api.MLA_PATH_SIMT}


def full_rollout(cfg, path, rows=None, check_positions=True):
    g = GpuRun(cfg, path)
    o = OracleRun(cfg, g.lw)
    rows = np.arange(cfg.n_q) if rows is None else rows
    report = {}
    for ch in range(cfg.n_chunks):
        x = inputs.chunk_x(cfg, ch)
        first = cfg.first_frame(ch)
        if check_positions:
            pos = g.key_positions(ch)
            for b in range(cfg.batch):
                np.testing.assert_array_equal(pos[b], expected_key_positions(cfg, o.windows[b], first))
        gres = g.attend(ch, x)
        ores = o.step(ch, x, rows)
        check_chunk(f"chunk{ch}", cfg, gres, ores, rows, report)
        g.append(ch)
        check_ring(cfg, g, o, report)
    return report


def test_toy_fp32_rollout_wraps_and_matches():
    """Config 0: 4 chunks of 1 frame, window of 2 frames (the ring wraps at chunk 2)."""
    full_rollout(inputs.CONFIGS[0], api.MLA_PATH_AUTO)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_small_frames_bf16_rollout(path):
    """Wan layer widths on 6x10 frames: 180 queries (2 tiles, ragged), 0..240 ring keys."""
    full_rollout(inputs.small_bf16_config(), PATHS[path])


LATENT_SHAPES = [(dc, dr) for dc in (128, 192, 256) for dr in (16, 32, 64)]


@pytest.mark.parametrize("fused_q", [False, True])
def test_window_of_one_chunk_replaces_the_whole_ring(fused_q):
    """Degenerate window: W = C = 3 frames, so every append overwrites every slot of the ring and
    each chunk attends to exactly the previous chunk plus itself.  A 5-chunk rollout of 2
    samples on both paths (unfused; the 3-launch step), every row and the ring against the
    oracle."""
    cfg = dataclasses.replace(inputs.small_bf16_config(), window_frames=3, n_chunks=5,
                              name="wan_layer_small_frames_w3")
    g = GpuRun(cfg)
    o = OracleRun(cfg, g.lw)
    rows = np.arange(cfg.n_q)
    for ch in range(cfg.n_chunks):
        x = inputs.chunk_x(cfg, ch)
        check_chunk(f"w3.chunk{ch}", cfg, g.attend(ch, x, fused_q=fused_q), o.step(ch, x, rows), rows)
        g.append(ch)
        check_ring(cfg, g, o)
    assert int(g.ring.slot_frame.min()) == 3 * (cfg.n_chunks - 1)


@pytest.mark.parametrize("path", ["tc", "pair"])
@pytest.mark.parametrize("d_c,d_rope", LATENT_SHAPES)
def test_latent_shape_sweep_tensor_cores_match_oracle(d_c, d_rope, path):
    """The latent-size ablation shapes (d_c in {128, 192, 256} x d_rope in {16, 32, 64}) run on
    the tensor-core kernels (the one-CTA kernel on the default path, and the CTA-pair kernel for
    d_c 128 and 192) and match the oracle over a 4-chunk rollout whose ring wraps."""
    if path == "pair" and d_c == 256:
        pytest.skip("d_c 256 has no CTA-pair kernel (no TMEM room for two S buffers)")
    cfg = inputs.with_latent_shape(inputs.small_bf16_config(), d_c, d_rope)
    c = api.make_config(cfg, kernel_path=PATHS[path])
    assert api.mla_attention_uses_tensor_cores(c, True)
    assert api.mla_attention_uses_tensor_cores(c, False)
    report = full_rollout(cfg, PATHS[path])
    worst = max(v[1] for k, v in report.items() if k.endswith(".o"))
    assert worst <= 5e-3


def prefilled(cfg, path, upto):
    g = GpuRun(cfg, path)
    o = OracleRun(cfg, g.lw)
    for ch in range(upto):
        x = inputs.chunk_x(cfg, ch)
        g.prefill(ch, x)
        o.prefill(ch, x)
    return g, o


def test_wan_config1_sampled_rows():
    """Config 1 at full size (B1, window 6 frames full, chunk of 3 frames), 384 sampled rows."""
    cfg = inputs.CONFIGS[1]
    g, o = prefilled(cfg, api.MLA_PATH_AUTO, cfg.measured_chunk)
    check_ring(cfg, g, o)
    ch = cfg.measured_chunk
    x = inputs.chunk_x(cfg, ch)
    rows = inputs.sample_rows(cfg.n_q, 384, tag=1)
    pos = g.key_positions(ch)
    np.testing.assert_array_equal(pos[0], expected_key_positions(cfg, o.windows[0], cfg.first_frame(ch)))
    check_chunk("cfg1", cfg, g.attend(ch, x), o.step(ch, x, rows), rows)
    g.append(ch)
    check_ring(cfg, g, o)


def test_largest_accepted_batch_on_the_bench_path():
    """The largest batch the library accepts for the Wan preset (170 samples; at 171 the unfused
    path's Q' array would reach 2^31 elements) through the bench's 3-launch step, one chunk after
    the window filled: the kernels' address arithmetic at the largest legal offsets.  The first
    and the last sample get their seeded inputs and are compared with the oracle on sampled rows
    (every 128-row query tile represented); the other samples get arbitrary values, which
    cannot reach the checked ones (samples are independent)."""
    cfg = inputs.CONFIGS[1]
    top = 170
    c = api.make_config(cfg, batch=top)
    lw = inputs.layer_weights(cfg)
    w = rollout.upload_weights(c, lw)
    ring, buf = rollout.Ring(c), rollout.ChunkBuffers(c)
    d = oracle.dims_from(cfg)
    checked = (0, top - 1)
    windows = {b: oracle.SlidingWindow(d) for b in checked}
    gen = torch.Generator(device="cuda").manual_seed(1234)
    rows = inputs.sample_rows(cfg.n_q, 192, tag=170)
    assert len(set(rows // 128)) == -(-cfg.n_q // 128)
    for ch in range(cfg.measured_chunk + 1):
        buf.x.normal_(generator=gen)
        xs = {}
        for b in checked:
            xs[b] = inputs.chunk_x(cfg, ch, samples=range(b, b + 1))[0]
            buf.x[b].copy_(torch.from_numpy(xs[b]).to(torch.bfloat16))
        first = cfg.first_frame(ch)
        if ch < cfg.measured_chunk:
            rollout.prefill_chunk(c, w, ring, buf, ch)
            for b in checked:
                c_kv, k_r = oracle.down_project(xs[b], lw.w_dkv, lw.w_kr)
                windows[b].append_chunk(first, c_kv, k_r)
            continue
        out = rollout.attend_chunk(c, w, ring, buf, ch)
        torch.cuda.synchronize()
        rollout.check_device_status(buf)
        for b in checked:
            r = oracle.chunk_step(d, lw, xs[b], windows[b], first, rows=rows, append=False)
            compare(f"batch{top}.o[b{b}]", to_np(out[b])[rows], r["o"], cfg.dtype)
            compare(f"batch{top}.lse[b{b}]", to_np(buf.lse[b])[:, rows], r["lse"], "bf16")


def test_wan_config3_batch8_sampled_rows():
    """Config 3: 8 independent samples, window 9 frames, chunk 3 frames, on the bench's path
    (rotated keys from the x-projection, query heads formed in the attention kernel); 512
    sampled rows of every sample (every 128-row query tile holds some) against the oracle, every
    row against the unfused path, then the append and every sample's ring (slots bit-exact,
    contents within tolerance)."""
    cfg = inputs.CONFIGS[3]
    g, o = prefilled(cfg, api.MLA_PATH_AUTO, cfg.measured_chunk)
    check_ring(cfg, g, o)
    ch = cfg.measured_chunk
    x = inputs.chunk_x(cfg, ch)
    rows = inputs.sample_rows(cfg.n_q, 512, tag=3)
    assert len(set(rows // 128)) == -(-cfg.n_q // 128)
    pos = g.key_positions(ch)
    for b in range(cfg.batch):
        np.testing.assert_array_equal(pos[b], expected_key_positions(cfg, o.windows[b], cfg.first_frame(ch)))
    rf = g.attend(ch, x, fused_q=True)
    check_chunk("cfg3", cfg, rf, o.step(ch, x, rows), rows)
    ra = g.attend(ch, x)
    for k in ("o", "o_lat", "lse"):
        assert np.abs(ra[k] - rf[k]).max() <= 2.0 ** -8 * max(1.0, np.abs(ra[k]).max()), k
    g.append(ch)
    check_ring(cfg, g, o)


def test_wan_config2_long_rollout_sampled():
    """Config 2: 80 chunks, window 21 frames; temporal positions reach t = 239 and the ring
    wraps every 7 chunks.  Every chunk runs the whole path on the GPU as the bench runs it
    (rotated keys from the x-projection, query heads formed in the attention kernel).  The
    oracle evaluates 512
    sampled rows (every query tile holds some) with all heads at chunks 0-8 (the window fills,
    then the first wraps) and 76-79 (t up to 239), with the key positions; after every chunk's
    append the whole ring is compared (slots bit-exact, contents within tolerance)."""
    cfg = inputs.CONFIGS[2]
    g = GpuRun(cfg, api.MLA_PATH_AUTO)
    o = OracleRun(cfg, g.lw)
    checked = set(range(9)) | set(range(76, 80))
    rows = inputs.sample_rows(cfg.n_q, 512, tag=2)
    assert len(set(rows // 128)) == -(-cfg.n_q // 128)
    for ch in range(cfg.n_chunks):
        x = inputs.chunk_x(cfg, ch)
        if ch in checked:
            pos = g.key_positions(ch)
            np.testing.assert_array_equal(pos[0], expected_key_positions(cfg, o.windows[0], cfg.first_frame(ch)))
            check_chunk(f"cfg2.chunk{ch}", cfg, g.attend(ch, x, want_latent=False, fused_q=True),
                        o.step(ch, x, rows), rows)
        else:
            g.attend(ch, x, want_latent=False, fused_q=True)
            o.prefill(ch, x)
        g.append(ch)
        check_ring(cfg, g, o)
    assert int(g.ring.slot_frame.max()) == 239


def test_pair_and_single_cta_attention_agree_on_config1():
    """Diagnostic cross-check on every row, head and output of config 1: the CTA-pair kernel
    against the one-CTA tensor-core kernel (same operands, same fp32 accumulation; only the
    order of the MMA pipeline's additions may differ, so a last-place bf16 difference at most)."""
    cfg = inputs.CONFIGS[1]
    outs = []
    for path in (api.MLA_PATH_TC_PAIR, api.MLA_PATH_AUTO):
        g, _ = prefilled(cfg, path, cfg.measured_chunk)
        outs.append(g.attend(cfg.measured_chunk, inputs.chunk_x(cfg, cfg.measured_chunk)))
    for k in ("o", "o_lat", "lse"):
        a, b = outs[0][k], outs[1][k]
        err = np.abs(a - b)
        assert np.isfinite(a).all(), k
        assert err.max() <= 2 * 2.0 ** -8 * max(1.0, np.abs(b).max()), (k, err.max())
        assert np.linalg.norm(a - b) / np.linalg.norm(b) <= 1e-3, k


FUSED_Q_SHAPES = [(dc, dr) for dc in (128, 192) for dr in (16, 32, 64)]


@pytest.mark.parametrize("d_c,d_rope", FUSED_Q_SHAPES)
def test_fused_query_heads_match_the_q_gemm(d_c, d_rope):
    """mla_attention_fwd_from_cq forms each CTA's query tile inside the attention kernel (c_Q x
    w_qcat[h] on the tensor cores, 3D-RoPE, one rounding to bf16) instead of reading Q' from the
    Q' GEMM.  Same operands, same fp32 accumulation order, same rotation code: outputs and lse
    agree with mla_project_chunk + mla_attention_fwd to the last place (checked to a bf16 ulp),
    over a 4-chunk rollout whose ring wraps, with and without the W_UV epilogue; and both match
    the oracle."""
    cfg = inputs.with_latent_shape(inputs.small_bf16_config(), d_c, d_rope)
    a, f = GpuRun(cfg), GpuRun(cfg)
    o = OracleRun(cfg, a.lw)
    rows = np.arange(cfg.n_q)
    identical = True
    for ch in range(cfg.n_chunks):
        x = inputs.chunk_x(cfg, ch)
        ra = a.attend(ch, x)
        rf = f.attend(ch, x, fused_q=True)
        for k in ("o", "o_lat", "lse", "c_q", "chunk_lat"):
            err = np.abs(ra[k] - rf[k])
            identical = identical and bool((err == 0).all())
            assert err.max() <= 2.0 ** -8 * max(1.0, np.abs(ra[k]).max()), (ch, k, err.max())
        check_chunk(f"fused.chunk{ch}", cfg, rf, o.step(ch, x, rows), rows)
        a.append(ch)
        f.append(ch)
    print("fused query heads bit-identical to the Q' GEMM path:", identical)


@pytest.mark.parametrize("d_c,d_rope", FUSED_Q_SHAPES)
def test_rotated_keys_from_the_projection_epilogue(d_c, d_rope):
    """mla_project_latents_rotated writes the chunk's rotated positional keys from the
    x-projection's epilogue and the ring's from its idle epilogue warps.  Over a 4-chunk rollout
    of 2 samples whose ring fills and wraps (chunk 0 has no ring keys): c_q and chunk_lat equal
    mla_project_latents; the workspace equals what the rotation pass of mla_attention_fwd_from_cq
    writes (padding rows included), with rotate_ring=1 from a poisoned workspace and with
    rotate_ring=0 on top of mla_rotate_ring_keys; and mla_attention_fwd_from_cq_prerotated gives
    exactly the outputs and lse of mla_attention_fwd_from_cq."""
    cfg = inputs.with_latent_shape(inputs.small_bf16_config(), d_c, d_rope)
    g = GpuRun(cfg)
    c, b, w = g.c, g.buf, g.w
    cq2, lat2 = torch.empty_like(b.c_q), torch.empty_like(b.chunk_lat)
    o2, lse2 = torch.empty_like(b.o), torch.empty_like(b.lse)
    for ch in range(cfg.n_chunks):
        first, n_valid = rollout.chunk_schedule(cfg.chunk_frames, cfg.window_frames, ch)
        nbytes = api.mla_attention_workspace_bytes(c, n_valid)
        g.load_x(inputs.chunk_x(cfg, ch))
        b.dev_status.zero_()
        # reference: plain projection, then the attention with its own rotation pass
        ws_ref = torch.full_like(b.workspace, 0x5A)
        api.mla_project_latents(c, b.x, w.w_x, b.c_q, b.chunk_lat)
        api.mla_attention_fwd_from_cq(c, b.c_q, w.w_qcat, b.chunk_lat, g.ring.cache,
                                      g.ring.slot_frame, n_valid, first, w.w_uv, b.o, b.lse,
                                      ws_ref, b.dev_status)
        # the fused projection, from a poisoned workspace
        ws = torch.full_like(b.workspace, 0xA5)
        api.mla_project_latents_rotated(c, b.x, w.w_x, cq2, lat2, g.ring.cache, g.ring.slot_frame,
                                        n_valid, first, ws, dev_status=b.dev_status)
        api.mla_attention_fwd_from_cq(c, cq2, w.w_qcat, lat2, g.ring.cache, g.ring.slot_frame,
                                      n_valid, first, w.w_uv, o2, lse2, ws, b.dev_status,
                                      prerotated=True)
        # frozen ring: ring part from mla_rotate_ring_keys, the rest from the projection
        ws_frozen = torch.full_like(b.workspace, 0x3C)
        api.mla_rotate_ring_keys(c, g.ring.cache, g.ring.slot_frame, n_valid, ws_frozen)
        api.mla_project_latents_rotated(c, b.x, w.w_x, cq2, lat2, g.ring.cache, g.ring.slot_frame,
                                        n_valid, first, ws_frozen, rotate_ring=False,
                                        dev_status=b.dev_status)
        torch.cuda.synchronize()
        assert torch.equal(cq2, b.c_q) and torch.equal(lat2, b.chunk_lat), ch
        assert torch.equal(ws[:nbytes], ws_ref[:nbytes]), ch
        assert torch.equal(ws_frozen[:nbytes], ws_ref[:nbytes]), ch
        assert torch.equal(o2, b.o) and torch.equal(lse2, b.lse), ch
        rollout.check_device_status(b)
        g.append(ch)


@pytest.mark.parametrize("which", ["fp32_toy", "bf16_cuda_cores"])
def test_rotated_keys_without_the_fused_epilogue(which):
    """Where the tensor-core GEMM does not serve (fp32, or the CUDA-core path forced),
    mla_project_latents_rotated runs the projection GEMMs and then the rotation pass; over a
    rollout whose ring wraps, its outputs and workspace equal those of mla_project_chunk and the
    rotation pass inside mla_attention_fwd."""
    cfg = inputs.CONFIGS[0] if which == "fp32_toy" else inputs.small_bf16_config()
    g = GpuRun(cfg, api.MLA_PATH_SIMT if which == "bf16_cuda_cores" else api.MLA_PATH_AUTO)
    c, b, w = g.c, g.buf, g.w
    cq2, lat2 = torch.empty_like(b.c_q), torch.empty_like(b.chunk_lat)
    for ch in range(cfg.n_chunks):
        first, n_valid = rollout.chunk_schedule(cfg.chunk_frames, cfg.window_frames, ch)
        nbytes = api.mla_attention_workspace_bytes(c, n_valid)
        g.load_x(inputs.chunk_x(cfg, ch))
        ws_ref = torch.full_like(b.workspace, 0x5A)
        api.mla_project_chunk(c, b.x, w.w_x, w.w_qcat, b.c_q, b.q, b.chunk_lat, first)
        api.mla_attention_fwd(c, b.q, b.chunk_lat, g.ring.cache, g.ring.slot_frame, n_valid,
                              first, w.w_uv, b.o, b.lse, ws_ref, b.dev_status)
        ws = torch.full_like(b.workspace, 0xA5)
        api.mla_project_latents_rotated(c, b.x, w.w_x, cq2, lat2, g.ring.cache, g.ring.slot_frame,
                                        n_valid, first, ws, dev_status=b.dev_status)
        torch.cuda.synchronize()
        assert torch.equal(cq2, b.c_q) and torch.equal(lat2, b.chunk_lat), ch
        assert torch.equal(ws[:nbytes], ws_ref[:nbytes]), ch
        rollout.check_device_status(b)
        g.append(ch)


def test_fused_query_heads_config1_sampled_rows():
    """The bench's step on config 1 (query heads formed in the attention kernel): 384 sampled
    rows against the oracle, and every row against the unfused path."""
    cfg = inputs.CONFIGS[1]
    g, o = prefilled(cfg, api.MLA_PATH_AUTO, cfg.measured_chunk)
    ch = cfg.measured_chunk
    x = inputs.chunk_x(cfg, ch)
    rows = inputs.sample_rows(cfg.n_q, 384, tag=1)
    rf = g.attend(ch, x, fused_q=True)
    check_chunk("cfg1.fused", cfg, rf, o.step(ch, x, rows, append=False), rows)
    ra = g.attend(ch, x)
    for k in ("o", "o_lat", "lse"):
        assert np.abs(ra[k] - rf[k]).max() <= 2.0 ** -8 * max(1.0, np.abs(ra[k]).max()), k


def test_tensor_core_and_cuda_core_paths_agree_on_config1():
    """Diagnostic cross-check on every row of config 1 (GPU against GPU)."""
    cfg = inputs.CONFIGS[1]
    outs = []
    for path in (api.MLA_PATH_AUTO, api.MLA_PATH_SIMT):
        g, _ = prefilled(cfg, path, cfg.measured_chunk)
        outs.append(g.attend(cfg.measured_chunk, inputs.chunk_x(cfg, cfg.measured_chunk)))
    # two correct bf16 results may differ by one or two units in the last place of a value
    for k in ("o", "o_lat", "q", "chunk_lat"):
        a, b = outs[0][k], outs[1][k]
        err = a - b
        assert np.abs(err).max() <= 2 * 2.0 ** -8 * max(1.0, np.abs(b).max()), k
        assert np.linalg.norm(err) / np.linalg.norm(b) <= 5e-3, k


@pytest.mark.parametrize("cfg_id,path", [("small", "tc"), ("small", "simt"), ("1", "tc")])
def test_project_chunk_matches_separate_projections(cfg_id, path):
    """mla_project_chunk (one pass over x, two outputs) gives the results of mla_query_proj and
    mla_cache_append(MLA_PROJECT), and both match the oracle."""
    cfg = inputs.small_bf16_config() if cfg_id == "small" else inputs.CONFIGS[int(cfg_id)]
    g = GpuRun(cfg, PATHS[path])
    ch = cfg.measured_chunk
    x = inputs.chunk_x(cfg, ch)
    g.load_x(x)
    first = cfg.first_frame(ch)
    b = g.buf
    api.mla_project_chunk(g.c, b.x, g.w.w_x, g.w.w_qcat, b.c_q, b.q, b.chunk_lat, first)
    fused = {k: to_np(getattr(b, k)) for k in ("c_q", "q", "chunk_lat")}
    for k in fused:
        getattr(b, k).zero_()
    api.mla_query_proj(g.c, b.x, g.w.w_dq, g.w.w_qcat, b.c_q, b.q, first)
    api.mla_cache_append(g.c, b.x, g.w.w_dkv_kr, b.chunk_lat, g.ring.cache, g.ring.slot_frame,
                         first, api.MLA_PROJECT)
    sep = {k: to_np(getattr(b, k)) for k in ("c_q", "q", "chunk_lat")}
    for k in fused:
        err = np.abs(fused[k] - sep[k])
        # same operands and fp32 accumulation; at most a last-place difference of a rounding
        assert err.max() <= 2.0 ** -7 * max(1.0, np.abs(sep[k]).max()), k
    rows = inputs.sample_rows(cfg.n_q, 96, tag=11)
    d = oracle.dims_from(cfg)
    for bi in range(cfg.batch):
        xb = x[bi][rows]
        c_kv, k_r = oracle.down_project(xb, g.lw.w_dkv, g.lw.w_kr)
        c_q = oracle.query_latent(xb, g.lw.w_dq)
        pos = oracle.token_positions(range(first, first + cfg.chunk_frames), d)[rows]
        q_ref = oracle.absorbed_query(c_q, g.lw.w_uq, g.lw.w_uk, g.lw.w_qr, pos, d)
        compare("fused.chunk_lat", fused["chunk_lat"][bi][rows],
                np.concatenate([c_kv, k_r], axis=1), cfg.dtype)
        compare("fused.c_q", fused["c_q"][bi][rows], c_q, cfg.dtype)
        compare("fused.q", fused["q"][bi][rows], q_ref, cfg.dtype)


@pytest.mark.parametrize("cfg_id", ["small", "3"])
def test_fused_project_and_append_matches_separate_calls(cfg_id):
    """mla_cache_append(MLA_PROJECT_AND_APPEND) on the tensor cores stores every projected row
    to its ring slot from the GEMM's epilogue; the ring, slot_frame and chunk latents are
    bit-identical to MLA_PROJECT followed by MLA_APPEND, over chunks whose frames wrap the ring
    (and, for the small frames, wrap inside a chunk)."""
    cfg = inputs.small_bf16_config() if cfg_id == "small" else inputs.CONFIGS[3]
    a, b = GpuRun(cfg), GpuRun(cfg)
    n = cfg.n_chunks if cfg_id == "small" else cfg.window_frames // cfg.chunk_frames + 2
    for ch in range(n):
        x = inputs.chunk_x(cfg, ch)
        first = cfg.first_frame(ch)
        a.load_x(x)
        b.load_x(x)
        api.mla_cache_append(a.c, a.buf.x, a.w.w_dkv_kr, a.buf.chunk_lat, a.ring.cache,
                             a.ring.slot_frame, first, api.MLA_PROJECT_AND_APPEND)
        api.mla_cache_append(b.c, b.buf.x, b.w.w_dkv_kr, b.buf.chunk_lat, b.ring.cache,
                             b.ring.slot_frame, first, api.MLA_PROJECT)
        api.mla_cache_append(b.c, None, None, b.buf.chunk_lat, b.ring.cache, b.ring.slot_frame,
                             first, api.MLA_APPEND)
        torch.cuda.synchronize()
        assert torch.equal(a.buf.chunk_lat, b.buf.chunk_lat), ch
        assert torch.equal(a.ring.slot_frame, b.ring.slot_frame), ch
        assert torch.equal(a.ring.cache, b.ring.cache), ch


def test_host_streamer_matches_serial_rollout():
    """rollout.HostStreamer (pinned host tokens in, output out, copies overlapped with the
    neighbouring chunks' compute) gives bit-identical outputs to run_chunk one chunk at a time."""
    cfg = inputs.small_bf16_config()
    xs = [torch.from_numpy(inputs.chunk_x(cfg, ch)).to(torch.bfloat16) for ch in range(cfg.n_chunks)]
    a = GpuRun(cfg)
    ref = []
    for ch in range(cfg.n_chunks):
        a.buf.x.copy_(xs[ch])
        ref.append(rollout.run_chunk(a.c, a.w, a.ring, a.buf, ch).cpu().clone())
    b = GpuRun(cfg)
    st = rollout.HostStreamer(b.c, b.w, b.ring)
    outs = [torch.empty_like(r).pin_memory() for r in ref]
    for ch in range(cfg.n_chunks):
        st.submit(ch, xs[ch].pin_memory(), outs[ch])
    st.finish()
    torch.cuda.synchronize()
    st.check_device_status()
    for ch in range(cfg.n_chunks):
        assert torch.equal(outs[ch], ref[ch]), ch
    assert torch.equal(a.ring.cache, b.ring.cache)
    assert torch.equal(a.ring.slot_frame, b.ring.slot_frame)


def test_host_streamer_serves_independent_rollouts_in_turn():
    """One HostStreamer serving two rollouts with their own rings, chunks interleaved (the
    bench's end-to-end form): each rollout's outputs and ring are bit-identical to that rollout
    run alone with run_chunk."""
    cfg = inputs.small_bf16_config()
    xs = [[torch.from_numpy(inputs.chunk_x(cfg, ch, layer=r)).to(torch.bfloat16)
           for ch in range(cfg.n_chunks)] for r in range(2)]
    a = GpuRun(cfg)
    refs, rings = [], []
    for r in range(2):
        ring = rollout.Ring(a.c)
        out = []
        for ch in range(cfg.n_chunks):
            a.buf.x.copy_(xs[r][ch])
            out.append(rollout.run_chunk(a.c, a.w, ring, a.buf, ch).cpu().clone())
        refs.append(out)
        rings.append(ring)
    b = GpuRun(cfg)
    served = [rollout.Ring(b.c) for _ in range(2)]
    st = rollout.HostStreamer(b.c, b.w, b.ring)
    outs = [[torch.empty_like(refs[0][0]).pin_memory() for _ in range(cfg.n_chunks)]
            for _ in range(2)]
    for ch in range(cfg.n_chunks):
        for r in range(2):
            st.submit(ch, xs[r][ch].pin_memory(), outs[r][ch], ring=served[r])
    st.finish()
    torch.cuda.synchronize()
    st.check_device_status()
    for r in range(2):
        for ch in range(cfg.n_chunks):
            assert torch.equal(outs[r][ch], refs[r][ch]), (r, ch)
        assert torch.equal(served[r].cache, rings[r].cache), r
        assert torch.equal(served[r].slot_frame, rings[r].slot_frame), r


def test_chunk_graph_replay_matches_eager_rollout():
    """rollout.ChunkGraph (a chunk's projections, attention and append captured as one CUDA
    graph per chunk index) replays to bit-identical outputs and ring state as the eager calls."""
    cfg = inputs.small_bf16_config()
    xs = [torch.from_numpy(inputs.chunk_x(cfg, ch)).to(torch.bfloat16).cuda()
          for ch in range(cfg.n_chunks)]
    a = GpuRun(cfg)
    ref = []
    for ch in range(cfg.n_chunks):
        a.buf.x.copy_(xs[ch])
        ref.append(rollout.run_chunk(a.c, a.w, a.ring, a.buf, ch).clone())
    b = GpuRun(cfg)
    graphs = [rollout.ChunkGraph(b.c, b.w, b.ring, b.buf, ch, x=xs[ch], events=True)
              for ch in range(cfg.n_chunks)]
    for ch in range(cfg.n_chunks):
        out = graphs[ch].replay().clone()
        torch.cuda.synchronize()
        assert torch.equal(out, ref[ch]), ch
        assert graphs[ch].attention_ms() > 0.0
    assert torch.equal(a.ring.cache, b.ring.cache)
    assert torch.equal(a.ring.slot_frame, b.ring.slot_frame)
    rollout.check_device_status(b.buf)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_cached_ring_attention_is_bit_identical(path):
    """mla_rotate_ring_keys once, then mla_attention_fwd_cached_ring, gives exactly the outputs
    and lse of mla_attention_fwd, on a ring that has wrapped."""
    cfg = inputs.small_bf16_config()
    g = GpuRun(cfg, PATHS[path])
    for ch in range(3):
        g.prefill(ch, inputs.chunk_x(cfg, ch))
    ch = 3
    first, n_valid = rollout.chunk_schedule(cfg.chunk_frames, cfg.window_frames, ch)
    g.load_x(inputs.chunk_x(cfg, ch))
    b = g.buf
    api.mla_project_chunk(g.c, b.x, g.w.w_x, g.w.w_qcat, b.c_q, b.q, b.chunk_lat, first)
    api.mla_attention_fwd(g.c, b.q, b.chunk_lat, g.ring.cache, g.ring.slot_frame, n_valid, first,
                          g.w.w_uv, b.o, b.lse, b.workspace, b.dev_status)
    o_ref, lse_ref = b.o.clone(), b.lse.clone()
    ws = torch.full_like(b.workspace, 0x5A)          # contents on entry must not matter
    api.mla_rotate_ring_keys(g.c, g.ring.cache, g.ring.slot_frame, n_valid, ws)
    for _ in range(2):                               # two steps against the same frozen ring
        b.o.zero_()
        api.mla_attention_fwd_cached_ring(g.c, b.q, b.chunk_lat, g.ring.cache, g.ring.slot_frame,
                                          n_valid, first, g.w.w_uv, b.o, b.lse, ws, b.dev_status)
        torch.cuda.synchronize()
        assert torch.equal(b.o, o_ref)
        assert torch.equal(b.lse, lse_ref)
    rollout.check_device_status(b)


def test_layer_stack_graph_matches_eager():
    """A 3-layer, 2-step stack over 4 chunks (rings wrap): each chunk captured as one CUDA graph
    replays to the eager run's rings and last outputs exactly."""
    cfg = inputs.small_bf16_config()
    c = api.make_config(cfg)
    n_layers, n_steps = 3, 2
    lws = [inputs.layer_weights(cfg, l) for l in range(n_layers)]
    xs = {(ch, s, l): torch.from_numpy(inputs.chunk_x(cfg, ch, s, l)).to(torch.bfloat16).cuda()
          for ch in range(cfg.n_chunks) for s in range(n_steps) for l in range(n_layers)}
    eager = rollout.LayerStack(c, [rollout.upload_weights(c, lw) for lw in lws])
    graphed = rollout.LayerStack(c, [rollout.upload_weights(c, lw) for lw in lws])
    for ch in range(cfg.n_chunks):
        x_of = lambda s, l, ch=ch: xs[(ch, s, l)]
        eager.run_chunk(ch, n_steps, x_of)
        o_eager = eager.buf.o.clone()
        graphed.capture_chunk(ch, n_steps, x_of).replay()
        torch.cuda.synchronize()
        assert torch.equal(graphed.buf.o, o_eager), ch
        for l in range(n_layers):
            assert torch.equal(graphed.rings[l].cache, eager.rings[l].cache), (ch, l)
            assert torch.equal(graphed.rings[l].slot_frame, eager.rings[l].slot_frame), (ch, l)
    rollout.check_device_status(graphed.buf)


def test_layer_stack_fused_query_matches_q_gemm():
    """The layer stack's default form (the chunk's rotated keys from the x-projection,
    mla_project_latents_rotated with rotate_ring=0 beside the ring keys rotated once per chunk,
    then the attention forming the query heads itself) against mla_project_chunk +
    mla_attention_fwd_cached_ring: identical rings and outputs to a bf16 ulp over 4 chunks (rings
    wrap)."""
    cfg = inputs.small_bf16_config()
    c = api.make_config(cfg)
    n_layers, n_steps = 2, 2
    lws = [inputs.layer_weights(cfg, l) for l in range(n_layers)]
    xs = {(ch, s, l): torch.from_numpy(inputs.chunk_x(cfg, ch, s, l)).to(torch.bfloat16).cuda()
          for ch in range(cfg.n_chunks) for s in range(n_steps) for l in range(n_layers)}
    fused = rollout.LayerStack(c, [rollout.upload_weights(c, lw) for lw in lws], fused_q=True)
    plain = rollout.LayerStack(c, [rollout.upload_weights(c, lw) for lw in lws], fused_q=False)
    for ch in range(cfg.n_chunks):
        x_of = lambda s, l, ch=ch: xs[(ch, s, l)]
        fused.run_chunk(ch, n_steps, x_of)
        plain.run_chunk(ch, n_steps, x_of)
        torch.cuda.synchronize()
        a, b = fused.buf.o.float(), plain.buf.o.float()
        assert (a - b).abs().max().item() <= 2.0 ** -8 * max(1.0, b.abs().max().item()), ch
        for l in range(n_layers):
            assert torch.equal(fused.rings[l].cache, plain.rings[l].cache), (ch, l)
    rollout.check_device_status(fused.buf)


def test_standalone_rope3d_and_out_proj():
    cfg = inputs.small_bf16_config()
    g = GpuRun(cfg, api.MLA_PATH_AUTO)
    o = OracleRun(cfg, g.lw)
    d = oracle.dims_from(cfg)
    x = inputs.chunk_x(cfg, 0)
    g.prefill(0, x)
    o.prefill(0, x)
    # rotate the ring's positional keys in place (frames from slot_frame) and compare
    rot = g.ring.cache.clone()
    api.mla_rope3d(g.c, rot, n_vec=1, col_offset=cfg.d_c, vec_stride=0,
                   frame_table=g.ring.slot_frame)
    tpf = cfg.tokens_per_frame
    sf = g.ring.slot_frame.cpu().numpy()
    got = to_np(rot)
    for b in range(cfg.batch):
        for s, t in enumerate(sf[b]):
            if t < 0:
                np.testing.assert_array_equal(got[b, s * tpf:(s + 1) * tpf],
                                              to_np(g.ring.cache)[b, s * tpf:(s + 1) * tpf])
                continue
            rec = [r for r in o.windows[b].frames if r.t == t][0]
            ref = oracle.rope3d(rec.k_r, oracle.token_positions([t], d), d)
            compare("rope3d", got[b, s * tpf:(s + 1) * tpf, cfg.d_c:], ref, "bf16")
    # out_proj of a latent output and the optional W_O
    x1 = inputs.chunk_x(cfg, 1)
    res = g.attend(1, x1)
    ores = o.step(1, x1, np.arange(cfg.n_q))
    y = torch.empty((cfg.batch, cfg.n_q, cfg.d_model), device="cuda", dtype=torch.bfloat16)
    api.mla_out_proj(g.c, g.buf.o_lat, g.w.w_uv, g.buf.o, w_o=g.w.w_o, y=y)
    torch.cuda.synchronize()
    for b in range(cfg.batch):
        compare("out_proj.o", to_np(g.buf.o)[b], ores[b]["o"], "bf16")
        compare("out_proj.y", to_np(y)[b], oracle.output_projection(ores[b]["o"], g.lw.w_o), "bf16")


def test_ring_checkpoint_resume_is_bit_identical():
    cfg = inputs.small_bf16_config()
    a = GpuRun(cfg)
    outs_a = []
    for ch in range(cfg.n_chunks):
        outs_a.append(a.attend(ch, inputs.chunk_x(cfg, ch), want_latent=False)["o"])
        a.append(ch)
        if ch == 1:
            saved = a.ring.state_dict()
    b = GpuRun(cfg)
    b.ring.load_state_dict(saved)
    for ch in range(2, cfg.n_chunks):
        ob = b.attend(ch, inputs.chunk_x(cfg, ch), want_latent=False)["o"]
        np.testing.assert_array_equal(ob, outs_a[ch])
        b.append(ch)


def test_bad_arguments_on_device():
    cfg = inputs.small_bf16_config()
    g = GpuRun(cfg)
    x = inputs.chunk_x(cfg, 0)
    g.load_x(x)
    host = torch.empty_like(g.buf.chunk_lat, device="cpu")
    with pytest.raises(api.MLAError) as e:
        api.mla_cache_append(g.c, g.buf.x, g.w.w_dkv_kr, host, g.ring.cache, g.ring.slot_frame, 0,
                             api.MLA_PROJECT)
    assert e.value.status == 1
    small_ws = torch.empty((64,), device="cuda", dtype=torch.uint8)
    with pytest.raises(api.MLAError) as e:
        api.mla_attention_fwd(g.c, g.buf.q, g.buf.chunk_lat, g.ring.cache, g.ring.slot_frame, 0, 0,
                              None, g.buf.o_lat, workspace=small_ws)
    assert e.value.status == 6
    from mla_latent_kv_attn_b200 import _lib
    import ctypes
    st = _lib.lib().mla_rope3d(ctypes.byref(g.c), g.buf.chunk_lat.data_ptr() + 2, 1, cfg.n_q,
                               224, 192, 1, 0, None, 0, 0, None)
    assert st == 3
    torch.cuda.synchronize()
    assert int(g.buf.dev_status.item()) == 0


def test_wan_config4_thirty_layer_stack():
    """Config 4: 30 layers, each with its own weights and ring, batch 2, window 12 frames; every
    chunk runs 4 denoising steps through all 30 layers against the frozen rings, then each layer
    appends its last step's latents.  All 1200 attention calls run on the GPU through
    rollout.LayerStack (ring keys rotated once per chunk and layer, cached-ring attention).  The oracle checks
    sampled rows of layer 29 at the last chunk (steps 0 and 3, ring wrapped, 23,400 keys) and of
    layer 0 at chunks 0 and 1 (256 sampled rows, both samples), plus both layers' ring slots."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    from parity_util import expected_slot_frame

    cfg = inputs.CONFIGS[4]
    c = api.make_config(cfg)
    layers = [inputs.layer_weights(cfg, l) for l in range(cfg.n_layers)]
    stack = rollout.LayerStack(c, [rollout.upload_weights(c, lw) for lw in layers])
    buf = stack.buf
    rings = stack.rings
    last = cfg.n_steps - 1
    checks = {(cfg.n_chunks - 1, 0, 29), (cfg.n_chunks - 1, last, 29), (0, 0, 0), (0, last, 0),
              (1, last, 0)}
    history = {29: range(cfg.n_chunks), 0: range(2)}
    rows = inputs.sample_rows(cfg.n_q, 256, tag=4)
    order = [(ch, s, l) for ch in range(cfg.n_chunks) for s in range(cfg.n_steps)
             for l in range(cfg.n_layers)]
    kept, gpu_out = {}, {}
    workers = min(16, os.cpu_count() or 4)
    pool = ThreadPoolExecutor(max_workers=workers)
    futs = {}
    for i, key in enumerate(order):
        for k in order[i:i + workers + 4]:
            if k not in futs:
                futs[k] = pool.submit(inputs.chunk_x, cfg, k[0], k[1], k[2])
        ch, s, l = key
        x = futs.pop(key).result()
        if key in checks or (l in history and s == last and ch in history[l]):
            kept[key] = x
        if s == 0 and l == 0:
            stack.begin_chunk(ch)       # each layer's ring keys rotated once per chunk
        buf.x.copy_(torch.from_numpy(x).to(torch.bfloat16))
        stack.attend(ch, l, buf.x, append=(s == last))
        if key in checks:
            gpu_out[key] = (to_np(buf.o)[:, rows], to_np(buf.lse)[:, :, rows])
    pool.shutdown()
    torch.cuda.synchronize()
    rollout.check_device_status(buf)

    for l, chunks in history.items():
        o = OracleRun(cfg, layers[l])
        for ch in chunks:
            for s in (0, last):
                if (ch, s, l) in checks:
                    res = o.step(ch, kept[(ch, s, l)], rows, append=False)
                    g_o, g_lse = gpu_out[(ch, s, l)]
                    for b in range(cfg.batch):
                        compare(f"cfg4.l{l}.c{ch}.s{s}.b{b}.o", g_o[b], res[b]["o"], "bf16")
                        compare(f"cfg4.l{l}.c{ch}.s{s}.b{b}.lse", g_lse[b], res[b]["lse"], "bf16")
            o.prefill(ch, kept[(ch, last, l)])
        if l == 29:
            gpu_sf = rings[l].slot_frame.cpu().numpy()
            for b in range(cfg.batch):
                np.testing.assert_array_equal(gpu_sf[b], expected_slot_frame(cfg, o.windows[b]))


def test_device_wait_timeout_is_reported_and_context_survives():
    """A bounded wait that runs out inside a kernel reports MLA_ERR_DEVICE_TIMEOUT through the
    status word; nothing traps and the context keeps working afterwards."""
    from mla_latent_kv_attn_b200 import _lib
    status = torch.zeros(1, device="cuda", dtype=torch.int32)
    st = _lib.lib().mla_selftest_wait_timeout(status.data_ptr(), 2000,
                                              torch.cuda.current_stream().cuda_stream)
    assert st == 0, _lib.last_error()
    torch.cuda.synchronize()
    assert int(status.item()) == _lib.MLA_ERR_DEVICE_TIMEOUT
    # the device is still usable: a small rollout chunk runs and matches the oracle
    cfg = inputs.CONFIGS[0]
    g = GpuRun(cfg)
    o = OracleRun(cfg, g.lw)
    x = inputs.chunk_x(cfg, 0)
    check_chunk("after_timeout", cfg, g.attend(0, x), o.step(0, x, np.arange(cfg.n_q)),
                np.arange(cfg.n_q))
