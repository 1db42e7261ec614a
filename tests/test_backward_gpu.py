"""GPU parity of the attention backward (mla_attention_bwd) against the float64 oracle's
latent_attention_backward, on identical seeded inputs: queries, chunk latents and ring contents
drawn directly (the ring filled through mla_cache_append so that it wraps), and a seeded upstream
gradient.  The GPU takes o_lat and lse from its own forward on those inputs; the oracle
recomputes everything it needs in float64."""
import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_attn_b200 import api, inputs, rollout
from parity_util import compare, to_np

pytestmark = pytest.mark.gpu


def _run(cfg, chunk, path=api.MLA_PATH_AUTO, grad_std=1.0):
    c = api.make_config(cfg, kernel_path=path)
    dt = api.torch_dtype(c)
    dev = torch.device("cuda")
    ring = rollout.Ring(c)
    d = oracle.dims_from(cfg)
    windows = [oracle.SlidingWindow(d) for _ in range(cfg.batch)]
    lat_buf = torch.empty((cfg.batch, cfg.n_q, cfg.d_latent), device=dev, dtype=dt)
    for ch in range(chunk):                      # earlier chunks enter the ring (it wraps)
        lat = inputs.direct_latents(cfg, ch)
        lat_buf.copy_(torch.from_numpy(lat).to(dt))
        api.mla_cache_append(c, None, None, lat_buf, ring.cache, ring.slot_frame,
                             cfg.first_frame(ch), api.MLA_APPEND)
        for b in range(cfg.batch):
            windows[b].append_chunk(cfg.first_frame(ch), lat[b][:, :cfg.d_c], lat[b][:, cfg.d_c:])
    first, n_valid = rollout.chunk_schedule(cfg.chunk_frames, cfg.window_frames, chunk)
    q_np = inputs.direct_queries(cfg, chunk)
    lat_np = inputs.direct_latents(cfg, chunk)
    g_np = inputs.upstream_gradient(cfg, chunk, cfg.d_c, std=grad_std)
    q = torch.from_numpy(q_np).to(device=dev, dtype=dt)
    lat_buf.copy_(torch.from_numpy(lat_np).to(dt))
    g = torch.from_numpy(g_np).to(device=dev, dtype=dt)
    o_lat = torch.empty((cfg.batch, cfg.n_q, cfg.n_heads, cfg.d_c), device=dev, dtype=dt)
    lse = torch.empty((cfg.batch, cfg.n_heads, cfg.n_q), device=dev, dtype=torch.float32)
    ws = torch.empty(max(api.mla_attention_workspace_bytes(c, n_valid), 256), device=dev,
                     dtype=torch.uint8)
    api.mla_attention_fwd(c, q, lat_buf, ring.cache, ring.slot_frame, n_valid, first, None, o_lat,
                          lse, ws)
    d_q = torch.full_like(q, float("nan"))
    d_lat = torch.full_like(lat_buf, float("nan"))
    sentinel = 7.0
    d_cache = torch.full_like(ring.cache, sentinel)
    bws = torch.empty(api.mla_attention_bwd_workspace_bytes(c, n_valid), device=dev,
                      dtype=torch.uint8)
    api.mla_attention_bwd(c, q, lat_buf, ring.cache, ring.slot_frame, n_valid, first, o_lat, lse, g,
                          d_q, d_lat, d_cache, bws)
    torch.cuda.synchronize()
    got = dict(d_q=to_np(d_q), d_lat=to_np(d_lat), d_cache=to_np(d_cache),
               slot_frame=ring.slot_frame.cpu().numpy())
    tpf = cfg.tokens_per_frame
    nc = n_valid * tpf
    for b in range(cfg.batch):
        recs = {r.t: r for r in windows[b].frames}
        slots = got["slot_frame"][b][:n_valid]
        c_ring = np.concatenate([recs[t].c_kv for t in slots]) if n_valid else np.zeros((0, cfg.d_c))
        k_ring = np.concatenate([recs[t].k_r for t in slots]) if n_valid else np.zeros((0, cfg.d_rope))
        pos_ring = oracle.token_positions(list(slots), d)
        pos_chunk = oracle.token_positions(range(first, first + cfg.chunk_frames), d)
        ref = oracle.latent_attention_backward(
            q_np[b], np.concatenate([c_ring, lat_np[b][:, :cfg.d_c]]),
            np.concatenate([k_ring, lat_np[b][:, cfg.d_c:]]), np.concatenate([pos_ring, pos_chunk]),
            g_np[b], d)
        dk = np.concatenate([ref["d_c"], ref["d_k_r"]], axis=1)
        tag = f"{cfg.name}[b{b}]"
        compare(tag + ".d_q", got["d_q"][b], ref["d_q"], cfg.dtype)
        compare(tag + ".d_chunk_lat", got["d_lat"][b], dk[nc:], cfg.dtype)
        if nc:
            compare(tag + ".d_cache", got["d_cache"][b][:nc], dk[:nc], cfg.dtype)
        assert (got["d_cache"][b][nc:] == sentinel).all(), "rows beyond the attended slots changed"
    return got


def test_backward_toy_fp32_wrapped_ring():
    cfg = inputs.CONFIGS[0]
    _run(cfg, chunk=3)          # window of 2 frames after 3 one-frame chunks: wrapped


@pytest.mark.parametrize("path", ["tc", "simt"])
@pytest.mark.parametrize("chunk", [0, 3])
def test_backward_small_frames_bf16(chunk, path):
    """Wan widths on 6x10 frames, 12 heads: chunk 0 (no ring) and chunk 3 (ring wrapped), on
    the tensor-core kernels and on the CUDA-core kernels."""
    _run(inputs.small_bf16_config(), chunk=chunk,
         path=api.MLA_PATH_AUTO if path == "tc" else api.MLA_PATH_SIMT)


def test_backward_wan_config1_full_size():
    """The Wan preset at full size on the tensor-core backward (4680 queries, 14,040 keys, 12
    heads, the launch grid and head-group split of the benchmark workload), one chunk after the
    window filled so that the ring has wrapped (slots 3..5 hold the oldest frames, 0..2 the
    newest).  Every gradient is compared element by element with the float64 oracle, which
    evaluates all rows and keys: d_q of every query row, and the latent gradient of every
    attended key (ring keys from the oldest and newest slots, the ragged last ring tile, every
    chunk key).  Besides, two identities that hold at any size, since every row's
    probabilities sum to one (so every row's dS sums to zero): summed over all keys, the content
    gradients equal the summed upstream gradient and the positional ones, rotated back to the
    keys' frames, sum to zero."""
    cfg = inputs.CONFIGS[1]
    c = api.make_config(cfg)
    dt = api.torch_dtype(c)
    dev = torch.device("cuda")
    ring = rollout.Ring(c)
    d = oracle.dims_from(cfg)
    chunk = cfg.measured_chunk + 1
    tpf = cfg.tokens_per_frame
    lat_buf = torch.empty((1, cfg.n_q, cfg.d_latent), device=dev, dtype=dt)
    recs = {}
    for ch in range(chunk):
        lat = inputs.direct_latents(cfg, ch)
        lat_buf.copy_(torch.from_numpy(lat).to(dt))
        api.mla_cache_append(c, None, None, lat_buf, ring.cache, ring.slot_frame,
                             cfg.first_frame(ch), api.MLA_APPEND)
        for f in range(cfg.chunk_frames):
            recs[cfg.first_frame(ch) + f] = lat[0][f * tpf:(f + 1) * tpf]
    first, n_valid = rollout.chunk_schedule(cfg.chunk_frames, cfg.window_frames, chunk)
    q_np = inputs.direct_queries(cfg, chunk)
    lat_np = inputs.direct_latents(cfg, chunk)
    g_np = inputs.upstream_gradient(cfg, chunk, cfg.d_c)
    q = torch.from_numpy(q_np).to(device=dev, dtype=dt)
    lat_buf.copy_(torch.from_numpy(lat_np).to(dt))
    g = torch.from_numpy(g_np).to(device=dev, dtype=dt)
    o_lat = torch.empty((1, cfg.n_q, cfg.n_heads, cfg.d_c), device=dev, dtype=dt)
    lse = torch.empty((1, cfg.n_heads, cfg.n_q), device=dev, dtype=torch.float32)
    ws = torch.empty(api.mla_attention_workspace_bytes(c, n_valid), device=dev, dtype=torch.uint8)
    api.mla_attention_fwd(c, q, lat_buf, ring.cache, ring.slot_frame, n_valid, first, None, o_lat,
                          lse, ws)
    d_q = torch.full_like(q, float("nan"))
    d_lat = torch.full_like(lat_buf, float("nan"))
    d_cache = torch.full_like(ring.cache, float("nan"))
    status = torch.zeros(1, device=dev, dtype=torch.int32)
    bws = torch.empty(api.mla_attention_bwd_workspace_bytes(c, n_valid), device=dev,
                      dtype=torch.uint8)
    api.mla_attention_bwd(c, q, lat_buf, ring.cache, ring.slot_frame, n_valid, first, o_lat, lse, g,
                          d_q, d_lat, d_cache, bws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    slots = ring.slot_frame.cpu().numpy()[0][:n_valid]
    assert list(slots) == [first - cfg.window_frames + (s - first) % cfg.window_frames
                           for s in range(cfg.window_frames)], "ring has not wrapped"
    c_ring = np.concatenate([recs[t][:, :cfg.d_c] for t in slots])
    k_ring = np.concatenate([recs[t][:, cfg.d_c:] for t in slots])
    pos_k = np.concatenate([oracle.token_positions(list(slots), d),
                            oracle.token_positions(range(first, first + cfg.chunk_frames), d)])
    ref = oracle.latent_attention_backward(
        q_np[0], np.concatenate([c_ring, lat_np[0][:, :cfg.d_c]]),
        np.concatenate([k_ring, lat_np[0][:, cfg.d_c:]]), pos_k, g_np[0], d)
    nc = n_valid * tpf
    dk = np.concatenate([ref["d_c"], ref["d_k_r"]], axis=1)              # [keys, D]
    got_dq, got_cache, got_lat = to_np(d_q)[0], to_np(d_cache)[0], to_np(d_lat)[0]
    compare("cfg1.d_q", got_dq, ref["d_q"], "bf16")
    compare("cfg1.d_cache", got_cache[:nc], dk[:nc], "bf16")
    compare("cfg1.d_chunk_lat", got_lat, dk[nc:], "bf16")
    # the oldest and newest ring frames and the chunk's last (ragged) key tile on their own
    oldest, newest = int(np.argmin(slots)), int(np.argmax(slots))
    for name, lo, hi in (("oldest", oldest * tpf, (oldest + 1) * tpf),
                         ("newest", newest * tpf, (newest + 1) * tpf),
                         ("ring tail tile", nc - nc % 128, nc)):
        compare(f"cfg1.d_cache[{name}]", got_cache[lo:hi], dk[lo:hi], "bf16")
    compare("cfg1.d_chunk_lat[tail tile]", got_lat[cfg.n_q - cfg.n_q % 128:],
            dk[nc + cfg.n_q - cfg.n_q % 128:], "bf16")
    grads = np.concatenate([got_cache[:nc], got_lat])
    content_sum = grads[:, :cfg.d_c].sum(axis=0)
    expect = g_np[0].astype(np.float64).sum(axis=(0, 1))
    assert np.linalg.norm(content_sum - expect) <= 2e-2 * np.linalg.norm(expect)
    rope_back = oracle.rope3d(grads[:, cfg.d_c:], pos_k, d).sum(axis=0)
    scale_ref = np.abs(grads[:, cfg.d_c:]).sum(axis=0)
    assert (np.abs(rope_back) <= 2e-2 * scale_ref + 1e-3).all()
