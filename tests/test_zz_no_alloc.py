"""The allocation-free attention entry point agrees with the regular one.

Some callers cannot call cudaMalloc: plugins whose host framework hands them only their own
input and output buffers, and services that forbid device allocation once they are running.
For them the library offers
mla_attention_fwd_static_scratch, which keeps the attention scratch (the rotated positional
keys) in a 16 MiB array built into the library instead of a caller-provided workspace.

This file checks that call through the C ABI against mla_attention_fwd on two calls in a row
with different work (so the second call cannot pass on what the first left in the shared
array), with the tolerances of the other parity tests, and that a call needing more than the
built-in 16 MiB is refused on the host.  It is collected last and needs nothing from the other
test files.
"""
import numpy as np
import pytest
import torch

from mla_latent_kv_attn_b200 import _lib, api, inputs, rollout

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


def close(name, got, ref):
    got = got.float().cpu().numpy().astype(np.float64)
    ref = ref.float().cpu().numpy().astype(np.float64)
    err = got - ref
    assert np.isfinite(got).all(), name
    assert np.abs(err).max() <= MAX_ABS, f"{name}: max-abs {np.abs(err).max():.3e}"
    assert np.linalg.norm(err) <= REL_L2 * np.linalg.norm(ref), f"{name}: rel-L2"


def prepared(cfg, chunk):
    """Weights, ring and per-chunk buffers with the ring filled up to `chunk` and the chunk's
    query and latents computed."""
    c = api.make_config(cfg)
    w = rollout.upload_weights(c, inputs.layer_weights(cfg))
    ring = rollout.Ring(c)
    buf = rollout.ChunkBuffers(c)
    for ch in range(chunk):
        buf.x.copy_(torch.from_numpy(inputs.chunk_x(cfg, ch)).to(torch.bfloat16))
        rollout.prefill_chunk(c, w, ring, buf, ch)
    buf.x.copy_(torch.from_numpy(inputs.chunk_x(cfg, chunk)).to(torch.bfloat16))
    first, n_valid = rollout.chunk_schedule(cfg.chunk_frames, cfg.window_frames, chunk)
    api.mla_query_proj(c, buf.x, w.w_dq, w.w_qcat, buf.c_q, buf.q, first)
    api.mla_cache_append(c, buf.x, w.w_dkv_kr, buf.chunk_lat, ring.cache, ring.slot_frame, first,
                         api.MLA_PROJECT)
    return c, w, ring, buf, first, n_valid


def run_both(cfg, chunk, fuse_uv):
    c, w, ring, buf, first, n_valid = prepared(cfg, chunk)
    w_uv = w.w_uv if fuse_uv else None
    ref = buf.o if fuse_uv else buf.o_lat
    api.mla_attention_fwd(c, buf.q, buf.chunk_lat, ring.cache, ring.slot_frame, n_valid, first,
                          w_uv, ref, buf.lse, buf.workspace, buf.dev_status)
    lse_ref = buf.lse.clone()
    out = torch.full_like(ref, float("nan"))
    lse = torch.full_like(buf.lse, float("nan"))
    api.mla_attention_fwd_static_scratch(c, buf.q, buf.chunk_lat, ring.cache, ring.slot_frame,
                                         n_valid, first, w_uv, out, lse, buf.dev_status)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    return out, ref, lse, lse_ref


def test_static_scratch_matches_workspace_call_twice_in_a_row():
    # first call: the Wan-shaped layer at full size, window full, W_UV fused
    out1, ref1, lse1, lse_ref1 = run_both(inputs.CONFIGS[1], inputs.CONFIGS[1].measured_chunk,
                                          fuse_uv=True)
    # second call right after it: other frame geometry, two samples, a partly filled ring and
    # the latent output, so its scratch layout differs from the first call's
    small = inputs.small_bf16_config()
    out2, ref2, lse2, lse_ref2 = run_both(small, 1, fuse_uv=False)
    close("call1.out", out1, ref1)
    close("call1.lse", lse1, lse_ref1)
    close("call2.out", out2, ref2)
    close("call2.lse", lse2, lse_ref2)


def test_static_scratch_refuses_work_beyond_its_size():
    cfg = inputs.CONFIGS[3]
    c = api.make_config(cfg, batch=16)            # needs about 19 MB of scratch
    assert api.mla_attention_workspace_bytes(c, cfg.window_frames) > 16 * 1024 * 1024
    tpf, n_q, D = cfg.tokens_per_frame, cfg.n_q, cfg.d_latent
    B, H = 16, cfg.n_heads
    q = torch.zeros((B, n_q, H, D), device="cuda", dtype=torch.bfloat16)
    lat = torch.zeros((B, n_q, D), device="cuda", dtype=torch.bfloat16)
    cache = torch.zeros((B, cfg.window_frames * tpf, D), device="cuda", dtype=torch.bfloat16)
    sf = torch.zeros((B, cfg.window_frames), device="cuda", dtype=torch.int32)
    out = torch.zeros((B, n_q, H, cfg.d_c), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(api.MLAError) as e:
        api.mla_attention_fwd_static_scratch(c, q, lat, cache, sf, cfg.window_frames, 27, None, out)
    assert e.value.status == _lib.MLA_ERR_WORKSPACE
    assert "16777216" in str(e.value)
