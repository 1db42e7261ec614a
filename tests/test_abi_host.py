"""The C-ABI library on a machine without a GPU: it loads, exports every entry point that
include/mla.h declares, and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

from mla_latent_kv_attn_b200 import _lib, api, inputs
from mla_latent_kv_attn_b200.rollout import chunk_schedule

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = _lib.lib()
    names = declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_abi_version_matches_header():
    m = re.search(r"#define MLA_ABI_VERSION (\d+)", open(HEADER).read())
    assert _lib.lib().mla_abi_version() == int(m.group(1))


def test_struct_layout_matches_header():
    text = open(HEADER).read()
    body = text[text.index("typedef struct mla_config {"):text.index("} mla_config;")]
    fields = re.findall(r"\b(int32_t|float)\s+(\w+);", body)
    assert [f for _, f in fields] == [f for f, _ in _lib.MLAConfigC._fields_]
    assert ctypes.sizeof(_lib.MLAConfigC) == 4 * len(fields)


def test_status_strings():
    assert _lib.status_string(0) == "MLA_OK"
    assert _lib.status_string(6) == "MLA_ERR_WORKSPACE"
    assert _lib.status_string(99) == "MLA_ERR_UNKNOWN"


@pytest.mark.parametrize("i", sorted(inputs.CONFIGS))
def test_presets_are_valid_configs(i):
    api.mla_config_check(api.make_config(inputs.CONFIGS[i]))


@pytest.mark.parametrize("field,value", [
    ("d_rope", 30), ("chunk_frames", 7), ("dtype", 5), ("batch", 0), ("rope_base", 1.0),
    ("softmax_scale", -1.0), ("kernel_path", 4), ("frame_w", 0),
])
def test_bad_configs_are_rejected(field, value):
    c = api.make_config(inputs.CONFIGS[1])
    setattr(c, field, value)
    with pytest.raises(api.MLAError) as e:
        api.mla_config_check(c)
    assert e.value.status == _lib.MLA_ERR_INVALID_ARG
    assert _lib.last_error()


def test_oversized_workload_is_rejected():
    c = api.make_config(inputs.CONFIGS[1])
    c.batch = 4096
    with pytest.raises(api.MLAError):
        api.mla_config_check(c)


def test_largest_accepted_batch_is_the_int32_element_limit():
    # Wan preset: the largest array per sample is Q' = n_q * H * (d_c + d_rope) = 12,579,840
    # elements; every array must hold fewer than 2^31 - 1 elements
    cfg = inputs.CONFIGS[1]
    per_sample = cfg.n_q * cfg.n_heads * (cfg.d_c + cfg.d_rope)
    assert per_sample == 12_579_840
    top = (2**31 - 2) // per_sample
    assert top == 170
    c = api.make_config(cfg, batch=top)
    api.mla_config_check(c)
    c = api.make_config(cfg, batch=top + 1)
    with pytest.raises(api.MLAError) as e:
        api.mla_config_check(c)
    assert e.value.status == _lib.MLA_ERR_INVALID_ARG and "2^31" in _lib.last_error()


def test_null_pointers_rejected_without_a_device():
    c = api.make_config(inputs.CONFIGS[1])
    lib = _lib.lib()
    st = lib.mla_cache_append(ctypes.byref(c), None, None, None, None, None, 0, 1, None)
    assert st == _lib.MLA_ERR_INVALID_ARG and "null" in _lib.last_error()
    st = lib.mla_cache_append(ctypes.byref(c), None, None, None, None, None, 0, 9, None)
    assert st == _lib.MLA_ERR_INVALID_ARG and "mode" in _lib.last_error()
    st = lib.mla_attention_fwd(ctypes.byref(c), None, None, None, None, 7, 0, None, None, None,
                               None, 0, None, None)
    assert st == _lib.MLA_ERR_INVALID_ARG and "n_valid_frames" in _lib.last_error()
    st = lib.mla_query_proj(ctypes.byref(c), None, None, None, None, None, -1, None)
    assert st == _lib.MLA_ERR_INVALID_ARG
    st = lib.mla_key_positions(ctypes.byref(c), None, 2, 0, None, None)
    assert st == _lib.MLA_ERR_INVALID_ARG


def test_projection_with_rotated_keys_checks_without_a_device():
    """mla_project_latents_rotated and mla_attention_fwd_from_cq_prerotated refuse bad
    arguments on the host before any device call."""
    c = api.make_config(inputs.CONFIGS[1])
    lib = _lib.lib()
    st = lib.mla_project_latents_rotated(ctypes.byref(c), None, None, None, None, None, None, 7,
                                         0, 1, None, 0, None, None)
    assert st == _lib.MLA_ERR_INVALID_ARG and "n_valid_frames" in _lib.last_error()
    st = lib.mla_project_latents_rotated(ctypes.byref(c), None, None, None, None, None, None, 6,
                                         0, 2, None, 0, None, None)
    assert st == _lib.MLA_ERR_INVALID_ARG and "rotate_ring" in _lib.last_error()
    st = lib.mla_project_latents_rotated(ctypes.byref(c), None, None, None, None, None, None, 6,
                                         -1, 1, None, 0, None, None)
    assert st == _lib.MLA_ERR_INVALID_ARG and "first_frame" in _lib.last_error()
    st = lib.mla_project_latents_rotated(ctypes.byref(c), None, None, None, None, None, None, 6,
                                         6, 1, None, 0, None, None)
    assert st == _lib.MLA_ERR_INVALID_ARG and "x is null" in _lib.last_error()
    st = lib.mla_attention_fwd_from_cq_prerotated(ctypes.byref(c), None, None, None, None, None,
                                                  7, 0, None, None, None, None, 0, None, None)
    assert st == _lib.MLA_ERR_INVALID_ARG and "n_valid_frames" in _lib.last_error()
    fp32 = api.make_config(inputs.CONFIGS[0])
    st = lib.mla_attention_fwd_from_cq_prerotated(ctypes.byref(fp32), None, None, None, None,
                                                  None, 0, 0, None, None, None, None, 0, None,
                                                  None)
    assert st == _lib.MLA_ERR_UNSUPPORTED


def test_frame_index_overflow_rejected_without_a_device():
    c = api.make_config(inputs.CONFIGS[1])              # chunk_frames 3
    lib = _lib.lib()
    top = 2**31 - 1
    for ff in (top, top - 2, -1):
        st = lib.mla_cache_append(ctypes.byref(c), None, None, None, None, None, ff, 3, None)
        assert st == _lib.MLA_ERR_INVALID_ARG and "first_frame" in _lib.last_error()
        st = lib.mla_attention_fwd(ctypes.byref(c), None, None, None, None, 0, ff, None, None,
                                   None, None, 0, None, None)
        assert st == _lib.MLA_ERR_INVALID_ARG and "first_frame" in _lib.last_error()
        st = lib.mla_query_proj(ctypes.byref(c), None, None, None, None, None, ff, None)
        assert st == _lib.MLA_ERR_INVALID_ARG and "first_frame" in _lib.last_error()
        st = lib.mla_key_positions(ctypes.byref(c), None, 0, ff, None, None)
        assert st == _lib.MLA_ERR_INVALID_ARG and "first_frame" in _lib.last_error()
    # the largest chunk start whose last frame still fits passes the frame check and then
    # fails on the first null pointer
    st = lib.mla_cache_append(ctypes.byref(c), None, None, None, None, None, top - 3, 3, None)
    assert st == _lib.MLA_ERR_INVALID_ARG and "chunk_lat is null" in _lib.last_error()


def test_workspace_size():
    for i in (0, 1, 2, 3):
        cfg = inputs.CONFIGS[i]
        c = api.make_config(cfg)
        tpf = cfg.tokens_per_frame
        for n_valid in (0, 1, cfg.window_frames):
            nc = n_valid * tpf
            rows = -(-nc // 128) * 128 + -(-cfg.n_q // 128) * 128
            es = 4 if cfg.dtype == "fp32" else 2
            assert api.mla_attention_workspace_bytes(c, n_valid) == cfg.batch * rows * cfg.d_rope * es
        assert api.mla_attention_workspace_bytes(c, cfg.window_frames + 1) == 0


def _bwd_head_groups(cfg, n_valid):
    """The key-gradient kernel's head-group count: the divisor g of H whose (key tile, group,
    sample) CTAs fill whole waves of 148 SMs best, the fewest on ties."""
    nc = n_valid * cfg.tokens_per_frame
    tiles = (-(-nc // 128) + -(-cfg.n_q // 128)) * cfg.batch
    best, best_eff = 1, -1.0
    for g in range(1, cfg.n_heads + 1):
        if cfg.n_heads % g:
            continue
        ctas = tiles * g
        eff = ctas / (-(-ctas // 148) * 148)
        if eff > best_eff + 1e-9:
            best, best_eff = g, eff
    return best


def test_backward_workspace_size():
    """Delta, the rotated keys, and (tensor-core path: bf16, d_c 192, d_rope 32, n_q % 4 == 0)
    the 256-wide padded key copy plus the head groups' fp32 partial key gradients."""
    cases = [(inputs.CONFIGS[0], api.MLA_PATH_AUTO, False),      # fp32: CUDA cores
             (inputs.CONFIGS[1], api.MLA_PATH_AUTO, True),       # the Wan preset: tensor cores
             (inputs.CONFIGS[1], api.MLA_PATH_SIMT, False),      # forced onto CUDA cores
             (inputs.small_bf16_config(), api.MLA_PATH_AUTO, True)]
    for cfg, path, tc in cases:
        c = api.make_config(cfg, kernel_path=path)
        es = 4 if cfg.dtype == "fp32" else 2
        for n_valid in (0, 1, cfg.window_frames):
            nc = n_valid * cfg.tokens_per_frame
            rows = -(-nc // 128) * 128 + -(-cfg.n_q // 128) * 128
            delta = -(-(cfg.batch * cfg.n_heads * cfg.n_q) // 64) * 64 * 4
            keys = cfg.batch * rows * cfg.d_rope * es
            expect = delta + keys
            if tc:
                groups = _bwd_head_groups(cfg, n_valid)
                expect += cfg.batch * rows * 256 * 2
                expect += groups * cfg.batch * rows * cfg.d_latent * 4
            assert api.mla_attention_bwd_workspace_bytes(c, n_valid) == expect, (cfg.name, path, n_valid)


def test_schedule_matches_oracle_window():
    """The driver's (first_frame, n_valid) per chunk equals the oracle's window contents."""
    import numpy as np
    import oracle
    for i in (0, 1, 2, 3):
        cfg = inputs.CONFIGS[i]
        d = oracle.dims_from(cfg)
        win = oracle.SlidingWindow(d)
        tpf = d.tokens_per_frame
        for ch in range(cfg.n_chunks):
            first, n_valid = chunk_schedule(cfg.chunk_frames, cfg.window_frames, ch)
            frames = win.frame_indices()
            assert n_valid == len(frames)
            assert frames == list(range(first - n_valid, first))
            # ring model: frame f lives in slot f mod W, so the filled slots are 0..n_valid-1
            assert sorted(f % cfg.window_frames for f in frames) == list(range(n_valid))
            z = np.zeros((cfg.chunk_frames * tpf, 1))
            win.frames.extend(oracle.FrameRecord(first + j, z[:tpf], z[:tpf])
                              for j in range(cfg.chunk_frames))
