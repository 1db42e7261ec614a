"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute: numbers
the VideoMLA pages print (tests/golden/), a library routine (torch's
scaled_dot_product_attention, the GPT-J rotary embedding in transformers),
closed-form properties of rotations and of softmax, and brute-force scalar
loops on tiny inputs.  A plausible slip in the oracle (a transposed weight, a
wrong head order, a dropped term, a flipped rotation, a wrong window) fails at
least one of them; ``test_planted_mistakes_are_caught`` checks that claim for a
list of slips planted into a copy of the oracle.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_attn_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def toy():
    cfg = inputs.CONFIGS[0]
    return cfg, oracle.dims_from(cfg)


def random_dims(**kw):
    base = dict(d_model=24, n_heads=3, d_head=5, d_c=7, d_rope=8, d_cq=6, pairs_t=2,
                pairs_h=1, pairs_w=1, rope_base=10000.0, frame_h=2, frame_w=3,
                chunk_frames=2, window_frames=3)
    base.update(kw)
    return oracle.Dims(**base)


def random_weights(d, rng, zero_rope=False):
    g = lambda *s: rng.standard_normal(s)
    w = inputs.LayerWeights(
        w_dkv=g(d.d_c, d.d_model), w_kr=g(d.d_rope, d.d_model) * (0 if zero_rope else 1),
        w_dq=g(d.d_cq, d.d_model), w_uq=g(d.n_heads, d.d_head, d.d_cq),
        w_uk=g(d.n_heads, d.d_head, d.d_c), w_uv=g(d.n_heads, d.d_head, d.d_c),
        w_qr=g(d.n_heads, d.d_rope, d.d_cq) * (0 if zero_rope else 1),
        w_o=g(d.d_model, d.n_heads * d.d_head))
    return w


# --------------------------------------------------------------------------
# numbers the pages print

def test_cache_size_matches_pages():
    gold = json.load(open(os.path.join(GOLDEN, "cache_size.json")))
    d = oracle.dims_from(inputs.CONFIGS[1])
    assert d.d_c == gold["d_c"]
    assert oracle.dense_scalars_per_token(d) == gold["dense_scalars_per_token"]
    assert oracle.latent_scalars_per_token(d) == gold["latent_scalars_per_token"]
    assert round(100 * oracle.kv_reduction(d), 1) == gold["reduction_percent_one_decimal"]


def test_every_wan_config_has_the_page_cache_layout():
    gold = json.load(open(os.path.join(GOLDEN, "cache_size.json")))
    for i in (1, 2, 3, 4):
        d = oracle.dims_from(inputs.CONFIGS[i])
        assert oracle.latent_scalars_per_token(d) == gold["latent_scalars_per_token"]


# --------------------------------------------------------------------------
# 3D-RoPE: closed-form properties and the textbook rotary embedding per band

def rot_inputs(seed=0, n=37):
    rng = np.random.default_rng(seed)
    d = oracle.dims_from(inputs.CONFIGS[1])
    pos = np.stack([rng.integers(0, 240, n), rng.integers(0, 30, n), rng.integers(0, 52, n)], 1)
    return d, rng, pos


def test_rope_identity_at_origin():
    d, rng, _ = rot_inputs()
    v = rng.standard_normal((5, d.d_rope))
    np.testing.assert_allclose(oracle.rope3d(v, np.zeros((5, 3), int), d), v, rtol=0, atol=0)


def test_rope_preserves_pair_norms():
    d, rng, pos = rot_inputs(1)
    v = rng.standard_normal((len(pos), d.d_rope))
    r = oracle.rope3d(v, pos, d)
    np.testing.assert_allclose((r[:, 0::2] ** 2 + r[:, 1::2] ** 2),
                               (v[:, 0::2] ** 2 + v[:, 1::2] ** 2), rtol=1e-12)


def test_rope_score_depends_only_on_relative_position():
    d, rng, pos = rot_inputs(2)
    a = rng.standard_normal((len(pos), d.d_rope))
    b = rng.standard_normal((len(pos), d.d_rope))
    pos2 = pos[::-1].copy()
    shift = np.array([17, 5, 11])
    s0 = np.sum(oracle.rope3d(a, pos, d) * oracle.rope3d(b, pos2, d), axis=1)
    s1 = np.sum(oracle.rope3d(a, pos + shift, d) * oracle.rope3d(b, pos2 + shift, d), axis=1)
    np.testing.assert_allclose(s1, s0, rtol=1e-10, atol=1e-10)


def test_rope_composes_additively():
    d, rng, pos = rot_inputs(3)
    v = rng.standard_normal((len(pos), d.d_rope))
    other = pos[::-1].copy()
    np.testing.assert_allclose(oracle.rope3d(oracle.rope3d(v, pos, d), other, d),
                               oracle.rope3d(v, pos + other, d), rtol=1e-9, atol=1e-9)


def test_rope_axes_touch_only_their_band():
    d, rng, pos = rot_inputs(4)
    v = rng.standard_normal((len(pos), d.d_rope))
    base = oracle.rope3d(v, pos, d)
    bounds = np.cumsum([0, 2 * d.pairs_t, 2 * d.pairs_h, 2 * d.pairs_w])
    for axis in range(3):
        moved = pos.copy()
        moved[:, axis] += 3
        r = oracle.rope3d(v, moved, d)
        lo, hi = bounds[axis], bounds[axis + 1]
        outside = np.r_[0:lo, hi:d.d_rope]
        np.testing.assert_array_equal(r[:, outside], base[:, outside])
        assert np.abs(r[:, lo:hi] - base[:, lo:hi]).max() > 1e-3


def test_rope_band_equals_textbook_rotary():
    """Each band is the interleaved-pair rotary embedding of GPT-J (the
    textbook RoFormer rotation, inverse frequency base^(-2i/dim)) applied to
    that band's channels at that axis' position."""
    from transformers.models.gptj.modeling_gptj import (apply_rotary_pos_emb,
                                                        create_sinusoidal_positions)
    d, rng, pos = rot_inputs(5)
    v = rng.standard_normal((len(pos), d.d_rope))
    r = oracle.rope3d(v, pos, d)
    lo = 0
    for axis, n_pairs in enumerate((d.pairs_t, d.pairs_h, d.pairs_w)):
        dim = 2 * n_pairs
        table = create_sinusoidal_positions(int(pos[:, axis].max()) + 1, dim)  # [P, dim]
        sincos = table[torch.from_numpy(pos[:, axis])]                            # [N, dim]
        sin, cos = sincos[:, :n_pairs][None], sincos[:, n_pairs:][None]            # [1, N, n]
        band = torch.from_numpy(v[:, lo:lo + dim])[None, :, None, :]               # [1,N,1,dim]
        ref = apply_rotary_pos_emb(band, sin.double(), cos.double())[0, :, 0].numpy()
        np.testing.assert_allclose(r[:, lo:lo + dim], ref, rtol=0, atol=2e-4)
        lo += dim


def test_rope_worked_example():
    """One pair at t = 1 on the first temporal pair (inverse frequency 1):
    (1, 0) turns by one radian counter-clockwise."""
    d = random_dims()
    v = np.zeros((1, d.d_rope))
    v[0, 0] = 1.0
    r = oracle.rope3d(v, np.array([[1, 0, 0]]), d)
    np.testing.assert_allclose(r[0, :2], [math.cos(1.0), math.sin(1.0)], rtol=1e-15)


# --------------------------------------------------------------------------
# softmax and absorption

def toy_chunk(seed=0, d=None, chunk=2):
    d = d or random_dims()
    rng = np.random.default_rng(seed)
    w = random_weights(d, rng)
    win = oracle.SlidingWindow(d)
    n_q = d.chunk_frames * d.tokens_per_frame
    res = None
    for c in range(chunk + 1):
        x = rng.standard_normal((n_q, d.d_model))
        res = oracle.chunk_step(d, w, x, win, c * d.chunk_frames, keep_p=True)
    return d, w, res


def test_softmax_rows_sum_to_one():
    _, _, r = toy_chunk(1)
    np.testing.assert_allclose(r["p"].sum(axis=2), 1.0, rtol=0, atol=1e-12)
    assert (r["p"] >= 0).all()


def test_lse_is_log_of_denominator():
    d, w, r = toy_chunk(2)
    s = (np.einsum("nhd,mhd->hnm", r["q_nope"], oracle.key_value_heads(r["c_keys"], w.w_uk,
                                                                        w.w_uv)[0])
         + np.einsum("nhr,mr->hnm", r["q_rope"], r["k_rope"])) * d.softmax_scale
    np.testing.assert_allclose(np.exp(s - r["lse"][..., None]), r["p"], rtol=1e-10, atol=1e-15)


def test_absorbed_form_equals_non_absorbed():
    d, w, r = toy_chunk(3)
    qp = oracle.absorbed_query(r["c_q"], w.w_uq, w.w_uk, w.w_qr, r["pos_q"], d)
    k_lat = np.concatenate([r["c_keys"], r["k_rope"]], axis=1)
    s_abs = np.einsum("nhc,mc->hnm", qp, k_lat) * d.softmax_scale
    k_nope, _ = oracle.key_value_heads(r["c_keys"], w.w_uk, w.w_uv)
    s_dir = (np.einsum("nhd,mhd->hnm", r["q_nope"], k_nope)
             + np.einsum("nhr,mr->hnm", r["q_rope"], r["k_rope"])) * d.softmax_scale
    np.testing.assert_allclose(s_abs, s_dir, rtol=1e-12, atol=1e-12)
    o_abs = oracle.up_project_output(r["o_lat"], w.w_uv)
    np.testing.assert_allclose(o_abs, r["o"], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# special case that reduces to textbook multi-head attention

def test_mha_special_case_matches_library_sdpa():
    """With W_down^KV = W_down^Q = I and zero positional projections the layer
    is plain multi-head attention with projections W_UQ_h, W_UK_h, W_UV_h over
    the window's tokens plus the chunk's; torch's SDPA is the reference.  The
    window is kept here as a plain list of past chunks (no deque, no slots)."""
    d = random_dims(d_model=10, d_c=10, d_cq=10, d_head=4, n_heads=3)
    rng = np.random.default_rng(7)
    w = random_weights(d, rng, zero_rope=True)
    w.w_dkv = np.eye(d.d_model)
    w.w_dq = np.eye(d.d_model)
    win = oracle.SlidingWindow(d)
    tpf = d.tokens_per_frame
    n_q = d.chunk_frames * tpf
    past_frames = []
    for c in range(5):
        x = rng.standard_normal((n_q, d.d_model))
        r = oracle.chunk_step(d, w, x, win, c * d.chunk_frames)
        window = past_frames[len(past_frames) - min(len(past_frames), d.window_frames):]
        keys = torch.from_numpy(np.concatenate(window + [x]))
        xq = torch.from_numpy(x)
        q = torch.einsum("hdk,nk->hnd", torch.from_numpy(w.w_uq), xq)
        k = torch.einsum("hdk,nk->hnd", torch.from_numpy(w.w_uk), keys)
        v = torch.einsum("hdk,nk->hnd", torch.from_numpy(w.w_uv), keys)
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=d.softmax_scale)
        ref = ref.permute(1, 0, 2).reshape(n_q, -1).numpy()
        np.testing.assert_allclose(r["o"], ref, rtol=1e-10, atol=1e-12)
        past_frames += [x[f * tpf:(f + 1) * tpf] for f in range(d.chunk_frames)]


# --------------------------------------------------------------------------
# brute force on tiny inputs

def brute_force_chunk(d, w, past_x, x, first_frame):
    """Scalar loops over tokens, heads and channels; the window is the last W
    frames of an explicit list of every earlier frame's tokens."""
    tpf = d.tokens_per_frame
    frames = [(f, past_x[f * tpf:(f + 1) * tpf]) for f in range(len(past_x) // tpf)]
    frames = frames[max(0, len(frames) - d.window_frames):]
    frames += [(first_frame + f, x[f * tpf:(f + 1) * tpf]) for f in range(d.chunk_frames)]

    def matvec(m, v):
        return [sum(m[i][j] * v[j] for j in range(len(v))) for i in range(len(m))]

    def rotate(vec, t, hh, ww):
        out = list(vec)
        pair = 0
        for axis_pos, n in ((t, d.pairs_t), (hh, d.pairs_h), (ww, d.pairs_w)):
            for i in range(n):
                ang = axis_pos * d.rope_base ** (-i / n)
                a, b = vec[2 * pair], vec[2 * pair + 1]
                out[2 * pair] = a * math.cos(ang) - b * math.sin(ang)
                out[2 * pair + 1] = a * math.sin(ang) + b * math.cos(ang)
                pair += 1
        return out

    keys = []
    for f, toks in frames:
        for i, tok in enumerate(toks):
            c = matvec(w.w_dkv, tok)
            kr = rotate(matvec(w.w_kr, tok), f, i // d.frame_w, i % d.frame_w)
            keys.append((c, kr))
    out = []
    for i, tok in enumerate(x):
        f = first_frame + i // tpf
        j = i % tpf
        cq = matvec(w.w_dq, tok)
        row = []
        for h in range(d.n_heads):
            qn = matvec(w.w_uq[h], cq)
            qr = rotate(matvec(w.w_qr[h], cq), f, j // d.frame_w, j % d.frame_w)
            scores = []
            for c, kr in keys:
                kn = matvec(w.w_uk[h], c)
                s = sum(a * b for a, b in zip(qn, kn)) + sum(a * b for a, b in zip(qr, kr))
                scores.append(s * d.softmax_scale)
            m = max(scores)
            e = [math.exp(s - m) for s in scores]
            z = sum(e)
            acc = [0.0] * d.d_head
            for p, (c, _) in zip(e, keys):
                vv = matvec(w.w_uv[h], c)
                for k in range(d.d_head):
                    acc[k] += p / z * vv[k]
            row.extend(acc)
        out.append(row)
    return np.array(out)


def test_brute_force_rollout_with_wraparound():
    d = random_dims(window_frames=3, chunk_frames=2, frame_h=2, frame_w=2)
    rng = np.random.default_rng(11)
    w = random_weights(d, rng)
    win = oracle.SlidingWindow(d)
    n_q = d.chunk_frames * d.tokens_per_frame
    past = np.zeros((0, d.d_model))
    for c in range(4):   # frames 0..7, window of 3: wraps twice
        x = rng.standard_normal((n_q, d.d_model))
        r = oracle.chunk_step(d, w, x, win, c * d.chunk_frames)
        ref = brute_force_chunk(d, w, past, x, c * d.chunk_frames)
        np.testing.assert_allclose(r["o"], ref, rtol=1e-10, atol=1e-12)
        past = np.concatenate([past, x])
    assert win.frame_indices() == [5, 6, 7]


def test_window_holds_the_last_w_frames():
    cfg, d = toy()
    win = oracle.SlidingWindow(d)
    tpf = d.tokens_per_frame
    for c in range(6):
        seen = win.frame_indices()
        assert seen == list(range(max(0, c - d.window_frames), c))
        win.append_chunk(c, np.full((tpf, d.d_c), c, float), np.zeros((tpf, d.d_rope)))
    assert [int(r.c_kv[0, 0]) for r in win.frames] == [4, 5]


def test_positions_row_major():
    d = random_dims(frame_h=2, frame_w=3)
    p = oracle.token_positions([4, 9], d)
    assert p.tolist() == [[4, 0, 0], [4, 0, 1], [4, 0, 2], [4, 1, 0], [4, 1, 1], [4, 1, 2],
                          [9, 0, 0], [9, 0, 1], [9, 0, 2], [9, 1, 0], [9, 1, 1], [9, 1, 2]]


def test_output_projection_brute_force():
    rng = np.random.default_rng(5)
    o = rng.standard_normal((3, 4))
    w_o = rng.standard_normal((5, 4))
    y = oracle.output_projection(o, w_o)
    for n in range(3):
        for i in range(5):
            assert abs(y[n, i] - sum(w_o[i, k] * o[n, k] for k in range(4))) < 1e-12


# --------------------------------------------------------------------------
# gradients (training use): pinned to finite differences of the forward, to the non-absorbed
# chain rule, and to the adjoint property of a rotation

def _latent_forward(q, c, k_r, pos_k, d):
    """O_lat through the (separately pinned) forward pieces: attention_probabilities with the
    content latent as both the content key and the value, and the rotated positional key."""
    n_heads = q.shape[1]
    keys = np.repeat(c[:, None, :], n_heads, axis=1)
    return oracle.attend(q[:, :, :d.d_c], q[:, :, d.d_c:], keys, oracle.rope3d(k_r, pos_k, d),
                         keys, d.softmax_scale, c_keys=c)["o_lat"]


def _backward_case(seed=3, n=4, m=6):
    d = random_dims()
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n, d.n_heads, d.d_c + d.d_rope))
    c = rng.standard_normal((m, d.d_c))
    k_r = rng.standard_normal((m, d.d_rope))
    pos_k = rng.integers(0, 5, size=(m, 3))
    g = rng.standard_normal((n, d.n_heads, d.d_c))
    return d, q, c, k_r, pos_k, g


def test_backward_matches_finite_differences():
    d, q, c, k_r, pos_k, g = _backward_case()
    res = oracle.latent_attention_backward(q, c, k_r, pos_k, g, d)
    loss = lambda q_, c_, k_: float((g * _latent_forward(q_, c_, k_, pos_k, d)).sum())
    eps = 1e-6
    for name, arr, grad in (("q", q, res["d_q"]), ("c", c, res["d_c"]), ("k_r", k_r, res["d_k_r"])):
        num = np.zeros_like(arr)
        for i in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[i] += eps
            minus[i] -= eps
            args_p = {"q": (plus, c, k_r), "c": (q, plus, k_r), "k_r": (q, c, plus)}[name]
            args_m = {"q": (minus, c, k_r), "c": (q, minus, k_r), "k_r": (q, c, minus)}[name]
            num[i] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)
    np.testing.assert_allclose(res["o_lat"], _latent_forward(q, c, k_r, pos_k, d), atol=1e-12)


def test_backward_absorbed_equals_non_absorbed():
    """The latent-space gradients are those of the layer with per-head keys and values rebuilt
    from c_KV: w.r.t. c_KV and k_R directly, w.r.t. c_Q through the absorbed query weights."""
    d = random_dims()
    rng = np.random.default_rng(11)
    w = random_weights(d, rng)
    n, m = 5, 7
    c_q = rng.standard_normal((n, d.d_cq))
    pos_q = rng.integers(0, 6, size=(n, 3))
    c = rng.standard_normal((m, d.d_c))
    k_r = rng.standard_normal((m, d.d_rope))
    pos_k = rng.integers(0, 6, size=(m, 3))
    d_o = rng.standard_normal((n, d.n_heads, d.d_head))
    ref = oracle.layer_backward_nonabsorbed(d, w, c_q, pos_q, c, k_r, pos_k, d_o)
    q = oracle.absorbed_query(c_q, w.w_uq, w.w_uk, w.w_qr, pos_q, d)
    d_o_lat = np.einsum("hdc,nhd->nhc", w.w_uv, d_o)           # o_h = W_UV_h O_lat,h
    lat = oracle.latent_attention_backward(q, c, k_r, pos_k, d_o_lat, d)
    np.testing.assert_allclose(lat["d_c"], ref["d_c"], rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(lat["d_k_r"], ref["d_k_r"], rtol=1e-10, atol=1e-10)
    d_q_lat, d_q_rope = lat["d_q"][..., :d.d_c], lat["d_q"][..., d.d_c:]
    d_c_q = (np.einsum("hdk,hdc,nhc->nk", w.w_uq, w.w_uk, d_q_lat) +
             np.einsum("hdk,nhd->nk", w.w_qr, oracle.rope3d_adjoint(d_q_rope, pos_q, d)))
    np.testing.assert_allclose(d_c_q, ref["d_c_q"], rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(oracle.up_project_output(lat["o_lat"], w.w_uv),
                               ref["o"].reshape(n, -1), rtol=1e-10, atol=1e-10)


def test_rope_adjoint_is_the_transpose():
    d = random_dims()
    rng = np.random.default_rng(5)
    x, y = rng.standard_normal((9, d.d_rope)), rng.standard_normal((9, d.d_rope))
    pos = rng.integers(-4, 9, size=(9, 3))
    lhs = (oracle.rope3d(x, pos, d) * y).sum(axis=1)
    rhs = (x * oracle.rope3d_adjoint(y, pos, d)).sum(axis=1)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def test_backward_is_linear_in_the_upstream_gradient():
    d, q, c, k_r, pos_k, g = _backward_case(seed=8)
    a = oracle.latent_attention_backward(q, c, k_r, pos_k, g, d)
    b = oracle.latent_attention_backward(q, c, k_r, pos_k, -2.5 * g, d)
    for k in ("d_q", "d_c", "d_k_r"):
        np.testing.assert_allclose(b[k], -2.5 * a[k], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# the pins above catch planted slips

PINS = [test_rope_identity_at_origin, test_rope_preserves_pair_norms,
        test_rope_score_depends_only_on_relative_position, test_rope_composes_additively,
        test_rope_axes_touch_only_their_band, test_rope_band_equals_textbook_rotary,
        test_rope_worked_example, test_softmax_rows_sum_to_one, test_lse_is_log_of_denominator,
        test_absorbed_form_equals_non_absorbed, test_mha_special_case_matches_library_sdpa,
        test_brute_force_rollout_with_wraparound, test_window_holds_the_last_w_frames,
        test_positions_row_major, test_cache_size_matches_pages,
        test_output_projection_brute_force, test_backward_matches_finite_differences,
        test_backward_absorbed_equals_non_absorbed, test_rope_adjoint_is_the_transpose,
        test_backward_is_linear_in_the_upstream_gradient]


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(oracle.mla_oracle, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def _mutants():
    M = oracle.mla_oracle
    orig_rope, orig_angles, orig_attn = M.rope3d, M.rope3d_angles, M.attention_probabilities
    orig_kv, orig_qh, orig_pos = M.key_value_heads, M.query_heads, M.token_positions
    orig_attend = M.attend
    orig_sbw, orig_lab = M.softmax_backward, M.latent_attention_backward

    def rope_flipped(vec, pos, d):
        return orig_rope(vec, -np.asarray(pos), d)

    def angles_wrong_exponent(pos, d):
        pos = np.asarray(pos, np.float64)
        bands = []
        for axis, n in enumerate((d.pairs_t, d.pairs_h, d.pairs_w)):
            bands.append(pos[:, axis:axis + 1] * d.rope_base ** (-2 * np.arange(n) / n)[None])
        return np.concatenate(bands, 1)

    def angles_bands_swapped(pos, d):
        pos = np.asarray(pos)[:, [1, 0, 2]]
        return orig_angles(pos, d)

    def attn_no_rope_term(qn, qr, kn, kr, scale):
        return orig_attn(qn, qr * 0, kn, kr, scale)

    def attn_wrong_scale(qn, qr, kn, kr, scale):
        return orig_attn(qn, qr, kn, kr, scale * 1.25)

    def attn_lse_without_max(qn, qr, kn, kr, scale):
        p, lse = orig_attn(qn, qr, kn, kr, scale)
        s = (qn @ kn.T + qr @ kr.T) * scale
        return p, lse - s.max(axis=1)

    def kv_swapped(c, w_uk, w_uv):
        k, v = orig_kv(c, w_uk, w_uv)
        return v, k

    def q_heads_reversed(c_q, w_uq, w_qr):
        qn, qr = orig_qh(c_q, w_uq, w_qr)
        return qn[:, ::-1], qr

    def positions_column_major(frames, d):
        p = orig_pos(frames, d)
        return p[:, [0, 2, 1]] if d.frame_h == d.frame_w else np.concatenate(
            [p[:, :1], (np.arange(len(p)) % d.tokens_per_frame % d.frame_h)[:, None],
             (np.arange(len(p)) % d.tokens_per_frame // d.frame_h)[:, None]], 1)

    def attend_heads_interleaved(qn, qr, kn, kr, v, scale, c_keys=None, keep_p=False):
        out = orig_attend(qn, qr, kn, kr, v, scale, c_keys, keep_p)
        n, hd = out["o"].shape
        h = qn.shape[1]
        out["o"] = out["o"].reshape(n, h, hd // h).transpose(0, 2, 1).reshape(n, hd)
        return out

    class ShortWindow(M.SlidingWindow):
        def __init__(self, d):
            super().__init__(d)
            import collections
            self.frames = collections.deque(maxlen=max(1, d.window_frames - 1))

    def dense_wrong(d):
        return d.n_heads * d.d_head

    def out_proj_transposed(o, w_o):
        return np.asarray(o, np.float64) @ np.asarray(w_o, np.float64)[:, :np.asarray(o).shape[1]]

    def softmax_bw_no_row_term(p, d_p):
        return p * d_p

    def rope_adjoint_same_direction(vec, pos, d):
        return orig_rope(vec, pos, d)

    def backward_value_gradient_dropped(q, c, k_r, pos_k, g, d):
        res = orig_lab(q, c, k_r, pos_k, g, d)
        p_t = []
        for h in range(q.shape[1]):
            k_full = np.concatenate([c, orig_rope(k_r, pos_k, d)], axis=1)
            s = q[:, h] @ k_full.T * d.softmax_scale
            e = np.exp(s - s.max(axis=1, keepdims=True))
            p_t.append((e / e.sum(axis=1, keepdims=True)).T @ g[:, h])
        return dict(res, d_c=res["d_c"] - sum(p_t))

    def backward_unscaled_query_gradient(q, c, k_r, pos_k, g, d):
        res = orig_lab(q, c, k_r, pos_k, g, d)
        return dict(res, d_q=res["d_q"] / d.softmax_scale)

    return {
        "softmax gradient without the row term": [("softmax_backward", softmax_bw_no_row_term)],
        "rope adjoint turns the same way": [("rope3d_adjoint", rope_adjoint_same_direction)],
        "value gradient dropped": [("latent_attention_backward", backward_value_gradient_dropped)],
        "query gradient without the scale": [("latent_attention_backward",
                                              backward_unscaled_query_gradient)],
        "rope rotates the wrong way": [("rope3d", rope_flipped)],
        "rope frequency exponent doubled": [("rope3d_angles", angles_wrong_exponent)],
        "rope bands t/h swapped": [("rope3d_angles", angles_bands_swapped)],
        "positional score term dropped": [("attention_probabilities", attn_no_rope_term)],
        "softmax scale wrong": [("attention_probabilities", attn_wrong_scale)],
        "lse without the row max": [("attention_probabilities", attn_lse_without_max)],
        "keys and values swapped": [("key_value_heads", kv_swapped)],
        "query heads reversed": [("query_heads", q_heads_reversed)],
        "tokens column-major": [("token_positions", positions_column_major)],
        "head outputs interleaved": [("attend", attend_heads_interleaved)],
        "window one frame short": [("SlidingWindow", ShortWindow)],
        "dense cache counted once": [("dense_scalars_per_token", dense_wrong)],
        "output projection transposed": [("output_projection", out_proj_transposed)],
    }


@pytest.mark.parametrize("name", sorted(_mutants().keys()))
def test_planted_mistakes_are_caught(name, monkeypatch):
    for attr, fn in _mutants()[name]:
        _patch(monkeypatch, attr, fn)
    failed = []
    for pin in PINS:
        try:
            pin()
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted slip: {name}"

