"""The library's two hand-written approximations, held to their error bounds on the device.

Both are evaluated by the very device functions the kernels call, through the test-only entry
points mla_selftest_exp2 / mla_selftest_sincos / mla_selftest_rope_angles:

* the softmax's FMA-pipe exponential (exp2_poly_pair): 2^x = 2^n * q(f), n = rint(x),
  f = x - n in [-1/2, 1/2], q the cubic interpolating 2^f at the four Chebyshev nodes of
  [-1/2, 1/2] (tests/test_approx_host.py pins the constants to that definition and finds the
  interpolant's largest relative error, 9.97e-5).  On the device the cubic is evaluated in
  float32 by three FMAs and scaled exactly through the exponent field, so it may add a few
  float32 roundings.  Checked against float64 2^x and against CUDA's exp2f over the whole range
  the softmax passes ([-125, 8]), at the clamp and at both ends.
* 3D-RoPE's angle and sine/cosine (rope_angle, rope_sincos): the angle pos_a * base^(-i/n_a) in
  float (the inverse frequency rounded once on the host, the product once on the device), then
  a two-constant Cody-Waite reduction by 2 pi and the hardware sine/cosine on [-pi, pi].
  Checked against float64 over every position the Wan workloads produce (t up to 239, every
  row and column of a 30 x 52 frame) for the three rotary splits of the latent-size presets.
"""
import ctypes

import numpy as np
import pytest
import torch

from mla_latent_kv_attn_b200 import _lib, api, inputs

pytestmark = pytest.mark.gpu

# the interpolant's own worst relative error (float64, tests/test_approx_host.py) plus four
# float32 roundings of its evaluation
POLY_REL = 9.975e-5 + 4 * 2.0 ** -24


def _exp2(x: np.ndarray):
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    outs = [torch.empty_like(xd) for _ in range(3)]
    st = _lib.lib().mla_selftest_exp2(xd.data_ptr(), outs[0].data_ptr(), outs[1].data_ptr(),
                                      outs[2].data_ptr(), xd.numel(),
                                      torch.cuda.current_stream().cuda_stream)
    assert st == 0, _lib.last_error()
    torch.cuda.synchronize()
    return [o.cpu().numpy().astype(np.float64) for o in outs]


def test_exp2_polynomial_within_its_bound_over_the_softmax_range():
    grid = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    special = np.array([-125.0, -124.5, -124.0, -1.0, -0.5, -0.25, 0.0, 0.25, 0.5, 1.0, 7.5, 8.0],
                       dtype=np.float32)
    # both sides of every rounding boundary n + 1/2 (f changes sign there)
    halves = np.arange(-125, 8, dtype=np.float32) + np.float32(0.5)
    edges = np.concatenate([np.nextafter(halves, np.float32(-200)), halves,
                            np.nextafter(halves, np.float32(200))])
    x = np.concatenate([grid, special, edges])
    y_poly, y_sfu, y_exp2f = _exp2(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y_poly - ref) / ref
    assert np.isfinite(y_poly).all()
    assert rel.max() <= POLY_REL, f"max relative error {rel.max():.3e} at x = {x[rel.argmax()]}"
    # against CUDA's own exp2f, as the kernels would otherwise use it
    rel_cuda = np.abs(y_poly - y_exp2f) / y_exp2f
    assert rel_cuda.max() <= POLY_REL + 2.0 ** -21
    # the SFU path of the same softmax (ex2.approx) for comparison: far tighter
    rel_sfu = np.abs(y_sfu - ref) / ref
    assert rel_sfu.max() <= 2.0 ** -20
    # at x = 0 the result is q(0) (n = 0, the exponent field untouched)
    assert y_poly[x == 0.0][0] == pytest.approx(1.0, rel=POLY_REL)


def test_exp2_polynomial_clamps_below_minus_125():
    x = np.array([-125.0, -125.5, -126.0, -130.0, -149.0, -200.0, -1e4, -np.inf],
                 dtype=np.float32)
    y_poly, _, _ = _exp2(x)
    at_clamp = y_poly[0]
    assert at_clamp > 0.0 and at_clamp <= 2.0 ** -124
    # every argument below the clamp gives the clamp's value: a normal float, never negative,
    # never a garbage exponent
    np.testing.assert_array_equal(y_poly, np.full_like(y_poly, at_clamp))


def _sincos(a: np.ndarray):
    ad = torch.from_numpy(a.astype(np.float32)).cuda()
    s, c = torch.empty_like(ad), torch.empty_like(ad)
    st = _lib.lib().mla_selftest_sincos(ad.data_ptr(), s.data_ptr(), c.data_ptr(), ad.numel(),
                                        torch.cuda.current_stream().cuda_stream)
    assert st == 0, _lib.last_error()
    torch.cuda.synchronize()
    return s.cpu().numpy().astype(np.float64), c.cpu().numpy().astype(np.float64)


# error of rope_sincos for a float angle: hardware sine/cosine on [-pi, pi] (2^-21.4) plus the two
# roundings of the Cody-Waite reduction (half an ulp of a value below 4 each)
SINCOS_ABS = 1.0e-6


def test_rope_sincos_of_float_angles():
    rng = np.random.default_rng(5)
    a = np.concatenate([
        rng.uniform(-2.0 ** 15, 2.0 ** 15, 1_000_000),
        rng.uniform(-300.0, 300.0, 1_000_000),
        np.pi / 2 * np.arange(-2000, 2001),                    # quadrant points
        np.pi * (2 * np.arange(-2000, 2001) + 1),               # reduction boundaries (k + 1/2)
    ]).astype(np.float32)
    s, c = _sincos(a)
    ad = a.astype(np.float64)
    err_s = np.abs(s - np.sin(ad))
    err_c = np.abs(c - np.cos(ad))
    assert err_s.max() <= SINCOS_ABS, f"sin: {err_s.max():.3e} at {a[err_s.argmax()]}"
    assert err_c.max() <= SINCOS_ABS, f"cos: {err_c.max():.3e} at {a[err_c.argmax()]}"


@pytest.mark.parametrize("d_rope", [16, 32, 64])
def test_rope_angles_over_every_wan_position(d_rope):
    cfg = inputs.with_latent_shape(inputs.CONFIGS[2], inputs.CONFIGS[2].d_c, d_rope)
    c = api.make_config(cfg)
    t, h, w = np.meshgrid(np.arange(240), np.arange(cfg.frame_h), np.arange(cfg.frame_w),
                          indexing="ij")
    pos = np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1).astype(np.int32)
    n, n_pairs = len(pos), d_rope // 2
    pd = torch.from_numpy(pos).cuda()
    ang = torch.empty((n, n_pairs), device="cuda", dtype=torch.float32)
    s, co = torch.empty_like(ang), torch.empty_like(ang)
    st = _lib.lib().mla_selftest_rope_angles(
        ctypes.byref(c), pd.data_ptr(), n, ang.data_ptr(), s.data_ptr(),
        co.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, _lib.last_error()
    torch.cuda.synchronize()
    # float64 angles of the same reading: pair i of axis a turns by pos_a * base^(-i / n_a)
    pt, ph, pw = cfg.rope_pairs
    freq, axis = [], []
    for a_idx, n_a in enumerate((pt, ph, pw)):
        for i in range(n_a):
            freq.append(cfg.rope_base ** (-i / n_a))
            axis.append(a_idx)
    exact = pos[:, axis].astype(np.float64) * np.array(freq)[None, :]
    got = ang.cpu().numpy().astype(np.float64)
    # two float roundings (the inverse frequency, the product): 2^-24 relative each
    assert (np.abs(got - exact) <= np.abs(exact) * 2.0 ** -23 + 1e-30).all()
    bound = np.abs(exact) * 2.0 ** -23 + SINCOS_ABS
    assert (np.abs(s.cpu().numpy() - np.sin(exact)) <= bound).all()
    assert (np.abs(co.cpu().numpy() - np.cos(exact)) <= bound).all()
