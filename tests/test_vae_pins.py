"""Pins of the VAE-decode oracle (oracle/vae.py) against routes independent of it.

* The causal convolution equals PyTorch's conv3d in fp64 on the same bf16 values,
  with the history frames (or zeros) placed in front of the chunk and one zero
  row / column of padding: a library route.
* A delta kernel (identity channels at the current frame's centre tap) returns
  the input plus the bias exactly; the same delta at the oldest frame's tap
  shifts the sequence two frames back, so the first two output frames are the
  history (or zeros); a delta at a corner tap shifts the frame by one row and one
  column and fills the border with zeros: the causal and spatial padding in
  closed form.
* A brute-force sum over every tap and channel in plain Python on a tiny shape.
* Causality: changing input frame t0 changes no output frame before t0.
* Streaming: two chunks decoded one after the other, the second with the last
  two input frames of the first as its history, give the convolution of the
  concatenated sequence (the property the chunk-pipelined decode relies on).
* RMSNorm + SiLU equals torch's rms_norm followed by silu in fp64.
* The residual block streamed over chunks equals the block applied to the
  whole sequence at once.
"""
import itertools

import numpy as np
import torch

import oracle
import oracle.vae as ov


def _bits(a):
    return oracle.f64_to_bf16(np.asarray(a, np.float64))


def _rand_bits(rng, shape, scale=1.0):
    return _bits(rng.standard_normal(shape) * scale)


def _torch_conv(x_bits, hist_bits, w_bits, bias):
    x = oracle.bf16_to_f64(x_bits)
    T, H, W, C = x.shape
    hist = np.zeros((2, H, W, C)) if hist_bits is None else oracle.bf16_to_f64(hist_bits)
    xe = torch.from_numpy(np.concatenate([hist, x], 0))          # [T+2, H, W, C]
    xe = xe.permute(3, 0, 1, 2)[None]                            # [1, C, T+2, H, W]
    xe = torch.nn.functional.pad(xe, (1, 1, 1, 1, 0, 0))
    w = torch.from_numpy(oracle.bf16_to_f64(w_bits)).permute(0, 4, 1, 2, 3)   # [O, C, 3, 3, 3]
    y = torch.nn.functional.conv3d(xe, w, torch.from_numpy(np.asarray(bias, np.float64)))
    return y[0].permute(1, 2, 3, 0).numpy()


def test_conv_equals_library_conv3d():
    rng = np.random.default_rng(0)
    for T, H, W, Cin, Cout, with_hist in [(3, 5, 7, 4, 6, True), (1, 4, 4, 3, 2, False),
                                          (4, 3, 9, 8, 5, True)]:
        x = _rand_bits(rng, (T, H, W, Cin))
        hist = _rand_bits(rng, (2, H, W, Cin)) if with_hist else None
        w = _rand_bits(rng, (Cout, 3, 3, 3, Cin), 0.3)
        b = rng.standard_normal(Cout).astype(np.float32)
        got = ov.causal_conv3d_f64(x, hist, w, b)
        ref = _torch_conv(x, hist, w, b)
        assert np.allclose(got, ref, rtol=0, atol=1e-12), np.abs(got - ref).max()


def test_delta_kernels_closed_forms():
    rng = np.random.default_rng(1)
    T, H, W, C = 4, 5, 6, 3
    x = _rand_bits(rng, (T, H, W, C))
    hist = _rand_bits(rng, (2, H, W, C))
    b = np.array([0.5, -0.25, 2.0], np.float32)
    eye = np.eye(C)
    # current frame, centre tap: identity
    w = np.zeros((C, 3, 3, 3, C))
    w[:, 2, 1, 1, :] = eye
    y = ov.causal_conv3d_f64(x, hist, _bits(w), b)
    assert np.array_equal(y, oracle.bf16_to_f64(x) + b.astype(np.float64))
    # oldest frame: a shift by two frames, the history first
    w = np.zeros((C, 3, 3, 3, C))
    w[:, 0, 1, 1, :] = eye
    y = ov.causal_conv3d_f64(x, hist, _bits(w))
    xs = oracle.bf16_to_f64(x)
    hs = oracle.bf16_to_f64(hist)
    assert np.array_equal(y[:2], hs) and np.array_equal(y[2:], xs[:T - 2])
    y0 = ov.causal_conv3d_f64(x, None, _bits(w))
    assert np.array_equal(y0[:2], np.zeros_like(hs)) and np.array_equal(y0[2:], xs[:T - 2])
    # corner tap (dy = 0, dx = 0): out[i, j] = in[i-1, j-1], zero on the first row / column
    w = np.zeros((C, 3, 3, 3, C))
    w[:, 2, 0, 0, :] = eye
    y = ov.causal_conv3d_f64(x, hist, _bits(w))
    assert np.array_equal(y[:, 1:, 1:], xs[:, :-1, :-1])
    assert not y[:, 0, :].any() and not y[:, :, 0].any()


def test_conv_brute_force_tiny():
    rng = np.random.default_rng(2)
    T, H, W, Cin, Cout = 2, 3, 4, 3, 2
    x = _rand_bits(rng, (T, H, W, Cin))
    hist = _rand_bits(rng, (2, H, W, Cin))
    w = _rand_bits(rng, (Cout, 3, 3, 3, Cin))
    b = rng.standard_normal(Cout).astype(np.float32)
    r = _rand_bits(rng, (T, H, W, Cout))
    xf, hf, wf_, rf = (oracle.bf16_to_f64(a) for a in (x, hist, w, r))

    def X(t, i, j, c):
        if not (0 <= i < H and 0 <= j < W):
            return 0.0
        return float(hf[t + 2, i, j, c]) if t < 0 else float(xf[t, i, j, c])

    got = ov.causal_conv3d_f64(x, hist, w, b, resid_bits=r)
    for t, i, j, o in itertools.product(range(T), range(H), range(W), range(Cout)):
        acc = float(b[o]) + float(rf[t, i, j, o])
        for dt, dy, dx, c in itertools.product(range(3), range(3), range(3), range(Cin)):
            acc += float(wf_[o, dt, dy, dx, c]) * X(t + dt - 2, i + dy - 1, j + dx - 1, c)
        assert abs(got[t, i, j, o] - acc) <= 1e-12 * (1 + abs(acc))


def test_conv_causality_and_streaming():
    rng = np.random.default_rng(3)
    T1, T2, H, W, Cin, Cout = 3, 4, 4, 5, 4, 3
    x = _rand_bits(rng, (T1 + T2, H, W, Cin))
    w = _rand_bits(rng, (Cout, 3, 3, 3, Cin), 0.3)
    b = rng.standard_normal(Cout).astype(np.float32)
    full = ov.causal_conv3d_f64(x, None, w, b)
    # causality: a change at frame t0 leaves frames < t0 bit-identical
    for t0 in range(T1 + T2):
        x2 = x.copy()
        x2[t0] = _rand_bits(rng, (H, W, Cin))
        y2 = ov.causal_conv3d_f64(x2, None, w, b)
        assert np.array_equal(y2[:t0], full[:t0])
        assert not np.array_equal(y2[t0:], full[t0:])
    # streaming: chunk 2 with chunk 1's last two frames as history
    y1 = ov.causal_conv3d_f64(x[:T1], None, w, b)
    y2 = ov.causal_conv3d_f64(x[T1:], x[T1 - 2:T1], w, b)
    assert np.allclose(np.concatenate([y1, y2]), full, rtol=0, atol=1e-12)


def test_conv_at_matches_full_and_bounds_terms():
    rng = np.random.default_rng(4)
    T, H, W, Cin, Cout = 3, 5, 6, 8, 4
    x = _rand_bits(rng, (T, H, W, Cin))
    hist = _rand_bits(rng, (2, H, W, Cin))
    w = _rand_bits(rng, (Cout, 3, 3, 3, Cin), 0.2)
    b = rng.standard_normal(Cout).astype(np.float32)
    r = _rand_bits(rng, (T, H, W, Cout))
    full = ov.causal_conv3d_f64(x, hist, w, b, resid_bits=r)
    px = np.array([[0, 0, 0], [2, 4, 5], [1, 2, 3], [0, 4, 0]])
    y, s = ov.causal_conv3d_at(x, hist, w, px, b, resid_bits=r)
    assert np.allclose(y, full[px[:, 0], px[:, 1], px[:, 2]], rtol=0, atol=1e-12)
    assert (s >= np.abs(y - oracle.bf16_to_f64(r)[px[:, 0], px[:, 1], px[:, 2]]) - 1e-12).all()


def test_rms_norm_silu_equals_torch():
    rng = np.random.default_rng(5)
    x = _rand_bits(rng, (2, 3, 4, 96), 3.0)
    g = (1 + 0.1 * rng.standard_normal(96)).astype(np.float32)
    got = ov.rms_norm_silu_f64(x, g)
    t = torch.from_numpy(oracle.bf16_to_f64(x))
    ref = torch.nn.functional.silu(torch.nn.functional.rms_norm(
        t, (96,), torch.from_numpy(g.astype(np.float64)), eps=1e-6)).numpy()
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-14)


def test_res_block_streams_like_the_whole_sequence():
    rng = np.random.default_rng(6)
    T1, T2, H, W, C = 3, 2, 4, 5, 8
    x = _rand_bits(rng, (T1 + T2, H, W, C))
    wts = dict(gamma1=(1 + 0.1 * rng.standard_normal(C)).astype(np.float32),
               gamma2=(1 + 0.1 * rng.standard_normal(C)).astype(np.float32),
               w1=_rand_bits(rng, (C, 3, 3, 3, C), 0.1), w2=_rand_bits(rng, (C, 3, 3, 3, C), 0.1),
               b1=(0.02 * rng.standard_normal(C)).astype(np.float32),
               b2=(0.02 * rng.standard_normal(C)).astype(np.float32))
    whole, _, _ = ov.res_block(x, wts)
    o1, _, h = ov.res_block(x[:T1], wts)
    o2, _, _ = ov.res_block(x[T1:], wts, h)
    assert np.array_equal(np.concatenate([o1, o2]), whole)
    # a one-frame chunk reaches into the history for its last two frames
    o1, _, h = ov.res_block(x[:T1], wts)
    oa, _, h = ov.res_block(x[T1:T1 + 1], wts, h)
    ob, _, _ = ov.res_block(x[T1 + 1:], wts, h)
    assert np.array_equal(np.concatenate([o1, oa, ob]), whole)
