"""CPU fp64 oracle for the streaming VAE-decode stage.

TEST INFRASTRUCTURE ONLY (the same rule as the rest of ``oracle/``): only
``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` call it.

"Wave Forcing: Towards Speed-of-Light Streaming Video Generation" (abstract)
lists pipelined VAE decoding as one of the three parts of its runtime; the
airadar.tv summary (usage section) takes the VAE from the Wan2.1 base model,
splits its decode into ``--vae-stages 2`` or ``3`` pipeline stages, and decodes
399 latent frames into 1593 video frames.  The pages print no layer of the
decoder.  The readings taken here (plain definitions of a causal 3D-conv
decoder stage, each stated once):

* Activations are channels-last ``[T, H, W, C]`` bf16; one chunk is the frames
  decoded from one output chunk of the wave.
* The decoder's convolution is a 3x3x3 convolution that is causal in time:
  output frame ``t`` reads input frames ``t-2, t-1, t`` and rows/columns
  ``i-1..i+1``, ``j-1..j+1`` (zero outside the frame).  Frames before the
  chunk (``t-2 < 0``) come from the last two input frames of the previous chunk
  (``hist``), or are zero at the start of the video.  Streaming the video chunk
  by chunk this way gives exactly the convolution of the whole sequence, which
  is what lets the decode run as a pipeline over chunks.
* Weights are ``[Cout, 3, 3, 3, Cin]`` bf16 (tap ``(dt, dy, dx)``, ``dt = 0``
  the oldest frame), bias ``[Cout]`` fp32; the product of the bf16 operands is
  formed exactly in fp64 and the result (bias and an optional residual added)
  is rounded once to bf16.
* The normalisation before each convolution is an RMSNorm over the channels of
  each pixel with a learned gain ``gamma [C]`` (eps 1e-6), followed by SiLU,
  ``y * sigmoid(y)``; rounded once to bf16.
* A residual block is ``x + conv2(norm_silu2(conv1(norm_silu1(x))))``, with
  conv1's output rounded to bf16 before the second norm.

Pins: ``tests/test_vae_pins.py``.
"""
from __future__ import annotations

import numpy as np

from . import bf16_to_f64, f64_to_bf16

VAE_EPS = 1e-6
KT = 3          # taps in time (causal: t-2, t-1, t)
KS = 3          # taps in each spatial direction (centred)


def _extended(x_bits, hist_bits):
    """fp64 input with the two history frames in front: [T + 2, H, W, C]."""
    x = bf16_to_f64(x_bits)
    T, H, W, C = x.shape
    if hist_bits is None:
        hist = np.zeros((KT - 1, H, W, C))
    else:
        hist = bf16_to_f64(hist_bits)
        if hist.shape != (KT - 1, H, W, C):
            raise ValueError("hist must be [2, H, W, C], got %r" % (hist.shape,))
    return np.concatenate([hist, x], axis=0)


def causal_conv3d_f64(x_bits, hist_bits, w_bits, bias=None, resid_bits=None):
    """Exact causal 3x3x3 convolution (see the module docstring), fp64, not rounded.

    x_bits [T, H, W, Cin], hist_bits [2, H, W, Cin] or None, w_bits
    [Cout, 3, 3, 3, Cin] (bf16 bit patterns); bias [Cout] fp32 or None;
    resid_bits [T, H, W, Cout] or None.  Returns [T, H, W, Cout] float64.
    """
    xe = _extended(x_bits, hist_bits)
    w = bf16_to_f64(w_bits)
    Cout = w.shape[0]
    T = xe.shape[0] - (KT - 1)
    H, W = xe.shape[1], xe.shape[2]
    # zero padding of one row / column on each side
    xp = np.zeros((xe.shape[0], H + 2, W + 2, xe.shape[3]))
    xp[:, 1:H + 1, 1:W + 1, :] = xe
    y = np.zeros((T, H, W, Cout))
    for dt in range(KT):
        for dy in range(KS):
            for dx in range(KS):
                win = xp[dt:dt + T, dy:dy + H, dx:dx + W, :]       # X(t+dt-2, i+dy-1, j+dx-1)
                y += win @ w[:, dt, dy, dx, :].T
    if bias is not None:
        y += np.asarray(bias, np.float32).astype(np.float64)
    if resid_bits is not None:
        y += bf16_to_f64(resid_bits)
    return y


def causal_conv3d(x_bits, hist_bits, w_bits, bias=None, resid_bits=None):
    """bf16 bits of :func:`causal_conv3d_f64` (one rounding)."""
    return f64_to_bf16(causal_conv3d_f64(x_bits, hist_bits, w_bits, bias, resid_bits))


def causal_conv3d_at(x_bits, hist_bits, w_bits, pixels, bias=None, resid_bits=None):
    """:func:`causal_conv3d_f64` at selected output pixels only.

    pixels: int array [n, 3] of (t, i, j).  Returns (y [n, Cout] float64,
    s [n, Cout] float64) where s = sum of |w x| over the taps plus |bias| (the
    size of the terms the sum adds up, for error bars of a floating-point
    accumulation).  Only the input pixels these outputs read are widened to fp64.
    """
    x_bits = np.asarray(x_bits, np.uint16)
    T, H, W, _ = x_bits.shape
    w = bf16_to_f64(w_bits)
    pixels = np.asarray(pixels, np.int64).reshape(-1, 3)
    Cout = w.shape[0]

    def X(tau, ii, jj):
        """Input pixel vector at frame tau (tau < 0: history frame tau + 2)."""
        if tau < 0:
            if hist_bits is None:
                return None
            return bf16_to_f64(np.asarray(hist_bits, np.uint16)[tau + KT - 1, ii, jj])
        return bf16_to_f64(x_bits[tau, ii, jj])

    y = np.zeros((len(pixels), Cout))
    s = np.zeros((len(pixels), Cout))
    for n, (t, i, j) in enumerate(pixels):
        for dt in range(KT):
            for dy in range(KS):
                for dx in range(KS):
                    ii, jj = i + dy - 1, j + dx - 1
                    if not (0 <= ii < H and 0 <= jj < W):
                        continue
                    v = X(t + dt - (KT - 1), ii, jj)
                    if v is None:
                        continue
                    y[n] += w[:, dt, dy, dx, :] @ v
                    s[n] += np.abs(w[:, dt, dy, dx, :]) @ np.abs(v)
    if bias is not None:
        b = np.asarray(bias, np.float32).astype(np.float64)
        y += b
        s += np.abs(b)
    if resid_bits is not None:
        r = np.asarray(resid_bits, np.uint16)[pixels[:, 0], pixels[:, 1], pixels[:, 2]]
        y += bf16_to_f64(r)
    return y, s


def rms_norm_silu_f64(x_bits, gamma, eps=VAE_EPS):
    """Per pixel: y = x / sqrt(mean_c x^2 + eps) * gamma, then y * sigmoid(y) (fp64)."""
    x = bf16_to_f64(x_bits)
    g = np.asarray(gamma, np.float32).astype(np.float64)
    y = x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * g
    return y / (1.0 + np.exp(-y))


def rms_norm_silu(x_bits, gamma, eps=VAE_EPS):
    return f64_to_bf16(rms_norm_silu_f64(x_bits, gamma, eps))


def res_block(x_bits, wts, hist=None):
    """One residual block of the decode stage over one chunk.

    wts: dict of gamma1, gamma2 [C] fp32, w1, w2 [C, 3, 3, 3, C] bf16 bits,
    b1, b2 [C] fp32.  hist: None (start of the video) or the dict this function
    returned for the previous chunk.  Returns (out bf16 bits [T, H, W, C],
    intermediates, the history for the next chunk: the last two frames of each
    convolution's input).
    """
    h1 = rms_norm_silu(x_bits, wts["gamma1"])
    c1 = causal_conv3d(h1, None if hist is None else hist["h1"], wts["w1"], wts["b1"])
    h2 = rms_norm_silu(c1, wts["gamma2"])
    out = causal_conv3d(h2, None if hist is None else hist["h2"], wts["w2"], wts["b2"],
                        resid_bits=x_bits)
    nxt = {"h1": _last_two(h1, hist, "h1"), "h2": _last_two(h2, hist, "h2")}
    return out, dict(h1=h1, c1=c1, h2=h2), nxt


def _last_two(frames, hist, key):
    """The last two frames of a conv input, reaching into the history when the
    chunk is shorter than two frames."""
    if frames.shape[0] >= KT - 1:
        return frames[-(KT - 1):].copy()
    prev = np.zeros((KT - 1,) + frames.shape[1:], frames.dtype) if hist is None else hist[key]
    return np.concatenate([prev, frames], axis=0)[-(KT - 1):].copy()


def conv_flops(T, H, W, Cin, Cout):
    """Useful FLOPs of one causal 3x3x3 convolution (every tap, zeros included)."""
    return 2.0 * T * H * W * Cout * Cin * KT * KS * KS
