"""Seeded synthetic inputs shaped like the TurboQuant KV-cache workloads.

This module only draws random numbers: it holds none of the method's
arithmetic, and both the tests (for the CUDA library and for the CPU
oracle) and the benchmark take their inputs from it.

Recipes
-------
* ``single_head_fp32``: one head, d = 128, fp32 K and V drawn N(0,1), four
  outlier channels (a seeded permutation, the same for K and V) scaled x20,
  one N(0,1) query.
* ``lognormal_kv``: bf16 K or V of shape [batch, tokens, heads, d] with
  value z * exp(w[h, c]); z ~ N(0,1) per element, w ~ N(0,1) per
  (layer, K-or-V, head, channel): log-normal per-channel scales, sigma 1.
* ``queries``: N(0,1) queries [batch, heads, d] in the given dtype.
* ``ragged_lengths``: integer lengths uniform in [lo, hi].

CPU generation is bit-reproducible across machines (torch's CPU
generator); a CUDA generator gives the same distribution, faster, for
benchmark-sized tensors.
"""

import torch

_K, _V = 0, 1


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & ((1 << 63) - 1))
    return g


def _mix(*parts):
    h = 0x243F6A8885A308D3
    for p in parts:
        h = (h * 0x100000001B3 + (int(p) + 1) * 0x9E3779B97F4A7C15) & ((1 << 63) - 1)
    return h


def single_head_fp32(seed=0, tokens=4096, d=128, n_outliers=4, outlier_scale=20.0):
    """Return (k [tokens, d], v [tokens, d], q [d], outlier_channels) fp32 on CPU."""
    g = _gen("cpu", seed)
    k = torch.randn(tokens, d, generator=g, dtype=torch.float32)
    v = torch.randn(tokens, d, generator=g, dtype=torch.float32)
    q = torch.randn(d, generator=g, dtype=torch.float32)
    channels = torch.randperm(d, generator=_gen("cpu", seed))[:n_outliers]
    k[:, channels] *= outlier_scale
    v[:, channels] *= outlier_scale
    return k, v, q, channels


def channel_log_scales(heads, d, seed, layer, which, device="cpu"):
    """w[h, c] ~ N(0,1) for one (layer, K-or-V) pair, fp32."""
    g = _gen(device, _mix(seed, layer, which, 1))
    return torch.randn(heads, d, generator=g, dtype=torch.float32, device=device)


def lognormal_kv(batch, tokens, heads, d, seed, layer, which, device="cpu",
                 dtype=torch.bfloat16, token_offset_seed=0):
    """bf16 tensor [batch, tokens, heads, d] = z * exp(w[h, c]).

    ``which`` is 0 for K and 1 for V.  ``token_offset_seed`` selects an
    independent z stream (for example the token appended at a decode step)
    while keeping the per-channel scales of the layer.
    """
    w = channel_log_scales(heads, d, seed, layer, which, device)
    g = _gen(device, _mix(seed, layer, which, 2, token_offset_seed))
    z = torch.randn(batch, tokens, heads, d, generator=g, dtype=torch.float32, device=device)
    z.mul_(torch.exp(w))
    return z.to(dtype)


def queries(batch, heads, d, seed, layer=0, step=0, device="cpu", dtype=torch.bfloat16):
    """N(0,1) queries [batch, heads, d]."""
    g = _gen(device, _mix(seed, layer, 7, step))
    return torch.randn(batch, heads, d, generator=g, dtype=torch.float32, device=device).to(dtype)


def ragged_lengths(batch, lo, hi, seed):
    """Integer lengths uniform in [lo, hi] (inclusive), int32 CPU tensor."""
    g = _gen("cpu", _mix(seed, 11))
    return torch.randint(lo, hi + 1, (batch,), generator=g, dtype=torch.int32)


K, V = _K, _V
