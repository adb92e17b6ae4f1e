"""Frequency tables for scaled-RoPE tests (test inputs; no attention arithmetic).

The pages derive each model's window table from its RoPE configuration,
rope_scaling included ("Porting to something else").  The scaled tables here
follow the frequency-scaling rule published with Llama 3.1 and used by the
Llama-3.2 family: wavelengths 2*pi/theta_r shorter than orig_ctx/high keep
their frequency, wavelengths longer than orig_ctx/low are divided by `factor`,
and the frequencies in between blend the two linearly in orig_ctx/wavelength.
"""
import numpy as np


def base_theta(D, base):
    return base ** (-2.0 * np.arange(D // 2, dtype=np.float64) / D)


def llama3_scaled_theta(D, base, factor=32.0, low=1.0, high=4.0, orig_ctx=8192.0):
    theta = base_theta(D, base)
    wavelen = 2.0 * np.pi / theta
    smooth = (orig_ctx / wavelen - low) / (high - low)
    blended = (1.0 - smooth) * theta / factor + smooth * theta
    return np.where(wavelen < orig_ctx / high, theta, np.where(wavelen > orig_ctx / low, theta / factor, blended))
