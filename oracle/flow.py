"""Flow-matching x0 conversion and renoise, fp64 (oracle; test infrastructure only).

[P2] §2 (4 步采样): each step predicts the flow ``flow_pred`` with one forward,
converts it to the clean latent in closed form, ``x0 = xt - sigma_t * flow_pred``,
and, unless it is the last step, re-noises x0 to the next (smaller) timestep; the
last step outputs x0. [P2] §精度: the flow->x0 conversion runs in double.
Re-noising follows the flow-matching interpolation xt = (1 - sigma) x0 + sigma eps
(the same convention that makes x0 = xt - sigma * (eps - x0)).

The sigma schedule is sigma = t / 1000 for the distilled timesteps
``denoising_step_list: [1000, 750, 500, 250]`` ([P4] §机制二 and §关键参数速查表).

Operation order (no fused multiply-add; numpy does not contract):
    x0  = xt - (sigma * v)
    xt' = ((1 - sigma') * x0) + (sigma' * eps)
    v   = u + (scale * (c - u))          (guided prediction, when CFG is used)
x0 used for renoising is the fp64 value, not its bf16 rounding.
"""
from __future__ import annotations

import numpy as np

from . import bf16

DENOISING_STEP_LIST = (1000, 750, 500, 250)


def sigmas(step_list=DENOISING_STEP_LIST):
    return [t / 1000.0 for t in step_list]


def x0_renoise_f64(xt, v, eps, sigma: float, sigma_next: float):
    """fp64 core. sigma_next < 0 marks the last step (returns (x0, None))."""
    xt = np.asarray(xt, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    x0 = xt - sigma * v
    if sigma_next < 0:
        return x0, None
    eps = np.asarray(eps, dtype=np.float64)
    return x0, (1.0 - sigma_next) * x0 + sigma_next * eps


def cfg_combine_f64(v_cond, v_uncond, scale: float):
    """Classifier-free guidance: v = v_uncond + scale * (v_cond - v_uncond), fp64, no FMA.

    The causal pre-training mode runs 40 steps with CFG scale 5.0, i.e. two DiT forwards per
    step, one per KV cache ([P2] §为什么需要: "40 步 ... scale5.0 ... 40 × 2 = 80 次";
    [P3] §两种推理模式: cond / uncond each keep their own KV cache)."""
    c = np.asarray(v_cond, dtype=np.float64)
    u = np.asarray(v_uncond, dtype=np.float64)
    return u + scale * (c - u)


def cfg_x0_renoise_bf16(xt_bits, vc_bits, vu_bits, eps_bits, scale: float, sigma: float, sigma_next: float):
    """Guided flow prediction, then the x0 / renoise step; bf16 in / out, fp64 arithmetic."""
    v = cfg_combine_f64(bf16.to_f64(vc_bits), bf16.to_f64(vu_bits), scale)
    x0, xn = x0_renoise_f64(bf16.to_f64(xt_bits), v, None if sigma_next < 0 else bf16.to_f64(eps_bits),
                            sigma, sigma_next)
    return bf16.from_f64(x0), (None if xn is None else bf16.from_f64(xn))


def x0_renoise_bf16(xt_bits, v_bits, eps_bits, sigma: float, sigma_next: float):
    """bf16 in, bf16 out (uint16 bit patterns); fp64 arithmetic, RNE on output."""
    x0, xn = x0_renoise_f64(bf16.to_f64(xt_bits), bf16.to_f64(v_bits),
                            None if sigma_next < 0 else bf16.to_f64(eps_bits), sigma, sigma_next)
    return bf16.from_f64(x0), (None if xn is None else bf16.from_f64(xn))
