"""Partial re-noise and the three-step Euler refinement (oracle side, FP64).

Page: "Open-H3-Regenerate-2K: High-Resolution Video Refinement with
Few-Step Diffusion" (agientry.com, English article).

* Section "Training: learn what degradation removed": the linear
  flow-matching path z_sigma = (1 - sigma) z0 + sigma eps with velocity
  target v = eps - z0.
* Section "Three steps instead of dozens": the enlarged latent is re-noised
  to sigma0 = 0.909 by z = (1 - sigma0) z_up + sigma0 eps, then three Euler
  updates z_{k+1} = z_k + (sigma_{k+1} - sigma_k) v follow the schedule
  0.909 -> 0.857 -> 0.667 -> 0.

Page "Open-H3-Regenerate-2K-IC" (wujieai.com), section
"三步接着放大的草稿画，八步从噪声重画": the IC variant starts from
sigma = 0.835 (up3) or 0.923 (up4) with the same blend, or from pure noise
(sigma = 1, hf8); all three routes share HyperFlow's eight-step noise table
with video shift 12; up3 then takes the last three steps of that table, up4
one step more, hf8 all eight; the reference row is blended with 0.1 % noise
(sigma = 0.001).

Reading of the table (the page names it but prints no formula): "video
shift 12" is the flow-matching time shift sigma = s t / (1 + (s - 1) t) on
the uniform grid t_k = 1 - k/8, k = 0..8.  At t = 1/2 it gives 12/13 =
0.923..., the printed up4 start.  A route starts at its printed sigma0 and
then visits every table point strictly below it, which yields three steps
for up3 (0.835 -> 0.8 -> 0.632 -> 0), four for up4 and eight for hf8, as the
page counts them.

Reading of the decimals (the pages print decimals only): each sigma is the
FP32 value nearest to the printed decimal, and both the kernels and this
oracle use exactly that binary value.  The oracle evaluates every blend in
FP64 from those exact inputs.
"""

import numpy as np

from oracle import lora

# Printed schedule, "Three steps instead of dozens".
SCHEDULE_DECIMAL = (0.909, 0.857, 0.667, 0.0)
# IC starts, "三步接着放大的草稿画，八步从噪声重画".
IC_STARTS_DECIMAL = (0.835, 0.923)
# Same section: the shared eight-step table, its video shift, the three
# routes' printed starts and the reference row's noise share.
HYPERFLOW_STEPS = 8
HYPERFLOW_SHIFT = 12.0
IC_ROUTES_DECIMAL = {"up3": 0.835, "up4": 0.923, "hf8": 1.0}
REFERENCE_ROW_SIGMA_DECIMAL = 0.001


def as_fp32(value):
    """The FP32 value nearest to a printed decimal, as an exact float64."""
    return float(np.float32(value))


SCHEDULE = tuple(as_fp32(s) for s in SCHEDULE_DECIMAL)
SIGMA0 = SCHEDULE[0]


def renoise(up, eps, sigma):
    """x = (1 - sigma) up + sigma eps, in FP64."""
    up = np.asarray(up, dtype=np.float64)
    eps = np.asarray(eps, dtype=np.float64)
    sigma = float(sigma)
    return (1.0 - sigma) * up + sigma * eps


def euler_step(x, v, sigma, sigma_next):
    """x + (sigma_next - sigma) v, in FP64."""
    x = np.asarray(x, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    return x + (float(sigma_next) - float(sigma)) * v


def projection_euler_step(x, W, A_cat, B_cat, z, frame_tokens, sigma, sigma_next):
    """The step's last projection followed by its Euler update (FP64).

    The projection v = lora.lora_linear(x, W, A_cat, B_cat) [M, C] gives each
    token its C velocity channels.  Token m is cell p = m mod T of frame
    f = m div T (T = frame_tokens, the H W cells of a frame); the latent z
    keeps the [F, C, H W] layout, so v[f T + p, c] is the velocity of
    z[f, c, p].  Returns euler_step(z, that velocity, sigma, sigma_next) with
    z's shape.  The pages fold nothing here; this is the plain composition of
    the layer ("The four-stage refinement pipeline") and the update ("Three
    steps instead of dozens").
    """
    v = lora.lora_linear(x, W, A_cat, B_cat)
    M, C = v.shape
    T = int(frame_tokens)
    v_latent = v.reshape(M // T, T, C).transpose(0, 2, 1)
    z = np.asarray(z, np.float64)
    return euler_step(z.reshape(M // T, C, T), v_latent, sigma, sigma_next).reshape(z.shape)


def flow_point(z0, eps, sigma):
    """The linear flow path z_sigma = (1 - sigma) z0 + sigma eps (FP64)."""
    return (1.0 - float(sigma)) * np.asarray(z0, np.float64) + float(sigma) * np.asarray(eps, np.float64)


def exact_velocity(z0, eps):
    """The flow-matching velocity target eps - z0 (FP64)."""
    return np.asarray(eps, np.float64) - np.asarray(z0, np.float64)


def refine(up, eps, schedule, velocity):
    """Re-noise at schedule[0], then one Euler step per schedule interval.

    velocity(z, k) returns the velocity used at step k.  Returns the list of
    iterates [z_0, z_1, ..., z_last].
    """
    z = renoise(up, eps, schedule[0])
    out = [z]
    for k in range(len(schedule) - 1):
        z = euler_step(z, velocity(z, k), schedule[k], schedule[k + 1])
        out.append(z)
    return out


def shifted_sigma(t, shift):
    """Time shift of the flow-matching grid: sigma = s t / (1 + (s - 1) t), FP64."""
    t = float(t)
    return shift * t / (1.0 + (shift - 1.0) * t)


def hyperflow_table(n_steps=HYPERFLOW_STEPS, shift=HYPERFLOW_SHIFT):
    """sigma at t_k = 1 - k / n_steps for k = 0..n_steps (FP64, from 1 down to 0)."""
    return [shifted_sigma(1.0 - k / n_steps, shift) for k in range(n_steps + 1)]


def ic_ladder(sigma0_decimal, n_steps=HYPERFLOW_STEPS, shift=HYPERFLOW_SHIFT):
    """The sigmas a route visits: its printed start, then every table point
    strictly below it; each the exact FP32 value (see as_fp32)."""
    start = as_fp32(sigma0_decimal)
    return [start] + [as_fp32(s) for s in hyperflow_table(n_steps, shift) if as_fp32(s) < start]
