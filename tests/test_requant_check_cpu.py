"""The SwiGLU-requantisation parity check (gpu_cases.requant_mismatches) on
the CPU, with the oracle standing in for both sides: it accepts differences
that a few-ulp change of h near a UE4M3 / E2M1 decision point causes, and it
flags every planted mistake (a misplaced code block, a wrong scale away from
a decision point, a code flipped by an error larger than the band)."""
import numpy as np

import oracle as O
import synthetic as S
from gpu_cases import E2M1_DECISION_POINTS, SWIGLU_BAND, requant_mismatches


def _case(R=32, I=256, seed=3):
    rng = np.random.default_rng(seed)
    y = S.f32_to_bf16_bits_np(rng.normal(0, 2, size=(R, 2 * I)).astype(np.float32))
    h = O.swiglu(y)
    g = np.float32(O.global_scale(float(np.abs(h).max())))
    return h, g


def _quant(h, g):
    return O.quantize_rows(h, g)        # codes [R, I/2], scales [R, I/32]


def _put_on_decisions(h, g, rng, n=200):
    """Moves n values of h onto an E2M1 decision point of their block's step
    (exactly representable cases are rounded to binary32), so that a tiny
    change of h flips their codes."""
    h = h.copy()
    R, I = h.shape
    _, sc = _quant(h, g)
    for _ in range(n):
        r, i = rng.integers(R), rng.integers(I)
        s_b = np.float32(O.ue4m3_value(int(sc[r, i // 32]))) / g
        tau = E2M1_DECISION_POINTS[rng.integers(len(E2M1_DECISION_POINTS))]
        v = np.float32(tau * s_b)
        if abs(v) < np.abs(h[r, (i // 32) * 32:(i // 32 + 1) * 32]).max():   # keep the block amax
            h[r, i] = v * np.float32(np.sign(h[r, i]) or 1.0)
    return h


def test_accepts_band_limited_changes_of_h():
    rng = np.random.default_rng(1)
    h, g = _case()
    h = _put_on_decisions(h, g, rng)
    oc, os_ = _quant(h, g)
    eps = rng.uniform(-2.0 ** -19, 2.0 ** -19, size=h.shape)
    h2 = (h.astype(np.float64) * (1 + eps)).astype(np.float32)
    gc, gs = _quant(h2, g)
    bad_s, bad_c, sd, cd = requant_mismatches(h, np.full(h.shape[0], g), os_, oc, gs, gc)
    assert cd.any()                      # the perturbation did flip codes
    assert not bad_s.any() and not bad_c.any()


def test_flags_a_misplaced_code_block():
    h, g = _case()
    oc, os_ = _quant(h, g)
    gc = oc.copy()
    gc[5, 0:16], gc[5, 16:32] = oc[5, 16:32], oc[5, 0:16]          # two 32-element blocks swapped
    bad_s, bad_c, _, _ = requant_mismatches(h, np.full(h.shape[0], g), os_, oc, os_, gc)
    assert bad_c.any()


def test_flags_a_wrong_scale_away_from_a_decision_point():
    h, g = _case()
    oc, os_ = _quant(h, g)
    gs = os_.copy()
    gs[7, 3] = (int(os_[7, 3]) + 1) & 0x7F
    bad_s, _, _, _ = requant_mismatches(h, np.full(h.shape[0], g), os_, oc, gs, oc)
    assert bad_s[7, 3]


def test_flags_a_code_flipped_by_an_error_beyond_the_band():
    rng = np.random.default_rng(2)
    h, g = _case()
    h = _put_on_decisions(h, g, rng)
    oc, os_ = _quant(h, g)
    h2 = (h.astype(np.float64) * (1 + 2.0 ** -14)).astype(np.float32)   # 4x the band
    # move the values that sit on a decision point just outside the band first
    h_ref = (h.astype(np.float64) * (1 - 2 * SWIGLU_BAND)).astype(np.float32)
    oc, os_ = _quant(h_ref, g)
    gc, gs = _quant(h2, g)
    keep = gs == os_
    bad_s, bad_c, sd, cd = requant_mismatches(h_ref, np.full(h.shape[0], g), os_, oc, np.where(keep, gs, os_), gc)
    assert bad_c.any()
