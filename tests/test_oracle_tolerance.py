"""Pins of the layer tolerance (oracle.layer.e2e_error_bound and its stages).

The MoE parity tests gate on e2e_error_bound: the bound on a route's output change when
each projection is off by at most eps * (|W| . |input|) elementwise (the projection
criterion |y - y_ref| <= 1e-3 * (|W| . |x'|)).  These tests pin it against the mathematics
rather than against itself:

  * soundness: perturbations inside the allowed box (random ones, and ones whose signs are
    chosen adversarially for one output) are pushed through the exact layer arithmetic
    (silu, the rotation, the matrix products); the change never exceeds the bound;
  * attainment: at each stage a perturbation exists that reaches the stage's bound (the
    SwiGLU remainder to first order, the rotation exactly, the down contraction exactly),
    and on a layer built so that every inequality of the chain is tight the end-to-end
    change reaches >= 0.9 of the bound;
  * planted mistakes (a rotation bound summed over the whole row instead of the 128-chunk,
    a SiLU term with silu in place of silu', a missing rotation factor) make one of the
    checks above fail.
"""
import numpy as np
import pytest

from oracle import layer as OL
from trellis_quantized_moe_gemv_b200 import inputs

H = OL.hadamard_matrix()


def perturbed_route(stage_in, a_g, a_u, c_y, signs=None):
    """Exact layer arithmetic of one route with the raw gate/up outputs off by a_g, a_u and
    the raw down output off by c_y (same shapes as the raw projections)."""
    two = signs is not None
    g_raw, u_raw = stage_in["g_raw"] + a_g, stage_in["u_raw"] + a_u
    g = OL.rotate_out(g_raw, signs["gu"] if two else None)
    u = OL.rotate_out(u_raw, signs["gu"] if two else None)
    h = OL.silu(g) * u
    h_rot = OL.rotate_in(h, signs["h"] if two else None)
    y_raw = OL.project(stage_in["Wd"], h_rot) + c_y
    y = OL.rotate_out(y_raw, signs["y"] if two else None)
    return y, h_rot


def route_stage(layer, e, x_rot):
    weights = OL.ExpertWeights(layer)
    signs = layer.signs
    st = OL.expert_forward(weights, e, x_rot, signs=signs)
    st["g_raw"] = OL.project(weights.matrix(e, "gate"), x_rot)
    st["u_raw"] = OL.project(weights.matrix(e, "up"), x_rot)
    return st


def budget_draws(rng, st, eps, target_row=None, n_random=6):
    """Perturbations of the raw projections inside the budget: random signs, and (for a
    target output row) signs aligned with the first-order sensitivity of that row."""
    dg = eps * st["bound_g"]
    du = eps * st["bound_u"]
    draws = []
    for _ in range(n_random):
        draws.append((dg * rng.choice([-1.0, 1.0], dg.shape), du * rng.choice([-1.0, 1.0], du.shape)))
    if target_row is not None and not st["two_sided"]:
        # d y_i / d h_m = sum_j Wd[i, j] R[j, m] (R the blockwise orthonormal rotation)
        Wd = st["Wd"]
        sens_h = OL.rotate(Wd[target_row:target_row + 1])[0]   # R is symmetric
        sg = np.sign(sens_h * OL.silu_prime(st["g"][0]) * st["u"][0])
        su = np.sign(sens_h * OL.silu(st["g"][0]))
        draws.append((dg * sg, du * su))
        draws.append((-dg * sg, -du * su))
    return draws


@pytest.mark.parametrize("two_sided", [False, True])
@pytest.mark.parametrize("scale", [1.0, 30.0])
def test_e2e_bound_holds_for_perturbations_inside_the_budget(two_sided, scale):
    layer = inputs.small_layer(4101, E=3, D=256, F=256, split={2: 1, 3: 1, 4: 1})
    if two_sided:
        inputs.with_signs(layer, 4102)
    rng = np.random.default_rng(4103)
    eps = 1e-3
    for e in range(3):
        x = rng.standard_normal((1, 256)) * scale
        x_rot = OL.rotate_in(x, layer.signs["x"] if two_sided else None)
        st = route_stage(layer, e, x_rot)
        bound = OL.e2e_error_bound(st, eps, np.ones(1))[0]
        Wd_abs_hrot = np.abs(st["Wd"])
        for target in (None, 0, 17):
            for a_g, a_u in budget_draws(rng, st, eps, target):
                # the down projection's budget on its (perturbed) input, with both signs
                _, h_rot_p = perturbed_route(st, a_g, a_u, 0.0, layer.signs)
                c_budget = eps * (np.abs(h_rot_p) @ Wd_abs_hrot.T)
                for c_sign in (1.0, -1.0):
                    y, _ = perturbed_route(st, a_g, a_u, c_sign * c_budget, layer.signs)
                    err = np.abs(y - st["y"])[0]
                    assert np.all(err <= bound * (1 + 1e-9)), (e, target, (err / bound).max())


def test_e2e_bound_is_attained_on_a_tight_chain():
    """A route built so that every inequality of the chain is tight: gate/up budgets only
    at intermediate channel m0 (chunk 0), a second budget at m1 in chunk 1 that row i of
    the down projection never reads, and row i of W_d equal to row m0 of H_128 on chunk 0.
    Sign-aligned perturbations then change y_i by >= 0.9 of the bound."""
    F, D, eps = 256, 4, 1e-3
    m0, m1, i = 5, 128 + 9, 0
    g = np.zeros((1, F)); u = np.zeros((1, F))
    g[0, m0], u[0, m0] = 0.7, 1.3
    g[0, m1], u[0, m1] = -0.4, 2.0
    bound_g = np.zeros((1, F)); bound_u = np.zeros((1, F))
    bound_g[0, [m0, m1]] = 3.0
    bound_u[0, [m0, m1]] = 2.5
    Wd = np.zeros((D, F))
    Wd[i, :128] = 0.02 * H[m0]
    Wd[1:, :] = 0.01
    h_rot = OL.rotate(OL.silu(g) * u)
    stage = dict(g=g, u=u, bound_g=bound_g, bound_u=bound_u, bound_y=np.abs(h_rot) @ np.abs(Wd).T,
                 Wd=Wd, two_sided=False, down_rows=None)
    bound = OL.e2e_error_bound(stage, eps, np.ones(1))[0]
    st_in = dict(g_raw=g, u_raw=u, Wd=Wd)
    y_ref, _ = perturbed_route(st_in, 0.0, 0.0, 0.0)
    dg, du = eps * bound_g, eps * bound_u
    sens = OL.rotate(Wd[i:i + 1])[0]
    a_g = dg * np.sign(sens * OL.silu_prime(g[0]) * u[0])
    a_u = du * np.sign(sens * OL.silu(g[0]))
    y0, h_rot_p = perturbed_route(st_in, a_g, a_u, 0.0)
    # the down budget on the perturbed input, in the direction of the change so far
    c = eps * (np.abs(h_rot_p) @ np.abs(Wd).T) * np.sign(y0 - y_ref)
    y_p, _ = perturbed_route(st_in, a_g, a_u, c)
    ratio = abs(y_p[0, i] - y_ref[0, i]) / bound[i]
    assert ratio <= 1 + 1e-9
    assert ratio >= 0.9, ratio


def test_swiglu_bound_holds_on_a_grid_and_is_attained_to_first_order():
    rng = np.random.default_rng(4201)
    # g around 0 (largest |silu''|), 2.4 (largest silu'), negative and large values
    g = np.concatenate([np.linspace(-8, 8, 161), [0.0, 2.3994, -1.2785], rng.normal(0, 3, 40)])
    u = rng.normal(0, 2, g.size)
    for rel in (1e-4, 1e-2, 0.3):
        dg = rel * (1 + np.abs(g))
        du = rel * (1 + np.abs(u))
        bound = OL.swiglu_error_bound(g, u, dg, du)
        worst = np.zeros_like(g)
        for a in np.linspace(-1, 1, 21):
            for b in np.linspace(-1, 1, 21):
                ch = np.abs(OL.silu(g + a * dg) * (u + b * du) - OL.silu(g) * u)
                worst = np.maximum(worst, ch)
        assert np.all(worst <= bound * (1 + 1e-12)), (rel, (worst / bound).max())
        if rel == 1e-4:
            # the grid's corners reach the first-order part of the bound, and what the bound
            # adds beyond it is second order
            first = np.abs(OL.silu_prime(g)) * dg * np.abs(u) + np.abs(OL.silu(g)) * du
            assert np.all(worst >= 0.999 * first), (worst / first).min()
            # where the first-order part dominates the second-order scale, the bound is
            # no looser than the grid's worst change
            dom = first >= 100.0 * (dg * dg + dg * du) * (1 + np.abs(u))
            assert dom.sum() > 100
            assert np.all(bound[dom] <= 1.02 * worst[dom]), (bound[dom] / worst[dom]).max()


def test_rotation_bound_holds_and_is_attained_at_every_index():
    rng = np.random.default_rng(4301)
    v = np.abs(rng.normal(size=(1, 384)))
    bound = OL.rot_abs_bound(v)[0]
    for _ in range(20):
        d = v * rng.choice([-1.0, 1.0], v.shape)
        assert np.all(np.abs(OL.rotate(d))[0] <= bound * (1 + 1e-12))
    for j in (0, 1, 77, 127, 128, 200, 383):
        c = j // 128
        d = np.zeros_like(v)
        d[0, 128 * c:128 * c + 128] = v[0, 128 * c:128 * c + 128] * H[j % 128]
        assert abs(abs(OL.rotate(d)[0, j]) - bound[j]) <= 1e-12 * bound[j]


# ------------------------------------------------------------------ planted mistakes

def _whole_row_rot_abs(v):
    v = np.asarray(v, dtype=np.float64)
    return np.repeat(v.sum(-1, keepdims=True), v.shape[-1], axis=-1) / np.sqrt(128.0)


def _silu_in_place_of_silu_prime(g, u, dg, du):
    g, u = np.asarray(g, dtype=np.float64), np.asarray(u, dtype=np.float64)
    return (np.abs(OL.silu(g)) * dg + 0.25 * dg * dg) * (np.abs(u) + du) + np.abs(OL.silu(g)) * du


_ROT_ABS_BOUND = OL.rot_abs_bound


def _rot_abs_over_128(v):
    return _ROT_ABS_BOUND(v) / np.sqrt(128.0)


def _fails(test, *args):
    try:
        test(*args)
    except AssertionError:
        return True
    return False


def test_planted_whole_row_rotation_bound_is_caught(monkeypatch):
    monkeypatch.setattr(OL, "rot_abs_bound", _whole_row_rot_abs)
    assert _fails(test_e2e_bound_is_attained_on_a_tight_chain)
    assert _fails(test_rotation_bound_holds_and_is_attained_at_every_index)


def test_planted_silu_term_is_caught(monkeypatch):
    monkeypatch.setattr(OL, "swiglu_error_bound", _silu_in_place_of_silu_prime)
    assert _fails(test_swiglu_bound_holds_on_a_grid_and_is_attained_to_first_order)
    assert _fails(test_e2e_bound_is_attained_on_a_tight_chain)


def test_planted_missing_rotation_factor_is_caught(monkeypatch):
    monkeypatch.setattr(OL, "rot_abs_bound", _rot_abs_over_128)
    assert _fails(test_rotation_bound_holds_and_is_attained_at_every_index)
    assert _fails(test_e2e_bound_is_attained_on_a_tight_chain)
