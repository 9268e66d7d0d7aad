"""The oracle's pins have teeth: each plausible mistake, planted in a temporary copy of the
oracle's source and compiled on the CPU, makes at least one pin fail.

The committed oracle is never modified; each variant lives in pytest's tmp_path.
"""
import pytest

from tests import test_oracle_langevin as lv_pins
from tests import test_oracle_md as md_pins
from tests import test_oracle_model as model_pins
from tests import test_oracle_neighbors as nb_pins

from schnet_gnn_molecular_cell_b200 import synth


def _closed_form(O):
    for d in (1.3, 2.71, 4.4):
        model_pins.test_closed_form_two_atoms(O, d)
    model_pins.test_message_direction_matters(O)


def _fd(O):
    for kind, seed in (("chain", 101), ("box", 103)):
        model_pins.test_forces_match_central_differences(O, kind, seed)


def _invariances(O):
    model_pins.test_invariances_open_chains(O)
    model_pins.test_periodic_translation_and_image_invariance(O)


def _readout(O):
    model_pins.test_T0_is_readout_of_embedding(O)


def _cutoff(O):
    model_pins.test_energy_continuous_at_cutoff(O)


def _neighbors(O):
    for case in nb_pins.CASES:
        nb_pins.test_brute_matches_numpy_all_pairs(O, *case)
        if case[1].periodic:
            nb_pins.test_cells_equal_brute(O, *case)
    nb_pins.test_strict_cutoff_and_exclusions(O)


def _md(O):
    md_pins.test_free_flight(O)
    md_pins.test_time_reversible(O)
    md_pins.test_energy_error_is_second_order(O)


def _langevin(O):
    for case in [([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8])]:
        lv_pins.test_philox_known_answers(O, *case)
    lv_pins.test_noise_is_standard_normal(O)
    lv_pins.test_zero_friction_is_velocity_verlet(O)
    lv_pins.test_free_particles_thermalise(O)


ALL = [_closed_form, _fd, _invariances, _readout, _cutoff, _neighbors, _md, _langevin]

# (name, original text, planted text)
MUTATIONS = [
    ("message_from_dst", "h[f] += xt[j * F + f] * sc.w[f];", "h[f] += xt[i * F + f] * sc.w[f];"),
    ("filter_bias_dropped", "linear(bw->W1, bw->b1, bt, a, m->F, m->K);", "linear(bw->W1, NULL, bt, a, m->F, m->K);"),
    ("W2_transposed", "linear(bw->W2, bw->b2, s, w, m->F, m->F);",
     "linear_t(bw->W2, s, w, m->F, m->F); for (int f = 0; f < m->F; ++f) w[f] += bw->b2[f];"),
    ("envelope_dropped", "bt[k] = phi * C;", "bt[k] = phi;"),
    ("centres_off_by_one", "double mu = (double)k * m->r_cut / (double)(m->K - 1);",
     "double mu = (double)k * m->r_cut / (double)(m->K);"),
    ("residual_dropped", "xn[i * F + f] = xt[i * F + f] + sc.tmp[F + f];", "xn[i * F + f] = sc.tmp[F + f];"),
    ("update_bias_dropped", "linear(bw->U2, bw->c2, sc.tmp, sc.tmp + F, F, F);",
     "linear(bw->U2, NULL, sc.tmp, sc.tmp + F, F, F);"),
    ("readout_sigma_dropped", "ob[k] = m.R2[k] * sigm(o[i * H + k]);", "ob[k] = m.R2[k];"),
    ("gaussian_derivative_sign", "double dphi = -2.0 * m->gamma * (d - mu) * phi;",
     "double dphi = 2.0 * m->gamma * (d - mu) * phi;"),
    ("envelope_derivative_dropped", "if (dbt) dbt[k] = dphi * C + phi * dC;", "if (dbt) dbt[k] = dphi * C;"),
    ("filter_sigma_dropped", "sc.abar[f] = sc.sbar[f] * sigm(sc.a[f]);", "sc.abar[f] = sc.sbar[f];"),
    ("backward_residual_dropped", "for (int f = 0; f < F; ++f) acc[f] = xbar[j * F + f];",
     "for (int f = 0; f < F; ++f) acc[f] = 0.0;"),
    ("wbar_uses_dst_features", "sc.wbar[f] = hbar[i * F + f] * xt[j * F + f];",
     "sc.wbar[f] = hbar[i * F + f] * xt[i * F + f];"),
    ("src_force_sign", "for (int a = 0; a < 3; ++a) g[a] -= dbar[e] * u[a] / d;",
     "for (int a = 0; a < 3; ++a) g[a] += dbar[e] * u[a] / d;"),
    ("min_image_sign", "dx = dx - shift;", "dx = dx + shift;"),
    ("cells_half_stencil", "for (int oz = -1; oz <= 1; ++oz)", "for (int oz = -1; oz <= 0; ++oz)"),
    ("cutoff_inclusive", "return r2 < rc2;", "return r2 <= rc2;"),
    ("full_kick", "const double c = 0.5 * dt * SNO_KAPPA / mass;\n    int st = SNO_OK;",
     "const double c = dt * SNO_KAPPA / mass;\n    int st = SNO_OK;"),
    ("philox_weyl_constant", "k1 += 0xBB67AE85u;", "k1 += 0xBB67AE84u;"),
    ("box_muller_sin_cos", "xi[1] = rad0 * sin(2.0 * SNO_PI * u[1]);", "xi[1] = rad0 * cos(2.0 * SNO_PI * u[1]);"),
    ("noise_same_for_all_atoms", "sno_langevin_noise(seed, step0 + s, i, xi);", "sno_langevin_noise(seed, step0 + s, 0, xi);"),
    ("ou_variance_without_sqrt", "const double b = sqrt((1.0 - a * a) * kB * temperature * SNO_KAPPA / mass);",
     "const double b = (1.0 - a * a) * kB * temperature * SNO_KAPPA / mass;"),
    ("drift_before_kick", "vel[q] += c * forces[q];\n            pos[q] += dt * vel[q];",
     "pos[q] += dt * vel[q];\n            vel[q] += c * forces[q];"),
]


@pytest.mark.parametrize("name,orig,planted", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(oracle, tmp_path, name, orig, planted):
    src = oracle.SRC.read_text()
    assert src.count(orig) == 1, f"mutation anchor for {name} not found exactly once"
    lib = oracle.compile_variant(src.replace(orig, planted), tmp_path / f"mut_{name}.so")
    failed = []
    with oracle.using(lib):
        for pin in ALL:
            try:
                pin(oracle)
            except (AssertionError, ValueError):
                failed.append(pin.__name__)
            except Exception as e:  # pytest.skip inside a pin counts as not catching
                if type(e).__name__ == "Skipped":
                    continue
                raise
    assert failed, f"planted mistake {name!r} passed every pin"
