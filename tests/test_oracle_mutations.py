"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a private copy of the oracle's C source (on
the CPU, in a temporary directory), loads it in place of the real oracle and
checks that at least one pin fails.  The real oracle is restored afterwards.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

MUTATIONS = {
    "drop last segment": ("for (int64_t q = 0; q + 1 < m; ++q)", "for (int64_t q = 0; q + 2 < m; ++q)"),
    "column offset sign": ("p[k] = dc[k] + cc * du[k] + rr * dv[k];", "p[k] = dc[k] - cc * du[k] + rr * dv[k];"),
    "row offset sign": ("p[k] = dc[k] + cc * du[k] + rr * dv[k];", "p[k] = dc[k] + cc * du[k] - rr * dv[k];"),
    "voxel index x<->z": ("int64_t flat = (idx[2] * g->n[1] + idx[1]) * g->n[0] + idx[0];",
                          "int64_t flat = (idx[0] * g->n[1] + idx[1]) * g->n[2] + idx[2];"),
    "weight in t units": ("emit(ctx, flat, (ts[q + 1] - ts[q]) * len);", "emit(ctx, flat, (ts[q + 1] - ts[q]));"),
    "isotropic pitch": ("double x = (a[k] + tm * d[k] - g->origin[k]) / g->spacing[k];",
                        "double x = (a[k] + tm * d[k] - g->origin[k]) / g->spacing[0];"),
    "segment start not midpoint": ("double tm = 0.5 * (ts[q] + ts[q + 1]);", "double tm = ts[q];"),
    "cylinder angle unscaled": ("double gam = cc * nu / R;", "double gam = cc * nu;"),
    "cylinder axial dropped": ("p[k] = s[k] + axial * vhat[k] + R *", "p[k] = s[k] + R *"),
    "back sinogram transposed": (
        "back_ctx b = {vol, (double)sino[((v - v0) * g->n_rows + r) * g->n_cols + c], power};",
        "back_ctx b = {vol, (double)sino[((v - v0) * g->n_cols + c) * g->n_rows + r], power};"),
    "clip ignores far face": ("if (tmax < t_out) t_out = tmax;", "(void)tmax;"),
    "last interior plane dropped": ("for (int64_t q = 0; q <= g->n[k]; ++q)", "for (int64_t q = 0; q <= g->n[k] - 2; ++q)"),
    "cone segment taken as a line": ("double t_in = 0.0, t_out = 1.0;", "double t_in = -1e30, t_out = 1e30;"),
    "power 2 ignored": ("b->power == 1 ? w : w * w", "b->power == 1 ? w : w"),
    "cylinder columns reversed": ("R * (cos(gam) * what[k] + sin(gam) * uhat[k])", "R * (cos(gam) * what[k] - sin(gam) * uhat[k])"),
}

PIN_TESTS = [
    lambda: pins.test_flat_pixel_centres_are_affine_in_row_and_column(),
    lambda: pins.test_cylindrical_pixel_centres_lie_on_the_source_centred_cylinder(),
    lambda: pins.test_uniform_box_central_chord(0.3),
    lambda: pins.test_uniform_box_offset_chords_against_rectangle_geometry(),
    lambda: pins.test_textbook_reduction_axis_aligned_views(),
    lambda: pins.test_single_voxel_chord_matches_brute_force(),
    lambda: pins.test_random_volume_matches_brute_force("helical_cyl"),
    lambda: pins.test_dense_transpose_8cubed_every_geometry_kind(),
    lambda: pins.test_cone_segment_ends_at_an_endpoint_inside_the_box(),
    lambda: pins.test_back_coefficient_powers(),
]


def _load_mutant(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "siddon_oracle.c")).read()
    assert src.count(old) >= 1, name
    mutated = src.replace(old, new)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "mutant.so"
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-fPIC", "-shared", "-o", str(so_path), str(c_path), "-lm"])
    return so_path


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    so_path = _load_mutant(tmp_path, name, old, new)
    real = oracle._load()
    mutant = ctypes.CDLL(str(so_path))
    for fn in ("oracle_pixel_centre", "oracle_ray_endpoints", "oracle_forward", "oracle_forward_rays",
               "oracle_back", "oracle_ray_segments", "oracle_count_updates"):
        getattr(mutant, fn).argtypes = getattr(real, fn).argtypes
        getattr(mutant, fn).restype = getattr(real, fn).restype
    oracle._lib = mutant
    try:
        failed = 0
        for t in PIN_TESTS:
            try:
                t()
            except AssertionError:
                failed += 1
        assert failed > 0, f"no pin caught mutation '{name}'"
    finally:
        oracle._lib = real
