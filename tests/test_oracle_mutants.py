"""Plant plausible mistakes in a copy of the oracle (CPU only) and check that
the pin suite notices every one of them. The oracle source itself is never
modified: each mutant is compiled from a temporary copy."""
import os

import pytest

import oracle
import oracle_pins as pins
from oracle import build as obuild

SRC = open(obuild.SRC).read()

MUTANTS = {
    "z_transposed": ("qbar[i * d + c] * kbar[j * d + c]", "qbar[j * d + c] * kbar[i * d + c]"),
    "z_scale_dropped": ("double z = scale * dot;", "double z = dot;"),
    "compressed_wrong_values": ("acc += w[j] * vbar[j * d + c]", "acc += w[j] * kbar[j * d + c]"),
    "compressed_not_normalised": ("o_cg[r * d + c] = acc / denom;", "o_cg[r * d + c] = acc;"),
    "ties_to_higher_index": ("return (a->j < b->j) ? -1 : (a->j > b->j);",
                             "return (a->j > b->j) ? -1 : (a->j < b->j);"),
    "topn_ascending": ("if (a->z > b->z) return -1;\n    if (a->z < b->z) return 1;",
                       "if (a->z < b->z) return -1;\n    if (a->z > b->z) return 1;"),
    "gap_wrong_ranks": ("sb[n - 1].z - sb[n].z", "sb[0].z - sb[n].z"),
    "pool_divides_by_d": ("xbar[j * d + c] = s / (double)block;", "xbar[j * d + c] = s / (double)d;"),
    "pool_skips_last_token": ("t < (j + 1) * block; ++t) s += x", "t < (j + 1) * block - 1; ++t) s += x"),
    "window_right_edge_dropped": ("int64_t hi = (i + w > m - 1) ? m - 1 : i + w;",
                                  "int64_t hi = (i + w > m - 1) ? m - 1 : i;"),
    "window_wraps_left": ("int64_t lo = (i - w < 0) ? 0 : i - w;", "int64_t lo = (i - w < 0) ? i : i - w;"),
    "fine_not_normalised": ("double p = scores[b * block + t] / denom;", "double p = scores[b * block + t];"),
    "fine_no_scale": ("double s = scale * dot;", "double s = dot;"),
    "selection_uses_row0": ("sel[t] = idx[i * n + t];", "sel[t] = idx[t];"),
    "gates_fg_l_swapped": ("g[1] * ofg[c] + g[2] * ol[c]", "g[2] * ofg[c] + g[1] * ol[c]"),
    "cg_term_dropped": ("g[0] * o_cg[i * d + c] + g[1]", "0.0 * o_cg[i * d + c] + g[1]"),
    "cg_wrong_block": ("g[0] * o_cg[i * d + c]", "g[0] * o_cg[(m - 1 - i) * d + c]"),
    # backward
    "bwd_fine_D_dropped": ("double ds = p[e] * (dp[e] - D);", "double ds = p[e] * dp[e];"),
    "bwd_dk_no_scale": ("dk[u * d + c] += scale * ds * qt[c];", "dk[u * d + c] += ds * qt[c];"),
    "bwd_dv_uses_dp": ("dv[u * d + c] += p[e] * dO[c];", "dv[u * d + c] += dp[e] * dO[c];"),
    "bwd_dq_uses_v": ("dq_t[c] += scale * ds * k[u * d + c];", "dq_t[c] += scale * ds * v[u * d + c];"),
    "bwd_compressed_D_dropped": ("double dz = a[j] * (da[j] - D);", "double dz = a[j] * da[j];"),
    "bwd_dkbar_uses_kbar": ("dkb_p[j * d + c] += scale * dz * qb[i * d + c];",
                            "dkb_p[j * d + c] += scale * dz * kb[i * d + c];"),
    "bwd_docg_wrong_gate": ("g += gates[t * 3] * dout[t * d + c];", "g += gates[t * 3 + 1] * dout[t * d + c];"),
    "bwd_local_gets_fg_gate": ("dO[c] = g[2] * dy[c];", "dO[c] = g[1] * dy[c];"),
    "bwd_pool_grad_not_divided": ("dk[t * d + c] += dkb[j * d + c] / (double)block;", "dk[t * d + c] += dkb[j * d + c];"),
    "bwd_dgates_fg_gets_l": ("dgates[t * 3 + 1] = s1;", "dgates[t * 3 + 1] = s2;"),
    "bwd_window_right_edge_dropped": ("int64_t lo = i - w, hi = i + w;", "int64_t lo = i - w, hi = i;"),
    "bwd_window_wraps_left": ("if (lo < 0) lo = 0;", "if (lo < 0) lo = i;"),
    "bwd_selection_uses_row0": ("sel[t] = (int64_t)idx[i * n + t];", "sel[t] = (int64_t)idx[t];"),
    # lat-lon -> HEALPix interpolation
    "hp_ring_off_by_one": ("int64_t ring = face_row[f] * nside - x - y - 1;", "int64_t ring = face_row[f] * nside - x - y;"),
    "hp_equatorial_z": ("*z = 4.0 / 3.0 - 2.0 * (double)ring / (3.0 * (double)nside);",
                        "*z = 1.0 - 2.0 * (double)ring / (3.0 * (double)nside);"),
    "hp_face_columns_shifted": ("static const int face_col[12] = {1, 3, 5, 7, 0, 2, 4, 6, 1, 3, 5, 7};",
                                "static const int face_col[12] = {1, 3, 5, 7, 1, 3, 5, 7, 1, 3, 5, 7};"),
    "hp_bits_not_interleaved": ("y |= ((ipf >> (2 * b + 1)) & 1) << b;", "y |= ((ipf >> (2 * b + 1)) & 1) << (b + 1);"),
    "plan_window_off_by_one": ("int64_t r = r0 + a, c = ((c0 - 1 + b) % nlon + nlon) % nlon;",
                               "int64_t r = r0 + a, c = ((c0 + 1 + b) % nlon + nlon) % nlon;"),
    "plan_rel_unscaled": ("rel[e * 3 + t] = (xj[t] - xi[t]) / h;", "rel[e * 3 + t] = (xj[t] - xi[t]);"),
    "interp_not_normalised": ("out[i * d + c] = acc / denom;", "out[i * d + c] = acc;"),
    "interp_values_are_keys": ("acc += s[j] * vsrc[(int64_t)nbr[i * K + j] * d + c];",
                               "acc += s[j] * ksrc[(int64_t)nbr[i * K + j] * d + c];"),
    "interp_query_column": ("double qc = wq[c * 3] * p[0] + wq[c * 3 + 1] * p[1] + wq[c * 3 + 2] * p[2];",
                            "double qc = wq[c * 3] * p[0] + wq[c * 3 + 1] * p[2] + wq[c * 3 + 2] * p[1];"),
    "bwd_softmax_not_normalised": ("for (int64_t e = 0; e < nk; ++e) p[e] /= denom;", "(void)denom;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation anchor for {name} not unique in the oracle source"
    src = tmp_path / "mutant.c"
    src.write_text(SRC.replace(old, new))
    lib = oracle.load(obuild.build(str(src), str(tmp_path / "libmutant.so"), force=True))
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, ValueError) as e:
            caught.append(f"{check.__name__}: {str(e)[:80]}")
    assert caught, f"no pin detects mutant {name}"


def test_unmutated_copy_passes(tmp_path):
    src = tmp_path / "copy.c"
    src.write_text(SRC)
    lib = oracle.load(obuild.build(str(src), str(tmp_path / "libcopy.so"), force=True))
    for check in pins.ALL_CHECKS:
        check(lib)
