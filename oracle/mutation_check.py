"""Mutation check of the oracle's pins (CPU only, run by hand; not a test).

Plants one plausible mistake at a time in a COPY of sage_oracle.c in a
temporary directory, builds that copy to a temporary shared library, and runs
tests/test_oracle_pins.py against it (SAGE_ORACLE_LIB points the oracle
package at the broken build).  The tracked source is never written.  Every
mistake listed must make at least one pin fail:

    python oracle/mutation_check.py [name ...]

Exit status 1 when some mistake goes uncaught.
"""
import os
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "sage_oracle.c")

# Eq. 6 radius replaced by the unweighted fit (p.c)/(c.c) of the chosen codeword
# before it reaches the grid and the codes.
_UNWEIGHTED = ("                idx[(size_t)o * S + j] = (uint16_t)oracle_assign(p8, omega + (size_t)j * SV, cb, K, &rs[t]);",
               "                idx[(size_t)o * S + j] = (uint16_t)oracle_assign(p8, omega + (size_t)j * SV, cb, K, &rs[t]);\n"
               "                { double nu = 0.0, de = 0.0; const int zz = idx[(size_t)o * S + j];\n"
               "                  for (int i = 0; i < SV; ++i) { nu += p8[i] * cb[zz * SV + i]; de += cb[zz * SV + i] * cb[zz * SV + i]; }\n"
               "                  rs[t] = de > 0.0 ? nu / de : 0.0; }")
# Eq. 2 evaluated against the grid before its fp16 rounding.
_UNROUNDED = ("            for (int t = 0; t < GROUP_SV; ++t)\n"
              "                q[(size_t)o * S + g * GROUP_SV + t] =\n"
              "                    (uint8_t)oracle_quantize(rs[t], mu[(size_t)o * G + g], delta[(size_t)o * G + g], V);",
              "            { double lo = rs[0], hi = rs[0];\n"
              "              for (int t = 1; t < GROUP_SV; ++t) { if (rs[t] < lo) lo = rs[t]; if (rs[t] > hi) hi = rs[t]; }\n"
              "              const double dd = (hi - lo) / (double)((1 << V) - 1);\n"
              "              for (int t = 0; t < GROUP_SV; ++t) {\n"
              "                double qq = dd > 0.0 ? floor((rs[t] - lo) / dd + 0.5) : 0.0;\n"
              "                if (qq < 0.0) qq = 0.0;\n"
              "                if (qq > (double)((1 << V) - 1)) qq = (double)((1 << V) - 1);\n"
              "                q[(size_t)o * S + g * GROUP_SV + t] = (uint8_t)qq; } }")

PLANTS = {
    "moe_combine_unweighted": ("                acc += w[(size_t)t * topk + k] * oracle_half_to_double(y[((size_t)t * topk + k) * d + c]);",
                               "                acc += oracle_half_to_double(y[((size_t)t * topk + k) * d + c]);"),
    "moe_combine_wrong_token": ("                acc += w[(size_t)t * topk + k] * oracle_half_to_double(y[((size_t)t * topk + k) * d + c]);",
                                "                acc += w[(size_t)t * topk + k] * oracle_half_to_double(y[((size_t)k * T + t) * d + c]);"),
    "dequant_sign_flip": ("const double sgn = ((s >> i) & 1) ? -1.0 : 1.0;", "const double sgn = ((s >> i) & 1) ? 1.0 : -1.0;"),
    "dequant_group_index": ("            const int g = j / GROUP_SV;", "            const int g = j / 8;"),
    "dequant_radius_no_q": ("const double r_hat = m + (double)q[(size_t)o * S + j] * d;", "const double r_hat = m + (double)q[(size_t)o * S + j] * d * 0.5;"),
    "gemv_bound_no_abs": ("                b += fabs(w32) * fabs(xp[p]);", "                b += w32 * xp[p];"),
    "gemv_fields_no_fp32_round": ("                const double w32 = (double)(float)W[p];", "                const double w32 = W[p];"),
    "assign_unsquared": ("        const double score = num * num / den;", "        const double score = num / den;"),
    "assign_radius_wrong": ("best_r = num / den; }", "best_r = num; }"),
    "grid_off_by_one": ("*delta16 = oracle_double_to_half((hi - lo) / (double)((1 << V) - 1));", "*delta16 = oracle_double_to_half((hi - lo) / (double)(1 << V));"),
    "quantize_truncate": ("    double qq = floor((r - mu) / d + 0.5);", "    double qq = floor((r - mu) / d);"),
    "quantize_no_clamp_top": ("    if (qq < 0.0) qq = 0.0;\n    if (qq > (double)((1 << V) - 1)) qq = (double)((1 << V) - 1);",
                              "    if (qq < 0.0) qq = 0.0;\n    if (qq > (double)((1 << V))) qq = (double)((1 << V));"),
    "omega_no_gamma": ("    for (int i = 0; i < SV; ++i) w8[i] = pow(e8[i], gamma) / mean;", "    for (int i = 0; i < SV; ++i) w8[i] = e8[i] / mean;"),
    "esg_ascending": ("    if (ea > eb) return -1;\n    if (ea < eb) return 1;", "    if (ea > eb) return 1;\n    if (ea < eb) return -1;"),
    "half_ties_away": ("    double s = nearbyint(ldexp(a, 10 - e));", "    double s = floor(ldexp(a, 10 - e) + 0.5);"),
    "kmeans_scalar_weight": ("            for (int i = 0; i < SV; ++i) acc[z[s] * SV + i] += Wt[(size_t)s * SV + i] * p[i] / nn;",
                             "            for (int i = 0; i < SV; ++i) acc[z[s] * SV + i] += Wt[(size_t)s * SV + 0] * p[i] / nn;"),
    "kmeans_empty_cluster_reset": ("            if (nn <= 0.0) continue;\n            nn = sqrt(nn);\n            for (int i = 0; i < SV; ++i) cb[k * SV + i] = acc[k * SV + i] / nn;",
                                   "            if (nn <= 0.0) { for (int i = 0; i < SV; ++i) cb[k * SV + i] = 0.0; continue; }\n            nn = sqrt(nn);\n            for (int i = 0; i < SV; ++i) cb[k * SV + i] = acc[k * SV + i] / nn;"),
    "pack_q_one_bit_low": ("            if (!isB) w |= (z << 7) | (qq << (23 - V));", "            if (!isB) w |= (z << 7) | (qq << (22 - V));"),
    "pack_aux_pair_swapped": ("            meta_plane[ai] |= (((s >> 6) & 1u) << tj) | (((s >> 7) & 1u) << (tj + 16));",
                              "            meta_plane[ai] |= (((s >> 7) & 1u) << tj) | (((s >> 6) & 1u) << (tj + 16));"),
    "rmsnorm_no_eps": ("        const double inv = 1.0 / sqrt(ss / (double)d + eps);", "        const double inv = 1.0 / sqrt(ss / (double)d);"),
    "rmsnorm_sum_not_mean": ("        const double inv = 1.0 / sqrt(ss / (double)d + eps);", "        const double inv = 1.0 / sqrt(ss + eps);"),
    "silu_sign": ("        out[i] = oracle_double_to_half(t / (1.0 + exp(-t)) * oracle_half_to_double(up[i]));",
                  "        out[i] = oracle_double_to_half(t / (1.0 + exp(t)) * oracle_half_to_double(up[i]));"),
    "attend_head_map": ("                out[((size_t)m * n_heads + h) * hd + e] = v[((size_t)m * n_kv + h / grp) * hd + e];",
                        "                out[((size_t)m * n_heads + h) * hd + e] = v[((size_t)m * n_kv + h % n_kv) * hd + e];"),
    "qdq_angle_no_eps": ("    return QDQ_EPS + (QDQ_HALF_PI - 2.0 * QDQ_EPS) / (1.0 + exp(-alpha));",
                         "    return QDQ_HALF_PI / (1.0 + exp(-alpha));"),
    "qdq_sine_product_off_by_one": ("            cb[(size_t)k * SV + i] = s * cos(t);\n            s *= sin(t);",
                                    "            s *= sin(t);\n            cb[(size_t)k * SV + i] = s * cos(t);"),
    "softplus_negative_branch": ("    return rho > 0.0 ? rho + log1p(exp(-rho)) : log1p(exp(rho));",
                                 "    return rho > 0.0 ? rho + log1p(exp(-rho)) : log1p(exp(-rho));"),
    "qdq_grid_step_2V": ("            const double delta = (hi - lo) / (double)((1 << V) - 1);",
                         "            const double delta = (hi - lo) / (double)(1 << V);"),
    "qdq_sign_component_reversed": ("                    W[(size_t)o * d_in + (size_t)j * SV + i] = (((s >> i) & 1) ? -rh : rh) * c[i];",
                                    "                    W[(size_t)o * d_in + (size_t)j * SV + i] = (((s >> (SV - 1 - i)) & 1) ? -rh : rh) * c[i];"),
    "abs_perm_direction": ("            const int c = perm ? perm[p] : p;\n            const double w = W[(size_t)o * d_in + c], d = w - Wh[(size_t)o * d_in + p];",
                           "            const int c = perm ? perm[p] : p;\n            const double w = W[(size_t)o * d_in + p], d = w - Wh[(size_t)o * d_in + p];"),
    "abs_energy_storage_order": ("            num += energy[c] * d * d;", "            num += energy[p] * d * d;"),
    "abs_denominator_unweighted": ("            den += energy[c] * w * w;", "            den += w * w;"),
    "encode_grid_unweighted_radius": _UNWEIGHTED,
    "encode_quantize_unrounded_grid": _UNROUNDED,
}


def run(name: str, tmp: str) -> bool:
    """True when the planted mistake makes at least one pin fail."""
    a, b = PLANTS[name]
    src = open(SRC).read()
    assert src.count(a) == 1, (name, src.count(a))
    c = os.path.join(tmp, f"{name}.c")
    so = os.path.join(tmp, f"{name}.so")
    with open(c, "w") as fh:
        fh.write(src.replace(a, b))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
                           "-o", so, c, "-lm"])
    env = dict(os.environ, SAGE_ORACLE_LIB=so)
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-q",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    failed = [ln.split("::")[1][:60] for ln in r.stdout.splitlines() if ln.startswith("FAILED")]
    print(f"{name:32s} rc={r.returncode} caught by {failed}")
    return r.returncode != 0


def main(argv):
    names = argv or list(PLANTS)
    with tempfile.TemporaryDirectory() as tmp:
        missed = [n for n in names if not run(n, tmp)]
    if missed:
        print("uncaught:", missed)
    return 1 if missed else 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
