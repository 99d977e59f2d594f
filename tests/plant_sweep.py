"""Mutation check of the oracle's pins (CPU only; not collected by pytest).

Plants one plausible mistake at a time in oracle/sage_oracle.c, runs the
oracle pin tests, and reports which tests catch it; the original source is
restored afterwards (also on interruption).  Every mistake listed must be
caught by at least one pin:

    python tests/plant_sweep.py [name ...]
"""
import os
import subprocess, shutil, sys
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sage_oracle.c")
BACKUP = SRC + ".orig"
shutil.copy(SRC, BACKUP)
PLANTS = {
    "dequant_sign_flip": ("const double sgn = ((s >> i) & 1) ? -1.0 : 1.0;", "const double sgn = ((s >> i) & 1) ? 1.0 : -1.0;"),
    "dequant_group_index": ("            const int g = j / GROUP_SV;", "            const int g = j / 8;"),
    "dequant_radius_no_q": ("const double r_hat = m + (double)q[(size_t)o * S + j] * d;", "const double r_hat = m + (double)q[(size_t)o * S + j] * d * 0.5;"),
    "gemv_bound_no_abs": ("                b += fabs(w32) * fabs(xp[p]);", "                b += w32 * xp[p];"),
    "gemv_fields_no_fp32_round": ("                const double w32 = (double)(float)W[p];", "                const double w32 = W[p];"),
    "assign_unsquared": ("        const double score = num * num / den;", "        const double score = num / den;"),
    "assign_radius_wrong": ("best_r = num / den; }", "best_r = num; }"),
    "grid_off_by_one": ("*delta16 = oracle_double_to_half((hi - lo) / (double)((1 << V) - 1));", "*delta16 = oracle_double_to_half((hi - lo) / (double)(1 << V));"),
    "quantize_truncate": ("    double qq = floor((r - mu) / d + 0.5);", "    double qq = floor((r - mu) / d);"),
    "quantize_no_clamp_top": ("    if (qq > (double)((1 << V) - 1)) qq = (double)((1 << V) - 1);", "    if (qq > (double)((1 << V))) qq = (double)((1 << V));"),
    "omega_no_gamma": ("    for (int i = 0; i < SV; ++i) w8[i] = pow(e8[i], gamma) / mean;", "    for (int i = 0; i < SV; ++i) w8[i] = e8[i] / mean;"),
    "esg_ascending": ("    if (ea > eb) return -1;\n    if (ea < eb) return 1;", "    if (ea > eb) return 1;\n    if (ea < eb) return -1;"),
    "half_ties_away": ("    double s = nearbyint(ldexp(a, 10 - e));", "    double s = floor(ldexp(a, 10 - e) + 0.5);"),
    "kmeans_scalar_weight": ("            for (int i = 0; i < SV; ++i) acc[z[s] * SV + i] += Wt[(size_t)s * SV + i] * p[i] / nn;",
                             "            for (int i = 0; i < SV; ++i) acc[z[s] * SV + i] += Wt[(size_t)s * SV + 0] * p[i] / nn;"),
    "kmeans_empty_cluster_reset": ("            if (nn <= 0.0) continue;\n            nn = sqrt(nn);\n            for (int i = 0; i < SV; ++i) cb[k * SV + i] = acc[k * SV + i] / nn;",
                                   "            if (nn <= 0.0) { for (int i = 0; i < SV; ++i) cb[k * SV + i] = 0.0; continue; }\n            nn = sqrt(nn);\n            for (int i = 0; i < SV; ++i) cb[k * SV + i] = acc[k * SV + i] / nn;"),
}
names = sys.argv[1:] or list(PLANTS)
uncaught = set()
try:
    for name in names:
        a, b = PLANTS[name]
        s = open(BACKUP).read()
        assert s.count(a) == 1, (name, s.count(a))
        open(SRC, "w").write(s.replace(a, b))
        r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-q",
                            "-p", "no:cacheprovider"], cwd=ROOT,
                           capture_output=True, text=True, timeout=900)
        last = [l for l in r.stdout.splitlines() if l.strip()][-1]
        failed = [l for l in r.stdout.splitlines() if l.startswith("FAILED")]
        if r.returncode == 0:
            uncaught.add(name)
        print(f"{name:28s} rc={r.returncode} {last[:40]} {[f.split('::')[1][:45] for f in failed]}")
finally:
    shutil.copy(BACKUP, SRC)
    os.remove(BACKUP)
missed = [n for n in names if n in uncaught]
sys.exit(1 if missed else 0)
