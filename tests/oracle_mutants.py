"""Planted-mistake check of the oracle pins (run by hand, not collected by
pytest: about ten minutes).  Each entry below makes one plausible mistake in a
copy of oracle/ (a dropped term, a wrong sign, index or operand, a changed tie
rule or rounding); the CPU pins (test_oracle_pins.py, test_hva_oracle_pins.py)
must fail on every one.  Exit status 1 if any mistake goes unnoticed.

    python tests/oracle_mutants.py [name ...]
"""
import os
import shutil
import subprocess
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
P, H = "oracle/park_oracle.py", "oracle/hva_oracle.py"

MUTS = [
    ("metric_n1", P, "return (Q.T @ Q) / Q.shape[0]", "return (Q.T @ Q) / (Q.shape[0] - 1)"),
    ("init_offset", P, "[(np.arange(K) * N) // K]", "[(np.arange(K) * N + N // (2 * K)) // K]"),
    ("dist_l1", P, "np.sum(diff * diff, axis=2)", "np.sum(np.abs(diff), axis=2)"),
    ("metric_transpose", P, "        X = X @ F\n        C = C @ F\n    X = np.ascontiguousarray(X)",
     "        X = X @ F.T\n        C = C @ F.T\n    X = np.ascontiguousarray(X)"),
    ("query_factor_T", P, "self.F = R.T / math.sqrt(Q.shape[0])", "self.F = R / math.sqrt(Q.shape[0])"),
    ("assign_c_l1", "oracle/assign.c", "                s[0] = s[0] + d0 * d0;", "                s[0] = s[0] + (d0 < 0 ? -d0 : d0);"),
    ("tie_last", "oracle/assign.c", "if (arg < 0 || s[u] < best) { /* strict", "if (arg < 0 || s[u] <= best) { /* strict"),
    ("mean_double_round", P, "return round_to(sums / float(n), dtype)",
     "return round_to(np.float64(np.float32(sums / float(n))), dtype)"),
    ("empty_zero", P, "        if n:\n            C[k] = exact_mean(X[order[start:start + n]], dtype)",
     "        C[k] = exact_mean(X[order[start:start + n]], dtype) if n else 0.0"),
    ("iters_minus1", P, "    for _ in range(iters):\n        hist.append(C.copy())\n        labels = assign(X, C, M)",
     "    for _ in range(max(1, iters - 1)):\n        hist.append(C.copy())\n        labels = assign(X, C, M)"),
    ("perm_unstable", P, "    for i, a in enumerate(labels.tolist()):\n        perm[cursor[a]] = i",
     "    for i, a in reversed(list(enumerate(labels.tolist()))):\n        perm[cursor[a]] = i"),
    ("pama_all_clusters", P, "    live = np.nonzero(np.asarray(k_counts) > 0)[0]\n    NK = CK.shape[0]",
     "    live = np.arange(len(k_counts))\n    NK = CK.shape[0]"),
    ("pama_no_scale", P, "Z = scale * (Q[i0:i0 + row_block] @ CK[live].T) + prior", "Z = (Q[i0:i0 + row_block] @ CK[live].T) + prior"),
    ("pama_sum_not_mean", P, "sums[nz] / q_counts[nz, None]", "sums[nz]"),
    ("pama_no_norm", P, "        P /= P.sum(axis=1, keepdims=True)\n        np.add.at", "        np.add.at"),
    ("topp_strict", P, "            if acc >= p:\n                break", "            if acc > p:\n                break"),
    ("topp_drop_crossing", P, "            mask[r, m] = True\n            acc += I[r, m]\n            if acc >= p:\n                break",
     "            acc += I[r, m]\n            if acc >= p:\n                break\n            mask[r, m] = True"),
    ("topp_tie_high", P, "        order = sorted(live, key=lambda m: (-I[r, m], m))\n        acc = 0.0",
     "        order = sorted(live, key=lambda m: (-I[r, m], -m))\n        acc = 0.0"),
    ("topk_floor", P, "k = max(1, int(math.ceil(rho * len(live))))", "k = max(1, int(math.floor(rho * len(live))))"),
    ("sip_c", P, "c = (budget - t) / tail[t]", "c = budget / tail[t]"),
    ("sip_weight", P, "                weight[r, m] = 1.0 / pm", "                weight[r, m] = pm"),
    ("sip_budget_floor", P, "B = max(1, int(math.ceil(ratio * len(live))))", "B = max(1, int(math.floor(ratio * len(live))))"),
    ("attn_mask_T", P, "keys = np.nonzero(mask[r][k_labels])[0]", "keys = np.nonzero(mask[:, r][k_labels])[0]"),
    ("attn_no_scale", P, "        S = scale * (Q[want[sel]] @ K[keys].T)", "        S = (Q[want[sel]] @ K[keys].T)"),
    ("attn_weight_sign", P, "S += np.log(weight[r][k_labels[keys]])[None, :]", "S -= np.log(weight[r][k_labels[keys]])[None, :]"),
    ("dense_no_norm", P, "O[i0:i0 + 2048] = (P @ V) / P.sum(axis=1, keepdims=True)", "O[i0:i0 + 2048] = (P @ V)"),
    ("win_order", H, "win = ((t // wt) * nWh + (y // wh)) * nWw + (w // ww)", "win = ((w // ww) * nWh + (y // wh)) * (-(-T // wt)) + (t // wt)"),
    ("win_starts_ceil", H, "return np.array([(w * K) // nW for w in range(nW + 1)], dtype=np.int64)",
     "return np.array([-(-(w * K) // nW) for w in range(nW + 1)], dtype=np.int64)"),
    ("local_init_off", H, "C[k0[w] + j] = X[members[(j * len(members)) // Kw]]", "C[k0[w] + j] = X[members[min(len(members) - 1, (j * len(members)) // Kw + 1)]]"),
    ("text_local", H, "        labels[text] = po.assign(X[text], C, M)", "        labels[text] = k0[0] + po.assign(X[text], C[k0[0]:k0[1]], M)"),
    ("pad_16", H, "KEY_GROUP = 8 ", "KEY_GROUP = 16 "),
    ("cost_no_ceil_q", H, "return -(-n // TILE_ROWS) * -(-L // TILE_ROWS)", "return max(1, n // TILE_ROWS) * -(-L // TILE_ROWS)"),
    ("merge_tie_high", H, "                if gain > top:\n                    top, best[g] = gain, h", "                if gain >= top and gain > 0:\n                    top, best[g] = gain, h"),
    ("merge_inter", H, "inter = (S * wk) @ S.T", "inter = 0 * (S * wk) @ S.T"),
    ("merge_no_mutual", H, "if h > g and best[h] == g:", "if h > g and alive[h] and alive[g]:"),
    ("apply_no_union", H, "        new_mask[root[r]] |= np.asarray(mask[r], dtype=bool)", "        new_mask[r] |= np.asarray(mask[r], dtype=bool) if root[r] == r else False"),
]

MUTS2 = [
    ("bf16_ties_away", P, "return np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)",
     "return np.ldexp(np.sign(x) * np.floor(np.abs(np.ldexp(x, 8 - e)) + 0.5), e - 8)"),
    ("bf16_7bits", P, "return np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)", "return np.ldexp(np.rint(np.ldexp(x, 7 - e)), e - 7)"),
    ("bf16_no_subnormal", P, "    e = np.maximum(e, -125)                 # below", "    e = np.maximum(e, -1000)                 # below"),
    ("factor_sqrt_missing", P, "return V * np.sqrt(np.clip(lam, 0.0, None))", "return V * np.clip(lam, 0.0, None)"),
    ("cq_no_scale", P, "z = scale * (np.asarray(CK, dtype=np.float64)[live] @ np.asarray(CQ[r], dtype=np.float64)) + prior",
     "z = (np.asarray(CK, dtype=np.float64)[live] @ np.asarray(CQ[r], dtype=np.float64)) + prior"),
    ("prior_sign", P, "    prior = np.log(np.asarray(k_counts, dtype=np.float64)[live]) if size_prior else 0.0\n    for i0",
     "    prior = -np.log(np.asarray(k_counts, dtype=np.float64)[live]) if size_prior else 0.0\n    for i0"),
    ("topk_tie_high", P, "        order = sorted(live, key=lambda m: (-I[r, m], m))\n        mask[r, order[:k]] = True",
     "        order = sorted(live, key=lambda m: (-I[r, m], -m))\n        mask[r, order[:k]] = True"),
    ("sip_fallback_worst", P, "            best = min(live, key=lambda m: (-I[r, m], m))", "            best = max(live, key=lambda m: (-I[r, m], m))"),
    ("topp_p1_all", P, "        if p >= 1.0:\n            mask[r, live] = True\n            continue", "        if p > 1.0:\n            mask[r, live] = True\n            continue"),
    ("recall_no_norm", P, "        A /= A.sum(axis=1, keepdims=True)\n        keep", "        keep"),
    ("mass_qlabels_T", P, "    np.add.at(mass.T, np.asarray(k_labels), A.T)", "    np.add.at(mass.T, np.asarray(k_labels)[::-1], A.T)"),
    ("tv_no_half", P, "return float(np.mean(0.5 * np.sum(np.abs(P - mass[:, live]), axis=1)))", "return float(np.mean(np.sum(np.abs(P - mass[:, live]), axis=1)))"),
    ("keyerr_raw_qk", P, "    qk = float(np.mean((Q @ R.T) ** 2))", "    qk = float(np.mean((Q @ R.T)) ** 2)"),
    ("wincount_floor", H, "return -(-T // wt), -(-Hg // wh), -(-W // ww)", "return max(1, T // wt), max(1, Hg // wh), max(1, W // ww)"),
    ("apply_old_centroids", H, "    C = po.update(Q, labels, CQ, dtype)\n    return labels, C, new_mask", "    C = np.array(CQ, dtype=np.float64)\n    return labels, C, new_mask"),
    ("merge_rounds_plus", H, "    for _ in range(rounds):", "    for _ in range(rounds + 1):"),
    ("merge_root_nofollow", H, "        while root[g] != g:\n            g = root[g]", "        pass"),
    ("padded_floor", H, "return KEY_GROUP * ((k_counts + KEY_GROUP - 1) // KEY_GROUP)", "return KEY_GROUP * (k_counts // KEY_GROUP)"),
    ("q_kmeans_metric", P, "q_labels, CQ, q_hist = kmeans(Q, NQ, iters, None, dtype,",
     "q_labels, CQ, q_hist = kmeans(Q, NQ, iters, qm, dtype,"),
    ("k_kmeans_euclid", P, "k_labels, CK, k_hist = kmeans(K, NK, iters, km, dtype,",
     "k_labels, CK, k_hist = kmeans(K, NK, iters, None, dtype,"),
    ("pama_query_centroids", P, "        I = pama(Q, q_labels, NQ, CK, k_counts, scale, size_prior=size_prior)",
     "        I = pama(Q, q_labels, NQ, CQ, k_counts, scale, size_prior=size_prior)"),
    ("layer_scale_n", P, "    scale = 1.0 / math.sqrt(np.asarray(Q).shape[1])\n    r[\"O\"]", "    scale = 1.0 / math.sqrt(np.asarray(Q).shape[0])\n    r[\"O\"]"),
    ("local_assign_euclid", H, "labels[rows] = k0[w] + po.assign(X[rows], C[k0[w]:k0[w + 1]], M)",
     "labels[rows] = k0[w] + po.assign(X[rows], C[k0[w]:k0[w + 1]], None)"),
    ("local_update_local", H, "        C = po.update(X, labels, C, dtype)\n    return (labels, C, hist)", "        C = po.update(X, labels, C, None)\n    return (labels, C, hist)"),
]


def run(name, f, old, new):
    with tempfile.TemporaryDirectory(prefix=".oracle_mutants_", dir=ROOT) as dst:
        for d in ("oracle", "tests", "synth"):
            shutil.copytree(os.path.join(ROOT, d), os.path.join(dst, d), ignore=shutil.ignore_patterns("__pycache__", "*.so"))
        shutil.copy(os.path.join(ROOT, "pytest.ini"), dst)
        path = os.path.join(dst, f)
        s = open(path).read()
        if s.count(old) != 1:
            return False, f"pattern found {s.count(old)} times"
        open(path, "w").write(s.replace(old, new))
        p = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                            "tests/test_oracle_pins.py", "tests/test_hva_oracle_pins.py"], cwd=dst,
                           capture_output=True, text=True, timeout=900)
        failed = [ln[7:] for ln in p.stdout.splitlines() if ln.startswith("FAILED")]
        return p.returncode != 0, (failed[0][:100] if failed else p.stdout.strip().splitlines()[-1])


def main(names):
    missed = 0
    for name, f, old, new in MUTS + MUTS2:
        if names and name not in names:
            continue
        caught, why = run(name, f, old, new)
        missed += not caught
        print(f"{name:22s} {'caught' if caught else 'MISSED'}  {why}", flush=True)
    return 1 if missed else 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
