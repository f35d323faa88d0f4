"""The pins catch plausible mistakes in the oracle: each case below plants
one mistake in a copy of oracle/kv2d_oracle.c (a dropped term, a wrong
index or bound, a reversed tie rule, a swapped operand, a step that should
stop but goes on), rebuilds that copy in a scratch directory and runs the
CPU pin files against it; every mutant must fail at least one pin, and the
unmutated copy must pass them all.  The mistakes are planted on the CPU
only, in the scratch copy; nothing here touches the GPU or the product
library's sources."""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PIN_FILES = ["tests/test_oracle_pins.py", "tests/test_oracle_select_pins.py",
             "tests/test_oracle_chunk_pins.py", "tests/test_golden.py"]

# (name, exact text, replacement, which occurrence)
MUTATIONS = [
    ("a_d without |.|", "acc += fabs(qw[(int64_t)row * p->d + k]);",
     "acc += qw[(int64_t)row * p->d + k];", 0),
    ("causal window one key short", "int nvis = last - r0 + 1;", "int nvis = last - r0;", 0),
    ("s_t normalised by the max, not the lse", "s[t] += exp(l[t] - lz);", "s[t] += exp(l[t] - mx);", 0),
    ("channel ties to the higher index", "if (best < 0 || e[x] > e[best]) best = x;",
     "if (best < 0 || e[x] >= e[best]) best = x;", 0),
    ("g_t from the kept channels", "if (!sel[x]) drop += e[x];", "if (sel[x]) drop += e[x];", 0),
    ("token ties to the higher index", "if (best < 0 || s_seg[t] > s_seg[best]) best = t;",
     "if (best < 0 || s_seg[t] >= s_seg[best]) best = t;", 0),
    ("E_BOTH without the dropped tokens", "E[ORC_BOTH] = etok + ekept;", "E[ORC_BOTH] = ekept;", 0),
    ("hull keeps points above the chord", "if (lhs <= rhs) --nh; else break;",
     "if (lhs >= rhs) --nh; else break;", 0),
    ("budget goes on after the first step that does not fit", "if (list[i].db > rem) break;",
     "if (list[i].db > rem) continue;", 0),
    ("value rows packed from K",
     "memcpy(o + (int64_t)j * d * 2, V16 + (int64_t)tok[j] * d, (size_t)d * 2);",
     "memcpy(o + (int64_t)j * d * 2, K16 + (int64_t)tok[j] * d, (size_t)d * 2);", 0),
    ("decode softmax not normalised", "double w = exp(logit[t] - mx) / z;",
     "double w = exp(logit[t] - mx);", 0),
    ("stage-2 score from the first head only", "if (l > best) best = l;", "if (g == 0) best = l;", 0),
    ("Token2Chunk span cap one short", "t - prev + 1 <= gamma", "t - prev + 1 < gamma", 0),
    ("Token2Chunk stops at the first gap that does not fit", "if (cg[i] > rem) continue;",
     "if (cg[i] > rem) break;", 0),
    ("fp16 subnormals one binade low", "v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);", 0),
    ("budget ties to the higher segment", "if (u->seg != v->seg) return u->seg < v->seg ? -1 : 1;",
     "if (u->seg != v->seg) return u->seg > v->seg ? -1 : 1;", 0),
    ("hull keeps options no better than its last point", "if (E[o] >= E[last]) continue;",
     "if (E[o] > E[last]) continue;", 0),
    ("budget bytes rounded up", "return (int64_t)floor(p->beta * (double)((int64_t)nseg * full));",
     "return (int64_t)ceil(p->beta * (double)((int64_t)nseg * full));", 0),
    ("decode segment logits unscaled", "logit[n + t] = p->scale * dot;", "logit[n + t] = dot;", 0),
    ("decode tail logits unscaled", "logit[n + t] = p->scale * dot;", "logit[n + t] = dot;", 1),
    ("stage-2 count rounded down", "double want = ceil(rho * (double)((int64_t)nseg * p->S));",
     "double want = floor(rho * (double)((int64_t)nseg * p->S));", 0),
    ("stage-2 ties to the higher slot", "if (arg < 0 || score[s] > score[arg]) arg = s;",
     "if (arg < 0 || score[s] >= score[arg]) arg = s;", 0),
    ("E_CH without s_t", "for (int t = 0; t < S; ++t) ech += s_seg[t] * g_seg[t];",
     "for (int t = 0; t < S; ++t) ech += g_seg[t];", 0),
    ("a_d divided by rows - 1", "a[k] = acc / (double)rows;", "a[k] = acc / (double)(rows - 1);", 0),
    ("an over-budget start not infeasible", "if (base > Bu) { *used = 0; return ORC_INFEASIBLE; }",
     "if (base > Bu + 1000000) { *used = 0; return ORC_INFEASIBLE; }", 0),
    ("Token2Chunk merit ties to the later gap", "(cm[k] == cm[best] && ca[k] < ca[best])",
     "(cm[k] == cm[best] && ca[k] > ca[best])", 0),
    ("Token2Chunk leftover budget by position, not score",
     "if (sel[order[k]]) continue;\n        sel[order[k]] = 1;", "if (sel[k]) continue;\n        sel[k] = 1;", 0),
    ("stage-2 candidate keys not cleared", "for (int x = 0; x < d; ++x) k[x] = 0.0;", "", 0),
    ("channel values packed from the wrong token", "kv[(int64_t)j * c + x] = K16[(int64_t)tok[j] * d + ch];",
     "kv[(int64_t)j * c + x] = K16[(int64_t)j * d + ch];", 0),
    ("sparse keys decoded at their position, not their channel", "dot += qg[ci[x]] * orc_half_to_double(h);",
     "dot += qg[x] * orc_half_to_double(h);", 0),
    ("beta = 1 through the greedy, not all FULL", "if (p->beta >= 1.0) {", "if (p->beta > 1.0) {", 0),
    ("E_TOK over the kept tokens", "if (!kept[t]) etok += s_seg[t];", "if (kept[t]) etok += s_seg[t];", 0),
    ("hull efficiency with its sign flipped", "eff[k - 1] = (E[h[k - 1]] - E[h[k]]) / (double)dbytes[k - 1];",
     "eff[k - 1] = (E[h[k]] - E[h[k - 1]]) / (double)dbytes[k - 1];", 0),
    ("channel importance from k, not |k|", "e[x] = fabs(k[x]) * a[x];", "e[x] = k[x] * a[x];", 0),
    ("lse without the max", "double lz = mx + log(sum);", "double lz = log(sum);", 0),
]
# Not listed, because they cannot change a result: the budget's tie rule on
# the step index (a segment's hull steps have strictly decreasing
# efficiency, so two of them never tie), and Token2Chunk gaps of length 0
# as candidates (filling one keeps nothing more).


def _replace_nth(src, old, new, n):
    pos = -1
    for _ in range(n + 1):
        pos = src.index(old, pos + 1)
    return src[:pos] + new + src[pos + len(old):]


def _scratch_tree(dst, mutation):
    for sub in ("oracle", "tests", "kv_cache_compression_kv2d_b200"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(dst, sub),
                        ignore=shutil.ignore_patterns("liboracle.so*", "__pycache__", "*.tmp"))
    path = os.path.join(dst, "oracle", "kv2d_oracle.c")
    if mutation is not None:
        _, old, new, n = mutation
        with open(path) as f:
            src = f.read()
        assert src.count(old) > n, f"mutation site not found: {old}"
        with open(path, "w") as f:
            f.write(_replace_nth(src, old, new, n))


def _run_pins(cwd):
    env = dict(os.environ)
    env.pop("PYTHONPATH", None)
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           "-m", "not gpu"] + PIN_FILES,
                          cwd=cwd, env=env, capture_output=True, text=True, timeout=600)


def test_unmutated_copy_passes(tmp_path):
    _scratch_tree(str(tmp_path), None)
    res = _run_pins(str(tmp_path))
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-2000:]


def test_every_mutant_fails_a_pin(tmp_path):
    # the mutants are independent builds and runs: several at a time
    def one(i):
        dst = str(tmp_path / f"m{i}")
        os.makedirs(dst)
        _scratch_tree(dst, MUTATIONS[i])
        return MUTATIONS[i][0], _run_pins(dst).returncode
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(one, range(len(MUTATIONS))))
    survivors = [name for name, rc in results if rc == 0]
    assert not survivors, f"mistakes no pin caught: {survivors}"
