"""Mutation check of the oracle's CPU pins (test infrastructure, not collected by pytest).

Plants one plausible mistake at a time (a dropped term, a wrong tie rule, an off-by-one, a
swapped operand) in a temporary copy of ``oracle/ckv_oracle.c``, rebuilds it there, and runs
the ``tests/test_oracle_*.py`` pins against the copy. Every mistake should make a pin fail.
The repository's own oracle is never modified.

    python tests/oracle_mutations.py            # all mutations (a few minutes)
    python tests/oracle_mutations.py "fit strict" "assign ties high"   # selected ones

Exit status 1 if a mistake survives. The stream-key layout (``unit << 32``) is a definition
shared with the CUDA side, not a computation; the GPU parity tests catch a mismatch there,
and it is not listed.
"""
import os, shutil, subprocess, sys, tempfile
REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = open(os.path.join(REPO, 'oracle/ckv_oracle.c')).read()
M = [
 ("bf16 ties away", "double r = nearbyint(ax / quantum) * quantum; /* default", "double r = round(ax / quantum) * quantum; /* default", 0),
 ("splitmix gamma", "uint64_t z = (*state += 0x9E3779B97F4A7C15ULL);", "uint64_t z = (*state += 0x9E3779B97F4A7C16ULL);", 0),
 ("bounded low bits", "return (uint32_t)(((x >> 32) * (uint64_t)r) >> 32);", "return (uint32_t)(((x & 0xffffffffULL) * (uint64_t)r) >> 32);", 0),
 ("fisher-yates range", "int64_t j = i + (int64_t)orc_bounded(x, (uint32_t)(m - i));", "int64_t j = i + (int64_t)orc_bounded(x, (uint32_t)(m - i - 1));", 0),
 ("normalise no sqrt", "double nrm = sqrt(ss);", "double nrm = ss;", 0),
 ("assign ties high", "if (s > best) { best = s; arg = c; }", "if (s >= best) { best = s; arg = c; }", 0),
 ("mean off by one", "acc[d] / (double)(hi - lo);", "acc[d] / (double)(hi - lo + 1);", 0),
 ("empty resets mu", "if (hi == lo) continue;\n        double acc[ORC_D] = {0};", "if (hi == lo) { for (int d = 0; d < ORC_D; d++) mu[(int64_t)c * ORC_D + d] = 0.0; continue; }\n        double acc[ORC_D] = {0};", 0),
 ("init row shifted", "orc_bf16_to_double(keys[(int64_t)init[c] * ORC_D + d]);", "orc_bf16_to_double(keys[(int64_t)((init[c] + 1) % m) * ORC_D + d]);", 0),
 ("prefill ids", "ids[j] = (int32_t)src;", "ids[j] = (int32_t)(src - n_sink);", 0),
 ("window ids", "ids[j] = (int32_t)(first_id + perm[j]);", "ids[j] = (int32_t)(first_id + perm[j] + 1);", 0),
 ("pending id", "(int32_t)(s->n_sink + s->m + (i - s->n_sink))", "(int32_t)(s->n_sink + (i - s->n_sink))", 0),
 ("remaining drops pending", "int64_t remaining = (int64_t)budget - s->n_sink - s->pending;", "int64_t remaining = (int64_t)budget - s->n_sink;", 0),
 ("cluster ties high", "return (x->idx > y->idx) - (x->idx < y->idx);", "return (x->idx < y->idx) - (x->idx > y->idx);", 0),
 ("token ties high", "return (x->id > y->id) - (x->id < y->id);", "return (x->id < y->id) - (x->id > y->id);", 0),
 ("fit strict", "if (size <= remaining) {", "if (size < remaining) {", 0),
 ("partial lowest", "sel_ids[count] = tk[j].id;\n                sel_rows[count] = tk[j].idx;", "sel_ids[count] = tk[size - 1 - j].id;\n                sel_rows[count] = tk[size - 1 - j].idx;", 0),
 ("skip-ahead", "            free(tk);\n            break;", "            free(tk);\n            continue;", 0),
 ("attend scale", "const double scale = 1.0 / sqrt((double)ORC_D);", "const double scale = 1.0 / (double)ORC_D;", 0),
 ("dense scale", "const double scale = 1.0 / sqrt((double)ORC_D);", "const double scale = 1.0 / (double)ORC_D;", 1),
 ("group query one head", "for (int32_t g = 0; g < G; g++) s += orc_bf16_to_double(q[(int64_t)g * ORC_D + d]);", "for (int32_t g = 0; g < 1; g++) s += orc_bf16_to_double(q[(int64_t)g * ORC_D + d]);", 0),
 ("drift plus cos", "acc += 1.0 - cosv;", "acc += 1.0 + cosv;", 0),
 ("drift no mu norm", "dot / (sqrt(kk) * sqrt(mm))", "dot / (sqrt(kk))", 0),
 ("drift no key norm", "dot / (sqrt(kk) * sqrt(mm))", "dot / (sqrt(mm))", 0),
 ("split room le", "n_split < room;", "n_split <= room;", 0),
 ("split size 1", "size >= 2 && n_split < room", "size >= 1 && n_split < room", 0),
 ("split key c", "((uint64_t)(c + 1) * 0x9E3779B97F4A7C15ULL)", "((uint64_t)(c) * 0x9E3779B97F4A7C15ULL)", 0),
 ("split mid", "offsets2[out + 1] = lo + coff[1];", "offsets2[out + 1] = lo + coff[1] - 1;", 0),
 ("split threshold ge", "split[c] = drift[c] > threshold &&", "split[c] = drift[c] >= threshold - 1e-3 &&", 0),
 ("e4m3 subnormal quantum", "if (ex < -6) ex = -6;     /* subnormals", "if (ex < -7) ex = -7;     /* subnormals", 0),
 ("e4m3 ties away", "double r = nearbyint(ax / quantum) * quantum;\n    if (r > 448.0)", "double r = round(ax / quantum) * quantum;\n    if (r > 448.0)", 0),
 ("quant scale 447", "float scale = mx / 448.0f;", "float scale = mx / 447.0f;", 0),
 ("mixed rank gt", "if (r >= 0 && row_rank[i] >= n_near) {\n                for (int d = 0; d < ORC_D; d++)\n                    dot +=", "if (r >= 0 && row_rank[i] > n_near) {\n                for (int d = 0; d < ORC_D; d++)\n                    dot +=", 0),
 ("mixed rank gt v", "if (r >= 0 && row_rank[i] >= n_near) {\n                for (int d = 0; d < ORC_D; d++)\n                    acc[d] +=", "if (r >= 0 && row_rank[i] > n_near) {\n                for (int d = 0; d < ORC_D; d++)\n                    acc[d] +=", 0),
 ("mixed v from k", "acc[d] += p * (orc_e4m3_to_double(v8[", "acc[d] += p * (orc_e4m3_to_double(k8[", 0),
("update perm descending", "    for (int64_t i = 0; i < m; i++) {\n        int32_t c = assign[i];\n        perm[", "    for (int64_t i = m - 1; i >= 0; i--) {\n        int32_t c = assign[i];\n        perm[", 0),
 ("assign gap sign", "gap[i] = (best - so)", "gap[i] = (so - best)", 0),
 ("attend denominator", "out[(int64_t)g * ORC_D + d] = acc[d] / den;", "out[(int64_t)g * ORC_D + d] = acc[d] / (den + 1e-3);", 0),
 ("dense denominator", "out[(int64_t)g * ORC_D + d] = acc[d] / den;", "out[(int64_t)g * ORC_D + d] = acc[d] / (den + 1e-3);", 1),
 ("attend v from kp", "const uint16_t* v = r >= 0 ? s->vp + (int64_t)r * ORC_D", "const uint16_t* v = r >= 0 ? s->kp + (int64_t)r * ORC_D", 0),
 ("select skips pending rows", "for (int32_t i = 0; i < s->n_sink + s->pending; i++) {", "for (int32_t i = 0; i < s->n_sink; i++) {", 0),
 ("score dims swapped", "sc += qbar[d] * s->mu[(int64_t)c * ORC_D + d];", "sc += qbar[d] * s->mu[(int64_t)c * ORC_D + (d ^ 1)];", 0),
 ("partial score next row", "t += qbar[d] * orc_bf16_to_double(s->kp[(int64_t)j * ORC_D + d]);", "t += qbar[d] * orc_bf16_to_double(s->kp[(int64_t)(j + 1 < hi ? j + 1 : j) * ORC_D + d]);", 0),
 ("prefill clusters sinks", "const uint16_t* keys = K + (int64_t)n_sink * ORC_D;", "const uint16_t* keys = K;", 0),
 ("drift empty one", "drift[c] = 0.0;", "drift[c] = 1.0;", 0),
 ("split rows unpermuted", "int64_t src = (int64_t)lo + cperm[j],", "int64_t src = (int64_t)lo + j,", 0),
 ("e4m3 decode subnormal", "ldexp((double)mant, -9)", "ldexp((double)mant, -10)", 0),
 ("e4m3 decode bias", "ldexp(1.0 + mant / 8.0, ex - 7)", "ldexp(1.0 + mant / 8.0, ex - 8)", 0),
 ("batch sp no pending", "int64_t sp = (int64_t)n_sink + pending;", "int64_t sp = (int64_t)n_sink;", 0),
 ("batch offsets stride C", "s.offsets = offsets + (int64_t)u * (C + 1);", "s.offsets = offsets + (int64_t)u * C;", 0),
 ("prefill batch offsets stride C", "offsets + (int64_t)u * (C + 1),\n                         mu", "offsets + (int64_t)u * C,\n                         mu", 0),
 ("batch qbar stride", "orc_group_query(q + (int64_t)u * G * ORC_D, G, qbar);", "orc_group_query(q + (int64_t)u * ORC_D, G, qbar);", 0),
 ("batch attend q stride", "orc_attend(&s, q + (int64_t)u * G * ORC_D", "orc_attend(&s, q + (int64_t)u * ORC_D", 0),
 ("mixed v path bf16 from k", "const uint16_t* v = r >= 0 ? s->vp + (int64_t)r * ORC_D", "const uint16_t* v = r >= 0 ? s->kp + (int64_t)r * ORC_D", 1),
]

def nth_replace(s, old, new, n):
    i = -1
    for _ in range(n + 1):
        i = s.find(old, i + 1)
        if i < 0:
            return None
    return s[:i] + new + s[i + len(old):]

only = sys.argv[1:]
survivors = []
for name, old, new, n in M:
    if only and name not in only:
        continue
    mutated = nth_replace(SRC, old, new, n)
    if mutated is None:
        print(f"!! pattern not found: {name}"); continue
    d = tempfile.mkdtemp(prefix='mut_')
    for sub in ('oracle', 'tests'):
        shutil.copytree(os.path.join(REPO, sub), os.path.join(d, sub), ignore=shutil.ignore_patterns('*.so', '__pycache__'))
    for f in ('synth_inputs.py', 'pytest.ini'):
        shutil.copy(os.path.join(REPO, f), d)
    open(os.path.join(d, 'oracle/ckv_oracle.c'), 'w').write(mutated)
    tests = sorted(os.path.join('tests', f) for f in os.listdir(os.path.join(d, 'tests')) if f.startswith('test_oracle'))
    r = subprocess.run([sys.executable, '-m', 'pytest', '-x', '-q', '-m', 'not gpu', '-p', 'no:cacheprovider', *tests],
                       cwd=d, capture_output=True, text=True, timeout=900)
    caught = r.returncode != 0
    first = ''
    for line in r.stdout.splitlines():
        if line.startswith('FAILED') or line.startswith('ERROR'):
            first = line[:110]; break
    print(f"{'caught ' if caught else 'SURVIVED'} {name:28s} {first}", flush=True)
    if not caught:
        survivors.append(name)
    shutil.rmtree(d)
print("survivors:", survivors)
sys.exit(1 if survivors else 0)
