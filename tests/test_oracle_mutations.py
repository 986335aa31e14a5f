"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle (on the CPU, in a scratch
directory, never in the repository's copy), runs the pin suite against the
mutant in a subprocess and requires at least one pin to fail.  A control run of
the unmodified copy must pass.  The mistakes are the ones a transcription of the
method is likely to make: a wrong divisor, a dropped term, a flipped sign, a
wrong index or slice, an off-by-one in a mask, rounding at the wrong point.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join("oracle", "kalm_oracle.py")

MUTATIONS = [
    ("partial chunk divided by the chunk size",
     "enc[base + lo: base + hi].sum(axis=0) / (hi - lo)", "enc[base + lo: base + hi].sum(axis=0) / chunk"),
    ("pooled count rounded down",
     "return (doc_len + chunk - 1) // chunk", "return doc_len // chunk"),
    ("causal diagonal dropped",
     "causal = np.tril(np.ones((Lq, Lq), dtype=bool))", "causal = np.tril(np.ones((Lq, Lq), dtype=bool), -1)"),
    ("future self keys visible",
     "causal = np.tril(np.ones((Lq, Lq), dtype=bool))", "causal = np.tril(np.ones((Lq, Lq), dtype=bool), 1)"),
    ("query heads mapped to KV heads by modulo",
     "g = h // G", "g = h % n_kv"),
    ("logits scaled twice",
     "logits = (q[:, h, :] @ keys.T) * scale", "logits = (q[:, h, :] @ keys.T) * scale * scale"),
    ("log-sum-exp without the row max",
     "lse[:, h] = (m + np.log(s))[:, 0]", "lse[:, h] = np.log(s)[:, 0]"),
    ("cross values taken from the cross keys",
     "np.asarray(v_cross, np.float64)[:, g, :]], axis=0)", "np.asarray(k_cross, np.float64)[:, g, :]], axis=0)"),
    ("bf16 with one significant bit too many",
     "step = np.ldexp(1.0, e - 8)", "step = np.ldexp(1.0, e - 9)"),
    ("bf16 rounding by truncation",
     "out[normal] = np.sign(x[normal]) * np.rint(a[normal] / step) * step",
     "out[normal] = np.sign(x[normal]) * np.floor(a[normal] / step) * step"),
    ("residual added after the rounding",
     "    if residual is not None:\n        y = y + np.asarray(residual, np.float64)\n"
     "    return bf16_round(y) if round_out else y",
     "    y = bf16_round(y) if round_out else y\n    if residual is not None:\n"
     "        y = y + np.asarray(residual, np.float64)\n    return y"),
    ("sigmoid of the negated margin",
     "out[pos] = 1.0 / (1.0 + np.exp(-m[pos]))", "out[pos] = 1.0 / (1.0 + np.exp(m[pos]))"),
    ("margin as no - yes",
     "    margin = yes - no\n    return yes, no, margin", "    margin = no - yes\n    return yes, no, margin"),
    ("readout from the first decoder row",
     "yes_no_score(X[Lq - 1:Lq], w_yes, w_no)", "yes_no_score(X[0:1], w_yes, w_no)"),
    ("self K read from the V slice",
     "ks = qkv[:, n_q * D:(n_q + n_kv) * D].reshape(Lq, n_kv, D)", "ks = qkv[:, (n_q + n_kv) * D:].reshape(Lq, n_kv, D)"),
    ("rotation in the opposite direction",
     "out = np.concatenate([a * c - b * s, b * c + a * s], axis=-1)",
     "out = np.concatenate([a * c + b * s, b * c - a * s], axis=-1)"),
    ("rotary frequencies with exponent i / D",
     "return float(theta) ** (-2.0 * i / head_dim)", "return float(theta) ** (-1.0 * i / head_dim)"),
    ("default logit scale 1 / head_dim",
     "scale = 1.0 / math.sqrt(D) if scale is None else scale", "scale = 1.0 / D if scale is None else scale"),
    ("each document's last encoder row dropped",
     "a, b = int(query.tok_off[d]), int(query.tok_off[d + 1])",
     "a, b = int(query.tok_off[d]), int(query.tok_off[d + 1]) - 1"),
    ("decoder residual dropped",
     "Xn = linear(o.reshape(Lq, n_q * D), w_o_l, residual=X)", "Xn = linear(o.reshape(Lq, n_q * D), w_o_l)"),
    ("every layer reads the first layer's cross weights",
     "w_o[l], w_kv_cross[l], n_q", "w_o[l], w_kv_cross[0], n_q"),
    ("softmax left unnormalised",
     "o[:, h, :] = (e / s) @ vals", "o[:, h, :] = e @ vals"),
    ("cross keys masked out",
     "np.ones((Lq, Nc), dtype=bool)], axis=1)", "np.zeros((Lq, Nc), dtype=bool)], axis=1)"),
    ("pooled chunks overlapping by one token",
     "hi = min(lo + chunk, n)", "hi = min(lo + chunk + 1, n)"),
    ("batched attention reading the next document's cross rows",
     "k_cross[c0:c1], v_cross[c0:c1], scale,", "k_cross[c0 + 1:c1 + 1], v_cross[c0 + 1:c1 + 1], scale,"),
    ("yes logit read with the no row",
     "yes = x @ np.asarray(w_yes, np.float64)", "yes = x @ np.asarray(w_no, np.float64)"),
    ("cross keys and values swapped",
     "merged_attention_doc(q, ks, vs, kv[:, 0], kv[:, 1], scale)", "merged_attention_doc(q, ks, vs, kv[:, 1], kv[:, 0], scale)"),
]


def _copy_tree(dst):
    for d in ("oracle", "tests", "synthetic"):
        shutil.copytree(os.path.join(ROOT, d), os.path.join(dst, d),
                        ignore=shutil.ignore_patterns("__pycache__", "*.pyc", "test_oracle_mutations.py"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), dst)


def _run_pins(tree):
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join("tests", "test_oracle_pins.py"), "-x", "-q",
                           "-p", "no:cacheprovider"], cwd=tree, env=env, capture_output=True, text=True, timeout=600)


def _mutant_result(base, i):
    """Exit status of the pin suite on copy i (-1: the unmodified copy)."""
    tree = os.path.join(base, f"m{i + 1}")
    _copy_tree(tree)
    if i >= 0:
        name, old, new = MUTATIONS[i]
        path = os.path.join(tree, ORACLE)
        src = open(path).read()
        if src.count(old) != 1:
            return "site"
        open(path, "w").write(src.replace(old, new))
    return _run_pins(tree).returncode


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    from concurrent.futures import ThreadPoolExecutor
    base = str(tmp_path_factory.mktemp("oracle_mutants"))
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        codes = list(ex.map(lambda i: _mutant_result(base, i), range(-1, len(MUTATIONS))))
    return dict(zip(range(-1, len(MUTATIONS)), codes))


def test_pins_pass_on_an_unmodified_copy(results):
    assert results[-1] == 0


@pytest.mark.parametrize("i", range(len(MUTATIONS)), ids=[m[0] for m in MUTATIONS])
def test_a_planted_mistake_fails_a_pin(results, i):
    assert results[i] != "site", f"mutation site not unique: {MUTATIONS[i][0]}"
    assert results[i] != 0, f"no pin caught: {MUTATIONS[i][0]}"
