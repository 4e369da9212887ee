"""The oracle's pins catch plausible mistakes: each case below plants one
mistake in a copy of the C oracle (a dropped term, a flipped sign, a wrong
index or bit order, a wrong tie rule, a skipped rounding), builds it, points
the oracle wrapper at it and checks that at least one pin of
tests/test_oracle_pins.py fails.  The NumPy attention, merge and full-layer
attention get the same treatment: a mutated copy of the function's source
replaces it while the pins run.  CPU only; the real oracle is restored after
every case."""

import inspect
import os
import subprocess
import tempfile

import pytest

from oracle import build as OB
from oracle import oracle as O
from tests import test_oracle_pins as P

# (name, text in kvq_oracle.c, replacement)
MUTATIONS = [
    ("distance drops the last channel",
     "for (int c = 0; c < d; ++c) {\n        float e = x[c] - mu[c];",
     "for (int c = 0; c < d - 1; ++c) {\n        float e = x[c] - mu[c];"),
    ("distance subtracts the squared term", "acc = acc + sq;", "acc = acc - sq;"),
    ("argmin ties go to the highest index", "        if (dj < bd) {\n            bd = dj;",
     "        if (dj <= bd) {\n            bd = dj;"),
    ("zero point with the wrong sign", "float z = rintf(-mn * inv);", "float z = rintf(mn * inv);"),
    ("codes without the zero point", "float v = rintf(r[c] * inv) + z;", "float v = rintf(r[c] * inv);"),
    ("dequantisation adds the zero point", "float t = (float)q - z;", "float t = (float)q + z;"),
    ("codes packed high bits first", "<< (i * bits);", "<< ((per - 1 - i) * bits);"),
    ("k-means mean over n + 1", "/ (double)counts[j];", "/ (double)(counts[j] + 1);"),
    ("empty centre zeroed instead of kept",
     "                if (counts[j] == 0)\n                    continue;",
     "                if (counts[j] == 0) {\n                    for (int c = 0; c < d; ++c)\n"
     "                        cent_h[(int64_t)j * d + c] = 0;\n                    continue;\n                }"),
    ("joint residual not rounded to bf16", "res[h * d + c] = bf16_widen(bf16_round(e));", "res[h * d + c] = e;"),
    ("joint decoder forgets the centre", "out[(t * H + h) * (int64_t)d + c] = mu + (float)acc;",
     "out[(t * H + h) * (int64_t)d + c] = (float)acc;"),
    ("QSAC distance without the channel weight", "const float term = w[c] * diff2;", "const float term = diff2;"),
    ("QSAC score without the group weight", "const float term = wg * range2;", "const float term = range2;"),
    ("QSAC group range without its minimum", "const float range = hi - lo;", "const float range = hi;"),
    ("QSAC score ties to the worse-ranked candidate", "if (k == 0 || sc < best) {", "if (k == 0 || sc <= best) {"),
    ("QSAC ranking ties to the higher index", "while (pos > 0 && dj < cand_dist[pos - 1])",
     "while (pos > 0 && dj <= cand_dist[pos - 1])"),
    ("second stage error with the wrong sign", "e[c] = r[c] - kvqo_dequant(q[c], s1, z1);",
     "e[c] = kvqo_dequant(q[c], s1, z1) - r[c];"),
    ("second stage quantises the residual again", "kvqo_quant_group(e + g * G, G, bits, &s2, &z2, q + g * G);",
     "kvqo_quant_group(r + g * G, G, bits, &s2, &z2, q + g * G);"),
    ("two-stage decode drops the second stage",
     "stage1 + kvqo_dequant(q2[c], meta2[(th * ng + g) * 2], meta2[(th * ng + g) * 2 + 1]);", "stage1;"),
    ("compact codec takes 1/s from the unrounded scale", "const float inv = 1.0f / sf;", "const float inv = 1.0f / s;"),
    ("binary16 rounding truncates", "if (rem > 0x1000u || (rem == 0x1000u && (h & 1u)))\n            h += 1u;",
     "(void)rem;"),
    ("binary16 overflow goes to infinity", "return (uint16_t)(sign | 0x7bffu);", "return (uint16_t)(sign | 0x7c00u);"),
    ("compact codec keeps a scale that rounds to zero", " || (s16 & 0x7fffu) == 0u", ""),
    ("compact decode forgets the zero point", "float z = kvqo_f16_widen(meta16[(th * ng + g) * 2 + 1]);",
     "float z = 0.0f;"),
    ("bf16 rounding ties away from zero", "u += 0x7fffu + keep_lsb;", "u += 0x8000u + 0u * keep_lsb;"),
    ("bf16 rounding truncates", "u += 0x7fffu + keep_lsb;", "u += 0u * keep_lsb;"),
]


def _pins():
    return [(n, f) for n, f in inspect.getmembers(P, inspect.isfunction)
            if n.startswith("test_") and not inspect.signature(f).parameters]


def _build_mutant(src: str, out_dir: str) -> str:
    path_c = os.path.join(out_dir, "kvq_oracle_mutant.c")
    with open(path_c, "w") as f:
        f.write(src)
    path_so = os.path.join(out_dir, "libkvq_oracle_mutant.so")
    subprocess.run(["gcc", *OB.CFLAGS, "-o", path_so, path_c, "-lm"], check=True)
    return path_so


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, old, new):
    with open(OB.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site not unique or missing: {name}"
    saved_path, saved_lib = O._LIB_PATH, O._lib
    failed = []
    with tempfile.TemporaryDirectory() as d:
        so = _build_mutant(src.replace(old, new), d)
        try:
            O._LIB_PATH, O._lib = so, None
            for pin_name, pin in _pins():
                try:
                    pin()
                except (AssertionError, RuntimeError, ValueError):
                    failed.append(pin_name)
        finally:
            O._LIB_PATH, O._lib = saved_path, saved_lib
    assert failed, f"no pin fails with the planted mistake: {name}"


def test_unmutated_oracle_passes_every_pin():
    for _, pin in _pins():
        pin()


# (function in oracle.py, name, text in its source, replacement): mistakes
# planted in the NumPy attention, merge and full-layer attention
PY_MUTATIONS = [
    ("attention", "softmax scale dropped", "@ kf[:, h, :].T) * sc", "@ kf[:, h, :].T)"),
    ("attention", "keys of head 0 for every head", "qf[:, h, :] @ kf[:, h, :].T", "qf[:, h, :] @ kf[:, 0, :].T"),
    ("attention", "output not normalised", "O[:, h, :] = (p @ vf[:, h, :]) / l", "O[:, h, :] = (p @ vf[:, h, :])"),
    ("attention", "lse without the max shift", "lse[h, :] = (m + np.log(l))[:, 0]", "lse[h, :] = (np.log(l))[:, 0]"),
    ("lse_merge", "merge weights not normalised", "w / np.where(finite, tot, 1.0)[None]", "w"),
    ("lse_merge", "merged lse without the max", "msafe + np.log(np.where(finite, tot, 1.0))",
     "np.log(np.where(finite, tot, 1.0))"),
    ("layer_attention", "chunk keys and values ignored",
     "k = np.concatenate([_widen(k_hist), _widen(k_cur)], axis=0)\n    v = np.concatenate([_widen(v_hist), "
     "_widen(v_cur)], axis=0)", "k = _widen(k_hist)\n    v = _widen(v_hist)"),
    ("layer_attention", "chunk values read as raw bf16 bits", "_widen(v_cur)], axis=0)",
     "v_cur.astype(np.float64)], axis=0)"),
    ("query_moments", "query moments not averaged", "/ max(n, 1)", ""),
    ("psac_basis", "PSAC keeps the smallest eigenvalues", 'np.argsort(-lam, kind="stable")',
     'np.argsort(lam, kind="stable")'),
    ("psac_coefficients", "PSAC error with the wrong sign", "e = _widen(x) - _widen(k_hat)",
     "e = _widen(k_hat) - _widen(x)"),
    ("bf16_bits", "bf16 rounding truncates", "q = np.rint(np.ldexp(a, 8 - e))", "q = np.trunc(np.ldexp(a, 8 - e))"),
    ("fast_maps_analytical", "analytical maps keep the smallest singular vectors", "V = vt[:d_low].T",
     "V = vt[-d_low:].T"),
    ("fast_reduce_queries", "reduced queries left unrounded",
     'return bf16_bits(np.einsum("thc,hcl->thl", _widen(q), _widen(P)))',
     'return np.einsum("thc,hcl->thl", _widen(q), _widen(P))'),
    ("fast_attention", "softmax scale of the low dimension", "d = _widen(P).shape[1]", "d = _widen(P).shape[2]"),
    ("fast_attention", "output restored with the query map", "_widen(R))", "np.transpose(_widen(P), (0, 2, 1)))"),
    ("fast_history_mac_ratio", "MACs not weighted by the head dim", "int(n) * int(dh)", "int(n) * d"),
    ("attention_psac", "PSAC correction dropped", 'kc = _widen(k_hat) + np.einsum("hdr,thr->thd", U, coef.astype(np.float64))',
     "kc = _widen(k_hat)"),
]


@pytest.mark.parametrize("fn,name,old,new", PY_MUTATIONS, ids=[m[1] for m in PY_MUTATIONS])
def test_pins_catch_planted_mistake_in_numpy_oracle(fn, name, old, new):
    src = inspect.getsource(getattr(O, fn))
    assert src.count(old) == 1, f"mutation site not unique or missing: {name}"
    scope = {}
    exec(compile(src.replace(old, new), O.__file__, "exec"), O.__dict__, scope)
    saved = getattr(O, fn)
    failed = []
    try:
        setattr(O, fn, scope[fn])
        for pin_name, pin in _pins():
            try:
                pin()
            except (AssertionError, RuntimeError, ValueError, FloatingPointError):
                failed.append(pin_name)
    finally:
        setattr(O, fn, saved)
    assert failed, f"no pin fails with the planted mistake: {name}"
