"""The pins are strong enough: for each plausible mistake planted in a copy
of the oracle (a wrong split of the tree, a dropped term, a transposed
index, an unstable sort, a misplaced eps ...), at least one pin of
test_oracle_pins.py fails.  The mutant is compiled into a temporary library
and swapped into the oracle module for the duration of the test; the
checked-in oracle is untouched.  CPU only.

Not in the list, because no CPU pin can see it: a change that stays inside
the accuracy bounds of the written exp/log (a coefficient of the log
series changed from 1/9 to 1/8 moves its result by far less than an ulp).
The GPU parity tests, which compare the kernels with the oracle bit for
bit, would catch it."""
import inspect

import pytest

import oracle
import test_oracle_pins as pins

# (name, text in oracle.c, replacement): each text occurs exactly once
MUTANTS = [
    ("tree split floor(n/2)", "long h = (n + 1) / 2;", "long h = n / 2;"),
    ("bf16 rounding half-up", "if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u)))", "if (rest >= 0x8000u)"),
    ("lane chain reversed inside a vector", "p = p + v[j * V + e];", "p = p + v[j * V + (V - 1 - e)];"),
    ("exp: wrong 1/3! coefficient", "const float c3 = (float)(1.0 / 6.0);", "const float c3 = (float)(1.0 / 5.0);"),
    ("exp: ln2 tail dropped", "    r = fmaf(-n, ln2_tl, r);\n", "\n"),
    ("log: no reduction to [sqrt(1/2), sqrt(2))", "if (m > sqrt2) { m = m * 0.5f; e = e + 1; }", ""),
    ("rmsnorm: eps outside the sqrt", "return 1.0f / sqrtf(ms + eps);", "return 1.0f / (sqrtf(ms) + eps);"),
    ("rmsnorm: final products reassociated", "float v = or_bf16_to_f32(xr[k]) * inv;\n            y[i * n + k] = or_f32_to_bf16(v * or_bf16_to_f32(w[k]));",
     "float v = inv * or_bf16_to_f32(w[k]);\n            y[i * n + k] = or_f32_to_bf16(or_bf16_to_f32(xr[k]) * v);"),
    ("log_softmax: reassociated output", "for (long k = 0; k < n; k++) out[i * n + k] = (xr[k] - m) - L;",
     "for (long k = 0; k < n; k++) out[i * n + k] = xr[k] - (m + L);"),
    ("log_softmax: 1024 lanes", "float S = or_canon_sum(e, n, 4096, 4);", "float S = or_canon_sum(e, n, 1024, 4);"),
    ("mean: divides by n - 1", "out[i] = or_canon_sum(x + i * n, n, 1024, 4) / (float)n;",
     "out[i] = or_canon_sum(x + i * n, n, 1024, 4) / (float)(n - 1);"),
    ("mean exact: divides by n + 1", "out[i] = s / (double)n;", "out[i] = s / (double)(n + 1);"),
    ("shrink: adapter and rank indices swapped", "const uint16_t *ar = at + (a * r + j) * K;",
     "const uint16_t *ar = at + (j * n_ad + a) * K;"),
    ("expand: y not rounded to bf16", "yb[j] = (double)or_bf16_to_f32(or_f32_to_bf16(y[m * r + j]));",
     "yb[j] = (double)y[m * r + j];"),
    ("gemm: W read transposed", "double p = av[k] * bf(wr[k]);", "double p = av[k] * bf(W[k * N + n]);"),
    ("addmm: bias indexed by row", "C[i * N + n] += bf(bias[n]);", "C[i * N + n] += bf(bias[i % N]);"),
    ("attention: running sum inside a chunk",
     "oc[c * D + d] = or_frame_tree(tmp, 256);",
     "{ float acc = 0.0f; for (long i = 0; i < 256; i++) acc = acc + tmp[i]; oc[c * D + d] = acc; }"),
    ("attention: chunk weights dropped", "for (long c = 0; c < n; c++) ac[c] = or_exp(mc[c] - M);",
     "for (long c = 0; c < n; c++) ac[c] = 1.0f;"),
    ("attention exact: softmax without the max shift", "for (long j = 0; j < L; j++) { s[j] = exp(s[j] - m); den += s[j]; }",
     "for (long j = 0; j < L; j++) { s[j] = exp(s[j]); den += s[j] * (1.0 + 1e-9); }"),
    ("segment: tokens scattered in reverse order",
     "if (ids[t] >= 0 && ids[t] < n_ad) perm[count[ids[t]]++] = (int32_t)t;",
     "if (ids[M - 1 - t] >= 0 && ids[M - 1 - t] < n_ad) perm[count[ids[M - 1 - t]]++] = (int32_t)(M - 1 - t);"),
    ("tree combine over the wrong axis", "out[i] = or_tree_f32(parts + i, s, count);",
     "out[i] = or_tree_f32(parts + i * s, s, 1);"),
]


def _pin_calls():
    """Every pin as a zero-argument callable (parametrized pins expanded)."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = list(inspect.signature(fn).parameters)
        marks = getattr(fn, "pytestmark", [])
        grid = [m for m in marks if m.name == "parametrize"]
        if params == ["oracle_mod"]:
            calls.append((name, lambda fn=fn: fn(oracle)))
        elif grid and len(grid) == 1 and params[0] == "oracle_mod":
            argname = grid[0].args[0]
            for v in grid[0].args[1]:
                calls.append((f"{name}[{v}]", lambda fn=fn, v=v, a=argname: fn(oracle, **{a: v})))
    return calls


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_a_pin_catches_the_mistake(name, old, new, tmp_path, monkeypatch):
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique for {name!r}"
    mutant = tmp_path / "oracle_mutant.c"
    mutant.write_text(src.replace(old, new))
    monkeypatch.setattr(oracle, "_SRC", str(mutant))
    monkeypatch.setattr(oracle, "_LIB", str(tmp_path / "liboracle_mutant.so"))
    monkeypatch.setattr(oracle, "_lib", None)
    caught = None
    for pin, call in _pin_calls():
        try:
            call()
        except AssertionError:
            caught = pin
            break
    assert caught is not None, f"no pin fails with the planted mistake {name!r}"
