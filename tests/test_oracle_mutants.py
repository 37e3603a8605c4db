"""Planted mistakes in the oracle, on the CPU.

Each mutant below is a copy of ``oracle/tq_oracle.cpp`` with one plausible mistake
planted in it -- a dropped term, a wrong sign, a transposed operand, a flipped tie,
a wrong constant or offset -- compiled on its own and loaded by a separate pytest
process in place of the oracle (``TQ_ORACLE_LIB``).  The pins named beside the
mutant must fail on it; the unmutated source, compiled and loaded the same way,
passes every one of them.  This is the evidence that the pins constrain what the
oracle computes, not only restate it: a mistake of one of these kinds anywhere in
the listed functions turns a pin red.

Nothing here touches a GPU or the CUDA library.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor
from pathlib import Path


ROOT = Path(__file__).resolve().parent.parent
SRC = ROOT / "oracle" / "tq_oracle.cpp"
P, Q = "tests/test_oracle_params.py::", "tests/test_oracle_quantizer.py::"
F3, WIN = "tests/test_oracle_f3.py::", "tests/test_oracle_window.py::"

# (mistake, text of the source, text planted instead, pins that must fail)
MUTANTS = [
    ("SplitMix64: wrong golden-gamma increment",
     "state += 0x9E3779B97F4A7C15ull;", "state += 0x9E3779B97F4A7C17ull;",
     [P + "test_splitmix64_published_outputs"]),
    ("QJL / Hadamard signs: top bit read inverted",
     "int sign() { return (next() >> 63) ? -1 : 1; }", "int sign() { return (next() >> 63) ? 1 : -1; }",
     [P + "test_signs_top_bit"]),
    ("Box-Muller: sine for the first normal of a pair",
     "out[k] = rad * std::cos(two_pi * u2);", "out[k] = rad * std::sin(two_pi * u2);",
     [P + "test_box_muller_pair_formula"]),
    ("Haar: sign fix of Q's columns dropped",
     "double s = (alpha[k] < 0.0) ? -1.0 : 1.0;", "double s = 1.0;",
     [P + "test_haar_is_the_positive_diagonal_qr_factor"]),
    ("FWHT: butterfly difference with the wrong sign",
     "x[j + h] = a - b;", "x[j + h] = b - a;",
     [P + "test_fwht_equals_sylvester_matrix"]),
    ("Hadamard rotation: 1/d instead of 1/sqrt(d)",
     "Rm[(size_t)i * d + j] = e[j] / std::sqrt((double)d);", "Rm[(size_t)i * d + j] = e[j] / (double)d;",
     [P + "test_hadamard_rotation_matrix"]),
    ("Gaussian Lloyd-Max: centroid numerator phi(a) + phi(b)",
     "double nc = (pa - pb) / cell_prob(a, b);", "double nc = (pa + pb) / cell_prob(a, b);",
     [P + "test_textbook_table"]),
    ("Gaussian cell probability: wrong tail on the positive side",
     "if (a >= 0.0) return 0.5 * (std::erfc(a / r2) - std::erfc(b / r2));",
     "if (a >= 0.0) return 0.5 * (std::erfc(b / r2) - std::erfc(a / r2));",
     [P + "test_textbook_table"]),
    ("Beta Lloyd-Max: first moment with the cell's ends swapped",
     "beta_first_moment(d, tt[j], tt[j + 1])", "beta_first_moment(d, tt[j + 1], tt[j])",
     [F3 + "test_lloyd_conditions_of_the_beta_law"]),
    ("Dense 3-bit layout ignored: 3-bit codes stay in nibbles",
     "return (dense3 && b == 3) ? 3 : container_width(b);", "return container_width(b);",
     [F3 + "test_dense3_chunk_sizes"]),
    ("Pack: bits written most significant first",
     "out[(i * w + k) / 8] |= (uint8_t)(1u << ((i * w + k) % 8));",
     "out[(i * w + k) / 8] |= (uint8_t)(1u << (7 - (i * w + k) % 8));",
     [Q + "test_pack_bit_order_convention"]),
    ("Chunk size: sign bits not counted",
     "+ (size_t)16 * d / 8 + 128;", "+ 128;",
     [Q + "test_chunk_sizes_match_the_pages_byte_counts"]),
    ("Chunk layout: gamma stored over the norms",
     "std::memcpy(chunk + off + 64 + 4 * row, &gf, 4);", "std::memcpy(chunk + off + 4 * row, &gf, 4);",
     [Q + "test_paged_store_matches_vector_compress"]),
    ("Norm: squared norm used as the norm",
     "const double n = std::sqrt(n2);", "const double n = n2;",
     [Q + "test_scale_invariance_of_codes"]),
    ("Zero vector: the cell above 0",
     "codes[i] = L / 2 - 1;", "codes[i] = L / 2;",
     [Q + "test_zero_vector"]),
    ("Rotation: R x instead of R^T x (transposed operand)",
     "for (int i = 0; i < d; ++i) s += P.R[(size_t)i * d + j] * x[i];",
     "for (int i = 0; i < d; ++i) s += P.R[(size_t)j * d + i] * x[i];",
     [Q + "test_rotation_direction_is_R_transpose"]),
    ("Bucketize: ties go to the upper cell",
     "if (t[k] < v) ++idx;", "if (t[k] <= v) ++idx;",
     [Q + "test_tie_goes_to_the_lower_cell"]),
    ("QJL: residual taken as k_hat - k",
     "r[i] = x[i] - khat[i];", "r[i] = khat[i] - x[i];",
     [Q + "test_qjl_signs_are_signs_of_the_residual_sketch"]),
    ("QJL: gamma = ||r||^2",
     "o.gamma = std::sqrt(g2);", "o.gamma = g2;",
     [Q + "test_gamma_equals_rotated_domain_residual"]),
    ("QJL: sign bits inverted",
     "signs[j] = (s >= 0.0) ? 1 : 0;", "signs[j] = (s >= 0.0) ? 0 : 1;",
     [Q + "test_qjl_estimator_unbiased_over_1000_seeds"]),
    ("QJL key decompress: pi/2 without the square root",
     "const double coef = gamma * std::sqrt(3.14159265358979323846 / 2.0) / d;",
     "const double coef = gamma * (3.14159265358979323846 / 2.0) / d;",
     [Q + "test_qjl_decompress_matches_estimator"]),
    ("Decode: QJL term subtracted",
     "dot += g * qjl * sg;", "dot -= g * qjl * sg;",
     [Q + "test_decode_forms_agree_and_match_bruteforce"]),
    ("Decode: QJL scale sqrt(pi/2)/sqrt(d) instead of /d",
     "const double qjl = std::sqrt(3.14159265358979323846 / 2.0) / d;",
     "const double qjl = std::sqrt(3.14159265358979323846 / 2.0) / sd;",
     [Q + "test_decode_forms_agree_and_match_bruteforce"]),
    ("Decode: softmax scale dropped",
     "sc[t] = scale * dot;", "sc[t] = dot;",
     [Q + "test_decode_forms_agree_and_match_bruteforce"]),
    ("Decode: query head h read against kv head h % Hkv (GQA grouping)",
     "hq = (int)(bh % Hq), hk = hq / G;", "hq = (int)(bh % Hq), hk = hq % Hkv;",
     [Q + "test_decode_forms_agree_and_match_bruteforce"]),
    ("Decode (rotated form): value norm dropped",
     "acc[j] += p * n * P->cv[codes[j]] / sd;", "acc[j] += p * P->cv[codes[j]] / sd;",
     [Q + "test_decode_forms_agree_and_match_bruteforce"]),
    ("Decode (rotated form): un-rotated by R^T instead of R",
     "for (int j = 0; j < d; ++j) s += P->R[(size_t)i * d + j] * acc[j];",
     "for (int j = 0; j < d; ++j) s += P->R[(size_t)j * d + i] * acc[j];",
     [Q + "test_decode_forms_agree_and_match_bruteforce"]),
    ("Residual window: window scores not scaled",
     "sc[Tn + u] = scale * dot;", "sc[Tn + u] = dot;",
     [WIN + "test_window_matches_bruteforce"]),
]


def _compile(src_text: str, out: Path):
    cpp = out.with_suffix(".cpp")
    cpp.write_text(src_text)
    subprocess.run(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
                    str(cpp), "-o", str(out)], check=True, capture_output=True)


def _run_pins(lib: Path, pins):
    env = dict(os.environ, TQ_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *pins],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


def _one(args):
    i, src, tmp, find, repl, pins = args
    lib = tmp / ("mutant%02d.so" % i if find is not None else "control.so")
    _compile(src if find is None else src.replace(find, repl), lib)
    return _run_pins(lib, pins)


def test_every_planted_mistake_fails_its_pin(tmp_path):
    src = SRC.read_text()
    for name, find, repl, _ in MUTANTS:
        assert src.count(find) == 1, "%s: the planted text must occur exactly once in the oracle" % name
        assert repl != find
    all_pins = sorted({p for m in MUTANTS for p in m[3]})
    jobs = [(-1, src, tmp_path, None, None, all_pins)]
    jobs += [(i, src, tmp_path, m[1], m[2], m[3]) for i, m in enumerate(MUTANTS)]
    with ThreadPoolExecutor(max_workers=max(2, min(8, os.cpu_count() or 2))) as ex:
        results = list(ex.map(_one, jobs))
    rc, out = results[0]
    assert rc == 0, "the unmutated oracle must pass every pin used here:\n" + out
    # caught = a pin's assertion failed (pytest exit status 1, "failed" in its summary
    # line and no collection or setup error)
    survived = []
    for i, (rc, out) in enumerate(results[1:]):
        summary = out.strip().splitlines()[-1] if out.strip() else ""
        if not (rc == 1 and " failed" in summary and "error" not in summary):
            survived.append((MUTANTS[i][0], rc, summary))
    assert not survived, "planted mistakes that no pin caught (or that broke the run): %s" % survived
