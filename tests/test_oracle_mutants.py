"""The oracle's pins catch planted slips.

Each case compiles a copy of oracle/pa_oracle.c with one plausible mistake
(an off-by-one window edge or query position, a dropped or misplaced scale,
a wrong GQA head map, K and V swapped, a wrong block slot, a wrong e4m3 bias
or subnormal exponent, an unweighted or truncated split-K merge, one q row
for every query token, a rounded-up dead-block count) and runs the pin suite
(tests/test_oracle_pins.py) against that build, on the CPU: every mutant must
fail it.  A control build of the unchanged source must pass it, so a failure
means the pins saw the slip, not that the harness broke.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "pa_oracle.c")
PINS = os.path.join(HERE, "test_oracle_pins.py")

MUTANTS = {
    "window_edge": ("start = end - window;", "start = end - window + 1;"),
    "query_position": ("int p = seq_len - query_len + i;", "int p = seq_len - query_len + i - 1;"),
    "dropped_scale": ("return pr->scale * acc;", "return acc;"),
    "gqa_head_map": ("int g = h / (pr->hq / pr->hkv);", "int g = h % pr->hkv;"),
    "k_v_swapped": ("kv_value(pr, pr->vc, v + x, pr->v_scale)", "kv_value(pr, pr->kc, v + x, pr->v_scale)"),
    "block_slot": ("int slot = t % pr->bs;", "int slot = (t + 1) % pr->bs;"),
    "e4m3_bias": ("else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
                  "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_subnormal": ("if (e == 0) v = ldexp((double)m / 8.0, -6);",
                       "if (e == 0) v = ldexp((double)m / 8.0, -7);"),
    "v_scale_dropped": ("kv_value(pr, pr->vc, v + x, pr->v_scale)", "kv_value(pr, pr->vc, v + x, 1.0)"),
    "k_scale_for_v": ("acc += q_value(pr, qrow + x) * kv_value(pr, pr->kc, k + x, pr->k_scale);",
                      "acc += q_value(pr, qrow + x) * kv_value(pr, pr->kc, k + x, pr->v_scale);"),
    "q_scale_dropped": ("if (pr->q_fp8) return pr->q_scale * e4m3_bits_to_double(",
                        "if (pr->q_fp8) return e4m3_bits_to_double("),
    "unweighted_merge": ("double wt = exp(lse[p] - mmax);", "double wt = 1.0;"),
    "split_union_short": ("    uhi = S;\n", "    uhi = S - 1;\n"),
    "one_q_row_per_row": ("    tok += (size_t)i;\n", ""),
    "normaliser_unshifted": ("for (int j = 0; j < n; ++j) z += exp(s[j] - m);",
                             "for (int j = 0; j < n; ++j) z += exp(s[j] - m) + 1e-3;"),
    "dead_blocks_rounded_up": ("count[b] = lowest / bs;", "count[b] = (lowest + bs - 1) / bs;"),
}


def _build(src_text, tmp_path, name):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", str(so),
                    str(c), "-lm"], check=True)
    return str(so)


def _run_pins(so):
    env = dict(os.environ, PA_ORACLE_LIB=so, OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q",
                           "-p", "no:cacheprovider"], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=900)


@pytest.fixture(scope="module")
def pin_runs(tmp_path_factory):
    """Every build's pin-suite run, the control's and each mutant's, run side
    by side in separate processes (each starts its own interpreter)."""
    from concurrent.futures import ThreadPoolExecutor
    tmp = tmp_path_factory.mktemp("mutants")
    src = open(SRC).read()
    sources = {"control": src}
    for name, (old, new) in MUTANTS.items():
        assert src.count(old) == 1, f"mutation site of {name} not found once"
        sources[name] = src.replace(old, new)
    libs = {name: _build(text, tmp, name) for name, text in sources.items()}
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        futures = {name: ex.submit(_run_pins, so) for name, so in libs.items()}
        return {name: f.result() for name, f in futures.items()}


def test_control_build_passes_the_pins(pin_runs):
    r = pin_runs["control"]
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pins_catch_a_planted_slip(name, pin_runs):
    r = pin_runs[name]
    # exit code 1: tests ran and at least one failed (not a collection error)
    assert r.returncode == 1 and " failed" in r.stdout, r.stdout[-3000:] + r.stderr[-2000:]
