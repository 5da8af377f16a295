"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in a temporary copy of the oracle (never in the
repository's file), runs the pin suites against that copy in a subprocess and
requires them to fail. A mutation that survives means a gap in the pins.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle", "gdr_oracle.py")
PIN_FILES = ["test_oracle_pins.py", "test_oracle_rounding_and_gate.py"]

DECAY = "S = S * np.exp(g_t)[:, None, None] * np.exp(gk[b, :, t, :])[:, :, None]"
READ = 'kv_mem = np.einsum("hij,hi->hj", S, k_t)'
DELTA = "delta = (v_t - kv_mem) * beta_t[:, None]"
OUTL = 'out[b, :, t, :] = rnd_out(np.einsum("hij,hi->hj", S, q_t))'
UPD = "S = S + k_t[:, :, None] * delta[:, None, :]"

# (name, [(old, new), ...]) - every `old` must occur in the oracle source.
MUTATIONS = [
    ("tokens_capped_at_eight", [("for t in range(L):", "for t in range(min(L, 8)):")]),
    ("decay_without_gk", [(DECAY, "S = S * np.exp(g_t)[:, None, None]")]),
    ("decay_without_g", [(DECAY, "S = S * np.exp(gk[b, :, t, :])[:, :, None]")]),
    ("read_before_decay", [(DECAY, "S_prev = S\n            " + DECAY),
                           (READ, 'kv_mem = np.einsum("hij,hi->hj", S_prev, k_t)')]),
    ("delta_sign", [(DELTA, "delta = (kv_mem - v_t) * beta_t[:, None]")]),
    ("beta_on_memory_only", [(DELTA, "delta = v_t - kv_mem * beta_t[:, None]")]),
    ("output_before_update", [(UPD, "S_dec = S\n            " + UPD),
                              (OUTL, 'out[b, :, t, :] = rnd_out(np.einsum("hij,hi->hj", '
                                     'S_dec, q_t))')]),
    ("output_reads_key_not_query", [(OUTL, 'out[b, :, t, :] = rnd_out(np.einsum("hij,hi->hj", '
                                           'S, k_t))')]),
    ("update_transposed_roles", [(UPD, "S = S + q_t[:, :, None] * delta[:, None, :]")]),
    ("gqa_modulo", [("hq = np.arange(H_v) // group", "hq = np.arange(H_v) % H_qk")]),
    ("scale_missing", [("q_t = query[b, hq, t, :] * scale_value",
                        "q_t = query[b, hq, t, :]")]),
    ("scale_on_key_too", [("k_t = key[b, hq, t, :]  #",
                           "k_t = key[b, hq, t, :] * scale_value  #")]),
    ("state_rounded_every_token", [(OUTL, OUTL + "\n            S = bf16_round(S)")]),
    ("lengths_ignored", [("L = int(min(max(asl[b], 0), T))", "L = T")]),
    ("committed_count_ignored", [("if t == n - 1:", "if t == L - 1:")]),
    ("committed_one_token_late", [("if t == n - 1:", "if t == n:")]),
    ("bad_slot_wraps", [("s = int(idx[b])", "s = int(idx[b]) % P")]),
    ("softplus_no_linear_part", [("return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))",
                                  "return np.log1p(np.exp(-np.abs(x)))")]),
    ("sigmoid_sign", [("return np.where(x >= 0.0, 1.0 / (1.0 + z), z / (1.0 + z))",
                       "return np.where(x >= 0.0, z / (1.0 + z), 1.0 / (1.0 + z))")]),
    ("gate_without_dt_bias", [("decay = decay_scale * softplus(a + dt_bias)\n    beta = None",
                               "decay = decay_scale * softplus(a)\n    beta = None")]),
    ("bf16_truncates", [("np.rint(scaled)", "np.trunc(scaled)")]),
    ("bf16_seven_bits", [("_BF16_SIG_BITS = 8", "_BF16_SIG_BITS = 7")]),
    ("bf16_no_subnormal_floor", [("e_eff = np.maximum(e - 1, _BF16_MIN_NORMAL_EXP)",
                                  "e_eff = e - 1")]),
]


def _run_pins_against(mutated_source: str, workdir: str) -> int:
    os.makedirs(os.path.join(workdir, "oracle"))
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), os.path.join(workdir, "oracle"))
    with open(os.path.join(workdir, "oracle", "gdr_oracle.py"), "w") as f:
        f.write(mutated_source)
    shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(workdir, "tests"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           *[os.path.join(workdir, "tests", p) for p in PIN_FILES]]
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
    return subprocess.run(cmd, cwd=workdir, env=env, capture_output=True, timeout=600).returncode


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with open(ORACLE) as f:
        src = f.read()
    jobs = []
    for name, edits in MUTATIONS:
        mutated = src
        for old, new in edits:
            assert mutated.count(old) == 1, f"{name}: target not found once: {old!r}"
            mutated = mutated.replace(old, new)
        jobs.append((name, mutated, str(tmp_path / name)))
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        codes = list(ex.map(lambda j: _run_pins_against(j[1], j[2]), jobs))
    survivors = [name for (name, _, _), rc in zip(jobs, codes) if rc == 0]
    assert not survivors, f"mutations not caught by any pin: {survivors}"


def test_unmutated_copy_passes(tmp_path):
    with open(ORACLE) as f:
        src = f.read()
    assert _run_pins_against(src, str(tmp_path / "clean")) == 0
