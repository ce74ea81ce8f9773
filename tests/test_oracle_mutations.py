"""The oracle's pins catch plausible mistakes (CPU).

Each case plants one mistake in a copy of the oracle (an exact source edit: a
dropped term, a wrong sign or index, a transposed operand), runs the pin tests
against that copy in a separate process, and requires them to fail. An
unmodified copy must pass, so a broken copy mechanism cannot make every mutant
look caught. The mistakes are planted in the oracle only, on the CPU.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "rmsnorm drops eps": ("return x / np.sqrt(ms + eps) * w", "return x / np.sqrt(ms) * w"),
    "rope sign": ("out[..., 0] = x0 * c - x1 * s", "out[..., 0] = x0 * c + x1 * s"),
    "rope frequency exponent": ("freqs = theta ** (-2.0 * i / head_dim)", "freqs = theta ** (-1.0 * i / head_dim)"),
    "mask off by one": ("future = k_pos[None, :] > q_pos[:, None]", "future = k_pos[None, :] >= q_pos[:, None]"),
    "gqa head map": ("        g = h // G\n", "        g = h % Hk\n"),
    "score scale": ("s = (q[:, h, :] @ k[:, g, :].T) / math.sqrt(d)", "s = (q[:, h, :] @ k[:, g, :].T) / d"),
    "layer swaps w1 and w3": ('silu(x @ w["w1"].T) * (x @ w["w3"].T)', 'silu(x @ w["w3"].T) * (x @ w["w1"].T)'),
    "ffn swaps w1 and w3": ("(silu(x @ w1.T) * (x @ w3.T)) @ w2.T", "(silu(x @ w3.T) * (x @ w1.T)) @ w2.T"),
    "wq transposed": ('q = (x[b] @ w["wq"].T)', 'q = (x[b] @ w["wq"])'),
    "wo transposed": ('h = h + out @ w["wo"].T', 'h = h + out @ w["wo"]'),
    "ffn norm dropped": ('x = self._norm_in(h, w["ffn_norm"])', 'x = h * w["ffn_norm"]'),
    "attention residual dropped": ('h = h + out @ w["wo"].T', 'h = out @ w["wo"].T'),
    "final norm dropped": ('x = self._norm_in(h[:, -1, :], f64(self.glob["norm"]))', "x = h[:, -1, :]"),
    "bf16 rounding keeps 9 bits": ("return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)",
                                   "return np.ldexp(np.rint(np.ldexp(m, 9)), e - 9)"),
    "bf16 rounding truncates": ("np.rint(np.ldexp(m, 8))", "np.trunc(np.ldexp(m, 8))"),
    "argmax ties to the highest index": ("return np.argmax(logits, axis=-1)",
                                         "return logits.shape[-1] - 1 - np.argmax(logits[..., ::-1], axis=-1)"),
}


def _run_pins(tree, mutation):
    for d in ("oracle", "seeded_inputs"):
        shutil.copytree(os.path.join(ROOT, d), tree / d, ignore=shutil.ignore_patterns("__pycache__"))
    (tree / "tests").mkdir()
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), tree / "tests" / f)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), tree / "tests" / "golden")
    if mutation is not None:
        src_path = tree / "oracle" / "__init__.py"
        src = src_path.read_text()
        old, new = mutation
        assert src.count(old) == 1, f"mutation site not unique or missing: {old!r}"
        src_path.write_text(src.replace(old, new))
    env = {k: v for k, v in os.environ.items() if k != "PYTHONPATH"}
    env["OMP_NUM_THREADS"] = "1"   # the copies run side by side
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-q", "-x", "-p", "no:cacheprovider"],
                       cwd=tree, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    """Exit code and output tail of the pins on the unmodified copy (key None) and
    on every mutant, run as independent processes side by side."""
    cases = [None] + sorted(MUTATIONS)
    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        futs = {name: ex.submit(_run_pins, tmp_path_factory.mktemp("tree"),
                                None if name is None else MUTATIONS[name]) for name in cases}
        return {name: f.result() for name, f in futs.items()}


def test_unmodified_copy_passes(results):
    rc, out = results[None]
    assert rc == 0, out


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(results, name):
    rc, out = results[name]
    assert rc == 1, f"{name}: pins still pass (exit {rc})\n{out}"
