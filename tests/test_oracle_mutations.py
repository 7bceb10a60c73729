"""Strength of the oracle's pins.  Each plausible mistake below (a wrong sign, a dropped term, a
wrong index, a permuted operand, a bookkeeping slip) is planted in a copy of the oracle, on the
CPU, and tests/test_oracle_pins.py is run against that copy: at least one pin must fail.  A
control run of the unmodified copy must pass, so that a broken harness cannot pass for a
caught mistake.  The committed oracle is never modified."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle", "mla_oracle.py")

# (what the mistake is, text in the oracle, text it becomes)
MUTATIONS = [
    ("RoPE: sign of the sine in the imaginary part",
     "out[..., 1::2] = re * sn + im * cs", "out[..., 1::2] = -re * sn + im * cs"),
    ("RoPE: band frequencies shifted by one",
     "freqs.append(float(base) ** (-2.0 * i / d_a))", "freqs.append(float(base) ** (-2.0 * (i + 1) / d_a))"),
    ("RoPE: query height and width coordinates swapped",
     'q_rope = self._rope(xq @ self.W["w_qr"][h * dr:(h + 1) * dr].T, tq, hq, wq)',
     'q_rope = self._rope(xq @ self.W["w_qr"][h * dr:(h + 1) * dr].T, tq, wq, hq)'),
    ("keys lose their RoPE part",
     "K = np.concatenate([k_nope, k_rope], axis=1)", "K = np.concatenate([k_nope, 0 * k_rope], axis=1)"),
    ("positional key stored with the wrong sign",
     'r = x @ self.W["w_kr"].T\n        return c, r', 'r = x @ self.W["w_kr"].T\n        return c, -r'),
    ("softmax scale from d_nope alone",
     "1.0 / math.sqrt(dn + dr)", "1.0 / math.sqrt(dn)"),
    ("softmax normalised over the wrong axis",
     "S = S - S.max(axis=1, keepdims=True)\n            E = np.exp(S)",
     "S = S - S.max(axis=0, keepdims=True)\n            E = np.exp(S)"),
    ("value up-projection with its rows permuted",
     'v = ctx["c"] @ w_uv.T', 'v = ctx["c"] @ w_uv[::-1].T'),
    ("output projection with its columns permuted",
     'out = O.reshape(nq, nh * dv) @ self.W["w_o"].T', 'out = O.reshape(nq, nh * dv) @ self.W["w_o"][:, ::-1].T'),
    ("low-rank query down-projection with its rows permuted",
     'return x @ self.W["w_dq"].T if "w_dq" in self.W else x',
     'return x @ self.W["w_dq"][::-1].T if "w_dq" in self.W else x'),
    ("window-local temporal positions reversed",
     "t_of_frame = np.arange(len(frame_ids), dtype=np.float64)",
     "t_of_frame = np.arange(len(frame_ids), dtype=np.float64)[::-1].copy()"),
    ("the window evicts the wrong frame",
     'if len(self.frames) > self.d["window_frames"]:\n                self.frames.pop(0)',
     'if len(self.frames) > self.d["window_frames"]:\n                self.frames.pop(-2)'),
    ("frame index off by one at append",
     "            entry = (self.frames_appended, c[sl], r[sl])\n            self.frames_appended += 1",
     "            self.frames_appended += 1\n            entry = (self.frames_appended, c[sl], r[sl])"),
    ("sink frames never kept", "if len(self.sink) < self.n_sink:", "if len(self.sink) < self.n_sink and False:"),
    ("sink frames ordered after the window", "return self.sink + self.frames", "return self.frames + self.sink"),
    ("token grid transposed (column-major h, w)", "return k // frame_w, k % frame_w", "return k % frame_w, k // frame_w"),
    ("ring slot one frame ahead", "return (frame % window_frames) * tokens_per_frame + token",
     "return ((frame + 1) % window_frames) * tokens_per_frame + token"),
    ("RoPE axes in the order h, t, w", "for a, d_a in enumerate((rope_t, rope_h, rope_w)):",
     "for a, d_a in enumerate((rope_h, rope_t, rope_w)):"),
    ("ring contents rotated at the window-local index instead of the absolute one",
     "for f, c, r in self.active_frames():\n            out.append((f, c.copy(), self._rope(r, f, hh, ww)))",
     "for i, (f, c, r) in enumerate(self.active_frames()):\n            out.append((f, c.copy(), self._rope(r, i, hh, ww)))"),
    ("ring contents with h and w swapped", "out.append((f, c.copy(), self._rope(r, f, hh, ww)))",
     "out.append((f, c.copy(), self._rope(r, f, ww, hh)))"),
    ("ring contents left unrotated", "out.append((f, c.copy(), self._rope(r, f, hh, ww)))",
     "out.append((f, c.copy(), r.copy()))"),
    ("ring contents one frame ahead in time", "out.append((f, c.copy(), self._rope(r, f, hh, ww)))",
     "out.append((f, c.copy(), self._rope(r, f + 1, hh, ww)))"),
    ("a head subset drops all but its first head", "for h in (range(nh) if heads is None else heads):",
     "for h in (range(nh) if heads is None else heads[:1]):"),
    ("dense baseline without the softmax scale", "S = (q[:, h, :] @ k[:, h, :].T) * scale",
     "S = (q[:, h, :] @ k[:, h, :].T)"),
    ("dense baseline normalising over queries", "out[:, h, :] = (E / E.sum(axis=1, keepdims=True)) @ v[:, h, :]",
     "out[:, h, :] = (E / E.sum(axis=0, keepdims=True)) @ v[:, h, :]"),
]

# Loads the given oracle source as the `oracle` package, then runs the pins in this process.
RUNNER = r"""
import importlib.util, sys, types
root, src = sys.argv[1], sys.argv[2]
sys.path.insert(0, root)
try:
    pkg = types.ModuleType("oracle")
    pkg.__path__ = []
    sys.modules["oracle"] = pkg
    spec = importlib.util.spec_from_file_location("oracle.mla_oracle", src)
    mod = importlib.util.module_from_spec(spec)
    sys.modules["oracle.mla_oracle"] = mod
    spec.loader.exec_module(mod)
    for name in dir(mod):
        if not name.startswith("_"):
            setattr(pkg, name, getattr(mod, name))
except Exception as e:
    print("could not load the oracle copy:", e)
    sys.exit(7)
import pytest
sys.exit(int(pytest.main([root + "/tests/test_oracle_pins.py", "-q", "-x", "-p", "no:cacheprovider"])))
"""


def _launch(tmp_path, name, source):
    path = tmp_path / f"{name}.py"
    path.write_text(source)
    env = dict(os.environ, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
    return subprocess.Popen([sys.executable, "-c", RUNNER, ROOT, str(path)], cwd=str(tmp_path), env=env,
                            stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)


def test_every_planted_mistake_fails_a_pin(tmp_path):
    original = open(ORACLE).read()
    procs = [("control", _launch(tmp_path, "control", original))]
    for i, (what, old, new) in enumerate(MUTATIONS):
        assert original.count(old) == 1, f"mutation anchor not found once: {what}"
        procs.append((what, _launch(tmp_path, f"mutant{i}", original.replace(old, new))))
    results = {}
    for what, p in procs:
        out, _ = p.communicate(timeout=600)
        results[what] = (p.returncode, out.strip().splitlines()[-1:] if out else [])
    assert results["control"][0] == 0, f"the unmodified oracle copy must pass its pins: {results['control']}"
    survivors = {w: r for w, r in results.items() if w != "control" and r[0] != 1}
    assert not survivors, f"mistakes no pin caught (exit 1 expected): {survivors}"
