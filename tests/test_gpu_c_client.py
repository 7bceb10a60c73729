"""GPU: the plain C client of the whole path (tests/c_abi_rollout.c) runs a 5-frame rollout of a
small layer through libmla.so - create, append, attention, commit, sync, destroy, with device
buffers of the CUDA runtime - and writes its host-generated inputs and its outputs; the fp64
oracle replays the same rollout on those inputs and every output element must match."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from oracle import OracleLayer
from tests.harness import assert_close

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mla_latent_kv_window_b200")


def _load(d, name, shape):
    raw = np.fromfile(os.path.join(d, name + ".bin"), dtype=np.uint16)
    return torch.from_numpy(raw.astype(np.int16)).view(torch.bfloat16).reshape(shape)


def test_c_client_rollout_matches_oracle(tmp_path):
    gcc = shutil.which("gcc")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    if gcc is None:
        pytest.skip("no C compiler")
    from mla_latent_kv_window_b200 import load_library
    load_library()
    exe = str(tmp_path / "c_abi_rollout")
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c_abi_rollout.c"),
                    "-L", PKG, "-lmla", "-L", os.path.join(cuda, "lib64"), "-lcudart", "-lm",
                    "-Wl,-rpath," + PKG, "-o", exe], check=True)
    dump = tmp_path / "dump"
    dump.mkdir()
    r = subprocess.run([exe, str(dump)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "frames_appended 5 valid_frames 2 non_finite 0" in r.stdout

    d, nh, F = 1536, 12, 24
    shapes = {"w_q": (nh * 128, d), "w_qr": (nh * 32, d), "w_dkv": (192, d), "w_kr": (32, d),
              "w_uk": (nh * 128, 192), "w_uv": (nh * 128, 192), "w_o": (d, nh * 128)}
    wts = {k: _load(dump, k, s) for k, s in shapes.items()}
    dims = dict(hidden=d, n_heads=nh, d_head=128, d_nope=128, d_latent=192, d_rope=32, rope_t=8,
                rope_h=12, rope_w=12, rope_base=10000.0, frame_h=4, frame_w=6, window_frames=2)
    orc = OracleLayer(dims, wts)
    for frame in range(5):
        x = _load(dump, f"x{frame}", (F, d))
        if frame > 0:
            got = _load(dump, f"out{frame}", (F, d))
            assert_close(got, orc.attention(x), f"C client, frame {frame}")
        orc.append(x)
