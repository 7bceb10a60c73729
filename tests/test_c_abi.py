"""The C ABI from plain C: tests/c_abi_host.c is compiled as C99 against include/mla.h, linked
against the in-tree libmla.so and run (host-only calls, no GPU).  Every value it prints must
agree with the Python binding of the same call and, for the ring slots without a sink, with the
oracle's definition of the frame ring."""
import os
import shutil
import subprocess
import tempfile

import pytest

from mla_latent_kv_window_b200 import binding as B
from oracle import ring_slot

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mla_latent_kv_window_b200")


@pytest.fixture(scope="module")
def c_output(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    B.load_library()   # raises if libmla.so is not built
    exe = str(tmp_path_factory.mktemp("c_abi") / "c_abi_host")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_host.c"),
                    "-L", PKG, "-lmla", "-Wl,-rpath," + PKG, "-o", exe], check=True)
    run = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=60)
    out = {}
    for line in run.stdout.splitlines():
        key, *vals = line.split()
        out[key] = vals
    return out


def wan(sink_frames=0, **over):
    import mla_synth
    d = dict(mla_synth.DIMS_WAN13B)
    d.update(over)
    return B.make_config(d, frame_h=30, frame_w=52, window_frames=21, max_chunk_frames=3, batch=1,
                         sink_frames=sink_frames)


def test_config_checks_from_c(c_output):
    assert int(c_output["check_wan"][0]) == 0 == B.mla_config_check(wan())
    assert int(c_output["check_odd_rope"][0]) == 1 == B.mla_config_check(wan(rope_t=7, rope_h=13))
    assert int(c_output["check_latent_128"][0]) == 2 == B.mla_config_check(wan(d_latent=128))
    assert int(c_output["check_null"][0]) == 1


def test_sizes_from_c(c_output):
    assert int(c_output["ring_bytes"][0]) == 21 * 1560 * 224 * 2 == B.mla_ring_bytes(wan())
    assert int(c_output["device_bytes"][0]) == B.mla_cache_device_bytes(wan())


def test_ring_slots_from_c(c_output):
    slots = {k: v for k, v in c_output.items() if k.startswith("slot_") and k != "slot_bad_token"}
    assert len(slots) == 2 * 8 * 4
    for key, (status, slot) in slots.items():
        _, sink, frame, token = key.split("_")
        sink, frame, token = int(sink), int(frame), int(token)
        assert int(status) == 0
        assert int(slot) == B.mla_ring_slot(wan(sink), frame, token), key
        if sink == 0:
            assert int(slot) == ring_slot(frame, token, 21, 1560), key


def test_errors_from_c(c_output):
    status, has_message = c_output["slot_bad_token"]
    assert int(status) == 1 and int(has_message) == 1
    assert c_output["status_name_0"] == ["MLA_OK"]
    assert c_output["status_name_5"] == ["MLA_ERR_DEVICE_TIMEOUT"]


def test_full_path_client_compiles_and_links():
    """tests/c_abi_rollout.c drives create / append / attention / sync / destroy from C with
    device buffers of the CUDA runtime; here it must compile and link against libmla.so (it
    needs a GPU to run)."""
    gcc = shutil.which("gcc")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    if gcc is None or not os.path.exists(os.path.join(cuda, "include", "cuda_runtime_api.h")):
        pytest.skip("no C compiler or CUDA headers")
    B.load_library()
    exe = os.path.join(tempfile.mkdtemp(), "c_abi_rollout")
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c_abi_rollout.c"),
                    "-L", PKG, "-lmla", "-L", os.path.join(cuda, "lib64"), "-lcudart", "-lm",
                    "-Wl,-rpath," + PKG, "-o", exe], check=True)
    assert os.path.getsize(exe) > 0
