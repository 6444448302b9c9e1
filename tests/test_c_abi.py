"""The library through its C ABI alone: tests/c_abi_host.c is compiled as C99
against include/pv.h with gcc (-Wall -Wextra -Werror), linked with libpv.so,
and run; it calls the host-only entry points (sizes, the stream state
machine, the attention plan, the sigma schedule) and prints the results,
which are checked here against closed forms and the pages' printed values.
No GPU is needed."""
import os
import shutil
import subprocess

import pytest

from golden_io import load

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "same_step_kv_b200")


@pytest.fixture(scope="module")
def output(tmp_path_factory):
    if not os.path.exists(os.path.join(LIBDIR, "libpv.so")):
        pytest.fail("libpv.so is not built")
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.fail("gcc is not available")
    exe = str(tmp_path_factory.mktemp("cabi") / "cabi")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_host.c"), "-o", exe, "-L", LIBDIR, "-l:libpv.so",
                    f"-Wl,-rpath,{LIBDIR}"], check=True, capture_output=True, text=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    out = {}
    for line in run.stdout.splitlines():
        key, _, rest = line.partition(" ")
        out[key] = rest.split()
    return out


def test_header_and_library_from_c(output):
    assert output["failures"] == ["0"]
    assert output["version"][0] == "pv"


def test_store_size_closed_form(output):
    # K and V regions: 2 x layers x steps x streams x H x (F0 + R) x T x D bf16
    assert int(output["kv_bytes"][0]) == 2 * 30 * 4 * 1 * 24 * (3 + 18) * 880 * 128 * 2


def test_state_machine_at_chunk_28(output):
    g = load("profile_geometry.txt")
    phase, chunk, fill, slot, frame0, n_keys = (int(x) for x in output["state"])
    R = g["recent_chunks_in_history"]
    assert chunk == g["chunks_per_generation"] - 1
    assert (fill, slot) == (min(chunk, R), (chunk - 1) % R)
    assert frame0 == g["first_chunk_latent_frames"] - 1 + chunk
    assert n_keys == (g["first_chunk_latent_frames"] + R) * 40 * 22
    assert phase == 3


def test_misuse_is_a_status(output):
    status, has_message = (int(x) for x in output["misuse"])
    assert status != 0 and has_message == 1


def test_plan_of_the_steady_chunk(output):
    grid, mode, r37, total = (int(x) for x in output["plan"])
    assert (grid, mode, total) == (148, 0, 24 * 4 * 145)
    assert r37 == 37 * total // grid


def test_sigma_schedule_printed_timesteps(output):
    g = load("shift_schedule.txt")
    assert [int(x) for x in output["timesteps"]] == [g[f"t{i}"] for i in range(6)]
    assert float(output["sigma_end"][0]) == 0.0
