"""The C ABI from C: include/mxa.h compiles as C, and a C program linked
against libmxa.so gets the same plans and refusals as the Python binding
(host-side calls only; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from decode_attention_packed_b200 import mxa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def abi_check(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("cabi") / "abi_check")
    lib_dir = os.path.dirname(mxa.LIBRARY)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c", "abi_check.c"), "-o", exe, "-L", lib_dir, "-lmxa",
                           "-Wl,-rpath," + lib_dir])
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return dict(line.split(" ", 1) for line in out.strip().splitlines())


def test_c_caller_gets_the_python_binding_plan(abi_check):
    p = mxa.mxa_decode_params_t(2, 1, 64, 8, 128, 512, 64, 256, 16384, mxa.MXA_BF16)
    plan = mxa.mxa_plan(p, 0, sm_count=148)
    want = (f"{mxa.MXA_OK} schedule {plan.schedule} grid {plan.grid} units {plan.units} unit_cost "
            f"{plan.unit_cost} combine {plan.needs_combine} ws {plan.workspace_bytes}")
    assert abi_check["plan"] == want
    u = mxa.mxa_plan(p, 4, sm_count=148)
    assert abi_check["uniform"] == f"{mxa.MXA_OK} schedule {u.schedule} grid {u.grid} splits {u.num_splits}"
    # mxa_decode_workspace_size agrees with the plan mxa_plan returns, and refuses num_splits < 0
    assert u.workspace_bytes > 0
    assert abi_check["wsize"] == f"{u.workspace_bytes} {u.workspace_bytes} 1"


def test_c_caller_gets_the_rules_and_refusals(abi_check):
    assert abi_check["pack"] == "1 0"
    assert abi_check["splits"] == (f"{mxa._lib.mxa_num_splits_heuristic(16, 148, 296, 128, 128, 0, 1, 8388608.0)} "
                                   f"{mxa._lib.mxa_num_splits_heuristic(256, 148, 296, 32, 64, 0, 1, 1048576.0)}")
    assert abi_check["unsupported"] == str(mxa.MXA_ERR_UNSUPPORTED)
    assert abi_check["no"].startswith(f"workspace {mxa.MXA_ERR_WORKSPACE} MXA_ERR_WORKSPACE")
