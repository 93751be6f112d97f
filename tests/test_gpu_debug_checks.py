"""The range-checked build (libsdpa_debug.so, compiled with SDPA_DEBUG_CHECKS) on the GPU.

It stands in for a memory checker: every index the kernels take from data is checked on the
device, and a violation becomes SDPA_ERR_DEVICE_CHECK in the status word instead of an access.
The small parity files run once more in a child process that loads it (SDPA_DEBUG_CHECKS=1);
then a block classification whose row count was raised past its row is reported. That input
stays inside every buffer even unchecked (it reads the next row's list), so it cannot fault.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FILES = ["tests/test_gpu_prefill.py", "tests/test_gpu_generic_decode.py", "tests/test_gpu_packed.py"]


def test_small_parity_cases_pass_under_range_checks():
    env = dict(os.environ, SDPA_DEBUG_CHECKS="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *FILES,
           os.path.abspath(__file__) + "::test_corrupt_row_count_is_reported"]
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = "\n".join((res.stdout + res.stderr).splitlines()[-15:])
    assert res.returncode == 0, tail
    assert " passed" in res.stdout and "skipped" not in res.stdout.split("passed")[-1], tail


def test_corrupt_row_count_is_reported():
    import head_scaled_dot_sdpa_b200 as sdpa
    if not sdpa.DEBUG_CHECKS:
        pytest.skip("runs in the child process that loads the range-checked build")
    assert sdpa.lib.sdpa_debug_checks() == 1
    rng = np.random.Generator(np.random.PCG64(9))
    H, L, D = 1, 512, 128
    mask = torch.from_numpy((rng.random((H, L, L)) < 0.5).astype(np.uint8)).cuda()
    info = sdpa.build_block_mask_info(mask)
    q, k, v = (torch.from_numpy(rng.standard_normal((1, L, H, D), dtype=np.float32)).to(torch.bfloat16).cuda()
               for _ in range(3))
    ws = sdpa.Workspace("cuda")
    sdpa.sdpa_forward(q, k, v, block_info=info, workspace=ws)
    assert sdpa.read_device_status(ws) == sdpa.SDPA_OK
    count = info.arrays()["count"]
    count[0, 0] = info.struct.nkb + 1  # row 0 claims one more block than a row holds
    torch.cuda.synchronize()
    sdpa.sdpa_forward(q, k, v, block_info=info, workspace=ws)
    assert sdpa.last_kernel() == "prefill_tcgen05"
    assert sdpa.read_device_status(ws) == sdpa.SDPA_ERR_DEVICE_CHECK
