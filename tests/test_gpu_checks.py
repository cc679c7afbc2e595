"""The checked build (libmoe_checks.so, compiled with MOE_CHECKS=1): the small
parity cases pass in it with device status OK, and its checks turn an
inconsistent caller-supplied offsets table into MOE_ERR_DEVICE_CHECK.  Run in
a child process with MOE_LIB_VARIANT=checks, so this process keeps the normal
library."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_small_parity_cases_pass_in_the_checked_build():
    from routed_expert_layer_route_b200 import build
    build.build(checks=True)
    env = dict(os.environ, MOE_LIB_VARIANT="checks")
    sel = ("test_layer_small_all_tokens or test_decode_path_single_token or "
           "test_decode_path_few_tokens or "
           "test_layer_grouped_all_tokens or test_expert_ffn_grouped_per_slot or "
           "test_expert_ffn_and_combine_steps")
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(ROOT, "tests", "test_gpu_layer.py"),
           os.path.join(ROOT, "tests", "test_gpu_cascade.py"),
           os.path.join(ROOT, "tests", "test_gpu_checks_only.py"), "-k",
           sel + " or test_cascade or test_checked_build"]
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert out.returncode == 0, out.stdout[-3000:] + out.stderr[-2000:]
    summary = [l for l in out.stdout.splitlines() if l.strip()][-1]
    assert " passed" in summary and "skipped" not in summary, summary
