"""The device-side timeout path, made to run out on purpose without faulting or hanging anything.

Every wait in the GEMM kernels is bounded: past its time limit (NVFP4_WAIT_TIMEOUT_MS, 1 s by default) a
role gives up, records NVFP4_ERR_DEVICE_TIMEOUT in the library's sticky device word and leaves the kernel
cleanly (its copies drained, TMEM freed).  The test build of the library (libnvfp4_testhooks.so, the same
sources compiled with NVFP4_TEST_HOOKS) has a switch that makes the first unit of every split-K tile park
its partial sum without publishing it, so the second unit's poll of the ready bit waits for a flag that
nothing sets.  The test runs in a child process with a 100 ms wait limit and checks that the call
reports the timeout, that the next ordinary call on the same context gives the earlier bits and a clean
status, and that nothing else went wrong.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import ctypes, sys
sys.path.insert(0, {root!r})
import torch
from epilogue_gemm_nvfp4_b200 import binding as B
from epilogue_gemm_nvfp4_b200 import build as BLD
from epilogue_gemm_nvfp4_b200 import workloads as W

B.LIB_PATH = BLD.TEST_LIB
lib = B.load()
lib.nvfp4_test_withhold_split_ready.argtypes = [ctypes.c_int32]
lib.nvfp4_test_withhold_split_ready.restype = None
torch.cuda.set_device(0)
for kind, N in (("bias", 256), ("bias", 384)):   # CTA pairs, then 128-wide tiles on single CTAs
    case = W.case_bias(130, N, 32768, seed=N, w_std=0.005, x_dist="student_t")
    assert B.split_k(N, 32768, kind) == 2
    aq, wq = B.quantize(case.x.cuda()), B.quantize(case.w.cuda())
    bias = case.bias.cuda()
    ref = B.linear(aq, wq, kind, bias=bias)
    clean = B.get_device_error()
    lib.nvfp4_test_withhold_split_ready(1)
    B.linear(aq, wq, kind, bias=bias)
    timed_out = B.get_device_error()
    lib.nvfp4_test_withhold_split_ready(0)
    again = B.linear(aq, wq, kind, bias=bias)
    after = B.get_device_error()
    torch.cuda.synchronize()
    print("RESULT", N, clean, timed_out, after, int(torch.equal(again, ref)), flush=True)
"""


def test_split_k_wait_runs_out_and_reports_a_device_timeout(tmp_path):
    script = tmp_path / "timeout_child.py"
    script.write_text(CHILD.format(root=ROOT))
    env = dict(os.environ, NVFP4_WAIT_TIMEOUT_MS="100")
    res = subprocess.run([sys.executable, str(script)], env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    from epilogue_gemm_nvfp4_b200 import binding as B
    results = [line.split()[1:] for line in res.stdout.splitlines() if line.startswith("RESULT")]
    assert len(results) == 2, res.stdout + res.stderr
    for n, clean, timed_out, after, same in results:
        assert int(clean) == B.OK, (n, clean)
        assert int(timed_out) == B.ERR_DEVICE_TIMEOUT, (n, timed_out)
        assert int(after) == B.OK, (n, after)
        assert same == "1", n
