"""The debug build, libw8a8_debug.so: the same sources with device-side index
checks that record W8A8_ERR_DEVICE_BOUNDS and skip the access instead of
faulting (the substitute for a memory checker on this GPU pool).

Its self-test check (one index one past the end, no memory touched) must be
reported; then a representative set of the library's calls (every forward
kernel form, input gradients, the chain epilogue, the quantizers, Q8_0,
requants, weight-only types, SVDQuant) must run with no check failing and
give the release build's results bit for bit.  The checked library runs in a
child process (the binding loads one library per process)."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, torch
sys.path.insert(0, %(root)r); sys.path.insert(0, %(tests)r)
import w8a8_quantized_linear_b200 as w8
import _debug_calls
assert w8.debug_checks(), "the child must load the checked library"
assert w8.device_status() == 0
out = _debug_calls.run_all(w8, "cuda:0")
st = w8.device_status()
assert st == 0, "an index check failed: %%s" %% w8.lib().w8a8_last_error()
w8.selftest_bounds()
st = w8.device_status()
assert st == 8, st                      # W8A8_ERR_DEVICE_BOUNDS
assert b"0xbfff" in w8.lib().w8a8_last_error()
assert w8.device_status() == 0          # cleared by the read
torch.save(out, %(path)r)
print("debug child ok", len(out))
'''


def test_debug_build_runs_clean_and_matches_release(tmp_path):
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w8a8_quantized_linear_b200 import _build
    _build.build()
    _build.build(debug=True)
    path = str(tmp_path / "debug_out.pt")
    env = dict(os.environ, W8A8_LIBRARY="debug")
    code = CHILD % {"root": ROOT, "tests": os.path.join(ROOT, "tests"), "path": path}
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import _debug_calls
    import w8a8_quantized_linear_b200 as w8
    assert not w8.debug_checks()
    w8.selftest_bounds()
    assert w8.device_status() == 0          # the release build has no checks
    want = _debug_calls.run_all(w8, "cuda:0")
    got = torch.load(path)
    assert list(got) == list(want)
    for k in want:
        assert torch.equal(got[k], want[k]), k
