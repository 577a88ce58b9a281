"""The unsupported-device path on a B200.

Every entry point that launches work first asks the device gate whether the current
device is compute capability 10.x ([FRLP] section "5.2": a preflight rejects hardware
the path does not support).  A child process started with FP8_B200_FORCE_CC_MAJOR=9
sees a Hopper-class major in the gate: fp8_device_check and every compute entry point
must return FP8_ERR_UNSUPPORTED_DEVICE without launching anything (their outputs stay
as they were).  With the override at 10 or malformed, the calls go through."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json
import torch
import fp8_dynamic_scaled_b200.binding as fp8

R, E4 = fp8.FP8_SCALE_ROW, fp8.FP8_E4M3


def status(fn):
    try:
        fn()
        return 0
    except fp8.FP8Error as e:
        return e.status


res = {"check": fp8.fp8_device_check()}
x = torch.ones((128, 256), dtype=torch.bfloat16, device="cuda")
q, s, _ = fp8.empty_quant_outputs(128, 256, R)
q.fill_(7)
w = torch.zeros((256, 256), dtype=torch.uint8, device="cuda")
ws = torch.ones(256, device="cuda")
y = torch.full((128, 256), 3.0, dtype=torch.bfloat16, device="cuda")
lws = fp8.workspace_for(2, 128, 256, 256, R)
res["quantize"] = status(lambda: fp8.fp8_quantize(x, E4, R, q, s))
torch.cuda.synchronize()
res["q_untouched"] = bool((q == 7).all().item())
res["gemm"] = status(lambda: fp8.fp8_scaled_gemm(q, s, R, E4, w, ws, R, E4, y))
res["weight_only"] = status(lambda: fp8.fp8_weight_only_linear(x[:4], w, ws, R, E4, y[:4]))
res["linear"] = status(lambda: fp8.fp8_linear_forward(x, E4, R, w, ws, R, E4, y, lws))
torch.cuda.synchronize()
res["y_untouched"] = bool((y == 3.0).all().item())
print(json.dumps(res))
'''


def run_child(value):
    env = dict(os.environ)
    env["FP8_B200_FORCE_CC_MAJOR"] = value
    out = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_forced_older_device_is_refused_everywhere():
    import fp8_dynamic_scaled_b200.binding as fp8
    r = run_child("9")
    for k in ("check", "quantize", "gemm", "weight_only", "linear"):
        assert r[k] == fp8.FP8_ERR_UNSUPPORTED_DEVICE, (k, r)
    assert r["q_untouched"] and r["y_untouched"], r


@pytest.mark.parametrize("value", ["10", "not-a-number"])
def test_blackwell_or_malformed_override_goes_through(value):
    r = run_child(value)
    for k in ("check", "quantize", "gemm", "weight_only", "linear"):
        assert r[k] == 0, (k, r)
    assert not r["q_untouched"] and not r["y_untouched"], r
