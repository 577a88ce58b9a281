"""The encode step of the quantize kernels over every fp32 bit pattern of a range.

Each quantize kernel turns x / s (fp32) into a code by one helper: round to nearest
even, saturating to +-F_max ([FFS] "Scale 怎样把 Tensor 塞进 E4M3": X_fp8 =
cast(clip(X / s))).  The testing entry point fp8_testing_encode_f32_range applies that
helper to the fp32 values first, first + 1, ... (by bit pattern).  Here every pattern
from +0 up to twice F_max, and the same magnitudes negative, goes through it and is
compared byte for byte with the oracle's clip-then-encode (quant_scaled with s = 1):
about 2.3e9 values for E4M3 and 2.4e9 for E5M2, every rounding midpoint, the fp32
subnormals, both zeros and the saturation range included.  The chunks are generated on
the device, so no input array is held."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
import fp8_dynamic_scaled_b200.binding as fp8  # noqa: E402

CHUNK = 1 << 26
F_MAX = {fp8.FP8_E4M3: 448.0, fp8.FP8_E5M2: 57344.0}


def f32_bits(x: float) -> int:
    return int(np.array([x], np.float32).view(np.uint32)[0])


@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2])
@pytest.mark.parametrize("negative", [False, True])
def test_encode_every_fp32_pattern_up_to_twice_fmax(fmt, negative):
    top = f32_bits(2.0 * F_MAX[fmt])               # every magnitude from +0 to 2 F_max
    sign = 0x80000000 if negative else 0
    q = torch.empty(CHUNK, dtype=torch.uint8, device="cuda")
    checked = 0
    for start in range(0, top + 1, CHUNK):
        n = min(CHUNK, top + 1 - start)
        fp8.fp8_testing_encode_f32_range(sign + start, q[:n], fmt)
        got = q[:n].cpu().numpy()
        bits = np.arange(start, start + n, dtype=np.uint32)
        if negative:
            bits |= np.uint32(sign)
        want = oracle.quant_scaled(bits.view(np.float32), 1.0, fmt)
        if not np.array_equal(got, want):
            i = int(np.flatnonzero(got != want)[0])
            pytest.fail(f"fmt {fmt}: pattern {int(bits[i]):#010x} ({float(bits[i:i + 1].view(np.float32)[0])!r}) "
                        f"-> {int(got[i]):#04x}, oracle {int(want[i]):#04x}")
        checked += n
    assert checked == top + 1


def test_encode_range_argument_errors():
    q = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_testing_encode_f32_range(0xFFFFFFF8, q, fp8.FP8_E4M3)     # past 2^32
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_testing_encode_f32_range(0, q, 7)
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG
    fp8.fp8_testing_encode_f32_range(0, q[:0], fp8.FP8_E4M3)                # nothing to do
