"""GPU tests of the library's runtime behaviour: the bounded-wait path sets
the device status word without faulting, calls honour the caller's stream,
and repeated calls are deterministic."""
import numpy as np
import pytest

from gpu_util import dev, host, need_gpu
from w8a8_int8_quantized_qk_b200 import qk, synth

pytestmark = pytest.mark.gpu

import torch  # noqa: E402


def test_bounded_wait_reports_timeout():
    need_gpu()
    assert qk.device_status() == qk.QK_OK
    s = torch.cuda.current_stream()
    assert qk.qk_selftest_bounded_wait(20000, qk._stream(s)) == qk.QK_OK  # 20 ms
    assert qk.device_status() == qk.QK_ERR_TIMEOUT
    assert qk.device_status() == qk.QK_OK  # read clears it
    # the context is still usable afterwards
    x = torch.ones((4, 64), dtype=torch.bfloat16, device="cuda")
    q, sc = qk.quantize_per_token(x)
    torch.cuda.synchronize()
    assert int(q.min()) == 127


def test_side_stream_and_determinism():
    need_gpu()
    w = synth.make_linear(512, 1024, 2048, seed=9)
    x = dev(w.x.view(np.int16)).view(torch.bfloat16)
    wq, sw = dev(w.w_q), dev(w.sw)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out1 = qk.linear(x, wq, sw)
    s.synchronize()
    out2 = qk.linear(x, wq, sw)
    torch.cuda.synchronize()
    assert np.array_equal(host(out1), host(out2))
    assert qk.device_status() == qk.QK_OK
