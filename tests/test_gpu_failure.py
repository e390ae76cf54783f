"""Failure detection on the GPU without a fault: the prefill kernel bounds
every wait, so a K tile that never arrives makes its waits run out (~2 s),
the launch records FATTN_ERR_TIMEOUT in the device status word and exits
cleanly, and the context stays usable for the next launch."""
import numpy as np
import pytest
import torch

from io_aware_exact_34_b200 import synth
from tests._compare import BF16_O_MAXABS, BF16_O_RELL2, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from io_aware_exact_34_b200 import build
    build.build()
    from io_aware_exact_34_b200 import fattn
    return fattn


def test_expired_wait_reports_timeout_and_context_survives(fl, oracle):
    q, k, v = synth.random_qkv(1, 2, 512, 512, 128, "bf16", seed=77)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    assert fl.fattn_device_status() == fl.FATTN_OK
    fl.fattn_debug_inject_stall(True)
    fl.attn_fwd(qd, kd, vd, causal=True)          # enqueues; the kernel times out inside
    assert fl.fattn_device_status() == fl.FATTN_ERR_TIMEOUT
    assert fl.fattn_device_status() == fl.FATTN_OK  # reading clears the word
    # the hook applies to one launch only; the next launch is correct
    o, lse = fl.attn_fwd(qd, kd, vd, causal=True)
    torch.cuda.synchronize()
    assert fl.fattn_device_status() == fl.FATTN_OK
    o_ref, lse_ref = oracle.attn(q, k, v, 128 ** -0.5, True)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, BF16_O_MAXABS, BF16_O_RELL2,
            label="after timeout")
    assert torch.cuda.current_stream().query() in (True, False)  # stream still usable
    x = torch.ones(4, device="cuda") * 2
    assert float(x.sum().item()) == 8.0 and np.isfinite(float(x.sum().item()))
