"""The failure path of the bounded device-side waits, made to run on purpose.

lh_selftest_wait_timeout enqueues one CTA that waits, through the same
bounded mbarrier wait as the tcgen05 attention kernels, on a barrier that
nothing signals.  The wait must give up by itself (about 2 s), the kernel
must return, lh_device_status must report LH_ERR_TIMEOUT once and then be
clear, and the CUDA context must stay usable.  Nothing here faults, traps or
hangs the GPU: the wait is bounded by the kernel's own cycle budget.
"""
import pytest
import torch

from long_context_hierarchical_b200.synth import make_inputs
from tests.helpers import assert_close, np64

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_timeout():
    from long_context_hierarchical_b200 import lh
    lh.device_status(reset=True)  # start from a clear status word
    lh.selftest_wait_timeout()
    with pytest.raises(lh.LighthouseError) as e:
        lh.device_status(reset=True)
    assert e.value.status == lh.LH_ERR_TIMEOUT
    lh.device_status()  # the reset cleared it
    # the context still runs the attention kernels, whose waits now all succeed
    Q, K, V, _ = make_inputs(1, 2, 256, 64, "bf16", seed=1, device="cuda", with_grad=False)
    O, lse = lh.attn_fwd(Q, K, V)
    ref = torch.nn.functional.scaled_dot_product_attention(Q.float(), K.float(), V.float(),
                                                           is_causal=True)
    assert_close(np64(O), np64(ref), torch.bfloat16, "O vs SDPA")
    lh.device_status()
