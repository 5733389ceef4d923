"""Device-side failure path of the tensor-core scan, exercised without a fault.

Every wait inside the scan kernel is bounded (2 s).  The test hook
kda_debug_drop_handoff makes each CTA's producer warps withhold their first "tiles
ready" signal, so the consumer's wait runs out: the kernel records a timeout in the
device status word, stops waiting, drains its own tensor-core and TMA work and exits.
The host must then read KDA_ERR_TIMEOUT, and the next call (hook off) must run
normally on the same context and match the oracle.
"""
import pytest
import torch

from linear_attention_sequence_mshortconv_b200 import kda
from oracle import oracle as O
from tests.parity import compare_heads, to_np
from tests.test_gpu_kda_parity import _custom

pytestmark = pytest.mark.gpu
KDA_ERR_TIMEOUT = 4


@pytest.mark.parametrize("H", [80, 4])   # 80 heads: one pass (P = 1); 4 heads: state + output passes
def test_bounded_wait_runs_out_reports_timeout_and_recovers(H):
    inp = _custom(1, 192, H, 128, 128, torch.bfloat16, seed=7 + H)
    t = {k: v.cuda() for k, v in inp.items()}
    assert kda.last_device_error() == 0
    kda.debug_drop_handoff(True)
    try:
        kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], o_dtype=torch.float32)
        torch.cuda.synchronize()
    finally:
        kda.debug_drop_handoff(False)
    assert kda.last_device_error() == KDA_ERR_TIMEOUT
    assert kda.last_device_error() == 0          # reading the word clears it

    o, ST = kda.forward(t["q"], t["k"], t["v"], t["g"], t["beta"], o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kda.last_device_error() == 0
    pairs = [(0, 0), (0, H - 1)]
    o_ref, S_ref = O.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], pairs=pairs)
    compare_heads(to_np(o), o_ref, to_np(ST), S_ref, "bf16", pairs=pairs, what="after a timeout")
