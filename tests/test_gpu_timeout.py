"""The bounded-wait path on the GPU: a kernel whose wait runs out records
GDR_ERR_TIMEOUT in the device status word, returns normally, the host reads
the status through gdr_check_status, and the context keeps working.  No
fault, trap or hang is involved: the wait is on a barrier nothing arrives on,
with a 50 ms bound."""
import ctypes

import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import synth
from gpu_common import dev

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    L = gdr.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    gdr.check_status()  # clean to start with
    gdr.check(L.gdr_debug_wait_timeout(50, s))
    st = L.gdr_check_status(s)
    assert st == gdr.GDR_ERR_TIMEOUT
    assert L.gdr_check_status(s) == gdr.GDR_OK  # read-and-clear
    x = synth.gdr_inputs(1, 70, 2, 128, 128, "bf16", seed=3)
    o, _ = gdr.gdr_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]), dev(x["beta"]))
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    gdr.check_status()
