"""Failure path on the GPU without a fault: every wait inside the kernel is
bounded in time.  A test-only launch flag makes the TMA producer withhold
the first V block, so the MMA warp's bounded wait runs out; the kernel then
records a timeout in its status word, drains what it started, frees its
tensor memory and exits.  The checked entry reports VITATTN_ERR_TIMEOUT and
the CUDA context stays usable: the next call is correct."""
import numpy as np
import pytest

import oracle
from vit_bidirectional_attention_b200 import synth, vitattn

pytestmark = pytest.mark.gpu

SKIP_FIRST_V_LOAD = 1


def _dev(bits, dtype):
    import torch

    tdt = torch.bfloat16 if dtype == synth.BF16 else torch.float16
    return torch.from_numpy(bits.view(np.int16).copy()).view(tdt).cuda()


@pytest.mark.parametrize("dtype", [synth.BF16, synth.F16])
def test_withheld_block_times_out_and_context_survives(cuda_device, dtype):
    """bf16: the V converter's wait runs out first (or the MMA warp's, whose
    V-ready barrier the converter never signals); f16: the MMA warp's."""
    import torch

    q, k, v = synth.random_qkv(1, 64, 1, 64, dtype, seed=4001)
    tq, tk, tv = (_dev(x, dtype) for x in (q, k, v))
    out = torch.zeros_like(tq)
    s = torch.cuda.current_stream()
    rc = vitattn.forward_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(), 1, 64, 1,
                             64, 0.125, dtype, s.cuda_stream, flags=SKIP_FIRST_V_LOAD)
    assert rc == -8, vitattn.strerror(rc)
    # the context is intact: a normal checked call succeeds and is right
    rc = vitattn.forward_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(), 1, 64, 1,
                             64, 0.125, dtype, s.cuda_stream, checked=True)
    assert rc == 0, vitattn.strerror(rc)
    got = synth.bits_to_float32(out.view(torch.int16).cpu().numpy().view(np.uint16), dtype)
    ref = oracle.attention(q, k, v, 0.125, dtype)
    assert np.max(np.abs(got - ref)) <= 1e-2
