"""Failure handling of the decode kernel's bounded waits, without a GPU fault.

Every pipeline wait of the staged decode kernel is bounded in time; a wait that
runs out sets KQ_DEV_TIMEOUT in the library status word and the kernel winds
down, letting the copies it issued land, instead of hanging.  The test makes a
wait run out on purpose by shortening the limit to 1 ns (kq_set_wait_limit):
nothing is withheld and no kernel is altered, the first wait that is not
complete at its first poll simply runs out.  It runs on the q8_0 M=1 kernel,
which uses neither clusters nor tensor memory.  The context must stay usable:
the next call on the same stream is exact again."""
import numpy as np
import pytest
import torch

import gguf_quant_dequant_q4_b200 as kq
import oracle
import synth
from tests._util import check_qmv, dev_bf16, dev_u8

pytestmark = pytest.mark.gpu


def test_decode_wait_runs_out_and_next_call_is_exact():
    n, k = 14336, 4096
    w = synth.weights(kq.Q8_0, n, k)
    x = synth.activations(1, k)
    wd, xd = dev_u8(w), dev_bf16(x)
    torch.cuda.synchronize()
    kq.read_device_status(clear=True)
    try:
        kq.set_wait_limit(1)
        kq.qmv(xd, wd, kq.Q8_0)
        torch.cuda.synchronize()
        status = kq.read_device_status(clear=True)
    finally:
        kq.set_wait_limit(0)
    assert status & kq.DEV_TIMEOUT
    y = kq.qmv(xd, wd, kq.Q8_0).cpu().numpy()
    ref, absdot = oracle.matmul(kq.Q8_0, w, k, x, absdot=True)
    check_qmv(y, ref, absdot)
    assert kq.read_device_status(clear=True) == 0
