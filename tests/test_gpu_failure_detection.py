"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every mbarrier wait in the library's kernels gives up after a cycle limit,
records a code in the per-device error word and unwinds, so a lost arrival
shows up on the host as VSA_ERR_DEVICE_TIMEOUT from vsa_device_status()
instead of a hung GPU.  vsa_wait_probe runs that path on purpose with a short
limit (a wait on an mbarrier nobody arrives at); the context must stay usable
and the next calls must succeed."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import content_adaptive_block_fractal_b200 as vsa
from content_adaptive_block_fractal_b200 import _lib, workloads

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported():
    L = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    _lib.check(L.vsa_device_status(stream))                 # start from a clear word
    _lib.check(L.vsa_wait_probe(1 << 21, stream))            # ~1 ms limit
    st = L.vsa_device_status(stream)
    assert st == 5, st                                       # VSA_ERR_DEVICE_TIMEOUT
    assert b"0x20" in L.vsa_last_error()
    # the word was cleared, and the context still works: a normal call is exact
    _lib.check(L.vsa_device_status(stream))
    wl = workloads.get("tiny")
    q, _, _ = workloads.make_qkv(wl)
    shape = vsa.Shape.of(wl)
    qf = vsa.fractal_flatten(q.cuda(), shape)
    _lib.check(L.vsa_device_status(stream))
    np.testing.assert_array_equal(oracle.as_u16(qf.cpu()), oracle.flatten(q, wl.T, wl.H, wl.W))


def test_two_probes_report_once():
    """Codes accumulate in the word until read; one status reports them all."""
    L = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    _lib.check(L.vsa_wait_probe(1 << 20, stream))
    _lib.check(L.vsa_wait_probe(1 << 20, stream))
    assert L.vsa_device_status(stream) == 5
    assert L.vsa_device_status(stream) == 0
