"""The library on every device of one process, and from fresh host threads.

Kernel attributes (the opt-in to large dynamic shared memory) belong to one
device's context, so the library sets them per (kernel, device).  This runs
the whole path (lengths, flags, lists, forward, backward) on each visible
device in turn from one process, and on device 0 from two fresh threads,
and checks that every run gives the first run's results bit for bit."""
import threading

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gsa():
    from content_adaptive_block_b200 import build
    build.build()
    import content_adaptive_block_b200 as g
    return g


def _path(gsa, dev):
    wl = W.WORKLOADS["b8_4k"]
    x = torch.from_numpy(W.batch_bytes(wl)[:2]).to(dev)
    hc = [int(c) for c in wl.head_classes()]
    lengths = gsa.gsa_block_lengths(x, wl.b)
    flags = gsa.gsa_literal_flags(lengths)
    csr = gsa.gsa_build_block_csr(flags, wl.w)
    q, k, v, do = (t[:2].contiguous() for t in W.qkv(wl, seed=4, device=dev, grad=True))
    outs = []
    for d in (64, 128):
        qd, kd, vd, dod = (t[..., :d].contiguous() if d == 64 else torch.cat([t, t], -1) for t in (q, k, v, do))
        o, lse = gsa.gsa_attn_fwd(qd, kd, vd, csr, hc, wl.b)
        outs += [o, lse, *gsa.gsa_attn_bwd(qd, kd, vd, o, lse, dod, csr, hc, wl.b)]
    torch.cuda.synchronize(dev)
    return [t.cpu() for t in [lengths, flags] + outs]


def test_every_device_and_fresh_threads(gsa):
    ref = _path(gsa, torch.device("cuda", 0))
    assert gsa.gsa_device_error() == 0
    for i in range(1, torch.cuda.device_count()):
        with torch.cuda.device(i):
            got = _path(gsa, torch.device("cuda", i))
            assert gsa.gsa_device_error() == 0
        for a, b in zip(got, ref):
            assert torch.equal(a, b), i

    results, errors = [], []

    def worker():
        try:
            torch.cuda.set_device(0)
            results.append(_path(gsa, torch.device("cuda", 0)))
        except Exception as e:  # reported below
            errors.append(repr(e))

    for _ in range(2):
        t = threading.Thread(target=worker)
        t.start()
        t.join()
    assert not errors, errors
    for got in results:
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
