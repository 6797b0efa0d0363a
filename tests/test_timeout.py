"""The bounded pipeline waits give up with an error status instead of hanging.

A test build of the library (libmla_shortwait.so, built by
``build.build_short_wait``) lets the indexer kernel's pipeline waits run out
after 200 ns, far less than a TMA load takes, so that a normal call takes the
error path: the waiting thread records MLA_DEVERR_TIMEOUT in the caller's
error word and raises the CTA's abort flag, every other wait returns at once,
the copies and MMAs already in flight are waited for (with the normal 2 s
limit), TMEM is freed and the kernel returns. Nothing faults or hangs: the
same device then runs a normal-build call whose results match the oracle.

The indexer kernel is the one exercised: it is a single-CTA pipeline whose
in-flight work (TMA loads, MMAs) completes on its own barriers, so an abort
leaves nothing in flight when the CTA exits.
"""

import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def test_short_waits_report_timeout_and_device_stays_usable(libmla):
    from mla_latent_kv_26_b200 import build
    from mla_latent_kv_26_b200.workloads import indexer_inputs

    short = libmla.load_library(build.build_short_wait())
    dev = torch.device("cuda", torch.cuda.current_device())
    d = indexer_inputs(batch=4, q_len=1, heads=64, num_keys=20000, seed=81)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    desc = libmla.make_index_desc(batch=4, q_len=1, num_heads=64, num_keys=20000)
    out = torch.zeros(4, 1, 20000, dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream(dev)
    st = short.mla_index_scores(desc, g["q"].data_ptr(), g["q_s"].data_ptr(), g["k"].data_ptr(), g["k_s"].data_ptr(),
                                out.data_ptr(), err.data_ptr(), s.cuda_stream)
    assert st == libmla.MLA_OK
    torch.cuda.synchronize(dev)  # the kernel returned
    assert int(err.item()) & libmla.MLA_DEVERR_TIMEOUT
    # the device and the context are fine: the normal build computes correct scores
    err.zero_()
    out.zero_()
    assert libmla.mla_index_scores(desc, g["q"], g["q_s"], g["k"], g["k_s"], out, err, s) == libmla.MLA_OK
    torch.cuda.synchronize(dev)
    assert int(err.item()) == 0
    ref = oracle.index_scores(d["q"][:1], d["q_s"][:1], d["k"][:1], d["k_s"][:1])
    mag = oracle.index_scores(d["q"][:1].to(torch.float32).abs(), d["q_s"][:1].abs(), d["k"][:1].to(torch.float32).abs(),
                              d["k_s"][:1])
    assert ((out[:1].double().cpu() - ref).abs() <= 2.0 ** -9 * mag).all()
