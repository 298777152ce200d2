"""The device-timeout path of the attention kernel, exercised without a fault.

s2o_attention_bounded runs the planned-stop attention kernel with every
pipeline wait limited to a given number of polls.  With 0 polls every wait
gives up at once, so the call must report S2O_ERR_DEVICE_TIMEOUT; with a few
polls some waits give up while tensor-core products, Q tiles and gathers are
in flight.  Either way each CTA must wind down (wait for its own started
work, free its tensor memory, end) so that the next launch on every SM can
allocate tensor memory again: a normal call afterwards must return exactly
what it returned before, and match the oracle.  The shapes launch more CTAs
than the GPU has SMs, so later CTAs allocate tensor memory after earlier ones
gave up.
"""
import numpy as np
import pytest
import torch

import score_keys_pooled_b200 as s2o
from score_keys_pooled_b200 import synth
from oracle import s2o_oracle as O
from tests import parity

pytestmark = pytest.mark.gpu

TIMEOUT = 5  # S2O_ERR_DEVICE_TIMEOUT


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    s2o.lib()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def test_every_wait_giving_up_reports_timeout_and_leaves_the_device_usable():
    B, Hq, Hkv, N, tau = 1, 16, 4, 4096, 1e-3
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=True, band=True, n_stripe=16, seed=31)
    q, k, v = _dev(Q), _dev(K), _dev(V)
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=tau)
    bufs = s2o.plan(cfg, q, k)
    ref = s2o.attention(cfg, q, k, v, bufs["perm"], bufs["nblocks"])
    assert s2o.last_device_error() == 0
    ncta = B * Hkv * s2o.num_segments(cfg) * (Hq // Hkv // 2)
    assert ncta > torch.cuda.get_device_properties(0).multi_processor_count

    s2o.attention_bounded(cfg, q, k, v, bufs["perm"], bufs["nblocks"], 0)
    assert s2o.last_device_error() == TIMEOUT
    assert s2o.last_device_error() == 0  # read and cleared

    out = s2o.attention(cfg, q, k, v, bufs["perm"], bufs["nblocks"])
    assert s2o.last_device_error() == 0
    assert torch.equal(out, ref)


@pytest.mark.parametrize("polls", [1, 2, 4, 16, 64, 256])
def test_waits_giving_up_mid_pipeline_wind_down(polls):
    B, Hq, Hkv, N, tau = 1, 16, 4, 4096, 1e-3
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=True, band=True, n_stripe=16, seed=32)
    q, k, v = _dev(Q), _dev(K), _dev(V)
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=tau)
    bufs = s2o.plan(cfg, q, k)
    ref = s2o.attention(cfg, q, k, v, bufs["perm"], bufs["nblocks"])
    assert s2o.last_device_error() == 0
    for _ in range(3):
        s2o.attention_bounded(cfg, q, k, v, bufs["perm"], bufs["nblocks"], polls)
        assert s2o.last_device_error() in (0, TIMEOUT)
    out = s2o.attention(cfg, q, k, v, bufs["perm"], bufs["nblocks"])
    assert s2o.last_device_error() == 0
    assert torch.equal(out, ref)
    # and the result is the oracle's on sampled segments
    p = O.Params(tau=tau)
    G = Hq // Hkv
    T, S = s2o.num_candidates(cfg), s2o.num_segments(cfg)
    perm = bufs["perm"][:B * Hkv * T].cpu().numpy().reshape(B, Hkv, T)
    nb = bufs["nblocks"].cpu().numpy().reshape(B, Hkv, S)
    off = O.candidate_offsets(N, p)
    got = out.float().cpu().numpy()
    for kvh in (0, Hkv - 1):
        for s in (0, 5, S - 1):
            keep = O.keep_set(N, s, perm[0, kvh, off[s]:off[s + 1]], int(nb[0, kvh, s]), p)
            want = O.attention_segment(Q, K, V, 0, kvh, s, G, keep, p)
            r0, r1 = O.segment_rows(N, s, p)
            parity.assert_output_close(got[0, kvh * G:(kvh + 1) * G, r0:r1], want, f"kvh={kvh} s={s}")


def test_bounded_entry_checks_its_arguments():
    cfg = s2o.make_config(1, 3, 1, 512, tau=1e-3)  # odd group: the kernel without the limit
    x = torch.zeros(16, dtype=torch.int16, device="cuda")
    with pytest.raises(s2o.S2OError) as e:
        s2o.attention_bounded(cfg, x, x, x, x.int(), x.int(), 0, O=x)
    assert e.value.code == 2
    cfg = s2o.make_config(1, 4, 1, 512, tau=1e-3)
    with pytest.raises(s2o.S2OError) as e:
        s2o.attention_bounded(cfg, x, x, x, x.int(), x.int(), (1 << 24) + 1, O=x)
    assert e.value.code == 1
