"""Two GPU checks that run after the rest of the suite: decode attention for more than
64 sequences, which runs on the mma.sync split-K kernels instead of the tensor-core
kernel, and the failure path of the kernels' bounded waits.  Both compare with the
fp64 oracle through the C ABI; the parity tests they reuse live in test_gpu_parity.
"""
import time

import pytest
import torch

import synth
from sparse_top_kv_std_b200 import binding as B
from tests import test_gpu_parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    B.lib()
    B.std_get_device_error(clear=True)
    yield
    torch.cuda.synchronize()


# ----------------------------------------------------------------------------- more than 64 sequences

B65 = P.small_wl("b65_splitk", Bsz=65, Hq=8, Hkv=2, nvis=tuple(300 + 11 * b for b in range(65)), T=5, K=32,
                 gamma=3, wl_id=107)


@pytest.mark.parametrize("splits", [1, 3, 0])
def test_more_than_64_sequences_run_the_split_k_kernels(splits, monkeypatch):
    """65 ragged sequences: more than the tensor-core kernel's 64, so bf16 verify and draft
    attention run on the mma.sync split-K kernel (plus its merge kernel when a call has more
    than one split); both match the oracle."""
    monkeypatch.setitem(P.ATTN_CASES, B65.name, B65)
    n0 = B.std_launch_count()
    P.test_dense_verify_matches_oracle(B65.name, splits)
    # the verify's cache has 1024 rows: automatic splits give 4 key ranges, so the split-K
    # path launches the attention kernel and the merge kernel (the tensor-core kernel: one)
    assert B.std_launch_count() - n0 == (1 if splits == 1 else 2)
    P.test_sparse_decode_matches_oracle(B65.name, splits)


# ----------------------------------------------------------------------------- bounded waits

def test_bounded_wait_gives_up_and_the_context_stays_usable():
    """Failure detection without a GPU fault: a wait that nothing completes (the probe's
    mbarrier gets no arrival) goes through the bounded wait of the tensor-core kernels, gives
    up after its 0.5 s limit, reports STD_DEVERR_TIMEOUT through the device error word, and
    the kernel returns; afterwards the same context still runs a selection that matches the
    oracle."""
    B.std_get_device_error(clear=True)
    done = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    B.std_probe_wait_timeout(done)
    flags = B.std_get_device_error(clear=True)          # synchronises the stream
    waited = time.perf_counter() - t0
    assert done.item() == 0
    assert flags == B.STD_DEVERR_TIMEOUT
    assert 0.4 < waited < 30.0, waited
    assert B.std_get_device_error() == 0
    wl = P.SELECT_CASES["ragged_bf16"]
    P._check_select(wl, synth.host_inputs(wl, seed=0))
