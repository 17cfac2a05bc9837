"""Failure detection on the GPU without a fault: a bounded wait that nothing completes gives up,
records DSA_ERR_TIMEOUT with its site, and leaves the context usable for the next launch."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_keys_b200")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    assert dsa.dsa_device_supported(), "libdsa needs an sm_100 device"
    assert dsa.dsa_get_device_status() == 0
    return torch.device("cuda", 0)


def test_wait_timeout_is_reported_with_its_site(dev):
    dsa.dsa_selftest_wait_timeout()
    assert dsa.dsa_get_device_status() == 4              # DSA_ERR_TIMEOUT
    d = dsa.dsa_get_error_detail()
    assert d["site_name"] == "selftest" and d["block"] == 0
    assert 900_000 <= d["wait_us"] <= 10_000_000, d      # the one-second bound, not a hang
    assert dsa.dsa_get_device_status() == 0              # read-and-clear


def test_context_usable_after_timeout(dev):
    dsa.dsa_selftest_wait_timeout()
    assert dsa.dsa_get_device_status() == 4
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 64, 128)).astype(np.float32)
    pos = np.array([0, 17, 4000], np.int32)
    table = O.rope_table(16384)
    codes, scales = dsa.dsa_index_keys(P.to_dev(x), P.to_dev(pos), torch.from_numpy(table).to(dev))
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_status() == 0
    P.check_codes(codes.cpu().numpy(), scales.cpu().numpy(), x, pos[:, None], table, True)
