"""Host-side argument checks of the Python binding: wrong types, devices and shapes are rejected
before any device call (so these run without a GPU)."""
import pytest
import torch


@pytest.fixture(scope="module")
def dsa():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import sparse_attention_keys_b200 as m
    return m


def test_index_keys_rejects_wrong_dtype_and_host_tensors(dsa):
    with pytest.raises(TypeError):
        dsa.dsa_index_keys(torch.zeros(2, 128, dtype=torch.float16), torch.zeros(2, dtype=torch.int32),
                           torch.zeros(8, 32, 2))
    with pytest.raises(ValueError):          # host tensors: the binding wants device memory
        dsa.dsa_index_keys(torch.zeros(2, 128), torch.zeros(2, dtype=torch.int32), torch.zeros(8, 32, 2))


def test_sparse_mla_rejects_wrong_dtypes(dsa):
    q = torch.zeros(1, 1, 128, 576, dtype=torch.float32)
    with pytest.raises(TypeError):
        dsa.dsa_sparse_mla(q, torch.zeros(1, 8, 576, dtype=torch.bfloat16), torch.zeros(1, 1, 4, dtype=torch.int32))


def test_absorb_weights_must_be_bf16_device_tensors(dsa):
    with pytest.raises(TypeError):
        dsa._head_weights(torch.zeros(128, 128, 512), "w_uk")                     # fp32
    with pytest.raises(TypeError):
        dsa._head_weights(torch.zeros(128, 128, 512, dtype=torch.bfloat16), "w_uk")   # host memory
    with pytest.raises(ValueError):                                                 # activations on the host
        dsa.dsa_mla_out_absorb(torch.zeros(1, 128, 512, dtype=torch.bfloat16),
                               torch.zeros(128, 128, 512, dtype=torch.bfloat16))


def test_noncontiguous_inputs_are_rejected(dsa):
    x = torch.zeros(4, 256)[:, :128]         # a strided view
    assert not x.is_contiguous()
    with pytest.raises(ValueError):
        dsa.dsa_index_keys(x, torch.zeros(4, dtype=torch.int32), torch.zeros(8, 32, 2))


def test_status_strings_cover_every_site(dsa):
    assert all(isinstance(v, str) and v for v in dsa.SITE_NAMES.values())
    assert {0x41, 0x42, 0x43, 0x44, 0x45} <= set(dsa.SITE_NAMES)


def test_sparse_mla_shape_checks(dsa):
    """Mismatched sparse-MLA buffers raise before any pointer reaches the library (checked on host
    tensors: the shape rules do not depend on the device)."""
    bf = torch.bfloat16
    q = torch.zeros(2, 3, 128, 576, dtype=bf)
    kv = torch.zeros(2, 64, 576, dtype=bf)
    idx = torch.zeros(2, 3, 16, dtype=torch.int32)
    out = torch.zeros(2, 3, 128, 512, dtype=bf)
    lse = torch.zeros(2, 3, 128)
    assert dsa._mla_shapes(q, kv, idx, out, lse) == (2, 3, 16)
    assert dsa._mla_shapes(q, kv, idx, None, None) == (2, 3, 16)
    bad = [
        (torch.zeros(2, 3, 64, 576, dtype=bf), kv, idx, out, lse),        # q heads
        (torch.zeros(2, 3, 128, 512, dtype=bf), kv, idx, out, lse),       # q width
        (q, torch.zeros(2, 64, 512, dtype=bf), idx, out, lse),            # kv width
        (q, kv, torch.zeros(2, 2, 16, dtype=torch.int32), out, lse),      # idx queries
        (q, kv, torch.zeros(3, 3, 16, dtype=torch.int32), out, lse),      # idx batch
        (q, kv, idx, torch.zeros(2, 3, 128, 256, dtype=bf), lse),         # out too small
        (q, kv, idx, torch.zeros(2, 2, 128, 512, dtype=bf), lse),         # out queries
        (q, kv, idx, out, torch.zeros(2, 3, 64)),                         # lse heads
    ]
    for args in bad:
        with pytest.raises(ValueError):
            dsa._mla_shapes(*args)
    with pytest.raises(ValueError):                                         # not on one device
        dsa._mla_shapes(q, kv.to("meta"), idx, out, lse)
