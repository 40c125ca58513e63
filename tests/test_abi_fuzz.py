"""Host-side robustness of the boundary (no GPU): arbitrary, mostly invalid
configurations are either accepted with a consistent ledger or rejected
with ZERO_ERR_ARG — never a crash."""
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from zero_partitioned_mixed_02_b200 import _abi as A

i32 = st.integers(-3, 70)


@settings(max_examples=500, deadline=None)
@given(psi=st.integers(-5, 100_000), nd=st.integers(-2, 2000), stage=i32, view=st.integers(-3, 40),
       variant=st.integers(-1, 5), precision=st.integers(-1, 3), view_outputs=st.integers(-1, 40),
       tensors=st.one_of(st.none(), st.lists(st.tuples(st.integers(-3, 40_000), st.integers(-1, 6),
                                                       st.integers(-1, 3)), max_size=10)))
def test_state_bytes_accepts_or_rejects(psi, nd, stage, view, variant, precision, view_outputs, tensors):
    cfg = A.Config(psi, nd, stage, rank_view=view, variant=variant, tensors=tensors, precision=precision,
                   view_outputs=view_outputs)
    try:
        L = A.zero_state_bytes(cfg)
    except A.ZeroError as e:
        assert e.code == A.ZERO_ERR_ARG
        return
    # accepted: the basic facts hold
    assert 1 <= nd <= A.ZERO_MAX_ND and stage in (1, 2, 3) and psi >= 1
    assert L.workspace_bytes > 0 and L.state_elems >= 0
    if view < 0:
        assert L.state_elems == psi
    if tensors:
        assert sum(t[0] for t in tensors) == psi


def _has_gpu():
    import torch
    return torch.cuda.is_available()


# host-side validation only: where a GPU is present, random IPC handles would
# reach the driver, which this test has no reason to probe
@pytest.mark.skipif(_has_gpu(), reason="host-side validation test; not run where a GPU is present")
@settings(max_examples=300, deadline=None)
@given(raw=st.binary(min_size=104, max_size=104), magic=st.booleans(), offset=st.integers(0, 1 << 40),
       nbytes=st.integers(0, 1 << 40), address=st.integers(0, (1 << 64) - 1))
def test_peer_descriptors_from_the_wire(raw, magic, offset, nbytes, address):
    """zero_peer_open/close take descriptors received from other processes:
    any 104 bytes are refused with an error code (ZERO_ERR_ARG, or
    ZERO_ERR_CUDA where no device can map them), never a crash."""
    d = A.zero_peer_desc.from_buffer_copy(raw)
    if magic:
        d.magic = A.ZERO_PEER_MAGIC
        d.offset, d.bytes, d.address = offset, nbytes, address
    desc = bytes(d)
    try:
        ptr = A.zero_peer_open(desc)
    except A.ZeroError as e:
        assert e.code in (A.ZERO_ERR_ARG, A.ZERO_ERR_CUDA)
    else:  # only a descriptor naming this very process opens without a device
        assert ptr == d.address
    try:
        A.zero_peer_close(desc, 16)
    except A.ZeroError as e:
        assert e.code in (A.ZERO_ERR_ARG, A.ZERO_ERR_CUDA)
    assert A.zero_peer_open_count() == 0
