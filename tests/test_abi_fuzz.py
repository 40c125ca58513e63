"""Host-side robustness of the boundary (no GPU): arbitrary, mostly invalid
configurations are either accepted with a consistent ledger or rejected
with ZERO_ERR_ARG — never a crash."""
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
