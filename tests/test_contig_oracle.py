"""CPU checks of the contiguous-KV inputs: the contiguous cache read as one page per
sequence and the same tokens scattered into a shuffled page pool give the same
oracle result (bit for bit), and poisoned slots past each length are never read."""
import numpy as np
import pytest

import oracle
import workloads


@pytest.mark.parametrize("layout", ["blhd", "bhld"])
def test_contig_and_paged_forms_agree_in_the_oracle(layout):
    w = workloads.make_contig(name="c", seed=3, batch=4, num_q_heads=8, num_kv_heads=2, head_dim=32,
                              seq_lens=[1, 33, 0, 70], lmax=77, layout=layout)
    a = oracle.paged_decode(w)
    assert np.isfinite(a).all()
    wp = workloads.paged_from_contig(w, page_size=32, seed=1)
    b = oracle.paged_decode(wp)
    assert np.array_equal(a, b)
    assert np.all(a[2] == 0)
