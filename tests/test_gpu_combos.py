"""Feature combinations on the CUDA path against the oracle: several query tokens per sequence
with more than 64 heads and a paged cache."""
import pytest
import torch

import oracle
from tests.gpu_helpers import assert_close, assert_lse_close
from tests.test_gpu_multi import multi_inputs, run_multi

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("q,B,heads,page_size", [(2, 1, 128, 64), (3, 4, 96, 0)])
def test_multi_token_with_head_groups(q, B, heads, page_size):
    w, inp, q_lat, q_rope = multi_inputs(q, [q, 190, 1500], B=B, heads=heads, page_size=page_size,
                                         seed=81)
    out, lse = run_multi(w, inp, q_lat, q_rope)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.decode_multi(q_lat, q_rope, inp.c_kv, inp.k_rope, inp.seq_lens,
                                       inp.page_table, w.num_branches, w.sigma, w.gamma,
                                       page_size=page_size, max_seq_len=inp.max_seq_len)
    assert_close(out, ref, f"q={q} H={heads}")
    assert_lse_close(lse, ref_lse, f"q={q} H={heads} lse")
