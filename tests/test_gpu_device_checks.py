"""Device-side checks report through the workspace error word, with no GPU fault.

A workspace whose header was never initialised (all zeros: no magic number, no RoPE
rows) is in bounds for every read the kernels make; each kernel must notice the bad
header, write zeros instead of attention output, set the workspace bit of the error
word, and leave the context usable.  recsa_check_device_errors reports and clears it.
"""

import pytest
import torch

import hierarchical_sparse_attention_build_b200 as R
import recsa_inputs as I

pytestmark = pytest.mark.gpu


def _case(batch=1, length=3000, queries=2):
    c = I.random_case(batch=batch, length=length, kv_heads=2, q_heads=8, queries=queries, seed=77, device="cuda")
    p = R.params(num_kv_heads=2, num_q_heads=8, branching=4, top_k=4)
    tree = R.RecsaTree(p, c["k_tok"], c["v_tok"], c["pooler"], length)
    R.build_tree(p, tree)
    return p, tree, c["q"]


@pytest.mark.parametrize("kernel", [R.KERNEL_CTA, R.KERNEL_WARP])
def test_uninitialised_workspace_sets_the_error_word(kernel):
    p, tree, q = _case()
    good = R.Workspace(p, tree.capacity, "cuda")
    bad = torch.zeros(good.nbytes, dtype=torch.uint8, device="cuda")
    bad_ws = R.Workspace.__new__(R.Workspace)
    bad_ws.nbytes, bad_ws.buf = good.nbytes, bad
    out = torch.full(q.shape, 5.0, dtype=torch.float32, device="cuda")
    R.decode(p, tree, q, out, bad_ws, kernel=kernel)
    with pytest.raises(R.RecsaError) as e:
        R.check_device_errors(bad_ws)
    assert e.value.code == 6 and "workspace" in str(e.value)
    assert torch.count_nonzero(out).item() == 0
    R.check_device_errors(bad_ws)  # the word was cleared by the report
    # the context is still usable: the same call on a valid workspace succeeds
    R.decode(p, tree, q, out, good, kernel=kernel)
    R.check_device_errors(good)
    assert torch.isfinite(out).all() and torch.count_nonzero(out).item() > 0
