"""ds4g_moe_permute_static -- the expert permutation for callers that cannot
allocate device memory (not even a workspace of their own), whose scratch is
the library's file-scope device array.  Checked through the C ABI against
the workspace-taking ds4g_moe_permute and against the oracle's permutation of
the same inputs, on two calls in a row (the array keeps the previous call's
contents), on problems that take the multi-CTA path (the one that uses the
scratch) and the single-CTA path.  Collected last on purpose."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _problem(T, k, E, K, seed_stream):
    lg = synth.logits(T, E, 0, 1.5)
    idx, _ = oracle.route_topk(lg, k)
    xq = oracle.quantize(synth.normal_f32((T, K), 0, seed_stream), oracle.MX)
    return idx, xq


@pytest.mark.parametrize("T,k,E", [(2048, 6, 256), (700, 6, 64), (5, 6, 256)])
def test_permute_static_matches_workspace_version(T, k, E):
    from block_scaled_fp4_topk_b200 import ds4g
    dev = torch.device("cuda:0")
    for call, stream in enumerate((61, 62)):           # two calls in a row, different inputs
        idx, xq = _problem(T, k, E, 256, stream + T)
        idx_d = torch.from_numpy(idx).to(dev)
        x_d = ds4g.Fp4Tensor(torch.from_numpy(xq.data).to(dev), torch.from_numpy(xq.scales).to(dev), None, 0)
        ref = ds4g.ds4g_moe_permute(idx_d, E, x_d)
        got = ds4g.ds4g_moe_permute_static(idx_d, E, x_d)
        torch.cuda.synchronize()
        for r, g in zip(ref[:3], got[:3]):
            assert torch.equal(r, g), f"call {call}"
        assert torch.equal(ref[3].data, got[3].data) and torch.equal(ref[3].scales, got[3].scales)
        # and against the oracle's permutation and gather, bit for bit
        offs, r2s, s2r = oracle.moe_permute(idx, E)
        assert np.array_equal(got[0].cpu().numpy(), offs), f"call {call}: offsets"
        assert np.array_equal(got[1].cpu().numpy(), r2s), f"call {call}: row_to_slot"
        assert np.array_equal(got[2].cpu().numpy(), s2r), f"call {call}: slot_to_row"
        a = oracle.gather_rows(xq, r2s, k)
        assert np.array_equal(got[3].data.cpu().numpy(), a.data) and np.array_equal(got[3].scales.cpu().numpy(),
                                                                                   a.scales), f"call {call}: rows"


def test_permute_static_rejects_too_large():
    from block_scaled_fp4_topk_b200 import ds4g
    dev = torch.device("cuda:0")
    E, k = 4096, 6
    T = 20000                                           # E * ceil(T*k/256) * 4 B > 256 KiB
    assert ds4g._lib.ds4g_permute_workspace_bytes(T, k, E) > ds4g._lib.ds4g_permute_static_max_bytes()
    idx = torch.zeros((T, k), dtype=torch.int32, device=dev)
    xq = ds4g.Fp4Tensor.empty(T, 64, 0, dev)
    with pytest.raises(ds4g.Ds4gError) as ei:
        ds4g.ds4g_moe_permute_static(idx, E, xq)
    assert ei.value.status == 6
