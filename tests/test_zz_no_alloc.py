"""moe_permute_noalloc: the dispatch for callers that cannot pass a workspace.

Such callers (a plug-in that only receives tensors from a host framework that
owns all device memory, or a serving loop that may not allocate once it runs)
get the same counting sort and row gather as moe_permute, with the histogram
kept in a fixed array inside the library.  This checks, through the C ABI, that
two calls in a row give exactly what moe_permute gives on the same inputs --
the second call with a different shape, so stale contents of the shared array
would show -- and that a request larger than the array is refused.  The file
is named to be collected last.
"""
import numpy as np
import pytest
import torch

import top_routing_expert_gemm_b200 as moe
from top_routing_expert_gemm_b200 import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    moe.lib()


def _case(T, E, k, d, seed):
    rng = np.random.default_rng(seed)
    keys = rng.random((T, E))
    keys[:, 0] += 0.5  # one hot expert, some cold ones
    ids = np.argsort(-keys, axis=1, kind="stable")[:, :k].astype(np.int32)
    x = torch.from_numpy(rng.standard_normal((T, d)).astype(np.float32)).to(torch.bfloat16).cuda()
    return torch.from_numpy(ids).cuda(), x


def _outputs(T, E, k, d):
    return dict(counts=torch.full((E,), -1, dtype=torch.int32, device="cuda"),
                offsets=torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
                perm=torch.full((T * k,), -1, dtype=torch.int32, device="cuda"),
                row_of=torch.full((T * k,), -2, dtype=torch.int32, device="cuda"),
                x_perm=torch.zeros(T * k, d, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("order", ["large_then_small", "small_then_large"])
def test_noalloc_permute_matches_moe_permute_on_two_calls(order):
    cases = [(4099, 256, 8, 512), (1000, 8, 2, 264)]
    if order == "small_then_large":
        cases = cases[::-1]
    for call, (T, E, k, d) in enumerate(cases):
        cfg = moe.make_config(T, d, E, k, 8, moe.MOE_BF16, moe.MOE_SOFTMAX_TOPK)
        ids, x = _case(T, E, k, d, seed=call + 7)
        ref = _outputs(T, E, k, d)
        ws = torch.zeros(moe.moe_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
        moe.moe_permute(cfg, ids, x, ref["counts"], ref["offsets"], ref["perm"], ref["row_of"], ref["x_perm"], ws)
        got = _outputs(T, E, k, d)
        moe.moe_permute_noalloc(cfg, ids, x, got["counts"], got["offsets"], got["perm"], got["row_of"],
                                got["x_perm"])
        torch.cuda.synchronize()
        # integer outputs and the copied rows: exact, the tolerance the dispatch tests use
        for name in ("counts", "offsets", "perm", "row_of"):
            assert torch.equal(got[name], ref[name]), (call, name)
        assert torch.equal(got["x_perm"].view(torch.int16), ref["x_perm"].view(torch.int16)), call


def test_noalloc_permute_refuses_more_than_its_array_holds():
    # 1024 experts x ceil(2^17 * 8 / 2048) chunks = 524288 entries > 65536
    cfg = moe.make_config(1 << 17, 64, 1024, 8, 8, moe.MOE_BF16, moe.MOE_SOFTMAX_TOPK)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_permute_noalloc(cfg, dummy, dummy, dummy, dummy, dummy, dummy, dummy)
    assert e.value.status == 2
