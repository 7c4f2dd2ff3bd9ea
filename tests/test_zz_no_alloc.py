"""moe_permute_noalloc: the dispatch for callers that cannot pass a workspace.

Such callers (a plug-in that only receives tensors from a host framework that
owns all device memory, or a serving loop that may not allocate once it runs)
get the same counting sort and row gather as moe_permute, with the histogram
kept in a fixed array inside the library.  This checks, through the C ABI, that
two calls in a row give exactly what moe_permute gives on the same inputs --
the second call with a different shape, so stale contents of the shared array
would show -- and that a request larger than the array is refused.  Further
cases reach the single-block path of decode-sized batches, an empty batch,
expert ids outside [0, E), a capacity factor and fp32 rows, and check that
the caller's current device and a side stream are honoured.  The file is
named to be collected last.
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


def _case(T, E, k, d, seed, dtype=torch.bfloat16):
    rng = np.random.default_rng(seed)
    keys = rng.random((T, E))
    keys[:, 0] += 0.5  # one hot expert, some cold ones
    ids = np.argsort(-keys, axis=1, kind="stable")[:, :k].astype(np.int32)
    x = torch.from_numpy(rng.standard_normal((T, d)).astype(np.float32)).to(dtype).cuda()
    return torch.from_numpy(ids).cuda(), x


def _outputs(T, E, k, d, dtype=torch.bfloat16):
    return dict(counts=torch.full((E,), -1, dtype=torch.int32, device="cuda"),
                offsets=torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
                perm=torch.full((max(1, T * k),), -1, dtype=torch.int32, device="cuda"),
                row_of=torch.full((max(1, T * k),), -2, dtype=torch.int32, device="cuda"),
                x_perm=torch.zeros(max(1, T * k), d, dtype=dtype, device="cuda"))


def _both(cfg, ids, x, T, E, k, d, dtype=torch.bfloat16, stream=None):
    """moe_permute (workspace) and moe_permute_noalloc on the same inputs."""
    ref = _outputs(T, E, k, d, dtype)
    got = _outputs(T, E, k, d, dtype)
    ws = torch.zeros(moe.moe_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()  # the buffers are filled on the current stream; the calls may use another
    moe.moe_permute(cfg, ids, x, ref["counts"], ref["offsets"], ref["perm"], ref["row_of"], ref["x_perm"], ws,
                    stream=stream)
    moe.moe_permute_noalloc(cfg, ids, x, got["counts"], got["offsets"], got["perm"], got["row_of"], got["x_perm"],
                            stream=stream)
    torch.cuda.synchronize()
    return ref, got


def _assert_same(ref, got, what):
    # integer outputs and the copied rows: exact, the tolerance the dispatch tests use
    for name in ("counts", "offsets", "perm", "row_of"):
        assert torch.equal(got[name], ref[name]), (what, name)
    bits = torch.int16 if got["x_perm"].dtype == torch.bfloat16 else torch.int32
    assert torch.equal(got["x_perm"].view(bits), ref["x_perm"].view(bits)), what


@pytest.mark.parametrize("order", ["large_then_small", "small_then_large"])
def test_noalloc_permute_matches_moe_permute_on_two_calls(order):
    cases = [(4099, 256, 8, 512), (1000, 8, 2, 264)]
    if order == "small_then_large":
        cases = cases[::-1]
    for call, (T, E, k, d) in enumerate(cases):
        cfg = moe.make_config(T, d, E, k, 8, moe.MOE_BF16, moe.MOE_SOFTMAX_TOPK)
        ids, x = _case(T, E, k, d, seed=call + 7)
        ref, got = _both(cfg, ids, x, T, E, k, d)
        _assert_same(ref, got, call)


def test_noalloc_permute_refuses_more_than_its_array_holds():
    # 1024 experts x ceil(2^17 * 8 / 2048) chunks = 524288 entries > 65536
    cfg = moe.make_config(1 << 17, 64, 1024, 8, 8, moe.MOE_BF16, moe.MOE_SOFTMAX_TOPK)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_permute_noalloc(cfg, dummy, dummy, dummy, dummy, dummy, dummy, dummy)
    assert e.value.status == 2


def test_noalloc_decode_sized_batch_single_block_path_two_calls():
    """At most 1024 assignments take the one-block dispatch kernel."""
    for call, (T, E, k, d) in enumerate([(4, 8, 2, 4096), (64, 8, 2, 4096), (1, 256, 8, 512)]):
        cfg = moe.make_config(T, d, E, k, 8, moe.MOE_BF16, moe.MOE_SOFTMAX_TOPK)
        ids, x = _case(T, E, k, d, seed=40 + call)
        ref, got = _both(cfg, ids, x, T, E, k, d)
        _assert_same(ref, got, ("decode", call))
        assert int(got["offsets"][E]) == T * k


def test_noalloc_empty_batch_zeroes_counts_and_offsets():
    E, k, d = 16, 2, 64
    cfg = moe.make_config(0, d, E, k, 8, moe.MOE_BF16, moe.MOE_SOFTMAX_TOPK)
    got = _outputs(0, E, k, d)
    moe.moe_permute_noalloc(cfg, None, None, got["counts"], got["offsets"], None, None, None)
    torch.cuda.synchronize()
    assert int(got["counts"].abs().sum()) == 0 and int(got["offsets"].abs().sum()) == 0


@pytest.mark.parametrize("T", [40, 3000, 5000])  # one-warp, all-warp single-block and three-kernel paths
def test_noalloc_skips_expert_ids_out_of_range_like_moe_permute(T):
    E, k, d = 8, 2, 256
    cfg = moe.make_config(T, d, E, k, 8, moe.MOE_BF16, moe.MOE_SOFTMAX_TOPK)
    ids, x = _case(T, E, k, d, seed=T)
    ids[3, 1] = -3
    ids[T // 2, 0] = E + 1
    ids[T - 1, 1] = E
    ref, got = _both(cfg, ids, x, T, E, k, d)
    _assert_same(ref, got, "bad ids")
    row_of = got["row_of"].cpu().numpy()
    assert row_of[3 * k + 1] == -1 and row_of[(T // 2) * k] == -1 and row_of[(T - 1) * k + 1] == -1
    assert int(got["offsets"][E]) == T * k - 3


@pytest.mark.parametrize("T", [300, 2000, 5000])
def test_noalloc_with_capacity_factor_matches_moe_permute(T):
    E, k, d = 8, 2, 128
    cfg = moe.make_config(T, d, E, k, 8, moe.MOE_BF16, moe.MOE_SOFTMAX_TOPK, capacity_factor=0.5)
    ids, x = _case(T, E, k, d, seed=T + 1)
    ref, got = _both(cfg, ids, x, T, E, k, d)
    _assert_same(ref, got, "capacity")
    cap = moe.moe_expert_capacity(cfg)
    assert int(got["offsets"][E]) == int(torch.clamp(got["counts"], max=cap).sum())
    assert int((got["row_of"] < 0).sum()) > 0  # the hot expert dropped its late tokens


def test_noalloc_fp32_rows_on_a_side_stream_keep_the_current_device():
    T, E, k, d = 2500, 32, 4, 96
    cfg = moe.make_config(T, d, E, k, 8, moe.MOE_F32, moe.MOE_SOFTMAX_TOPK)
    ids, x = _case(T, E, k, d, seed=5, dtype=torch.float32)
    dev_before = torch.cuda.current_device()
    side = torch.cuda.Stream()
    ref, got = _both(cfg, ids, x, T, E, k, d, dtype=torch.float32, stream=side)
    _assert_same(ref, got, "fp32")
    assert torch.cuda.current_device() == dev_before
