"""moe_permute_noalloc: the dispatch call for callers that cannot allocate
device memory (a host program with no device allocator of its own, or a
serving loop on a fixed memory plan that must not call cudaMalloc/cudaFree
while running).  It takes no workspace; its scratch is a fixed array inside
the library.  Checked through the C ABI against moe_permute, which uses a
caller workspace, on two calls in a row with different layers, so stale
scratch contents from the first call would show up in the second."""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_bias_b200 import binding as B
from mixture_experts_ffn_bias_b200 import build as build_mod
from mixture_experts_ffn_bias_b200 import inputs as I
from mixture_experts_ffn_bias_b200.layer import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build_mod.build()
    B.lib()


def _routing(T, E, k, seed):
    rng = np.random.default_rng(seed)
    # skewed choice of distinct experts per token, so segments are ragged
    p = rng.dirichlet(np.full(E, 0.3))
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def _buffers(T, k, E, d):
    kw = dict(device="cuda")
    return (torch.full((E,), -7, dtype=torch.int32, **kw),
            torch.full((E + 1,), -7, dtype=torch.int32, **kw),
            torch.full((T, k), -7, dtype=torch.int32, **kw),
            torch.full((T * k,), -7, dtype=torch.int32, **kw),
            torch.zeros((T * k, d), dtype=torch.bfloat16, **kw))


def _compare_one(T, d, E, k, seed):
    cfg = B.make_config(T, d, E, 128, k)
    idx = torch.from_numpy(_routing(T, E, k, seed)).cuda()
    rng = np.random.default_rng(seed + 1)
    x = to_device(I.round_to_bf16(rng.standard_normal((T, d)).astype(np.float32)),
                  torch.bfloat16, "cuda")
    ref = _buffers(T, k, E, d)
    ws = torch.empty(B.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    B.moe_permute(cfg, idx, x, *ref, ws)
    got = _buffers(T, k, E, d)
    B.moe_permute_noalloc(cfg, idx, x, *got)
    torch.cuda.synchronize()
    for a, b in zip(ref[:3], got[:3]):
        assert torch.equal(a, b)
    R = int(ref[1][-1])
    assert R == T * k
    assert torch.equal(ref[3][:R], got[3][:R])
    assert torch.equal(ref[4][:R], got[4][:R])


def test_noalloc_matches_workspace_permute_on_two_calls_in_a_row():
    _compare_one(T=600, d=256, E=128, k=8, seed=11)
    _compare_one(T=1000, d=512, E=64, k=6, seed=12)


def test_noalloc_rejects_sizes_beyond_its_fixed_scratch():
    E = 128
    T = 256 * (B.NOALLOC_MAX_BLOCK_COUNTS // E) + 1     # one block more than fits
    cfg = B.make_config(T, 128, E, 128, 2)
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    st = B.moe_permute_noalloc(cfg, dummy, dummy, dummy, dummy, dummy, dummy, dummy, check=False)
    assert st == B.MOE_ERR_WORKSPACE
