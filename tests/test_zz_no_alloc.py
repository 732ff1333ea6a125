"""moe_permute_noalloc: the dispatch step for callers that cannot allocate
device memory (allocator callbacks, fixed-footprint runtimes, hosts without
an allocator).  Its scratch is a fixed array inside the library, so its
results must equal the oracle's stable expert-major order -- and those of
moe_permute with a caller workspace -- call after call, although the array
keeps whatever the previous call left in it."""
import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_renormalised_b200 as moe

pytestmark = pytest.mark.gpu


def _routing(T, E, k, seed, skew):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g)
    if skew:
        logits = logits + 3.0 * (torch.arange(E, dtype=torch.float32) + 1.0) ** -0.3
    return torch.topk(logits, k, dim=1).indices.to(torch.int32).cuda()


def _outputs(T, E, k, L):
    dev = "cuda"
    return (torch.empty(E + 1, dtype=torch.int32, device=dev), torch.empty(T * k, dtype=torch.int32, device=dev),
            torch.empty(T * k, dtype=torch.int32, device=dev), torch.empty(T * k, L, dtype=torch.bfloat16, device=dev))


def _check_fault_free():
    st, code = moe.moe_device_error()
    assert st == moe.MOE_OK and code == 0, f"device fault {code}"


@pytest.mark.parametrize("T,E,k,L", [(4096, 128, 8, 1024), (16384, 896, 16, 256)])
def test_noalloc_permute_matches_workspace_permute_twice(T, E, k, L):
    d = moe.Dims(T=T, H=2048, L=L, E=E, k=k, I=768, S=2, Is=1024)
    ws = torch.empty(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    for call, (seed, skew) in enumerate(((1, False), (2, True))):  # two calls in a row, different routings
        idx = _routing(T, E, k, seed + T, skew)
        z = torch.randn(T, L, device="cuda").to(torch.bfloat16)
        want = _outputs(T, E, k, L)
        got = _outputs(T, E, k, L)
        for t in got:
            t.fill_(-7)  # stale contents must not leak into any output
        assert moe.moe_permute(d, idx, z, want[0], want[1], want[2], want[3], ws) == moe.MOE_OK
        assert moe.moe_permute_noalloc(d, idx, z, got[0], got[1], got[2], got[3]) == moe.MOE_OK
        torch.cuda.synchronize()
        _check_fault_free()
        # against the oracle's stable counting sort of the (token, slot) pairs
        _, offsets, perm_token, inv_perm = oracle.permute(idx.cpu().numpy(), E)
        assert np.array_equal(got[0].cpu().numpy(), offsets), f"call {call}: expert_offsets differ from the oracle"
        assert np.array_equal(got[1].cpu().numpy(), perm_token), f"call {call}: perm_token differs from the oracle"
        assert np.array_equal(got[2].cpu().numpy(), inv_perm), f"call {call}: inv_perm differs from the oracle"
        assert torch.equal(got[3].cpu(), z.cpu()[torch.as_tensor(perm_token)]), f"call {call}: z_perm differs"
        # and against the workspace variant
        for a, b, name in zip(got, want, ("expert_offsets", "perm_token", "inv_perm", "z_perm")):
            assert torch.equal(a, b), f"call {call}: {name} differs from moe_permute"


def test_noalloc_permute_rejects_dims_beyond_its_scratch():
    # 100k tokens at the K3 shape need about 9 MB of scratch: more than the 4 MiB array holds.
    d = moe.Dims(T=100_000, H=7168, L=3584, E=896, k=16, I=3072, S=2, Is=3072)
    fake = 1 << 20  # never dereferenced: the size check comes first
    assert moe.moe_permute_noalloc(d, fake, None, fake, fake, fake, None) == moe.MOE_ERR_INVALID_ARG
