"""The allocation-free grouping entry point, moe_permute_noalloc.

It exists for callers that cannot allocate device memory (code inside an
allocator callback, plugins whose host owns all device memory, serving loops
that forbid allocation): its scratch is a static array in the library.  The
test calls it through the C ABI several times in a row, on different inputs
(multi-chunk and one-CTA grouping, no slots, exactly the slot limit, small
after large), and checks each result bit for bit against moe_permute with a
workspace (the tolerance of all index work).  This file is collected last on
purpose.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

CASES = [
    # (T, E, top_k, capacity factor, seed), run in this order, each call
    # right after the previous one: a smaller call after a larger one would
    # show stale scratch from the earlier call
    (3000, 128, 8, 1.25, 1),    # several chunks: histogram, scans, scatter
    (777, 32, 4, 0.0, 2),
    (1, 32, 4, 0.0, 3),         # decode size: the one-CTA grouping kernel
    (200, 64, 8, 0.5, 4),       # 1600 slots, one chunk, capacity drops
    (0, 16, 2, 0.0, 5),         # no slots: counts and offsets cleared
    (131072, 64, 8, 1.0, 6),    # exactly the limit: all 512 chunks of the scratch
    (5, 8, 2, 0.0, 7),          # small again after the largest call
]


def seeded_topk(T, E, k, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    if T == 0:
        return torch.empty((0, k), dtype=torch.int32, device="cuda")
    return torch.argsort(torch.rand((T, E), device="cuda", generator=g), dim=1)[:, :k].to(torch.int32).contiguous()


def outputs(T, E, k):
    return [torch.full((n,), -7, dtype=torch.int32, device="cuda") for n in (E, E + 1, T * k, T * k, E)]


def test_noalloc_permute_matches_workspace_permute_twice(gpu_lib):
    moe = gpu_lib
    assert CASES[-2][0] * CASES[-2][2] == 1 << 20
    for T, E, k, cf, seed in CASES:
        cfg = moe.config(T, 256, 256, E, k, 0, cf, "bf16")
        idx = seeded_topk(T, E, k, seed)
        ref = outputs(T, E, k)
        moe.moe_permute(cfg, idx, *ref, moe.workspace(cfg))
        got = outputs(T, E, k)
        moe.moe_permute_noalloc(cfg, idx, *got)
        torch.cuda.synchronize()
        for name, a, b in zip(("counts", "offsets", "perm_rows", "row_of", "dropped"), ref, got):
            assert np.array_equal(a.cpu().numpy(), b.cpu().numpy()), (T, name)
        if T == 0:
            assert got[0].cpu().numpy().tolist() == [0] * E and got[1].cpu().numpy().tolist() == [0] * (E + 1)


def test_noalloc_permute_rejects_too_many_slots(gpu_lib):
    moe = gpu_lib
    cfg = moe.config(131073, 256, 256, 64, 8)  # 1048584 slots > 1048576
    fake = 0x7f0000000000
    with pytest.raises(moe.MoeError) as e:
        moe.moe_permute_noalloc(cfg, fake, fake, fake, fake, fake, fake)
    assert e.value.status == 2 and "1048576" in str(e.value)
