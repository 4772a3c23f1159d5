"""GPU: attention from host buffers through the copy-overlapped pipeline
must give, bit for bit, what the device path gives (same plans, kernels and
inputs), with ragged head chunks, B > 1 and repeated runs."""
import numpy as np
import pytest

import workloads as W
from _helpers import torch_bf16

pytestmark = pytest.mark.gpu

S = W.mask_spec


@pytest.mark.parametrize("chunk", [1, 2, 5])
def test_pipeline_matches_device_path(chunk):
    import torch
    import block_sparse_attention_mask_b200 as vsa
    specs = [S("spatial", 1, rt=1), S("temporal", 1, rh=2, rw=3, layout=1), S("full"),
             S("stripe", 1, Tw=1, To=0, Ts=2, Sw=5, So=1, Ss=11), S("temporal", 0, rh=1, rw=2)]
    grid, unit, B, D = (3, 9, 20), (1, 8, 16), 2, 128
    N = int(np.prod(grid))
    g = np.random.Generator(np.random.PCG64(9))
    host = [W.bf16_bits_from_f32(g.standard_normal((B, len(specs), N, D), dtype=np.float32)) for _ in range(3)]
    plan = vsa.Plan(specs, grid, unit, 128, 128)
    o_ref, lse_ref = vsa.attention(plan, *(torch_bf16(x) for x in host), scale=D ** -0.5)
    torch.cuda.synchronize()
    o_ref = o_ref.cpu().view(torch.int16)
    lse_ref = lse_ref.cpu()
    pinned = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in host]
    pipe = vsa.Pipeline(specs, grid, unit, 128, 128, B=B, D=D, chunk_heads=chunk)
    for _ in range(2):
        o = torch.empty((B, len(specs), N, D), dtype=torch.bfloat16).pin_memory()
        lse = torch.empty((B, len(specs), plan.n_slots), dtype=torch.float32).pin_memory()
        pipe.run(*pinned, o, lse, D ** -0.5)
        torch.cuda.synchronize()
        pipe.check()
        assert torch.equal(o.view(torch.int16), o_ref)
        # lse rows of padding slots are unspecified; compare the real ones
        for h, spec in enumerate(specs):
            import oracle
            perm = oracle.tile_major_order(grid, unit, plan.n_slots, layout=spec["layout"])
            real = torch.from_numpy(perm >= 0)
            assert torch.equal(lse[:, h][:, real], lse_ref[:, h][:, real])
    pipe.close()
    plan.close()
