"""moe_permute_static_ws: the permutation for callers that cannot allocate
device memory at the call site (their memory belongs to a framework
allocator, or they must not risk the implicit synchronisation of cudaMalloc,
or their plugin interface passes only inputs and outputs). It keeps its
scratch in the library's own fixed 1 MiB device array.

Checked through the C ABI against moe_permute with a caller workspace, on two
calls in a row with different sizes (the shared array keeps the previous
call's contents), plus the size limit. This file is collected last on
purpose and also runs alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_limited_b200 import native as N

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _outputs(T, k, E, H):
    R = T * k
    return dict(offsets=torch.full((E + 1,), -7, dtype=torch.int32, device=DEV),
                src=torch.full((R,), -7, dtype=torch.int32, device=DEV),
                s2r=torch.full((R,), -7, dtype=torch.int32, device=DEV),
                roww=torch.full((R,), -7.0, dtype=torch.float32, device=DEV),
                xp=torch.zeros(R, H, dtype=torch.bfloat16, device=DEV))


def _inputs(T, k, E, H, seed):
    rng = np.random.default_rng(seed)
    L = rng.standard_normal((T, E)).astype(np.float32)
    r = oracle.route_from_logits(L, k, 1, 1, "softmax", False, 1.0)
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    x = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    return (torch.from_numpy(r.ids).to(DEV), torch.from_numpy(r.weights.astype(np.float32)).to(DEV), x)


def test_static_workspace_permute_matches_allocating_entry_point():
    lib = N.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, (T, k, E, H, seed) in enumerate([(8192, 8, 256, 512, 1), (1000, 6, 64, 256, 2)]):
        ids, tw, x = _inputs(T, k, E, H, seed)
        ref = _outputs(T, k, E, H)
        ws = torch.empty(N.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=DEV)
        N.moe_permute(T, k, E, H, ids, tw, x, N.MOE_BF16, None, ref["xp"], None, ref["offsets"],
                      ref["src"], ref["s2r"], ref["roww"], ws)
        got = _outputs(T, k, E, H)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        rc = lib.moe_permute_static_ws(T, k, E, H, _ptr(ids), _ptr(tw), _ptr(x), N.MOE_BF16, None,
                                       _ptr(got["xp"]), None, _ptr(got["offsets"]), _ptr(got["src"]),
                                       _ptr(got["s2r"]), _ptr(got["roww"]), _ptr(status), stream)
        assert rc == N.MOE_OK, f"call {call}: status {rc}"
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for key in ref:
            assert torch.equal(got[key], ref[key]), f"call {call}: {key} differs"


def test_static_workspace_rejects_sizes_beyond_its_array():
    lib = N.load_library()
    fake = ctypes.c_void_p(0x1000)      # never dereferenced: the size check comes first
    # ceil(70000 / 64) * 256 = 280064 int32 > 262144
    rc = lib.moe_permute_static_ws(70000, 8, 256, 512, fake, fake, fake, N.MOE_BF16, None, fake, None,
                                   fake, fake, fake, fake, None, None)
    assert rc == N.MOE_ERR_UNSUPPORTED
