"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/moe.h declares, and rejects bad arguments on the host before any
launch (nothing here touches a device)."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_limited_b200 import native as N
from mixture_experts_layer_limited_b200.build import lib_path

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

pytestmark = pytest.mark.skipif(not os.path.exists(lib_path()),
                                reason="libmoe.so not built (run the package build)")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src, flags=re.M)))


def test_header_declarations_match_binding_list():
    assert declared_functions() == sorted(N.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(lib_path())
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_abi_version_and_status_strings():
    lib = N.load_library()
    assert lib.moe_abi_version() == 3
    assert lib.moe_status_string(0) == b"ok"
    assert b"invalid" in lib.moe_status_string(N.MOE_ERR_INVALID_ARG)
    assert lib.moe_status_string(99) == b"unknown status"
    assert lib.moe_last_cuda_error() == 0


def test_workspace_size_is_host_only():
    assert N.moe_permute_workspace_size(8192, 8, 256) == (8192 // 64) * 256 * 4
    assert N.moe_permute_workspace_size(65, 8, 16) == 2 * 16 * 4
    with pytest.raises(N.MoEError):
        N.moe_permute_workspace_size(0, 8, 256)


def test_ffn_sync_size_and_host_validation():
    """The one-launch FFN's scratch: an int32 counter per possible token block
    of the routed rows (one partial block per group at most) and of the
    shared rows, plus the tile counter; short, misaligned or missing scratch
    and a non-bf16 layer are rejected on the host, before any launch."""
    R, E, T = 65536, 256, 8192
    assert N.moe_swiglu_ffn_sync_size(R, E, T) == 4 * ((R + 255) // 256 + E + (T + 255) // 256 + 1)
    with pytest.raises(N.MoEError):
        N.moe_swiglu_ffn_sync_size(0, E, T)
    lib = N.load_library()
    P = ctypes.c_void_p
    fake = P(0x1000)
    w = N.FFNWeights(fake, fake, None, None, N.MOE_BF16, 4, 256)
    sw = N.FFNWeights(fake, fake, None, None, N.MOE_BF16, 1, 256)
    need = N.moe_swiglu_ffn_sync_size(64, 4, 16)

    def call(sync, nbytes, weights=w):
        return lib.moe_swiglu_ffn_with_shared(64, 512, ctypes.byref(weights), fake, fake, None, fake, fake,
                                              16, ctypes.byref(sw), fake, fake, fake, sync, nbytes, None, None)
    assert call(fake, need - 4) == N.MOE_ERR_INVALID_ARG
    assert call(None, need) == N.MOE_ERR_INVALID_ARG
    assert call(P(0x1004), need) == N.MOE_ERR_ALIGNMENT
    e4 = N.FFNWeights(fake, fake, fake, fake, N.MOE_E4M3, 4, 256)
    assert call(fake, need, e4) != N.MOE_OK


def test_tiled_weights_host_validation():
    """moe_tile_ffn_weights and the GEMM calls check the weight layout flag on
    the host: only bf16 weights tile, a tiled source or a flag other than 0/1
    is refused, shapes outside the GEMM limits or past int32 tiled rows are
    unsupported, and misaligned buffers are caught, all before any launch."""
    lib = N.load_library()
    P = ctypes.c_void_p
    fake, odd = P(0x1000), P(0x1004)

    def w(dtype=N.MOE_BF16, groups=4, I=256, tiled=0, w13=fake, scale=None):
        f = N.FFNWeights(w13, fake, scale, scale, dtype, groups, I)
        f.tiled = tiled
        return f

    def tile(H, src, w13_t=fake, w2_t=fake):
        return lib.moe_tile_ffn_weights(H, ctypes.byref(src) if src is not None else None, w13_t, w2_t, None)
    assert tile(512, None) == N.MOE_ERR_INVALID_ARG
    assert tile(512, w(tiled=1)) == N.MOE_ERR_INVALID_ARG                 # already tiled
    assert tile(512, w(dtype=N.MOE_E4M3, scale=fake)) == N.MOE_ERR_UNSUPPORTED
    assert tile(384, w()) == N.MOE_ERR_UNSUPPORTED                        # H % 256
    assert tile(512, w(I=192)) == N.MOE_ERR_UNSUPPORTED                   # I % 128
    assert tile(65536, w(groups=512, I=8192)) == N.MOE_ERR_UNSUPPORTED    # tiled rows past int32
    assert tile(512, w(w13=None)) == N.MOE_ERR_INVALID_ARG                # w13_t without w13
    assert tile(512, w(), w13_t=odd) == N.MOE_ERR_ALIGNMENT
    # outputs may not overlap the inputs or each other (w13 at 0x1000 spans 4*512*512*2 bytes)
    assert tile(512, w(), w13_t=P(0x1000 + 4096), w2_t=P(0x10000000)) == N.MOE_ERR_INVALID_ARG
    assert tile(512, w(), w13_t=P(0x10000000), w2_t=P(0x10000000 + 4096)) == N.MOE_ERR_INVALID_ARG

    def gate_up(weights, H=512):
        return lib.moe_gate_up_swiglu(64, H, ctypes.byref(weights), fake, None, fake, fake, None, None, None)
    assert gate_up(w(tiled=2)) == N.MOE_ERR_INVALID_ARG
    assert gate_up(w(tiled=-1)) == N.MOE_ERR_INVALID_ARG
    assert gate_up(w(dtype=N.MOE_E4M3, scale=fake, tiled=1)) == N.MOE_ERR_UNSUPPORTED
    assert gate_up(w(groups=512, I=8192, tiled=1), H=65536) == N.MOE_ERR_UNSUPPORTED
    assert lib.moe_last_cuda_error() == 0      # nothing above reached the CUDA runtime


def _raw(lib, fn, *args):
    return getattr(lib, fn)(*args)


def test_host_validation_rejects_before_launch():
    lib = N.load_library()
    P = ctypes.c_void_p
    fake = P(0x1000)          # never dereferenced: every call below fails validation first
    odd = P(0x1004)
    # moe_route: no params / k > E / unsupported E / misaligned pointer
    assert lib.moe_route(None, fake, fake, None, None, fake, fake, fake, None) == N.MOE_ERR_INVALID_ARG
    p = N.RouteParams(16, 256, 16, 17, 1, 1, N.MOE_SOFTMAX, 0, 1.0, None)
    assert lib.moe_route(ctypes.byref(p), fake, fake, None, fake, fake, fake, fake, None) == N.MOE_ERR_INVALID_ARG
    p = N.RouteParams(16, 256, 24, 4, 1, 1, N.MOE_SOFTMAX, 0, 1.0, None)
    assert lib.moe_route(ctypes.byref(p), fake, fake, None, fake, fake, fake, fake, None) == N.MOE_ERR_UNSUPPORTED
    p = N.RouteParams(16, 256, 256, 8, 8, 4, N.MOE_SIGMOID, 1, 2.5, None)
    assert lib.moe_route(ctypes.byref(p), odd, fake, None, fake, fake, fake, fake, None) == N.MOE_ERR_ALIGNMENT
    # logits are required (the gate GEMM writes them, routing reads them)
    p = N.RouteParams(16, 256, 16, 4, 1, 1, N.MOE_SOFTMAX, 0, 1.0, None)
    assert lib.moe_route(ctypes.byref(p), fake, fake, None, None, fake, fake, fake, None) == N.MOE_ERR_INVALID_ARG
    # group limit makes k impossible: 4 groups of 4, keep 1 -> at most 4 candidates
    p = N.RouteParams(16, 256, 16, 5, 4, 1, N.MOE_SIGMOID, 1, 2.5, None)
    assert lib.moe_route(ctypes.byref(p), fake, fake, None, fake, fake, fake, fake, None) == N.MOE_ERR_INVALID_ARG
    # moe_gate_logits: T, H not a multiple of 64, E beyond 256, misaligned logits
    assert lib.moe_gate_logits(0, 256, 16, fake, fake, fake, None, None) == N.MOE_ERR_INVALID_ARG
    assert lib.moe_gate_logits(8, 200, 16, fake, fake, fake, None, None) == N.MOE_ERR_UNSUPPORTED
    assert lib.moe_gate_logits(8, 256, 512, fake, fake, fake, None, None) == N.MOE_ERR_UNSUPPORTED
    assert lib.moe_gate_logits(8, 256, 16, fake, None, fake, None, None) == N.MOE_ERR_INVALID_ARG
    assert lib.moe_gate_logits(8, 256, 16, fake, fake, odd, None, None) == N.MOE_ERR_ALIGNMENT
    # moe_permute: missing workspace, too small workspace, unsupported E
    args = [fake, fake, fake, N.MOE_BF16, None, fake, N.MOE_BF16, None, None, None, fake, fake, fake, fake]
    assert lib.moe_permute(64, 4, 16, 256, *args, None, 0, None, None) == N.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(64, 4, 16, 256, *args, fake, 4, None, None) == N.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(64, 4, 2048, 256, *args, fake, 1 << 20, None, None) == N.MOE_ERR_UNSUPPORTED
    # perm_dtype: E4M3 codes cannot become bf16 rows; quantising needs x_perm_scale and H % 128;
    # x_q only when quantising, and with its scales
    def perm(x_dt, p_dt, xps, xq, xqs, H=256):
        return lib.moe_permute(64, 4, 16, H, fake, fake, fake, x_dt, fake, fake, p_dt, xps, xq, xqs,
                               fake, fake, fake, fake, fake, 1 << 20, None, None)
    assert perm(N.MOE_E4M3, N.MOE_BF16, None, None, None) == N.MOE_ERR_UNSUPPORTED
    assert perm(N.MOE_BF16, N.MOE_E4M3, None, None, None) == N.MOE_ERR_INVALID_ARG
    assert perm(N.MOE_BF16, N.MOE_E4M3, fake, None, None, H=200) == N.MOE_ERR_UNSUPPORTED
    assert perm(N.MOE_BF16, N.MOE_BF16, None, fake, fake) == N.MOE_ERR_INVALID_ARG
    assert perm(N.MOE_BF16, N.MOE_E4M3, fake, fake, None) == N.MOE_ERR_INVALID_ARG
    assert perm(N.MOE_BF16, 7, fake, None, None) == N.MOE_ERR_INVALID_ARG
    # moe_grouped_swiglu: H not a multiple of 256, offsets NULL with groups > 1
    w = N.FFNWeights(fake, fake, None, None, N.MOE_BF16, 4, 128)
    assert lib.moe_grouped_swiglu(64, 200, ctypes.byref(w), fake, None, fake, None, fake, None, fake,
                                  None, None) == N.MOE_ERR_UNSUPPORTED
    assert lib.moe_grouped_swiglu(64, 256, ctypes.byref(w), fake, None, None, None, fake, None, fake,
                                  None, None) == N.MOE_ERR_INVALID_ARG
    w8 = N.FFNWeights(fake, fake, None, None, N.MOE_E4M3, 4, 128)
    assert lib.moe_grouped_swiglu(64, 256, ctypes.byref(w8), fake, None, fake, None, fake, None, fake,
                                  None, None) == N.MOE_ERR_INVALID_ARG
    # moe_down_proj_combine: T, the token map, the shared expert's groups, H, alignment, E4M3
    w2 = N.FFNWeights(None, fake, None, None, N.MOE_BF16, 4, 128)
    sw2 = N.FFNWeights(None, fake, None, None, N.MOE_BF16, 2, 128)
    w2e = N.FFNWeights(None, fake, None, None, N.MOE_E4M3, 4, 128)
    def dpc(T, H, w, src, sw, y):
        return lib.moe_down_proj_combine(64, T, H, ctypes.byref(w), fake, fake, fake, src,
                                         ctypes.byref(sw) if sw is not None else None, fake, fake, y,
                                         None, None)
    assert dpc(0, 256, w2, fake, None, fake) == N.MOE_ERR_INVALID_ARG
    assert dpc(16, 256, w2, None, None, fake) == N.MOE_ERR_INVALID_ARG
    assert dpc(16, 256, w2, fake, sw2, fake) == N.MOE_ERR_INVALID_ARG
    assert dpc(16, 200, w2, fake, None, fake) == N.MOE_ERR_UNSUPPORTED
    assert dpc(16, 256, w2, fake, None, odd) == N.MOE_ERR_ALIGNMENT
    assert dpc(16, 256, w2e, fake, None, fake) != N.MOE_OK
    # moe_combine / moe_bias_update / quantisers
    assert lib.moe_combine(0, 4, 256, fake, fake, None, None, fake, None) == N.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(8, 4, 252, fake, fake, None, None, fake, None) == N.MOE_ERR_UNSUPPORTED
    assert lib.moe_bias_update(2048, 8, 4, fake, fake, ctypes.c_float(0.001), None, None) == N.MOE_ERR_UNSUPPORTED
    assert lib.moe_bias_update(16, 8, 4, None, fake, ctypes.c_float(0.001), None, None) == N.MOE_ERR_INVALID_ARG
    # moe_aux_loss: seq_len must divide T, workspace too small, E beyond 256, scoring
    assert N.moe_aux_loss_workspace_size(256, 16, 128) == 2 * 16 * 12
    with pytest.raises(N.MoEError):
        N.moe_aux_loss_workspace_size(100, 16, 30)
    assert lib.moe_aux_loss(100, 16, 4, 30, N.MOE_SOFTMAX, fake, fake, ctypes.c_float(1.0), fake, fake,
                            1 << 20, None, None) == N.MOE_ERR_INVALID_ARG
    assert lib.moe_aux_loss(256, 16, 4, 128, N.MOE_SOFTMAX, fake, fake, ctypes.c_float(1.0), fake, fake,
                            16, None, None) == N.MOE_ERR_INVALID_ARG
    assert lib.moe_aux_loss(256, 512, 4, 256, N.MOE_SIGMOID, fake, fake, ctypes.c_float(1.0), fake, fake,
                            1 << 20, None, None) == N.MOE_ERR_UNSUPPORTED
    assert lib.moe_aux_loss(256, 16, 4, 256, 7, fake, fake, ctypes.c_float(1.0), fake, fake,
                            1 << 20, None, None) == N.MOE_ERR_INVALID_ARG
    assert lib.moe_quantize_blocks(1, 100, 128, fake, fake, fake, None) == N.MOE_ERR_UNSUPPORTED
    assert lib.moe_quantize_rows(4, 128, odd, fake, fake, None) == N.MOE_ERR_ALIGNMENT
    assert lib.moe_read_device_status(None, None, None) == N.MOE_ERR_INVALID_ARG
    assert lib.moe_last_cuda_error() == 0


def test_header_is_plain_c_and_a_c_program_links_and_calls_it(tmp_path):
    """include/moe.h compiles as C99 (no C++ or torch types in the
    boundary), and a C program linked against libmoe.so calls it: the ABI
    version, a workspace size, and an argument check that fails before any
    launch (no GPU needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    from mixture_experts_layer_limited_b200.build import lib_path
    lib = lib_path()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "use_moe.c"
    src.write_text(r'''
#include <stdio.h>
#include "moe.h"
int main(void) {
  size_t ws = 0;
  moe_status s = moe_permute_workspace_size(8192, 8, 256, &ws);
  moe_status bad = moe_combine(0, 8, 7168, NULL, NULL, NULL, NULL, NULL, NULL);
  printf("%d %d %zu %d %s\n", (int)moe_abi_version(), (int)s, ws, (int)bad, moe_status_string(bad));
  return 0;
}
''')
    exe = tmp_path / "use_moe"
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"), str(src), "-o", str(exe),
           lib, "-Wl,-rpath," + os.path.dirname(lib)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    ver, s, ws, bad, *msg = out.stdout.split()
    assert int(ver) == N.load_library().moe_abi_version()
    assert int(s) == N.MOE_OK and int(ws) == N.moe_permute_workspace_size(8192, 8, 256)
    assert int(bad) == N.MOE_ERR_INVALID_ARG


def test_wait_limit_knob_round_trip_is_host_only():
    """moe_set_wait_limit_ns only records the limit for later launches."""
    assert N.moe_wait_limit_ns() == 2_000_000_000
    try:
        N.moe_set_wait_limit_ns(12345)
        assert N.moe_wait_limit_ns() == 12345
    finally:
        N.moe_set_wait_limit_ns(0)
    assert N.moe_wait_limit_ns() == 2_000_000_000
