"""The C-ABI library builds for sm_100a, loads without a GPU and exports every
entry point declared in include/*.h (no compute calls here)."""
import ctypes
import glob
import os
import re


from combine_moe_dispatch_05_b200 import build as B
from combine_moe_dispatch_05_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        names += re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", open(h).read(), re.M)
    return names


def test_header_declares_the_entry_points():
    names = set(declared_symbols())
    for n in ["moe_dispatch_layout", "moe_dispatch_permute", "moe_combine", "moe_combine_bwd",
              "moe_dispatch_bwd"]:
        assert n in names


def test_library_loads_and_exports_every_declared_symbol():
    B.build()
    L = ctypes.CDLL(ops.LIB_PATH)
    names = declared_symbols()
    assert names
    for n in names:
        assert hasattr(L, n), n
        assert n in ops.SIGNATURES, f"binding lacks {n}"
    assert set(ops.SIGNATURES) == set(names)


def test_host_only_entry_points():
    B.build()
    assert ops.lib().moe_version() >= 100
    assert ops.padded_capacity(5, 2, 4) == 640
    assert ops.padded_capacity(4096, 8, 256) == 65280
    assert ops.padded_capacity(0, 8, 256) == 0
    assert ops.lib().moe_padded_capacity(1, 17, 4) == -1
    assert ops.layout_workspace_bytes(4096, 8, 256) > 0
    assert ops.status_string(ops.ERR_TIMEOUT) == "device-side wait timed out"


def test_dispatch_in_one_call_checks_both_halves_before_launching():
    """moe_dispatch checks the layout's and the permute's arguments before it
    launches either kernel: a bad permute argument returns its own code, not
    a launch failure of the layout (there is no GPU here, so any launch would
    return ERR_CUDA)."""
    B.build()
    L = ops.lib()
    f = ctypes.c_void_p(256)
    T, K, E, R, H = 4, 2, 4, 2, 64
    ws = ops.layout_workspace_bytes(T, K, E)

    def call(E=E, R=R, dtype=0, stride=H, P_cap=1024, work=f, ws_bytes=ws):
        return L.moe_dispatch(f, T, K, E, R, f, dtype, H, stride, None, 0, f, f, f, f, f, f, f,
                              P_cap, f, ws_bytes, f, None, work, None, None)

    assert call(E=6, R=4) == ops.ERR_INVALID_ARG           # E % R != 0 (layout)
    assert call(P_cap=128) == ops.ERR_CAPACITY             # P_cap below the bound (layout)
    assert call(ws_bytes=ws - 4) == ops.ERR_INVALID_ARG    # workspace too small (layout)
    assert call(dtype=7) == ops.ERR_UNSUPPORTED            # unknown dtype (permute)
    assert call(stride=H - 8) == ops.ERR_INVALID_ARG       # row stride below H (permute)
    assert call(work=None) == ops.ERR_INVALID_ARG          # no scheduling words (permute)


def test_layout_workspace_follows_the_block_size():
    """The layout scratch holds per-block expert counts (one int32 per expert
    per block) and one int32 rank per slot, each region padded to 256 bytes.
    Blocks own 1024 slots when the batch has at most 65536, 2048 above."""
    B.build()

    def expect(T, K, E):
        per_block = (1024 if T * K <= 65536 else 2048) // K  # whole tokens per block
        nb = (T + per_block - 1) // per_block if T else 1
        pad = lambda n: (n + 255) // 256 * 256
        return pad(nb * E * 4) + pad(max(T, 1) * K * 4)

    for T, K, E in [(4096, 8, 256), (8192, 8, 256), (8193, 8, 256), (21845, 3, 9),
                    (21846, 3, 9), (65536, 1, 4), (65537, 1, 4), (32768, 8, 256), (1, 16, 512),
                    (0, 4, 8), (116480, 8, 256)]:
        assert ops.layout_workspace_bytes(T, K, E) == expect(T, K, E), (T, K, E)


def test_host_argument_errors_launch_nothing():
    """Argument checks return before any CUDA call, so they run without a GPU."""
    B.build()
    L = ops.lib()
    null = None
    # E % R != 0
    assert L.moe_dispatch_layout(null, 4, 2, 6, 4, null, null, null, null, null, null, null,
                                 1024, null, null, 0, null) == ops.ERR_INVALID_ARG
    # capacity too small
    fake = ctypes.c_void_p(256)
    assert L.moe_dispatch_layout(fake, 4, 2, 4, 1, fake, fake, fake, fake, fake, fake, fake,
                                 128, fake, fake, 1 << 20, null) == ops.ERR_CAPACITY
    # K out of range
    assert L.moe_combine(fake, fake, fake, null, 4, 17, 64, 1024, fake, null,
                         null) == ops.ERR_INVALID_ARG
    # H not a multiple of 8
    assert L.moe_combine(fake, fake, fake, null, 4, 2, 12, 1024, fake, null,
                         null) == ops.ERR_INVALID_ARG
    # misaligned output
    assert L.moe_combine(fake, fake, fake, null, 4, 2, 64, 1024, ctypes.c_void_p(260), null,
                         null) == ops.ERR_INVALID_ARG
    # bad dtype
    assert L.moe_dispatch_permute(fake, 7, 4, 64, 64, null, 0, fake, 2, fake, fake, 4, fake,
                                  null, 1024, null, fake, null, null) == ops.ERR_UNSUPPORTED
    # E4M3 needs H % 128 == 0
    assert L.moe_dispatch_permute(fake, 1, 4, 64, 64, fake, 0, fake, 2, fake, fake, 4, fake,
                                  fake, 1024, null, fake, null, null) == ops.ERR_INVALID_ARG
    # row stride smaller than H
    assert L.moe_dispatch_permute(fake, 0, 4, 64, 32, null, 0, fake, 2, fake, fake, 4, fake,
                                  null, 1024, null, fake, null, null) == ops.ERR_INVALID_ARG
    # no scheduling words
    assert L.moe_dispatch_permute(fake, 0, 4, 64, 64, null, 0, fake, 2, fake, fake, 4, fake,
                                  null, 1024, null, null, null, null) == ops.ERR_INVALID_ARG
    assert L.moe_quantize_e4m3(fake, 4, 100, 100, fake, fake, null, null) == ops.ERR_INVALID_ARG
    assert L.moe_combine_bwd(fake, fake, fake, fake, fake, fake, 4, 4, 2, 64, 128, fake, fake,
                             null, null) == ops.ERR_CAPACITY
