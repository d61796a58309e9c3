"""The C-ABI library loads without a GPU and exports every entry point that
include/moe.h declares (no compute calls)."""
import ctypes
import os
import re

import quantized_moe_route_b200 as moe
from quantized_moe_route_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ["moe_pack_w4", "moe_route", "moe_permute", "moe_ffn_w4a16_decode",
                 "moe_ffn_grouped_prefill", "moe_unpermute_combine"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    moe_build.build()
    L = ctypes.CDLL(moe.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing
    assert set(declared_functions()) <= set(moe.SIGNATURES)


def test_host_only_queries():
    L = moe.lib()
    assert L.moe_w4_packed_bytes(1024, 2048) == 1179648
    assert L.moe_status_string(2) == b"MOE_ERR_UNSUPPORTED_SHAPE"
    assert L.moe_version().startswith(b"moe-w4-b200")
    assert L.moe_decode_workspace_bytes(1, 8, 512) >= 8 * 512 * 8  # one 8-byte h word per value
    # fused layer: h words and one 8-byte output word per (row, channel)
    assert L.moe_decode_layer_workspace_bytes(1, 8, 2048, 512) >= 8 * 8 * (512 + 2048)
