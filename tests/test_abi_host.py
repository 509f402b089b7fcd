"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point the header declares, sizes workspaces, and rejects bad
arguments before launching anything."""

import ctypes

import pytest

from bit_expert_gemm_b200 import abi


def test_library_exports_every_header_symbol():
    lib = abi.load()
    names = abi.header_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(abi._SIGS)  # the binding covers exactly the header
    assert lib.moe_abi_version() == 2


def test_workspace_sizes():
    lib = abi.load()
    assert lib.moe_workspace_size(abi.MOE_OP_ROUTE_TOPK, 8192, 2048, 512, 10, 640) >= 8192 * 512 * 4
    big = lib.moe_workspace_size(abi.MOE_OP_SWIGLU_BF16, 8192, 2048, 512, 10, 640)
    assert big >= 81920 * 640 * 2  # h between the GEMMs (GEMM1 gathers x rows itself)
    # routed + shared experts: h [rows, I] for prefill, h [rows + T, I] (shared rows appended) for decode
    assert lib.moe_workspace_size(abi.MOE_OP_EXPERTS_BF16, 8192, 2048, 512, 10, 640) >= 81920 * 640 * 2
    assert lib.moe_workspace_size(abi.MOE_OP_EXPERTS_BF16, 64, 2048, 512, 10, 640) >= (640 + 64) * 640 * 2  # 16-bit h
    # T <= 16: FP32 split-K partials [I/64][rows + T][H]
    assert lib.moe_workspace_size(abi.MOE_OP_EXPERTS_BF16, 1, 2048, 512, 10, 640) >= 10 * 11 * 2048 * 4
    assert lib.moe_workspace_size(abi.MOE_OP_PERMUTE, 32768, 2048, 512, 11, 640) >= 512 * 1024 * 8
    assert lib.moe_workspace_size(99, 1, 1, 1, 1, 1) == 0
    assert lib.moe_workspace_size(abi.MOE_OP_ROUTE_TOPK, -1, 1, 1, 1, 1) == 0


def _code(fn, *args):
    return getattr(abi.load(), fn)(*args)


@pytest.mark.parametrize("k,extra,E,H", [(0, 0, 16, 256), (17, 0, 512, 256), (10, 1, 10, 256), (2, 0, 2048, 256),
                                         (2, 0, 16, 100), (2, 3, 16, 256)])
def test_route_rejects_bad_shapes(k, extra, E, H):
    rc = _code("moe_route_topk", None, 4, H, None, None, E, k, extra, 0, None, None, None, None, 0, None)
    assert rc in (abi.MOE_ERR_UNSUPPORTED, abi.MOE_ERR_INVALID_ARG)
    assert abi.load().moe_last_error().decode()
    off = ctypes.c_void_p(256)  # never dereferenced: the shape check comes first
    rc = _code("moe_route_permute", None, 4, H, None, None, E, k, extra, 0, None, None, None, off, None, None, None,
               0, None)
    assert rc in (abi.MOE_ERR_UNSUPPORTED, abi.MOE_ERR_INVALID_ARG)


def test_calls_reject_null_pointers_and_bad_sizes():
    assert _code("moe_route_topk", None, 4, 256, None, None, 16, 2, 0, 0, None, None, None, None, 0, None) == \
        abi.MOE_ERR_INVALID_ARG
    assert _code("moe_permute", None, 4, 2, 2000, None, None, None, None, 0, None) == abi.MOE_ERR_UNSUPPORTED
    assert _code("moe_route_permute", None, 4, 256, None, None, 16, 2, 0, 0, None, None, None, None, None, None, None,
                 0, None) == abi.MOE_ERR_INVALID_ARG  # expert_offsets is null
    assert _code("moe_route_permute", None, 4, 256, None, None, 16, 2, 0, 0, None, None, None, ctypes.c_void_p(256),
                 None, None, None, 0, None) == abi.MOE_ERR_INVALID_ARG  # x is null
    assert _code("moe_permute", None, 4, 2, 16, None, None, None, None, 0, None) == abi.MOE_ERR_INVALID_ARG
    assert _code("moe_grouped_swiglu_bf16", None, None, None, 4, 8, 100, 64, 4, None, None, 0, 0, None, None, 0,
                 None) == abi.MOE_ERR_UNSUPPORTED
    assert _code("moe_grouped_swiglu_bf16", None, None, None, 4, 8, 256, 64, 4, None, None, 0, 0, None, None, 0,
                 None) == abi.MOE_ERR_INVALID_ARG  # identity rows need rows == T
    assert _code("moe_combine", None, 0, None, 2, None, None, None, 4, 3, 256, 0, None, None) == \
        abi.MOE_ERR_INVALID_ARG  # k > k_slots
    assert _code("razor_select", None, None, 16, 17, None, None, None, None) == abi.MOE_ERR_INVALID_ARG
    assert _code("razor_select", None, None, 0, 0, None, None, None, None) == abi.MOE_ERR_UNSUPPORTED
    assert _code("moe_nvfp4_quantize", None, 1, 4, 24, 0, None, None, None, None, None, 0, None) == \
        abi.MOE_ERR_UNSUPPORTED
    # the bounded-wait self-test checks its limit and output before launching
    assert _code("moe_selftest_bounded_wait", 50, ctypes.c_void_p(256), None) == abi.MOE_ERR_UNSUPPORTED
    assert _code("moe_selftest_bounded_wait", 2_000_000, ctypes.c_void_p(256), None) == abi.MOE_ERR_UNSUPPORTED
    assert _code("moe_selftest_bounded_wait", 2000, None, None) == abi.MOE_ERR_INVALID_ARG


def test_zero_sized_calls_are_no_ops():
    # nothing to do: returns OK without touching the device
    assert _code("moe_route_topk", None, 0, 256, None, None, 16, 2, 0, 0, None, None, None, None, 0, None) == abi.MOE_OK
    assert _code("moe_grouped_swiglu_bf16", None, ctypes.c_void_p(16), None, 0, 0, 256, 64, 4, None, None, 0, 0, None,
                 None, 0, None) == abi.MOE_OK
    assert _code("moe_combine", None, 0, None, 2, None, None, None, 0, 2, 256, 0, None, None) == abi.MOE_OK


def test_nvfp4_prepack_sizes_and_checks():
    lib = abi.load()
    # one 2 KB scale tile per 128 rows and 256 K per expert
    assert lib.moe_nvfp4_packed_sf_bytes(512, 1280, 2048, 1) == 512 * 10 * 8 * 2048
    assert lib.moe_nvfp4_packed_sf_bytes(512, 2048, 640, 0) == 512 * 16 * 3 * 2048
    assert lib.moe_nvfp4_packed_sf_bytes(4, 100, 256, 0) == 0
    buf = ctypes.c_void_p(256)  # never dereferenced: the checks come first
    assert _code("moe_nvfp4_prepack_sf", buf, 4, 100, 256, 0, buf, 1 << 20, None) == abi.MOE_ERR_UNSUPPORTED
    assert _code("moe_nvfp4_prepack_sf", buf, 4, 128, 256, 2, buf, 1 << 20, None) == abi.MOE_ERR_INVALID_ARG
    assert _code("moe_nvfp4_prepack_sf", None, 4, 128, 256, 0, buf, 1 << 20, None) == abi.MOE_ERR_INVALID_ARG
    assert _code("moe_nvfp4_prepack_sf", buf, 4, 128, 256, 0, buf, 4 * 2048 - 1, None) == abi.MOE_ERR_WORKSPACE
    assert _code("moe_grouped_swiglu_nvfp4_prepacked", None, None, None, 4, 8, 256, 100, 4, None, None, None, None,
                 None, None, None, None, 0, None, None, 0, None) == abi.MOE_ERR_UNSUPPORTED
    assert _code("moe_grouped_swiglu_nvfp4_prepacked", buf, None, buf, 4, 4, 256, 128, 4, buf, None, buf, buf, buf,
                 buf, None, None, 0, buf, None, 0, None) == abi.MOE_ERR_INVALID_ARG  # packed gate/up scales missing
    assert _code("moe_grouped_swiglu_nvfp4_prepacked", None, None, None, 0, 0, 256, 128, 4, None, None, None, None,
                 None, None, None, None, 0, None, None, 0, None) == abi.MOE_OK


def test_awq_prepack_sizes_and_checks():
    lib = abi.load()
    # packed units: I/64 x (H/64 + H/128) per expert, 4736 bytes each = the AWQ bytes of an expert
    assert lib.moe_awq_packed_bytes(512, 2048, 640) == 512 * 10 * 48 * 4736 == 512 * 2273280
    assert lib.moe_awq_packed_bytes(4, 100, 64) == 0
    buf = ctypes.c_void_p(256)  # never dereferenced: the checks come first
    assert _code("moe_awq_prepack_g32", buf, buf, buf, buf, buf, buf, 4, 2048, 100, buf, 1 << 30, None) == \
        abi.MOE_ERR_UNSUPPORTED
    assert _code("moe_awq_prepack_g32", buf, buf, buf, None, buf, buf, 4, 2048, 640, buf, 1 << 30, None) == \
        abi.MOE_ERR_INVALID_ARG
    assert _code("moe_awq_prepack_g32", buf, buf, buf, buf, buf, buf, 4, 2048, 640, buf, 1000, None) == \
        abi.MOE_ERR_WORKSPACE
    assert _code("moe_experts_awq_g32_prepacked", buf, buf, buf, 1, 10, 2048, 640, 16, buf, buf, buf, buf, buf, buf,
                 None, buf, buf, abi.MOE_DTYPE_F16, 0, buf, buf, buf, 1 << 30, None) == \
        abi.MOE_ERR_INVALID_ARG  # awq_packed is null
    # the AWQ calls take FP16 or (BF16 mode) BF16 activations, nothing else
    assert _code("moe_experts_awq_g32", buf, buf, buf, 1, 10, 2048, 640, 16, buf, buf, buf, buf, buf, buf, buf, buf,
                 7, 0, buf, buf, buf, 1 << 30, None) == abi.MOE_ERR_INVALID_ARG
    assert _code("moe_grouped_swiglu_awq_g32", buf, buf, buf, 1, 10, 2048, 640, 16, buf, buf, buf, buf, buf, buf,
                 7, 0, buf, buf, 1 << 30, None) == abi.MOE_ERR_INVALID_ARG
    assert _code("moe_awq_dequant_g32", buf, buf, buf, 1, 64, 64, 7, buf, None) == abi.MOE_ERR_INVALID_ARG


def test_razor_slice_and_router_norm_reject_bad_arguments():
    p = ctypes.c_void_p
    # keep above E, negative keep, E <= 0
    assert _code("razor_slice", p(256), 4, 16, p(512), 5, p(1 << 20), None) == abi.MOE_ERR_INVALID_ARG
    assert _code("razor_slice", p(256), 4, 16, p(512), -1, p(1 << 20), None) == abi.MOE_ERR_INVALID_ARG
    assert _code("razor_slice", p(256), 0, 16, p(512), 0, p(1 << 20), None) == abi.MOE_ERR_INVALID_ARG
    # null pointers, and a dst that overlaps src (E * 4096 bytes from 4096)
    assert _code("razor_slice", None, 4, 16, p(512), 2, p(1 << 20), None) == abi.MOE_ERR_INVALID_ARG
    assert _code("razor_slice", p(4096), 4, 4096, None, 2, p(1 << 20), None) == abi.MOE_ERR_INVALID_ARG
    assert _code("razor_slice", p(4096), 4, 4096, p(512), 2, p(8192), None) == abi.MOE_ERR_INVALID_ARG
    assert "overlaps" in abi.load().moe_last_error().decode()
    # nothing to copy: accepted without touching memory
    assert _code("razor_slice", None, 4, 16, None, 0, None, None) == abi.MOE_OK
    assert _code("razor_router_norm", None, 16, 256, 0, p(256), None, None) == abi.MOE_ERR_INVALID_ARG
    assert _code("razor_router_norm", p(256), 16, 256, 7, p(256), None, None) == abi.MOE_ERR_INVALID_ARG
    assert _code("razor_router_norm", p(256), 0, 256, 0, p(256), None, None) == abi.MOE_ERR_INVALID_ARG


def test_keep_manifest():
    from bit_expert_gemm_b200.layer import keep_manifest

    m = keep_manifest([1, 4, 7], 8, scores=[0.0, 2.0, 0.5, 0.1, 3.0, 0.0, 0.0, 1.0])
    assert m["kept_expert_indices"] == [1, 4, 7] and m["experts_kept"] == 3 and m["experts_before"] == 8
    assert m["aggregation"] == "rms" and m["kept_scores"] == [2.0, 3.0, 1.0]
    assert keep_manifest([0, 2], 4, policy="router_norm")["policy"] == "router_norm"
    for bad in ([2, 1], [1, 1], [0, 8]):
        with pytest.raises(ValueError):
            keep_manifest(bad, 8)


def test_rmsnorm_rejects_bad_arguments():
    p = ctypes.c_void_p
    assert _code("moe_rmsnorm", p(256), 4, 100, p(512), ctypes.c_float(1e-6), 0, p(1024), None) == \
        abi.MOE_ERR_UNSUPPORTED  # H % 8 != 0
    assert _code("moe_rmsnorm", p(256), 4, 64, p(512), ctypes.c_float(1e-6), 9, p(1024), None) == \
        abi.MOE_ERR_INVALID_ARG  # dtype
    assert _code("moe_rmsnorm", p(260), 4, 64, p(512), ctypes.c_float(1e-6), 0, p(1024), None) == \
        abi.MOE_ERR_INVALID_ARG  # misaligned x
    assert _code("moe_rmsnorm", None, 0, 64, None, ctypes.c_float(1e-6), 0, None, None) == abi.MOE_OK  # empty batch


def test_header_is_plain_c_and_links(tmp_path):
    """include/moe.h compiles as strict C99, and a C program links against
    libmoe_b200.so and calls it (moe_abi_version needs no GPU)."""
    import os
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    inc = os.path.dirname(abi.HEADER)
    libdir = os.path.dirname(abi.LIB_PATH)
    src = tmp_path / "use_moe.c"
    src.write_text('#include "moe.h"\nint main(void) { return moe_abi_version() == 2 ? 0 : 1; }\n')
    exe = tmp_path / "use_moe"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", f"-I{inc}", str(src),
                        f"-L{libdir}", "-lmoe_b200", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert subprocess.run([str(exe)]).returncode == 0
