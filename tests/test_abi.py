"""The C-ABI library loads, exports every entry point its header declares, and
validates descriptors on the host (no GPU needed)."""
import ctypes
import os
import re

import pytest

from expert_routed_ffn_route_b200 import _build, binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return binding.load_library()


def header_functions():
    src = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_exports_match_header(lib):
    names = header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(binding.EXPORTS)
    assert lib.moe_abi_version() == 2


def _desc(**kw):
    fake = 1 << 20  # aligned non-NULL host-side stand-ins: validation never dereferences
    bank = lambda n, fmt=4: binding.MoeBank(fmt, 128, n, 0, fake, fake, fake, fake, fake, fake)
    d = binding.MoeLayer(16, 2560, 1024, 512, 10, 0, fake, None, bank(512), bank(1))
    for k, v in kw.items():
        setattr(d, k, v)
    return d


@pytest.mark.parametrize("field,value,code", [
    ("T", 0, -1), ("d", 100, -1), ("f", 130, -1), ("k", 0, -1), ("k", 33, -2),
    ("E", 2048, -2), ("path", 7, -1), ("router_w", None, -1), ("router_w", (1 << 20) + 2, -1),
])
def test_validation_codes(lib, field, value, code):
    d = _desc(**{field: value})
    assert lib.moe_validate(ctypes.byref(d)) == code
    assert lib.moe_workspace_size(ctypes.byref(d)) == 0


def test_validation_banks(lib):
    d = _desc()
    assert lib.moe_validate(ctypes.byref(d)) == 0
    d.routed.group = 64
    assert lib.moe_validate(ctypes.byref(d)) == -1
    d = _desc()
    d.shared.n_exp = 2
    assert lib.moe_validate(ctypes.byref(d)) == -2
    d = _desc()
    d.shared.fmt = 8  # an int8 shared expert beside int4 routed experts
    assert lib.moe_validate(ctypes.byref(d)) == 0
    d.shared.group = 64
    assert lib.moe_validate(ctypes.byref(d)) == -1
    d = _desc()
    d.routed.s_up = None
    assert lib.moe_validate(ctypes.byref(d)) == -1
    d = _desc()
    d.routed.fmt = 16
    d.routed.s_gate = d.routed.s_up = d.routed.s_down = None
    d.shared.fmt = 16
    assert lib.moe_validate(ctypes.byref(d)) == 0


def _nvfp4_desc(**kw):
    fake = 1 << 20
    d = _desc(**kw)
    d.routed = binding.MoeBank(41, 16, 512, 0, fake, fake, fake, fake, fake, fake,
                               fake, fake, fake)
    d.shared.fmt = 16
    d.shared.s_gate = d.shared.s_up = d.shared.s_down = None
    return d


def test_validation_nvfp4_bank(lib):
    d = _nvfp4_desc()
    assert lib.moe_validate(ctypes.byref(d)) == 0
    nv_ws = lib.moe_workspace_size(ctypes.byref(d))
    d.path = binding.PATH_CODE["tc"]
    assert lib.moe_validate(ctypes.byref(d)) == 0
    for path in ("gemv", "fused"):  # the FP4 tensor-core kernels only
        d.path = binding.PATH_CODE[path]
        assert lib.moe_validate(ctypes.byref(d)) == -2
    d = _nvfp4_desc()
    d.routed.group = 128  # NVFP4 blocks are 16 values
    assert lib.moe_validate(ctypes.byref(d)) == -1
    d = _nvfp4_desc()
    d.routed.g_up = None  # tensor scales required
    assert lib.moe_validate(ctypes.byref(d)) == -1
    d = _nvfp4_desc()
    d.routed.s_down = (1 << 20) + 8  # packed scales are read by bulk copies: 16-byte aligned
    assert lib.moe_validate(ctypes.byref(d)) == -1
    d = _nvfp4_desc(d=2560 + 128)  # stages of 256 K values
    assert lib.moe_validate(ctypes.byref(d)) == -2
    d = _nvfp4_desc()
    d.shared = binding.MoeBank(41, 16, 1, 0, *([1 << 20] * 9))  # routed experts only
    assert lib.moe_validate(ctypes.byref(d)) == -2
    # the NVFP4 intermediates (quantised x and h, fp32 h) add to the integer layer's workspace
    assert nv_ws > lib.moe_workspace_size(ctypes.byref(_desc()))


def test_nvfp4_helpers_validate_on_host(lib):
    fake = 1 << 20
    pack = lib.moe_nvfp4_pack_scales
    assert pack(None, fake, 1, 128, 64, None) == -1
    assert pack(fake, fake + (1 << 20), 1, 100, 64, None) == -1   # rows % 128
    assert pack(fake, fake + (1 << 20), 1, 128, 48, None) == -1    # K % 64
    assert pack(fake, fake + 64, 1, 128, 64, None) == -1           # overlapping buffers
    q = lib.moe_nvfp4_quantize_rows
    assert q(fake, 4, 40, fake, fake, fake, None) == -1            # K % 16
    assert q(fake, 0, 64, fake, fake, fake, None) == -1            # rows
    assert q(fake + 8, 4, 64, fake, fake, fake, None) == -1        # alignment


def test_launch_counts_follow_the_automatic_path(lib):
    """Host-side path choice (no GPU needed above one row): up to 32 rows the fused routing
    kernel, the two GEMV kernels and the combine (4 launches); from 33 rows router, top-k, the
    plan, the tensor-core prep, gate/up and down, and the combine; a W8 shared expert beside
    W4 routed experts runs each GEMM once per bank; NVFP4 routed experts add the activation
    quantisers and the shared expert's own GEMMs."""
    for T in (2, 16, 32):
        assert lib.moe_launches_per_call(ctypes.byref(_desc(T=T))) == 4, T
    assert lib.moe_launches_per_call(ctypes.byref(_desc(T=33))) == 7  # 330 assignments: one plan kernel
    assert lib.moe_launches_per_call(ctypes.byref(_desc(T=512))) == 9  # the plan in 3 kernels
    d = _desc(T=16)
    d.shared.fmt = 8
    assert lib.moe_launches_per_call(ctypes.byref(d)) == 6
    d = _desc(T=16)
    d.path = binding.PATH_CODE["tc"]
    assert lib.moe_launches_per_call(ctypes.byref(d)) == 5
    assert lib.moe_launches_per_call(ctypes.byref(_nvfp4_desc(T=16))) == 1 + 5 + 2 + 1


def test_workspace_size_grows_with_T(lib):
    a = lib.moe_workspace_size(ctypes.byref(_desc(T=1)))
    b = lib.moe_workspace_size(ctypes.byref(_desc(T=4096)))
    assert 0 < a < b
    assert a % 256 == 0 and b % 256 == 0


def test_calls_reject_bad_arguments_before_any_cuda_call(lib):
    d = _desc()
    # NULL workspace / NULL x: rejected on the host, nothing enqueued
    assert lib.moe_layer_forward(ctypes.byref(d), 1 << 20, 1 << 20, None, None, None, None,
                                 None, 0, None) == -5
    assert lib.moe_layer_forward(ctypes.byref(d), None, 1 << 20, None, None, None, None,
                                 1 << 20, 1 << 40, None) == -1
    assert lib.moe_route(None, None, None, None, None, 0, None) == -1
    assert lib.moe_status_str(-4) == b"device-side wait timed out"


@pytest.mark.parametrize("path,single", [(2, 5), (1, 4)])
def test_launch_count_of_mixed_bank_formats(lib, path, single):
    """16 tokens: routing (one launch), the grouped products, the combine; a shared bank in
    another format than the routed one runs each of the two GEMMs once per bank."""
    d = _desc(path=path)
    assert lib.moe_launches_per_call(ctypes.byref(d)) == single
    d.shared.fmt = 8
    assert lib.moe_launches_per_call(ctypes.byref(d)) == single + 2


def test_header_is_plain_c(tmp_path):
    """The boundary is a C ABI: the header compiles as C99 (no C++ types in the signatures),
    and the struct layout the binding declares matches the compiler's."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "moe_b200.h"\n'
                   'int main(void) { printf("%zu %zu %zu %zu\\n", sizeof(moe_bank), sizeof(moe_layer),'
                   ' offsetof(moe_layer, routed), offsetof(moe_bank, g_gate)); return 0; }\n')
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    sizes = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                            check=True).stdout.split()]
    assert sizes == [ctypes.sizeof(binding.MoeBank), ctypes.sizeof(binding.MoeLayer),
                     binding.MoeLayer.routed.offset, binding.MoeBank.g_gate.offset]
