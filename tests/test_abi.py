"""The C-ABI library loads, exports every entry point include/mx.h declares,
and rejects invalid arguments on the host (no GPU needed: these calls return
before any CUDA call)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mx():
    from microscaling_block_quantization_b200 import build
    build.build()
    import microscaling_block_quantization_b200 as m
    m.lib()
    return m


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(mx_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(mx):
    names = declared_functions()
    assert {"mx_quantize", "mx_dequantize", "mx_hadamard_quantize", "mx_qsnr",
            "mx_gemm_qsnr"} <= set(names)
    L = C.CDLL(mx.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n


def test_version_and_strerror(mx):
    assert "sm_100a" in mx.mx_version()
    assert mx.mx_strerror(0) == "ok"
    assert "aligned" in mx.mx_strerror(-3)


def test_query_sizes_host_only(mx):
    s = mx.query_sizes(mx.MXFP4, 256, 256)
    assert s.codes_bytes == 256 * 128 and s.n_scales == 256 * 8 and s.workspace_bytes > 0
    s = mx.query_sizes(mx.NVFP4, 8192, 4096)
    assert s.n_scales == 8192 * 256
    s = mx.query_sizes(mx.Config(elem=mx.E2M3, axis=mx.AXIS_COL), 64, 96)
    assert s.codes_bytes == 64 * 96 and s.n_scales == 2 * 96
    s = mx.query_sizes(mx.Config(axis=mx.AXIS_2D, macro_block=128), 64, 256)
    assert s.n_scales == 2 * 8 and s.n_macro == 64 * 2
    s = mx.query_sizes(mx.Config(elem=mx.INT4, asymmetric=1, rule=mx.RULE_CEIL), 32, 64)
    assert s.n_offsets == 64


@pytest.mark.parametrize("cfg,rows,cols,rc", [
    (dict(block=24), 64, 96, -2),                         # unsupported block
    (dict(axis=2, block=16), 64, 64, -2),                 # 2D is 32 x 32
    (dict(rule=3), 64, 64, -1),                           # NEAREST needs UE4M3/UE5M3
    (dict(scale_fmt=1, rule=3, asymmetric=1), 64, 64, -2),
    (dict(tensor_scale=1), 64, 64, -1),                   # tensor scale with E8M0
    (dict(macro_block=64), 64, 128, -1),
    (dict(macro_block=128), 64, 96, -1),                  # cols % 128
    (dict(block=32), 64, 48, -1),                         # cols % block
    (dict(block=16), 64, 16, -1),                         # cols % 32 (lanes walk 32-element chunks)
    (dict(rule=2, oas_tau=float("nan")), 64, 64, -1),
    (dict(elem=9), 64, 64, -1),
    (dict(rule=5), 64, 64, -1),
    (dict(rule=4, block=16), 64, 64, -2),                 # MSE rule: blocks of 32 only
    (dict(rule=4, round=2), 64, 64, -2),                  # ... and nearest-even rounding
    (dict(rule=4, axis=1), 64, 64, -2),
])
def test_invalid_configs_rejected_on_host(mx, cfg, rows, cols, rc):
    c = mx.Config(**cfg)
    got = mx.mx_quantize(c, C.c_void_p(4096), 0, rows, cols, C.c_void_p(4096), C.c_void_p(4096),
                         C.c_void_p(4096), C.c_void_p(4096), C.c_void_p(4096), None, None, 0, None)
    assert got == rc


def test_alignment_and_workspace_rejected_on_host(mx):
    c = mx.MXFP4
    P = C.c_void_p
    assert mx.mx_quantize(c, P(4100), 0, 64, 64, P(4096), P(4096), None, None, None, None, None, 0,
                          None) == -3
    # stats requested without a workspace
    assert mx.mx_quantize(c, P(4096), 0, 64, 64, P(4096), P(4096), None, None, None, P(4096), None,
                          0, None) == -5
    # hadamard config on the plain entry point, and the reverse
    assert mx.mx_quantize(mx.Config(hadamard=32), P(4096), 0, 64, 64, P(4096), P(4096), None, None,
                          None, None, None, 0, None) == -1
    assert mx.mx_hadamard_quantize(c, P(4096), 0, 64, 64, P(4096), P(4096), None, None, None, None,
                                   None, None, 0, None) == -1
    # column-axis rotation longer than the block
    assert mx.mx_hadamard_quantize(mx.Config(axis=1, block=8, hadamard=16), P(4096), 0, 64, 64,
                                   P(4096), P(4096), None, None, None, None, None, None, 0,
                                   None) == -2


def test_gemm_operand_pairs_checked_on_host(mx):
    """mx_gemm rejects operand pairs it has no tensor-core kind for, and the
    misaligned packed E2M1 operand of the FP6 x FP4 kind, before any launch."""
    P = C.c_void_p
    def gemm(ca, cb, a=4096, b=4096, M=128, N=256, K=256):
        return mx.mx_gemm(ca, cb, P(a), P(4096), P(b), P(4096), None, None, M, N, K, P(4096), 1, None)
    g = dict(sf_layout=1)
    assert gemm(mx.Config(hadamard=32, **g), mx.Config(**g)) == -2         # rotation on one side only
    assert gemm(mx.Config(hadamard=16, **g), mx.Config(hadamard=32, **g)) == -2
    assert gemm(mx.Config(elem=2, **g), mx.Config(elem=4, **g)) == -2       # FP6 x INT4
    nv = mx.Config(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_NEAREST, tensor_scale=mx.TS_COMPUTE, **g)
    assert gemm(mx.Config(elem=2, **g), nv) == -2                           # FP6 x NVFP4
    assert gemm(mx.Config(elem=2, **g), mx.Config(**g), b=4112) == -3       # packed E2M1 wants 32 bytes
    assert gemm(mx.Config(elem=2, **g), mx.Config(**g), N=128) == -2        # FP6 kinds: N % 256
    assert gemm(mx.Config(**g), mx.Config(**g), K=128) == -1                # K % 256


def test_sharding_entry_points_checked_on_host(mx):
    P = C.c_void_p
    amax_cfg = mx.Config(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_NEAREST, tensor_scale=mx.TS_AMAX)
    # the amax pass wants the amax mode and a workspace
    assert mx.mx_tensor_amax(mx.NVFP4, P(4096), 0, 64, 64, P(4096), 4096, None) == -1
    assert mx.mx_tensor_amax(amax_cfg, P(4096), 0, 64, 64, None, 0, None) == -5
    assert mx.mx_tensor_amax(amax_cfg, P(4100), 0, 64, 64, P(4096), 1 << 20, None) == -3
    # the given-amax mode: a workspace carries the amax; not through the no-alloc entry
    assert mx.mx_quantize(amax_cfg, P(4096), 0, 64, 64, P(4096), P(4096), P(4096), None, None, None,
                          None, 0, None) == -5
    assert mx.mx_quantize_noalloc(amax_cfg, P(4096), 0, 64, 64, P(4096), P(4096), P(4096), None, None,
                                  None, None) == -2
    # rotation is not covered by the no-alloc entry: unsupported, not invalid
    for n in (16, 32):
        assert mx.mx_quantize_noalloc(mx.Config(hadamard=n), P(4096), 0, 64, 64, P(4096), P(4096), None,
                                      None, None, P(4096), None) == -2
    assert mx.mx_quantize(mx.Config(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_NEAREST, tensor_scale=4),
                          P(4096), 0, 64, 64, P(4096), P(4096), P(4096), None, None, None, None, 0, None) == -1
    assert mx.mx_stats_finalize(None, None) == -1
    assert mx.mx_stats_finalize(P(4100), None) == -3


def test_group_checked_on_host(mx):
    """mx_quantize_group checks every item before anything is queued: an
    invalid item fails the whole call with that item's error, and two items
    whose statistics would share one workspace are rejected."""
    P = C.c_void_p
    WS = 1 << 20

    def item(x=4096, rows=64, cols=64, stats=None, ws=None, wsb=0):
        return mx.mx_quantize_item(x, rows, cols, 4096, 4096, 4096, None, None, stats, ws, wsb)

    def call(cfg, *its):
        arr = (mx.mx_quantize_item * max(len(its), 1))(*its)
        return mx.mx_quantize_group(cfg, 0, arr, len(its), None)

    assert mx.lib().mx_quantize_group(None, 0, None, 1, None) == -1
    assert mx.mx_quantize_group(mx.MXFP4, 0, None, 1, None) == -1
    assert call(mx.MXFP4) == -1                                         # no items
    assert call(mx.MXFP4, item(), item(cols=48)) == -1                  # cols % 32
    assert call(mx.MXFP4, item(), item(x=4100)) == -3                   # misaligned input
    assert call(mx.MXFP4, item(), item(stats=4096)) == -5               # statistics without a workspace
    assert call(mx.MXFP4, item(stats=4096, ws=1 << 24, wsb=WS),
                item(stats=8192, ws=(1 << 24) + 4096, wsb=WS)) == -1    # one workspace for two tensors
    assert call(mx.NVFP4, item(ws=1 << 24, wsb=WS), item(ws=1 << 24, wsb=WS)) == -1
    assert call(mx.Config(elem=9), item()) == -1
    assert call(mx.Config(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_NEAREST, tensor_scale=4), item()) == -1


def test_element_limit_checked_on_host(mx):
    """Calls take fewer than 2^32 elements (32-bit indices in the kernels)."""
    P = C.c_void_p
    s = mx.mx_sizes()
    assert mx.lib().mx_query_sizes(C.byref(mx.MXFP4.c()), 1 << 16, (1 << 16) - 32, C.byref(s)) == 0
    assert mx.lib().mx_query_sizes(C.byref(mx.MXFP4.c()), 1 << 16, 1 << 16, C.byref(s)) == -1
    assert mx.mx_quantize(mx.MXFP4, P(4096), 0, 1 << 17, 1 << 15, P(4096), P(4096), None, None, None, None,
                          None, 0, None) == -1
    ws = 1 << 20
    assert mx.mx_qsnr(P(4096), 0, P(4096), 0, 1 << 17, 1 << 15, 0, 0, P(4096), None, P(4096), ws, None) == -1


def test_header_is_plain_c_and_links(tmp_path):
    """include/mx.h compiles as strict C11 (no C++ in the boundary), and a C
    program calling every declared entry point links against the library."""
    import re
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no gcc")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    hdr = open(os.path.join(root, "include", "mx.h")).read()
    names = sorted(set(re.findall(r"^\s*(?:int|int64_t|const char \*)\s*\**(mx_\w+)\(", hdr, re.M)))
    assert "mx_quantize" in names and "mx_gemm_qsnr" in names
    src = tmp_path / "use.c"
    src.write_text('#include "mx.h"\n#include <stdio.h>\ntypedef void (*fn)(void);\n'
                   + "static const fn all[] = {" + ", ".join(f"(fn){n}" for n in names) + "};\n"
                   + "int main(void) {\n    unsigned i, k = 0;\n"
                   + "    for (i = 0; i < sizeof all / sizeof all[0]; ++i) k += all[i] != 0;\n"
                   + '    printf("%u\\n", k);\n    return 0;\n}\n')
    lib = os.path.dirname(mx_lib_path())
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(root, "include"),
           "-I", "/usr/local/cuda/include", str(src), "-o", str(tmp_path / "use"), "-L", lib, "-lmx_b200",
           "-Wl,--unresolved-symbols=ignore-in-shared-libs"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def mx_lib_path():
    import microscaling_block_quantization_b200 as m
    return m.LIB_PATH


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    import microscaling_block_quantization_b200 as m
    monkeypatch.setattr(m, "_lib", None)
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError):
        m.lib()


def test_group_binding_checks_on_host(mx):
    """The grouped binding rejects CPU tensors and mixed dtypes before any
    library call, and an empty group is an empty result."""
    import torch
    assert mx.quantize_group([], mx.MXFP4) == []
    with pytest.raises(ValueError):
        mx.quantize_group([torch.zeros(32, 64, dtype=torch.bfloat16)], mx.MXFP4)
    with pytest.raises(ValueError):
        mx.quantize_group([torch.zeros(2, 32, 64, dtype=torch.bfloat16)], mx.MXFP4)
