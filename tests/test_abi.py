"""The C-ABI library loads and exports every entry point include/ft_moe.h
declares; argument validation works without a GPU."""
import ctypes
import os
import re

import pytest
import torch

import sparse_moe_expert_topk_b200 as ft
from conftest import ROOT


@pytest.fixture(scope="module")
def lib():
    from sparse_moe_expert_topk_b200 import build
    build.build()
    return ft.lib()


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z_0-9]*\s*\*?\s*(ft_[a-z_0-9]+)\s*\(", src, re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert len(declared) >= 14
    assert sorted(ft.EXPORTS) == declared
    for name in declared:
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr), name


def test_slot_bytes(lib):
    for wtype, n in ((ft.FT_W_F32, 98304), (ft.FT_W_BF16, 37748736), (ft.FT_W_NVFP4, 10616832)):
        d, dff = (64, 128) if wtype == ft.FT_W_F32 else (4096, 1536)
        cfg = ft.make_config(1, 8, 2, d, dff, wtype, 4, 16)
        assert ft.ft_moe_slot_bytes(cfg) == n


@pytest.mark.parametrize("field,value", [("n_layers", 0), ("n_experts", 0), ("n_experts", 513), ("top_k", 0),
                                         ("top_k", 9), ("d_model", 100), ("d_ff", 32), ("wtype", 3),
                                         ("cache_slots", -1), ("cache_slots", 17), ("max_tokens", 0),
                                         ("device", -1)])
def test_config_validation(lib, field, value):
    cfg = ft.make_config(1, 8, 2, 64, 128, ft.FT_W_F32, 4, 16)
    setattr(cfg, field, value)
    with pytest.raises(ft.FtError) as ei:
        ft.ft_moe_slot_bytes(cfg)
    assert ei.value.status == ft.FT_EINVAL


def test_status_strings(lib):
    assert ft.status_str(ft.FT_OK) == "ok"
    assert ft.status_str(ft.FT_ETIMEOUT) == "timed out"
    assert ft.status_str(99) == "unknown status"


def test_null_arguments_are_rejected(lib):
    P = ctypes.c_void_p
    assert lib.ft_moe_set_router(None, 0, P(1)) == ft.FT_EINVAL
    assert lib.ft_set_bandwidths(None, 1, 1) == ft.FT_EINVAL
    assert lib.ft_cache_stats(None, None) == ft.FT_EINVAL
    assert lib.ft_moe_layer_forward(None, 0, 0, None, 0, None, 0, None, None, None) == ft.FT_EINVAL
    assert lib.ft_moe_layer_forward_host(None, 0, 0, None, 0, None, 0, None) == ft.FT_EINVAL
    assert lib.ft_moe_expert_rows(None, 0, 0, None, None, 0, 0, None) == ft.FT_EINVAL
    lib.ft_moe_destroy(None)


def test_ep_argument_checks_without_a_gpu(lib):
    """The expert-parallel entry points reject bad sizes before touching the
    device; the pack's scratch covers its arrays."""
    u = ctypes.c_uint64()
    for T, k, E in [(0, 6, 256), (1, 6, 256), (4096, 6, 256), (5, 1, 8)]:
        assert lib.ft_ep_pack_scratch_bytes(T, k, E, ctypes.byref(u)) == ft.FT_OK
        n = T * k
        chunks = -(-n // 1024) * E
        assert u.value >= 4 * (n + E + (E + 1) + n + chunks) and u.value % 256 == 0
    small = ft.ft_ep_pack_scratch_bytes(1, 6, 256)
    assert ft.ft_ep_pack_scratch_bytes(4096, 6, 256) > small
    for T, k, E in [(-1, 6, 256), (1, 0, 256), (1, 17, 256), (1, 6, 0), (1, 6, 513)]:
        assert lib.ft_ep_pack_scratch_bytes(T, k, E, ctypes.byref(u)) == ft.FT_EINVAL
    assert lib.ft_ep_pack_scratch_bytes(1, 6, 256, None) == ft.FT_EINVAL
    P = ctypes.c_void_p
    pack = lambda T, k, E, G, d, wt, counts: lib.ft_ep_pack(  # noqa: E731
        P(16), T, k, E, G, P(16), d, wt, P(16), P(16), counts, P(16), None, P(256), 1 << 20, None)
    assert pack(1, 6, 256, 3, 64, ft.FT_W_BF16, P(16)) == ft.FT_EINVAL   # 3 does not divide 256
    assert pack(1, 6, 8, 16, 64, ft.FT_W_BF16, P(16)) == ft.FT_EINVAL    # more owners than experts
    assert pack(1, 6, 256, 8, 60, ft.FT_W_BF16, P(16)) == ft.FT_EINVAL   # d not a multiple of 8
    assert pack(1, 6, 256, 8, 64, 7, P(16)) == ft.FT_EINVAL              # no such weight type
    assert pack(1, 6, 256, 8, 64, ft.FT_W_BF16, None) == ft.FT_EINVAL    # counts output missing
    assert pack(1, 0, 256, 8, 64, ft.FT_W_BF16, P(16)) == ft.FT_EINVAL
    comb = lambda T, k, d, wt, y: lib.ft_ep_combine(P(16), P(16), P(16), T, k, d, wt, y, None)  # noqa: E731
    assert comb(0, 6, 64, ft.FT_W_BF16, None) == ft.FT_OK                # no tokens, nothing launched
    assert comb(1, 6, 62, ft.FT_W_BF16, P(32)) == ft.FT_EINVAL
    assert comb(1, 17, 64, ft.FT_W_BF16, P(32)) == ft.FT_EINVAL
    assert comb(1, 6, 64, ft.FT_W_BF16, None) == ft.FT_EINVAL
    assert comb(1, 6, 64, ft.FT_W_BF16, P(16)) == ft.FT_EINVAL           # y aliases the rows


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_init_without_gpu_fails_cleanly(lib):
    cfg = ft.make_config(1, 8, 2, 64, 128, ft.FT_W_F32, 4, 16)
    with pytest.raises(ft.FtError) as ei:
        ft.ft_moe_init(cfg, None, 1)
    assert ei.value.status == ft.FT_ECUDA


def test_header_is_plain_c_and_links(lib, tmp_path):
    """The boundary is a C ABI: a C99 translation unit that includes the header
    and takes the address of every declared entry point compiles with warnings
    as errors and links against the library (no C++ in any signature)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    names = _declared()
    src = tmp_path / "use_abi.c"
    src.write_text('#include "ft_moe.h"\n#include <stdio.h>\n'
                   "typedef void (*fn_t)(void);\n"
                   "int main(void) {\n  const fn_t fns[] = {\n"
                   + "".join(f"    (fn_t)&{n},\n" for n in names)
                   + "  };\n  printf(\"%d %s\\n\", (int)(sizeof fns / sizeof fns[0]), ft_status_str(FT_EINVAL));\n"
                   "  return 0;\n}\n")
    lib_dir = os.path.join(ROOT, "sparse_moe_expert_topk_b200")
    exe = tmp_path / "use_abi"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                        str(src), "-o", str(exe), "-L", lib_dir, "-lft_moe", f"-Wl,-rpath,{lib_dir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    n, msg = out.stdout.strip().split(" ", 1)
    assert int(n) == len(names) and msg == "invalid argument"


def test_struct_layouts_match_the_binding(lib, tmp_path):
    """sizeof and field offsets of ft_config, ft_stats and ft_kernel_time as
    a C compiler lays them out equal the ctypes mirrors of the binding."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    mirrors = {"ft_config": ft.FtConfig, "ft_stats": ft.FtStats, "ft_kernel_time": ft.FtKernelTime}
    lines = []
    for cname, py in mirrors.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            lines.append(f'  printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    src = tmp_path / "layout.c"
    src.write_text('#include "ft_moe.h"\n#include <stdio.h>\n#include <stddef.h>\nint main(void) {\n'
                   + "\n".join(lines) + "\n  return 0;\n}\n")
    exe = tmp_path / "layout"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                        str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l.strip()}
    for cname, py in mirrors.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for f, _ in py._fields_:
            assert got[(cname, f)] == getattr(py, f).offset, (cname, f)
