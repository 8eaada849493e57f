"""The C-ABI library loads and exports every function include/gs.h declares,
and its host-only calls (sizes, carving, error strings) behave as documented.
No compute call is made: these run without a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gs.h")


@pytest.fixture(scope="module")
def lib():
    from gaussian_splatting_differentiable_tile_b200 import build as B
    B.build()
    from gaussian_splatting_differentiable_tile_b200 import _abi
    return _abi.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gs_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 14
    for name in names:
        assert hasattr(lib, name), name


def test_binding_declares_exactly_the_header(lib):
    from gaussian_splatting_differentiable_tile_b200 import _abi
    assert sorted(_abi.PROTOTYPES) == _declared()


def test_struct_sizes_match_header_layout():
    from gaussian_splatting_differentiable_tile_b200 import _abi
    assert ctypes.sizeof(_abi.GsCamera) == 4 * (16 + 4 + 2 + 1 + 3 + 1)
    assert ctypes.sizeof(_abi.GsProjected) == 5 * 8
    assert ctypes.sizeof(_abi.GsBins) == 5 * 8 + 8 + 8 + 4 + 4 + 8 + 8


def test_error_strings(lib):
    from gaussian_splatting_differentiable_tile_b200 import _abi
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        s = lib.gs_error_string(code).decode()
        assert s and s != "unknown error code"
    assert lib.gs_error_string(-99).decode() == "unknown error code"
    assert lib.gs_version() == 1
    assert _abi.GS_ERR_CAPACITY == -2


def test_projected_carve_is_host_arithmetic(lib):
    from gaussian_splatting_differentiable_tile_b200 import _abi
    n = 1001
    nbytes = lib.gs_projected_bytes(n)
    assert nbytes >= n * (16 * 4 + 4)
    s = _abi.GsProjected()
    base = 1 << 40  # never dereferenced
    assert lib.gs_projected_carve(ctypes.c_void_p(base), n, ctypes.byref(s)) == 0
    ptrs = [s.xy_opacity_depth, s.conic_radius, s.rgb, s.rect, s.count]
    assert ptrs == sorted(ptrs) and ptrs[0] == base
    assert all(p % 256 == 0 for p in ptrs)
    assert ptrs[1] - ptrs[0] >= 16 * n and base + nbytes >= ptrs[4] + 4 * n
    assert lib.gs_projected_carve(ctypes.c_void_p(base + 16), n, ctypes.byref(s)) == _abi.GS_ERR_ALIGNMENT
    assert lib.gs_projected_carve(ctypes.c_void_p(base), 1 << 30, ctypes.byref(s)) == _abi.GS_ERR_TOO_LARGE


def test_bins_carve_is_host_arithmetic(lib):
    from gaussian_splatting_differentiable_tile_b200 import _abi
    n, mp, W, H = 400_000, 3_000_000, 980, 545
    nbytes = lib.gs_bins_bytes(n, mp, W, H)
    b = _abi.GsBins()
    base = 1 << 40
    assert lib.gs_bins_carve(ctypes.c_void_p(base), n, mp, W, H, ctypes.byref(b)) == 0
    assert b.max_tiles == 62 * 35 and b.max_pairs == mp and b.max_n == n
    assert b.scratch == base and b.scratch_bytes == nbytes
    for p, size in ((b.pair_tile, 4 * mp), (b.pair_gid, 4 * mp), (b.ranges, 8 * b.max_tiles)):
        assert base <= p and p + size <= base + nbytes
    assert lib.gs_bins_carve(ctypes.c_void_p(base), n, 1 << 30, W, H, ctypes.byref(b)) == _abi.GS_ERR_TOO_LARGE
    assert lib.gs_bins_carve(ctypes.c_void_p(base), n, mp, 0, H, ctypes.byref(b)) == _abi.GS_ERR_INVALID_ARG
    assert lib.gs_bins_bytes(-1, mp, W, H) == 0


def test_binding_fails_loudly_without_library(tmp_path):
    from gaussian_splatting_differentiable_tile_b200 import _abi
    with pytest.raises(ImportError):
        _abi._LIB, saved = None, _abi._LIB
        try:
            _abi.load(str(tmp_path / "missing.so"))
        finally:
            _abi._LIB = saved


def test_ctypes_layouts_match_the_c_compiler(tmp_path):
    """Every struct of include/gs.h, as the C compiler lays it out (size and
    the offset of every field), equals the binding's ctypes declaration."""
    import shutil
    import subprocess
    from gaussian_splatting_differentiable_tile_b200 import _abi
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = {"gs_camera": _abi.GsCamera, "gs_params": _abi.GsParams, "gs_grads": _abi.GsGrads,
               "gs_projected": _abi.GsProjected, "gs_bins": _abi.GsBins, "gs_profile_stat": _abi.GsProfileStat,
               "gs_adam_config": _abi.GsAdamConfig, "gs_train_lane": _abi.GsTrainLane}
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "gs.h"', "int main(void) {"]
    for cname, cls in structs.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in cls._fields_:
            lines.append(f'printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {tuple(line.split()[:2]): int(line.split()[2]) for line in out if line.strip()}
    for cname, cls in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(cls), cname
        for field, _ in cls._fields_:
            assert got[(cname, field)] == getattr(cls, field).offset, (cname, field)


def test_sort_bytes_is_the_bins_layout_for_any_n(lib):
    """gs_sort_bytes (the size query under its plain name) equals gs_bins_bytes
    for the same pairs and tile grid, whatever N."""
    W, H = 1960, 1090
    tiles = ((W + 15) // 16) * ((H + 15) // 16)
    for n, mp in ((0, 0), (1000, 5000), (400_000, 21_000_000)):
        assert lib.gs_sort_bytes(mp, tiles) == lib.gs_bins_bytes(n, mp, W, H)
    assert lib.gs_sort_bytes(-1, tiles) == 0 and lib.gs_sort_bytes(10, 0) == 0


def test_static_binding_refuses_short_arrays_before_any_launch():
    """gs_bin_and_sort_static cannot see the sizes of its output arrays, so the
    binding refuses a pair_gid shorter than pair_tile, or ranges with fewer
    than two entries per tile, before anything reaches the library."""
    import torch

    import gaussian_splatting_differentiable_tile_b200 as G
    from scenes import tiny_camera

    cam = tiny_camera(100, 40)  # 7 x 3 tiles
    pt = torch.empty(64, dtype=torch.int32)
    with pytest.raises(ValueError, match="pair_gid"):
        G.gs_bin_and_sort_static(cam, 8, None, pt, torch.empty(63, dtype=torch.int32),
                                 torch.empty(21, 2, dtype=torch.int32))
    with pytest.raises(ValueError, match="ranges"):
        G.gs_bin_and_sort_static(cam, 8, None, pt, pt.clone(), torch.empty(20, 2, dtype=torch.int32))
