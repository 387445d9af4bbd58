"""The C ABI without a GPU: every symbol the header declares is exported, the
host-side argument checks return the documented codes, and no call that is
checked here launches a kernel."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "oft.h")


@pytest.fixture(scope="module")
def lib():
    from orthogonal_fine_tuning_b200 import _lib
    return _lib.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_]\w*\s*\*?\s+\*?([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_path(lib):
    names = _declared()
    for required in ("oft_build_rotation", "oft_linear_fwd", "oft_linear_bwd", "moe_chunked_oft_fwd"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    from orthogonal_fine_tuning_b200 import _lib
    names = _declared()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(_lib.EXPORTS)


def test_version(lib):
    assert b"sm_100a" in lib.oft_version()


def _w(lib, fmt=1, codes=0x1000, scales=0x2000, d_in=256, d_out=384, group=32, n=0):
    from orthogonal_fine_tuning_b200 import _lib
    return _lib.CWeight(fmt, codes, scales, d_in, d_out, group, n)


def _s(sizes):
    from orthogonal_fine_tuning_b200 import _lib
    s = _lib.CSplit()
    s.n = len(sizes)
    for i, v in enumerate(sizes):
        s.sizes[i] = v
    return s


def _fwd(lib, w, s, b=32, X=0x3000, R=0x4000, Y=0x5000, ws=0x6000, nbytes=1 << 40, M=64):
    return lib.oft_linear_fwd(X, M, ctypes.byref(w), ctypes.byref(s), b, R, Y, ws, nbytes, None)


def test_argument_checks(lib):
    from orthogonal_fine_tuning_b200 import _lib as L
    s = _s([128, 128, 128])
    assert _fwd(lib, _w(lib, codes=0), s) == L.OFT_ERR_INVALID_ARG                  # NULL codes
    assert _fwd(lib, _w(lib, codes=0x1001), s) == L.OFT_ERR_INVALID_ARG             # misaligned
    assert _fwd(lib, _w(lib), s, b=48) == L.OFT_ERR_UNSUPPORTED                     # b not supported
    assert _fwd(lib, _w(lib, d_in=160), s, b=64) == L.OFT_ERR_UNSUPPORTED                # K % b
    assert _fwd(lib, _w(lib, group=48), s) == L.OFT_ERR_UNSUPPORTED                 # INT4 group
    assert _fwd(lib, _w(lib, fmt=9), s) == L.OFT_ERR_UNSUPPORTED                    # format
    assert _fwd(lib, _w(lib, d_in=250), s) == L.OFT_ERR_UNSUPPORTED                 # K % 32
    assert _fwd(lib, _w(lib), _s([128, 128, 120])) == L.OFT_ERR_INVALID_ARG         # sizes != d_out
    assert _fwd(lib, _w(lib), _s([128, 128, 124, 4])) == L.OFT_ERR_UNSUPPORTED      # size % 8
    s5 = _s([128] * 4)
    s5.n = 5
    assert _fwd(lib, _w(lib, d_out=640), s5) == L.OFT_ERR_UNSUPPORTED               # > 4 splits
    assert _fwd(lib, _w(lib), s, X=0) == L.OFT_ERR_INVALID_ARG                      # NULL X
    assert _fwd(lib, _w(lib), s, Y=0x5008) == L.OFT_ERR_INVALID_ARG                 # misaligned Y
    assert _fwd(lib, _w(lib), s, nbytes=16) == L.OFT_ERR_WORKSPACE                  # workspace too small
    assert _fwd(lib, _w(lib), s, M=-1) == L.OFT_ERR_INVALID_ARG
    assert _fwd(lib, _w(lib), s, M=0) == L.OFT_OK                                   # nothing to do
    assert lib.oft_last_error() != b""


def test_workspace_sizes(lib):
    w, s = _w(lib, d_in=2560, d_out=6144, group=0, fmt=2), _s([4096, 1024, 1024])
    fwd = lib.oft_linear_fwd_workspace(4096, ctypes.byref(w), ctypes.byref(s), 32)
    # 4096 tokens: rotated activations for 3 sub-projections + the bf16 weight copy of the plain GEMM
    assert 2 * 3 * 4096 * 2560 + 2 * 6144 * 2560 <= fwd < 2 * 3 * 4096 * 2560 + 2 * 6144 * 2560 + 4096
    bwd = lib.oft_linear_bwd_workspace(4096, ctypes.byref(w), ctypes.byref(s), 32)
    # fp32 dX' for 3 sub-projections + the transposed bf16 weight copy + dR partials
    assert bwd >= 4 * 3 * 4096 * 2560 + 2 * 6144 * 2560
    # 1024 tokens: the fused-decode kernels, so no bf16 weight copy; packed FP8 codes in the backward
    fwd1 = lib.oft_linear_fwd_workspace(1024, ctypes.byref(w), ctypes.byref(s), 32)
    assert 2 * 3 * 1024 * 2560 <= fwd1 < 2 * 3 * 1024 * 2560 + 4096
    bwd1 = lib.oft_linear_bwd_workspace(1024, ctypes.byref(w), ctypes.byref(s), 32)
    assert 4 * 3 * 1024 * 2560 + 6144 * 2560 <= bwd1 < 4 * 3 * 1024 * 2560 + 2 * 6144 * 2560
    assert lib.oft_linear_fwd_workspace(0, ctypes.byref(w), ctypes.byref(s), 32) == 0


def test_moe_argument_checks(lib):
    from orthogonal_fine_tuning_b200 import _lib as L
    w = _w(lib, d_in=256, d_out=64, group=32, n=16)
    p = [0x10000 * (i + 1) for i in range(11)]

    def call(E=16, top_k=4, chunk=4, b=32, w=w):
        args = [p[0], 32, p[1], E, top_k, chunk, ctypes.byref(w), b, p[2], p[3], p[4], p[5], p[6], p[7], p[8],
                p[9], p[10], 1 << 40, None]
        return lib.moe_chunked_oft_fwd(*args)

    assert call(E=600, w=_w(lib, d_in=256, d_out=64, n=600)) == L.OFT_ERR_UNSUPPORTED
    assert call(top_k=9) == L.OFT_ERR_UNSUPPORTED
    assert call(chunk=17) == L.OFT_ERR_UNSUPPORTED
    assert call(E=8) == L.OFT_ERR_UNSUPPORTED                       # bank size mismatch
    assert call(w=_w(lib, fmt=2, d_in=256, d_out=64, n=16)) == L.OFT_ERR_UNSUPPORTED


def test_chunk_dequant_hook_checks(lib):
    """oft_moe_chunk_dequant rejects bad arguments on the host, before any launch."""
    from orthogonal_fine_tuning_b200 import _lib as L
    w = _w(lib, d_in=256, d_out=64, group=32, n=16)
    assert lib.oft_moe_chunk_dequant(ctypes.byref(w), 0, 0, 4, 0, 0x20000, None) == L.OFT_ERR_INVALID_ARG
    assert lib.oft_moe_chunk_dequant(ctypes.byref(w), 0x10000, 0, 4, 0, 0x20008, None) == L.OFT_ERR_INVALID_ARG
    assert lib.oft_moe_chunk_dequant(ctypes.byref(w), 0x10000, -1, 4, 0, 0x20000, None) == L.OFT_ERR_INVALID_ARG
    assert lib.oft_moe_chunk_dequant(ctypes.byref(w), 0x10000, 0, 17, 0, 0x20000, None) == L.OFT_ERR_UNSUPPORTED
    fp8 = _w(lib, fmt=2, d_in=256, d_out=64, n=16)
    assert lib.oft_moe_chunk_dequant(ctypes.byref(fp8), 0x10000, 0, 4, 0, 0x20000, None) == L.OFT_ERR_UNSUPPORTED
    odd = _w(lib, d_in=256, d_out=40, group=32, n=16)
    assert lib.oft_moe_chunk_dequant(ctypes.byref(odd), 0x10000, 0, 4, 1, 0x20000, None) == L.OFT_ERR_UNSUPPORTED


def test_rotation_and_debug_checks(lib):
    from orthogonal_fine_tuning_b200 import _lib as L
    assert lib.oft_build_rotation(0x1000, 4, 24, 0x2000, None) == L.OFT_ERR_UNSUPPORTED
    assert lib.oft_build_rotation(0, 4, 32, 0x2000, None) == L.OFT_ERR_INVALID_ARG
    assert lib.oft_build_rotation(0x1000, 0, 32, 0x2000, None) == L.OFT_OK
    assert lib.oft_debug_bounded_wait(0, None) == L.OFT_ERR_INVALID_ARG


def test_moe_backward_and_layer_argument_checks(lib):
    """Each call below fails a host-side check before any launch."""
    from orthogonal_fine_tuning_b200 import _lib as L
    w = _w(lib, d_in=256, d_out=64, group=32, n=16)
    p = [0x10000 * (i + 1) for i in range(12)]

    def bwd(E=16, top_k=4, chunk=4, b=32, w=w, dY=p[0], ws_bytes=1 << 40, dlogits=p[6]):
        return lib.moe_chunked_oft_bwd(dY, p[1], 32, p[2], E, top_k, chunk, ctypes.byref(w), b, p[3], p[4], p[5],
                                       dlogits, p[7], ws_bytes, None)

    assert bwd(E=600, w=_w(lib, d_in=256, d_out=64, n=600)) == L.OFT_ERR_UNSUPPORTED
    assert bwd(top_k=9) == L.OFT_ERR_UNSUPPORTED
    assert bwd(chunk=17) == L.OFT_ERR_UNSUPPORTED
    assert bwd(E=8) == L.OFT_ERR_UNSUPPORTED                        # bank size mismatch
    assert bwd(w=_w(lib, fmt=2, d_in=256, d_out=64, n=16)) == L.OFT_ERR_UNSUPPORTED
    assert bwd(b=24) == L.OFT_ERR_UNSUPPORTED
    assert bwd(dY=0) == L.OFT_ERR_INVALID_ARG
    assert bwd(dlogits=p[6] + 4) == L.OFT_ERR_INVALID_ARG           # misaligned
    assert bwd(ws_bytes=1024) == L.OFT_ERR_WORKSPACE
    need = lib.moe_chunked_oft_bwd_workspace(32, 16, 4, 4, ctypes.byref(w), 32)
    assert need > 2 * 4 * 32 * 4 * 256                              # D = dY W^T alone is 2 x T*k x K fp32

    wd = _w(lib, d_in=32, d_out=256, group=32, n=16)                # n_proj = 32 -> K = 256

    def layer(w=w, wd=wd, b=32, X=p[0], ws_bytes=1 << 40):
        return lib.moe_chunked_oft_layer_fwd(X, 32, p[1], 16, 4, 4, ctypes.byref(w), ctypes.byref(wd), b, p[2],
                                             p[3], p[4], p[5], ws_bytes, None)

    assert layer(wd=_w(lib, d_in=64, d_out=256, group=32, n=16)) == L.OFT_ERR_INVALID_ARG   # d_in != n_proj
    assert layer(wd=_w(lib, d_in=32, d_out=128, group=32, n=16)) == L.OFT_ERR_INVALID_ARG   # d_out != K
    assert layer(wd=_w(lib, d_in=32, d_out=256, group=32, n=8)) == L.OFT_ERR_INVALID_ARG    # experts differ
    assert layer(wd=_w(lib, fmt=2, d_in=32, d_out=256, group=0, n=16)) == L.OFT_ERR_UNSUPPORTED
    assert layer(X=0) == L.OFT_ERR_INVALID_ARG
    assert layer(ws_bytes=1024) == L.OFT_ERR_WORKSPACE
    lneed = lib.moe_chunked_oft_layer_workspace(32, 16, 4, 4, ctypes.byref(w), ctypes.byref(wd), 32)
    assert lneed > lib.moe_chunked_oft_workspace(32, 16, 4, 4, ctypes.byref(w), 32)


def _schedule(lib, groups, grid, rows=128):
    ng = len(groups)
    arr = ctypes.c_int * ng
    m, n, k = (arr(*[g[i] for g in groups]) for i in range(3))
    total = sum(-(-g[0] // rows) * -(-g[1] // 256) for g in groups)
    used = ctypes.c_int(-1)
    off = (ctypes.c_int * (grid + 1))()
    tiles = (ctypes.c_int * max(total, 1))()
    rc = lib.oft_gemm_schedule(ng, m, n, k, rows, grid, ctypes.byref(used), off, tiles)
    depth = []
    for g in groups:
        depth += [-(-g[2] // 64)] * (-(-g[0] // rows) * -(-g[1] // 256))
    return rc, used.value, list(off), list(tiles)[:off[grid]] if used.value == 1 else [], depth


def test_gemm_schedule_balances_unequal_depths(lib):
    # dX' of the fused-QKV workload: 320 tiles 64 k-steps deep (Q), 2 x 320 tiles 16 deep
    rc, used, off, tiles, depth = _schedule(lib, [(4096, 2560, 4096), (4096, 2560, 1024), (4096, 2560, 1024)], 148)
    assert rc == 0 and used == 1
    assert sorted(tiles) == list(range(960))
    assert off[0] == 0 and all(a <= b for a, b in zip(off, off[1:]))
    loads = [sum(depth[t] for t in tiles[off[c]:off[c + 1]]) for c in range(148)]
    round_robin = max(sum(depth[t] for t in range(c, 960, 148)) for c in range(148))
    # two deep tiles per CTA, 24 CTAs take a third; shallow ones fill the rest up to 208
    assert max(loads) == 208 and round_robin == 256
    for c in range(148):  # deepest first within a CTA
        d = [depth[t] for t in tiles[off[c]:off[c + 1]]]
        assert d == sorted(d, reverse=True)


def test_gemm_schedule_pairs(lib):
    # the same dX' on 74 CTA pairs with 256 x 256 tiles: 160 tiles 64 deep, 320 tiles 16 deep
    rc, used, off, tiles, depth = _schedule(lib, [(4096, 2560, 4096), (4096, 2560, 1024), (4096, 2560, 1024)], 74,
                                            rows=256)
    assert rc == 0 and used == 1 and sorted(tiles) == list(range(480))
    loads = [sum(depth[t] for t in tiles[off[c]:off[c + 1]]) for c in range(74)]
    assert max(loads) == 208 and sum(loads) == 160 * 64 + 320 * 16


def test_gemm_schedule_ragged_groups(lib):
    groups = [(300, 352, 264), (300, 352, 8), (300, 352, 136)]  # 6 tiles each, depths 5, 1, 3
    rc, used, off, tiles, depth = _schedule(lib, groups, 18)
    assert rc == 0 and used == 1 and sorted(tiles) == list(range(18))
    loads = [sum(depth[t] for t in tiles[off[c]:off[c + 1]]) for c in range(18)]
    assert max(loads) == 5  # one tile per CTA


def test_gemm_schedule_falls_back_to_round_robin(lib):
    assert _schedule(lib, [(4096, 4096, 2560), (4096, 1024, 2560)], 148)[:2] == (0, 0)  # equal depths
    assert _schedule(lib, [(16384, 7168, 9216), (16384, 7168, 4096)], 148)[:2] == (0, 0)  # 7168 tiles
    assert _schedule(lib, [(4096, 2560, 4096), (4096, 2560, 1024)], 161)[:2] == (0, 0)  # too many CTAs
    used = ctypes.c_int()
    one = (ctypes.c_int * 1)(1)
    assert lib.oft_gemm_schedule(0, one, one, one, 128, 4, ctypes.byref(used), one, one) == 1
    assert lib.oft_gemm_schedule(1, one, one, one, 128, 0, ctypes.byref(used), one, one) == 1
    assert lib.oft_gemm_schedule(1, one, one, one, 64, 4, ctypes.byref(used), one, one) == 1
    assert lib.oft_gemm_schedule(1, None, one, one, 256, 4, ctypes.byref(used), one, one) == 1


def test_gemm_mode_range(lib):
    for mode in range(5):
        assert lib.oft_set_gemm_mode(mode) == 0
    assert lib.oft_set_gemm_mode(5) == 1 and lib.oft_set_gemm_mode(-1) == 1
    assert lib.oft_set_gemm_mode(0) == 0
