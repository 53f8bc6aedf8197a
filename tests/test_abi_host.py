"""Host-only checks of the C ABI (no GPU needed): the library loads, exports every symbol that
include/*.h declares, and its host-side layout and argument checks behave as documented."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def native():
    from adaptive_sparse_attention_b200 import build, _native
    build.build()
    return _native


def declared_functions():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if not f.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"\b(entmax_attn_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(native):
    lib = native.lib()
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    # and every binding signature names a declared function
    assert set(native.SIGNATURES) == set(names)


def test_strerror(native):
    lib = native.lib()
    for code in range(6):
        assert lib.entmax_attn_strerror(code)
    assert b"unknown" in lib.entmax_attn_strerror(99)


@pytest.mark.parametrize("B,Hq,T,packed", [(1, 2, 256, 0), (2, 32, 16384, 0), (1, 3, 1, 0),
                                           (4, 32, 32192, 1), (1, 8, 129, 0), (3, 1, 10, 1),
                                           (1, 32, 131072, 0)])
def test_mask_layout_matches_documentation(native, B, Hq, T, packed):
    from adaptive_sparse_attention_b200 import api
    nt = -(-T // 128)
    slots = T // 128 + B if packed else nt
    W = -(-nt // 32)
    assert api.mask_layout(B, Hq, T, bool(packed)) == (slots, W)
    assert api.mask_words(B, Hq, T, bool(packed)) == (1 if packed else B) * Hq * slots * W
    ws = api.workspace_bytes(B, Hq, T, bool(packed))
    tiles = (1 if packed else B) * Hq * slots
    assert ws >= 4 * tiles * (2 + nt)


def test_packed_slots_never_overlap():
    """The slot base floor(cu[s] / 128) + s leaves room for every query tile of sequence s."""
    from adaptive_sparse_attention_b200.api import tile_slot_table
    rng = np.random.default_rng(0)
    for _ in range(200):
        lens = rng.integers(0, 700, size=rng.integers(1, 9))
        cu = np.concatenate([[0], np.cumsum(lens)])
        T = int(cu[-1])
        if T == 0:
            continue
        tab = tile_slot_table(len(lens), T, cu)
        used = set()
        for slot0, nqt, start, length in tab:
            for i in range(nqt):
                assert slot0 + i not in used
                assert slot0 + i < T // 128 + len(lens)
                used.add(slot0 + i)


def test_decode_block_mask_bit_order():
    from adaptive_sparse_attention_b200.api import decode_block_mask
    B, Hq, T = 1, 1, 128 * 40  # 40 key tiles -> 2 words per query tile
    words = np.zeros((40, 2), dtype=np.uint32)
    words[3, 0] = 1 | (1 << 31)
    words[39, 1] = 1 << 7  # key tile 39
    bits = decode_block_mask(words.view(np.int32), B, Hq, T)
    assert bits.shape == (1, 1, 40, 40)
    assert list(np.nonzero(bits[0, 0, 3])[0]) == [0, 31]
    assert list(np.nonzero(bits[0, 0, 39])[0]) == [39]


def _fake(addr):
    return ctypes.c_void_p(addr)


@pytest.mark.parametrize("case", ["d96", "hq_not_multiple", "alpha1", "alpha_nan", "niter0",
                                  "dtype", "null_q", "causal2", "too_long"])
def test_argument_errors_are_reported_before_any_launch(native, case):
    lib = native.lib()
    args = dict(B=1, Hq=4, Hkv=2, T=256, d=64, alpha=1.5, n_iter=10, causal=1, dtype=1, q=0x1000)
    if case == "d96":
        args["d"] = 96
    elif case == "hq_not_multiple":
        args["Hq"] = 3
    elif case == "alpha1":
        args["alpha"] = 1.0
    elif case == "alpha_nan":
        args["alpha"] = float("nan")
    elif case == "niter0":
        args["n_iter"] = 0
    elif case == "dtype":
        args["dtype"] = 7
    elif case == "null_q":
        args["q"] = 0
    elif case == "causal2":
        args["causal"] = 2
    elif case == "too_long":
        args["T"] = 128 * 32 * 64 + 1  # more key tiles than the kernels' mask words
    a = args
    rc = lib.entmax_attn_tau_pass(_fake(a["q"]) if a["q"] else None, _fake(0x2000),
                                  _fake(0x3000), _fake(0x4000), _fake(0x10000), 1 << 40,
                                  a["B"], a["Hq"], a["Hkv"], a["T"], a["d"], a["alpha"],
                                  a["n_iter"], a["causal"], None, a["dtype"], 0, None)
    assert rc == native.EINVAL
    rc = lib.entmax_attn_fwd(_fake(a["q"]) if a["q"] else None, _fake(0x2000), _fake(0x3000),
                             _fake(0x5000), _fake(0x6000), _fake(0x7000), a["B"], a["Hq"],
                             a["Hkv"], a["T"], a["d"], a["alpha"], a["n_iter"], a["causal"],
                             None, a["dtype"], None)
    assert rc == native.EINVAL
    rc = lib.entmax_attn_fwd_no_block_mask(_fake(a["q"]) if a["q"] else None, _fake(0x2000),
                                           _fake(0x3000), _fake(0x5000), _fake(0x6000), a["B"],
                                           a["Hq"], a["Hkv"], a["T"], a["d"], a["alpha"],
                                           a["n_iter"], a["causal"], None, a["dtype"], None)
    assert rc == native.EINVAL


def test_block_mask_is_required_unless_the_variant_says_otherwise(native):
    """A NULL block_mask is an argument error of the masked passes; with
    ENTMAX_ATTN_FLAG_NO_BLOCK_MASK the same call passes the argument checks (it then needs a
    device, so only the misaligned workspace below is seen)."""
    lib = native.lib()
    rc = lib.entmax_attn_tau_pass(_fake(0x1000), _fake(0x2000), _fake(0x3000), None,
                                  _fake(0x10000), 1 << 40, 1, 2, 2, 256, 64, 1.5, 10, 1, None, 1,
                                  0, None)
    assert rc == native.EINVAL
    rc = lib.entmax_attn_fwd(_fake(0x1000), _fake(0x2000), _fake(0x3000), _fake(0x5000),
                             _fake(0x6000), None, 1, 2, 2, 256, 64, 1.5, 10, 1, None, 1, None)
    assert rc == native.EINVAL
    rc = lib.entmax_attn_tau_pass(_fake(0x1000), _fake(0x2000), _fake(0x3000), None,
                                  _fake(0x10010), 1 << 40, 1, 2, 2, 256, 64, 1.5, 10, 1, None, 1,
                                  native.FLAG_NO_BLOCK_MASK, None)
    assert rc == native.EALIGN


@pytest.mark.parametrize("case", ["rows0", "n0", "ldx_small", "ldp_small", "alpha1", "niter0",
                                  "dtype", "null_x", "misaligned"])
def test_rows_argument_errors(native, case):
    lib = native.lib()
    a = dict(x=0x1000, p=0x2000, tau=0x3000, rows=4, n=8, ldx=8, ldp=8, alpha=1.5, n_iter=10,
             dtype=0)
    want = native.EINVAL
    if case == "rows0":
        a["rows"] = 0
    elif case == "n0":
        a["n"] = 0
    elif case == "ldx_small":
        a["ldx"] = 7
    elif case == "ldp_small":
        a["ldp"] = 7
    elif case == "alpha1":
        a["alpha"] = 1.0
    elif case == "niter0":
        a["n_iter"] = 0
    elif case == "dtype":
        a["dtype"] = 5
    elif case == "null_x":
        a["x"] = 0
    elif case == "misaligned":
        a["p"] = 0x2002
        want = native.EALIGN
    rc = lib.entmax_attn_rows(_fake(a["x"]) if a["x"] else None, a["ldx"], _fake(a["p"]), a["ldp"],
                              _fake(a["tau"]), a["rows"], a["n"], a["alpha"], a["n_iter"],
                              a["dtype"], None)
    assert rc == want


def test_misaligned_pointers_are_rejected(native):
    lib = native.lib()
    rc = lib.entmax_attn_tau_pass(_fake(0x1008), _fake(0x2000), _fake(0x3000), _fake(0x4000),
                                  _fake(0x10000), 1 << 40, 1, 2, 2, 256, 64, 1.5, 10, 1, None, 1,
                                  0, None)
    assert rc == native.EALIGN
    rc = lib.entmax_attn_tau_pass(_fake(0x1000), _fake(0x2000), _fake(0x3000), _fake(0x4000),
                                  _fake(0x10010), 1 << 40, 1, 2, 2, 256, 64, 1.5, 10, 1, None, 1,
                                  0, None)
    assert rc == native.EALIGN  # workspace must be 256-byte aligned


def test_small_workspace_is_rejected(native):
    lib = native.lib()
    need = lib.entmax_attn_workspace_min_bytes(1, 2, 256, 0)
    for fn in ("entmax_attn_tau_pass",):
        rc = getattr(lib, fn)(_fake(0x1000), _fake(0x2000), _fake(0x3000), _fake(0x4000),
                              _fake(0x10000), need - 1, 1, 2, 2, 256, 64, 1.5, 10, 1, None, 1,
                              0, None)
        assert rc == native.ENOMEM
    rc = lib.entmax_attn_out_pass(_fake(0x1000), _fake(0x2000), _fake(0x3000), _fake(0x4000),
                                  _fake(0x10000), need - 1, _fake(0x5000), 1, 2, 2, 256, 64, 1.5,
                                  1, None, 1, 0, None)
    assert rc == native.ENOMEM


@pytest.mark.parametrize("B,Hq,T,packed", [(1, 2, 256, 0), (2, 32, 16384, 0), (4, 32, 32192, 1),
                                           (1, 32, 131072, 0), (1, 8, 1023, 0)])
def test_workspace_sizes_nest(native, B, Hq, T, packed):
    """The full workspace adds to the smallest one the warm-up sections -- squared norms of
    (B or 1) * Hq * T key rows and B * Hq * levels warm-up tiles of 128 x 128 bf16, levels being
    the ranges 1024 * 2^j that fit in T keys -- and the support sections: one int32 index per
    query row and 2048 eight-byte entries per query tile (slot)."""
    from adaptive_sparse_attention_b200 import api
    lo, hi = api.workspace_min_bytes(B, Hq, T, bool(packed)), api.workspace_bytes(B, Hq, T, bool(packed))
    levels = 0
    while (1024 << levels) <= T:
        levels += 1
    rows = (1 if packed else B) * Hq * T
    slots = (T // 128 + B) if packed else -(-T // 128)
    tiles = (1 if packed else B) * Hq * slots
    def up(x):
        return (x + 255) // 256 * 256
    assert 0 < lo <= hi
    assert hi - lo == (up(4 * rows) + up(B * Hq * levels * 128 * 128 * 2) + up(4 * rows)
                       + up(8 * 2048 * tiles))


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from adaptive_sparse_attention_b200 import _native
    monkeypatch.setattr(_native, "_lib", None)
    monkeypatch.setattr(_native, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(_native.NativeLibraryError):
        _native.lib()


def test_backward_argument_checks(native):
    """entmax_attn_bwd returns its argument errors before any launch (fake pointers)."""
    lib = native.lib()
    p = _fake(0x10000)
    rc = lib.entmax_attn_bwd(p, p, p, None, p, p, 1 << 30, p, p, p, p, 1, 2, 2, 256, 64, 1.5, 1,
                             None, native.BF16, 0, None)
    assert rc == native.EINVAL  # null dout
    rc = lib.entmax_attn_bwd(p, p, p, p, p, p, 1 << 30, p, p, p, p, 1, 2, 2, 256, 48, 1.5, 1,
                             None, native.BF16, 0, None)
    assert rc == native.EINVAL  # d not in {64, 128}
    rc = lib.entmax_attn_bwd(p, p, p, p, p, _fake(0x10010), 1 << 30, p, p, p, p, 1, 2, 2, 256, 64,
                             1.5, 1, None, native.BF16, 0, None)
    assert rc == native.EALIGN  # workspace not 256-byte aligned
    need = lib.entmax_attn_workspace_min_bytes(1, 2, 256, 0)
    rc = lib.entmax_attn_bwd(p, p, p, p, p, p, need - 1, p, p, p, p, 1, 2, 2, 256, 64, 1.5, 1,
                             None, native.BF16, 0, None)
    assert rc == native.ENOMEM


def test_product_never_reaches_the_oracle():
    """The package (Python binding and CUDA sources) imports, includes and loads nothing from
    oracle/, and the oracle nothing from the package but the seeded input generators."""
    import ast
    import pathlib
    root = pathlib.Path(__file__).resolve().parent.parent
    pkg = root / "adaptive_sparse_attention_b200"
    for f in pkg.rglob("*.py"):
        for node in ast.walk(ast.parse(f.read_text())):
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            else:
                continue
            assert not any(n == "oracle" or n.startswith("oracle.") for n in names), f
    for f in list(pkg.rglob("*.cu")) + list(pkg.rglob("*.cuh")) + list(pkg.rglob("*.h")):
        text = f.read_text()
        assert "oracle" not in text.lower(), f
    for f in (root / "oracle").rglob("*.py"):
        for node in ast.walk(ast.parse(f.read_text())):
            if isinstance(node, ast.ImportFrom) and (node.module or "").startswith(
                    "adaptive_sparse_attention_b200"):
                assert node.module == "adaptive_sparse_attention_b200.workloads", f
            if isinstance(node, ast.Import):
                for a in node.names:
                    assert not a.name.startswith("adaptive_sparse_attention_b200") or \
                        a.name == "adaptive_sparse_attention_b200.workloads", f


def test_route_chunks_argument_checks(native):
    """entmax_attn_route_chunks returns its argument errors before any launch (fake pointers)."""
    lib = native.lib()
    p = _fake(0x10000)
    good = [p, p, p, p, 1, 4, 2, 300, 64, 16, 1.5, 10, 1, 1, 1.0, native.BF16, None]

    def call(**kw):
        a = list(good)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return lib.entmax_attn_route_chunks(*a)

    assert call(a1=None) == native.EINVAL       # null summaries
    assert call(a2=None) == native.EINVAL       # null pi
    assert call(a5=3) == native.EINVAL          # Hq not a multiple of Hkv
    assert call(a4=65536) == native.EINVAL      # B above the search grid's 65535
    assert call(a5=65536, a6=1) == native.EINVAL  # Hq above it
    assert call(a8=2000) == native.EINVAL       # d > 1024
    assert call(a9=0) == native.EINVAL          # chunk_size < 1
    assert call(a10=1.0) == native.EINVAL       # alpha <= 1
    assert call(a11=0) == native.EINVAL         # n_iter < 1
    assert call(a13=2) == native.EINVAL         # estimate_diagonal not 0/1
    assert call(a14=float("inf")) == native.EINVAL  # scaling_factor not finite
    assert call(a15=7) == native.EINVAL         # dtype
    assert call(a1=_fake(0x10001)) == native.EALIGN  # bf16 summaries on an odd address
    assert call(a2=_fake(0x10002)) == native.EALIGN  # pi not 4-byte aligned


def test_host_entry_point_argument_checks(native):
    """entmax_attn_fwd_host checks its arguments, host cu_seqlens included, before it touches
    the GPU (fake pointers: never dereferenced on these paths)."""
    import ctypes
    lib = native.lib()
    p = _fake(0x10000)

    def call(B=2, Hq=4, Hkv=2, T=300, d=64, cu=None, dtype=native.BF16, null=None):
        a = [p] * 6
        if null is not None:
            a[null] = None
        return lib.entmax_attn_fwd_host(*a, B, Hq, Hkv, T, d, 1.5, 10, 1, cu, dtype, None)

    for i in range(6):
        assert call(null=i) == native.EINVAL  # a null host pointer
    assert call(Hq=3) == native.EINVAL        # Hq not a multiple of Hkv
    assert call(T=0) == native.EINVAL
    assert call(dtype=9) == native.EINVAL

    def cu(vals):
        arr = (ctypes.c_int32 * len(vals))(*vals)
        return ctypes.cast(arr, ctypes.c_void_p), arr

    bad = [[1, 100, 300], [0, 200, 100, 300], [0, 100, 299]]  # start, order, end
    for vals in bad:
        ptr, keep = cu(vals)
        assert call(B=len(vals) - 1, T=300, cu=ptr) == native.EINVAL, vals


def test_screened_tau_pass_argument_checks(native):
    """entmax_attn_tau_pass_screened: bf16 on the tensor cores with d = 128 only, a 256-byte
    aligned screen buffer of entmax_attn_screen_bytes() bytes (fake pointers, never launched)."""
    lib = native.lib()
    p = _fake(0x10000)
    need = lib.entmax_attn_screen_bytes(1, 2, 1, 300, 0)
    assert need > 0
    assert lib.entmax_attn_screen_bytes(1, 3, 2, 300, 0) == 0  # Hq not a multiple of Hkv
    ws = lib.entmax_attn_workspace_bytes(1, 2, 300, 0)

    def call(d=128, dtype=native.BF16, flags=0, screen=p, sbytes=need):
        return lib.entmax_attn_tau_pass_screened(p, p, p, p, p, ws, screen, sbytes, 1, 2, 1, 300,
                                                 d, 1.5, 10, 1, None, dtype, flags, None)

    assert call(d=64) == native.EINVAL
    assert call(dtype=native.FP32) == native.EINVAL
    assert call(flags=native.FLAG_CUDA_CORES) == native.EINVAL
    assert call(screen=None) == native.EINVAL
    assert call(screen=_fake(0x10010)) == native.EALIGN
    assert call(sbytes=need - 1) == native.ENOMEM
