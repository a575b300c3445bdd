"""The C ABI without a GPU: the library loads, exports every symbol that
include/jetlong.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jetlong.h")

FAKE = 0x10000  # an aligned non-null address; validation never dereferences it


@pytest.fixture(scope="module")
def lib():
    from long_context_attention_bifocal_b200 import build
    build.build()
    import long_context_attention_bifocal_b200 as jl
    return jl.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(jl_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("jl_bifocal_prefill", "jl_bifocal_prefill_ex", "jl_bifocal_decode",
              "jl_bifocal_decode_workspace_size", "jl_bifocal_prefill_workspace_size",
              "jl_last_error", "jl_check_device_status", "jl_finalize", "jl_group_size"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in jetlong.h but not exported"


def test_group_size_host(lib):
    assert lib.jl_group_size(65536, 32768) == 2
    assert lib.jl_group_size(131072, 32768) == 4
    assert lib.jl_group_size(32768, 32768) == 1
    assert lib.jl_group_size(98304, 32768) == 3
    assert lib.jl_group_size(0, 5) == -1
    assert lib.jl_group_size(5, 0) == -1
    # no overflow at the top of the 64-bit range
    big = 2**63 - 1
    assert lib.jl_group_size(big, 2) == big // 2 + 1
    assert lib.jl_group_size(big, big) == 1
    assert lib.jl_group_size(big - 1, big) == 1
    assert lib.jl_group_size(big, 1) == big


def _prefill(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, L=256, Hq=4, Hkv=2, D=128,
             w_local=64, w_pretrained=128, base=1e6, dtype=0, scale=0.0, flags=0,
             ws=None, ws_bytes=0)
    a.update(kw)
    return lib.jl_bifocal_prefill_ex(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"],
                                     a["L"], a["Hq"], a["Hkv"], a["D"], a["w_local"],
                                     a["w_pretrained"], a["base"], a["dtype"], a["scale"],
                                     a["flags"], a["ws"], a["ws_bytes"], None)


INVALID, UNSUPPORTED = 1, 2


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=3, Hkv=2), INVALID),
    (dict(B=0), INVALID),
    (dict(L=0), INVALID),
    (dict(D=7), INVALID),
    (dict(D=64), UNSUPPORTED),            # bf16 path is head dim 128
    (dict(D=256, dtype=1), UNSUPPORTED),  # fp32 path is 64 or 128
    (dict(w_local=-1), INVALID),
    (dict(w_pretrained=0), INVALID),
    (dict(base=1.0), INVALID),
    (dict(base=float("nan")), INVALID),
    (dict(q=None), INVALID),
    (dict(k=FAKE + 2), INVALID),          # misaligned
    (dict(flags=1 << 7), INVALID),
    (dict(flags=1 << 31), INVALID),       # the decode-only test flag
    (dict(dtype=5), INVALID),
    (dict(flags=1 << 2), INVALID),                                    # keys rotated once: no workspace
    (dict(flags=1 << 2, ws=FAKE + 16, ws_bytes=1 << 30), INVALID),    # workspace not 256-aligned
    (dict(flags=1 << 2, ws=FAKE, ws_bytes=10), INVALID),              # workspace too small
])
def test_prefill_rejects(lib, kw, code):
    assert _prefill(lib, **kw) == code
    assert lib.jl_last_error()  # a message is left


def _decode(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, pos=100, cap=200, out=FAKE, lse=FAKE, ws=FAKE,
             ws_bytes=1 << 30, B=1, Hq=8, Hkv=2, D=128, w_local=16, w_pretrained=64,
             base=1e6, flags=0)
    a.update(kw)
    return lib.jl_bifocal_decode(a["q"], a["kc"], a["vc"], a["pos"], a["cap"], a["out"],
                                 a["lse"], a["ws"], a["ws_bytes"], a["B"], a["Hq"],
                                 a["Hkv"], a["D"], a["w_local"], a["w_pretrained"],
                                 a["base"], a["flags"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(pos=200), INVALID),
    (dict(pos=-1), INVALID),
    (dict(Hq=6, Hkv=4), INVALID),
    (dict(D=64), UNSUPPORTED),
    (dict(ws=None), INVALID),
    (dict(ws_bytes=8), INVALID),
    (dict(kc=FAKE + 4), INVALID),
    (dict(w_local=-3), INVALID),
    (dict(flags=2), INVALID),
    (dict(Hq=18, Hkv=2, flags=1 << 31), UNSUPPORTED),  # group 9: no tensor-core kernel
])
def test_decode_rejects(lib, kw, code):
    assert _decode(lib, **kw) == code
    assert lib.jl_last_error()


def test_workspace_sizes(lib):
    # keys are rotated inside the prefill kernels: no workspace at any size
    assert lib.jl_bifocal_prefill_workspace_size(1, 131072, 8, 128, 0) == 0
    assert lib.jl_bifocal_prefill_workspace_size(1, 100, 8, 64, 1) == 0
    assert lib.jl_bifocal_prefill_chunk_workspace_size(1, 131072 - 16384, 16384, 8, 128) == 0
    # the opt-in mode that rotates the keys once: two bf16 copies, 256-aligned each
    assert lib.jl_bifocal_prefill_rotated_keys_bytes(1, 131072, 8, 128) == 2 * 131072 * 8 * 128 * 2
    assert lib.jl_bifocal_prefill_rotated_keys_bytes(1, 3, 1, 128) == 2 * 768
    assert lib.jl_bifocal_prefill_rotated_keys_bytes(0, 3, 1, 128) == 0
    n = lib.jl_bifocal_decode_workspace_size(1, 32, 8, 128, 131071)
    assert n > 0 and n % 4 == 0
    assert lib.jl_bifocal_decode_workspace_size(1, 32, 8, 128, -1) == 0


def test_product_path_has_no_oracle_or_fallback():
    """The library package never imports the oracle and has no CPU path."""
    pkg = os.path.join(ROOT, "long_context_attention_bifocal_b200")
    for name in os.listdir(pkg):
        if name.endswith(".py"):
            src = open(os.path.join(pkg, name)).read()
            assert "import oracle" not in src and "from oracle" not in src, name


def _prefill_3pass(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, L=256, Hq=4, Hkv=2, D=128,
             w_local=64, w_pretrained=128, base=1e6, flags=0, ws=FAKE, ws_bytes=1 << 32)
    a.update(kw)
    return lib.jl_bifocal_prefill_3pass(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"],
                                        a["L"], a["Hq"], a["Hkv"], a["D"], a["w_local"],
                                        a["w_pretrained"], a["base"], a["flags"], a["ws"],
                                        a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=64), UNSUPPORTED),
    (dict(ws=None), INVALID),
    (dict(ws=FAKE + 16), INVALID),          # workspace not 256-aligned
    (dict(ws_bytes=100), INVALID),          # workspace too small
    (dict(flags=1 << 31), INVALID),
    (dict(Hq=3), INVALID),
    (dict(w_local=-1), INVALID),
])
def test_prefill_3pass_rejects(lib, kw, code):
    assert _prefill_3pass(lib, **kw) == code
    assert lib.jl_last_error()


def test_prefill_3pass_workspace_size(lib):
    B, L, Hq, Hkv, D = 1, 1000, 4, 2, 128
    n = lib.jl_bifocal_prefill_3pass_workspace_size(B, L, Hq, Hkv, D)
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    # O_B and O_C (bf16) and their lse; the keys are rotated inside the kernels
    assert n == 2 * up(B * L * Hq * D * 2) + 2 * up(B * Hq * L * 4)


def _decode_batched(lib, pos=(100, 5), **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, cap=200, out=FAKE, lse=FAKE, ws=FAKE,
             ws_bytes=1 << 30, B=len(pos) if pos else 2, Hq=8, Hkv=2, D=128, w_local=16,
             w_pretrained=64,
             base=1e6, flags=0)
    a.update(kw)
    arr = (ctypes.c_int * len(pos))(*pos) if pos is not None else None
    return lib.jl_bifocal_decode_batched(a["q"], a["kc"], a["vc"], arr, a["cap"], a["out"],
                                         a["lse"], a["ws"], a["ws_bytes"], a["B"], a["Hq"],
                                         a["Hkv"], a["D"], a["w_local"], a["w_pretrained"],
                                         a["base"], a["flags"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(pos=(100, 200)), INVALID),          # pos >= cap
    (dict(pos=(100, -1)), INVALID),
    (dict(pos=None, B=2), INVALID),
    (dict(D=64), UNSUPPORTED),
    (dict(Hq=18, Hkv=2), UNSUPPORTED),        # group 9: no tensor-core kernel
    (dict(ws_bytes=64), INVALID),
    (dict(ws=FAKE + 16), INVALID),            # not 256-aligned
    (dict(flags=1 << 31), INVALID),
])
def test_decode_batched_rejects(lib, kw, code):
    pos = kw.pop("pos", (100, 5))
    assert _decode_batched(lib, pos=pos, **kw) == code
    assert lib.jl_last_error()


def test_decode_batched_workspace_size(lib):
    n = lib.jl_bifocal_decode_batched_workspace_size(4, 32, 8, 128)
    assert n >= (148 + 8) * 32 * 132 * 4
    assert lib.jl_bifocal_decode_batched_workspace_size(4, 32, 8, 64) == 0


def _prefill_chunk(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, q_offset=256, cap=1024, out=FAKE, lse=FAKE, B=1, Lq=300,
             Hq=4, Hkv=2, D=128, w_local=64, w_pretrained=128, base=1e6, flags=0, ws=None,
             ws_bytes=0)
    a.update(kw)
    return lib.jl_bifocal_prefill_chunk(a["q"], a["kc"], a["vc"], a["q_offset"], a["cap"],
                                        a["out"], a["lse"], a["B"], a["Lq"], a["Hq"], a["Hkv"],
                                        a["D"], a["w_local"], a["w_pretrained"], a["base"],
                                        a["flags"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q_offset=100), UNSUPPORTED),       # not a multiple of 128
    (dict(q_offset=-128), UNSUPPORTED),
    (dict(cap=500), INVALID),                # q_offset + Lq > cap
    (dict(D=64), UNSUPPORTED),
    (dict(Lq=0), INVALID),
    (dict(flags=1 << 31), INVALID),
])
def test_prefill_chunk_rejects(lib, kw, code):
    assert _prefill_chunk(lib, **kw) == code
    assert lib.jl_last_error()


def _decode_paged(lib, pos=(100, 5), **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, num_pages=64, page_size=16, bt=FAKE, max_pages=8,
             out=FAKE, lse=FAKE, ws=FAKE, ws_bytes=1 << 30, B=len(pos) if pos else 2, Hq=8,
             Hkv=2, D=128, w_local=16, w_pretrained=64, base=1e6, flags=0)
    a.update(kw)
    arr = (ctypes.c_int * len(pos))(*pos) if pos is not None else None
    return lib.jl_bifocal_decode_paged(a["q"], a["kc"], a["vc"], a["num_pages"],
                                       a["page_size"], a["bt"], a["max_pages"], arr, a["out"],
                                       a["lse"], a["ws"], a["ws_bytes"], a["B"], a["Hq"],
                                       a["Hkv"], a["D"], a["w_local"], a["w_pretrained"],
                                       a["base"], a["flags"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(pos=(100, 128)), INVALID),          # pos >= max_pages * page_size
    (dict(pos=(100, -1)), INVALID),
    (dict(pos=None, B=2), INVALID),
    (dict(page_size=8), INVALID),             # not a multiple of 16
    (dict(page_size=40), INVALID),
    (dict(page_size=0), INVALID),
    (dict(num_pages=0), INVALID),
    (dict(max_pages=0), INVALID),
    (dict(num_pages=1 << 27, page_size=32), INVALID),   # 2^32 rows
    (dict(bt=None), INVALID),
    (dict(bt=FAKE + 2), INVALID),             # block table not 4-byte aligned
    (dict(kc=FAKE + 8), INVALID),
    (dict(D=64), UNSUPPORTED),
    (dict(Hq=18, Hkv=2), UNSUPPORTED),
    (dict(ws_bytes=64), INVALID),
    (dict(flags=1 << 31), INVALID),
])
def test_decode_paged_rejects(lib, kw, code):
    pos = kw.pop("pos", (100, 5))
    assert _decode_paged(lib, pos=pos, **kw) == code
    assert lib.jl_last_error()


def test_decode_batched_device_positions_must_be_aligned(lib):
    """With JL_FLAG_DEVICE_POS the positions are a device pointer: it must be
    4-byte aligned (its values are checked on the device, not here)."""
    B = 2
    rc = lib.jl_bifocal_decode_batched(FAKE, FAKE, FAKE, ctypes.c_void_p(FAKE + 2), 200, FAKE,
                                       FAKE, FAKE, 1 << 30, B, 8, 2, 128, 16, 64, 1e6, 1 << 1,
                                       None)
    assert rc == INVALID
    assert lib.jl_last_error()
    rc = lib.jl_bifocal_decode_paged(FAKE, FAKE, FAKE, 64, 16, FAKE, 8, ctypes.c_void_p(FAKE + 2),
                                     FAKE, FAKE, FAKE, 1 << 30, B, 8, 2, 128, 16, 64, 1e6, 1 << 1,
                                     None)
    assert rc == INVALID
