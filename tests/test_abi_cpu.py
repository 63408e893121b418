"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad arguments on the host before launching anything (no GPU needed)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(packkv_\w+)\s*\(", text, flags=re.M))
    return sorted(names)


@pytest.fixture(scope="module")
def pk():
    from decode_gemv_packkv_b200 import build
    build.build()
    from decode_gemv_packkv_b200 import packkv
    return packkv


def test_header_declares_the_four_calls():
    names = _declared_functions()
    for call in ("packkv_encode_block", "packkv_append_token", "packkv_qk_gemv", "packkv_pv_gemv"):
        assert call in names


@pytest.mark.parametrize("lang,std", [("c", "-std=c99"), ("c++", "-std=c++17")])
def test_header_is_plain_c_and_cxx(lang, std, tmp_path):
    """include/*.h compile on their own as strict C99 and as C++ (no torch or CUDA types)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = tmp_path / ("use.c" if lang == "c" else "use.cc")
        src.write_text(f'#include "{os.path.basename(hdr)}"\nint main(void) {{ return 0; }}\n')
        r = subprocess.run([cc, std, "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only",
                            "-I", os.path.dirname(hdr), str(src)], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_library_exports_every_declared_symbol(pk):
    lib = ctypes.CDLL(pk.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(pk.EXPORTED) <= set(_declared_functions())


def test_abi_constants(pk):
    lib = pk._lib
    assert lib.packkv_abi_version() == 3
    assert lib.packkv_cache_struct_size() == ctypes.sizeof(pk.CacheStruct)
    assert [lib.packkv_record_bytes_max(b) for b in (1, 2, 3, 4, 5)] == [0, 4624, 6672, 8720, 0]
    assert lib.packkv_status_string(3) == b"capacity exceeded"


def _fake_cache(pk, **over):
    s = pk.CacheStruct()
    s.fmt = pk.Format(1, 4, 128, 32, 128, 1)
    s.batch, s.kv_heads, s.max_blocks, s.n_blocks, s.tail_len = 2, 2, 4, 0, 0
    base = 0x10000000
    for i, f in enumerate(["k_arena", "v_arena", "k_index", "v_index", "k_tail", "v_tail", "ctrl"]):
        setattr(s, f, base + i * 0x100000)
    s.arena_bytes = 1 << 20
    for k, v in over.items():
        if k in ("bits", "version", "reorder_key", "head_dim", "unit_mode"):
            setattr(s.fmt, k, v)
        else:
            setattr(s, k, v)
    return s


def test_host_checks_reject_before_launch(pk):
    lib = pk._lib
    ok = _fake_cache(pk)
    assert lib.packkv_cache_check(ctypes.byref(ok)) == pk.OK
    assert lib.packkv_cache_check(ctypes.byref(_fake_cache(pk, unit_mode=pk.UNITS_WIDTH_ONLY))) == pk.OK
    bad_cases = {
        "bits": (dict(bits=5), pk.ERR_UNSUPPORTED),
        "version": (dict(version=2), pk.ERR_UNSUPPORTED),
        "head_dim": (dict(head_dim=64), pk.ERR_UNSUPPORTED),
        "key": (dict(reorder_key=7), pk.ERR_UNSUPPORTED),
        "unit mode": (dict(unit_mode=2), pk.ERR_UNSUPPORTED),
        "misaligned": (dict(k_arena=0x10000008), pk.ERR_INVALID_ARG),
        "null": (dict(ctrl=0), pk.ERR_INVALID_ARG),
        "arena": (dict(arena_bytes=1000), pk.ERR_INVALID_ARG),
        "tail": (dict(tail_len=128), pk.ERR_INVALID_ARG),
        "blocks": (dict(n_blocks=5), pk.ERR_INVALID_ARG),
    }
    for name, (over, want) in bad_cases.items():
        s = _fake_cache(pk, **over)
        assert lib.packkv_cache_check(ctypes.byref(s)) == want, name
    # call-level checks (all return before any CUDA call)
    k = ctypes.c_void_p(0x20000000)
    s = _fake_cache(pk, tail_len=3)
    assert lib.packkv_encode_block(ctypes.byref(s), k, k, 1, None) == pk.ERR_INVALID_ARG  # tail not empty
    s = _fake_cache(pk, n_blocks=4)
    assert lib.packkv_encode_block(ctypes.byref(s), k, k, 1, None) == pk.ERR_CAPACITY
    s = _fake_cache(pk, n_blocks=4, tail_len=127)
    assert lib.packkv_append_token(ctypes.byref(s), k, k, None) == pk.ERR_CAPACITY
    s = _fake_cache(pk)
    assert lib.packkv_encode_block(ctypes.byref(s), ctypes.c_void_p(0x20000004), k, 1, None) == pk.ERR_INVALID_ARG
    assert lib.packkv_encode_block(ctypes.byref(s), k, k, 0, None) == pk.OK  # no-op
    assert s.n_blocks == 0
    # GEMVs: bad head grouping, bad leading dimension
    s = _fake_cache(pk, n_blocks=2)
    assert lib.packkv_qk_gemv(ctypes.byref(s), k, 3, 1.0, k, 256, None, 0, None) == pk.ERR_INVALID_ARG
    assert lib.packkv_qk_gemv(ctypes.byref(s), k, 6, 1.0, k, 256, None, 0, None) == pk.ERR_UNSUPPORTED
    assert lib.packkv_qk_gemv(ctypes.byref(s), k, 2, 1.0, k, 255, None, 0, None) == pk.ERR_INVALID_ARG
    assert lib.packkv_qk_gemv(ctypes.byref(s), k, 2, 1.0, k, 254, None, 0, None) == pk.ERR_INVALID_ARG
    assert lib.packkv_pv_gemv(ctypes.byref(s), k, 256, 2, k, k, 0, None) == pk.ERR_INVALID_ARG  # ws too small
    s = _fake_cache(pk)  # empty cache: q·Kᵀ is a no-op
    assert lib.packkv_qk_gemv(ctypes.byref(s), k, 2, 1.0, k, 0, None, 0, None) == pk.OK
    # fused attention: an empty cache has no softmax; bad grouping; misaligned output;
    # a workspace below the size the library reports
    att = lib.packkv_attention_decode
    assert att(ctypes.byref(s), k, 2, 1.0, k, k, 1 << 30, None) == pk.ERR_INVALID_ARG
    s = _fake_cache(pk, n_blocks=2)
    assert att(ctypes.byref(s), k, 3, 1.0, k, k, 1 << 30, None) == pk.ERR_INVALID_ARG
    assert att(ctypes.byref(s), k, 6, 1.0, k, k, 1 << 30, None) == pk.ERR_UNSUPPORTED
    assert att(ctypes.byref(s), k, 2, 1.0, ctypes.c_void_p(0x20000004), k, 1 << 30, None) == pk.ERR_INVALID_ARG
    need = lib.packkv_attention_workspace_bytes(ctypes.byref(s), 2)
    assert need > 0
    assert att(ctypes.byref(s), k, 2, 1.0, k, k, need - 16, None) == pk.ERR_INVALID_ARG


def test_ragged_host_checks(pk):
    """Ragged caches (host counters per sequence): malformed counters, appends that
    would overflow a sequence's blocks, calls that need an empty tail, and calls that
    do not take ragged caches are refused on the host, before any launch."""
    lib = pk._lib
    B = 2
    blocks = (ctypes.c_int32 * B)(1, 3)
    tail = (ctypes.c_int32 * B)(0, 127)
    P = ctypes.POINTER(ctypes.c_int32)

    def ragged(**over):
        s = _fake_cache(pk, **over)
        s.seq_blocks, s.seq_tail = ctypes.cast(blocks, P), ctypes.cast(tail, P)
        return s

    assert lib.packkv_cache_check(ctypes.byref(ragged())) == pk.OK
    assert lib.packkv_cache_check(ctypes.byref(ragged(n_blocks=1))) == pk.ERR_INVALID_ARG
    half = _fake_cache(pk)
    half.seq_blocks = ctypes.cast(blocks, P)
    assert lib.packkv_cache_check(ctypes.byref(half)) == pk.ERR_INVALID_ARG      # seq_tail missing
    tail[1] = 128
    assert lib.packkv_cache_check(ctypes.byref(ragged())) == pk.ERR_INVALID_ARG  # tail out of range
    tail[1] = 127
    blocks[0] = 5
    assert lib.packkv_cache_check(ctypes.byref(ragged())) == pk.ERR_INVALID_ARG  # beyond max_blocks
    blocks[0] = 1
    big = ragged(batch=pk.RAGGED_MAX_BATCH + 1)
    assert lib.packkv_cache_check(ctypes.byref(big)) == pk.ERR_UNSUPPORTED
    k = ctypes.c_void_p(0x20000000)
    s = ragged()
    assert lib.packkv_encode_block(ctypes.byref(s), k, k, 1, None) == pk.ERR_INVALID_ARG  # a tail is not empty
    blocks[1], tail[1] = 4, 127                         # sequence 1 completes a block it has no room for
    act = (ctypes.c_uint8 * B)(0, 1)
    assert lib.packkv_append_token_masked(ctypes.byref(ragged()), k, k, act, None) == pk.ERR_CAPACITY
    assert list(blocks) == [1, 4] and list(tail) == [0, 127]   # nothing advanced
    u = _fake_cache(pk)
    assert lib.packkv_append_token_masked(ctypes.byref(u), k, k, act, None) == pk.ERR_UNSUPPORTED
    assert lib.packkv_pv_gemv_noalloc(ctypes.byref(ragged()), k, 1024, 2, k, None) == pk.ERR_UNSUPPORTED
    s = _fake_cache(pk, n_blocks=1)
    s.block_table = 0x30000002                          # misaligned table
    assert lib.packkv_cache_check(ctypes.byref(s)) == pk.ERR_INVALID_ARG
