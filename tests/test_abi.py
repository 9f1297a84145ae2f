"""C-ABI checks that need no GPU: the library loads, exports every entry point
the header declares, and rejects bad arguments on the host before any CUDA
call is made."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "uf.h")


@pytest.fixture(scope="module")
def uf(built_lib):
    return built_lib


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(uf_[a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("uf_kv_append", "uf_block_mask", "uf_block_sparse_attn"):
        assert n in names
    assert len(names) >= 10


def test_library_exports_every_declared_symbol(uf):
    lib = ctypes.CDLL(os.path.join(ROOT, "block_sparse_causal_b200", "libuf.so"))
    for n in declared_functions():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (uf_[a-z_0-9]+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported


def declared_arity():
    """Number of parameters of every uf_ prototype in the header."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"(uf_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_signatures_match_the_header(uf):
    # every call the ctypes binding declares has the header's parameter count,
    # and every declared call is bound
    from block_sparse_causal_b200 import _uf
    arity = declared_arity()
    assert set(arity) == set(declared_functions())
    for name, n in arity.items():
        fn = getattr(_uf.lib, name)
        assert fn.argtypes is not None, f"{name} is not bound"
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)


def test_version_and_strerror(uf):
    assert uf.uf_version() >= 100
    for code in range(6):
        assert uf.strerror(code).startswith("UF_")
    assert uf.strerror(99) == "UF_UNKNOWN"


def test_cache_bytes(uf):
    kv, kp, meta = uf.uf_kv_cache_bytes(1, 12, 128, 2, 18720, 128)
    assert kv == 1 * 12 * 2 * (147 * 128) * 128 * 2
    assert kp == 1 * 12 * 2 * 147 * 128 * 4
    assert meta == 16
    kv, kp, _ = uf.uf_kv_cache_bytes(1, 2, 128, 2, 256, 64)
    assert kv == 2 * 2 * 256 * 128 * 2 and kp == 2 * 2 * 4 * 128 * 4
    for bad in [(0, 12, 128, 2, 100, 128), (1, 12, 64, 2, 100, 128), (1, 12, 128, 0, 100, 128),
                (1, 12, 128, 65, 100, 128), (1, 12, 128, 2, 0, 128), (1, 12, 128, 2, 100, 32)]:
        with pytest.raises(uf.UfError) as e:
            uf.uf_kv_cache_bytes(*bad)
        assert e.value.status == uf.UF_EINVAL


class FakeTensor:
    """Stands in for a device tensor: only its address is read on the host."""

    def __init__(self, addr):
        self.addr = addr

    def data_ptr(self):
        return self.addr


def _cache(uf, **kw):
    d = dict(B=1, G=2, D=128, W=2, Lc=300, blk=128)
    d.update(kw)
    return uf.uf_kv_cache_init(FakeTensor(0x100000), FakeTensor(0x200000), FakeTensor(0x300000),
                               FakeTensor(0x400000), d["B"], d["G"], d["D"], d["W"], d["Lc"], d["blk"])


def test_cache_init_validates_on_host(uf):
    c = _cache(uf)
    assert (c.B, c.G, c.W, c.Lc, c.blk, c.host_n_valid) == (1, 2, 2, 300, 128, 0)
    with pytest.raises(uf.UfError):
        uf.uf_kv_cache_init(FakeTensor(0x100008), FakeTensor(0x200000), FakeTensor(0x300000),
                            FakeTensor(0x400000), 1, 2, 128, 2, 300, 128)     # misaligned k
    with pytest.raises(uf.UfError):
        uf.uf_kv_cache_init(None, FakeTensor(0x200000), FakeTensor(0x300000), FakeTensor(0x400000),
                            1, 2, 128, 2, 300, 128)
    with pytest.raises(uf.UfError):
        _cache(uf, D=64)


def test_calls_reject_bad_arguments_before_launch(uf):
    c = _cache(uf)
    q = FakeTensor(0x500000)
    kn, vn = FakeTensor(0x600000), FakeTensor(0x700000)
    # append: keep_chunks out of range, unknown flag, replace on an empty window, misaligned input
    for keep, flags, k_new in [(0, 0, kn), (3, 0, kn), (2, 4, kn), (2, uf.UF_APPEND_REPLACE_NEWEST, kn),
                               (2, 0, FakeTensor(0x600002))]:
        with pytest.raises(uf.UfError) as e:
            uf.uf_kv_append(c, k_new, vn, keep, flags, stream=0)
        assert e.value.status == uf.UF_EINVAL
    # anchor: with replace, on a non-empty window, and keep_chunks 1 while an anchor is pinned
    with pytest.raises(uf.UfError) as e:
        uf.uf_kv_append(c, kn, vn, 2, uf.UF_APPEND_ANCHOR | uf.UF_APPEND_REPLACE_NEWEST, stream=0)
    assert e.value.status == uf.UF_EINVAL
    c.host_n_valid = 1
    with pytest.raises(uf.UfError) as e:
        uf.uf_kv_append(c, kn, vn, 2, uf.UF_APPEND_ANCHOR, stream=0)
    assert e.value.status == uf.UF_EINVAL
    c.host_anchor = 1
    with pytest.raises(uf.UfError) as e:
        uf.uf_kv_append(c, kn, vn, 1, 0, stream=0)
    assert e.value.status == uf.UF_EINVAL
    c.host_n_valid, c.host_anchor = 0, 0
    # FP8 append: NULL or misaligned e4m3 buffer, scale not finite and positive
    for k8, ks in [(None, 1.0), (FakeTensor(0xB00008), 1.0), (FakeTensor(0xB00000), 0.0),
                   (FakeTensor(0xB00000), -2.0), (FakeTensor(0xB00000), float("nan")),
                   (FakeTensor(0xB00000), float("inf"))]:
        with pytest.raises(uf.UfError) as e:
            uf.uf_kv_append_fp8k(c, k8, ks, kn, vn, 2, 0, stream=0)
        assert e.value.status == uf.UF_EINVAL
    # RoPE: negative or too large position, base <= 1 or not finite, misaligned or empty input
    for pos0, base in [(-1, 10000.0), (1 << 40, 10000.0), (0, 1.0), (0, 0.5), (0, float("nan")), (0, float("inf"))]:
        with pytest.raises(uf.UfError) as e:
            uf.uf_kv_append_rope(c, kn, vn, 2, 0, pos0, base, stream=0)
        assert e.value.status == uf.UF_EINVAL
        with pytest.raises(uf.UfError) as e:
            uf.uf_rope(q, q, 1, 4, 2, pos0, base, stream=0)
        assert e.value.status == uf.UF_EINVAL
    for args in [(FakeTensor(0x500008), q, 1, 4, 2), (q, q, 0, 4, 2), (q, q, 1, 0, 2), (q, q, 1, 4, 0)]:
        with pytest.raises(uf.UfError) as e:
            uf.uf_rope(*args, 0, 10000.0, stream=0)
        assert e.value.status == uf.UF_EINVAL
    idx, cnt = FakeTensor(0x800000), FakeTensor(0x900000)
    # mask / attention on an empty window (host mirror) are rejected
    with pytest.raises(uf.UfError):
        uf.uf_block_mask(q, 2, c, 2, idx, cnt, None, stream=0)
    with pytest.raises(uf.UfError):
        uf.uf_block_sparse_attn(q, 2, c, None, None, 0, 0.088, FakeTensor(0xA00000), None, stream=0)
    c.host_n_valid = 1   # pretend one chunk is in the window; still no launch below
    for H, k in [(3, 2), (0, 2), (2, 0), (2, 7)]:        # H % G != 0, H < 1, k < 1, k > W * nb (= 6)
        with pytest.raises(uf.UfError) as e:
            uf.uf_block_mask(q, H, c, k, idx, cnt, None, stream=0)
        assert e.value.status == uf.UF_EINVAL
    # local band: wider than k, negative radius, unknown flag (every case is invalid: nothing launches)
    for k, local, flags in [(2, 1, 0), (5, -1, 0), (5, 1, 2), (6, 3, 0), (3, 1, uf.UF_MASK_LOCAL_ONLY | 4)]:
        with pytest.raises(uf.UfError) as e:
            uf.uf_block_mask_local(q, 2, c, k, local, flags, idx, cnt, None, stream=0)
        assert e.value.status == uf.UF_EINVAL
    for scale in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(uf.UfError) as e:
            uf.uf_block_sparse_attn(q, 2, c, None, None, 0, scale, FakeTensor(0xA00000), None, stream=0)
        assert e.value.status == uf.UF_EINVAL
    # FP8 scores: NULL or misaligned e4m3 K, either scale not finite and positive
    for k8, qs, ks in [(None, 1.0, 1.0), (FakeTensor(0xB00004), 1.0, 1.0), (FakeTensor(0xB00000), 0.0, 1.0),
                       (FakeTensor(0xB00000), 1.0, -1.0), (FakeTensor(0xB00000), float("nan"), 1.0),
                       (FakeTensor(0xB00000), 1.0, float("inf"))]:
        with pytest.raises(uf.UfError) as e:
            uf.uf_block_sparse_attn_fp8k(q, 2, c, k8, qs, ks, None, None, 0, 0.088, FakeTensor(0xA00000), None,
                                         stream=0)
        assert e.value.status == uf.UF_EINVAL
    with pytest.raises(uf.UfError):
        uf.uf_block_sparse_attn(q, 2, c, idx, cnt, 9, 0.088, FakeTensor(0xA00000), None, stream=0)
    # balanced schedule: a workspace is required
    with pytest.raises(uf.UfError) as e:
        uf.uf_block_sparse_attn_balanced(q, 2, c, None, None, 0, 0.088, FakeTensor(0xA00000), None, None, stream=0)
    assert e.value.status == uf.UF_EINVAL
    with pytest.raises(uf.UfError):
        uf.uf_block_sparse_attn(q, 2, c, None, None, 0, 0.088, FakeTensor(0xA00001), None, stream=0)


def test_mask_beyond_1024_window_blocks_is_unsupported(uf):
    # 5 chunks of 205 blocks = 1025 window blocks: one more than the selection holds
    c = _cache(uf, G=1, W=5, Lc=205 * 128)
    c.host_n_valid = 1
    with pytest.raises(uf.UfError) as e:
        uf.uf_block_mask(FakeTensor(0x500000), 1, c, 2, FakeTensor(0x800000), FakeTensor(0x900000), None, stream=0)
    assert e.value.status == uf.UF_EUNSUPPORTED


def test_wait_limit_bounds(uf):
    with pytest.raises(uf.UfError):
        uf.uf_set_wait_limit(10)
    uf.uf_set_wait_limit(1 << 31)
    with pytest.raises(uf.UfError):
        uf.uf_debug_wait_timeout(5, stream=0)


def test_binding_fails_loudly_without_library(tmp_path):
    # a copy of the package without libuf.so must refuse to import (no CPU fallback)
    import shutil
    import sys
    pkg = os.path.join(ROOT, "block_sparse_causal_b200")
    dst = tmp_path / "block_sparse_causal_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc"))
    code = "import block_sparse_causal_b200"
    res = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True)
    assert res.returncode != 0 and "not built" in res.stderr


def test_library_is_built_from_this_tree(uf):
    # the source hash compiled into libuf.so is the hash of csrc/ and include/
    from conftest import load_builder
    assert uf.uf_source_hash() == load_builder().source_hash()


def test_stale_library_is_refused(uf, monkeypatch):
    # a library whose compiled-in hash differs from the tree's sources is refused
    from block_sparse_causal_b200 import _uf, build
    monkeypatch.setattr(build, "source_hash", lambda: "0" * 16)
    with pytest.raises(ImportError, match="other sources"):
        _uf._check_source_hash()


def test_build_rejects_an_attention_register_count_it_cannot_split():
    from conftest import load_builder
    b = load_builder()
    ok = ("ptxas info    : Compiling entry function '_ZN2uf11attn_kernelILi128ELb0EEEv' for 'sm_100a'\n"
          "ptxas info    : Used 168 registers, used 1 barriers\n")
    b.check_attention_registers(ok)
    with pytest.raises(RuntimeError, match="160 registers"):
        b.check_attention_registers(ok.replace("Used 168", "Used 160"))
    with pytest.raises(RuntimeError):
        b.check_attention_registers("ptxas info    : Used 64 registers\n")


def test_error_word_calls_validate_on_host(uf):
    # misaligned or NULL error words are refused before anything is enqueued
    with pytest.raises(uf.UfError):
        uf.uf_check_error(FakeTensor(0), stream=0)
    with pytest.raises(uf.UfError):
        uf.uf_check_error(FakeTensor(0xB00002), stream=0)
    c = uf.uf_kv_cache_init(FakeTensor(0xA00000), FakeTensor(0xA10000), FakeTensor(0xA20000),
                            FakeTensor(0xA30000), 1, 2, 128, 2, 256, 64)
    assert c.err is None
    with pytest.raises(uf.UfError):
        uf.uf_kv_cache_set_error_word(c, FakeTensor(0xB00002))
    uf.uf_kv_cache_set_error_word(c, FakeTensor(0xB00004))
    assert c.err == 0xB00004
    uf.uf_kv_cache_set_error_word(c, None)
    assert c.err is None


def test_clock_counters_validate_on_host(uf):
    # a misaligned counter pair is refused; NULL (off) is always accepted
    lib = uf._uf.lib
    assert lib.uf_set_clock_counters(0xB00004) == uf.UF_EINVAL
    try:
        assert lib.uf_set_clock_counters(0xB00008) == uf.UF_OK
    finally:
        assert lib.uf_set_clock_counters(None) == uf.UF_OK
    with pytest.raises(ValueError):
        uf.uf_set_clock_counters(torch.zeros(2, dtype=torch.int64))      # host memory
