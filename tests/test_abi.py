"""libpkv.so loads and exports the C ABI of include/*.h; host-side
validation returns its status codes without touching a device (CPU only)."""

import ctypes
import os
import re

import pytest

from paged_kv_cache_407_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")


def declared_functions():
    names = set()
    for f in sorted(os.listdir(INCLUDE)):
        if f.endswith(".h"):
            text = open(os.path.join(INCLUDE, f), encoding="utf-8").read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(pkv_[a-z_0-9]+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_407_b200.build import build
    build()
    return bd.library()


def test_header_declares_the_hot_path():
    names = declared_functions()
    for n in ("pkv_reshape_and_cache", "pkv_paged_attention_decode", "pkv_copy_blocks",
              "pkv_paged_attention_workspace_size", "pkv_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(bd.SIGNATURES), "binding and header disagree"


def test_only_declared_symbols_are_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", bd.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if l.split()[-2:-1] == ["T"]}
    ours = {s for s in exported if s.startswith("pkv_")}
    assert ours == set(declared_functions())


def test_status_strings_and_version(lib):
    for code in range(13):
        assert lib.pkv_status_string(code) != b"unknown pkv_status"
    assert lib.pkv_status_string(0) == b"ok"
    assert bd.version() >= 100


@pytest.fixture(scope="module")
def check_lib():
    from paged_kv_cache_407_b200.build import build_check
    build_check()
    return bd.check_library()


def test_check_build_exports_the_same_abi(lib, check_lib):
    """libpkv_check.so (PKV_CHECK) declares and exports exactly what
    libpkv.so does, and says which build it is."""
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", bd.CHECK_LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if l.split()[-2:-1] == ["T"]}
    assert {s for s in exported if s.startswith("pkv_")} == set(declared_functions())
    assert check_lib.pkv_check_build() == 1 and lib.pkv_check_build() == 0
    assert check_lib.pkv_status_string(bd.ERR_ALIAS) == lib.pkv_status_string(bd.ERR_ALIAS)


def test_check_build_validates_arguments_before_its_alias_checks(check_lib):
    """The host-side argument checks come first and are the regular build's;
    calls with nothing to write or copy return at once, touching no device."""
    null = None
    d = bd.CacheDesc(16, 16, 4, 64, 0)
    assert check_lib.pkv_reshape_and_cache(null, null, 0, 0, null, null, d, null, 1, null, null) == 1
    assert check_lib.pkv_reshape_and_cache(null, null, 0, 0, null, null, d, null, 0, null, null) == 0
    assert check_lib.pkv_copy_blocks(null, null, d, null, 0, null, null) == 0
    assert check_lib.pkv_copy_blocks(null, null, d, null, 2, null, null) == 1
    assert check_lib.pkv_copy_blocks(null, null, bd.CacheDesc(16, 12, 4, 64, 0), null, 2, null, null) == 3


def _desc(N=16, B=16, H=4, D=64, dt=0):
    return bd.CacheDesc(N, B, H, D, dt)


def test_host_validation_without_device(lib):
    null = None
    # NULL key with tokens to write
    assert lib.pkv_reshape_and_cache(null, null, 0, 0, null, null, _desc(), null, 1, null, null) == 1
    # zero tokens: nothing to do, no device needed
    assert lib.pkv_reshape_and_cache(null, null, 0, 0, null, null, _desc(), null, 0, null, null) == 0
    # bad dtype / block size / head dim
    assert lib.pkv_copy_blocks(null, null, _desc(dt=7), null, 1, null, null) == 2
    assert lib.pkv_copy_blocks(null, null, _desc(B=12), null, 1, null, null) == 3
    assert lib.pkv_copy_blocks(null, null, _desc(D=96), null, 1, null, null) == 3
    dec = lib.pkv_paged_attention_decode
    args = lambda **k: [k.get("out"), null, null, null, k.get("desc", _desc()), null, 4, null,
                        k.get("S", 2), k.get("Hq", 4), 64, ctypes.c_float(k.get("scale", 0.125)),
                        k.get("P", 0), null, 0, null, null]
    assert dec(*args(P=24)) == 6            # not a multiple of block_size
    assert dec(*args(Hq=6)) == 3            # Hq not a multiple of Hkv
    assert dec(*args(Hq=4 * 17, desc=_desc(H=4))) == 3  # group larger than 16
    assert dec(*args(scale=0.0)) == 3
    assert dec(*args(S=0)) == 0             # nothing to do
    assert dec(*args()) == 1                # NULL pointers


def test_workspace_and_partition_queries(lib):
    # automatic partitions of 1024 tokens, smaller when the grid would be thin
    assert bd.partition_size(64, 32, 16, 2048) == 2048  # enough (seq, kv head) units: no split
    assert bd.partition_size(64, 32, 16, 2035) == 2048
    assert bd.partition_size(256, 8, 16, 4096) == 1024  # long tail: split
    assert bd.partition_size(32, 32, 16, 2048) == 1024  # too few units
    assert bd.partition_size(4, 8, 32, 131072) == 1024
    assert bd.partition_size(1, 8, 16, 32768) == 256
    assert bd.partition_size(4, 8, 16, 32768) == 512
    assert bd.partition_size(4, 8, 32, 131072, 512) == 512
    assert bd.partition_size(4, 8, 32, 131072, 500) == -1
    # no split, no workspace
    assert bd.workspace_size(4, 4, 4, 64, 16, 33) == 0
    # 131072 tokens in 512-token partitions: one int32 arrival counter per
    # (seq, kv head), then 256 partials of (D + 2) floats per (seq, head)
    # [arrival counters + unit count, 16-byte padded][unit list (int2), padded][partials]
    assert bd.workspace_size(4, 32, 8, 128, 32, 131072, 512) == 144 + 4 * 256 * 8 + 4 * 32 * 256 * 130 * 4
    assert bd.workspace_size(3, 4, 1, 64, 16, 2000, 256) == 16 + 3 * 8 * 8 + 3 * 4 * 8 * 66 * 4
    assert bd.workspace_size(4, 32, 8, 128, 32, 131072, 24) == 0  # invalid partition


def test_prefill_host_validation_without_device(lib):
    """pkv_paged_prefill checks its arguments on the host before it looks for
    a device: each broken rule returns its status, empty calls return OK."""
    null = None
    A = ctypes.c_void_p(0x10000)       # 16-byte aligned stand-ins, never dereferenced
    odd = ctypes.c_void_p(0x10008)     # 8-byte aligned only
    pre = lib.pkv_paged_prefill

    def call(desc=None, out=A, q=A, k=A, v=A, tables=A, qs=A, lens=A, S=2, T=64, maxq=32, Hq=8,
             scale=0.125, ws=null, ws_bytes=0):
        return pre(out, q, k, v, desc or _desc(N=64, B=16, H=4, D=128), tables, 8, qs, lens, S, T, maxq, Hq,
                   ctypes.c_float(scale), ws, ws_bytes, null, null)

    assert call(desc=_desc(D=64)) == 3                 # head_dim must be 128
    assert call(desc=_desc(D=128, dt=2)) == 2          # 8-bit pools: not for prefill
    assert call(Hq=6) == 3                             # Hq not a multiple of Hkv
    assert call(Hq=4 * 32) == 3                        # group of 32 > 16
    assert call(Hq=12, desc=_desc(N=64, B=16, H=4, D=128)) == 3  # group of 3 does not divide 128 rows
    assert call(scale=0.0) == 3
    assert call(scale=float("inf")) == 3
    assert call(S=0) == 0 and call(T=0) == 0 and call(maxq=0) == 0  # nothing to do
    assert call(q=null) == 1 and call(lens=null) == 1 and call(qs=null) == 1
    assert call(k=odd) == 4 and call(out=odd) == 4     # pools and rows must be 16-byte aligned
    assert call(ws=ctypes.c_void_p(0x10002), ws_bytes=16) == 4   # workspace: 4-byte aligned
    assert call(ws=A, ws_bytes=bd.PREFILL_WORKSPACE_BYTES - 1) == 5  # workspace too small
    # query tiles x kv heads x sequences beyond 2^31 - 1
    assert call(S=40, maxq=2**31 - 1, Hq=4) == 7


def test_split_state_calls_validate_on_the_host(lib):
    """The attention-state entry points of the cross-GPU split check their
    arguments before any device work."""
    null = None
    A = ctypes.c_void_p(0x10000)
    merge = lib.pkv_merge_attention_states
    assert merge(A, 2, A, 129, 2, 1, 128, null) == 2        # 8-bit output: not accepted
    assert merge(A, 0, A, 97, 2, 1, 96, null) == 3          # head_dim 96
    assert merge(A, 0, A, 128, 2, 1, 128, null) == 3        # stride below rows * (D + 1)
    assert merge(A, 0, A, 0, 2, 0, 128, null) == 0          # no rows: nothing to do
    assert merge(null, 0, A, 129, 2, 1, 128, null) == 1
    assert merge(A, 0, null, 129, 2, 1, 128, null) == 1
    assert merge(A, 1, ctypes.c_void_p(0x10002), 129, 2, 1, 128, null) == 4
    lse = lib.pkv_paged_attention_decode_lse
    desc = _desc(N=16, B=16, H=4, D=64)
    # NULL log-sum-exp output with sequences to do
    assert lse(A, null, A, A, A, desc, A, 4, A, 2, 4, 64, ctypes.c_float(0.125), 0, null, 0, null, null) == 1
    # otherwise the decode rules: partition not a multiple of the block size
    assert lse(A, A, A, A, A, desc, A, 4, A, 2, 4, 64, ctypes.c_float(0.125), 24, null, 0, null, null) == 6


def test_fp8_calls_validate_on_the_host(lib):
    """The 8-bit write and decode check pool dtype, shapes, scales, pointers,
    alignment and workspace on the host."""
    null = None
    A = ctypes.c_void_p(0x10000)
    f8 = _desc(N=16, B=16, H=4, D=128, dt=2)
    wr = lib.pkv_reshape_and_cache_fp8
    f = ctypes.c_float

    def write(desc=f8, in_dt=0, T=3, ks=0.5, vs=0.5, key=A):
        return wr(key, A, 0, 0, in_dt, A, A, desc, A, T, f(ks), f(vs), null, null)

    assert write(desc=_desc(N=16, B=16, H=4, D=128, dt=0)) == 2   # 16-bit pool
    assert write(in_dt=2) == 2                                      # 8-bit input
    assert write(desc=_desc(N=16, B=8, H=4, D=128, dt=2)) == 3      # 8-token blocks
    assert write(ks=0.0) == 3 and write(vs=float("nan")) == 3
    assert write(T=0) == 0
    assert write(key=null) == 1
    dec = lib.pkv_paged_attention_decode_fp8

    def decode(desc=f8, q_dt=1, ks=0.5, P=0, ws=null, ws_bytes=0, maxlen=64, out=A):
        return dec(out, A, q_dt, A, A, desc, A, 64, A, 2, 8, maxlen, f(0.125), f(ks), f(0.5), P, ws, ws_bytes,
                   null, null)

    assert decode(desc=_desc(N=16, B=16, H=4, D=64, dt=2)) == 3    # head_dim 64 on 8-bit pools
    assert decode(q_dt=2) == 2
    assert decode(ks=-1.0) == 3
    assert decode(P=24) == 6
    assert decode(out=ctypes.c_void_p(0x10002)) == 4
    # a call that splits needs its workspace
    need = bd.workspace_size(2, 8, 4, 128, 16, 1024, 256)
    assert need > 0
    assert decode(P=256, maxlen=1024) == 5
    assert decode(P=256, maxlen=1024, ws=A, ws_bytes=need - 1) == 5


def test_withheld_load_entry_validates_on_the_host(lib):
    """The fault-injection entry point accepts only its one kernel instance
    (fp16 pools, head_dim 128, 16-token blocks, up to 8 query heads per kv
    head), a wait limit of 1 us .. 1 s and a withheld block inside the first
    partition; each rule is checked before any device work."""
    null = None
    A = ctypes.c_void_p(0x10000)
    fn = lib.pkv_test_decode_withheld_load

    def call(desc=None, Hq=8, maxlen=300, P=512, block=3, wait_us=3000):
        return fn(A, A, A, A, desc or _desc(N=64, B=16, H=2, D=128), A, 32, A, 4, Hq, maxlen,
                  ctypes.c_float(0.1), P, null, 0, block, wait_us, null, null)

    assert call(desc=_desc(N=64, B=16, H=2, D=128, dt=1)) == 3   # bf16 pools
    assert call(desc=_desc(N=64, B=32, H=2, D=128)) == 3         # 32-token blocks
    assert call(desc=_desc(N=64, B=16, H=2, D=64)) == 3          # head_dim 64
    assert call(Hq=2 * 16) == 3                                  # 16 query heads per kv head
    assert call(wait_us=0) == 3 and call(wait_us=2_000_000) == 3
    assert call(block=-1) == 3
    assert call(block=32) == 6                                   # past the first 512-token partition


def test_binding_can_route_every_call_to_the_check_build(check_lib):
    """use_check_build() before the first call makes library() serve
    libpkv_check.so; after the regular build is in use it refuses."""
    import subprocess
    import sys
    code = ("from paged_kv_cache_407_b200 import binding as bd; bd.use_check_build(); "
            "assert bd.library().pkv_check_build() == 1; assert bd.library()._name == bd.CHECK_LIB_PATH; "
            "print('ok')")
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stderr
    code = ("from paged_kv_cache_407_b200 import binding as bd; bd.library()\n"
            "try:\n    bd.use_check_build()\nexcept RuntimeError:\n    print('refused')")
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert res.returncode == 0 and res.stdout.strip() == "refused", res.stderr


def test_headers_are_plain_c_and_usable_from_c(lib, tmp_path):
    """tests/native/c_client.c includes both headers as strict C99 (no
    warning with -pedantic), links libpkv.so and checks the calls that need
    no GPU: status text, version, host-side argument checks, and the block
    manager through a prompt, a fork, a copy-on-write step and a free."""
    import shutil
    import subprocess
    from paged_kv_cache_407_b200.build import INCLUDE, LIB_PATH
    cc = os.environ.get("CC") or shutil.which("gcc") or shutil.which("cc")
    assert cc, "a host C compiler is needed"
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "native", "c_client.c")
    exe = str(tmp_path / "c_client")
    libdir = os.path.dirname(LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", INCLUDE, src, "-L", libdir,
                    "-lpkv", f"-Wl,-rpath,{libdir}", "-o", exe], check=True, capture_output=True, text=True)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0 and res.stdout.strip() == "c client ok", (res.stdout, res.stderr)
