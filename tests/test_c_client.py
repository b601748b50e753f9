"""A plain C99 program (tests/c_abi_client.c) compiled with gcc against
include/*.h and linked with the in-tree libpaged_attn.so: the headers are
valid C, the entry points have C linkage, and the host block manager called
from C gives, line by line, what the oracle's block manager gives for the
same scenario (page "5.KV Cache 管理 & PagedAttention": Q12 growth, Q18 fork
and copy-on-write, Q20 prefix cache, LRU release).  CPU only."""

import os
import shutil
import subprocess

import pytest

from oracle.block_manager import BlockManager as Oracle
from oracle.block_manager import BlockManagerError
from paged_kv_cache_463_b200 import binding as b
from paged_kv_cache_463_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _oracle_lines():
    nb, bs = 8, 16
    o = Oracle(nb, bs)
    out = []

    def app(what, st, slots, copies):
        out.append(" ".join([what, str(st), "slots", *map(str, slots), "copies",
                             *[f"{s}:{d}" for s, d in copies]]))

    def state(what):
        out.append(" ".join([what, "free", str(o.num_free()), "cached", str(o.cached_blocks()), "refs",
                             *[str(o.ref_counts[k]) for k in range(nb)]]))

    o.add_sequence(1)
    app("grow", b.PA_OK, *o.append_tokens(1, 20))
    o.fork(1, 2)
    state("forked")
    app("child_write", b.PA_OK, *o.append_tokens(2, 1))
    app("parent_write", b.PA_OK, *o.append_tokens(1, 1))
    tables, lens = o.build_batch([1, 2], 4)
    out.append(" ".join(["batch", "lens", str(lens[0]), str(lens[1]), "tables", *map(str, tables[0] + tables[1])]))
    slots, copies = [], []
    for sid in (2, 1):
        s, c = o.append_tokens(sid, 1)
        slots += s
        copies += c
    app("append_batch", b.PA_OK, slots, copies)
    state("after_appends")
    o.free_sequence(1)
    o.free_sequence(2)
    a = [100 + k for k in range(40)]
    bb = [100 + k if k < 32 else 900 + k for k in range(36)]
    m, s = o.allocate_with_prefix(3, a)
    out.append(" ".join(["prefix_a", "matched", str(m), "slots", *map(str, s)]))
    m, s = o.allocate_with_prefix(4, bb)
    out.append(" ".join(["prefix_b", "matched", str(m), "slots", *map(str, s)]))
    state("prefixed")
    out.append(f"evicted {o.evict_lru_sequence(exclude=4)}")
    state("final")
    try:
        o.free_sequence(77)
        out.append("unknown 0")
    except BlockManagerError:
        out.append(f"unknown {b.PA_ERR_INVALID_ARG}")
    return out


@pytest.fixture(scope="module")
def client(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    lib = build.build()
    exe = str(tmp_path_factory.mktemp("c_client") / "c_abi_client")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(HERE, "c_abi_client.c"), "-o", exe, "-L", os.path.dirname(lib), "-lpaged_attn",
           "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_headers_compile_as_cxx():
    """The same client compiles as C++ too (the headers' extern "C" guards)."""
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    r = subprocess.run(["g++", "-x", "c++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-I",
                        os.path.join(ROOT, "include"), os.path.join(HERE, "c_abi_client.c")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_c_client_matches_the_oracle(client):
    r = subprocess.run([client], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = r.stdout.strip().splitlines()
    assert lines[-1].startswith("create ")
    st, rest = lines[-1].split(" ", 2)[1], lines[-1].split(" ", 2)[2]
    assert int(st) == b.PA_ERR_INVALID_ARG and rest.endswith(" 1")  # refused, no context returned
    assert lines[:-1] == _oracle_lines()
