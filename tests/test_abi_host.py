"""CPU-only checks of the C-ABI library: it loads, exports every entry point
that include/semicrf.h declares, and rejects bad arguments on the host before
launching anything (no GPU needed for any of this)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "semicrf.h")


@pytest.fixture(scope="module")
def lib():
    from semi_markov_crf_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*SEMICRF_API\s+(?:const\s+)?\w+\s*\*?\s*(semicrf_\w+)\s*\(", text, re.M)))


def test_header_declares_the_four_steps():
    names = declared_functions()
    for n in ("semicrf_prefix_center", "semicrf_forward", "semicrf_backward", "semicrf_viterbi",
              "semicrf_workspace_bytes", "semicrf_get_status", "semicrf_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_loaded_library_is_built_from_the_current_sources():
    from semi_markov_crf_b200 import semicrf
    from semi_markov_crf_b200.build import source_digest
    got = semicrf.source_digest()
    assert len(got) == 64 and got == source_digest(), (
        "the loaded library was built from other kernel sources: rebuild it")


def _ws_bytes(lib, B, T, C, K, flags=0):
    n = ctypes.c_size_t(0)
    rc = lib.semicrf_workspace_bytes(B, T, C, K, ctypes.c_uint(flags), ctypes.byref(n))
    return rc, n.value


def test_workspace_bytes_and_limits(lib):
    rc, n = _ws_bytes(lib, 32, 800, 39, 30)
    assert rc == 0 and n > 32 * 801 * 39 * 8  # at least the split prefix sums
    rc2, n2 = _ws_bytes(lib, 1, 1_000_000, 6, 200)
    assert rc2 == 0
    assert _ws_bytes(lib, 1, 10, 129, 4)[0] == 2          # C above the limit
    assert _ws_bytes(lib, 1, 10, 128, 65)[0] == 2         # K above the limit for C=128
    assert _ws_bytes(lib, 1, 10, 16, 512)[0] == 0
    assert _ws_bytes(lib, 1, 10, 16, 513)[0] == 2
    assert _ws_bytes(lib, 1, 10, 8, 2048)[0] == 0          # long durations, few labels
    assert _ws_bytes(lib, 1, 10, 8, 8192)[0] == 0          # ... up to 8192 (pipelined kernels)
    assert _ws_bytes(lib, 1, 10, 8, 8193)[0] == 2
    assert _ws_bytes(lib, 1, 10, 9, 1024)[0] == 2
    assert _ws_bytes(lib, 1, 10, 9, 2049)[0] == 2
    assert _ws_bytes(lib, -1, 10, 4, 4)[0] == 1
    assert _ws_bytes(lib, 1, 10, 0, 4)[0] == 1
    assert _ws_bytes(lib, 1, 10, 4, 4, flags=0x80)[0] == 1
    assert lib.semicrf_workspace_bytes(1, 10, 4, 4, ctypes.c_uint(0), None) == 1


def _groups(B, T, C, K):
    from semi_markov_crf_b200 import semicrf
    return semicrf.workspace_itemize(B, T, C, K)


def test_workspace_groups_add_up_and_scale_as_designed(lib):
    """Where the workspace goes, from semicrf_workspace_itemize: the groups
    add up to semicrf_workspace_bytes; the checkpoints of the log-domain
    walk grow like the number of checkpoint segments (their K x C rings,
    about sqrt(T) of them at the pages' spacing) while the per-position
    arrays (prefix sums, kept ring rows, decoder rows) grow like T."""
    for B, T, C, K in ((32, 800, 39, 30), (1, 1_000_000, 6, 200), (8, 10_000, 128, 64)):
        g = _groups(B, T, C, K)
        assert sum(g.values()) == _ws_bytes(lib, B, T, C, K)[1]
        assert g["prefix_sums"] >= B * (T + 1) * C * 8
    small, big = _groups(1, 250_000, 6, 200), _groups(1, 1_000_000, 6, 200)
    for key in ("prefix_sums", "kept_rows", "viterbi"):      # O(T C)
        assert 3.9 < big[key] / small[key] < 4.1, key
    # checkpoints: one K x C ring pair per segment; segments grow more slowly
    # than T (sqrt(T K), capped for one wave of the posterior pass)
    assert big["checkpoints"] / small["checkpoints"] < 3.0
    assert big["checkpoints"] < big["prefix_sums"] / 4


def test_host_side_argument_errors_launch_nothing(lib):
    vp = ctypes.c_void_p
    fake = vp(256 * 1024)  # never dereferenced: every call below fails validation first
    # null pointers
    assert lib.semicrf_forward(None, fake, fake, fake, 1, 8, 2, 2, ctypes.c_uint(0), fake,
                               ctypes.c_size_t(1 << 30), fake, None) == 1
    # workspace too small
    assert lib.semicrf_forward(fake, fake, fake, fake, 1, 8, 2, 2, ctypes.c_uint(0), fake,
                               ctypes.c_size_t(16), fake, None) == 3
    # unsupported size
    assert lib.semicrf_viterbi(fake, fake, fake, fake, 1, 8, 200, 2, ctypes.c_uint(0), fake,
                               ctypes.c_size_t(1 << 30), fake, fake, fake, None) == 2
    # unknown flag
    assert lib.semicrf_backward(fake, fake, fake, 1, 8, 2, 2, ctypes.c_uint(0x40), fake,
                                ctypes.c_size_t(1 << 30), None, fake, fake, fake, None, None, None,
                                None) == 1
    # misaligned workspace
    assert lib.semicrf_forward(fake, fake, fake, fake, 1, 8, 2, 2, ctypes.c_uint(0), vp(256 * 1024 + 8),
                               ctypes.c_size_t(1 << 30), fake, None) == 1


def test_host_side_argument_errors_of_the_loss_and_projection_calls(lib):
    vp = ctypes.c_void_p
    fake = vp(256 * 1024)  # never dereferenced: every call below fails validation first
    big = ctypes.c_size_t(1 << 30)
    u0 = ctypes.c_uint(0)
    # path score: missing labels / workspace too small / unknown flag
    assert lib.semicrf_path_score(fake, fake, fake, fake, None, fake, 1, 8, 2, 2, u0, fake, big,
                                  None, fake, None, None, None, None) == 1
    assert lib.semicrf_path_score(fake, fake, fake, fake, fake, fake, 1, 8, 2, 2, u0, fake,
                                  ctypes.c_size_t(16), None, fake, None, None, None, None) == 3
    assert lib.semicrf_path_score(fake, fake, fake, fake, fake, fake, 1, 8, 2, 2,
                                  ctypes.c_uint(0x40), fake, big, None, fake, None, None, None,
                                  None) == 1
    assert lib.semicrf_path_score_proj(fake, None, fake, fake, fake, fake, fake, fake, 1, 8, 2, 2,
                                       u0, fake, big, None, fake, None, None, None, None, None,
                                       None) == 1
    # projection entry points: null inputs, unsupported sizes, misaligned workspace
    assert lib.semicrf_forward_proj(None, fake, fake, fake, fake, fake, 1, 8, 2, 2, u0, fake, big,
                                    fake, None) == 1
    assert lib.semicrf_forward_proj(fake, fake, fake, fake, fake, fake, 1, 8, 2, 9000, u0, fake,
                                    big, fake, None) == 2
    assert lib.semicrf_forward_proj(fake, fake, fake, fake, fake, fake, 1, 8, 2, 2, u0,
                                    vp(256 * 1024 + 8), big, fake, None) == 1
    assert lib.semicrf_viterbi_proj(fake, fake, fake, fake, fake, fake, 1, 8, 2, 2, u0, fake, big,
                                    None, fake, fake, None) == 1
    assert lib.semicrf_backward_proj(fake, fake, fake, 1, 8, 2, 2, u0, fake, ctypes.c_size_t(16),
                                     None, fake, fake, fake, None, None, None, None, None,
                                     None) == 3


def test_strerror_names_every_status(lib):
    lib.semicrf_strerror.restype = ctypes.c_char_p
    seen = {lib.semicrf_strerror(i).decode() for i in range(8)}
    assert len(seen) == 8 and "unknown status" not in seen
    assert lib.semicrf_strerror(99).decode() == "unknown status"


def test_binding_argument_lists_match_the_header():
    import re
    torch = pytest.importorskip("torch")  # noqa: F841  (the binding imports it)
    from semi_markov_crf_b200 import semicrf
    header = open(os.path.join(ROOT, "include", "semicrf.h")).read()
    header = re.sub(r"/\*.*?\*/", "", header, flags=re.S)
    decls = re.findall(r"SEMICRF_API\s+[\w\s\*]+?\b(semicrf_\w+)\s*\(([^;]*?)\)\s*;", header, flags=re.S)
    assert len(decls) >= 15
    for name, params in decls:
        n = 0 if params.strip() in ("", "void") else params.count(",") + 1
        fn = getattr(semicrf.lib, name)
        if fn.argtypes is None:
            continue  # declared but not bound by the Python layer
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
