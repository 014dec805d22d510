"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any CUDA call.

Pointers below are fake integers: every rejection tested here happens in the
library's pure host checks (null, sizes, dims, dtype, chunk, alignment,
overlap), so nothing is dereferenced and no device is touched.
"""
import ctypes
import os
import re

import pytest

from gated_deltanet_linear_chunked_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = header_symbols()
    for name in ("gdn_chunk_fwd", "gdn_chunk_bidir", "gdn_state_reset", "gdn_status_string"):
        assert name in syms


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for name in header_symbols():
        assert hasattr(lib, name), name
    assert set(header_symbols()) == set(_lib.SIGNATURES)


def test_status_strings_and_version():
    lib = _lib.load()
    names = [lib.gdn_status_string(i).decode() for i in range(6)]
    assert names == ["GDN_OK", "GDN_ERR_INVALID_ARG", "GDN_ERR_UNSUPPORTED",
                     "GDN_ERR_ALIAS", "GDN_ERR_CUDA", "GDN_ERR_TIMEOUT"]
    assert lib.gdn_status_string(6).decode() == "GDN_ERR_SCRATCH_LIMIT"
    assert lib.gdn_status_string(99).decode() == "GDN_ERR_UNKNOWN"
    assert lib.gdn_version() >= 100


# Fake, 16-byte aligned, non-overlapping "device" addresses.
MB = 1 << 20
BASE = 0x7F0000000000


def fake(i):
    return BASE + i * 256 * MB


def call(entry="gdn_chunk_fwd", q=fake(0), k=fake(1), v=fake(2), g=fake(3), beta=fake(4),
         s_in=fake(5), s_out=fake(6), out=fake(7), B=1, T=64, H=2, Dk=64, Dv=64,
         dtype=_lib.GDN_BF16, chunk=0):
    lib = _lib.load()
    return getattr(lib, entry)(q, k, v, g, beta, s_in, s_out, out, B, T, H, Dk, Dv,
                               dtype, chunk, None)


@pytest.mark.parametrize("entry", ["gdn_chunk_fwd", "gdn_chunk_bidir"])
def test_null_pointers_rejected(entry):
    for name in ("q", "k", "v", "g", "beta", "out"):
        assert call(entry, **{name: None}) == _lib.GDN_ERR_INVALID_ARG, name


@pytest.mark.parametrize("entry", ["gdn_chunk_fwd", "gdn_chunk_bidir"])
def test_bad_sizes_and_dims(entry):
    assert call(entry, B=-1) == _lib.GDN_ERR_INVALID_ARG
    assert call(entry, T=-5) == _lib.GDN_ERR_INVALID_ARG
    assert call(entry, H=-2) == _lib.GDN_ERR_INVALID_ARG
    for d in (0, 8, 24, 100, 144, 256):
        assert call(entry, Dk=d) == _lib.GDN_ERR_UNSUPPORTED, d
        assert call(entry, Dv=d) == _lib.GDN_ERR_UNSUPPORTED, d
    assert call(entry, dtype=7) == _lib.GDN_ERR_INVALID_ARG
    for c in (-1, 8, 48, 128):
        assert call(entry, chunk=c) == _lib.GDN_ERR_INVALID_ARG, c


def test_empty_batch_is_a_no_op():
    # nothing to do: returns before touching any pointer or device
    assert call(B=0, q=None, k=None, v=None, g=None, beta=None, out=None) == _lib.GDN_OK
    assert call(H=0, q=None, k=None, v=None, g=None, beta=None, out=None) == _lib.GDN_OK


def test_misaligned_pointers_rejected():
    for name in ("q", "k", "v", "g", "beta", "s_in", "s_out", "out"):
        assert call(**{name: fake(0 if name != "q" else 9) + 8}) == _lib.GDN_ERR_INVALID_ARG, name


def test_overlaps_rejected():
    # out overlapping any input or the state
    for name in ("q", "k", "v", "g", "beta", "s_in", "s_out"):
        assert call(**{name: fake(7) + 1024}) == _lib.GDN_ERR_ALIAS, name
    # state_out overlapping an input
    for name in ("q", "k", "v", "g", "beta"):
        assert call(**{name: fake(6)}) == _lib.GDN_ERR_ALIAS, name
    # state_out partially overlapping state_in (exact equality is allowed)
    assert call(s_out=fake(5) + 4096) == _lib.GDN_ERR_ALIAS


def test_valid_arguments_reach_the_device_checks_without_a_gpu():
    # All host checks pass; with no usable device the call reports a CUDA
    # error instead of crashing (on a machine with a GPU the fake pointers are rejected
    # as not device memory).  Either way nothing is launched.
    st = call()
    assert st in (_lib.GDN_ERR_CUDA, _lib.GDN_ERR_INVALID_ARG)


def test_state_reset_host_checks():
    lib = _lib.load()
    assert lib.gdn_state_reset(None, 0, 4, 16, 16, None) == _lib.GDN_OK
    assert lib.gdn_state_reset(None, 1, 4, 16, 16, None) == _lib.GDN_ERR_INVALID_ARG
    assert lib.gdn_state_reset(fake(1) + 4, 1, 4, 16, 16, None) == _lib.GDN_ERR_INVALID_ARG
    assert lib.gdn_state_reset(fake(1), -1, 4, 16, 16, None) == _lib.GDN_ERR_INVALID_ARG


def test_wait_limit_hook_round_trips():
    lib = _lib.load()
    old = lib.gdn_set_wait_limit(1234)
    assert lib.gdn_set_wait_limit(0) == 1234
    assert lib.gdn_set_wait_limit(old) > 0


@pytest.mark.parametrize("entry", ["gdn_chunk_fwd_logits", "gdn_chunk_bidir_logits"])
def test_logit_entry_points_validate_like_the_others(entry):
    for name in ("q", "k", "v", "g", "beta", "out"):
        assert call(entry, **{name: None}) == _lib.GDN_ERR_INVALID_ARG, name
    assert call(entry, Dk=24) == _lib.GDN_ERR_UNSUPPORTED
    assert call(entry, g=fake(7) + 64) == _lib.GDN_ERR_ALIAS       # logits overlap out
    assert call(entry, beta=fake(3) + 8) == _lib.GDN_ERR_INVALID_ARG  # misaligned
    assert call(entry) in (_lib.GDN_ERR_CUDA, _lib.GDN_ERR_INVALID_ARG)


def test_time_segment_hook_round_trips():
    lib = _lib.load()
    old = lib.gdn_set_time_segments(7)
    assert lib.gdn_set_time_segments(-3) == 7      # negative means automatic
    assert lib.gdn_set_time_segments(old) == 0
    assert lib.gdn_kernel_name(4).decode() == "gdn_segment_prefix_kernel"


def swa(q=fake(0), k=fake(1), v=fake(2), kc=fake(3), vc=fake(4), out=fake(5), B=1, Tc=64, H=2,
        D=64, n_sink=1, window=2, c=3, dtype=_lib.GDN_BF16):
    return _lib.load().gdn_sink_window_attention(q, k, v, kc, vc, out, B, Tc, H, D, n_sink,
                                                 window, c, dtype, None)


def test_sink_window_slots_by_hand():
    lib = _lib.load()
    # one sink chunk, window 2: chunk 0 in the sink slot, then the ring 1, 2, 1, 2, ...
    assert [lib.gdn_sink_window_slot(c, 1, 2) for c in range(7)] == [0, 1, 2, 1, 2, 1, 2]
    # two sink chunks, window 3: ring slots 2, 3, 4
    assert [lib.gdn_sink_window_slot(c, 2, 3) for c in range(8)] == [0, 1, 2, 3, 4, 2, 3, 4]
    assert [lib.gdn_sink_window_slot(c, 0, 1) for c in range(3)] == [0, 0, 0]
    assert lib.gdn_sink_window_slot(-1, 1, 2) == -1
    assert lib.gdn_sink_window_slot(0, -1, 2) == -1
    assert lib.gdn_sink_window_slot(0, 1, 0) == -1


def test_sink_window_host_checks():
    assert swa(window=0) == _lib.GDN_ERR_INVALID_ARG
    assert swa(n_sink=-1) == _lib.GDN_ERR_INVALID_ARG
    assert swa(n_sink=9, window=8) == _lib.GDN_ERR_INVALID_ARG
    assert swa(c=-1) == _lib.GDN_ERR_INVALID_ARG
    assert swa(B=-1) == _lib.GDN_ERR_INVALID_ARG
    assert swa(Tc=-1) == _lib.GDN_ERR_INVALID_ARG
    assert swa(dtype=7) == _lib.GDN_ERR_INVALID_ARG
    assert swa(dtype=_lib.GDN_F32) == _lib.GDN_ERR_UNSUPPORTED
    for d in (0, 8, 100, 144):
        assert swa(D=d) == _lib.GDN_ERR_UNSUPPORTED, d
    assert swa(B=2, H=40000) == _lib.GDN_ERR_UNSUPPORTED
    # nothing to do
    assert swa(Tc=0, q=None, k=None, v=None, kc=None, vc=None, out=None) == _lib.GDN_OK
    assert swa(B=0, q=None) == _lib.GDN_OK
    for name in ("q", "k", "v", "kc", "vc", "out"):
        assert swa(**{name: None}) == _lib.GDN_ERR_INVALID_ARG, name
        assert swa(**{name: fake(0 if name != "q" else 9) + 8}) == _lib.GDN_ERR_INVALID_ARG, name


def test_sink_window_overlaps():
    chunk = 64 * 2 * 64 * 2          # bytes of one chunk (B1 Tc64 H2 D64 bf16)
    for name in ("q", "k", "v", "kc", "vc"):
        assert swa(**{name: fake(5) + 1024}) == _lib.GDN_ERR_ALIAS, name   # out overlaps it
    assert swa(vc=fake(3) + chunk) == _lib.GDN_ERR_ALIAS                  # the caches overlap
    assert swa(q=fake(3) + chunk) == _lib.GDN_ERR_ALIAS                   # q inside k_cache
    slot = _lib.load().gdn_sink_window_slot(3, 1, 2)
    assert swa(k=fake(3) + (slot ^ 3) * chunk) == _lib.GDN_ERR_ALIAS      # k in another slot
    assert swa(k=fake(4) + slot * chunk) == _lib.GDN_ERR_ALIAS            # k inside v_cache
    assert swa(k=fake(3) + slot * chunk, B=2) == _lib.GDN_ERR_ALIAS       # a slot is strided for B > 1
    # k, v exactly this chunk's slots (B = 1): the host checks pass; with no
    # usable device the device checks report it, and nothing is launched
    st = swa(k=fake(3) + slot * chunk, v=fake(4) + slot * chunk)
    assert st in (_lib.GDN_ERR_CUDA, _lib.GDN_ERR_INVALID_ARG)


# ---------------------------------------------------------------- backward
# Gradient outputs at their own fake addresses, apart from the forward's.
def bwd(entry="gdn_chunk_fwd_backward", q=fake(0), k=fake(1), v=fake(2), g=fake(3),
        beta=fake(4), s_in=fake(5), d_out=fake(6), d_s_out=fake(7), dq=fake(8), dk=fake(9),
        dv=fake(10), dg=fake(11), dbeta=fake(12), d_s_in=fake(13), B=1, T=64, H=2, Dk=64,
        Dv=64, dtype=_lib.GDN_BF16):
    lib = _lib.load()
    return getattr(lib, entry)(q, k, v, g, beta, s_in, d_out, d_s_out, dq, dk, dv, dg, dbeta,
                               d_s_in, B, T, H, Dk, Dv, dtype, None)


BWD_ENTRIES = ["gdn_chunk_fwd_backward", "gdn_chunk_bidir_backward"]
GRADS = ("dq", "dk", "dv", "dg", "dbeta", "d_s_in")


@pytest.mark.parametrize("entry", BWD_ENTRIES)
def test_backward_null_pointers_rejected(entry):
    for name in ("q", "k", "v", "g", "beta", "d_out", "dq", "dk", "dv", "dg", "dbeta"):
        assert bwd(entry, **{name: None}) == _lib.GDN_ERR_INVALID_ARG, name


@pytest.mark.parametrize("entry", BWD_ENTRIES)
def test_backward_sizes_dims_and_dtype(entry):
    assert bwd(entry, B=-1) == _lib.GDN_ERR_INVALID_ARG
    assert bwd(entry, T=-3) == _lib.GDN_ERR_INVALID_ARG
    assert bwd(entry, dtype=5) == _lib.GDN_ERR_INVALID_ARG
    for d in (0, 8, 40, 144):
        assert bwd(entry, Dk=d) == _lib.GDN_ERR_UNSUPPORTED, d
        assert bwd(entry, Dv=d) == _lib.GDN_ERR_UNSUPPORTED, d
    # nothing to do: no pointer is looked at
    nulls = {n: None for n in ("q", "k", "v", "g", "beta", "d_out") + GRADS}
    assert bwd(entry, B=0, **nulls) == _lib.GDN_OK
    assert bwd(entry, H=0, **nulls) == _lib.GDN_OK


@pytest.mark.parametrize("entry", BWD_ENTRIES)
def test_backward_misaligned_pointers_rejected(entry):
    for i, name in enumerate(("q", "k", "v", "g", "beta", "s_in", "d_out", "d_s_out") + GRADS):
        assert bwd(entry, **{name: fake(i) + 8}) == _lib.GDN_ERR_INVALID_ARG, name


@pytest.mark.parametrize("entry", BWD_ENTRIES)
def test_backward_gradients_may_not_overlap_anything(entry):
    reads = {"q": 0, "k": 1, "v": 2, "g": 3, "beta": 4, "s_in": 5, "d_out": 6, "d_s_out": 7}
    for grad in GRADS:
        for name, i in reads.items():      # a gradient inside an input
            assert bwd(entry, **{grad: fake(i) + 256}) == _lib.GDN_ERR_ALIAS, (grad, name)
        for other in GRADS:                # two gradients sharing memory
            if other != grad:
                slot = 8 + GRADS.index(other)
                assert bwd(entry, **{grad: fake(slot) + 256}) == _lib.GDN_ERR_ALIAS, (grad, other)
    # d_state_in exactly on state_in is an overlap too (it is written while
    # state_in is still read)
    assert bwd(entry, d_s_in=fake(5)) == _lib.GDN_ERR_ALIAS


@pytest.mark.parametrize("entry", BWD_ENTRIES)
def test_backward_valid_arguments_reach_the_device_checks(entry):
    # optional buffers absent or present: the host checks pass and, with no
    # usable device, the device checks report it; nothing is launched
    for extra in ({}, {"s_in": None}, {"d_s_out": None}, {"d_s_in": None}):
        assert bwd(entry, **extra) in (_lib.GDN_ERR_CUDA, _lib.GDN_ERR_INVALID_ARG), extra


def test_allocation_free_entry_host_checks():
    entry = "gdn_chunk_fwd_noalloc"
    for name in ("q", "k", "v", "g", "beta", "out"):
        assert call(entry, **{name: None}) == _lib.GDN_ERR_INVALID_ARG, name
    assert call(entry, Dk=24) == _lib.GDN_ERR_UNSUPPORTED
    assert call(entry, dtype=_lib.GDN_F32) == _lib.GDN_ERR_UNSUPPORTED   # bf16 only
    assert call(entry, s_out=fake(7) + 64) == _lib.GDN_ERR_ALIAS
    assert call(entry, q=fake(0) + 8) == _lib.GDN_ERR_INVALID_ARG
    assert call(entry, B=0, q=None, k=None, v=None, g=None, beta=None, out=None) == _lib.GDN_OK
    assert call(entry) in (_lib.GDN_ERR_CUDA, _lib.GDN_ERR_INVALID_ARG)


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "gdn.h"

#define CHECK(cond) do { if (!(cond)) { printf("failed: %s\n", #cond); return 1; } } while (0)

int main(void) {
    /* fake, aligned, disjoint addresses: every status below comes from the
       host checks, before any CUDA call */
    char* base = (char*)0x7f0000000000ULL;
    const void* q = base;
    const void* k = base + (1 << 24);
    const void* v = base + (2 << 24);
    const float* g = (const float*)(base + (3 << 24));
    const float* beta = (const float*)(base + (4 << 24));
    void* out = base + (5 << 24);
    CHECK(gdn_version() >= 100);
    CHECK(strcmp(gdn_status_string(GDN_ERR_ALIAS), "GDN_ERR_ALIAS") == 0);
    CHECK(gdn_chunk_fwd(NULL, k, v, g, beta, NULL, NULL, out, 1, 64, 2, 64, 64, GDN_BF16, 0,
                        NULL) == GDN_ERR_INVALID_ARG);
    CHECK(gdn_chunk_bidir(q, k, v, g, beta, NULL, NULL, out, 1, 64, 2, 24, 64, GDN_BF16, 0,
                          NULL) == GDN_ERR_UNSUPPORTED);
    CHECK(gdn_chunk_fwd(q, k, v, g, beta, NULL, NULL, (void*)q, 1, 64, 2, 64, 64, GDN_BF16, 0,
                        NULL) == GDN_ERR_ALIAS);
    CHECK(gdn_chunk_fwd(q, k, v, g, beta, NULL, NULL, out, 0, 64, 2, 64, 64, GDN_BF16, 0,
                        NULL) == GDN_OK);
    CHECK(gdn_sink_window_slot(5, 1, 2) == 1);  /* 1 + (5 - 1) mod 2 */
    printf("ok\n");
    return 0;
}
"""


def test_header_is_plain_c_and_the_library_links_from_c(tmp_path):
    """A C99 program (no C++, no CUDA headers) includes gdn.h, links
    libgdn.so and gets the documented statuses back from the host checks."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(_lib.library_path())
    _lib.load()  # builds the library if it is missing
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    cc = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(src), "-L", lib_dir, "-lgdn",
                         "-Wl,-rpath," + lib_dir, "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
