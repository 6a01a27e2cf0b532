"""The C-ABI library builds, loads without a GPU, exports every declared symbol, and rejects
bad arguments on the host before touching the device (no compute calls here)."""
import ctypes
import os
import re

import pytest

from attention_kl_divergence_02_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(streamkl_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"streamkl_fwd", "streamkl_bwd", "streamkl_bwd_workspace_bytes"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert set(binding.EXPORTS) == set(names)


def test_status_strings_and_version(lib):
    assert binding.version() >= 100
    for code in range(5):
        assert binding.status_string(code)
    assert binding.status_string(99) == "unknown status"


def test_workspace_bytes(lib):
    # the dK accumulator: B * Hkv * whole 128-row key tiles * d fp32 ...
    assert binding.streamkl_bwd_workspace_bytes(1, 32, 32, 16384, 16384, 128) == 32 * 16384 * 128 * 4
    assert binding.streamkl_bwd_workspace_bytes(2, 6, 3, 5, 5, 64) == 2 * 3 * 128 * 64 * 4
    assert binding.streamkl_bwd_workspace_bytes(4, 32, 8, 2048, 32768, 64) == 4 * 8 * 32768 * 64 * 4
    # ... plus, when the query tiles alone would leave SMs idle and their keys are split into
    # ranges, the dQ partial sums: B * Hq * whole 128-row query tiles * d fp32
    assert binding.streamkl_bwd_workspace_bytes(1, 1, 1, 7, 129, 128) == 256 * 128 * 4 + 128 * 128 * 4
    assert binding.streamkl_bwd_workspace_bytes(1, 16, 16, 512, 65536, 128) == (
        16 * 65536 * 128 * 4 + 16 * 512 * 128 * 4)
    assert binding.streamkl_bwd_workspace_bytes(1, 1, 1, 1, 1, 96) == 0
    assert binding.streamkl_bwd_workspace_bytes(0, 1, 1, 1, 1, 64) == 0


FAKE = 1 << 20  # 16-byte aligned, never dereferenced: every call below fails its checks first
HOST_REJECTIONS = (binding.ERR_INVALID_ARG, binding.ERR_UNSUPPORTED)


def fwd_call(**kw):
    assert kw.pop("_expect") in HOST_REJECTIONS   # never reach a launch with fake pointers
    args = dict(q1=FAKE, k1=FAKE, q2=FAKE, k2=FAKE, B=1, Hq=2, Hkv=1, NQ=8, NK=8, d=64,
                scale=0.125, causal=0, kl=FAKE, lse1=FAKE, lse2=FAKE, stream=0)
    args.update(kw)
    return binding.streamkl_fwd(**args)


@pytest.mark.parametrize("kw,want", [
    (dict(q1=None), binding.ERR_INVALID_ARG),
    (dict(kl=None), binding.ERR_INVALID_ARG),
    (dict(B=0), binding.ERR_INVALID_ARG),
    (dict(NQ=-1), binding.ERR_INVALID_ARG),
    (dict(d=96), binding.ERR_UNSUPPORTED),
    (dict(d=256), binding.ERR_UNSUPPORTED),
    (dict(Hq=3, Hkv=2), binding.ERR_UNSUPPORTED),
    (dict(causal=1, NQ=8, NK=9), binding.ERR_UNSUPPORTED),
    (dict(scale=0.0), binding.ERR_UNSUPPORTED),
    (dict(scale=float("nan")), binding.ERR_UNSUPPORTED),
    (dict(scale=-1.0), binding.ERR_UNSUPPORTED),
    (dict(q2=FAKE + 8), binding.ERR_UNSUPPORTED),
    (dict(lse1=FAKE + 4), binding.ERR_UNSUPPORTED),
    (dict(B=1 << 20, Hq=1 << 6, Hkv=1, NQ=1 << 6), binding.ERR_UNSUPPORTED),
])
def test_fwd_rejects_on_host(lib, kw, want):
    assert fwd_call(_expect=want, **kw) == want


WS_NEED = 1 * 1 * 128 * 64 * 4   # B=1, Hkv=1, one 128-row key tile, d=64


def bwd_call(**kw):
    assert kw.pop("_expect") in HOST_REJECTIONS   # never reach a launch with fake pointers
    args = dict(mode=1, q1=FAKE, k1=FAKE, q2=FAKE, k2=FAKE, kl=FAKE, lse1=FAKE, lse2=FAKE,
                dkl=FAKE, B=1, Hq=2, Hkv=1, NQ=8, NK=8, d=64, scale=0.125, causal=0, dq=FAKE,
                dk=FAKE, workspace=FAKE, workspace_bytes=WS_NEED, stream=0)
    args.update(kw)
    return binding.streamkl_bwd(**args)


@pytest.mark.parametrize("kw,want", [
    (dict(mode=0), binding.ERR_INVALID_ARG),
    (dict(mode=3), binding.ERR_INVALID_ARG),
    (dict(dq=None), binding.ERR_INVALID_ARG),
    (dict(workspace=None), binding.ERR_INVALID_ARG),
    (dict(workspace_bytes=WS_NEED - 4), binding.ERR_INVALID_ARG),
    (dict(d=32), binding.ERR_UNSUPPORTED),
    (dict(causal=1, NK=7), binding.ERR_UNSUPPORTED),
    (dict(dk=FAKE + 2), binding.ERR_UNSUPPORTED),
    (dict(workspace=FAKE + 4), binding.ERR_UNSUPPORTED),
])
def test_bwd_rejects_on_host(lib, kw, want):
    assert binding.streamkl_bwd_workspace_bytes(1, 2, 1, 8, 8, 64) == WS_NEED
    assert bwd_call(_expect=want, **kw) == want


def test_splitk_workspace_and_choice(lib):
    # 5 fp32 per row per range actually used; ranges are whole 128-key tiles
    assert binding.streamkl_fwd_splitk_workspace_bytes(2, 4, 1, 5000, 3) == 3 * 5 * 2 * 4 * 1 * 4
    assert binding.streamkl_fwd_splitk_workspace_bytes(1, 2, 1, 300, 64) == 3 * 5 * 2 * 4   # 3 tiles
    assert binding.streamkl_fwd_splitk_workspace_bytes(1, 1, 5, 1, 8) == 0                  # one tile
    assert binding.streamkl_fwd_splitk_workspace_bytes(1, 2, 1, 1000, 1) == 0
    # 40 tiles in 6 ranges of 7 -> 6 used; in 7 ranges of 6 -> 7 used
    assert binding.streamkl_fwd_splitk_workspace_bytes(1, 1, 1, 5000, 6) == 6 * 5 * 4
    assert binding.streamkl_fwd_splitk_workspace_bytes(1, 1, 1, 5000, 7) == 7 * 5 * 4
    assert binding.streamkl_fwd_splitk_workspace_bytes(1, 1, 1, 1, -1) == 0
    # the library's choice: none when the query blocks fill the GPU, several otherwise
    assert binding.streamkl_fwd_splits(1, 32, 16384, 16384) == 1
    assert binding.streamkl_fwd_splits(1, 1, 1, 128) == 1
    # at most 8 query rows (keys as MMA rows, two CTAs per SM): one wave of 2 x 148 CTAs
    assert binding.streamkl_fwd_splits(4, 32, 1, 32768) == 2     # 128 heads -> 256 CTAs
    assert binding.streamkl_fwd_splits(8, 40, 1, 32768) == 1     # 320 heads fill the wave
    s = binding.streamkl_fwd_splits(1, 16, 1, 131072)
    assert s == 18                                               # 16 x 18 = 288 CTAs
    assert binding.streamkl_fwd_splitk_workspace_bytes(1, 16, 1, 131072, 0) == s * 5 * 16 * 4
    # more rows: the query-block kernel's model (waves x (tiles per range + 8))
    s = binding.streamkl_fwd_splits(1, 16, 32, 131072)
    assert 4 <= s <= 64


def splitk_call(**kw):
    assert kw.pop("_expect") in HOST_REJECTIONS   # never reach a launch with fake pointers
    args = dict(q1=FAKE, k1=FAKE, q2=FAKE, k2=FAKE, B=1, Hq=2, Hkv=1, NQ=1, NK=4096, d=128,
                scale=0.088, causal=0, splits=4, kl=FAKE, lse1=FAKE, lse2=FAKE, workspace=FAKE,
                workspace_bytes=4 * 5 * 2 * 4, stream=0)
    args.update(kw)
    return binding.streamkl_fwd_splitk(**args)


@pytest.mark.parametrize("kw,want", [
    (dict(splits=-1), binding.ERR_INVALID_ARG),
    (dict(workspace=None), binding.ERR_INVALID_ARG),
    (dict(workspace_bytes=4 * 5 * 2 * 4 - 4), binding.ERR_INVALID_ARG),
    (dict(workspace=FAKE + 4), binding.ERR_UNSUPPORTED),
    (dict(kl=None), binding.ERR_INVALID_ARG),
    (dict(d=96), binding.ERR_UNSUPPORTED),
    (dict(causal=1), binding.ERR_UNSUPPORTED),
])
def test_splitk_rejects_on_host(lib, kw, want):
    assert splitk_call(_expect=want, **kw) == want


@pytest.mark.parametrize("args, want", [
    ((0, 50_000, 1 << 20, 8), binding.ERR_INVALID_ARG),              # duration below 1 us
    ((20_000_000_000, 50_000, 1 << 20, 8), binding.ERR_INVALID_ARG),  # above 10 s
    ((1_000_000, 500, 1 << 20, 8), binding.ERR_INVALID_ARG),          # interval below 1 us
    ((1_000_000, 2_000_000, 1 << 20, 8), binding.ERR_INVALID_ARG),    # interval above duration
    ((1_000_000, 50_000, 1 << 20, 1), binding.ERR_INVALID_ARG),       # fewer than 2 pairs
    ((1_000_000, 50_000, None, 8), binding.ERR_INVALID_ARG),          # no buffer
    ((1_000_000, 50_000, (1 << 20) + 4, 8), binding.ERR_UNSUPPORTED),  # misaligned buffer
])
def test_clock_probe_rejects_on_host(lib, args, want):
    """The clock probe validates its arguments before launching anything."""
    dur, iv, ptr, pairs = args
    assert lib.streamkl_probe_clock(dur, iv, ptr, pairs, None) == want
    for kind, iters in ((2, 10), (-1, 10), (0, 0)):
        assert lib.streamkl_probe_exp2(kind, iters, None, None) == binding.ERR_INVALID_ARG


def test_header_is_plain_c():
    """The public header compiles as C99 with no CUDA or torch headers."""
    import subprocess
    import tempfile
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "t.c")
        with open(src, "w") as f:
            f.write('#include "streamkl.h"\n'
                    'int (*volatile vfn)(void) = streamkl_version;\n'
                    'int main(void){return vfn != streamkl_version;}\n')
        subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-c", "-I",
                               os.path.join(ROOT, "include"), src, "-o", os.path.join(td, "t.o")])


def test_plain_c_program_links_and_calls_the_library(lib):
    """A C99 program (no CUDA or torch headers) links libstreamkl.so and calls the host-only
    entry points: version, status strings, workspace sizes, the split choice, and argument
    rejection before any device work."""
    import subprocess
    import tempfile
    libdir = os.path.dirname(build.LIB)
    src = r'''
#include <stdio.h>
#include <string.h>
#include "streamkl.h"
int main(void) {
    if (streamkl_version() < 100) return 1;
    if (strcmp(streamkl_status_string(STREAMKL_OK), "ok") != 0) return 2;
    if (streamkl_bwd_workspace_bytes(1, 32, 32, 16384, 16384, 128) != (size_t)32 * 16384 * 128 * 4) return 3;
    if (streamkl_fwd_splits(1, 32, 16384, 16384) != 1) return 4;
    if (streamkl_fwd_splitk_workspace_bytes(1, 1, 1, 5000, 7) != (size_t)7 * 5 * 4) return 5;
    /* null pointers and bad shapes are refused on the host */
    if (streamkl_fwd(NULL, NULL, NULL, NULL, 1, 1, 1, 8, 8, 64, 0.125f, 0, NULL, NULL, NULL, NULL)
        != STREAMKL_ERR_INVALID_ARG) return 6;
    if (streamkl_bwd(3, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 8, 8, 64, 0.125f, 0,
                     NULL, NULL, NULL, 0, NULL) != STREAMKL_ERR_INVALID_ARG) return 7;
    printf("ok\n");
    return 0;
}
'''
    with tempfile.TemporaryDirectory() as td:
        c = os.path.join(td, "t.c")
        exe = os.path.join(td, "t")
        with open(c, "w") as f:
            f.write(src)
        subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), c,
                               "-L", libdir, "-lstreamkl", "-Wl,-rpath," + libdir, "-o", exe])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
        assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
        assert out.stdout.strip() == "ok"
