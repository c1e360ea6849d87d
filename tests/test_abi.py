"""The C ABI without a GPU: every symbol the header declares is exported, and
host-side argument checks answer before any CUDA call."""

import ctypes
import os
import re

import pytest

from dynamic_block_sparse_variance_b200 import build, prism as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared():
    names = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"^(?:int|const char \*|size_t|void)\s*\*?\s*(prism_\w+)\(", text, re.M)
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return P.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(P.ENTRY_POINTS) <= set(names)


def test_workspace_sizes(lib):
    p = P.make_params(64, 96, 160, 24, 128, 32, 0.9)
    ind, _ = P.prism_workspace_size(p, P.PRISM_WS_INDICATOR)
    sel_min, sel_all = P.prism_workspace_size(p, P.PRISM_WS_SELECT)
    bwd, _ = P.prism_workspace_size(p, P.PRISM_WS_BWD, 10**8)
    cap = 8 * (64 * 96 * 160 // 512)
    assert ind > 0 and sel_min >= cap * cap * 4 and sel_all >= 24 * cap * cap * 4
    assert bwd >= 4 * 10**8
    N = 64 * 96 * 160
    rows = 24 * N
    # head_dim 128: fp16 copies of V and dO, the fp32 dQ accumulator, three padded per-row stats
    assert bwd >= 10**8 * 4 + rows * 128 * (2 * 2 + 4) + 3 * (rows + 128) * 4
    bwd64, _ = P.prism_workspace_size(P.make_params(64, 96, 160, 24, 64, 32, 0.9), P.PRISM_WS_BWD, 10**8)
    assert bwd64 < bwd - rows * 128 * 8 // 2      # the warp-MMA backward has no copies or accumulator
    fwd, _ = P.prism_workspace_size(p, P.PRISM_WS_FWD)
    assert 24 * N * 128 * 2 <= fwd <= 24 * N * 128 * 2 + 4096    # fp16 copy of V, per-head maxima
    p64 = P.make_params(8, 16, 16, 2, 64, 2, 0.9)
    assert P.prism_workspace_size(p64, P.PRISM_WS_FWD)[0] == 0


@pytest.mark.parametrize("bad", [dict(T=7), dict(H=0), dict(head_dim=96), dict(heads=0)])
def test_invalid_params_rejected_on_host(lib, bad):
    kw = dict(T=8, H=16, W=16, heads=2, head_dim=64, top_k=2, top_p=0.9)
    kw.update(bad)
    p = P.make_params(**kw)
    with pytest.raises(P.PrismError) as e:
        P.prism_workspace_size(p, P.PRISM_WS_INDICATOR)
    assert e.value.code == P.PRISM_EINVAL
    rc = lib.prism_zone_indicator(ctypes.byref(p), None, 0, None, None, None, None, None, 0, None)
    assert rc == P.PRISM_EINVAL
    assert lib.prism_last_error()


def test_null_and_misaligned_pointers_rejected(lib):
    p = P.make_params(8, 16, 16, 2, 64, 2, 0.9)
    assert lib.prism_permute(ctypes.byref(p), None, None, None, 0, None, None, None) == P.PRISM_EINVAL
    fake = ctypes.c_void_p(0x1001)
    assert lib.prism_permute(ctypes.byref(p), fake, fake, fake, 0, fake, None, None) == P.PRISM_EINVAL
    assert b"aligned" in lib.prism_last_error()
    bad_p = P.make_params(8, 16, 16, 2, 64, 0, 0.9)
    assert lib.prism_block_select(ctypes.byref(bad_p), fake, fake, fake, fake, fake, 0, fake, fake, 1 << 30,
                                  None) == P.PRISM_EINVAL


@pytest.mark.parametrize("bad", [dict(fixed_shape=-1), dict(fixed_shape=17), dict(sparsity=-0.1),
                                 dict(sparsity=1.5), dict(sparsity=float("nan"))])
def test_variant_params_rejected_on_host(lib, bad):
    kw = dict(T=8, H=16, W=16, heads=2, head_dim=64, top_k=2, top_p=0.9)
    kw.update(bad)
    with pytest.raises(P.PrismError) as e:
        P.prism_workspace_size(P.make_params(**kw), P.PRISM_WS_INDICATOR)
    assert e.value.code == P.PRISM_EINVAL


def test_variant_params_accepted(lib):
    for kw in (dict(fixed_shape=P.PRISM_FIXED_444), dict(fixed_shape=16), dict(sparsity=0.75),
               dict(sparsity=1.0, top_k=0)):
        p = P.make_params(8, 16, 16, 2, 64, kw.pop("top_k", 2), 0.9, **kw)
        assert P.prism_workspace_size(p, P.PRISM_WS_SELECT)[0] > 0
    # dynamic shapes need g and rho; a fixed shape does not read them
    p = P.make_params(8, 16, 16, 2, 64, 2, 0.9)
    assert lib.prism_assign_blocks(ctypes.byref(p), None, None, None, None, None, None, None) == P.PRISM_EINVAL
    assert b"NULL" in lib.prism_last_error()


def test_audio_norms_host_checks(lib):
    fake = ctypes.c_void_p(0x1000)
    assert lib.prism_audio_norms(fake, P.PRISM_BF16, 10, 12, fake, None) == P.PRISM_EINVAL    # C % 8
    assert lib.prism_audio_norms(fake, P.PRISM_F32, 10, 6, fake, None) == P.PRISM_EINVAL      # C % 4
    assert lib.prism_audio_norms(fake, 7, 10, 8, fake, None) == P.PRISM_EINVAL                # dtype
    assert lib.prism_audio_norms(ctypes.c_void_p(0x1008), P.PRISM_BF16, 10, 8, fake, None) == P.PRISM_EINVAL
    assert b"aligned" in lib.prism_last_error()
    assert lib.prism_audio_norms(None, P.PRISM_BF16, 10, 8, fake, None) == P.PRISM_EINVAL
    assert lib.prism_audio_norms(fake, P.PRISM_BF16, -1, 8, fake, None) == P.PRISM_EINVAL
    assert lib.prism_audio_norms(None, P.PRISM_BF16, 0, 8, None, None) == P.PRISM_OK          # empty: no launch


def test_selection_beyond_its_shared_memory_rejected_on_host(lib):
    """A head's score row is sorted in shared memory: 4 bytes per block, 8 blocks
    per zone.  8000 zones (T x H x W = 8 x 800 x 640) need 256 KB, beyond the
    227 KB a CTA can have; the call says so before any launch."""
    p = P.make_params(8, 800, 640, 1, 64, 4, 0.9)
    fake = ctypes.c_void_p(0x1000)
    rc = lib.prism_block_select(ctypes.byref(p), fake, fake, fake, fake, None, 0, fake, fake, 1 << 40, None)
    assert rc == P.PRISM_EINVAL and b"too many blocks" in lib.prism_last_error()


def test_header_is_c99_and_links(lib, tmp_path):
    """include/prism.h is a C header: a C99 program (-pedantic, warnings as errors)
    includes it, links the library and calls the host-only entry points."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "prism.h"
int main(void) {
  prism_params p = {64, 96, 160, 24, 128, 0.5f, 0.25f, 1e-4f, 32, 0.9f, 0.f, PRISM_FIXED_444, 0.75f};
  size_t a = 0, b = 0;
  if (prism_workspace_size(&p, PRISM_WS_SELECT, 0, &a, &b) != PRISM_OK || a == 0 || b < a) return 1;
  p.T = 7;
  if (prism_workspace_size(&p, PRISM_WS_SELECT, 0, &a, &b) != PRISM_EINVAL) return 2;
  if (strstr(prism_last_error(), "multiples of 8") == NULL) return 3;
  if (prism_audio_norms(NULL, PRISM_BF16, 0, 8, NULL, NULL) != PRISM_OK) return 4;
  printf("ok\n");
  return 0;
}
''')
    libdir = os.path.dirname(P.LIB_PATH)
    exe = tmp_path / "abi"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lprism_b200", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)
