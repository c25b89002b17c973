"""The C ABI library builds, loads and exports every entry point of
include/ksa.h; host-side validation rejects bad arguments before touching the
device.  Runs without a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "ksa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ksa_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def ksa():
    from block_top_sparse_ksa_b200 import build
    build.build()
    import block_top_sparse_ksa_b200 as k
    return k


def test_header_declares_the_hot_path():
    names = declared_functions()
    for n in ("ksa_build_block_summaries", "ksa_select_blocks", "ksa_sparse_decode_attn",
              "ksa_unified_select"):
        assert n in names


def test_library_exports_every_declared_symbol(ksa):
    lib = ctypes.CDLL(ksa.library_path)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_wraps_every_entry_point(ksa):
    for n in declared_functions():
        assert hasattr(ksa, n), n


def test_status_strings_and_version(ksa):
    assert ksa.ksa_status_string(0) == "KSA_OK"
    assert ksa.ksa_status_string(2) == "KSA_ERR_UNSUPPORTED"
    assert ksa.ksa_version() >= 100


def _shape(ksa, B=1, Hq=4, Hkv=2, D=128, T=64, bs=16):
    return ksa.Shape(B, Hq, Hkv, D, T, bs)


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first


def test_validation_rejects_bad_shapes(ksa):
    lib = ksa.lib()
    assert lib.ksa_select_blocks(None, FAKE, FAKE, FAKE, 4, FAKE, FAKE, None, 0, None, None) == 1
    for kw, want in [(dict(D=96), 2), (dict(Hq=3, Hkv=2), 1), (dict(bs=8), 2), (dict(B=0), 1)]:
        sh = _shape(ksa, **kw)
        st = lib.ksa_select_blocks(ctypes.byref(sh), FAKE, FAKE, FAKE, 4, FAKE, FAKE, None, 0,
                                   None, None)
        assert st == want, (kw, st, ksa.ksa_last_error())
        assert ksa.ksa_last_error() != ""


def test_validation_rejects_bad_arguments(ksa):
    lib = ksa.lib()
    sh = _shape(ksa)
    # k_blocks < 1
    assert lib.ksa_select_blocks(ctypes.byref(sh), FAKE, FAKE, FAKE, 0, FAKE, FAKE, None, 0,
                                 None, None) == 1
    # NULL output
    assert lib.ksa_select_blocks(ctypes.byref(sh), FAKE, FAKE, FAKE, 4, None, FAKE, None, 0,
                                 None, None) == 1
    # summaries mode out of range
    assert lib.ksa_build_block_summaries(ctypes.byref(sh), FAKE, FAKE, 7, FAKE, None, None) == 1
    # attention: G = 16 unsupported, tokens_per_idx not a power of two, bad dtype
    sh16 = _shape(ksa, Hq=32, Hkv=2)
    assert lib.ksa_sparse_decode_attn(ctypes.byref(sh16), FAKE, FAKE, FAKE, FAKE, None, None, 0,
                                      1, 0, 0.0, 0, FAKE, None, None, 0, None, None) == 2
    assert lib.ksa_sparse_decode_attn(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 3,
                                      0, 0.0, 0, FAKE, None, None, 0, None, None) == 2
    assert lib.ksa_sparse_decode_attn(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, None, None, 0, 1,
                                      0, 0.0, 5, FAKE, None, None, 0, None, None) == 1
    assert lib.ksa_sparse_decode_attn(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, None, None, 0, 1,
                                      0, -1.0, 0, FAKE, None, None, 0, None, None) == 1
    # unified: recent > budget, budget > capacity, missing workspace
    assert lib.ksa_unified_select(ctypes.byref(sh), FAKE, FAKE, FAKE, 8, 16, 17, FAKE, FAKE, FAKE,
                                  1 << 20, None, None) == 1
    assert lib.ksa_unified_select(ctypes.byref(sh), FAKE, FAKE, FAKE, 8, 65, 1, FAKE, FAKE, FAKE,
                                  1 << 20, None, None) == 1
    assert lib.ksa_unified_select(ctypes.byref(sh), FAKE, FAKE, FAKE, 8, 16, 4, FAKE, FAKE, None,
                                  0, None, None) == 3


def test_workspace_sizes(ksa):
    lib = ksa.lib()
    sh = _shape(ksa, B=16, Hq=32, Hkv=8, D=128, T=20000)
    ws = lib.ksa_unified_select_workspace(ctypes.byref(sh), 4000, 4000)
    assert ws >= 16 * 32 * 20000 * 4 + 16 * 20000 * 4
    sh16 = _shape(ksa, B=32, Hq=32, Hkv=8, D=128, T=32768, bs=16)
    assert lib.ksa_select_blocks_workspace(ctypes.byref(sh16), 128) >= 32 * 8 * 2048 * 4 + 32 * 8 * 4
    assert lib.ksa_sparse_decode_attn_workspace(ctypes.byref(sh16), 128, 16) >= 32 * 8 * 4
    bad = _shape(ksa, D=96)
    assert lib.ksa_select_blocks_workspace(ctypes.byref(bad), 8) == 0


def test_missing_workspace_is_rejected(ksa):
    lib = ksa.lib()
    sh = _shape(ksa)
    assert lib.ksa_select_blocks(ctypes.byref(sh), FAKE, FAKE, FAKE, 4, FAKE, FAKE, None, 0, None,
                                 None) == 3
    assert lib.ksa_sparse_decode_attn(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, None, None, 0, 1,
                                      0, 0.0, 0, FAKE, None, None, 0, None, None) == 3


def test_validation_of_the_newer_entry_points(ksa):
    """Storage type, window, per-head top-k, paged caches and list layouts are checked on the
    host before any device work."""
    lib = ksa.lib()
    sh = _shape(ksa)
    BIG = 1 << 30
    # summary storage type out of range
    assert lib.ksa_build_block_summaries_ex(ctypes.byref(sh), FAKE, FAKE, 0, 7, FAKE, None,
                                            None) == 1
    assert lib.ksa_select_blocks_ex(ctypes.byref(sh), FAKE, FAKE, 3, FAKE, 4, FAKE, FAKE, FAKE,
                                    BIG, None, None) == 1
    # fp8 summaries (2) need head_dim 128
    sh64 = _shape(ksa, D=64)
    assert lib.ksa_build_block_summaries_ex(ctypes.byref(sh64), FAKE, FAKE, 0, 2, FAKE, None,
                                            None) == 2
    assert lib.ksa_select_blocks_ex(ctypes.byref(sh64), FAKE, FAKE, 2, FAKE, 4, FAKE, FAKE, FAKE,
                                    BIG, None, None) == 2
    # window: k < 1, NULL output, unsupported block size
    assert lib.ksa_select_window(ctypes.byref(sh), FAKE, 0, FAKE, FAKE, None, None) == 1
    assert lib.ksa_select_window(ctypes.byref(sh), FAKE, 4, None, FAKE, None, None) == 1
    assert lib.ksa_select_window(ctypes.byref(_shape(ksa, bs=8)), FAKE, 4, FAKE, FAKE, None,
                                 None) == 2
    # per-head top-k: k < 1, G > 8, capacity above 65536
    assert lib.ksa_select_tokens_per_head(ctypes.byref(sh), FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE,
                                          BIG, None, None) == 1
    assert lib.ksa_select_tokens_per_head(ctypes.byref(_shape(ksa, Hq=32, Hkv=2)), FAKE, FAKE,
                                          FAKE, 4, FAKE, FAKE, FAKE, BIG, None, None) == 2
    assert lib.ksa_select_tokens_per_head(ctypes.byref(_shape(ksa, T=70000)), FAKE, FAKE, FAKE, 4,
                                          FAKE, FAKE, FAKE, BIG, None, None) == 2
    # paged caches: no pages, capacity != max_blocks * block_size, empty pool
    assert lib.ksa_build_block_summaries_paged(ctypes.byref(sh), FAKE, None, FAKE, 0, 0, FAKE,
                                               None, None) == 1
    bad_cap = ksa.Pages(FAKE, 3, 10)  # 3 * 16 != 64
    assert lib.ksa_build_block_summaries_paged(ctypes.byref(sh), FAKE, ctypes.byref(bad_cap),
                                               FAKE, 0, 0, FAKE, None, None) == 1
    no_pages = ksa.Pages(FAKE, 4, 0)
    assert lib.ksa_build_block_summaries_paged(ctypes.byref(sh), FAKE, ctypes.byref(no_pages),
                                               FAKE, 0, 0, FAKE, None, None) == 1
    assert lib.ksa_decode_select_blocks_paged(ctypes.byref(sh), FAKE, FAKE, ctypes.byref(bad_cap),
                                              FAKE, 0, FAKE, 4, FAKE, FAKE, FAKE, BIG, None,
                                              None) == 1
    # attention list layout out of range
    assert lib.ksa_sparse_decode_attn(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 1,
                                      3, 0.0, 0, FAKE, None, None, 0, None, None) == 1


def test_sizes_past_32_bit_row_indices_are_refused(ksa):
    """K/V row coordinates are 32-bit on the device: caches of 2^31 rows or more, and page
    pools of that size, are refused on the host (KSA_ERR_UNSUPPORTED), never run."""
    lib = ksa.lib()
    big = _shape(ksa, B=1024, Hq=16, Hkv=8, T=1 << 18, bs=16)  # 1024 * 8 * 2^18 = 2^31 rows
    assert lib.ksa_select_blocks(ctypes.byref(big), FAKE, FAKE, FAKE, 4, FAKE, FAKE, FAKE,
                                 1 << 30, None, None) == 2
    assert lib.ksa_sparse_decode_attn(ctypes.byref(big), FAKE, FAKE, FAKE, FAKE, None, None, 0,
                                      1, 0, 0.0, 0, FAKE, None, None, 0, None, None) == 2
    assert lib.ksa_select_blocks_workspace(ctypes.byref(big), 4) == 0
    just_under = _shape(ksa, B=1023, Hq=16, Hkv=8, T=1 << 18, bs=16)
    assert lib.ksa_select_blocks_workspace(ctypes.byref(just_under), 4) > 0
    sh = _shape(ksa, B=1, Hq=4, Hkv=2, D=128, T=64, bs=16)
    pool = ksa.Pages(FAKE, 4, 1 << 26)  # 2^26 pages * 2 kv-heads * 16 rows = 2^31
    assert lib.ksa_sparse_decode_attn_paged(ctypes.byref(sh), FAKE, FAKE, FAKE,
                                            ctypes.byref(pool), FAKE, FAKE, FAKE, 4, 16, 0, 0.0,
                                            0, FAKE, None, FAKE, 1 << 30, None, None) == 2


C_CALLER = r"""
#include <stdio.h>
#include <string.h>
#include "ksa.h"

int main(void) {
  ksa_shape sh;
  ksa_status st;
  memset(&sh, 0, sizeof sh);
  if (ksa_version() < 100) return 1;
  if (strcmp(ksa_status_string(KSA_ERR_UNSUPPORTED), "KSA_ERR_UNSUPPORTED") != 0) return 2;
  /* a NULL shape and an empty batch are refused on the host, with a message */
  st = ksa_select_blocks(NULL, NULL, NULL, NULL, 4, NULL, NULL, NULL, 0, NULL, NULL);
  if (st != KSA_ERR_INVALID_ARG || ksa_last_error()[0] == '\0') return 3;
  sh.batch = 0; sh.num_q_heads = 4; sh.num_kv_heads = 2; sh.head_dim = 128;
  sh.capacity = 64; sh.block_size = 16;
  st = ksa_sparse_decode_attn(&sh, NULL, NULL, NULL, NULL, NULL, NULL, 0, 1, KSA_IDX_PER_KV_HEAD,
                              0.0f, KSA_OUT_F32, NULL, NULL, NULL, 0, NULL, NULL);
  if (st != KSA_ERR_INVALID_ARG) return 4;
  sh.batch = 2;
  if (ksa_select_blocks_workspace(&sh, 4) == 0) return 5;
  printf("ok %d\n", (int)ksa_version());
  return 0;
}
"""


@pytest.mark.parametrize("lang", ["c99", "c++11"])
def test_c_caller_builds_links_and_runs(ksa, tmp_path, lang):
    """A plain C (and C++) program includes include/ksa.h, links libksa.so and makes the
    host-only calls: version, status strings, validation errors, workspace sizes."""
    import shutil
    import subprocess
    src = tmp_path / ("caller.c" if lang == "c99" else "caller.cpp")
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(ksa.library_path)
    cc = "gcc" if lang == "c99" else "g++"
    if shutil.which(cc) is None:
        pytest.skip(f"{cc} not found")
    cmd = [cc, f"-std={lang}", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", libdir, "-l:" + os.path.basename(ksa.library_path), "-Wl,-rpath," + libdir]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.startswith("ok ")


def test_no_fallback_without_the_library_or_a_gpu(tmp_path):
    """The product path has no CPU fallback: CPU tensors are refused before any call, and a
    missing library is an error naming the build step (checked in a fresh interpreter)."""
    import subprocess
    import sys
    code = (
        "import sys, torch\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "import block_top_sparse_ksa_b200 as k\n"
        "q = torch.zeros((1, 4, 128), dtype=torch.bfloat16)\n"
        "K = torch.zeros((1, 2, 64, 128), dtype=torch.bfloat16)\n"
        "L = torch.full((1,), 64, dtype=torch.int32)\n"
        "try:\n"
        "    k.ksa_sparse_decode_attn(q, K, K, L)\n"
        "    sys.exit('CPU tensors were accepted')\n"
        "except TypeError as e:\n"
        "    assert 'CUDA tensor' in str(e), e\n"
        f"k.library_path = {str(tmp_path / 'libksa_absent.so')!r}\n"
        "k._LIB = None\n"
        "try:\n"
        "    k.lib()\n"
        "    sys.exit('a missing library loaded')\n"
        "except RuntimeError as e:\n"
        "    assert 'missing' in str(e) and 'build' in str(e), e\n"
        "print('ok')\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip().endswith("ok")


def test_validation_of_random_head_selection(ksa):
    """The host array of heads is checked row by row before any launch."""
    lib = ksa.lib()
    sh = _shape(ksa, B=3, Hq=8, Hkv=2)
    good = (ctypes.c_int32 * 3)(0, 7, 3)
    bad = (ctypes.c_int32 * 3)(0, 8, 3)  # head 8 of 8
    neg = (ctypes.c_int32 * 3)(-1, 0, 0)
    BIG = 1 << 30
    call = lambda heads, k, ws, n: lib.ksa_select_tokens_one_head(
        ctypes.byref(sh), FAKE, FAKE, FAKE, heads, k, FAKE, FAKE, ws, n, None, None)
    assert call(None, 4, FAKE, BIG) == 1
    assert call(bad, 4, FAKE, BIG) == 1 and "head_of_row[1]" in ksa.ksa_last_error()
    assert call(neg, 4, FAKE, BIG) == 1
    assert call(good, 0, FAKE, BIG) == 1
    assert call(good, 4, None, 0) == 3
    per_head = lib.ksa_select_tokens_per_head_workspace(ctypes.byref(sh), 4)
    one_head = lib.ksa_select_tokens_one_head_workspace(ctypes.byref(sh), 4)
    assert one_head >= per_head + 3 * 8 * 4 * 4 + 3 * 8 * 4 + 3 * 4  # lists, counts, heads
    assert call(good, 4, FAKE, one_head - 1) == 3


def test_every_entry_point_refuses_a_null_shape(ksa):
    """Driven by the binding's signature table: each call that takes a shape first returns
    KSA_ERR_INVALID_ARG (status calls) or 0 bytes (workspace queries) for a NULL shape, with
    every other pointer NULL and every number 0 -- validation first, nothing dereferenced."""
    lib = ksa.lib()
    checked = 0
    for name, (res, args) in ksa._SIGS.items():
        if not args or args[0] is not ctypes.POINTER(ksa.Shape):
            continue
        rest = []
        for t in args[1:]:
            if t in (ctypes.c_float, ctypes.c_double):
                rest.append(0.0)
            elif t in (ctypes.c_int32, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint32):
                rest.append(0)
            else:
                rest.append(None)
        got = getattr(lib, name)(None, *rest)
        want = 0 if res is ctypes.c_size_t else 1
        assert got == want, (name, got)
        checked += 1
    assert checked >= 20


def test_device_status_read_back_validation(ksa):
    lib = ksa.lib()
    flags = ctypes.c_uint32(7)
    assert lib.ksa_get_device_status(None, None, 0, ctypes.byref(flags)) == 1
    assert lib.ksa_get_device_status(FAKE, None, 0, None) == 1
    assert flags.value == 7  # untouched on a refused call


# The one kernel allowed a spill: the token-list attention at head_dim 128 runs two producer
# warps, so three CTAs of six warps hold at most 96 registers a thread (five warps of one
# sub-partition share its 16K registers), and it spills a few words; measured against the
# one-producer form without spills it is faster (65.5 -> 59.9 us per LessIsMore layer).
SPILL_ALLOWED = {"sparse_decode_attn_kernelILi128ELi2E": 64}  # kernel -> max bytes


def test_no_kernel_spills_registers(ksa):
    """The last build's ptxas report: every kernel fits its registers (the selection and pick
    kernels keep whole rows of keys in registers; a spill would send them to local memory),
    but for the listed one, within its bound."""
    from block_top_sparse_ksa_b200 import build
    if not os.path.exists(build.REPORT):
        build.build(force=True)
    text = open(build.REPORT).read()
    blocks = re.split(r"Compiling entry function '", text)[1:]
    assert len(blocks) >= 30
    for blk in blocks:
        name = blk.split("'", 1)[0]
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", blk)
        assert m, name
        allowed = max([v for k, v in SPILL_ALLOWED.items() if k in name], default=0)
        assert int(m.group(1)) <= allowed and int(m.group(2)) <= allowed, (name, m.groups())


def test_validation_of_the_decode_step_and_append(ksa):
    """ksa_decode_step checks the arguments of both calls it stands for, then its own
    workspace; ksa_append_kv checks pointers and alignment.  Nothing reaches the device."""
    lib = ksa.lib()
    sh = _shape(ksa, B=2, Hq=8, Hkv=2, D=128, T=256, bs=16)
    args = lambda **kw: [kw.get("q", FAKE), kw.get("K", FAKE), FAKE, FAKE, 0, FAKE,
                         kw.get("k", 8), FAKE, FAKE, kw.get("scale", 0.0), 0, FAKE, None,
                         kw.get("ws", None), kw.get("ws_bytes", 0), None, None]
    assert lib.ksa_decode_step(None, *args()) == 1
    assert lib.ksa_decode_step(ctypes.byref(sh), *args(K=None)) == 1
    assert lib.ksa_decode_step(ctypes.byref(sh), *args(k=0)) == 1
    assert lib.ksa_decode_step(ctypes.byref(sh), *args(scale=-1.0)) == 1
    assert lib.ksa_decode_step(ctypes.byref(sh), *args()) == 3  # no workspace
    need = lib.ksa_decode_step_workspace(ctypes.byref(sh), 8)
    assert need >= (lib.ksa_select_blocks_workspace(ctypes.byref(sh), 8) +
                    lib.ksa_sparse_decode_attn_workspace(ctypes.byref(sh), 8, 16))
    assert lib.ksa_decode_step(ctypes.byref(sh), *args(ws=FAKE, ws_bytes=need - 1)) == 3
    bad = _shape(ksa, B=2, Hq=8, Hkv=2, D=128, T=256, bs=8)
    assert lib.ksa_decode_step(ctypes.byref(bad), *args()) == 2
    assert lib.ksa_append_kv(ctypes.byref(sh), FAKE, None, FAKE, FAKE, FAKE, None, None) == 1
    odd = ctypes.c_void_p(0x1008)  # 8-byte aligned only
    assert lib.ksa_append_kv(ctypes.byref(sh), odd, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert "aligned" in ksa.ksa_last_error()
