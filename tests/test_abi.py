"""Host-side checks of the C ABI (no GPU needed): libkvq.so loads, exports every
function include/kvq.h declares, and rejects bad arguments before touching the
device.  Pointers passed here are never dereferenced: every call is expected to
fail validation (or be a no-op) on the host."""
from __future__ import annotations

import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvq(kvq_built):
    return kvq_built


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", text):
            names.add(m.group(1))
    return names


def test_header_declares_the_four_conversions():
    names = _declared_functions()
    for n in ("kvq_fp16_to_fp8", "kvq_fp8_to_fp16", "kvq_fp16_to_q_kv", "kvq_q_to_fp16_kv",
              "kvq_status_string", "kvq_poll_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol(kvq):
    lib = ctypes.CDLL(kvq.LIB_PATH)
    for n in _declared_functions():
        assert hasattr(lib, n), n


def test_status_strings(kvq):
    L = kvq.library()
    for s in range(8):
        assert L.kvq_status_string(s)
    assert L.kvq_status_string(99) == b"unknown status"


def _desc(kvq, d0=2, d1=16, H=2, D=64, stride=0):
    return kvq._Desc(d0, d1, H, D, stride)


FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced


def test_fp8_validation(kvq):
    L = kvq.library()
    d = _desc(kvq)
    by = ctypes.byref
    assert L.kvq_fp16_to_fp8(None, FAKE, by(d), 2, 0, 16, None) == 1
    assert L.kvq_fp16_to_fp8(FAKE, FAKE, None, 2, 0, 16, None) == 1
    assert L.kvq_fp16_to_fp8(FAKE + 8, FAKE, by(d), 2, 0, 16, None) == 5
    assert L.kvq_fp8_to_fp16(FAKE, FAKE, by(d), 3, 0, 16, None) == 4   # batch > dim0
    assert L.kvq_fp8_to_fp16(FAKE, FAKE, by(d), 2, 8, 9, None) == 4    # window past the end
    assert L.kvq_fp8_to_fp16(FAKE, FAKE, by(d), 2, -1, 2, None) == 4   # negative offset
    assert L.kvq_fp8_to_fp16(FAKE, FAKE, by(_desc(kvq, D=12)), 2, 0, 1, None) == 2
    assert L.kvq_fp8_to_fp16(FAKE, FAKE, by(_desc(kvq, H=0)), 2, 0, 1, None) == 2
    # empty windows are accepted and enqueue nothing
    assert L.kvq_fp16_to_fp8(FAKE, FAKE, by(d), 2, 3, 0, None) == 0
    assert L.kvq_fp16_to_fp8(FAKE, FAKE, by(d), 0, 0, 16, None) == 0


def test_q_validation(kvq):
    L = kvq.library()
    d = _desc(kvq)
    by = ctypes.byref
    P = [FAKE] * 6
    assert L.kvq_fp16_to_q_kv(*P, by(d), 2, 0, 16, 0, None, None, 5, None) == 3
    assert L.kvq_fp16_to_q_kv(*P, by(d), 2, 0, 16, 0, None, None, 7, None) == 3
    assert L.kvq_q_to_fp16_kv(*P, by(_desc(kvq, D=48)), 2, 0, 16, 0, None, None, 4, None) == 2
    assert L.kvq_fp16_to_q_kv(*P[:5], None, by(d), 2, 0, 16, 0, None, None, 4, None) == 1
    assert L.kvq_fp16_to_q_kv(*P[:3], FAKE + 4, *P[4:], by(d), 2, 0, 16, 0, None, None, 4, None) == 5
    assert L.kvq_fp16_to_q_kv(*P, by(d), 2, 10, 7, 0, None, None, 4, None) == 4
    # paged: needs seqlens + block_table, page_size == dim1, stride >= 1
    dp = _desc(kvq, d0=10, d1=16, stride=4)
    assert L.kvq_fp16_to_q_kv(*P, by(dp), 2, 0, 16, 16, None, FAKE, 4, None) == 1
    assert L.kvq_fp16_to_q_kv(*P, by(dp), 2, 0, 16, 8, FAKE, FAKE, 4, None) == 4
    assert L.kvq_fp16_to_q_kv(*P, by(_desc(kvq, d0=10, d1=16, stride=0)), 2, 0, 16, 16, FAKE, FAKE, 4,
                              None) == 4
    assert L.kvq_fp16_to_q_kv(*P, by(dp), 2, 0, 16, 16, FAKE + 2, FAKE, 4, None) == 5
    assert L.kvq_fp16_to_q_kv(*P, by(dp), 2, 0, 16, -1, FAKE, FAKE, 4, None) == 4
    # paged offsets may be negative (windows end at cache_seqlens); empty is a no-op
    assert L.kvq_fp16_to_q_kv(*P, by(dp), 2, -5, 0, 16, FAKE, FAKE, 4, None) == 0
    assert L.kvq_q_to_fp16_kv(*P, by(dp), 0, -5, 5, 16, FAKE, FAKE, 6, None) == 0


def test_selfcheck_validation(kvq):
    L = kvq.library()
    assert L.kvq_selfcheck_code_rounding(4, None, None) == 1
    assert L.kvq_selfcheck_code_rounding(5, FAKE, None) == 3
    assert L.kvq_selfcheck_wait_timeout(None, None) == 1
    assert L.kvq_poll_device_error(None, None) == 1


def test_python_binding_checks_dtypes(kvq):
    import torch

    k = torch.zeros(1, 4, 1, 32, dtype=torch.float16)
    with pytest.raises(ValueError):
        kvq.fp16_to_fp8(k, torch.zeros(1, 4, 1, 32, dtype=torch.uint8), 1, 0, 4)  # CPU tensors
    with pytest.raises(ValueError):
        kvq.fp16_to_fp8(k.float(), k, 1, 0, 4)


def test_fp8_kv_validation(kvq):
    L = kvq.library()
    by = ctypes.byref
    d = _desc(kvq)
    P = [FAKE] * 4
    assert L.kvq_fp16_to_fp8_kv(None, *P[1:], by(d), 2, 0, 16, 0, None, None, None) == 1
    assert L.kvq_fp16_to_fp8_kv(*P, by(_desc(kvq, D=12)), 2, 0, 16, 0, None, None, None) == 2
    assert L.kvq_fp16_to_fp8_kv(*P, by(d), 3, 0, 16, 0, None, None, None) == 4
    assert L.kvq_fp8_to_fp16_kv(FAKE + 8, *P[1:], by(d), 2, 0, 16, 0, None, None, None) == 5
    dp = _desc(kvq, d0=10, d1=16, stride=4)
    assert L.kvq_fp16_to_fp8_kv(*P, by(dp), 2, 0, 16, 16, None, FAKE, None) == 1
    assert L.kvq_fp16_to_fp8_kv(*P, by(dp), 2, 0, 16, 8, FAKE, FAKE, None) == 4
    assert L.kvq_fp8_to_fp16_kv(*P, by(dp), 2, -3, 0, 16, FAKE, FAKE, None) == 0   # empty window
    assert L.kvq_set_engine(9) == 4 and L.kvq_get_engine() == 0


def test_decode_attention_validation(kvq):
    L = kvq.library()
    by = ctypes.byref
    d = _desc(kvq, d0=2, d1=16, H=2, D=64)
    P = [FAKE] * 6  # q, k_codes, k_scales, v_codes, v_scales, out
    ws = kvq.attention_workspace_bytes((2, 16, 2, 64), 2, 4)
    assert ws == L.kvq_decode_attention_workspace_size(by(d), 2, 4, 0) > 0
    # one (2 + head_dim)-float entry per (sequence, query head, 128-position chunk slot)
    assert ws == 2 * 4 * 1 * (2 + 64) * 4
    big = _desc(kvq, d0=64, d1=16384, H=8, D=128)
    assert L.kvq_decode_attention_workspace_size(by(big), 64, 32, 0) == 64 * 32 * 128 * 130 * 4
    paged = _desc(kvq, d0=2048, d1=256, H=8, D=128, stride=65)
    assert L.kvq_decode_attention_workspace_size(by(paged), 32, 32, 256) == 32 * 32 * 130 * 130 * 4

    def call(*args, desc=d, bs=2, nh=4, ps=0, lens=FAKE, bt=None, wbits=4, wsp=FAKE, wsb=ws):
        return L.kvq_decode_attention_q(*(args or P), by(desc) if desc else None, bs, nh, ps, lens, bt, wbits,
                                        ctypes.c_float(0.125), wsp, wsb, None)

    assert call(None, *P[1:]) == 1
    assert call(lens=None) == 1
    assert call(wsp=None) == 1                          # workspace needed for a non-empty batch
    assert call(wbits=5) == 3
    assert call(desc=_desc(kvq, D=96)) == 2             # head_dim 64, 128 or 256
    assert call(nh=3) == 2                              # query heads must split over the kv heads
    assert call(nh=18) == 2                             # at most 8 query heads per kv head
    assert call(bs=3) == 4                              # batch > dim0 (contiguous)
    assert call(wsb=ws - 1) == 4                        # workspace too small
    assert call(P[0] + 8, *P[1:]) == 5
    assert call(lens=FAKE + 2) == 5
    dp = _desc(kvq, d0=10, d1=16, H=2, D=64, stride=4)
    assert call(desc=dp, ps=16) == 1                    # paged needs a block table
    assert call(desc=dp, ps=8, bt=FAKE) == 4            # page_size must equal dim1
    assert call(bs=0, wsp=None, wsb=0) == 0             # empty batch enqueues nothing


def test_decode_attention_workspace_size_overflow(kvq):
    """A geometry whose workspace size overflows size_t: the size query returns SIZE_MAX and
    the attention call is rejected before anything is enqueued, whatever workspace it is
    handed (a wrapped size would otherwise admit a small one)."""
    L = kvq.library()
    by = ctypes.byref
    # paged: 65535 sequences x 524280 query heads x (2^31 - 1) chunk slots x 258 floats
    d = _desc(kvq, d0=1, d1=256, H=65535, D=256, stride=(1 << 31) - 1)
    size_max = (1 << (8 * ctypes.sizeof(ctypes.c_size_t))) - 1
    assert L.kvq_decode_attention_workspace_size(by(d), 65535, 8 * 65535, 256) == size_max
    P = [FAKE] * 6
    st = L.kvq_decode_attention_q(*P, by(d), 65535, 8 * 65535, 256, FAKE, FAKE, 4, ctypes.c_float(1.0), FAKE,
                                  1 << 20, None)
    assert st == 4  # KVQ_ERR_RANGE
    assert L.kvq_decode_attention_q_noalloc(*P, by(d), 65535, 8 * 65535, 256, FAKE, FAKE, 4, ctypes.c_float(1.0),
                                            None) == 4


def test_decode_attention_fp8_validation(kvq):
    L = kvq.library()
    by = ctypes.byref
    d = _desc(kvq, d0=2, d1=16, H=2, D=64)
    ws = kvq.attention_workspace_bytes((2, 16, 2, 64), 2, 4)
    P = [FAKE] * 4  # q, k_fp8, v_fp8, out

    def call(*args, desc=d, bs=2, nh=4, ps=0, lens=FAKE, bt=None, wsp=FAKE, wsb=ws):
        return L.kvq_decode_attention_fp8(*(args or P), by(desc) if desc else None, bs, nh, ps, lens, bt,
                                          ctypes.c_float(0.125), wsp, wsb, None)

    assert call(None, *P[1:]) == 1
    assert call(FAKE, None, *P[2:]) == 1
    assert call(lens=None) == 1
    assert call(desc=None) == 1
    assert call(wsp=None) == 1
    assert call(desc=_desc(kvq, D=96)) == 2             # head_dim 64, 128 or 256
    assert call(nh=3) == 2
    assert call(bs=3) == 4
    assert call(wsb=ws - 1) == 4
    assert call(P[0], P[1] + 4, *P[2:]) == 5            # 16-byte alignment
    dp = _desc(kvq, d0=10, d1=16, H=2, D=64, stride=4)
    assert call(desc=dp, ps=16) == 1                    # paged needs a block table
    assert call(desc=dp, ps=8, bt=FAKE) == 4            # page_size must equal dim1
    assert call(bs=0, wsp=None, wsb=0) == 0             # empty batch enqueues nothing


def test_decode_attention_noalloc_validation(kvq):
    L = kvq.library()
    by = ctypes.byref
    P = [FAKE] * 6
    big = _desc(kvq, d0=64, d1=1 << 20, H=8, D=128)
    assert L.kvq_decode_attention_workspace_size(by(big), 64, 64, 0) > kvq.ATTENTION_SCRATCH_BYTES
    assert L.kvq_decode_attention_q_noalloc(*P, None, 2, 4, 0, FAKE, None, 4, ctypes.c_float(1.0), None) == 1
    # beyond the scratch array: rejected on the host, nothing enqueued
    assert L.kvq_decode_attention_q_noalloc(*P, by(big), 64, 64, 0, FAKE, None, 4, ctypes.c_float(1.0), None) == 4


def test_scratch_size_matches_the_header(kvq):
    """The binding's pre-check uses the scratch size include/kvq.h defines: the two must
    not drift apart (the binding would then reject valid calls, or pass calls the
    library refuses)."""
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    m = re.search(r"#define\s+KVQ_ATTENTION_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", text)
    assert m, "KVQ_ATTENTION_SCRATCH_BYTES not found in include/kvq.h"
    assert kvq.ATTENTION_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
    # and the library agrees at the boundary: the largest geometry that fits is accepted by
    # the size check, one entry more is refused (host-side validation only)
    L = kvq.library()
    by = ctypes.byref
    d = _desc(kvq, d0=1, d1=128, H=1, D=126)  # one 128-position chunk, 128 floats per entry
    per_head = L.kvq_decode_attention_workspace_size(by(d), 1, 1, 0)
    assert per_head == 128 * 4
    heads_fit = kvq.ATTENTION_SCRATCH_BYTES // per_head
    assert L.kvq_decode_attention_workspace_size(by(d), 1, heads_fit, 0) <= kvq.ATTENTION_SCRATCH_BYTES
    assert L.kvq_decode_attention_workspace_size(by(d), 1, heads_fit + 1, 0) > kvq.ATTENTION_SCRATCH_BYTES


def test_binding_rejects_dimensions_beyond_int32(kvq):
    """A cache dimension the int32 descriptor cannot hold is refused by the binding
    instead of wrapping into another geometry."""
    with pytest.raises(ValueError, match="int32"):
        kvq._desc(1, (1 << 32) + 5, 8, 128, 0)
    with pytest.raises(ValueError, match="int32"):
        kvq._desc(1, 16, 8, 128, -1)
    d = kvq._desc(2, 16, 2, 64, 0)
    assert (d.dim0, d.dim1, d.kv_heads, d.head_dim, d.block_table_stride) == (2, 16, 2, 64, 0)


def test_binding_rejects_int_arguments_beyond_int32(kvq):
    assert kvq._i32(-5, "offset") == -5
    with pytest.raises(ValueError, match="width"):
        kvq._i32(1 << 32, "width")


def test_header_is_plain_c_and_links(kvq, tmp_path):
    """include/kvq.h compiles as C99 with warnings as errors, and a C program links against
    libkvq.so and calls the host-only entry points (no device work)."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_kvq.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "kvq.h"
int main(void) {
  const long long a[4] = {1, 2, 3, 4}, b[4] = {1, 2, 9, 4};
  kvq_cache_desc d = {2, 16, 2, 64, 0};
  if (kvq_count_match((const int64_t*)a, 4, (const int64_t*)b, 4, 4) != 2) return 1;
  if (kvq_decode_attention_workspace_size(&d, 2, 4, 0) == 0) return 2;
  if (strcmp(kvq_status_string(KVQ_OK), kvq_status_string(KVQ_ERR_NULL)) == 0) return 3;
  if (kvq_fp16_to_fp8(NULL, NULL, &d, 1, 0, 1, NULL) != KVQ_ERR_NULL) return 4;
  puts("ok");
  return 0;
}
''')
    exe = tmp_path / "use_kvq"
    lib = os.path.dirname(kvq.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", lib, "-lkvq", f"-Wl,-rpath,{lib}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)
