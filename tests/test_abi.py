"""The C-ABI library loads, exports every entry point include/ring_attn.h
declares, and rejects bad arguments on the host before touching CUDA (these
calls never reach a kernel, so they run without a GPU)."""

import ctypes
import math
import os
import re

import pytest

import blockwise_exact_attention_attn_b200 as ra

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "ring_attn.h")

# an aligned, never-dereferenced fake device address
FAKE = 0x10000


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ring_attn_\w+)\s*\(", text)))


def test_header_and_export_list_agree():
    assert declared_functions() == sorted(ra.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in enumerate(["RA_OK", "RA_ERR_INVALID", "RA_ERR_UNSUPPORTED", "RA_ERR_CUDA",
                                 "RA_ERR_TIMEOUT"]):
        assert lib.ring_attn_status_string(code).decode() == name
    assert lib.ring_attn_status_string(99).decode() == "RA_ERR_UNKNOWN"


def test_withhold_hook_toggles_on_the_host(lib):
    # host-only setting: returns the previous value, never touches CUDA
    assert lib.ring_attn_test_withhold_q(1) == 0
    assert lib.ring_attn_test_withhold_q(7) == 1
    assert lib.ring_attn_test_withhold_q(0) == 1
    assert lib.ring_attn_test_withhold_q(0) == 0
    assert ra.ring_attn_test_withhold_q(False) is False


def fwd(lib, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, batch=1, heads=2, seqlen=256, d_head=128,
             n=4, layout=0, causal=1, scale=0.1, passes=4, cu=None, dtype=1, stream=None)
    a.update(over)
    return lib.ring_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["batch"], a["heads"],
                             a["seqlen"], a["d_head"], a["n"], a["layout"], a["causal"],
                             a["scale"], a["passes"], a["cu"], a["dtype"], a["stream"])


@pytest.mark.parametrize("over", [
    dict(q=None), dict(k=None), dict(v=None), dict(out=None), dict(lse=None),
    dict(q=FAKE + 4), dict(out=FAKE + 8), dict(lse=FAKE + 2),
    dict(batch=0), dict(heads=0), dict(seqlen=0), dict(n=0), dict(passes=0),
    dict(seqlen=250),                    # dense seqlen not a multiple of N
    dict(d_head=48), dict(d_head=0), dict(layout=2), dict(causal=2), dict(dtype=5),
    dict(scale=math.inf), dict(scale=math.nan), dict(cu=FAKE + 2),
])
def test_fwd_rejects_invalid_arguments(lib, over):
    assert fwd(lib, **over) == ra.RA_ERR_INVALID


@pytest.mark.parametrize("over", [
    dict(batch=2, seqlen=1 << 30),       # batch * seqlen = 2^31 rows: past 32-bit row indices
    dict(batch=1 << 16, heads=1 << 15, seqlen=4),   # batch * heads = 2^31
])
def test_fwd_refuses_sizes_past_32_bit_indices(lib, over):
    # maximum sizes: refused on the host before any CUDA call
    assert fwd(lib, **over) == ra.RA_ERR_UNSUPPORTED


def test_merge_refuses_rows_past_32_bit_indices(lib):
    # batch * seqlen * heads = 2^31 rows
    assert lib.ring_attn_merge(FAKE, FAKE, FAKE, FAKE, 2, 1 << 10, 1 << 20, 128, 0,
                               None) == ra.RA_ERR_UNSUPPORTED
    assert lib.ring_attn_merge(FAKE, FAKE, FAKE, FAKE, 1, 1 << 11, 1 << 20, 128, 0,
                               None) == ra.RA_ERR_UNSUPPORTED


def test_qkvpacked_and_simt_reject_invalid_arguments(lib):
    st = lib.ring_attn_qkvpacked_fwd(None, FAKE, FAKE, 1, 2, 256, 128, 4, 0, 1, 0.1, 4, None, 1,
                                     None)
    assert st == ra.RA_ERR_INVALID
    st = lib.ring_attn_fwd_simt(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 256, 100, 4, 0, 1, 0.1, 4,
                                None, 0, None)
    assert st == ra.RA_ERR_INVALID


@pytest.mark.parametrize("heads,heads_kv", [(4, 3), (4, 0), (4, -2), (2, 4)])
def test_gqa_rejects_heads_that_do_not_group(lib, heads, heads_kv):
    st = lib.ring_attn_gqa_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, heads, heads_kv, 256, 128, 4, 0,
                               1, 0.1, 4, None, 1, None)
    assert st == ra.RA_ERR_INVALID


def test_gqa_shares_the_forward_validation(lib):
    # the same checks as ring_attn_fwd run first (null pointer, bad seqlen)
    assert lib.ring_attn_gqa_fwd(None, FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 256, 128, 4, 0, 1, 0.1,
                                 4, None, 1, None) == ra.RA_ERR_INVALID
    assert lib.ring_attn_gqa_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 250, 128, 4, 0, 1, 0.1,
                                 4, None, 1, None) == ra.RA_ERR_INVALID


@pytest.mark.parametrize("over,want", [
    (dict(q_block=4), "invalid"), (dict(kv_block=-1), "invalid"), (dict(acc=2), "invalid"),
    (dict(seqlen=960), "unsupported"),       # blocks of 240 rows: not whole tiles
    (dict(dtype=0), "unsupported"),          # fp32 has no tensor-core step
    (dict(scale=0.0), "unsupported"),
    (dict(out=None), "invalid"), (dict(seqlen=1002), "invalid"),   # not a multiple of N
])
def test_step_validation(lib, over, want):
    a = dict(q=FAKE, out=FAKE, batch=1, heads=2, seqlen=1024, d=128, n=4, layout=0, causal=1,
             scale=0.1, q_block=1, kv_block=0, acc=1, dtype=1)
    a.update(over)
    st = lib.ring_attn_fwd_step(a["q"], FAKE, FAKE, a["out"], FAKE, a["batch"], a["heads"],
                                a["seqlen"], a["d"], a["n"], a["layout"], a["causal"],
                                a["scale"], a["q_block"], a["kv_block"], a["acc"], a["dtype"],
                                None)
    assert st == {"invalid": ra.RA_ERR_INVALID, "unsupported": ra.RA_ERR_UNSUPPORTED}[want]


@pytest.mark.parametrize("args", [
    (None, FAKE, FAKE, FAKE, 1, 1, 8, 128, 0),         # null
    (FAKE, FAKE + 4, FAKE, FAKE, 1, 1, 8, 128, 0),     # misaligned lse
    (FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 3, 0),           # row not whole 16-byte chunks
    (FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 256, 0),         # fp32 row of 64 chunks (> 32)
    (FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 24, 1),          # 3 chunks: not a power of two
    (FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 128, 0),         # empty batch
    (FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 128, 7),         # dtype
])
def test_merge_rejects_invalid_arguments(lib, args):
    assert lib.ring_attn_merge(*args, None) == ra.RA_ERR_INVALID


def test_binding_refuses_host_tensors():
    import torch
    x = torch.zeros(1, 128, 1, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 128)
    with pytest.raises(ValueError):
        ra.ring_attn_fwd(x, x, x, x, lse, 1, 1, 128, 64, 1)


C_CONSUMER = r"""
#include <stdio.h>
#include <string.h>
#include "ring_attn.h"
int main(void) {
  int32_t qt[8], kt[8];
  int8_t cl[8];
  int64_t n;
  if (strcmp(ring_attn_status_string(RA_ERR_TIMEOUT), "RA_ERR_TIMEOUT") != 0) return 1;
  if (ring_attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 128, 128, 1, RA_LAYOUT_CONTIGUOUS, 0,
                    0.1f, 1, NULL, RA_BF16, NULL) != RA_ERR_INVALID)
    return 2;
  /* causal, 256 rows, 128-row tiles: (0,0) partial, (1,0) full, (1,1) partial */
  n = ring_attn_schedule(256, 2, RA_LAYOUT_CONTIGUOUS, 1, 2, 128, 128, 1, qt, kt, cl, 8);
  if (n != 3 || cl[0] != 2) return 3;
  if (ring_attn_test_withhold_q(0) != 0) return 4;
  printf("ok\n");
  return 0;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    # the boundary from C itself: strict C99 against the header, linked to the
    # library, host-only calls (no CUDA call is made)
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "consumer.c"
    src.write_text(C_CONSUMER)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(ra.library_path())
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.dirname(HEADER), str(src), "-L", libdir, "-lringattn",
                    "-Wl,-rpath," + libdir, "-o", str(exe)], check=True, capture_output=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_host_workspace_size_is_two_slots_of_one_chunk(lib):
    # one slot: q, k, v, out of one chunk ([B, S, hc, D] each, 256-byte
    # rounded) and its lse ([B, hc, S] fp32); two slots unless one chunk
    def slot(B, S, hc, D, es):
        up = lambda x: (x + 255) // 256 * 256
        return 4 * up(B * S * hc * D * es) + up(B * hc * S * 4)
    assert lib.ring_attn_fwd_host_workspace(2, 8, 1024, 128, ra.BF16, 0) == 2 * slot(2, 1024, 1, 128, 2)
    assert lib.ring_attn_fwd_host_workspace(1, 16, 512, 64, ra.F16, 0) == 2 * slot(1, 512, 2, 64, 2)
    assert lib.ring_attn_fwd_host_workspace(1, 5, 100, 16, ra.F32, 3) == 2 * slot(1, 100, 3, 16, 4)
    assert lib.ring_attn_fwd_host_workspace(1, 2, 256, 128, ra.BF16, 8) == slot(1, 256, 2, 128, 2)
    for bad in [(0, 1, 1, 16, ra.F32, 0), (1, 1, 1, 16, 9, 0), (1, 0, 1, 16, ra.F32, 0)]:
        assert lib.ring_attn_fwd_host_workspace(*bad) == 0


def test_host_call_rejects_invalid_arguments_before_cuda(lib):
    def call(**over):
        a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, batch=1, heads=2, seqlen=256,
                 d_head=128, n=4, layout=0, causal=1, scale=0.1, passes=4, dtype=1, hc=0,
                 ws=FAKE * 16, nbytes=1 << 30, stream=None)
        a.update(over)
        return lib.ring_attn_fwd_host(a["q"], a["k"], a["v"], a["out"], a["lse"], a["batch"],
                                      a["heads"], a["seqlen"], a["d_head"], a["n"], a["layout"],
                                      a["causal"], a["scale"], a["passes"], a["dtype"], a["hc"],
                                      a["ws"], a["nbytes"], a["stream"])
    for over in [dict(q=None), dict(ws=None), dict(ws=FAKE + 16), dict(seqlen=250),
                 dict(hc=-1), dict(nbytes=0), dict(d_head=48)]:
        assert call(**over) == ra.RA_ERR_INVALID, over


def test_noalloc_status_is_exported_with_a_stream_argument(lib):
    assert lib.ring_attn_noalloc_status.argtypes == [ctypes.c_void_p]


def test_schedule_dump_hook_validates_on_the_host(lib):
    assert lib.ring_attn_test_dump_schedule(None, 5) == ra.RA_ERR_INVALID
    assert lib.ring_attn_test_dump_schedule(FAKE, -1) == ra.RA_ERR_INVALID
    assert lib.ring_attn_test_dump_schedule(None, 0) == ra.RA_OK   # off
