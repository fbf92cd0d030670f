"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/tp.h declares, and rejects bad arguments with the
documented status before touching the device."""
import ctypes
import os
import re

import pytest

import tensor_transformer_layers_b200 as tp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tp.h")

A = 1 << 20  # a fake, 256-byte aligned "device address" (never dereferenced: checks fail first)


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tp_[a-z0-9_]+)\s*\(", text)))


def test_library_builds_and_loads():
    assert os.path.exists(tp.LIB_PATH), "libtp.so missing; run python -m tensor_transformer_layers_b200.build"
    assert tp.tp_abi_version() == 1


def test_every_declared_symbol_is_exported():
    names = header_functions()
    assert len(names) >= 20
    lib = ctypes.CDLL(tp.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert missing == []
    assert set(names) == set(tp.SIGNATURES), "binding and header disagree"


def test_status_strings():
    for code in range(len(tp.STATUS)):
        assert tp.tp_status_string(code) not in ("", "unknown status")
    assert tp.tp_status_string(99) == "unknown status"


def test_workspace_sizes():
    up = lambda n: (n + 255) // 256 * 256  # noqa: E731
    M, D, F, T = 4608, 3072, 12288, 4
    assert tp.tp_mlp_workspace_bytes(M, D, F, T) == up(F * D * 2) + up(F * 2) + up(D * F * 2) + up(M * F * 2)
    assert tp.tp_mlp_run_workspace_bytes(M, D, F, T) == up(M * F * 2)
    assert tp.tp_attn_workspace_bytes(M, D, 24, T) == up(3 * D * D * 2) + up(D * D * 2) + up(M * 3 * D * 2) + up(M * D * 2)
    assert tp.tp_attn_run_workspace_bytes(M, D, 24, T) == up(M * 3 * D * 2) + up(M * D * 2)
    # invalid shapes report 0
    assert tp.tp_swiglu_workspace_bytes(M, D, F, T) == (up(2 * F * D * 2) + up(2 * F * 2) + up(D * F * 2)
                                                        + up(M * F * 2))
    assert tp.tp_swiglu_workspace_bytes(M, D, F, 5) == 0
    assert tp.tp_mlp_workspace_bytes(M, D, F, 5) == 0
    assert tp.tp_attn_workspace_bytes(M, D, 24, 5) == 0
    assert tp.tp_attn_workspace_bytes(M, 3000, 24, 4) == 0


S = {v: k for k, v in tp.STATUS.items()}


@pytest.mark.parametrize("args,want", [
    ((0, 8, 8, tp.TP_COLWISE, 2, 0, A), "TP_ERR_NULL"),
    ((A, 8, 8, 7, 2, 0, A), "TP_ERR_BAD_STYLE"),
    ((A, 8, 8, tp.TP_COLWISE, 0, 0, A), "TP_ERR_BAD_DEGREE"),
    ((A, 8, 8, tp.TP_COLWISE, 2, 2, A), "TP_ERR_BAD_RANK"),
    ((A, 8, 8, tp.TP_COLWISE, 2, -1, A), "TP_ERR_BAD_RANK"),
    ((A, 0, 8, tp.TP_COLWISE, 1, 0, A), "TP_ERR_BAD_SHAPE"),
    ((A, 9, 8, tp.TP_COLWISE, 2, 0, A), "TP_ERR_INDIVISIBLE"),
    ((A, 8, 24, tp.TP_ROWWISE, 5, 0, A), "TP_ERR_INDIVISIBLE"),
    ((A + 2, 8, 8, tp.TP_COLWISE, 2, 0, A), "TP_ERR_ALIGNMENT"),
    ((A, 8, 12, tp.TP_COLWISE, 2, 0, A), "TP_ERR_ALIGNMENT"),
    ((A, 8, 24, tp.TP_ROWWISE, 2, 0, A), "TP_ERR_ALIGNMENT"),  # 12-element shard rows
])
def test_shard_weight_checks(args, want):
    assert tp.tp_shard_weight(*args, stream=0) == S[want]


def test_qkv_and_bias_checks():
    assert tp.tp_shard_qkv_heads(A, 384, 3, 2, 0, A, stream=0) == S["TP_ERR_HEADS_INDIVISIBLE"]
    assert tp.tp_shard_qkv_heads(A, 300, 3, 1, 0, A, stream=0) == S["TP_ERR_BAD_SHAPE"]
    assert tp.tp_shard_qkv_heads(A, 384, 3, 3, 3, A, stream=0) == S["TP_ERR_BAD_RANK"]
    assert tp.tp_shard_bias(A, 100, 3, 0, A, stream=0) == S["TP_ERR_INDIVISIBLE"]
    assert tp.tp_shard_bias(A, 24, 2, 0, A, stream=0) == S["TP_ERR_ALIGNMENT"]


def test_layer_checks():
    ws = 1 << 30
    # MLP pair
    assert tp.tp_mlp_pair(A, 64, 128, 512, A, A, A, A, 3, A, A, ws, stream=0) == S["TP_ERR_INDIVISIBLE"]
    assert tp.tp_mlp_pair(A, 64, 128, 512, A, A, A, A, 0, A, A, ws, stream=0) == S["TP_ERR_BAD_DEGREE"]
    assert tp.tp_mlp_pair(A, 64, 128, 520, A, A, A, A, 4, A, A, ws, stream=0) == S["TP_ERR_ALIGNMENT"]
    assert tp.tp_mlp_pair(A, -1, 128, 512, A, A, A, A, 2, A, A, ws, stream=0) == S["TP_ERR_BAD_SHAPE"]
    assert tp.tp_mlp_pair(None, 64, 128, 512, A, A, A, A, 2, A, A, ws, stream=0) == S["TP_ERR_NULL"]
    assert tp.tp_mlp_pair(A, 64, 128, 512, A, A, A, A, 2, A, A, 100, stream=0) == S["TP_ERR_WORKSPACE"]
    assert tp.tp_mlp_pair(A, 64, 128, 512, A, A, A, A, 2, A, A + 16, ws, stream=0) == S["TP_ERR_WORKSPACE"]
    assert tp.tp_mlp_pair(A, 64, 128, 512, A, A + 8, A, A, 2, A, A, ws, stream=0) == S["TP_ERR_ALIGNMENT"]
    # an empty input is valid and does nothing (no device access)
    assert tp.tp_mlp_pair(A, 0, 128, 512, A, A, A, A, 2, A, None, 0, stream=0) == 0
    # attention block: the degree must divide the head count, D must be heads*128
    assert tp.tp_attn_block(A, 64, 768, A, A, 6, 4, A, A, ws, stream=0) == S["TP_ERR_HEADS_INDIVISIBLE"]
    assert tp.tp_attn_block(A, 64, 700, A, A, 6, 2, A, A, ws, stream=0) == S["TP_ERR_BAD_SHAPE"]
    assert tp.tp_attn_block(A, 64, 768, A, A, 6, 2, A, A, 10, stream=0) == S["TP_ERR_WORKSPACE"]
    assert tp.tp_attn_block(A, 0, 768, A, A, 6, 2, A, None, 0, stream=0) == 0
    # step-level calls
    assert tp.tp_colwise_linear(A, 64, 100, A, None, 64, 2, 1, 0, A, stream=0) == S["TP_ERR_ALIGNMENT"]
    assert tp.tp_colwise_linear(A, 64, 128, A, None, 64, 2, 1, 7, A, stream=0) == S["TP_ERR_BAD_STYLE"]
    assert tp.tp_rowwise_linear_sum(A, 64, 64, A, 100, None, 2, A, stream=0) == S["TP_ERR_ALIGNMENT"]
    assert tp.tp_sdpa_shards(A, 64, 6, 4, A, stream=0) == S["TP_ERR_HEADS_INDIVISIBLE"]
    assert tp.tp_reduce_partials(A, 64, 100, 2, None, A, stream=0) == S["TP_ERR_ALIGNMENT"]
    assert tp.tp_reduce_partials(A, 64, 64, 0, None, A, stream=0) == S["TP_ERR_BAD_DEGREE"]
    # handles
    assert tp.tp_mlp_run(None, A, 64, A, A, ws, stream=0) == S["TP_ERR_BAD_HANDLE"]
    assert tp.tp_attn_run(None, A, 64, A, A, ws, stream=0) == S["TP_ERR_BAD_HANDLE"]
    st, h = tp.tp_mlp_prepare(A, A, A, A, 128, 512, 3, stream=0)
    assert st == S["TP_ERR_INDIVISIBLE"] and not h
    st, h = tp.tp_attn_prepare(A, A, 768, 6, 4, stream=0)
    assert st == S["TP_ERR_HEADS_INDIVISIBLE"] and not h
    tp.tp_destroy(None)


@pytest.mark.parametrize("args,want", [
    # (W, rows, cols, style, blocks, T, rank, out)
    ((0, 36, 8, tp.TP_COLWISE, [1, 1, 1, 3, 3], 2, 0, A), "TP_ERR_NULL"),
    ((A, 36, 8, tp.TP_COLWISE, None, 2, 0, A), "TP_ERR_NULL"),
    ((A, 36, 8, tp.TP_ROWWISE_SPLIT_INPUT, [1, 1], 2, 0, A), "TP_ERR_BAD_STYLE"),
    ((A, 36, 8, tp.TP_COLWISE, [1, 1, 1, 3, 3], 0, 0, A), "TP_ERR_BAD_DEGREE"),
    ((A, 0, 8, tp.TP_COLWISE, [1], 1, 0, A), "TP_ERR_BAD_SHAPE"),
    ((A, 36, 8, tp.TP_COLWISE, [], 2, 0, A), "TP_ERR_BAD_BLOCKS"),
    ((A, 36, 8, tp.TP_COLWISE, [1, 0, 1], 2, 0, A), "TP_ERR_BAD_BLOCKS"),
    ((A, 36, 8, tp.TP_COLWISE, [1, -1, 2], 2, 0, A), "TP_ERR_BAD_BLOCKS"),
    ((A, 36, 8, tp.TP_COLWISE, [1, 1, 3], 2, 0, A), "TP_ERR_BAD_BLOCKS"),      # sum 5 does not divide 36
    ((A, 36, 8, tp.TP_COLWISE, [1] * 65, 1, 0, A), "TP_ERR_BAD_BLOCKS"),       # more than 64 blocks
    ((A, 18, 8, tp.TP_COLWISE, [1, 1, 1, 3, 3], 3, 0, A), "TP_ERR_INDIVISIBLE"),  # blocks 2,2,2,6,6 by 3
    ((A, 12, 8, tp.TP_COLWISE, [5, 1], 4, 0, A), "TP_ERR_INDIVISIBLE"),      # 12 % 4 == 0, 10 % 4 != 0
    ((A, 36, 12, tp.TP_COLWISE, [1, 1, 1, 3, 3], 2, 0, A), "TP_ERR_ALIGNMENT"),
    ((A, 8, 48, tp.TP_ROWWISE, [1, 5], 2, 0, A), "TP_ERR_ALIGNMENT"),        # per-shard widths 4 and 20
    ((A, 36, 8, tp.TP_COLWISE, [1, 1, 1, 3, 3], 2, 2, A), "TP_ERR_BAD_RANK"),
])
def test_shard_packed_checks(args, want):
    W, rows, cols, style, blocks, T, rank, out = args
    assert tp.tp_shard_packed(W, rows, cols, style, blocks, T, rank, out, stream=0) == S[want]
    if want != "TP_ERR_BAD_RANK":
        assert tp.tp_shard_packed_all(W, rows, cols, style, blocks, T, out, stream=0) == S[want]


def test_swiglu_and_split_input_checks():
    ws = 1 << 30
    assert tp.tp_swiglu_mlp_pair(A, 64, 128, 512, A, A, A, A, 3, A, A, ws, stream=0) == S["TP_ERR_INDIVISIBLE"]
    assert tp.tp_swiglu_mlp_pair(A, 64, 128, 520, A, A, A, A, 4, A, A, ws, stream=0) == S["TP_ERR_ALIGNMENT"]
    assert tp.tp_swiglu_mlp_pair(None, 64, 128, 512, A, A, A, A, 2, A, A, ws, stream=0) == S["TP_ERR_NULL"]
    assert tp.tp_swiglu_mlp_pair(A, 64, 128, 512, A, A, A, A, 2, A, A, 100, stream=0) == S["TP_ERR_WORKSPACE"]
    assert tp.tp_swiglu_mlp_pair(A, 0, 128, 512, A, A, A, A, 2, A, None, 0, stream=0) == 0
    st, h = tp.tp_swiglu_prepare(A, A, A, A, 128, 512, 3, stream=0)
    assert st == S["TP_ERR_INDIVISIBLE"] and not h
    assert tp.tp_colwise_swiglu(A, 64, 100, A, None, 64, 2, A, stream=0) == S["TP_ERR_ALIGNMENT"]
    assert tp.tp_colwise_swiglu(A, 64, 128, A, None, 60, 2, A, stream=0) == S["TP_ERR_ALIGNMENT"]
    assert tp.tp_colwise_swiglu(A, 64, 128, A, None, 64, 0, A, stream=0) == S["TP_ERR_BAD_DEGREE"]
    assert tp.tp_colwise_swiglu(A, -1, 128, A, None, 64, 2, A, stream=0) == S["TP_ERR_BAD_SHAPE"]
    assert tp.tp_rowwise_split_input_linear(A, 64, 100, A, 64, None, 3, A, stream=0) == S["TP_ERR_INDIVISIBLE"]
    assert tp.tp_rowwise_split_input_linear(A, 64, 60, A, 64, None, 3, A, stream=0) == S["TP_ERR_ALIGNMENT"]
    assert tp.tp_rowwise_split_input_linear(A, 64, 128, A, 60, None, 2, A, stream=0) == S["TP_ERR_ALIGNMENT"]
    assert tp.tp_rowwise_split_input_linear(None, 64, 128, A, 64, None, 2, A, stream=0) == S["TP_ERR_NULL"]
    # the split-input style slices its weight like rowwise
    assert tp.tp_shard_weight(A, 8, 24, tp.TP_ROWWISE_SPLIT_INPUT, 5, 0, A, stream=0) == S["TP_ERR_INDIVISIBLE"]


def test_joint_attn_checks():
    ws = 1 << 30
    up = lambda n: (n + 255) // 256 * 256  # noqa: E731
    Mi, Mt, D = 4096, 512, 3072
    assert tp.tp_joint_attn_workspace_bytes(Mi, Mt, D, 24, 4) == (2 * up(3 * D * D * 2) + 2 * up(D * D * 2)
                                                                  + up((Mi + Mt) * 3 * D * 2) + up((Mi + Mt) * D * 2))
    assert tp.tp_joint_attn_run_workspace_bytes(Mi, Mt, D, 24, 4) == up((Mi + Mt) * 3 * D * 2) + up((Mi + Mt) * D * 2)
    assert tp.tp_joint_attn_workspace_bytes(Mi, -1, D, 24, 4) == 0
    assert tp.tp_joint_attn_workspace_bytes(Mi, Mt, D, 24, 5) == 0
    j = tp.tp_joint_attn_block
    assert j(A, 64, A, 32, 768, A, A, A, A, 6, 4, A, A, A, ws, stream=0) == S["TP_ERR_HEADS_INDIVISIBLE"]
    assert j(A, 64, A, 32, 700, A, A, A, A, 6, 2, A, A, A, ws, stream=0) == S["TP_ERR_BAD_SHAPE"]
    assert j(A, 64, A, -2, 768, A, A, A, A, 6, 2, A, A, A, ws, stream=0) == S["TP_ERR_BAD_SHAPE"]
    assert j(A, 64, A, 32, 768, A, None, A, A, 6, 2, A, A, A, ws, stream=0) == S["TP_ERR_NULL"]
    assert j(A, 64, None, 32, 768, A, A, A, A, 6, 2, A, A, A, ws, stream=0) == S["TP_ERR_NULL"]
    assert j(A, 64, A, 32, 768, A, A, A, A, 6, 2, A, A, A, 10, stream=0) == S["TP_ERR_WORKSPACE"]
    assert j(A, 64, A, 32, 768, A, A, A, A, 6, 2, A + 8, A, A, ws, stream=0) == S["TP_ERR_ALIGNMENT"]
    # an empty text stream may pass NULL pointers for it; both empty is a no-op
    assert j(A, 0, None, 0, 768, A, A, A, A, 6, 2, None, None, None, 0, stream=0) == 0
    st, h = tp.tp_joint_attn_prepare(A, A, A, A, 768, 6, 4, stream=0)
    assert st == S["TP_ERR_HEADS_INDIVISIBLE"] and not h
    assert tp.tp_joint_attn_run(None, A, 64, A, 32, A, A, A, ws, stream=0) == S["TP_ERR_BAD_HANDLE"]


def test_header_is_plain_c(tmp_path):
    # The ABI header must compile as C99 on its own (no C++ constructs outside
    # the extern "C" guard) and as C++.
    import shutil
    import subprocess
    src = tmp_path / "use.c"
    src.write_text('#include "tp.h"\nint main(void) { return tp_abi_version() == TP_ABI_VERSION ? 0 : 1; }\n')
    for cc, std in (("gcc", "-std=c99"), ("g++", "-std=c++17")):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not available")
        r = subprocess.run([cc, std, "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x",
                            "c" if cc == "gcc" else "c++", "-I", os.path.join(ROOT, "include"), str(src)],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_shard_batch_checks():
    ok = (A, 8, 8, tp.TP_COLWISE, A)
    assert tp.tp_shard_weights_batch([], 2, stream=0) == S["TP_ERR_NULL"]
    assert tp.tp_shard_weights_batch([ok] * 9, 2, stream=0) == S["TP_ERR_BAD_SHAPE"]
    assert tp.tp_shard_weights_batch([ok], 0, stream=0) == S["TP_ERR_BAD_DEGREE"]
    # a bad job anywhere in the list rejects the whole call before any launch
    assert tp.tp_shard_weights_batch([ok, (A, 8, 8, 7, A)], 2, stream=0) == S["TP_ERR_BAD_STYLE"]
    assert tp.tp_shard_weights_batch([ok, (A, 9, 8, tp.TP_COLWISE, A)], 2, stream=0) == S["TP_ERR_INDIVISIBLE"]
    assert tp.tp_shard_weights_batch([ok, (A, 8, 24, tp.TP_ROWWISE, A)], 2, stream=0) == S["TP_ERR_ALIGNMENT"]
    assert tp.tp_shard_weights_batch([ok, (0, 8, 8, tp.TP_COLWISE, A)], 2, stream=0) == S["TP_ERR_NULL"]
    # packed jobs are checked like tp_shard_packed_all
    assert tp.tp_shard_weights_batch([ok, (A, 36, 8, tp.TP_COLWISE, A, [1, 1, 3])], 2, stream=0) == \
        S["TP_ERR_BAD_BLOCKS"]
    assert tp.tp_shard_weights_batch([ok, (A, 18, 8, tp.TP_COLWISE, A, [1, 1, 1, 3, 3])], 3, stream=0) == \
        S["TP_ERR_INDIVISIBLE"]


def test_c_program_links_and_gets_errors(tmp_path):
    # A plain C program against libtp.so: status strings and argument errors,
    # which are decided on the host before any CUDA call.
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = tmp_path / "abi.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "tp.h"
int main(void) {
  uint16_t* fake = (uint16_t*)(uintptr_t)(1u << 20);
  int64_t blocks[2] = {1, 4};  /* sum 5 does not divide 36 */
  if (tp_abi_version() != TP_ABI_VERSION) return 1;
  if (tp_shard_weight(NULL, 8, 8, TP_COLWISE, 2, 0, fake, NULL) != TP_ERR_NULL) return 2;
  if (tp_shard_weight(fake, 9, 8, TP_COLWISE, 2, 0, fake, NULL) != TP_ERR_INDIVISIBLE) return 3;
  if (tp_shard_packed_all(fake, 36, 8, TP_COLWISE, blocks, 2, 2, fake, NULL) != TP_ERR_BAD_BLOCKS) return 4;
  if (tp_attn_block(fake, 64, 768, fake, fake, 6, 4, fake, fake, 1 << 30, NULL) != TP_ERR_HEADS_INDIVISIBLE) return 5;
  if (tp_mlp_pair(fake, 0, 128, 512, fake, fake, fake, fake, 2, fake, NULL, 0, NULL) != TP_OK) return 6;
  if (strcmp(tp_status_string(TP_ERR_NULL), "a required pointer is NULL") != 0) return 7;
  puts("ok");
  return 0;
}
""")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(tp.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                        "-L", libdir, "-l:libtp.so", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
