"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every function that
``include/s2o.h`` declares, sizes its buffers as documented and rejects bad arguments before
enqueueing any device work; the header compiles in a plain C99 client that links the library."""
import ctypes
import os
import re

import pytest

import long_context_sparse_stripe_b200 as s2o

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "s2o.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(s2o_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = s2o._load()
    names = declared_functions()
    assert len(names) >= 13
    for name in names:
        assert hasattr(lib, name), name


def test_library_is_the_in_tree_build():
    path = s2o.library_path()
    assert os.path.isfile(path)
    assert os.path.dirname(path) == os.path.dirname(os.path.abspath(s2o.__file__))


def test_status_strings():
    lib = s2o._load()
    for code, name in s2o.STATUS.items():
        assert lib.s2o_status_string(code).decode() == name
    assert lib.s2o_status_string(99).decode() == "S2O_ERR_UNKNOWN"


LLAMA_128K = s2o.Config(1, 32, 8, 131072, 128, 2048, 128, 0.01)


def test_index_sizes_and_workspace_are_documented_shapes():
    cfg = LLAMA_128K
    nB = 1024
    assert s2o.index_sizes(cfg) == [32 * 131072, 32 * 131072, 32 * nB, 32 * nB * nB, 32 * nB]
    ws = s2o.workspace_size(cfg)
    # kappa/rho/keys (2 x 8-byte) per query slot, Qbar/Kbar/chunks, block scores and counts
    lower = 32 * 131072 * (4 + 4 + 16) + 32 * nB * nB * 4 + 32 * 64 * nB * 4
    assert lower <= ws <= lower + 96 * 2**20


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 96, 2), ("block_size", 32, 2), ("n_kv_heads", 3, 2), ("segment_len", 192, 2),
    ("seq_len", 131072 + 2048 * 0 + 64, 2), ("tau", -0.1, 1), ("tau", float("nan"), 1),
    ("tau", float("inf"), 1), ("batch", 0, 1), ("query_perm", 2, 1),
])
def test_bad_config_rejected(field, value, code):
    cfg = s2o.Config(**{**LLAMA_128K.__dict__, field: value})
    n = ctypes.c_size_t(0)
    assert s2o._load().s2o_workspace_size(ctypes.byref(cfg._c()), ctypes.byref(n)) == code


def test_tau_above_one_is_legal():
    cfg = s2o.Config(**{**LLAMA_128K.__dict__, "tau": 1.5})
    assert s2o.workspace_size(cfg) > 0


def test_null_and_misaligned_pointers_rejected_before_launch():
    lib = s2o._load()
    c = LLAMA_128K._c()
    idx = s2o._Indices(0x1000, 0x2000, 0x3000, 0x4000, 0x5000)
    # null q
    assert lib.s2o_build_indices(ctypes.byref(c), None, 0x1000, ctypes.byref(idx), 0x1000,
                                 1 << 40, None) == 1
    # misaligned k
    assert lib.s2o_build_indices(ctypes.byref(c), 0x1000, 0x1008, ctypes.byref(idx), 0x1000,
                                 1 << 40, None) == 1
    # null index array
    bad = s2o._Indices(0x1000, 0, 0x3000, 0x4000, 0x5000)
    assert lib.s2o_build_indices(ctypes.byref(c), 0x1000, 0x1000, ctypes.byref(bad), 0x1000,
                                 1 << 40, None) == 1
    assert lib.s2o_attention_prefill_with_indices(ctypes.byref(c), 0x1000, 0x1000, None,
                                                  ctypes.byref(idx), 0x1000, None) == 1
    assert lib.s2o_dense_causal_prefill(ctypes.byref(c), 0x1000, 0x1000, 0x1000, None, None) == 1
    assert lib.s2o_exp64_eval(None, None, 4, None) == 1


def test_workspace_too_small_rejected_before_launch():
    lib = s2o._load()
    c = LLAMA_128K._c()
    idx = s2o._Indices(0x1000, 0x2000, 0x3000, 0x4000, 0x5000)
    need = s2o.workspace_size(LLAMA_128K)
    assert lib.s2o_build_indices(ctypes.byref(c), 0x1000, 0x1000, ctypes.byref(idx), 0x1000,
                                 need - 1, None) == 3
    assert lib.s2o_attention_prefill(ctypes.byref(c), 0x1000, 0x1000, 0x1000, 0x1000,
                                     ctypes.byref(idx), 0x1000, need - 1, None) == 3
    assert lib.s2o_validate_indices(ctypes.byref(c), ctypes.byref(idx), 0x1000, need - 1,
                                    None) == 3
    st = s2o._Stats()
    assert lib.s2o_index_stats(ctypes.byref(c), ctypes.byref(idx), 0x1000, need - 1,
                               ctypes.byref(st), None) == 3


def test_workspace_views_are_inside_the_workspace():
    cfg = LLAMA_128K
    need = s2o.workspace_size(cfg)
    view = s2o._View()
    base = 1 << 32
    assert s2o._load().s2o_workspace_views(ctypes.byref(cfg._c()), base, need,
                                           ctypes.byref(view)) == 0
    ptrs = [getattr(view, f) for f, _ in s2o._View._fields_]
    assert all(base <= p < base + need for p in ptrs)
    assert len(set(ptrs)) == len(ptrs)


# ----------------------------------------------------------------------------- prefill + layer


def test_prefill_workspace_holds_the_merge_and_packed_stream_buffers():
    cfg = LLAMA_128K
    base = s2o.workspace_size(cfg)
    full = s2o.prefill_workspace_size(cfg)
    Hq, N, d, B, S = 32, 131072, 128, 128, 2048
    nB, nSeg = N // B, N // S
    lse = Hq * N * 4                          # per-row log2-sum-exps of the merge path
    copy = 2 * Hq * N * d * 2                 # K and V in each query head's key order
    positions = Hq * N * 4 + Hq * nSeg * nB   # block-ordered key positions, visible counts
    pairs = Hq * nB // 2
    chunks = pairs * (2 * nB * (B // 16) + 3 * (B // 16)) * 4 + pairs * 16  # chunk lists, counts
    want = lse + copy + positions + chunks
    assert want <= full - base <= want + 4096


def test_permuted_copy_modes_are_accepted():
    lib = s2o._load()
    for mode in (0, 1, 2, 3, 7, -1):
        s2o.set_permuted_copy(mode)
    s2o.set_permuted_copy(1)
    assert lib is s2o._load()


def _layer_size(cfg, shape, dense=False):
    n = ctypes.c_size_t(0)
    lc = s2o._layer_config(shape, dense)
    return s2o._load().s2o_layer_workspace_size(ctypes.byref(cfg._c()), ctypes.byref(lc),
                                                ctypes.byref(n)), n.value


def test_layer_workspace_size_and_argument_checks():
    import gen
    shape = gen.LAYER_8B
    st, s2o_bytes = _layer_size(LLAMA_128K, shape)
    assert st == 0
    st, dense_bytes = _layer_size(LLAMA_128K, shape, dense=True)
    assert st == 0
    rows, H, I = 131072, 4096, 14336
    # activations: h, qkv, q, k, v, o, o_rows, gate|up, silu product (bf16)
    acts = rows * 2 * (H + 6144 + H + 1024 + 1024 + H + H + 2 * I + I)
    assert dense_bytes >= acts
    # the S2O layer adds the attention's prefill workspace
    assert s2o_bytes - dense_bytes >= s2o.prefill_workspace_size(LLAMA_128K) - 1024
    assert _layer_size(LLAMA_128K, shape.replace(intermediate=100))[0] == 1   # not a multiple of 8
    assert _layer_size(LLAMA_128K, shape.replace(rms_eps=0.0))[0] == 1
    # the dense baseline ignores the segment length; S2O does not
    bad_seg = s2o.Config(**{**LLAMA_128K.__dict__, "segment_len": 192})
    assert _layer_size(bad_seg, shape)[0] == 2
    assert _layer_size(bad_seg, shape, dense=True)[0] == 0


def test_layer_prefill_rejects_null_weights_before_launch():
    import gen
    lib = s2o._load()
    shape = gen.LAYER_8B
    lc = s2o._layer_config(shape, False)
    w = s2o._LayerWeights(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0)  # w_down missing
    st = lib.s2o_layer_prefill(ctypes.byref(LLAMA_128K._c()), ctypes.byref(lc), ctypes.byref(w),
                               0x10000, 0x20000, 1 << 40, None)
    assert st == 1
    w = s2o._LayerWeights(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000)
    st = lib.s2o_layer_prefill(ctypes.byref(LLAMA_128K._c()), ctypes.byref(lc), ctypes.byref(w),
                               0x10000, 0x20000, 1024, None)
    assert st == 3  # workspace too small


def test_attention_work_rejects_bad_arguments_before_device_work():
    cfg = LLAMA_128K
    lib = s2o._load()
    idx = s2o._Indices(0x1000, 0x2000, 0x3000, 0x4000, 0x5000)
    out = s2o._Work()
    small = s2o.prefill_workspace_size(cfg) - 1
    assert lib.s2o_attention_work(ctypes.byref(cfg._c()), ctypes.byref(idx), 0x10000, small,
                                  ctypes.byref(out), None) == 3
    assert lib.s2o_attention_work(ctypes.byref(cfg._c()), ctypes.byref(idx), 0x10000, small + 1,
                                  None, None) == 1
    assert lib.s2o_attention_work(ctypes.byref(cfg._c()), None, 0x10000, small + 1,
                                  ctypes.byref(out), None) == 1


C_CLIENT = r"""
#include "s2o.h"
#include <stdio.h>

int main(void) {
  s2o_config c = {1, 32, 8, 131072, 128, 2048, 128, 0.01f, 1, 0, 0};
  size_t ws = 0, pws = 0, counts[5], bad = 0;
  if (s2o_workspace_size(&c, &ws) != S2O_OK) return 1;
  if (s2o_prefill_workspace_size(&c, &pws) != S2O_OK) return 2;
  if (s2o_index_sizes(&c, counts) != S2O_OK) return 3;
  c.head_dim = 96;
  if (s2o_workspace_size(&c, &bad) != S2O_ERR_UNSUPPORTED) return 4;
  printf("%zu %zu %zu %zu %zu %zu %zu %s %u\n", ws, pws, counts[0], counts[1], counts[2],
         counts[3], counts[4], s2o_status_string(S2O_ERR_UNSUPPORTED),
         (unsigned)S2O_STATIC_WORKSPACE_BYTES);
  return 0;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    """A C99 client (no C++, no torch) includes the header with warnings as errors, links the
    in-tree library and makes host-only calls; it sees the sizes the binding sees."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(s2o.library_path())
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                    "-L", libdir, "-l:" + os.path.basename(s2o.library_path()),
                    "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    cfg = LLAMA_128K
    want = [s2o.workspace_size(cfg), s2o.prefill_workspace_size(cfg), *s2o.index_sizes(cfg)]
    assert [int(x) for x in out[:7]] == want
    assert out[7] == "S2O_ERR_UNSUPPORTED" and int(out[8]) == s2o.STATIC_WORKSPACE_BYTES
