"""The C-ABI library loads, exports every declared symbol and validates
configs on the host, all without a GPU."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import synth
import classifier_scoring_b200 as rm
from classifier_scoring_b200 import build
from tests.helpers import config_for

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(rm_[a-z0-9_]+)\s*\(",
                                text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 15, names
    out = subprocess.run(["nm", "-D", "--defined-only", rm.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (rm_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    L = rm.lib()
    for n in names:
        assert hasattr(L, n)


def test_library_links_no_cudart_shared_object():
    out = subprocess.run(["ldd", rm.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_weights_bytes_match_layout(name):
    shape = synth.WORKLOADS[name].shape
    esz = 4 if shape.weight_dtype == synth.W_F32 else 2
    assert rm.weights_bytes(config_for(shape)) == synth.n_weight_elems(shape) * esz


@pytest.mark.parametrize("field,value", [
    ("arch", 2), ("n_layers", 0), ("hidden", 100), ("n_heads", 7), ("ffn", 12), ("vocab", 0),
    ("max_pos", 10), ("weight_dtype", 3), ("gelu", 5), ("ln_eps", 0.0), ("max_batch_seqs", 0),
    ("max_tokens", 0), ("max_len", 0), ("max_len", 2000), ("sched_max_batch", 0), ("sched_c0", -1),
])
def test_invalid_config_is_rejected_on_host(field, value):
    cfg = config_for(synth.TINY, max_len=32)
    setattr(cfg, field, value)
    assert rm.weights_bytes(cfg) == 0
    h = ctypes.c_void_p()
    buf = np.zeros(16, dtype=np.uint8)
    rc = rm.lib().rm_create(ctypes.byref(cfg), buf.ctypes.data, 16, ctypes.byref(h))
    assert rc == rm.RM_E_INVAL
    assert h.value is None
    assert rm.lib().rm_last_error().decode()


def test_head_dim_limits():
    cfg = config_for(synth.TINY, max_len=32)
    cfg.hidden, cfg.n_heads = 264, 1          # d = 264 > 128
    assert rm.weights_bytes(cfg) == 0
    cfg.hidden, cfg.n_heads = 120, 8          # d = 15, odd
    assert rm.weights_bytes(cfg) == 0


def test_create_checks_weight_size_before_the_device():
    cfg = config_for(synth.TINY, max_len=32)
    n = rm.weights_bytes(cfg)
    buf = np.zeros(n - 4, dtype=np.uint8)
    h = ctypes.c_void_p()
    assert rm.lib().rm_create(ctypes.byref(cfg), buf.ctypes.data, n - 4, ctypes.byref(h)) == rm.RM_E_INVAL
    assert "weights_bytes" in rm.lib().rm_last_error().decode()


def test_null_arguments_are_errors_not_crashes():
    L = rm.lib()
    assert L.rm_score(None, None, None, 1, None, None) == rm.RM_E_INVAL
    assert L.rm_score_host(None, None, None, 1, None, None) == rm.RM_E_INVAL
    assert L.rm_schedule(None, None, 0, None) == rm.RM_E_INVAL
    assert L.rm_get_device_error(None, None) == rm.RM_E_INVAL
    assert L.rm_arena_stats(None, None) == rm.RM_E_INVAL
    L.rm_destroy(None)
    assert L.rm_op_gemm(None, None, None, None, 1, 1, 8, 8, 0, None) == rm.RM_E_INVAL
    assert L.rm_op_res_ln(None, None, None, None, None, 1, 8, 1e-5, 1, 0, None) == rm.RM_E_INVAL


def test_varlen_meta_layout():
    lens = np.array([1, 7, 64, 65, 130, 8])
    off = synth.offsets_from_lengths(lens)
    rb, so = rm.ops.varlen_meta(off, 3)
    Lp = (lens + 7) // 8 * 8
    assert rb.tolist() == [0] + np.cumsum((lens + 63) // 64).tolist()
    assert so.tolist() == [0] + np.cumsum(3 * lens * Lp).tolist()
    bad = off.copy()
    bad[2] = bad[1]
    with pytest.raises(rm.RmError):
        rm.ops.varlen_meta(bad, 3)


@pytest.mark.parametrize("seed", range(6))
def test_attn_tc_tiles_cut_whole_sequences_greedily(seed):
    """Tiles of the tensor-core attention: consecutive runs of whole sequences
    that cover the batch, each at most 128 rows, and maximal (the next
    sequence would not have fit) -- checked against the definition, not a
    second implementation of the cut."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 129, int(rng.integers(1, 400)))
    if seed == 0:
        lens = np.array([128, 1, 127, 128, 64, 64, 65])
    off = synth.offsets_from_lengths(lens)
    tiles = rm.ops.attn_tc_tiles(off)
    assert tiles[0] == 0 and tiles[-1] == len(lens)
    assert np.all(np.diff(tiles) >= 1)
    rows = off[tiles[1:]] - off[tiles[:-1]]
    assert np.all(rows <= 128)
    # greedy: each tile but the last could not take the next tile's first sequence
    assert np.all(rows[:-1] + lens[tiles[1:-1]] > 128)


def test_attn_tcl_items_cover_every_query_tile_heaviest_first():
    rng = np.random.default_rng(5)
    for causal in (0, 1):
        lens = rng.integers(1, 513, 40)
        off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        items = rm.ops.attn_tcl_items(off, causal)
        want = sorted((i, q) for i, L in enumerate(lens) for q in range((L + 127) // 128))
        assert sorted((int(it) >> 2, int(it) & 3) for it in items) == want
        chunks = [(min(lens[it >> 2], 128 * ((it & 3) + 1)) if causal else lens[it >> 2]) for it in items]
        chunks = [(c + 127) // 128 for c in chunks]
        assert chunks == sorted(chunks, reverse=True)


def test_attn_tcl_items_reject_long_or_empty_sequences():
    out = np.zeros(8, dtype=np.int32)
    for lens in ([513], [3, 0, 2]):
        off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        rc = rm.lib().rm_attn_tcl_items(off.ctypes.data, len(lens), 0, out.ctypes.data)
        assert rc < 0


def test_attn_tc_tiles_reject_long_or_empty_sequences():
    for lens in ([5, 129, 3], [4, 0, 2]):
        off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        with pytest.raises(rm.RmError):
            rm.ops.attn_tc_tiles(off)


def test_gemm_tile_pick_is_a_known_tile():
    tiles = {(1, bn) for bn in (64, 96, 128, 160, 192, 224, 256)} | {(2, bn) for bn in (128, 192, 256)}
    for M in (1, 77, 128, 300, 3328, 26112):
        for N in (8, 312, 768, 2304, 3072, 8192):
            for K in (8, 768, 2048, 8192):
                for sms in (1, 2, 148):
                    t = rm.ops.gemm_tile(M, N, K, sms)
                    assert t in tiles, (M, N, K, sms, t)
                    if sms == 1:
                        assert t[0] == 1            # a pair needs two SMs
    with pytest.raises(rm.RmError):
        rm.ops.gemm_tile(0, 8, 8, 148)


def test_gemm_tiled_rejects_unknown_tiles_on_host():
    # rejected before any device call: the pointers are never dereferenced
    fake = 1 << 20
    for cg, bn in [(2, 64), (2, 96), (1, 72), (3, 128), (-1, 128)]:
        rc = rm.lib().rm_op_gemm_tiled(fake, fake, None, fake, rm.F32, 128, 128, 64, 0, cg, bn, None)
        assert rc == -1, (cg, bn, rc)
        assert b"tile" in rm.lib().rm_last_error()


def test_headers_compile_as_c_and_host_calls_run_without_a_gpu(tmp_path):
    """include/*.h as plain C11 (-Wall -Werror), linked against the library;
    the host-only calls run here.  The latency objective on four equal
    requests with T = 2 + b*L takes batches [2, 1, 1] (a worked example of the
    oracle's pins)."""
    exe = tmp_path / "abi_from_c"
    src = os.path.join(ROOT, "tests", "c", "abi_from_c.c")
    libdir = os.path.join(ROOT, "classifier_scoring_b200")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    src, "-o", str(exe), "-L", libdir, "-lrmscore", f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    cfg = config_for(synth.TINY)
    assert int(out[0]) == rm.lib().rm_weights_bytes(ctypes.byref(cfg))
    assert out[1:] == ["3", "0", "0", "1", "2"]
